"""CPU checks of the stream planner's refusals (they happen before any CUDA
call): stream_buffers outside [2, 8], a plan that does not fit the device cap,
misaligned sizes, missing host blobs.  Refuse, never clamp."""
import ctypes

import pytest

from layer_streamed_qlora_b200 import _lib as L


def _desc(n_layers=4, layer_bytes=1 << 20, n_buffers=2, cap=0, reserve=0, vocab=0, null_layer=False):
    ptrs = (ctypes.c_void_p * n_layers)(*[0x1000 * (i + 1) for i in range(n_layers)])
    if null_layer:
        ptrs[1] = None
    d = L.StreamDesc(n_layers, layer_bytes, ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p)), vocab, None, None,
                     n_buffers, cap, reserve)
    return d, ptrs


def _plan_status(d):
    h = ctypes.c_void_p()
    st = L.lib().soup_stream_plan(ctypes.byref(d), ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("nb", [0, 1, 9, 16])
def test_buffers_out_of_range_refused(nb):
    d, keep = _desc(n_buffers=nb)
    st, h = _plan_status(d)
    assert st == 1 and not h.value
    assert b"[2, 8]" in L.lib().soup_last_error()


def test_cap_too_small_refused():
    # 2 slots x 100 MiB + 50 MiB reserve > 200 MiB cap
    d, keep = _desc(layer_bytes=100 << 20, n_buffers=2, cap=200 << 20, reserve=50 << 20)
    st, h = _plan_status(d)
    assert st == 5 and not h.value  # SOUP_ERR_OOM_PLAN
    assert b"cap" in L.lib().soup_last_error()


def test_misaligned_and_missing_refused():
    d, keep = _desc(layer_bytes=1000)
    assert _plan_status(d)[0] == 3  # SOUP_ERR_ALIGN
    d, keep = _desc(null_layer=True)
    assert _plan_status(d)[0] == 1
    d, keep = _desc(vocab=100)
    assert _plan_status(d)[0] == 3


def test_blob_layout_sizes_match_the_shapes():
    import soup_synth as ss
    c = L.layer_cfg(ss.LLAMA8B_LAYER)
    nf4 = L.soup_layer_blob_bytes(c, L.SOUP_WEIGHT_NF4)
    bf = L.soup_layer_blob_bytes(c, L.SOUP_WEIGHT_BF16)
    params = 6144 * 4096 + 4096 * 4096 + 2 * 14336 * 4096 + 4096 * 14336
    assert params == 218_103_808
    # codes (1/2 byte) + absmax (4 bytes / 64) + two norms, each part 256-aligned
    assert abs(nf4 - (params // 2 + params // 16 + 2 * 4096 * 2)) < 10 * 256
    assert abs(bf - (params * 2 + 2 * 4096 * 2)) < 10 * 256
    v = L.soup_layer_blob_views(c, L.SOUP_WEIGHT_NF4, 0)
    assert v.qkv.out_features == 6144 and v.down.in_features == 14336
    assert v.norm2 + 4096 * 2 <= nf4
    cq = L.layer_cfg(ss.QWEN3B_LAYER)
    assert abs(L.soup_layer_blob_bytes(cq, L.SOUP_WEIGHT_BF16) - 154_148_864) < 10 * 256


def test_kept_layer_count_respects_the_device_cap():
    from layer_streamed_qlora_b200.model import kept_layer_count
    per = 25_165_824  # q|k|v of an 8B layer at 2048 tokens, fp16
    arena = 2 * 122_700_000 + 1_050_700_000
    assert kept_layer_count(32, per, arena, 2_000_000_000, 0) == 32          # no cap: every layer
    assert kept_layer_count(32, per, arena, 2_000_000_000, 1 << 32) == 32    # 4 GiB: all fit
    k = kept_layer_count(32, per, arena, 2_000_000_000, 4_000_000_000)       # 4e9 bytes: some
    assert 0 < k < 32 and arena + 2_000_000_000 + k * per <= 4_000_000_000
    assert arena + 2_000_000_000 + (k + 1) * per > 4_000_000_000
    assert kept_layer_count(32, per, arena, 3_000_000_000, 4_000_000_000) == 0  # no room
    assert kept_layer_count(32, 0, arena, 0, 0) == 0


def test_plan_without_host_layers_passes_validation():
    # the disk tier's plan holds no host copies of the layers (they arrive
    # through soup_stream_prefetch_from); validation accepts a NULL array.
    # Without a GPU the arena allocation that follows fails with SOUP_ERR_CUDA.
    d = L.StreamDesc(4, 1 << 20, None, 0, None, None, 2, 0, 0)
    st, h = _plan_status(d)
    if st == 0:
        L.lib().soup_stream_plan_free(h)
    assert st in (0, 7), L.lib().soup_last_error()


def test_model_refuses_unknown_settings_before_touching_the_gpu():
    # refuse, never ignore: checked before any allocation
    from layer_streamed_qlora_b200.model import ModelConfig, StreamedLoRAModel
    cfg = ModelConfig(hidden=512, n_q_heads=4, n_kv_heads=2, head_dim=128, intermediate=1024, rank=16, alpha=32.0,
                      vocab=512, n_layers=2)
    for kw in ({"stream_source": "nvme"}, {"stream_source": "disk"}, {"task": "kto"}):
        with pytest.raises(ValueError):
            StreamedLoRAModel(cfg, 2, 16, **kw)


def test_model_precheck_refuses_a_cap_below_the_lower_bound_before_any_work():
    from layer_streamed_qlora_b200.model import ModelConfig, StreamedLoRAModel, device_bytes_lower_bound
    cfg = ModelConfig(hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, intermediate=14336, rank=16,
                      alpha=32.0, vocab=128256, n_layers=32)
    lb = device_bytes_lower_bound(cfg, 4, 512, 2, 256)
    # 2 slots x 122.7 MB + the 1050.7 MB vocab slot + 33 checkpoints x 16.8 MB + workspaces
    assert 2 * 122_699_776 + 1_050_673_152 + 33 * 2048 * 4096 * 2 < lb < 4 << 30
    with pytest.raises(ValueError, match="device cap"):
        StreamedLoRAModel(cfg, 4, 512, n_buffers=2, device_cap_bytes=1 << 30)  # refused at once, no GPU needed


def test_keep_plan_modes_and_the_cap():
    from layer_streamed_qlora_b200.model import plan_keep
    qkv, saved = 25_165_824, 455_000_000
    arena, reserve = 1_296_000_000, 2_500_000_000
    # no cap: auto keeps everything
    assert plan_keep(32, qkv, saved, arena, reserve, 0) == ["saved"] * 32
    assert plan_keep(32, qkv, saved, arena, reserve, 0, "recompute") == [None] * 32
    assert plan_keep(32, qkv, saved, arena, reserve, 0, "keep") == ["saved"] * 32
    # 4 GiB: q|k|v for the layers that fit, nothing saved
    cap = 1 << 32
    p = plan_keep(32, qkv, saved, arena, reserve, cap)
    k = p.count("qkv")
    assert 0 < k < 32 and p.count("saved") == 0 and p[:k] == ["qkv"] * k
    assert arena + reserve + k * qkv <= cap < arena + reserve + (k + 1) * qkv
    # room for every q|k|v and two upgrades: the first two layers are saved
    cap2 = arena + reserve + 32 * qkv + 2 * (saved - qkv) + 1000
    p2 = plan_keep(32, qkv, saved, arena, reserve, cap2)
    assert p2[:2] == ["saved", "saved"] and p2[2:] == ["qkv"] * 30
    assert arena + reserve + 2 * saved + 30 * qkv <= cap2
    # keep refuses a cap that cannot hold every saved layer; unknown modes refused
    with pytest.raises(ValueError):
        plan_keep(32, qkv, saved, arena, reserve, cap, "keep")
    with pytest.raises(ValueError):
        plan_keep(32, qkv, saved, arena, reserve, cap, "sometimes")


def test_prompt_dedup_indices_brute_force():
    """The shared-prompt layout's index arrays against a direct construction:
    pairs (2p chosen, 2p+1 rejected) whose prompts are equal, laid out as
    [prompt | chosen continuation | rejected continuation]."""
    import numpy as np

    from layer_streamed_qlora_b200.model import prompt_dedup_indices, token_rows
    B, S, Lp = 6, 11, 4
    Lc = S - Lp
    rng = np.random.default_rng(0)
    ids = rng.integers(0, 1000, size=(B, S))
    ids[1::2, :Lp] = ids[0::2, :Lp]  # each pair shares its prompt
    phys, hrows, hids, start, src = prompt_dedup_indices(B, S, Lp)
    T = token_rows(B, S, Lp)
    assert T == (B // 2) * (Lp + 2 * Lc) == phys.size
    flat = ids.reshape(-1)
    tok = flat[phys]
    expect = np.concatenate([np.concatenate([ids[2 * p, :Lp], ids[2 * p, Lp:], ids[2 * p + 1, Lp:]])
                             for p in range(B // 2)])
    assert np.array_equal(tok, expect)
    # the head reads, per sequence, positions Lp-1 .. S-1 of that sequence
    assert hrows.size == B * (Lc + 1) and np.array_equal(flat[hids], ids[:, Lp - 1:].reshape(-1))
    for v in range(B):
        for j in range(Lc + 1):
            t = Lp - 1 + j
            assert tok[hrows[v * (Lc + 1) + j]] == ids[v, t]
    # the CSR lists every head row once, under the token row it reads
    assert start[0] == 0 and start[-1] == hrows.size and np.array_equal(np.sort(src), np.arange(hrows.size))
    for d in range(T):
        for h in src[start[d]:start[d + 1]]:
            assert hrows[h] == d
    # the last prompt row of each pair is read by both sequences
    for p in range(B // 2):
        d = p * (Lp + 2 * Lc) + Lp - 1
        assert start[d + 1] - start[d] == 2
