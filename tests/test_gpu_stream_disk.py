"""The disk tier on the GPU: a plan made without host copies of the layers is
fed from shard files through the shard reader's page-locked staging buffers
(soup_stream_prefetch_from with the buffer's copy-done event); the slots hold
the files' bytes, only the copied visits are read, and a streamed training
step from disk gives the same bits as the same step from pinned RAM."""
import numpy as np
import pytest
import torch

import soup_synth as ss
from tests.model_fixture import NumpyWeights

pytestmark = pytest.mark.gpu
L = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global L
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from layer_streamed_qlora_b200 import _lib as lib
    lib.lib()
    L = lib
    yield
    assert lib.device_error() == 0


def _bring(plan, disk, l):
    if plan.resident(l):
        plan.prefetch(l)
        return
    host, ev = disk.acquire(l)
    plan.prefetch_from(l, host, ev)
    disk.release(l)


def test_disk_slots_hold_the_shard_bytes(tmp_path):
    nb = 9 << 20  # two read requests; a copy split over both copy streams
    n, N = 5, 2
    data, paths = [], []
    for i in range(n):
        b = np.random.default_rng(i).integers(0, 256, nb, dtype=np.uint8)
        p = tmp_path / f"layer_{i:03d}.bin"
        b.tofile(p)
        data.append(torch.from_numpy(b))
        paths.append(str(p))
    plan = L.Plan(None, nb, N, n_layers=n)
    disk = L.Disk(paths, nb, read_ahead=2, n_slots=N, io_threads=4, pinned=True, direct=True)
    rows = nb // 16
    ids = torch.arange(rows, dtype=torch.int32, device="cuda")
    out = torch.empty((rows, 8), dtype=torch.bfloat16, device="cuda")
    try:
        with pytest.raises(L.SoupError):
            plan.prefetch(0)  # no host copy in this plan: layers come from the reader
        order = list(range(n)) + list(range(n - 1, -1, -1))
        disk.schedule(order)
        for direction in (range(n), range(n - 1, -1, -1)):  # forward, then backward, as a training step
            seq = list(direction)
            for l in seq[:N]:
                _bring(plan, disk, l)
            for i, l in enumerate(seq):
                ptr = plan.wait(l)
                L.soup_embed(ptr, rows, 8, ids, rows, out)
                torch.cuda.synchronize()
                assert torch.equal(out.view(torch.uint8).reshape(-1).cpu(), data[l]), l
                plan.release(l)
                if i + N < n:
                    _bring(plan, disk, seq[i + N])
        torch.cuda.synchronize()
        st, ps = disk.stats(), plan.stats()
        assert ps["copies"] == 2 * n - N and ps["reuses"] == N
        assert st["acquires"] == ps["copies"] and st["skipped"] == 0
    finally:
        plan.free()
        disk.close()


def test_disk_model_matches_ram_model_bit_exact(tmp_path):
    from layer_streamed_qlora_b200 import model as M
    cfg = M.ModelConfig(hidden=512, n_q_heads=4, n_kv_heads=2, head_dim=128, intermediate=1024, rank=16,
                        alpha=32.0, vocab=512, n_layers=4, kind="nf4")
    B, S = 2, 64
    ids = torch.from_numpy(ss.uniform_ids(3, "ids", (B, S), cfg.vocab).astype(np.int32))
    out = {}
    for src in ("ram", "disk"):
        m = M.StreamedLoRAModel(cfg, B, S, n_buffers=2, weights=NumpyWeights(cfg, 4), head_chunk=48,
                                stream_source=src, shard_dir=str(tmp_path / "shards") if src == "disk" else None,
                                read_ahead=2)
        try:
            m.ids.copy_(ids)
            losses = []
            for _ in range(2):  # two steps: the step boundary's resident layers too
                losses.append(m.sft_step().clone())
                m.optimizer_step()
            torch.cuda.synchronize()
            out[src] = (torch.stack(losses), m.lora_flat.clone(), m.master_flat.clone(),
                        m.disk.stats() if m.disk is not None else None)
        finally:
            m.close()
    a, b = out["ram"], out["disk"]
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    st = b[3]
    n, N = cfg.n_layers, 2
    assert st["acquires"] == (2 * n - N) + (2 * n - 2 * N) and st["skipped"] == 0
