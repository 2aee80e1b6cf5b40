"""Host-side pieces of bench.py (no GPU): the roofline denominators, the
per-launch DRAM traffic read from the committed ncu summary (only while the
GEMM source is the one it was taken on), the workload table and the JSON
config, the probe shapes, and the projection of the oracle's timed sample to
the whole stack."""
import hashlib
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)  # defines only; main() runs under __main__
    return mod


def test_peaks_are_the_measured_ones_when_present(bench):
    pk, kind = bench.peaks()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        assert kind == "measured" and pk == json.load(open(path))
    else:
        assert kind == "fallback"
    assert pk["bf16_tflops_sustained"] > 0 and pk["hbm_gbs"] > 0


def test_traffic_only_for_the_gemm_source_it_was_taken_on(bench):
    md = open(os.path.join(ROOT, "profiles", "gemm_nf4_fwd_traffic.md")).read()
    src = open(os.path.join(ROOT, "layer_streamed_qlora_b200", "csrc", "gemm.cu"), "rb").read()
    tr = bench.gemm_traffic()
    if hashlib.sha256(src).hexdigest() in md:
        assert tr is not None and 0 < tr["bytes_per_launch"] < 1e9
    else:
        assert tr is None


def test_workloads_and_config(bench):
    assert bench.DEFAULT in bench.WORKLOADS
    w = bench.WORKLOADS[bench.DEFAULT]
    # the 8B NF4 stream: 32 layers, 2048 tokens per step, 2 slots, 4 GiB cap
    assert (w["n_layers"], w["batch"] * w["seq"], w["buffers"], w["cap_gb"], w["kind"]) == (32, 2048, 2, 4.0, "nf4")
    for name, wl in bench.WORKLOADS.items():
        assert wl["task"] in ("sft", "dpo", "simpo", "orpo"), name
        if wl["task"] != "sft":
            assert wl["batch"] % 2 == 0 and 0 < wl["prompt"] < wl["seq"], name
        c = bench.bench_config(wl, name, 2, kept_layers=3)
        assert c["workload"] == name and c["global_batch"] == 2 * wl["batch"] and c["parallelism"] == "dp2"
        assert c["kept_qkv_layers"] == 3 and "optimizer" in c and "l2" in c
        assert not {"model"} & set(c)
    shapes = bench.probe_shapes(w)
    assert shapes == {"qkv": (6144, 4096), "o": (4096, 4096), "gate_up": (28672, 4096), "down": (4096, 14336)}
    assert set(bench.PROBE_WEIGHTS) == set(shapes)


def test_oracle_projection(bench):
    w = dict(bench.WORKLOADS[bench.DEFAULT])
    # a layer sample of 256 tokens taking 2 s and an AdamW step of 0.5 s per
    # 2048-token step, over 32 layers; a head sample of 64 tokens over 1/8 of
    # the vocabulary taking 0.25 s
    per_tok = bench.oracle_seconds_per_token(w, 2.0, 0.5, 0.25, 256)
    assert bench.HEAD_SAMPLE_TOKENS == 64 and bench.HEAD_VOCAB_FRACTION == 8
    assert per_tok == pytest.approx((2.0 / 256 + 0.5 / 2048) * 32 + 0.25 * 8 / 64, rel=1e-12)


def test_gpus_n_spawns_n_ranks_itself():
    """`bench.py --gpus 2` without a launcher starts two ranks itself (RANK /
    WORLD_SIZE / MASTER_* set for each), which join one process group; here
    with the gloo backend and the launcher check only (no GPU)."""
    import subprocess
    import sys
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dist-check",
                          "--backend", "gloo"], env=env, capture_output=True, text=True, timeout=240)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout  # rank 0 alone prints
    d = lines[0]
    assert d["n_gpus"] == 2 and d["ranks_joined"] == 2 and d["rank_sum"] == 3.0 and d["backend"] == "gloo"
