"""GPU checks of the slot ring: bytes arrive intact, resident items are reused
without a copy, the host wait times out instead of hanging, an injected copy
failure surfaces as a status, and a full ring refuses another prefetch.
Nothing here faults or hangs the GPU: the delayed copy waits on an event
recorded on another stream after a short, bounded spin (torch.cuda._sleep)."""
import time

import pytest
import torch

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


def _blobs(n, nbytes):
    out = []
    for i in range(n):
        t = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
        t.copy_(torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=torch.Generator().manual_seed(i)))
        out.append(t)
    return out


def test_round_trip_reuse_and_refusal():
    nb = 1 << 20
    blobs = _blobs(5, nb)
    plan = L.Plan(blobs, nb, 2)
    seen = {}
    for item in range(5):
        if item >= 2:
            plan.release(item - 2)
        plan.prefetch(item)
        ptr = plan.wait(item)
        seen[item] = ptr
    torch.cuda.synchronize()
    s = plan.stats()
    assert s["copies"] == 5 and s["reuses"] == 0 and s["bytes_copied"] == 5 * nb
    # both slots hold unreleased items: a third prefetch is refused
    with pytest.raises(L.SoupError):
        plan.prefetch(0)
    plan.release(3)
    plan.release(4)
    plan.prefetch(4)  # still resident: reused, no copy
    assert plan.stats()["reuses"] == 1
    plan.release(4)
    plan.free()


def test_slot_contents_are_the_host_bytes():
    nb = 1 << 16
    blobs = _blobs(3, nb)
    plan = L.Plan(blobs, nb, 2)
    # read the slot back with the embedding gather: the slot viewed as
    # [nb/16, 8] bf16 rows (16 bytes each), ids = every row
    rows = nb // 16
    ids = torch.arange(rows, dtype=torch.int32, device="cuda")
    out = torch.empty((rows, 8), dtype=torch.bfloat16, device="cuda")
    for item in range(3):
        if item >= 2:
            plan.release(item - 2)
        plan.prefetch(item)
        ptr = plan.wait(item)
        L.soup_embed(ptr, rows, 8, ids, rows, out)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.uint8).reshape(-1).cpu(), blobs[item])
    plan.free()


def test_host_wait_times_out_then_completes():
    nb = 1 << 20
    blobs = _blobs(2, nb)
    plan = L.Plan(blobs, nb, 2)
    gate_stream = torch.cuda.Stream()
    ev = torch.cuda.Event()
    with torch.cuda.stream(gate_stream):
        torch.cuda._sleep(int(4e8))  # ~0.2 s of bounded device-side spinning on the gate stream only
        ev.record()
    plan.debug_gate_next_copy(ev.cuda_event)
    plan.prefetch(0)
    t0 = time.time()
    with pytest.raises(L.SoupError) as e:
        plan.wait_host(0, 10)
    assert e.value.status == 6  # SOUP_ERR_TIMEOUT
    assert time.time() - t0 < 0.15
    plan.wait_host(0, 30000)  # the copy does finish once the gate opens
    plan.free()


def test_injected_copy_failure_is_a_status():
    nb = 1 << 16
    plan = L.Plan(_blobs(2, nb), nb, 2)
    plan.debug_fail_next_copy()
    with pytest.raises(L.SoupError) as e:
        plan.prefetch(0)
    assert e.value.status == 7
    plan.prefetch(0)  # the next one works
    plan.wait_host(0, 10000)
    plan.free()


def test_timing_events_stay_bounded_and_totals_survive_the_ring():
    """1,200 prefetch / wait / release cycles (more than four laps of the
    256-entry timing rings): the plan holds at most 1,024 events, and the
    statistics still count every copy and wait, with totals no smaller
    than those of the first 200 cycles."""
    nb = 1 << 12
    blobs = _blobs(3, nb)
    plan = L.Plan(blobs, nb, 2)
    n = 1200
    for i in range(n):
        item = i % 3
        plan.prefetch(item)
        plan.wait(item)
        plan.release(item)
        if i == 199:
            torch.cuda.synchronize()
            early = plan.stats()
    torch.cuda.synchronize()
    s = plan.stats()
    assert plan.timing_events() <= 1024
    assert s["copies"] + s["reuses"] == n and s["waits"] == n
    assert s["bytes_copied"] == s["copies"] * nb
    assert s["copy_ms"] >= early["copy_ms"] and s["stall_ms"] >= early["stall_ms"]
    plan.reset_stats()
    assert plan.stats()["waits"] == 0 and plan.stats()["copy_ms"] == 0.0
    plan.free()


def test_timing_totals_after_a_reset_count_only_new_pairs():
    """After soup_stream_stats_reset the rings still hold a lap of older
    event pairs; the totals of the next few copies must not include them:
    20 copies of 1 MiB after the reset take about 20/600 of the 600 copies
    before it (the copies are identical), not twice that."""
    nb = 1 << 20
    plan = L.Plan(_blobs(3, nb), nb, 2)

    def cycles(n):
        for i in range(n):
            item = i % 3
            plan.prefetch(item)
            plan.wait(item)
            plan.release(item)
        torch.cuda.synchronize()

    cycles(600)
    before = plan.stats()
    plan.reset_stats()
    cycles(20)
    after = plan.stats()
    assert after["copies"] == 20 and after["waits"] == 20
    expect = before["copy_ms"] * 20 / 600
    assert 0.5 * expect <= after["copy_ms"] <= 1.6 * expect, (after["copy_ms"], expect)
    plan.free()


def test_gemm_bounded_wait_runs_out_and_the_context_survives():
    """The producer of a one-CTA tcgen05 GEMM is told to skip its arrivals and
    the kernel's mbarrier waits are limited to 2e6 SM cycles (~1 ms): the MMA
    warp's wait runs out, the kernel records code 1 in the device error word
    and returns (no MMA, tensor memory freed, output untouched).  The same
    device then runs the GEMM normally, and it matches a float64 reference."""
    g = torch.Generator(device="cuda").manual_seed(3)
    M, N, K = 256, 128, 192
    A = torch.randn(M, K, device="cuda", generator=g).bfloat16()
    B = torch.randn(N, K, device="cuda", generator=g).bfloat16()
    C = torch.full((M, N), 7.0, device="cuda")
    assert L.device_error() == 0
    t0 = time.time()
    L.soup_debug_gemm_bounded_wait(A, B, C, wait_limit_cycles=2_000_000, skip_producer_arrivals=True)
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert L.device_error() == 1
    assert torch.all(C == 7.0)  # nothing was written
    L.soup_debug_gemm_bounded_wait(A, B, C, wait_limit_cycles=2_000_000, skip_producer_arrivals=False)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref = A.double() @ B.double().T
    err = (C.double() - ref).norm() / ref.norm()
    assert err < 1e-4, float(err)
