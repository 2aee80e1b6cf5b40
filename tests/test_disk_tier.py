"""The disk tier's shard reader on the host (no GPU): plain page-aligned
staging buffers and no CUDA call (the reader opened without SOUP_DISK_PINNED).

A consumer here follows the stream plan's slot policy with its own small LRU
ring (n_slots slots, least recently used first): a visit whose layer is in
the ring is served without a copy, any other visit acquires the layer's
staging buffer, checks every byte against the shard file and releases it.
The reader must hand out exactly the copied visits, in order, with no read
wasted, and keep handing out correct bytes when the consumer strays from the
schedule."""
import ctypes
import os
import time

import numpy as np
import pytest

from layer_streamed_qlora_b200 import _lib as L

LAYER_BYTES = 2 * (8 << 20) + 4096 + 256  # three I/O requests, the last one ragged


@pytest.fixture(scope="module")
def shards(tmp_path_factory):
    d = tmp_path_factory.mktemp("shards")
    paths, data = [], []
    rng = np.random.default_rng(0)
    for l in range(6):
        b = rng.integers(0, 256, LAYER_BYTES, dtype=np.uint8).tobytes()
        p = d / f"layer_{l:03d}.bin"
        p.write_bytes(b)
        paths.append(str(p))
        data.append(b)
    return paths, data


def _open(paths, read_ahead=2, n_slots=2, io_threads=3, direct=False):
    return L.Disk(paths, LAYER_BYTES, read_ahead=read_ahead, n_slots=n_slots, io_threads=io_threads, pinned=False,
                  direct=direct)


def _consume(disk, data, visits, n_slots):
    """Visits layers in order through an LRU slot ring; returns the number of copies."""
    ring, copies = [], 0
    for l in visits:
        if l in ring:
            ring.remove(l)
        else:
            host, ev = disk.acquire(l, timeout_ms=5000)
            assert ev is None
            assert ctypes.string_at(host, LAYER_BYTES) == data[l], f"layer {l}: wrong bytes"
            disk.release(l)
            copies += 1
        ring.append(l)
        if len(ring) > n_slots:
            ring.pop(0)
    return copies


def _sft_order(n):
    return list(range(n)) + list(range(n - 1, -1, -1))


@pytest.mark.parametrize("read_ahead,n_slots", [(1, 2), (2, 2), (3, 4), (8, 2)])
def test_reads_exactly_the_copied_visits(shards, read_ahead, n_slots):
    paths, data = shards
    disk = _open(paths, read_ahead, n_slots)
    try:
        order = _sft_order(len(paths))
        disk.schedule(order)
        copies = _consume(disk, data, order * 3, n_slots)  # three training steps
        n = len(paths)
        assert copies == (2 * n - n_slots) + 2 * (2 * n - 2 * n_slots)  # first step, then steady state
        st = disk.stats()
        assert st["acquires"] == copies and st["reads"] >= copies and st["skipped"] == 0
        assert st["reads"] - copies <= read_ahead  # only read-ahead of the next step is in flight
        assert st["bytes_read"] == st["reads"] * LAYER_BYTES
    finally:
        disk.close()


def test_dpo_two_pass_order(shards):
    # reference forward, policy forward, backward: three visits per layer
    paths, data = shards
    n = len(paths)
    order = list(range(n)) * 2 + list(range(n - 1, -1, -1))
    disk = _open(paths, 2, 2)
    try:
        disk.schedule(order)
        copies = _consume(disk, data, order * 2, 2)
        assert copies == (3 * n - 2) + (3 * n - 4)
        assert disk.stats()["skipped"] == 0
    finally:
        disk.close()


def test_consumer_off_schedule_still_gets_the_right_bytes(shards):
    # schedule says forward + backward, the consumer runs forward-only passes
    # and then a shuffled order: visits it passes over are dropped, every
    # acquired buffer still holds the requested layer
    paths, data = shards
    n = len(paths)
    disk = _open(paths, 2, 2)
    try:
        disk.schedule(_sft_order(n))
        _consume(disk, data, list(range(n)) * 3, 2)
        _consume(disk, data, [3, 0, 5, 1, 4, 2, 2, 0, 5], 2)
        assert disk.stats()["skipped"] > 0
    finally:
        disk.close()


@pytest.mark.parametrize("read_ahead,n_slots", [(2, 4), (8, 8)])
def test_every_layer_fits_the_ring(shards, read_ahead, n_slots):
    # (8, 8): more staging buffers than copied visits, so the reader runs out
    # of visits to read in the same pass that queues the first reads; those
    # reads must still start
    paths, data = shards
    disk = _open(paths[:3], read_ahead, n_slots)
    try:
        order = _sft_order(3)
        time.sleep(0.2)  # let the I/O threads go idle first: the queued reads must wake them
        disk.schedule(order)
        assert _consume(disk, data, order * 4, n_slots) == 3  # read once, resident afterwards
        assert disk.stats()["reads"] == 3
    finally:
        disk.close()


def test_direct_reads_when_the_file_system_takes_them(shards):
    paths, data = shards
    disk = _open(paths, 2, 2, direct=True)
    try:
        order = _sft_order(len(paths))
        disk.schedule(order)
        _consume(disk, data, order * 2, 2)
        assert 0 <= disk.stats()["direct_files"] <= len(paths)
    finally:
        disk.close()


def test_acquire_times_out_when_no_buffer_can_be_filled(shards):
    paths, data = shards
    disk = _open(paths, 1, 2)
    try:
        disk.schedule(_sft_order(len(paths)))
        host, _ = disk.acquire(0)
        with pytest.raises(L.SoupError) as e:
            disk.acquire(1, timeout_ms=300)  # the only staging buffer is still held
        assert e.value.status == 6  # SOUP_ERR_TIMEOUT
        disk.release(0)
        host, _ = disk.acquire(1)  # released: the reader goes on
        assert ctypes.string_at(host, LAYER_BYTES) == data[1]
        disk.release(1)
    finally:
        disk.close()


def test_refusals(shards, tmp_path):
    paths, data = shards
    with pytest.raises(L.SoupError) as e:
        L.Disk(paths[:2] + [str(tmp_path / "missing.bin")], LAYER_BYTES, pinned=False)
    assert e.value.status == 8  # SOUP_ERR_IO
    short = tmp_path / "short.bin"
    short.write_bytes(b"\0" * 4096)
    with pytest.raises(L.SoupError) as e:
        L.Disk([paths[0], str(short)], LAYER_BYTES, pinned=False)
    assert e.value.status == 2  # SOUP_ERR_SHAPE
    for ra in (0, 9):
        with pytest.raises(L.SoupError) as e:
            L.Disk(paths, LAYER_BYTES, read_ahead=ra, pinned=False)
        assert e.value.status == 1
    disk = _open(paths[:4], 2, 2)
    try:
        with pytest.raises(L.SoupError):
            disk.acquire(0)  # no schedule yet
        disk.schedule([0, 1, 2, 1, 0])
        with pytest.raises(L.SoupError):
            disk.acquire(3)  # not in the schedule
        with pytest.raises(L.SoupError):
            disk.release(0)  # not held
        disk.acquire(0)
        with pytest.raises(L.SoupError):
            disk.acquire(0)  # already held
        with pytest.raises(L.SoupError):
            disk.schedule([0, 1])  # a buffer is held
        disk.release(0)
        with pytest.raises(L.SoupError):
            disk.schedule([0, 7])  # layer out of range
    finally:
        disk.close()


def test_read_error_is_reported_by_the_acquire(shards, tmp_path):
    # a shard truncated after the reader opened it: the read of that visit
    # fails and its acquire says so; the reader carries on with the others
    paths, data = shards
    p = tmp_path / "shrinks.bin"
    p.write_bytes(data[1])
    disk = _open([paths[0], str(p), paths[2]], 1, 2)
    try:
        os.truncate(p, 8192)
        disk.schedule([0, 1, 2])
        host, _ = disk.acquire(0)
        assert ctypes.string_at(host, LAYER_BYTES) == data[0]
        disk.release(0)
        with pytest.raises(L.SoupError) as e:
            disk.acquire(1)
        assert e.value.status == 8 and b"end of file" in L.lib().soup_last_error()
        host, _ = disk.acquire(2)
        assert ctypes.string_at(host, LAYER_BYTES) == data[2]
        disk.release(2)
    finally:
        disk.close()


def test_randomized_settings_orders_and_idle_threads(tmp_path):
    # seeded random read-ahead / slot / thread counts, O_DIRECT on or off,
    # I/O threads idle or not when the schedule arrives, and consumers that
    # stray from the schedule: every acquired buffer must hold its layer
    import random
    lb = (8 << 20) + 4352  # two requests, the second ragged
    rng = np.random.default_rng(21)
    paths, marks = [], []
    for l in range(7):
        b = rng.integers(0, 256, lb, dtype=np.uint8)
        p = tmp_path / f"r{l}.bin"
        b.tofile(p)
        paths.append(str(p))
        marks.append((b[:64].tobytes(), b[lb // 2:lb // 2 + 64].tobytes(), b[-64:].tobytes()))
    n = len(paths)
    order = _sft_order(n)
    for trial in range(24):
        rnd = random.Random(trial)
        ra, ns, io = rnd.randint(1, 8), rnd.randint(2, 8), rnd.randint(1, 8)
        disk = L.Disk(paths, lb, read_ahead=ra, n_slots=ns, io_threads=io, pinned=False, direct=bool(trial % 2))
        try:
            if trial % 3 == 0:
                time.sleep(0.02)
            disk.schedule(order)
            visits = order * 3
            if trial % 4 == 1:
                visits = visits[:9] + rnd.sample(range(n), n) + visits[9:]
            ring = []
            for l in visits:
                if l in ring:
                    ring.remove(l)
                else:
                    host, _ = disk.acquire(l, timeout_ms=5000)
                    got = (ctypes.string_at(host, 64), ctypes.string_at(host + lb // 2, 64),
                           ctypes.string_at(host + lb - 64, 64))
                    assert got == marks[l], (trial, l)
                    disk.release(l)
                ring.append(l)
                if len(ring) > ns:
                    ring.pop(0)
        finally:
            disk.close()
