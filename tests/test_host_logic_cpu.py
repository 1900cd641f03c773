"""Host-side logic that needs no GPU: the overlapped sweep's row blocks and the
benchmark's stamped ncu traffic (reported only while the kernel's sources
hash as they did at the capture)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from activation_sparse_gemm_lynx_b200.sweep import LinearSweep  # noqa: E402


def _sweep_of(shapes):
    # work_items reads only each layer's (M, K, N); no device tensors needed
    sw = object.__new__(LinearSweep)
    sw.layers = [{"shape": s} for s in shapes]
    return sw


@pytest.mark.parametrize("M", [1, 255, 256, 384, 4608, 8192, 8193])
@pytest.mark.parametrize("chunks", [1, 2, 3, 4])
def test_row_blocks_cover_each_layer_in_order(M, chunks):
    sw = _sweep_of([(M, 3072, 3072), (M, 12288, 3072)])
    items = sw.work_items(chunks)
    for t in sw.layers:
        blocks = [(r0, r1) for (tt, r0, r1) in items if tt is t]
        assert blocks[0][0] == 0 and blocks[-1][1] == M
        for (a0, a1), (b0, b1) in zip(blocks, blocks[1:]):
            assert a1 == b0
        # every block but the last is a whole number of 256-row CTA-pair tiles
        assert all((r1 - r0) % 256 == 0 for (r0, r1) in blocks[:-1])
        assert all(r1 > r0 for (r0, r1) in blocks)
        assert len(blocks) <= chunks
    # items keep the layers' order
    order = [sw.layers.index(tt) for (tt, _r0, _r1) in items]
    assert order == sorted(order)


def test_one_chunk_is_the_whole_layer():
    sw = _sweep_of([(384, 3072, 9216)])
    assert [(r0, r1) for (_t, r0, r1) in sw.work_items(1)] == [(0, 384)]
    assert [(r0, r1) for (_t, r0, r1) in sw.work_items(2)] == [(0, 256), (256, 384)]


def test_stamped_traffic_follows_the_sources(monkeypatch):
    for kernel in ("gemm", "sparsify"):
        rec = bench.DRAM_TRAFFIC[kernel]
        now = bench.src_hash(bench.KERNEL_SOURCES[kernel])
        for workload in rec["bytes"]:
            value, note = bench.stored_traffic(kernel, workload)
            if rec["src"] == now:
                assert value == rec["bytes"][workload] and rec["src"] in note
            else:
                assert value is None and "stale" in note
        assert bench.stored_traffic(kernel, "no-such-workload")[0] is None
        # a stamp taken on other sources is never reported
        monkeypatch.setitem(bench.DRAM_TRAFFIC, kernel, dict(rec, src="0" * 12))
        for workload in rec["bytes"]:
            value, note = bench.stored_traffic(kernel, workload)
            assert value is None and "stale" in note
