"""bench.py reports ncu DRAM traffic only while the kernel sources hash to the ones the counters
were taken on. These checks fail when a kernel source changes and its counters have not been
re-taken (the constants and hashes in bench.py updated together), so a stale figure is never
reported by accident, and a null one never shipped unnoticed."""
import bench


def test_split_kernel_traffic_matches_current_sources():
    t = bench.measured_traffic()
    assert t is not None, "kda_chunk_split.cu / kda_chunk_common.cuh / sm100.cuh changed: re-take its ncu DRAM bytes"
    # read + write of one 8192 x 32 launch: the inputs are the floor, the ring stays in L2
    assert 3.3e8 < t < 4.5e8


def test_decode_side_traffic_matches_current_sources():
    for k in ("decode", "verify", "commit", "commit_verify"):
        t = bench.decode_side_traffic(k)
        assert t is not None, "kda_decode.cu / kda_internal.cuh changed: re-take the decode-side ncu DRAM bytes"
        assert 5.0e8 < t < 1.5e9, (k, t)
