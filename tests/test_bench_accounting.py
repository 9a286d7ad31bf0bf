"""The benchmark's algorithmic byte counts (the numerators of its roofline
fractions), checked against the sums written out term by term from the
workload shapes.  CPU only."""
import bench
from long_context_compressed_06_b200 import workloads as W


def test_decode_step_bytes_per_query_128k():
    wl = W.CSA_DECODE                         # N = 32768 entries, indexer 64 x 128, k = 1024, W = 128, 128 x 512 heads
    keys = 32768 * 128 * 2                    # indexer keys, bf16
    q_idx = 64 * 128 * 2                      # indexer query heads
    w = 64 * 4                                # head weights, fp32
    gather = 1024 * 512 * 2                   # the selected compressed rows
    window = 128 * 512 * 2                    # the sliding-window rows
    q_out = 2 * 128 * 512 * 2                 # query heads in, output heads out
    idx = 1024 * 4                            # selected indices
    per_query = keys + q_idx + w + gather + window + q_out + idx
    assert per_query == 9_851_136
    assert bench.decode_step_bytes(wl) == wl.batch * wl.nq * per_query


def test_index_bytes_bf16_and_fp4():
    wl = W.CSA_DECODE
    per_seq = 32768 * 128 * 2 + 64 * 128 * 2 + 64 * 4 + 32768 * 4      # keys, q_I, w, fp32 scores out
    assert bench.index_bytes(wl) == wl.batch * per_seq == 8 * 8_536_320
    f4 = W.FP4_DECODE                                                     # 262144 entries
    keys4 = 262144 * (128 // 2 + 128 // 16)                              # packed e2m1 + e4m3 block scales
    q4 = 64 * (128 // 2 + 128 // 16)
    assert keys4 == 18_874_368
    assert bench.index_bytes(f4, fp4=True) == f4.batch * (keys4 + q4 + 64 * 4 + 262144 * 4)
