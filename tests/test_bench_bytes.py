"""The bench's algorithmic byte counts (the numerators of every roofline
fraction) against the library's own operand sizes (qgemm_operand_bytes,
independent code in the C ABI), and the MoE suite's routing generator.  CPU
only."""
import numpy as np
import pytest

import bench
import precision_quantized_gemm_b200 as qg


def _operand_bytes(fmt, is_w, rows, K):
    q, s = qg.qgemm_operand_bytes(fmt, is_w, rows, K)
    return q + s


@pytest.mark.parametrize("fmt", [qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_BLOCK_FP8])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (8, 1792, 5120), (32, 5120, 640), (4096, 5120, 5120)])
def test_shape_bytes_equal_operand_sizes_plus_output(fmt, M, N, K):
    want = _operand_bytes(fmt, True, N, K) + _operand_bytes(fmt, False, M, K) + 2 * M * N
    assert bench.shape_bytes(fmt, M, N, K) == want


@pytest.mark.parametrize("M,N,K", [(1, 896, 1024), (64, 1792, 5120), (512, 1280, 8192)])
def test_nvfp4_shape_bytes_are_the_unpadded_operands(M, N, K):
    # the library pads NVFP4 scale atoms to 128 rows x 4 columns; the
    # algorithmic count takes one e4m3 scale per 16 elements and the two
    # fp32 tensor scales, so it is at most the padded size
    padded = _operand_bytes(qg.QG_NVFP4, True, N, K) + _operand_bytes(qg.QG_NVFP4, False, M, K) + 2 * M * N
    algo = bench.shape_bytes(qg.QG_NVFP4, M, N, K)
    assert algo == (N + M) * K // 2 + (N + M) * K // 16 + 8 + 2 * M * N
    assert algo <= padded + 8


def test_decode_step_bytes_follow_the_int8_gemm_and_quantiser():
    for m in bench.MS:
        assert bench.gemm_bytes(m) == bench.shape_bytes(qg.QG_W8A8_INT8, m, bench.N, bench.K)
        assert bench.quant_bytes(m) == 2 * m * bench.K + _operand_bytes(qg.QG_W8A8_INT8, False, m, bench.K)
    assert bench.step_bytes() == sum(bench.gemm_bytes(m) + bench.quant_bytes(m) for m in bench.MS)


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_moe_routing_picks_distinct_experts_per_token(T):
    counts = bench.moe_routing(T, seed=1000 + T)
    assert counts.shape == (bench.MOE_EXPERTS,)
    assert counts.sum() == T * bench.MOE_TOPK
    assert counts.max() <= T                      # an expert at most once per token
    assert np.array_equal(counts, bench.moe_routing(T, seed=1000 + T))


def test_kernel_source_hash_ignores_comments_but_not_code():
    src = "// header\nint f(int x) {  // doubles\n  return 2 * x;\n}\n\n"
    same = "int f(int x) {\n\n  return 2 * x;   // twice\n}\n"
    other = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench.kernel_source_code(src) == bench.kernel_source_code(same)
    assert bench.kernel_source_code(src) != bench.kernel_source_code(other)
    assert len(bench.kernel_source_hash()) == 12


def test_all_cores_oracle_baseline_reassembles_the_single_process_result():
    # the pool splits each oracle GEMM by output-column blocks; the function
    # asserts that the blocks reassemble into the single-process result
    cb = bench.cpu_baseline_all_cores(1)
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
