"""The tcgen05 GEMM (tensor-core linear) against the oracle.

The linear of the LLAISYS report's operator list ("linear", Y = X W^T + b)
and the two epilogues the model fuses into it (SwiGLU over interleaved
gate/up rows, residual add).  Sizes span several 128-feature and BN-token
tiles with ragged tails in every dimension, K not a multiple of the 64-wide
k-block, and the token tile widths 64, 128, 192 and 256 the kernel picks by
M and by how full the last wave of tiles is (192 wherever it cuts the
wave-quantised work by a tenth: most of the shapes below from M = 257 up;
the 4096-token chunks keep 256 for q/k/v and take 192 for o and down).
"""
import pytest
import torch

import oracle
import qwen2_decode_step_b200 as q2
from synth import normal
from tol import assert_close, assert_op_close, bits_equal

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    pass


def cuda(t):
    return None if t is None else t.to("cuda")


@pytest.mark.parametrize("M,N,K", [
    (64, 128, 64),        # one tile of each, BN = 64
    (100, 200, 136),      # ragged M, N and K (K % 64 = 8)
    (128, 384, 1536),     # BN = 128, Qwen2 hidden K
    (300, 1000, 520),     # BN = 256 with a partial token tile, ragged N
    (512, 2048, 1536),    # the q/k/v projection of a 512-token prefill
    (512, 1536, 8960),    # the down projection, long K
])
@pytest.mark.parametrize("bias", [False, True])
@pytest.mark.parametrize("split", [False, True])
def test_tc_gemm_plain_bf16(M, N, K, bias, split):
    x = normal((M, K), 1.0, 101, "bf16")
    w = normal((N, K), 0.02, 102, "bf16")
    b = normal((N,), 0.01, 103, "bf16") if bias else None
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q2.q2_test_tc_gemm(out, cuda(x), cuda(w), cuda(b), split=split)
    assert_op_close(out, oracle.linear(x, w, b), f"tc gemm {M}x{N}x{K} split={split}")


# The prefill chunk's products at full size, on sampled rows: both sides of
# every 192- and 256-token tile edge the rows cross, and the last tile (4096
# = 21 x 192 + 64: a partial 192-token tile).
ROWS_4096 = [0, 1, 127, 128, 191, 192, 255, 256, 383, 384, 2047, 2048, 3839, 3840, 4031, 4032, 4095]


@pytest.mark.parametrize("N,K", [
    (2048, 1536),   # q/k/v: 256 tiles of 256 tokens (two full waves)
    (1536, 1536),   # o: 264 tiles of 192 tokens (192 of 256 would leave the second wave a third full)
    (1536, 8960),   # down
])
def test_tc_gemm_prefill_chunk_4096_sampled_rows(N, K):
    M = 4096
    x = normal((M, K), 1.0, 171, "bf16")
    w = normal((N, K), 0.02, 172, "bf16")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q2.q2_linear(out, cuda(x), cuda(w))
    rows = torch.tensor(ROWS_4096)
    assert_op_close(out.cpu()[rows], oracle.linear(x[rows], w, None), f"tc gemm {M}x{N}x{K} sampled rows")


def test_tc_gemm_split_k_is_deterministic():
    """Split-K partials are added in split order: repeated calls agree bit for bit."""
    M, N, K = 64, 1536, 8960
    x = cuda(normal((M, K), 1.0, 161, "bf16"))
    w = cuda(normal((N, K), 0.02, 162, "bf16"))
    outs = []
    for _ in range(3):
        out = torch.empty((M, N), dtype=torch.float32, device="cuda")
        q2.q2_test_tc_gemm(out, x, w, split=True)
        outs.append(out)
    assert bits_equal(outs[0], outs[1]) and bits_equal(outs[0], outs[2])


@pytest.mark.parametrize("M,N,K", [(64, 256, 1536), (257, 640, 1536)])
def test_tc_gemm_plain_f32_out(M, N, K):
    x = normal((M, K), 1.0, 111, "bf16")
    w = normal((N, K), 0.02, 112, "bf16")
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q2.q2_test_tc_gemm(out, cuda(x), cuda(w))
    ref = oracle.linear(x, w, None, out_dtype=torch.float32)
    # bf16 products are exact in fp32; what is left is the fp32 summation
    # order of 1536 terms (relative error ~ K * 2^-24 at worst, far below this)
    assert_close(out, ref, 1e-4, f"tc gemm fp32 out {M}x{N}x{K}")


def test_tc_gemm_one_hot_is_exact():
    """A one-hot row of x selects a column of W exactly (no rounding on the way)."""
    M, N, K = 64, 256, 1536
    w = normal((N, K), 1.0, 121, "bf16")
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    for m in range(M):
        x[m, (37 * m) % K] = 1.0
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q2.q2_test_tc_gemm(out, cuda(x), cuda(w))
    assert bits_equal(out, oracle.linear(x, w, None))


@pytest.mark.parametrize("M", [64, 200, 512])
def test_tc_gemm_swiglu_epilogue(M):
    """Interleaved gate/up rows: out = silu(gate) * up, each rounded to bf16 first."""
    I, K = 320, 1536
    x = normal((M, K), 1.0, 131, "bf16")
    wg = normal((I, K), 0.02, 132, "bf16")
    wu = normal((I, K), 0.02, 133, "bf16")
    w = torch.stack([wg, wu], dim=1).reshape(2 * I, K)  # row 2j gate j, 2j + 1 up j
    out = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    q2.q2_test_tc_gemm(out, cuda(x), cuda(w), epilogue="swiglu", split=M == 64)
    ref = oracle.swiglu(oracle.linear(x, wg), oracle.linear(x, wu))
    # Two operators in one kernel: the gate and up values are each rounded to
    # bf16 from an fp32 (not fp64) sum, so either may land one bf16 ulp away
    # from the oracle's (2^-7 relative at worst), and SwiGLU then rounds once
    # more: the composed bound is twice the single-operator 1e-2.
    assert_close(out, ref, 2e-2, f"tc gemm swiglu M={M}")


@pytest.mark.parametrize("M", [64, 300])
def test_tc_gemm_residual_epilogue(M):
    N, K = 1536, 8960
    x = normal((M, K), 1.0, 141, "bf16")
    w = normal((N, K), 0.02, 142, "bf16")
    r = normal((M, N), 1.0, 143, "bf16")
    out = cuda(r.clone())
    q2.q2_test_tc_gemm(out, cuda(x), cuda(w), epilogue="resid", split=M == 64)
    ref = oracle.add(r, oracle.linear(x, w))
    # Two operators in one kernel (linear rounded to bf16, then the add): the
    # linear's rounding may differ by one ulp from the oracle's, so the
    # composed bound is twice the single-operator 1e-2.
    assert_close(out, ref, 2e-2, f"tc gemm residual M={M}")


def test_linear_entry_point_takes_the_tensor_core_path_at_prefill_sizes():
    """q2_linear at M >= 64 runs the tcgen05 kernel; its result matches the oracle."""
    M, N, K = 96, 256, 1536
    x = normal((M, K), 1.0, 151, "bf16")
    w = normal((N, K), 0.02, 152, "bf16")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q2.q2_linear(out, cuda(x), cuda(w))
    assert_op_close(out, oracle.linear(x, w, None), "q2_linear tensor-core path")
