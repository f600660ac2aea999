"""Per-operator parity: each CUDA entry point (through the C ABI) against the
CPU oracle on the same seeded inputs, at sizes spanning several tiles with
ragged tails, plus edge cases.  GPU only."""

import math

import pytest
import torch

import oracle
import qwen2_decode_step_b200 as q2
from synth import normal, uniform_ids
from tol import RTOL, assert_op_close, assert_close, bits_equal

pytestmark = pytest.mark.gpu

DTS = ["f32", "bf16"]
TD = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    yield
    torch.cuda.synchronize()


def cuda(t):
    return t.cuda()


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("n", [1, 7, 4096, 1_000_003])
def test_add(dt, n):
    a, b = normal((n,), 1.0, 1, dt), normal((n,), 1.0, 2, dt)
    c = torch.empty_like(cuda(a))
    q2.q2_add(c, cuda(a), cuda(b))
    assert_op_close(c, oracle.add(a, b), "add")


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("n", [5, 8960, 573_447])
def test_swiglu(dt, n):
    g, u = normal((n,), 3.0, 3, dt), normal((n,), 1.0, 4, dt)
    out = torch.empty_like(cuda(g))
    q2.q2_swiglu(out, cuda(g), cuda(u))
    assert_op_close(out, oracle.swiglu(g, u), "swiglu")


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("M,d", [(1, 1536), (3, 128), (17, 1536), (64, 1000)])
def test_rms_norm(dt, M, d):
    x = normal((M, d), 1.0, 5, dt)
    w = normal((d,), 0.05, 6, dt, mean=1.0)
    out = torch.empty_like(cuda(x))
    q2.q2_rms_norm(out, cuda(x), cuda(w), 1e-6)
    assert_op_close(out, oracle.rms_norm(x, w, 1e-6), "rms_norm")


@pytest.mark.parametrize("dt", DTS)
def test_add_rms_norm(dt):
    M, d = 9, 1536
    x, y = normal((M, d), 1.0, 7, dt), normal((M, d), 1.0, 8, dt)
    w = normal((d,), 0.05, 9, dt, mean=1.0)
    r, h = cuda(x).clone(), torch.empty((M, d), dtype=TD[dt], device="cuda")
    q2.q2_add_rms_norm(r, cuda(y), h, cuda(w), 1e-6)
    r_ref = oracle.add(x, y)
    assert_op_close(r, r_ref, "residual")
    assert_op_close(h, oracle.rms_norm(r_ref, w, 1e-6), "norm")


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("ntok,nh,hd", [(5, 12, 128), (33, 2, 128), (4, 4, 32), (3, 1, 2)])
def test_rope(dt, ntok, nh, hd):
    x = normal((ntok, nh, hd), 1.0, 10, dt)
    pos = torch.tensor([0, 1, 4095, 32767, 511] * 7)[:ntok]
    out = torch.empty_like(cuda(x))
    q2.q2_rope(out, cuda(x), cuda(pos), 10000.0)
    assert_op_close(out, oracle.rope(x, pos, 10000.0), "rope")


@pytest.mark.parametrize("dt", DTS)
def test_rope_in_place(dt):
    x = normal((6, 12, 128), 1.0, 11, dt)
    pos = torch.arange(6) * 1000
    y = cuda(x).clone()
    q2.q2_rope(y, y, cuda(pos), 10000.0)
    assert_op_close(y, oracle.rope(x, pos, 10000.0), "rope in place")


@pytest.mark.parametrize("dt", DTS)
def test_embedding_bit_exact(dt):
    V, d = 151936, 1536 if dt == "bf16" else 128
    table = normal((V, d), 0.02, 12, dt)
    ids = torch.cat([torch.tensor([0, V - 1, 5, 5]), uniform_ids(60, V, 13)])
    out = torch.empty((ids.numel(), d), dtype=TD[dt], device="cuda")
    q2.q2_embedding(out, cuda(ids), cuda(table))
    q2.q2_check_device_error()
    assert bits_equal(out, oracle.embedding(ids, table))


def test_embedding_out_of_range_sets_the_error_flag():
    table = normal((100, 64), 1.0, 14, "bf16")
    ids = torch.tensor([3, 100, -1, 7])
    out = torch.full((4, 64), 9.0, dtype=torch.bfloat16, device="cuda")
    q2.q2_embedding(out, cuda(ids), cuda(table))
    with pytest.raises(q2.Q2Error) as e:
        q2.q2_check_device_error()
    assert e.value.status == "Q2_ERR_INDEX"
    ref, rc = oracle.embedding(ids, table, allow_range_error=True)
    assert rc == -2 and bits_equal(out, ref)
    q2.q2_check_device_error()  # the flag was cleared


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("M,N,K,bias", [
    (1, 2048, 1536, True), (1, 1536, 8960, False), (3, 1000, 1536, True), (8, 17920, 1536, False),
    (9, 333, 1536, True), (64, 2048, 1536, True), (130, 1000, 128, False), (1, 1024, 128, False),
])
def test_linear(dt, M, N, K, bias):
    x = normal((M, K), 1.0, 15, dt)
    w = normal((N, K), 0.02, 16, dt)
    b = normal((N,), 0.01, 17, dt) if bias else None
    out = torch.empty((M, N), dtype=TD[dt], device="cuda")
    q2.q2_linear(out, cuda(x), cuda(w), cuda(b) if bias else None)
    assert_op_close(out, oracle.linear(x, w, b), f"linear {M}x{N}x{K}")


def test_linear_one_hot_exact():
    K, N = 1536, 256
    w = normal((N, K), 1.0, 18, "bf16")
    b = normal((N,), 1.0, 19, "bf16")
    x = torch.zeros((2, K), dtype=torch.bfloat16)
    x[0, 5] = 1.0
    x[1, K - 1] = 1.0
    out = torch.empty((2, N), dtype=torch.bfloat16, device="cuda")
    q2.q2_linear(out, cuda(x), cuda(w), cuda(b))
    assert bits_equal(out, oracle.linear(x, w, b))


def _attn_case(dt, S, T, nh, nkv, hd, seed):
    q = normal((S, nh, hd), 1.0, seed, dt)
    k = normal((T, nkv, hd), 1.0, seed + 1, dt)
    v = normal((T, nkv, hd), 1.0, seed + 2, dt)
    out = torch.empty((S, nh, hd), dtype=TD[dt], device="cuda")
    scale = 1.0 / math.sqrt(hd)
    q2.q2_self_attention(out, cuda(q), cuda(k), cuda(v), scale)
    return out, oracle.self_attention(q, k, v, scale)


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("S,T,nh,nkv,hd", [
    (1, 1, 12, 2, 128),        # one position: returns v
    (1, 4096, 12, 2, 128),     # decode row, many splits
    (1, 4097, 12, 2, 128),     # ragged last tile
    (7, 100, 12, 2, 128),      # cache offset
    (65, 65, 12, 2, 128),      # square causal, ragged
    (16, 16, 4, 2, 32),        # tiny-model shape
    (5, 300, 8, 8, 64),        # plain MHA
    (3, 77, 8, 1, 64),         # MQA (group 8)
    (16, 16, 12, 2, 128),      # one warp's rows (bf16: tensor-core prefill kernel)
    (128, 128, 12, 2, 128),    # two full row blocks, square causal
    (100, 612, 12, 2, 128),    # prefill chunk after 512 cached positions, ragged
    (300, 4096, 12, 2, 128),   # long cache, ragged row block and key tile
])
def test_self_attention(dt, S, T, nh, nkv, hd):
    out, ref = _attn_case(dt, S, T, nh, nkv, hd, 20)
    assert_op_close(out, ref, f"attention S={S} T={T}")


@pytest.mark.parametrize("S", [4, 40])  # 40 rows: the tensor-core prefill kernel
def test_self_attention_constant_v_and_future_independence(S):
    T, nh, nkv, hd = 300, 12, 2, 128
    q = normal((S, nh, hd), 2.0, 30, "bf16")
    k = normal((T, nkv, hd), 2.0, 31, "bf16")
    v = torch.ones((T, nkv, hd), dtype=torch.bfloat16)
    out = torch.empty((S, nh, hd), dtype=torch.bfloat16, device="cuda")
    q2.q2_self_attention(out, cuda(q), cuda(k), cuda(v), 1 / math.sqrt(hd))
    assert torch.equal(out.float().cpu(), torch.ones(S, nh, hd))
    # keys after row 0's position (T - S) cannot change row 0, bit for bit
    v2 = normal((T, nkv, hd), 1.0, 32, "bf16")
    k3, v3 = k.clone(), v2.clone()
    k3[T - S + 1:] = 100.0
    v3[T - S + 1:] = -100.0
    a = torch.empty_like(out)
    q2.q2_self_attention(a, cuda(q), cuda(k), cuda(v2), 1 / math.sqrt(hd))
    b = torch.empty_like(out)
    q2.q2_self_attention(b, cuda(q), cuda(k3), cuda(v3), 1 / math.sqrt(hd))
    assert bits_equal(a[:1], b[:1])
    assert not bits_equal(a[1:], b[1:])


@pytest.mark.parametrize("rows,n", [(1, 151936), (64, 151936), (3, 1000), (2, 1)])
def test_argmax_bit_exact(rows, n):
    x = normal((rows, n), 1.0, 40, "f32")
    idx = torch.empty(rows, dtype=torch.int64, device="cuda")
    val = torch.empty(rows, dtype=torch.float32, device="cuda")
    q2.q2_argmax(idx, val, cuda(x))
    ri, rv = oracle.argmax(x)
    assert torch.equal(idx.cpu(), ri) and bits_equal(val, rv)


def test_argmax_ties_nan_and_bf16():
    n = 151936
    x = torch.zeros((4, n))
    x[0, 100] = x[0, 100000] = 3.0          # tie: the lowest index wins
    x[1, n - 1] = 1.0                        # last element
    x[2, 7] = float("nan")                   # NaN wins
    x[2, 9] = float("nan")
    x[3, :] = -1.0                           # all equal -> index 0
    idx = torch.empty(4, dtype=torch.int64, device="cuda")
    q2.q2_argmax(idx, None, cuda(x))
    assert idx.cpu().tolist() == oracle.argmax(x)[0].tolist() == [100, n - 1, 7, 0]
    xb = normal((5, 4097), 1.0, 41, "bf16")
    idx = torch.empty(5, dtype=torch.int64, device="cuda")
    val = torch.empty(5, dtype=torch.bfloat16, device="cuda")
    q2.q2_argmax(idx, val, cuda(xb))
    ri, rv = oracle.argmax(xb)
    assert torch.equal(idx.cpu(), ri) and bits_equal(val, rv)


@pytest.mark.parametrize("es", [1, 2, 4, 8, 16])
def test_rearrange_permutation_bit_exact(es):
    import ctypes
    shape, n = (3, 5, 7, 2), 3 * 5 * 7 * 2
    src = torch.randint(0, 255, (n * es,), dtype=torch.uint8,
                        generator=torch.Generator().manual_seed(es))
    in_str, out_str = (70, 14, 2, 1), (1, 3, 15, 105)  # out[d, c, b, a] = in[a, b, c, d]
    arr = ctypes.c_int64 * 4
    g_src, g_dst = cuda(src), torch.zeros(n * es, dtype=torch.uint8, device="cuda")
    rc = q2.lib().q2_rearrange(g_dst.data_ptr(), g_src.data_ptr(), 4, arr(*shape), arr(*out_str),
                               arr(*in_str), es, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    ref = torch.zeros(n * es, dtype=torch.uint8)
    assert oracle.lib().oracle_rearrange(ref.data_ptr(), src.data_ptr(), 4, arr(*shape),
                                         arr(*out_str), arr(*in_str), es) == 0
    assert torch.equal(g_dst.cpu(), ref)


def test_rearrange_contiguous_fast_path_and_kv_rows():
    cache = torch.zeros((10, 2, 8), dtype=torch.bfloat16)
    k = normal((3, 2, 8), 1.0, 50, "bf16")
    g = cuda(cache.clone())
    q2.q2_rearrange(g[4:7], cuda(k), (3, 2, 8), (16, 8, 1), (16, 8, 1))
    oracle.rearrange(cache[4:7], k, (3, 2, 8), (16, 8, 1), (16, 8, 1))
    assert bits_equal(g, cache)
