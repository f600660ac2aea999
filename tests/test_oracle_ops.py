"""Pins of the CPU oracle's operators against things other than itself:
library routines (torch in float64, numpy), closed forms, invariants and
brute force on tiny inputs.  CPU only."""

import math

import numpy as np
import pytest
import torch

import oracle
from synth import normal

pytestmark = pytest.mark.filterwarnings("ignore")


def bf16_ulp(x: torch.Tensor) -> torch.Tensor:
    """Spacing of bf16 values around |x| (8 significant bits)."""
    ax = x.abs().double().clamp_min(2.0 ** -126)
    return torch.pow(2.0, torch.floor(torch.log2(ax)) - 7)


# ------------------------------------------------------------- storage types

def test_bf16_rounding_matches_torch_on_float_values():
    g = torch.Generator().manual_seed(7)
    x = torch.randn(200_000, generator=g) * torch.exp(torch.randn(200_000, generator=g) * 8)
    x = torch.cat([x, torch.tensor([0.0, -0.0, 1.0, 3.3895314e38, 3.39e38, 1e-40, -1e-41,
                                    float("inf"), float("-inf")])])
    ours = oracle.round_to(x.double().numpy(), torch.bfloat16)
    ref = x.to(torch.bfloat16)  # torch's RNE cast, a library routine
    assert torch.equal(ours.view(torch.int16), ref.view(torch.int16))


def test_bf16_rounding_ties_go_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: the even neighbour is 1.
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    vals = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 2.0 ** -134,
                     3 * 2.0 ** -134, 2.0 ** 128, (2 - 2.0 ** -8) * 2.0 ** 127])
    got = oracle.round_to(vals, torch.bfloat16).double().numpy()
    want = np.array([1.0, 1 + 2.0 ** -6, -1.0, 0.0, 2 * 2.0 ** -133, np.inf, np.inf])
    assert np.array_equal(got, want)


def test_bf16_rounding_is_direct_not_through_float():
    # A double just above a bf16 tie that float rounding would land exactly on
    # the tie: direct rounding must go up.
    x = 1 + 2.0 ** -8 + 2.0 ** -40
    got = oracle.round_to(np.array([x]), torch.bfloat16).double().item()
    assert got == 1 + 2.0 ** -7


# ---------------------------------------------------------------------- add

@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_add_exact_on_small_integers(dt):
    a = torch.arange(-50, 50, dtype=dt)
    b = torch.arange(100, 0, -1, dtype=dt)
    # (-50 + i) + (100 - i) = 50 for every i
    assert torch.equal(oracle.add(a, b), torch.full((100,), 50.0, dtype=dt))


def test_add_rounds_once():
    a = torch.tensor([1.0], dtype=torch.bfloat16)
    b = torch.tensor([2.0 ** -8], dtype=torch.bfloat16)   # exact sum is a tie -> 1.0
    c = torch.tensor([3 * 2.0 ** -9], dtype=torch.bfloat16)  # 1 + 0.75 ulp -> 1 + ulp
    assert oracle.add(a, b).item() == 1.0
    assert oracle.add(a, c).item() == 1 + 2.0 ** -7


# ------------------------------------------------------------------- argmax

def test_argmax_matches_numpy_and_tie_rule():
    g = torch.Generator().manual_seed(3)
    x = torch.randint(-5, 5, (64, 1000), generator=g).float()  # many ties
    idx, val = oracle.argmax(x)
    assert np.array_equal(idx.numpy(), np.argmax(x.numpy(), axis=1))  # numpy: first max
    assert torch.equal(val, x.max(dim=1).values)


def test_argmax_edges():
    n = 151936
    x = torch.zeros(3, n)
    x[0, 0] = 1.0
    x[1, n - 1] = 1.0
    x[2, 7] = 2.0
    x[2, 9] = 2.0
    idx, _ = oracle.argmax(x)
    assert idx.tolist() == [0, n - 1, 7]
    y = torch.tensor([[1.0, float("nan"), 5.0, float("nan")], [-0.0, 0.0, -1.0, -2.0]])
    idx, _ = oracle.argmax(y)
    assert idx.tolist() == [1, 0]  # first NaN wins; -0 == +0 -> lowest index
    assert idx.tolist() == np.argmax(y.numpy(), axis=1).tolist()


def test_argmax_bf16_single_row():
    x = normal((1, 1000), 1.0, 5, "bf16")
    idx, val = oracle.argmax(x)
    assert idx.item() == int(np.argmax(x.float().numpy()))
    assert val.dtype == torch.bfloat16 and val.item() == x.max().item()


# ---------------------------------------------------------------- embedding

@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_embedding_is_row_gather(dt):
    table = normal((1000, 96), 1.0, 11, "f32" if dt == torch.float32 else "bf16")
    ids = torch.tensor([0, 999, 5, 5, 123])
    out = oracle.embedding(ids, table)
    assert torch.equal(out.view(torch.int16) if dt == torch.bfloat16 else out,
                       table[ids].view(torch.int16) if dt == torch.bfloat16 else table[ids])


def test_embedding_out_of_range_reports_and_zeroes():
    table = torch.ones((10, 4))
    out, rc = oracle.embedding(torch.tensor([1, 10, -1]), table, allow_range_error=True)
    assert rc == -2
    assert out[0].tolist() == [1.0] * 4 and out[1].abs().sum() == 0 and out[2].abs().sum() == 0


# ------------------------------------------------------------------- linear

def test_linear_one_hot_picks_a_column_plus_bias():
    N, K = 37, 53
    w = normal((N, K), 1.0, 21, "f32")
    b = normal((N,), 1.0, 22, "f32")
    for k in (0, 17, K - 1):
        x = torch.zeros(1, K)
        x[0, k] = 1.0
        y = oracle.linear(x, w, b)
        want = (w[:, k].double() + b.double()).float()  # one rounding of an exact sum
        assert torch.equal(y[0], want)


def test_linear_identity_weight_returns_x_plus_b():
    K = 64
    x = normal((5, K), 1.0, 23, "bf16")
    y = oracle.linear(x, torch.eye(K, dtype=torch.bfloat16), None)
    assert torch.equal(y.view(torch.int16), x.view(torch.int16))


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_linear_matches_torch_float64_matmul(dt):
    M, N, K = 7, 129, 300
    x = normal((M, K), 1.0, 24, dt)
    w = normal((N, K), 0.05, 25, dt)
    b = normal((N,), 0.1, 26, dt)
    y = oracle.linear(x, w, b)
    ref = x.double() @ w.double().T + b.double()  # library routine in float64
    tol = bf16_ulp(ref) * 0.5 + 1e-12 if dt == "bf16" else ref.abs() * 2 ** -24 + 1e-12
    assert ((y.double() - ref).abs() <= tol).all()
    # no bias + fp32 output
    y32 = oracle.linear(x, w, None, out_dtype=torch.float32)
    ref32 = (x.double() @ w.double().T)
    assert ((y32.double() - ref32).abs() <= ref32.abs() * 2 ** -24 + 1e-12).all()


# ----------------------------------------------------------------- rms_norm

@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_rms_norm_invariants(dt):
    d = 1536
    x = normal((4, d), 1.0, 31, dt)
    ones = torch.ones(d, dtype=x.dtype)
    y = oracle.rms_norm(x, ones, 1e-6).double()
    # unit RMS output when w = 1
    rms = y.pow(2).mean(dim=1).sqrt()
    assert torch.allclose(rms, torch.ones(4, dtype=torch.float64), atol=3e-3 if dt == "bf16" else 1e-6)
    # scale invariance: with eps = 0 a power-of-two scale is exact end to end;
    # with eps = 1e-6 it holds to about eps / mean(x^2)
    y0 = oracle.rms_norm(x, ones, 0.0).double()
    y8 = oracle.rms_norm((x.double() * 8).to(x.dtype), ones, 0.0).double()
    assert torch.equal(y0, y8)
    y8e = oracle.rms_norm((x.double() * 8).to(x.dtype), ones, 1e-6).double()
    assert torch.allclose(y, y8e, rtol=1e-5 if dt == "f32" else 2 ** -7, atol=0)
    # direction preserved: y is a positive multiple of x
    cos = torch.nn.functional.cosine_similarity(y, x.double(), dim=1)
    assert (cos > 1 - 1e-4).all()


def test_rms_norm_special_cases():
    w = torch.tensor([2.0, -1.0, 0.5, 3.0])
    # all-equal row c: mean(x^2) = c^2, so y = w * c / sqrt(c^2 + eps) -> w * sign(c)
    y = oracle.rms_norm(torch.full((1, 4), -3.0), w, 0.0)
    assert torch.equal(y[0], -w)
    # the zero row stays zero (eps keeps the division finite)
    assert torch.equal(oracle.rms_norm(torch.zeros(1, 4), w, 1e-6)[0], torch.zeros(4))
    # eps sits inside the square root: for x = (e, e, e, e) and eps = 3 e^2,
    # y = w * e / sqrt(4 e^2) = w / 2
    e = 0.25
    y = oracle.rms_norm(torch.full((1, 4), e), w, 3 * e * e)
    assert torch.equal(y[0], w / 2)


# --------------------------------------------------------------------- rope

def test_rope_position_zero_is_identity():
    x = normal((3, 4, 64), 1.0, 41, "f32")
    assert torch.equal(oracle.rope(x, torch.zeros(3, dtype=torch.int64), 10000.0), x)


def test_rope_head_dim_two_is_a_plane_rotation():
    # hd = 2: the only frequency is theta^0 = 1, so the pair (a, b) is the
    # complex number a + ib multiplied by e^{i pos}.
    x = normal((5, 3, 2), 1.0, 42, "f32")
    pos = torch.tensor([0, 1, 2, 100, 32767])
    y = oracle.rope(x, pos, 10000.0)
    z = torch.complex(x[..., 0].double(), x[..., 1].double()) * torch.exp(1j * pos.double())[:, None]
    assert torch.allclose(y[..., 0].double(), z.real, atol=1e-6)
    assert torch.allclose(y[..., 1].double(), z.imag, atol=1e-6)


def test_rope_pairs_are_half_split_with_known_frequency():
    # hd = 4, theta = 10000: frequencies 1 and 10000^(-1/2) = 0.01.
    # pos = 157: second pair angle = 1.57 rad.  A one-hot at j = 1 must move
    # into index j + hd/2 = 3 (half-split pairing), not into index 2.
    x = torch.zeros(1, 1, 4)
    x[0, 0, 1] = 1.0
    y = oracle.rope(x, torch.tensor([157]), 10000.0)[0, 0].double()
    assert abs(y[1] - math.cos(1.57)) < 1e-7 and abs(y[3] - math.sin(1.57)) < 1e-7
    assert y[0] == 0 and y[2] == 0


def test_rope_preserves_pair_norms_and_relative_positions():
    hd = 128
    q = normal((1, 1, hd), 1.0, 43, "f32")
    k = normal((1, 1, hd), 1.0, 44, "f32")
    def rot(x, p):
        return oracle.rope(x, torch.tensor([p]), 10000.0)[0, 0].double()
    for p in (1, 77, 4095):
        y = rot(q, p)
        n0 = q[0, 0, :64].double() ** 2 + q[0, 0, 64:].double() ** 2
        n1 = y[:64] ** 2 + y[64:] ** 2
        assert torch.allclose(n0, n1, rtol=1e-6, atol=1e-7)
    # <rope(q, m), rope(k, n)> depends on m - n only
    d1 = torch.dot(rot(q, 10), rot(k, 3))
    d2 = torch.dot(rot(q, 1010), rot(k, 1003))
    assert abs(d1 - d2) < 1e-4


# ----------------------------------------------------------- self_attention

def _sdpa_reference(q, k, v, scale):
    """torch's scaled_dot_product_attention in float64 with an explicit
    causal mask for a cache offset; GQA by repeating kv heads."""
    S, nh, hd = q.shape
    T, nkv, _ = k.shape
    G = nh // nkv
    qq = q.double().permute(1, 0, 2)
    kk = k.double().repeat_interleave(G, dim=1).permute(1, 0, 2)
    vv = v.double().repeat_interleave(G, dim=1).permute(1, 0, 2)
    pos_q = torch.arange(S) + (T - S)
    mask = torch.arange(T)[None, :] <= pos_q[:, None]
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale)
    return o.permute(1, 0, 2)


@pytest.mark.parametrize("S,T,nh,nkv,hd,dt", [
    (7, 7, 4, 2, 32, "f32"),       # square causal, GQA 2
    (3, 10, 12, 2, 16, "f32"),     # cache offset, GQA 6
    (1, 33, 6, 6, 8, "f32"),       # decode row, plain MHA
    (5, 20, 12, 2, 128, "bf16"),
])
def test_attention_matches_torch_sdpa(S, T, nh, nkv, hd, dt):
    q = normal((S, nh, hd), 1.0, 51, dt)
    k = normal((T, nkv, hd), 1.0, 52, dt)
    v = normal((T, nkv, hd), 1.0, 53, dt)
    scale = 1 / math.sqrt(hd)
    out = oracle.self_attention(q, k, v, scale).double()
    ref = _sdpa_reference(q, k, v, scale)
    if dt == "f32":
        assert torch.allclose(out, ref, rtol=2 ** -23, atol=1e-7)
    else:
        assert ((out - ref).abs() <= bf16_ulp(ref) * 0.5 + 1e-12).all()


def test_attention_single_position_returns_v():
    v = normal((1, 2, 64), 1.0, 54, "bf16")
    q = normal((1, 12, 64), 3.0, 55, "bf16")
    k = normal((1, 2, 64), 3.0, 56, "bf16")
    out = oracle.self_attention(q, k, v)
    want = v.repeat_interleave(6, dim=1)
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))


def test_attention_constant_v_gives_constant_rows():
    q = normal((4, 4, 32), 2.0, 57, "f32")
    k = normal((9, 2, 32), 2.0, 58, "f32")
    v = torch.full((9, 2, 32), 1.0)
    out = oracle.self_attention(q, k, v)
    assert torch.allclose(out.double(), torch.ones_like(out).double(), atol=2 ** -23)


def test_attention_ignores_future_positions_bitwise():
    S, T = 4, 12
    q = normal((S, 4, 32), 1.0, 59, "bf16")
    k = normal((T, 2, 32), 1.0, 60, "bf16")
    v = normal((T, 2, 32), 1.0, 61, "bf16")
    base = oracle.self_attention(q[:1], k[:T - S + 1], v[:T - S + 1])  # row 0 sees keys <= T-S
    k2, v2 = k.clone(), v.clone()
    k2[T - S + 1:] = 100.0
    v2[T - S + 1:] = -100.0
    full = oracle.self_attention(q, k2, v2)
    assert torch.equal(full[:1].view(torch.int16), base.view(torch.int16))


def test_attention_brute_force_loops_tiny():
    # explicit per-(i, h) loops with python floats: masked scores, softmax, sum
    S, T, nh, nkv, hd = 3, 5, 4, 2, 4
    q = normal((S, nh, hd), 1.0, 62, "f32")
    k = normal((T, nkv, hd), 1.0, 63, "f32")
    v = normal((T, nkv, hd), 1.0, 64, "f32")
    out = oracle.self_attention(q, k, v, 0.5)
    for i in range(S):
        for h in range(nh):
            g = h // (nh // nkv)
            vis = range(T - S + i + 1)
            s = [0.5 * sum(float(q[i, h, d]) * float(k[j, g, d]) for d in range(hd)) for j in vis]
            e = [math.exp(x - max(s)) for x in s]
            z = sum(e)
            for d in range(hd):
                want = sum(e[j] / z * float(v[j, g, d]) for j in vis)
                assert abs(float(out[i, h, d]) - want) <= 1e-6 * max(1.0, abs(want))


# ------------------------------------------------------------------- swiglu

@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_swiglu_matches_torch_silu(dt):
    gate = normal((5000,), 3.0, 71, dt)
    up = normal((5000,), 1.0, 72, dt)
    out = oracle.swiglu(gate, up).double()
    ref = torch.nn.functional.silu(gate.double()) * up.double()
    if dt == "f32":
        assert torch.allclose(out, ref, rtol=2 ** -23, atol=1e-30)
    else:
        assert ((out - ref).abs() <= bf16_ulp(ref) * 0.5 + 1e-30).all()


def test_swiglu_special_values():
    gate = torch.tensor([0.0, 80.0, -80.0, -1000.0])
    up = torch.tensor([5.0, 2.0, 2.0, 3.0])
    out = oracle.swiglu(gate, up)
    assert out[0] == 0 and out[1] == 160.0 and abs(out[2]) < 1e-30 and out[3] == 0


# ---------------------------------------------------------------- rearrange

def test_rearrange_transpose_and_round_trip():
    a = torch.arange(2 * 3 * 5, dtype=torch.float32).reshape(2, 3, 5)
    out = torch.empty(5, 3, 2)
    # out[k, j, i] = a[i, j, k]: iterate over a's shape with out's strides permuted
    oracle.rearrange(out, a, (2, 3, 5), (1, 2, 6), (15, 5, 1))
    assert torch.equal(out, a.permute(2, 1, 0))
    back = torch.empty(2, 3, 5)
    oracle.rearrange(back, out, (5, 3, 2), (1, 5, 15), (6, 2, 1))
    assert torch.equal(back, a)


def test_rearrange_bf16_slice_into_cache_rows():
    cache = torch.zeros(10, 2, 8, dtype=torch.bfloat16)
    k = normal((3, 2, 8), 1.0, 81, "bf16")
    view = cache[4:7]
    oracle.rearrange(view, k, (3, 2, 8), (16, 8, 1), (16, 8, 1))
    assert torch.equal(cache[4:7].view(torch.int16), k.view(torch.int16))
    assert cache[:4].abs().sum() == 0 and cache[7:].abs().sum() == 0
