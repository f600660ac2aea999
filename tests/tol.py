"""Tolerances of the parity tests.

Per operator: |gpu - oracle| <= rtol * max(|oracle|, rms(oracle)) element by
element, rtol = 1e-5 for fp32 storage and 1e-2 for bf16 (the rms floor keeps
near-zero elements from failing on absolute noise).  Logits: 1e-4 (fp32) by
the same rule; bf16 logits max-abs <= 5e-2 and cosine >= 0.9995.
Integer / index / byte results: bit-exact.
"""

import torch

RTOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}


def rel_err(got: torch.Tensor, ref: torch.Tensor) -> float:
    g = got.detach().double().cpu()
    r = ref.detach().double().cpu()
    if r.numel() == 0:
        return 0.0
    scale = torch.maximum(r.abs(), r.pow(2).mean().sqrt().expand_as(r))
    err = (g - r).abs()
    ratio = torch.where(scale > 0, err / scale, torch.where(err > 0, torch.inf, 0.0))
    return float(ratio.max())


def assert_close(got: torch.Tensor, ref: torch.Tensor, rtol: float, what: str = ""):
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    e = rel_err(got, ref)
    assert e <= rtol, f"{what}: max scaled error {e:.3e} > {rtol:.1e}"


def assert_op_close(got: torch.Tensor, ref: torch.Tensor, what: str = ""):
    assert_close(got, ref, RTOL[ref.dtype], what)


def assert_bf16_logits(got: torch.Tensor, ref: torch.Tensor, what: str = ""):
    g = got.detach().double().cpu().reshape(-1)
    r = ref.detach().double().cpu().reshape(-1)
    mx = float((g - r).abs().max())
    cos = float(torch.nn.functional.cosine_similarity(g, r, dim=0))
    assert mx <= 5e-2 and cos >= 0.9995, f"{what}: max-abs {mx:.3e}, cosine {cos:.6f}"
    return mx, cos


def bits_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    a, b = a.detach().cpu().contiguous(), b.detach().cpu().contiguous()
    if a.dtype != b.dtype or a.shape != b.shape:
        return False
    if a.dtype in (torch.bfloat16, torch.float16):
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a, b)
