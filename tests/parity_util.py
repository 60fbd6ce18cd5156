"""Helpers of the parity tests: move seeded inputs to the GPU in the library's
layout and compare CUDA results with the CPU oracle.

Tolerances (the floating-point bar of the parity tests):
  * routing indices, counts, offsets and the permutation: bit-exact;
  * routing weights r: relative 2e-5. r = exp(l_e - m) / sum, so its
    relative error is about twice the absolute error of the logits, and a
    float32 logit (d_model products accumulated in float32) carries up to
    ~1e-5 of rounding at d_model of a few thousand -- the selection itself
    stays exact (near ties are re-decided in float64);
  * bf16 outputs: max abs error <= 2e-2 and relative Frobenius error <= 5e-3
    against the float64 oracle. The full-size workloads are held to exactly
    that. The synthetic test shapes and the bf16 intermediate h can reach
    magnitudes |v| > 4, where rounding a value to bf16 alone moves it by up
    to 2^-9 |v| (> 8e-3); for them the absolute bound is
    max(2e-2, 2^-7 max|reference|) -- two bf16 half-ulps of the largest
    value -- and the relative Frobenius bound stays 5e-3;
  * float32 outputs: relative Frobenius error <= 1e-5 and max abs error
    <= 1e-5 * max(1, max |reference|).
"""
from __future__ import annotations

import numpy as np
import torch

from mixture_experts_projections_b200.inputs import bf16_bits

BF16_MAX_ABS = 2e-2
BF16_REL_FRO = 5e-3
F32_REL = 1e-5
TOPK_W_RTOL = 2e-5


def to_dev(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """float32 numpy (bf16-exact when dtype == "bf16") -> torch tensor."""
    if a is None:
        return None
    if dtype == "bf16":
        bits = torch.from_numpy(bf16_bits(a).view(np.int16).copy())
        return bits.view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def weights_to_dev(w_pages: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """[E, K, N] in the pages' notation -> [E, N, K] contiguous on the device."""
    t = to_dev(w_pages, dtype, device)
    return t.transpose(1, 2).contiguous()


def block_to_dev(inp: dict, dtype: str, device="cuda") -> dict:
    return dict(
        x=to_dev(inp["x"], dtype, device),
        w_r=to_dev(inp["w_r"], "f32", device),
        bias=None if inp.get("bias") is None else to_dev(inp["bias"], "f32", device),
        w_conv=weights_to_dev(inp["w_conv"], dtype, device),
        w_gate=weights_to_dev(inp["w_gate"], dtype, device),
        w_out=weights_to_dev(inp["w_out"], dtype, device),
    )


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    d = got - ref
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def assert_close(got, ref, dtype: str, what: str, magnitude_scaled_abs: bool = False):
    max_abs, rel = errors(got, ref)
    if dtype == "bf16":
        bound = BF16_MAX_ABS
        if magnitude_scaled_abs and np.size(ref):
            bound = max(BF16_MAX_ABS, 2.0 ** -7 * float(np.max(np.abs(ref))))
        assert max_abs <= bound and rel <= BF16_REL_FRO, \
            f"{what}: max abs {max_abs:.3e} (<= {bound:.3e}), rel Frobenius {rel:.3e} (<= {BF16_REL_FRO})"
    else:
        scale = max(1.0, float(np.max(np.abs(ref)))) if np.size(ref) else 1.0
        assert rel <= F32_REL and max_abs <= F32_REL * scale, \
            f"{what}: max abs {max_abs:.3e}, rel Frobenius {rel:.3e} (<= {F32_REL})"
    return max_abs, rel


def assert_routing_matches(gpu_idx: np.ndarray, gpu_w: np.ndarray, rt: dict, band=1e-9):
    """Exact index equality; tokens whose oracle decision margin is below
    `band` (numerically ambiguous in float64) may differ only to another
    valid choice. Returns the number of such ambiguous tokens."""
    ref_idx = rt["topk_idx"]
    ambiguous = rt["margin"] <= band
    mism = np.any(gpu_idx != ref_idx, axis=1)
    bad = mism & ~ambiguous
    assert not np.any(bad), (f"{int(bad.sum())} tokens routed differently, first at "
                             f"{np.nonzero(bad)[0][:5]}: gpu {gpu_idx[bad][:3]} ref {ref_idx[bad][:3]}")
    for t in np.nonzero(mism & ambiguous)[0]:
        lg = rt["logits"][t]
        chosen = lg[gpu_idx[t]]
        assert np.all(np.diff(chosen) <= band), "ambiguous token: slots not in descending order"
    ok = ~mism
    np.testing.assert_allclose(gpu_w[ok], rt["topk_w"][ok], rtol=TOPK_W_RTOL, atol=1e-7)
    return int(ambiguous.sum())
