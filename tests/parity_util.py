"""Helpers of the parity tests: move seeded inputs to the GPU in the library's
layout and compare CUDA results with the CPU oracle.

Tolerances (the floating-point bar of the parity tests):
  * routing indices, counts, offsets and the permutation: bit-exact;
  * routing weights r: a per-token relative bound derived from the float32
    arithmetic of the routers (``routing_weight_rtol``): twice the largest
    rounding error a float32 logit can carry (gamma_n * sum_i |x_i w_ie|,
    n = the longest accumulation chain of any router), plus the softmax's own
    rounding ((E + 8) u and 2 u times the logit spread, u = 2^-24). It holds
    for every token whatever the router; the largest measured error and its
    ratio to the bound are printed at the end of the run;
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
U32 = 2.0 ** -24  # unit roundoff of float32

# Largest routing-weight errors seen in this run (printed by conftest.py).
ROUTING_WEIGHT_STATS = {"checks": 0, "tokens": 0, "max_rel": 0.0, "max_ratio": 0.0}


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


# Every output comparison of this run: (what, max abs, its bound, rel Frobenius,
# its bound), printed by conftest.py at the end of the run.
PARITY_LOG = []


def assert_close(got, ref, dtype: str, what: str, magnitude_scaled_abs: bool = False):
    max_abs, rel = errors(got, ref)
    if dtype == "bf16":
        bound = BF16_MAX_ABS
        if magnitude_scaled_abs and np.size(ref):
            bound = max(BF16_MAX_ABS, 2.0 ** -7 * float(np.max(np.abs(ref))))
        PARITY_LOG.append((what, max_abs, bound, rel, BF16_REL_FRO))
        assert max_abs <= bound and rel <= BF16_REL_FRO, \
            f"{what}: max abs {max_abs:.3e} (<= {bound:.3e}), rel Frobenius {rel:.3e} (<= {BF16_REL_FRO})"
    else:
        scale = max(1.0, float(np.max(np.abs(ref)))) if np.size(ref) else 1.0
        PARITY_LOG.append((what, max_abs, F32_REL * scale, rel, F32_REL))
        assert rel <= F32_REL and max_abs <= F32_REL * scale, \
            f"{what}: max abs {max_abs:.3e}, rel Frobenius {rel:.3e} (<= {F32_REL})"
    return max_abs, rel


def routing_weight_rtol(x, w_r, bias=None) -> np.ndarray:
    """Per-token bound on |r_gpu - r| / r for the float32 routing weights.

    A float32 logit accumulated over d_model products in a chain of at most n
    roundings is off by at most gamma_n * sum_i |x_i w_ie| (+ u |b_e| for the
    bias add); a token decided on float64 logits carries at most u |l_e| from
    the final cast. Every router's chain is shorter than
    n = d_model / 32 + 32 (per-token router: features per thread + 5 + 8 + 2;
    streaming router: 16 + d_model / 128 + 9, or 8 + d_model / 64 + 9 for
    16 experts; register-tiled router: the lane's slice + 7), and gamma_n
    gets the 1 % slack the kernels use.
    ln r = l_j - logsumexp(l), so logit errors move ln r by at most twice the
    largest one. The softmax itself adds at most (E + 8) u (expf within 2 ulp
    per term, the sum of E positive terms, the division) plus u |l - max l|
    for each of the two exponent arguments.
    """
    x = np.asarray(x, np.float64)
    w = np.asarray(w_r, np.float64)
    E = w.shape[1]
    n = x.shape[1] / 32.0 + 32.0
    gamma = 1.01 * n * U32 / (1.0 - n * U32)
    logits = x @ w
    delta = gamma * (np.abs(x) @ np.abs(w))
    if bias is not None:
        b = np.asarray(bias, np.float64)
        logits = logits + b[None, :]
        delta = delta + U32 * np.abs(b)[None, :]
    delta = delta + 2.0 * U32 * np.abs(logits)
    spread = logits.max(axis=1) - logits.min(axis=1)
    return 2.0 * delta.max(axis=1) + (E + 8) * U32 + 2.0 * U32 * spread


def assert_routing_matches(gpu_idx: np.ndarray, gpu_w: np.ndarray, rt: dict, *, x, w_r,
                           bias=None, band=1e-9):
    """Exact index equality; tokens whose oracle decision margin is below
    `band` (numerically ambiguous in float64) may differ only to another
    valid choice. Routing weights within ``routing_weight_rtol`` of the
    oracle's, token by token. Returns the number of ambiguous tokens."""
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
    ref_w = np.asarray(rt["topk_w"], np.float64)
    rel = np.abs(np.asarray(gpu_w, np.float64) - ref_w) / np.maximum(ref_w, 1e-300)
    bound = routing_weight_rtol(x, w_r, bias)[:, None]
    bad_w = ok[:, None] & (rel > bound)
    assert not np.any(bad_w), (f"routing weights of {int(bad_w.any(axis=1).sum())} tokens exceed "
                               f"the bound: worst rel {rel[bad_w].max():.3e}")
    if np.any(ok):
        st = ROUTING_WEIGHT_STATS
        st["checks"] += 1
        st["tokens"] += int(ok.sum())
        st["max_rel"] = max(st["max_rel"], float(rel[ok].max()))
        st["max_ratio"] = max(st["max_ratio"], float((rel / bound)[ok].max()))
    return int(ambiguous.sum())
