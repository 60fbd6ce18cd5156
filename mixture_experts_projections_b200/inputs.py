"""Seeded synthetic inputs for the RoM projection block.

This module only draws random numbers and rounds them to the storage type.
It holds none of the block's arithmetic, so both the CUDA path and the CPU
oracle can take their inputs from it without sharing any computation.

Recipe (the same for every workload):
  * one ``numpy.random.default_rng(seed)`` stream, standard normals drawn in
    float32 in the fixed order X, W_r, W_conv, W_gate, W_out, then dO
    (for the Swimba in-projection workload: X, W_r, W);
  * X ~ N(0, 1); router W_r ~ N(0, 0.02^2); expert weights ~ N(0, 1/fan_in)
    with fan_in = the contraction length of that matrix (d_model for the Conv,
    Gate and Swimba in-projections, d_inner for Out); dO ~ N(0, 1);
  * bf16 workloads round X, the expert weights and dO to bf16 (round to
    nearest, ties to even); the router weight stays float32;
  * expert weights are returned in the paper's notation: W_conv, W_gate and
    the Swimba W as [E, d_model, d_out] (x W), W_out as [E, d_inner, d_model].

Everything is returned as float32 numpy arrays whose values are exactly
representable in the storage type, so upcasting them is exact.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    """One synthetic workload of the RoM projection block."""

    name: str
    kind: str  # "block" (Conv/Gate/Out) or "inproj" (Swimba X|B|C in-projection)
    T: int  # tokens
    Dm: int  # d_model
    De: int  # d_inner (block) or output width of the in-projection
    E: int  # experts
    k: int  # experts selected per token
    dtype: str  # "bf16" or "f32"
    renorm: bool = False  # renormalise the selected probabilities
    router_std: float = 0.02
    # additive router bias: tuple of (expert, value); empty means no bias
    bias: tuple = field(default_factory=tuple)
    backward: bool = False
    # Swimba stream widths (X, B, C) when kind == "inproj"
    streams: tuple = field(default_factory=tuple)
    # kind == "variant": "independent" (a router per projection, each
    # projection a conventional MoE layer) or "gate_out" (dense Conv, one
    # router shared by Gate and Out)
    variant: str = ""
    # the dense core (conv + selective scan) between the projections instead
    # of the identity, over sequences of seq_len tokens (0: one sequence)
    core: bool = False
    seq_len: int = 0
    # the core's x and dt projections expertized too ("RoM (Conv, Gate, dt,
    # x, Out)")
    core_routed: bool = False


# Router-bias constants of the load-imbalanced workload. They were found by
# bisection on the seed-0 inputs with oracle/make_imbalance_bias.py so that
# about 40 % of the tokens pick expert 0 and expert 7 receives about
# 1.5 % (seed-0 load: 40.0 % on expert 0, 1.5 % on expert 7).
IMBALANCE_BIAS_E0 = 0.6279296875
IMBALANCE_BIAS_E7 = -0.5830078125

WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", "block", T=256, Dm=64, De=128, E=8, k=1, dtype="f32"),
    "prefill_16k": Workload("prefill_16k", "block", T=16384, Dm=2048, De=4096, E=8, k=1,
                            dtype="bf16"),
    "imbalanced_8x4096": Workload(
        "imbalanced_8x4096", "block", T=8 * 4096, Dm=1024, De=2048, E=8, k=1, dtype="bf16",
        bias=((0, IMBALANCE_BIAS_E0), (7, IMBALANCE_BIAS_E7))),
    "decode_swimba_inproj": Workload(
        "decode_swimba_inproj", "inproj", T=64, Dm=4096, De=8192 + 8 * 128 + 8 * 128, E=4, k=1,
        dtype="bf16", streams=(8192, 8 * 128, 8 * 128)),
    "top2_fwd_bwd": Workload("top2_fwd_bwd", "block", T=32768, Dm=2560, De=5120, E=16, k=2,
                             dtype="bf16", renorm=True, backward=True),
    # The prefill shapes with the comparison configurations of the pages:
    # independent routing of Conv, Gate and Out, and RoM (Gate, Out).
    "independent_moe_16k": Workload("independent_moe_16k", "variant", T=16384, Dm=2048, De=4096,
                                    E=8, k=1, dtype="bf16", variant="independent"),
    "rom_gate_out_16k": Workload("rom_gate_out_16k", "variant", T=16384, Dm=2048, De=4096, E=8,
                                 k=1, dtype="bf16", variant="gate_out"),
    # The prefill block with the dense core between the projections.
    "prefill_16k_core": Workload("prefill_16k_core", "block", T=16384, Dm=2048, De=4096, E=8,
                                 k=1, dtype="bf16", core=True, seq_len=16384),
    "prefill_16k_core_dtx": Workload("prefill_16k_core_dtx", "block", T=16384, Dm=2048, De=4096,
                                     E=8, k=1, dtype="bf16", core=True, seq_len=16384,
                                     core_routed=True),
}

# Sizes of the core: state size, convolution taps and the rank of the dt
# projection (d_model / 16, rounded up to a multiple of 8).
CORE_STATE = 16
CORE_TAPS = 4

# The order the workloads are listed in (the small fp32 case first).
WORKLOAD_ORDER = ["tiny_fp32", "prefill_16k", "imbalanced_8x4096", "decode_swimba_inproj",
                  "top2_fwd_bwd", "independent_moe_16k", "rom_gate_out_16k"]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # finite inputs only: the largest finite pattern + 0x8000 stays below 2^32
    r = (u >> 16) & 1
    r += 0x7FFF
    r += u
    r &= 0xFFFF0000
    return r.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns (uint16) of float32 values that are bf16-exact."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _draw(rng, shape, std, bf16):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return round_to_bf16(a) if bf16 else a


def bias_vector(E: int, bias_items) -> np.ndarray | None:
    """The additive router bias as a float32 [E] vector, or None."""
    if not bias_items:
        return None
    b = np.zeros(E, dtype=np.float32)
    for e, v in bias_items:
        b[e] = np.float32(v)
    return b


def make_block_inputs(T, Dm, De, E, *, seed=0, dtype="bf16", router_std=0.02, bias=None,
                      with_dout=False, zero_router=False, extra_routers=False):
    """Inputs of the Conv/Gate/Out block in the paper's notation.

    Returns a dict with x [T,Dm], w_r [Dm,E] (float32), bias [E] or None,
    w_conv and w_gate [E,Dm,De], w_out [E,De,Dm] and, if asked, dout [T,Dm].
    With ``extra_routers`` two more router weights w_r_gate and w_r_out
    [Dm,E] are drawn last (after everything above), so the other arrays are
    those of the same seed without them.
    """
    bf = dtype == "bf16"
    rng = np.random.default_rng(seed)
    x = _draw(rng, (T, Dm), 1.0, bf)
    w_r = _draw(rng, (Dm, E), router_std, False)
    if zero_router:
        w_r[:] = 0.0
    w_conv = _draw(rng, (E, Dm, De), 1.0 / np.sqrt(Dm), bf)
    w_gate = _draw(rng, (E, Dm, De), 1.0 / np.sqrt(Dm), bf)
    w_out = _draw(rng, (E, De, Dm), 1.0 / np.sqrt(De), bf)
    out = dict(x=x, w_r=w_r, bias=None if bias is None else np.asarray(bias, np.float32),
               w_conv=w_conv, w_gate=w_gate, w_out=w_out)
    if with_dout:
        out["dout"] = _draw(rng, (T, Dm), 1.0, bf)
    if extra_routers:
        out["w_r_gate"] = _draw(rng, (Dm, E), router_std, False)
        out["w_r_out"] = _draw(rng, (Dm, E), router_std, False)
    return out


def make_inproj_inputs(T, Dm, N_out, E, *, seed=0, dtype="bf16", router_std=0.02):
    """Inputs of the Swimba in-projection: x [T,Dm], w_r [Dm,E], w [E,Dm,N_out]."""
    bf = dtype == "bf16"
    rng = np.random.default_rng(seed)
    x = _draw(rng, (T, Dm), 1.0, bf)
    w_r = _draw(rng, (Dm, E), router_std, False)
    w = _draw(rng, (E, Dm, N_out), 1.0 / np.sqrt(Dm), bf)
    return dict(x=x, w_r=w_r, bias=None, w=w)


def core_dt_rank(Dm: int) -> int:
    """Rank of the dt projection: ceil(d_model / 16), rounded up to a multiple of 8."""
    r = -(-Dm // 16)
    return max(8, -(-r // 8) * 8)


def make_core_params(De, Dm, *, seed=0, N=CORE_STATE, K=CORE_TAPS, experts=None):
    """Parameters of the dense core for d_inner = De (float32 numpy, in the
    pages' x W notation), from their own generator (seeded by (seed, 1)) so
    the block's other inputs do not change:
      conv_w [De, K] ~ N(0, 1/K), conv_b [De] ~ N(0, 0.1^2),
      w_x [De, R + 2N] ~ N(0, 1/De) and w_dt [R, De] ~ N(0, 1/R), both
      rounded to bf16 (the library's projection dtype), R = core_dt_rank(Dm),
      b_dt [De] ~ U[ln 1e-3, ln 1e-1] (softplus then gives delta of about
      1e-3 .. 1e-1), a_log [De, N] ~ U[0, 3], d [De] ~ U[0.5, 1.5].
    With ``experts`` = E, w_x and w_dt hold one matrix per expert
    ([E, De, R + 2N] and [E, R, De]: the x and dt projections expertized)."""
    rng = np.random.default_rng([seed, 1])
    R = core_dt_rank(Dm)
    lead = () if experts is None else (experts,)
    return dict(
        conv_w=_draw(rng, (De, K), 1.0 / np.sqrt(K), False),
        conv_b=_draw(rng, (De,), 0.1, False),
        w_x=_draw(rng, lead + (De, R + 2 * N), 1.0 / np.sqrt(De), True),
        w_dt=_draw(rng, lead + (R, De), 1.0 / np.sqrt(R), True),
        b_dt=rng.uniform(np.log(1e-3), np.log(1e-1), De).astype(np.float32),
        a_log=rng.uniform(0.0, 3.0, (De, N)).astype(np.float32),
        d=rng.uniform(0.5, 1.5, De).astype(np.float32))


def make_workload_inputs(wl: Workload, seed=0):
    """Inputs of a named workload at its full size."""
    T = wl.T
    if wl.kind == "inproj":
        return make_inproj_inputs(T, wl.Dm, wl.De, wl.E, seed=seed, dtype=wl.dtype,
                                  router_std=wl.router_std)
    inp = make_block_inputs(T, wl.Dm, wl.De, wl.E, seed=seed, dtype=wl.dtype,
                            router_std=wl.router_std, bias=bias_vector(wl.E, wl.bias),
                            with_dout=wl.backward, extra_routers=wl.variant == "independent")
    if wl.core:
        inp["core"] = make_core_params(wl.De, wl.Dm, seed=seed,
                                       experts=wl.E if wl.core_routed else None)
    return inp

