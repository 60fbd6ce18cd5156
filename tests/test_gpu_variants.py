"""GPU parity of the projection-block variants the RoM page compares RoM
with: independently routed MoE on Conv, Gate and Out (Knowl 4, a router per
projection) and RoM (Gate, Out) with a dense Conv projection (Knowl 3).
Every routing is compared bit-exactly with the oracle's, the block output
within the bf16 / float32 bars of the other parity tests. Calls go through the
C ABI (rom_route, rom_dispatch, rom_expert_proj with ROM_PROJ_SLOTS,
rom_combine)."""
import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import WORKLOADS, make_block_inputs, \
    make_workload_inputs
from oracle import rom_oracle as orc
from parity_util import assert_close, assert_routing_matches, to_dev, to_np, weights_to_dev

pytestmark = pytest.mark.gpu


def _spec(variant, inp):
    """Which router drives which projection, and which are r-weighted."""
    if variant == "independent":
        return ({"conv": inp["w_r"], "gate": inp["w_r_gate"], "out": inp["w_r_out"]},
                {"conv": True, "gate": True, "out": True})
    if variant == "gate_out":
        return ({"conv": None, "gate": inp["w_r"], "out": inp["w_r"]},
                {"conv": False, "gate": False, "out": True})
    if variant == "conv_only":  # independent MoE on Conv alone (Knowl 4, first row)
        return ({"conv": inp["w_r"], "gate": None, "out": None},
                {"conv": True, "gate": False, "out": False})
    if variant == "gate_and_out":  # independent MoE on Gate and Out (Knowl 4)
        return ({"conv": None, "gate": inp["w_r_gate"], "out": inp["w_r_out"]},
                {"conv": False, "gate": True, "out": True})
    if variant == "rom":
        return ({"conv": inp["w_r"], "gate": inp["w_r"], "out": inp["w_r"]},
                {"conv": False, "gate": False, "out": True})
    raise ValueError(variant)


def _run(inp, variant, k, renorm, dtype):
    routers, weighted = _spec(variant, inp)
    dense = {n: routers[n] is None for n in routers}
    w = {"conv": inp["w_conv"], "gate": inp["w_gate"], "out": inp["w_out"]}
    w = {n: (a[:1] if dense[n] else a) for n, a in w.items()}
    ref = orc.variant_block_forward(inp["x"], w["conv"], w["gate"], w["out"], k, routers,
                                    weighted, bias=inp.get("bias"), renorm=renorm)
    dev_r = {}
    for n, r in routers.items():  # the same array -> the same device tensor (shared routing)
        if r is not None and id(r) not in dev_r:
            dev_r[id(r)] = to_dev(r, "f32")
    d_routers = {n: (None if r is None else dev_r[id(r)]) for n, r in routers.items()}
    out = rom.variant_block_forward(
        to_dev(inp["x"], dtype), d_routers, weighted, weights_to_dev(w["conv"], dtype),
        weights_to_dev(w["gate"], dtype), weights_to_dev(w["out"], dtype), k, renorm=renorm,
        bias=None if inp.get("bias") is None else to_dev(inp["bias"], "f32"))
    torch.cuda.synchronize()
    assert rom.rom_get_status() == rom.ROM_OK
    for n, r in routers.items():
        if r is None:
            continue
        rb = next(b for key, b in out.routings.items() if key == id(d_routers[n]))
        assert_routing_matches(rb.topk_idx.cpu().numpy(),
                               rb.topk_w.cpu().numpy().astype(np.float64), ref["routing"][n],
                               x=inp["x"], w_r=r, bias=inp.get("bias"))
    return out, ref


CASES = [
    # variant, T, Dm, De, E, k, renorm, dtype
    ("independent", 1500, 256, 256, 8, 1, False, "bf16"),   # SM-pair GEMMs
    ("independent", 600, 256, 384, 8, 1, False, "bf16"),    # swap-AB GEMMs (<= 1024 rows)
    ("independent", 1100, 256, 256, 8, 2, True, "bf16"),
    ("independent", 300, 64, 128, 8, 1, False, "f32"),
    ("independent", 257, 64, 96, 5, 2, True, "f32"),
    ("gate_out", 1500, 256, 256, 8, 1, False, "bf16"),
    ("gate_out", 700, 256, 256, 8, 2, True, "bf16"),
    ("gate_out", 300, 64, 128, 8, 1, False, "f32"),
    ("conv_only", 1300, 256, 256, 4, 1, False, "bf16"),
    ("gate_and_out", 1300, 256, 256, 4, 1, False, "bf16"),
    ("rom", 1500, 256, 256, 8, 1, False, "bf16"),
    ("rom", 900, 256, 256, 8, 2, True, "bf16"),
]


@pytest.mark.parametrize("variant,T,Dm,De,E,k,renorm,dtype", CASES)
def test_variant_matches_oracle(variant, T, Dm, De, E, k, renorm, dtype):
    inp = make_block_inputs(T, Dm, De, E, seed=T + De + E, dtype=dtype, router_std=0.05,
                            extra_routers=True)
    out, ref = _run(inp, variant, k, renorm, dtype)
    assert_close(to_np(out.out), ref["O"], dtype, f"{variant} O", magnitude_scaled_abs=True)


def test_rom_through_the_variant_path_equals_the_fused_block():
    """One shared router with RoM's weighting, run as separate Conv and Gate
    projections and a gate combine, agrees with the fused RoM block (same
    routing bit for bit; outputs within bf16 rounding of each other)."""
    T, Dm, De, E = 2000, 256, 256, 8
    inp = make_block_inputs(T, Dm, De, E, seed=4, router_std=0.05, extra_routers=True)
    out, ref = _run(inp, "rom", 1, False, "bf16")
    d = {n: weights_to_dev(inp[n], "bf16") for n in ("w_conv", "w_gate", "w_out")}
    fused = rom.block_forward(to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"), None,
                              d["w_conv"], d["w_gate"], d["w_out"], k=1)
    torch.cuda.synchronize()
    rb = next(iter(out.routings.values()))
    assert torch.equal(rb.topk_idx, fused.routing.topk_idx)
    assert torch.equal(rb.sorted_slot[:T], fused.routing.sorted_slot[:T])
    assert_close(to_np(out.out), to_np(fused.out), "bf16", "variant vs fused",
                 magnitude_scaled_abs=True)


@pytest.mark.parametrize("name", ["independent_moe_16k", "rom_gate_out_16k"])
def test_variant_workload_full_size(name):
    """The prefill-shaped comparison workloads at full size: every token's
    routing exact for every router, and the whole block output."""
    wl = WORKLOADS[name]
    inp = make_workload_inputs(wl)
    out, _ = _run_full(inp, wl)
    routers, weighted = _spec(wl.variant, inp)
    dense = {n: routers[n] is None for n in routers}
    w = {"conv": inp["w_conv"], "gate": inp["w_gate"], "out": inp["w_out"]}
    w = {n: (a[:1] if dense[n] else a) for n, a in w.items()}
    ref = orc.variant_block_forward(inp["x"], w["conv"], w["gate"], w["out"], wl.k, routers,
                                    weighted)
    assert_close(to_np(out.out), ref["O"], wl.dtype, f"{name} O (whole)")


def _run_full(inp, wl):
    """Like _run, but the routing of every token is checked against the
    oracle's router alone (the full-size block output is sampled)."""
    routers, weighted = _spec(wl.variant, inp)
    dense = {n: routers[n] is None for n in routers}
    w = {"conv": inp["w_conv"], "gate": inp["w_gate"], "out": inp["w_out"]}
    w = {n: (a[:1] if dense[n] else a) for n, a in w.items()}
    dev_r = {}
    for n, r in routers.items():
        if r is not None and id(r) not in dev_r:
            dev_r[id(r)] = to_dev(r, "f32")
    d_routers = {n: (None if r is None else dev_r[id(r)]) for n, r in routers.items()}
    out = rom.variant_block_forward(
        to_dev(inp["x"], wl.dtype), d_routers, weighted, weights_to_dev(w["conv"], wl.dtype),
        weights_to_dev(w["gate"], wl.dtype), weights_to_dev(w["out"], wl.dtype), wl.k)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == rom.ROM_OK
    for n, r in routers.items():
        if r is None:
            continue
        rb = out.routings[id(d_routers[n])]
        rt = orc.route(inp["x"], r, wl.k)
        amb = assert_routing_matches(rb.topk_idx.cpu().numpy(),
                                     rb.topk_w.cpu().numpy().astype(np.float64), rt, x=inp["x"],
                                     w_r=r)
        assert amb == 0
    return out, None
