"""GPU parity of the RoM block backward (renormalised top-k) against the
float64 oracle's exact gradient, through the C ABI.

Gradients: dX (bf16), d(router logits) (float32) and the expert weight
gradients dW_conv, dW_gate, dW_out (float32, in the library's weight layout,
i.e. the pages' matrices transposed). Each is held to the bf16 bar of the
forward outputs, per tensor: relative Frobenius <= 5e-3 and max abs <=
max(2e-2, 2^-7 max|ref|).
"""
import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import WORKLOADS, make_block_inputs, make_workload_inputs
from oracle import rom_oracle as orc
from parity_util import assert_close, block_to_dev, to_dev, to_np

pytestmark = pytest.mark.gpu


def run_fwd_bwd(inp, k, renorm=True):
    d = block_to_dev(inp, "bf16")
    fwd = rom.block_forward(d["x"], d["w_r"], d["bias"], d["w_conv"], d["w_gate"], d["w_out"],
                            k=k, renorm=renorm)
    dout = to_dev(inp["dout"], "bf16")
    bwd = rom.block_backward(fwd, dout, d["w_r"], d["w_conv"], d["w_gate"], d["w_out"],
                             renorm=renorm)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    return fwd, bwd


def check_grads(bwd, ref, tokens=None, experts=None):
    sel = slice(None) if tokens is None else torch.from_numpy(np.asarray(tokens)).cuda()
    assert_close(to_np(bwd.dx[sel]), ref["dX"], "bf16", "dX", magnitude_scaled_abs=True)
    assert_close(to_np(bwd.dlogits[sel]), ref["dlogits"], "bf16", "dlogits",
                 magnitude_scaled_abs=True)
    es = range(bwd.dw_out.shape[0]) if experts is None else experts
    for e in es:
        assert_close(to_np(bwd.dw_conv[e]), ref["dW_in"][e].T, "bf16", f"dW_conv[{e}]",
                     magnitude_scaled_abs=True)
        assert_close(to_np(bwd.dw_gate[e]), ref["dW_g"][e].T, "bf16", f"dW_gate[{e}]",
                     magnitude_scaled_abs=True)
        assert_close(to_np(bwd.dw_out[e]), ref["dW_out"][e].T, "bf16", f"dW_out[{e}]",
                     magnitude_scaled_abs=True)


BWD_CASES = [
    # T, Dm, De, E, k, router_std, bias
    (600, 256, 256, 8, 2, 0.05, None),
    (1000, 512, 256, 16, 2, 0.05, None),
    (333, 256, 512, 6, 3, 0.1, None),
    (257, 256, 256, 8, 2, 0.05, {2: -40.0}),  # one expert without rows
    (300, 256, 256, 64, 8, 0.1, None),        # the largest E and k: 64 experts of ~37 rows
]


@pytest.mark.parametrize("T,Dm,De,E,k,std,bias", BWD_CASES)
def test_backward_matches_oracle(T, Dm, De, E, k, std, bias):
    b = None
    if bias is not None:
        b = np.zeros(E, np.float32)
        for e, v in bias.items():
            b[e] = v
    inp = make_block_inputs(T, Dm, De, E, seed=7 * T + E, router_std=std, bias=b, with_dout=True)
    fwd, bwd = run_fwd_bwd(inp, k)
    ref = orc.block_backward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                             inp["dout"], k=k, bias=inp["bias"], renorm=True)
    assert np.array_equal(fwd.routing.topk_idx.cpu().numpy(), ref["forward"]["topk_idx"])
    check_grads(bwd, ref)
    if bias is not None:
        for e, v in bias.items():
            assert torch.count_nonzero(bwd.dw_out[e]) == 0


def test_backward_is_deterministic():
    inp = make_block_inputs(700, 256, 256, 8, seed=3, router_std=0.05, with_dout=True)
    _, a = run_fwd_bwd(inp, 2)
    snap = {n: getattr(a, n).clone() for n in ("dx", "dlogits", "dw_conv", "dw_gate", "dw_out")}
    _, b = run_fwd_bwd(inp, 2)
    for n, v in snap.items():
        assert torch.equal(v, getattr(b, n)), n


def test_top2_workload_full_size_backward():
    """Full top-2 workload, whole gradients: every token's dX and dlogits,
    every expert's dW_conv, dW_gate and dW_out, and the whole forward O. The
    oracle runs on batches of tokens (a token's forward and its dX, dlogits
    depend on that token only; the weight gradients are sums over tokens, so
    the batches' sums add up to them)."""
    wl = WORKLOADS["top2_fwd_bwd"]
    inp = make_workload_inputs(wl)
    fwd, bwd = run_fwd_bwd(inp, wl.k, wl.renorm)
    E, Dm, De = wl.E, wl.Dm, wl.De
    dX = np.empty((wl.T, Dm))
    dl = np.empty((wl.T, E))
    O = np.empty((wl.T, Dm))
    dW = {n: np.zeros((E, a, b)) for n, a, b in (("dW_in", Dm, De), ("dW_g", Dm, De),
                                                   ("dW_out", De, Dm))}
    step = 4096
    for a in range(0, wl.T, step):
        b = min(wl.T, a + step)
        ref = orc.block_backward(inp["x"][a:b], inp["w_r"], inp["w_conv"], inp["w_gate"],
                                 inp["w_out"], inp["dout"][a:b], k=wl.k, renorm=wl.renorm)
        assert np.array_equal(fwd.routing.topk_idx[a:b].cpu().numpy(),
                              ref["forward"]["topk_idx"])
        dX[a:b], dl[a:b], O[a:b] = ref["dX"], ref["dlogits"], ref["forward"]["O"]
        for n in dW:
            dW[n] += ref[n]
    assert_close(to_np(fwd.out), O, "bf16", "top2 O (whole)")
    assert_close(to_np(bwd.dx), dX, "bf16", "top2 dX (whole)", magnitude_scaled_abs=True)
    assert_close(to_np(bwd.dlogits), dl, "bf16", "top2 dlogits (whole)",
                 magnitude_scaled_abs=True)
    for e in range(E):
        assert_close(to_np(bwd.dw_conv[e]), dW["dW_in"][e].T, "bf16", f"top2 dW_conv[{e}]",
                     magnitude_scaled_abs=True)
        assert_close(to_np(bwd.dw_gate[e]), dW["dW_g"][e].T, "bf16", f"top2 dW_gate[{e}]",
                     magnitude_scaled_abs=True)
        assert_close(to_np(bwd.dw_out[e]), dW["dW_out"][e].T, "bf16", f"top2 dW_out[{e}]",
                     magnitude_scaled_abs=True)


ROUTER_GRAD_CASES = [
    # T, Dm, De, E, k, renorm, bias
    (600, 256, 256, 8, 1, False, None),       # top-1, r = p (the formula of Knowl 1)
    (500, 256, 256, 8, 2, False, None),       # top-2 without renormalisation
    (700, 256, 512, 8, 1, True, None),        # top-1 renormalised: r = 1, dlogits = 0
    (400, 512, 256, 16, 2, True, {3: 0.5}),   # with a router bias
]


@pytest.mark.parametrize("T,Dm,De,E,k,renorm,bias", ROUTER_GRAD_CASES)
def test_backward_without_renormalisation_and_router_weight_gradients(T, Dm, De, E, k, renorm,
                                                                      bias):
    """r = p (no renormalisation) through rom_route_probs and rom_route_bwd,
    top-1 through the forward that keeps u and z, and the router weight
    gradients dW_r, dbias (rom_route_wgrad), all against the oracle."""
    b = None
    if bias is not None:
        b = np.zeros(E, np.float32)
        for e, v in bias.items():
            b[e] = v
    inp = make_block_inputs(T, Dm, De, E, seed=11 * T + k, router_std=0.05, bias=b,
                            with_dout=True)
    d = block_to_dev(inp, "bf16")
    fwd = rom.block_forward(d["x"], d["w_r"], d["bias"], d["w_conv"], d["w_gate"], d["w_out"],
                            k=k, renorm=renorm, keep_uz=True)
    bwd = rom.block_backward(fwd, to_dev(inp["dout"], "bf16"), d["w_r"], d["w_conv"],
                             d["w_gate"], d["w_out"], renorm=renorm, x=d["x"], bias=d["bias"])
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    ref = orc.block_backward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                             inp["dout"], k=k, bias=inp["bias"], renorm=renorm)
    assert np.array_equal(fwd.routing.topk_idx.cpu().numpy(), ref["forward"]["topk_idx"])
    assert_close(to_np(fwd.out), ref["forward"]["O"], "bf16", "O (kept u, z)",
                 magnitude_scaled_abs=True)
    check_grads(bwd, ref)
    assert_close(to_np(bwd.dw_r), ref["dW_r"], "bf16", "dW_r", magnitude_scaled_abs=True)
    assert_close(to_np(bwd.dbias), ref["dbias"], "bf16", "dbias", magnitude_scaled_abs=True)
