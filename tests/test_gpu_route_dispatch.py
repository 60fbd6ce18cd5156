"""GPU parity of the router and the dispatch against the oracle (bit-exact
indices, counts, offsets and permutation). Calls go through the C ABI."""
import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import make_block_inputs
from oracle import rom_oracle as orc
from parity_util import assert_routing_matches, to_dev, to_np

pytestmark = pytest.mark.gpu

ROUTE_CASES = [
    # T, Dm, E, k, renorm, dtype, router_std
    (256, 64, 8, 1, False, "f32", 0.02),
    (1000, 256, 8, 1, False, "bf16", 0.02),
    (1000, 256, 8, 2, True, "bf16", 0.05),
    (777, 512, 16, 2, True, "bf16", 0.02),
    (300, 128, 4, 1, False, "bf16", 0.1),
    (129, 2048, 8, 1, False, "bf16", 0.02),
    (300, 1024, 64, 4, False, "bf16", 0.05),  # router weight read from global memory
    (513, 128, 33, 3, True, "f32", 0.2),
    (200, 256, 1, 1, False, "bf16", 0.02),
    (1, 64, 5, 2, False, "f32", 0.3),
    # above the small-batch limit (1024 tokens): the chunk-per-CTA routers
    (2100, 512, 8, 1, False, "bf16", 0.02),
    (1500, 512, 16, 2, True, "bf16", 0.02),
    (1300, 256, 4, 1, False, "bf16", 0.1),
    (1200, 256, 8, 2, False, "f32", 0.05),
    # small batches with 16 experts, float32 data, a 64-token decode shape
    (64, 4096, 4, 1, False, "bf16", 0.02),
    (333, 512, 16, 2, True, "f32", 0.05),
]


def run_route(x, w_r, bias, E, k, renorm):
    T = x.shape[0]
    bufs = rom.RoutingBuffers(T, x.shape[1], E, k, x.dtype, x.device)
    rom.rom_route(x, w_r, bias, k, renorm, bufs.topk_idx, bufs.topk_w, bufs.counts, bufs.ws)
    return bufs


@pytest.mark.parametrize("T,Dm,E,k,renorm,dtype,std", ROUTE_CASES)
def test_route_matches_oracle(T, Dm, E, k, renorm, dtype, std):
    inp = make_block_inputs(T, Dm, 1, E, seed=T + Dm + E, dtype=dtype, router_std=std)
    rt = orc.route(inp["x"], inp["w_r"], k, renorm=renorm)
    b = run_route(to_dev(inp["x"], dtype), to_dev(inp["w_r"], "f32"), None, E, k, renorm)
    torch.cuda.synchronize()
    idx = b.topk_idx.cpu().numpy()
    amb = assert_routing_matches(idx, b.topk_w.cpu().numpy().astype(np.float64), rt)
    assert amb == 0
    assert np.array_equal(b.counts.cpu().numpy(), np.bincount(idx.reshape(-1), minlength=E))


def test_route_with_bias_and_empty_expert():
    T, Dm, E = 700, 256, 8
    inp = make_block_inputs(T, Dm, 1, E, seed=3)
    bias = np.zeros(E, np.float32)
    bias[0], bias[3] = 0.8, -50.0  # expert 3 never chosen
    rt = orc.route(inp["x"], inp["w_r"], 2, bias=bias)
    b = run_route(to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"), to_dev(bias, "f32"), E, 2,
                  False)
    idx = b.topk_idx.cpu().numpy()
    assert_routing_matches(idx, b.topk_w.cpu().numpy().astype(np.float64), rt)
    assert b.counts.cpu().numpy()[3] == 0


@pytest.mark.parametrize("k,renorm", [(1, False), (2, False), (2, True)])
def test_route_zero_router_tie_rule(k, renorm):
    """W_r = 0: all logits tie exactly; the lower expert index wins."""
    T, Dm, E = 300, 128, 6
    inp = make_block_inputs(T, Dm, 1, E, seed=9, zero_router=True)
    b = run_route(to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"), None, E, k, renorm)
    assert np.array_equal(b.topk_idx.cpu().numpy(), np.tile(np.arange(k), (T, 1)))
    np.testing.assert_allclose(b.topk_w.cpu().numpy(), (1.0 / k) if renorm else 1.0 / E,
                               rtol=1e-6)


@pytest.mark.parametrize("T", [512, 2048])
def test_route_near_ties_are_decided_exactly(T):
    """Two router columns that differ by a tiny perturbation give float32
    logit gaps below the float32 rounding bound; the kernel must fall back to
    float64 and agree with the oracle on every token (T = 512: the per-token
    router; T = 2048: the streaming router)."""
    Dm, E = 1024, 4
    inp = make_block_inputs(T, Dm, 1, E, seed=17)
    w = inp["w_r"].copy()
    rng = np.random.default_rng(5)
    w[:, 1] = w[:, 0] + np.float32(3e-7) * rng.standard_normal(Dm).astype(np.float32)
    w[:, 2] = w[:, 0] * np.float32(0.5)
    w[:, 3] = -w[:, 0]
    rt = orc.route(inp["x"], w, 1)
    assert np.mean(rt["margin"] < 1e-4) > 0.3  # many tokens are near-ties in float32 terms
    b = run_route(to_dev(inp["x"], "bf16"), to_dev(w, "f32"), None, E, 1, False)
    amb = assert_routing_matches(b.topk_idx.cpu().numpy(),
                                 b.topk_w.cpu().numpy().astype(np.float64), rt)
    assert amb == 0


DISPATCH_CASES = [
    # T, Dm, E, k, dtype
    (1000, 256, 8, 1, "bf16"),
    (1000, 256, 8, 2, "bf16"),
    (333, 512, 16, 3, "bf16"),
    (256, 64, 8, 1, "f32"),
    (129, 128, 5, 1, "f32"),
    (4096, 128, 64, 8, "bf16"),
]


@pytest.mark.parametrize("T,Dm,E,k,dtype", DISPATCH_CASES)
def test_dispatch_matches_oracle(T, Dm, E, k, dtype):
    inp = make_block_inputs(T, Dm, 1, E, seed=T * k + E, dtype=dtype, router_std=0.3)
    x = to_dev(inp["x"], dtype)
    bufs = rom.route_and_dispatch(x, to_dev(inp["w_r"], "f32"), None, E, k, False)
    torch.cuda.synchronize()
    idx = bufs.topk_idx.cpu().numpy()
    d = orc.dispatch(idx, E)
    R = T * k
    assert np.array_equal(bufs.offsets.cpu().numpy(), d["offsets"])
    assert np.array_equal(bufs.sorted_slot.cpu().numpy()[:R], d["sorted_slot"])
    assert np.array_equal(bufs.slot_pos.cpu().numpy()[:R], d["slot_pos"])
    src = torch.from_numpy(d["sorted_slot"] // k).long().to(x.device)
    assert torch.equal(bufs.x_sorted[:R], x[src])


def test_dispatch_is_deterministic():
    T, Dm, E, k = 2000, 256, 8, 2
    inp = make_block_inputs(T, Dm, 1, E, seed=1, router_std=0.3)
    x = to_dev(inp["x"], "bf16")
    w_r = to_dev(inp["w_r"], "f32")
    a = rom.route_and_dispatch(x, w_r, None, E, k, True)
    b = rom.route_and_dispatch(x, w_r, None, E, k, True)
    for n in ("topk_idx", "topk_w", "offsets", "sorted_slot", "slot_pos", "x_sorted"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n
