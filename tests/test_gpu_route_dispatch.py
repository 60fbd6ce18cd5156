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
    # more 128-token tiles than SMs: CTAs of the streaming router take a second
    # tile (the weight norms come from the first)
    (20000, 192, 16, 2, True, "bf16", 0.05),
    (19001, 128, 4, 1, False, "bf16", 0.1),
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
    amb = assert_routing_matches(idx, b.topk_w.cpu().numpy().astype(np.float64), rt,
                                 x=inp["x"], w_r=inp["w_r"])
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
    assert_routing_matches(idx, b.topk_w.cpu().numpy().astype(np.float64), rt, x=inp["x"],
                           w_r=inp["w_r"], bias=bias)
    assert b.counts.cpu().numpy()[3] == 0


@pytest.mark.parametrize("k,renorm,T,E", [(1, False, 300, 6), (2, False, 300, 6),
                                           (2, True, 300, 6),
                                           # the streaming router: every token of every
                                           # tile is re-decided in float64, in batches
                                           (1, False, 2100, 8), (2, True, 2100, 16)])
def test_route_zero_router_tie_rule(k, renorm, T, E):
    """W_r = 0: all logits tie exactly; the lower expert index wins."""
    Dm = 128
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
                                 b.topk_w.cpu().numpy().astype(np.float64), rt, x=inp["x"],
                                 w_r=w)
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


def _wide_bound_router(T, Dm, E, dtype, seed):
    """Inputs whose true top expert f = 2 has a weight column of huge norm.

    Features 0 and Dm-1 of every token are 1 and feature 1 is 1. Column a = 0
    is random; column b = 1 equals a except at feature 1, where it is lower by
    about g = 1e-3; column f = 2 equals a except for +B at feature 0, -B at
    feature Dm-1 (B = 2^14; a and b are zero there) and about +d = 5e-4 at
    feature 1. So exactly l_f = l_a + d and l_b = l_a - g: the true order is
    f > a > b, the other experts far below. But |w_f| is ~23000, so f's float32
    logit is accumulated next to partial sums of magnitude 2^14 and can land
    below l_b, while the rounding bound of f is far wider than those of a and
    b. A certification that compares only adjacent ranks then accepts a
    float32 order with f in third place; a sound one re-decides in float64.
    """
    inp = make_block_inputs(T, Dm, 1, E, seed=seed, dtype=dtype, router_std=0.02)
    x = inp["x"].copy()
    x[:, 0] = 1.0
    x[:, 1] = 1.0
    x[:, Dm - 1] = 1.0
    w = inp["w_r"].copy()
    w[0, :] = 0.0
    w[Dm - 1, :] = 0.0
    w[:, 1] = w[:, 0]
    w[1, 1] = w[1, 0] - np.float32(1e-3)
    w[:, 2] = w[:, 0]
    w[1, 2] = w[1, 0] + np.float32(5e-4)
    w[0, 2] = np.float32(16384.0)
    w[Dm - 1, 2] = np.float32(-16384.0)
    w[1, 3:] -= np.float32(10.0)
    return x, w


@pytest.mark.parametrize("T,Dm,E,k,dtype", [
    (512, 1024, 8, 1, "bf16"),    # per-token router (T <= 1024)
    (512, 1024, 8, 2, "bf16"),
    (2048, 1024, 8, 1, "bf16"),   # streaming router (bf16, E in {4, 8, 16})
    (2048, 1024, 16, 2, "bf16"),
    (2048, 1024, 5, 1, "bf16"),   # register-tiled router (other E)
    (2048, 1024, 8, 1, "f32"),    # register-tiled router (float32 data)
    (300, 1024, 8, 2, "f32"),     # per-token router, float32 data
])
def test_route_wide_bound_expert_is_decided_exactly(T, Dm, E, k, dtype):
    """Router columns of very different norms: the top-k certification must
    bound every lower-ranked expert, not only the next one."""
    x, w = _wide_bound_router(T, Dm, E, dtype, seed=T + E + k)
    rt = orc.route(x, w, k)
    assert np.all(rt["topk_idx"][:, 0] == 2)
    # A plain float32 running sum (features in order) ranks f below b for
    # many tokens: the float32 order alone cannot be trusted here.
    acc = np.zeros((T, 3), np.float32)
    for i in range(Dm):
        acc = (acc + x[:, i:i + 1] * w[i, :3]).astype(np.float32)
    assert np.mean(acc[:, 2] < acc[:, 1]) > 0.2
    b = run_route(to_dev(x, dtype), to_dev(w, "f32"), None, E, k, False)
    torch.cuda.synchronize()
    idx = b.topk_idx.cpu().numpy()
    assert np.array_equal(idx, rt["topk_idx"])
    amb = assert_routing_matches(idx, b.topk_w.cpu().numpy().astype(np.float64), rt, x=x, w_r=w)
    assert amb == 0


def _checked_dispatch_outputs(bufs, T, E, k):
    """The dispatch outputs stay in range even when its inputs were refused."""
    R = T * k
    off = bufs.offsets.cpu().numpy().astype(np.int64)
    assert off[0] == 0 and np.all(np.diff(off) >= 0) and off[E] <= R
    for n in ("sorted_slot", "slot_pos"):
        v = getattr(bufs, n).cpu().numpy()[:R]
        assert v.min() >= 0 and v.max() < R, n
    return off


@pytest.mark.parametrize("bad", ["index_minus_one", "index_past_E", "histogram_garbage",
                                 "histogram_negative", "histogram_of_other_tokens"])
def test_dispatch_refuses_inconsistent_routing(bad):
    """rom_dispatch checks the expert indices and the router's histograms
    before it uses them as indices: bad ones are reported as ROM_ERR_ROUTING
    through the status word, every output stays in range, and the next
    correct call works."""
    T, Dm, E, k = 1000, 256, 8, 2
    inp = make_block_inputs(T, Dm, 1, E, seed=21, router_std=0.3)
    x = to_dev(inp["x"], "bf16")
    w_r = to_dev(inp["w_r"], "f32")
    assert rom.rom_get_status() == rom.ROM_OK
    bufs = rom.RoutingBuffers(T, Dm, E, k, x.dtype, x.device)
    rom.rom_route(x, w_r, None, k, False, bufs.topk_idx, bufs.topk_w, bufs.counts, bufs.ws)
    if bad == "index_minus_one":
        bufs.topk_idx[5:300] = -1
    elif bad == "index_past_E":
        bufs.topk_idx[700, 1] = E + 3
    elif bad == "histogram_garbage":
        bufs.ws.fill_(1 << 20)
    elif bad == "histogram_negative":
        bufs.ws[3] = -5
    else:
        other = make_block_inputs(T, Dm, 1, E, seed=22, router_std=0.3)
        ob = rom.RoutingBuffers(T, Dm, E, k, x.dtype, x.device)
        rom.rom_route(to_dev(other["x"], "bf16"), w_r, None, k, False, ob.topk_idx, ob.topk_w,
                      ob.counts, ob.ws)
        bufs.ws.copy_(ob.ws)
    rom.rom_dispatch(x, E, k, bufs.topk_idx, bufs.ws, bufs.offsets, bufs.sorted_slot,
                     bufs.slot_pos, bufs.x_sorted)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == rom.ROM_ERR_ROUTING
    off = _checked_dispatch_outputs(bufs, T, E, k)
    if bad in ("histogram_garbage", "histogram_negative"):
        assert np.all(off == 0)  # no expert gets rows
    # the context is intact and the status word was reset
    good = rom.route_and_dispatch(x, w_r, None, E, k, False)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == rom.ROM_OK
    d = orc.dispatch(good.topk_idx.cpu().numpy(), E)
    assert np.array_equal(good.offsets.cpu().numpy(), d["offsets"])
    assert np.array_equal(good.sorted_slot.cpu().numpy()[:T * k], d["sorted_slot"])
