"""Edge cases of the block on the GPU, through the C ABI: an empty batch,
a single token, the largest expert and top-k counts the library takes
(E = 64, k = 8), one token per expert, and every token on one expert."""
import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import make_block_inputs
from oracle import rom_oracle as orc
from parity_util import assert_close, assert_routing_matches, block_to_dev, to_np

pytestmark = pytest.mark.gpu


def _bias(E, entries):
    if entries is None:
        return None
    b = np.zeros(E, np.float32)
    for e, v in entries.items():
        b[e] = v
    return b


def _run_and_compare(T, Dm, De, E, k, renorm, bias=None, std=0.05, seed=0):
    inp = make_block_inputs(T, Dm, De, E, seed=seed, router_std=std, bias=_bias(E, bias))
    ref = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                            k=k, bias=inp["bias"], renorm=renorm)
    d = block_to_dev(inp, "bf16")
    out = rom.block_forward(d["x"], d["w_r"], d["bias"], d["w_conv"], d["w_gate"], d["w_out"],
                            k=k, renorm=renorm)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    rb = out.routing
    assert_routing_matches(rb.topk_idx.cpu().numpy(), rb.topk_w.cpu().numpy().astype(np.float64),
                           ref, x=inp["x"], w_r=inp["w_r"], bias=inp["bias"])
    assert_close(to_np(out.out), ref["O"], "bf16", f"O (T={T}, E={E}, k={k})",
                 magnitude_scaled_abs=True)
    return out, ref


def test_empty_batch_enqueues_nothing_and_leaves_zero_offsets():
    """T = 0: every entry point of the forward accepts it; the router's counts
    and the dispatch's offsets are all zero and the status word stays clean."""
    Dm, De, E, k = 128, 128, 8, 2
    x = torch.empty((0, Dm), dtype=torch.bfloat16, device="cuda")
    inp = make_block_inputs(4, Dm, De, E, seed=1)
    d = block_to_dev(inp, "bf16")
    b = rom.RoutingBuffers(0, Dm, E, k, x.dtype, x.device)
    b.offsets.fill_(7)
    b.counts.fill_(5)
    rom.rom_route(x, d["w_r"], None, k, True, b.topk_idx, b.topk_w, b.counts, b.ws)
    rom.rom_dispatch(x, E, k, b.topk_idx, b.ws, b.offsets, b.sorted_slot, b.slot_pos, b.x_sorted)
    uz = torch.empty((2, 1, De), dtype=torch.float32, device="cuda")
    rom.rom_expert_proj(rom.ROM_PROJ_CONV_GATE, b.x_sorted[:0], d["w_conv"], d["w_gate"], E, k,
                        b.offsets, b.sorted_slot, b.topk_w, uz)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    assert torch.equal(b.offsets.cpu(), torch.zeros(E + 1, dtype=torch.int32))
    assert torch.equal(b.counts.cpu(), torch.zeros(E, dtype=torch.int32))


@pytest.mark.parametrize("k,renorm", [(1, False), (2, True)])
def test_single_token(k, renorm):
    _run_and_compare(1, 256, 256, 8, k, renorm, seed=3)


def test_largest_expert_and_topk_counts():
    """E = 64 experts with k = 8 slots per token, renormalised: every token
    reaches 8 experts, most experts get a few dozen rows (ragged tiles)."""
    out, ref = _run_and_compare(300, 128, 128, 64, 8, True, std=0.1, seed=5)
    counts = out.routing.counts.cpu().numpy()
    assert counts.sum() == 300 * 8 and counts.min() > 0


def test_one_token_per_expert():
    """8 tokens, 8 experts, biases that send token t to expert t: every expert
    holds exactly one row (a 256-row tile with 255 rows past its end)."""
    T = E = 8
    Dm = 128  # the bf16 projections take output widths in multiples of 128
    inp = make_block_inputs(T, Dm, 128, E, seed=9, router_std=0.0)
    # x_t = 4 e_t (one-hot on feature t) and W_r = identity columns: logit e = 4 [t == e]
    x = np.zeros((T, Dm), np.float32)
    x[np.arange(T), np.arange(T)] = 4.0
    w_r = np.zeros((Dm, E), np.float32)
    w_r[np.arange(E), np.arange(E)] = 1.0
    inp["x"], inp["w_r"] = x, w_r
    ref = orc.block_forward(x, w_r, inp["w_conv"], inp["w_gate"], inp["w_out"], k=1)
    assert np.array_equal(ref["topk_idx"][:, 0], np.arange(T))
    d = block_to_dev(inp, "bf16")
    out = rom.block_forward(d["x"], d["w_r"], None, d["w_conv"], d["w_gate"], d["w_out"], k=1)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    assert np.array_equal(out.routing.topk_idx.cpu().numpy()[:, 0], np.arange(T))
    assert np.array_equal(out.routing.offsets.cpu().numpy(), np.arange(E + 1))
    assert_close(to_np(out.out), ref["O"], "bf16", "O (one token per expert)",
                 magnitude_scaled_abs=True)


def test_every_token_on_one_expert():
    """A bias of +40 on expert 5: all 2000 tokens go there (one expert's rows
    span many tiles, the other seven are empty), with the streaming router."""
    out, ref = _run_and_compare(2000, 256, 256, 8, 1, False, bias={5: 40.0}, seed=11)
    counts = out.routing.counts.cpu().numpy()
    assert counts[5] == 2000 and counts.sum() == 2000
