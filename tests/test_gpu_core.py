"""GPU parity of the dense core between the projections (rom_ssm_core: the
causal depthwise convolution, SiLU, the x and dt projections, softplus and the
selective scan) and of the RoM block with the core in place of the identity,
against the float64 oracle, through the C ABI.

The library rounds X and dt to bf16 for its two projections (tensor cores),
so Y is held to the bf16 bar (relative Frobenius 5e-3, max abs
max(2e-2, 2^-7 max|ref|)) like the block outputs."""
import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import (WORKLOADS, make_block_inputs,
                                                     make_core_params, make_workload_inputs)
from oracle import rom_oracle as orc
from parity_util import assert_close, block_to_dev, to_np

pytestmark = pytest.mark.gpu

CORE_CASES = [
    # T, De, Dm (sets the dt rank), seq_len, N, K
    (300, 128, 128, 300, 16, 4),     # one sequence, ragged last chunk
    (1000, 256, 256, 250, 16, 4),    # four sequences
    (777, 128, 512, 777, 5, 2),      # small state, two taps
    (2048, 384, 1024, 1024, 16, 4),  # several chunks per sequence, 3 channel blocks
]


@pytest.mark.parametrize("T,De,Dm,L,N,K", CORE_CASES)
def test_core_matches_oracle(T, De, Dm, L, N, K):
    rng = np.random.default_rng(T + De)
    H = rng.standard_normal((T, De)).astype(np.float32)
    p = make_core_params(De, Dm, seed=T, N=N, K=K)
    ref = orc.ssm_core(H, p, seq_len=L)
    core = rom.CoreParams(p)
    h = torch.from_numpy(H).cuda()
    y = torch.empty_like(h)
    ws = rom.core_workspace(T, De, L, core, "cuda")
    rom.rom_ssm_core(h, L, core, y, ws)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == rom.ROM_OK
    assert_close(to_np(y), ref["Y"], "bf16", "core Y", magnitude_scaled_abs=True)
    # in place (y = h) gives the same bits
    rom.rom_ssm_core(h, L, core, h, ws)
    torch.cuda.synchronize()
    assert torch.equal(h, y)


BLOCK_CASES = [
    # T, Dm, De, E, k, renorm, seq_len
    (600, 256, 256, 8, 1, False, 300),
    (1500, 256, 384, 8, 1, False, 1500),   # SM-pair GEMMs, one sequence
    (512, 256, 256, 8, 2, True, 256),
]


@pytest.mark.parametrize("T,Dm,De,E,k,renorm,L", BLOCK_CASES)
def test_block_with_core_matches_oracle(T, Dm, De, E, k, renorm, L):
    inp = make_block_inputs(T, Dm, De, E, seed=T + k, router_std=0.05)
    p = make_core_params(De, Dm, seed=3)
    ref = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], k,
                            renorm=renorm, core=p, seq_len=L)
    d = block_to_dev(inp, "bf16")
    out = rom.block_forward(d["x"], d["w_r"], None, d["w_conv"], d["w_gate"], d["w_out"], k,
                            renorm=renorm, core=rom.CoreParams(p), seq_len=L)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == rom.ROM_OK
    assert np.array_equal(out.routing.topk_idx.cpu().numpy(), ref["topk_idx"])
    assert_close(to_np(out.out), ref["O"], "bf16", "block with core O", magnitude_scaled_abs=True)


def test_prefill_with_core_full_size():
    """The prefill workload with the core (one sequence of 16384 tokens): the
    whole block output against the oracle."""
    wl = WORKLOADS["prefill_16k_core"]
    inp = make_workload_inputs(wl)
    ref = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                            wl.k, core=inp["core"], seq_len=wl.seq_len)
    d = block_to_dev(inp, "bf16")
    out = rom.block_forward(d["x"], d["w_r"], None, d["w_conv"], d["w_gate"], d["w_out"], wl.k,
                            core=rom.CoreParams(inp["core"]), seq_len=wl.seq_len)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == rom.ROM_OK
    assert np.array_equal(out.routing.topk_idx.cpu().numpy(), ref["topk_idx"])
    assert_close(to_np(out.out), ref["O"], "bf16", "prefill_16k_core O (whole)")


ROUTED_CASES = [
    # T, Dm, De, E, k, renorm, seq_len
    (600, 256, 256, 8, 1, False, 300),     # swap-AB GEMMs for the x / dt projections
    (1500, 256, 256, 4, 1, False, 1500),   # SM-pair GEMMs
    (512, 256, 256, 8, 2, True, 256),
]


@pytest.mark.parametrize("T,Dm,De,E,k,renorm,L", ROUTED_CASES)
def test_block_with_expertized_core_matches_oracle(T, Dm, De, E, k, renorm, L):
    """RoM (Conv, Gate, dt, x, Out): the core's x and dt projections follow
    the block's routing."""
    inp = make_block_inputs(T, Dm, De, E, seed=T + 7 * k, router_std=0.05)
    p = make_core_params(De, Dm, seed=4, experts=E)
    ref = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], k,
                            renorm=renorm, core=p, seq_len=L)
    d = block_to_dev(inp, "bf16")
    core = rom.CoreParams(p)
    assert core.routed and core.E == E
    out = rom.block_forward(d["x"], d["w_r"], None, d["w_conv"], d["w_gate"], d["w_out"], k,
                            renorm=renorm, core=core, seq_len=L)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == rom.ROM_OK
    assert np.array_equal(out.routing.topk_idx.cpu().numpy(), ref["topk_idx"])
    assert_close(to_np(out.out), ref["O"], "bf16", "block with expertized core O",
                 magnitude_scaled_abs=True)
