"""Parity at the full workload sizes, in the launch configuration the bench
times: routing and dispatch are compared with the oracle on every token
(bit-exact), and the whole block output element by element (the top-2
workload's whole output and gradients are in test_gpu_backward.py)."""
import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import WORKLOADS, make_workload_inputs
from oracle import rom_oracle as orc
from parity_util import (assert_close, assert_routing_matches, block_to_dev, to_dev, to_np,
                         weights_to_dev)

pytestmark = pytest.mark.gpu

@pytest.mark.parametrize("name", ["prefill_16k", "imbalanced_8x4096"])
def test_block_workload_full_size(name):
    wl = WORKLOADS[name]
    inp = make_workload_inputs(wl)
    d = block_to_dev(inp, wl.dtype)
    out = rom.block_forward(d["x"], d["w_r"], d["bias"], d["w_conv"], d["w_gate"], d["w_out"],
                            k=wl.k, renorm=wl.renorm)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    rb = out.routing
    rt = orc.route(inp["x"], inp["w_r"], wl.k, bias=inp["bias"], renorm=wl.renorm)
    idx = rb.topk_idx.cpu().numpy()
    amb = assert_routing_matches(idx, rb.topk_w.cpu().numpy().astype(np.float64), rt,
                                 x=inp["x"], w_r=inp["w_r"], bias=inp["bias"])
    assert amb == 0
    dsp = orc.dispatch(idx, wl.E)
    R = wl.T * wl.k
    assert np.array_equal(rb.offsets.cpu().numpy(), dsp["offsets"])
    assert np.array_equal(rb.sorted_slot.cpu().numpy()[:R], dsp["sorted_slot"])
    if name == "imbalanced_8x4096":
        load = np.bincount(idx[:, 0], minlength=wl.E) / wl.T
        assert 0.38 < load[0] < 0.42 and load[7] < 0.02
    ref = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                            k=wl.k, bias=inp["bias"], renorm=wl.renorm)
    assert_close(to_np(out.out), ref["O"], wl.dtype, f"{name} O (whole)")


def test_decode_swimba_inproj_full():
    wl = WORKLOADS["decode_swimba_inproj"]
    inp = make_workload_inputs(wl)
    ref = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=wl.k)
    out, rb = rom.inproj_forward(to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"),
                                 weights_to_dev(inp["w"], "bf16"), k=wl.k)
    torch.cuda.synchronize()
    assert_routing_matches(rb.topk_idx.cpu().numpy(), rb.topk_w.cpu().numpy().astype(np.float64),
                           ref, x=inp["x"], w_r=inp["w_r"])
    assert_close(to_np(out), ref["S"], "bf16", "decode S (whole)")
