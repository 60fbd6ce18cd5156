"""The no-allocation routing entry point, rom_route_dispatch_noalloc.

Callers that cannot allocate device memory (a plugin handed only its host
framework's buffers, or a process whose memory is fully reserved by its own
pool) cannot pass the workspace that rom_route() and rom_dispatch() exchange.
rom_route_dispatch_noalloc keeps that scratch in a fixed device array inside
the library instead. These tests call it through the C ABI, twice in a row
(the array keeps the previous call's contents), and check that it returns
exactly what the two workspace-based calls return: bit-identical routing
indices, counts, offsets, permutation and gathered rows, and routing weights
within the routing-weight tolerance of the other parity tests.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import make_block_inputs
from parity_util import TOPK_W_RTOL, to_dev

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc_call(lib, x, w_r, bias, E, k, renorm):
    T, Dm = x.shape
    R = T * k
    out = dict(
        topk_idx=torch.full((T, k), -1, dtype=torch.int32, device="cuda"),
        topk_w=torch.zeros((T, k), dtype=torch.float32, device="cuda"),
        counts=torch.full((E,), -1, dtype=torch.int32, device="cuda"),
        offsets=torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
        sorted_slot=torch.full((R,), -1, dtype=torch.int32, device="cuda"),
        slot_pos=torch.full((R,), -1, dtype=torch.int32, device="cuda"),
        x_sorted=torch.zeros((R, Dm), dtype=x.dtype, device="cuda"),
    )
    code = lib.rom_route_dispatch_noalloc(
        _p(x), rom.ROM_BF16 if x.dtype == torch.bfloat16 else rom.ROM_F32, T, Dm, _p(w_r),
        _p(bias), E, k, int(renorm), _p(out["topk_idx"]), _p(out["topk_w"]), _p(out["counts"]),
        _p(out["offsets"]), _p(out["sorted_slot"]), _p(out["slot_pos"]), _p(out["x_sorted"]),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == rom.ROM_OK, lib.rom_status_string(code)
    return out


CASES = [
    # T, Dm, E, k, renorm, dtype
    (1000, 256, 8, 1, False, "bf16"),
    (777, 512, 16, 2, True, "bf16"),
    (300, 64, 5, 2, False, "f32"),
]


@pytest.mark.parametrize("T,Dm,E,k,renorm,dtype", CASES)
def test_noalloc_matches_workspace_entry_points_on_two_calls(T, Dm, E, k, renorm, dtype):
    lib = rom.load_library()
    inp = make_block_inputs(T, Dm, 1, E, seed=T + E, dtype=dtype, router_std=0.1)
    x = to_dev(inp["x"], dtype)
    w_r = to_dev(inp["w_r"], "f32")
    ref = rom.route_and_dispatch(x, w_r, None, E, k, renorm)
    R = T * k
    for _ in range(2):
        got = _noalloc_call(lib, x, w_r, None, E, k, renorm)
        torch.cuda.synchronize()
        assert torch.equal(got["topk_idx"], ref.topk_idx)
        np.testing.assert_allclose(got["topk_w"].cpu().numpy(), ref.topk_w.cpu().numpy(),
                                   rtol=TOPK_W_RTOL, atol=0)
        assert torch.equal(got["counts"], ref.counts)
        assert torch.equal(got["offsets"], ref.offsets)
        assert torch.equal(got["sorted_slot"], ref.sorted_slot[:R])
        assert torch.equal(got["slot_pos"], ref.slot_pos[:R])
        assert torch.equal(got["x_sorted"], ref.x_sorted[:R])
    assert rom.rom_get_status() == rom.ROM_OK


def test_noalloc_refuses_sizes_beyond_its_scratch():
    """ceil(T / 128) * E above the fixed scratch size is refused before any
    work is enqueued (the pointers are never dereferenced)."""
    lib = rom.load_library()
    fake = ctypes.c_void_p(1 << 20)
    E, T = 64, 128 * 1024 + 1  # 1025 chunks x 64 experts > 65536 entries
    code = lib.rom_route_dispatch_noalloc(fake, rom.ROM_BF16, T, 64, fake, None, E, 1, 0, fake,
                                          fake, None, fake, fake, fake, fake, None)
    assert code == rom.ROM_ERR_WORKSPACE
