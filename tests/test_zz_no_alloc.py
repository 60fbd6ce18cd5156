"""The no-allocation routing entry point, rom_route_dispatch_noalloc.

Callers that cannot allocate device memory (a plugin handed only its host
framework's buffers, or a process whose memory is fully reserved by its own
pool) cannot pass the workspace that rom_route() and rom_dispatch() exchange.
rom_route_dispatch_noalloc keeps that scratch in a fixed device array inside
the library instead. These tests call it through the C ABI, twice in a row
(the array keeps the previous call's contents), and check that it returns
exactly what the two workspace-based calls return: the same kernels run on
the same inputs, so routing indices and weights, counts, offsets,
permutation and gathered rows are bit-identical. They also check that a call
leaves the device's free memory unchanged, and that a sequence of calls of
different sizes and expert counts never sees the previous call's scratch.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import make_block_inputs
from parity_util import to_dev

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


def _assert_same(got, ref, R):
    for n in ("topk_idx", "topk_w", "counts", "offsets"):
        assert torch.equal(got[n], getattr(ref, n)), n
    for n in ("sorted_slot", "slot_pos", "x_sorted"):
        assert torch.equal(got[n], getattr(ref, n)[:R]), n


CASES = [
    # T, Dm, E, k, renorm, dtype
    (1000, 256, 8, 1, False, "bf16"),     # per-token router
    (777, 512, 16, 2, True, "bf16"),
    (300, 64, 5, 2, False, "f32"),        # register-tiled router
    (4096, 2048, 8, 1, False, "bf16"),    # streaming router (32 chunks of histograms)
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
        _assert_same(got, ref, R)
    assert rom.rom_get_status() == rom.ROM_OK


def test_noalloc_sequence_of_sizes_never_reads_stale_scratch():
    """A large call with 16 experts, then smaller ones with 5 and 8 experts,
    then the large one again: each equals the workspace-based calls, although
    the shared array still holds the previous call's histograms."""
    lib = rom.load_library()
    seq = [(3000, 512, 16, 2, True, "bf16"), (500, 256, 5, 1, False, "bf16"),
           (2100, 512, 8, 1, False, "bf16"), (130, 128, 8, 2, False, "f32"),
           (3000, 512, 16, 2, True, "bf16")]
    for i, (T, Dm, E, k, renorm, dtype) in enumerate(seq):
        inp = make_block_inputs(T, Dm, 1, E, seed=100 + i, dtype=dtype, router_std=0.1)
        x = to_dev(inp["x"], dtype)
        w_r = to_dev(inp["w_r"], "f32")
        ref = rom.route_and_dispatch(x, w_r, None, E, k, renorm)
        got = _noalloc_call(lib, x, w_r, None, E, k, renorm)
        torch.cuda.synchronize()
        _assert_same(got, ref, T * k)
        assert rom.rom_get_status() == rom.ROM_OK


def test_noalloc_call_allocates_no_device_memory():
    """After a first call (which loads the kernels and looks up the array's
    address), a call leaves the device's free memory exactly as it was."""
    lib = rom.load_library()
    T, Dm, E, k = 4096, 2048, 8, 1
    inp = make_block_inputs(T, Dm, 1, E, seed=5, router_std=0.1)
    x = to_dev(inp["x"], "bf16")
    w_r = to_dev(inp["w_r"], "f32")
    first = _noalloc_call(lib, x, w_r, None, E, k, False)
    torch.cuda.synchronize()
    out = {n: torch.empty_like(t) for n, t in first.items()}
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    code = lib.rom_route_dispatch_noalloc(
        _p(x), rom.ROM_BF16, T, Dm, _p(w_r), None, E, k, 0, _p(out["topk_idx"]),
        _p(out["topk_w"]), _p(out["counts"]), _p(out["offsets"]), _p(out["sorted_slot"]),
        _p(out["slot_pos"]), _p(out["x_sorted"]),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == rom.ROM_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    for n in first:
        assert torch.equal(out[n], first[n]), n
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
