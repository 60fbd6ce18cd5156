"""Host-side checks of the C ABI (no GPU needed): the library builds and loads,
exports every entry point that include/rom.h declares, and rejects invalid
arguments before it enqueues anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from mixture_experts_projections_b200.build import build
    build()
    from mixture_experts_projections_b200 import rom
    return rom.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "rom.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(rom_\w+)\s*\(", text,
                                 flags=re.M)))


def test_header_declares_the_four_block_entry_points():
    names = declared_functions()
    for n in ("rom_route", "rom_dispatch", "rom_expert_proj", "rom_combine"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from mixture_experts_projections_b200 import rom
    names = declared_functions()
    assert names, "no declarations parsed from include/rom.h"
    for n in names:
        assert hasattr(lib, n), f"librom.so does not export {n}"
        assert n in rom.SIGNATURES, f"the Python binding does not declare {n}"


def test_status_strings_and_version(lib):
    assert lib.rom_status_string(0) == b"ROM_OK"
    assert lib.rom_status_string(5) == b"ROM_ERR_TIMEOUT"
    assert lib.rom_status_string(6) == b"ROM_ERR_ROUTING"
    assert lib.rom_status_string(99) == b"ROM_ERR_UNKNOWN"
    assert lib.rom_version() >= 2


def test_workspace_size(lib):
    assert lib.rom_workspace_size(0, 8) == 0
    assert lib.rom_workspace_size(1, 8) == 8 * 4
    assert lib.rom_workspace_size(128, 8) == 8 * 4
    assert lib.rom_workspace_size(129, 8) == 2 * 8 * 4
    assert lib.rom_workspace_size(16384, 8) == 128 * 8 * 4


FAKE = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced by these calls


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), 1), (dict(E=0), 1), (dict(E=65), 1), (dict(k=9, E=16), 1), (dict(k=3, E=2), 1),
    (dict(renorm=2), 1), (dict(Dm=0), 1), (dict(T=-1), 1), (dict(Dm=12), 2), (dict(x=None), 1),
    # a NULL workspace is accepted (no chunk histograms); a short one is not
    (dict(ws_bytes=4), 3), (dict(x=ctypes.c_void_p((1 << 20) + 2)), 2),
])
def test_route_rejects_bad_arguments(lib, kw, code):
    a = dict(x=FAKE, dtype=1, T=256, Dm=64, w_r=FAKE, bias=None, E=8, k=1, renorm=0,
             topk_idx=FAKE, topk_w=FAKE, counts=None, ws=FAKE, ws_bytes=1 << 20, stream=None)
    a.update(kw)
    assert lib.rom_route(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(proj=5), 1), (dict(dtype=2), 1), (dict(K=0), 1), (dict(N=0), 1), (dict(k=2, R=7), 1),
    # ROM_PROJ_SLOTS: a dense projection (no routing arrays) needs E == 1; a
    # routed one needs both offsets and sorted_slot
    (dict(proj=3, offsets=None, sorted_slot=None), 1), (dict(proj=3, offsets=None), 1),
    (dict(proj=3, sorted_slot=None), 1),
    (dict(w1=None), 1), (dict(offsets=None), 1), (dict(N=200), 2), (dict(K=12), 2),
    (dict(out=ctypes.c_void_p((1 << 20) + 8)), 2),
    (dict(proj=1, N=320), 2),
    (dict(proj=1, topk_w=None), 1),
])
def test_expert_proj_rejects_bad_arguments(lib, kw, code):
    a = dict(proj=0, dtype=1, a_sorted=FAKE, R=256, K=64, w0=FAKE, w1=FAKE, N=256, E=8, k=1,
             offsets=FAKE, sorted_slot=FAKE, topk_w=FAKE, out=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_expert_proj(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(mode=3), 1), (dict(dtype=3), 1), (dict(k=0), 1), (dict(k=9), 1), (dict(N=6), 2),
    (dict(inp=None), 1), (dict(mode=2, out=None), 1),
])
def test_combine_rejects_bad_arguments(lib, kw, code):
    a = dict(mode=0, dtype=1, inp=FAKE, T=10, k=2, N=64, slot_pos=FAKE, out=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_combine(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(E=0), 1), (dict(k=3, E=2), 1), (dict(offsets=None), 1), (dict(x_sorted=None), 1),
    (dict(ws_bytes=0), 3), (dict(Dm=4), 2),
])
def test_dispatch_rejects_bad_arguments(lib, kw, code):
    a = dict(x=FAKE, dtype=1, T=300, Dm=64, E=8, k=1, topk_idx=FAKE, ws=FAKE, ws_bytes=1 << 20,
             offsets=FAKE, sorted_slot=FAKE, slot_pos=FAKE, x_sorted=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_dispatch(*a.values()) == code


def test_debug_wait_rejects_out_of_range_limits(lib):
    assert lib.rom_debug_wait_timeout(10, None) == 1
    assert lib.rom_debug_wait_timeout(10 ** 11, None) == 1


def test_binding_fails_loudly_without_library(tmp_path):
    from mixture_experts_projections_b200 import rom
    with pytest.raises(rom.RomError):
        old = rom._lib
        rom._lib = None
        try:
            rom.load_library(str(tmp_path / "missing.so"))
        finally:
            rom._lib = old


# Every case below fails validation, so nothing reaches the device (the
# pointers are never dereferenced).
@pytest.mark.parametrize("kw,code", [
    (dict(k=0), 1), (dict(k=9), 1), (dict(N=0), 1), (dict(T=-1), 1), (dict(N=12), 2),
    (dict(dout=None), 1), (dict(rdo_sorted=ctypes.c_void_p((1 << 20) + 4)), 2),
])
def test_bwd_gather_rejects_bad_arguments(lib, kw, code):
    a = dict(dout=FAKE, T=10, k=2, N=64, sorted_slot=FAKE, topk_w=FAKE, rdo_sorted=FAKE,
             stream=None)
    a.update(kw)
    assert lib.rom_bwd_gather(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(R=255), 1), (dict(E=0), 1), (dict(E=65), 1), (dict(k=9), 1), (dict(Dm=100), 2),
    (dict(De=128), 2), (dict(offsets=None), 1), (dict(g_slots=ctypes.c_void_p((1 << 20) + 4)), 2),
])
def test_bwd_dgrad_out_rejects_bad_arguments(lib, kw, code):
    a = dict(rdo_sorted=FAKE, R=256, Dm=256, w_out=FAKE, De=256, E=8, k=2, offsets=FAKE,
             sorted_slot=FAKE, h_sorted=FAKE, g_slots=FAKE, dr_part=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_bwd_dgrad_out(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), 1), (dict(De=0), 1), (dict(De=6), 2), (dict(uz=None), 1),
    (dict(dhz_sorted=ctypes.c_void_p((1 << 20) + 2)), 2),
])
def test_bwd_gate_rejects_bad_arguments(lib, kw, code):
    a = dict(uz=FAKE, g_slots=FAKE, T=10, k=2, De=64, slot_pos=FAKE, dhz_sorted=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_bwd_gate(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(R=-1), 1), (dict(k=3, E=2), 1), (dict(De=100), 2), (dict(Dm=128), 2),
    (dict(w_g=None), 1), (dict(dx_slots=ctypes.c_void_p((1 << 20) + 4)), 2),
])
def test_bwd_dgrad_in_rejects_bad_arguments(lib, kw, code):
    a = dict(dhz_sorted=FAKE, R=256, De=256, w_in=FAKE, w_g=FAKE, Dm=256, E=8, k=2,
             offsets=FAKE, sorted_slot=FAKE, dx_slots=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_bwd_dgrad_in(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(n_parts=0), 1), (dict(renorm=2), 1), (dict(renorm=0, probs=None), 1), (dict(Dm=6), 2),
    (dict(k=9), 1), (dict(w_r=None), 1), (dict(dx=ctypes.c_void_p((1 << 20) + 2)), 2),
])
def test_route_bwd_rejects_bad_arguments(lib, kw, code):
    a = dict(T=10, k=2, E=8, Dm=64, renorm=1, topk_idx=FAKE, topk_w=FAKE, probs=None,
             dr_part=FAKE, n_parts=1, dx_slots=FAKE, w_r=FAKE, dlogits=FAKE, dx=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_route_bwd(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=3), 1), (dict(E=0), 1), (dict(E=65), 1), (dict(Dm=0), 1), (dict(x=None), 1),
    (dict(probs=None), 1),
])
def test_route_probs_rejects_bad_arguments(lib, kw, code):
    a = dict(x=FAKE, dtype=1, T=10, Dm=64, w_r=FAKE, bias=None, E=8, probs=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_route_probs(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=3), 1), (dict(E=0), 1), (dict(T=-1), 1), (dict(dw_r=None), 1),
    (dict(dlogits=None), 1),
])
def test_route_wgrad_rejects_bad_arguments(lib, kw, code):
    a = dict(x=FAKE, dtype=1, T=10, Dm=64, E=8, dlogits=FAKE, dw_r=FAKE, dbias=None, stream=None)
    a.update(kw)
    assert lib.rom_route_wgrad(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(M=0), 1), (dict(m_split=-1), 1), (dict(m_split=384), 1), (dict(M=200), 2),
    (dict(N=128), 2), (dict(m_split=64), 2), (dict(out1=None), 1), (dict(out0=None), 1),
])
def test_bwd_wgrad_rejects_bad_arguments(lib, kw, code):
    a = dict(a_sorted=FAKE, M=256, b_sorted=FAKE, N=256, R=512, E=8, offsets=FAKE, m_split=128,
             out0=FAKE, out1=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_bwd_wgrad(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), 1), (dict(E=0), 1), (dict(k=9), 1), (dict(renorm=2), 1), (dict(Dm=12), 2),
    (dict(offsets=None), 1), (dict(x_sorted=None), 1), (dict(x=ctypes.c_void_p((1 << 20) + 2)), 2),
    (dict(T=128 * 65537, E=1), 3),  # more chunk histograms than the fixed scratch holds
])
def test_route_dispatch_noalloc_rejects_bad_arguments(lib, kw, code):
    a = dict(x=FAKE, dtype=1, T=300, Dm=64, w_r=FAKE, bias=None, E=8, k=1, renorm=0,
             topk_idx=FAKE, topk_w=FAKE, counts=None, offsets=FAKE, sorted_slot=FAKE,
             slot_pos=FAKE, x_sorted=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_route_dispatch_noalloc(*a.values()) == code


def _declared_arity():
    """Number of parameters of every function declared in include/rom.h."""
    text = open(os.path.join(ROOT, "include", "rom.h")).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    out = {}
    for m in re.finditer(r"(?:int|size_t|const char\*)\s+(rom_\w+)\s*\(([^)]*)\)\s*;", text):
        params = [p for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        out[m.group(1)] = len(params)
    return out


def test_binding_signatures_match_the_header_arity():
    from mixture_experts_projections_b200 import rom
    arity = _declared_arity()
    assert arity, "no declarations parsed"
    for name, n in arity.items():
        assert len(rom.SIGNATURES[name][1]) == n, (name, len(rom.SIGNATURES[name][1]), n)


@pytest.mark.parametrize("kw,code", [
    (dict(proj=0), 1), (dict(dtype=5), 1), (dict(E=0), 1), (dict(k=3, E=2), 1),
    (dict(T=65), 2), (dict(dtype=0), 2), (dict(N=200), 2), (dict(K=12), 2),
    (dict(topk_idx=None), 1), (dict(out=ctypes.c_void_p((1 << 20) + 4)), 2),
])
def test_expert_proj_dense_rejects_bad_arguments(lib, kw, code):
    a = dict(proj=2, dtype=1, x=FAKE, T=64, K=64, w=FAKE, N=256, E=4, k=1, topk_idx=FAKE,
             topk_w=FAKE, out=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_expert_proj_dense(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    # the tile-major weights (ROM_W_TILED) need whole 64-element K blocks
    (dict(proj=2 | 0x100, K=96), 2), (dict(proj=1 | 0x100, K=72), 2), (dict(proj=0 | 0x100), 1),
    (dict(proj=2 | 0x200), 1),
])
def test_expert_proj_dense_tiled_flag(lib, kw, code):
    a = dict(proj=2, dtype=1, x=FAKE, T=64, K=64, w=FAKE, N=256, E=4, k=1, topk_idx=FAKE,
             topk_w=FAKE, out=FAKE, stream=None)
    a.update(kw)
    assert lib.rom_expert_proj_dense(*a.values()) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), 1), (dict(E=0), 1), (dict(N=0), 1), (dict(K=-64), 1),
    (dict(dtype=0), 2), (dict(N=192), 2), (dict(K=96), 2), (dict(w=None), 1),
    (dict(w_tiled=ctypes.c_void_p((1 << 22) + 8)), 2),
    # the copy must not overlap its source
    (dict(w_tiled=ctypes.c_void_p((1 << 20) + 4096)), 1),
])
def test_pack_expert_weights_rejects_bad_arguments(lib, kw, code):
    a = dict(dtype=1, w=FAKE, E=2, N=128, K=64, w_tiled=ctypes.c_void_p(1 << 22), stream=None)
    a.update(kw)
    assert lib.rom_pack_expert_weights(*a.values()) == code
