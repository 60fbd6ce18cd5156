"""GPU parity of the whole RoM block forward and of the Swimba in-projection
against the float64 oracle, on sizes that span several tiles with ragged
tails, through the C ABI."""
import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import (WORKLOADS, make_block_inputs,
                                                     make_inproj_inputs, make_workload_inputs)
from oracle import rom_oracle as orc
from parity_util import (assert_close, assert_routing_matches, block_to_dev, to_dev, to_np,
                         weights_to_dev)

pytestmark = pytest.mark.gpu

BLOCK_CASES = [
    # T, Dm, De, E, k, renorm, dtype, router_std, bias
    (1000, 256, 384, 8, 1, False, "bf16", 0.02, None),
    (700, 512, 256, 4, 1, False, "bf16", 0.05, {0: 1.0}),
    (600, 256, 256, 16, 2, True, "bf16", 0.05, None),
    (300, 128, 128, 8, 2, False, "bf16", 0.1, None),
    (333, 256, 128, 6, 3, True, "bf16", 0.1, None),
    (200, 256, 256, 1, 1, False, "bf16", 0.02, None),
    (517, 64, 128, 8, 1, False, "f32", 0.05, None),
    (300, 96, 72, 5, 2, True, "f32", 0.2, None),
    (150, 512, 512, 8, 1, False, "bf16", 0.02, {3: -40.0, 5: -40.0}),  # two empty experts
    # over 1024 routed rows (the SM-pair Out GEMM) with d_model % 256 == 128:
    # a last tile of 128 output columns
    (1300, 384, 256, 8, 1, False, "bf16", 0.02, None),
    (800, 640, 256, 8, 2, True, "bf16", 0.05, None),
    # few routed rows (the swap-AB Out GEMM) over d_inner = 1024 and 1536
    (500, 512, 1024, 8, 1, False, "bf16", 0.02, None),
    (400, 256, 1536, 4, 2, True, "bf16", 0.05, None),
]


def oracle_block(inp, k, renorm):
    return orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                             k=k, bias=inp["bias"], renorm=renorm)


@pytest.mark.parametrize("T,Dm,De,E,k,renorm,dtype,std,bias", BLOCK_CASES)
def test_block_forward_matches_oracle(T, Dm, De, E, k, renorm, dtype, std, bias):
    b = None
    if bias is not None:
        b = np.zeros(E, np.float32)
        for e, v in bias.items():
            b[e] = v
    inp = make_block_inputs(T, Dm, De, E, seed=T + De, dtype=dtype, router_std=std, bias=b)
    ref = oracle_block(inp, k, renorm)
    d = block_to_dev(inp, dtype)
    out = rom.block_forward(d["x"], d["w_r"], d["bias"], d["w_conv"], d["w_gate"], d["w_out"],
                            k=k, renorm=renorm)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    rb = out.routing
    assert_routing_matches(rb.topk_idx.cpu().numpy(), rb.topk_w.cpu().numpy().astype(np.float64),
                           ref, x=inp["x"], w_r=inp["w_r"], bias=inp["bias"])
    assert_close(to_np(out.out), ref["O"], dtype, "O", magnitude_scaled_abs=True)
    if k == 1:
        # the intermediate h in sorted order matches Y (.) G of the oracle
        R = T
        srt = rb.sorted_slot.cpu().numpy()[:R]
        assert_close(to_np(out.h_sorted[:R]), ref["YG"][srt], dtype, "h", magnitude_scaled_abs=True)


def test_tiny_fp32_workload():
    wl = WORKLOADS["tiny_fp32"]
    inp = make_workload_inputs(wl)
    ref = oracle_block(inp, wl.k, wl.renorm)
    d = block_to_dev(inp, "f32")
    out = rom.block_forward(d["x"], d["w_r"], d["bias"], d["w_conv"], d["w_gate"], d["w_out"],
                            k=wl.k)
    assert_routing_matches(out.routing.topk_idx.cpu().numpy(),
                           out.routing.topk_w.cpu().numpy().astype(np.float64), ref, x=inp["x"],
                           w_r=inp["w_r"])
    assert_close(to_np(out.out), ref["O"], "f32", "O")


def test_block_forward_is_deterministic_and_repeatable():
    inp = make_block_inputs(900, 256, 256, 8, seed=2, router_std=0.05)
    d = block_to_dev(inp, "bf16")
    args = (d["x"], d["w_r"], None, d["w_conv"], d["w_gate"], d["w_out"])
    a = rom.block_forward(*args, k=2, renorm=True).out.clone()
    bufs = rom.BlockBuffers(900, 256, 256, 8, 2, torch.bfloat16, "cuda")
    for _ in range(3):
        b = rom.block_forward(*args, k=2, renorm=True, bufs=bufs).out
        assert torch.equal(a, b)


INPROJ_CASES = [
    # T, Dm, N, E, k, renorm
    (64, 512, 1280, 4, 1, False),
    (200, 256, 768, 4, 2, True),
    (37, 1024, 512, 8, 1, False),
    # several 64-token tiles per expert, float32 slots
    (300, 1024, 768, 4, 2, True),
    # ragged last K block (K = 1000), partial token tiles of both 32-column halves
    (700, 1000, 512, 4, 1, False),
    # more weight tiles than SMs (several tiles per CTA)
    (300, 1024, 2560, 8, 2, True),
]


@pytest.mark.parametrize("T,Dm,N,E,k,renorm", INPROJ_CASES)
def test_inproj_matches_oracle(T, Dm, N, E, k, renorm):
    inp = make_inproj_inputs(T, Dm, N, E, seed=T + N, router_std=0.05)
    ref = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=k, renorm=renorm)
    out, rb = rom.inproj_forward(to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"),
                                 weights_to_dev(inp["w"], "bf16"), k=k, renorm=renorm)
    torch.cuda.synchronize()
    assert_routing_matches(rb.topk_idx.cpu().numpy(), rb.topk_w.cpu().numpy().astype(np.float64),
                           ref, x=inp["x"], w_r=inp["w_r"])
    assert_close(to_np(out), ref["S"], "bf16", "S", magnitude_scaled_abs=True)


def test_inproj_is_deterministic():
    """The in-projection accumulates in a fixed order and writes every output
    once: two calls give identical bits."""
    inp = make_inproj_inputs(64, 4096, 1024, 4, seed=7, router_std=0.05)
    args = (to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"), weights_to_dev(inp["w"], "bf16"))
    a, _ = rom.inproj_forward(*args, k=1, renorm=False)
    a = a.clone()
    b, _ = rom.inproj_forward(*args, k=1, renorm=False)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    assert torch.equal(a, b)


def test_inproj_skewed_routing_small_batch():
    """96 tokens over 4 experts (the swap-AB GEMM path); with this seed one
    expert receives 36 of them and another 17."""
    T, Dm, N, E = 96, 256, 512, 4
    inp = make_inproj_inputs(T, Dm, N, E, seed=615, router_std=0.05)
    ref = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=1, renorm=False)
    assert np.bincount(ref["topk_idx"].reshape(-1), minlength=E).max() > 32
    out, rb = rom.inproj_forward(to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"),
                                 weights_to_dev(inp["w"], "bf16"), k=1, renorm=False)
    torch.cuda.synchronize()
    assert_routing_matches(rb.topk_idx.cpu().numpy(), rb.topk_w.cpu().numpy().astype(np.float64),
                           ref, x=inp["x"], w_r=inp["w_r"])
    assert_close(to_np(out), ref["S"], "bf16", "S", magnitude_scaled_abs=True)


@pytest.mark.parametrize("T,Dm,De,E,k,renorm", [(5000, 256, 256, 8, 1, False),
                                                (3000, 256, 384, 8, 2, True),
                                                (900, 256, 256, 4, 1, False)])
def test_host_pipeline_matches_single_call(T, Dm, De, E, k, renorm):
    """Chunked, multi-stream forward on pinned host buffers gives every
    token's routing exactly and its output within the forward's bar."""
    inp = make_block_inputs(T, Dm, De, E, seed=T, router_std=0.05)
    d = block_to_dev(inp, "bf16")
    ref = rom.block_forward(d["x"], d["w_r"], None, d["w_conv"], d["w_gate"], d["w_out"], k=k,
                            renorm=renorm).out
    x_h = d["x"].cpu().pin_memory()
    out_h = torch.empty((T, Dm), dtype=torch.bfloat16, pin_memory=True)
    pipe = rom.HostPipeline(T, Dm, None, E, k, torch.bfloat16, "cuda", chunks=5, De=De)
    # first call eager, second captured into a CUDA graph, third replayed
    for call in range(3):
        out_h.zero_()
        pipe.block_forward(x_h, d["w_r"], None, d["w_conv"], d["w_gate"], d["w_out"], out_h,
                           renorm=renorm)
        torch.cuda.synchronize()
        assert_close(out_h.float().numpy(), to_np(ref), "bf16",
                     f"O (pipelined vs single call, call {call})", magnitude_scaled_abs=True)
    orc_ref = oracle_block(inp, k, renorm)
    assert_close(out_h.float().numpy().astype(np.float64), orc_ref["O"], "bf16", "O (pipelined)",
                 magnitude_scaled_abs=True)



@pytest.mark.parametrize("T,Dm,N,E,k,renorm", [(5000, 256, 512, 4, 1, False),
                                               (3000, 512, 768, 8, 2, True)])
def test_host_pipeline_inproj_matches_single_call(T, Dm, N, E, k, renorm):
    """The in-projection on pinned host buffers (chunks over three streams;
    eager, captured and replayed calls) matches one call on the whole batch
    and the oracle within the forward's bar (a short last chunk may take the
    swap-AB GEMM where the whole batch takes the SM-pair one)."""
    inp = make_inproj_inputs(T, Dm, N, E, seed=T + 1, router_std=0.05)
    x = to_dev(inp["x"], "bf16")
    w_r = to_dev(inp["w_r"], "f32")
    w = weights_to_dev(inp["w"], "bf16")
    ref, _ = rom.inproj_forward(x, w_r, w, k=k, renorm=renorm)
    ref = ref.clone()
    x_h = x.cpu().pin_memory()
    out_h = torch.empty((T, N), dtype=torch.bfloat16, pin_memory=True)
    pipe = rom.HostPipeline(T, Dm, N, E, k, torch.bfloat16, "cuda", chunks=5)
    for call in range(3):
        out_h.zero_()
        pipe.inproj_forward(x_h, w_r, w, out_h, renorm=renorm)
        torch.cuda.synchronize()
        assert rom.rom_get_status() == 0
        assert_close(out_h.float().numpy(), to_np(ref), "bf16",
                     f"S (pipelined vs single call, call {call})", magnitude_scaled_abs=True)
    orc_ref = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=k, renorm=renorm)
    assert_close(out_h.float().numpy().astype(np.float64), orc_ref["S"], "bf16", "S (pipelined)",
                 magnitude_scaled_abs=True)

@pytest.mark.parametrize("T,Dm,N,E,k,renorm", [
    (64, 512, 1280, 4, 1, False),
    (37, 1024, 512, 8, 1, False),
    (1, 256, 256, 4, 1, False),
    (50, 256, 768, 4, 2, True),
    (64, 1024, 1024, 16, 2, False),
    # more weight tiles than SMs (several tiles per CTA), ragged K = 1000
    (50, 1000, 5120, 4, 1, False),
    (64, 2048, 2560, 8, 2, True),
])
def test_inproj_without_dispatch_for_small_batches(T, Dm, N, E, k, renorm):
    """rom_expert_proj_dense (every expert's weights meet all tokens, the
    routing selects in the epilogue, launched as a dependent of the router)
    against the oracle and against the dispatched path on the same inputs."""
    inp = make_inproj_inputs(T, Dm, N, E, seed=3 * T + N + k, router_std=0.05)
    ref = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=k, renorm=renorm)
    args = (to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"), weights_to_dev(inp["w"], "bf16"))
    dense, rb = rom.inproj_forward(*args, k=k, renorm=renorm)
    sparse, _ = rom.inproj_forward(*args, k=k, renorm=renorm, dense_small=False)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    assert_routing_matches(rb.topk_idx.cpu().numpy(), rb.topk_w.cpu().numpy().astype(np.float64),
                           ref, x=inp["x"], w_r=inp["w_r"])
    assert_close(to_np(dense), ref["S"], "bf16", "S (no dispatch)", magnitude_scaled_abs=True)
    assert_close(to_np(dense), to_np(sparse), "bf16", "no dispatch vs dispatched",
                 magnitude_scaled_abs=True)


@pytest.mark.parametrize("dense_small", [True, False])
def test_few_token_inproj_graph_replays_match_eager(dense_small):
    """The few-token projection over more weight tiles than SMs, captured in a
    CUDA graph and replayed: every replay must reproduce the eager bits."""
    T, Dm, N, E = 64, 4096, 5120, 4  # 160 weight tiles
    inp = make_inproj_inputs(T, Dm, N, E, seed=11, router_std=0.05)
    x, w_r, w = (to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"),
                 weights_to_dev(inp["w"], "bf16"))
    eager, bufs = rom.inproj_forward(x, w_r, w, k=1, renorm=False, dense_small=dense_small)
    eager = eager.clone()
    out = torch.empty_like(eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        rom.inproj_forward(x, w_r, w, k=1, renorm=False, bufs=bufs, out=out,
                           dense_small=dense_small)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        rom.inproj_forward(x, w_r, w, k=1, renorm=False, bufs=bufs, out=out,
                           dense_small=dense_small)
    for _ in range(4):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert rom.rom_get_status() == 0
        assert torch.equal(out, eager)
    ref = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=1, renorm=False)
    assert_close(to_np(eager), ref["S"], "bf16", "S (160 weight tiles)", magnitude_scaled_abs=True)
    del g


def test_pack_expert_weights_layout():
    """rom_pack_expert_weights writes every 128 x 64 weight tile as one
    contiguous block: element (e, n, c) at
    ((((e * N/128 + n/128) * K/64 + c/64) * 128 + n % 128) * 64 + c % 64)."""
    E, N, K = 3, 384, 320
    g = torch.Generator(device="cpu").manual_seed(5)
    w = torch.randn((E, N, K), generator=g).to(torch.bfloat16).cuda()
    t = rom.pack_expert_weights(w)
    torch.cuda.synchronize()
    ref = w.view(E, N // 128, 128, K // 64, 64).permute(0, 1, 3, 2, 4).reshape(-1)
    assert torch.equal(t.reshape(-1), ref)
    # the element formula, checked at a few places
    flat = t.reshape(-1).cpu()
    for e, n, c in [(0, 0, 0), (2, 383, 319), (1, 130, 65), (2, 127, 64)]:
        i = (((e * (N // 128) + n // 128) * (K // 64) + c // 64) * 128 + n % 128) * 64 + c % 64
        assert flat[i].item() == w[e, n, c].item()


@pytest.mark.parametrize("T,Dm,N,E,k,renorm", [
    (64, 4096, 2560, 4, 1, False),
    (33, 1024, 1280, 8, 2, True),
])
def test_tiled_weights_give_the_same_projection(T, Dm, N, E, k, renorm):
    """The dispatch-free projection reading the tile-major weights computes
    the same tiles in the same order: identical bits to the row-major read."""
    inp = make_inproj_inputs(T, Dm, N, E, seed=T + E, router_std=0.05)
    x, w_r, w = (to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"),
                 weights_to_dev(inp["w"], "bf16"))
    wt = rom.pack_expert_weights(w)
    a, _ = rom.inproj_forward(x, w_r, w, k=k, renorm=renorm)
    a = a.clone()
    b, _ = rom.inproj_forward(x, w_r, w, k=k, renorm=renorm, w_tiled=wt)
    torch.cuda.synchronize()
    assert rom.rom_get_status() == 0
    assert torch.equal(a, b)
    ref = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=k, renorm=renorm)
    assert_close(to_np(b), ref["S"], "bf16", "S (tiled weights)", magnitude_scaled_abs=True)
