"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test fixes the oracle to a closed form, a library routine, a brute-force
evaluation on tiny inputs, an invariant of the method, or finite differences.
Sources: "Routing Mamba: Scaling State Space Models with Mixture-of-Experts
Projection" (chapterpal summary page), Knowl 1; "Swimba: Switch Mamba Model
Scales State Space Models" (project page), Extended abstract.
"""
import itertools
import math

import numpy as np
import pytest
from scipy.special import expit, softmax as sp_softmax

from mixture_experts_projections_b200.inputs import make_block_inputs, make_inproj_inputs
from oracle import rom_oracle as orc


def _silu_ref(z):
    return z * expit(z)


# ---------------------------------------------------------------- closed forms


def test_worked_example_closed_form():
    """A 2-expert, d_model=2, d_inner=2 block evaluated by hand from Knowl 1.

    Token 0: x=[1,0], logits [ln3, 0] -> p=[3/4,1/4], S={0}, r=3/4.
      H = x W_in,0 = [2, 1]; z = x W_g,0 = [ln3, 0]; G = [ln3*3/4, 0]
      Y(.)G = [1.5 ln3, 0];  (Y(.)G) W_out,0 = [1.5 ln3, -3 ln3];  O = 3/4 of that.
    Token 1: x=[-1,0], logits [-ln3, 0] -> p=[1/4,3/4], S={1}, r=3/4.
      H = x W_in,1 = [-1, 3]; z = x W_g,1 = [0, ln3]; G = [0, ln3*3/4]
      Y(.)G = [0, 2.25 ln3]; (Y(.)G) W_out,1 = 2.25 ln3 * [4, -1]; O = 3/4 of that.
    Token 2: x=[0,1], logits [0,0] (tie) -> expert 0, r = 1/2.
      H = x W_in,0 = [0, 5]; z = x W_g,0 = [0, 0] -> G = 0 -> O = 0.
    """
    l3 = math.log(3.0)
    x = np.array([[1.0, 0.0], [-1.0, 0.0], [0.0, 1.0]])
    w_r = np.array([[l3, 0.0], [0.0, 0.0]])
    w_in = np.array([[[2.0, 1.0], [0.0, 5.0]], [[1.0, -3.0], [7.0, 7.0]]])
    w_g = np.array([[[l3, 0.0], [0.0, 0.0]], [[0.0, -l3], [1.0, 1.0]]])
    w_out = np.array([[[1.0, -2.0], [5.0, 7.0]], [[9.0, 9.0], [4.0, -1.0]]])
    fw = orc.block_forward(x, w_r, w_in, w_g, w_out, k=1)
    assert fw["topk_idx"][:, 0].tolist() == [0, 1, 0]
    np.testing.assert_allclose(fw["topk_w"][:, 0], [0.75, 0.75, 0.5], rtol=1e-15)
    exp = np.array([[0.75 * 1.5 * l3, -0.75 * 3 * l3],
                    [0.75 * 2.25 * l3 * 4, -0.75 * 2.25 * l3],
                    [0.0, 0.0]])
    np.testing.assert_allclose(fw["O"], exp, rtol=1e-14, atol=1e-14)


def test_silu_closed_forms_and_extremes():
    """SiLU(z) = z sigma(z): SiLU(ln 3) = (3/4) ln 3, SiLU(z) - SiLU(-z) = z,
    SiLU'(0) = 1/2 and SiLU'(z) + SiLU'(-z) = 1; no overflow for |z| ~ 1e3
    (SiLU -> z above, -> 0 below)."""
    l3 = math.log(3.0)
    assert orc.silu(np.array([l3]))[0] == pytest.approx(0.75 * l3, rel=1e-15)
    z = np.linspace(-40.0, 40.0, 161)
    np.testing.assert_allclose(orc.silu(z) - orc.silu(-z), z, rtol=1e-14, atol=1e-14)
    assert orc.silu_grad(np.array([0.0]))[0] == pytest.approx(0.5, rel=1e-15)
    np.testing.assert_allclose(orc.silu_grad(z) + orc.silu_grad(-z), 1.0, rtol=1e-14)
    with np.errstate(over="raise", invalid="raise", divide="raise"):
        big = np.array([-1000.0, -750.0, 750.0, 1000.0])
        out = orc.silu(big)
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out, [0.0, 0.0, 750.0, 1000.0], atol=1e-300)


def test_softmax_sums_to_one_and_matches_scipy():
    inp = make_block_inputs(64, 32, 16, 8, seed=3)
    rt = orc.route(inp["x"], inp["w_r"], 2)
    np.testing.assert_allclose(rt["p"].sum(1), 1.0, atol=1e-12)
    ref = sp_softmax(inp["x"].astype(np.float64) @ inp["w_r"].astype(np.float64), axis=1)
    np.testing.assert_allclose(rt["p"], ref, rtol=1e-12)


def test_renormalised_weights_are_softmax_over_selected_logits():
    inp = make_block_inputs(50, 16, 8, 6, seed=5, router_std=0.5)
    rt = orc.route(inp["x"], inp["w_r"], 2, renorm=True)
    np.testing.assert_allclose(rt["topk_w"].sum(1), 1.0, atol=1e-12)
    rows = np.arange(50)[:, None]
    sel_logits = rt["logits"][rows, rt["topk_idx"]]
    np.testing.assert_allclose(rt["topk_w"], sp_softmax(sel_logits, axis=1), rtol=1e-12)


# ---------------------------------------------------------------- brute force


def _bruteforce_topk(logits, k):
    """Rank of expert i = number of experts that beat it (larger logit, or
    equal logit and lower index). S = ranks < k, slot = rank."""
    T, E = logits.shape
    idx = np.full((T, k), -1)
    for t in range(T):
        for i in range(E):
            rank = sum(1 for j in range(E)
                       if logits[t, j] > logits[t, i] or (logits[t, j] == logits[t, i] and j < i))
            if rank < k:
                idx[t, rank] = i
    return idx


@pytest.mark.parametrize("k", [1, 2, 3])
def test_topk_matches_bruteforce_rank(k):
    inp = make_block_inputs(40, 8, 4, 5, seed=11, router_std=1.0)
    rt = orc.route(inp["x"], inp["w_r"], k)
    assert np.array_equal(rt["topk_idx"], _bruteforce_topk(rt["logits"], k))
    # p_{S_j} are the k largest probabilities
    srt = np.sort(rt["p"], axis=1)[:, ::-1][:, :k]
    np.testing.assert_allclose(rt["p"][np.arange(40)[:, None], rt["topk_idx"]], srt, rtol=0)


def _bruteforce_block(x, w_r, w_in, w_g, w_out, k, renorm):
    """Evaluate every expert densely for every token, then mask by S_t."""
    x = x.astype(np.float64)
    logits = x @ w_r.astype(np.float64)
    p = sp_softmax(logits, axis=1)
    S = _bruteforce_topk(logits, k)
    T = x.shape[0]
    E, Dm, De = w_in.shape
    out = np.zeros((T, Dm))
    for t in range(T):
        mask = np.zeros(E)
        mask[S[t]] = 1.0
        r = p[t] * mask
        if renorm:
            r = r / r.sum()
        u_all = np.stack([x[t] @ w_in[i] for i in range(E)])  # [E, De]
        z_all = np.stack([x[t] @ w_g[i] for i in range(E)])
        h = (mask @ u_all) * _silu_ref(mask @ z_all)
        for i in range(E):
            out[t] += r[i] * (h @ w_out[i])
    return out


@pytest.mark.parametrize("E,k,renorm", [(1, 1, False), (2, 1, False), (4, 1, False),
                                        (8, 1, False), (4, 2, False), (4, 2, True),
                                        (8, 2, True), (3, 3, False)])
def test_block_matches_dense_bruteforce(E, k, renorm):
    inp = make_block_inputs(24, 12, 10, E, seed=E * 10 + k, router_std=0.7)
    args = (inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"])
    fw = orc.block_forward(*args, k=k, renorm=renorm)
    ref = _bruteforce_block(*args, k=k, renorm=renorm)
    np.testing.assert_allclose(fw["O"], ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- special cases


def test_single_expert_is_dense_mamba_projection():
    inp = make_block_inputs(33, 16, 24, 1, seed=2)
    x = inp["x"].astype(np.float64)
    fw = orc.block_forward(x, inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], k=1)
    assert np.all(fw["topk_idx"] == 0)
    np.testing.assert_allclose(fw["topk_w"], 1.0, rtol=0, atol=0)
    u = x @ inp["w_conv"][0].astype(np.float64)
    z = x @ inp["w_gate"][0].astype(np.float64)
    ref = (u * _silu_ref(z)) @ inp["w_out"][0].astype(np.float64)
    np.testing.assert_allclose(fw["O"], ref, rtol=1e-12, atol=1e-13)


def test_top1_output_is_p_times_dense_block_of_chosen_expert():
    """For K=1 the block equals p_{t,e} times the dense block of expert e:
    only Out is routing-weighted, Conv and Gate use the indicator."""
    inp = make_block_inputs(40, 16, 20, 4, seed=9, router_std=0.5)
    x = inp["x"].astype(np.float64)
    fw = orc.block_forward(x, inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], k=1)
    logits = x @ inp["w_r"].astype(np.float64)
    e = np.argmax(logits, axis=1)
    p = sp_softmax(logits, axis=1)[np.arange(40), e]
    for t in range(40):
        we = [inp[n][e[t]].astype(np.float64) for n in ("w_conv", "w_gate", "w_out")]
        dense = ((x[t] @ we[0]) * _silu_ref(x[t] @ we[1])) @ we[2]
        np.testing.assert_allclose(fw["O"][t], p[t] * dense, rtol=1e-12, atol=1e-13)


def test_all_experts_selected_sums_before_silu():
    """K = E: indicators are all one, so H = x sum_i W_in,i and
    G = SiLU(x sum_i W_g,i) (SiLU after the sum over experts)."""
    inp = make_block_inputs(20, 8, 6, 2, seed=4, router_std=0.5)
    x = inp["x"].astype(np.float64)
    fw = orc.block_forward(x, inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], k=2)
    p = sp_softmax(x @ inp["w_r"].astype(np.float64), axis=1)
    h = (x @ inp["w_conv"].astype(np.float64).sum(0)) * _silu_ref(
        x @ inp["w_gate"].astype(np.float64).sum(0))
    ref = p[:, :1] * (h @ inp["w_out"][0].astype(np.float64)) + \
        p[:, 1:] * (h @ inp["w_out"][1].astype(np.float64))
    np.testing.assert_allclose(fw["O"], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("k,renorm", [(1, False), (2, False), (2, True)])
def test_zero_router_tie_rule(k, renorm):
    """W_r = 0: every logit ties, so S_t = {0..k-1} in index order, p = 1/E."""
    inp = make_block_inputs(10, 8, 4, 5, seed=1, zero_router=True)
    rt = orc.route(inp["x"], inp["w_r"], k, renorm=renorm)
    assert np.array_equal(rt["topk_idx"], np.tile(np.arange(k), (10, 1)))
    np.testing.assert_allclose(rt["topk_w"], (1.0 / k) if renorm else 0.2, rtol=1e-15)


def test_zero_gate_gives_zero_output():
    inp = make_block_inputs(16, 8, 8, 4, seed=6)
    fw = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], np.zeros_like(inp["w_gate"]),
                           inp["w_out"], k=2)
    assert np.all(fw["O"] == 0.0)


# ---------------------------------------------------------------- invariants


def test_token_permutation_equivariance():
    inp = make_block_inputs(30, 8, 6, 4, seed=12, router_std=0.5)
    perm = np.random.default_rng(0).permutation(30)
    a = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], k=2)
    b = orc.block_forward(inp["x"][perm], inp["w_r"], inp["w_conv"], inp["w_gate"],
                          inp["w_out"], k=2)
    np.testing.assert_allclose(b["O"], a["O"][perm], rtol=1e-13, atol=1e-14)
    assert np.array_equal(b["topk_idx"], a["topk_idx"][perm])


def test_expert_relabel_invariance():
    inp = make_block_inputs(30, 8, 6, 5, seed=13, router_std=0.5)
    pi = np.array([3, 0, 4, 1, 2])  # new expert n is old expert pi[n]
    a = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], k=2)
    b = orc.block_forward(inp["x"], inp["w_r"][:, pi], inp["w_conv"][pi], inp["w_gate"][pi],
                          inp["w_out"][pi], k=2)
    np.testing.assert_allclose(b["O"], a["O"], rtol=1e-13, atol=1e-14)
    assert np.array_equal(pi[b["topk_idx"]], a["topk_idx"])


@pytest.mark.parametrize("k", [1, 2])
def test_dispatch_is_stable_counting_sort(k):
    inp = make_block_inputs(97, 8, 4, 6, seed=21, router_std=1.0)
    idx = orc.route(inp["x"], inp["w_r"], k)["topk_idx"]
    d = orc.dispatch(idx, 6)
    flat = idx.reshape(-1)
    assert np.array_equal(d["counts"], np.bincount(flat, minlength=6))
    assert np.array_equal(d["offsets"], np.concatenate([[0], np.cumsum(d["counts"])]))
    assert np.array_equal(d["sorted_slot"], np.argsort(flat, kind="stable"))
    R = flat.size
    assert np.array_equal(np.sort(d["sorted_slot"]), np.arange(R))  # bijection
    assert np.array_equal(d["slot_pos"][d["sorted_slot"]], np.arange(R))  # inverse


def test_dispatch_empty_expert_and_no_tokens():
    idx = np.array([[2], [2], [0]], dtype=np.int32)
    d = orc.dispatch(idx, 4)
    assert d["counts"].tolist() == [1, 0, 2, 0]
    assert d["offsets"].tolist() == [0, 1, 1, 3, 3]
    assert d["sorted_slot"].tolist() == [2, 0, 1]
    d0 = orc.dispatch(np.zeros((0, 1), np.int32), 3)
    assert d0["offsets"].tolist() == [0, 0, 0, 0]


# ---------------------------------------------------------------- Swimba in-projection


def test_inproj_top1_is_p_times_dense_projection():
    inp = make_inproj_inputs(20, 16, 12, 4, seed=7, router_std=0.5)
    x = inp["x"].astype(np.float64)
    res = orc.inproj_forward(x, inp["w_r"], inp["w"], k=1)
    logits = x @ inp["w_r"].astype(np.float64)
    e = np.argmax(logits, axis=1)
    p = sp_softmax(logits, axis=1)[np.arange(20), e]
    for t in range(20):
        np.testing.assert_allclose(res["S"][t], p[t] * (x[t] @ inp["w"][e[t]].astype(np.float64)),
                                   rtol=1e-12, atol=1e-13)


def test_inproj_all_experts_is_probability_weighted_mix():
    """K = E: the layer applies the p-weighted mixture of expert matrices
    (parameter-space mixing: one projection with W = sum_i p_i W_i)."""
    inp = make_inproj_inputs(15, 8, 10, 3, seed=8, router_std=0.5)
    x = inp["x"].astype(np.float64)
    res = orc.inproj_forward(x, inp["w_r"], inp["w"], k=3)
    p = sp_softmax(x @ inp["w_r"].astype(np.float64), axis=1)
    for t in range(15):
        wmix = np.tensordot(p[t], inp["w"].astype(np.float64), axes=(0, 0))
        np.testing.assert_allclose(res["S"][t], x[t] @ wmix, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- backward


def _loss(inp, k, renorm, **over):
    a = {n: over.get(n, inp[n]) for n in ("x", "w_r", "w_conv", "w_gate", "w_out")}
    fw = orc.block_forward(a["x"], a["w_r"], a["w_conv"], a["w_gate"], a["w_out"], k=k,
                           renorm=renorm)
    return float(np.sum(fw["O"] * inp["dout"])), fw["topk_idx"]


@pytest.mark.parametrize("k,renorm", [(1, False), (2, False), (2, True)])
def test_backward_matches_central_differences(k, renorm):
    inp = make_block_inputs(6, 5, 4, 3, seed=31 + k, router_std=0.8, with_dout=True)
    inp = {n: (v.astype(np.float64) if v is not None else None) for n, v in inp.items()}
    fw = orc.route(inp["x"], inp["w_r"], k)
    assert fw["margin"].min() > 1e-3  # the selection cannot flip under the steps below
    g = orc.block_backward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                           inp["dout"], k=k, renorm=renorm)
    names = {"x": "dX", "w_r": "dW_r", "w_conv": "dW_in", "w_gate": "dW_g", "w_out": "dW_out"}
    h = 1e-6
    _, idx0 = _loss(inp, k, renorm)
    for n, gn in names.items():
        base = inp[n]
        fd = np.zeros_like(base)
        for pos in itertools.product(*[range(s) for s in base.shape]):
            plus = base.copy()
            plus[pos] += h
            minus = base.copy()
            minus[pos] -= h
            lp, ip = _loss(inp, k, renorm, **{n: plus})
            lm, im = _loss(inp, k, renorm, **{n: minus})
            assert np.array_equal(ip, idx0) and np.array_equal(im, idx0)
            fd[pos] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[gn], fd, rtol=1e-6, atol=1e-8, err_msg=n)


def test_backward_router_gradient_closed_form_top1():
    """K=1 without renormalisation: r = p_e, so dl_m = dr (delta_{m,e} - p_m) p_e."""
    inp = make_block_inputs(9, 6, 5, 4, seed=40, router_std=0.5, with_dout=True)
    g = orc.block_backward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                           inp["dout"], k=1)
    fw = g["forward"]
    e = fw["topk_idx"][:, 0]
    p = fw["p"]
    pe = p[np.arange(9), e]
    exp = -p * (g["dr"][:, 0] * pe)[:, None]
    exp[np.arange(9), e] += g["dr"][:, 0] * pe
    np.testing.assert_allclose(g["dlogits"], exp, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g["dlogits"].sum(1), 0.0, atol=1e-12)  # softmax shift-invariance


# ---------------------------------------------------------------- regression fixture


def test_oracle_regression_fixture():
    """Frozen oracle results (tests/golden/make_golden.py) still reproduce."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_regression.json")
    cases = json.load(open(path))["cases"]
    for name, c in cases.items():
        if name.startswith("independent"):
            inp = make_block_inputs(c["T"], c["Dm"], c["De"], c["E"], seed=c["seed"],
                                    router_std=c["router_std"], extra_routers=True)
            v = orc.variant_block_forward(inp["x"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                                          c["k"], {"conv": inp["w_r"], "gate": inp["w_r_gate"],
                                                   "out": inp["w_r_out"]},
                                          {"conv": True, "gate": True, "out": True})
            np.testing.assert_allclose(v["O"], c["O"], rtol=1e-12, atol=1e-14)
            continue
        if name.startswith("core"):
            from mixture_experts_projections_b200.inputs import make_core_params
            inp = make_block_inputs(c["T"], c["Dm"], c["De"], c["E"], seed=c["seed"],
                                    router_std=c["router_std"])
            core = make_core_params(c["De"], c["Dm"], seed=c["seed"], N=c["N"], K=c["K"])
            r = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"],
                                  inp["w_out"], c["k"], core=core, seq_len=c["seq_len"])
            np.testing.assert_allclose(r["O"], c["O"], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(r["Y"], c["Y"], rtol=1e-12, atol=1e-14)
            continue
        if name.startswith("inproj"):
            inp = make_inproj_inputs(c["T"], c["Dm"], c["N"], c["E"], seed=c["seed"],
                                     router_std=c["router_std"])
            s = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=c["k"])
            np.testing.assert_allclose(s["S"], c["S"], rtol=1e-12, atol=1e-14)
            continue
        inp = make_block_inputs(c["T"], c["Dm"], c["De"], c["E"], seed=c["seed"],
                                router_std=c["router_std"], with_dout=True)
        bw = orc.block_backward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"],
                                inp["w_out"], inp["dout"], k=c["k"], renorm=c["renorm"])
        assert bw["forward"]["topk_idx"].tolist() == c["topk_idx"]
        np.testing.assert_allclose(bw["forward"]["O"], c["O"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(bw["dX"], c["dX"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(bw["dlogits"], c["dlogits"], rtol=1e-12, atol=1e-14)


# ------------------------------------------- projection variants (Knowl 3, Knowl 4)


def _brute_routing(x, w_r, k, renorm):
    """Selection mask and weights [T, E] by a rank count: expert e is chosen
    when fewer than k experts beat it (larger logit, or equal logit and a
    lower index); weights from scipy's softmax."""
    lg = x @ w_r
    T, E = lg.shape
    p = sp_softmax(lg, axis=1)
    mask = np.zeros((T, E))
    for t in range(T):
        for e in range(E):
            beats = sum(1 for f in range(E) if lg[t, f] > lg[t, e] or (lg[t, f] == lg[t, e] and f < e))
            mask[t, e] = 1.0 if beats < k else 0.0
    w = p * mask
    if renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return mask, w


def _brute_variant(x, w_in, w_g, w_out, k, routers, weighted, renorm):
    """Every expert of every projection evaluated densely, then masked."""
    x = x.astype(np.float64)

    def proj(name, a, w):
        if routers[name] is None:
            return a @ w[0].astype(np.float64)
        mask, wt = _brute_routing(x, routers[name].astype(np.float64), k, renorm)
        c = wt if weighted[name] else mask
        return sum(c[:, [e]] * (a @ w[e].astype(np.float64)) for e in range(w.shape[0]))

    H = proj("conv", x, w_in)
    G = _silu_ref(proj("gate", x, w_g))
    return proj("out", H * G, w_out)


def _three_routers(Dm, E, seed, std=0.5):
    rng = np.random.default_rng(seed)
    return [(std * rng.standard_normal((Dm, E))).astype(np.float32) for _ in range(3)]


@pytest.mark.parametrize("k,renorm", [(1, False), (2, False), (2, True)])
def test_variant_with_one_shared_router_is_rom(k, renorm):
    inp = make_block_inputs(40, 12, 10, 5, seed=31, router_std=0.4)
    w_r = inp["w_r"]
    rom = orc.block_forward(inp["x"], w_r, inp["w_conv"], inp["w_gate"], inp["w_out"], k=k,
                            renorm=renorm)
    var = orc.variant_block_forward(inp["x"], inp["w_conv"], inp["w_gate"], inp["w_out"], k,
                                    {"conv": w_r, "gate": w_r, "out": w_r},
                                    {"conv": False, "gate": False, "out": True}, renorm=renorm)
    np.testing.assert_allclose(var["O"], rom["O"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("k,renorm,E", [(1, False, 4), (2, False, 5), (2, True, 3), (3, False, 6)])
def test_independent_moe_matches_brute_force(k, renorm, E):
    inp = make_block_inputs(30, 10, 9, E, seed=40 + E)
    rc, rg, ro = _three_routers(10, E, seed=E)
    routers = {"conv": rc, "gate": rg, "out": ro}
    weighted = {"conv": True, "gate": True, "out": True}
    var = orc.variant_block_forward(inp["x"], inp["w_conv"], inp["w_gate"], inp["w_out"], k,
                                    routers, weighted, renorm=renorm)
    ref = _brute_variant(inp["x"], inp["w_conv"], inp["w_gate"], inp["w_out"], k, routers,
                         weighted, renorm)
    np.testing.assert_allclose(var["O"], ref, rtol=1e-12, atol=1e-12)


def test_independent_moe_top1_closed_form():
    """Top-1: each projection is its own router's winner, scaled by its
    probability: O = p^o ((p^c x W_in,c) (.) SiLU(p^g x W_g,g)) W_out,o."""
    E = 4
    inp = make_block_inputs(25, 8, 6, E, seed=7)
    rc, rg, ro = _three_routers(8, E, seed=3)
    var = orc.variant_block_forward(inp["x"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                                    {"conv": rc, "gate": rg, "out": ro},
                                    {"conv": True, "gate": True, "out": True})
    x = inp["x"].astype(np.float64)
    for t in range(x.shape[0]):
        pc, pg, po = (sp_softmax(x[t] @ r.astype(np.float64)) for r in (rc, rg, ro))
        c, g, o = int(np.argmax(pc)), int(np.argmax(pg)), int(np.argmax(po))
        h = pc[c] * (x[t] @ inp["w_conv"][c])
        gg = _silu_ref(pg[g] * (x[t] @ inp["w_gate"][g]))
        np.testing.assert_allclose(var["O"][t], po[o] * ((h * gg) @ inp["w_out"][o]), rtol=1e-12,
                                   atol=1e-13)


def test_all_dense_variant_is_the_dense_projection():
    inp = make_block_inputs(20, 8, 6, 1, seed=2)
    var = orc.variant_block_forward(inp["x"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                                    {"conv": None, "gate": None, "out": None},
                                    {"conv": True, "gate": True, "out": True})
    x = inp["x"].astype(np.float64)
    dense = ((x @ inp["w_conv"][0]) * _silu_ref(x @ inp["w_gate"][0])) @ inp["w_out"][0]
    np.testing.assert_allclose(var["O"], dense, rtol=1e-13, atol=1e-13)


def test_rom_gate_out_variant_top1_closed_form():
    """RoM (Gate, Out): Conv dense, Gate and Out share one router; top-1:
    O = p_e ((x W_in) (.) SiLU(x W_g,e)) W_out,e."""
    E = 4
    inp = make_block_inputs(25, 8, 6, E, seed=8, router_std=0.4)
    w_in_dense = inp["w_conv"][:1]
    var = orc.variant_block_forward(inp["x"], w_in_dense, inp["w_gate"], inp["w_out"], 1,
                                    {"conv": None, "gate": inp["w_r"], "out": inp["w_r"]},
                                    {"conv": False, "gate": False, "out": True})
    x = inp["x"].astype(np.float64)
    for t in range(x.shape[0]):
        p = sp_softmax(x[t] @ inp["w_r"].astype(np.float64))
        e = int(np.argmax(p))
        h = (x[t] @ w_in_dense[0]) * _silu_ref(x[t] @ inp["w_gate"][e])
        np.testing.assert_allclose(var["O"][t], p[e] * (h @ inp["w_out"][e]), rtol=1e-12,
                                   atol=1e-13)


def test_independent_routers_relabel_one_projection_alone():
    """Permuting the expert labels of the Gate router together with the Gate
    experts, and nothing else, leaves O unchanged: each projection follows its
    own router."""
    E = 5
    inp = make_block_inputs(30, 10, 8, E, seed=12)
    rc, rg, ro = _three_routers(10, E, seed=9)
    weighted = {"conv": True, "gate": True, "out": True}
    a = orc.variant_block_forward(inp["x"], inp["w_conv"], inp["w_gate"], inp["w_out"], 2,
                                  {"conv": rc, "gate": rg, "out": ro}, weighted)
    perm = np.array([3, 0, 4, 1, 2])
    b = orc.variant_block_forward(inp["x"], inp["w_conv"], inp["w_gate"][perm], inp["w_out"], 2,
                                  {"conv": rc, "gate": rg[:, perm], "out": ro}, weighted)
    np.testing.assert_allclose(a["O"], b["O"], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------- dense core (Knowl 1, Knowl 9)


def test_causal_conv1d_matches_numpy_convolve_and_shifts():
    rng = np.random.default_rng(0)
    L, D, K = 37, 5, 4
    h = rng.standard_normal((L, D))
    w = rng.standard_normal((D, K))
    b = rng.standard_normal(D)
    out = orc.causal_conv1d(h, w, b)
    for d in range(D):
        ref = np.convolve(h[:, d], w[d, ::-1], mode="full")[:L] + b[d]
        np.testing.assert_allclose(out[:, d], ref, rtol=1e-13, atol=1e-13)
    delta = np.zeros((D, K))
    delta[:, K - 1] = 1.0
    np.testing.assert_array_equal(orc.causal_conv1d(h, delta, np.zeros(D)), h)
    shift = np.zeros((D, K))
    shift[:, K - 2] = 1.0
    s = orc.causal_conv1d(h, shift, np.zeros(D))
    np.testing.assert_array_equal(s[1:], h[:-1])
    np.testing.assert_array_equal(s[0], 0.0)


def test_softplus_matches_logaddexp_without_overflow():
    v = np.linspace(-800.0, 800.0, 3201)
    with np.errstate(over="raise"):
        np.testing.assert_allclose(orc.softplus(v), np.logaddexp(0.0, v), rtol=1e-14, atol=1e-300)


def _scan_brute(u, delta, A, B, C, D):
    """y_t = sum_{s <= t} sum_n C_t[n] exp(A[:, n] sum_{r=s+1..t} delta_r) delta_s u_s B_s[n]
    + D u_t, summed directly (no recurrence)."""
    L, Dd = u.shape
    y = np.zeros((L, Dd))
    for t in range(L):
        for s in range(t + 1):
            decay = np.exp(A * delta[s + 1:t + 1].sum(axis=0)[:, None])  # [D, N]
            y[t] += (decay * (delta[s] * u[s])[:, None] * B[s][None, :]) @ C[t]
        y[t] += D * u[t]
    return y


def test_selective_scan_matches_the_direct_sum():
    rng = np.random.default_rng(1)
    L, Dd, N = 12, 3, 4
    u = rng.standard_normal((L, Dd))
    delta = rng.uniform(0.01, 0.5, (L, Dd))
    A = -rng.uniform(0.2, 3.0, (Dd, N))
    B = rng.standard_normal((L, N))
    C = rng.standard_normal((L, N))
    D = rng.standard_normal(Dd)
    np.testing.assert_allclose(orc.selective_scan(u, delta, A, B, C, D),
                               _scan_brute(u, delta, A, B, C, D), rtol=1e-12, atol=1e-12)


def test_selective_scan_first_step_and_causality():
    rng = np.random.default_rng(2)
    L, Dd, N = 20, 4, 3
    u = rng.standard_normal((L, Dd))
    delta = rng.uniform(0.01, 0.5, (L, Dd))
    A = -rng.uniform(0.2, 3.0, (Dd, N))
    B = rng.standard_normal((L, N))
    C = rng.standard_normal((L, N))
    D = rng.standard_normal(Dd)
    y = orc.selective_scan(u, delta, A, B, C, D)
    # first step: h_1 = delta u B, y = delta u (B . C) + D u
    np.testing.assert_allclose(y[0], delta[0] * u[0] * (B[0] @ C[0]) + D * u[0], rtol=1e-14)
    u2 = u.copy()
    u2[9] += 5.0
    y2 = orc.selective_scan(u2, delta, A, B, C, D)
    np.testing.assert_array_equal(y2[:9], y[:9])
    assert np.all(np.abs(y2[9:] - y[9:]).max(axis=1) > 0)


def test_selective_scan_time_invariant_is_a_convolution():
    """Constant delta, B, C (one state): y = u * k + D u with the geometric
    kernel k_j = C exp(delta A)^j delta B."""
    rng = np.random.default_rng(3)
    L = 30
    u = rng.standard_normal((L, 1))
    dlt, a, b, c, d = 0.3, -0.7, 1.3, -0.4, 0.25
    y = orc.selective_scan(u, np.full((L, 1), dlt), np.array([[a]]), np.full((L, 1), b),
                           np.full((L, 1), c), np.array([d]))
    kern = c * np.exp(dlt * a) ** np.arange(L) * dlt * b
    ref = np.convolve(u[:, 0], kern, mode="full")[:L] + d * u[:, 0]
    np.testing.assert_allclose(y[:, 0], ref, rtol=1e-12, atol=1e-13)


def _core_params(De, N=4, R=3, K=4, seed=0):
    rng = np.random.default_rng(seed)
    return dict(conv_w=rng.standard_normal((De, K)) / 2, conv_b=0.1 * rng.standard_normal(De),
                w_x=rng.standard_normal((De, R + 2 * N)) / np.sqrt(De),
                w_dt=rng.standard_normal((R, De)) / np.sqrt(R),
                b_dt=rng.uniform(np.log(1e-3), np.log(1e-1), De),
                a_log=rng.uniform(0.0, 2.0, (De, N)), d=rng.uniform(0.5, 1.5, De))


def test_core_restarts_at_every_sequence():
    rng = np.random.default_rng(4)
    H = rng.standard_normal((24, 6))
    core = _core_params(6)
    both = orc.ssm_core(H, core, seq_len=12)["Y"]
    np.testing.assert_allclose(both[:12], orc.ssm_core(H[:12], core)["Y"], rtol=1e-14)
    np.testing.assert_allclose(both[12:], orc.ssm_core(H[12:], core)["Y"], rtol=1e-14)


def test_core_without_state_input_is_the_gated_skip():
    """B = 0 (its columns of W_x zero): the state stays 0 and Y = D (.)
    SiLU(conv(H)); with a delta kernel and no bias, Y = D (.) SiLU(H)."""
    rng = np.random.default_rng(5)
    De, N, R = 6, 4, 3
    H = rng.standard_normal((15, De))
    core = _core_params(De, N=N, R=R)
    core["w_x"][:, R:R + N] = 0.0
    core["conv_w"][:] = 0.0
    core["conv_w"][:, -1] = 1.0
    core["conv_b"][:] = 0.0
    np.testing.assert_allclose(orc.ssm_core(H, core)["Y"], core["d"] * _silu_ref(H), rtol=1e-14)


def test_block_with_core_uses_y_in_place_of_h():
    """E = 1 block with the core: O = (core(x W_in) (.) SiLU(x W_g)) W_out,
    the core evaluated on its own; and with a core that reduces to
    Y = D (.) SiLU(H) the block output follows in closed form."""
    inp = make_block_inputs(20, 8, 6, 1, seed=6)
    core = _core_params(6)
    x = inp["x"].astype(np.float64)
    o = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                          core=core)["O"]
    H = x @ inp["w_conv"][0]
    Y = orc.ssm_core(H, core)["Y"]
    np.testing.assert_allclose(o, (Y * _silu_ref(x @ inp["w_gate"][0])) @ inp["w_out"][0],
                               rtol=1e-12, atol=1e-13)
    core["w_x"][:, 3:7] = 0.0
    core["conv_w"][:] = 0.0
    core["conv_w"][:, -1] = 1.0
    core["conv_b"][:] = 0.0
    o2 = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                           core=core)["O"]
    ref = ((core["d"] * _silu_ref(H)) * _silu_ref(x @ inp["w_gate"][0])) @ inp["w_out"][0]
    np.testing.assert_allclose(o2, ref, rtol=1e-12, atol=1e-13)
    with pytest.raises(ValueError):
        orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                          core=core, tokens=[0, 1])


def test_core_equals_its_pieces_computed_independently():
    """The core's composition -- SiLU(conv), [dt | B | C] = X W_x in that
    order, delta = softplus(dt W_dt + b_dt), A = -exp(A_log), the scan --
    evaluated with numpy's convolution, logaddexp and the scan's direct sum."""
    rng = np.random.default_rng(7)
    De, N, R, L = 5, 3, 2, 14
    H = rng.standard_normal((L, De))
    core = _core_params(De, N=N, R=R, seed=8)
    X = np.stack([np.convolve(H[:, d], core["conv_w"][d, ::-1], mode="full")[:L]
                  for d in range(De)], axis=1) + core["conv_b"]
    X = _silu_ref(X)
    dbc = X @ core["w_x"]
    delta = np.logaddexp(0.0, dbc[:, :R] @ core["w_dt"] + core["b_dt"])
    ref = _scan_brute(X, delta, -np.exp(core["a_log"]), dbc[:, R:R + N], dbc[:, R + N:],
                      core["d"])
    np.testing.assert_allclose(orc.ssm_core(H, core)["Y"], ref, rtol=1e-11, atol=1e-12)


def test_core_is_stable_over_long_sequences():
    """A = -exp(A_log) < 0 makes every step contractive: with bounded inputs
    the output stays bounded over a long sequence (the stability the Swimba
    page states for a contractive transition)."""
    rng = np.random.default_rng(9)
    H = rng.standard_normal((600, 4))
    core = _core_params(4, seed=10)
    y = orc.ssm_core(H, core)["Y"]
    assert np.all(np.isfinite(y)) and np.abs(y).max() < 50.0


def test_block_with_core_restarts_per_sequence():
    inp = make_block_inputs(24, 8, 6, 3, seed=11, router_std=0.5)
    core = _core_params(6, seed=12)
    both = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                             core=core, seq_len=12)["O"]
    for a in (0, 12):
        one = orc.block_forward(inp["x"][a:a + 12], inp["w_r"], inp["w_conv"], inp["w_gate"],
                                inp["w_out"], 1, core=core)["O"]
        np.testing.assert_allclose(both[a:a + 12], one, rtol=1e-13, atol=1e-14)


def _routed_core_params(De, E, N=3, R=2, seed=0):
    base = _core_params(De, N=N, R=R, seed=seed)
    rng = np.random.default_rng(seed + 100)
    base["w_x"] = rng.standard_normal((E, De, R + 2 * N)) / np.sqrt(De)
    base["w_dt"] = rng.standard_normal((E, R, De)) / np.sqrt(R)
    return base


def test_routed_core_with_identical_experts_is_the_shared_core():
    rng = np.random.default_rng(13)
    De, E = 5, 4
    H = rng.standard_normal((30, De))
    p = _routed_core_params(De, E)
    p["w_x"][:] = p["w_x"][0]
    p["w_dt"][:] = p["w_dt"][0]
    shared = dict(p, w_x=p["w_x"][0], w_dt=p["w_dt"][0])
    S = rng.integers(0, E, (30, 1))
    np.testing.assert_allclose(orc.ssm_core(H, p, topk_idx=S)["Y"], orc.ssm_core(H, shared)["Y"],
                               rtol=1e-13, atol=1e-14)


def test_routed_core_top1_uses_each_tokens_expert():
    """Top-1: token t's [dt | B | C] is X_t W_x[e_t] and its dt projection
    uses W_dt[e_t]; built token by token and fed to the scan's direct sum."""
    rng = np.random.default_rng(14)
    De, E, N, R, L = 4, 3, 3, 2, 12
    H = rng.standard_normal((L, De))
    p = _routed_core_params(De, E, N=N, R=R, seed=15)
    S = rng.integers(0, E, (L, 1))
    X = _silu_ref(orc.causal_conv1d(H, p["conv_w"], p["conv_b"]))
    dbc = np.stack([X[t] @ p["w_x"][S[t, 0]] for t in range(L)])
    pre = np.stack([dbc[t, :R] @ p["w_dt"][S[t, 0]] for t in range(L)])
    delta = np.logaddexp(0.0, pre + p["b_dt"])
    ref = _scan_brute(X, delta, -np.exp(p["a_log"]), dbc[:, R:R + N], dbc[:, R + N:], p["d"])
    np.testing.assert_allclose(orc.ssm_core(H, p, topk_idx=S)["Y"], ref, rtol=1e-11, atol=1e-12)


def test_block_with_routed_core_uses_the_block_routing():
    """In the block, the expertized x and dt projections follow S_t: with
    k = E every expert is selected, so they see the sum of all experts'
    matrices (a shared core with the summed weights)."""
    E = 3
    inp = make_block_inputs(16, 8, 6, E, seed=16, router_std=0.5)
    p = _routed_core_params(6, E, seed=17)
    summed = dict(p, w_x=p["w_x"].sum(axis=0), w_dt=p["w_dt"].sum(axis=0))
    a = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], E,
                          core=p)["O"]
    b = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], E,
                          core=summed)["O"]
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_block_with_routed_core_top1_follows_its_router():
    """Top-1 block with an expertized core equals its pieces: the routing of
    the block's router drives Conv, Gate, the x and dt projections and Out."""
    E = 3
    inp = make_block_inputs(16, 8, 6, E, seed=18, router_std=0.5)
    p = _routed_core_params(6, E, seed=19)
    o = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                          core=p)["O"]
    x = inp["x"].astype(np.float64)
    pr = sp_softmax(x @ inp["w_r"].astype(np.float64), axis=1)
    e = np.argmax(pr, axis=1)
    H = np.stack([x[t] @ inp["w_conv"][e[t]] for t in range(16)])
    G = _silu_ref(np.stack([x[t] @ inp["w_gate"][e[t]] for t in range(16)]))
    Y = orc.ssm_core(H, p, topk_idx=e[:, None])["Y"]
    ref = np.stack([pr[t, e[t]] * ((Y[t] * G[t]) @ inp["w_out"][e[t]]) for t in range(16)])
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)
