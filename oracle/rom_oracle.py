"""CPU oracle of the Routing Mamba (RoM) mixture-of-experts projection block.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` call it. It shares no code with the CUDA library.

Plain, slow, float64 numpy. Every function follows a passage of the pages:

* "Routing Mamba: Scaling State Space Models with Mixture-of-Experts
  Projection" (chapterpal summary page), Knowl 1 -- the router
  p_t = Softmax(x_t W_r), the top-K set S_t, the routing weights
  r_{t,i} = p_{t,i} 1[i in S_t], the shared-selection input and gate
  projections H_t and G_t = SiLU(sum ...), and the block output
  O_t = sum_i r_{t,i} (Y_t (.) G_t) W_out,i.
* Same page, Knowl 12 -- dropless dispatch: no expert parallelism, no
  capacity factor, no token dropping (every selected (token, expert) pair is
  computed).
* "Swimba: Switch Mamba Model Scales State Space Models" (project page),
  Extended abstract, second paragraph -- expert in-projections emit the X, B
  and C streams, and the routing-weighted streams are summed.

Readings taken where the pages are silent:

* The short convolution and selective scan between the projections are not
  changed by the method; the oracle stands the identity in for them (Y = H).
* S_t is chosen on the logits (softmax is strictly increasing, so the K
  largest logits are the K largest probabilities); equal logits go to the
  lower expert index, and the slots of S_t are ordered by descending logit.
* ``renorm=True`` divides the selected probabilities by their sum (the top-2
  workload); otherwise r = p as the formula states.
* An optional additive router bias is added to the logits before softmax.
* The expert permutation is expert-major and, inside an expert, ascending
  in token (slot) index.
* The backward treats S_t as fixed (piecewise-constant selection) and returns
  the exact gradient of the forward above.

Weights are taken in the pages' notation: W_in,i and W_g,i are [D_m, D_e]
(used as x W), W_out,i is [D_e, D_m]. Arrays are stacked on a leading expert
axis.
"""
from __future__ import annotations

import numpy as np


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def sigmoid(z):
    """Logistic function 1 / (1 + exp(-z)), written to avoid overflow."""
    z = np.asarray(z, dtype=np.float64)
    out = np.empty_like(z)
    pos = z >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-z[pos]))
    ez = np.exp(z[~pos])
    out[~pos] = ez / (1.0 + ez)
    return out


def silu(z):
    """SiLU(z) = z * sigmoid(z) (Elfwing et al., cited by the RoM page for SiLU)."""
    return np.asarray(z, dtype=np.float64) * sigmoid(z)


def silu_grad(z):
    """d/dz SiLU(z) = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    s = sigmoid(z)
    return s * (1.0 + np.asarray(z, np.float64) * (1.0 - s))


def softmax(logits):
    """Row-wise softmax exp(l - max) / sum exp(l - max)."""
    l = _f64(logits)
    m = l.max(axis=-1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=-1, keepdims=True)


def route(x, w_r, k, bias=None, renorm=False):
    """RoM router (RoM page, Knowl 1): logits, probabilities, S_t and r_{t,i}.

    Returns a dict with
      logits [T,E], p [T,E],
      topk_idx [T,k] int32: S_t, slot j holds the j-th largest logit
        (equal logits: lower expert index first),
      topk_w [T,k] float64: r_{t,S_t[j]} (= p, or p / sum_S p if renorm),
      margin [T]: the smallest logit gap that decides S_t and its slot order
        (used to flag tokens whose choice is numerically ambiguous).
    """
    x = _f64(x)
    logits = x @ _f64(w_r)
    if bias is not None:
        logits = logits + _f64(bias)[None, :]
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("k must be in [1, E]")
    p = softmax(logits)
    # Order experts per token by (descending logit, ascending index).
    order = np.empty((T, E), dtype=np.int64)
    for t in range(T):
        order[t] = sorted(range(E), key=lambda i: (-logits[t, i], i))
    topk_idx = order[:, :k].astype(np.int32)
    rows = np.arange(T)[:, None]
    r = p[rows, topk_idx]
    if renorm:
        r = r / r.sum(axis=1, keepdims=True)
    # Decision margin: gaps between consecutive sorted logits up to slot k.
    srt = logits[rows, order]
    ngaps = k if k < E else k - 1
    if ngaps > 0:
        gaps = srt[:, :ngaps] - srt[:, 1:ngaps + 1]
        margin = gaps.min(axis=1)
    else:
        margin = np.full(T, np.inf)
    return dict(logits=logits, p=p, topk_idx=topk_idx, topk_w=r, margin=margin)


def dispatch(topk_idx, E):
    """Dropless dispatch order (RoM page, Knowl 12; order reading in the header).

    Slots are numbered s = t*k + j. Returns
      counts [E]: number of slots routed to each expert,
      offsets [E+1]: exclusive prefix sum of counts,
      sorted_slot [R]: sorted position -> slot (expert-major, ascending slot),
      slot_pos [R]: slot -> sorted position.
    Written as a counting sort with explicit loops.
    """
    idx = np.asarray(topk_idx).reshape(-1)
    R = idx.shape[0]
    counts = np.zeros(E, dtype=np.int64)
    for s in range(R):
        counts[int(idx[s])] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    cursor = offsets[:E].copy()
    sorted_slot = np.empty(R, dtype=np.int64)
    slot_pos = np.empty(R, dtype=np.int64)
    for s in range(R):
        e = int(idx[s])
        sorted_slot[cursor[e]] = s
        slot_pos[s] = cursor[e]
        cursor[e] += 1
    return dict(counts=counts.astype(np.int32), offsets=offsets.astype(np.int32),
                sorted_slot=sorted_slot.astype(np.int32), slot_pos=slot_pos.astype(np.int32))


def block_forward(x, w_r, w_in, w_g, w_out, k, bias=None, renorm=False, tokens=None,
                  core=None, seq_len=None):
    """RoM projection block forward (RoM page, Knowl 1).

    H_t = sum_i 1[i in S_t] x_t W_in,i ;  G_t = SiLU(sum_i 1[i in S_t] x_t W_g,i)
    Y_t = H_t (identity stand-in for the unchanged conv + SSM core), or
    Y = ssm_core(H) when ``core`` holds the core's parameters
    O_t = sum_i r_{t,i} (Y_t (.) G_t) W_out,i

    ``tokens`` (optional index array) evaluates only those tokens; without
    the core every token is independent of the others in this block (with
    the core, ``tokens`` is refused: a token depends on its sequence's past).
    ``seq_len``: the tokens are consecutive sequences of that length (for
    the core). A core whose w_x and w_dt hold one matrix per expert
    ([E, ...]) has its x and dt projections routed with S_t as well.
    Returns a dict with O [T,Dm], H, Gpre (the sum before SiLU), G, YG [T,De]
    and the router outputs.
    """
    x = _f64(x)
    if tokens is not None:
        x = x[np.asarray(tokens)]
    rt = route(x, w_r, k, bias=bias, renorm=renorm)
    S, r = rt["topk_idx"], rt["topk_w"]
    T = x.shape[0]
    E, Dm, De = np.shape(w_in)
    H = np.zeros((T, De))
    Gpre = np.zeros((T, De))
    for i in range(E):
        for j in range(k):
            sel = np.nonzero(S[:, j] == i)[0]
            if sel.size == 0:
                continue
            H[sel] += x[sel] @ _f64(w_in[i])
            Gpre[sel] += x[sel] @ _f64(w_g[i])
    G = silu(Gpre)
    if core is None:
        Y = H
    else:
        if tokens is not None:
            raise ValueError("the core mixes tokens over time: evaluate whole sequences")
        routed = np.ndim(core["w_x"]) == 3  # x and dt projections expertized
        Y = ssm_core(H, core, seq_len, topk_idx=S if routed else None)["Y"]
    YG = Y * G
    O = np.zeros((T, Dm))
    for i in range(E):
        for j in range(k):
            sel = np.nonzero(S[:, j] == i)[0]
            if sel.size == 0:
                continue
            O[sel] += r[sel, j][:, None] * (YG[sel] @ _f64(w_out[i]))
    return dict(O=O, H=H, Gpre=Gpre, G=G, Y=Y, YG=YG, **rt)


def inproj_forward(x, w_r, w, k=1, bias=None, renorm=False, tokens=None):
    """Swimba routed in-projection (Swimba page, Extended abstract, paragraph 2).

    s_t = sum_i r_{t,i} x_t W_i, with W_i [D_m, N_out] producing the X | B | C
    streams side by side. Returns a dict with S [T,N_out] and router outputs.
    """
    x = _f64(x)
    if tokens is not None:
        x = x[np.asarray(tokens)]
    rt = route(x, w_r, k, bias=bias, renorm=renorm)
    idx, r = rt["topk_idx"], rt["topk_w"]
    T = x.shape[0]
    E, Dm, N = np.shape(w)
    s = np.zeros((T, N))
    for i in range(E):
        for j in range(k):
            sel = np.nonzero(idx[:, j] == i)[0]
            if sel.size == 0:
                continue
            s[sel] += r[sel, j][:, None] * (x[sel] @ _f64(w[i]))
    return dict(S=s, **rt)


def block_backward(x, w_r, w_in, w_g, w_out, dout, k, bias=None, renorm=False):
    """Exact gradient of ``block_forward`` for L = sum_t <O_t, dO_t>, S_t held fixed.

    With g_{t,j} = dO_t W_out,S_j^T and dr_{t,j} = <Y_t (.) G_t, g_{t,j}>:
      d(YG)_t = sum_j r_{t,j} g_{t,j};  dH = d(YG) (.) G;  dGpre = d(YG) (.) Y (.) SiLU'(Gpre)
      dW_in,i  = sum_{t: i in S_t} x_t^T dH_t
      dW_g,i   = sum_{t: i in S_t} x_t^T dGpre_t
      dW_out,i = sum_{(t,j): S_tj = i} r_{t,j} (Y_t (.) G_t)^T dO_t
      dlogits  = Jacobian of r w.r.t. the logits applied to dr
                 (full softmax if not renorm; softmax over S_t if renorm)
      dX = sum_j (dH W_in,S_j^T + dGpre W_g,S_j^T) + dlogits W_r^T
      dW_r = X^T dlogits, dbias = sum_t dlogits_t
    """
    x = _f64(x)
    dout = _f64(dout)
    fw = block_forward(x, w_r, w_in, w_g, w_out, k, bias=bias, renorm=renorm)
    S, r, p = fw["topk_idx"], fw["topk_w"], fw["p"]
    H, G, Gpre, YG = fw["H"], fw["G"], fw["Gpre"], fw["YG"]
    T, Dm = x.shape
    E, _, De = np.shape(w_in)
    dYG = np.zeros((T, De))
    dr = np.zeros((T, k))
    dW_out = np.zeros((E, De, Dm))
    for i in range(E):
        for j in range(k):
            sel = np.nonzero(S[:, j] == i)[0]
            if sel.size == 0:
                continue
            g = dout[sel] @ _f64(w_out[i]).T
            dr[sel, j] = np.sum(YG[sel] * g, axis=1)
            dYG[sel] += r[sel, j][:, None] * g
            dW_out[i] += (r[sel, j][:, None] * YG[sel]).T @ dout[sel]
    dH = dYG * G
    dGpre = dYG * H * silu_grad(Gpre)
    dX = np.zeros((T, Dm))
    dW_in = np.zeros((E, Dm, De))
    dW_g = np.zeros((E, Dm, De))
    for i in range(E):
        for j in range(k):
            sel = np.nonzero(S[:, j] == i)[0]
            if sel.size == 0:
                continue
            dW_in[i] += x[sel].T @ dH[sel]
            dW_g[i] += x[sel].T @ dGpre[sel]
            dX[sel] += dH[sel] @ _f64(w_in[i]).T + dGpre[sel] @ _f64(w_g[i]).T
    dlogits = np.zeros((T, E))
    rows = np.arange(T)
    if renorm:
        # r_j = exp(l_Sj) / sum_{i in S} exp(l_i): softmax over the selected logits.
        inner = np.sum(r * dr, axis=1)
        for j in range(k):
            dlogits[rows, S[:, j]] += r[:, j] * (dr[:, j] - inner)
    else:
        # r_j = p_{S_j}, p = softmax(l): dl_m = sum_j dr_j p_Sj (delta_{m,Sj} - p_m).
        inner = np.sum(dr * p[rows[:, None], S], axis=1)
        dlogits -= p * inner[:, None]
        for j in range(k):
            dlogits[rows, S[:, j]] += dr[:, j] * p[rows, S[:, j]]
    dX += dlogits @ _f64(w_r).T
    dW_r = x.T @ dlogits
    dbias = dlogits.sum(axis=0)
    return dict(dX=dX, dW_in=dW_in, dW_g=dW_g, dW_out=dW_out, dlogits=dlogits, dr=dr,
                dW_r=dW_r, dbias=dbias, forward=fw)


def variant_block_forward(x, w_in, w_g, w_out, k, routers, weighted, bias=None, renorm=False,
                          tokens=None):
    """Mamba projection block whose three projections are each dense or routed.

    Covers the configurations the RoM page compares (Knowl 3 and Knowl 4):
      * RoM (Conv, Gate, Out): one router shared by the three projections;
        only Out is weighted by r (Knowl 1). Equals ``block_forward``.
      * RoM (Gate, Out): Conv is a dense projection; Gate and Out share one
        router (Knowl 3, "Samba + RoM (Gate, Out)").
      * Independent MoE on Conv, Gate and Out: each projection is a
        conventional MoE layer with its own router, its experts' outputs
        weighted by that router's probabilities (Knowl 4).

    ``routers`` maps "conv", "gate" and "out" to a router weight [D_m, E] or
    to None for a dense projection (the weight stack then holds one matrix
    and it is applied to every token with weight 1). Routers are evaluated
    separately for each projection; passing the same matrix twice shares the
    decision, since it is the same computation. ``weighted`` maps the three
    names to True when that projection's expert outputs are scaled by r.
    ``bias`` is an optional additive logit bias used by every router.

    H_t = sum_{i in S^conv_t} w^conv_{t,i} x_t W_in,i
    G_t = SiLU(sum_{i in S^gate_t} w^gate_{t,i} x_t W_g,i)
    O_t = sum_{i in S^out_t} w^out_{t,i} (Y_t (.) G_t) W_out,i,   Y = H,
    with w = r for a weighted projection, 1 otherwise.
    Returns a dict with O, H, Gpre, G, YG and the three routings.
    """
    x = _f64(x)
    if tokens is not None:
        x = x[np.asarray(tokens)]
    T = x.shape[0]

    def routing(name):
        w_r = routers.get(name)
        if w_r is None:
            return None
        return route(x, w_r, k, bias=bias, renorm=renorm)

    def project(name, a, w):
        """Sum over the projection's selected experts of (weight) * a W_i."""
        rt = rts[name]
        N = np.shape(w)[2]
        out = np.zeros((T, N))
        if rt is None:
            return out + a @ _f64(w[0])
        S, r = rt["topk_idx"], rt["topk_w"]
        for i in range(np.shape(w)[0]):
            for j in range(k):
                sel = np.nonzero(S[:, j] == i)[0]
                if sel.size == 0:
                    continue
                part = a[sel] @ _f64(w[i])
                if weighted[name]:
                    part = r[sel, j][:, None] * part
                out[sel] += part
        return out

    rts = {n: routing(n) for n in ("conv", "gate", "out")}
    H = project("conv", x, w_in)
    Gpre = project("gate", x, w_g)
    G = silu(Gpre)
    YG = H * G
    O = project("out", YG, w_out)
    return dict(O=O, H=H, Gpre=Gpre, G=G, YG=YG, routing=rts)


def softplus(v):
    """softplus(v) = ln(1 + e^v), written to avoid overflow."""
    v = np.asarray(v, dtype=np.float64)
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def causal_conv1d(h, w, b):
    """Short causal depthwise convolution over time (one sequence).

    h [L, D]; w [D, K] (tap K-1 multiplies the current step, tap K-1-j the
    step j back); b [D]. out_t = b + sum_j w[:, K-1-j] * h_{t-j}, with
    h_{t-j} = 0 before the start of the sequence.
    """
    h = _f64(h)
    w = _f64(w)
    L, D = h.shape
    K = w.shape[1]
    out = np.zeros((L, D)) + _f64(b)[None, :]
    for j in range(K):
        out[j:] += w[:, K - 1 - j][None, :] * h[:L - j]
    return out


def selective_scan(u, delta, A, B, C, D):
    """Selective state-space recurrence of one sequence (Mamba, Gu and Dao
    2023, Section 3: zero-order hold for A, Euler step for the input).

    u, delta [L, D]; A [D, N]; B, C [L, N]; D [D]. With the state
    h_t [D, N] (h_0 = 0 before the first step):
      h_t = exp(delta_t A) (.) h_{t-1} + (delta_t u_t) B_t
      y_t = h_t C_t + D (.) u_t
    Returns y [L, D].
    """
    u, delta, A, B, C, D = (_f64(a) for a in (u, delta, A, B, C, D))
    L, Dd = u.shape
    h = np.zeros(A.shape)
    y = np.empty((L, Dd))
    for t in range(L):
        h = np.exp(delta[t][:, None] * A) * h + (delta[t] * u[t])[:, None] * B[t][None, :]
        y[t] = h @ C[t] + D * u[t]
    return y


def _routed_projection(a, w, topk_idx):
    """sum_j a_t W[S_tj] for every token t (unweighted, like the Conv and
    Gate projections of RoM): a [T, K], w [E, K, N], topk_idx [T, k]."""
    T = a.shape[0]
    E, _, N = np.shape(w)
    out = np.zeros((T, N))
    for i in range(E):
        for j in range(topk_idx.shape[1]):
            sel = np.nonzero(topk_idx[:, j] == i)[0]
            if sel.size:
                out[sel] += a[sel] @ _f64(w[i])
    return out


def ssm_core(H, core, seq_len=None, topk_idx=None):
    """The dense core between the projections (RoM page, Knowl 1: the short
    convolution and selective state-space computation applied to H_t give
    Y_t; Knowl 9: the 1D convolution, x projection and dt projection are
    shared, not expertized), in the original Mamba form:

      X = SiLU(conv1d(H));  [dt | B | C] = X W_x;
      delta = softplus(dt W_dt + b_dt);  A = -exp(A_log);
      Y = selective_scan(X, delta, A, B, C, D).

    ``core`` holds conv_w [D_e, K], conv_b [D_e], w_x [D_e, R + 2N],
    w_dt [R, D_e], b_dt [D_e], a_log [D_e, N] and d [D_e]. The T rows of H
    are consecutive sequences of ``seq_len`` tokens (one sequence if None);
    the convolution and the state restart at every sequence.

    With ``topk_idx`` [T, k] (the block's routing) the x and dt projections
    are expertized too, like Conv and Gate (RoM page, Knowl 3 and Knowl 9:
    "RoM (Conv, Gate, dt, x, Out)"): w_x [E, D_e, R + 2N] and w_dt [E, R, D_e]
    hold one matrix per expert, and each token's [dt | B | C] and dt
    projection are the sums over its selected experts (unweighted).
    Returns Y [T, D_e] and the intermediates (X, delta, B, C).
    """
    H = _f64(H)
    T, De = H.shape
    L = T if seq_len is None else int(seq_len)
    if T % L:
        raise ValueError("T must be a multiple of seq_len")
    N = np.shape(core["a_log"])[1]
    R = np.shape(core["w_dt"])[-2]
    A = -np.exp(_f64(core["a_log"]))
    Y = np.empty((T, De))
    X = np.empty((T, De))
    dl = np.empty((T, De))
    Bs = np.empty((T, N))
    Cs = np.empty((T, N))
    for s0 in range(0, T, L):
        sl = slice(s0, s0 + L)
        xs = silu(causal_conv1d(H[sl], core["conv_w"], core["conv_b"]))
        if topk_idx is None:
            dbc = xs @ _f64(core["w_x"])
            pre = dbc[:, :R] @ _f64(core["w_dt"])
        else:
            S = np.asarray(topk_idx)[sl]
            dbc = _routed_projection(xs, core["w_x"], S)
            pre = _routed_projection(dbc[:, :R], core["w_dt"], S)
        delta = softplus(pre + _f64(core["b_dt"])[None, :])
        B, C = dbc[:, R:R + N], dbc[:, R + N:R + 2 * N]
        Y[sl] = selective_scan(xs, delta, A, B, C, core["d"])
        X[sl], dl[sl], Bs[sl], Cs[sl] = xs, delta, B, C
    return dict(Y=Y, X=X, delta=dl, B=Bs, C=Cs)
