/*
 * rom.h -- C ABI of librom.so, the sm_100a (B200) implementation of the
 * Routing Mamba (RoM) mixture-of-experts projection block.
 *
 * Method: "Routing Mamba: Scaling State Space Models with Mixture-of-Experts
 * Projection" (chapterpal summary page), Knowl 1. For a token x_t in R^{D_m},
 * a router W_r in R^{D_m x E} gives p_t = Softmax(x_t W_r) and the set S_t of
 * the K largest probabilities; r_{t,i} = p_{t,i} 1[i in S_t]. The same S_t
 * drives the input (Conv) and Gate projections
 *     H_t = sum_i 1[i in S_t] x_t W_in,i,   G_t = SiLU(sum_i 1[i in S_t] x_t W_g,i)
 * and, after the (unchanged, here identity) conv + SSM core Y_t, the output
 *     O_t = sum_i r_{t,i} (Y_t (.) G_t) W_out,i.
 * Knowl 12 of the same page: dropless (no capacity factor, no token dropping).
 * The Swimba in-projection ("Swimba: Switch Mamba Model Scales State Space
 * Models", project page, Extended abstract, paragraph 2) is the routed,
 * routing-weighted projection s_t = sum_i r_{t,i} x_t W_i of the X|B|C streams.
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers unless stated otherwise. The caller owns all
 *    memory; the library allocates nothing on these paths.
 *  - Row-major, contiguous. bf16 data is passed as raw 16-bit words.
 *  - Expert weights are stored [E][N][K] ("output feature major", the
 *    nn.Linear layout): row n of expert e holds the K weights of output
 *    feature n. In the pages' notation W_i in R^{K x N}, so the stored matrix
 *    is W_i transposed.
 *  - Slots: token t's j-th selected expert is slot s = t*k + j.
 *  - Every call is asynchronous on `stream` (a cudaStream_t, may be NULL for
 *    the legacy default stream) and enqueues no host synchronisation.
 *  - The return value reports argument validation and launch errors
 *    (rom_status). Errors found on the device (a bounded wait that ran out)
 *    are recorded in a per-device status word read by rom_get_status().
 *  - Arguments are checked before anything is launched; on a non-zero return
 *    nothing was enqueued, unless the code is ROM_ERR_CUDA from a launch.
 */
#ifndef ROM_H_
#define ROM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ROM_OK = 0,
  ROM_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad enum, k > E, ... */
  ROM_ERR_UNSUPPORTED = 2, /* valid but not implemented (shape or alignment limit) */
  ROM_ERR_WORKSPACE = 3,   /* workspace missing or smaller than rom_workspace_size() */
  ROM_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  ROM_ERR_TIMEOUT = 5,     /* device side: a bounded wait ran out (see rom_get_status) */
  ROM_ERR_ROUTING = 6      /* device side: rom_dispatch found expert indices outside [0, E) or
                              histograms that do not match them (see rom_get_status) */
} rom_status;

typedef enum { ROM_F32 = 0, ROM_BF16 = 1 } rom_dtype;

typedef enum {
  ROM_PROJ_CONV_GATE = 0, /* Conv (input) and Gate projections, shared selection */
  ROM_PROJ_OUT = 1,       /* Out projection, weighted by r */
  ROM_PROJ_INPROJ = 2,    /* Swimba routed in-projection, weighted by r */
  ROM_PROJ_SLOTS = 3,     /* one projection to float32 slot rows (Conv or Gate on their own) */
  ROM_PROJ_CONV_GATE_SLOTS = 4 /* Conv and Gate to float32 u, z slot rows for any k */
} rom_proj;

/* Flag OR'd into `proj` of rom_expert_proj_dense: the weights are in the
 * tile-major layout written by rom_pack_expert_weights. */
#define ROM_W_TILED 0x100

typedef enum {
  ROM_COMBINE_SUM = 0,       /* out[t] = sum_j in[t*k+j]                     */
  ROM_COMBINE_GATE = 1,      /* h_t = (sum_j u_{t,j}) * SiLU(sum_j z_{t,j}) */
  ROM_COMBINE_GATE_DENSE = 2 /* h_t = u_t * SiLU(sum_j z_{t,j}), u_t dense  */
} rom_combine_mode;

/* Human-readable name of a rom_status value (static string). */
const char* rom_status_string(int status);

/* ABI version of this library (incremented on incompatible changes). */
int rom_version(void);

/*
 * Bytes of workspace that rom_route() fills and rom_dispatch() reads for T
 * tokens and E experts (the per-chunk expert histograms). Host function.
 */
size_t rom_workspace_size(int64_t T, int E);

/*
 * rom_route -- router: logits, softmax, top-k selection and expert histogram
 * (RoM page, Knowl 1: p_t = Softmax(x_t W_r), S_t, r_{t,i}).
 *
 *  x        [T][Dm]   activations, dtype (ROM_BF16 words or float)
 *  w_r      [Dm][E]   router weight, float32 (both dtypes)
 *  bias     [E]       optional additive logit bias, float32, or NULL
 *  k                  experts per token, 1 <= k <= min(E, 8); E <= 64
 *  renorm             0: r = p (the formula); 1: r = p / sum_{S_t} p
 *  topk_idx [T][k]    out, int32: S_t, slot j = j-th largest logit; equal
 *                     logits go to the lower expert index
 *  topk_w   [T][k]    out, float32: r_{t, topk_idx[t][j]}
 *  counts   [E]       out, int32 per-expert slot count, or NULL (not written)
 *  ws, ws_bytes       workspace of at least rom_workspace_size(T, E) bytes;
 *                     rom_dispatch() must receive the same workspace, unchanged,
 *                     on the same stream, after this call. NULL when no
 *                     rom_dispatch follows (rom_expert_proj_dense): the per-chunk
 *                     histograms are then not formed.
 *
 * Precision: logits are accumulated in float32 in a fixed order together with
 * a rigorous bound on their rounding error; a token whose top-k decision is
 * not certain under that bound has its logits recomputed in float64 before
 * the decision. The softmax is evaluated in float32.
 * Requires Dm % 8 == 0 for bf16 and Dm % 4 == 0 for float32 (16-byte rows).
 */
int rom_route(const void* x, int dtype, int64_t T, int Dm, const float* w_r, const float* bias,
              int E, int k, int renorm, int32_t* topk_idx, float* topk_w, int32_t* counts,
              void* ws, size_t ws_bytes, void* stream);

/*
 * rom_dispatch -- dropless permutation into expert-contiguous order
 * (RoM page, Knowl 12: no capacity factor, no token dropping).
 * Order: expert-major, ascending slot index inside an expert (stable).
 *
 *  x           [T][Dm]   activations (as given to rom_route)
 *  topk_idx    [T][k]    from rom_route
 *  ws, ws_bytes          the workspace rom_route filled
 *  offsets     [E+1]     out, int32: exclusive prefix of the per-expert counts;
 *                        offsets[E] = T*k
 *  sorted_slot [T*k]     out, int32: sorted position -> slot
 *  slot_pos    [T*k]     out, int32: slot -> sorted position
 *  x_sorted    [T*k][Dm] out, dtype: x_sorted[p] = x[sorted_slot[p] / k]
 *
 * The kernel checks topk_idx and the workspace before using them as indices:
 * every index must lie in [0, E), and the histograms must be the ones
 * rom_route() wrote for these indices. If not (for example after the router
 * gave up on a bounded wait), it records ROM_ERR_ROUTING in the device status
 * word (rom_get_status) and writes outputs that stay in range for the kernels
 * that read them (offsets monotone in [0, T*k], sorted_slot and slot_pos in
 * [0, T*k)); their values then carry no meaning.
 */
int rom_dispatch(const void* x, int dtype, int64_t T, int Dm, int E, int k,
                 const int32_t* topk_idx, const void* ws, size_t ws_bytes, int32_t* offsets,
                 int32_t* sorted_slot, int32_t* slot_pos, void* x_sorted, void* stream);

/*
 * rom_expert_proj -- grouped expert projection over the dispatched rows.
 * For expert e, rows offsets[e] .. offsets[e+1]-1 of `a_sorted` ([R][K],
 * R = T*k) are multiplied by expert e's matrix; the experts' row counts are
 * read on the device (no host synchronisation).
 *
 *  ROM_PROJ_CONV_GATE (RoM page, Knowl 1, H_t and G_t):
 *     w0 = W_in [E][N][K], w1 = W_g [E][N][K]  (K = D_m, N = D_e)
 *     k == 1: out = h_sorted [R][N] dtype, h = u * SiLU(z) with u = x W_in,e,
 *             z = x W_g,e (the identity stands in for the conv + SSM core);
 *     k  > 1: out = float32 [2][R][N] in SLOT order: out[0][s] = u, out[1][s] = z
 *             of slot s; rom_combine(ROM_COMBINE_GATE) then sums over the
 *             slots before SiLU.
 *  ROM_PROJ_CONV_GATE_SLOTS: as ROM_PROJ_CONV_GATE with k > 1 (u and z as
 *     float32 [2][R][N] in slot order) for any k, including k == 1: the
 *     input of the dense core (rom_ssm_core), which needs H before the gate.
 *  ROM_PROJ_OUT (RoM page, Knowl 1, O_t): w0 = W_out [E][N][K] (K = D_e, N = D_m),
 *     w1 = NULL. Each row is scaled by r = topk_w[slot] in float32.
 *     k == 1: out = O [T][N] dtype in token order;
 *     k  > 1: out = float32 [R][N] in slot order (rom_combine(ROM_COMBINE_SUM)).
 *  ROM_PROJ_INPROJ (Swimba page, Extended abstract): w0 = W [E][N][K], the
 *     X|B|C in-projection; same weighting and outputs as ROM_PROJ_OUT.
 *  ROM_PROJ_SLOTS: w0 = W [E][N][K], w1 = NULL: one projection on its own,
 *     out = float32 [R][N] in SLOT order for any k, row s = the slot's sorted
 *     row times W_e^T, scaled by topk_w[s] when topk_w is not NULL and
 *     unscaled when it is NULL. With a router of its own this is the Conv or
 *     the Gate projection of independently routed MoE-Mamba, a conventional
 *     MoE layer per projection (RoM page, Knowl 4); with offsets == NULL,
 *     sorted_slot == NULL and E == 1 it is a dense projection of the R rows
 *     in row order (RoM page, Knowl 3: "RoM (Gate, Out)" keeps Conv dense).
 *     rom_combine(ROM_COMBINE_GATE or ROM_COMBINE_GATE_DENSE) then forms h.
 *  bf16 (tensor cores, tcgen05 + TMA): requires K % 8 == 0, N % 128 == 0 and
 *  16-byte aligned a_sorted, w0, w1 and out. float32 (CUDA-core FMA): any K, N.
 */
int rom_expert_proj(int proj, int dtype, const void* a_sorted, int64_t R, int K, const void* w0,
                    const void* w1, int N, int E, int k, const int32_t* offsets,
                    const int32_t* sorted_slot, const float* topk_w, void* out, void* stream);

/*
 * rom_expert_proj_dense -- the routed projection for a few tokens (T <= 64)
 * without a dispatch (Swimba page, Extended abstract: s_t = sum_j r_{t,j}
 * x_t W_{S_j}; RoM page, Knowl 1 for the Out projection). Every expert's
 * weight tiles meet all T tokens, taken in token order, and the routing
 * only selects in the epilogue: token t keeps expert e's result exactly when
 * e is one of its k selected experts. The weights stream once, as in
 * rom_expert_proj. Nothing before the epilogue depends on the routing, so
 * the kernel is launched as a programmatic dependent of the kernel before it
 * on the stream (the router: decode steps need no rom_dispatch) and only its
 * epilogue waits for that kernel's results.
 *
 *  proj      ROM_PROJ_INPROJ or ROM_PROJ_OUT (both weighted by r), optionally
 *            | ROM_W_TILED
 *  x         [T][K] bf16, token order (as given to rom_route)
 *  w         [E][N][K] bf16, or with ROM_W_TILED the same weights in the
 *            tile-major layout of rom_pack_expert_weights (which requires
 *            K % 64 == 0); the results are identical, the tiled weights
 *            stream as whole 16 KB blocks
 *  topk_idx, topk_w [T][k] from rom_route
 *  out       k == 1: [T][N] bf16, token order; k > 1: float32 [T*k][N] in slot
 *            order (then rom_combine(ROM_COMBINE_SUM))
 * Requires dtype ROM_BF16, 1 <= T <= 64, K % 8 == 0, N % 128 == 0 and
 * 16-byte aligned x, w and out.
 */
int rom_expert_proj_dense(int proj, int dtype, const void* x, int64_t T, int K, const void* w,
                          int N, int E, int k, const int32_t* topk_idx, const float* topk_w,
                          void* out, void* stream);

/*
 * rom_pack_expert_weights -- a one-time copy of expert weights into the
 * tile-major layout that rom_expert_proj_dense takes with ROM_W_TILED: the
 * 128 x 64 weight tiles the projection's kernel reads (128 output rows, 64
 * contraction elements) stored one after another, 16 KB each, so that every
 * tile is one contiguous read. No counterpart in the source pages: it is a
 * storage layout of the same W, not part of the method.
 *  w         [E][N][K] bf16 (as for rom_expert_proj_dense)
 *  w_tiled   out, E*N*K bf16 elements: element (e, n, c) at
 *            ((((e * N/128 + n/128) * K/64 + c/64) * 128 + n % 128) * 64 + c % 64)
 * Requires dtype ROM_BF16, N % 128 == 0, K % 64 == 0, 16-byte aligned
 * pointers and w_tiled not overlapping w.
 */
int rom_pack_expert_weights(int dtype, const void* w, int E, int N, int K, void* w_tiled,
                            void* stream);

/*
 * rom_combine -- reduce the k slots of each token in slot order 0..k-1.
 *  ROM_COMBINE_SUM:  in = float32 [T*k][N] (slot order); out = [T][N] dtype,
 *                    out[t] = sum_j in[t*k+j]. slot_pos is unused (may be NULL).
 *  ROM_COMBINE_GATE: in = float32 [2][T*k][N] (u then z, slot order);
 *                    h_t = (sum_j u[t*k+j]) * SiLU(sum_j z[t*k+j]) (RoM page,
 *                    Knowl 1: SiLU after the sum over the selected experts);
 *                    out = h_sorted [T*k][N] dtype with h_t written to row
 *                    slot_pos[t*k+j] for every j. u and z may come from
 *                    different routings (ROM_PROJ_SLOTS, each in its own slot
 *                    order); slot_pos is then the Out projection's. With
 *                    slot_pos == NULL, h_t is written once, to row t (a dense
 *                    Out projection reads h in token order).
 *  ROM_COMBINE_GATE_DENSE: in = float32 [T + T*k][N]: rows 0..T-1 hold the
 *                    dense Conv projection u_t (token order), rows T.. the
 *                    Gate partials z in slot order; h_t = u_t * SiLU(sum_j
 *                    z[t*k+j]) written like ROM_COMBINE_GATE (RoM page,
 *                    Knowl 3, "RoM (Gate, Out)": Conv is not expertized).
 *  Requires N % 4 == 0.
 */
int rom_combine(int mode, int dtype, const void* in, int64_t T, int k, int N,
                const int32_t* slot_pos, void* out, void* stream);

/*
 * rom_get_status -- synchronises `stream`, copies the calling device's status
 * word to *host_status (host pointer) and resets it to ROM_OK. One word per
 * device, shared by all streams.
 */
int rom_get_status(void* stream, int32_t* host_status);

/*
 * rom_debug_wait_timeout -- launches one CTA that waits on an mbarrier that
 * nothing arrives on, with a limit of `limit_ns` nanoseconds (1e3 .. 1e10).
 * The wait must run out and record ROM_ERR_TIMEOUT in the status word; used
 * to test the bounded-wait path without hanging the GPU.
 */
int rom_debug_wait_timeout(uint64_t limit_ns, void* stream);

/* ------------------------------------------------------------------------
 * Backward of the block (bf16), for the loss L = sum_t <O_t, dO_t> with the
 * selection S_t held fixed (RoM page, Knowl 1, differentiated). With
 * g_{t,j} = dO_t W_out,S_j^T:
 *   dr_{t,j} = <Y_t (.) G_t, g_{t,j}>,   d(Y(.)G)_t = sum_j r_{t,j} g_{t,j},
 *   dH = d(Y(.)G) (.) G,   dZ = d(Y(.)G) (.) H (.) SiLU'(Z)   (Z: the gate sum),
 *   dlogit_{t,j} = r_j (dr_j - sum_i r_i dr_i)   (renormalised top-k weights),
 *   dX_t = sum_j (dH W_in,S_j^T + dZ W_g,S_j^T) + sum_j dlogit_j W_r[:, S_j],
 *   dW_in,e = sum_{t->e} x_t^T dH_t,   dW_g,e = sum_{t->e} x_t^T dZ_t,
 *   dW_out,e = sum_{(t,j)->e} r_{t,j} (Y(.)G)_t^T dO_t.
 * Call order: rom_bwd_gather, rom_bwd_dgrad_out, rom_bwd_gate,
 * rom_bwd_dgrad_in, rom_route_bwd, rom_bwd_wgrad (twice). Every buffer is a
 * caller-owned device buffer; the sorted arrays use the forward's offsets,
 * sorted_slot and slot_pos. R = T*k, Dm = d_model, De = d_inner.
 * ------------------------------------------------------------------------ */

/* rdo_sorted[p] = r_s * dO[s / k] (bf16), s = sorted_slot[p]; dout [T][N]
 * bf16. Requires N % 8 == 0. */
int rom_bwd_gather(const void* dout, int64_t T, int k, int N, const int32_t* sorted_slot,
                   const float* topk_w, void* rdo_sorted, void* stream);

/*
 * Out dgrad: g'_s = rdo_sorted_s W_out,e^T (= r_s g_s) for the rows of each
 * expert. w_out [E][Dm][De] (forward layout); h_sorted [R][De] bf16 (the
 * forward's Y(.)G rows). Outputs: g_slots float32 [R][De] in slot order, and
 * dr_part float32 [R][De/256], the partial dots <h_s, g'_s> of each
 * 256-column tile. Requires Dm % 64 == 0 and De % 256 == 0.
 */
int rom_bwd_dgrad_out(const void* rdo_sorted, int64_t R, int Dm, const void* w_out, int De, int E,
                      int k, const int32_t* offsets, const int32_t* sorted_slot,
                      const void* h_sorted, float* g_slots, float* dr_part, void* stream);

/*
 * Gate backward. uz: float32 [2][R][De], the u and z of every slot in slot
 * order (the forward's rom_expert_proj(ROM_PROJ_CONV_GATE) output for k > 1);
 * g_slots from rom_bwd_dgrad_out. Writes dhz_sorted bf16 [R][2*De]: row
 * slot_pos[s] = [dH_t | dZ_t] of the slot's token t. Requires De % 4 == 0.
 */
int rom_bwd_gate(const float* uz, const float* g_slots, int64_t T, int k, int De,
                 const int32_t* slot_pos, void* dhz_sorted, void* stream);

/*
 * In/Gate dgrad: dx_slots_s = dhz_sorted_s [W_in,e ; W_g,e]^T (K = 2*De);
 * w_in, w_g [E][De][Dm] (forward layout). Output float32 [R][Dm], slot order.
 * Requires De % 64 == 0 and Dm % 256 == 0.
 */
int rom_bwd_dgrad_in(const void* dhz_sorted, int64_t R, int De, const void* w_in,
                     const void* w_g, int Dm, int E, int k, const int32_t* offsets,
                     const int32_t* sorted_slot, float* dx_slots, void* stream);

/*
 * Router backward and dX: dr_{t,j} = (sum of dr_part[s][0 .. n_parts)) / r_s,
 * s = sum_j r_{t,j} dr_{t,j};
 *   renorm = 1 (r = softmax over the selected logits):
 *     dlogit = r_j (dr_j - s) on S_t, 0 elsewhere; probs unused (may be NULL);
 *   renorm = 0 (r = p, the formula of Knowl 1): dlogit_m = p_m (dr_j - s) for
 *     m = S_j and -p_m s off S_t, which needs probs [T][E] float32, the
 *     softmax over all E experts (rom_route_probs).
 * dlogits [T][E] float32 (may be NULL);
 * dx [T][Dm] bf16 = sum_j dx_slots[t*k+j] + sum_m dlogit_{t,m} w_r[:, m].
 * Requires Dm % 4 == 0.
 */
int rom_route_bwd(int64_t T, int k, int E, int Dm, int renorm, const int32_t* topk_idx,
                  const float* topk_w, const float* probs, const float* dr_part, int n_parts,
                  const float* dx_slots, const float* w_r, float* dlogits, void* dx,
                  void* stream);

/*
 * probs [T][E] float32 = softmax(x W_r + bias) over all E experts (float32
 * logits accumulated in a fixed order): what rom_route_bwd needs for r = p.
 * x, w_r, bias as for rom_route.
 */
int rom_route_probs(const void* x, int dtype, int64_t T, int Dm, const float* w_r,
                    const float* bias, int E, float* probs, void* stream);

/*
 * Router weight gradients (the router is trained through the Out
 * projection's routing weights): dw_r [Dm][E] = sum_t x_t^T dlogit_t and
 * dbias [E] = sum_t dlogit_t (may be NULL), float32, summed over the tokens
 * in order. x [T][Dm] as given to rom_route (dtype); dlogits [T][E] float32
 * from rom_route_bwd. With T == 0 both are written as zeros.
 */
int rom_route_wgrad(const void* x, int dtype, int64_t T, int Dm, int E, const float* dlogits,
                    float* dw_r, float* dbias, void* stream);

/*
 * Weight gradients of every expert: out[e] = A_e^T B_e, A_e and B_e the rows
 * offsets[e] .. offsets[e+1]-1 of a_sorted [R][M] and b_sorted [R][N]
 * (bf16). float32 result rows m < m_split go to out0 [E][m_split][N], the
 * others to out1 [E][M - m_split][N] (out1 may be NULL when m_split == M).
 * Experts without rows get zeros. dW_out = wgrad(rdo_sorted, h_sorted);
 * [dW_in ; dW_g] = wgrad(dhz_sorted, x_sorted, m_split = De).
 * Requires M % 128 == 0, N % 256 == 0 and m_split % 128 == 0.
 */
int rom_bwd_wgrad(const void* a_sorted, int M, const void* b_sorted, int N, int64_t R, int E,
                  const int32_t* offsets, int m_split, float* out0, float* out1, void* stream);

/* ------------------------------------------------------------------------
 * The dense core between the projections (RoM page, Knowl 1: the short
 * convolution and the selective state-space computation applied to H_t
 * produce Y_t; Knowl 9: the 1D convolution and the x and dt projections are
 * shared by all experts), in the original Mamba form (zero-order hold for A,
 * Euler step for the input):
 *   X = SiLU(conv1d(H) + conv_b);  [dt | B | C] = X W_x;
 *   delta = softplus(dt W_dt + b_dt);  A = -exp(A_log);
 *   h_t = exp(delta_t A) (.) h_{t-1} + (delta_t x_t) B_t,  Y_t = h_t C_t + D (.) x_t.
 * ------------------------------------------------------------------------ */

/* Bytes of workspace rom_ssm_core needs (0 for invalid sizes). Host function. */
size_t rom_ssm_core_workspace_size(int64_t T, int De, int seq_len, int R, int N, int Np);

/*
 * rom_ssm_core -- Y = core(H) for T = (T / seq_len) consecutive sequences of
 * seq_len tokens each (the convolution and the state restart at every
 * sequence).
 *
 *  h       [T][De] float32, token order (the Conv projection H)
 *  conv_w  [De][K] float32: tap K-1 multiplies the current step, tap K-1-j
 *          the step j back;  conv_b [De] float32;  K <= 8
 *  w_x     bf16 [Np][De]: row j < R + 2N is column j of W_x ([De][R + 2N] in
 *          the pages' x W notation: dt, then B, then C); rows R + 2N .. Np-1
 *          zero; Np % 128 == 0
 *  w_dt    bf16 [De][R]: W_dt ([R][De]) transposed; R % 8 == 0
 *  b_dt    [De], a_log [De][N] (N <= 16), d [De]: float32
 *  y       [T][De] float32 out; may be the same buffer as h
 *  ws      workspace of rom_ssm_core_workspace_size() bytes, 256-byte aligned
 * The two projections run on the bf16 tensor cores with X and dt split into
 * two bf16 parts each (hi + lo, so the products are accurate to ~2^-16);
 * the convolution, softplus and the scan run in float32. Requires
 * De % 128 == 0.
 */
int rom_ssm_core(const float* h, int64_t T, int De, int seq_len, const float* conv_w,
                 const float* conv_b, int K, const void* w_x, int R, int N, int Np,
                 const void* w_dt, const float* b_dt, const float* a_log, const float* d,
                 float* y, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace rom_ssm_core_routed needs (0 for invalid sizes). */
size_t rom_ssm_core_routed_workspace_size(int64_t T, int De, int seq_len, int R, int N, int Np,
                                          int E, int k);

/*
 * rom_ssm_core_routed -- rom_ssm_core with the x and dt projections
 * expertized, routed by the block's own selection (RoM page, Knowl 3: "RoM
 * (Conv, Gate, dt, x, Out)"; Knowl 9: the dt and x ablation). w_x holds E
 * matrices [E][Np][De] and w_dt [E][De][R]; offsets, sorted_slot (from
 * rom_dispatch of the block, k slots per token) select each token's experts,
 * and its [dt | B | C] and dt projection are the sums over its k selected
 * experts, unweighted (as H and G). Other arguments as rom_ssm_core.
 */
int rom_ssm_core_routed(const float* h, int64_t T, int De, int seq_len, const float* conv_w,
                        const float* conv_b, int K, const void* w_x, int R, int N, int Np,
                        const void* w_dt, const float* b_dt, const float* a_log, const float* d,
                        int E, int k, const int32_t* offsets, const int32_t* sorted_slot,
                        float* y, void* ws, size_t ws_bytes, void* stream);

/*
 * rom_route_dispatch_noalloc -- rom_route() followed by rom_dispatch(), for
 * callers that cannot allocate device memory. The paper has no counterpart:
 * this is a deployment variant of the two calls above.
 *
 * Who needs it: code that may not call cudaMalloc or any allocator (for
 * example a plugin that only receives the host framework's buffers, or a
 * process whose memory is fully reserved by its own pool) cannot provide the
 * workspace that rom_route() and rom_dispatch() exchange. This entry point
 * keeps that scratch (the router's per-chunk expert histograms) in a fixed
 * array of ROM_NOALLOC_SCRATCH_WORDS int32 in the library's own device
 * memory, which every GPU that loads the library holds until the process
 * exits. It allocates nothing and calls no allocating routine; the caller
 * still passes every input and output.
 *
 * Arguments, layouts and outputs are those of rom_route() (x, dtype, T, Dm,
 * w_r, bias, E, k, renorm, topk_idx, topk_w, counts) and rom_dispatch()
 * (offsets, sorted_slot, slot_pos, x_sorted), without the workspace.
 *
 * Limits and errors: ceil(T / 128) * E must not exceed
 * ROM_NOALLOC_SCRATCH_WORDS (e.g. T <= 1,048,576 tokens at E = 8), else the
 * call returns ROM_ERR_WORKSPACE and enqueues nothing. Other argument errors
 * are those of rom_route() and rom_dispatch().
 *
 * Sharing: every call on a device uses the same array. Calls that can
 * overlap on the GPU (unordered streams) race on it and must not be issued;
 * calls on one stream are safe. The array keeps the last call's contents,
 * which is harmless: the router rewrites every entry the dispatch reads, and
 * if the router gives up on a bounded wait the dispatch's own checks catch
 * stale entries (ROM_ERR_ROUTING). Device-side errors go to the same status
 * word as for rom_route() and rom_dispatch() (rom_get_status).
 *
 * Set-up: the first call on a device looks up the array's device address
 * (with that device current) and caches it; make that first call before
 * any stream capture on the device.
 */
#define ROM_NOALLOC_SCRATCH_WORDS 65536
int rom_route_dispatch_noalloc(const void* x, int dtype, int64_t T, int Dm, const float* w_r,
                               const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                               float* topk_w, int32_t* counts, int32_t* offsets,
                               int32_t* sorted_slot, int32_t* slot_pos, void* x_sorted,
                               void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ROM_H_ */
