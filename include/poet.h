/*
 * poet.h -- C ABI of libpoet, the B200 (sm_100a) hot path of the POET
 * reparameterized linear layer   y = R . W0 . P . x
 *
 * Sources (web pages on POET / POET-X; cited by page title and section):
 *   [P1] "Reparameterized LLM Training via Orthogonal Equivalence
 *        Transformation" (atlas.scime.ai summary of arXiv 2506.08001):
 *        Approach, Key results, Measured effects table, Limitations.
 *   [P2] mlsanity page for arXiv 2506.08001: Abstract.
 *   [P3] "POET-X: Memory-efficient LLM Training by Scaling Orthogonal
 *        Transformation" (pith.science review): Core claim, What carries the
 *        argument.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument named "device" is CUDA device memory on the
 *    current device; the caller owns all memory.  The library never
 *    allocates device memory: scratch comes from the caller's workspace.
 *  - Every call is asynchronous and ordered on the given stream (NULL = the
 *    legacy default stream).  Inputs must stay valid until the work is done.
 *  - Row-major everywhere.  W0 is m x n (out x in).  Activations are
 *    token-major: x is T x n, y is T x m (one row per token), so the per-token
 *    y_t = R W0 P x_t of [P1] Approach is  Y = X P^T W0^T R^T.
 *  - Element type: POET_F32 (float) or POET_BF16 (bfloat16, round to nearest
 *    even) for W0, activations and materialized primitives.  Skew parameters
 *    theta and their gradients are always float32.  Accumulation is float32.
 *  - Status: arguments are validated on the host before anything is
 *    launched; a bad argument returns POET_EINVAL and launches nothing.  A
 *    failed CUDA launch returns POET_ECUDA.  Device-side errors (a bounded
 *    wait that ran out, a perm entry out of range) are recorded in a device
 *    status word that poet_sync_status() reads; kernels never dereference an
 *    index they found out of range.  poet_last_error() describes the last
 *    failure of the calling thread.
 *  - The library caches per-device addresses of its own device variables
 *    (the status word, the allocation-free entry point's scratch).  Do not
 *    use it across a cudaDeviceReset of a device it has run on.
 *
 * One side (R: dim = m, P: dim = n) -- readings of [P1] Key results
 * ("POET-FS (b=1/2)", "POET-BS (b=256)"); the pages fix no layout:
 *  - perm is a permutation of 0..dim-1.
 *  - POET_BS: floor(dim/b) primitives of size b; primitive j acts on the
 *    natural indices perm[j*b .. j*b+b-1]; the dim mod b leftover indices are
 *    left unchanged (identity).
 *  - POET_FS: one primitive of size s = floor(dim/2) acting on perm[0..s-1].
 *  - As a matrix the side is  Pi^T diag(B_0, ..., B_{q-1}, I) Pi  with
 *    (Pi v)_i = v[perm[i]].
 *  - theta holds, for each primitive in order, size*(size-1)/2 floats: the
 *    strict upper triangle of U packed row by row; Q = U - U^T.
 *  - Each primitive is the truncated Cayley-Neumann map of order k >= 0
 *    ([P1] Approach, Limitations):  B = (I + Q)(I + Q + Q^2 + ... + Q^k).
 *
 * The permuted frame.  The library keeps a copy of W0 with rows ordered by
 * R.perm and columns by P.perm (W0f[i][j] = W0[R.perm[i]][P.perm[j]]), so
 * that every primitive acts on a contiguous range of frame indices and every
 * contraction on the hot path reads contiguous tiles.
 *
 * Two plans compute the same layer (the pages fix what is computed, not the
 * order of the products; both are exact rearrangements of y = R W0 P x):
 *  - token plan: the primitives act on the activations.  Activations are
 *    gathered into the frame once on entry, pass through the blocks of P,
 *    W0f and the blocks of R, and are scattered out once on exit.  Cost per
 *    token ~ 2mn + 2(sum of primitive sizes squared) flops plus four
 *    activation-sized permutation passes (forward and backward).
 *  - weight plan: the primitives act on W0.  The forward forms the
 *    effective weight E = R W0 P (weight-sized work) and runs one GEMM
 *    y = x E^T; the backward runs dx = dy E and D = dy^T x and takes the
 *    per-primitive gradients from D (weight-sized work again).  Cost per
 *    token ~ 3 x 2mn flops and no activation permutation.
 *  poet_layer.plan selects one; POET_PLAN_AUTO picks the cheaper for the
 *  token count (poet_plan_for tells which).
 */
#ifndef POET_H
#define POET_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define POET_API __attribute__((visibility("default")))
#else
#define POET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t (a CUDA runtime stream handle). */
typedef struct CUstream_st *poet_stream;

typedef enum {
  POET_OK = 0,
  POET_EINVAL = 1,     /* bad argument; nothing was launched */
  POET_ECUDA = 2,      /* a CUDA call or launch failed */
  POET_ETIMEOUT = 3,   /* a device-side bounded wait ran out (see poet_sync_status) */
  POET_ENOMEM_WS = 4,  /* the workspace passed is smaller than required */
  POET_EBOUNDS = 5     /* a kernel met an index out of range in a caller-written perm
                          (outside [0, dim)) and skipped it (see poet_sync_status) */
} poet_status;

typedef enum { POET_F32 = 0, POET_BF16 = 1 } poet_dtype;
typedef enum { POET_BS = 0, POET_FS = 1 } poet_mode;
typedef enum { POET_PLAN_AUTO = 0, POET_PLAN_TOKEN = 1, POET_PLAN_WEIGHT = 2 } poet_plan;

typedef struct {
  int32_t dim;     /* m for R, n for P; 1 <= dim <= 16384 */
  int32_t mode;    /* POET_BS or POET_FS */
  int32_t b;       /* POET_BS: block size, 1 <= b; ignored for POET_FS */
  int32_t k;       /* Neumann order, 0 <= k <= 16 */
  int32_t *perm;   /* device int32[dim]; written by poet_prepare/poet_resample */
  float *theta;    /* device float[nprim * size*(size-1)/2]; zeroed by poet_merge */
  void *state;     /* device, poet_side_state_bytes() bytes, written by
                      poet_cayley_neumann.  It starts with the materialized
                      primitives, element type dtype, [nprim][ld][ld] with
                      ld = size rounded up to a multiple of 8 (padding zero);
                      the rest (Neumann terms for the backward) is opaque. */
} poet_side;

typedef struct {
  int64_t m;       /* output features (rows of W0) */
  int64_t n;       /* input features (columns of W0) */
  int32_t dtype;   /* poet_dtype of W0, W0f, activations, primitives */
  int32_t layer_id;/* >= 0; keys the permutation draw */
  int32_t epoch;   /* >= 0; advanced by poet_resample */
  int32_t plan;    /* poet_plan: POET_PLAN_AUTO (0), _TOKEN or _WEIGHT */
  uint64_t seed;   /* keys the permutation draw */
  void *W0;        /* device m x n, row-major, natural order (the fixed weight) */
  void *W0f;       /* device, poet_frame_bytes() bytes: W0 in the permuted frame */
  poet_side R;     /* left side, dim = m */
  poet_side P;     /* right side, dim = n */
} poet_layer;

/* ---------------------------------------------------------------- sizes */

/* Bytes of side->state for element type dtype (0 if the side is invalid). */
POET_API size_t poet_side_state_bytes(const poet_side *side, int32_t dtype);

/* Bytes of L->W0f (0 if the layer is invalid). */
POET_API size_t poet_frame_bytes(const poet_layer *L);

/* The plan poet_forward / poet_backward run for this layer at T tokens
 * (POET_PLAN_TOKEN or POET_PLAN_WEIGHT; -1 if the layer is invalid).  With
 * POET_PLAN_AUTO the choice depends only on the shapes, the sides' geometry
 * and T: the plan with the smaller estimated device time, counting flops at
 * the tensor-core rate and activation or weight passes at the HBM rate. */
POET_API int32_t poet_plan_for(const poet_layer *L, int64_t T);

/* Bytes of the buffer poet_forward saves for poet_backward at T tokens
 * (token plan: the frame copies of x and of W0 P x; weight plan: the
 * effective weight and two weight-sized factors, plus a 16-byte aligned copy
 * of x when n is not a multiple of 8). */
POET_API size_t poet_saved_bytes(const poet_layer *L, int64_t T);

/* Bytes of workspace that poet_forward, poet_backward, poet_merge and
 * poet_cayley_neumann(_grad) on this layer's sides need at T tokens
 * (one size covers all of them; T may be 0 for merge / Cayley-Neumann). */
POET_API size_t poet_workspace_bytes(const poet_layer *L, int64_t T);

/* Bytes of workspace poet_cayley_neumann_grad needs for one side alone. */
POET_API size_t poet_side_workspace_bytes(const poet_side *side, int32_t dtype);

/* ---------------------------------------------------------------- a1 / a8 */

/* a1: materialize every primitive of one side from side->theta into
 * side->state ([P1] Approach: truncated Neumann-series Cayley
 * parameterization).  ws: device scratch of ws_bytes bytes (may be NULL when
 * poet_workspace_bytes(.., 0) is 0).  Overwrites side->state only. */
POET_API poet_status poet_cayley_neumann(const poet_side *side, int32_t dtype,
                                void *ws, size_t ws_bytes, poet_stream stream);

/* a8: gradient of <G, B(Q)> with respect to the packed parameters of every
 * primitive of one side (chain rule through the map of poet_cayley_neumann).
 * G: device float[nprim][size][size] (dL/dB of each primitive, row-major).
 * dtheta: device float[nprim * size*(size-1)/2], overwritten.
 * Requires side->state from poet_cayley_neumann of the same theta. */
POET_API poet_status poet_cayley_neumann_grad(const poet_side *side, int32_t dtype,
                                     const float *G, float *dtheta,
                                     void *ws, size_t ws_bytes, poet_stream stream);

/* The same computation as poet_cayley_neumann_grad, for callers that cannot
 * allocate device memory (a host framework that owns all device memory and
 * hands out none, a plug-in whose host forbids allocations, a caller that
 * cannot keep a workspace between calls).  The POET pages have no counterpart
 * of this call; it exists for those callers only.  Inputs and outputs as in
 * poet_cayley_neumann_grad; the scratch is a 32 MiB array built into the
 * library, which every GPU that loads the library holds until the process
 * exits.  A side whose workspace (poet_side_workspace_bytes) exceeds 32 MiB is
 * rejected with POET_EINVAL.  No allocation happens in this call.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and may load the library's code on that device:
 *    make that first call before any stream capture begins.
 *  - All calls on a device share the one array, which keeps the last call's
 *    contents (nothing in it needs to start at zero).  Calls whose work
 *    overlaps on the GPU race on it: order them on one stream. */
POET_API poet_status poet_cayley_neumann_grad_noalloc(const poet_side *side, int32_t dtype,
                                                      const float *G, float *dtheta,
                                                      poet_stream stream);

/* ---------------------------------------------------------------- a2..a4 */

/* Forward: y = R W0 P x for T tokens ([P1] Approach; [P2] Abstract).
 * x: device T x n (dtype), y: device T x m (dtype), both row-major and
 * contiguous.  saved: device, poet_saved_bytes(L, T) bytes, written here and
 * read by poet_backward.  Requires both sides' state from
 * poet_cayley_neumann and W0f from poet_prepare/poet_resample/poet_merge.
 * T = 0 is allowed (nothing is launched). */
POET_API poet_status poet_forward(const poet_layer *L, const void *x, int64_t T, void *y,
                         void *saved, void *ws, size_t ws_bytes, poet_stream stream);

/* ---------------------------------------------------------------- a5..a8 */

/* Backward for upstream gradient dy (device T x m, dtype): writes
 * dx = P^T W0^T R^T dy (device T x n, dtype) and the gradients of the loss
 * with respect to both sides' packed parameters (device float, overwritten,
 * same layout as theta).  W0 is fixed ([P1] Approach), so there is no dW0.
 * x: the forward's input (device T x n), read by the weight plan (D = dy^T x)
 * and ignored by the token plan (may be NULL there).  saved: the buffer
 * poet_forward filled for the same x and T.  The layer's plan, state and
 * W0f must be those of that forward. */
POET_API poet_status poet_backward(const poet_layer *L, const void *x, const void *saved,
                          const void *dy, int64_t T, void *dx, float *dtheta_R,
                          float *dtheta_P, void *ws, size_t ws_bytes, poet_stream stream);

/* ---------------------------------------------------------------- many layers at once
 *
 * Training steps run a1 for every primitive of every layer and a8 for every
 * layer; the calls below let many sides share each tensor-core launch (the
 * primitives of one side are often too few to fill the GPU).  The per-side
 * gradient G of a primitive is laid out like the materialized primitives at
 * the start of the side state: float [nprim][ld][ld], ld = size rounded up to
 * a multiple of 8 (padding ignored). */

/* Bytes of the per-primitive gradient G of one side (float [nprim][ld][ld]). */
POET_API size_t poet_block_grad_bytes(const poet_side *side);

/* a1 for count sides (same result as poet_cayley_neumann on each). */
POET_API poet_status poet_cayley_neumann_many(const poet_side *sides, int32_t count, int32_t dtype,
                                              poet_stream stream);

/* a5..a7 of poet_backward: writes dx and the per-primitive gradients
 * G_R = dL/dR_j and G_P = dL/dP_j (device, poet_block_grad_bytes each,
 * 16-byte aligned, overwritten) instead of dtheta. */
POET_API poet_status poet_backward_blocks(const poet_layer *L, const void *x, const void *saved,
                                          const void *dy, int64_t T, void *dx, float *G_R,
                                          float *G_P, void *ws, size_t ws_bytes, poet_stream stream);

/* ---- many layers' forward and backward
 *
 * The forward and a5..a7 of count independent layers (for example every
 * linear of a layer set whose inputs are all at hand, or q, k and v of one
 * block, which share their input).  Same results as poet_forward and
 * poet_backward_blocks on each layer (the per-primitive gradients, whose
 * products are summed over split ranges, agree to rounding); the difference
 * is the launches: under the weight plan the weight-sized products of every
 * layer share grouped tensor-core launches, their permutations share one
 * launch, and the T-sized GEMMs of all layers run as one grouped launch.
 * Token-plan layers in the list run one after another.
 *  - layers: count complete layers of one element type (state from
 *    poet_cayley_neumann, W0f from poet_prepare / poet_resample / poet_merge),
 *    each with its plan as poet_plan_for(&layers[i], T) says.
 *  - x[i] (T x n_i), y[i] (T x m_i), dy[i] (T x m_i), dx[i] (T x n_i): device,
 *    row-major with row strides ldx[i], ldy[i], lddy[i], lddx[i] elements
 *    (>= the width; a NULL stride list means contiguous rows).  Rows whose
 *    start is 16-byte aligned (stride x element size a multiple of 16, base
 *    16-byte aligned) are read and written in place; other x and dy rows are
 *    first copied into 16-byte aligned rows.
 *  - saved[i]: device, poet_saved_bytes(&layers[i], T) bytes, 256-byte aligned.
 *  - G_R[i], G_P[i]: device, poet_block_grad_bytes each, 16-byte aligned,
 *    overwritten.
 *  - ws: device, poet_many_workspace_bytes(layers, count, T, lddy) bytes,
 *    256-byte aligned; one size serves both calls. */
POET_API size_t poet_many_workspace_bytes(const poet_layer *layers, int32_t count, int64_t T, const int64_t *lddy);

POET_API poet_status poet_forward_many(const poet_layer *layers, int32_t count, const void *const *x,
                                       const int64_t *ldx, int64_t T, void *const *y, const int64_t *ldy,
                                       void *const *saved, void *ws, size_t ws_bytes, poet_stream stream);

POET_API poet_status poet_backward_blocks_many(const poet_layer *layers, int32_t count, const void *const *x,
                                               const int64_t *ldx, const void *const *saved,
                                               const void *const *dy, const int64_t *lddy, int64_t T,
                                               void *const *dx, const int64_t *lddx, float *const *G_R,
                                               float *const *G_P, void *ws, size_t ws_bytes, poet_stream stream);

/* Workspace bytes of poet_cayley_neumann_grad_many for these sides. */
POET_API size_t poet_cayley_neumann_grad_many_workspace_bytes(const poet_side *sides, int32_t count,
                                                              int32_t dtype);

/* a8 for count sides: dtheta[i] (device float, theta layout, overwritten) from
 * G[i] (device, layout above).  The same gradient as poet_cayley_neumann_grad;
 * its matrix products are grouped differently (every product of one Neumann
 * order, across all sides, in one launch), so the two agree to rounding of
 * the operand type, not bitwise. */
POET_API poet_status poet_cayley_neumann_grad_many(const poet_side *sides, const float *const *G,
                                                   float *const *dtheta, int32_t count, int32_t dtype,
                                                   void *ws, size_t ws_bytes, poet_stream stream);

/* ---------------------------------------------------------------- a9 */

/* Merge-then-reinitialize ([P1] Approach: "merged periodically"; Measured
 * effects: merge-then-reinitialize frequency):  W0 <- R W0 P using the
 * primitives currently materialized in the side states (the same ones the
 * forward used), then theta <- 0 for both sides and both states are
 * re-materialized, so R = P = I exactly for any k.  Updates W0 and W0f;
 * the permutations are unchanged (call poet_resample next for new ones). */
POET_API poet_status poet_merge(poet_layer *L, void *ws, size_t ws_bytes, poet_stream stream);

/* ---------------------------------------------------------------- a10 */

/* Draw both sides' permutations for L->epoch and rebuild W0f from W0.
 * Use once on a fresh layer; does not change L->epoch. */
POET_API poet_status poet_prepare(poet_layer *L, poet_stream stream);

/* Reinitialize's new sampling ([P1] Approach, "sampled sub-block
 * primitives"): L->epoch += 1 (host struct), then as poet_prepare. */
POET_API poet_status poet_resample(poet_layer *L, poet_stream stream);

/* The permutation draw on its own (a reading: the pages fix no generator).
 * key_i = i-th output of SplitMix64 (Steele, Lea, Flood 2014) seeded with
 *   h = sm(seed ^ sm((layer_id << 32) ^ (epoch << 1) ^ side)),
 * where sm(z) is one SplitMix64 step from state z; perm lists 0..dim-1
 * ordered by (key_i, i) ascending.  side: 0 = R, 1 = P.
 * perm: device int32[dim], overwritten.  1 <= dim <= 16384. */
POET_API poet_status poet_draw_perm(uint64_t seed, int32_t layer_id, int32_t side, int32_t epoch,
                           int32_t dim, int32_t *perm, poet_stream stream);

/* ---------------------------------------------------------------- optimizer step (adjacent) */

/* One AdamW step on n packed parameters in place: the pages name no
 * optimizer for the primitives' parameters, so this is the textbook update
 * (Loshchilov & Hutter, "Decoupled Weight Decay Regularization"):
 *   m <- beta1 m + (1 - beta1) g,   v <- beta2 v + (1 - beta2) g^2,
 *   theta <- theta - lr * ( (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps)
 *                           + weight_decay * theta ).
 * theta, m, v: device float[n], updated; grad: device float[n] (e.g. the
 * dtheta of poet_backward).  step >= 1 counts the updates so far including
 * this one.  After poet_merge resets theta, the caller resets m, v and step.
 * Host validation: n >= 0; pointers non-NULL and 4-byte aligned when n > 0;
 * 0 <= beta1, beta2 < 1; eps > 0; lr, weight_decay >= 0 and finite. */
POET_API poet_status poet_adamw_step(float *theta, const float *grad, float *m, float *v, int64_t n,
                                     float lr, float beta1, float beta2, float eps, float weight_decay,
                                     int32_t step, poet_stream stream);

/* AdamW hyperparameters of one step (see poet_adamw_step). */
typedef struct {
  float lr, beta1, beta2, eps, weight_decay;
  int32_t step;    /* >= 1: updates so far including this one */
} poet_adamw_hparams;

/* a8 for count sides, with the AdamW step of poet_adamw_step applied to each
 * side's theta (in place, side->theta) in the same kernel that packs the
 * gradient: per parameter the gradient is formed, the moments m[i], v[i]
 * (device float, theta layout) are updated and theta moves, with no pass of
 * the gradient through memory.  dtheta[i] may be NULL (not written) or a
 * buffer that also receives the gradient.  Same gradient as
 * poet_cayley_neumann_grad_many, same update as poet_adamw_step on it.
 * Workspace as poet_cayley_neumann_grad_many.  For data-parallel training,
 * where the gradient is summed over ranks before the update, use
 * poet_cayley_neumann_grad_many, the all-reduce, then poet_adamw_step. */
POET_API poet_status poet_cayley_neumann_grad_many_adamw(const poet_side *sides, const float *const *G,
                                                         float *const *m, float *const *v,
                                                         float *const *dtheta, int32_t count, int32_t dtype,
                                                         const poet_adamw_hparams *h, void *ws, size_t ws_bytes,
                                                         poet_stream stream);

/* poet_merge, then the AdamW moments of both sides reset to zero (the
 * parameters restart at theta = 0; the caller restarts its step count).
 * m_R, v_R: device float[R's theta length]; m_P, v_P: the same for P (any of
 * them may be NULL when that side has no parameters). */
POET_API poet_status poet_merge_reset_moments(poet_layer *L, float *m_R, float *v_R, float *m_P, float *v_P,
                                              void *ws, size_t ws_bytes, poet_stream stream);

/* The workspace size query under the name of the pages' boundary sketch: the
 * same value as poet_workspace_bytes. */
POET_API size_t poet_workspace_size(const poet_layer *L, int64_t T);

/* ---------------------------------------------------------------- one LLaMA block (adjacent)
 *
 * The pages train LLaMA models whose linears are POET layers ([P1]
 * Experimental setup); these calls run one such block on synthetic tokens,
 * forward and backward, with the published LLaMA design around the seven
 * linears: pre-normalization by RMSNorm (gains 1, not trained; eps inside the
 * square root), rotary position embedding on interleaved pairs (2i, 2i+1) of
 * each head (angle pos * rope_base^(-2i/head_dim), positions counted within
 * each sequence of seq_len tokens), causal multi-head attention with scores
 * scaled by 1/sqrt(head_dim), SwiGLU (down(silu(gate(x)) * up(x))) and
 * residual connections.  The readings are the library's; the pages restate
 * none of the block.  Attention materializes the scores (float) and the
 * probabilities (bf16, kept for the backward) of every head: T/seq_len x heads
 * x seq_len^2 each.  bf16 only. */
typedef struct {
  int32_t seq_len;    /* tokens per sequence (a multiple of 8); T must be a multiple of it */
  int32_t heads;      /* attention heads */
  int32_t head_dim;   /* width of one head (a multiple of 8); heads * head_dim = hidden */
  float rope_base;    /* rotary base (LLaMA: 10000) */
  float norm_eps;     /* RMSNorm epsilon (LLaMA: 1e-6) */
  poet_layer lin[7];  /* q, k, v, o (hidden x hidden), gate, up (ffn x hidden), down (hidden x ffn),
                         each prepared (poet_prepare) with its sides materialized */
} poet_llama_block;

/* Bytes of the buffer the block's forward saves for its backward at T tokens (0 if invalid). */
POET_API size_t poet_llama_block_saved_bytes(const poet_llama_block *blk, int64_t T);

/* Bytes of workspace the block's forward and backward need at T tokens (0 if invalid). */
POET_API size_t poet_llama_block_workspace_bytes(const poet_llama_block *blk, int64_t T);

/* out = the block applied to h (device T x hidden bf16, contiguous rows, 16-byte
 * aligned); saved: device, poet_llama_block_saved_bytes, 256-byte aligned;
 * ws: device, poet_llama_block_workspace_bytes, 256-byte aligned. */
POET_API poet_status poet_llama_block_forward(const poet_llama_block *blk, const void *h, int64_t T, void *out,
                                              void *saved, void *ws, size_t ws_bytes, poet_stream stream);

/* For upstream gradient dout (device T x hidden bf16): dh (device T x hidden
 * bf16) and every linear's per-primitive gradients G[2i] = G_R, G[2i+1] = G_P
 * of lin[i] (device, poet_block_grad_bytes each, 16-byte aligned, overwritten);
 * the skew-parameter gradients follow with poet_cayley_neumann_grad_many on
 * the fourteen sides.  saved: the buffer the forward filled for the same h. */
POET_API poet_status poet_llama_block_backward(const poet_llama_block *blk, const void *saved, const void *dout,
                                               int64_t T, void *dh, float *const *G, void *ws, size_t ws_bytes,
                                               poet_stream stream);

/* ---------------------------------------------------------------- utilities */

/* Batched dense product on the library's GEMM engine, exported so that the
 * engine can be tested on its own (it is the same code the layer uses):
 *   C[b][i][j] = alpha * sum_l A(b,i,l) * B(b,j,l) (+ beta * C[b][i][j])
 * A(b,i,l) = A[b*sAb + i*sAm + l*sAk], B(b,j,l) = B[b*sBb + j*sBn + l*sBk]
 * (element strides), C row-major with row stride ldc and batch stride sCb.
 * dtype: element type of A, B and C.  Returns POET_EINVAL on a bad shape. */
POET_API poet_status poet_gemm(int32_t dtype, int32_t M, int32_t N, int32_t K, int32_t batch,
                      const void *A, int64_t sAm, int64_t sAk, int64_t sAb,
                      const void *B, int64_t sBn, int64_t sBk, int64_t sBb,
                      void *C, int64_t ldc, int64_t sCb, float alpha, float beta,
                      poet_stream stream);

/* Which GEMM engine poet_gemm and the layer use for dtype:
 * 1 = tcgen05 tensor cores (bf16 with a supported operand layout),
 * 0 = CUDA-core FMA (float32, and layouts tcgen05 cannot read). */
POET_API int32_t poet_gemm_engine(int32_t dtype);

/* ---------------------------------------------------------------- accounting */

/* One kind of work with its recorded launches, CUDA-event time and
 * algorithmic flops / bytes (the operation's own operand sizes, not counters).
 * flop_tc sums the flops of the launches whose flop / byte ratio is at or
 * above the ridge set by poet_trace_set_ridge, bytes_hbm the bytes of the
 * others, so that flop_tc / (tensor peak) + bytes_hbm / (copy peak) is the
 * kind's roofline time with every launch held to its own bound. */
typedef struct {
  char kind[32];
  int64_t launches;
  double ms;
  double flop;
  double bytes;
  double flop_tc;
  double bytes_hbm;
} poet_trace_row;

/* Kernels this library has launched since it was loaded (all devices). */
POET_API int64_t poet_launch_count(void);

/* Start (on != 0) or stop recording a CUDA event pair on the launch stream
 * around each unit of work, tagged by kind.  Recording adds host calls
 * between launches but no device work. */
POET_API poet_status poet_trace_enable(int32_t on);

/* The flop / byte ratio that splits launches into flop_tc and bytes_hbm
 * (the tensor peak over the copy peak; 216 until set).  EINVAL unless > 0. */
POET_API poet_status poet_trace_set_ridge(double flop_per_byte);

/* Wait for the recorded events, aggregate them by kind into rows (at most
 * max_rows, sorted by kind), forget them, and return the rows written. */
POET_API int32_t poet_trace_read(poet_trace_row *rows, int32_t max_rows);

/* Failure-detection self test.  Launches one CTA that waits, through the
 * library's bounded mbarrier wait, on a barrier that nothing arrives on, with
 * the limit set to timeout_us (1 .. 1e6).  The wait runs out, records a
 * timeout in the device status word and the kernel returns normally, so the
 * next poet_sync_status returns POET_ETIMEOUT and the context stays usable. */
POET_API poet_status poet_selftest_bounded_wait(uint32_t timeout_us, poet_stream stream);

/* Synchronize the stream, then read and clear the device status word.
 * Returns POET_ETIMEOUT if a kernel gave up a bounded wait since the last
 * call, else POET_EBOUNDS if a kernel skipped an index out of range (a
 * permutation entry outside [0, dim); the results of that call are not
 * meaningful), POET_ECUDA on a CUDA error, POET_OK otherwise. */
POET_API poet_status poet_sync_status(poet_stream stream);

/* Text of the last failure on the calling thread ("" if none). */
POET_API const char *poet_last_error(void);

/* Library version string. */
POET_API const char *poet_version(void);

#ifdef __cplusplus
}
#endif

#endif /* POET_H */
