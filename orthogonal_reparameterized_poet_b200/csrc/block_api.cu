// C ABI of one LLaMA block around seven POET linears (poet_llama_block_*):
// the order of the steps, the saved-buffer and workspace layouts, and the
// attention products on the GEMM engine.  The element-wise and row kernels
// are in block.cu; the linears run through poet_forward_many /
// poet_backward_blocks_many (q, k, v in one call; gate, up in one call).
//
//   forward   n1 = norm(h); q, k, v = POET(n1); qr, kr = rope(q), rope(k);
//             P = causal softmax(qr kr^T / sqrt(hd)); att = P v;
//             h1 = h + POET_o(att); n2 = norm(h1); g, u = POET(n2);
//             mlp = silu(g) u; out = h1 + POET_down(mlp)
//   backward  the chain rule through the same steps in reverse; every
//             linear's per-primitive gradients G_R, G_P are written (a8, the
//             skew-parameter gradients, is the caller's grouped call)
#include <cmath>
#include <vector>

#include "poet_internal.cuh"

namespace poet {

poet_status block_rmsnorm(const bf16 *x, int64_t ldx, int64_t rows, int d, float eps, bf16 *y, int64_t ldy, float *r,
                          cudaStream_t st);
poet_status block_rmsnorm_bwd(const bf16 *g0, const bf16 *g1, const bf16 *g2, int64_t ldg, const bf16 *y, int64_t ldy,
                              const float *r, const bf16 *resid, int64_t ldr, int64_t rows, int d, bf16 *dx,
                              int64_t lddx, cudaStream_t st);
poet_status block_rope(bf16 *x, int64_t ldx, int64_t rows, int d, int head_dim, int seq_len, float base, bool inverse,
                       cudaStream_t st);
poet_status block_softmax(const float *s, int64_t rows, int S, bf16 *p, cudaStream_t st);
poet_status block_softmax_bwd(const bf16 *p, const float *dp, int64_t rows, int S, float scale, bf16 *ds,
                              cudaStream_t st);
poet_status block_swiglu(const bf16 *g, const bf16 *u, int64_t ld, int64_t rows, int d, bf16 *m, int64_t ldm,
                         cudaStream_t st);
poet_status block_swiglu_bwd(const bf16 *dm, int64_t lddm, const bf16 *g, const bf16 *u, int64_t ld, int64_t rows,
                             int d, bf16 *dg, bf16 *du, int64_t ldo, cudaStream_t st);
poet_status block_add(const bf16 *a, int64_t lda, const bf16 *b, int64_t ldb, int64_t rows, int d, bf16 *out,
                      int64_t ldo, cudaStream_t st);

namespace {

enum { LQ = 0, LK, LV, LO, LGATE, LUP, LDOWN, NLIN };

struct BlockGeom {
  int64_t T = 0, hidden = 0, ffn = 0, ldh = 0, ldf = 0;
  int S = 0, H = 0, hd = 0, B = 0;
};

// Validation of the block's shape (pointers of the linears are checked by the
// grouped calls); fills g.
poet_status check_block(const poet_llama_block *blk, int64_t T, BlockGeom *g) {
  POET_REQUIRE(blk != nullptr, "llama block: NULL");
  const poet_layer *L = blk->lin;
  const int64_t hidden = L[LQ].m, ffn = L[LGATE].m;
  POET_REQUIRE(blk->seq_len >= 8 && blk->seq_len % 8 == 0, "llama block: seq_len %d must be a positive multiple of 8",
               blk->seq_len);
  POET_REQUIRE(blk->head_dim >= 8 && blk->head_dim % 8 == 0 && blk->heads >= 1 &&
                   int64_t(blk->heads) * blk->head_dim == hidden,
               "llama block: heads (%d) x head_dim (%d) must equal hidden (%lld), head_dim a multiple of 8",
               blk->heads, blk->head_dim, (long long)hidden);
  POET_REQUIRE(std::isfinite(blk->rope_base) && blk->rope_base > 1.f && std::isfinite(blk->norm_eps) &&
                   blk->norm_eps >= 0.f,
               "llama block: rope_base must be > 1 and norm_eps >= 0");
  POET_REQUIRE(T >= 0 && T % blk->seq_len == 0, "llama block: T=%lld is not a multiple of seq_len %d", (long long)T,
               blk->seq_len);
  for (int i = 0; i < NLIN; ++i) POET_REQUIRE(L[i].dtype == POET_BF16, "llama block: linear %d is not bf16", i);
  POET_REQUIRE(L[LQ].n == hidden && L[LK].m == hidden && L[LK].n == hidden && L[LV].m == hidden &&
                   L[LV].n == hidden && L[LO].m == hidden && L[LO].n == hidden && L[LGATE].n == hidden &&
                   L[LUP].m == ffn && L[LUP].n == hidden && L[LDOWN].m == hidden && L[LDOWN].n == ffn &&
                   hidden % 8 == 0,
               "llama block: linear shapes must be q, k, v, o: h x h; gate, up: f x h; down: h x f (h a multiple of 8)");
  g->T = T;
  g->hidden = hidden;
  g->ffn = ffn;
  g->ldh = round_up(hidden, 8);
  g->ldf = round_up(ffn, 8);
  g->S = blk->seq_len;
  g->H = blk->heads;
  g->hd = blk->head_dim;
  g->B = int(T / blk->seq_len);
  return POET_OK;
}

struct SavedLayout {
  size_t n1, r1, sv[NLIN], qr, kr, v, P, att, n2, r2, g, u, mlp, bytes;
};
SavedLayout saved_layout(const poet_llama_block *blk, const BlockGeom &g) {
  SavedLayout s{};
  const size_t th = align256(size_t(g.T) * g.ldh * 2), tf = align256(size_t(g.T) * g.ldf * 2);
  const size_t tr = align256(size_t(g.T) * 4);
  size_t off = 0;
  auto take = [&](size_t b) { const size_t o = off; off += align256(b); return o; };
  s.n1 = take(th);
  s.r1 = take(tr);
  for (int i : {int(LQ), int(LK), int(LV)}) s.sv[i] = take(poet_saved_bytes(&blk->lin[i], g.T));
  s.qr = take(th);
  s.kr = take(th);
  s.v = take(th);
  s.P = take(size_t(g.B) * g.H * g.S * g.S * 2);
  s.att = take(th);
  s.sv[LO] = take(poet_saved_bytes(&blk->lin[LO], g.T));
  s.n2 = take(th);
  s.r2 = take(tr);
  for (int i : {int(LGATE), int(LUP)}) s.sv[i] = take(poet_saved_bytes(&blk->lin[i], g.T));
  s.g = take(tf);
  s.u = take(tf);
  s.mlp = take(tf);
  s.sv[LDOWN] = take(poet_saved_bytes(&blk->lin[LDOWN], g.T));
  s.bytes = off;
  return s;
}

struct WsLayoutB {
  size_t many, scores, dS, t1, t2, dmlp, dg, du, dn2g, dn2u, dh1, datt, dqr, dkr, dv, dn1q, dn1k, dn1v, bytes;
};
// The grouped calls' workspace first, then the block's own buffers (the
// forward uses scores, t1 = h1 and t2; the backward all but t1, t2).
WsLayoutB ws_layout_block(const poet_llama_block *blk, const BlockGeom &g) {
  WsLayoutB w{};
  const poet_layer *L = blk->lin;
  const int64_t ldh3[3] = {g.ldh, g.ldh, g.ldh}, ldf2[2] = {g.ldf, g.ldf};
  size_t many = poet_many_workspace_bytes(L + LQ, 3, g.T, ldh3);
  many = std::max(many, poet_many_workspace_bytes(L + LO, 1, g.T, ldh3));
  many = std::max(many, poet_many_workspace_bytes(L + LGATE, 2, g.T, ldf2));
  many = std::max(many, poet_many_workspace_bytes(L + LDOWN, 1, g.T, &g.hidden));
  const size_t th = align256(size_t(g.T) * g.ldh * 2), tf = align256(size_t(g.T) * g.ldf * 2);
  size_t off = 0;
  auto take = [&](size_t b) { const size_t o = off; off += align256(b); return o; };
  w.many = take(many);
  w.scores = take(size_t(g.B) * g.H * g.S * g.S * 4);
  w.dS = take(size_t(g.B) * g.H * g.S * g.S * 2);
  w.t1 = take(th);
  w.t2 = take(th);
  w.dmlp = take(tf);
  w.dg = take(tf);
  w.du = take(tf);
  w.dn2g = take(th);
  w.dn2u = take(th);
  w.dh1 = take(th);
  w.datt = take(th);
  w.dqr = take(th);
  w.dkr = take(th);
  w.dv = take(th);
  w.dn1q = take(th);
  w.dn1k = take(th);
  w.dn1v = take(th);
  w.bytes = off;
  return w;
}

// The attention products of every sequence: one grouped GEMM launch per
// product kind, each problem batched over the heads (batch stride head_dim
// columns of the token-major activations, S x S per head for the scores).
Gemm attn_gemm(const BlockGeom &g, const char *tag) {
  Gemm p;
  p.tag = tag;
  p.dtype = POET_BF16;
  p.batch = g.H;
  return p;
}

}  // namespace
}  // namespace poet

using namespace poet;

extern "C" {

size_t poet_llama_block_saved_bytes(const poet_llama_block *blk, int64_t T) {
  BlockGeom g;
  if (check_block(blk, T, &g) != POET_OK) return 0;
  return saved_layout(blk, g).bytes;
}

size_t poet_llama_block_workspace_bytes(const poet_llama_block *blk, int64_t T) {
  BlockGeom g;
  if (check_block(blk, T, &g) != POET_OK) return 0;
  return ws_layout_block(blk, g).bytes;
}

poet_status poet_llama_block_forward(const poet_llama_block *blk, const void *h, int64_t T, void *out, void *saved,
                                     void *ws, size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_llama_block_forward");
  clear_error();
  BlockGeom g;
  POET_TRY(check_block(blk, T, &g));
  if (T == 0) return POET_OK;
  POET_REQUIRE(h && out && (reinterpret_cast<uintptr_t>(h) & 15) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0,
               "poet_llama_block_forward: h/out NULL or not 16-byte aligned");
  POET_REQUIRE(saved && (reinterpret_cast<uintptr_t>(saved) & 255) == 0,
               "poet_llama_block_forward: saved NULL or not 256-byte aligned");
  const SavedLayout s = saved_layout(blk, g);
  const WsLayoutB w = ws_layout_block(blk, g);
  if (!ws || ws_bytes < w.bytes || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) {
    set_error("poet_llama_block_forward: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, w.bytes);
    return POET_ENOMEM_WS;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *sv = static_cast<char *>(saved);
  char *wb = static_cast<char *>(ws);
  const poet_layer *L = blk->lin;
  auto B16 = [](void *p) { return static_cast<bf16 *>(p); };
  bf16 *n1 = B16(sv + s.n1), *qr = B16(sv + s.qr), *kr = B16(sv + s.kr), *v = B16(sv + s.v);
  bf16 *att = B16(sv + s.att), *n2 = B16(sv + s.n2), *gg = B16(sv + s.g), *uu = B16(sv + s.u);
  bf16 *mlp = B16(sv + s.mlp), *P = B16(sv + s.P);
  float *r1 = reinterpret_cast<float *>(sv + s.r1), *r2 = reinterpret_cast<float *>(sv + s.r2);
  bf16 *h1 = B16(wb + w.t1), *tmp = B16(wb + w.t2);
  float *scores = reinterpret_cast<float *>(wb + w.scores);
  void *many = wb + w.many;
  const size_t many_bytes = w.scores - w.many;
  const bf16 *hin = static_cast<const bf16 *>(h);
  // n1 = norm(h); q, k, v
  POET_TRY(block_rmsnorm(hin, g.hidden, T, int(g.hidden), blk->norm_eps, n1, g.ldh, r1, st));
  {
    const void *x3[3] = {n1, n1, n1};
    void *y3[3] = {qr, kr, v};
    void *s3[3] = {sv + s.sv[LQ], sv + s.sv[LK], sv + s.sv[LV]};
    const int64_t ld3[3] = {g.ldh, g.ldh, g.ldh};
    POET_TRY(poet_forward_many(L + LQ, 3, x3, ld3, T, y3, ld3, s3, many, many_bytes, stream));
  }
  POET_TRY(block_rope(qr, g.ldh, T, int(g.hidden), g.hd, g.S, blk->rope_base, false, st));
  POET_TRY(block_rope(kr, g.ldh, T, int(g.hidden), g.hd, g.S, blk->rope_base, false, st));
  // attention: scores = qr kr^T / sqrt(hd), P = causal softmax, att = P v
  const int64_t SS = int64_t(g.S) * g.S;
  const float scale = 1.f / std::sqrt(float(g.hd));
  std::vector<Gemm> gs;
  for (int b = 0; b < g.B; ++b) {
    Gemm p = attn_gemm(g, "attn");
    p.M = g.S; p.N = g.S; p.K = g.hd; p.alpha = scale;
    p.A = qr + int64_t(b) * g.S * g.ldh; p.a_m = g.ldh; p.a_k = 1; p.a_b = g.hd;
    p.B = kr + int64_t(b) * g.S * g.ldh; p.b_n = g.ldh; p.b_k = 1; p.b_b = g.hd;
    p.outF = scores + int64_t(b) * g.H * SS; p.of_m = g.S; p.of_b = SS;
    gs.push_back(p);
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  POET_TRY(block_softmax(scores, int64_t(g.B) * g.H * g.S, g.S, P, st));
  gs.clear();
  for (int b = 0; b < g.B; ++b) {
    Gemm p = attn_gemm(g, "attn");
    p.M = g.S; p.N = g.hd; p.K = g.S;
    p.A = P + int64_t(b) * g.H * SS; p.a_m = g.S; p.a_k = 1; p.a_b = SS;
    p.B = v + int64_t(b) * g.S * g.ldh; p.b_n = 1; p.b_k = g.ldh; p.b_b = g.hd;
    p.outD = att + int64_t(b) * g.S * g.ldh; p.od_m = g.ldh; p.od_b = g.hd;
    gs.push_back(p);
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  // h1 = h + o(att); n2 = norm(h1)
  {
    const void *x1[1] = {att};
    void *y1[1] = {tmp};
    void *s1[1] = {sv + s.sv[LO]};
    const int64_t ld1[1] = {g.ldh};
    POET_TRY(poet_forward_many(L + LO, 1, x1, ld1, T, y1, ld1, s1, many, many_bytes, stream));
  }
  POET_TRY(block_add(hin, g.hidden, tmp, g.ldh, T, int(g.hidden), h1, g.ldh, st));
  POET_TRY(block_rmsnorm(h1, g.ldh, T, int(g.hidden), blk->norm_eps, n2, g.ldh, r2, st));
  // gate, up; mlp = silu(gate) up; out = h1 + down(mlp)
  {
    const void *x2[2] = {n2, n2};
    void *y2[2] = {gg, uu};
    void *s2[2] = {sv + s.sv[LGATE], sv + s.sv[LUP]};
    const int64_t ldx2[2] = {g.ldh, g.ldh}, ldy2[2] = {g.ldf, g.ldf};
    POET_TRY(poet_forward_many(L + LGATE, 2, x2, ldx2, T, y2, ldy2, s2, many, many_bytes, stream));
  }
  POET_TRY(block_swiglu(gg, uu, g.ldf, T, int(g.ffn), mlp, g.ldf, st));
  {
    const void *x1[1] = {mlp};
    void *y1[1] = {tmp};
    void *s1[1] = {sv + s.sv[LDOWN]};
    const int64_t ldx1[1] = {g.ldf}, ldy1[1] = {g.ldh};
    POET_TRY(poet_forward_many(L + LDOWN, 1, x1, ldx1, T, y1, ldy1, s1, many, many_bytes, stream));
  }
  return block_add(h1, g.ldh, tmp, g.ldh, T, int(g.hidden), static_cast<bf16 *>(out), g.hidden, st);
}

poet_status poet_llama_block_backward(const poet_llama_block *blk, const void *saved, const void *dout, int64_t T,
                                      void *dh, float *const *G, void *ws, size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_llama_block_backward");
  clear_error();
  BlockGeom g;
  POET_TRY(check_block(blk, T, &g));
  POET_REQUIRE(G != nullptr, "poet_llama_block_backward: G list is NULL");
  const poet_layer *L = blk->lin;
  float *GR[NLIN], *GP[NLIN];
  for (int i = 0; i < NLIN; ++i) {
    GR[i] = G[2 * i];
    GP[i] = G[2 * i + 1];
  }
  if (T == 0) {  // no tokens: every per-primitive gradient is zero
    const void *none[NLIN] = {};
    void *nonev[NLIN] = {};
    for (int i = 0; i < NLIN; ++i)
      POET_TRY(poet_backward_blocks_many(L + i, 1, none, nullptr, none, none, nullptr, 0, nonev, nullptr, GR + i,
                                         GP + i, nullptr, 0, stream));
    return POET_OK;
  }
  POET_REQUIRE(dout && dh && (reinterpret_cast<uintptr_t>(dout) & 15) == 0 && (reinterpret_cast<uintptr_t>(dh) & 15) == 0,
               "poet_llama_block_backward: dout/dh NULL or not 16-byte aligned");
  POET_REQUIRE(saved && (reinterpret_cast<uintptr_t>(saved) & 255) == 0,
               "poet_llama_block_backward: saved NULL or not 256-byte aligned");
  const SavedLayout s = saved_layout(blk, g);
  const WsLayoutB w = ws_layout_block(blk, g);
  if (!ws || ws_bytes < w.bytes || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) {
    set_error("poet_llama_block_backward: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, w.bytes);
    return POET_ENOMEM_WS;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const char *sv = static_cast<const char *>(saved);
  char *wb = static_cast<char *>(ws);
  auto C16 = [](const void *p) { return static_cast<const bf16 *>(p); };
  auto B16 = [](void *p) { return static_cast<bf16 *>(p); };
  const bf16 *n1 = C16(sv + s.n1), *qr = C16(sv + s.qr), *kr = C16(sv + s.kr), *v = C16(sv + s.v);
  const bf16 *att = C16(sv + s.att), *n2 = C16(sv + s.n2), *gg = C16(sv + s.g), *uu = C16(sv + s.u);
  const bf16 *mlp = C16(sv + s.mlp), *P = C16(sv + s.P);
  const float *r1 = reinterpret_cast<const float *>(sv + s.r1), *r2 = reinterpret_cast<const float *>(sv + s.r2);
  bf16 *dmlp = B16(wb + w.dmlp), *dg = B16(wb + w.dg), *du = B16(wb + w.du);
  bf16 *dn2g = B16(wb + w.dn2g), *dn2u = B16(wb + w.dn2u), *dh1 = B16(wb + w.dh1), *datt = B16(wb + w.datt);
  bf16 *dqr = B16(wb + w.dqr), *dkr = B16(wb + w.dkr), *dv = B16(wb + w.dv);
  bf16 *dn1q = B16(wb + w.dn1q), *dn1k = B16(wb + w.dn1k), *dn1v = B16(wb + w.dn1v);
  float *dP = reinterpret_cast<float *>(wb + w.scores);
  bf16 *dS = B16(wb + w.dS);
  void *many = wb + w.many;
  const size_t many_bytes = w.scores - w.many;
  const bf16 *dO = static_cast<const bf16 *>(dout);
  // down: dmlp; gate, up through SwiGLU
  {
    const void *x1[1] = {mlp}, *s1[1] = {sv + s.sv[LDOWN]}, *d1[1] = {dO};
    void *o1[1] = {dmlp};
    const int64_t ldx1[1] = {g.ldf}, ldd1[1] = {g.hidden}, ldo1[1] = {g.ldf};
    POET_TRY(poet_backward_blocks_many(L + LDOWN, 1, x1, ldx1, s1, d1, ldd1, T, o1, ldo1, GR + LDOWN, GP + LDOWN,
                                       many, many_bytes, stream));
  }
  POET_TRY(block_swiglu_bwd(dmlp, g.ldf, gg, uu, g.ldf, T, int(g.ffn), dg, du, g.ldf, st));
  {
    const void *x2[2] = {n2, n2}, *s2[2] = {sv + s.sv[LGATE], sv + s.sv[LUP]}, *d2[2] = {dg, du};
    void *o2[2] = {dn2g, dn2u};
    const int64_t ldx2[2] = {g.ldh, g.ldh}, ldd2[2] = {g.ldf, g.ldf}, ldo2[2] = {g.ldh, g.ldh};
    POET_TRY(poet_backward_blocks_many(L + LGATE, 2, x2, ldx2, s2, d2, ldd2, T, o2, ldo2, GR + LGATE, GP + LGATE,
                                       many, many_bytes, stream));
  }
  // dh1 = dout + norm backward of (dn2g + dn2u)
  POET_TRY(block_rmsnorm_bwd(dn2g, dn2u, nullptr, g.ldh, n2, g.ldh, r2, dO, g.hidden, T, int(g.hidden), dh1, g.ldh,
                             st));
  // o: datt
  {
    const void *x1[1] = {att}, *s1[1] = {sv + s.sv[LO]}, *d1[1] = {dh1};
    void *o1[1] = {datt};
    const int64_t ld1[1] = {g.ldh};
    POET_TRY(poet_backward_blocks_many(L + LO, 1, x1, ld1, s1, d1, ld1, T, o1, ld1, GR + LO, GP + LO, many,
                                       many_bytes, stream));
  }
  // attention backward: dP = datt v^T, dv = P^T datt, dS = softmax backward, dqr = dS kr, dkr = dS^T qr
  const int64_t SS = int64_t(g.S) * g.S;
  const float scale = 1.f / std::sqrt(float(g.hd));
  std::vector<Gemm> gs;
  for (int b = 0; b < g.B; ++b) {
    const int64_t ro = int64_t(b) * g.S * g.ldh, po = int64_t(b) * g.H * SS;
    Gemm p = attn_gemm(g, "attn");  // dP (float)
    p.M = g.S; p.N = g.S; p.K = g.hd;
    p.A = datt + ro; p.a_m = g.ldh; p.a_k = 1; p.a_b = g.hd;
    p.B = v + ro; p.b_n = g.ldh; p.b_k = 1; p.b_b = g.hd;
    p.outF = dP + po; p.of_m = g.S; p.of_b = SS;
    gs.push_back(p);
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  gs.clear();
  for (int b = 0; b < g.B; ++b) {
    const int64_t ro = int64_t(b) * g.S * g.ldh, po = int64_t(b) * g.H * SS;
    Gemm p = attn_gemm(g, "attn");  // dv = P^T datt: P read transposed (MN-major)
    p.M = g.S; p.N = g.hd; p.K = g.S;
    p.A = P + po; p.a_m = 1; p.a_k = g.S; p.a_b = SS;
    p.B = datt + ro; p.b_n = 1; p.b_k = g.ldh; p.b_b = g.hd;
    p.outD = dv + ro; p.od_m = g.ldh; p.od_b = g.hd;
    gs.push_back(p);
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  POET_TRY(block_softmax_bwd(P, dP, int64_t(g.B) * g.H * g.S, g.S, scale, dS, st));
  gs.clear();
  for (int b = 0; b < g.B; ++b) {
    const int64_t ro = int64_t(b) * g.S * g.ldh, po = int64_t(b) * g.H * SS;
    Gemm p = attn_gemm(g, "attn");  // dqr = dS kr
    p.M = g.S; p.N = g.hd; p.K = g.S;
    p.A = dS + po; p.a_m = g.S; p.a_k = 1; p.a_b = SS;
    p.B = kr + ro; p.b_n = 1; p.b_k = g.ldh; p.b_b = g.hd;
    p.outD = dqr + ro; p.od_m = g.ldh; p.od_b = g.hd;
    gs.push_back(p);
    Gemm q = attn_gemm(g, "attn");  // dkr = dS^T qr: dS read transposed
    q.M = g.S; q.N = g.hd; q.K = g.S;
    q.A = dS + po; q.a_m = 1; q.a_k = g.S; q.a_b = SS;
    q.B = qr + ro; q.b_n = 1; q.b_k = g.ldh; q.b_b = g.hd;
    q.outD = dkr + ro; q.od_m = g.ldh; q.od_b = g.hd;
    gs.push_back(q);
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  POET_TRY(block_rope(dqr, g.ldh, T, int(g.hidden), g.hd, g.S, blk->rope_base, true, st));
  POET_TRY(block_rope(dkr, g.ldh, T, int(g.hidden), g.hd, g.S, blk->rope_base, true, st));
  // q, k, v: dn1 parts; dh = dh1 + norm backward of their sum
  {
    const void *x3[3] = {n1, n1, n1}, *s3[3] = {sv + s.sv[LQ], sv + s.sv[LK], sv + s.sv[LV]},
               *d3[3] = {dqr, dkr, dv};
    void *o3[3] = {dn1q, dn1k, dn1v};
    const int64_t ld3[3] = {g.ldh, g.ldh, g.ldh};
    POET_TRY(poet_backward_blocks_many(L + LQ, 3, x3, ld3, s3, d3, ld3, T, o3, ld3, GR + LQ, GP + LQ, many,
                                       many_bytes, stream));
  }
  return block_rmsnorm_bwd(dn1q, dn1k, dn1v, g.ldh, n1, g.ldh, r1, dh1, g.ldh, T, int(g.hidden),
                           static_cast<bf16 *>(dh), g.hidden, st);
}

}  // extern "C"
