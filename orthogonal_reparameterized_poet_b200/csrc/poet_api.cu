// libpoet C ABI: argument validation and the order of the steps of the POET
// layer y = R W0 P x (POET summary page, Approach).  Every arithmetic step
// runs in this library's CUDA kernels; nothing falls back to the host.
//
// Data flow of one layer (frame = indices ordered by the side's permutation,
// see poet.h), T tokens, q_R / q_P primitives of size s_R / s_P:
//   forward   x --gather(P.perm)--> xf --blocks P_j--> uf --W0f--> vf
//             --blocks R_j--> yf --scatter(R.perm)--> y           (saved: xf, vf)
//   backward  dy --gather(R.perm)--> dyf --blocks R_j^T--> dvf --W0f^T--> duf
//             --blocks P_j^T--> dxf --scatter(P.perm)--> dx
//             G_R[j] = dyf_j^T vf_j,  G_P[j] = duf_j^T xf_j  (summed over tokens)
//             dtheta = Cayley-Neumann backward of G
// Frame indices past q*s (the leftover identity part) pass through unchanged.
//
// The weight plan computes the same layer with the primitives applied to W0:
//   forward   H = R W0f, F = W0f P, E_f = H P (frame, weight-sized),
//             E = E_f unframed (natural order),  y = x E^T       (saved: E, F, H)
//   backward  dx = dy E,  D = dy^T x (natural),  D_f = D framed,
//             G_R[j] = D_f[rows j] F[rows j]^T,  G_P[j] = H[:, cols j]^T D_f[:, cols j]
// (G_R = sum_t dyf_t vf_t^T with vf_t = F xf_t, and G_P = sum_t duf_t xf_t^T with
// duf_t = H^T dyf_t, so both plans give the same gradients.)
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "poet_internal.cuh"

namespace poet {

// ------------------------------------------------------------------ errors

static thread_local char g_last_error[512] = "";

void set_error(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}
void clear_error() { g_last_error[0] = 0; }

poet_status launch_status(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("%s: launch failed: %s", what, cudaGetErrorString(e));
    return POET_ECUDA;
  }
  return POET_OK;
}

__device__ unsigned g_errword;

unsigned *device_errword() {
  static std::mutex mu;
  static std::vector<unsigned *> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (int(cache.size()) <= dev) cache.resize(dev + 1, nullptr);
  if (!cache[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_errword) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<unsigned *>(p);
  }
  return cache[dev];
}

int num_sms() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (int(cache.size()) <= dev) cache.resize(dev + 1, 0);
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

// ------------------------------------------------------------------ geometry

bool side_geom(const poet_side *s, SideGeom *g) {
  if (!s || s->dim < 1 || s->dim > 16384 || s->k < 0 || s->k > 16) return false;
  SideGeom r;
  if (s->mode == POET_FS) {
    r.size = s->dim / 2;
    r.nprim = r.size >= 1 ? 1 : 0;
  } else if (s->mode == POET_BS) {
    if (s->b < 1) return false;
    r.size = s->b;
    r.nprim = s->dim / s->b;
  } else {
    return false;
  }
  if (r.nprim == 0) r.size = 0;
  r.ld = int(round_up(r.size, 8));
  r.covered = r.nprim * r.size;
  r.k = s->k;
  *g = r;
  return true;
}

StateLayout state_layout(const SideGeom &g, int dtype) {
  StateLayout L;
  L.term = align256(size_t(g.all_elems()) * esize(dtype));
  L.R = 0;
  L.Q = L.term;
  L.S1 = 2 * L.term;
  L.bytes = size_t(2 + g.k) * L.term;
  return L;
}

namespace {

bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }
bool aligned_elem(const void *p, int dtype) { return (reinterpret_cast<uintptr_t>(p) % esize(dtype)) == 0; }

struct LayerGeom {
  SideGeom R, P;
  int64_t m = 0, n = 0, ldm = 0, ldn = 0;
  int dtype = 0;
  int plan = POET_PLAN_AUTO;  // as requested; resolve_plan() gives the one that runs
};

poet_status check_layer(const poet_layer *L, LayerGeom *lg, bool need_state) {
  POET_REQUIRE(L != nullptr, "layer is NULL");
  POET_REQUIRE(L->m >= 1 && L->n >= 1 && L->m <= 16384 && L->n <= 16384, "layer shape %lld x %lld outside [1,16384]^2",
               (long long)L->m, (long long)L->n);
  POET_REQUIRE(L->dtype == POET_F32 || L->dtype == POET_BF16, "dtype %d is not POET_F32 or POET_BF16", L->dtype);
  POET_REQUIRE(L->R.dim == L->m && L->P.dim == L->n, "side dims (%d, %d) do not match W0 (%lld x %lld)", L->R.dim,
               L->P.dim, (long long)L->m, (long long)L->n);
  POET_REQUIRE(side_geom(&L->R, &lg->R), "malformed R side (mode %d, b %d, k %d)", L->R.mode, L->R.b, L->R.k);
  POET_REQUIRE(side_geom(&L->P, &lg->P), "malformed P side (mode %d, b %d, k %d)", L->P.mode, L->P.b, L->P.k);
  POET_REQUIRE(L->layer_id >= 0 && L->epoch >= 0, "layer_id/epoch must be >= 0");
  POET_REQUIRE(L->plan == POET_PLAN_AUTO || L->plan == POET_PLAN_TOKEN || L->plan == POET_PLAN_WEIGHT,
               "plan %d is not a poet_plan", L->plan);
  POET_REQUIRE(L->R.perm && L->P.perm, "perm pointers must not be NULL");
  POET_REQUIRE(L->W0 && aligned_elem(L->W0, L->dtype), "W0 is NULL or misaligned");
  POET_REQUIRE(L->W0f && aligned256(L->W0f), "W0f is NULL or not 256-byte aligned");
  if (need_state) {
    POET_REQUIRE(lg->R.nprim == 0 || (L->R.state && aligned256(L->R.state)), "R.state is NULL or not 256-byte aligned");
    POET_REQUIRE(lg->P.nprim == 0 || (L->P.state && aligned256(L->P.state)), "P.state is NULL or not 256-byte aligned");
  }
  lg->m = L->m;
  lg->n = L->n;
  lg->ldm = frame_ld(L->m);
  lg->ldn = frame_ld(L->n);
  lg->dtype = L->dtype;
  lg->plan = L->plan;
  return POET_OK;
}

// Plan choice for POET_PLAN_AUTO: estimated device time of fwd + bwd in
// tensor-core flop equivalents, one HBM byte counted as kFlopPerByte flops
// (about the ratio of the B200's dense bf16 rate to its HBM bandwidth).
constexpr double kFlopPerByte = 200.0;
int resolve_plan(const LayerGeom &lg, int64_t T) {
  if (lg.plan == POET_PLAN_TOKEN || lg.plan == POET_PLAN_WEIGHT) return lg.plan;
  const double m = double(lg.m), n = double(lg.n), t = double(T), es = double(esize(lg.dtype));
  const double cR = double(lg.R.nprim) * lg.R.size * lg.R.size, cP = double(lg.P.nprim) * lg.P.size * lg.P.size;
  // token plan: W0f forward and backward, three block products per side,
  // four permutation passes and the block passes' activation traffic
  const double tok = t * (4.0 * m * n + 6.0 * (cR + cP) + kFlopPerByte * es * 8.0 * (m + n));
  // weight plan: three T x m x n GEMMs, the weight-sized block products and
  // passes, and re-striding copies of x / dy whose rows are not 16-byte aligned
  double wt = t * 6.0 * m * n + 4.0 * n * cR + 6.0 * m * cP + kFlopPerByte * es * 12.0 * m * n;
  if (lg.n % 8) wt += kFlopPerByte * es * 2.0 * t * n;
  if (lg.m % 8) wt += kFlopPerByte * es * 2.0 * t * m;
  return wt < tok ? POET_PLAN_WEIGHT : POET_PLAN_TOKEN;
}

struct WsLayout {
  size_t act1 = 0, act2 = 0, act3 = 0, GR = 0, GP = 0, cnp = 0, Z = 0, D = 0, D2 = 0, bytes = 0;
};

// token plan: act1..act3 activation frames;  weight plan: act1 = re-strided
// dy, D = float m x ldn, D2 = its framed copy (float layers; bf16 layers frame
// D into Z).  Both: GR, GP, the Cayley-Neumann scratch and Z (m x ldn: merge,
// the weight plan's E_f and framed D).
WsLayout ws_layout(const LayerGeom &lg, int64_t T, int plan) {
  WsLayout w;
  const size_t es = esize(lg.dtype);
  const int64_t ldmax = lg.ldm > lg.ldn ? lg.ldm : lg.ldn;
  const size_t wsz = size_t(lg.m) * lg.ldn;
  size_t off = 0;
  if (plan == POET_PLAN_WEIGHT) {
    w.act1 = off; off += align256(size_t(T) * lg.ldm * es);
  } else {
    w.act1 = off; off += align256(size_t(T) * ldmax * es);
    w.act2 = off; off += align256(size_t(T) * lg.ldm * es);
    w.act3 = off; off += align256(size_t(T) * lg.ldn * es);
  }
  w.GR = off; off += align256(size_t(lg.R.all_elems()) * 4);
  w.GP = off; off += align256(size_t(lg.P.all_elems()) * 4);
  w.cnp = off;
  const size_t cr = cnp_scratch_bytes(lg.R, lg.dtype), cp = cnp_scratch_bytes(lg.P, lg.dtype);
  off += cr > cp ? cr : cp;
  w.Z = off; off += align256(wsz * es);
  if (plan == POET_PLAN_WEIGHT) {
    w.D = off; off += align256(wsz * 4);
    if (lg.dtype == POET_F32) { w.D2 = off; off += align256(wsz * 4); }  // bf16 frames D into Z
  }
  w.bytes = off;
  return w;
}

// Weight plan saved buffer: E (natural), F, H (frame), all m x ldn, then a
// T x ldn re-strided copy of x (used when x's rows are not 16-byte aligned).
struct WeightSaved {
  size_t E = 0, F = 0, H = 0, xp = 0, bytes = 0;
};
WeightSaved weight_saved(const LayerGeom &lg, int64_t T) {
  WeightSaved v;
  const size_t w = align256(size_t(lg.m) * lg.ldn * esize(lg.dtype));
  v.E = 0; v.F = w; v.H = 2 * w; v.xp = 3 * w;
  v.bytes = 3 * w + align256(size_t(T) * lg.ldn * esize(lg.dtype));
  return v;
}

bool rows16(const void *p, int64_t ld, int dtype) {
  return (reinterpret_cast<uintptr_t>(p) & 15) == 0 && (ld * int64_t(esize(dtype))) % 16 == 0;
}

size_t side_ws_bytes(const SideGeom &g, int dtype) {
  return align256(size_t(g.all_elems()) * 4) + cnp_scratch_bytes(g, dtype);
}

// token-parallel block-diagonal product in the frame:
//   C[t][j*s + a] = sum_c X[t][j*s + c] * (trans ? Blk_j[c][a] : Blk_j[a][c])
Gemm blockdiag(const SideGeom &g, int dtype, int64_t T, const void *X, int64_t ldx, const void *Blk, bool trans,
               void *C, int64_t ldc) {
  Gemm p;
  p.tag = trans ? "blk_bwd" : "blk_fwd";
  p.M = int(T); p.N = g.size; p.K = g.size; p.batch = g.nprim;
  p.dtype = dtype;
  p.A = X; p.a_m = ldx; p.a_k = 1; p.a_b = g.size;
  p.B = Blk;
  if (trans) { p.b_n = 1; p.b_k = g.ld; } else { p.b_n = g.ld; p.b_k = 1; }
  p.b_b = g.blk_elems();
  p.outD = C; p.od_m = ldc; p.od_b = g.size;
  return p;
}

// per-primitive gradient summed over tokens:
//   Gout[j][a][c] += sum_t D[t][j*s + a] * V[t][j*s + c]
Gemm blockgrad(const SideGeom &g, int dtype, int64_t T, const void *D, const void *V, int64_t ld, float *Gout) {
  Gemm p;
  p.tag = "blk_grad";
  p.M = g.size; p.N = g.size; p.K = int(T); p.batch = g.nprim;
  p.dtype = dtype;
  p.A = D; p.a_m = 1; p.a_k = ld; p.a_b = g.size;
  p.B = V; p.b_n = 1; p.b_k = ld; p.b_b = g.size;
  p.outF = Gout; p.of_m = g.ld; p.of_b = g.blk_elems();
  p.atomic = true;
  return p;
}

const void *state_R(const poet_side *s, const SideGeom &g, int dtype) {
  return static_cast<const char *>(s->state) + state_layout(g, dtype).R;
}

// out = blockdiag(R) src on the rows of an m x ldn frame matrix: the rows of
// each R primitive are multiplied by it, the leftover rows are copied.
Gemm left_blocks(const poet_layer *L, const LayerGeom &lg, const void *src, void *out, const char *tag) {
  const SideGeom &g = lg.R;
  const int64_t ldw = lg.ldn;
  Gemm p;
  p.tag = tag;
  p.M = g.size; p.N = int(lg.n); p.K = g.size; p.batch = g.nprim; p.dtype = lg.dtype;
  p.A = state_R(&L->R, g, lg.dtype); p.a_m = g.ld; p.a_k = 1; p.a_b = g.blk_elems();
  p.B = src; p.b_n = 1; p.b_k = ldw; p.b_b = int64_t(g.size) * ldw;
  p.outD = out; p.od_m = ldw; p.od_b = int64_t(g.size) * ldw;
  return p;
}
poet_status left_tail(const LayerGeom &lg, const void *src, void *out, cudaStream_t st) {
  if (lg.R.covered >= lg.m) return POET_OK;
  const size_t es = esize(lg.dtype), row = size_t(lg.ldn) * es;
  POET_CUDA_TRY(cudaMemcpyAsync(static_cast<char *>(out) + size_t(lg.R.covered) * row,
                                static_cast<const char *>(src) + size_t(lg.R.covered) * row,
                                size_t(lg.m - lg.R.covered) * row, cudaMemcpyDeviceToDevice, st));
  return POET_OK;
}

// out = src blockdiag(P) on the columns of an m x ldn frame matrix: the
// columns of each P primitive are multiplied by it, the leftover columns are
// copied.
Gemm right_blocks(const poet_layer *L, const LayerGeom &lg, const void *src, void *out, const char *tag) {
  const SideGeom &g = lg.P;
  const int64_t ldw = lg.ldn;
  Gemm p;
  p.tag = tag;
  p.M = int(lg.m); p.N = g.size; p.K = g.size; p.batch = g.nprim; p.dtype = lg.dtype;
  p.A = src; p.a_m = ldw; p.a_k = 1; p.a_b = g.size;
  p.B = state_R(&L->P, g, lg.dtype); p.b_n = 1; p.b_k = g.ld; p.b_b = g.blk_elems();
  p.outD = out; p.od_m = ldw; p.od_b = g.size;
  return p;
}
poet_status right_tail(const LayerGeom &lg, const void *src, void *out, cudaStream_t st) {
  if (lg.P.covered >= lg.n) return POET_OK;
  const size_t es = esize(lg.dtype), row = size_t(lg.ldn) * es;
  POET_CUDA_TRY(cudaMemcpy2DAsync(static_cast<char *>(out) + size_t(lg.P.covered) * es, row,
                                  static_cast<const char *>(src) + size_t(lg.P.covered) * es, row,
                                  size_t(lg.n - lg.P.covered) * es, size_t(lg.m), cudaMemcpyDeviceToDevice, st));
  return POET_OK;
}

}  // namespace

poet_status gemm_run(const Gemm &g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return POET_OK;
  const double mnb = double(g.M) * g.N * g.batch;
  const double bytes = double(esize(g.dtype)) * (double(g.M) + g.N) * g.K * g.batch +
                       mnb * ((g.outF ? 4.0 : 0.0) + (g.outD ? double(esize(g.dtype)) : 0.0) +
                              (g.add ? double(esize(g.add_dtype)) : 0.0));
  TraceScope ts(g.tag, 2.0 * mnb * g.K, bytes, st);
  if (gemm_tc_enabled() && gemm_tc_supported(g)) return gemm_tc(g, st);
  return gemm_simt(g, st);
}

poet_status gemm_run_many(const Gemm *gs, int count, cudaStream_t st) {
  if (count <= 0) return POET_OK;
  double flop = 0.0, bytes = 0.0;
  for (int i = 0; i < count; ++i) {
    const Gemm &g = gs[i];
    const double mnb = double(g.M) * g.N * g.batch;
    flop += 2.0 * mnb * g.K;
    bytes += double(esize(g.dtype)) * (double(g.M) + g.N) * g.K * g.batch +
             mnb * ((g.outF ? 4.0 : 0.0) + (g.outD ? double(esize(g.dtype)) : 0.0) +
                    (g.add ? double(esize(g.add_dtype)) : 0.0));
  }
  TraceScope ts(gs[0].tag, flop, bytes, st);
  return gemm_tc_many(gs, count, st);
}

}  // namespace poet

using namespace poet;

// ====================================================================== C ABI

extern "C" {

const char *poet_last_error(void) { return g_last_error; }

// The kernel revisions name the code that profiles/ counters were taken on.
const char *poet_version(void) { return "libpoet 0.3 (sm_100a; gemm_tc r9; permute r3; restride r1; cnp r2)"; }

size_t poet_side_state_bytes(const poet_side *side, int32_t dtype) {
  SideGeom g;
  if (!side_geom(side, &g) || (dtype != POET_F32 && dtype != POET_BF16)) return 0;
  return state_layout(g, dtype).bytes;
}

size_t poet_frame_bytes(const poet_layer *L) {
  if (!L || L->m < 1 || L->n < 1) return 0;
  return align256(size_t(L->m) * frame_ld(L->n) * esize(L->dtype));
}

// Shapes only, so that sizes can be queried before the pointers exist.
static bool shape_geom(const poet_layer *L, LayerGeom *lg) {
  if (!L || L->m < 1 || L->n < 1 || L->m > 16384 || L->n > 16384) return false;
  if (L->dtype != POET_F32 && L->dtype != POET_BF16) return false;
  if (L->plan != POET_PLAN_AUTO && L->plan != POET_PLAN_TOKEN && L->plan != POET_PLAN_WEIGHT) return false;
  if (!side_geom(&L->R, &lg->R) || !side_geom(&L->P, &lg->P)) return false;
  lg->m = L->m; lg->n = L->n; lg->ldm = frame_ld(L->m); lg->ldn = frame_ld(L->n);
  lg->dtype = L->dtype; lg->plan = L->plan;
  return true;
}

int32_t poet_plan_for(const poet_layer *L, int64_t T) {
  LayerGeom lg;
  if (T < 0 || !shape_geom(L, &lg)) return -1;
  return resolve_plan(lg, T);
}

size_t poet_saved_bytes(const poet_layer *L, int64_t T) {
  LayerGeom lg;
  if (T < 0 || !shape_geom(L, &lg)) return 0;
  if (resolve_plan(lg, T) == POET_PLAN_WEIGHT) return weight_saved(lg, T).bytes;
  const size_t es = esize(L->dtype);
  return align256(size_t(T) * lg.ldn * es) + align256(size_t(T) * lg.ldm * es);
}

size_t poet_workspace_bytes(const poet_layer *L, int64_t T) {
  LayerGeom lg;
  if (T < 0 || !shape_geom(L, &lg)) return 0;
  return ws_layout(lg, T, resolve_plan(lg, T)).bytes;
}

size_t poet_side_workspace_bytes(const poet_side *side, int32_t dtype) {
  SideGeom g;
  if (!side_geom(side, &g) || (dtype != POET_F32 && dtype != POET_BF16)) return 0;
  return side_ws_bytes(g, dtype);
}

poet_status poet_cayley_neumann(const poet_side *side, int32_t dtype, void *ws, size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_cayley_neumann");
  (void)ws; (void)ws_bytes;
  clear_error();
  SideGeom g;
  POET_REQUIRE(side_geom(side, &g), "poet_cayley_neumann: malformed side");
  POET_REQUIRE(dtype == POET_F32 || dtype == POET_BF16, "poet_cayley_neumann: bad dtype %d", dtype);
  if (g.nprim == 0) return POET_OK;
  POET_REQUIRE((side->theta || g.packed_per() == 0) && side->state && aligned256(side->state),
               "poet_cayley_neumann: theta/state NULL or state not 256-byte aligned");
  return cnp_forward(side, g, dtype, reinterpret_cast<cudaStream_t>(stream));
}

poet_status poet_cayley_neumann_grad(const poet_side *side, int32_t dtype, const float *G, float *dtheta, void *ws,
                                     size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_cayley_neumann_grad");
  clear_error();
  SideGeom g;
  POET_REQUIRE(side_geom(side, &g), "poet_cayley_neumann_grad: malformed side");
  POET_REQUIRE(dtype == POET_F32 || dtype == POET_BF16, "poet_cayley_neumann_grad: bad dtype %d", dtype);
  if (g.nprim == 0 || g.size < 2) return POET_OK;
  POET_REQUIRE(side->state && aligned256(side->state) && G && dtheta, "poet_cayley_neumann_grad: NULL argument");
  const size_t need = side_ws_bytes(g, dtype);
  if (ws_bytes < need || !ws || !aligned256(ws)) {
    set_error("poet_cayley_neumann_grad: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, need);
    return POET_ENOMEM_WS;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float *Gpad = static_cast<float *>(ws);
  POET_TRY(pad_blocks(G, g, Gpad, st));
  void *scratch = static_cast<char *>(ws) + align256(size_t(g.all_elems()) * 4);
  return cnp_backward(side, g, dtype, Gpad, dtheta, scratch, st);
}

// ------------------------------------------------------------------ weight plan

// E_f = R W0f P in the frame (H = R W0f and F = W0f P kept for the backward),
// then E = E_f in natural order.  Weight-sized work only.
static poet_status weight_factors(const poet_layer *L, const LayerGeom &lg, char *sv, const WeightSaved &ly, void *Ef,
                                  cudaStream_t st) {
  const int dt = lg.dtype;
  const void *W0f = L->W0f;
  const void *Hs = W0f, *Es = W0f;
  if (lg.R.nprim > 0) {
    POET_TRY(gemm_run(left_blocks(L, lg, W0f, sv + ly.H, "w_prep"), st));
    POET_TRY(left_tail(lg, W0f, sv + ly.H, st));
    Hs = sv + ly.H;
    Es = Hs;
  }
  if (lg.P.nprim > 0) {
    Gemm two[2] = {right_blocks(L, lg, W0f, sv + ly.F, "w_prep"), right_blocks(L, lg, Hs, Ef, "w_prep")};
    POET_TRY(gemm_run_many(two, 2, st));
    POET_TRY(right_tail(lg, W0f, sv + ly.F, st));
    POET_TRY(right_tail(lg, Hs, Ef, st));
    Es = Ef;
  }
  // E[R.perm[i]][P.perm[j]] = E_f[i][j]
  return scatter_cols(dt, Es, lg.ldn, Es, lg.ldn, int(lg.n), lg.m, int(lg.n), L->P.perm, sv + ly.E, lg.ldn,
                      L->R.perm, st, "unframe");
}

static poet_status forward_weight(const poet_layer *L, const LayerGeom &lg, const void *x, int64_t T, void *y,
                                  void *saved, char *wb, const WsLayout &w, cudaStream_t st) {
  const int dt = lg.dtype;
  char *sv = static_cast<char *>(saved);
  const WeightSaved ly = weight_saved(lg, T);
  POET_TRY(weight_factors(L, lg, sv, ly, wb + w.Z, st));
  // x as a GEMM operand needs 16-byte aligned rows
  const void *xa = x;
  int64_t ldx = lg.n;
  if (!rows16(x, lg.n, dt)) {
    POET_TRY(copy_rows(dt, x, lg.n, T, int(lg.n), sv + ly.xp, lg.ldn, st));
    xa = sv + ly.xp;
    ldx = lg.ldn;
  }
  Gemm p;  // y = x E^T
  p.tag = "w0_fwd";
  p.M = int(T); p.N = int(lg.m); p.K = int(lg.n); p.dtype = dt;
  p.A = xa; p.a_m = ldx; p.a_k = 1;
  p.B = sv + ly.E; p.b_n = lg.ldn; p.b_k = 1;
  p.outD = y; p.od_m = lg.m;
  return gemm_run(p, st);
}

static poet_status backward_weight(const poet_layer *L, const LayerGeom &lg, char *wb, const WsLayout &w,
                                   const void *x, const void *saved, const void *dy, int64_t T, void *dx, float *GR,
                                   float *GP, cudaStream_t st) {
  const int dt = lg.dtype;
  const SideGeom &gR = lg.R, &gP = lg.P;
  const char *sv = static_cast<const char *>(saved);
  const WeightSaved ly = weight_saved(lg, T);
  const void *xa = x;
  int64_t ldx = lg.n;
  if (!rows16(x, lg.n, dt)) { xa = sv + ly.xp; ldx = lg.ldn; }  // the forward's re-strided copy
  const void *dya = dy;
  int64_t ldy = lg.m;
  if (!rows16(dy, lg.m, dt)) {
    POET_TRY(copy_rows(dt, dy, lg.m, T, int(lg.m), wb + w.act1, lg.ldm, st));
    dya = wb + w.act1;
    ldy = lg.ldm;
  }
  {  // dx = dy E
    Gemm p;
    p.tag = "w0_bwd";
    p.M = int(T); p.N = int(lg.n); p.K = int(lg.m); p.dtype = dt;
    p.A = dya; p.a_m = ldy; p.a_k = 1;
    p.B = sv + ly.E; p.b_n = 1; p.b_k = lg.ldn;
    p.outD = dx; p.od_m = lg.n;
    POET_TRY(gemm_run(p, st));
  }
  if (gR.nprim == 0 && gP.nprim == 0) return POET_OK;
  // D = dy^T x (natural order, float, split over tokens)
  float *D = reinterpret_cast<float *>(wb + w.D);
  float *D2 = reinterpret_cast<float *>(wb + w.D2);
  const size_t wsz = size_t(lg.m) * lg.ldn;
  POET_CUDA_TRY(cudaMemsetAsync(D, 0, wsz * 4, st));
  {
    Gemm p;
    p.tag = "w_grad";
    p.M = int(lg.m); p.N = int(lg.n); p.K = int(T); p.dtype = dt;
    p.A = dya; p.a_m = 1; p.a_k = ldy;
    p.B = xa; p.b_n = 1; p.b_k = ldx;
    p.outF = D; p.of_m = lg.ldn;
    p.atomic = true;
    POET_TRY(gemm_run(p, st));
  }
  // D_f[i][j] = D[R.perm[i]][P.perm[j]], in the element type of the GEMMs
  const void *Df;
  if (dt == POET_BF16) {
    POET_TRY(frame_f32_to_bf16(D, lg.ldn, L->R.perm, lg.m, int(lg.n), L->P.perm, wb + w.Z, lg.ldn, st));
    Df = wb + w.Z;
  } else {
    POET_TRY(gather_cols(POET_F32, D, lg.ldn, L->R.perm, lg.m, int(lg.n), L->P.perm, D2, lg.ldn, nullptr, 0,
                         int(lg.n), st, "frame"));
    Df = D2;
  }
  const void *Fs = gP.nprim > 0 ? static_cast<const void *>(sv + ly.F) : L->W0f;
  const void *Hs = gR.nprim > 0 ? static_cast<const void *>(sv + ly.H) : L->W0f;
  // the per-primitive products are small (K = n or m): split over K, summed in place
  Gemm g2[2];
  int ng = 0;
  if (gR.nprim > 0) POET_CUDA_TRY(cudaMemsetAsync(GR, 0, size_t(gR.all_elems()) * 4, st));
  if (gP.nprim > 0) POET_CUDA_TRY(cudaMemsetAsync(GP, 0, size_t(gP.all_elems()) * 4, st));
  if (gR.nprim > 0) {  // G_R[j] = D_f[rows j] F[rows j]^T
    Gemm &p = g2[ng++];
    p.tag = "blk_grad";
    p.M = gR.size; p.N = gR.size; p.K = int(lg.n); p.batch = gR.nprim; p.dtype = dt;
    p.A = Df; p.a_m = lg.ldn; p.a_k = 1; p.a_b = int64_t(gR.size) * lg.ldn;
    p.B = Fs; p.b_n = lg.ldn; p.b_k = 1; p.b_b = int64_t(gR.size) * lg.ldn;
    p.outF = GR; p.of_m = gR.ld; p.of_b = gR.blk_elems();
    p.atomic = true;
  }
  if (gP.nprim > 0) {  // G_P[j] = H[:, cols j]^T D_f[:, cols j]
    Gemm &p = g2[ng++];
    p.tag = "blk_grad";
    p.M = gP.size; p.N = gP.size; p.K = int(lg.m); p.batch = gP.nprim; p.dtype = dt;
    p.A = Hs; p.a_m = 1; p.a_k = lg.ldn; p.a_b = gP.size;
    p.B = Df; p.b_n = 1; p.b_k = lg.ldn; p.b_b = gP.size;
    p.outF = GP; p.of_m = gP.ld; p.of_b = gP.blk_elems();
    p.atomic = true;
  }
  return gemm_run_many(g2, ng, st);
}

poet_status poet_forward(const poet_layer *L, const void *x, int64_t T, void *y, void *saved, void *ws,
                         size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_forward");
  clear_error();
  LayerGeom lg;
  POET_TRY(check_layer(L, &lg, true));
  POET_REQUIRE(T >= 0 && T <= (int64_t(1) << 31) - 1, "poet_forward: T=%lld out of range", (long long)T);
  if (T == 0) return POET_OK;
  POET_REQUIRE(x && y && aligned_elem(x, lg.dtype) && aligned_elem(y, lg.dtype), "poet_forward: x/y NULL or misaligned");
  POET_REQUIRE(saved && aligned256(saved), "poet_forward: saved NULL or not 256-byte aligned");
  const int plan = resolve_plan(lg, T);
  const WsLayout w = ws_layout(lg, T, plan);
  if (!ws || ws_bytes < w.bytes || !aligned256(ws)) {
    set_error("poet_forward: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, w.bytes);
    return POET_ENOMEM_WS;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (plan == POET_PLAN_WEIGHT) return forward_weight(L, lg, x, T, y, saved, static_cast<char *>(ws), w, st);
  const int dt = lg.dtype;
  const size_t es = esize(dt);
  char *sv = static_cast<char *>(saved);
  void *xf = sv;
  void *vf = sv + align256(size_t(T) * lg.ldn * es);
  char *wb = static_cast<char *>(ws);
  void *uf = wb + w.act1;
  void *yf = wb + w.act2;
  const SideGeom &gR = lg.R, &gP = lg.P;

  // a2: gather x into the P frame; the identity tail goes straight to uf
  const bool tailP = gP.nprim > 0 && gP.covered < lg.n;
  POET_TRY(gather_cols(dt, x, lg.n, nullptr, T, int(lg.n), L->P.perm, xf, lg.ldn, tailP ? uf : nullptr, lg.ldn,
                       gP.covered, st));
  const void *u = xf;
  if (gP.nprim > 0) {
    POET_TRY(gemm_run(blockdiag(gP, dt, T, xf, lg.ldn, state_R(&L->P, gP, dt), false, uf, lg.ldn), st));
    u = uf;
  }
  // a3: v = u W0f^T
  {
    Gemm p;
    p.tag = "w0_fwd";
    p.M = int(T); p.N = int(lg.m); p.K = int(lg.n); p.dtype = dt;
    p.A = u; p.a_m = lg.ldn; p.a_k = 1;
    p.B = L->W0f; p.b_n = lg.ldn; p.b_k = 1;
    p.outD = vf; p.od_m = lg.ldm;
    POET_TRY(gemm_run(p, st));
  }
  // a4: R blocks, then scatter to natural order (tail straight from vf)
  const void *ysrc = vf;
  if (gR.nprim > 0) {
    POET_TRY(gemm_run(blockdiag(gR, dt, T, vf, lg.ldm, state_R(&L->R, gR, dt), false, yf, lg.ldm), st));
    ysrc = yf;
  }
  return scatter_cols(dt, ysrc, lg.ldm, vf, lg.ldm, gR.covered, T, int(lg.m), L->R.perm, y, lg.m, nullptr, st);
}

static poet_status backward_core(const poet_layer *L, const LayerGeom &lg, int plan, char *wb, const WsLayout &w,
                                 const void *x, const void *saved, const void *dy, int64_t T, void *dx, float *GR,
                                 float *GP, cudaStream_t st) {
  const int dt = lg.dtype;
  const size_t es = esize(dt);
  const SideGeom &gR = lg.R, &gP = lg.P;
  if (T > 0 && plan == POET_PLAN_WEIGHT) {
    POET_REQUIRE(dy && dx && aligned_elem(dy, dt) && aligned_elem(dx, dt), "backward: dy/dx NULL or misaligned");
    POET_REQUIRE(x && aligned_elem(x, dt), "backward: x NULL or misaligned (the weight plan reads x)");
    POET_REQUIRE(saved && aligned256(saved), "backward: saved NULL or not 256-byte aligned");
    return backward_weight(L, lg, wb, w, x, saved, dy, T, dx, GR, GP, st);
  }
  if (T > 0) {
    POET_REQUIRE(dy && dx && aligned_elem(dy, dt) && aligned_elem(dx, dt), "backward: dy/dx NULL or misaligned");
    POET_REQUIRE(saved && aligned256(saved), "backward: saved NULL or not 256-byte aligned");
    const char *sv = static_cast<const char *>(saved);
    const void *xf = sv;
    const void *vf = sv + align256(size_t(T) * lg.ldn * es);
    void *dyf = wb + w.act1, *dvf = wb + w.act2, *duf = wb + w.act3, *dxf = wb + w.act1;

    // a5: gather dy into the R frame (tail straight to dvf), dv = R^T dy, G_R
    const bool tailR = gR.nprim > 0 && gR.covered < lg.m;
    POET_TRY(gather_cols(dt, dy, lg.m, nullptr, T, int(lg.m), L->R.perm, dyf, lg.ldm, tailR ? dvf : nullptr, lg.ldm,
                         gR.covered, st));
    const void *dv = dyf;
    if (gR.nprim > 0) {
      POET_TRY(gemm_run(blockdiag(gR, dt, T, dyf, lg.ldm, state_R(&L->R, gR, dt), true, dvf, lg.ldm), st));
      dv = dvf;
      POET_CUDA_TRY(cudaMemsetAsync(GR, 0, size_t(gR.all_elems()) * 4, st));
      POET_TRY(gemm_run(blockgrad(gR, dt, T, dyf, vf, lg.ldm, GR), st));
    }
    // a6: du = dv W0f
    {
      Gemm p;
      p.tag = "w0_bwd";
      p.M = int(T); p.N = int(lg.n); p.K = int(lg.m); p.dtype = dt;
      p.A = dv; p.a_m = lg.ldm; p.a_k = 1;
      p.B = L->W0f; p.b_n = 1; p.b_k = lg.ldn;
      p.outD = duf; p.od_m = lg.ldn;
      POET_TRY(gemm_run(p, st));
    }
    // a7: G_P, dx = P^T du, scatter (tail straight from du)
    const void *dxsrc = duf;
    if (gP.nprim > 0) {
      POET_CUDA_TRY(cudaMemsetAsync(GP, 0, size_t(gP.all_elems()) * 4, st));
      POET_TRY(gemm_run(blockgrad(gP, dt, T, duf, xf, lg.ldn, GP), st));
      POET_TRY(gemm_run(blockdiag(gP, dt, T, duf, lg.ldn, state_R(&L->P, gP, dt), true, dxf, lg.ldn), st));
      dxsrc = dxf;
    }
    POET_TRY(scatter_cols(dt, dxsrc, lg.ldn, duf, lg.ldn, gP.covered, T, int(lg.n), L->P.perm, dx, lg.n, nullptr, st));
  } else {
    if (gR.nprim > 0) POET_CUDA_TRY(cudaMemsetAsync(GR, 0, size_t(gR.all_elems()) * 4, st));
    if (gP.nprim > 0) POET_CUDA_TRY(cudaMemsetAsync(GP, 0, size_t(gP.all_elems()) * 4, st));
  }
  return POET_OK;
}

poet_status poet_backward(const poet_layer *L, const void *x, const void *saved, const void *dy, int64_t T,
                          void *dx, float *dtheta_R, float *dtheta_P, void *ws, size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_backward");
  clear_error();
  LayerGeom lg;
  POET_TRY(check_layer(L, &lg, true));
  POET_REQUIRE(T >= 0 && T <= (int64_t(1) << 31) - 1, "poet_backward: T=%lld out of range", (long long)T);
  const SideGeom &gR = lg.R, &gP = lg.P;
  POET_REQUIRE(gR.nprim == 0 || gR.size < 2 || dtheta_R, "poet_backward: dtheta_R is NULL");
  POET_REQUIRE(gP.nprim == 0 || gP.size < 2 || dtheta_P, "poet_backward: dtheta_P is NULL");
  const int plan = resolve_plan(lg, T);
  const WsLayout w = ws_layout(lg, T, plan);
  if (!ws || ws_bytes < w.bytes || !aligned256(ws)) {
    set_error("poet_backward: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, w.bytes);
    return POET_ENOMEM_WS;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *wb = static_cast<char *>(ws);
  float *GR = reinterpret_cast<float *>(wb + w.GR);
  float *GP = reinterpret_cast<float *>(wb + w.GP);
  POET_TRY(backward_core(L, lg, plan, wb, w, x, saved, dy, T, dx, GR, GP, st));
  // a8: through the Cayley-Neumann map to the packed parameters
  void *scratch = wb + w.cnp;
  if (gR.nprim > 0 && gR.size >= 2) POET_TRY(cnp_backward(&L->R, gR, lg.dtype, GR, dtheta_R, scratch, st));
  if (gP.nprim > 0 && gP.size >= 2) POET_TRY(cnp_backward(&L->P, gP, lg.dtype, GP, dtheta_P, scratch, st));
  return POET_OK;
}

poet_status poet_backward_blocks(const poet_layer *L, const void *x, const void *saved, const void *dy, int64_t T,
                                 void *dx, float *G_R, float *G_P, void *ws, size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_backward_blocks");
  clear_error();
  LayerGeom lg;
  POET_TRY(check_layer(L, &lg, true));
  POET_REQUIRE(T >= 0 && T <= (int64_t(1) << 31) - 1, "poet_backward_blocks: T=%lld out of range", (long long)T);
  POET_REQUIRE(lg.R.nprim == 0 || (G_R && (reinterpret_cast<uintptr_t>(G_R) & 15) == 0),
               "poet_backward_blocks: G_R NULL or not 16-byte aligned");
  POET_REQUIRE(lg.P.nprim == 0 || (G_P && (reinterpret_cast<uintptr_t>(G_P) & 15) == 0),
               "poet_backward_blocks: G_P NULL or not 16-byte aligned");
  const int plan = resolve_plan(lg, T);
  const WsLayout w = ws_layout(lg, T, plan);
  if (!ws || ws_bytes < w.bytes || !aligned256(ws)) {
    set_error("poet_backward_blocks: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, w.bytes);
    return POET_ENOMEM_WS;
  }
  return backward_core(L, lg, plan, static_cast<char *>(ws), w, x, saved, dy, T, dx, G_R, G_P,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t poet_block_grad_bytes(const poet_side *side) {
  SideGeom g;
  if (!side_geom(side, &g)) return 0;
  return size_t(g.all_elems()) * 4;
}

poet_status poet_cayley_neumann_many(const poet_side *sides, int32_t count, int32_t dtype, poet_stream stream) {
  CallRange nvtx_range("poet_cayley_neumann_many");
  clear_error();
  POET_REQUIRE(count >= 0 && (count == 0 || sides), "poet_cayley_neumann_many: bad side list");
  POET_REQUIRE(dtype == POET_F32 || dtype == POET_BF16, "poet_cayley_neumann_many: bad dtype %d", dtype);
  std::vector<SideGeom> geoms(count);
  for (int i = 0; i < count; ++i) {
    POET_REQUIRE(side_geom(&sides[i], &geoms[i]), "poet_cayley_neumann_many: side %d malformed", i);
    if (geoms[i].nprim == 0) continue;
    POET_REQUIRE((sides[i].theta || geoms[i].packed_per() == 0) && sides[i].state && aligned256(sides[i].state),
                 "poet_cayley_neumann_many: side %d theta/state NULL or misaligned", i);
  }
  return cnp_forward_many(sides, geoms.data(), count, dtype, reinterpret_cast<cudaStream_t>(stream));
}

size_t poet_cayley_neumann_grad_many_workspace_bytes(const poet_side *sides, int32_t count, int32_t dtype) {
  if (count < 0 || (count > 0 && !sides) || (dtype != POET_F32 && dtype != POET_BF16)) return 0;
  size_t total = 0;
  for (int i = 0; i < count; ++i) {
    SideGeom g;
    if (!side_geom(&sides[i], &g)) return 0;
    total += align256(cnp_many_scratch_bytes(g, dtype));
  }
  return total;
}

poet_status poet_cayley_neumann_grad_many(const poet_side *sides, const float *const *G, float *const *dtheta,
                                          int32_t count, int32_t dtype, void *ws, size_t ws_bytes,
                                          poet_stream stream) {
  CallRange nvtx_range("poet_cayley_neumann_grad_many");
  clear_error();
  POET_REQUIRE(count >= 0 && (count == 0 || (sides && G && dtheta)), "poet_cayley_neumann_grad_many: bad lists");
  POET_REQUIRE(dtype == POET_F32 || dtype == POET_BF16, "poet_cayley_neumann_grad_many: bad dtype %d", dtype);
  std::vector<SideGeom> geoms(count);
  std::vector<void *> scratch(count, nullptr);
  size_t off = 0;
  for (int i = 0; i < count; ++i) {
    POET_REQUIRE(side_geom(&sides[i], &geoms[i]), "poet_cayley_neumann_grad_many: side %d malformed", i);
    if (geoms[i].nprim == 0 || geoms[i].size < 2) continue;
    POET_REQUIRE(sides[i].state && aligned256(sides[i].state) && G[i] && dtheta[i] &&
                     (reinterpret_cast<uintptr_t>(G[i]) & 15) == 0,
                 "poet_cayley_neumann_grad_many: side %d state/G/dtheta NULL or misaligned", i);
    scratch[i] = static_cast<char *>(ws) + off;
    off += align256(cnp_many_scratch_bytes(geoms[i], dtype));
  }
  if (off > 0 && (!ws || ws_bytes < off || !aligned256(ws))) {
    set_error("poet_cayley_neumann_grad_many: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, off);
    return POET_ENOMEM_WS;
  }
  return cnp_backward_many(sides, geoms.data(), count, dtype, G, dtheta, scratch.data(),
                           reinterpret_cast<cudaStream_t>(stream));
}

poet_status poet_prepare(poet_layer *L, poet_stream stream) {
  CallRange nvtx_range("poet_prepare");
  clear_error();
  LayerGeom lg;
  POET_TRY(check_layer(L, &lg, false));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  POET_TRY(draw_perm_dev(L->seed, L->layer_id, 0, L->epoch, int(lg.m), L->R.perm, st));
  POET_TRY(draw_perm_dev(L->seed, L->layer_id, 1, L->epoch, int(lg.n), L->P.perm, st));
  // W0f[i][j] = W0[R.perm[i]][P.perm[j]]
  return gather_cols(lg.dtype, L->W0, lg.n, L->R.perm, lg.m, int(lg.n), L->P.perm, L->W0f, lg.ldn, nullptr, 0,
                     int(lg.n), st);
}

poet_status poet_resample(poet_layer *L, poet_stream stream) {
  CallRange nvtx_range("poet_resample");
  clear_error();
  POET_REQUIRE(L != nullptr, "poet_resample: layer is NULL");
  POET_REQUIRE(L->epoch >= 0 && L->epoch < 0x7FFFFFFF, "poet_resample: epoch %d cannot advance", L->epoch);
  L->epoch += 1;
  poet_status s = poet_prepare(L, stream);
  if (s != POET_OK) L->epoch -= 1;
  return s;
}

poet_status poet_draw_perm(uint64_t seed, int32_t layer_id, int32_t side, int32_t epoch, int32_t dim, int32_t *perm,
                           poet_stream stream) {
  CallRange nvtx_range("poet_draw_perm");
  clear_error();
  return draw_perm_dev(seed, layer_id, side, epoch, dim, perm, reinterpret_cast<cudaStream_t>(stream));
}

poet_status poet_merge(poet_layer *L, void *ws, size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_merge");
  clear_error();
  LayerGeom lg;
  POET_TRY(check_layer(L, &lg, true));
  POET_REQUIRE(lg.R.nprim == 0 || lg.R.packed_per() == 0 || L->R.theta, "poet_merge: R.theta is NULL");
  POET_REQUIRE(lg.P.nprim == 0 || lg.P.packed_per() == 0 || L->P.theta, "poet_merge: P.theta is NULL");
  const WsLayout w = ws_layout(lg, 0, POET_PLAN_TOKEN);
  if (!ws || ws_bytes < w.bytes || !aligned256(ws)) {
    set_error("poet_merge: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, w.bytes);
    return POET_ENOMEM_WS;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int dt = lg.dtype;
  const size_t es = esize(dt);
  const SideGeom &gR = lg.R, &gP = lg.P;
  char *W0f = static_cast<char *>(L->W0f);
  char *Z = static_cast<char *>(ws) + w.Z;
  const int64_t ldw = lg.ldn;
  if (gR.nprim > 0 || gP.nprim > 0) {
    // Z = blockdiag(R) W0f
    const char *src = W0f;
    if (gR.nprim > 0) {
      POET_TRY(gemm_run(left_blocks(L, lg, W0f, Z, "merge"), st));
      POET_TRY(left_tail(lg, W0f, Z, st));
      src = Z;
    }
    // W0f = src blockdiag(P)
    if (gP.nprim > 0) {
      if (src == W0f) {  // R had no primitives: the product cannot be written in place
        POET_CUDA_TRY(cudaMemcpyAsync(Z, W0f, size_t(lg.m) * ldw * es, cudaMemcpyDeviceToDevice, st));
        src = Z;
      }
      POET_TRY(gemm_run(right_blocks(L, lg, src, W0f, "merge"), st));
      POET_TRY(right_tail(lg, src, W0f, st));
    } else {
      POET_CUDA_TRY(cudaMemcpyAsync(W0f, Z, size_t(lg.m) * ldw * es, cudaMemcpyDeviceToDevice, st));
    }
    // W0[R.perm[i]][P.perm[j]] = W0f[i][j]
    POET_TRY(scatter_cols(dt, W0f, ldw, W0f, ldw, int(lg.n), lg.m, int(lg.n), L->P.perm, L->W0, lg.n, L->R.perm, st));
  }
  // reinitialize: theta <- 0 and re-materialize (every primitive becomes I)
  if (gR.nprim > 0) {
    if (gR.packed_per() > 0)
      POET_CUDA_TRY(cudaMemsetAsync(L->R.theta, 0, size_t(gR.nprim) * gR.packed_per() * 4, st));
    POET_TRY(cnp_forward(&L->R, gR, dt, st));
  }
  if (gP.nprim > 0) {
    if (gP.packed_per() > 0)
      POET_CUDA_TRY(cudaMemsetAsync(L->P.theta, 0, size_t(gP.nprim) * gP.packed_per() * 4, st));
    POET_TRY(cnp_forward(&L->P, gP, dt, st));
  }
  return POET_OK;
}

poet_status poet_gemm(int32_t dtype, int32_t M, int32_t N, int32_t K, int32_t batch, const void *A, int64_t sAm,
                      int64_t sAk, int64_t sAb, const void *B, int64_t sBn, int64_t sBk, int64_t sBb, void *C,
                      int64_t ldc, int64_t sCb, float alpha, float beta, poet_stream stream) {
  CallRange nvtx_range("poet_gemm");
  clear_error();
  POET_REQUIRE(dtype == POET_F32 || dtype == POET_BF16, "poet_gemm: bad dtype %d", dtype);
  POET_REQUIRE(M >= 0 && N >= 0 && K >= 0 && batch >= 0, "poet_gemm: negative size");
  if (M == 0 || N == 0 || batch == 0) return POET_OK;
  POET_REQUIRE(A && B && C && ldc >= N, "poet_gemm: NULL operand or ldc < N");
  Gemm p;
  p.M = M; p.N = N; p.K = K; p.batch = batch; p.dtype = dtype;
  p.A = A; p.a_m = sAm; p.a_k = sAk; p.a_b = sAb;
  p.B = B; p.b_n = sBn; p.b_k = sBk; p.b_b = sBb;
  p.alpha = alpha;
  if (beta != 0.f) { p.add = C; p.add_dtype = dtype; p.add_m = ldc; p.add_b = sCb; p.beta = beta; }
  p.outD = C; p.od_m = ldc; p.od_b = sCb;
  return gemm_run(p, reinterpret_cast<cudaStream_t>(stream));
}

poet_status poet_adamw_step(float *theta, const float *grad, float *m, float *v, int64_t n, float lr, float beta1,
                            float beta2, float eps, float weight_decay, int32_t step, poet_stream stream) {
  CallRange nvtx_range("poet_adamw_step");
  clear_error();
  POET_REQUIRE(n >= 0, "poet_adamw_step: n=%lld < 0", (long long)n);
  POET_REQUIRE(step >= 1, "poet_adamw_step: step=%d < 1", step);
  POET_REQUIRE(std::isfinite(lr) && lr >= 0.f && std::isfinite(weight_decay) && weight_decay >= 0.f,
               "poet_adamw_step: lr and weight_decay must be finite and >= 0");
  POET_REQUIRE(beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f, "poet_adamw_step: betas outside [0, 1)");
  POET_REQUIRE(std::isfinite(eps) && eps > 0.f, "poet_adamw_step: eps must be > 0");
  if (n == 0) return POET_OK;
  auto ok = [](const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 3) == 0; };
  POET_REQUIRE(ok(theta) && ok(grad) && ok(m) && ok(v), "poet_adamw_step: NULL or misaligned buffer");
  return adamw_step(theta, grad, m, v, n, lr, beta1, beta2, eps, weight_decay, step,
                    reinterpret_cast<cudaStream_t>(stream));
}

poet_status poet_selftest_bounded_wait(uint32_t timeout_us, poet_stream stream) {
  clear_error();
  return selftest_bounded_wait(timeout_us, reinterpret_cast<cudaStream_t>(stream));
}

int32_t poet_gemm_engine(int32_t dtype) { return (dtype == POET_BF16 && gemm_tc_enabled()) ? 1 : 0; }

poet_status poet_sync_status(poet_stream stream) {
  clear_error();
  POET_CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  unsigned *ew = device_errword();
  POET_REQUIRE(ew != nullptr, "poet_sync_status: no device status word");
  unsigned word = 0;
  POET_CUDA_TRY(cudaMemcpy(&word, ew, sizeof(word), cudaMemcpyDeviceToHost));
  if (word) {
    unsigned zero = 0;
    POET_CUDA_TRY(cudaMemcpy(ew, &zero, sizeof(zero), cudaMemcpyHostToDevice));
    set_error("device status word 0x%x (%s%s)", word, (word & ERR_TIMEOUT) ? "bounded wait ran out " : "",
              (word & ERR_BOUNDS) ? "index out of range skipped" : "");
    return (word & ERR_TIMEOUT) ? POET_ETIMEOUT : POET_EBOUNDS;
  }
  return POET_OK;
}

}  // extern "C"
