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
  p.small = SMALL_RIGHT;
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
  p.small = SMALL_GRAD;
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
  p.small = SMALL_LEFT;
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
  p.small = SMALL_RIGHT;
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
  bool done = false;
  POET_TRY(smallb_dispatch(g, st, &done));
  if (done) return POET_OK;
  const double mnb = double(g.M) * g.N * g.batch;
  const double bytes = double(esize(g.dtype)) * (double(g.M) + g.N) * g.K * g.batch +
                       mnb * ((g.outF ? 4.0 : 0.0) + (g.outD ? double(esize(g.dtype)) : 0.0) +
                              (g.add ? double(esize(g.add_dtype)) : 0.0) +
                              (g.add2 ? double(esize(g.add2_dtype)) : 0.0));
  TraceScope ts(g.tag, 2.0 * mnb * g.K, bytes, st);
  if (gemm_tc_enabled() && gemm_tc_supported(g)) return gemm_tc(g, st);
  return gemm_simt(g, st);
}

poet_status gemm_run_many(const Gemm *gs, int count, cudaStream_t st) {
  if (count <= 0) return POET_OK;
  std::vector<Gemm> rest;  // what the small-block kernels do not take
  for (int i = 0; i < count; ++i) {
    bool done = false;
    if (gs[i].M > 0 && gs[i].N > 0 && gs[i].batch > 0) POET_TRY(smallb_dispatch(gs[i], st, &done));
    if (!done) rest.push_back(gs[i]);
  }
  if (rest.empty()) return POET_OK;
  gs = rest.data();
  count = int(rest.size());
  double flop = 0.0, bytes = 0.0;
  for (int i = 0; i < count; ++i) {
    const Gemm &g = gs[i];
    const double mnb = double(g.M) * g.N * g.batch;
    flop += 2.0 * mnb * g.K;
    bytes += double(esize(g.dtype)) * (double(g.M) + g.N) * g.K * g.batch +
             mnb * ((g.outF ? 4.0 : 0.0) + (g.outD ? double(esize(g.dtype)) : 0.0) +
                    (g.add ? double(esize(g.add_dtype)) : 0.0) + (g.add2 ? double(esize(g.add2_dtype)) : 0.0));
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
const char *poet_version(void) { return "libpoet 0.4 (sm_100a; gemm_tc r27; permute r9; restride r1; cnp r7; smallb r6; block r1)"; }

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
//
// Every weight-plan call works on a list of layers, so that the weight-sized
// products of many layers share grouped tensor-core launches and their
// permutations share one launch; the single-layer entry points pass a list of
// one.  With c_R = R.covered and c_P = P.covered (frame indices acted on):
//   H = R W0f on the rows [0, c_R)            (the other rows of H are W0f's)
//   F = W0f P on the columns [0, c_P)         (the other columns are W0f's)
//   E_f = H P on the rows [0, c_R) and columns [0, c_P)
// and E = E_f unframed, reading E_f / H on the rows [0, c_R) and F / W0f on
// the others, each split at the column c_P.  The backward's per-primitive
// products read whole rows of F and whole columns of H, so H's leftover rows
// and F's leftover columns are copied from W0f once (one grouped launch):
// reading them from W0f in place would split each product's K range into two
// problems summed into one output, i.e. float reductions where one plain store
// suffices.

namespace {

struct WFwd {          // one layer of a grouped weight-plan forward
  const poet_layer *L;
  LayerGeom lg;
  const void *x; int64_t ldx;
  void *y; int64_t ldy;
  char *sv;            // saved buffer (weight_saved layout)
  void *Ef;            // m x ldn scratch in the storage type (E_f)
};

struct WBwd {          // one layer of a grouped weight-plan backward
  const poet_layer *L;
  LayerGeom lg;
  const void *x; int64_t ldx;
  const char *sv;
  const void *dy; int64_t lddy;
  void *dx; int64_t lddx;
  float *GR, *GP;      // per-primitive gradients (overwritten)
  void *act1;          // T x ldm scratch for a re-strided dy (used when dy's rows are not 16-byte aligned)
  float *D;            // m x ldn float scratch
  void *Df;            // m x ldn scratch in the storage type (D framed)
};

const char *at(const void *base, int64_t elems, int dtype) {
  return static_cast<const char *>(base) + elems * int64_t(esize(dtype));
}

poet_status forward_weight_many(std::vector<WFwd> &v, int64_t T, cudaStream_t st) {
  std::vector<Gemm> gs;
  std::vector<RowPermute> perms;
  if (v.empty()) return POET_OK;
  const int dt = v[0].lg.dtype;
  // H = R W0f (rows < c_R) and F = W0f P (columns < c_P), every layer in one grouped launch
  for (WFwd &f : v) {
    const WeightSaved ly = weight_saved(f.lg, T);
    if (f.lg.R.nprim > 0) gs.push_back(left_blocks(f.L, f.lg, f.L->W0f, f.sv + ly.H, "w_prep"));
    if (f.lg.P.nprim > 0) gs.push_back(right_blocks(f.L, f.lg, f.L->W0f, f.sv + ly.F, "w_prep"));
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  // H's leftover rows and F's leftover columns (the identity part of each side), for the backward
  for (WFwd &f : v) {
    const WeightSaved ly = weight_saved(f.lg, T);
    const int64_t cR = f.lg.R.covered, cP = f.lg.P.covered;
    if (f.lg.R.nprim > 0 && f.lg.P.nprim > 0 && cR < f.lg.m) {
      RowPermute r;
      r.src1 = at(f.L->W0f, cR * f.lg.ldn, dt); r.ld1 = f.lg.ldn;
      r.rows = f.lg.m - cR; r.d = int(f.lg.n);
      r.dst = const_cast<char *>(at(f.sv + ly.H, cR * f.lg.ldn, dt)); r.ldd = f.lg.ldn;
      perms.push_back(r);
    }
    if (f.lg.P.nprim > 0 && f.lg.R.nprim > 0 && cP < f.lg.n) {
      RowPermute r;
      r.src1 = at(f.L->W0f, cP, dt); r.ld1 = f.lg.ldn;
      r.rows = f.lg.m; r.d = int(f.lg.n - cP);
      r.dst = const_cast<char *>(at(f.sv + ly.F, cP, dt)); r.ldd = f.lg.ldn;
      perms.push_back(r);
    }
  }
  POET_TRY(permute_many(dt, perms, st, "copy"));
  // E_f = H P on the rows < c_R
  gs.clear();
  for (WFwd &f : v) {
    if (f.lg.R.nprim == 0 || f.lg.P.nprim == 0) continue;
    const WeightSaved ly = weight_saved(f.lg, T);
    Gemm p = right_blocks(f.L, f.lg, f.sv + ly.H, f.Ef, "w_prep");
    p.M = f.lg.R.covered;
    gs.push_back(p);
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  // E[R.perm[i]][P.perm[j]] = E_f[i][j], every layer in one launch
  perms.clear();
  for (WFwd &f : v) {
    const LayerGeom &lg = f.lg;
    const WeightSaved ly = weight_saved(lg, T);
    const int64_t cR = lg.R.covered, cP = lg.P.covered;
    const char *W0f = static_cast<const char *>(f.L->W0f);
    RowPermute r;
    r.ld1 = r.ld2 = lg.ldn;
    r.d = int(lg.n);
    r.perm = f.L->P.perm; r.inverse = 1;
    r.dst = f.sv + ly.E; r.ldd = lg.ldn;
    r.map_rows = lg.m;
    if (cR > 0) {  // rows acted on by R: E_f (columns < c_P) and H
      RowPermute a = r;
      a.src1 = cP > 0 ? static_cast<const void *>(f.Ef) : f.sv + ly.H;
      a.src2 = cP > 0 && cP < lg.n ? f.sv + ly.H : nullptr;
      a.split = int(cP);
      a.rows = cR;
      a.dst_rowmap = f.L->R.perm;
      perms.push_back(a);
    }
    if (cR < lg.m) {  // the other rows: F (columns < c_P) and W0f
      RowPermute b = r;
      b.src1 = at(cP > 0 ? static_cast<const void *>(f.sv + ly.F) : W0f, cR * lg.ldn, dt);
      b.src2 = cP > 0 && cP < lg.n ? at(W0f, cR * lg.ldn, dt) : nullptr;
      b.split = int(cP);
      b.rows = lg.m - cR;
      b.dst_rowmap = f.L->R.perm + cR;
      perms.push_back(b);
    }
  }
  POET_TRY(permute_many(dt, perms, st, "unframe"));
  // y = x E^T, every layer in one grouped launch (x re-strided first where its rows are not 16-byte aligned)
  gs.clear();
  for (WFwd &f : v) {
    const LayerGeom &lg = f.lg;
    const WeightSaved ly = weight_saved(lg, T);
    const void *xa = f.x;
    int64_t ldx = f.ldx;
    if (!rows16(f.x, f.ldx, dt)) {
      POET_TRY(copy_rows(dt, f.x, f.ldx, T, int(lg.n), f.sv + ly.xp, lg.ldn, st));
      xa = f.sv + ly.xp;
      ldx = lg.ldn;
    }
    Gemm p;
    p.tag = "w0_fwd";
    p.M = int(T); p.N = int(lg.m); p.K = int(lg.n); p.dtype = dt;
    p.A = xa; p.a_m = ldx; p.a_k = 1;
    p.B = f.sv + ly.E; p.b_n = lg.ldn; p.b_k = 1;
    p.outD = f.y; p.od_m = f.ldy;
    gs.push_back(p);
  }
  return gemm_run_many(gs.data(), int(gs.size()), st);
}

poet_status backward_weight_many(std::vector<WBwd> &v, int64_t T, cudaStream_t st) {
  if (v.empty()) return POET_OK;
  const int dt = v[0].lg.dtype;
  std::vector<Gemm> gs;
  std::vector<const void *> xa(v.size()), dya(v.size());
  std::vector<int64_t> ldxa(v.size()), ldya(v.size());
  // dx = dy E, every layer in one grouped launch
  for (size_t i = 0; i < v.size(); ++i) {
    WBwd &b = v[i];
    const LayerGeom &lg = b.lg;
    const WeightSaved ly = weight_saved(lg, T);
    xa[i] = b.x; ldxa[i] = b.ldx;
    if (!rows16(b.x, b.ldx, dt)) { xa[i] = b.sv + ly.xp; ldxa[i] = lg.ldn; }  // the forward's re-strided copy
    dya[i] = b.dy; ldya[i] = b.lddy;
    if (!rows16(b.dy, b.lddy, dt)) {
      POET_TRY(copy_rows(dt, b.dy, b.lddy, T, int(lg.m), b.act1, lg.ldm, st));
      dya[i] = b.act1; ldya[i] = lg.ldm;
    }
    Gemm p;
    p.tag = "w0_bwd";
    p.M = int(T); p.N = int(lg.n); p.K = int(lg.m); p.dtype = dt;
    p.A = dya[i]; p.a_m = ldya[i]; p.a_k = 1;
    p.B = b.sv + ly.E; p.b_n = 1; p.b_k = lg.ldn;
    p.outD = b.dx; p.od_m = b.lddx;
    gs.push_back(p);
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  // D = dy^T x (natural order, float) for the layers with primitives
  gs.clear();
  for (size_t i = 0; i < v.size(); ++i) {
    WBwd &b = v[i];
    const LayerGeom &lg = b.lg;
    if (lg.R.nprim == 0 && lg.P.nprim == 0) continue;
    Gemm p;
    p.tag = "w_grad";
    p.M = int(lg.m); p.N = int(lg.n); p.K = int(T); p.dtype = dt;
    p.A = dya[i]; p.a_m = 1; p.a_k = ldya[i];
    p.B = xa[i]; p.b_n = 1; p.b_k = ldxa[i];
    p.outF = b.D; p.of_m = lg.ldn;
    p.atomic = true;
    gs.push_back(p);
  }
  if (gs.empty()) return POET_OK;
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  // D_f[i][j] = D[R.perm[i]][P.perm[j]] in the storage type, every layer in one launch
  if (dt == POET_BF16) {
    std::vector<FrameItem> fr;
    for (WBwd &b : v) {
      if (b.lg.R.nprim == 0 && b.lg.P.nprim == 0) continue;
      fr.push_back(FrameItem{b.D, b.lg.ldn, b.L->R.perm, b.lg.m, int(b.lg.n), b.L->P.perm, b.Df, b.lg.ldn});
    }
    POET_TRY(frame_many(fr, st));
  } else {
    std::vector<RowPermute> fr;
    for (WBwd &b : v) {
      if (b.lg.R.nprim == 0 && b.lg.P.nprim == 0) continue;
      RowPermute r;
      r.src1 = b.D; r.ld1 = b.lg.ldn;
      r.src_rowmap = b.L->R.perm;
      r.rows = b.lg.m; r.d = int(b.lg.n);
      r.perm = b.L->P.perm;
      r.dst = b.Df; r.ldd = b.lg.ldn;
      fr.push_back(r);
    }
    POET_TRY(permute_many(POET_F32, fr, st, "frame"));
  }
  // G_R[j] = D_f[rows j] F[rows j]^T,  G_P[j] = H[:, cols j]^T D_f[:, cols j]
  // (the engine splits K only for launches of less than two waves)
  gs.clear();
  for (WBwd &b : v) {
    const LayerGeom &lg = b.lg;
    const SideGeom &gR = lg.R, &gP = lg.P;
    const WeightSaved ly = weight_saved(lg, T);
    const char *W0f = static_cast<const char *>(b.L->W0f);
    if (gR.nprim > 0) {  // G_R[j] = D_f[rows j] F[rows j]^T  (F = W0f when P has no primitives)
      Gemm p;
      p.tag = "blk_grad";
      p.M = gR.size; p.N = gR.size; p.K = int(lg.n); p.batch = gR.nprim; p.dtype = dt;
      p.A = b.Df; p.a_m = lg.ldn; p.a_k = 1; p.a_b = int64_t(gR.size) * lg.ldn;
      p.B = gP.nprim > 0 ? static_cast<const void *>(b.sv + ly.F) : W0f;
      p.b_n = lg.ldn; p.b_k = 1; p.b_b = int64_t(gR.size) * lg.ldn;
      p.outF = b.GR; p.of_m = gR.ld; p.of_b = gR.blk_elems();
      p.atomic = true;
      gs.push_back(p);
    }
    if (gP.nprim > 0) {  // G_P[j] = H[:, cols j]^T D_f[:, cols j]  (H = W0f when R has no primitives)
      Gemm p;
      p.small = SMALL_GRAD;  // the sum runs over the rows
      p.tag = "blk_grad";
      p.M = gP.size; p.N = gP.size; p.K = int(lg.m); p.batch = gP.nprim; p.dtype = dt;
      p.A = gR.nprim > 0 ? static_cast<const void *>(b.sv + ly.H) : W0f;
      p.a_m = 1; p.a_k = lg.ldn; p.a_b = gP.size;
      p.B = b.Df; p.b_n = 1; p.b_k = lg.ldn; p.b_b = gP.size;
      p.outF = b.GP; p.of_m = gP.ld; p.of_b = gP.blk_elems();
      p.atomic = true;
      gs.push_back(p);
    }
  }
  return gemm_run_many(gs.data(), int(gs.size()), st);
}

}  // namespace

// Token plan forward (the primitives act on the activations); x and y rows
// ldx and ldy elements apart.
static poet_status forward_token(const poet_layer *L, const LayerGeom &lg, const void *x, int64_t ldx, int64_t T,
                                 void *y, int64_t ldy, void *saved, char *wb, const WsLayout &w, cudaStream_t st) {
  const int dt = lg.dtype;
  const size_t es = esize(dt);
  char *sv = static_cast<char *>(saved);
  void *xf = sv;
  void *vf = sv + align256(size_t(T) * lg.ldn * es);
  void *uf = wb + w.act1;
  void *yf = wb + w.act2;
  const SideGeom &gR = lg.R, &gP = lg.P;

  // a2: gather x into the P frame; the identity tail goes straight to uf
  const bool tailP = gP.nprim > 0 && gP.covered < lg.n;
  POET_TRY(gather_cols(dt, x, ldx, nullptr, T, int(lg.n), L->P.perm, xf, lg.ldn, tailP ? uf : nullptr, lg.ldn,
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
  return scatter_cols(dt, ysrc, lg.ldm, vf, lg.ldm, gR.covered, T, int(lg.m), L->R.perm, y, ldy, nullptr, st);
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
  if (plan == POET_PLAN_WEIGHT) {
    std::vector<WFwd> one{WFwd{L, lg, x, lg.n, y, lg.m, static_cast<char *>(saved), static_cast<char *>(ws) + w.Z}};
    return forward_weight_many(one, T, st);
  }
  return forward_token(L, lg, x, lg.n, T, y, lg.m, saved, static_cast<char *>(ws), w, st);
}

// Token plan backward a5..a7 (dx and the per-primitive gradients); dy and dx
// rows lddy and lddx elements apart.
static poet_status backward_token(const poet_layer *L, const LayerGeom &lg, char *wb, const WsLayout &w,
                                  const void *saved, const void *dy, int64_t lddy, int64_t T, void *dx, int64_t lddx,
                                  float *GR, float *GP, cudaStream_t st) {
  const int dt = lg.dtype;
  const size_t es = esize(dt);
  const SideGeom &gR = lg.R, &gP = lg.P;
  const char *sv = static_cast<const char *>(saved);
  const void *xf = sv;
  const void *vf = sv + align256(size_t(T) * lg.ldn * es);
  void *dyf = wb + w.act1, *dvf = wb + w.act2, *duf = wb + w.act3, *dxf = wb + w.act1;

  // a5: gather dy into the R frame (tail straight to dvf), dv = R^T dy, G_R
  const bool tailR = gR.nprim > 0 && gR.covered < lg.m;
  POET_TRY(gather_cols(dt, dy, lddy, nullptr, T, int(lg.m), L->R.perm, dyf, lg.ldm, tailR ? dvf : nullptr, lg.ldm,
                       gR.covered, st));
  const void *dv = dyf;
  if (gR.nprim > 0) {
    POET_TRY(gemm_run(blockdiag(gR, dt, T, dyf, lg.ldm, state_R(&L->R, gR, dt), true, dvf, lg.ldm), st));
    dv = dvf;
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
    POET_TRY(gemm_run(blockgrad(gP, dt, T, duf, xf, lg.ldn, GP), st));
    POET_TRY(gemm_run(blockdiag(gP, dt, T, duf, lg.ldn, state_R(&L->P, gP, dt), true, dxf, lg.ldn), st));
    dxsrc = dxf;
  }
  POET_TRY(scatter_cols(dt, dxsrc, lg.ldn, duf, lg.ldn, gP.covered, T, int(lg.n), L->P.perm, dx, lddx, nullptr, st));
  return POET_OK;
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
    std::vector<WBwd> one{WBwd{L, lg, x, lg.n, static_cast<const char *>(saved), dy, lg.m, dx, lg.n, GR, GP,
                               wb + w.act1, reinterpret_cast<float *>(wb + w.D),
                               lg.dtype == POET_BF16 ? static_cast<void *>(wb + w.Z) : static_cast<void *>(wb + w.D2)}};
    return backward_weight_many(one, T, st);
  }
  if (T > 0) {
    POET_REQUIRE(dy && dx && aligned_elem(dy, dt) && aligned_elem(dx, dt), "backward: dy/dx NULL or misaligned");
    POET_REQUIRE(saved && aligned256(saved), "backward: saved NULL or not 256-byte aligned");
    POET_TRY(backward_token(L, lg, wb, w, saved, dy, lg.m, T, dx, lg.n, GR, GP, st));
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

// Workspace of the grouped calls.  Token-plan layers run one after another,
// each with its single-layer workspace at offset 0; every weight-plan layer
// has a region of its own after that: D (float m x ldn), D_f (m x ldn in the
// storage type; the forward keeps E_f there) and, when dy's rows are not
// 16-byte aligned, a re-strided copy of dy (T x ldm).
struct ManyLayout {
  std::vector<int> plan;
  std::vector<size_t> region;   // weight-plan layers: offset of the layer's region
  std::vector<char> dy_copy;    // weight-plan layers: the region holds a re-strided dy
  size_t D_bytes(const LayerGeom &lg) const { return align256(size_t(lg.m) * lg.ldn * 4); }
  size_t Df_bytes(const LayerGeom &lg) const { return align256(size_t(lg.m) * lg.ldn * esize(lg.dtype)); }
  size_t bytes = 0;
};

// dy_copies: reserve re-strided dy copies (the backward); the forward never reads dy.
static ManyLayout many_layout(const std::vector<LayerGeom> &geoms, int64_t T, const int64_t *lddy,
                              bool dy_copies = true) {
  ManyLayout M;
  const size_t n = geoms.size();
  M.plan.resize(n);
  M.region.assign(n, 0);
  M.dy_copy.assign(n, 0);
  size_t token = 0;
  for (size_t i = 0; i < n; ++i) {
    M.plan[i] = resolve_plan(geoms[i], T);
    if (M.plan[i] == POET_PLAN_TOKEN) {
      const size_t b = ws_layout(geoms[i], T, POET_PLAN_TOKEN).bytes;
      if (b > token) token = b;
    }
  }
  size_t off = align256(token);
  for (size_t i = 0; i < n; ++i) {
    if (M.plan[i] != POET_PLAN_WEIGHT) continue;
    const LayerGeom &lg = geoms[i];
    const int64_t ld = lddy ? lddy[i] : lg.m;
    M.region[i] = off;
    off += M.D_bytes(lg) + M.Df_bytes(lg);
    if (dy_copies && (ld * int64_t(esize(lg.dtype))) % 16 != 0) {
      M.dy_copy[i] = 1;
      off += align256(size_t(T) * lg.ldm * esize(lg.dtype));
    }
  }
  M.bytes = off;
  return M;
}

// Validation shared by the grouped calls: every layer complete and of one
// element type, T in range, row strides at least the rows' widths.
static poet_status check_many(const char *fn, const poet_layer *layers, int32_t count, int64_t T,
                              std::vector<LayerGeom> *geoms) {
  POET_REQUIRE(count >= 0 && (count == 0 || layers), "%s: bad layer list", fn);
  POET_REQUIRE(T >= 0 && T <= (int64_t(1) << 31) - 1, "%s: T=%lld out of range", fn, (long long)T);
  geoms->resize(count);
  for (int i = 0; i < count; ++i) {
    poet_status st = check_layer(&layers[i], &(*geoms)[i], true);
    if (st != POET_OK) return st;
    POET_REQUIRE(layers[i].dtype == layers[0].dtype, "%s: layer %d has another element type than layer 0", fn, i);
  }
  return POET_OK;
}

static poet_status check_rows(const char *fn, const char *what, int i, const void *p, int64_t ld, int64_t width,
                              int dtype) {
  POET_REQUIRE(p && aligned_elem(p, dtype), "%s: %s[%d] NULL or misaligned", fn, what, i);
  POET_REQUIRE(ld >= width, "%s: row stride of %s[%d] (%lld) below its width %lld", fn, what, i, (long long)ld,
               (long long)width);
  return POET_OK;
}

size_t poet_block_grad_bytes(const poet_side *side) {
  SideGeom g;
  if (!side_geom(side, &g)) return 0;
  return size_t(g.all_elems()) * 4;
}

size_t poet_many_workspace_bytes(const poet_layer *layers, int32_t count, int64_t T, const int64_t *lddy) {
  if (count < 0 || (count > 0 && !layers) || T < 0) return 0;
  std::vector<LayerGeom> geoms(count);
  for (int i = 0; i < count; ++i)
    if (!shape_geom(&layers[i], &geoms[i])) return 0;
  return many_layout(geoms, T, lddy).bytes;
}

poet_status poet_forward_many(const poet_layer *layers, int32_t count, const void *const *x, const int64_t *ldx,
                              int64_t T, void *const *y, const int64_t *ldy, void *const *saved, void *ws,
                              size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_forward_many");
  clear_error();
  std::vector<LayerGeom> geoms;
  POET_TRY(check_many("poet_forward_many", layers, count, T, &geoms));
  if (count == 0 || T == 0) return POET_OK;
  POET_REQUIRE(x && y && saved, "poet_forward_many: x, y and saved lists must not be NULL");
  for (int i = 0; i < count; ++i) {
    const LayerGeom &lg = geoms[i];
    POET_TRY(check_rows("poet_forward_many", "x", i, x[i], ldx ? ldx[i] : lg.n, lg.n, lg.dtype));
    POET_TRY(check_rows("poet_forward_many", "y", i, y[i], ldy ? ldy[i] : lg.m, lg.m, lg.dtype));
    POET_REQUIRE(saved[i] && aligned256(saved[i]), "poet_forward_many: saved[%d] NULL or not 256-byte aligned", i);
  }
  const ManyLayout M = many_layout(geoms, T, nullptr, false);
  if (!ws || ws_bytes < M.bytes || !aligned256(ws)) {
    set_error("poet_forward_many: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, M.bytes);
    return POET_ENOMEM_WS;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *wb = static_cast<char *>(ws);
  std::vector<WFwd> wl;
  for (int i = 0; i < count; ++i) {
    if (M.plan[i] != POET_PLAN_WEIGHT) continue;
    const LayerGeom &lg = geoms[i];
    wl.push_back(WFwd{&layers[i], lg, x[i], ldx ? ldx[i] : lg.n, y[i], ldy ? ldy[i] : lg.m,
                      static_cast<char *>(saved[i]), wb + M.region[i] + M.D_bytes(lg)});
  }
  POET_TRY(forward_weight_many(wl, T, st));
  for (int i = 0; i < count; ++i) {  // token-plan layers, one after another
    if (M.plan[i] != POET_PLAN_TOKEN) continue;
    const LayerGeom &lg = geoms[i];
    POET_TRY(forward_token(&layers[i], lg, x[i], ldx ? ldx[i] : lg.n, T, y[i], ldy ? ldy[i] : lg.m, saved[i], wb,
                           ws_layout(lg, T, POET_PLAN_TOKEN), st));
  }
  return POET_OK;
}

poet_status poet_backward_blocks_many(const poet_layer *layers, int32_t count, const void *const *x,
                                      const int64_t *ldx, const void *const *saved, const void *const *dy,
                                      const int64_t *lddy, int64_t T, void *const *dx, const int64_t *lddx,
                                      float *const *G_R, float *const *G_P, void *ws, size_t ws_bytes,
                                      poet_stream stream) {
  CallRange nvtx_range("poet_backward_blocks_many");
  clear_error();
  std::vector<LayerGeom> geoms;
  POET_TRY(check_many("poet_backward_blocks_many", layers, count, T, &geoms));
  if (count == 0) return POET_OK;
  POET_REQUIRE(G_R && G_P, "poet_backward_blocks_many: G_R and G_P lists must not be NULL");
  for (int i = 0; i < count; ++i) {
    POET_REQUIRE(geoms[i].R.nprim == 0 || (G_R[i] && (reinterpret_cast<uintptr_t>(G_R[i]) & 15) == 0),
                 "poet_backward_blocks_many: G_R[%d] NULL or not 16-byte aligned", i);
    POET_REQUIRE(geoms[i].P.nprim == 0 || (G_P[i] && (reinterpret_cast<uintptr_t>(G_P[i]) & 15) == 0),
                 "poet_backward_blocks_many: G_P[%d] NULL or not 16-byte aligned", i);
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {  // no tokens: every per-primitive gradient is zero
    std::vector<std::pair<float *, int64_t>> zero;
    for (int i = 0; i < count; ++i) {
      if (geoms[i].R.nprim > 0) zero.emplace_back(G_R[i], geoms[i].R.all_elems());
      if (geoms[i].P.nprim > 0) zero.emplace_back(G_P[i], geoms[i].P.all_elems());
    }
    return zero_many(zero, st);
  }
  POET_REQUIRE(x && saved && dy && dx, "poet_backward_blocks_many: x, saved, dy and dx lists must not be NULL");
  const ManyLayout M = many_layout(geoms, T, lddy);
  for (int i = 0; i < count; ++i) {
    const LayerGeom &lg = geoms[i];
    const int64_t ld_dy = lddy ? lddy[i] : lg.m;
    POET_TRY(check_rows("poet_backward_blocks_many", "dy", i, dy[i], ld_dy, lg.m, lg.dtype));
    POET_TRY(check_rows("poet_backward_blocks_many", "dx", i, dx[i], lddx ? lddx[i] : lg.n, lg.n, lg.dtype));
    POET_REQUIRE(saved[i] && aligned256(saved[i]), "poet_backward_blocks_many: saved[%d] NULL or not 256-byte aligned",
                 i);
    if (M.plan[i] == POET_PLAN_WEIGHT) {
      POET_TRY(check_rows("poet_backward_blocks_many", "x", i, x[i], ldx ? ldx[i] : lg.n, lg.n, lg.dtype));
      POET_REQUIRE(M.dy_copy[i] || rows16(dy[i], ld_dy, lg.dtype),
                   "poet_backward_blocks_many: dy[%d] must start on a 16-byte boundary (its row stride is)", i);
    }
  }
  if (!ws || ws_bytes < M.bytes || !aligned256(ws)) {
    set_error("poet_backward_blocks_many: workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, M.bytes);
    return POET_ENOMEM_WS;
  }
  char *wb = static_cast<char *>(ws);
  std::vector<WBwd> wl;
  for (int i = 0; i < count; ++i) {
    if (M.plan[i] != POET_PLAN_WEIGHT) continue;
    const LayerGeom &lg = geoms[i];
    char *r = wb + M.region[i];
    wl.push_back(WBwd{&layers[i], lg, x[i], ldx ? ldx[i] : lg.n, static_cast<const char *>(saved[i]), dy[i],
                      lddy ? lddy[i] : lg.m, dx[i], lddx ? lddx[i] : lg.n, G_R[i], G_P[i],
                      r + M.D_bytes(lg) + M.Df_bytes(lg), reinterpret_cast<float *>(r), r + M.D_bytes(lg)});
  }
  POET_TRY(backward_weight_many(wl, T, st));
  for (int i = 0; i < count; ++i) {  // token-plan layers, one after another
    if (M.plan[i] != POET_PLAN_TOKEN) continue;
    const LayerGeom &lg = geoms[i];
    POET_TRY(backward_token(&layers[i], lg, wb, ws_layout(lg, T, POET_PLAN_TOKEN), saved[i], dy[i],
                            lddy ? lddy[i] : lg.m, T, dx[i], lddx ? lddx[i] : lg.n, G_R[i], G_P[i], st));
  }
  return POET_OK;
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

static poet_status grad_many_impl(const char *fn, const poet_side *sides, const float *const *G,
                                  float *const *dtheta, int32_t count, int32_t dtype, void *ws, size_t ws_bytes,
                                  cudaStream_t st, const AdamW *adam, float *const *m, float *const *v) {
  POET_REQUIRE(count >= 0 && (count == 0 || (sides && G && (dtheta || adam))), "%s: bad lists", fn);
  POET_REQUIRE(!adam || count == 0 || (m && v), "%s: moment lists must not be NULL", fn);
  POET_REQUIRE(dtype == POET_F32 || dtype == POET_BF16, "%s: bad dtype %d", fn, dtype);
  std::vector<SideGeom> geoms(count);
  std::vector<void *> scratch(count, nullptr);
  size_t off = 0;
  auto ok4 = [](const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 3) == 0; };
  for (int i = 0; i < count; ++i) {
    POET_REQUIRE(side_geom(&sides[i], &geoms[i]), "%s: side %d malformed", fn, i);
    if (geoms[i].nprim == 0 || geoms[i].size < 2) continue;
    POET_REQUIRE(sides[i].state && aligned256(sides[i].state) && G[i] && (reinterpret_cast<uintptr_t>(G[i]) & 15) == 0,
                 "%s: side %d state/G NULL or misaligned", fn, i);
    if (adam) {
      POET_REQUIRE(ok4(sides[i].theta) && ok4(m[i]) && ok4(v[i]) && (!dtheta || !dtheta[i] || ok4(dtheta[i])),
                   "%s: side %d theta/m/v NULL or misaligned", fn, i);
    } else {
      POET_REQUIRE(dtheta[i] != nullptr, "%s: side %d dtheta is NULL", fn, i);
    }
    scratch[i] = static_cast<char *>(ws) + off;
    off += align256(cnp_many_scratch_bytes(geoms[i], dtype));
  }
  if (off > 0 && (!ws || ws_bytes < off || !aligned256(ws))) {
    set_error("%s: workspace %zu bytes, need %zu (256-byte aligned)", fn, ws_bytes, off);
    return POET_ENOMEM_WS;
  }
  return cnp_backward_many(sides, geoms.data(), count, dtype, G, dtheta, scratch.data(), st, adam, m, v);
}

poet_status poet_cayley_neumann_grad_many(const poet_side *sides, const float *const *G, float *const *dtheta,
                                          int32_t count, int32_t dtype, void *ws, size_t ws_bytes,
                                          poet_stream stream) {
  CallRange nvtx_range("poet_cayley_neumann_grad_many");
  clear_error();
  return grad_many_impl("poet_cayley_neumann_grad_many", sides, G, dtheta, count, dtype, ws, ws_bytes,
                        reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr);
}

static poet_status check_adamw(const char *fn, float lr, float beta1, float beta2, float eps, float weight_decay,
                               int32_t step) {
  POET_REQUIRE(step >= 1, "%s: step=%d < 1", fn, step);
  POET_REQUIRE(std::isfinite(lr) && lr >= 0.f && std::isfinite(weight_decay) && weight_decay >= 0.f,
               "%s: lr and weight_decay must be finite and >= 0", fn);
  POET_REQUIRE(beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f, "%s: betas outside [0, 1)", fn);
  POET_REQUIRE(std::isfinite(eps) && eps > 0.f, "%s: eps must be > 0", fn);
  return POET_OK;
}

poet_status poet_cayley_neumann_grad_many_adamw(const poet_side *sides, const float *const *G, float *const *m,
                                                float *const *v, float *const *dtheta, int32_t count,
                                                int32_t dtype, const poet_adamw_hparams *h, void *ws,
                                                size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_cayley_neumann_grad_many_adamw");
  clear_error();
  const char *fn = "poet_cayley_neumann_grad_many_adamw";
  POET_REQUIRE(h != nullptr, "%s: hyperparameters are NULL", fn);
  POET_TRY(check_adamw(fn, h->lr, h->beta1, h->beta2, h->eps, h->weight_decay, h->step));
  const AdamW a = adamw_of(h->lr, h->beta1, h->beta2, h->eps, h->weight_decay, h->step);
  return grad_many_impl(fn, sides, G, dtheta, count, dtype, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream),
                        &a, m, v);
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

poet_status poet_merge_reset_moments(poet_layer *L, float *m_R, float *v_R, float *m_P, float *v_P, void *ws,
                                     size_t ws_bytes, poet_stream stream) {
  CallRange nvtx_range("poet_merge_reset_moments");
  clear_error();
  LayerGeom lg;
  POET_TRY(check_layer(L, &lg, true));
  const int64_t nR = int64_t(lg.R.nprim) * lg.R.packed_per(), nP = int64_t(lg.P.nprim) * lg.P.packed_per();
  auto ok4 = [](const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 3) == 0; };
  POET_REQUIRE(nR == 0 || (ok4(m_R) && ok4(v_R)), "poet_merge_reset_moments: R moments NULL or misaligned");
  POET_REQUIRE(nP == 0 || (ok4(m_P) && ok4(v_P)), "poet_merge_reset_moments: P moments NULL or misaligned");
  POET_TRY(poet_merge(L, ws, ws_bytes, stream));
  std::vector<std::pair<float *, int64_t>> zero;
  if (nR > 0) { zero.emplace_back(m_R, nR); zero.emplace_back(v_R, nR); }
  if (nP > 0) { zero.emplace_back(m_P, nP); zero.emplace_back(v_P, nP); }
  return zero_many(zero, reinterpret_cast<cudaStream_t>(stream));
}

size_t poet_workspace_size(const poet_layer *L, int64_t T) { return poet_workspace_bytes(L, T); }

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
  POET_TRY(check_adamw("poet_adamw_step", lr, beta1, beta2, eps, weight_decay, step));
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
