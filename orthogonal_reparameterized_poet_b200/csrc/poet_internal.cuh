// Internal declarations of libpoet (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include <utility>
#include <vector>

#include "poet.h"

namespace poet {

using bf16 = __nv_bfloat16;

// ------------------------------------------------------------------ errors

void set_error(const char *fmt, ...);
void clear_error();

#define POET_REQUIRE(cond, ...)                 \
  do {                                          \
    if (!(cond)) {                              \
      ::poet::set_error(__VA_ARGS__);           \
      return POET_EINVAL;                       \
    }                                           \
  } while (0)

#define POET_CUDA_TRY(call)                                                         \
  do {                                                                              \
    cudaError_t e_ = (call);                                                        \
    if (e_ != cudaSuccess) {                                                        \
      ::poet::set_error("%s failed: %s", #call, cudaGetErrorString(e_));            \
      return POET_ECUDA;                                                            \
    }                                                                               \
  } while (0)

#define POET_TRY(expr)                 \
  do {                                 \
    poet_status s_ = (expr);           \
    if (s_ != POET_OK) return s_;      \
  } while (0)

// Checks the last launch.
poet_status launch_status(const char *what);

// Device status word: kernels with bounded waits OR bits into it.
enum : unsigned { ERR_TIMEOUT = 1u, ERR_BOUNDS = 2u };
unsigned *device_errword();   // device address for the current device (nullptr on failure)

// Multiprocessor count of the current device (cached per device).
int num_sms();

// ------------------------------------------------------------------ accounting
//
// Every kernel launch of the library is counted.  When tracing is on, a
// TraceScope records a CUDA event pair on the launch stream around the work
// it encloses, tagged with a kind and the work's algorithmic flops and bytes.
void count_launch();
bool trace_on();
struct TraceScope {
  TraceScope(const char *kind, double flop, double bytes, cudaStream_t st);
  ~TraceScope();
  int slot = -1;
  cudaStream_t st = nullptr;
};

// An NVTX range around one ABI call on the calling thread (the kernels it
// launches carry the call's name in a profiler's NVTX filters; TraceScope adds
// a nested range per kernel kind).  No-ops unless a profiler is attached.
struct CallRange {
  explicit CallRange(const char *name);
  ~CallRange();
  CallRange(const CallRange &) = delete;
  CallRange &operator=(const CallRange &) = delete;
};

// ------------------------------------------------------------------ geometry

inline size_t esize(int dtype) { return dtype == POET_BF16 ? 2 : 4; }
inline int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// One side's primitives: nprim primitives of size `size`, stored with row
// stride `ld` (size rounded up to 8 so that rows are 16-byte aligned);
// covered = nprim * size frame indices are acted on, the rest is identity.
struct SideGeom {
  int nprim = 0, size = 0, ld = 0, covered = 0, k = 0;
  int64_t blk_elems() const { return int64_t(ld) * ld; }          // one primitive
  int64_t all_elems() const { return blk_elems() * nprim; }       // one side
  int64_t packed_per() const { return int64_t(size) * (size - 1) / 2; }
};
bool side_geom(const poet_side *s, SideGeom *g);   // false if the side is malformed

// Frame row stride of a dimension (elements): rows start on 128-byte lines.
inline int64_t frame_ld(int64_t dim) { return round_up(dim, 64); }

// Layout of a side's state buffer (byte offsets).
struct StateLayout {
  size_t R = 0, Q = 0, S1 = 0, bytes = 0;   // S_l at S1 + (l-1)*term
  size_t term = 0;                          // bytes of one nprim x ld x ld array
};
StateLayout state_layout(const SideGeom &g, int dtype);

// ------------------------------------------------------------------ GEMM engine
//
//   v(b,i,j) = alpha * sum_l A(b,i,l) * B(b,j,l)  (+ beta * Add(b,i,j)) (+ beta2 * Add2(b,i,j))
//              (+ diag if i == j)
//   A(b,i,l) = A[b*a_b + i*a_m + l*a_k], B(b,j,l) = B[b*b_b + j*b_n + l*b_k]
// then v is stored to outF (float) and/or outD (element type `dtype`).  With
// `atomic` (outF only, no addend or diagonal) the engine may split K: it then
// zeroes outF and adds the partial sums into it; outF's prior content is never
// used.
struct Gemm {
  int M = 0, N = 0, K = 0, batch = 1;
  int dtype = POET_F32;                       // type of A, B, outD
  const void *A = nullptr; int64_t a_m = 0, a_k = 0, a_b = 0;
  const void *B = nullptr; int64_t b_n = 0, b_k = 0, b_b = 0;
  float alpha = 1.f;
  const void *add = nullptr; int add_dtype = POET_F32; int64_t add_m = 0, add_b = 0; float beta = 0.f;
  const void *add2 = nullptr; int add2_dtype = POET_F32; int64_t add2_m = 0, add2_b = 0; float beta2 = 0.f;
  float diag = 0.f;
  float *outF = nullptr; int64_t of_m = 0, of_b = 0;
  void *outD = nullptr; int64_t od_m = 0, od_b = 0;
  bool atomic = false;
  const char *tag = "gemm";                   // kind for tracing
  // A block-diagonal product of one side's primitives, which primitives of
  // size <= 32 run on the small-block kernels instead:
  //   SMALL_RIGHT: out[r][j*s + a] = sum_c A[r][j*s + c] B_j(a, c)  (M = rows, N = K = s)
  //   SMALL_LEFT:  out[j*s + a][k] = sum_c A_j[a][c] B[j*s + c][k]  (M = K = s, N = columns)
  //   SMALL_GRAD:  outF_j[a][c] += sum_r A[r][j*s + a] B[r][j*s + c] (M = N = s, K = rows)
  int small = 0;
};
enum { SMALL_RIGHT = 1, SMALL_LEFT = 2, SMALL_GRAD = 3 };

poet_status gemm_run(const Gemm &g, cudaStream_t st);       // picks the engine
// out[b*ldb + r*ldm + c] = 0 for b < batch, r < M, c < N (an output about to
// receive reductions).
poet_status zero_output(float *out, int M, int N, int64_t ldm, int batch, int64_t ldb, cudaStream_t st);
struct ZeroRegion {
  float *out; int M, N; int64_t ldm; int batch; int64_t ldb;
};
poet_status zero_outputs(const std::vector<ZeroRegion> &v, cudaStream_t st);  // many regions, one launch
poet_status gemm_simt(const Gemm &g, cudaStream_t st);      // CUDA-core FMA engine
bool gemm_tc_supported(const Gemm &g);                      // tcgen05 engine can take g
poet_status gemm_tc(const Gemm &g, cudaStream_t st);        // tcgen05 engine
// Many independent problems: grouped tcgen05 launches where possible, the rest
// on the CUDA-core engine.  gemm_run_many adds tracing around it.
poet_status gemm_tc_many(const Gemm *gs, int count, cudaStream_t st);
poet_status gemm_run_many(const Gemm *gs, int count, cudaStream_t st);
// One CTA whose bounded wait on a barrier nothing arrives on runs out (tests failure detection).
poet_status selftest_bounded_wait(uint32_t timeout_us, cudaStream_t st);
bool gemm_tc_enabled();

// Small-block kernels (primitive size <= 32, CUDA cores; see smallb.cu).
bool smallb_supported(int size);
poet_status smallb_right(int dtype, const void *X, int64_t ldx, int64_t rows, const void *M, int64_t ldm,
                         int64_t bstride, int nprim, int s, bool trans, void *out, int64_t ldo, cudaStream_t st,
                         const char *kind);
poet_status smallb_left(int dtype, const void *X, int64_t ldx, int64_t cols, const void *M, int64_t ldm,
                        int64_t bstride, int nprim, int s, bool trans, void *out, int64_t ldo, cudaStream_t st,
                        const char *kind);
poet_status smallb_grad(int dtype, const void *D, const void *V, int64_t ld, int64_t rows, int nprim, int s, float *G,
                        int64_t ldg, int64_t gstride, cudaStream_t st);
// Runs g on the small-block kernels if it is a marked block product they serve (*done = true).
poet_status smallb_dispatch(const Gemm &g, cudaStream_t st, bool *done);

// ------------------------------------------------------------------ data movement

// dst[r][i] = src[srcrow(r)][perm[i]] for i < d, r < rows; srcrow(r) = rowmap ? rowmap[r] : r.
// If dst2 != nullptr, columns i >= split are also written to dst2.  Rows of
// dst/dst2 are zero-padded up to round_up(d, 8).
poet_status gather_cols(int dtype, const void *src, int64_t ld_src, const int32_t *rowmap,
                        int64_t rows, int d, const int32_t *perm,
                        void *dst, int64_t ld_dst, void *dst2, int64_t ld_dst2, int split,
                        cudaStream_t st, const char *kind = "gather");

// dst[r][j] = src[r][j] for j < d: rows re-strided to 16-byte aligned rows.
poet_status copy_rows(int dtype, const void *src, int64_t ld_src, int64_t rows, int d, void *dst, int64_t ld_dst,
                      cudaStream_t st);

// out[a][c] = bf16(D[rowmap[a]][perm[c]]) for a < rows, c < d (out: bf16).
poet_status frame_f32_to_bf16(const float *D, int64_t ldD, const int32_t *rowmap, int64_t rows, int d,
                              const int32_t *perm, void *out, int64_t ld_out, cudaStream_t st);

// dst[dstrow(r)][perm[i]] = (i < split ? src1[r][i] : src2[r][i]); dstrow(r) = rowmap ? rowmap[r] : r.
poet_status scatter_cols(int dtype, const void *src1, int64_t ld1, const void *src2, int64_t ld2,
                         int split, int64_t rows, int d, const int32_t *perm,
                         void *dst, int64_t ld_dst, const int32_t *rowmap, cudaStream_t st,
                         const char *kind = "scatter");

// Many row permutations in one launch (weight-sized matrices of several
// layers).  Output row r of item i: dst[dstrow(r)][j] = src(r)[map[j]] for
// j < d, where src(r) = row srcrow(r) of src1 for columns < split and of src2
// for columns >= split (src2 = nullptr: src1 only), map = perm (inverse = 0),
// perm^-1 (inverse = 1) or the identity (perm = nullptr), and srcrow/dstrow
// are the row maps (nullptr: r) whose entries must lie in [0, map_rows)
// (map_rows = 0: [0, rows)).  Rows may start at any element boundary.
struct RowPermute {
  const void *src1 = nullptr; int64_t ld1 = 0;
  const void *src2 = nullptr; int64_t ld2 = 0; int split = 0;
  const int32_t *src_rowmap = nullptr;
  int64_t rows = 0; int d = 0;
  const int32_t *perm = nullptr; int inverse = 0;
  void *dst = nullptr; int64_t ldd = 0;
  const int32_t *dst_rowmap = nullptr;
  int64_t map_rows = 0;
};
poet_status permute_many(int dtype, const std::vector<RowPermute> &v, cudaStream_t st, const char *kind);

// out[a][c] = bf16(D[rowmap[a]][perm[c]]) for several matrices in one launch.
struct FrameItem {
  const float *D; int64_t ldD;
  const int32_t *rowmap; int64_t rows; int d;
  const int32_t *perm;
  void *out; int64_t ld_out;
};
poet_status frame_many(const std::vector<FrameItem> &v, cudaStream_t st);

// Zero several float buffers in one launch.
poet_status zero_many(const std::vector<std::pair<float *, int64_t>> &v, cudaStream_t st);

// ------------------------------------------------------------------ optimizer step

// AdamW hyperparameters of one step with the bias corrections 1 - beta^step.
struct AdamW {
  float lr, beta1, beta2, eps, wd;
  float bc1, bc2;
};
AdamW adamw_of(float lr, float beta1, float beta2, float eps, float weight_decay, int32_t step);

// One parameter's AdamW update (decoupled weight decay, bias-corrected moments).
// Every operation is an explicitly rounded single-precision intrinsic, so the
// compiler contracts none of them into fused multiply-adds and every kernel
// that calls this function performs exactly the same arithmetic.
__device__ __forceinline__ void adamw_one(float &theta, float g, float &m, float &v, const AdamW &h) {
  m = __fadd_rn(__fmul_rn(h.beta1, m), __fmul_rn(__fsub_rn(1.f, h.beta1), g));
  v = __fadd_rn(__fmul_rn(h.beta2, v), __fmul_rn(__fmul_rn(__fsub_rn(1.f, h.beta2), g), g));
  const float m_hat = __fdiv_rn(m, h.bc1);
  const float v_hat = __fdiv_rn(v, h.bc2);
  const float step = __fadd_rn(__fdiv_rn(m_hat, __fadd_rn(__fsqrt_rn(v_hat), h.eps)), __fmul_rn(h.wd, theta));
  theta = __fsub_rn(theta, __fmul_rn(h.lr, step));
}

// One AdamW step on n float parameters in place (see poet_adamw_step).
poet_status adamw_step(float *theta, const float *grad, float *m, float *v, int64_t n, float lr, float beta1,
                       float beta2, float eps, float weight_decay, int32_t step, cudaStream_t st);

// ------------------------------------------------------------------ Cayley-Neumann

poet_status cnp_forward(const poet_side *side, const SideGeom &g, int dtype, cudaStream_t st);
// G: float [nprim][ld][ld]; scratch: cnp_scratch_bytes(g, dtype) bytes.
poet_status cnp_backward(const poet_side *side, const SideGeom &g, int dtype, const float *G,
                         float *dtheta, void *scratch, cudaStream_t st);
size_t cnp_scratch_bytes(const SideGeom &g, int dtype);
// The same for many sides at once; their GEMM steps share grouped launches.
// G[i]: float [nprim][ld][ld]; scratch[i]: cnp_many_scratch_bytes(geoms[i], dtype) bytes each.
poet_status cnp_forward_many(const poet_side *sides, const SideGeom *geoms, int count, int dtype, cudaStream_t st);
// With adam != nullptr the packing also applies that AdamW step to each side's
// theta with moments m[i], v[i] (dtheta[i] may then be nullptr).
poet_status cnp_backward_many(const poet_side *sides, const SideGeom *geoms, int count, int dtype,
                              const float *const *G, float *const *dtheta, void *const *scratch, cudaStream_t st,
                              const AdamW *adam = nullptr, float *const *m = nullptr, float *const *v = nullptr);
size_t cnp_many_scratch_bytes(const SideGeom &g, int dtype);
// out = G (dense [nprim][size][size]) re-laid as [nprim][ld][ld] with zero padding
poet_status pad_blocks(const float *G, const SideGeom &g, float *out, cudaStream_t st);

// ------------------------------------------------------------------ permutations

poet_status draw_perm_dev(uint64_t seed, int32_t layer_id, int32_t side, int32_t epoch,
                          int32_t dim, int32_t *perm, cudaStream_t st);

}  // namespace poet
