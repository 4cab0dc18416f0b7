// One LLaMA block around seven POET linears: the non-linear pieces.
//
// The POET pages train LLaMA models whose linears are POET layers (POET
// summary page, Experimental setup); the block follows the published LLaMA
// design (pre-normalization with RMSNorm, rotary position embeddings, causal
// multi-head attention, SwiGLU feed-forward, residual connections).  Readings
// (the pages fix none of them): RMSNorm gains 1 and untrained, eps inside the
// square root; rotary embedding on interleaved pairs (2i, 2i+1) of each head,
// angle pos * base^(-2i/head_dim), positions counted within each sequence;
// attention scores scaled by 1/sqrt(head_dim) with a causal mask.
//
// Row kernels (RMSNorm, softmax) give one warp to one row and accumulate in
// float; element-wise kernels (rotary, SwiGLU, residual) use 16-byte vectors
// of bf16 where rows allow.  The attention products run on the library's
// GEMM engine (block_api.cu): scores and their gradient in float, the
// probabilities and the score gradient in bf16.
#include "poet_internal.cuh"

namespace poet {
namespace {

constexpr int ROW_WARPS = 8;  // rows per CTA for the row kernels

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

int row_grid(int64_t rows) {
  const int64_t want = (rows + ROW_WARPS - 1) / ROW_WARPS, cap = int64_t(num_sms()) * 16;
  return int(want < 1 ? 1 : (want < cap ? want : cap));
}

// y = x / r, r = sqrt(mean(x^2) + eps) per row (r stored as float).
__global__ void __launch_bounds__(ROW_WARPS * 32) rmsnorm_kernel(const bf16 *__restrict__ x, int64_t ldx,
                                                                 int64_t rows, int d, float eps, bf16 *__restrict__ y,
                                                                 int64_t ldy, float *__restrict__ r) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int64_t row = int64_t(blockIdx.x) * ROW_WARPS + warp; row < rows; row += int64_t(gridDim.x) * ROW_WARPS) {
    const bf16 *xr = x + row * ldx;
    float ss = 0.f;
    for (int c = lane; c < d; c += 32) {
      const float v = __bfloat162float(xr[c]);
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    const float rr = sqrtf(ss / float(d) + eps);
    const float inv = 1.f / rr;
    bf16 *yr = y + row * ldy;
    for (int c = lane; c < d; c += 32) yr[c] = __float2bfloat16_rn(__bfloat162float(xr[c]) * inv);
    if (lane == 0) r[row] = rr;
  }
}

// dx = resid + (g - y * mean(g * y)) / r with g = g0 + g1 + g2 (g1, g2 may be
// null; resid may be null): the gradient through y = x / r(x), with the sum of
// the incoming gradients and the residual branch folded in.
__global__ void __launch_bounds__(ROW_WARPS * 32) rmsnorm_bwd_kernel(
    const bf16 *__restrict__ g0, const bf16 *__restrict__ g1, const bf16 *__restrict__ g2, int64_t ldg,
    const bf16 *__restrict__ y, int64_t ldy, const float *__restrict__ r, const bf16 *__restrict__ resid,
    int64_t ldr, int64_t rows, int d, bf16 *__restrict__ dx, int64_t lddx) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int64_t row = int64_t(blockIdx.x) * ROW_WARPS + warp; row < rows; row += int64_t(gridDim.x) * ROW_WARPS) {
    const int64_t og = row * ldg, oy = row * ldy;
    auto grad = [&](int c) {
      float v = __bfloat162float(g0[og + c]);
      if (g1) v += __bfloat162float(g1[og + c]);
      if (g2) v += __bfloat162float(g2[og + c]);
      return v;
    };
    float dot = 0.f;
    for (int c = lane; c < d; c += 32) dot = fmaf(grad(c), __bfloat162float(y[oy + c]), dot);
    const float mean = warp_sum(dot) / float(d);
    const float inv = 1.f / r[row];
    for (int c = lane; c < d; c += 32) {
      float v = (grad(c) - __bfloat162float(y[oy + c]) * mean) * inv;
      if (resid) v += __bfloat162float(resid[row * ldr + c]);
      dx[row * lddx + c] = __float2bfloat16_rn(v);
    }
  }
}

// Rotate the interleaved pairs (2i, 2i+1) of each head of x in place by
// angle pos * base^(-2i/head_dim) (or minus it: the inverse, and the backward).
// The angle is formed and reduced in double.
__global__ void rope_kernel(bf16 *__restrict__ x, int64_t ldx, int64_t rows, int d, int head_dim, int seq_len,
                            double log_base, int inverse) {
  const int pairs_row = d / 2, half = head_dim / 2;
  const int64_t total = rows * pairs_row;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = e / pairs_row;
    const int pr = int(e % pairs_row);
    const int i = pr % half;  // pair index inside its head
    const int pos = int(row % seq_len);
    const double ang = double(pos) * exp(-2.0 * double(i) / double(head_dim) * log_base);
    double s, c;
    sincos(ang, &s, &c);
    if (inverse) s = -s;
    __nv_bfloat162 *p = reinterpret_cast<__nv_bfloat162 *>(x + row * ldx) + pr;
    const float2 v = __bfloat1622float2(*p);
    *p = __floats2bfloat162_rn(float(v.x * c - v.y * s), float(v.x * s + v.y * c));
  }
}

// P = causal softmax of each row of the float scores (rows of width S; row i
// of every S x S matrix keeps columns j <= i), stored in bf16.
__global__ void __launch_bounds__(ROW_WARPS * 32) causal_softmax_kernel(const float *__restrict__ s, int64_t rows,
                                                                        int S, bf16 *__restrict__ p) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int64_t row = int64_t(blockIdx.x) * ROW_WARPS + warp; row < rows; row += int64_t(gridDim.x) * ROW_WARPS) {
    const int i = int(row % S);  // query position: columns 0..i are kept
    const float *sr = s + row * S;
    float mx = -INFINITY;
    for (int c = lane; c <= i; c += 32) mx = fmaxf(mx, sr[c]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int c = lane; c <= i; c += 32) sum += expf(sr[c] - mx);
    sum = warp_sum(sum);
    const float inv = 1.f / sum;
    bf16 *pr = p + row * S;
    for (int c = lane; c < S; c += 32) pr[c] = __float2bfloat16_rn(c <= i ? expf(sr[c] - mx) * inv : 0.f);
  }
}

// dS = scale * P .* (dP - rowsum(P .* dP)) per row (bf16 out; zero above the diagonal through P).
__global__ void __launch_bounds__(ROW_WARPS * 32) softmax_bwd_kernel(const bf16 *__restrict__ p,
                                                                     const float *__restrict__ dp, int64_t rows, int S,
                                                                     float scale, bf16 *__restrict__ ds) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int64_t row = int64_t(blockIdx.x) * ROW_WARPS + warp; row < rows; row += int64_t(gridDim.x) * ROW_WARPS) {
    const bf16 *pr = p + row * S;
    const float *dr = dp + row * S;
    float dot = 0.f;
    for (int c = lane; c < S; c += 32) dot = fmaf(__bfloat162float(pr[c]), dr[c], dot);
    dot = warp_sum(dot);
    bf16 *o = ds + row * S;
    for (int c = lane; c < S; c += 32) o[c] = __float2bfloat16_rn(scale * __bfloat162float(pr[c]) * (dr[c] - dot));
  }
}

__device__ __forceinline__ float sigmoid(float z) { return 1.f / (1.f + expf(-z)); }

// m = silu(g) * u,  silu(z) = z * sigmoid(z)
__global__ void swiglu_kernel(const bf16 *__restrict__ g, const bf16 *__restrict__ u, int64_t ld, int64_t rows, int d,
                              bf16 *__restrict__ m, int64_t ldm) {
  const int64_t total = rows * d;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = e / d;
    const int c = int(e % d);
    const float gv = __bfloat162float(g[row * ld + c]), uv = __bfloat162float(u[row * ld + c]);
    m[row * ldm + c] = __float2bfloat16_rn(gv * sigmoid(gv) * uv);
  }
}

// dg = dm * u * silu'(g),  du = dm * silu(g),  silu'(z) = sigmoid(z) (1 + z (1 - sigmoid(z)))
__global__ void swiglu_bwd_kernel(const bf16 *__restrict__ dm, int64_t lddm, const bf16 *__restrict__ g,
                                  const bf16 *__restrict__ u, int64_t ld, int64_t rows, int d, bf16 *__restrict__ dg,
                                  bf16 *__restrict__ du, int64_t ldo) {
  const int64_t total = rows * d;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = e / d;
    const int c = int(e % d);
    const float gv = __bfloat162float(g[row * ld + c]), uv = __bfloat162float(u[row * ld + c]);
    const float dmv = __bfloat162float(dm[row * lddm + c]);
    const float sg = sigmoid(gv);
    dg[row * ldo + c] = __float2bfloat16_rn(dmv * uv * sg * (1.f + gv * (1.f - sg)));
    du[row * ldo + c] = __float2bfloat16_rn(dmv * gv * sg);
  }
}

// out = a + b (row-wise, bf16, float add)
__global__ void add_kernel(const bf16 *__restrict__ a, int64_t lda, const bf16 *__restrict__ b, int64_t ldb,
                           int64_t rows, int d, bf16 *__restrict__ out, int64_t ldo) {
  const int64_t total = rows * d;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = e / d;
    const int c = int(e % d);
    out[row * ldo + c] = __float2bfloat16_rn(__bfloat162float(a[row * lda + c]) + __bfloat162float(b[row * ldb + c]));
  }
}

int elem_grid(int64_t n) {
  const int64_t want = (n + 255) / 256, cap = int64_t(num_sms()) * 16;
  return int(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

poet_status block_rmsnorm(const bf16 *x, int64_t ldx, int64_t rows, int d, float eps, bf16 *y, int64_t ldy, float *r,
                          cudaStream_t st) {
  if (rows <= 0) return POET_OK;
  TraceScope ts("norm", 3.0 * double(rows) * d, double(rows) * d * 4.0, st);
  rmsnorm_kernel<<<row_grid(rows), ROW_WARPS * 32, 0, st>>>(x, ldx, rows, d, eps, y, ldy, r);
  count_launch();
  return launch_status("norm");
}

poet_status block_rmsnorm_bwd(const bf16 *g0, const bf16 *g1, const bf16 *g2, int64_t ldg, const bf16 *y, int64_t ldy,
                              const float *r, const bf16 *resid, int64_t ldr, int64_t rows, int d, bf16 *dx,
                              int64_t lddx, cudaStream_t st) {
  if (rows <= 0) return POET_OK;
  const int nin = 1 + (g1 ? 1 : 0) + (g2 ? 1 : 0) + (resid ? 1 : 0);
  TraceScope ts("norm", 6.0 * double(rows) * d, double(rows) * d * 2.0 * (nin + 2), st);
  rmsnorm_bwd_kernel<<<row_grid(rows), ROW_WARPS * 32, 0, st>>>(g0, g1, g2, ldg, y, ldy, r, resid, ldr, rows, d, dx,
                                                                lddx);
  count_launch();
  return launch_status("norm");
}

poet_status block_rope(bf16 *x, int64_t ldx, int64_t rows, int d, int head_dim, int seq_len, float base, bool inverse,
                       cudaStream_t st) {
  if (rows <= 0) return POET_OK;
  TraceScope ts("rope", 6.0 * double(rows) * d / 2, double(rows) * d * 4.0, st);
  rope_kernel<<<elem_grid(rows * (d / 2)), 256, 0, st>>>(x, ldx, rows, d, head_dim, seq_len, std::log(double(base)),
                                                         inverse ? 1 : 0);
  count_launch();
  return launch_status("rope");
}

poet_status block_softmax(const float *s, int64_t rows, int S, bf16 *p, cudaStream_t st) {
  if (rows <= 0) return POET_OK;
  TraceScope ts("softmax", 0.0, double(rows) * S * 6.0, st);
  causal_softmax_kernel<<<row_grid(rows), ROW_WARPS * 32, 0, st>>>(s, rows, S, p);
  count_launch();
  return launch_status("softmax");
}

poet_status block_softmax_bwd(const bf16 *p, const float *dp, int64_t rows, int S, float scale, bf16 *ds,
                              cudaStream_t st) {
  if (rows <= 0) return POET_OK;
  TraceScope ts("softmax", 0.0, double(rows) * S * 8.0, st);
  softmax_bwd_kernel<<<row_grid(rows), ROW_WARPS * 32, 0, st>>>(p, dp, rows, S, scale, ds);
  count_launch();
  return launch_status("softmax");
}

poet_status block_swiglu(const bf16 *g, const bf16 *u, int64_t ld, int64_t rows, int d, bf16 *m, int64_t ldm,
                         cudaStream_t st) {
  if (rows <= 0) return POET_OK;
  TraceScope ts("swiglu", 0.0, double(rows) * d * 6.0, st);
  swiglu_kernel<<<elem_grid(rows * d), 256, 0, st>>>(g, u, ld, rows, d, m, ldm);
  count_launch();
  return launch_status("swiglu");
}

poet_status block_swiglu_bwd(const bf16 *dm, int64_t lddm, const bf16 *g, const bf16 *u, int64_t ld, int64_t rows,
                             int d, bf16 *dg, bf16 *du, int64_t ldo, cudaStream_t st) {
  if (rows <= 0) return POET_OK;
  TraceScope ts("swiglu", 0.0, double(rows) * d * 10.0, st);
  swiglu_bwd_kernel<<<elem_grid(rows * d), 256, 0, st>>>(dm, lddm, g, u, ld, rows, d, dg, du, ldo);
  count_launch();
  return launch_status("swiglu");
}

poet_status block_add(const bf16 *a, int64_t lda, const bf16 *b, int64_t ldb, int64_t rows, int d, bf16 *out,
                      int64_t ldo, cudaStream_t st) {
  if (rows <= 0) return POET_OK;
  TraceScope ts("residual", 0.0, double(rows) * d * 6.0, st);
  add_kernel<<<elem_grid(rows * d), 256, 0, st>>>(a, lda, b, ldb, rows, d, out, ldo);
  count_launch();
  return launch_status("residual");
}

}  // namespace poet
