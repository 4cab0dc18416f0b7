// CUDA-core FMA engine of the batched GEMM (float32 accumulation).
//
// Serves float32 layers (where tensor-core inputs would not meet float32
// accuracy) and any operand layout the tcgen05 engine cannot read.  64x64
// output tiles, 16-deep K slices staged in shared memory, 4x4 outputs per
// thread; operands are read through arbitrary element strides.
#include "poet_internal.cuh"

namespace poet {
namespace {

constexpr int TM = 64, TN = 64, TK = 16, NT = 256;

template <typename T> __device__ __forceinline__ float ld_as_float(const T *p);
template <> __device__ __forceinline__ float ld_as_float<float>(const float *p) { return __ldg(p); }
template <> __device__ __forceinline__ float ld_as_float<bf16>(const bf16 *p) { return __bfloat162float(*p); }

template <typename T> __device__ __forceinline__ void st_from_float(T *p, float v);
template <> __device__ __forceinline__ void st_from_float<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void st_from_float<bf16>(bf16 *p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ float ld_any(const void *p, int dtype, int64_t i) {
  return dtype == POET_BF16 ? __bfloat162float(static_cast<const bf16 *>(p)[i]) : static_cast<const float *>(p)[i];
}

template <typename T>
__global__ void __launch_bounds__(NT) gemm_simt_kernel(Gemm g, int splitk, int kchunk) {
  const bool reduce = g.atomic && splitk > 1;  // partial sums added into the zeroed output
  __shared__ float As[TK][TM + 1];
  __shared__ float Bs[TK][TN + 1];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int bz = blockIdx.z;
  const int b = bz / splitk, split = bz % splitk;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int kbeg = split * kchunk;
  const int kend = min(g.K, kbeg + kchunk);
  const T *A = static_cast<const T *>(g.A) + int64_t(b) * g.a_b;
  const T *B = static_cast<const T *>(g.B) + int64_t(b) * g.b_b;
  const bool a_kfast = g.a_k == 1, b_kfast = g.b_k == 1;

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = kbeg; k0 < kend; k0 += TK) {
    for (int e = tid; e < TM * TK; e += NT) {
      int mm, kk;
      if (a_kfast) { kk = e % TK; mm = e / TK; } else { mm = e % TM; kk = e / TM; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < g.M && gk < kend) ? ld_as_float<T>(A + int64_t(gm) * g.a_m + int64_t(gk) * g.a_k) : 0.f;
    }
    for (int e = tid; e < TN * TK; e += NT) {
      int nn, kk;
      if (b_kfast) { kk = e % TK; nn = e / TK; } else { nn = e % TN; kk = e / TN; }
      const int gn = n0 + nn, gk = k0 + kk;
      Bs[kk][nn] = (gn < g.N && gk < kend) ? ld_as_float<T>(B + int64_t(gn) * g.b_n + int64_t(gk) * g.b_k) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= g.N) continue;
      float v = g.alpha * acc[i][j];
      if (reduce) {
        atomicAdd(g.outF + int64_t(b) * g.of_b + int64_t(gm) * g.of_m + gn, v);
        continue;
      }
      if (g.add) v += g.beta * ld_any(g.add, g.add_dtype, int64_t(b) * g.add_b + int64_t(gm) * g.add_m + gn);
      if (g.add2) v += g.beta2 * ld_any(g.add2, g.add2_dtype, int64_t(b) * g.add2_b + int64_t(gm) * g.add2_m + gn);
      if (gm == gn) v += g.diag;
      if (g.outF) g.outF[int64_t(b) * g.of_b + int64_t(gm) * g.of_m + gn] = v;
      if (g.outD) st_from_float<T>(static_cast<T *>(g.outD) + int64_t(b) * g.od_b + int64_t(gm) * g.od_m + gn, v);
    }
  }
}

}  // namespace

poet_status gemm_simt(const Gemm &g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return POET_OK;
  const int mt = (g.M + TM - 1) / TM, nt = (g.N + TN - 1) / TN;
  // split K only for atomically accumulated outputs with few tiles
  int splitk = 1;
  if (g.atomic && g.K > 0) {
    const int64_t tiles = int64_t(mt) * nt * g.batch;
    const int64_t want = (2 * int64_t(num_sms()) + tiles - 1) / tiles;
    const int64_t maxk = (g.K + 255) / 256;
    splitk = int(want < maxk ? want : maxk);
    if (splitk < 1) splitk = 1;
    if (splitk > 4096) splitk = 4096;
  }
  int kchunk = (g.K + splitk - 1) / splitk;
  kchunk = int(round_up(kchunk, TK));
  if (g.K == 0) kchunk = 0;
  POET_REQUIRE(int64_t(g.batch) * splitk <= 65535 && mt <= 65535, "gemm grid too large (M=%d batch=%d)", g.M, g.batch);
  dim3 grid(nt, mt, g.batch * splitk);
  if (g.atomic && splitk > 1) POET_TRY(zero_output(g.outF, g.M, g.N, g.of_m, g.batch, g.of_b, st));
  if (g.dtype == POET_BF16)
    gemm_simt_kernel<bf16><<<grid, NT, 0, st>>>(g, splitk, kchunk);
  else
    gemm_simt_kernel<float><<<grid, NT, 0, st>>>(g, splitk, kchunk);
  count_launch();
  return launch_status("gemm_simt");
}

}  // namespace poet
