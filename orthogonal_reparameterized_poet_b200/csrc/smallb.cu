// Block-diagonal products for small primitives (size <= 32): CUDA cores, and
// for bf16 blocks of 16 or 32 in the right product, mma.sync tensor-core tiles.
//
// POET summary page, Approach: the primitives are small orthogonal blocks
// acting on sampled index subsets; with blocks of 32 or fewer the products
// with them carry about 2 * size flops per element moved, far below the
// B200's flop/byte ridge, so they are bound by HBM bandwidth, and a
// tensor-core tile (128 rows) would be mostly empty.  These kernels move
// each element once and keep the arithmetic in registers:
//
//   right:  out[r][j*s + a] = sum_c X[r][j*s + c] * M_j(a, c)   (column blocks)
//   left:   out[j*s + a][k] = sum_c M_j(a, c) * X[j*s + c][k]   (row blocks)
//   grad:   G_j[a][c]      += sum_r D[r][j*s + a] * V[r][j*s + c]
//
// with M_j(a, c) = M_j[a][c], or M_j[c][a] when transposed.  Every global
// access is coalesced: a warp loads one row segment of a block per
// instruction (right, grad) or one element of 32 consecutive columns (left).
// Block rows (right), gradient rows (grad) or a column segment (left) sit in
// registers, the other operand is read from shared memory as warp-wide
// broadcasts, and the accumulation is float (fused multiply-add, in the order
// c = 0 .. s-1).
#include "poet_internal.cuh"

namespace poet {
namespace {

constexpr int SB = 32;        // largest primitive size served here
constexpr int SB_ROWS = 128;  // columns per CTA (left)
constexpr int SB_WARPS = 8;   // warps per CTA (right, grad)
constexpr int RU = 8;         // rows per warp iteration (right, grad): loads in flight

template <typename T> __device__ __forceinline__ float ldf(const T *p);
template <> __device__ __forceinline__ float ldf<float>(const float *p) { return __ldg(p); }
template <> __device__ __forceinline__ float ldf<bf16>(const bf16 *p) { return __bfloat162float(*p); }
template <typename T> __device__ __forceinline__ void stf(T *p, float v);
template <> __device__ __forceinline__ void stf<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void stf<bf16>(bf16 *p, float v) { *p = __float2bfloat16_rn(v); }

// Stage block j as float in shared memory, Ms[a][c] = M_j(a, c) (row stride SB);
// every entry outside the s x s block is zero, since the products read whole
// rows of SB entries (0 * an unset entry could be NaN).
template <typename T>
__device__ __forceinline__ void stage_block(const T *M, int64_t ldm, int64_t bstride, int j, int s, bool trans,
                                            float *Ms) {
  const T *Mj = M + int64_t(j) * bstride;
  for (int e = threadIdx.x; e < SB * SB; e += blockDim.x) {
    const int a = e / SB, c = e % SB;
    float v = 0.f;
    if (a < s && c < s) v = trans ? ldf(Mj + int64_t(c) * ldm + a) : ldf(Mj + int64_t(a) * ldm + c);
    Ms[e] = v;
  }
}

// right: blockIdx.y = block j, blockIdx.x = a range of rows.  Lane a of every
// warp keeps row a of the block (M_j(a, c), c < s) in registers; each warp
// takes RU rows at a time, lane c loading element c of each row segment
// (coalesced) into shared memory, then lane a forms output a of each row from
// broadcast reads.
template <typename T>
__global__ void __launch_bounds__(SB_WARPS * 32) smallb_right_kernel(const T *__restrict__ X, int64_t ldx,
                                                                     int64_t rows, int64_t rows_per_cta,
                                                                     const T *__restrict__ M, int64_t ldm,
                                                                     int64_t bstride, int s, int trans,
                                                                     T *__restrict__ out, int64_t ldo) {
  __shared__ __align__(16) float xs[SB_WARPS][RU][SB];
  const int j = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const T *Mj = M + int64_t(j) * bstride;
  float m[SB];
#pragma unroll
  for (int c = 0; c < SB; ++c)
    m[c] = (lane < s && c < s) ? (trans ? ldf(Mj + int64_t(c) * ldm + lane) : ldf(Mj + int64_t(lane) * ldm + c)) : 0.f;
  const int64_t r0 = int64_t(blockIdx.x) * rows_per_cta;
  const int64_t r1 = r0 + rows_per_cta < rows ? r0 + rows_per_cta : rows;
  const int64_t col = int64_t(j) * s + lane;
  for (int64_t rb = r0 + int64_t(warp) * RU; rb < r1; rb += int64_t(SB_WARPS) * RU) {
    float v[RU];
#pragma unroll
    for (int u = 0; u < RU; ++u) v[u] = (lane < s && rb + u < r1) ? ldf(X + (rb + u) * ldx + col) : 0.f;
#pragma unroll
    for (int u = 0; u < RU; ++u) xs[warp][u][lane] = v[u];
    __syncwarp();
#pragma unroll
    for (int u = 0; u < RU; ++u) {
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < SB; c += 4) {
        const float4 x4 = *reinterpret_cast<const float4 *>(&xs[warp][u][c]);  // a broadcast
        acc = fmaf(m[c], x4.x, acc);
        acc = fmaf(m[c + 1], x4.y, acc);
        acc = fmaf(m[c + 2], x4.z, acc);
        acc = fmaf(m[c + 3], x4.w, acc);
      }
      if (lane < s && rb + u < r1) stf(out + (rb + u) * ldo + col, acc);
    }
    __syncwarp();
  }
}

// left: blockIdx.y = block j, blockIdx.x = a chunk of SB_ROWS columns; one thread per column.
template <typename T>
__global__ void __launch_bounds__(SB_ROWS) smallb_left_kernel(const T *__restrict__ X, int64_t ldx, int64_t cols,
                                                              const T *__restrict__ M, int64_t ldm, int64_t bstride,
                                                              int s, int trans, T *__restrict__ out, int64_t ldo) {
  __shared__ float Ms[SB * SB];
  const int j = blockIdx.y;
  stage_block(M, ldm, bstride, j, s, trans != 0, Ms);
  __syncthreads();
  const int64_t k = int64_t(blockIdx.x) * SB_ROWS + threadIdx.x;
  if (k >= cols) return;
  const T *xc = X + int64_t(j) * s * ldx + k;
  float x[SB];
#pragma unroll
  for (int c = 0; c < SB; ++c) x[c] = c < s ? ldf(xc + int64_t(c) * ldx) : 0.f;  // coalesced across the warp
  T *ocol = out + int64_t(j) * s * ldo + k;
  for (int a = 0; a < s; ++a) {
    const float *m = Ms + a * SB;
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < SB; c += 4) {
      const float4 mv = *reinterpret_cast<const float4 *>(m + c);
      acc = fmaf(mv.x, x[c], acc);
      acc = fmaf(mv.y, x[c + 1], acc);
      acc = fmaf(mv.z, x[c + 2], acc);
      acc = fmaf(mv.w, x[c + 3], acc);
    }
    stf(ocol + int64_t(a) * ldo, acc);
  }
}

// grad: blockIdx.y = block j, blockIdx.x = a range of rows.  Lane a of each warp
// accumulates row a of G_j over the warp's rows, RU rows at a time: V's row
// segments are staged in shared memory (coalesced loads) and read as
// broadcasts; the CTA's warps are summed in shared memory and added to G with
// one float atomic per element.
template <typename T>
__global__ void __launch_bounds__(SB_WARPS * 32) smallb_grad_kernel(const T *__restrict__ D, const T *__restrict__ V,
                                                                    int64_t ld, int64_t rows, int64_t rows_per_cta,
                                                                    int s, float *__restrict__ G, int64_t ldg,
                                                                    int64_t gstride) {
  __shared__ __align__(16) float vs[SB_WARPS][RU][SB];
  __shared__ float red[SB_WARPS][SB][SB + 1];
  const int j = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t r0 = int64_t(blockIdx.x) * rows_per_cta;
  const int64_t r1 = r0 + rows_per_cta < rows ? r0 + rows_per_cta : rows;
  const int64_t col = int64_t(j) * s + lane;
  float acc[SB];
#pragma unroll
  for (int c = 0; c < SB; ++c) acc[c] = 0.f;
  for (int64_t rb = r0 + int64_t(warp) * RU; rb < r1; rb += int64_t(SB_WARPS) * RU) {
    float dv[RU], vv[RU];
#pragma unroll
    for (int u = 0; u < RU; ++u) {
      const bool ok = lane < s && rb + u < r1;
      dv[u] = ok ? ldf(D + (rb + u) * ld + col) : 0.f;
      vv[u] = ok ? ldf(V + (rb + u) * ld + col) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < RU; ++u) vs[warp][u][lane] = vv[u];
    __syncwarp();
#pragma unroll
    for (int u = 0; u < RU; ++u) {
#pragma unroll
      for (int c = 0; c < SB; c += 4) {
        const float4 v4 = *reinterpret_cast<const float4 *>(&vs[warp][u][c]);
        acc[c] = fmaf(dv[u], v4.x, acc[c]);
        acc[c + 1] = fmaf(dv[u], v4.y, acc[c + 1]);
        acc[c + 2] = fmaf(dv[u], v4.z, acc[c + 2]);
        acc[c + 3] = fmaf(dv[u], v4.w, acc[c + 3]);
      }
    }
    __syncwarp();
  }
#pragma unroll
  for (int c = 0; c < SB; ++c) red[warp][lane][c] = acc[c];
  __syncthreads();
  float *Gj = G + int64_t(j) * gstride;
  for (int e = threadIdx.x; e < s * s; e += blockDim.x) {
    const int a = e / s, c = e % s;
    float sum = 0.f;
    for (int w = 0; w < SB_WARPS; ++w) sum += red[w][a][c];
    atomicAdd(Gj + int64_t(a) * ldg + c, sum);
  }
}

__device__ __forceinline__ uint32_t bf16_pair(bf16 lo, bf16 hi) {
  return uint32_t(__bfloat16_as_ushort(lo)) | (uint32_t(__bfloat16_as_ushort(hi)) << 16);
}

__device__ __forceinline__ void ldsm_x4(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  const uint32_t a = uint32_t(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_trans(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  const uint32_t a = uint32_t(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}

// right for bf16 blocks of 16 or 32 with 16-byte aligned rows, on the tensor
// cores: mma.sync m16n8k16 (bf16 in, float accumulate) takes the s
// multiply-adds per output off the CUDA cores (the CUDA-core kernel above is
// bound by them and by its broadcast reads).  blockIdx.y = block j.  Each
// warp holds M_j's B fragments in registers, stages 32 rows of X_j in its own
// shared memory with 16-byte loads (rows padded to S + 8 elements, so that
// the eight row segments of an ldmatrix fall on distinct banks), takes the A
// fragments with ldmatrix, writes the outputs back over the same rows and
// stores them as 16-byte units.  Fragment layouts of m16n8k16 (g = lane / 4,
// q = lane % 4): A regs = X[g][2q..], X[g+8][2q..], X[g][2q+8..],
// X[g+8][2q+8..]; B regs = M(n=g, k=2q..), M(g, 2q+8..); C = out[g][2q..],
// out[g+8][2q..]; every register holds two consecutive bf16 (the lower
// column in the low half).  Fragments built from 4-byte global loads and
// stores instead kept L1/TEX at 87 % at half the copy peak.
template <int S>
__global__ void __launch_bounds__(SB_WARPS * 32) smallb_right_mma_staged_kernel(
    const bf16 *__restrict__ X, int64_t ldx, int64_t rows, int64_t rows_per_cta, const bf16 *__restrict__ M,
    int64_t ldm, int64_t bstride, int trans, bf16 *__restrict__ out, int64_t ldo) {
  constexpr int KS = S / 16, NT = S / 8, RW = 32, LDS = S + 8, CH = S / 8, PER = RW * CH / 32;
  __shared__ __align__(16) bf16 sx[SB_WARPS][RW][LDS];
  const int j = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, q = lane & 3, mi = lane >> 3, mr = lane & 7;
  const bf16 *Mj = M + int64_t(j) * bstride;
  auto m_at = [&](int a, int c) { return trans ? Mj[int64_t(c) * ldm + a] : Mj[int64_t(a) * ldm + c]; };
  uint32_t bfr[KS][NT][2];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int a = nt * 8 + g, c = ks * 16 + 2 * q;
      bfr[ks][nt][0] = bf16_pair(m_at(a, c), m_at(a, c + 1));
      bfr[ks][nt][1] = bf16_pair(m_at(a, c + 8), m_at(a, c + 9));
    }
  const int64_t r_begin = int64_t(blockIdx.x) * rows_per_cta;
  const int64_t r_end = r_begin + rows_per_cta < rows ? r_begin + rows_per_cta : rows;
  const bf16 *Xj = X + int64_t(j) * S;
  bf16 *Oj = out + int64_t(j) * S;
  bf16(*tile)[LDS] = sx[warp];
  for (int64_t r0 = r_begin + warp * RW; r0 < r_end; r0 += SB_WARPS * RW) {
    uint4 buf[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int idx = lane + 32 * i, r = idx / CH, ch = idx % CH;
      buf[i] = r0 + r < r_end ? *reinterpret_cast<const uint4 *>(Xj + (r0 + r) * ldx + ch * 8) : make_uint4(0, 0, 0, 0);
    }
    __syncwarp();  // the previous rows' outputs have left the tile
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int idx = lane + 32 * i, r = idx / CH, ch = idx % CH;
      *reinterpret_cast<uint4 *>(&tile[r][ch * 8]) = buf[i];
    }
    __syncwarp();
#pragma unroll
    for (int mt = 0; mt < RW / 16; ++mt) {
      uint32_t af[KS][4];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)  // matrix i: rows 16 mt + 8 (i & 1), columns 16 ks + 8 (i >> 1)
        ldsm_x4(&tile[mt * 16 + (mi & 1) * 8 + mr][ks * 16 + (mi >> 1) * 8], af[ks][0], af[ks][1], af[ks][2],
                af[ks][3]);
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
              "{%0, %1, %2, %3};"
              : "+f"(acc[nt][0]), "+f"(acc[nt][1]), "+f"(acc[nt][2]), "+f"(acc[nt][3])
              : "r"(af[ks][0]), "r"(af[ks][1]), "r"(af[ks][2]), "r"(af[ks][3]), "r"(bfr[ks][nt][0]),
                "r"(bfr[ks][nt][1]));
      }
      __syncwarp();  // every lane's fragments of these 16 rows are in registers
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int c = nt * 8 + 2 * q;
        *reinterpret_cast<__nv_bfloat162 *>(&tile[mt * 16 + g][c]) = __floats2bfloat162_rn(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<__nv_bfloat162 *>(&tile[mt * 16 + g + 8][c]) = __floats2bfloat162_rn(acc[nt][2], acc[nt][3]);
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int idx = lane + 32 * i, r = idx / CH, ch = idx % CH;
      if (r0 + r < r_end)
        *reinterpret_cast<uint4 *>(Oj + (r0 + r) * ldo + ch * 8) = *reinterpret_cast<const uint4 *>(&tile[r][ch * 8]);
    }
  }
}

// grad for bf16 blocks of 16 or 32 on the tensor cores: G_j = D_j^T V_j is a
// product over the rows, and both operands hold the rows as their strided
// dimension, so each warp stages 32 rows of D_j and V_j in its own shared
// memory (rows padded to S + 8 elements: eight 16-byte row segments of an
// ldmatrix then fall on distinct banks) and takes the fragments with
// ldmatrix.trans, which hands every lane two consecutive rows of one column.
// A(a, r) = D[r][j*S + a], B(r, c) = V[r][j*S + c]; the accumulators of the
// S x S block stay in registers over the CTA's rows, then the warps are summed
// with shared atomics and added to G with one float atomic per element.

template <int S>
__global__ void __launch_bounds__(SB_WARPS * 32) smallb_grad_mma_kernel(const bf16 *__restrict__ D,
                                                                        const bf16 *__restrict__ V, int64_t ld,
                                                                        int64_t rows, int64_t rows_per_cta,
                                                                        float *__restrict__ G, int64_t ldg,
                                                                        int64_t gstride) {
  constexpr int MT = S / 16, NT = S / 8, RW = 32, LDS = S + 8, CH = S / 8;  // CH: 16-byte chunks per row
  __shared__ __align__(16) bf16 sd[SB_WARPS][RW][LDS];
  __shared__ __align__(16) bf16 sv[SB_WARPS][RW][LDS];
  __shared__ float red[S][S + 1];
  const int j = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, q = lane & 3;
  for (int e = threadIdx.x; e < S * (S + 1); e += blockDim.x) (&red[0][0])[e] = 0.f;
  const int64_t r_begin = int64_t(blockIdx.x) * rows_per_cta;
  const int64_t r_end = r_begin + rows_per_cta < rows ? r_begin + rows_per_cta : rows;
  const bf16 *Dj = D + int64_t(j) * S;
  const bf16 *Vj = V + int64_t(j) * S;
  float acc[MT][NT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
  // ldmatrix addresses: lane i of matrix (lane / 8) gives row (lane % 8) of that 8 x 8 matrix
  const int mi = lane >> 3, mr = lane & 7;
  for (int64_t r0 = r_begin + warp * RW; r0 < r_end; r0 += SB_WARPS * RW) {
    uint4 dbuf[RW * CH / 32], vbuf[RW * CH / 32];
#pragma unroll
    for (int i = 0; i < RW * CH / 32; ++i) {
      const int idx = lane + 32 * i, r = idx / CH, ch = idx % CH;
      const bool ok = r0 + r < r_end;
      dbuf[i] = ok ? *reinterpret_cast<const uint4 *>(Dj + (r0 + r) * ld + ch * 8) : make_uint4(0, 0, 0, 0);
      vbuf[i] = ok ? *reinterpret_cast<const uint4 *>(Vj + (r0 + r) * ld + ch * 8) : make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < RW * CH / 32; ++i) {
      const int idx = lane + 32 * i, r = idx / CH, ch = idx % CH;
      *reinterpret_cast<uint4 *>(&sd[warp][r][ch * 8]) = dbuf[i];
      *reinterpret_cast<uint4 *>(&sv[warp][r][ch * 8]) = vbuf[i];
    }
    __syncwarp();
#pragma unroll
    for (int k0 = 0; k0 < RW; k0 += 16) {
      uint32_t af[MT][4], bfr[NT][2];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)  // matrix i: rows k0 + 8 (i & 2 ? 1 : 0), columns 16 mt + 8 (i & 1)
        ldsm_x4_trans(&sd[warp][k0 + ((mi & 2) ? 8 : 0) + mr][mt * 16 + ((mi & 1) ? 8 : 0)], af[mt][0], af[mt][1],
                      af[mt][2], af[mt][3]);
#pragma unroll
      for (int np = 0; np < NT / 2; ++np)  // matrix i: rows k0 + 8 (i & 1), columns 16 np + 8 (i & 2 ? 1 : 0)
        ldsm_x4_trans(&sv[warp][k0 + ((mi & 1) ? 8 : 0) + mr][np * 16 + ((mi & 2) ? 8 : 0)], bfr[2 * np][0],
                      bfr[2 * np][1], bfr[2 * np + 1][0], bfr[2 * np + 1][1]);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
              "{%0, %1, %2, %3};"
              : "+f"(acc[mt][nt][0]), "+f"(acc[mt][nt][1]), "+f"(acc[mt][nt][2]), "+f"(acc[mt][nt][3])
              : "r"(af[mt][0]), "r"(af[mt][1]), "r"(af[mt][2]), "r"(af[mt][3]), "r"(bfr[nt][0]), "r"(bfr[nt][1]));
    }
    __syncwarp();
  }
  __syncthreads();  // red zeroed
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int a = mt * 16 + g, c = nt * 8 + 2 * q;
      atomicAdd(&red[a][c], acc[mt][nt][0]);
      atomicAdd(&red[a][c + 1], acc[mt][nt][1]);
      atomicAdd(&red[a + 8][c], acc[mt][nt][2]);
      atomicAdd(&red[a + 8][c + 1], acc[mt][nt][3]);
    }
  __syncthreads();
  float *Gj = G + int64_t(j) * gstride;
  for (int e = threadIdx.x; e < S * S; e += blockDim.x) {
    const int a = e / S, c = e % S;
    atomicAdd(Gj + int64_t(a) * ldg + c, red[a][c]);
  }
}

// Row ranges per block for about four CTAs per SM over all blocks (at least 64 rows each).
int64_t rows_per_cta(int64_t rows, int nprim) {
  int64_t ranges = (int64_t(num_sms()) * 4 + nprim - 1) / nprim;
  int64_t per = (rows + ranges - 1) / ranges;
  return per < 64 ? 64 : per;
}

}  // namespace

bool smallb_supported(int size) { return size >= 1 && size <= SB; }

poet_status smallb_right(int dtype, const void *X, int64_t ldx, int64_t rows, const void *M, int64_t ldm,
                         int64_t bstride, int nprim, int s, bool trans, void *out, int64_t ldo, cudaStream_t st,
                         const char *kind) {
  if (rows <= 0 || nprim <= 0 || s <= 0) return POET_OK;
  POET_REQUIRE(smallb_supported(s) && nprim <= 65535, "smallb: primitive size %d or count %d out of range", s, nprim);
  const int64_t per = rows_per_cta(rows, nprim);
  const dim3 grid(unsigned((rows + per - 1) / per), unsigned(nprim));
  const double elems = double(rows) * nprim * s;
  TraceScope ts(kind, 2.0 * elems * s, elems * esize(dtype) * 2.0, st);
  const bool units_ok = ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(out)) & 15) == 0 &&
                        ldx % 8 == 0 && ldo % 8 == 0;
  if (dtype == POET_BF16 && (s == 16 || s == 32) && units_ok) {
    if (s == 32)
      smallb_right_mma_staged_kernel<32><<<grid, SB_WARPS * 32, 0, st>>>(
          static_cast<const bf16 *>(X), ldx, rows, per, static_cast<const bf16 *>(M), ldm, bstride, trans ? 1 : 0,
          static_cast<bf16 *>(out), ldo);
    else
      smallb_right_mma_staged_kernel<16><<<grid, SB_WARPS * 32, 0, st>>>(
          static_cast<const bf16 *>(X), ldx, rows, per, static_cast<const bf16 *>(M), ldm, bstride, trans ? 1 : 0,
          static_cast<bf16 *>(out), ldo);
  } else if (dtype == POET_BF16)
    smallb_right_kernel<bf16><<<grid, SB_WARPS * 32, 0, st>>>(static_cast<const bf16 *>(X), ldx, rows, per,
                                                              static_cast<const bf16 *>(M), ldm, bstride, s,
                                                              trans ? 1 : 0, static_cast<bf16 *>(out), ldo);
  else
    smallb_right_kernel<float><<<grid, SB_WARPS * 32, 0, st>>>(static_cast<const float *>(X), ldx, rows, per,
                                                               static_cast<const float *>(M), ldm, bstride, s,
                                                               trans ? 1 : 0, static_cast<float *>(out), ldo);
  count_launch();
  return launch_status(kind);
}

poet_status smallb_left(int dtype, const void *X, int64_t ldx, int64_t cols, const void *M, int64_t ldm,
                        int64_t bstride, int nprim, int s, bool trans, void *out, int64_t ldo, cudaStream_t st,
                        const char *kind) {
  if (cols <= 0 || nprim <= 0 || s <= 0) return POET_OK;
  POET_REQUIRE(smallb_supported(s) && nprim <= 65535, "smallb: primitive size %d or count %d out of range", s, nprim);
  const dim3 grid(unsigned((cols + SB_ROWS - 1) / SB_ROWS), unsigned(nprim));
  const double elems = double(cols) * nprim * s;
  TraceScope ts(kind, 2.0 * elems * s, elems * esize(dtype) * 2.0, st);
  if (dtype == POET_BF16)
    smallb_left_kernel<bf16><<<grid, SB_ROWS, 0, st>>>(static_cast<const bf16 *>(X), ldx, cols,
                                                       static_cast<const bf16 *>(M), ldm, bstride, s, trans ? 1 : 0,
                                                       static_cast<bf16 *>(out), ldo);
  else
    smallb_left_kernel<float><<<grid, SB_ROWS, 0, st>>>(static_cast<const float *>(X), ldx, cols,
                                                        static_cast<const float *>(M), ldm, bstride, s, trans ? 1 : 0,
                                                        static_cast<float *>(out), ldo);
  count_launch();
  return launch_status(kind);
}

poet_status smallb_grad(int dtype, const void *D, const void *V, int64_t ld, int64_t rows, int nprim, int s, float *G,
                        int64_t ldg, int64_t gstride, cudaStream_t st) {
  if (rows <= 0 || nprim <= 0 || s <= 0) return POET_OK;
  POET_REQUIRE(smallb_supported(s) && nprim <= 65535, "smallb: primitive size %d or count %d out of range", s, nprim);
  const int64_t per = rows_per_cta(rows, nprim);
  const dim3 grid(unsigned((rows + per - 1) / per), unsigned(nprim));
  POET_TRY(zero_output(G, s, s, ldg, nprim, gstride, st));  // the CTAs' sums are added into it
  const double elems = double(rows) * nprim * s;
  TraceScope ts("blk_grad", 2.0 * elems * s, elems * esize(dtype) * 2.0, st);
  const bool chunks_ok = ((reinterpret_cast<uintptr_t>(D) | reinterpret_cast<uintptr_t>(V)) & 15) == 0 && ld % 8 == 0;
  if (dtype == POET_BF16 && (s == 16 || s == 32) && chunks_ok) {
    if (s == 32)
      smallb_grad_mma_kernel<32><<<grid, SB_WARPS * 32, 0, st>>>(static_cast<const bf16 *>(D),
                                                                 static_cast<const bf16 *>(V), ld, rows, per, G, ldg,
                                                                 gstride);
    else
      smallb_grad_mma_kernel<16><<<grid, SB_WARPS * 32, 0, st>>>(static_cast<const bf16 *>(D),
                                                                 static_cast<const bf16 *>(V), ld, rows, per, G, ldg,
                                                                 gstride);
  } else if (dtype == POET_BF16)
    smallb_grad_kernel<bf16><<<grid, SB_WARPS * 32, 0, st>>>(
        static_cast<const bf16 *>(D), static_cast<const bf16 *>(V), ld, rows, per, s, G, ldg, gstride);
  else
    smallb_grad_kernel<float><<<grid, SB_WARPS * 32, 0, st>>>(
        static_cast<const float *>(D), static_cast<const float *>(V), ld, rows, per, s, G, ldg, gstride);
  count_launch();
  return launch_status("blk_grad");
}

poet_status smallb_dispatch(const Gemm &g, cudaStream_t st, bool *done) {
  *done = false;
  if (!g.small || g.alpha != 1.f || g.add || g.add2 || g.diag != 0.f) return POET_OK;
  if (g.small == SMALL_RIGHT) {
    // A = X (K contiguous, blocks s apart), B_j(a, c) = B[a][c] (b_n = ld) or B[c][a] (b_n = 1)
    if (!smallb_supported(g.K) || g.N != g.K || g.a_k != 1 || g.a_b != g.K || !g.outD || g.outF || g.od_b != g.K)
      return POET_OK;
    const bool trans = g.b_n == 1;
    *done = true;
    return smallb_right(g.dtype, g.A, g.a_m, g.M, g.B, trans ? g.b_k : g.b_n, g.b_b, g.batch, g.K, trans, g.outD,
                        g.od_m, st, g.tag);
  }
  if (g.small == SMALL_LEFT) {
    // A_j = the primitives (K contiguous), B = rows of the matrix (N contiguous, blocks s rows apart)
    if (!smallb_supported(g.K) || g.M != g.K || g.a_k != 1 || g.b_n != 1 || g.b_b != int64_t(g.K) * g.b_k ||
        !g.outD || g.outF || g.od_b != int64_t(g.K) * g.od_m)
      return POET_OK;
    *done = true;
    return smallb_left(g.dtype, g.B, g.b_k, g.N, g.A, g.a_m, g.a_b, g.batch, g.K, false, g.outD, g.od_m, st, g.tag);
  }
  if (g.small == SMALL_GRAD) {
    // A, B: token-major rows (M / N contiguous, blocks s apart), summed into outF
    if (!smallb_supported(g.M) || g.N != g.M || g.a_m != 1 || g.b_n != 1 || g.a_k != g.b_k || g.a_b != g.M ||
        g.b_b != g.M || !g.outF || !g.atomic || g.outD)
      return POET_OK;
    *done = true;
    return smallb_grad(g.dtype, g.A, g.B, g.a_k, g.K, g.batch, g.M, g.outF, g.of_m, g.of_b, st);
  }
  return POET_OK;
}

}  // namespace poet
