// Column permutations between natural order and the permuted frame.
//
// A side's primitives act on the natural indices perm[j*size .. j*size+size-1]
// (POET summary page, Approach: "sampled sub-block orthogonal primitives";
// the index layout is a reading).  These kernels move whole rows between the
// natural order and the frame order, so that every contraction downstream
// reads contiguous blocks.  Each CTA stages a few rows in shared memory:
// global reads and writes are 16-byte vectors on 16-byte boundaries (rows of
// odd length are split into an aligned body and scalar edges), and only the
// shared-memory side is accessed through the permutation.  HBM-bound.
#include "poet_internal.cuh"

namespace poet {
namespace {

constexpr int NT = 512;

__device__ __forceinline__ int perm_bytes_dev(int d) { return (d * 4 + 15) & ~15; }

// Row r of a chunk lives in shared memory at slot r (stride `slot` elements);
// element e of the global row sits at slot position off_r + e, where off_r is
// the row's misalignment (in elements) relative to 16 bytes, so that shared
// and global addresses agree modulo 16 and both sides can use 16-byte vectors.
template <typename T>
struct RowIO {
  static constexpr int VEC = 16 / sizeof(T);
  __device__ static int misalign(const T *row) { return int((reinterpret_cast<uintptr_t>(row) & 15) / sizeof(T)); }
  __device__ static int units(const T *row, int d) { return (misalign(row) + d + VEC - 1) / VEC; }
  // copy unit u of a global row into the slot (the slot is 16-byte aligned)
  __device__ static void load_unit(const T *row, int d, int u, T *slot) {
    const int off = misalign(row);
    const int first = u * VEC - off;  // row element of the unit's first lane
    if (first >= 0 && first + VEC <= d) {
      *reinterpret_cast<uint4 *>(slot + u * VEC) = __ldg(reinterpret_cast<const uint4 *>(row + first));
    } else {
      for (int v = 0; v < VEC; ++v) {
        const int e = first + v;
        if (e >= 0 && e < d) slot[u * VEC + v] = row[e];
      }
    }
  }
  __device__ static void store_unit(T *row, int d, int u, const T *slot) {
    const int off = misalign(row);
    const int first = u * VEC - off;
    if (first >= 0 && first + VEC <= d) {
      *reinterpret_cast<uint4 *>(row + first) = *reinterpret_cast<const uint4 *>(slot + u * VEC);
    } else {
      for (int v = 0; v < VEC; ++v) {
        const int e = first + v;
        if (e >= 0 && e < d) row[e] = slot[u * VEC + v];
      }
    }
  }
};

template <typename T>
__global__ void __launch_bounds__(NT) gather_cols_kernel(const T *__restrict__ src, int64_t ld_src,
                                                        const int32_t *__restrict__ rowmap, int64_t rows, int d,
                                                        const int32_t *__restrict__ perm, T *__restrict__ dst,
                                                        int64_t ld_dst, T *__restrict__ dst2, int64_t ld_dst2,
                                                        int split, int rows_per_cta, int slot) {
  using IO = RowIO<T>;
  constexpr int VEC = IO::VEC;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  int32_t *sperm = reinterpret_cast<int32_t *>(smem_raw);
  T *srows = reinterpret_cast<T *>(smem_raw + perm_bytes_dev(d));
  for (int i = threadIdx.x; i < d; i += NT) sperm[i] = perm[i];
  const int dpad = (d + VEC - 1) / VEC * VEC;  // frame columns written (zero padded)
  const int gpr = dpad / VEC;                  // vector groups per frame row
  const int64_t nchunks = (rows + rows_per_cta - 1) / rows_per_cta;
  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const int64_t r0 = c * rows_per_cta;
    const int nr = int(rows - r0 < rows_per_cta ? rows - r0 : rows_per_cta);
    __syncthreads();  // previous chunk's readers are done (and sperm is ready)
    // load: every unit of every row of the chunk
    const T *row0 = src + (rowmap ? int64_t(rowmap[r0]) : r0) * ld_src;
    const int upr = IO::units(row0, d) + 1;  // rows may differ in misalignment by one unit
    for (int idx = threadIdx.x; idx < nr * upr; idx += NT) {
      const int r = idx / upr, u = idx % upr;
      const T *row = src + (rowmap ? int64_t(rowmap[r0 + r]) : (r0 + r)) * ld_src;
      if (u < IO::units(row, d)) IO::load_unit(row, d, u, srows + int64_t(r) * slot);
    }
    __syncthreads();
    // write: frame row r, vector group q covers frame columns q*VEC .. q*VEC+VEC-1
    for (int idx = threadIdx.x; idx < nr * gpr; idx += NT) {
      const int r = idx / gpr, q = idx % gpr;
      const T *row = src + (rowmap ? int64_t(rowmap[r0 + r]) : (r0 + r)) * ld_src;
      const T *s = srows + int64_t(r) * slot + IO::misalign(row);
      alignas(16) T v[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const int i = q * VEC + e;
        v[e] = i < d ? s[sperm[i]] : T(0.f);
      }
      const int i0 = q * VEC;
      *reinterpret_cast<uint4 *>(dst + (r0 + r) * ld_dst + i0) = *reinterpret_cast<const uint4 *>(v);
      if (dst2) {
        if (i0 >= split) {
          *reinterpret_cast<uint4 *>(dst2 + (r0 + r) * ld_dst2 + i0) = *reinterpret_cast<const uint4 *>(v);
        } else if (i0 + VEC > split) {
          for (int e = split - i0; e < VEC; ++e) dst2[(r0 + r) * ld_dst2 + i0 + e] = v[e];
        }
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(NT) scatter_cols_kernel(const T *__restrict__ src1, int64_t ld1,
                                                         const T *__restrict__ src2, int64_t ld2, int split,
                                                         int64_t rows, int d, const int32_t *__restrict__ perm,
                                                         T *__restrict__ dst, int64_t ld_dst,
                                                         const int32_t *__restrict__ rowmap, int rows_per_cta,
                                                         int slot) {
  using IO = RowIO<T>;
  constexpr int VEC = IO::VEC;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  int32_t *sperm = reinterpret_cast<int32_t *>(smem_raw);
  T *srows = reinterpret_cast<T *>(smem_raw + perm_bytes_dev(d));
  for (int i = threadIdx.x; i < d; i += NT) sperm[i] = perm[i];
  const int gpr = (d + VEC - 1) / VEC;
  const int64_t nchunks = (rows + rows_per_cta - 1) / rows_per_cta;
  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const int64_t r0 = c * rows_per_cta;
    const int nr = int(rows - r0 < rows_per_cta ? rows - r0 : rows_per_cta);
    __syncthreads();
    // load frame rows (aligned vectors), scatter into the slot at natural positions
    for (int idx = threadIdx.x; idx < nr * gpr; idx += NT) {
      const int r = idx / gpr, q = idx % gpr;
      T *drow = dst + (rowmap ? int64_t(rowmap[r0 + r]) : (r0 + r)) * ld_dst;
      T *s = srows + int64_t(r) * slot + IO::misalign(drow);
      const int i0 = q * VEC;
      alignas(16) T v[VEC];
      if (i0 + VEC <= split) {
        *reinterpret_cast<uint4 *>(v) = __ldg(reinterpret_cast<const uint4 *>(src1 + (r0 + r) * ld1 + i0));
      } else if (i0 >= split) {
        *reinterpret_cast<uint4 *>(v) = __ldg(reinterpret_cast<const uint4 *>(src2 + (r0 + r) * ld2 + i0));
      } else {
        for (int e = 0; e < VEC; ++e) {
          const int i = i0 + e;
          if (i < d) v[e] = (i < split) ? src1[(r0 + r) * ld1 + i] : src2[(r0 + r) * ld2 + i];
        }
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const int i = i0 + e;
        if (i < d) s[sperm[i]] = v[e];
      }
    }
    __syncthreads();
    const T *drow0 = dst + (rowmap ? int64_t(rowmap[r0]) : r0) * ld_dst;
    const int upr = IO::units(drow0, d) + 1;
    for (int idx = threadIdx.x; idx < nr * upr; idx += NT) {
      const int r = idx / upr, u = idx % upr;
      T *drow = dst + (rowmap ? int64_t(rowmap[r0 + r]) : (r0 + r)) * ld_dst;
      if (u < IO::units(drow, d)) IO::store_unit(drow, d, u, srows + int64_t(r) * slot);
    }
  }
}

}  // namespace

// shared-memory plan: permutation (d ints, rounded to 16 bytes) + rows
static void plan_rows(int d, size_t esz, int64_t rows, int *rows_per_cta, int *slot, size_t *smem) {
  const int vec = int(16 / esz);
  *slot = int(round_up(d + 2 * vec, vec));  // misalignment offset + one spare unit
  const size_t perm_bytes = size_t(round_up(int64_t(d) * 4, 16));
  const size_t budget = 96 * 1024;
  int r = int((budget > perm_bytes ? budget - perm_bytes : 0) / (size_t(*slot) * esz));
  if (r < 1) r = 1;
  if (r > 16) r = 16;
  if (r > rows) r = int(rows > 0 ? rows : 1);
  *rows_per_cta = r;
  *smem = perm_bytes + size_t(r) * size_t(*slot) * esz;
}

poet_status gather_cols(int dtype, const void *src, int64_t ld_src, const int32_t *rowmap, int64_t rows, int d,
                        const int32_t *perm, void *dst, int64_t ld_dst, void *dst2, int64_t ld_dst2, int split,
                        cudaStream_t st) {
  if (rows <= 0 || d <= 0) return POET_OK;
  int rpc, slot;
  size_t smem;
  plan_rows(d, esize(dtype), rows, &rpc, &slot, &smem);
  const int64_t chunks = (rows + rpc - 1) / rpc;
  const int grid = int(chunks < 2 * num_sms() ? chunks : 2 * num_sms());
  TraceScope ts("gather", 0.0, double(rows) * d * esize(dtype) * 2.0, st);
  count_launch();
  if (dtype == POET_BF16) {
    POET_CUDA_TRY(cudaFuncSetAttribute(gather_cols_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    gather_cols_kernel<bf16><<<grid, NT, smem, st>>>(static_cast<const bf16 *>(src), ld_src, rowmap, rows, d, perm,
                                                     static_cast<bf16 *>(dst), ld_dst, static_cast<bf16 *>(dst2),
                                                     ld_dst2, split, rpc, slot);
  } else {
    POET_CUDA_TRY(cudaFuncSetAttribute(gather_cols_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    gather_cols_kernel<float><<<grid, NT, smem, st>>>(static_cast<const float *>(src), ld_src, rowmap, rows, d, perm,
                                                      static_cast<float *>(dst), ld_dst, static_cast<float *>(dst2),
                                                      ld_dst2, split, rpc, slot);
  }
  return launch_status("gather_cols");
}

poet_status scatter_cols(int dtype, const void *src1, int64_t ld1, const void *src2, int64_t ld2, int split,
                         int64_t rows, int d, const int32_t *perm, void *dst, int64_t ld_dst, const int32_t *rowmap,
                         cudaStream_t st) {
  if (rows <= 0 || d <= 0) return POET_OK;
  int rpc, slot;
  size_t smem;
  plan_rows(d, esize(dtype), rows, &rpc, &slot, &smem);
  const int64_t chunks = (rows + rpc - 1) / rpc;
  const int grid = int(chunks < 2 * num_sms() ? chunks : 2 * num_sms());
  TraceScope ts("scatter", 0.0, double(rows) * d * esize(dtype) * 2.0, st);
  count_launch();
  if (dtype == POET_BF16) {
    POET_CUDA_TRY(cudaFuncSetAttribute(scatter_cols_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    scatter_cols_kernel<bf16><<<grid, NT, smem, st>>>(static_cast<const bf16 *>(src1), ld1,
                                                      static_cast<const bf16 *>(src2), ld2, split, rows, d, perm,
                                                      static_cast<bf16 *>(dst), ld_dst, rowmap, rpc, slot);
  } else {
    POET_CUDA_TRY(cudaFuncSetAttribute(scatter_cols_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    scatter_cols_kernel<float><<<grid, NT, smem, st>>>(static_cast<const float *>(src1), ld1,
                                                       static_cast<const float *>(src2), ld2, split, rows, d, perm,
                                                       static_cast<float *>(dst), ld_dst, rowmap, rpc, slot);
  }
  return launch_status("scatter_cols");
}

}  // namespace poet
