// Permutation draw of one side (a10).
//
// POET summary page, Approach: the primitives act on sampled index subsets
// that are redrawn at every merge-then-reinitialize.  The pages fix no
// generator; the reading used here is counter-based SplitMix64 (Steele, Lea,
// Flood 2014): key_i is the i-th output of a SplitMix64 stream whose seed
// mixes (seed, layer_id, side, epoch), and the permutation lists 0..d-1
// ordered by (key_i, i).  One CTA draws and sorts one permutation in shared
// memory (bitonic network over the next power of two, padding keys sort last),
// so the result is bit-exact and independent of launch configuration.
#include "poet_internal.cuh"

namespace poet {
namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ __forceinline__ uint64_t splitmix64(uint64_t state) {
  uint64_t z = state + kGamma;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

constexpr int NT = 1024;

__global__ void __launch_bounds__(NT) draw_perm_kernel(uint64_t h, int d, int npow2, int32_t *__restrict__ perm) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint64_t *key = reinterpret_cast<uint64_t *>(smem_raw);
  uint32_t *idx = reinterpret_cast<uint32_t *>(key + npow2);
  for (int i = threadIdx.x; i < npow2; i += NT) {
    key[i] = i < d ? splitmix64(h + uint64_t(i) * kGamma) : ~0ull;
    idx[i] = uint32_t(i);
  }
  for (int size = 2; size <= npow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < (npow2 >> 1); t += NT) {
        const int lo = 2 * stride * (t / stride) + (t % stride);
        const int hi = lo + stride;
        const bool ascending = (lo & size) == 0;
        const uint64_t ka = key[lo], kb = key[hi];
        const uint32_t ia = idx[lo], ib = idx[hi];
        const bool a_gt_b = ka > kb || (ka == kb && ia > ib);
        if (a_gt_b == ascending) {
          key[lo] = kb; key[hi] = ka;
          idx[lo] = ib; idx[hi] = ia;
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < d; i += NT) perm[i] = int32_t(idx[i]);
}

}  // namespace

poet_status draw_perm_dev(uint64_t seed, int32_t layer_id, int32_t side, int32_t epoch, int32_t dim, int32_t *perm,
                          cudaStream_t st) {
  POET_REQUIRE(dim >= 1 && dim <= 16384, "poet_draw_perm: dim %d outside [1, 16384]", dim);
  POET_REQUIRE(perm != nullptr, "poet_draw_perm: perm is NULL");
  POET_REQUIRE(layer_id >= 0 && epoch >= 0 && (side == 0 || side == 1),
               "poet_draw_perm: need layer_id >= 0, epoch >= 0, side in {0,1}");
  const uint64_t inner = splitmix64((uint64_t(uint32_t(layer_id)) << 32) ^ (uint64_t(uint32_t(epoch)) << 1) ^
                                    uint64_t(side & 1));
  const uint64_t h = splitmix64(seed ^ inner);
  int npow2 = 1;
  while (npow2 < dim) npow2 <<= 1;
  if (npow2 < 2) npow2 = 2;
  const size_t smem = size_t(npow2) * (8 + 4);
  POET_CUDA_TRY(cudaFuncSetAttribute(draw_perm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
  draw_perm_kernel<<<1, NT, smem, st>>>(h, dim, npow2, perm);
  count_launch();
  return launch_status("draw_perm");
}

}  // namespace poet
