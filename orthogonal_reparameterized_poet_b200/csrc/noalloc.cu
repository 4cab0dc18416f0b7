// poet_cayley_neumann_grad_noalloc: the packed-skew gradient of one side
// (the same computation as poet_cayley_neumann_grad) for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where a cudaMalloc is not available or not
// allowed -- a host framework that owns and pre-partitions all device memory
// and hands out none, a plug-in whose host forbids device allocations, or a
// caller that cannot size and keep a workspace around between calls.  Such a
// caller still passes its inputs and outputs (theta, the side state, G and
// dtheta); the scratch comes from a fixed array compiled into this library.
//
// The scratch is one file-scope device array of kNoAllocScratchBytes
// (32 MiB).  Every GPU that loads this library holds it until the process
// exits, and every call on a device shares it: two calls whose work overlaps
// on the GPU (different streams, or different host threads) race on it, so
// order them on one stream.  It keeps the previous call's contents; nothing in
// it has to start at zero, because every call writes each scratch value before
// reading it.  No call here allocates: no cudaMalloc, cudaFree or allocating
// library routine.
#include <mutex>

#include "poet_internal.cuh"

namespace poet {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
poet_status scratch_address(void **out) {
  static std::mutex mu;
  static void *addr[64] = {};
  int dev = 0;
  POET_CUDA_TRY(cudaGetDevice(&dev));
  POET_REQUIRE(dev >= 0 && dev < 64, "poet_cayley_neumann_grad_noalloc: device %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_error("poet_cayley_neumann_grad_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      return POET_ECUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return POET_OK;
}

}  // namespace
}  // namespace poet

using namespace poet;

extern "C" {

poet_status poet_cayley_neumann_grad_noalloc(const poet_side *side, int32_t dtype, const float *G, float *dtheta,
                                             poet_stream stream) {
  CallRange nvtx_range("poet_cayley_neumann_grad_noalloc");
  clear_error();
  SideGeom g;
  POET_REQUIRE(side_geom(side, &g), "poet_cayley_neumann_grad_noalloc: malformed side");
  POET_REQUIRE(dtype == POET_F32 || dtype == POET_BF16, "poet_cayley_neumann_grad_noalloc: bad dtype %d", dtype);
  const size_t need = poet_side_workspace_bytes(side, dtype);
  POET_REQUIRE(need <= kNoAllocScratchBytes,
               "poet_cayley_neumann_grad_noalloc: this side needs %zu bytes of scratch, more than the %zu built in; "
               "use poet_cayley_neumann_grad with a caller workspace",
               need, kNoAllocScratchBytes);
  void *scratch = nullptr;
  POET_TRY(scratch_address(&scratch));
  return poet_cayley_neumann_grad(side, dtype, G, dtheta, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
