// tcgen05 (5th-generation tensor core) engine of the batched GEMM.
#include "poet_internal.cuh"

namespace poet {

bool gemm_tc_enabled() { return false; }
bool gemm_tc_supported(const Gemm &) { return false; }
poet_status gemm_tc(const Gemm &g, cudaStream_t st) { return gemm_simt(g, st); }

}  // namespace poet
