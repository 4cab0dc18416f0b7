// The optimizer step on the packed skew parameters: one AdamW update per
// element (decoupled weight decay, bias-corrected moments; Loshchilov & Hutter,
// "Decoupled Weight Decay Regularization").  The POET pages name no optimizer
// ([P1] Approach trains the primitives' parameters); this is the textbook
// update, applied to theta and its two moment buffers in place.
//
// HBM-bound: per element 16 B read (theta, grad, m, v) and 12 B written.  The
// grid covers whole waves of 148 SMs; four elements per thread move as 16-byte
// vectors when every buffer is 16-byte aligned.
#include <cmath>

#include "poet_internal.cuh"

namespace poet {
namespace {

__global__ void adamw_vec4_kernel(float4 *__restrict__ theta, const float4 *__restrict__ grad, float4 *__restrict__ m,
                                  float4 *__restrict__ v, int64_t n4, const AdamW h) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n4; i += int64_t(gridDim.x) * blockDim.x) {
    float4 t = theta[i], mm = m[i], vv = v[i];
    const float4 g = grad[i];
    adamw_one(t.x, g.x, mm.x, vv.x, h);
    adamw_one(t.y, g.y, mm.y, vv.y, h);
    adamw_one(t.z, g.z, mm.z, vv.z, h);
    adamw_one(t.w, g.w, mm.w, vv.w, h);
    theta[i] = t;
    m[i] = mm;
    v[i] = vv;
  }
}

__global__ void adamw_kernel(float *__restrict__ theta, const float *__restrict__ grad, float *__restrict__ m,
                             float *__restrict__ v, int64_t n, const AdamW h) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    adamw_one(theta[i], grad[i], m[i], v[i], h);
}

}  // namespace

AdamW adamw_of(float lr, float beta1, float beta2, float eps, float weight_decay, int32_t step) {
  AdamW h;
  h.lr = lr; h.beta1 = beta1; h.beta2 = beta2; h.eps = eps; h.wd = weight_decay;
  h.bc1 = float(1.0 - std::pow(double(beta1), double(step)));
  h.bc2 = float(1.0 - std::pow(double(beta2), double(step)));
  return h;
}

poet_status adamw_step(float *theta, const float *grad, float *m, float *v, int64_t n, float lr, float beta1,
                       float beta2, float eps, float weight_decay, int32_t step, cudaStream_t st) {
  if (n == 0) return POET_OK;
  const AdamW h = adamw_of(lr, beta1, beta2, eps, weight_decay, step);
  const bool vec = ((reinterpret_cast<uintptr_t>(theta) | reinterpret_cast<uintptr_t>(grad) |
                     reinterpret_cast<uintptr_t>(m) | reinterpret_cast<uintptr_t>(v)) & 15) == 0;
  const int threads = 256;
  const int64_t per_wave = int64_t(num_sms()) * 8;
  TraceScope ts("adamw", 0.0, double(n) * 28.0, st);
  if (vec) {
    const int64_t n4 = n / 4;
    if (n4 > 0) {
      const int64_t blocks = (n4 + threads - 1) / threads;
      adamw_vec4_kernel<<<int(blocks < per_wave ? blocks : per_wave), threads, 0, st>>>(
          reinterpret_cast<float4 *>(theta), reinterpret_cast<const float4 *>(grad), reinterpret_cast<float4 *>(m),
          reinterpret_cast<float4 *>(v), n4, h);
      count_launch();
      POET_TRY(launch_status("adamw"));
    }
    const int64_t tail = n - n4 * 4;
    if (tail > 0) {
      adamw_kernel<<<1, 32, 0, st>>>(theta + n4 * 4, grad + n4 * 4, m + n4 * 4, v + n4 * 4, tail, h);
      count_launch();
      POET_TRY(launch_status("adamw"));
    }
    return POET_OK;
  }
  const int64_t blocks = (n + threads - 1) / threads;
  adamw_kernel<<<int(blocks < per_wave ? blocks : per_wave), threads, 0, st>>>(theta, grad, m, v, n, h);
  count_launch();
  return launch_status("adamw");
}

}  // namespace poet
