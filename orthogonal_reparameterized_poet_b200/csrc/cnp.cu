// Cayley-Neumann parameterization of the orthogonal primitives (a1) and its
// gradient with respect to the packed skew parameters (a8).
//
// POET summary page, Approach and Limitations: each primitive is the Cayley
// map (I+Q)(I-Q)^-1 of a skew-symmetric Q with the inverse replaced by its
// Neumann series truncated after Q^k:  B = (I + Q)(I + Q + ... + Q^k).
//
// Forward, by Horner's rule on the series:
//   S_1 = I + Q,  S_{l+1} = I + Q S_l (l = 1..k-1),  B = (I + Q) S_k = S_1 S_k
// (k GEMMs of size^3; k = 0 gives B = I + Q).  Q and S_1..S_k are kept in
// the side state for the backward.
//
// Backward (reverse-mode through the same recurrence), G = dL/dB:
//   A_k = (I + Q)^T G = G - Q G            (Q^T = -Q)
//   dQ  = G S_k^T + sum_{l=k-1..0} A_{l+1} S_l^T,   A_l = Q^T A_{l+1} = -Q A_{l+1}
// with S_0 = I, then dtheta[a,c] = dQ[a,c] - dQ[c,a] (a < c) because
// Q[a,c] = theta and Q[c,a] = -theta.  2k GEMMs.
#include <vector>

#include "poet_internal.cuh"

namespace poet {
namespace {

// index of (a, c), a < c, in the row-major packed strict upper triangle
__device__ __forceinline__ int64_t packed_index(int a, int c, int size) {
  return int64_t(a) * size - int64_t(a) * (a + 1) / 2 + (c - a - 1);
}

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// Q and S_1 = I + Q (or B = I + Q when k == 0) for every primitive; padding is zero.
template <typename T>
__global__ void unpack_kernel(const float *__restrict__ theta, int nprim, int size, int ld,
                              T *__restrict__ Q, T *__restrict__ IplusQ) {
  const int64_t blk = int64_t(ld) * ld;
  const int64_t total = blk * nprim;
  const int64_t per = int64_t(size) * (size - 1) / 2;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int j = int(e / blk);
    const int a = int((e % blk) / ld), c = int(e % ld);
    float q = 0.f, eye = 0.f;
    if (a < size && c < size) {
      if (a < c) q = theta[j * per + packed_index(a, c, size)];
      else if (a > c) q = -theta[j * per + packed_index(c, a, size)];
      else eye = 1.f;
    }
    Q[e] = from_f<T>(q);
    IplusQ[e] = from_f<T>(q + eye);
  }
}

// dtheta[j][idx(a,c)] = D[a,c] - D[c,a] with D = dQ (+ A1 when given)
__global__ void pack_grad_kernel(const float *__restrict__ dQ, const float *__restrict__ A1, int nprim, int size,
                                 int ld, float *__restrict__ dtheta) {
  const int64_t blk = int64_t(ld) * ld;
  const int64_t per = int64_t(size) * (size - 1) / 2;
  const int64_t total = int64_t(nprim) * size * size;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int j = int(e / (int64_t(size) * size));
    const int a = int((e / size) % size), c = int(e % size);
    if (a >= c) continue;
    const int64_t ac = j * blk + int64_t(a) * ld + c, ca = j * blk + int64_t(c) * ld + a;
    float v = dQ[ac] - dQ[ca];
    if (A1) v += A1[ac] - A1[ca];
    dtheta[j * per + packed_index(a, c, size)] = v;
  }
}

constexpr int PACK_T = 32;  // tile edge of the transposing pack

// out[j][a][c] = G[j][a][c] for a, c < size (G dense [nprim][size][size]); zero padding up to ld
__global__ void pad_blocks_kernel(const float *__restrict__ G, int nprim, int size, int ld, float *__restrict__ out) {
  const int64_t blk = int64_t(ld) * ld;
  const int64_t total = blk * nprim;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t j = e / blk;
    const int a = int((e % blk) / ld), c = int(e % ld);
    out[e] = (a < size && c < size) ? G[(j * size + a) * size + c] : 0.f;
  }
}

__global__ void f32_to_bf16_kernel(const float *__restrict__ in, bf16 *__restrict__ out, int64_t n) {
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x)
    out[e] = __float2bfloat16_rn(in[e]);
}

int grid_for(int64_t n, int threads) {
  int64_t g = (n + threads - 1) / threads;
  const int64_t cap = int64_t(num_sms()) * 8;
  return int(g < 1 ? 1 : (g > cap ? cap : g));
}

// C_j = alpha * X_j Y_j (+ beta * Add_j) (+ diag I), all ld x ld primitives of one side.
// transY: false -> B(n, l) = Y[l][n] (Y read column-wise, "MN-major");
//         true  -> B(n, l) = Y[n][l] (C = X Y^T).
Gemm prim_gemm(const SideGeom &g, int dtype, const void *X, const void *Y, bool transY, const char *tag) {
  Gemm p;
  p.tag = tag;
  p.M = p.N = p.K = g.size;
  p.batch = g.nprim;
  p.dtype = dtype;
  p.A = X; p.a_m = g.ld; p.a_k = 1; p.a_b = g.blk_elems();
  p.B = Y;
  if (transY) { p.b_n = g.ld; p.b_k = 1; } else { p.b_n = 1; p.b_k = g.ld; }
  p.b_b = g.blk_elems();
  return p;
}

}  // namespace

poet_status pad_blocks(const float *G, const SideGeom &g, float *out, cudaStream_t st) {
  const int64_t n = g.all_elems();
  pad_blocks_kernel<<<grid_for(n, 256), 256, 0, st>>>(G, g.nprim, g.size, g.ld, out);
  count_launch();
  return launch_status("pad blocks");
}

size_t cnp_scratch_bytes(const SideGeom &g, int dtype) {
  const size_t f = align256(size_t(g.all_elems()) * 4);
  const size_t d = align256(size_t(g.all_elems()) * esize(dtype));
  // G operand copy (dtype), A ping-pong (f32 + dtype each), dQ (f32)
  return d + 2 * (f + d) + f;
}

poet_status cnp_forward(const poet_side *side, const SideGeom &g, int dtype, cudaStream_t st) {
  if (g.nprim == 0) return POET_OK;
  const StateLayout L = state_layout(g, dtype);
  char *base = static_cast<char *>(side->state);
  void *R = base + L.R, *Q = base + L.Q;
  const int64_t n = g.all_elems();
  void *first = g.k == 0 ? R : static_cast<void *>(base + L.S1);
  if (dtype == POET_BF16)
    unpack_kernel<bf16><<<grid_for(n, 256), 256, 0, st>>>(side->theta, g.nprim, g.size, g.ld, static_cast<bf16 *>(Q),
                                                          static_cast<bf16 *>(first));
  else
    unpack_kernel<float><<<grid_for(n, 256), 256, 0, st>>>(side->theta, g.nprim, g.size, g.ld, static_cast<float *>(Q),
                                                           static_cast<float *>(first));
  count_launch();
  POET_TRY(launch_status("cnp unpack"));
  for (int l = 1; l <= g.k; ++l) {
    void *S = base + L.S1 + size_t(l - 1) * L.term;
    Gemm p;
    if (l < g.k) {                               // S_{l+1} = I + Q S_l
      p = prim_gemm(g, dtype, Q, S, false, "cnp_fwd");
      p.diag = 1.f;
      p.outD = base + L.S1 + size_t(l) * L.term;
    } else {                                     // B = (I + Q) S_k = S_1 S_k
      p = prim_gemm(g, dtype, base + L.S1, S, false, "cnp_fwd");
      p.outD = R;
    }
    p.od_m = g.ld; p.od_b = g.blk_elems();
    POET_TRY(gemm_run(p, st));
  }
  return POET_OK;
}

poet_status cnp_backward(const poet_side *side, const SideGeom &g, int dtype, const float *G, float *dtheta,
                         void *scratch, cudaStream_t st) {
  if (g.nprim == 0 || g.size < 2) return POET_OK;
  const StateLayout L = state_layout(g, dtype);
  char *base = static_cast<char *>(side->state);
  const void *Q = base + L.Q;
  const int64_t n = g.all_elems();
  if (g.k == 0) {  // B = I + Q  ->  dQ = G
    pack_grad_kernel<<<grid_for(n, 256), 256, 0, st>>>(G, nullptr, g.nprim, g.size, g.ld, dtheta);
    count_launch();
    return launch_status("cnp pack");
  }
  const size_t fb = align256(size_t(n) * 4), db = align256(size_t(n) * esize(dtype));
  char *s = static_cast<char *>(scratch);
  const void *Gop;
  if (dtype == POET_BF16) {
    f32_to_bf16_kernel<<<grid_for(n, 256), 256, 0, st>>>(G, reinterpret_cast<bf16 *>(s), n);
    count_launch();
    POET_TRY(launch_status("cnp G to bf16"));
    Gop = s;
  } else {
    Gop = G;
  }
  s += db;
  float *Af[2] = {reinterpret_cast<float *>(s), reinterpret_cast<float *>(s + fb + db)};
  void *Ad[2] = {s + fb, s + 2 * fb + db};
  if (dtype != POET_BF16) { Ad[0] = Af[0]; Ad[1] = Af[1]; }
  float *dQ = reinterpret_cast<float *>(s + 2 * (fb + db));
  auto S = [&](int l) -> const void * { return base + L.S1 + size_t(l - 1) * L.term; };

  // A_k = G - Q G
  {
    Gemm p = prim_gemm(g, dtype, Q, Gop, false, "cnp_bwd");
    p.alpha = -1.f;
    p.add = G; p.add_dtype = POET_F32; p.add_m = g.ld; p.add_b = g.blk_elems(); p.beta = 1.f;
    p.outF = Af[0]; p.of_m = g.ld; p.of_b = g.blk_elems();
    if (dtype == POET_BF16) { p.outD = Ad[0]; p.od_m = g.ld; p.od_b = g.blk_elems(); }
    POET_TRY(gemm_run(p, st));
  }
  // dQ = G S_k^T
  {
    Gemm p = prim_gemm(g, dtype, Gop, S(g.k), true, "cnp_bwd");
    p.outF = dQ; p.of_m = g.ld; p.of_b = g.blk_elems();
    POET_TRY(gemm_run(p, st));
  }
  int cur = 0;  // A_{l+1} lives in slot cur
  for (int l = g.k - 1; l >= 1; --l) {
    {  // dQ += A_{l+1} S_l^T
      Gemm p = prim_gemm(g, dtype, Ad[cur], S(l), true, "cnp_bwd");
      p.add = dQ; p.add_dtype = POET_F32; p.add_m = g.ld; p.add_b = g.blk_elems(); p.beta = 1.f;
      p.outF = dQ; p.of_m = g.ld; p.of_b = g.blk_elems();
      POET_TRY(gemm_run(p, st));
    }
    {  // A_l = -Q A_{l+1}
      Gemm p = prim_gemm(g, dtype, Q, Ad[cur], false, "cnp_bwd");
      p.alpha = -1.f;
      p.outF = Af[cur ^ 1]; p.of_m = g.ld; p.of_b = g.blk_elems();
      if (dtype == POET_BF16) { p.outD = Ad[cur ^ 1]; p.od_m = g.ld; p.od_b = g.blk_elems(); }
      POET_TRY(gemm_run(p, st));
    }
    cur ^= 1;
  }
  // dQ += A_1 S_0^T = A_1, folded into the packing
  pack_grad_kernel<<<grid_for(n, 256), 256, 0, st>>>(dQ, Af[cur], g.nprim, g.size, g.ld, dtheta);
  count_launch();
  return launch_status("cnp pack");
}

// ---------------------------------------------------------------- many sides
//
// The element-wise steps of many sides (unpacking theta, rounding G to the
// operand type, packing dQ into dtheta) run as one launch per step over a
// table of up to kSidesMax sides; each block works inside one side.

namespace {

constexpr int kSidesMax = 64;
constexpr int kItems = 4;  // elements per thread in the element-wise many-side kernels

struct SideTable {
  int count;
  int64_t block_start[kSidesMax + 1];
  const void *src[kSidesMax];
  void *dst[kSidesMax];
  void *dst2[kSidesMax];
  int nprim[kSidesMax], size[kSidesMax], ld[kSidesMax];
  int terms[kSidesMax];          // pack: partial products summed onto src
  int64_t stride[kSidesMax];     // pack: floats between partial products
};

__device__ __forceinline__ int side_of_block(const SideTable &t) {
  int lo = 0, hi = t.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (t.block_start[mid] <= int64_t(blockIdx.x)) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// unpack_kernel for many sides: src = theta, dst = Q, dst2 = S_1 (or B when k = 0)
template <typename T>
__global__ void __launch_bounds__(256) unpack_many_kernel(const __grid_constant__ SideTable t) {
  const int i = side_of_block(t);
  const int size = t.size[i], ld = t.ld[i];
  const int64_t blk = int64_t(ld) * ld, total = blk * t.nprim[i];
  const int64_t per = int64_t(size) * (size - 1) / 2;
  const float *theta = static_cast<const float *>(t.src[i]);
  T *Q = static_cast<T *>(t.dst[i]);
  T *IplusQ = static_cast<T *>(t.dst2[i]);
  const int64_t e0 = (int64_t(blockIdx.x) - t.block_start[i]) * (256 * kItems);
  const int64_t e1 = e0 + 256 * kItems < total ? e0 + 256 * kItems : total;
  for (int64_t e = e0 + threadIdx.x; e < e1; e += 256) {
    const int j = int(e / blk);
    const int a = int((e % blk) / ld), c = int(e % ld);
    float q = 0.f, eye = 0.f;
    if (a < size && c < size) {
      if (a < c) q = theta[j * per + packed_index(a, c, size)];
      else if (a > c) q = -theta[j * per + packed_index(c, a, size)];
      else eye = 1.f;
    }
    Q[e] = from_f<T>(q);
    IplusQ[e] = from_f<T>(q + eye);
  }
}

// src = G (float), dst = its bf16 copy, nprim * ld * ld elements
__global__ void __launch_bounds__(256) round_many_kernel(const __grid_constant__ SideTable t) {
  const int i = side_of_block(t);
  const int64_t total = int64_t(t.ld[i]) * t.ld[i] * t.nprim[i];
  const float *G = static_cast<const float *>(t.src[i]);
  bf16 *out = static_cast<bf16 *>(t.dst[i]);
  const int64_t e0 = (int64_t(blockIdx.x) - t.block_start[i]) * (256 * kItems);
  const int64_t e1 = e0 + 256 * kItems < total ? e0 + 256 * kItems : total;
  for (int64_t e = e0 + threadIdx.x; e < e1; e += 256) out[e] = __float2bfloat16_rn(G[e]);
}

// dst = dtheta: dtheta[j][idx(a,c)] = D[a][c] - D[c][a] with D = src +
// sum_{t < terms} dst2 + t * stride (all float [nprim][ld][ld]).  One block
// per pair of 32 x 32 tiles (ta <= tc) of one primitive; both tiles are summed
// row-contiguously into shared memory and the transposed read comes from there.
__global__ void __launch_bounds__(256) pack_many_kernel(const __grid_constant__ SideTable t) {
  __shared__ float t1[PACK_T][PACK_T + 1], t2[PACK_T][PACK_T + 1];
  const int i = side_of_block(t);
  const int size = t.size[i], ld = t.ld[i];
  const int tiles = (size + PACK_T - 1) / PACK_T;
  const int pairs = tiles * (tiles + 1) / 2;
  const int64_t local = int64_t(blockIdx.x) - t.block_start[i];
  const int j = int(local / pairs);
  int ta = 0, rem = int(local % pairs);
  while (rem >= tiles - ta) { rem -= tiles - ta; ++ta; }
  const int tc = ta + rem;
  const int64_t off = int64_t(j) * ld * ld;
  const float *dQ = static_cast<const float *>(t.src[i]) + off;
  const int terms = t.terms[i];
  const float *P = terms ? static_cast<const float *>(t.dst2[i]) + off : nullptr;
  const int64_t stride = t.stride[i];
  float *dtheta = static_cast<float *>(t.dst[i]) + int64_t(j) * (int64_t(size) * (size - 1) / 2);
  const int x = threadIdx.x % PACK_T;
  for (int y = threadIdx.x / PACK_T; y < PACK_T; y += 256 / PACK_T) {
    const int a1 = ta * PACK_T + y, c1 = tc * PACK_T + x;
    const int a2 = tc * PACK_T + y, c2 = ta * PACK_T + x;
    float v1 = 0.f, v2 = 0.f;
    if (a1 < size && c1 < size) {
      const int64_t o = int64_t(a1) * ld + c1;
      v1 = dQ[o];
      for (int q = 0; q < terms; ++q) v1 += P[q * stride + o];
    }
    if (a2 < size && c2 < size) {
      const int64_t o = int64_t(a2) * ld + c2;
      v2 = dQ[o];
      for (int q = 0; q < terms; ++q) v2 += P[q * stride + o];
    }
    t1[y][x] = v1;
    t2[y][x] = v2;
  }
  __syncthreads();
  for (int y = threadIdx.x / PACK_T; y < PACK_T; y += 256 / PACK_T) {
    const int a = ta * PACK_T + y, c = tc * PACK_T + x;
    if (a < c && c < size) dtheta[packed_index(a, c, size)] = t1[y][x] - t2[x][y];
  }
}

// Fill a table with the sides of idx[0..n) (blocks per side from `blocks`) and launch.
template <typename Launch, typename Blocks>
poet_status many_launch(const std::vector<int> &idx, Blocks blocks, SideTable &t, Launch launch) {
  for (size_t c0 = 0; c0 < idx.size(); c0 += kSidesMax) {
    const int n = int(idx.size() - c0 < size_t(kSidesMax) ? idx.size() - c0 : size_t(kSidesMax));
    t.count = n;
    t.block_start[0] = 0;
    for (int q = 0; q < n; ++q) t.block_start[q + 1] = t.block_start[q] + blocks(idx[c0 + q], q);
    if (t.block_start[n] == 0) continue;
    POET_TRY(launch(t, int(c0), n));
  }
  return POET_OK;
}

}  // namespace

poet_status cnp_forward_many(const poet_side *sides, const SideGeom *geoms, int count, int dtype, cudaStream_t st) {
  std::vector<int> idx;
  int kmax = 0;
  for (int i = 0; i < count; ++i) {
    if (geoms[i].nprim == 0) continue;
    idx.push_back(i);
    if (geoms[i].k > kmax) kmax = geoms[i].k;
  }
  // theta -> Q and S_1 (or B when k = 0), every side in one launch
  static thread_local SideTable t;
  POET_TRY(many_launch(idx, [&](int i, int q) {
    const SideGeom &g = geoms[i];
    const StateLayout L = state_layout(g, dtype);
    char *base = static_cast<char *>(sides[i].state);
    t.src[q] = sides[i].theta;
    t.dst[q] = base + L.Q;
    t.dst2[q] = g.k == 0 ? base + L.R : base + L.S1;
    t.nprim[q] = g.nprim; t.size[q] = g.size; t.ld[q] = g.ld;
    return (g.all_elems() + 256 * kItems - 1) / (256 * kItems);
  }, t, [&](const SideTable &tt, int, int) {
    const int blocks = int(tt.block_start[tt.count]);
    if (dtype == POET_BF16) unpack_many_kernel<bf16><<<blocks, 256, 0, st>>>(tt);
    else unpack_many_kernel<float><<<blocks, 256, 0, st>>>(tt);
    count_launch();
    return launch_status("cnp unpack");
  }));
  std::vector<Gemm> gs;
  for (int l = 1; l <= kmax; ++l) {
    gs.clear();
    for (int i : idx) {
      const SideGeom &g = geoms[i];
      if (g.k < l) continue;
      const StateLayout L = state_layout(g, dtype);
      char *base = static_cast<char *>(sides[i].state);
      void *S = base + L.S1 + size_t(l - 1) * L.term;
      Gemm p;
      if (l < g.k) {  // S_{l+1} = I + Q S_l
        p = prim_gemm(g, dtype, base + L.Q, S, false, "cnp_fwd");
        p.diag = 1.f;
        p.outD = base + L.S1 + size_t(l) * L.term;
      } else {        // B = (I + Q) S_k = S_1 S_k
        p = prim_gemm(g, dtype, base + L.S1, S, false, "cnp_fwd");
        p.outD = base + L.R;
      }
      p.od_m = g.ld; p.od_b = g.blk_elems();
      gs.push_back(p);
    }
    POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  }
  return POET_OK;
}

// Many sides: the same gradient reorganised for grouped launches.  The chain
// A_k = S_1^T G, A_l = -Q A_{l+1} takes one grouped launch per order (all
// sides; S_1^T is read straight from the stored S_1 as a transposed operand).
// One more launch forms every partial product P_k = G S_k^T,
// P_l = A_{l+1} S_l^T (l < k) of every side, each into its own float buffer,
// and one launch packs D - D^T into dtheta with D = A_1 + P_1 + ... + P_k.
// Every product writes one plain output, which the tensor-core engine stores
// through its staged epilogue.
size_t cnp_many_scratch_bytes(const SideGeom &g, int dtype) {
  if (g.nprim == 0 || g.size < 2 || g.k == 0) return 0;
  const size_t f = align256(size_t(g.all_elems()) * 4);
  const size_t d = align256(size_t(g.all_elems()) * esize(dtype));
  // G operand copy, A_k..A_2 (dtype), A_1 (f32), P_1..P_k (f32)
  return d + size_t(g.k - 1) * d + f + size_t(g.k) * f;
}

poet_status cnp_backward_many(const poet_side *sides, const SideGeom *geoms, int count, int dtype,
                              const float *const *G, float *const *dtheta, void *const *scratch, cudaStream_t st) {
  struct Work {
    const void *Q, *Gop;
    const char *S1;
    size_t term;
    char *X;   // A_{l+1} for l = 1..k-1 at X + (l-1) * xb (dtype)
    size_t xb;
    float *A1;  // A_1
    float *P;   // P_l at P + (l-1) * pstride
    int64_t pstride;
  };
  std::vector<Work> w(count);
  std::vector<int> chain, all;  // sides with k >= 1; every side with parameters
  int kmax = 0;
  for (int i = 0; i < count; ++i) {
    const SideGeom &g = geoms[i];
    if (g.nprim == 0 || g.size < 2) continue;
    all.push_back(i);
    if (g.k == 0) continue;  // B = I + Q: dQ = G
    chain.push_back(i);
    const StateLayout L = state_layout(g, dtype);
    const char *base = static_cast<const char *>(sides[i].state);
    const size_t db = align256(size_t(g.all_elems()) * esize(dtype));
    const size_t fb = align256(size_t(g.all_elems()) * 4);
    char *s = static_cast<char *>(scratch[i]);
    Work &x = w[i];
    x.Q = base + L.Q;
    x.S1 = base + L.S1;
    x.term = L.term;
    x.Gop = dtype == POET_BF16 ? static_cast<const void *>(s) : static_cast<const void *>(G[i]);
    x.X = s + db;
    x.xb = db;
    x.A1 = reinterpret_cast<float *>(s + size_t(g.k) * db);
    x.P = reinterpret_cast<float *>(s + size_t(g.k) * db + fb);
    x.pstride = int64_t(fb / 4);
    if (g.k > kmax) kmax = g.k;
  }
  static thread_local SideTable t;
  if (dtype == POET_BF16) {  // G rounded to the operand type, every side in one launch
    POET_TRY(many_launch(chain, [&](int i, int q) {
      const SideGeom &g = geoms[i];
      t.src[q] = G[i];
      t.dst[q] = const_cast<void *>(w[i].Gop);
      t.nprim[q] = g.nprim; t.size[q] = g.size; t.ld[q] = g.ld;
      return (g.all_elems() + 256 * kItems - 1) / (256 * kItems);
    }, t, [&](const SideTable &tt, int, int) {
      round_many_kernel<<<int(tt.block_start[tt.count]), 256, 0, st>>>(tt);
      count_launch();
      return launch_status("cnp G to bf16");
    }));
  }
  // X_l, the left factor of P_l: G for l = k, else A_{l+1}
  auto Xop = [&](int i, int l) -> const void * {
    return l == geoms[i].k ? w[i].Gop : static_cast<const void *>(w[i].X + size_t(l - 1) * w[i].xb);
  };
  std::vector<Gemm> gs;
  // the chain, one order per launch (sides with a smaller k finish early)
  for (int step = 0; step < kmax; ++step) {
    gs.clear();
    for (int i : chain) {
      const SideGeom &g = geoms[i];
      const int l = g.k - step;  // order of the A made now
      if (l < 1) continue;
      const Work &x = w[i];
      Gemm a;
      if (l == g.k) {  // A_k = S_1^T G: S_1 read transposed (M contiguous)
        a = prim_gemm(g, dtype, x.S1, x.Gop, false, "cnp_bwd");
        a.a_m = 1; a.a_k = g.ld;
      } else {         // A_l = -Q A_{l+1}
        a = prim_gemm(g, dtype, x.Q, Xop(i, l), false, "cnp_bwd");
        a.alpha = -1.f;
      }
      if (l == 1) {
        a.outF = x.A1; a.of_m = g.ld; a.of_b = g.blk_elems();
      } else if (dtype == POET_BF16) {
        a.outD = x.X + size_t(l - 2) * x.xb; a.od_m = g.ld; a.od_b = g.blk_elems();
      } else {
        a.outF = reinterpret_cast<float *>(x.X + size_t(l - 2) * x.xb); a.of_m = g.ld; a.of_b = g.blk_elems();
      }
      gs.push_back(a);
    }
    POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  }
  // P_l = X_l S_l^T for every order of every side, in one launch
  gs.clear();
  for (int i : chain) {
    const SideGeom &g = geoms[i];
    for (int l = g.k; l >= 1; --l) {
      Gemm p = prim_gemm(g, dtype, Xop(i, l), w[i].S1 + size_t(l - 1) * w[i].term, true, "cnp_bwd");
      p.outF = w[i].P + (l - 1) * w[i].pstride; p.of_m = g.ld; p.of_b = g.blk_elems();
      gs.push_back(p);
    }
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  // dtheta = D - D^T with D = A_1 + sum P_l (k = 0: D = G), every side in one launch
  return many_launch(all, [&](int i, int q) {
    const SideGeom &g = geoms[i];
    t.src[q] = g.k == 0 ? static_cast<const void *>(G[i]) : static_cast<const void *>(w[i].A1);
    t.dst2[q] = g.k == 0 ? nullptr : static_cast<void *>(w[i].P);
    t.terms[q] = g.k;
    t.stride[q] = g.k == 0 ? 0 : w[i].pstride;
    t.dst[q] = dtheta[i];
    t.nprim[q] = g.nprim; t.size[q] = g.size; t.ld[q] = g.ld;
    const int64_t tiles = (g.size + PACK_T - 1) / PACK_T;
    return int64_t(g.nprim) * tiles * (tiles + 1) / 2;
  }, t, [&](const SideTable &tt, int, int) {
    pack_many_kernel<<<int(tt.block_start[tt.count]), 256, 0, st>>>(tt);
    count_launch();
    return launch_status("cnp pack");
  });
}

}  // namespace poet
