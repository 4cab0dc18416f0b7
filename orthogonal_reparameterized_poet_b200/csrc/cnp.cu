// Cayley-Neumann parameterization of the orthogonal primitives (a1) and its
// gradient with respect to the packed skew parameters (a8).
//
// POET summary page, Approach and Limitations: each primitive is the Cayley
// map (I+Q)(I-Q)^-1 of a skew-symmetric Q with the inverse replaced by its
// Neumann series truncated after Q^k:  B = (I + Q)(I + Q + ... + Q^k).
//
// Order 4 (the order the pages' LLaMA runs use) is evaluated by powers of
// S = Q^2, with T = S^2:  B = Q C + D0,  C = 2I + 2S + T,  D0 = I + 2S + 2T,
// as three GEMMs whose epilogues add the rest:
//   S = Q Q,   C' = S S + 2S,   B = (Q + 2I) C' + 2Q - 2S + I
// with C' = C - 2I (the last equals Q C + D0).  No stored matrix carries a
// multiple of I (Q + 2I differs from Q only on its zero diagonal, where 2 is
// exact), so bf16 storage rounds the small parts only: a stored C, whose
// diagonal is near 2, would put its rounding, doubled, on B's diagonal.  The
// state keeps Q, Q + 2I, S and C'.  Its
// gradient, G = dL/dB: theta enters Q antisymmetrically (Q[a,c] = theta =
// -Q[c,a]), so only the antisymmetric part of dL/dQ reaches dtheta; S, T and C
// are symmetric, so only the symmetric parts of dL/dS and dL/dT matter:
//   dT_s = sym(2G - QG),  W = dT_s S,  dS_s = sym(2G - 2QG) + W + W^T,
//   D = G C - 2 dS_s Q,  dtheta[a,c] = D[a,c] - D[c,a]   (sym(X) = (X + X^T)/2)
// evaluated as four GEMMs (three grouped launches) with the sums in their
// epilogues:  U = G - Q G and G C = G C' + 2G;  V = dT_s S + U with
// dT_s = sym(G + U);  D = G C - 2 (V + V^T) Q;  so the element-wise passes
// between them read one or two matrices each.
//
// Every other order, by Horner's rule on the series:
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
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }

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

}  // namespace

// Order 4 is evaluated by powers of S = Q^2 (see the top of this file).
bool by_powers(const SideGeom &g) { return g.k == 4; }

namespace {

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
  return cnp_forward_many(side, &g, 1, dtype, st);  // one code path: a single side is a list of one
}

poet_status cnp_backward(const poet_side *side, const SideGeom &g, int dtype, const float *G, float *dtheta,
                         void *scratch, cudaStream_t st) {
  if (g.nprim == 0 || g.size < 2) return POET_OK;
  if (by_powers(g)) {  // order 4: the grouped path on a list of one side (cnp_scratch_bytes >= its scratch)
    void *sc = scratch;
    float *dth = dtheta;
    return cnp_backward_many(side, &g, 1, dtype, &G, &dth, &sc, st);
  }
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
// operand type, the symmetric combinations of the order-4 gradient, packing
// dQ into dtheta) run as one launch per step over a table of up to kSidesMax
// sides; each block works inside one side.

namespace {

constexpr int kSidesMax = 64;

struct SideTable {
  int count;
  int64_t block_start[kSidesMax + 1];
  const void *src[kSidesMax];
  const void *src2[kSidesMax];
  void *dst[kSidesMax];
  void *dst2[kSidesMax];
  void *dst3[kSidesMax];
  int nprim[kSidesMax], size[kSidesMax], ld[kSidesMax];
  int terms[kSidesMax];          // pack: partial products summed onto src
  int64_t stride[kSidesMax];     // pack: floats between partial products
  float coef[kSidesMax];         // pack: weight of the partial products
  float *theta[kSidesMax];       // pack with an optimizer step: parameters, first and second moments
  float *m1[kSidesMax];
  float *m2[kSidesMax];
};
static_assert(sizeof(SideTable) <= 32000, "side table exceeds the kernel parameter limit");

__device__ __forceinline__ int side_of_block(const SideTable &t) {
  int lo = 0, hi = t.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (t.block_start[mid] <= int64_t(blockIdx.x)) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Tile pair (ta <= tc, 32 x 32 tiles over [0, span)) of primitive j handled by
// this block: the pairs of a primitive are numbered row by row (ta, then tc),
// and the row of a number comes from the quadratic formula, then is corrected
// by one step where float rounding put it off.
struct TilePair {
  int j, ta, tc;
};
__device__ __forceinline__ TilePair tile_pair(const SideTable &t, int i, int span) {
  const int tiles = (span + PACK_T - 1) / PACK_T;
  const int pairs = tiles * (tiles + 1) / 2;
  const int local = int(int64_t(blockIdx.x) - t.block_start[i]);  // 32-bit division below
  TilePair p;
  p.j = local / pairs;
  const int r = local - p.j * pairs;
  // row ta starts at start(ta) = ta * tiles - ta (ta - 1) / 2
  const float b = 2.f * float(tiles) + 1.f;
  int ta = int(0.5f * (b - sqrtf(fmaxf(b * b - 8.f * float(r), 0.f))));
  ta = ta < 0 ? 0 : (ta > tiles - 1 ? tiles - 1 : ta);
  while (ta + 1 < tiles && (ta + 1) * tiles - (ta + 1) * ta / 2 <= r) ++ta;
  while (ta > 0 && ta * tiles - ta * (ta - 1) / 2 > r) --ta;
  p.ta = ta;
  p.tc = ta + (r - (ta * tiles - ta * (ta - 1) / 2));
  return p;
}

// src = theta, dst = Q, dst2 = Q + coef I (Horner's S_1 = I + Q, or B = I + Q
// when k = 0, with coef 1; Q + 2I for order 4; nullptr: not written), dst3 = B
// whose padding (rows or columns >= size) is zeroed (nullptr: none).  Padding
// of Q and dst2 is zero.  One block per pair of 32 x 32 tiles (ta <= tc) over
// [0, ld): theta of the upper tile is read row-contiguously into shared
// memory, and the tile and its mirror (negated, transposed) are written.
template <typename T>
__global__ void __launch_bounds__(256) unpack_many_kernel(const __grid_constant__ SideTable t) {
  __shared__ float u[PACK_T][PACK_T + 1];
  const int i = side_of_block(t);
  const int size = t.size[i], ld = t.ld[i];
  const TilePair tp = tile_pair(t, i, ld);
  const int64_t per = int64_t(size) * (size - 1) / 2;
  const float *theta = static_cast<const float *>(t.src[i]) + int64_t(tp.j) * per;
  const int64_t off = int64_t(tp.j) * ld * ld;
  T *Q = static_cast<T *>(t.dst[i]) + off;
  T *Q2 = t.dst2[i] ? static_cast<T *>(t.dst2[i]) + off : nullptr;
  T *Bpad = t.dst3[i] ? static_cast<T *>(t.dst3[i]) + off : nullptr;
  const float coef = t.coef[i];
  const int x = threadIdx.x % PACK_T;
  // u[y][x] = Q[ta*32+y][tc*32+x] where a < c < size, else 0
  for (int y = threadIdx.x / PACK_T; y < PACK_T; y += 256 / PACK_T) {
    const int a = tp.ta * PACK_T + y, c = tp.tc * PACK_T + x;
    u[y][x] = (a < c && c < size) ? theta[packed_index(a, c, size)] : 0.f;
  }
  __syncthreads();
  for (int y = threadIdx.x / PACK_T; y < PACK_T; y += 256 / PACK_T) {
    {  // tile (ta, tc); on the diagonal tile the lower part is the mirror
      const int a = tp.ta * PACK_T + y, c = tp.tc * PACK_T + x;
      if (a < ld && c < ld) {
        const float q = (tp.ta == tp.tc && a > c) ? -u[x][y] : u[y][x];
        const float eye = (a == c && a < size) ? 1.f : 0.f;
        const int64_t e = int64_t(a) * ld + c;
        Q[e] = from_f<T>(q);
        if (Q2) Q2[e] = from_f<T>(q + coef * eye);
        if (Bpad && (a >= size || c >= size)) Bpad[e] = from_f<T>(0.f);
      }
    }
    if (tp.ta != tp.tc) {  // tile (tc, ta): Q[a][c] = -Q[c][a]
      const int a = tp.tc * PACK_T + y, c = tp.ta * PACK_T + x;
      if (a < ld && c < ld) {
        const float q = -u[x][y];
        const int64_t e = int64_t(a) * ld + c;
        Q[e] = from_f<T>(q);
        if (Q2) Q2[e] = from_f<T>(q);
        if (Bpad && (a >= size || c >= size)) Bpad[e] = from_f<T>(0.f);
      }
    }
  }
}

// src = G (float), dst = its bf16 copy, nprim * ld * ld elements; eight per
// thread, as two 16-byte loads and one 16-byte store where both are aligned
constexpr int kRoundItems = 8;
__global__ void __launch_bounds__(256) round_many_kernel(const __grid_constant__ SideTable t) {
  const int i = side_of_block(t);
  const int64_t total = int64_t(t.ld[i]) * t.ld[i] * t.nprim[i];
  const float *G = static_cast<const float *>(t.src[i]);
  bf16 *out = static_cast<bf16 *>(t.dst[i]);
  const bool vec = ((reinterpret_cast<uintptr_t>(G) | reinterpret_cast<uintptr_t>(out)) & 15) == 0;
  const int64_t e = (int64_t(blockIdx.x) - t.block_start[i]) * (256 * kRoundItems) + int64_t(threadIdx.x) * kRoundItems;
  if (vec && e + kRoundItems <= total) {
    const float4 lo = *reinterpret_cast<const float4 *>(G + e), hi = *reinterpret_cast<const float4 *>(G + e + 4);
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(lo.x, lo.y), h1 = __floats2bfloat162_rn(lo.z, lo.w);
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(hi.x, hi.y), h3 = __floats2bfloat162_rn(hi.z, hi.w);
    uint4 pk;
    pk.x = *reinterpret_cast<const uint32_t *>(&h0);
    pk.y = *reinterpret_cast<const uint32_t *>(&h1);
    pk.z = *reinterpret_cast<const uint32_t *>(&h2);
    pk.w = *reinterpret_cast<const uint32_t *>(&h3);
    *reinterpret_cast<uint4 *>(out + e) = pk;
  } else {
    for (int64_t q = e; q < e + kRoundItems && q < total; ++q) out[q] = __float2bfloat16_rn(G[q]);
  }
}

// The tile-pair kernels below give each thread four consecutive columns of
// one row of a 32 x 32 tile: threadIdx.x / 8 is the row, (threadIdx.x % 8) * 4
// the first column, so that a warp reads four rows x 128 contiguous bytes.

// v[e] = sum_q cf_q X_q[row][col + e] for e < 4 (0 outside [0, size)^2); one
// 16-byte load per matrix when the four columns are inside and aligned.
__device__ __forceinline__ void load_quad(const float *const *X, const float *cf, int nx, int row, int col, int size,
                                          int ld, bool vec, float (&v)[4]) {
  v[0] = v[1] = v[2] = v[3] = 0.f;
  if (row >= size || col >= size) return;
  const int64_t o = int64_t(row) * ld + col;
  for (int q = 0; q < nx; ++q) {
    if (!X[q]) continue;
    if (vec && col + 4 <= size) {
      const float4 f = *reinterpret_cast<const float4 *>(X[q] + o);
      v[0] += cf[q] * f.x; v[1] += cf[q] * f.y; v[2] += cf[q] * f.z; v[3] += cf[q] * f.w;
    } else {
      for (int e = 0; e < 4 && col + e < size; ++e) v[e] += cf[q] * X[q][o + e];
    }
  }
}

// out[row][col + e] = v[e] for the columns inside [0, size): one 8-byte
// (bf16) or 16-byte (float) store when all four are inside and aligned.
template <typename T>
__device__ __forceinline__ void store_quad(T *out, int row, int col, int size, int ld, bool vec, const float (&v)[4]) {
  if (row >= size || col >= size) return;
  T *o = out + int64_t(row) * ld + col;
  if (vec && col + 4 <= size) {
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t *>(&h0);
      pk.y = *reinterpret_cast<const uint32_t *>(&h1);
      *reinterpret_cast<uint2 *>(o) = pk;
    } else {
      *reinterpret_cast<float4 *>(o) = make_float4(v[0], v[1], v[2], v[3]);
    }
  } else {
    for (int e = 0; e < 4 && col + e < size; ++e) o[e] = from_f<T>(v[e]);
  }
}

// Order-4 gradient, symmetric combinations: dst = c0 (X_0 + X_0^T) + c1 (X_1 +
// X_1^T) over X_0 = src and X_1 = src2 (float [nprim][ld][ld]; src2 may be
// nullptr), in the operand type.  One block per pair of 32 x 32 tiles
// (ta <= tc) of one primitive; both tiles of every input are read
// row-contiguously into shared memory and both output tiles are written.
template <typename T>
__global__ void __launch_bounds__(256) sym_many_kernel(const __grid_constant__ SideTable t, float c0, float c1) {
  __shared__ float u1[PACK_T][PACK_T + 1], u2[PACK_T][PACK_T + 1];
  const int i = side_of_block(t);
  const int size = t.size[i], ld = t.ld[i];
  const TilePair tp = tile_pair(t, i, size);
  const int64_t off = int64_t(tp.j) * ld * ld;
  const float *X[2] = {static_cast<const float *>(t.src[i]) + off,
                       t.src2[i] ? static_cast<const float *>(t.src2[i]) + off : nullptr};
  const float cf[2] = {c0, c1};
  T *out = static_cast<T *>(t.dst[i]) + off;
  const bool vec = ((reinterpret_cast<uintptr_t>(X[0]) | reinterpret_cast<uintptr_t>(X[1]) |
                     reinterpret_cast<uintptr_t>(out)) & 15) == 0;
  const int y = threadIdx.x / 8, x = (threadIdx.x % 8) * 4;
  // u1[y][x] = sum c_q X_q[ta*32+y][tc*32+x],  u2[y][x] = sum c_q X_q[tc*32+y][ta*32+x]
  float v1[4], v2[4];
  load_quad(X, cf, 2, tp.ta * PACK_T + y, tp.tc * PACK_T + x, size, ld, vec, v1);
  load_quad(X, cf, 2, tp.tc * PACK_T + y, tp.ta * PACK_T + x, size, ld, vec, v2);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    u1[y][x + e] = v1[e];
    u2[y][x + e] = v2[e];
  }
  __syncthreads();
  // out[ta*32+y][tc*32+x] = u1[y][x] + u2[x][y];  out[tc*32+y][ta*32+x] = u2[y][x] + u1[x][y]
  float w1[4], w2[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    w1[e] = u1[y][x + e] + u2[x + e][y];
    w2[e] = u2[y][x + e] + u1[x + e][y];
  }
  store_quad(out, tp.ta * PACK_T + y, tp.tc * PACK_T + x, size, ld, vec, w1);
  if (tp.ta != tp.tc) store_quad(out, tp.tc * PACK_T + y, tp.ta * PACK_T + x, size, ld, vec, w2);
}

// dst = dtheta: dtheta[j][idx(a,c)] = D[a][c] - D[c][a] with D = src +
// coef * sum_{q < terms} dst2 + q * stride (all float [nprim][ld][ld]).  One
// block per pair of 32 x 32 tiles (ta <= tc) of one primitive; both tiles are
// summed row-contiguously into shared memory and the transposed read comes
// from there.  With ADAM, each parameter's gradient also drives its AdamW
// step (theta, m1, m2 updated in place; dst may be nullptr).
template <bool ADAM>
__global__ void __launch_bounds__(256) pack_many_kernel(const __grid_constant__ SideTable t, const AdamW h) {
  __shared__ float t1[PACK_T][PACK_T + 1], t2[PACK_T][PACK_T + 1];
  const int i = side_of_block(t);
  const int size = t.size[i], ld = t.ld[i];
  const TilePair tp = tile_pair(t, i, size);
  const int64_t off = int64_t(tp.j) * ld * ld;
  const float *dQ = static_cast<const float *>(t.src[i]) + off;
  const int terms = t.terms[i];
  const float coef = t.coef[i];
  const float *P = terms ? static_cast<const float *>(t.dst2[i]) + off : nullptr;
  const int64_t stride = t.stride[i];
  float *dtheta = t.dst[i] ? static_cast<float *>(t.dst[i]) + int64_t(tp.j) * (int64_t(size) * (size - 1) / 2)
                           : nullptr;
  const bool vec = ((reinterpret_cast<uintptr_t>(dQ) | reinterpret_cast<uintptr_t>(P)) & 15) == 0 && stride % 4 == 0;
  const int y = threadIdx.x / 8, x = (threadIdx.x % 8) * 4;
  // t1[y][x] = D[ta*32+y][tc*32+x],  t2[y][x] = D[tc*32+y][ta*32+x]
  auto load_d = [&](int row, int col, float (&v)[4]) {
    const float *one[1] = {dQ};
    const float cf1[1] = {1.f};
    load_quad(one, cf1, 1, row, col, size, ld, vec, v);
    if (terms == 0) return;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int q = 0; q < terms; ++q) {
      const float *pq[1] = {P + q * stride};
      float w[4];
      load_quad(pq, cf1, 1, row, col, size, ld, vec, w);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] += w[e];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] += coef * acc[e];
  };
  float v1[4], v2[4];
  load_d(tp.ta * PACK_T + y, tp.tc * PACK_T + x, v1);
  load_d(tp.tc * PACK_T + y, tp.ta * PACK_T + x, v2);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    t1[y][x + e] = v1[e];
    t2[y][x + e] = v2[e];
  }
  __syncthreads();
  const int64_t pbase = int64_t(tp.j) * (int64_t(size) * (size - 1) / 2);
  const int a = tp.ta * PACK_T + y;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c = tp.tc * PACK_T + x + e;
    if (a < c && c < size) {
      const int64_t idx = packed_index(a, c, size);
      const float g = t1[y][x + e] - t2[x + e][y];
      if (!ADAM || t.dst[i]) dtheta[idx] = g;
      if constexpr (ADAM) {
        const int64_t q = pbase + idx;
        float th = t.theta[i][q], mm = t.m1[i][q], vv = t.m2[i][q];
        adamw_one(th, g, mm, vv, h);
        t.theta[i][q] = th;
        t.m1[i][q] = mm;
        t.m2[i][q] = vv;
      }
    }
  }
}

// Logical elements (nprim * size^2) of the sides in a table, for the trace's bytes.
double table_elems(const SideTable &t) {
  double e = 0.0;
  for (int q = 0; q < t.count; ++q) e += double(t.nprim[q]) * t.size[q] * t.size[q];
  return e;
}

int64_t round_blocks(const SideGeom &g) { return (g.all_elems() + 256 * kRoundItems - 1) / (256 * kRoundItems); }
// tile pairs (ta <= tc) over [0, span) of every primitive
int64_t pairs_over(const SideGeom &g, int span) {
  const int64_t tiles = (span + PACK_T - 1) / PACK_T;
  return int64_t(g.nprim) * tiles * (tiles + 1) / 2;
}
int64_t pair_blocks(const SideGeom &g) { return pairs_over(g, g.size); }

// Fill a table with the sides of idx[0..n) (blocks per side from `blocks`) and launch.
template <typename Launch, typename Blocks>
poet_status many_launch(const std::vector<int> &idx, Blocks blocks, SideTable &t, Launch launch) {
  for (size_t c0 = 0; c0 < idx.size(); c0 += kSidesMax) {
    const int n = int(idx.size() - c0 < size_t(kSidesMax) ? idx.size() - c0 : size_t(kSidesMax));
    t.count = n;
    t.block_start[0] = 0;
    for (int q = 0; q < n; ++q) {
      t.src[q] = t.src2[q] = nullptr;
      t.dst[q] = t.dst2[q] = t.dst3[q] = nullptr;
      t.theta[q] = t.m1[q] = t.m2[q] = nullptr;
      t.terms[q] = 0;
      t.stride[q] = 0;
      t.coef[q] = 1.f;
      t.block_start[q + 1] = t.block_start[q] + blocks(idx[c0 + q], q);
    }
    if (t.block_start[n] == 0) continue;
    POET_TRY(launch(t, int(c0), n));
  }
  return POET_OK;
}

// Byte offsets of the order-4 terms in a side state: Q + 2I, S and C' = C - 2I
// take the slots of S_1..S_3.
struct PowersLayout {
  size_t Q2, S, C;
};
PowersLayout powers_layout(const StateLayout &L) { return {L.S1, L.S1 + L.term, L.S1 + 2 * L.term}; }

}  // namespace

poet_status cnp_forward_many(const poet_side *sides, const SideGeom *geoms, int count, int dtype, cudaStream_t st) {
  std::vector<int> idx, horner, pw;
  int kmax = 0;
  for (int i = 0; i < count; ++i) {
    if (geoms[i].nprim == 0) continue;
    idx.push_back(i);
    if (by_powers(geoms[i])) {
      pw.push_back(i);
    } else {
      horner.push_back(i);
      if (geoms[i].k > kmax) kmax = geoms[i].k;
    }
  }
  // theta -> Q, and S_1 (or B when k = 0) for Horner's rule; every side in one launch
  static thread_local SideTable t;
  POET_TRY(many_launch(idx, [&](int i, int q) {
    const SideGeom &g = geoms[i];
    const StateLayout L = state_layout(g, dtype);
    char *base = static_cast<char *>(sides[i].state);
    t.src[q] = sides[i].theta;
    t.dst[q] = base + L.Q;
    t.dst2[q] = g.k == 0 ? base + L.R : base + L.S1;  // B = I + Q, S_1 = I + Q, or Q + 2I (order 4)
    t.coef[q] = by_powers(g) ? 2.f : 1.f;
    t.dst3[q] = g.k == 0 ? nullptr : base + L.R;
    t.nprim[q] = g.nprim; t.size[q] = g.size; t.ld[q] = g.ld;
    return pairs_over(g, g.ld);
  }, t, [&](const SideTable &tt, int, int) {
    const int blocks = int(tt.block_start[tt.count]);
    TraceScope ts("cnp_elem", 0.0, table_elems(tt) * (2.0 * esize(dtype) + 2.0), st);
    if (dtype == POET_BF16) unpack_many_kernel<bf16><<<blocks, 256, 0, st>>>(tt);
    else unpack_many_kernel<float><<<blocks, 256, 0, st>>>(tt);
    count_launch();
    return launch_status("cnp unpack");
  }));
  std::vector<Gemm> gs;
  // Horner's rule: one grouped launch per order
  for (int l = 1; l <= kmax; ++l) {
    gs.clear();
    for (int i : horner) {
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
  if (pw.empty()) return POET_OK;
  // order 4 by powers: S = Q Q, C' = S S + 2S, B = (Q + 2I) C' + 2Q - 2S + I
  for (int step = 0; step < 3; ++step) {
    gs.clear();
    for (int i : pw) {
      const SideGeom &g = geoms[i];
      const StateLayout L = state_layout(g, dtype);
      const PowersLayout W = powers_layout(L);
      char *base = static_cast<char *>(sides[i].state);
      Gemm p;
      if (step == 0) {
        p = prim_gemm(g, dtype, base + L.Q, base + L.Q, false, "cnp_fwd");
        p.outD = base + W.S;
      } else if (step == 1) {
        p = prim_gemm(g, dtype, base + W.S, base + W.S, false, "cnp_fwd");
        p.add = base + W.S; p.add_dtype = dtype; p.add_m = g.ld; p.add_b = g.blk_elems(); p.beta = 2.f;
        p.outD = base + W.C;
      } else {
        p = prim_gemm(g, dtype, base + W.Q2, base + W.C, false, "cnp_fwd");
        p.add = base + L.Q; p.add_dtype = dtype; p.add_m = g.ld; p.add_b = g.blk_elems(); p.beta = 2.f;
        p.add2 = base + W.S; p.add2_dtype = dtype; p.add2_m = g.ld; p.add2_b = g.blk_elems(); p.beta2 = -2.f;
        p.diag = 1.f;
        p.outD = base + L.R;
      }
      p.od_m = g.ld; p.od_b = g.blk_elems();
      gs.push_back(p);
    }
    POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  }
  return POET_OK;
}

// Many sides: the same gradient reorganised for grouped launches.
//  - Horner's rule: the chain A_k = S_1^T G, A_l = -Q A_{l+1} takes one grouped
//    launch per order (all sides; S_1^T is read straight from the stored S_1
//    as a transposed operand).  One more launch forms every partial product
//    P_k = G S_k^T, P_l = A_{l+1} S_l^T (l < k) of every side, each into its
//    own float buffer, and one launch packs D - D^T into dtheta with
//    D = A_1 + P_1 + ... + P_k.
//  - order 4 by powers: U = G - Q G and G C = G C' + 2G in one launch, dT_s, V = dT_s S + U,
//    dS_s, D = G C - 2 dS_s Q, then D packed (see the top of this file).
// Every product writes one plain output, which the tensor-core engine stores
// through its staged epilogue.
size_t cnp_many_scratch_bytes(const SideGeom &g, int dtype) {
  if (g.nprim == 0 || g.size < 2 || g.k == 0) return 0;
  const size_t f = align256(size_t(g.all_elems()) * 4);
  const size_t d = align256(size_t(g.all_elems()) * esize(dtype));
  // order 4: G operand copy, U then D (f32), G C (f32), dT_s then dS_s (operand type), V (f32)
  if (by_powers(g)) return 2 * d + 3 * f;
  // G operand copy, A_k..A_2 (dtype), A_1 (f32), P_1..P_k (f32)
  return d + size_t(g.k - 1) * d + f + size_t(g.k) * f;
}

poet_status cnp_backward_many(const poet_side *sides, const SideGeom *geoms, int count, int dtype,
                              const float *const *G, float *const *dtheta, void *const *scratch, cudaStream_t st,
                              const AdamW *adam, float *const *m, float *const *v) {
  struct Work {
    const void *Q, *Gop;
    const char *S1;
    size_t term;
    char *X;   // Horner: A_{l+1} for l = 1..k-1 at X + (l-1) * xb (dtype)
    size_t xb;
    float *A1;  // Horner: A_1
    float *P;   // Horner: P_l at P + (l-1) * pstride
    int64_t pstride;
    // order 4 by powers
    const void *S, *C;   // S and C' = C - 2I
    float *UD, *GC, *V;  // U, then D; G C; V
    void *dT;            // dT_s, then dS_s (operand type)
  };
  std::vector<Work> w(count);
  std::vector<int> chain, all, pw, rounded;  // Horner sides with k >= 1; every side; order-4 sides; G to round
  int kmax = 0;
  for (int i = 0; i < count; ++i) {
    const SideGeom &g = geoms[i];
    if (g.nprim == 0 || g.size < 2) continue;
    all.push_back(i);
    if (g.k == 0) continue;  // B = I + Q: dQ = G
    rounded.push_back(i);
    const StateLayout L = state_layout(g, dtype);
    const char *base = static_cast<const char *>(sides[i].state);
    const size_t db = align256(size_t(g.all_elems()) * esize(dtype));
    const size_t fb = align256(size_t(g.all_elems()) * 4);
    char *s = static_cast<char *>(scratch[i]);
    Work &x = w[i];
    x.Q = base + L.Q;
    x.Gop = dtype == POET_BF16 ? static_cast<const void *>(s) : static_cast<const void *>(G[i]);
    if (by_powers(g)) {
      pw.push_back(i);
      const PowersLayout P = powers_layout(L);
      x.S = base + P.S;
      x.C = base + P.C;
      x.UD = reinterpret_cast<float *>(s + db);
      x.GC = reinterpret_cast<float *>(s + db + fb);
      x.dT = s + db + 2 * fb;
      x.V = reinterpret_cast<float *>(s + 2 * db + 2 * fb);
      continue;
    }
    chain.push_back(i);
    x.S1 = base + L.S1;
    x.term = L.term;
    x.X = s + db;
    x.xb = db;
    x.A1 = reinterpret_cast<float *>(s + size_t(g.k) * db);
    x.P = reinterpret_cast<float *>(s + size_t(g.k) * db + fb);
    x.pstride = int64_t(fb / 4);
    if (g.k > kmax) kmax = g.k;
  }
  static thread_local SideTable t;
  if (dtype == POET_BF16) {  // G rounded to the operand type, every side in one launch
    POET_TRY(many_launch(rounded, [&](int i, int q) {
      const SideGeom &g = geoms[i];
      t.src[q] = G[i];
      t.dst[q] = const_cast<void *>(w[i].Gop);
      t.nprim[q] = g.nprim; t.size[q] = g.size; t.ld[q] = g.ld;
      return round_blocks(g);
    }, t, [&](const SideTable &tt, int, int) {
      TraceScope ts("cnp_elem", 0.0, table_elems(tt) * 6.0, st);
      round_many_kernel<<<int(tt.block_start[tt.count]), 256, 0, st>>>(tt);
      count_launch();
      return launch_status("cnp G to bf16");
    }));
  }
  std::vector<Gemm> gs;
  auto fout = [](Gemm &p, const SideGeom &g, float *o) { p.outF = o; p.of_m = g.ld; p.of_b = g.blk_elems(); };
  // ---- order 4 by powers
  if (!pw.empty()) {
    gs.clear();
    for (int i : pw) {  // U = G - Q G, GC = G C' + 2G
      const SideGeom &g = geoms[i];
      Gemm a = prim_gemm(g, dtype, w[i].Q, w[i].Gop, false, "cnp_bwd");
      a.alpha = -1.f;
      a.add = G[i]; a.add_dtype = POET_F32; a.add_m = g.ld; a.add_b = g.blk_elems(); a.beta = 1.f;
      fout(a, g, w[i].UD);
      gs.push_back(a);
      Gemm b = prim_gemm(g, dtype, w[i].Gop, w[i].C, false, "cnp_bwd");
      b.add = G[i]; b.add_dtype = POET_F32; b.add_m = g.ld; b.add_b = g.blk_elems(); b.beta = 2.f;
      fout(b, g, w[i].GC);
      gs.push_back(b);
    }
    POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
    // dT_s = sym(G + U) = (G + G^T + U + U^T) / 2, then dS_s = V + V^T
    auto sym = [&](bool second) {
      return many_launch(pw, [&](int i, int q) {
        const SideGeom &g = geoms[i];
        t.src[q] = second ? static_cast<const void *>(w[i].V) : static_cast<const void *>(G[i]);
        t.src2[q] = second ? nullptr : w[i].UD;
        t.dst[q] = w[i].dT;
        t.nprim[q] = g.nprim; t.size[q] = g.size; t.ld[q] = g.ld;
        return pair_blocks(g);
      }, t, [&](const SideTable &tt, int, int) {
        const int blocks = int(tt.block_start[tt.count]);
        const float c0 = second ? 1.f : 0.5f, c1 = second ? 0.f : 0.5f;
        TraceScope ts("cnp_elem", 0.0, table_elems(tt) * ((second ? 4.0 : 8.0) + esize(dtype)), st);
        if (dtype == POET_BF16) sym_many_kernel<bf16><<<blocks, 256, 0, st>>>(tt, c0, c1);
        else sym_many_kernel<float><<<blocks, 256, 0, st>>>(tt, c0, c1);
        count_launch();
        return launch_status("cnp symmetric part");
      });
    };
    POET_TRY(sym(false));
    gs.clear();
    for (int i : pw) {  // V = dT_s S + U
      const SideGeom &g = geoms[i];
      Gemm a = prim_gemm(g, dtype, w[i].dT, w[i].S, false, "cnp_bwd");
      a.add = w[i].UD; a.add_dtype = POET_F32; a.add_m = g.ld; a.add_b = g.blk_elems(); a.beta = 1.f;
      fout(a, g, w[i].V);
      gs.push_back(a);
    }
    POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
    POET_TRY(sym(true));
    gs.clear();
    for (int i : pw) {  // D = GC - 2 dS_s Q (over U, which is no longer needed)
      const SideGeom &g = geoms[i];
      Gemm a = prim_gemm(g, dtype, w[i].dT, w[i].Q, false, "cnp_bwd");
      a.alpha = -2.f;
      a.add = w[i].GC; a.add_dtype = POET_F32; a.add_m = g.ld; a.add_b = g.blk_elems(); a.beta = 1.f;
      fout(a, g, w[i].UD);
      gs.push_back(a);
    }
    POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  }
  // ---- Horner's rule
  // X_l, the left factor of P_l: G for l = k, else A_{l+1}
  auto Xop = [&](int i, int l) -> const void * {
    return l == geoms[i].k ? w[i].Gop : static_cast<const void *>(w[i].X + size_t(l - 1) * w[i].xb);
  };
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
        fout(a, g, x.A1);
      } else if (dtype == POET_BF16) {
        a.outD = x.X + size_t(l - 2) * x.xb; a.od_m = g.ld; a.od_b = g.blk_elems();
      } else {
        fout(a, g, reinterpret_cast<float *>(x.X + size_t(l - 2) * x.xb));
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
      fout(p, g, w[i].P + (l - 1) * w[i].pstride);
      gs.push_back(p);
    }
  }
  POET_TRY(gemm_run_many(gs.data(), int(gs.size()), st));
  // dtheta = D - D^T, every side in one launch:  k = 0: D = G;  Horner: D = A_1 + sum P_l;
  // order 4: D as formed above
  return many_launch(all, [&](int i, int q) {
    const SideGeom &g = geoms[i];
    if (g.k == 0) {
      t.src[q] = G[i];
    } else if (by_powers(g)) {
      t.src[q] = w[i].UD;
    } else {
      t.src[q] = w[i].A1;
      t.dst2[q] = w[i].P;
      t.terms[q] = g.k;
      t.stride[q] = w[i].pstride;
    }
    t.dst[q] = dtheta ? dtheta[i] : nullptr;
    if (adam) {
      t.theta[q] = sides[i].theta;
      t.m1[q] = m[i];
      t.m2[q] = v[i];
    }
    t.nprim[q] = g.nprim; t.size[q] = g.size; t.ld[q] = g.ld;
    return pair_blocks(g);
  }, t, [&](const SideTable &tt, int, int) {
    const int blocks = int(tt.block_start[tt.count]);
    double terms = 0.0;
    for (int q = 0; q < tt.count; ++q) terms += double(tt.nprim[q]) * tt.size[q] * tt.size[q] * (1 + tt.terms[q]);
    TraceScope ts("cnp_elem", 0.0, terms * 4.0 + table_elems(tt) * (adam ? 14.0 : 2.0), st);
    if (adam) pack_many_kernel<true><<<blocks, 256, 0, st>>>(tt, *adam);
    else pack_many_kernel<false><<<blocks, 256, 0, st>>>(tt, AdamW{});
    count_launch();
    return launch_status("cnp pack");
  });
}

}  // namespace poet
