// Column permutations between natural order and the permuted frame.
//
// A side's primitives act on the natural indices perm[j*size .. j*size+size-1]
// (POET summary page, Approach: "sampled sub-block orthogonal primitives";
// the index layout is a reading).  These kernels move whole rows between the
// natural order and the frame order, so that every contraction downstream
// reads contiguous blocks.  HBM-bound: one read and one write of each row.
//
// One kernel serves both directions as a row gather out[r][j] = in[r][map[j]]:
//   gather  (natural -> frame): map = perm
//   scatter (frame -> natural): map = perm^-1, built in shared memory
// Indices come from the caller (perm, row maps): an entry out of range is
// never dereferenced.  A perm entry outside [0, d) leaves its map slot at 0 (a
// valid column), a row-map entry outside [0, rows) skips that output row, and
// either sets ERR_BOUNDS in the device status word (poet_sync_status reports
// POET_EBOUNDS).
// Each CTA keeps map (uint16) in shared memory and streams its rows through a
// ring of NB row slots filled by cp.async 16-byte copies, prefetching NB-1
// rows ahead, so the loads, the shared-memory gather and the 16-byte global
// stores of different rows overlap; several CTAs per SM add more rows in
// flight.  Rows whose start is not 16-byte aligned (natural rows of odd
// length) use 16-byte copies for the aligned body and scalar copies for the
// edges; shared and global addresses stay congruent modulo 16.
#include <algorithm>
#include <type_traits>
#include <vector>

#include "poet_internal.cuh"

namespace poet {
namespace {

constexpr int MAX_WARPS = 8;          // warps per CTA (fewer for very long rows); each warp owns whole rows
constexpr int NT = MAX_WARPS * 32;
constexpr int NBW = 2;                // row slots per warp (one row prefetched while one is processed)

template <typename T>
struct PermArgs {
  const T *src1; int64_t ld1;         // source row = src1[0:split) ++ src2[split:d)
  const T *src2; int64_t ld2; int split;
  const int32_t *src_rowmap;          // source row of output row r (nullptr: r)
  int64_t rows; int d;
  const int32_t *perm; int inverse;
  T *dst1; int64_t ldd1;              // output rows
  T *dst2; int64_t ldd2; int dsplit;  // columns >= dsplit also go here (nullptr: none)
  const int32_t *dst_rowmap;          // destination row of output row r (nullptr: r)
  int64_t map_rows;                   // row-map entries must lie in [0, map_rows) (0: rows)
  unsigned *errword;                  // ERR_BOUNDS is OR-ed in for an index out of range
};

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <typename T>
__device__ __forceinline__ int misalign(const T *p) {
  return int((reinterpret_cast<uintptr_t>(p) & 15) / sizeof(T));
}

// One warp copies elements [e0, e1) of a global row into slot[off + e]
// (off = misalignment of the row start; the same for every part of a row).
template <typename T>
__device__ __forceinline__ void load_part(const T *row, int e0, int e1, T *slot, int off, int lane) {
  constexpr int VEC = 16 / sizeof(T);
  if (e1 <= e0) return;
  const int b0 = ((off + e0 + VEC - 1) / VEC) * VEC - off;  // first 16B-aligned element >= e0
  const int b1 = ((off + e1) / VEC) * VEC - off;            // end of the last whole aligned unit
  if (b0 < b1)
    for (int e = b0 + lane * VEC; e < b1; e += 32 * VEC) cp_async16(slot + off + e, row + e);
  const int h1 = b0 < e1 ? b0 : e1;
  for (int e = e0 + lane; e < h1; e += 32) slot[off + e] = row[e];
  const int t0 = b1 > h1 ? b1 : h1;
  for (int e = t0 + lane; e < e1; e += 32) slot[off + e] = row[e];
}

// VEC consecutive map entries starting at j0 = u*VEC - DOFF, read as aligned
// vectors (two when the destination row is misaligned).
template <int VEC, int DOFF>
__device__ __forceinline__ void map_entries(const uint16_t *map, int u, uint16_t (&m)[VEC]) {
  if constexpr (VEC == 8) {
    if constexpr (DOFF == 0) {
      const uint4 a = *reinterpret_cast<const uint4 *>(map + 8 * u);
      const uint16_t *pa = reinterpret_cast<const uint16_t *>(&a);
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = pa[e];
    } else {
      const uint4 a = *reinterpret_cast<const uint4 *>(map + 8 * (u - 1));
      const uint4 b = *reinterpret_cast<const uint4 *>(map + 8 * u);
      const uint16_t *pa = reinterpret_cast<const uint16_t *>(&a);
      const uint16_t *pb = reinterpret_cast<const uint16_t *>(&b);
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = (8 - DOFF + e) < 8 ? pa[8 - DOFF + e] : pb[e - DOFF];
    }
  } else {  // VEC == 4: groups of four 16-bit entries
    if constexpr (DOFF == 0) {
      const uint2 a = *reinterpret_cast<const uint2 *>(map + 4 * u);
      const uint16_t *pa = reinterpret_cast<const uint16_t *>(&a);
#pragma unroll
      for (int e = 0; e < 4; ++e) m[e] = pa[e];
    } else {
      const uint2 a = *reinterpret_cast<const uint2 *>(map + 4 * (u - 1));
      const uint2 b = *reinterpret_cast<const uint2 *>(map + 4 * u);
      const uint16_t *pa = reinterpret_cast<const uint16_t *>(&a);
      const uint16_t *pb = reinterpret_cast<const uint16_t *>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) m[e] = (4 - DOFF + e) < 4 ? pa[4 - DOFF + e] : pb[e - DOFF];
    }
  }
}

// Output row = slot gathered through map; drow misaligned by DOFF elements.
// ident: the map is the identity and the staged row is congruent with drow
// modulo 16 bytes, so each unit is one 16-byte shared-memory read.
template <typename T, int DOFF>
__device__ __forceinline__ void emit_row(const PermArgs<T> &a, const uint16_t *map, const T *s, T *drow, T *d2row,
                                         int lane, bool ident) {
  constexpr int VEC = 16 / sizeof(T);
  const int d = a.d;
  const int units = (DOFF + d + VEC - 1) / VEC;
  for (int u = lane; u < units; u += 32) {
    const int j0 = u * VEC - DOFF;  // output column of the unit's first lane
    if (j0 >= 0 && j0 + VEC <= d) {
      alignas(16) T v[VEC];
      if (ident) {
        *reinterpret_cast<uint4 *>(v) = *reinterpret_cast<const uint4 *>(s + j0);
      } else {
        uint16_t m[VEC];
        map_entries<VEC, DOFF>(map, u, m);
#pragma unroll
        for (int e = 0; e < VEC; ++e) v[e] = s[m[e]];
      }
      *reinterpret_cast<uint4 *>(drow + j0) = *reinterpret_cast<const uint4 *>(v);
      if (d2row && j0 + VEC > a.dsplit) {
        if (DOFF == 0 && j0 >= a.dsplit) {
          *reinterpret_cast<uint4 *>(d2row + j0) = *reinterpret_cast<const uint4 *>(v);
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            if (j0 + e >= a.dsplit) d2row[j0 + e] = v[e];
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const int j = j0 + e;
        if (j >= 0 && j < d) {
          const T x = s[map[j]];
          drow[j] = x;
          if (d2row && j >= a.dsplit) d2row[j] = x;
        }
      }
    }
  }
}

// Up to MAXP independent row permutations in one launch.  Problem p owns the
// global rows [row_start[p], row_start[p+1]); CTA c works through the
// contiguous global rows [total*c/G, total*(c+1)/G), one segment per problem
// it touches, and rebuilds its shared-memory map at the start of each segment.
template <typename T, int MAXP>
struct PermGroup {
  PermArgs<T> prob[MAXP];
  int64_t row_start[MAXP + 1];
  int count;
  int slot;     // ring slot stride (elements, multiple of 16 bytes), for the widest problem
  int map_len;  // map entries allocated (>= round_up(max d, 8) + 8)
};

template <typename T, int MAXP>
__global__ void __launch_bounds__(NT) permute_rows_kernel(const __grid_constant__ PermGroup<T, MAXP> g) {
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint16_t *map = reinterpret_cast<uint16_t *>(smem_raw);
  const int nthr = blockDim.x, warps = nthr / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  T *ring = reinterpret_cast<T *>(smem_raw + size_t(g.map_len) * 2) + int64_t(warp) * NBW * g.slot;
  const int64_t total = g.row_start[g.count];
  const int64_t r0 = total * blockIdx.x / gridDim.x, r1 = total * (blockIdx.x + 1) / gridDim.x;
  int p = 0;
  for (int64_t seg = r0; seg < r1;) {
    while (g.row_start[p + 1] <= seg) ++p;
    const PermArgs<T> &a = g.prob[p];
    const int64_t seg_end = r1 < g.row_start[p + 1] ? r1 : g.row_start[p + 1];
    const int64_t lo = seg - g.row_start[p], hi = seg_end - g.row_start[p];  // rows [lo, hi) of problem p
    seg = seg_end;
    const int d = a.d;
    __syncthreads();  // the previous segment's readers of map are done
    for (int i = threadIdx.x; i < g.map_len; i += nthr) map[i] = 0;
    __syncthreads();
    bool bad = false;
    if (!a.perm) {  // identity: a plain row copy
      for (int i = threadIdx.x; i < d; i += nthr) map[i] = uint16_t(i);
    } else if (a.inverse) {
      for (int i = threadIdx.x; i < d; i += nthr) {
        const int pi = a.perm[i];
        if (unsigned(pi) < unsigned(d)) map[pi] = uint16_t(i);
        else bad = true;
      }
    } else {
      for (int i = threadIdx.x; i < d; i += nthr) {
        const int pi = a.perm[i];
        const bool ok = unsigned(pi) < unsigned(d);
        map[i] = ok ? uint16_t(pi) : uint16_t(0);
        bad |= !ok;
      }
    }
    if (bad && a.errword) atomicOr(a.errword, ERR_BOUNDS);
    __syncthreads();  // map is complete

    const int split = a.split < d ? a.split : d;
    const int64_t first = lo + warp, stride = warps;
    const int64_t count = first < hi ? (hi - first + stride - 1) / stride : 0;

    // source and destination row of output row r; -1 when a row map's entry is out of range
    const int64_t map_rows = a.map_rows > 0 ? a.map_rows : a.rows;
    auto src_row = [&](int64_t r) -> int64_t {
      if (!a.src_rowmap) return r;
      const int64_t s = a.src_rowmap[r];
      return s >= 0 && s < map_rows ? s : -1;
    };
    auto dst_row = [&](int64_t r) -> int64_t {
      if (!a.dst_rowmap) return r;
      const int64_t s = a.dst_rowmap[r];
      return s >= 0 && s < map_rows ? s : -1;
    };
    auto issue = [&](int64_t k) {
      const int64_t r = first + k * stride;
      const int64_t sr = src_row(r);
      if (sr < 0 || dst_row(r) < 0) return;  // skipped row: nothing to load
      T *slot = ring + int64_t(k % NBW) * g.slot;
      const T *row1 = a.src1 + sr * a.ld1;
      const int off = misalign(row1);
      load_part(row1, 0, split, slot, off, lane);
      if (split < d) load_part(a.src2 + sr * a.ld2, split, d, slot, off, lane);
    };

    if (count > 0) issue(0);
    cp_async_commit();
    for (int64_t k = 0; k < count; ++k) {
      if (k + 1 < count) issue(k + 1);
      cp_async_commit();
      cp_async_wait_one();  // this lane's copies of row k have landed
      __syncwarp();         // ... and every other lane's (scalar edges included)
      const int64_t r = first + k * stride;
      const int64_t sr = src_row(r), dr = dst_row(r);
      if (sr < 0 || dr < 0) {  // a row map entry out of range: skip the row, report it
        if (lane == 0 && a.errword) atomicOr(a.errword, ERR_BOUNDS);
        __syncwarp();
        continue;
      }
      const T *sl = ring + int64_t(k % NBW) * g.slot + misalign(a.src1 + sr * a.ld1);
      T *drow = a.dst1 + dr * a.ldd1;
      T *d2row = a.dst2 ? a.dst2 + r * a.ldd2 : nullptr;
      const bool ident = !a.perm && misalign(sl) == misalign(drow);
      switch (misalign(drow)) {
        case 0: emit_row<T, 0>(a, map, sl, drow, d2row, lane, ident); break;
        case 1: emit_row<T, 1>(a, map, sl, drow, d2row, lane, ident); break;
        case 2: emit_row<T, 2>(a, map, sl, drow, d2row, lane, ident); break;
        case 3: emit_row<T, 3>(a, map, sl, drow, d2row, lane, ident); break;
        case 4: if constexpr (VEC == 8) emit_row<T, 4>(a, map, sl, drow, d2row, lane, ident); break;
        case 5: if constexpr (VEC == 8) emit_row<T, 5>(a, map, sl, drow, d2row, lane, ident); break;
        case 6: if constexpr (VEC == 8) emit_row<T, 6>(a, map, sl, drow, d2row, lane, ident); break;
        default: if constexpr (VEC == 8) emit_row<T, 7>(a, map, sl, drow, d2row, lane, ident); break;
      }
      __syncwarp();  // slot k % NBW may be refilled by the next iteration's prefetch
    }
    cp_async_wait_all();
  }
}

// Plain row copy to 16-byte aligned destination rows (re-striding rows whose
// start is only element-aligned).  Destination unit u (16 bytes) of a row is
// assembled from the two aligned 16-byte source words u and u + 1 of that
// row, shifted by the row's misalignment; every word read overlaps the row.
// Columns past d in the last unit receive bytes of the source's next
// elements (padding, never read as data).
template <int H>  // shift by H 16-bit halves (0..7)
__device__ __forceinline__ uint4 shift_pair(const uint4 &a, const uint4 &b) {
  const uint32_t c[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (H % 2 == 0) o[i] = c[i + H / 2];
    else o[i] = __byte_perm(c[i + H / 2], c[i + H / 2 + 1], 0x5432);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void __launch_bounds__(256) restride_kernel(const unsigned char *__restrict__ src, int64_t ld_src_bytes,
                                                       int64_t rows, int row_bytes, unsigned char *__restrict__ dst,
                                                       int64_t ld_dst_bytes) {
  const int units = (row_bytes + 15) / 16;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const unsigned char *srow = src + r * ld_src_bytes;
    const int off = int(reinterpret_cast<uintptr_t>(srow) & 15);  // even: elements are >= 2 bytes
    const uint4 *wp = reinterpret_cast<const uint4 *>(srow - off);
    const int nwords = (off + row_bytes + 15) / 16;  // aligned words overlapping the row
    uint4 *drow = reinterpret_cast<uint4 *>(dst + r * ld_dst_bytes);
    for (int u = threadIdx.x; u < units; u += blockDim.x) {
      const uint4 w0 = wp[u];
      const uint4 w1 = u + 1 < nwords ? wp[u + 1] : make_uint4(0, 0, 0, 0);
      uint4 v;
      switch (off >> 1) {
        case 0: v = w0; break;
        case 1: v = shift_pair<1>(w0, w1); break;
        case 2: v = shift_pair<2>(w0, w1); break;
        case 3: v = shift_pair<3>(w0, w1); break;
        case 4: v = shift_pair<4>(w0, w1); break;
        case 5: v = shift_pair<5>(w0, w1); break;
        case 6: v = shift_pair<6>(w0, w1); break;
        default: v = shift_pair<7>(w0, w1); break;
      }
      drow[u] = v;
    }
  }
}

// out[a][c] = bf16(D[rowmap[a]][perm[c]]): a float matrix gathered into the
// frame and rounded in one pass, for up to kFrameMax matrices per launch
// (matrix p owns the global rows [row_start[p], row_start[p+1])).  One block
// per output row at a time; the source row is read through L1 (it is reused
// by the block's gathers).  An index out of range (rowmap outside [0, rows),
// perm outside [0, d)) is not read: its output is 0 and ERR_BOUNDS is set in
// the status word.
constexpr int kFrameMax = 64;
struct FrameGroup {
  const float *D[kFrameMax];
  int64_t ldD[kFrameMax];
  const int32_t *rowmap[kFrameMax];
  const int32_t *perm[kFrameMax];
  bf16 *out[kFrameMax];
  int64_t ld_out[kFrameMax];
  int64_t rows[kFrameMax];
  int d[kFrameMax];
  int64_t row_start[kFrameMax + 1];
  int count;
  unsigned *errword;
};
static_assert(sizeof(FrameGroup) <= 32000, "frame table exceeds the kernel parameter limit");

__global__ void __launch_bounds__(256) frame_f32_to_bf16_kernel(const __grid_constant__ FrameGroup g) {
  // a row of D is staged in shared memory with 16-byte copies (coalesced), then
  // gathered from there; rows whose start is not 16-byte aligned are gathered
  // from global memory directly
  extern __shared__ __align__(16) float srow[];
  bool bad = false;
  const int64_t total = g.row_start[g.count];
  int p = 0;
  for (int64_t gr = blockIdx.x; gr < total; gr += gridDim.x) {
    while (g.row_start[p + 1] <= gr) ++p;  // rows are visited in increasing order
    const int64_t a = gr - g.row_start[p], rows = g.rows[p];
    const int d = g.d[p];
    const int32_t *perm = g.perm[p];
    const int64_t sr = __ldg(g.rowmap[p] + a);
    const bool row_ok = sr >= 0 && sr < rows;
    bad |= !row_ok;
    const float *src = g.D[p] + (row_ok ? sr : 0) * g.ldD[p];
    const bool staged = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
    if (staged) {
      __syncthreads();  // the previous row's readers of srow are done
      const int units = d / 4;
      for (int u = threadIdx.x; u < units; u += blockDim.x) cp_async16(srow + 4 * u, src + 4 * u);
      for (int c = 4 * units + threadIdx.x; c < d; c += blockDim.x) srow[c] = src[c];
      cp_async_wait_all();
      __syncthreads();
    }
    bf16 *orow = g.out[p] + a * g.ld_out[p];
    for (int c = 2 * threadIdx.x; c < d; c += 2 * blockDim.x) {
      if (c + 1 < d) {
        const int2 pc = *reinterpret_cast<const int2 *>(perm + c);
        const bool okx = row_ok && unsigned(pc.x) < unsigned(d), oky = row_ok && unsigned(pc.y) < unsigned(d);
        bad |= !(okx && oky);
        const float vx = okx ? (staged ? srow[pc.x] : __ldg(src + pc.x)) : 0.f;
        const float vy = oky ? (staged ? srow[pc.y] : __ldg(src + pc.y)) : 0.f;
        *reinterpret_cast<__nv_bfloat162 *>(orow + c) = __floats2bfloat162_rn(vx, vy);
      } else {
        const int pc = perm[c];
        const bool ok = row_ok && unsigned(pc) < unsigned(d);
        bad |= !ok;
        orow[c] = __float2bfloat16_rn(ok ? (staged ? srow[pc] : __ldg(src + pc)) : 0.f);
      }
    }
  }
  if (bad && g.errword) atomicOr(g.errword, ERR_BOUNDS);
}

// dst[p][0 .. n[p]) = 0 for up to kFrameMax float buffers (16-byte vectors
// where a buffer is 16-byte aligned).
struct ZeroGroup {
  float *dst[kFrameMax];
  int64_t n[kFrameMax];
  int count;
};
__global__ void __launch_bounds__(256) zero_many_kernel(const __grid_constant__ ZeroGroup g) {
  for (int p = 0; p < g.count; ++p) {
    float *d = g.dst[p];
    const int64_t n = g.n[p];
    const int64_t tid = blockIdx.x * int64_t(blockDim.x) + threadIdx.x, nth = int64_t(gridDim.x) * blockDim.x;
    if ((reinterpret_cast<uintptr_t>(d) & 15) == 0) {
      const int64_t n4 = n / 4;
      for (int64_t i = tid; i < n4; i += nth) reinterpret_cast<float4 *>(d)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int64_t i = n4 * 4 + tid; i < n; i += nth) d[i] = 0.f;
    } else {
      for (int64_t i = tid; i < n; i += nth) d[i] = 0.f;
    }
  }
}

// out_p[b*ldb + r*ldm + c] = 0 for b < batch, r < M, c < N of up to kZeroMax
// regions p (blockIdx.z); 16-byte stores where rows allow.
constexpr int kZeroMax = 64;
struct ZeroTable {
  ZeroRegion reg[kZeroMax];
  int count;
};
__global__ void __launch_bounds__(256) zero_output_kernel(const __grid_constant__ ZeroTable t) {
  const ZeroRegion &r = t.reg[blockIdx.z];
  const bool vec = (reinterpret_cast<uintptr_t>(r.out) & 15) == 0 && r.ldm % 4 == 0 && (r.batch == 1 || r.ldb % 4 == 0);
  const int units = vec ? (r.N + 3) / 4 : r.N;  // 16-byte units (the last may be partial) or single columns
  const int64_t rows = int64_t(r.batch) * r.M;
  for (int64_t row = blockIdx.y * int64_t(blockDim.y) + threadIdx.y; row < rows; row += int64_t(gridDim.y) * blockDim.y) {
    float *o = r.out + (row / r.M) * r.ldb + (row % r.M) * r.ldm;
    for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < units; u += gridDim.x * blockDim.x) {
      if (vec && 4 * u + 4 <= r.N) *reinterpret_cast<float4 *>(o + 4 * u) = make_float4(0.f, 0.f, 0.f, 0.f);
      else if (vec) { for (int c = 4 * u; c < r.N; ++c) o[c] = 0.f; }
      else o[u] = 0.f;
    }
  }
}

// Launches the problems of one table: the ring slot fits the widest row, as
// many warps as shared memory allows (at most MAX_WARPS), and a grid of the
// CTAs that can be resident at once (fewer for little work).
template <typename T, int MAXP>
poet_status launch_permute_group(PermGroup<T, MAXP> &grp, cudaStream_t st, const char *kind) {
  constexpr int VEC = 16 / sizeof(T);
  int dmax = 0;
  double bytes = 0.0;
  grp.row_start[0] = 0;
  for (int i = 0; i < grp.count; ++i) {
    const PermArgs<T> &a = grp.prob[i];
    POET_REQUIRE(a.d >= 1 && a.d <= 65535, "permute: dimension %d outside [1, 65535]", a.d);
    if (a.d > dmax) dmax = a.d;
    grp.row_start[i + 1] = grp.row_start[i] + (a.rows > 0 ? a.rows : 0);
    bytes += double(a.rows) * a.d * sizeof(T) * 2.0;
  }
  const int64_t total = grp.row_start[grp.count];
  if (total <= 0) return POET_OK;
  grp.slot = int(round_up(dmax + VEC, VEC));
  grp.map_len = int(round_up(dmax, 8) + 8);
  const size_t budget = 220 * 1024, per_warp = size_t(NBW) * grp.slot * sizeof(T);
  int warps = int((budget - size_t(grp.map_len) * 2) / per_warp);
  if (warps > MAX_WARPS) warps = MAX_WARPS;
  POET_REQUIRE(warps >= 1, "permute: rows of %d elements do not fit in shared memory", dmax);
  const size_t smem = size_t(grp.map_len) * 2 + size_t(warps) * per_warp;
  auto kern = permute_rows_kernel<T, MAXP>;
  static int configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && configured[dev] < int(smem)) {
    POET_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    configured[dev] = int(smem);
  }
  int per_sm = 0;
  POET_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, warps * 32, smem));
  if (per_sm < 1) per_sm = 1;
  const int64_t want = (total + warps - 1) / warps;
  const int64_t cap = int64_t(num_sms()) * per_sm;
  const int grid = int(want < cap ? want : cap);
  unsigned *ew = device_errword();
  for (int i = 0; i < grp.count; ++i) grp.prob[i].errword = ew;
  TraceScope ts(kind, 0.0, bytes, st);
  kern<<<grid, warps * 32, smem, st>>>(grp);
  count_launch();
  return launch_status(kind);
}

template <typename T>
poet_status launch_permute(const PermArgs<T> &a, cudaStream_t st, const char *kind) {
  if (a.rows <= 0 || a.d <= 0) return POET_OK;
  PermGroup<T, 1> grp;
  grp.prob[0] = a;
  grp.count = 1;
  return launch_permute_group(grp, st, kind);
}

constexpr int kPermMax = 64;
static_assert(sizeof(PermGroup<float, kPermMax>) <= 32000, "permute table exceeds the kernel parameter limit");

// Problems are launched in buckets of similar row width (the ring slot of a
// launch fits its widest row, so a narrow row sharing a launch with a wide one
// would get fewer CTAs per SM than on its own), up to kPermMax per launch.
template <typename T>
poet_status launch_permute_many(const std::vector<PermArgs<T>> &v, cudaStream_t st, const char *kind) {
  static thread_local PermGroup<T, kPermMax> grp;  // large: keep it off the stack
  auto width_class = [](int d) {  // row bytes rounded up to a power of two
    int c = 0;
    while ((int64_t(1) << c) < int64_t(d) * int64_t(sizeof(T))) ++c;
    return c;
  };
  std::vector<int> classes;
  for (const PermArgs<T> &a : v)
    if (a.rows > 0 && a.d > 0) classes.push_back(width_class(a.d));
  std::sort(classes.begin(), classes.end());
  classes.erase(std::unique(classes.begin(), classes.end()), classes.end());
  for (int cls : classes) {
    grp.count = 0;
    for (const PermArgs<T> &a : v) {
      if (a.rows <= 0 || a.d <= 0 || width_class(a.d) != cls) continue;
      grp.prob[grp.count++] = a;
      if (grp.count == kPermMax) {
        POET_TRY(launch_permute_group(grp, st, kind));
        grp.count = 0;
      }
    }
    if (grp.count > 0) POET_TRY(launch_permute_group(grp, st, kind));
  }
  return POET_OK;
}

}  // namespace

poet_status gather_cols(int dtype, const void *src, int64_t ld_src, const int32_t *rowmap, int64_t rows, int d,
                        const int32_t *perm, void *dst, int64_t ld_dst, void *dst2, int64_t ld_dst2, int split,
                        cudaStream_t st, const char *kind) {
  POET_REQUIRE((reinterpret_cast<uintptr_t>(dst) & 15) == 0 && ld_dst * int64_t(esize(dtype)) % 16 == 0,
               "gather: frame rows must be 16-byte aligned");
  auto fill = [&](auto *tag) {
    using T = std::remove_pointer_t<decltype(tag)>;
    PermArgs<T> a{};
    a.src1 = static_cast<const T *>(src); a.ld1 = ld_src;
    a.src2 = nullptr; a.ld2 = 0; a.split = d;
    a.src_rowmap = rowmap;
    a.rows = rows; a.d = d;
    a.perm = perm; a.inverse = 0;
    a.dst1 = static_cast<T *>(dst); a.ldd1 = ld_dst;
    a.dst2 = static_cast<T *>(dst2); a.ldd2 = ld_dst2; a.dsplit = dst2 ? split : d;
    a.dst_rowmap = nullptr;
    return launch_permute<T>(a, st, kind);
  };
  return dtype == POET_BF16 ? fill(static_cast<bf16 *>(nullptr)) : fill(static_cast<float *>(nullptr));
}

poet_status frame_many(const std::vector<FrameItem> &v, cudaStream_t st) {
  static thread_local FrameGroup grp;
  for (size_t i0 = 0; i0 < v.size(); i0 += kFrameMax) {
    grp.count = 0;
    grp.row_start[0] = 0;
    double bytes = 0.0;
    for (size_t i = i0; i < v.size() && i < i0 + kFrameMax; ++i) {
      const FrameItem &f = v[i];
      if (f.rows <= 0 || f.d <= 0) continue;
      POET_REQUIRE((reinterpret_cast<uintptr_t>(f.out) & 3) == 0 && f.ld_out % 2 == 0 &&
                       (reinterpret_cast<uintptr_t>(f.perm) & 7) == 0,
                   "frame: output rows must be 4-byte aligned and perm 8-byte aligned");
      const int q = grp.count++;
      grp.D[q] = f.D; grp.ldD[q] = f.ldD; grp.rowmap[q] = f.rowmap; grp.perm[q] = f.perm;
      grp.out[q] = static_cast<bf16 *>(f.out); grp.ld_out[q] = f.ld_out; grp.rows[q] = f.rows; grp.d[q] = f.d;
      grp.row_start[q + 1] = grp.row_start[q] + f.rows;
      bytes += double(f.rows) * f.d * 6.0;
    }
    if (grp.count == 0) continue;
    grp.errword = device_errword();
    int dmax = 0;
    for (int q = 0; q < grp.count; ++q) dmax = grp.d[q] > dmax ? grp.d[q] : dmax;
    const size_t smem = size_t(dmax) * 4;  // one staged row of the widest matrix
    POET_REQUIRE(smem <= 200 * 1024, "frame: rows of %d floats do not fit in shared memory", dmax);
    static int configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (smem > 48 * 1024 && dev < 64 && configured[dev] < int(smem)) {
      POET_CUDA_TRY(cudaFuncSetAttribute(frame_f32_to_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem)));
      configured[dev] = int(smem);
    }
    int per_sm = 0;
    POET_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, frame_f32_to_bf16_kernel, 256, smem));
    if (per_sm < 1) per_sm = 1;
    const int64_t total = grp.row_start[grp.count];
    const int64_t cap = int64_t(num_sms()) * per_sm;
    const int grid = int(total < cap ? total : cap);
    TraceScope ts("frame", 0.0, bytes, st);
    frame_f32_to_bf16_kernel<<<grid, 256, smem, st>>>(grp);
    count_launch();
    POET_TRY(launch_status("frame"));
  }
  return POET_OK;
}

poet_status frame_f32_to_bf16(const float *D, int64_t ldD, const int32_t *rowmap, int64_t rows, int d,
                              const int32_t *perm, void *out, int64_t ld_out, cudaStream_t st) {
  return frame_many({FrameItem{D, ldD, rowmap, rows, d, perm, out, ld_out}}, st);
}

poet_status zero_outputs(const std::vector<ZeroRegion> &v, cudaStream_t st) {
  static thread_local ZeroTable t;
  for (size_t i0 = 0; i0 < v.size(); i0 += kZeroMax) {
    t.count = 0;
    int nmax = 1;
    int64_t rmax = 1;
    double bytes = 0.0;
    for (size_t i = i0; i < v.size() && i < i0 + kZeroMax; ++i) {
      const ZeroRegion &r = v[i];
      if (r.M <= 0 || r.N <= 0 || r.batch <= 0) continue;
      t.reg[t.count++] = r;
      nmax = r.N > nmax ? r.N : nmax;
      const int64_t rows = int64_t(r.batch) * r.M;
      rmax = rows > rmax ? rows : rmax;
      bytes += double(rows) * r.N * 4.0;
    }
    if (t.count == 0) continue;
    const dim3 block(32, 8);
    const int64_t gy_want = (rmax + 7) / 8, gy_cap = int64_t(num_sms()) * 8 / t.count + 1;
    const dim3 grid(unsigned(((nmax + 3) / 4 + 31) / 32), unsigned(gy_want < gy_cap ? gy_want : gy_cap),
                    unsigned(t.count));
    TraceScope ts("zero", 0.0, bytes, st);
    zero_output_kernel<<<grid, block, 0, st>>>(t);
    count_launch();
    POET_TRY(launch_status("zero"));
  }
  return POET_OK;
}

poet_status zero_output(float *out, int M, int N, int64_t ldm, int batch, int64_t ldb, cudaStream_t st) {
  return zero_outputs({ZeroRegion{out, M, N, ldm, batch, ldb}}, st);
}

poet_status zero_many(const std::vector<std::pair<float *, int64_t>> &v, cudaStream_t st) {
  static thread_local ZeroGroup grp;
  for (size_t i0 = 0; i0 < v.size(); i0 += kFrameMax) {
    grp.count = 0;
    int64_t most = 0;
    for (size_t i = i0; i < v.size() && i < i0 + kFrameMax; ++i) {
      if (!v[i].first || v[i].second <= 0) continue;
      grp.dst[grp.count] = v[i].first;
      grp.n[grp.count++] = v[i].second;
      if (v[i].second > most) most = v[i].second;
    }
    if (grp.count == 0) continue;
    const int64_t want = (most / 4 + 255) / 256, cap = int64_t(num_sms()) * 4;
    const int grid = int(want < 1 ? 1 : (want < cap ? want : cap));
    double bytes = 0.0;
    for (int q = 0; q < grp.count; ++q) bytes += double(grp.n[q]) * 4.0;
    TraceScope ts("zero", 0.0, bytes, st);
    zero_many_kernel<<<grid, 256, 0, st>>>(grp);
    count_launch();
    POET_TRY(launch_status("zero"));
  }
  return POET_OK;
}

poet_status permute_many(int dtype, const std::vector<RowPermute> &v, cudaStream_t st, const char *kind) {
  auto run = [&](auto *tag) {
    using T = std::remove_pointer_t<decltype(tag)>;
    std::vector<PermArgs<T>> args;
    args.reserve(v.size());
    for (const RowPermute &r : v) {
      PermArgs<T> a{};
      a.src1 = static_cast<const T *>(r.src1); a.ld1 = r.ld1;
      a.src2 = static_cast<const T *>(r.src2 ? r.src2 : r.src1); a.ld2 = r.src2 ? r.ld2 : r.ld1;
      a.split = r.src2 ? r.split : r.d;
      a.src_rowmap = r.src_rowmap;
      a.rows = r.rows; a.d = r.d;
      a.perm = r.perm; a.inverse = r.inverse;
      a.dst1 = static_cast<T *>(r.dst); a.ldd1 = r.ldd;
      a.dst2 = nullptr; a.ldd2 = 0; a.dsplit = r.d;
      a.dst_rowmap = r.dst_rowmap;
      a.map_rows = r.map_rows;
      args.push_back(a);
    }
    return launch_permute_many<T>(args, st, kind);
  };
  return dtype == POET_BF16 ? run(static_cast<bf16 *>(nullptr)) : run(static_cast<float *>(nullptr));
}

poet_status copy_rows(int dtype, const void *src, int64_t ld_src, int64_t rows, int d, void *dst, int64_t ld_dst,
                      cudaStream_t st) {
  const int64_t es = int64_t(esize(dtype));
  POET_REQUIRE((reinterpret_cast<uintptr_t>(dst) & 15) == 0 && ld_dst * es % 16 == 0 && ld_dst >= round_up(d, 16 / es),
               "copy_rows: destination rows must be 16-byte aligned and hold whole 16-byte units");
  POET_REQUIRE((reinterpret_cast<uintptr_t>(src) % es) == 0, "copy_rows: source misaligned");
  if (rows <= 0 || d <= 0) return POET_OK;
  TraceScope ts("pad", 0.0, double(rows) * d * es * 2.0, st);
  const int64_t cap = int64_t(num_sms()) * 8;
  const int grid = int(rows < cap ? rows : cap);
  restride_kernel<<<grid, 256, 0, st>>>(static_cast<const unsigned char *>(src), ld_src * es, rows, int(d * es),
                                        static_cast<unsigned char *>(dst), ld_dst * es);
  count_launch();
  return launch_status("pad");
}

poet_status scatter_cols(int dtype, const void *src1, int64_t ld1, const void *src2, int64_t ld2, int split,
                         int64_t rows, int d, const int32_t *perm, void *dst, int64_t ld_dst, const int32_t *rowmap,
                         cudaStream_t st, const char *kind) {
  const size_t es = esize(dtype);
  POET_REQUIRE((reinterpret_cast<uintptr_t>(src1) & 15) == 0 && ld1 * int64_t(es) % 16 == 0 &&
                   (split >= d || ((reinterpret_cast<uintptr_t>(src2) & 15) == 0 && ld2 * int64_t(es) % 16 == 0)),
               "scatter: frame rows must be 16-byte aligned");
  auto fill = [&](auto *tag) {
    using T = std::remove_pointer_t<decltype(tag)>;
    PermArgs<T> a{};
    a.src1 = static_cast<const T *>(src1); a.ld1 = ld1;
    a.src2 = static_cast<const T *>(src2); a.ld2 = ld2; a.split = split;
    a.src_rowmap = nullptr;
    a.rows = rows; a.d = d;
    a.perm = perm; a.inverse = 1;
    a.dst1 = static_cast<T *>(dst); a.ldd1 = ld_dst;
    a.dst2 = nullptr; a.ldd2 = 0; a.dsplit = d;
    a.dst_rowmap = rowmap;
    return launch_permute<T>(a, st, kind);
  };
  return dtype == POET_BF16 ? fill(static_cast<bf16 *>(nullptr)) : fill(static_cast<float *>(nullptr));
}

}  // namespace poet
