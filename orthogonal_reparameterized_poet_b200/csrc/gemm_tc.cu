// tcgen05 (5th-generation tensor core) engine of the batched GEMM, sm_100a.
//
//   C[b] = epilogue( A[b] . B[b]^T ),  A: M x K, B: N x K, bf16 in, fp32 accumulate
//
// Each operand is read by TMA (no multicast) in 64-element-wide slabs with the
// 128-byte swizzle, either K-major (K contiguous) or MN-major (M/N contiguous);
// the UMMA shared-memory descriptors describe both forms, so transposed
// operands (W0f^T in the backward, the token-contracted per-primitive
// gradients) need no transposed copy.
//
// Persistent, warp-specialized CTA (one per SM, 192 threads):
//   warp 0     TMA producer (one elected lane) filling a STAGES-deep ring
//   warp 1     TMEM allocator + MMA issuer (one elected lane):
//              tcgen05.mma.cta_group::1.kind::f16, M=128, N=BN, K=16
//   warps 2-5  epilogue: tcgen05.ld 32x32b rows out of TMEM, alpha/addends/
//              diagonal, bf16 and/or fp32 stores, or fp32 reductions (split-K);
//              single plain outputs are staged through shared memory so that
//              every store instruction covers four rows x 128 bytes
// The accumulator is double-buffered in TMEM (2 x BN columns), so the
// epilogue of one tile overlaps the MMAs of the next.
//
// CTA pairs (CG = 2, large streaming launches): two CTAs of a cluster run
// tcgen05.mma.cta_group::2 on 256 x 256 tiles.  Each loads its 128 rows of A
// and half of B; rank 0 issues the MMAs; stage and accumulator barriers are
// shared through multicast commits and remote arrivals; TMEM is allocated and
// freed by both CTAs together.
//
// Every mbarrier wait is bounded: after a time limit the CTA records
// ERR_TIMEOUT in the device status word, stops, drains what it issued (bounded
// too), frees TMEM and returns.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "poet_internal.cuh"

namespace poet {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;                      // one 128-byte swizzle row of bf16
constexpr int NTHREADS = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per wait

// One GEMM problem of a launch.
struct TcProblem {
  int M, N, K, batch;
  int num_m, num_n, nk, kchunk, splits;
  float alpha, beta, diag;
  const void *add; int add_f32; int64_t add_m, add_b;
  const void *add2; int add2_f32; int64_t add2_m, add2_b; float beta2;  // a second addend
  float *outF; int64_t of_m, of_b;
  bf16 *outD; int64_t od_m, od_b;
  int atomic;
  int coalesced;  // staged epilogue mode (0: per row; 1, 3: bf16; 2: fp32)
  int m_fast;     // tile order: M tiles fastest (N > M: CTAs of a wave share B slabs)
  int group_m;    // split-K: M tiles per group (a group runs all its splits before the next group)
};

// A launch: up to MAXP independent problems sharing operand majors and tile
// width, with their TMA descriptors, passed whole as a __grid_constant__
// kernel parameter.  Tiles of problem i are [tile_start[i], tile_start[i+1]).
template <int MAXP>
struct TcGroup {
  CUtensorMap ma[MAXP];
  CUtensorMap mb[MAXP];
  TcProblem prob[MAXP];
  int64_t tile_start[MAXP + 1];
  int count;
  unsigned *errword;
};

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false (after
// recording ERR_TIMEOUT and raising the CTA's abort flag) if it runs out, or
// if another role of the CTA has already aborted.
__device__ __noinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned *errword,
                                       uint64_t timeout_ns = kTimeoutNs) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > timeout_ns) {
        if (errword) atomicOr(errword, ERR_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---- CTA pairs (cta_group::2): two CTAs of a cluster share one 256-row MMA.
// The pair's MMAs are issued by rank 0; each CTA loads its half of A (128
// rows) and of B (half the N columns) and holds its 128 accumulator rows.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (no multicast)
__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the mbarrier at this offset in both CTAs of the pair once the pair's MMAs so far are done
__device__ __forceinline__ void umma_commit_pair_both(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(uint16_t(3))
      : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// UMMA shared-memory descriptor, 128-byte swizzle, sm_100 descriptor version.
//   K-major slab (rows of 64 elements = 128 B): SBO = 1024 B between 8-row groups.
//   MN-major slab (64 MN elements per 128-B row, one row per K):
//     LBO = bytes between 64-element MN chunks, SBO = 1024 B between 8-row K groups.
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFF);
  d |= uint64_t((lbo >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// Instruction descriptor, kind::f16: D f32, A and B bf16, M = MM, N = BN.
template <bool A_MN, bool B_MN, int BN, int MM = BM>
__device__ __forceinline__ uint32_t make_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(A_MN) << 15) | (uint32_t(B_MN) << 16) |
         (uint32_t(BN >> 3) << 17) | (uint32_t(MM >> 4) << 24);
}

struct TileCoord {
  int pi, b, s, mt, nt;
};
template <int MAXP>
__device__ __forceinline__ TileCoord decode(int64_t tile, const TcGroup<MAXP> &g) {
  int lo = 0, hi = g.count - 1;  // last problem with tile_start <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (g.tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  TileCoord c;
  c.pi = lo;
  const TcProblem &p = g.prob[lo];
  int64_t t = tile - g.tile_start[lo];
  if (p.splits > 1) {
    // split-K: groups of group_m M tiles; a group's tiles run split by split,
    // so its part of the float output is reduced into while it is in L2
    const int64_t per_b = int64_t(p.num_m) * p.num_n * p.splits;
    c.b = int(t / per_b);
    t %= per_b;
    const int64_t full = int64_t(p.group_m) * p.num_n * p.splits;
    const int grp = int(t / full);
    t %= full;
    const int m0 = grp * p.group_m;
    const int gm = p.num_m - m0 < p.group_m ? p.num_m - m0 : p.group_m;  // the last group may be smaller
    const int64_t per_split = int64_t(gm) * p.num_n;
    c.s = int(t / per_split);
    t %= per_split;
    if (p.m_fast) {
      c.mt = m0 + int(t % gm);
      c.nt = int(t / gm);
    } else {
      c.nt = int(t % p.num_n);
      c.mt = m0 + int(t / p.num_n);
    }
    return c;
  }
  if (p.m_fast) {
    c.mt = int(t % p.num_m);
    t /= p.num_m;
    c.nt = int(t % p.num_n);
    t /= p.num_n;
  } else {
    c.nt = int(t % p.num_n);
    t /= p.num_n;
    c.mt = int(t % p.num_m);
    t /= p.num_m;
  }
  c.s = int(t % p.splits);
  c.b = int(t / p.splits);
  return c;
}

// Shared-memory plan.  Streaming mode: a ring of (A slab, B slab) stages.
// B-stationary mode (BSTAT, problems with K <= 256 and one N tile): the whole
// B operand of the current (problem, batch) stays resident (KB_MAX slabs) and
// only A slabs stream through the ring.
constexpr int KB_MAX = 4;  // B-stationary: K <= 256
template <int BN, bool BSTAT = false, int CG = 1>
struct Smem {
  static constexpr int A_BYTES = BM * BK * 2;          // 16 KB
  static constexpr int B_BYTES = (BN / CG) * BK * 2;   // 32 KB (BN = 256), 16 KB per CTA of a pair
  static constexpr int STAGE_BYTES = BSTAT ? A_BYTES : A_BYTES + B_BYTES;
  static constexpr int STAGES = BSTAT ? 4 : (CG == 2 ? 6 : (BN == 256 ? 4 : 6));
  static constexpr int BRES_BYTES = BSTAT ? KB_MAX * B_BYTES : 0;  // resident B
  // epilogue staging: per epilogue warp 32 rows of one 64-column bf16 chunk
  // (plus up to 16 elements of shift and carry for rows that are not 16-byte
  // aligned), rows 176 B apart (11 16-byte units) so row-wise writes and
  // line-wise reads both take the minimum number of shared-memory wavefronts
  static constexpr int EPI_ROW = BSTAT ? 144 : 176;  // B-stationary launches have aligned rows only
  static constexpr int EPI_BYTES = 4 * 32 * EPI_ROW;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr size_t BYTES =
      size_t(STAGES) * STAGE_BYTES + BRES_BYTES + EPI_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// v[j] += beta * Add[off + j] for the j < nvalid values of one row chunk (Add
// float or bf16): 16-byte vector loads when the chunk is whole and aligned.
__device__ __forceinline__ void add_row(const void *add, int f32, int64_t off, float beta, int nvalid, float (&v)[32]) {
  if (f32) {
    const float *a = static_cast<const float *>(add) + off;
    if (nvalid == 32 && (reinterpret_cast<uintptr_t>(a) & 15) == 0) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 q = *reinterpret_cast<const float4 *>(a + j);
        v[j] += beta * q.x; v[j + 1] += beta * q.y; v[j + 2] += beta * q.z; v[j + 3] += beta * q.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nvalid) v[j] += beta * a[j];
    }
  } else {
    const uint16_t *a = static_cast<const uint16_t *>(add) + off;
    if (nvalid == 32 && (reinterpret_cast<uintptr_t>(a) & 15) == 0) {
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        const uint4 q = *reinterpret_cast<const uint4 *>(a + j);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[j + 2 * e] += beta * bf16_bits_to_float(uint16_t(w[e] & 0xFFFFu));
          v[j + 2 * e + 1] += beta * bf16_bits_to_float(uint16_t(w[e] >> 16));
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nvalid) v[j] += beta * bf16_bits_to_float(a[j]);
    }
  }
}

// out[0..3] += (a, b, c, d) as one 16-byte reduction at L2
__device__ __forceinline__ void red_add_v4(float *out, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(out), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

template <bool A_MN, bool B_MN, int BN, int MAXP, bool BSTAT, int CG>
__global__ void __launch_bounds__(NTHREADS, 1) gemm_tc_kernel(const __grid_constant__ TcGroup<MAXP> g) {
  static_assert(CG == 1 || (CG == 2 && BN == 256 && !BSTAT), "CTA pairs run 256 x 256 streaming tiles");
  using S = Smem<BN, BSTAT, CG>;
  constexpr int STAGES = S::STAGES;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char *stage_base = smem;
  unsigned char *bres = smem + size_t(STAGES) * S::STAGE_BYTES;  // resident B (B-stationary only)
  unsigned char *epi = bres + S::BRES_BYTES;                      // epilogue staging
  uint64_t *bars = reinterpret_cast<uint64_t *>(epi + S::EPI_BYTES);
  uint64_t *full = bars;                 // [STAGES]
  uint64_t *empty = bars + STAGES;       // [STAGES]
  uint64_t *tfull = bars + 2 * STAGES;   // [2]
  uint64_t *tempty = tfull + 2;          // [2]
  uint64_t *drain = tempty + 2;          // [1]
  uint64_t *bfull = drain + 1;           // [1] resident B landed
  uint64_t *bfree = bfull + 1;           // [1] MMAs reading the resident B are done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bfree + 1);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t tiles = g.tile_start[g.count];
  // CTA pairs: rank 0 issues the pair's MMAs; rank r holds rows r*128.. of each 256-row tile
  const uint32_t rank = CG == 2 ? cluster_rank() : 0;
  const bool leader = rank == 0;
  const int64_t units = CG == 2 ? int64_t(cluster_count()) : int64_t(gridDim.x);
  const int64_t unit = CG == 2 ? int64_t(cluster_id()) : int64_t(blockIdx.x);
  // Tiles of this CTA (pair): one contiguous range (B-stationary, so that
  // consecutive tiles share their B operand), or one tile of each wave of
  // `units` consecutive tiles (streaming), the waves taken in alternating
  // directions.  The host orders a launch's problems by decreasing K, so the
  // long tiles come first and the short ones of the later waves even out
  // what the long ones left; within a wave the tiles stay consecutive, which
  // keeps their shared operand slabs together in L2.
  const int64_t per_cta = (tiles + units - 1) / units;
  const int64_t t_first = BSTAT ? unit * per_cta : unit;
  const int64_t t_end = BSTAT ? (t_first + per_cta < tiles ? t_first + per_cta : tiles) : tiles;
  auto tile_of = [&](int64_t k) -> int64_t {
    if (BSTAT) return t_first + k;
    return k * units + ((k & 1) ? units - 1 - unit : unit);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4 * CG);  // the epilogue warps of every CTA of the pair
    }
    mbar_init(drain, 1);
    mbar_init(bfull, 1);
    mbar_init(bfree, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // a pair allocates collectively (the same warp of both CTAs)
    if constexpr (CG == 2) {
      tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, S::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync_all();  // barriers initialised in both CTAs before any remote use
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int last_stage = -1;
      uint32_t last_phase = 0;
      int last_pi = -1;
      int res_pi = -1, res_b = -1;   // B-stationary: operand currently resident
      uint32_t bfree_phase = 0;
      uint32_t bloads = 0;
      const uint32_t full0 = CG == 2 ? mapa_shared(smem_u32(full), 0) : 0;  // rank 0's full[0]
      for (int64_t k = 0;; ++k) {
        const int64_t tile = tile_of(k);
        if (tile >= t_end || *abort) break;
        const TileCoord c = decode(tile, g);
        const TcProblem &p = g.prob[c.pi];
        const CUtensorMap *ma = &g.ma[c.pi];
        const CUtensorMap *mb = &g.mb[c.pi];
        if (c.pi != last_pi) {
          tma_prefetch_desc(ma);
          tma_prefetch_desc(mb);
          last_pi = c.pi;
        }
        if constexpr (BSTAT) {
          if (c.pi != res_pi || c.b != res_b) {  // load this (problem, batch)'s whole B once
            if (res_pi >= 0) {
              if (!mbar_wait(bfree, bfree_phase, abort, g.errword)) break;
              bfree_phase ^= 1;
            }
            mbar_expect_tx(bfull, uint32_t(p.nk) * S::B_BYTES);
            ++bloads;
            for (int kb = 0; kb < p.nk; ++kb) {
              unsigned char *sb = bres + size_t(kb) * S::B_BYTES;
              if (!B_MN) {
                tma_load_3d(sb, mb, bfull, kb * BK, c.nt * BN, c.b);
              } else {
#pragma unroll
                for (int q = 0; q < BN / 64; ++q) tma_load_3d(sb + q * 8192, mb, bfull, c.nt * BN + 64 * q, kb * BK, c.b);
              }
            }
            res_pi = c.pi;
            res_b = c.b;
          }
        }
        const int kb0 = c.s * p.kchunk;
        const int kb1 = min(p.nk, kb0 + p.kchunk);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort, g.errword)) break;
          unsigned char *sa = stage_base + size_t(stage) * S::STAGE_BYTES;
          unsigned char *sb = sa + S::A_BYTES;
          if constexpr (CG == 2) {
            // both halves land on rank 0's full barrier, which expects the pair's bytes
            if (leader) mbar_expect_tx(&full[stage], 2 * S::STAGE_BYTES);
            const uint32_t fb = full0 + uint32_t(stage) * 8u;
            const int row0 = c.mt * (2 * BM) + int(rank) * BM;
            const int col0 = c.nt * BN + int(rank) * (BN / 2);
            if (!A_MN) {
              tma_load_3d_pair(sa, ma, fb, kb * BK, row0, c.b);
            } else {
#pragma unroll
              for (int q = 0; q < BM / 64; ++q) tma_load_3d_pair(sa + q * 8192, ma, fb, row0 + 64 * q, kb * BK, c.b);
            }
            if (!B_MN) {
              tma_load_3d_pair(sb, mb, fb, kb * BK, col0, c.b);
            } else {
#pragma unroll
              for (int q = 0; q < BN / 128; ++q) tma_load_3d_pair(sb + q * 8192, mb, fb, col0 + 64 * q, kb * BK, c.b);
            }
          } else {
          mbar_expect_tx(&full[stage], S::STAGE_BYTES);
          if (!A_MN) {
            tma_load_3d(sa, ma, &full[stage], kb * BK, c.mt * BM, c.b);
          } else {
#pragma unroll
            for (int q = 0; q < BM / 64; ++q) tma_load_3d(sa + q * 8192, ma, &full[stage], c.mt * BM + 64 * q, kb * BK, c.b);
          }
          if constexpr (!BSTAT) {
            if (!B_MN) {
              tma_load_3d(sb, mb, &full[stage], kb * BK, c.nt * BN, c.b);
            } else {
#pragma unroll
              for (int q = 0; q < BN / 64; ++q) tma_load_3d(sb + q * 8192, mb, &full[stage], c.nt * BN + 64 * q, kb * BK, c.b);
            }
          }
          }
          last_stage = stage;
          last_phase = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort && last_stage >= 0) {
        if (CG == 1 || leader) {
          // drain: the most recent copies (bounded)
          volatile int no_abort = 0;
          mbar_wait(&full[last_stage], last_phase, &no_abort, nullptr);
        } else {
          // the second CTA of a pair cannot wait on rank 0's barrier: give its
          // copies in flight a fixed 200 us to land
          const uint64_t t0 = globaltimer();
          while (globaltimer() - t0 < 200000ull) {
          }
        }
      }
      if (BSTAT && *abort && bloads > 0) {
        volatile int no_abort = 0;
        mbar_wait(bfull, (bloads - 1) & 1, &no_abort, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && (CG == 1 || leader)) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc = make_idesc<A_MN, B_MN, BN, BM * CG>();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      int res_pi = -1, res_b = -1;  // B-stationary: operand currently resident
      uint32_t bfull_phase = 0;
      bool ready = false;  // the next k-block's stage has been seen full
      for (int64_t k = 0;; ++k) {
        const int64_t tile = tile_of(k);
        if (tile >= t_end || *abort) break;
        const TileCoord c = decode(tile, g);
        const TcProblem &p = g.prob[c.pi];
        const int kb0 = c.s * p.kchunk;
        const int kb1 = min(p.nk, kb0 + p.kchunk);
        if constexpr (BSTAT) {
          if (c.pi != res_pi || c.b != res_b) {
            if (!mbar_wait(bfull, bfull_phase, abort, g.errword)) break;
            bfull_phase ^= 1;
            res_pi = c.pi;
            res_b = c.b;
          }
        }
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort, g.errword)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        bool ok = true;
        // The barrier of the next k-block's stage is tested before this
        // k-block's MMAs are issued, so that the test's round trip overlaps
        // the issue.  A test on the path between k-blocks left the tensor pipe
        // idle about a third of the time.
        auto issue_kb = [&](int kb) {
          const uint32_t sa = smem_u32(stage_base + size_t(stage) * S::STAGE_BYTES);
          const uint32_t sb = BSTAT ? smem_u32(bres + size_t(kb) * S::B_BYTES) : sa + S::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? make_desc(sa + kk * 2048, 8192, 1024) : make_desc(sa + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? make_desc(sb + kk * 2048, 8192, 1024) : make_desc(sb + kk * 32, 16, 1024);
            if constexpr (CG == 2) umma_bf16_pair(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
            else umma_bf16(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          if constexpr (CG == 2) umma_commit_pair_both(&empty[stage]);
          else umma_commit(&empty[stage]);
          issued = true;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        };
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!ready && !mbar_wait(&full[stage], phase, abort, g.errword)) { ok = false; break; }
          tc_fence_after();
          const int s1 = stage + 1 == STAGES ? 0 : stage + 1;
          const uint32_t ph1 = stage + 1 == STAGES ? phase ^ 1 : phase;
          ready = mbar_test(&full[s1], ph1);  // the ring runs on across tiles
          issue_kb(kb);
        }
        if (!ok) break;
        if constexpr (CG == 2) umma_commit_pair_both(&tfull[acc]);
        else umma_commit(&tfull[acc]);
        if constexpr (BSTAT) {
          // the resident B is released after the last tile that reads it
          bool last_use = tile_of(k + 1) >= t_end;
          if (!last_use) {
            const TileCoord nc = decode(tile_of(k + 1), g);
            last_use = nc.pi != c.pi || nc.b != c.b;
          }
          if (last_use) umma_commit(bfree);
        }
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (*abort && issued) {
        // drain: every MMA issued so far has completed once this commit arrives
        if constexpr (CG == 2) umma_commit_pair(drain);
        else umma_commit(drain);
        volatile int no_abort = 0;
        mbar_wait(drain, 0, &no_abort, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp % 4;
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t k = 0;; ++k) {
      const int64_t tile = tile_of(k);
      if (tile >= t_end || *abort) break;
      const TileCoord c = decode(tile, g);
      // A copy, not a reference: the problem's fields then live in registers.
      // Read in place, every use went back to the kernel's parameter space
      // (each asm with a memory clobber forces a reload), which cost about a
      // quarter of a tile's epilogue.
      const TcProblem p = g.prob[c.pi];
      if (!mbar_wait(&tfull[acc], acc_phase, abort, g.errword)) break;
      tc_fence_after();
      const int mrow0 = c.mt * (BM * CG) + int(rank) * BM;  // this CTA's first accumulator row
      const int gm = mrow0 + row;
      const bool row_ok = gm < p.M;
      const float alpha = p.alpha, beta = p.beta, diag = p.diag;
      if (p.coalesced == 1 || p.coalesced == 3) {
        // plain bf16 output: each 64-column chunk goes row-wise into this warp's
        // staging rows, then out with every store instruction covering four
        // rows x 128 contiguous bytes.
        // Mode 3 (rows not 16-byte aligned): a row's chunk is staged shifted by
        // the row's misalignment q (elements mod 8 of the tile's first column),
        // so that the 16-byte units of the output row are 16-byte units of the
        // staging row; the last q columns of a chunk carry over to the front of
        // the next one.  Units then go out exactly as in mode 1, and only the
        // first 8 - q and last q columns of a tile row (16-byte units shared
        // with the neighbouring tiles) are written as single elements.
        unsigned char *ew = epi + quarter * (32 * S::EPI_ROW);
        const int m_base = mrow0 + quarter * 32;
        bf16 *obase = p.outD + int64_t(c.b) * p.od_b;
        const int sub = lane & 7, rsub = lane >> 3;
        const int nt0 = c.nt * BN;
        const bool mis_rows = !BSTAT && p.coalesced == 3;  // B-stationary launches never get mode 3
        const bool my_row_ok = m_base + lane < p.M;
        uint16_t *myout = reinterpret_cast<uint16_t *>(obase + int64_t(m_base + lane) * p.od_m + nt0);
        const int qrow = mis_rows ? int((reinterpret_cast<uintptr_t>(myout) >> 1) & 7) : 0;
        for (int cc = 0; cc < BN / 64; ++cc) {
          uint32_t r0[32], r1[32];
          __syncwarp();
          const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN + cc * 64);
          tmem_ld32(taddr, r0);
          tmem_ld32(taddr + 32, r1);
          tmem_ld_wait();
          const int gn0 = nt0 + cc * 64;
          if (gn0 >= p.N) continue;  // the same for the whole warp
          unsigned char *myrow = ew + lane * S::EPI_ROW;
          uint16_t *row16 = reinterpret_cast<uint16_t *>(myrow);
          if (mis_rows && cc > 0) *reinterpret_cast<uint4 *>(myrow + 16) = *reinterpret_cast<const uint4 *>(myrow + 144);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t *src = q < 4 ? r0 + 8 * q : r1 + 8 * (q - 4);
            uint4 pk;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(alpha * __uint_as_float(src[0]), alpha * __uint_as_float(src[1]));
            __nv_bfloat162 h1 = __floats2bfloat162_rn(alpha * __uint_as_float(src[2]), alpha * __uint_as_float(src[3]));
            __nv_bfloat162 h2 = __floats2bfloat162_rn(alpha * __uint_as_float(src[4]), alpha * __uint_as_float(src[5]));
            __nv_bfloat162 h3 = __floats2bfloat162_rn(alpha * __uint_as_float(src[6]), alpha * __uint_as_float(src[7]));
            pk.x = *reinterpret_cast<uint32_t *>(&h0);
            pk.y = *reinterpret_cast<uint32_t *>(&h1);
            pk.z = *reinterpret_cast<uint32_t *>(&h2);
            pk.w = *reinterpret_cast<uint32_t *>(&h3);
            if (!mis_rows) {
              *reinterpret_cast<uint4 *>(myrow + q * 16) = pk;
            } else {  // elements 8 + qrow + 8q ... (2-byte aligned)
              uint16_t *d = row16 + 8 + qrow + 8 * q;
              d[0] = uint16_t(pk.x); d[1] = uint16_t(pk.x >> 16);
              d[2] = uint16_t(pk.y); d[3] = uint16_t(pk.y >> 16);
              d[4] = uint16_t(pk.z); d[5] = uint16_t(pk.z >> 16);
              d[6] = uint16_t(pk.w); d[7] = uint16_t(pk.w >> 16);
            }
          }
          if (mis_rows && cc == 0 && qrow > 0 && my_row_ok) {
            // head: columns [0, 8 - q) end the 16-byte unit the previous tile begins
            for (int e = 0; e < 8 - qrow; ++e)
              if (nt0 + e < p.N) myout[e] = row16[8 + qrow + e];
          }
          __syncwarp();
          if (mis_rows) {
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int rr = it * 4 + rsub;
              const int gm = m_base + rr;
              if (gm >= p.M) continue;
              uint16_t *orow = reinterpret_cast<uint16_t *>(obase + int64_t(gm) * p.od_m + nt0);
              const int qr = int((reinterpret_cast<uintptr_t>(orow) >> 1) & 7);
              if (cc == 0 && qr > 0 && sub == 0) continue;  // the head, written above
              const int col = cc * 64 - qr + 8 * sub;        // tile column of this 16-byte unit
              if (nt0 + col >= p.N) continue;
              const uint4 v = *reinterpret_cast<const uint4 *>(ew + rr * S::EPI_ROW + 16 + sub * 16);
              if (nt0 + col + 8 <= p.N) {
                *reinterpret_cast<uint4 *>(orow + col) = v;
              } else {
                const uint16_t *pv = reinterpret_cast<const uint16_t *>(&v);
                for (int e = 0; e < 8; ++e)
                  if (nt0 + col + e < p.N) orow[col + e] = pv[e];
              }
            }
            // tail after the tile's last chunk: its last q columns (staged at 72..)
            const bool last_chunk = cc == BN / 64 - 1 || gn0 + 64 >= p.N;
            if (last_chunk && qrow > 0 && my_row_ok) {
              for (int e = 0; e < qrow; ++e) {
                const int col = cc * 64 + 64 - qrow + e;
                if (nt0 + col < p.N) myout[col] = row16[72 + e];
              }
            }
            continue;
          }
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + rsub;
            const int gm = m_base + rr;
            const int gn = gn0 + sub * 8;
            const uint4 v = *reinterpret_cast<const uint4 *>(ew + rr * S::EPI_ROW + sub * 16);
            if (gm < p.M && gn < p.N) {
              bf16 *o = obase + int64_t(gm) * p.od_m + gn;
              if (gn + 8 <= p.N) {
                *reinterpret_cast<uint4 *>(o) = v;
              } else {
                const bf16 *pv = reinterpret_cast<const bf16 *>(&v);
                for (int e = 0; e < 8; ++e)
                  if (gn + e < p.N) o[e] = pv[e];
              }
            }
          }
        }
      } else if (p.coalesced == 2) {
        // plain fp32 output: each 32-column chunk (128 B per row) goes row-wise
        // into this warp's staging rows, then out four rows x 128 B at a time
        unsigned char *ew = epi + quarter * (32 * S::EPI_ROW);
        const int m_base = mrow0 + quarter * 32;
        float *obase = p.outF + int64_t(c.b) * p.of_b;
        const int sub = lane & 7, rsub = lane >> 3;
        unsigned char *myrow = ew + lane * S::EPI_ROW;
        for (int cc = 0; cc < BN / 32; ++cc) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld32(tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN + cc * 32), r);
          tmem_ld_wait();
          const int gn0 = c.nt * BN + cc * 32;
          if (gn0 >= p.N) continue;  // the same for the whole warp
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float4 f;
            f.x = alpha * __uint_as_float(r[4 * q]);
            f.y = alpha * __uint_as_float(r[4 * q + 1]);
            f.z = alpha * __uint_as_float(r[4 * q + 2]);
            f.w = alpha * __uint_as_float(r[4 * q + 3]);
            *reinterpret_cast<float4 *>(myrow + q * 16) = f;
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + rsub;
            const int gm = m_base + rr;
            const int gn = gn0 + sub * 4;
            const float4 f = *reinterpret_cast<const float4 *>(ew + rr * S::EPI_ROW + sub * 16);
            if (gm < p.M && gn < p.N) {
              float *o = obase + int64_t(gm) * p.of_m + gn;
              if (p.atomic) {  // split-K: float reductions at L2, four rows x 128 B per instruction
                if (gn + 4 <= p.N) {
                  red_add_v4(o, f.x, f.y, f.z, f.w);
                } else {
                  atomicAdd(o, f.x);  // gn < N
                  if (gn + 1 < p.N) atomicAdd(o + 1, f.y);
                  if (gn + 2 < p.N) atomicAdd(o + 2, f.z);
                }
              } else if (gn + 4 <= p.N) {
                *reinterpret_cast<float4 *>(o) = f;
              } else {
                o[0] = f.x;  // gn < N
                if (gn + 1 < p.N) o[1] = f.y;
                if (gn + 2 < p.N) o[2] = f.z;
              }
            }
          }
        }
      } else
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN + cc * 32), r);
        tmem_ld_wait();
        const int gn0 = c.nt * BN + cc * 32;
        if (!row_ok || gn0 >= p.N) continue;
        const int nvalid = min(32, p.N - gn0);
        if (p.atomic) {
          float *o = p.outF + int64_t(c.b) * p.of_b + int64_t(gm) * p.of_m + gn0;
          if (nvalid == 32 && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              red_add_v4(o + j, alpha * __uint_as_float(r[j]), alpha * __uint_as_float(r[j + 1]),
                         alpha * __uint_as_float(r[j + 2]), alpha * __uint_as_float(r[j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) atomicAdd(o + j, alpha * __uint_as_float(r[j]));
          }
          continue;
        }
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = alpha * __uint_as_float(r[j]);
        if (p.add) add_row(p.add, p.add_f32, int64_t(c.b) * p.add_b + int64_t(gm) * p.add_m + gn0, beta, nvalid, v);
        if (p.add2) add_row(p.add2, p.add2_f32, int64_t(c.b) * p.add2_b + int64_t(gm) * p.add2_m + gn0, p.beta2, nvalid, v);
        if (diag != 0.f && gm >= gn0 && gm < gn0 + 32) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (gn0 + j == gm) v[j] += diag;
        }
        if (p.outF) {
          float *o = p.outF + int64_t(c.b) * p.of_b + int64_t(gm) * p.of_m + gn0;
          if (nvalid == 32 && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4 *>(o + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) o[j] = v[j];
          }
        }
        if (p.outD) {
          bf16 *o = p.outD + int64_t(c.b) * p.od_b + int64_t(gm) * p.od_m + gn0;
          if (nvalid == 32 && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 pk;
              __nv_bfloat162 h0 = __floats2bfloat162_rn(v[j], v[j + 1]);
              __nv_bfloat162 h1 = __floats2bfloat162_rn(v[j + 2], v[j + 3]);
              __nv_bfloat162 h2 = __floats2bfloat162_rn(v[j + 4], v[j + 5]);
              __nv_bfloat162 h3 = __floats2bfloat162_rn(v[j + 6], v[j + 7]);
              pk.x = *reinterpret_cast<uint32_t *>(&h0);
              pk.y = *reinterpret_cast<uint32_t *>(&h1);
              pk.z = *reinterpret_cast<uint32_t *>(&h2);
              pk.w = *reinterpret_cast<uint32_t *>(&h3);
              *reinterpret_cast<uint4 *>(o + j) = pk;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) o[j] = __float2bfloat16_rn(v[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // the accumulator is released on the CTA that issues the MMAs
        if constexpr (CG == 2) mbar_arrive_remote(mapa_shared(smem_u32(&tempty[acc]), 0));
        else mbar_arrive(&tempty[acc]);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  // a pair frees its TMEM together, after every MMA of the pair has completed
  // and both CTAs' epilogues have read their accumulators
  if constexpr (CG == 2) cluster_sync_all();
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2) tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
    else tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

// Failure-detection self test: one thread waits, through the same bounded wait
// the GEMM roles use, on a barrier that nothing arrives on.  The wait runs out
// after timeout_ns, records ERR_TIMEOUT in the device status word and the
// kernel returns normally (no trap, no fault: the context stays usable).
__global__ void bounded_wait_selftest_kernel(unsigned *errword, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, errword, timeout_ns);
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 3-D map (inner, outer, batch) over a bf16 operand; strides in elements.
bool make_map(CUtensorMap *map, const void *base, int64_t inner, int64_t outer, int batch, int64_t outer_stride,
              int64_t batch_stride, uint32_t box_inner, uint32_t box_outer) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(inner), cuuint64_t(outer), cuuint64_t(batch)};
  int64_t bstride = batch > 1 ? batch_stride : outer_stride * outer;
  bstride = round_up(bstride > 0 ? bstride : 8, 8);
  cuuint64_t strides[2] = {cuuint64_t(outer_stride) * 2, cuuint64_t(bstride) * 2};
  cuuint32_t box[3] = {box_inner, box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// CTA pairs: POET_GEMM_PAIRS=0 turns them off (the single-CTA engine serves
// every shape), =2 uses them for every streaming launch with problems at least
// 256 rows tall (tests cover the pair engine at small sizes this way).
const int g_pairs_mode = [] {
  const char *e = std::getenv("POET_GEMM_PAIRS");
  if (e && e[0] == '0') return 0;
  if (e && e[0] == '2') return 2;
  return 1;
}();

// Split-K: POET_GEMM_SPLITK_MAX=n caps the number of K splits of a launch with
// float-reduced outputs (default 16; 1 turns split-K off).
const int g_splitk_max = [] {
  const char *e = std::getenv("POET_GEMM_SPLITK_MAX");
  const int v = e ? std::atoi(e) : 16;
  return v < 1 ? 1 : (v > 16 ? 16 : v);
}();

// POET_GEMM_BSTAT=0 turns the B-stationary kernels off (such problems stream
// both operands).
const bool g_bstat = [] {
  const char *e = std::getenv("POET_GEMM_BSTAT");
  return !(e && e[0] == '0');
}();

// Operand majors and tile width of a supported problem.
struct TcPlan {
  bool A_MN, B_MN;
  int BN;
  bool bstat;  // B-stationary (whole B of a batch resident; contiguous tiles per CTA)
  int cg = 1;  // CTAs per MMA: 2 = CTA pairs on 256 x 256 tiles
  bool operator==(const TcPlan &o) const {
    return A_MN == o.A_MN && B_MN == o.B_MN && BN == o.BN && bstat == o.bstat && cg == o.cg;
  }
};
TcPlan plan_of(const Gemm &g) {
  TcPlan t;
  t.A_MN = !(g.a_k == 1 && g.a_m % 8 == 0);
  t.B_MN = !(g.b_k == 1 && g.b_n % 8 == 0);
  t.BN = g.N <= 128 ? 128 : 256;
  // token-streaming products against a small operand (block-diagonal passes
  // with 256-wide blocks): keep B resident when it fits and many M tiles
  // share it
  t.bstat = g_bstat && t.BN == 256 && g.N <= 256 && g.K <= KB_MAX * BK && g.M >= 8 * BM && !g.atomic;
  return t;
}

// Fill one problem of a group (tiles use split-K only for atomic outputs).
bool fill_problem(const Gemm &g, const TcPlan &t, int split_want, TcProblem *p, CUtensorMap *ma, CUtensorMap *mb) {
  p->M = g.M; p->N = g.N; p->K = g.K; p->batch = g.batch;
  p->num_m = (g.M + BM * t.cg - 1) / (BM * t.cg);
  p->num_n = (g.N + t.BN - 1) / t.BN;
  p->nk = (g.K + BK - 1) / BK;
  int splits = g.atomic ? (split_want < p->nk ? split_want : p->nk) : 1;
  if (splits < 1) splits = 1;
  p->kchunk = (p->nk + splits - 1) / splits;
  p->splits = (p->nk + p->kchunk - 1) / p->kchunk;
  p->alpha = g.alpha; p->beta = g.beta; p->diag = g.diag;
  p->add = g.add; p->add_f32 = g.add_dtype == POET_F32; p->add_m = g.add_m; p->add_b = g.add_b;
  p->add2 = g.add2; p->add2_f32 = g.add2_dtype == POET_F32; p->add2_m = g.add2_m; p->add2_b = g.add2_b;
  p->beta2 = g.beta2;
  p->outF = g.outF; p->of_m = g.of_m; p->of_b = g.of_b;
  p->outD = static_cast<bf16 *>(g.outD); p->od_m = g.od_m; p->od_b = g.od_b;
  p->atomic = g.atomic && p->splits > 1 ? 1 : 0;  // one split: the zeroed output is simply stored
  // consecutive tiles (one wave of persistent CTAs) share the slabs of the
  // larger operand, which is then read from HBM about once
  p->m_fast = g.N > g.M ? 1 : 0;
  // split-K groups: about one wave of tile workers (CTAs or CTA pairs) per group
  {
    const int workers = num_sms() / t.cg;
    int gm = workers / (p->num_n > 0 ? p->num_n : 1);
    if (gm < 1) gm = 1;
    if (gm > p->num_m) gm = p->num_m;
    p->group_m = gm;
  }
  // staged epilogue for a single plain output (1: bf16, 16-byte aligned rows;
  // 3: bf16, any rows; 2: fp32, 16-byte aligned rows, stored or reduced); the
  // per-row path handles addends, pairs of outputs and unaligned fp32 rows
  p->coalesced = 0;
  const bool plain = !g.add && !g.add2 && !g.atomic && g.diag == 0.f;
  if (plain && g.outD && !g.outF) {
    p->coalesced = aligned16(g.outD) && g.od_m % 8 == 0 && (g.batch == 1 || g.od_b % 8 == 0) ? 1 : 3;
    if (t.bstat && p->coalesced == 3) p->coalesced = 0;  // the B-stationary kernels stage aligned rows only
  }
  // fp32: plain stores or split-K reductions
  if (!g.add && !g.add2 && g.diag == 0.f && g.outF && !g.outD && aligned16(g.outF) && g.of_m % 4 == 0 &&
      (g.batch == 1 || g.of_b % 4 == 0))
    p->coalesced = 2;
  bool ok;
  if (!t.A_MN) ok = make_map(ma, g.A, g.K, g.M, g.batch, g.a_m, g.a_b, 64, BM);
  else ok = make_map(ma, g.A, g.M, g.K, g.batch, g.a_k, g.a_b, 64, 64);
  if (ok) {
    if (!t.B_MN) ok = make_map(mb, g.B, g.K, g.N, g.batch, g.b_n, g.b_b, 64, t.BN / t.cg);
    else ok = make_map(mb, g.B, g.N, g.K, g.batch, g.b_k, g.b_b, 64, 64);
  }
  return ok;
}

template <bool A_MN, bool B_MN, int BN, int MAXP, bool BSTAT = false, int CG = 1>
poet_status launch(const TcGroup<MAXP> &grp, cudaStream_t st) {
  using S = Smem<BN, BSTAT, CG>;
  auto kern = gemm_tc_kernel<A_MN, B_MN, BN, MAXP, BSTAT, CG>;
  static bool configured[64] = {};
  static int max_pairs[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    POET_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(S::BYTES)));
    configured[dev] = true;
  }
  const int64_t tiles = grp.tile_start[grp.count];
  if constexpr (CG == 1) {
    const int64_t grid = tiles < num_sms() ? tiles : num_sms();
    kern<<<int(grid), NTHREADS, S::BYTES, st>>>(grp);
  } else {
    // persistent CTA pairs: one cluster of two CTAs per pair of SMs, as many
    // as can be resident at once
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = S::BYTES;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (dev < 64 && max_pairs[dev] == 0) {
      cfg.gridDim = dim3(2 * (num_sms() / 2));
      int n = 0;
      POET_CUDA_TRY(cudaOccupancyMaxActiveClusters(&n, kern, &cfg));
      max_pairs[dev] = n > 0 ? n : num_sms() / 2;
    }
    const int64_t cap = dev < 64 ? max_pairs[dev] : num_sms() / 2;
    const int64_t pairs = tiles < cap ? tiles : cap;
    cfg.gridDim = dim3(unsigned(2 * pairs));
    POET_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, grp));
  }
  count_launch();
  return launch_status("gemm_tc");
}

template <int MAXP>
poet_status run_group(const Gemm *gs, int n, const TcPlan &t, cudaStream_t st) {
  static thread_local TcGroup<MAXP> grp;  // large: keep it off the stack
  int64_t base_tiles = 0;
  double kb_sum = 0.0;  // k-blocks summed over the base tiles
  for (int i = 0; i < n; ++i) {
    const int64_t mt = (gs[i].M + BM * t.cg - 1) / (BM * t.cg), nt = (gs[i].N + t.BN - 1) / t.BN;
    base_tiles += mt * nt * gs[i].batch;
    kb_sum += double(mt * nt * gs[i].batch) * double((gs[i].K + BK - 1) / BK);
  }
  // Split K (atomic outputs only) into s parts, for launches of less than two
  // full waves only: on the weight plan's launches of 4-11 waves (tiles of
  // 16-512 k-blocks) one split beat every other.  A tile of k k-blocks takes
  // about max(k, kEpiKb) + 1 k-block times (its float reduction takes about
  // kEpiKb, overlapped with the next tile's products), the tiles run in
  // ceil(tiles / workers) waves, and each further split costs about 3.5% more
  // (the output is zeroed and reduced into through L2); s minimizes
  // waves(s) * (max(kavg / s, kEpiKb) + 1) * (1 + 0.035 (s - 1)), the smallest
  // s within 1% of the best.  (Filling waves alone picked up to 15 splits of
  // 2048-deep products whose every 3-k-block tile then waited on a whole
  // tile's reduction.)
  int split_want = 1;
  bool any_atomic = false;
  for (int i = 0; i < n; ++i) any_atomic |= gs[i].atomic;
  const int64_t workers = num_sms() / t.cg;  // concurrent tile workers: CTAs or CTA pairs
  if (any_atomic && base_tiles > 0 && base_tiles < 2 * workers) {
    constexpr double kEpiKb = 6.0;
    constexpr double kSplitCost = 0.035;  // each further split: zeroing and reducing the whole output
    const double kavg = kb_sum / double(base_tiles);
    double cost[17] = {};
    double best = 0.0;
    for (int sp = 1; sp <= g_splitk_max; ++sp) {
      const int64_t waves = (base_tiles * sp + workers - 1) / workers;
      const double per = kavg / sp;
      cost[sp] = double(waves) * ((per > kEpiKb ? per : kEpiKb) + 1.0) * (1.0 + kSplitCost * (sp - 1));
      if (sp == 1 || cost[sp] < best) best = cost[sp];
    }
    for (int sp = 1; sp <= g_splitk_max; ++sp)
      if (cost[sp] <= 1.01 * best) { split_want = sp; break; }
  }
  std::vector<ZeroRegion> zero;  // outputs of split problems, zeroed in one launch before the products
  // problems in decreasing K order (their tiles' length; ties keep the list order)
  int order[MAXP];
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order, order + n, [&](int a, int b) { return gs[a].K > gs[b].K; });
  grp.count = n;
  grp.errword = device_errword();
  grp.tile_start[0] = 0;
  for (int i = 0; i < n; ++i) {
    TcProblem &p = grp.prob[i];
    const Gemm &gi = gs[order[i]];
    if (!fill_problem(gi, t, split_want, &p, &grp.ma[i], &grp.mb[i])) {
      set_error("gemm_tc: tensor map encoding failed (M=%d N=%d K=%d)", gi.M, gi.N, gi.K);
      return POET_ECUDA;
    }
    grp.tile_start[i + 1] = grp.tile_start[i] + int64_t(p.num_m) * p.num_n * p.splits * p.batch;
    if (p.atomic) zero.push_back(ZeroRegion{gi.outF, gi.M, gi.N, gi.of_m, gi.batch, gi.of_b});  // split: reduced into
  }
  if (!zero.empty()) POET_TRY(zero_outputs(zero, st));
  if constexpr (MAXP == 1) {
    if (t.bstat && !t.A_MN) {
      if (!t.B_MN) return launch<false, false, 256, MAXP, true>(grp, st);
      return launch<false, true, 256, MAXP, true>(grp, st);
    }
  }
  if (t.BN == 128) {
    if (!t.A_MN && !t.B_MN) return launch<false, false, 128, MAXP>(grp, st);
    if (!t.A_MN && t.B_MN) return launch<false, true, 128, MAXP>(grp, st);
    if (t.A_MN && !t.B_MN) return launch<true, false, 128, MAXP>(grp, st);
    return launch<true, true, 128, MAXP>(grp, st);
  }
  if (t.cg == 2) {
    if (!t.A_MN && !t.B_MN) return launch<false, false, 256, MAXP, false, 2>(grp, st);
    if (!t.A_MN && t.B_MN) return launch<false, true, 256, MAXP, false, 2>(grp, st);
    if (t.A_MN && !t.B_MN) return launch<true, false, 256, MAXP, false, 2>(grp, st);
    return launch<true, true, 256, MAXP, false, 2>(grp, st);
  }
  if (!t.A_MN && !t.B_MN) return launch<false, false, 256, MAXP>(grp, st);
  if (!t.A_MN && t.B_MN) return launch<false, true, 256, MAXP>(grp, st);
  if (t.A_MN && !t.B_MN) return launch<true, false, 256, MAXP>(grp, st);
  return launch<true, true, 256, MAXP>(grp, st);
}

constexpr int kGroupMax = 64;  // ~25 KB of kernel parameters (limit 32 KB)
static_assert(sizeof(TcGroup<kGroupMax>) <= 32000, "grouped launch parameters exceed the kernel parameter limit");

}  // namespace

bool gemm_tc_enabled() { return encoder() != nullptr; }

bool gemm_tc_supported(const Gemm &g) {
  if (g.dtype != POET_BF16 || g.K < 1 || g.M < 1 || g.N < 1) return false;
  if (!aligned16(g.A) || !aligned16(g.B)) return false;
  const bool a_k = g.a_k == 1 && g.a_m % 8 == 0 && g.a_m >= 1;
  const bool a_mn = g.a_m == 1 && g.a_k % 8 == 0 && g.a_k >= 1;
  const bool b_k = g.b_k == 1 && g.b_n % 8 == 0 && g.b_n >= 1;
  const bool b_mn = g.b_n == 1 && g.b_k % 8 == 0 && g.b_k >= 1;
  if (!(a_k || a_mn) || !(b_k || b_mn)) return false;
  if (g.batch > 1 && (g.a_b % 8 != 0 || g.b_b % 8 != 0 || g.a_b <= 0 || g.b_b <= 0)) return false;
  if (g.atomic && (g.add || g.add2 || g.outD || !g.outF)) return false;
  if (g.add2 && !g.add) return false;
  return true;
}

// A launch whose 128 x 256 tiles would not give every SM one tile and that
// has no split-K output runs 128 x 128 tiles instead (twice as many CTAs).
int64_t wide_tiles(const Gemm &g) {
  return int64_t((g.M + BM - 1) / BM) * ((g.N + 255) / 256) * g.batch;
}
TcPlan narrowed(TcPlan t, int64_t tiles, bool any_atomic) {
  if (t.BN == 256 && !t.bstat && !any_atomic && tiles < num_sms()) t.BN = 128;
  return t;
}

// Large streaming launches run on CTA pairs (256 x 256 tiles, each CTA loading
// half of B): every problem at least 512 rows tall and enough pair tiles for
// every pair of SMs.
TcPlan paired(TcPlan t, const Gemm *gs, int n) {
  if (t.BN != 256 || t.bstat || g_pairs_mode == 0) return t;
  int64_t pair_tiles = 0;
  for (int i = 0; i < n; ++i) {
    if (gs[i].M < (g_pairs_mode == 2 ? 256 : 512)) return t;
    pair_tiles += int64_t((gs[i].M + 2 * BM - 1) / (2 * BM)) * ((gs[i].N + 255) / 256) * gs[i].batch;
  }
  if (g_pairs_mode == 2 || pair_tiles >= num_sms() / 2) t.cg = 2;
  return t;
}

poet_status gemm_tc(const Gemm &g, cudaStream_t st) {
  return run_group<1>(&g, 1, paired(narrowed(plan_of(g), wide_tiles(g), g.atomic), &g, 1), st);
}

// Runs many independent problems: tensor-core problems that share operand
// majors and tile width go into grouped launches of up to kGroupMax problems
// each (buckets in order of first appearance, list order kept inside a
// bucket); the others run one by one on the CUDA-core engine.
poet_status gemm_tc_many(const Gemm *gs, int count, cudaStream_t st) {
  std::vector<TcPlan> plans;
  std::vector<std::vector<Gemm>> buckets;
  for (int i = 0; i < count; ++i) {
    if (gs[i].M <= 0 || gs[i].N <= 0 || gs[i].batch <= 0) continue;
    if (!(gemm_tc_enabled() && gemm_tc_supported(gs[i]))) {
      POET_TRY(gemm_simt(gs[i], st));
      continue;
    }
    const TcPlan t = plan_of(gs[i]);
    size_t b = 0;
    while (b < plans.size() && !(plans[b] == t)) ++b;
    if (b == plans.size()) { plans.push_back(t); buckets.emplace_back(); }
    buckets[b].push_back(gs[i]);
  }
  for (size_t b = 0; b < plans.size(); ++b) {
    const std::vector<Gemm> &v = buckets[b];
    for (size_t i = 0; i < v.size(); i += kGroupMax) {
      const int n = int(v.size() - i < size_t(kGroupMax) ? v.size() - i : size_t(kGroupMax));
      int64_t tiles = 0;
      bool any_atomic = false;
      for (int j = 0; j < n; ++j) {
        tiles += wide_tiles(v[i + j]);
        any_atomic |= v[i + j].atomic;
      }
      // Only single-problem launches have a B-stationary kernel.  A grouped
      // launch of such problems (at most 256 columns, K <= 256) streams on
      // single CTAs with 256-wide tiles: their time goes to the epilogue (four
      // k-blocks of MMA per tile), which CTA pairs do not shorten, and pairs
      // measured 5-8 % slower on them.
      TcPlan t = plans[b];
      if (!(t.bstat && n > 1)) t = paired(narrowed(t, tiles, any_atomic), v.data() + i, n);
      else t.bstat = false;
      if (n == 1) POET_TRY(run_group<1>(v.data() + i, 1, t, st));
      else POET_TRY(run_group<kGroupMax>(v.data() + i, n, t, st));
    }
  }
  return POET_OK;
}

poet_status selftest_bounded_wait(uint32_t timeout_us, cudaStream_t st) {
  POET_REQUIRE(timeout_us >= 1 && timeout_us <= 1000000, "poet_selftest_bounded_wait: timeout %u us outside [1, 1e6]",
               timeout_us);
  unsigned *ew = device_errword();
  POET_REQUIRE(ew != nullptr, "poet_selftest_bounded_wait: no device status word");
  bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(ew, uint64_t(timeout_us) * 1000ull);
  count_launch();
  return launch_status("bounded_wait_selftest");
}

}  // namespace poet
