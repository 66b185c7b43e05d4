// Paged MLA decode on CTA pairs (tcgen05 cta_group::2) for latent heads with 128 or more
// query rows: the compute-bound decode shapes.
//
// A 1-SM tcgen05 MMA with 64 rows runs at half the tensor rate, and 128 rows of output
// (128 x 512 fp32) fill a whole SM's tensor memory.  A CTA pair shares each MMA instead:
// CTA c of the pair (cluster rank c) holds query rows 64c..64c+63 of a 128-row block, and a
// cta_group::2 MMA with M = 128 puts each CTA's 64 rows on all 128 lanes of its own tensor
// memory (columns 0..N/2-1 of the result on lanes 0-63, N/2..N-1 on lanes 64-127).  With
// N = 256 that runs at the full per-SM rate (measured: 68 cycles, as an M = 128 1-SM MMA
// with N = 256).  The B operand is split between the two CTAs (its first N/2 rows come from
// CTA 0's shared memory, the rest from CTA 1's, at the same offset).
//
// Per group of two pages (128 keys; "OpenSourceWeek Day 1 - FlashMLA", section II.1: fixed
// 64-token blocks):
//     S = Q K^T      M = 128 rows, N = 128 keys, K = 576: CTA 0 supplies the first page's
//                    keys, CTA 1 the second's (each loads its "own" page whole).  Row r's
//                    scores for the first page sit on lane r, for the second on lane 64 + r
//                    (absorbed-query score over the whole latent row, dpshk.com notes 2.1)
//     softmax        online, the running maximum refreshed only when it grows by more than
//                    8 in log2 units (same notes, 2.2); the two threads of a row exchange
//                    their maxima through shared memory; P -> bf16 in shared memory
//     O += P V       M = 128 rows, N = 256 value columns, K = 16 keys, twice (V = the first
//                    512 latent columns, read in place as an MN-major operand).  CTA 0
//                    supplies value columns 0-255, CTA 1 256-511, of BOTH pages: after the
//                    score, each CTA loads the partner page's half of the values into the
//                    ring slots whose columns it no longer needs, at the offsets where its
//                    partner keeps the same keys.  Row r's output: value columns 0-255 on
//                    lane r, 256-511 on lane 64 + r.
//
// Shared memory (per CTA, 8 KB blocks of 64 rows x 128 bytes, 128-byte swizzle):
//   ring: 2 stages x 10 slots: slots 0-8 = the own page's column blocks 0-8; after the score
//         CTA 0 reloads slots 4-7 with the partner page's column blocks 0-3 and CTA 1 slots
//         0-3 with the partner page's blocks 4-7; slot 8 (rope, free after the score) and
//         slot 9 hold the two pages' P tiles
//   query: column blocks 1-8 of the CTA's 64 query rows (TMA)
// Tensor memory (per CTA, 512 columns): O (value halves at 0 and 128), S (double-buffered
// at 256 and 320), query column block 0 at 384 (the TS operand, each row on lanes r and
// 64 + r).
//
// Warp roles (both CTAs):
//   warp 0      producer: own pages into the ring, the partner page's value half after
//               each score, L2 prefetch two groups ahead; both CTAs' copies complete on CTA
//               0's barriers (.cta_group::2 loads)
//   warp 1      TMEM owner; in CTA 0 the MMA issuer (one thread)
//   warps 2-5   softmax, O rescale and epilogue: thread (lane l of sub-partition q) owns row
//               l mod 64 and the l / 64 half (keys of the second page; value columns 256-511)
//   warps 6-9   query loaders: column block 0 into tensor memory, blocks 1-8 by TMA
// Cross-CTA signals: the MMA issuer's commits are multicast to both CTAs; CTA 1's copies and
// threads arrive on CTA 0's barriers through their cluster addresses.  Every wait is bounded.
#include "common.cuh"
#include "launch.h"

namespace pagedmla {

struct Pair128 {
  static constexpr int kThreads = 320;
  static constexpr int BM = 64;                 // query rows per CTA
  static constexpr int kSlots = 10;             // 8 KB blocks per ring stage
  static constexpr int kStageBytes = kSlots * kPageBlockBytes;
  static constexpr int kOffRing = 0;
  static constexpr int kOffQs = kOffRing + 2 * kStageBytes;      // query column blocks 1-8
  static constexpr int kOffX = kOffQs + 8 * kPageBlockBytes;      // row-max exchange [2][2][64] floats
  enum {
    FULL = 0, VFULL = FULL + 2, EMPTY = VFULL + 2, SFULL = EMPTY + 2, SFREE = SFULL + 2, PFULL = SFREE + 2,
    OFULL = PFULL + 2, OFREE = OFULL + 1, QFULL = OFREE + 1, QFREE = QFULL + 1, QTMA = QFREE + 1,
    FINAL = QTMA + 1, NBARS = FINAL + 1
  };
  static constexpr int kOffBar = kOffX + 2 * 2 * 64 * 4 + 2 * 64 * 4;  // + row-sum exchange [2][64]
  static constexpr int kOffTmem = kOffBar + NBARS * 8;
  static constexpr int kOffAbort = kOffTmem + 8;
  static constexpr int kSmemBytes = kOffAbort + 8 + 1024;   // + slack for 1 KB alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 0;         // value halves v at 128 v
  static constexpr uint32_t kTmemS = 256;       // score buffers b at 256 + 64 b
  static constexpr uint32_t kTmemQ = 384;       // query column block 0: 32 packed columns
  static constexpr uint32_t kOwnBytes = kColBlocks * kPageBlockBytes;   // a whole page
  static constexpr uint32_t kHalfVBytes = 4 * kPageBlockBytes;          // half of its values
  static_assert(kOffQs % 1024 == 0 && kOffX % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// ------------------------------------------------------------------------------------
// Cluster helpers (CTA pair).
// ------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Cluster address of the same shared-memory offset in CTA 0 of the pair.
__device__ __forceinline__ uint32_t in_cta0(uint32_t local) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(local));
  return r;
}

// Arrive on an mbarrier given by its cluster address (the default release semantics).  An
// explicit cluster-scope release measured about 0.6 us per arrive here, twice per page group
// on the softmax warps' path; the data these arrivals publish is read by the tensor cores
// (P tiles behind fence.proxy.async) or is tensor memory the arriving warp has finished with.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_test_cluster(uint32_t bar, uint32_t parity) { return mbar_test_wait(bar, parity); }

// TMA 3-D load into this CTA's shared memory whose completion (bytes) is counted on an
// mbarrier of CTA 0, given by its cluster address (.cta_group::2 form).
__device__ __forceinline__ void tma_load_3d_to_cta0(uint32_t dst, const CUtensorMap *map, uint32_t bar_cluster, int c0,
                                                    int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void umma2_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void umma2_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Arrive once on the barrier at this offset in both CTAs when all tcgen05 work issued so
// far by this thread is done.
__device__ __forceinline__ void umma2_commit_both(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint4 &a, const uint4 &b) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ bool warp_all_ok(bool v) { return __all_sync(0xffffffffu, v); }

// Shapes the pair kernel takes: whole 128-row blocks, and query rows of a CTA that form a
// rectangle of (position, head) for the query TMA box.
bool pair_supported(int R, int g) { return R >= 128 && R % 128 == 0 && g > 0 && (g % 64 == 0 || 64 % g == 0); }

struct PairPiece {
  int seq, L, t0, t1, ntiles, ngroups;  // groups = page pairs (the last may hold one page)
};

// One sequence piece of a part, trimmed to the keys the pair's 128 rows can see.
__device__ __forceinline__ PairPiece pair_piece(const DecodeParams &p, const PartCursor &pc, int seq, int prow0) {
  PairPiece w;
  w.seq = seq;
  w.L = p.seqlens[seq];
  w.t0 = seq == pc.bi ? pc.bt : 0;
  w.t1 = seq == pc.ei ? pc.et : w.L;
  if (p.causal) {
    const int last_row = min(p.R - 1, prow0 + 2 * Pair128::BM - 1);
    w.t1 = min(w.t1, w.L - (p.s_q - 1 - last_row / p.g));
  }
  w.ntiles = w.t1 > w.t0 ? (w.t1 - w.t0 + kPage - 1) / kPage : 0;
  w.ngroups = (w.ntiles + 1) / 2;
  return w;
}

// Walks the groups of a part in order, with a window of 32 block-table entries (one per
// lane) of the current piece.  All lanes of the warp call it together.
struct GroupWalker {
  int seq, j, ntiles, ngroups, t0;
  int win_base, win_val;
  bool done;
};

__device__ __forceinline__ void walker_seek(const DecodeParams &p, const PartCursor &pc, int prow0, GroupWalker &w,
                                            int seq) {
  for (; part_has(pc, seq); ++seq) {
    const PairPiece pp = pair_piece(p, pc, seq, prow0);
    if (pp.ngroups > 0) {
      w.seq = seq;
      w.j = 0;
      w.ntiles = pp.ntiles;
      w.ngroups = pp.ngroups;
      w.t0 = pp.t0;
      w.win_base = -64;
      w.done = false;
      return;
    }
  }
  w.done = true;
}

// Physical page of logical page `pg` (relative to the piece's first page).
__device__ __forceinline__ int walker_page(const DecodeParams &p, GroupWalker &w, int pg, int lane) {
  if (pg < w.win_base || pg >= w.win_base + 32) {
    w.win_base = pg & ~31;
    const int idx = w.win_base + lane;
    w.win_val = idx < w.ntiles ? p.block_table[(int64_t)w.seq * p.bt_stride + w.t0 / kPage + idx] : 0;
  }
  return __shfl_sync(0xffffffffu, w.win_val, pg - w.win_base);
}

__device__ __forceinline__ void walker_next(const DecodeParams &p, const PartCursor &pc, int prow0, GroupWalker &w) {
  if (++w.j == w.ngroups) walker_seek(p, pc, prow0, w, w.seq + 1);
}

// The pair is the cluster's x dimension (grid x = the CTAs of the 128-row blocks, y = parts,
// z = latent heads): a pair along y was refused at launch ("cluster misconfiguration").
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Pair128::kThreads, 1)
    decode_pair_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap q_map,
                       const DecodeParams p, int q_box_heads) {
  using T = Pair128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int rank = int(cluster_rank());
  const int part = blockIdx.y, pair = blockIdx.x / 2, kvh = blockIdx.z;
  const int prow0 = pair * 2 * T::BM;        // first row of the pair's 128-row block
  const int crow0 = prow0 + rank * T::BM;    // first row of this CTA
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + T::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  // barriers the other CTA arrives on live in CTA 0
  auto bar_cta0 = [&](int i) { return in_cta0(bar(i)); };
  volatile int *abort = reinterpret_cast<volatile int *>(smem + T::kOffAbort);
  const uint32_t sRing = sbase + T::kOffRing, sQs = sbase + T::kOffQs;
  auto slot = [&](int st, int k) { return sRing + uint32_t(st * T::kStageBytes + k * kPageBlockBytes); };
  float *xmax = reinterpret_cast<float *>(smem + T::kOffX);             // [2 parity][2 half][64 rows]
  float *xsum = xmax + 2 * 2 * 64;                                       // [2 half][64 rows]
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(T::FULL + i), 1);
      mbar_init(bar(T::VFULL + i), 1);
      mbar_init(bar(T::EMPTY + i), 1);
      mbar_init(bar(T::SFULL + i), 1);
      mbar_init(bar(T::SFREE + i), 8);
      mbar_init(bar(T::PFULL + i), 8);
    }
    mbar_init(bar(T::OFULL), 1);
    mbar_init(bar(T::OFREE), 8);
    mbar_init(bar(T::QFULL), 8);
    mbar_init(bar(T::QFREE), 1);
    mbar_init(bar(T::QTMA), 1);
    mbar_init(bar(T::FINAL), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc_pair(sbase + T::kOffTmem, T::kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + T::kOffTmem);
  grid_dependency_wait();  // the plan comes from the scheduler kernel just before
  const PartCursor pc = load_part(p.tile_md, part);
  const unsigned long long lim_ns = p.watchdog_ns;

  if (warp == 0) {
    // ------------------------- producer (both CTAs) -------------------------
    if (lane == 0) {
      prefetch_tensormap(&kv_map);
      prefetch_tensormap(&q_map);
    }
    // pages are read by both CTAs of the pair (one from HBM, the other's value half later
    // from L2), so they keep the normal L2 policy
    const uint64_t policy = l2_evict_normal_policy();
    const bool prefetch = p.h_kv == 1;
    GroupWalker wa, wb, wf;   // own pages, partner value halves, L2 prefetch two groups ahead
    walker_seek(p, pc, prow0, wa, pc.bi);
    wb = wa;
    wf = wa;
    int ga = 0, gb = 0, gf = 0;
    if (prefetch)
      for (; gf < 2 && !wf.done; ++gf) walker_next(p, pc, prow0, wf);
    int last_a[2] = {-1, -1}, last_b[2] = {-1, -1};
    bool ok = true;
    unsigned long long idle_since = 0;
    uint32_t spins = 0;
    while (ok && (!wa.done || gb < ga)) {
      bool progressed = false;
      // the partner page's value half for group gb, once its score is done
      if (gb < ga) {
        int ready = 0;
        if (lane == 0) ready = mbar_test_wait(bar(T::SFULL + (gb & 1)), (gb >> 1) & 1);
        if (__shfl_sync(0xffffffffu, ready, 0)) {
          const int pA = 2 * wb.j, pB = min(2 * wb.j + 1, wb.ntiles - 1);
          const int phys = walker_page(p, wb, rank == 0 ? pB : pA, lane);
          if (lane == 0) {
            const int st = gb & 1;
            if (leader) mbar_arrive_expect_tx(bar(T::VFULL + st), 2 * T::kHalfVBytes);
            // CTA 0 takes the partner's value blocks 0-3 into slots 4-7, CTA 1 blocks 4-7 into slots 0-3
            for (int c = 0; c < 4; ++c)
              tma_load_3d_to_cta0(slot(st, rank == 0 ? 4 + c : c), &kv_map, bar_cta0(T::VFULL + st),
                                  (rank == 0 ? c : 4 + c) * 64, kvh, phys * kPage, policy);
            last_b[st] = gb;
          }
          walker_next(p, pc, prow0, wb);
          ++gb;
          progressed = true;
        }
      }
      // the own page of group ga, once PV of group ga - 2 has freed the stage
      if (!progressed && !wa.done) {
        int ready = 1;
        if (lane == 0 && ga >= 2) ready = mbar_test_wait(bar(T::EMPTY + (ga & 1)), ((ga - 2) >> 1) & 1);
        if (__shfl_sync(0xffffffffu, ready, 0)) {
          const int pA = 2 * wa.j, pB = min(2 * wa.j + 1, wa.ntiles - 1);
          const int phys = walker_page(p, wa, rank == 0 ? pA : pB, lane);
          int pf = -1;
          if (prefetch && !wf.done) {
            const int fA = 2 * wf.j, fB = min(2 * wf.j + 1, wf.ntiles - 1);
            pf = walker_page(p, wf, rank == 0 ? fA : fB, lane);
          }
          if (lane == 0) {
            const int st = ga & 1;
            if (leader) mbar_arrive_expect_tx(bar(T::FULL + st), 2 * T::kOwnBytes);
            const uint32_t fb = bar_cta0(T::FULL + st);
#pragma unroll
            for (int c = 0; c < kColBlocks; ++c) tma_load_3d_to_cta0(slot(st, c), &kv_map, fb, c * 64, kvh, phys * kPage, policy);
            if (pf >= 0) prefetch_l2_bulk(p.kv_base + (int64_t)pf * kPage * p.kv_token_bytes, kPageBytes);
            last_a[st] = ga;
          }
          if (prefetch && !wf.done) walker_next(p, pc, prow0, wf);
          walker_next(p, pc, prow0, wa);
          ++ga;
          progressed = true;
        }
      }
      if (progressed) {
        idle_since = 0;
      } else {
        // nothing ready: sleep briefly so the polling warp leaves its issue slots to the
        // softmax warp on the same sub-partition
        __nanosleep(32);
      }
      if (!progressed && (++spins & 15u) == 0) {
        int stop = 0;
        if (lane == 0) {
          const unsigned long long now = global_ns();
          if (*abort) {
            stop = 1;
          } else if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > lim_ns) {
            *abort = 1;
            report_timeout(p.status);
            stop = 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, stop, 0) == 0;
      }
    }
    // every copy issued must land before the CTAs exit: CTA 0's barriers count both CTAs'
    // bytes, and CTA 1 leaves only after CTA 0 (final cluster barrier), so CTA 0 waits for all
    if (lane == 0 && leader) {
      int never = 0;
      for (int st = 0; st < 2; ++st) {
        if (last_a[st] >= 0) mbar_wait(bar(T::FULL + st), (last_a[st] >> 1) & 1, &never, p.status, lim_ns);
        if (last_b[st] >= 0) mbar_wait(bar(T::VFULL + st), (last_b[st] >> 1) & 1, &never, p.status, lim_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ------------------------- MMA issuer (CTA 0, one thread) -------------------------
      // QK of group g needs its pages in both CTAs (FULL), the query tile (QFULL) and its
      // score buffer read (SFREE); PV of group g needs both CTAs' P tiles (PFULL) and partner
      // value halves (VFULL), and at a piece's first group the previous epilogue (OFREE).
      // QK runs at most two groups ahead of PV; PV goes first when both are ready.
      const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
      GroupWalker wq, wv;
      walker_seek(p, pc, prow0, wq, pc.bi);
      wv = wq;
      int qg = 0, vg = 0, qpiece = 0, vpiece = 0;
      bool have_q = false, ok = true;
      unsigned long long idle_since = 0;
      uint32_t spins = 0;
      while (ok && !wv.done) {
        bool progressed = false;
        if (vg < qg) {
          const int b = vg & 1;
          const bool first = wv.j == 0;
          if (mbar_test_cluster(bar(T::PFULL + b), (vg >> 1) & 1) &&
              mbar_test_cluster(bar(T::VFULL + b), (vg >> 1) & 1) &&
              (!first || vpiece == 0 || mbar_test_cluster(bar(T::OFREE), (vpiece - 1) & 1))) {
            tc_fence_after();
            // a lone last page: the second page's keys are masked (P = 0), skip their MMAs
            const int halves = (2 * wv.j + 1 < wv.ntiles) ? 2 : 1;
            // descriptors step by (byte offset >> 4) in their address field
            const uint64_t pa = smem_desc_sw128(slot(b, 8), 16, 1024);
            const uint64_t vb = smem_desc_sw128(slot(b, 0), kPageBlockBytes, 1024);
            for (int h = 0; h < halves; ++h)
#pragma unroll
              for (int ks = 0; ks < kPage / 16; ++ks)
#pragma unroll
                for (int v = 0; v < 2; ++v)
                  umma2_ss(tmem + T::kTmemO + 128 * v, pa + uint64_t((h * kPageBlockBytes + ks * 32) >> 4),
                           vb + uint64_t(((4 * h + 2 * v) * kPageBlockBytes + ks * 2048) >> 4), idesc_pv,
                           (!first || h > 0 || ks > 0) ? 1u : 0u);
            umma2_commit_both(bar(T::EMPTY + b));
            if (wv.j + 1 == wv.ngroups) {
              umma2_commit_both(bar(T::OFULL));
              ++vpiece;
            }
            walker_next(p, pc, prow0, wv);
            ++vg;
            progressed = true;
          }
        }
        if (!progressed && !wq.done && qg < vg + 2) {
          const int b = qg & 1;
          if (!have_q) have_q = mbar_test_cluster(bar(T::QFULL), qpiece & 1);
          if (have_q && mbar_test_cluster(bar(T::FULL + b), (qg >> 1) & 1) &&
              (qg < 2 || mbar_test_cluster(bar(T::SFREE + b), ((qg - 2) >> 1) & 1))) {
            tc_fence_after();
            const uint32_t d = tmem + T::kTmemS + 64 * b;
            // query column block 0 from tensor memory, blocks 1-8 from shared memory
            const uint64_t kb = smem_desc_sw128(slot(b, 0), 16, 1024);
            const uint64_t qa = smem_desc_sw128(sQs, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) umma2_ts(d, tmem + T::kTmemQ + 8 * kk, kb + uint64_t(kk * 2), idesc_qk, kk > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 4; kk < kD / 16; ++kk) {
              const int cb = kk >> 2;
              umma2_ss(d, qa + uint64_t(((cb - 1) * kPageBlockBytes + (kk & 3) * 32) >> 4),
                       kb + uint64_t((cb * kPageBlockBytes + (kk & 3) * 32) >> 4), idesc_qk, 1u);
            }
            umma2_commit_both(bar(T::SFULL + b));
            if (wq.j + 1 == wq.ngroups) {
              umma2_commit_both(bar(T::QFREE));  // the query tile may be replaced
              have_q = false;
              ++qpiece;
            }
            walker_next(p, pc, prow0, wq);
            ++qg;
            progressed = true;
          }
        }
        if (progressed) {
          idle_since = 0;
        } else if (__nanosleep(32), (++spins & 15u) == 0) {
          const unsigned long long now = global_ns();
          if (*abort) {
            ok = false;
          } else if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > lim_ns) {
            *abort = 1;
            report_timeout(p.status);
            ok = false;
          }
        }
      }
      umma2_commit_both(bar(T::FINAL));
    }
    __syncwarp();
    // all tensor-core work (issued by CTA 0, writing both CTAs' tensor memory) is complete
    // before either CTA releases its tensor memory
    if (lane == 0) {
      int never = 0;
      mbar_wait(bar(T::FINAL), 0, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------- softmax / O rescale / epilogue -------------------------
    const int q = warp & 3;                 // TMEM sub-partition of this warp
    const int lrow = (32 * q + lane) & 63;  // row within the CTA's 64
    const int hf = q >> 1;                  // 0: first page's keys, values 0-255; 1: second page, 256-511
    const int row = crow0 + lrow;
    const bool active = row < p.R;
    const int s_row = row / p.g, h_row = kvh * p.g + row % p.g;
    const uint32_t lanes = tmem + (uint32_t(32 * q) << 16);
    const int xbar = 1 + (q & 1);           // named barrier of the two warps sharing rows
    const uint32_t sfree = bar_cta0(T::SFREE), pfull = bar_cta0(T::PFULL), ofree = bar_cta0(T::OFREE);
    int g = 0, qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      const PairPiece w = pair_piece(p, pc, seq, prow0);
      const int ns0 = split_base(p.num_splits, seq);
      const int nsplit = split_base(p.num_splits, seq + 1) - ns0;
      const int ord = seq == pc.bi ? pc.bord : 0;
      const int64_t acc_row = ((int64_t)(ns0 + ord) * p.h_kv + kvh) * p.R + row;
      if (w.ngroups == 0) {
        // no visible key in this piece: zero output (or partial) and lse = -inf
        if (active) {
          if (nsplit == 1) {
            uint4 *o = reinterpret_cast<uint4 *>(p.out + (((int64_t)seq * p.s_q + s_row) * p.h_q + h_row) * kDV + hf * 256);
            for (int i = 0; i < 32; ++i) o[i] = make_uint4(0u, 0u, 0u, 0u);
            if (hf == 0) p.lse[((int64_t)seq * p.h_q + h_row) * p.s_q + s_row] = -INFINITY;
          } else {
            float4 *o = reinterpret_cast<float4 *>(p.o_accum + acc_row * kDV + hf * 256);
            for (int i = 0; i < 64; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (hf == 0) p.lse_accum[acc_row] = -INFINITY;
          }
        }
        continue;
      }
      // rows past R and rows without a visible key get P = 0 (every key masked)
      const int lim = active ? min(w.t1, p.causal ? w.L - (p.s_q - 1 - s_row) : w.L) : -1;
      float m_used = -INFINITY, l = 0.f;  // l: this thread's half of the row sum
      for (int j = 0; j < w.ngroups; ++j, ++g) {
        const int b = g & 1;
        ok = warp_all_ok(ok && mbar_wait(bar(T::SFULL + b), (g >> 1) & 1, abort, p.status, lim_ns));
        tc_fence_after();
        float sv[64];
        if (ok) {
          float t[32];
          tmem_ld32(lanes + T::kTmemS + 64 * b, t);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[i] = t[i];
          tmem_ld32(lanes + T::kTmemS + 64 * b + 32, t);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[32 + i] = t[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(sfree + 8u * b);
        const int key0 = w.t0 + 128 * j + 64 * hf;
        // keys at or past this row's limit get -inf (only partial groups need the test)
        if (key0 + 64 > lim) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (key0 + i >= lim) sv[i] = -INFINITY;
        }
        // maximum of the raw scores (scale > 0), four independent chains
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 64; ++i) m4[i & 3] = fmaxf(m4[i & 3], sv[i]);
        float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.scale_log2;
        // the row's other half lives on the partner warp: exchange maxima
        xmax[(b * 2 + hf) * 64 + lrow] = mx;
        named_bar_sync(xbar, 64);
        mx = fmaxf(mx, xmax[(b * 2 + (hf ^ 1)) * 64 + lrow]);
        const float m_new = fmaxf(m_used, mx);
        const bool need = m_new > m_used + 8.f;
        float alpha = 1.f;
        if (need) {
          alpha = fast_exp2(m_used - m_new);
          m_used = m_new;
        }
        const float nbase = m_used == -INFINITY ? 0.f : -m_used;
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          sv[i] = fast_exp2(fmaf(sv[i], p.scale_log2, nbase));
          s4[i & 3] += sv[i];
        }
        l = l * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
        const bool rescale = __any_sync(0xffffffffu, need && j > 0);
        // O may be rescaled once the previous group's PV has completed (its commit arrives
        // on EMPTY of that group's stage; that barrier is at most one phase behind)
        if (rescale)
          ok = warp_all_ok(ok && mbar_wait(bar(T::EMPTY + ((g - 1) & 1)), ((g - 1) >> 1) & 1, abort, p.status, lim_ns));
        if (ok && rescale) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < 256; c0 += 32) {
            float v[32];
            tmem_ld32(lanes + T::kTmemO + c0, v);
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] *= alpha;
            tmem_st32(lanes + T::kTmemO + c0, v);
          }
          tmem_st_wait();
        }
        if (ok) {
          // P of this half into its tile (slot 8: first page's keys, slot 9: second page's)
          const uint32_t dst = slot(b, 8 + hf);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + sw128(lrow, c)),
                         "r"(pack_bf16x2(sv[8 * c], sv[8 * c + 1])), "r"(pack_bf16x2(sv[8 * c + 2], sv[8 * c + 3])),
                         "r"(pack_bf16x2(sv[8 * c + 4], sv[8 * c + 5])), "r"(pack_bf16x2(sv[8 * c + 6], sv[8 * c + 7]))
                         : "memory");
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(pfull + 8u * b);
      }

      // ---- epilogue: O / l -> output (or fp32 split partial), natural-log LSE ----
      xsum[hf * 64 + lrow] = l;
      named_bar_sync(xbar, 64);
      const float l_row = l + xsum[(hf ^ 1) * 64 + lrow];
      ok = warp_all_ok(ok && mbar_wait(bar(T::OFULL), qs & 1, abort, p.status, lim_ns));
      tc_fence_after();
      if (ok) {
        const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
        for (int c0 = 0; c0 < 256; c0 += 32) {
          float v[32];
          tmem_ld32(lanes + T::kTmemO + c0, v);
          if (!active) continue;
          if (nsplit == 1) {
            uint4 *o = reinterpret_cast<uint4 *>(p.out + (((int64_t)seq * p.s_q + s_row) * p.h_q + h_row) * kDV +
                                                 hf * 256 + c0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              o[k] = make_uint4(pack_bf16x2(v[8 * k] * inv, v[8 * k + 1] * inv),
                                pack_bf16x2(v[8 * k + 2] * inv, v[8 * k + 3] * inv),
                                pack_bf16x2(v[8 * k + 4] * inv, v[8 * k + 5] * inv),
                                pack_bf16x2(v[8 * k + 6] * inv, v[8 * k + 7] * inv));
          } else {
            float4 *o = reinterpret_cast<float4 *>(p.o_accum + acc_row * kDV + hf * 256 + c0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              o[k] = make_float4(v[4 * k] * inv, v[4 * k + 1] * inv, v[4 * k + 2] * inv, v[4 * k + 3] * inv);
          }
        }
        if (active && hf == 0) {
          const float lse_v = l_row > 0.f ? (m_used + fast_log2(l_row)) * 0.69314718055994531f : -INFINITY;
          if (nsplit == 1)
            p.lse[((int64_t)seq * p.h_q + h_row) * p.s_q + s_row] = lse_v;
          else
            p.lse_accum[acc_row] = lse_v;
        }
      }
      tc_fence_before();
      // the row-sum slots are rewritten by the next piece only after both warps have read them
      named_bar_sync(xbar, 64);
      if (lane == 0) mbar_arrive_cluster(ofree);
      ++qs;
    }
  } else {
    // ------------------------- query loaders -------------------------
    // Column block 0 of the CTA's 64 rows goes to tensor memory (row r on lanes r and
    // 64 + r, the TS operand of the score's first four K steps); blocks 1-8 come by TMA.
    const int q = warp & 3;
    const int lrow = (32 * q + lane) & 63;
    const int row = crow0 + lrow;
    const bool active = row < p.R;
    const uint32_t lanes = tmem + (uint32_t(32 * q) << 16);
    const uint32_t qfull = bar_cta0(T::QFULL);
    int qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      if (pair_piece(p, pc, seq, prow0).ngroups == 0) continue;
      const uint4 *src = reinterpret_cast<const uint4 *>(
          p.q + (int64_t)seq * p.q_sb + (int64_t)(row / p.g) * p.q_ss + (int64_t)(kvh * p.g + row % p.g) * p.q_sh);
      uint4 qv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) qv[i] = active ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
      if (qs > 0) ok = warp_all_ok(ok && mbar_wait(bar(T::QFREE), (qs - 1) & 1, abort, p.status, lim_ns));
      tc_fence_after();
      if (ok && warp == 6 && lane == 0) {
        // rows crow0.. as a (heads x positions) box: 64 heads of one position, or all g heads
        // of 64 / g positions
        const int s0 = crow0 / p.g, h0 = kvh * p.g + (q_box_heads == 64 ? crow0 % p.g : 0);
        mbar_arrive_expect_tx(bar(T::QTMA), 8 * kPageBlockBytes);
        for (int c = 1; c < kColBlocks; ++c)
          tma_load_4d(sQs + (c - 1) * kPageBlockBytes, &q_map, bar(T::QTMA), c * 64, h0, s0, seq);
      }
      if (ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_st8(lanes + T::kTmemQ + 8 * i, qv[2 * i], qv[2 * i + 1]);
        tmem_st_wait();
      }
      ok = warp_all_ok(ok && mbar_wait(bar(T::QTMA), qs & 1, abort, p.status, lim_ns));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(qfull);
      ++qs;
    }
  }
  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, T::kTmemCols);
  cluster_sync();
}

cudaError_t launch_decode_pair(const CUtensorMap &kv_map, const CUtensorMap &q_map, const DecodeParams &p,
                               int q_box_heads, cudaStream_t stream) {
  using T = Pair128;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(decode_pair_kernel), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  // grid x = two CTAs per 128-row block, paired by the kernel's compiled cluster shape
  return launch_early(decode_pair_kernel, dim3(p.R / T::BM, p.num_parts, p.h_kv), dim3(T::kThreads), T::kSmemBytes,
                      stream, kv_map, q_map, p, q_box_heads);
}

}  // namespace pagedmla
