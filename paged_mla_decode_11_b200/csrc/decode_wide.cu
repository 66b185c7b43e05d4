// Paged MLA decode on 5th-generation tensor cores (tcgen05, TMEM accumulators) for more
// than 16 query rows per latent head: the mixed and compute-bound decode shapes.
//
// One CTA per (split-KV part, block of 64 query rows, latent head).  The 64-row tile is
// what fits: 64 rows x 512 value columns of fp32 output take one lane half of TMEM.  An
// M = 64 accumulator occupies lanes 0-15 of each 32-lane sub-partition (row 16q + i on lane
// 32q + i) or, placed at lane 16, lanes 16-31; 128 rows of output would need all of TMEM.
// TMEM map (512 columns):
//     lanes 0-15 of each sub-partition    score buffers A (columns 0-127, a page pair) and
//                                         B (columns 128-191, one page); the 64-row query
//                                         tile as the MMA's A operand (columns 224-511:
//                                         576 bf16 = 288 packed columns)
//     lanes 16-31                         O: value columns 0-255 in TMEM columns 0-255,
//                                         256-511 in columns 256-511
// Shared memory holds a three-page ring laid out column block by column block across the
// slots: block c (64 columns) of slot s at c * 24 KB + s * 8 KB.  Slots 0-1 and 1-2 are
// then one 128-key operand with a uniform row stride, and an M = 64 MMA costs the same for
// N = 64 and N = 128, so the score of a page pair is one MMA per 16-column step at half the
// cost per key.  Each page's P tile is written into its own rope block (columns 512-575),
// which no MMA reads once the page's score is done.
// Per page ("OpenSourceWeek Day 1 - FlashMLA", section II.1: fixed 64-token blocks):
//     S = Q K^T          M = 64 rows, N = 128 keys (a page pair in slots 0-1 or 1-2 of one
//                        sequence piece) or 64 keys, K = 576, A from TMEM (absorbed-query
//                        score over the whole latent row, dpshk.com notes 2.1)
//     online softmax     running maximum refreshed only when it grows by more than 8 in
//                        log2 units (same notes 2.2); P -> bf16 tile in shared memory
//     O += P V           M = 64, N = 256 (two halves of the 512 value columns), K = 64
//                        keys, V = the page's first 512 columns read in place as an
//                        MN-major operand
// Warp roles:
//   warp 0      TMA producer: pages gathered through block_table into the ring (and, when
//               two or more row blocks share the pages, an L2 prefetch three pages ahead)
//   warp 1      TMEM owner and MMA issuer (one thread): scores run up to two groups ahead
//               of PV and each step issues whichever group is ready, so the softmax of one
//               group overlaps tensor-core work on the next
//   warps 2-5   softmax, O rescale and epilogue.  The warp on sub-partition q owns rows
//               16q..16q+15; lane i and lane i + 16 share row 16q + i: the two pages of a
//               pair (keys 0-31 / 32-63 of a single page), value columns 0-255 / 256-511
//   warps 6-9   query loaders: the next sequence piece's query rows are read into registers
//               while the current piece runs and written to TMEM once its last QK is done
// Every mbarrier wait is bounded (pagedmla watchdog); a warp whose wait gives up keeps
// walking the same barrier sequence without work.
#include "common.cuh"
#include "launch.h"

namespace pagedmla {

struct Wide64 {
  static constexpr int kThreads = 320;
  static constexpr int BM = 64;                             // query rows per CTA
  static constexpr int NS = 3;                              // page ring depth
  static constexpr int kPrefetchAhead = 3;                  // L2 prefetch distance in pages
  static constexpr int kBoxStride = NS * kPageBlockBytes;   // one column block of every slot
  static constexpr int kOffRing = 0;
  static constexpr int kOffRope = kOffRing + (kColBlocks - 1) * kBoxStride;  // P tiles
  enum {
    FULL = 0, EMPTY = FULL + NS, QFULL = EMPTY + NS, QFREE = QFULL + 1, SFULL = QFREE + 1,
    SFREE = SFULL + 2, PFULL = SFREE + 2, PVDONE = PFULL + 2, OFULL = PVDONE + 2, OFREE = OFULL + 1,
    FINAL = OFREE + 1, NBARS = FINAL + 1
  };
  static constexpr int kOffBar = kOffRing + NS * kPageBytes;
  static constexpr int kOffTmem = kOffBar + NBARS * 8;
  static constexpr int kOffAbort = kOffTmem + 8;
  static constexpr int kSmemBytes = kOffAbort + 8 + 1024;   // + slack for 1 KB alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemSA = 0;                    // score of a page pair: 128 columns
  static constexpr uint32_t kTmemSB = 128;                  // score of a single page: 64 columns
  static constexpr uint32_t kTmemQ = kTmemCols - kD / 2;    // query tile: columns 224-511
  static constexpr uint32_t kHalf1 = 16u << 16;             // lane offset of the O accumulators
  static_assert(kOffRope % 1024 == 0 && kPageBlockBytes % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kTmemSB + 64 <= kTmemQ, "tensor memory map");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Pages in the score group that starts at page n of a piece with ntiles pages, `it` being
// the CTA-wide page counter (slot it % 3): a pair when the page sits in slot 0 or 1 and
// the piece has a next page (the two slots are adjacent in every column block), else one.
__device__ __forceinline__ int wide_group(int it, int n, int ntiles) {
  return (it % Wide64::NS != Wide64::NS - 1 && n + 1 < ntiles) ? 2 : 1;
}

// Shapes the 64-row tensor-core kernel takes: more than 16 rows per latent head.
bool wide_supported(int R, int g) { return R > 16 && g > 0; }

struct WidePiece {
  int seq, L, t0, t1, ntiles;  // ntiles = 64-token pages in [t0, t1); t0 is page aligned
};

// One sequence piece of a part, trimmed to the keys the CTA's rows can see: under the
// causal mask the rows of this 64-row block see at most L - (s_q - 1 - s_last) keys.
__device__ __forceinline__ WidePiece wide_piece(const DecodeParams &p, const PartCursor &pc, int seq, int row0) {
  WidePiece w;
  w.seq = seq;
  w.L = p.seqlens[seq];
  w.t0 = seq == pc.bi ? pc.bt : 0;
  w.t1 = seq == pc.ei ? pc.et : w.L;
  if (p.causal) {
    const int last_row = min(p.R - 1, row0 + Wide64::BM - 1);
    w.t1 = min(w.t1, w.L - (p.s_q - 1 - last_row / p.g));
  }
  w.ntiles = w.t1 > w.t0 ? (w.t1 - w.t0 + kPage - 1) / kPage : 0;
  return w;
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// 16-lane TMEM accesses (.16x32bx2): lane i < 16 of the warp reaches TMEM lane base + i at
// column c + j, lane i + 16 the same TMEM lane at column c + OFF + j.  Both lane halves of a
// warp work on one 16-row half of its sub-partition, which is how an M = 64 accumulator
// (16 rows per sub-partition) is read without touching the other 16 lanes.
template <int OFF>
__device__ __forceinline__ void tmem_ld_half32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32], %33;\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr), "n"(OFF)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

template <int OFF>
__device__ __forceinline__ void tmem_st_half32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %1, "
      "{%2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, "
      "%18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33};" ::"r"(taddr),
      "n"(OFF), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
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

template <int OFF>
__device__ __forceinline__ void tmem_st_half16(uint32_t taddr, const uint4 (&v)[4]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %1, "
      "{%2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17};" ::"r"(taddr),
      "n"(OFF), "r"(v[0].x), "r"(v[0].y), "r"(v[0].z), "r"(v[0].w), "r"(v[1].x), "r"(v[1].y), "r"(v[1].z),
      "r"(v[1].w), "r"(v[2].x), "r"(v[2].y), "r"(v[2].z), "r"(v[2].w), "r"(v[3].x), "r"(v[3].y), "r"(v[3].z),
      "r"(v[3].w)
      : "memory");
}


__global__ void __launch_bounds__(Wide64::kThreads, 1)
    decode_wide_kernel(const __grid_constant__ CUtensorMap kv_map, const DecodeParams p) {
  using T = Wide64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int part = blockIdx.x, mb = blockIdx.y, kvh = blockIdx.z;
  const int row0 = mb * T::BM;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + T::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  volatile int *abort = reinterpret_cast<volatile int *>(smem + T::kOffAbort);
  const uint32_t sRing = sbase + T::kOffRing, sRope = sbase + T::kOffRope;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(bar(T::FULL + s), 1);
      mbar_init(bar(T::EMPTY + s), 1);
    }
    mbar_init(bar(T::QFULL), 4);
    mbar_init(bar(T::QFREE), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(T::SFULL + i), 1);
      mbar_init(bar(T::SFREE + i), 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(T::PFULL + i), 4);
      mbar_init(bar(T::PVDONE + i), 1);
    }
    mbar_init(bar(T::OFULL), 1);
    mbar_init(bar(T::OFREE), 4);
    mbar_init(bar(T::FINAL), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(sbase + T::kOffTmem, T::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + T::kOffTmem);
  grid_dependency_wait();  // the plan comes from the scheduler kernel just before
  const PartCursor pc = load_part(p.tile_md, part);
  const unsigned long long lim_ns = p.watchdog_ns;

  if (warp == 0) {
    // ------------------------- producer: pages -------------------------
    if (lane == 0) prefetch_tensormap(&kv_map);
    // pages are read once, unless another 64-row block of the same latent head reads them
    // too (from L2, shortly after)
    const uint64_t policy = gridDim.y == 1 ? l2_evict_first_policy() : l2_evict_normal_policy();
    // With one latent head a page's 64 token rows are one contiguous 72 KB range.  When two
    // or more 64-row blocks read the same pages, the first also asks L2 for the page
    // kPrefetchAhead pages ahead, so that the ring's copies, which can start only when a slot
    // frees, mostly hit L2.  A single row block streams from HBM, where the extra requests
    // only compete with the ring's own copies.
    const bool prefetch = p.h_kv == 1 && mb == 0 && gridDim.y > 1;
    int it = 0;
    int last_page[T::NS];
#pragma unroll
    for (int s = 0; s < T::NS; ++s) last_page[s] = -1;
    bool ok = true;
    for (int seq = pc.bi; ok && part_has(pc, seq); ++seq) {
      const WidePiece w = wide_piece(p, pc, seq, row0);
      if (w.ntiles == 0) continue;
      const int32_t *bt_row = p.block_table + (int64_t)seq * p.bt_stride + w.t0 / kPage;
      for (int base = 0; ok && base < w.ntiles; base += 32) {
        const int mine = base + lane < w.ntiles ? bt_row[base + lane] : 0;
        const int ahead = prefetch && base + lane + T::kPrefetchAhead < w.ntiles ? bt_row[base + lane + T::kPrefetchAhead] : -1;
        const int cnt = min(32, w.ntiles - base);
        for (int i = 0; ok && i < cnt; ++i, ++it) {
          const int phys = __shfl_sync(0xffffffffu, mine, i);
          const int pf = __shfl_sync(0xffffffffu, ahead, i);
          const int s = it % T::NS;
          int g2 = 1;
          if (lane == 0) {
            if (!mbar_wait(bar(T::EMPTY + s), ((it / T::NS) & 1) ^ 1, abort, p.status, lim_ns)) {
              g2 = 0;
            } else {
              mbar_arrive_expect_tx(bar(T::FULL + s), kPageBytes);
              const uint32_t dst = sRing + s * kPageBlockBytes;
#pragma unroll
              for (int c = 0; c < kColBlocks; ++c)
                tma_load_3d_hint(dst + c * T::kBoxStride, &kv_map, bar(T::FULL + s), c * 64, kvh, phys * kPage,
                                 policy);
              if (pf >= 0) prefetch_l2_bulk(p.kv_base + (int64_t)pf * kPage * p.kv_token_bytes, kPageBytes);
              last_page[s] = it;
            }
          }
          ok = __shfl_sync(0xffffffffu, g2, 0) != 0;
        }
      }
    }
    // every copy issued must land before the CTA exits
    if (lane == 0) {
      int never = 0;
      for (int s = 0; s < T::NS; ++s)
        if (last_page[s] >= 0)
          mbar_wait(bar(T::FULL + s), (last_page[s] / T::NS) & 1, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------- MMA issuer (one thread) -------------------------
    // Two cursors walk the part's score groups (wide_group): QK of group g is issued only
    // once PV of group g - 2 has been, so QK runs at most two groups ahead of PV.  The four
    // softmax warps publish P independently, and a warp may finish group g + 1 before a
    // slower one finishes group g; P hand-offs therefore alternate between two barriers by
    // group parity, and the bound keeps any warp from reaching group g + 2 before PV(g) is
    // issued (which needs all four arrivals for g).  Each step issues whichever MMA group
    // is ready, PV first: it frees ring slots sooner.  A fixed QK(n+1)-then-PV(n) order
    // would hold PV behind a QK that waits for a page whose load could only start after
    // the PV before.
    if (lane == 0) {
      const uint32_t idesc_qk1 = idesc_bf16_f32(64, 64, false, false);
      const uint32_t idesc_qk2 = idesc_bf16_f32(64, 128, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(64, 256, false, true);
      // first piece at or after `seq` with pages; -1 at the end of the part
      auto seek = [&](int seq, int &nt) -> int {
        for (; part_has(pc, seq); ++seq) {
          const int n = wide_piece(p, pc, seq, row0).ntiles;
          if (n > 0) {
            nt = n;
            return seq;
          }
        }
        return -1;
      };
      auto landed = [&](int it) { return mbar_test_wait(bar(T::FULL + it % T::NS), (it / T::NS) & 1); };
      int qk_nt = 0, qk_n = 0, qk_it = 0, qk_g = 0, qk_piece = 0;
      int uses_a = 0, uses_b = 0;  // score groups issued into buffer A (pairs) and B (single pages)
      int qk_seq = seek(pc.bi, qk_nt);
      int pv_nt = qk_nt, pv_n = 0, pv_it = 0, pv_g = 0, pv_piece = 0;
      int pv_seq = qk_seq;
      bool have_q = false, ok = true;
      unsigned long long idle_since = 0;
      uint32_t spins = 0;
      while (ok && pv_seq >= 0) {
        bool progressed = false;
        if (pv_g < qk_g) {
          // O += P V for the pages of group pv_g; the first page of a piece overwrites O
          // once the previous piece's epilogue has read it
          const int gsz = wide_group(pv_it, pv_n, pv_nt);
          const bool first = pv_n == 0;
          if (mbar_test_wait(bar(T::PFULL + (pv_g & 1)), (pv_g >> 1) & 1) &&
              (!first || pv_piece == 0 || mbar_test_wait(bar(T::OFREE), (pv_piece - 1) & 1))) {
            tc_fence_after();
            for (int j = 0; j < gsz; ++j) {
              const int s = (pv_it + j) % T::NS;
#pragma unroll
              for (int half = 0; half < 2; ++half)
#pragma unroll
                for (int ks = 0; ks < kPage / 16; ++ks) {
                  // V: value columns 256 half.. (4 column blocks, kBoxStride apart), keys
                  // 16 ks.. (two 8-row groups, 1 KB apart); P: keys 16 ks.. of the page's tile
                  const uint64_t b = smem_desc_sw128(sRing + s * kPageBlockBytes + half * 4 * T::kBoxStride + ks * 2048,
                                                     T::kBoxStride, 1024);
                  const uint64_t a = smem_desc_sw128(sRope + s * kPageBlockBytes + ks * 32, 16, 1024);
                  umma_bf16(tmem + T::kHalf1 + half * 256, a, b, idesc_pv, (!first || j > 0 || ks > 0) ? 1u : 0u);
                }
              umma_commit(bar(T::EMPTY + s));
            }
            umma_commit(bar(T::PVDONE + (pv_g & 1)));
            pv_n += gsz;
            pv_it += gsz;
            ++pv_g;
            if (pv_n == pv_nt) {
              umma_commit(bar(T::OFULL));
              pv_seq = seek(pv_seq + 1, pv_nt);
              pv_n = 0;
              ++pv_piece;
            }
            progressed = true;
          }
        }
        if (!progressed && qk_seq >= 0 && qk_g < pv_g + 2) {
          // S = Q K^T for group qk_g: its pages have landed and its score buffer has been read
          if (!have_q) have_q = mbar_test_wait(bar(T::QFULL), qk_piece & 1);
          const int gsz = wide_group(qk_it, qk_n, qk_nt);
          const int sb = gsz == 2 ? 0 : 1;
          const int uses = sb == 0 ? uses_a : uses_b;
          if (have_q && landed(qk_it) && (gsz == 1 || landed(qk_it + 1)) &&
              (uses == 0 || mbar_test_wait(bar(T::SFREE + sb), (uses - 1) & 1))) {
            tc_fence_after();
            const uint32_t keys = sRing + (qk_it % T::NS) * kPageBlockBytes;
            const uint32_t d = tmem + (sb == 0 ? T::kTmemSA : T::kTmemSB);
            const uint32_t idesc = gsz == 2 ? idesc_qk2 : idesc_qk1;
#pragma unroll 4
            for (int kk = 0; kk < kD / 16; ++kk) {
              // keys of the group: 8-row groups 1 KB apart, running on into the next slot
              const uint64_t b = smem_desc_sw128(keys + (kk >> 2) * T::kBoxStride + (kk & 3) * 32, 16, 1024);
              umma_bf16_ts(d, tmem + T::kTmemQ + kk * 8, b, idesc, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar(T::SFULL + sb));
            if (sb == 0) ++uses_a; else ++uses_b;
            qk_n += gsz;
            qk_it += gsz;
            ++qk_g;
            if (qk_n == qk_nt) {
              umma_commit(bar(T::QFREE));  // the query tile may be replaced by the next piece's
              have_q = false;
              qk_seq = seek(qk_seq + 1, qk_nt);
              qk_n = 0;
              ++qk_piece;
            }
            progressed = true;
          }
        }
        // watchdog: give up after lim_ns without progress, or when another warp has
        if (progressed) {
          idle_since = 0;
        } else if ((++spins & 255u) == 0) {
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
      // all issued tensor-core work completes before TMEM is released
      umma_commit(bar(T::FINAL));
      int never = 0;
      mbar_wait(bar(T::FINAL), 0, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------- softmax / O rescale / epilogue -------------------------
    const int q = warp & 3;                   // TMEM sub-partition of this warp
    const int hf = lane >> 4;                 // page hf of a pair (keys 32 hf.. of a single page); value columns 256 hf..
    const int rl = 16 * q + (lane & 15);      // row within the 64-row block
    const int row = row0 + rl;
    const bool active = row < p.R;
    const int s_row = row / p.g, h_row = kvh * p.g + row % p.g;
    const uint32_t lanes = tmem + (uint32_t(32 * q) << 16);   // S rows of this warp
    const uint32_t olanes = lanes + T::kHalf1;                // O rows of this warp
    int it = 0, g = 0, qs = 0;  // pages, score groups and pieces done
    int uses_a = 0, uses_b = 0;  // score groups read from buffer A (pairs) and B (single pages)
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      const WidePiece w = wide_piece(p, pc, seq, row0);
      const int ns0 = split_base(p.num_splits, seq);
      const int nsplit = split_base(p.num_splits, seq + 1) - ns0;
      const int ord = seq == pc.bi ? pc.bord : 0;
      const int64_t acc_row = ((int64_t)(ns0 + ord) * p.h_kv + kvh) * p.R + row;
      if (w.ntiles == 0) {
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
      float m_used = -INFINITY, l = 0.f;  // l: this lane's half of the row sum

      for (int n = 0; n < w.ntiles;) {
        const int gsz = wide_group(it, n, w.ntiles);
        const int sb = gsz == 2 ? 0 : 1;
        ok = warp_all(ok && mbar_wait(bar(T::SFULL + sb), (sb == 0 ? uses_a : uses_b) & 1, abort, p.status, lim_ns));
        tc_fence_after();
        // pair: lane i < 16 takes the first page (columns 0-63), lane i + 16 the second
        // (64-127); single page: keys 0-31 / 32-63
        float sv[2][32];
        if (ok) {
          if (gsz == 2) {
            tmem_ld_half32<64>(lanes + T::kTmemSA, sv[0]);
            tmem_ld_half32<64>(lanes + T::kTmemSA + 32, sv[1]);
          } else {
            tmem_ld_half32<32>(lanes + T::kTmemSB, sv[0]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::SFREE + sb));
        if (sb == 0) ++uses_a; else ++uses_b;

        const int nh = gsz;  // 32-key halves this lane holds
        bool need = false;
        float alpha = 1.f;
        if (ok) {
          const int key0 = w.t0 + n * kPage + 32 * gsz * hf;
          float mx = -INFINITY;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (h < nh) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float v = key0 + 32 * h + i < lim ? sv[h][i] * p.scale_log2 : -INFINITY;
                sv[h][i] = v;
                mx = fmaxf(mx, v);
              }
            }
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m_used, mx);
          need = m_new > m_used + 8.f;
          if (need) {
            alpha = fast_exp2(m_used - m_new);
            m_used = m_new;
          }
          const float base = m_used == -INFINITY ? 0.f : m_used;
          float sum = 0.f;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (h < nh) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                sv[h][i] = fast_exp2(sv[h][i] - base);
                sum += sv[h][i];
              }
            }
          l = l * alpha + sum;
        }
        const bool rescale = __any_sync(0xffffffffu, need && n > 0);
        // O may be rescaled once the previous group's PV has completed.  Groups alternate
        // between two PV-done barriers, and the score of group g (so this softmax) can only
        // have been issued after PV(g - 3) completed: its pages took slots that PV freed.
        // The barrier of group g - 1 is therefore at most one phase behind, and the wait is
        // needed only when rescaling.
        if (rescale)
          ok = warp_all(ok && mbar_wait(bar(T::PVDONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, abort, p.status, lim_ns));
        if (ok && rescale) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < 256; c0 += 32) {
            float v[32];
            tmem_ld_half32<256>(olanes + c0, v);
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] *= alpha;
            tmem_st_half32<256>(olanes + c0, v);
          }
          tmem_st_wait();
        }
        if (ok) {
          // P into the rope block of the page's slot (128-byte swizzle, 64 keys per row)
          const int slot = (it + (gsz == 2 ? hf : 0)) % T::NS;
          const int chunk0 = gsz == 2 ? 0 : 4 * hf;
          const uint32_t dst = sRope + slot * kPageBlockBytes;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (h < nh) {
#pragma unroll
              for (int c = 0; c < 4; ++c)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + sw128(rl, chunk0 + 4 * h + c)),
                             "r"(pack_bf16x2(sv[h][8 * c], sv[h][8 * c + 1])),
                             "r"(pack_bf16x2(sv[h][8 * c + 2], sv[h][8 * c + 3])),
                             "r"(pack_bf16x2(sv[h][8 * c + 4], sv[h][8 * c + 5])),
                             "r"(pack_bf16x2(sv[h][8 * c + 6], sv[h][8 * c + 7]))
                             : "memory");
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::PFULL + (g & 1)));
        ++g;
        n += gsz;
        it += gsz;
      }

      // ---- epilogue: O / l -> output (or fp32 split partial), natural-log LSE ----
      const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
      ok = warp_all(ok && mbar_wait(bar(T::OFULL), qs & 1, abort, p.status, lim_ns));
      tc_fence_after();
      if (ok) {
        const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
        for (int c0 = 0; c0 < 256; c0 += 32) {
          float v[32];
          tmem_ld_half32<256>(olanes + c0, v);
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
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::OFREE));
      ++qs;
    }
  } else {
    // ------------------------- query loaders -------------------------
    // Lane i and lane i + 16 of the warp on sub-partition q carry row 16q + i: query
    // elements 0-287 and 288-575 (144 packed bf16 pairs each).
    const int q = warp & 3;
    const int hf = lane >> 4;
    const int row = row0 + 16 * q + (lane & 15);
    const bool active = row < p.R;
    const uint32_t lanes = tmem + (uint32_t(32 * q) << 16);
    uint4 qv[36];
    int qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      if (wide_piece(p, pc, seq, row0).ntiles == 0) continue;
      // read this piece's rows while the previous piece still uses the tile in TMEM
      const uint4 *src = reinterpret_cast<const uint4 *>(
          p.q + (int64_t)seq * p.q_sb + (int64_t)(row / p.g) * p.q_ss + (int64_t)(kvh * p.g + row % p.g) * p.q_sh) +
          hf * 36;
#pragma unroll
      for (int i = 0; i < 36; ++i) qv[i] = active ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
      if (qs > 0) ok = warp_all(ok && mbar_wait(bar(T::QFREE), (qs - 1) & 1, abort, p.status, lim_ns));
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int j = 0; j < 9; ++j) {
          const uint4 v4[4] = {qv[4 * j], qv[4 * j + 1], qv[4 * j + 2], qv[4 * j + 3]};
          tmem_st_half16<144>(lanes + T::kTmemQ + 16 * j, v4);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::QFULL));
      ++qs;
    }
  }
  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, T::kTmemCols);
}

cudaError_t launch_decode_wide(const CUtensorMap &kv_map, const DecodeParams &p, cudaStream_t stream) {
  using T = Wide64;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(decode_wide_kernel), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_parts, (p.R + T::BM - 1) / T::BM, p.h_kv);
  return launch_early(decode_wide_kernel, grid, dim3(T::kThreads), T::kSmemBytes, stream, kv_map, p);
}

}  // namespace pagedmla
