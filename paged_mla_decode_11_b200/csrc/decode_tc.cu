// Paged MLA decode on 5th-generation tensor cores (tcgen05, TMEM accumulators) for up to
// 16 query rows per latent head (MLA_FLAG_TCGEN05; the 16-row warp-MMA kernel is the
// default there, and decode_wide.cu takes more rows).  The template covers up to 64 rows.
//
// Per CTA: one split-KV part of the scheduler's plan, all R = s_q * h_q / h_kv query rows
// of one latent head.  Warp roles:
//   warp 0      TMA producer: the query tile (4-D tensor map, once per sequence) and the
//               latent pages gathered through block_table ("OpenSourceWeek Day 1 -
//               FlashMLA", section II.1: fixed 64-token blocks), staged as 32-token
//               half pages (32 x 576 bf16 = 36,864 B) in a 3- to 5-deep ring so that two
//               to two and a half pages per SM are in flight from HBM.
//   warp 1      MMA issuer (one thread) and TMEM owner, per 32-key chunk:
//                 S   = Q K^T              M = 128 query rows, N = 32 keys, K = 576;
//                                          up to 32 rows Q is the A operand in TMEM
//                                          (tcgen05.cp once per sequence), so the
//                                          tensor core reads only the key slab from
//                                          shared memory
//                 O^T += V^T P^T           M = 128 value columns (x 4 blocks), N = R_pad,
//                                          K = 32 keys; V = the chunk's first 512 columns
//               (absorbed-query score over the whole latent row, dpshk.com notes 2.1).
//   warps 2-5   softmax / correction / epilogue warpgroup: thread = query row for S,
//               thread = value column for O^T.  Online softmax (same notes, 2.2) with the
//               running maximum refreshed only when it grows by more than 8 in log2 units;
//               O^T and the row sum always share the maximum they were scaled with, so the
//               result is exact.
// Accumulating O transposed keeps TMEM at 64 (S, double-buffered) + 4 * R_pad (O^T)
// columns, and lets V be read straight from the TMA chunk tile as an MN-major operand.
// QK of chunk n+1 is issued before PV of chunk n, so the softmax of one chunk overlaps
// tensor-core work on the next.
// Rows R .. 127 of the S tile read whatever follows the query tile in shared memory; they
// are never used.
//
// Every mbarrier wait is bounded (pagedmla watchdog); a warp whose wait gives up keeps
// walking the same barrier sequence without work, so no warp is left at a named barrier.
#include "common.cuh"
#include "launch.h"

namespace pagedmla {

template <int RP>
struct TcNarrow {
  static constexpr int kThreads = 192;
  static constexpr int KC = 32;                          // keys per chunk (half a page)
  static constexpr int kChunkBlock = KC * 128;           // one 64-column block of a chunk
  static constexpr int kChunkBytes = kColBlocks * kChunkBlock;  // 36,864 B
  // Up to 32 rows the query tile lives in TMEM (the A operand of S = Q K^T), copied there
  // once per sequence, so each QK MMA reads only its 1 KB key slab from shared memory.
  static constexpr bool kQinTmem = RP <= 32;
  static constexpr int NS = RP == 64 ? 3 : (RP == 48 ? 4 : 5);  // chunk ring depth
  static constexpr int NQ = 1;                           // shared-memory query tile buffers
  static constexpr int NP = 2;                           // P tile buffers
  static constexpr int kQBlock = RP * 128;               // one 64-column block of the query tile
  static constexpr int kQBytes = kColBlocks * kQBlock;
  static constexpr int kPBytes = RP * 128;               // 32 keys per 128-byte row (first half)
  static constexpr int kOffQ = 0;
  static constexpr int kOffP = NQ * kQBytes;
  static constexpr int kOffRing = ((kOffP + NP * kPBytes + 1023) / 1024) * 1024;
  static constexpr int kOffRows = kOffRing + NS * kChunkBytes;  // l, m, alpha [64] each
  enum {
    FULL = 0, EMPTY = FULL + NS, QFULL = EMPTY + NS, QFREE = QFULL + NQ,
    SFULL = QFREE + NQ, SFREE = SFULL + 2, PFULL = SFREE + 2, PFREE = PFULL + NP,
    OFULL = PFREE + NP, OFREE = OFULL + 1, FINAL = OFREE + 1, NBARS = FINAL + 1
  };
  static constexpr int kOffBar = kOffRows + 3 * 64 * 4;
  static constexpr int kOffTmem = kOffBar + NBARS * 8;
  static constexpr int kOffAbort = kOffTmem + 8;
  static constexpr int kSmemBytes = kOffAbort + 8 + 1024;  // + slack for 1 KB alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 2 * KC;  // O^T blocks start after the two S buffers
  static constexpr uint32_t kTmemQ = kTmemCols - kD / 2;  // Q: 288 columns (2 bf16 each)
  static_assert(!kQinTmem || kTmemO + 4 * RP <= kTmemQ, "tensor memory budget with Q");
  static_assert(RP % 16 == 0 && RP >= 16 && RP <= 64, "rows per tile");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kTmemO + 4 * RP <= kTmemCols, "tensor memory budget");
  // the M = 128 query-operand read of the last column block of the last buffer stays inside
  static_assert((NQ - 1) * kQBytes + (kColBlocks - 1) * kQBlock + 128 * 128 <= kOffRows, "Q over-read");
};

struct Segment {
  int seq, L, t0, t1, nch;  // nch = 32-key chunks in [t0, t1); t0 is page aligned
};

// One sequence piece of a part; the narrow kernel holds all query rows, so causal
// visibility never trims whole chunks (the last row sees every key).
__device__ __forceinline__ Segment make_segment(const DecodeParams &p, const PartCursor &pc, int seq) {
  Segment s;
  s.seq = seq;
  s.L = p.seqlens[seq];
  s.t0 = seq == pc.bi ? pc.bt : 0;
  s.t1 = seq == pc.ei ? pc.et : s.L;
  s.nch = s.t1 > s.t0 ? (s.t1 - s.t0 + 31) / 32 : 0;
  return s;
}

template <int RP>
__global__ void __launch_bounds__(TcNarrow<RP>::kThreads, 1)
    decode_tc_narrow_kernel(const __grid_constant__ CUtensorMap kv_map,
                            const __grid_constant__ CUtensorMap q_map, const DecodeParams p) {
  using T = TcNarrow<RP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int part = blockIdx.x, kvh = blockIdx.z;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + T::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  volatile int *abort = reinterpret_cast<volatile int *>(smem + T::kOffAbort);
  const uint32_t sQ = sbase + T::kOffQ, sP = sbase + T::kOffP, sRing = sbase + T::kOffRing;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(bar(T::FULL + s), 1);
      mbar_init(bar(T::EMPTY + s), 1);
    }
    for (int i = 0; i < T::NQ; ++i) {
      mbar_init(bar(T::QFULL + i), 1);
      mbar_init(bar(T::QFREE + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(T::SFULL + i), 1);
      mbar_init(bar(T::SFREE + i), 4);
    }
    for (int i = 0; i < T::NP; ++i) {
      mbar_init(bar(T::PFULL + i), 4);
      mbar_init(bar(T::PFREE + i), 1);
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
    // ------------------------- producer: query tiles and key chunks -------------------------
    if (lane == 0) {
      prefetch_tensormap(&kv_map);
      prefetch_tensormap(&q_map);
    }
    int it = 0, qs = 0;
    int last_chunk[T::NS], last_q[T::NQ];
#pragma unroll
    for (int s = 0; s < T::NS; ++s) last_chunk[s] = -1;
#pragma unroll
    for (int s = 0; s < T::NQ; ++s) last_q[s] = -1;
    bool ok = true;
    for (int seq = pc.bi; ok && part_has(pc, seq); ++seq) {
      const Segment sg = make_segment(p, pc, seq);
      if (sg.nch == 0) continue;
      const int qb = qs % T::NQ;
      int good = 1;
      if (lane == 0) {
        if (!mbar_wait(bar(T::QFREE + qb), ((qs / T::NQ) & 1) ^ 1, abort, p.status, lim_ns)) {
          good = 0;
        } else {
          mbar_arrive_expect_tx(bar(T::QFULL + qb), uint32_t(kColBlocks * p.R * 128));
#pragma unroll
          for (int c = 0; c < kColBlocks; ++c)
            tma_load_4d(sQ + qb * T::kQBytes + c * T::kQBlock, &q_map, bar(T::QFULL + qb), c * 64,
                        kvh * p.g, 0, seq);
          last_q[qb] = qs;
        }
      }
      ok = __shfl_sync(0xffffffffu, good, 0) != 0;
      ++qs;
      // chunk i of the segment = half (i & 1) of logical page t0/64 + i/2
      const int32_t *bt_row = p.block_table + (int64_t)seq * p.bt_stride + sg.t0 / kPage;
      for (int base = 0; ok && base < sg.nch; base += 32) {
        const int mine = base + lane < sg.nch ? bt_row[(base + lane) >> 1] : 0;
        const int cnt = min(32, sg.nch - base);
        for (int i = 0; ok && i < cnt; ++i, ++it) {
          const int phys = __shfl_sync(0xffffffffu, mine, i);
          const int s = it % T::NS;
          int g2 = 1;
          if (lane == 0) {
            if (!mbar_wait(bar(T::EMPTY + s), ((it / T::NS) & 1) ^ 1, abort, p.status, lim_ns)) {
              g2 = 0;
            } else {
              mbar_arrive_expect_tx(bar(T::FULL + s), T::kChunkBytes);
              const uint32_t dst = sRing + s * T::kChunkBytes;
              const int row = phys * kPage + ((base + i) & 1) * T::KC;
#pragma unroll
              for (int c = 0; c < kColBlocks; ++c)
                tma_load_3d(dst + c * T::kChunkBlock, &kv_map, bar(T::FULL + s), c * 64, kvh, row);
              last_chunk[s] = it;
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
        if (last_chunk[s] >= 0)
          mbar_wait(bar(T::FULL + s), (last_chunk[s] / T::NS) & 1, &never, p.status, lim_ns);
      for (int s = 0; s < T::NQ; ++s)
        if (last_q[s] >= 0)
          mbar_wait(bar(T::QFULL + s), (last_q[s] / T::NQ) & 1, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------- MMA issuer (one thread) -------------------------
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, T::KC, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, RP, true, false);
      int it = 0, qs = 0;
      bool ok = true;
      for (int seq = pc.bi; ok && part_has(pc, seq); ++seq) {
        const Segment sg = make_segment(p, pc, seq);
        if (sg.nch == 0) continue;
        const int qb = qs % T::NQ;
        if (!mbar_wait(bar(T::QFULL + qb), (qs / T::NQ) & 1, abort, p.status, lim_ns)) {
          ok = false;
          break;
        }
        const uint32_t qtile = sQ + qb * T::kQBytes;
        if constexpr (T::kQinTmem) {
          // Q (rows on lanes, 576 columns as 288 packed pairs) into TMEM; the shared-memory
          // tile is free again once the copies complete.
          tc_fence_after();
#pragma unroll 4
          for (int kk = 0; kk < kD / 16; ++kk)
            tmem_cp_128x256b(tmem + T::kTmemQ + kk * 8,
                             smem_desc_sw128(qtile + (kk >> 2) * T::kQBlock + (kk & 3) * 32, 16, 1024));
          umma_commit(bar(T::QFREE + qb));
        }
        auto issue_qk = [&](int cur) -> bool {
          const int s = cur % T::NS, sb = cur & 1;
          if (!mbar_wait(bar(T::FULL + s), (cur / T::NS) & 1, abort, p.status, lim_ns)) return false;
          if (!mbar_wait(bar(T::SFREE + sb), ((cur >> 1) & 1) ^ 1, abort, p.status, lim_ns)) return false;
          tc_fence_after();
          const uint32_t chunk = sRing + s * T::kChunkBytes;
          const uint64_t b0 = smem_desc_sw128(chunk, 16, 1024);
#pragma unroll 4
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * T::kChunkBlock + (kk & 3) * 32;
            const uint64_t b = b0 + (off >> 4);
            if constexpr (T::kQinTmem) {
              umma_bf16_ts(tmem + sb * T::KC, tmem + T::kTmemQ + kk * 8, b, idesc_qk, kk > 0 ? 1u : 0u);
            } else {
              const uint64_t a = smem_desc_sw128(qtile + (kk >> 2) * T::kQBlock + (kk & 3) * 32, 16, 1024);
              umma_bf16(tmem + sb * T::KC, a, b, idesc_qk, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(bar(T::SFULL + sb));
          return true;
        };
        if (!issue_qk(it)) {
          ok = false;
          break;
        }
        if (!T::kQinTmem && sg.nch == 1) umma_commit(bar(T::QFREE + qb));
        for (int n = 0; n < sg.nch; ++n) {
          const int cur = it + n;
          if (n + 1 < sg.nch) {
            if (!issue_qk(cur + 1)) {
              ok = false;
              break;
            }
            if (!T::kQinTmem && n + 2 == sg.nch) umma_commit(bar(T::QFREE + qb));
          }
          const int pb = cur & 1;
          if (!mbar_wait(bar(T::PFULL + pb), (cur >> 1) & 1, abort, p.status, lim_ns)) {
            ok = false;
            break;
          }
          if (n == 0 && !mbar_wait(bar(T::OFREE), (qs & 1) ^ 1, abort, p.status, lim_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t chunk = sRing + (cur % T::NS) * T::kChunkBytes;
          const uint32_t ptile = sP + pb * T::kPBytes;
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int ks = 0; ks < T::KC / 16; ++ks) {
              // V^T block j: MN-major over the chunk's column blocks 2j, 2j+1 (4 KB apart),
              // keys 16ks.. (two 8-row groups, 1 KB apart)
              const uint64_t a = smem_desc_sw128(chunk + (2 * j) * T::kChunkBlock + ks * 2048,
                                                 T::kChunkBlock, 1024);
              const uint64_t b = smem_desc_sw128(ptile + ks * 32, 16, 1024);
              umma_bf16(tmem + T::kTmemO + j * RP, a, b, idesc_pv, (n > 0 || ks > 0) ? 1u : 0u);
            }
          umma_commit(bar(T::PFREE + pb));
          umma_commit(bar(T::EMPTY + cur % T::NS));
          if (n == sg.nch - 1) umma_commit(bar(T::OFULL));
        }
        it += sg.nch;
        ++qs;
      }
      // all issued tensor-core work completes before TMEM is released
      umma_commit(bar(T::FINAL));
      int never = 0;
      mbar_wait(bar(T::FINAL), 0, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else {
    // ------------------------- softmax / correction / epilogue -------------------------
    const int wq = warp & 3;         // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;  // query row (S) and value column within a block (O^T)
    const int tid = threadIdx.x - 64;
    const bool warp_rows = wq * 32 < p.R;
    const bool active = row < p.R;
    float *l_sm = reinterpret_cast<float *>(smem + T::kOffRows);
    float *m_sm = l_sm + 64;
    float *a_sm = l_sm + 128;
    const uint32_t lanes = tmem + (uint32_t(wq * 32) << 16);
    int it = 0, qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      const Segment sg = make_segment(p, pc, seq);
      const int ns0 = split_base(p.num_splits, seq);
      const int nsplit = split_base(p.num_splits, seq + 1) - ns0;
      const int ord = seq == pc.bi ? pc.bord : 0;
      const int64_t acc_row0 = ((int64_t)(ns0 + ord) * p.h_kv + kvh) * p.R;
      if (sg.nch == 0) {
        for (int idx = tid; idx < p.R * kDV; idx += 128) {
          const int c = idx / kDV, dv = idx % kDV;
          if (nsplit == 1) {
            const int h = kvh * p.g + c % p.g;
            p.out[(((int64_t)seq * p.s_q + c / p.g) * p.h_q + h) * kDV + dv] = __float2bfloat16(0.f);
          } else {
            p.o_accum[(acc_row0 + c) * kDV + dv] = 0.f;
          }
        }
        if (active) {
          if (nsplit == 1)
            p.lse[((int64_t)seq * p.h_q + kvh * p.g + row % p.g) * p.s_q + row / p.g] = -INFINITY;
          else
            p.lse_accum[acc_row0 + row] = -INFINITY;
        }
        continue;
      }
      int lim = -1;
      if (active) lim = min(sg.t1, p.causal ? sg.L - (p.s_q - 1 - row / p.g) : sg.L);
      float m_used = -INFINITY, l = 0.f;

      for (int n = 0; n < sg.nch; ++n) {
        const int cur = it + n;
        const int sb = cur & 1;
        ok = ok && mbar_wait(bar(T::SFULL + sb), (cur >> 1) & 1, abort, p.status, lim_ns);
        tc_fence_after();
        float s[T::KC];
        if (ok && warp_rows) tmem_ld32(lanes + sb * T::KC, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::SFREE + sb));

        bool need = false;
        float alpha = 1.f;
        if (ok && warp_rows) {
          const int key0 = sg.t0 + n * T::KC;
          float mx = -INFINITY;
#pragma unroll
          for (int i = 0; i < T::KC; ++i) {
            const float v = key0 + i < lim ? s[i] * p.scale_log2 : -INFINITY;
            s[i] = v;
            mx = fmaxf(mx, v);
          }
          const float m_new = fmaxf(m_used, mx);
          need = m_new > m_used + 8.f;
          if (need) {
            alpha = fast_exp2(m_used - m_new);
            m_used = m_new;
          }
          const float base = m_used == -INFINITY ? 0.f : m_used;
          float sum = 0.f;
#pragma unroll
          for (int i = 0; i < T::KC; ++i) {
            s[i] = fast_exp2(s[i] - base);
            sum += s[i];
          }
          l = l * alpha + sum;
        }
        const int pb = cur & 1;
        ok = ok && mbar_wait(bar(T::PFREE + pb), ((cur >> 1) & 1) ^ 1, abort, p.status, lim_ns);
        if (ok && warp_rows && row < RP) {
          const uint32_t prow = sP + pb * T::kPBytes;
#pragma unroll
          for (int c = 0; c < T::KC / 8; ++c) {
            const uint32_t w0 = pack_bf16x2(s[8 * c + 0], s[8 * c + 1]);
            const uint32_t w1 = pack_bf16x2(s[8 * c + 2], s[8 * c + 3]);
            const uint32_t w2 = pack_bf16x2(s[8 * c + 4], s[8 * c + 5]);
            const uint32_t w3 = pack_bf16x2(s[8 * c + 6], s[8 * c + 7]);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + sw128(row, c)),
                         "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                         : "memory");
          }
        }
        // Rescale O^T when some row refreshed its maximum (after the previous PV is done).
        if (named_bar_or(1, 128, need && n > 0 && active)) {
          const int prv = cur - 1;
          ok = ok && mbar_wait(bar(T::PFREE + (prv & 1)), (prv >> 1) & 1, abort, p.status, lim_ns);
          if (row < RP) a_sm[row] = active ? alpha : 1.f;
          named_bar_sync(1, 128);
          tc_fence_after();
          if (ok) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              for (int c0 = 0; c0 < RP; c0 += 16) {
                const uint32_t ta = lanes + T::kTmemO + j * RP + c0;
                float v[16];
                tmem_ld16(ta, v);
#pragma unroll
                for (int k = 0; k < 16; ++k) v[k] *= a_sm[c0 + k];
                tmem_st16(ta, v);
              }
            tmem_st_wait();
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::PFULL + pb));
      }

      // ---- epilogue: O^T / l -> output (or fp32 split partial), natural-log LSE ----
      ok = ok && mbar_wait(bar(T::OFULL), qs & 1, abort, p.status, lim_ns);
      tc_fence_after();
      if (active) {
        l_sm[row] = l;
        m_sm[row] = m_used;
      }
      named_bar_sync(1, 128);
      if (ok) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int dv = j * 128 + row;
          for (int c0 = 0; c0 < RP; c0 += 16) {
            float v[16];
            tmem_ld16(lanes + T::kTmemO + j * RP + c0, v);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int c = c0 + k;
              if (c < p.R) {
                const float lt = l_sm[c];
                const float val = lt > 0.f ? v[k] / lt : 0.f;
                if (nsplit == 1) {
                  const int h = kvh * p.g + c % p.g;
                  p.out[(((int64_t)seq * p.s_q + c / p.g) * p.h_q + h) * kDV + dv] = __float2bfloat16(val);
                } else {
                  p.o_accum[(acc_row0 + c) * kDV + dv] = val;
                }
              }
            }
          }
        }
        if (active) {
          const float lse_v = l > 0.f ? (m_used + fast_log2(l)) * 0.69314718055994531f : -INFINITY;
          if (nsplit == 1)
            p.lse[((int64_t)seq * p.h_q + kvh * p.g + row % p.g) * p.s_q + row / p.g] = lse_v;
          else
            p.lse_accum[acc_row0 + row] = lse_v;
        }
      }
      tc_fence_before();
      named_bar_sync(1, 128);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::OFREE));
      it += sg.nch;
      ++qs;
    }
  }
  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, T::kTmemCols);
}

template <int RP>
static cudaError_t launch_tc(const CUtensorMap &kv_map, const CUtensorMap &q_map, const DecodeParams &p,
                             cudaStream_t stream) {
  using T = TcNarrow<RP>;
  auto kern = decode_tc_narrow_kernel<RP>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_parts, 1, p.h_kv);
  return launch_early(kern, grid, dim3(T::kThreads), T::kSmemBytes, stream, kv_map, q_map, p);
}

cudaError_t launch_decode_tc_narrow(const CUtensorMap &kv_map, const CUtensorMap &q_map,
                                    const DecodeParams &p, cudaStream_t stream) {
  // above 16 rows per latent head the 64-row tcgen05 kernel takes over
  if (p.R > 16) return cudaErrorInvalidValue;
  return launch_tc<16>(kv_map, q_map, p, stream);
}

}  // namespace pagedmla
