// Paged MLA decode on 5th-generation tensor cores (tcgen05, TMEM accumulators) for more
// than 16 query rows per latent head: the mixed and compute-bound decode shapes.
//
// One CTA per (split-KV part, block of 64 query rows, latent head).  The 64-row tile is
// what fits: the fp32 output accumulator of 64 rows x 512 value columns takes half of
// TMEM when it is held as two M = 64 accumulators interleaved in the lane halves of each
// 32-lane sub-partition (value columns 0-255 in lanes 0-15, 256-511 in lanes 16-31, both
// in TMEM columns 0-255), which leaves room for the score tiles; 128 rows would need all of
// TMEM for the output alone.  Per 64-token page (one tile, "OpenSourceWeek Day 1 - FlashMLA",
// section II.1: fixed 64-token blocks):
//     S = Q K^T          M = 64 rows, N = 64 keys, K = 576 (absorbed-query score over the
//                        whole latent row, dpshk.com notes 2.1); S double-buffered in TMEM
//     online softmax     running maximum refreshed only when it grows by more than 8 in
//                        log2 units (same notes 2.2); P -> bf16 tile in shared memory
//     O += P V           M = 64, N = 256 (two halves of the 512 value columns), K = 64
//                        keys, V = the page's first 512 columns read in place as an
//                        MN-major operand
// Warp roles:
//   warp 0      TMA producer: the 64-row query tile (once per sequence piece) and the pages
//               gathered through block_table into a two-page ring
//   warp 1      TMEM owner and MMA issuer (one thread); QK of page n+1 is issued before PV
//               of page n, so the softmax of one page overlaps tensor-core work on the next
//   warps 2-5   softmax, O rescale and epilogue: lanes 0-15 of the warp on sub-partition q
//               own rows 16q..16q+15 of the score tile; for the output both lane halves work,
//               each on one half of the value columns of the same row
// Every mbarrier wait is bounded (pagedmla watchdog); a warp whose wait gives up keeps
// walking the same barrier sequence without work.
#include "common.cuh"
#include "launch.h"

namespace pagedmla {

struct Wide64 {
  static constexpr int kThreads = 192;
  static constexpr int BM = 64;                             // query rows per CTA
  static constexpr int NS = 2;                              // page ring depth
  static constexpr int kQBlock = BM * 128;                  // 64 rows x 64 columns: 8 KB
  static constexpr int kQBytes = kColBlocks * kQBlock;      // 73,728 B
  static constexpr int kPBytes = BM * 128;                  // 64 rows x 64 keys bf16
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kOffQ + kQBytes;          // 1 KB aligned
  static constexpr int kOffP = kOffRing + NS * kPageBytes;
  enum {
    FULL = 0, EMPTY = FULL + NS, QFULL = EMPTY + NS, QFREE = QFULL + 1, SFULL = QFREE + 1,
    SFREE = SFULL + 2, PFULL = SFREE + 2, PFREE = PFULL + 1, OFULL = PFREE + 1, OFREE = OFULL + 1,
    FINAL = OFREE + 1, NBARS = FINAL + 1
  };
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr int kOffTmem = kOffBar + NBARS * 8;
  static constexpr int kOffAbort = kOffTmem + 8;
  static constexpr int kSmemBytes = kOffAbort + 8 + 1024;   // + slack for 1 KB alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemS = 256;                   // S buffers: columns 256 and 320
  static constexpr uint32_t kHalf1 = 16u << 16;             // lane offset of the second atom
  static_assert(kOffRing % 1024 == 0 && kOffP % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Shapes the 64-row tensor-core kernel takes: more than 16 rows per latent head, and a
// query tile of 64 rows that one 4-D TMA box covers (g a multiple or a divisor of 64).
bool wide_supported(int R, int g) { return R > 16 && (g % 64 == 0 || 64 % g == 0); }

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

__global__ void __launch_bounds__(Wide64::kThreads, 1)
    decode_wide_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap q_map,
                       const DecodeParams p) {
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
  const uint32_t sQ = sbase + T::kOffQ, sRing = sbase + T::kOffRing, sP = sbase + T::kOffP;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(bar(T::FULL + s), 1);
      mbar_init(bar(T::EMPTY + s), 1);
    }
    mbar_init(bar(T::QFULL), 1);
    mbar_init(bar(T::QFREE), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(T::SFULL + i), 1);
      mbar_init(bar(T::SFREE + i), 4);
    }
    mbar_init(bar(T::PFULL), 4);
    mbar_init(bar(T::PFREE), 1);
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
    // ------------------------- producer: query tiles and pages -------------------------
    if (lane == 0) {
      prefetch_tensormap(&kv_map);
      prefetch_tensormap(&q_map);
    }
    // the query tile of this block: rows row0.. in the order s * g + h
    const int s0 = row0 / p.g, h0 = kvh * p.g + row0 % p.g;
    int it = 0, qs = 0, last_q = -1;
    int last_page[T::NS];
#pragma unroll
    for (int s = 0; s < T::NS; ++s) last_page[s] = -1;
    bool ok = true;
    for (int seq = pc.bi; ok && part_has(pc, seq); ++seq) {
      const WidePiece w = wide_piece(p, pc, seq, row0);
      if (w.ntiles == 0) continue;
      int good = 1;
      if (lane == 0) {
        if (!mbar_wait(bar(T::QFREE), (qs & 1) ^ 1, abort, p.status, lim_ns)) {
          good = 0;
        } else {
          mbar_arrive_expect_tx(bar(T::QFULL), uint32_t(T::kQBytes));
#pragma unroll
          for (int c = 0; c < kColBlocks; ++c)
            tma_load_4d(sQ + c * T::kQBlock, &q_map, bar(T::QFULL), c * 64, h0, s0, seq);
          last_q = qs;
        }
      }
      ok = __shfl_sync(0xffffffffu, good, 0) != 0;
      ++qs;
      const int32_t *bt_row = p.block_table + (int64_t)seq * p.bt_stride + w.t0 / kPage;
      for (int base = 0; ok && base < w.ntiles; base += 32) {
        const int mine = base + lane < w.ntiles ? bt_row[base + lane] : 0;
        const int cnt = min(32, w.ntiles - base);
        for (int i = 0; ok && i < cnt; ++i, ++it) {
          const int phys = __shfl_sync(0xffffffffu, mine, i);
          const int s = it % T::NS;
          int g2 = 1;
          if (lane == 0) {
            if (!mbar_wait(bar(T::EMPTY + s), ((it / T::NS) & 1) ^ 1, abort, p.status, lim_ns)) {
              g2 = 0;
            } else {
              mbar_arrive_expect_tx(bar(T::FULL + s), kPageBytes);
              const uint32_t dst = sRing + s * kPageBytes;
#pragma unroll
              for (int c = 0; c < kColBlocks; ++c)
                tma_load_3d(dst + c * kPageBlockBytes, &kv_map, bar(T::FULL + s), c * 64, kvh, phys * kPage);
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
      if (last_q >= 0) mbar_wait(bar(T::QFULL), last_q & 1, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------- MMA issuer (one thread) -------------------------
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(64, 64, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(64, 256, false, true);
      int it = 0, qs = 0;
      bool ok = true;
      // O += P V for global page j; `first` = first page of a sequence piece (overwrites O,
      // after the previous piece's epilogue has read it)
      auto issue_pv = [&](int j, bool first) -> bool {
        if (!mbar_wait(bar(T::PFULL), j & 1, abort, p.status, lim_ns)) return false;
        if (first && qs > 0 && !mbar_wait(bar(T::OFREE), (qs - 1) & 1, abort, p.status, lim_ns)) return false;
        tc_fence_after();
        const uint32_t page = sRing + (j % T::NS) * kPageBytes;
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int ks = 0; ks < kPage / 16; ++ks) {
            // V: value columns 256 half.. (4 column blocks, 8 KB apart), keys 16 ks.. (two
            // 8-row groups, 1 KB apart); P: keys 16 ks.. of the 64-row tile
            const uint64_t b = smem_desc_sw128(page + half * 4 * kPageBlockBytes + ks * 2048, kPageBlockBytes, 1024);
            const uint64_t a = smem_desc_sw128(sP + ks * 32, 16, 1024);
            umma_bf16(tmem + (half ? T::kHalf1 : 0u), a, b, idesc_pv, (!first || ks > 0) ? 1u : 0u);
          }
        umma_commit(bar(T::PFREE));
        umma_commit(bar(T::EMPTY + j % T::NS));
        return true;
      };
      for (int seq = pc.bi; ok && part_has(pc, seq); ++seq) {
        const WidePiece w = wide_piece(p, pc, seq, row0);
        if (w.ntiles == 0) continue;
        if (!mbar_wait(bar(T::QFULL), qs & 1, abort, p.status, lim_ns)) {
          ok = false;
          break;
        }
        for (int n = 0; ok && n < w.ntiles; ++n) {
          const int cur = it + n, s = cur % T::NS, sb = cur & 1;
          if (!mbar_wait(bar(T::FULL + s), (cur / T::NS) & 1, abort, p.status, lim_ns) ||
              (cur >= 2 && !mbar_wait(bar(T::SFREE + sb), ((cur >> 1) - 1) & 1, abort, p.status, lim_ns))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t page = sRing + s * kPageBytes;
#pragma unroll 4
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kPageBlockBytes + (kk & 3) * 32;
            const uint64_t a = smem_desc_sw128(sQ + (kk >> 2) * T::kQBlock + (kk & 3) * 32, 16, 1024);
            const uint64_t b = smem_desc_sw128(page + off, 16, 1024);
            umma_bf16(tmem + T::kTmemS + sb * 64, a, b, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(T::SFULL + sb));
          if (n == w.ntiles - 1) umma_commit(bar(T::QFREE));
          if (n > 0 && !issue_pv(cur - 1, n == 1)) ok = false;
        }
        if (ok && !issue_pv(it + w.ntiles - 1, w.ntiles == 1)) ok = false;
        if (ok) umma_commit(bar(T::OFULL));
        it += w.ntiles;
        ++qs;
      }
      // all issued tensor-core work completes before TMEM is released
      umma_commit(bar(T::FINAL));
      int never = 0;
      mbar_wait(bar(T::FINAL), 0, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else {
    // ------------------------- softmax / O rescale / epilogue -------------------------
    const int q = warp & 3;                   // TMEM sub-partition of this warp
    const int hf = lane >> 4;                 // 0: score row and value columns 0-255; 1: columns 256-511
    const int rl = 16 * q + (lane & 15);      // row within the 64-row block
    const int row = row0 + rl;
    const bool active = row < p.R;
    const int s_row = row / p.g, h_row = kvh * p.g + row % p.g;
    const uint32_t lanes = tmem + (uint32_t(32 * q) << 16);
    int it = 0, qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      const WidePiece w = wide_piece(p, pc, seq, row0);
      const int ns0 = p.num_splits[seq];
      const int nsplit = p.num_splits[seq + 1] - ns0;
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
      float m_used = -INFINITY, l = 0.f;

      for (int n = 0; n < w.ntiles; ++n) {
        const int cur = it + n, sb = cur & 1;
        ok = warp_all(ok && mbar_wait(bar(T::SFULL + sb), (cur >> 1) & 1, abort, p.status, lim_ns));
        tc_fence_after();
        float sa[32], sc[32];
        if (ok) {
          tmem_ld32(lanes + T::kTmemS + sb * 64, sa);
          tmem_ld32(lanes + T::kTmemS + sb * 64 + 32, sc);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::SFREE + sb));

        bool need = false;
        float alpha = 1.f;
        if (ok && hf == 0) {
          const int key0 = w.t0 + n * kPage;
          float mx = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float va = key0 + i < lim ? sa[i] * p.scale_log2 : -INFINITY;
            const float vc = key0 + 32 + i < lim ? sc[i] * p.scale_log2 : -INFINITY;
            sa[i] = va;
            sc[i] = vc;
            mx = fmaxf(mx, fmaxf(va, vc));
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
          for (int i = 0; i < 32; ++i) {
            sa[i] = fast_exp2(sa[i] - base);
            sc[i] = fast_exp2(sc[i] - base);
            sum += sa[i] + sc[i];
          }
          l = l * alpha + sum;
        }
        // both lane halves hold the row's output; they share its rescale factor
        const float alpha_o = __shfl_sync(0xffffffffu, alpha, lane & 15);
        const bool rescale = __any_sync(0xffffffffu, need && n > 0);
        // P and O may be touched once the previous page's PV has completed
        if (cur > 0) ok = warp_all(ok && mbar_wait(bar(T::PFREE), (cur - 1) & 1, abort, p.status, lim_ns));
        if (ok && rescale) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < 256; c0 += 16) {
            float v[16];
            tmem_ld16(lanes + c0, v);
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] *= alpha_o;
            tmem_st16(lanes + c0, v);
          }
          tmem_st_wait();
        }
        if (ok && hf == 0) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float *src = c < 4 ? sa + 8 * c : sc + 8 * (c - 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sP + sw128(rl, c)),
                         "r"(pack_bf16x2(src[0], src[1])), "r"(pack_bf16x2(src[2], src[3])),
                         "r"(pack_bf16x2(src[4], src[5])), "r"(pack_bf16x2(src[6], src[7]))
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::PFULL));
      }

      // ---- epilogue: O / l -> output (or fp32 split partial), natural-log LSE ----
      const float l_row = __shfl_sync(0xffffffffu, l, lane & 15);
      const float m_row = __shfl_sync(0xffffffffu, m_used, lane & 15);
      ok = warp_all(ok && mbar_wait(bar(T::OFULL), qs & 1, abort, p.status, lim_ns));
      tc_fence_after();
      if (ok) {
        const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
        for (int c0 = 0; c0 < 256; c0 += 32) {
          float v[32];
          tmem_ld32(lanes + c0, v);
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
          const float lse_v = l_row > 0.f ? (m_row + fast_log2(l_row)) * 0.69314718055994531f : -INFINITY;
          if (nsplit == 1)
            p.lse[((int64_t)seq * p.h_q + h_row) * p.s_q + s_row] = lse_v;
          else
            p.lse_accum[acc_row] = lse_v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::OFREE));
      it += w.ntiles;
      ++qs;
    }
  }
  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, T::kTmemCols);
}

cudaError_t launch_decode_wide(const CUtensorMap &kv_map, const CUtensorMap &q_map, const DecodeParams &p,
                               cudaStream_t stream) {
  using T = Wide64;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(decode_wide_kernel), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_parts, (p.R + T::BM - 1) / T::BM, p.h_kv);
  return launch_early(decode_wide_kernel, grid, dim3(T::kThreads), T::kSmemBytes, stream, kv_map, q_map, p);
}

}  // namespace pagedmla
