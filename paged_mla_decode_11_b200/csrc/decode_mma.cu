// Paged MLA decode, warp-MMA variant (mma.sync m16n8k16 bf16, fp32 accumulate).
//
// One CTA per (split-KV part, 16- or 64-row block of query rows, latent head).  A
// producer warp streams whole 64-token latent pages (64 x 576 bf16 = 73,728 B) from the
// paged cache into a two-stage shared-memory ring with TMA (128-byte swizzle), each
// page addressed through block_table ("OpenSourceWeek Day 1 - FlashMLA", section II.1:
// fixed 64-token blocks).  Consumer warps compute per page
//     S = scale * Q K^T over all 576 columns (absorbed-query score, dpshk.com notes 2.1)
//     online softmax: running max m, running sum l, O <- O * 2^(m_old - m_new)
//     O += P V with V = the page's first 512 columns                (same notes, 2.2)
// and write either the final bf16 output and natural-log LSE or, when the scheduler
// split the sequence, an fp32 partial (O / l, lse) for the log-sum-exp combine.
//
// Warp layout: BM / 16 row groups x DVS value slices.  In a row group the DVS warps
// split the 64 keys of S (NK = 64 / DVS each) and the 512 value columns of O
// (NDV = 512 / DVS each); the row maximum and the P tile are exchanged through shared
// memory, the row sums only once per segment.
#include "common.cuh"
#include "launch.h"

namespace pagedmla {

template <int BM, int DVS>
struct MmaTile {
  static constexpr int RG = BM / 16;
  static constexpr int NCW = RG * DVS;      // consumer warps
  static constexpr int kThreads = (NCW + 1) * 32;
  static constexpr int NK = kPage / DVS;    // keys of S per warp
  static constexpr int NT = NK / 8;         // 8-key n-tiles of S per warp
  static constexpr int NDV = kDV / DVS;     // value columns per warp
  static constexpr int NO = NDV / 8;        // 8-column n-tiles of O per warp
  static constexpr int kStages = 2;
  static constexpr int kQBlock = BM * 128;  // one 64-column block of the Q tile
  static constexpr int kOffQ = kStages * kPageBytes;
  static constexpr int kOffP = kOffQ + kColBlocks * kQBlock;
  static constexpr int kOffRed = kOffP + BM * 128;
  static constexpr int kRedFloats = RG * DVS * 16;
  static constexpr int kOffBar = kOffRed + 2 * kRedFloats * 4;
  static constexpr int kOffAbort = kOffBar + 2 * kStages * 8;
  static constexpr int kSmemBytes = kOffAbort + 16 + 1024;  // + slack for 1 KB alignment
  static_assert(NT >= 1 && (NT == 1 || NT % 2 == 0), "S tiling");
  static_assert(NO % 2 == 0, "O tiling");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Last key (exclusive) any row of m-block `mb` may see: causal rows see fewer keys.
__device__ __forceinline__ int block_visible_end(const DecodeParams &p, int L, int mb, int BM) {
  if (!p.causal) return L;
  const int last_row = min(p.R - 1, mb * BM + BM - 1);
  return L - (p.s_q - 1 - last_row / p.g);
}

template <int BM, int DVS>
__global__ void __launch_bounds__(MmaTile<BM, DVS>::kThreads, 1)
    decode_mma_kernel(const __grid_constant__ CUtensorMap kv_map, const DecodeParams p) {
  using T = MmaTile<BM, DVS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int part = blockIdx.x, mb = blockIdx.y, kvh = blockIdx.z;
  const uint32_t full_bar = smem_u32(smem + T::kOffBar);
  const uint32_t empty_bar = full_bar + 8 * T::kStages;
  volatile int *abort = reinterpret_cast<volatile int *>(smem + T::kOffAbort);

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::kStages; ++s) {
      mbar_init(full_bar + 8 * s, 1);
      mbar_init(empty_bar + 8 * s, T::NCW);
    }
    *abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  grid_dependency_wait();  // the plan comes from the scheduler kernel just before
  const PartCursor pc = load_part(p.tile_md, part);

  if (warp == T::NCW) {
    // ---------------- producer warp: page gather through block_table ----------------
    if (lane == 0) prefetch_tensormap(&kv_map);
    int it = 0;
    int last_it[T::kStages];
#pragma unroll
    for (int s = 0; s < T::kStages; ++s) last_it[s] = -1;
    bool ok = true;
    for (int seq = pc.bi; ok && part_has(pc, seq); ++seq) {
      const int L = p.seqlens[seq];
      const int t0 = seq == pc.bi ? pc.bt : 0;
      const int t1 = min(seq == pc.ei ? pc.et : L, block_visible_end(p, L, mb, BM));
      const int npages = t1 > t0 ? (t1 - t0 + kPage - 1) / kPage : 0;
      const int32_t *bt_row = p.block_table + (int64_t)seq * p.bt_stride + t0 / kPage;
      for (int base = 0; ok && base < npages; base += 32) {
        const int mine = base + lane < npages ? bt_row[base + lane] : 0;
        const int cnt = min(32, npages - base);
        for (int i = 0; i < cnt; ++i) {
          const int phys = __shfl_sync(0xffffffffu, mine, i);
          const int s = it % T::kStages;
          const uint32_t ph = (it / T::kStages) & 1;
          int good = 1;
          if (lane == 0) {
            if (!mbar_wait(empty_bar + 8 * s, ph ^ 1, abort, p.status, p.watchdog_ns)) {
              good = 0;
            } else {
              mbar_arrive_expect_tx(full_bar + 8 * s, kPageBytes);
              const uint32_t dst = smem_u32(smem) + s * kPageBytes;
#pragma unroll
              for (int c = 0; c < kColBlocks; ++c)
                tma_load_3d(dst + c * kPageBlockBytes, &kv_map, full_bar + 8 * s, c * 64, kvh,
                            phys * kPage);
              last_it[s] = it;
            }
          }
          ok = __shfl_sync(0xffffffffu, good, 0) != 0;
          if (!ok) break;
          ++it;
        }
      }
    }
    // Wait (bounded) until every copy this warp issued has landed before the CTA exits.
    if (lane == 0) {
      int never = 0;
      for (int s = 0; s < T::kStages; ++s)
        if (last_it[s] >= 0)
          mbar_wait(full_bar + 8 * s, (last_it[s] / T::kStages) & 1, &never, p.status,
                    p.watchdog_ns);
    }
    __syncwarp();
  } else {
    // ---------------- consumer warps ----------------
    const int rg = warp / DVS, wd = warp % DVS;
    const int g4 = lane / 4, c4 = lane % 4;
    const uint32_t sPages = smem_u32(smem);
    const uint32_t sQ = smem_u32(smem + T::kOffQ);
    const uint32_t sP = smem_u32(smem + T::kOffP);
    float *red_max = reinterpret_cast<float *>(smem + T::kOffRed);
    float *red_sum = red_max + T::kRedFloats;
    const int rows[2] = {mb * BM + rg * 16 + g4, mb * BM + rg * 16 + g4 + 8};
    const int group_bar = 1 + rg, all_bar = 1 + T::RG;
    const int tid = threadIdx.x;
    int it = 0;
    bool ok = true;

    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      const int L = p.seqlens[seq];
      const int t0 = seq == pc.bi ? pc.bt : 0;
      const int t1 = min(seq == pc.ei ? pc.et : L, block_visible_end(p, L, mb, BM));
      const int npages = t1 > t0 ? (t1 - t0 + kPage - 1) / kPage : 0;
      int lim[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = rows[r];
        lim[r] = row < p.R ? min(t1, p.causal ? L - (p.s_q - 1 - row / p.g) : L) : -1;
      }

      // Q tile of this sequence: rows mb*BM.., all 576 columns, 128-byte swizzled.
      named_bar_sync(all_bar, T::NCW * 32);
      for (int idx = tid; idx < BM * 72; idx += T::NCW * 32) {
        const int row = idx / 72, ch = idx % 72;
        const int r = mb * BM + row;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < p.R) {
          const int s = r / p.g, h = kvh * p.g + r % p.g;
          v = __ldg(reinterpret_cast<const uint4 *>(p.q + (int64_t)seq * p.q_sb +
                                                    (int64_t)s * p.q_ss + (int64_t)h * p.q_sh) +
                    ch);
        }
        *reinterpret_cast<uint4 *>(smem + T::kOffQ + (ch / 8) * T::kQBlock + sw128(row, ch % 8)) = v;
      }
      named_bar_sync(all_bar, T::NCW * 32);

      float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
      float o[T::NO][4];
#pragma unroll
      for (int j = 0; j < T::NO; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

      for (int pg = 0; pg < npages; ++pg, ++it) {
        const int s = it % T::kStages;
        const uint32_t ph = (it / T::kStages) & 1;
        // After a failed wait the warp keeps walking the same named-barrier sequence
        // without touching the page, so no other warp is left waiting at a bar.sync.
        ok = ok && mbar_wait(full_bar + 8 * s, ph, abort, p.status, p.watchdog_ns);
        const uint32_t sK = sPages + s * kPageBytes;

        // ---- S = Q K^T over the warp's NK keys ----
        float sc[T::NT][4];
#pragma unroll
        for (int t = 0; t < T::NT; ++t) sc[t][0] = sc[t][1] = sc[t][2] = sc[t][3] = 0.f;
        if constexpr (T::NT == 1) {
#pragma unroll 2
          for (int kk = 0; kk < kD / 16; kk += 2) {
            uint32_t a0[4], a1[4], b[4];
            const int cb = kk / 4;
            const int qr = rg * 16 + (lane % 16);
            ldsm_x4(sQ + cb * T::kQBlock + sw128(qr, (kk % 4) * 2 + lane / 16), a0[0], a0[1], a0[2], a0[3]);
            ldsm_x4(sQ + cb * T::kQBlock + sw128(qr, ((kk + 1) % 4) * 2 + lane / 16), a1[0], a1[1], a1[2], a1[3]);
            ldsm_x4(sK + cb * kPageBlockBytes + sw128(wd * 8 + (lane % 8), (kk % 4) * 2 + lane / 8),
                    b[0], b[1], b[2], b[3]);
            mma_bf16_16816(sc[0], a0, b[0], b[1]);
            mma_bf16_16816(sc[0], a1, b[2], b[3]);
          }
        } else {
#pragma unroll 2
          for (int kk = 0; kk < kD / 16; ++kk) {
            uint32_t a[4];
            const int cb = kk / 4;
            ldsm_x4(sQ + cb * T::kQBlock + sw128(rg * 16 + (lane % 16), (kk % 4) * 2 + lane / 16),
                    a[0], a[1], a[2], a[3]);
#pragma unroll
            for (int np = 0; np < T::NT / 2; ++np) {
              uint32_t b[4];
              const int key = wd * T::NK + np * 16 + (lane % 8) + (lane / 16) * 8;
              ldsm_x4(sK + cb * kPageBlockBytes + sw128(key, (kk % 4) * 2 + (lane / 8) % 2), b[0],
                      b[1], b[2], b[3]);
              mma_bf16_16816(sc[2 * np], a, b[0], b[1]);
              mma_bf16_16816(sc[2 * np + 1], a, b[2], b[3]);
            }
          }
        }

        // ---- mask, scale to the log2 domain, row maximum across the row group ----
        const int key_base = (t0 / kPage + pg) * kPage + wd * T::NK;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int t = 0; t < T::NT; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = e / 2;
            const int key = key_base + t * 8 + c4 * 2 + (e & 1);
            const float v = key < lim[r] ? sc[t][e] * p.scale_log2 : -INFINITY;
            sc[t][e] = v;
            mx[r] = fmaxf(mx[r], v);
          }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
          mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        }
        if (c4 == 0) {
          red_max[(rg * DVS + wd) * 16 + g4] = mx[0];
          red_max[(rg * DVS + wd) * 16 + g4 + 8] = mx[1];
        }
        named_bar_sync(group_bar, DVS * 32);
        float alpha[2], base[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float mn = m[r];
#pragma unroll
          for (int w = 0; w < DVS; ++w) mn = fmaxf(mn, red_max[(rg * DVS + w) * 16 + g4 + 8 * r]);
          base[r] = mn == -INFINITY ? 0.f : mn;
          alpha[r] = fast_exp2(m[r] - base[r]);   // m = -inf -> 0
          m[r] = mn;
        }

        // ---- P = 2^(S - m) -> bf16 tile in shared memory; partial row sums ----
        float ps[2] = {0.f, 0.f};
#pragma unroll
        for (int t = 0; t < T::NT; ++t) {
          const float p0 = fast_exp2(sc[t][0] - base[0]), p1 = fast_exp2(sc[t][1] - base[0]);
          const float p2 = fast_exp2(sc[t][2] - base[1]), p3 = fast_exp2(sc[t][3] - base[1]);
          ps[0] += p0 + p1;
          ps[1] += p2 + p3;
          const int kl = wd * T::NK + t * 8 + c4 * 2;
          const uint32_t off = (kl % 8) * 2;
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + sw128(rg * 16 + g4, kl / 8) + off),
                       "r"(pack_bf16x2(p0, p1)));
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + sw128(rg * 16 + g4 + 8, kl / 8) + off),
                       "r"(pack_bf16x2(p2, p3)));
        }
        l[0] = l[0] * alpha[0] + ps[0];
        l[1] = l[1] * alpha[1] + ps[1];
        named_bar_sync(group_bar, DVS * 32);

        // ---- O = O * alpha + P V over the warp's NDV value columns ----
#pragma unroll
        for (int j = 0; j < T::NO; ++j) {
          o[j][0] *= alpha[0];
          o[j][1] *= alpha[0];
          o[j][2] *= alpha[1];
          o[j][3] *= alpha[1];
        }
#pragma unroll
        for (int ks = 0; ks < kPage / 16; ++ks) {
          uint32_t a[4];
          ldsm_x4(sP + sw128(rg * 16 + (lane % 16), ks * 2 + lane / 16), a[0], a[1], a[2], a[3]);
          const int key = ks * 16 + (lane % 8) + ((lane / 8) % 2) * 8;
#pragma unroll
          for (int jp = 0; jp < T::NO / 2; ++jp) {
            const int dv0 = wd * T::NDV + jp * 16;
            uint32_t b[4];
            ldsm_x4_t(sK + (dv0 / 64) * kPageBlockBytes + sw128(key, (dv0 % 64) / 8 + lane / 16),
                      b[0], b[1], b[2], b[3]);
            mma_bf16_16816(o[2 * jp], a, b[0], b[1]);
            mma_bf16_16816(o[2 * jp + 1], a, b[2], b[3]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar + 8 * s);
      }
      // ---- epilogue: total row sums, then final output or split partial ----
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
      }
      if (c4 == 0) {
        red_sum[(rg * DVS + wd) * 16 + g4] = l[0];
        red_sum[(rg * DVS + wd) * 16 + g4 + 8] = l[1];
      }
      named_bar_sync(group_bar, DVS * 32);
      const int ns0 = split_base(p.num_splits, seq);
      const int nsplit = split_base(p.num_splits, seq + 1) - ns0;
      const int ord = seq == pc.bi ? pc.bord : 0;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = rows[r];
        if (row >= p.R || !ok) continue;
        float lt = 0.f;
#pragma unroll
        for (int w = 0; w < DVS; ++w) lt += red_sum[(rg * DVS + w) * 16 + g4 + 8 * r];
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float lse_v = lt > 0.f ? (m[r] + fast_log2(lt)) * 0.69314718055994531f : -INFINITY;
        if (nsplit == 1) {
          const int s = row / p.g, h = kvh * p.g + row % p.g;
          __nv_bfloat16 *orow = p.out + (((int64_t)seq * p.s_q + s) * p.h_q + h) * kDV;
#pragma unroll
          for (int j = 0; j < T::NO; ++j) {
            const int dv = wd * T::NDV + j * 8 + c4 * 2;
            *reinterpret_cast<uint32_t *>(orow + dv) =
                pack_bf16x2(o[j][2 * r] * inv, o[j][2 * r + 1] * inv);
          }
          if (wd == 0 && c4 == 0) p.lse[((int64_t)seq * p.h_q + h) * p.s_q + s] = lse_v;
        } else {
          const int64_t sidx = ((int64_t)(ns0 + ord) * p.h_kv + kvh) * p.R + row;
          float *orow = p.o_accum + sidx * kDV;
#pragma unroll
          for (int j = 0; j < T::NO; ++j) {
            const int dv = wd * T::NDV + j * 8 + c4 * 2;
            *reinterpret_cast<float2 *>(orow + dv) = make_float2(o[j][2 * r] * inv, o[j][2 * r + 1] * inv);
          }
          if (wd == 0 && c4 == 0) p.lse_accum[sidx] = lse_v;
        }
      }
    }
  }
  grid_launch_dependents();
  __syncthreads();
}

// ---------------------------------------------------------------------------------------
// Up to 16 query rows: the memory-bound decode shape.  mma.sync's 16-row tile fits these
// rows exactly (a tcgen05 MMA pads them to 128 and costs at least a 128x128x16 tile).
// Keys stream as 32-token half pages through a 5-deep TMA ring (two and a half pages per
// SM in flight from HBM).  Three warp stages overlap across chunks:
//   - S warps 0-3: warp (kh, kn) keeps the A fragments of half the 576 columns of Q in
//     registers for a whole sequence and computes the partial scores of 16 keys of each
//     chunk into a double-buffered shared-memory tile;
//   - softmax warp 4: sums the two column halves, runs the online softmax (running max,
//     rescale factor, row sums) and writes the bf16 P tile, double-buffered;
//   - PV warps 5-8: O (16 rows x 128 value columns each) += P V from the same chunk.
// Each hand-off is a producer/consumer named barrier pair (full / empty), so the S warps
// run up to two chunks ahead of the softmax, which runs up to two chunks ahead of PV.
// ---------------------------------------------------------------------------------------
// Sparse variant (kSparse): the keys of a chunk are 32 listed token rows of one query token,
// gathered row by row with untiled bulk copies into a row-major chunk (rows of 576 bf16
// padded to 1,168 bytes, so that 8 consecutive rows of a ldmatrix fall in distinct banks) by
// two producer warps taking alternate chunks; a producer also records which of the chunk's 32
// entries are real keys (a validity mask).
template <bool kSparse>
struct Mma16T {
  static constexpr int KC = 32;                           // keys per chunk
  static constexpr int NS = 5;                            // ring depth
  static constexpr int kSWarps = 4, kSmWarp = 4, kPVWarp0 = 5, kPVWarps = 4, kProducer = 9;
  // sparse: two producer warps (9 and 10), chunk `it` issued by warp 9 + it % 2.  One warp's
  // row copies are issued one request at a time and top out near 2.9 TB/s over the GPU; two
  // warps reach about 5.1 TB/s (measured).  A third warp measured slower (33.6 against
  // 32.4 us on the random top-2048 workload): 162 registers, and the copies gain little.
  static constexpr int kNP = kSparse ? 2 : 1;
  static constexpr int kThreads = (kProducer + kNP) * 32;
  static constexpr int kChunkBlock = KC * 128;            // one 64-column block: 4 KB
  static constexpr int kChunkBytes = kColBlocks * kChunkBlock;  // bytes a chunk's copies deliver
  static constexpr int kRowBytes = kD * 2 + 16;           // sparse: padded row of a chunk
  // ring slot stride (1 KB multiple, so that the Q tile after the ring stays 1 KB aligned)
  static constexpr int kSlotBytes = kSparse ? (KC * kRowBytes + 1023) / 1024 * 1024 : kChunkBytes;
  static constexpr int kOffRing = 0;
  static constexpr int kOffQ = NS * kSlotBytes;           // 16 rows x 576, 9 blocks of 2 KB
  static constexpr int kOffP = kOffQ + kColBlocks * 16 * 128;   // 2 x [16 rows x 32 keys] bf16
  static constexpr int kOffS = kOffP + 2 * 16 * 128;            // 2 x [4 warps][8][32] f32 partial S
  static constexpr int kOffAlpha = kOffS + 2 * 4 * 8 * 32 * 4;  // alpha[2][16]
  static constexpr int kOffL = kOffAlpha + 2 * 16 * 4;          // l[2 segs][16]
  static constexpr int kOffM = kOffL + 2 * 16 * 4;              // m[2 segs][16]
  static constexpr int kOffBar = kOffM + 2 * 16 * 4;
  enum { FULL = 0, EMPTY = FULL + NS, QFULL = EMPTY + NS, QFREE = QFULL + 1, NBARS = QFREE + 1 };
  static constexpr int kOffAbort = kOffBar + NBARS * 8;
  static constexpr int kOffMask = kOffAbort + 16;          // sparse: vmask[NS] (per slot), smask[2]
  static constexpr int kSmemBytes = kOffMask + (NS + 2) * 4 + 1024;
  // named barriers (id, id + 1 for the two buffers): S tile full / empty, P tile full / empty
  static constexpr int kBarSFull = 1, kBarSEmpty = 3, kBarPFull = 5, kBarPEmpty = 7;
  static constexpr int kSPair = (kSWarps + 1) * 32, kPPair = (kPVWarps + 1) * 32;
  static_assert(kSmemBytes <= 232448, "shared memory budget");

  // Shared address of 16-byte column chunk col16 (0..71) of key row `row` of a ring chunk:
  // nine 128-byte-swizzled 32-row column blocks (tiled TMA), or padded rows (sparse).
  static __device__ __forceinline__ uint32_t key_addr(uint32_t chunk, int row, int col16) {
    if constexpr (kSparse) return chunk + row * kRowBytes + col16 * 16;
    else return chunk + (col16 >> 3) * kChunkBlock + sw128(row, col16 & 7);
  }
};
using Mma16 = Mma16T<false>;

__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Token range and 32-key chunk count of sequence `seq` within part `pc` (sparse: the range of
// entries of query token `seq`'s key list).
template <bool kSparse = false>
__device__ __forceinline__ int chunk_range(const DecodeParams &p, const PartCursor &pc, int seq, int &L,
                                           int &t0, int &t1) {
  L = kSparse ? p.row_ptr[seq + 1] - p.row_ptr[seq] : p.seqlens[seq];
  t0 = seq == pc.bi ? pc.bt : 0;
  t1 = seq == pc.ei ? pc.et : L;
  return t1 > t0 ? (t1 - t0 + Mma16::KC - 1) / Mma16::KC : 0;
}

template <bool kSparse>
__global__ void __launch_bounds__(Mma16T<kSparse>::kThreads, 1)
    decode_mma16_kernel(const __grid_constant__ CUtensorMap kv_map,
                        const __grid_constant__ CUtensorMap q_map, const DecodeParams p) {
  using T = Mma16T<kSparse>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int part = blockIdx.x, kvh = blockIdx.z;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + T::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  volatile int *abort = reinterpret_cast<volatile int *>(smem + T::kOffAbort);
  const uint32_t sRing = sbase + T::kOffRing, sQ = sbase + T::kOffQ, sP = sbase + T::kOffP;
  float *sbuf = reinterpret_cast<float *>(smem + T::kOffS);
  float *alpha_sm = reinterpret_cast<float *>(smem + T::kOffAlpha);
  float *l_sm = reinterpret_cast<float *>(smem + T::kOffL);
  float *m_sm = reinterpret_cast<float *>(smem + T::kOffM);
  uint32_t *vmask = reinterpret_cast<uint32_t *>(smem + T::kOffMask);  // [NS], then smask[2]
  const unsigned long long lim_ns = p.watchdog_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(bar(T::FULL + s), 1);
      mbar_init(bar(T::EMPTY + s), T::kPVWarps);
    }
    mbar_init(bar(T::QFULL), 1);
    mbar_init(bar(T::QFREE), T::kSWarps);
    *abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  grid_dependency_wait();  // the plan comes from the scheduler kernel just before
  const PartCursor pc = load_part(p.tile_md, part);
  const int g4 = lane >> 2, c4 = lane & 3;

  if (warp >= T::kProducer) {
    // ------------------------- producer: query tiles and key chunks -------------------------
    // (sparse: producer pid takes the chunks with it % kNP == pid; the first also loads Q)
    const int pid = warp - T::kProducer;
    if (lane == 0) {
      prefetch_tensormap(&kv_map);
      prefetch_tensormap(&q_map);
    }
    const uint64_t policy = l2_evict_first_policy();  // pages are read once
    int it = 0, qs = 0, last_q = -1;
    int last_chunk[T::NS];
#pragma unroll
    for (int s = 0; s < T::NS; ++s) last_chunk[s] = -1;
    bool ok = true;
    for (int seq = pc.bi; ok && part_has(pc, seq); ++seq) {
      int L, t0, t1;
      const int nch = chunk_range<kSparse>(p, pc, seq, L, t0, t1);
      if (nch == 0) continue;
      int good = 1;
      if (lane == 0 && pid == 0) {
        if (!mbar_wait(bar(T::QFREE), (qs & 1) ^ 1, abort, p.status, lim_ns)) {
          good = 0;
        } else {
          mbar_arrive_expect_tx(bar(T::QFULL), uint32_t(kColBlocks * p.R * 128));
#pragma unroll
          for (int c = 0; c < kColBlocks; ++c) {
            if constexpr (kSparse)  // one query token: position seq % s_q of sequence seq / s_q
              tma_load_4d(sQ + c * 16 * 128, &q_map, bar(T::QFULL), c * 64, kvh * p.g, seq % p.sq_fold,
                          seq / p.sq_fold);
            else
              tma_load_4d(sQ + c * 16 * 128, &q_map, bar(T::QFULL), c * 64, kvh * p.g, 0, seq);
          }
          last_q = qs;
        }
      }
      ok = __shfl_sync(0xffffffffu, good, 0) != 0;
      ++qs;
      if constexpr (kSparse) {
        // Entry t0 + 32 n + lane of the list goes to row `lane` of chunk n.  Lists are read four
        // chunks at a time (one coalesced index load and one block-table load per lane and
        // chunk), the next group's indices while the current group's copies are issued.
        const int b = seq / p.sq_fold, sq = seq % p.sq_fold;
        const int Lb = p.seqlens[b];
        const int nvis = p.causal ? Lb - (p.sq_fold - 1 - sq) : Lb;
        const int32_t *list = p.col_idx + p.row_ptr[seq];
        const int32_t *bt = p.block_table + (int64_t)b * p.bt_stride;
        auto fetch = [&](int grp, int (&idx)[4]) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int e = t0 + (grp * 4 + k) * T::KC + lane;
            idx[k] = e < t1 ? list[e] : -1;
          }
        };
        // a pruned entry copies token 0 of page 0 (finite data; its score is masked)
        auto resolve = [&](const int (&idx)[4], const uint8_t *(&src)[4], unsigned &valid) {
          valid = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const bool v = idx[k] >= 0 && idx[k] < nvis;
            const int64_t phys = v ? bt[idx[k] / kPage] : 0;
            const int64_t row = phys * kPage + (v ? idx[k] % kPage : 0);
            src[k] = p.kv_base + (row * p.h_kv + kvh) * (kD * 2);
            valid |= unsigned(v) << k;
          }
        };
        const int ngrp = (nch + 3) / 4;
        int idx[4];
        const uint8_t *src[4];
        unsigned valid;
        fetch(0, idx);
        resolve(idx, src, valid);
        for (int grp = 0; ok && grp < ngrp; ++grp) {
          if (grp + 1 < ngrp) fetch(grp + 1, idx);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int n = grp * 4 + k;
            if (!ok || n >= nch) break;
            if (it % T::kNP != pid) {  // another producer's chunk
              ++it;
              continue;
            }
            const unsigned vm = __ballot_sync(0xffffffffu, (valid >> k) & 1u);
            const int s = it % T::NS;
            int g2 = 1;
            if (lane == 0) {
              if (!mbar_wait(bar(T::EMPTY + s), ((it / T::NS) & 1) ^ 1, abort, p.status, lim_ns)) {
                g2 = 0;
              } else {
                vmask[s] = vm;
                mbar_arrive_expect_tx(bar(T::FULL + s), T::KC * kD * 2);
                last_chunk[s] = it;
              }
            }
            ok = __shfl_sync(0xffffffffu, g2, 0) != 0;
            if (ok) bulk_load_hint(sRing + s * T::kSlotBytes + lane * T::kRowBytes, src[k], kD * 2,
                                   bar(T::FULL + s), policy);
            ++it;
          }
          if (grp + 1 < ngrp) resolve(idx, src, valid);
        }
        continue;
      }
      const int32_t *bt_row = p.block_table + (int64_t)seq * p.bt_stride + t0 / kPage;
      for (int base = 0; ok && base < nch; base += 32) {
        const int mine = base + lane < nch ? bt_row[(base + lane) >> 1] : 0;
        const int cnt = min(32, nch - base);
        for (int i = 0; ok && i < cnt; ++i, ++it) {
          const int phys = __shfl_sync(0xffffffffu, mine, i);
          const int s = it % T::NS;
          int g2 = 1;
          if (lane == 0) {
            if (!mbar_wait(bar(T::EMPTY + s), ((it / T::NS) & 1) ^ 1, abort, p.status, lim_ns)) {
              g2 = 0;
            } else {
              mbar_arrive_expect_tx(bar(T::FULL + s), T::kChunkBytes);
              const uint32_t dst = sRing + s * T::kSlotBytes;
              const int row = phys * kPage + ((base + i) & 1) * T::KC;
#pragma unroll
              for (int c = 0; c < kColBlocks; ++c)
                tma_load_3d_hint(dst + c * T::kChunkBlock, &kv_map, bar(T::FULL + s), c * 64, kvh, row, policy);
              last_chunk[s] = it;
            }
          }
          ok = __shfl_sync(0xffffffffu, g2, 0) != 0;
        }
      }
    }
    // Wait (bounded) until every copy this warp issued has landed before the CTA exits: per
    // slot, the slot's final use, when this warp issued it (with two producers a slot's
    // earlier use may have been followed by the other warp's, and a parity wait can only
    // name the latest phase).
    if (lane == 0) {
      int never = 0;
      for (int s = 0; s < T::NS; ++s) {
        const int final_use = it - 1 - ((it - 1 - s) % T::NS + T::NS) % T::NS;
        if (final_use >= 0 && last_chunk[s] == final_use)
          mbar_wait(bar(T::FULL + s), (final_use / T::NS) & 1, &never, p.status, lim_ns);
      }
      if (last_q >= 0) mbar_wait(bar(T::QFULL), last_q & 1, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else if (warp < T::kSWarps) {
    // ------------------------- S warps: partial scores -------------------------
    const int kh = warp >> 1, kn = warp & 1;
    uint32_t qf[kD / 32][4];  // A fragments of this warp's 288 columns of Q
    int it = 0, qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      int L, t0, t1;
      const int nch = chunk_range<kSparse>(p, pc, seq, L, t0, t1);
      if (nch == 0) continue;
      ok = ok && mbar_wait(bar(T::QFULL), qs & 1, abort, p.status, lim_ns);
      if (ok) {
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk) {
          const int k = kh * (kD / 32) + kk;
          ldsm_x4(sQ + (k >> 2) * (16 * 128) + sw128(lane & 15, (k & 3) * 2 + (lane >> 4)), qf[kk][0],
                  qf[kk][1], qf[kk][2], qf[kk][3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::QFREE));
      for (int n = 0; n < nch; ++n, ++it) {
        const int sb = it & 1;
        ok = ok && mbar_wait(bar(T::FULL + it % T::NS), (it / T::NS) & 1, abort, p.status, lim_ns);
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if (ok) {
          // key fragments loaded one k-step ahead; four independent accumulator chains
          const uint32_t chunk = sRing + (it % T::NS) * T::kSlotBytes;
          float sd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          auto kaddr = [&](int k) {
            return T::key_addr(chunk, kn * 16 + (lane & 7) + (lane >> 4) * 8, 2 * k + ((lane >> 3) & 1));
          };
          uint32_t b[2][4];
          ldsm_x4(kaddr(kh * (kD / 32)), b[0][0], b[0][1], b[0][2], b[0][3]);
#pragma unroll
          for (int kk = 0; kk < kD / 32; ++kk) {
            if (kk + 1 < kD / 32)
              ldsm_x4(kaddr(kh * (kD / 32) + kk + 1), b[(kk + 1) & 1][0], b[(kk + 1) & 1][1],
                      b[(kk + 1) & 1][2], b[(kk + 1) & 1][3]);
            float(&a0)[4] = (kk & 1) ? sd[0] : sc[0];
            float(&a1)[4] = (kk & 1) ? sd[1] : sc[1];
            mma_bf16_16816(a0, qf[kk], b[kk & 1][0], b[kk & 1][1]);
            mma_bf16_16816(a1, qf[kk], b[kk & 1][2], b[kk & 1][3]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            sc[0][e] += sd[0][e];
            sc[1][e] += sd[1][e];
          }
        }
        if (it >= 2) named_bar_sync(T::kBarSEmpty + sb, T::kSPair);
        // the chunk's validity mask travels with the S tile (read after this warp's FULL wait)
        if (kSparse && warp == 0 && lane == 0) vmask[T::NS + sb] = ok ? vmask[it % T::NS] : 0u;
        float *dst = sbuf + (sb * 4 + warp) * 8 * 32;
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[e * 32 + lane] = sc[e >> 2][e & 3];
        named_bar_arrive(T::kBarSFull + sb, T::kSPair);
      }
      ++qs;
    }
    for (int c = max(it - 2, 0); c < it; ++c) named_bar_sync(T::kBarSEmpty + (c & 1), T::kSPair);
  } else if (warp == T::kSmWarp) {
    // ------------------------- softmax warp -------------------------
    int it = 0, qs = 0;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      int L, t0, t1;
      const int nch = chunk_range<kSparse>(p, pc, seq, L, t0, t1);
      if (nch == 0) continue;
      int lim[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = g4 + 8 * r;
        lim[r] = row < p.R ? min(t1, p.causal ? L - (p.s_q - 1 - row / p.g) : L) : -1;
      }
      float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
      for (int n = 0; n < nch; ++n, ++it) {
        const int sb = it & 1, pb = it & 1;
        named_bar_sync(T::kBarSFull + sb, T::kSPair);
        // this thread's 16 scores: key halves kn = 0, 1; per half 2 key tiles x 4 values
        float sc[2][8];
        const float *src = sbuf + sb * 4 * 8 * 32;
#pragma unroll
        for (int kn = 0; kn < 2; ++kn)
#pragma unroll
          for (int e = 0; e < 8; ++e)
            sc[kn][e] = src[(kn * 8 + e) * 32 + lane] + src[((2 + kn) * 8 + e) * 32 + lane];
        const unsigned vm = kSparse ? vmask[T::NS + sb] : 0u;
        named_bar_arrive(T::kBarSEmpty + sb, T::kSPair);
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int kn = 0; kn < 2; ++kn)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int r = (e >> 1) & 1;
            const int kc = kn * 16 + (e >> 2) * 8 + c4 * 2 + (e & 1);
            const bool vis = kSparse ? (lim[r] >= 0 && ((vm >> kc) & 1u)) : t0 + n * T::KC + kc < lim[r];
            const float v = vis ? sc[kn][e] * p.scale_log2 : -INFINITY;
            sc[kn][e] = v;
            mx[r] = fmaxf(mx[r], v);
          }
        float alpha[2], base[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
          mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
          const float mn = fmaxf(m[r], mx[r]);
          base[r] = mn == -INFINITY ? 0.f : mn;
          alpha[r] = fast_exp2(m[r] - base[r]);
          m[r] = mn;
          l[r] *= alpha[r];
        }
        if (it >= 2) named_bar_sync(T::kBarPEmpty + pb, T::kPPair);
        const uint32_t ptile = sP + pb * (16 * 128);
#pragma unroll
        for (int kn = 0; kn < 2; ++kn)
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const float p0 = fast_exp2(sc[kn][t * 4 + 0] - base[0]), p1 = fast_exp2(sc[kn][t * 4 + 1] - base[0]);
            const float p2 = fast_exp2(sc[kn][t * 4 + 2] - base[1]), p3 = fast_exp2(sc[kn][t * 4 + 3] - base[1]);
            l[0] += p0 + p1;
            l[1] += p2 + p3;
            const int kl = kn * 16 + t * 8 + c4 * 2;
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(ptile + sw128(g4, kl / 8) + (kl % 8) * 2),
                         "r"(pack_bf16x2(p0, p1)));
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(ptile + sw128(g4 + 8, kl / 8) + (kl % 8) * 2),
                         "r"(pack_bf16x2(p2, p3)));
          }
        if (c4 == 0) {
          alpha_sm[pb * 16 + g4] = alpha[0];
          alpha_sm[pb * 16 + g4 + 8] = alpha[1];
        }
        if (n == nch - 1) {
          // row sums and the row maximum for the epilogue of this sequence
          float lr[2] = {l[0], l[1]};
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            lr[r] += __shfl_xor_sync(0xffffffffu, lr[r], 1);
            lr[r] += __shfl_xor_sync(0xffffffffu, lr[r], 2);
          }
          if (c4 == 0) {
            l_sm[(qs & 1) * 16 + g4] = lr[0];
            l_sm[(qs & 1) * 16 + g4 + 8] = lr[1];
            m_sm[(qs & 1) * 16 + g4] = m[0];
            m_sm[(qs & 1) * 16 + g4 + 8] = m[1];
          }
        }
        named_bar_arrive(T::kBarPFull + pb, T::kPPair);
      }
      ++qs;
    }
    for (int c = max(it - 2, 0); c < it; ++c) named_bar_sync(T::kBarPEmpty + (c & 1), T::kPPair);
  } else {
    // ------------------------- PV warps -------------------------
    const int v = warp - T::kPVWarp0;  // value columns 128 v .. 128 v + 127
    int it = 0, qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      int L, t0, t1;
      const int nch = chunk_range<kSparse>(p, pc, seq, L, t0, t1);
      const int ns0 = split_base(p.num_splits, seq);
      const int nsplit = split_base(p.num_splits, seq + 1) - ns0;
      const int ord = seq == pc.bi ? pc.bord : 0;
      const int64_t acc_row0 = ((int64_t)(ns0 + ord) * p.h_kv + kvh) * p.R;
      if (nch == 0) {
        const int tid = threadIdx.x - T::kPVWarp0 * 32;
        for (int idx = tid; idx < p.R * kDV; idx += T::kPVWarps * 32) {
          const int c = idx / kDV, dv = idx % kDV;
          if (nsplit == 1)
            p.out[(((int64_t)seq * p.s_q + c / p.g) * p.h_q + kvh * p.g + c % p.g) * kDV + dv] =
                __float2bfloat16(0.f);
          else
            p.o_accum[(acc_row0 + c) * kDV + dv] = 0.f;
        }
        if (tid < p.R) {
          if (nsplit == 1)
            p.lse[lse_index(p, seq, tid / p.g, kvh * p.g + tid % p.g)] = -INFINITY;
          else
            p.lse_accum[acc_row0 + tid] = -INFINITY;
        }
        continue;
      }
      float o[16][4];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
      float lt[2] = {0.f, 0.f}, mr[2] = {-INFINITY, -INFINITY};
      for (int n = 0; n < nch; ++n, ++it) {
        const int s = it % T::NS, pb = it & 1;
        named_bar_sync(T::kBarPFull + pb, T::kPPair);
        const float a0 = alpha_sm[pb * 16 + g4], a1 = alpha_sm[pb * 16 + g4 + 8];
        if (n == nch - 1) {
          // this sequence's row sums and maxima, read before the P tile is released
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            lt[r] = l_sm[(qs & 1) * 16 + g4 + 8 * r];
            mr[r] = m_sm[(qs & 1) * 16 + g4 + 8 * r];
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          o[j][0] *= a0;
          o[j][1] *= a0;
          o[j][2] *= a1;
          o[j][3] *= a1;
        }
        const uint32_t chunk = sRing + s * T::kSlotBytes;
        const uint32_t ptile = sP + pb * (16 * 128);
        ok = ok && !*abort;
        if (ok) {
#pragma unroll
          for (int ks = 0; ks < T::KC / 16; ++ks) {
            // all fragments of this 16-key step first, then the 16 independent MMAs
            uint32_t a[4], b[8][4];
            ldsm_x4(ptile + sw128(lane & 15, ks * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
            const int key = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int jp = 0; jp < 8; ++jp) {
              const int dv0 = v * 128 + jp * 16;
              ldsm_x4_t(T::key_addr(chunk, key, dv0 / 8 + (lane >> 4)), b[jp][0], b[jp][1], b[jp][2], b[jp][3]);
            }
#pragma unroll
            for (int jp = 0; jp < 8; ++jp) {
              mma_bf16_16816(o[2 * jp], a, b[jp][0], b[jp][1]);
              mma_bf16_16816(o[2 * jp + 1], a, b[jp][2], b[jp][3]);
            }
          }
        }
        named_bar_arrive(T::kBarPEmpty + pb, T::kPPair);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::EMPTY + s));
      }
      // ---- epilogue: O / l -> output (or fp32 split partial), natural-log LSE ----
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = g4 + 8 * r;
        if (row >= p.R || !ok) continue;
        const float inv = lt[r] > 0.f ? 1.f / lt[r] : 0.f;
        const int sq = row / p.g, h = kvh * p.g + row % p.g;
        const float lse_v = lt[r] > 0.f ? (mr[r] + fast_log2(lt[r])) * 0.69314718055994531f : -INFINITY;
        if (nsplit == 1) {
          __nv_bfloat16 *orow = p.out + (((int64_t)seq * p.s_q + sq) * p.h_q + h) * kDV + v * 128 + c4 * 2;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            *reinterpret_cast<uint32_t *>(orow + j * 8) = pack_bf16x2(o[j][2 * r] * inv, o[j][2 * r + 1] * inv);
          if (v == 0 && c4 == 0) p.lse[lse_index(p, seq, sq, h)] = lse_v;
        } else {
          float *orow = p.o_accum + (acc_row0 + row) * kDV + v * 128 + c4 * 2;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            *reinterpret_cast<float2 *>(orow + j * 8) = make_float2(o[j][2 * r] * inv, o[j][2 * r + 1] * inv);
          if (v == 0 && c4 == 0) p.lse_accum[acc_row0 + row] = lse_v;
        }
      }
      ++qs;
    }
  }
  grid_launch_dependents();
  __syncthreads();
}

cudaError_t launch_decode_mma16(const CUtensorMap &kv_map, const CUtensorMap &q_map, const DecodeParams &p,
                                cudaStream_t stream) {
  using T = Mma16T<false>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(decode_mma16_kernel<false>), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_parts, 1, p.h_kv);
  return launch_early(decode_mma16_kernel<false>, grid, dim3(T::kThreads), T::kSmemBytes, stream, kv_map, q_map, p);
}

cudaError_t launch_decode_sparse16(const CUtensorMap &q_map, const DecodeParams &p, cudaStream_t stream) {
  using T = Mma16T<true>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(decode_mma16_kernel<true>), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_parts, 1, p.h_kv);
  // the key rows are addressed through p.kv_base; the tensor-map slot is unused
  return launch_early(decode_mma16_kernel<true>, grid, dim3(T::kThreads), T::kSmemBytes, stream, q_map, q_map, p);
}

template <int BM, int DVS>
static cudaError_t launch_mma(const CUtensorMap &map, const DecodeParams &p, int m_blocks,
                              cudaStream_t stream) {
  using T = MmaTile<BM, DVS>;
  auto kern = decode_mma_kernel<BM, DVS>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_parts, m_blocks, p.h_kv);
  return launch_early(kern, grid, dim3(T::kThreads), T::kSmemBytes, stream, map, p);
}

cudaError_t launch_decode_mma(const CUtensorMap &map, const DecodeParams &p, cudaStream_t stream) {
  return launch_mma<64, 2>(map, p, (p.R + 63) / 64, stream);
}

}  // namespace pagedmla
