// Paged MLA decode over an FP8 latent cache, up to 16 query rows per latent head (the
// memory-bound decode shape), warp MMA (mma.sync m16n8k16 bf16, fp32 accumulate).
//
// Cache format (this library's reading; the Baidu page on Flash MLA names FP8 storage of the
// cache, section 三.2, without a format): every token's 576-column latent row is stored as
// OCP E4M3 codes, [num_pages][64][h_kv][576] bytes, with one fp32 scale per token and latent
// head, [h_kv][num_pages][64]; the row the decode uses is scale * e4m3(code).  Half the
// bytes of the bf16 cache stream from HBM.
//
// The kernel is the 16-row warp-MMA pipeline of the bf16 cache (producer, four S warps, one
// softmax warp, four PV warps, chunks in a TMA ring) with these changes:
//   - a chunk is a whole 64-token page: 5 TMA boxes of 128 code columns x 64 tokens
//     (128-byte swizzle; the last box's columns 576-639 lie outside the tensor and are
//     filled with zeros) plus one box of the page's 64 scales.  At half the bytes of a bf16
//     page, twice the keys per chunk halve the stages' per-chunk costs (hand-offs between
//     warps, the accumulator rescale), which bound this pipeline rather than HBM;
//   - both MMAs run in f16 on the codes' exact f16 form (cvt.rn.f16x2.e4m3x2: one conversion
//     per two codes, every E4M3 value being an f16 value); the query tile is carried in f16
//     after a power-of-two scale of the tile (its largest |q| in [2^14, 2^15)), and P times
//     the key scale in f16 after a power-of-two scale of the chunk (every product below
//     2^15), the accumulator carrying that factor from chunk to chunk through the rescale;
//   - score: ldmatrix (no transpose) of a code tile gives each thread 4 consecutive columns
//     of one key, which is the B fragment of m16n8k16 up to a permutation of the 16 K
//     columns of each step; the Q fragments are read with the same permutation;
//   - PV: ldmatrix.trans of a code tile gives each thread 2 value columns of 2 keys; a byte
//     permute turns that into the B fragments of two 8-column tiles holding the even and the
//     odd value columns of a 16-column group, so a thread's accumulators cover 4 consecutive
//     value columns;
//   - the per-token scale multiplies the score (x_j = softmax_scale * s_j * q.code_j) and
//     the probability that enters P V (the row sum uses the probability itself).
// Every mbarrier wait is bounded (pagedmla watchdog).
#include "common.cuh"
#include "launch.h"

namespace pagedmla {

struct Fp8x16 {
  static constexpr int KC = 64;                           // keys per chunk (one page)
  static constexpr int NS = 4;                            // ring depth
  static constexpr int kSWarps = 4, kSmWarp = 4, kPVWarp0 = 5, kPVWarps = 4, kProducer = 9;
  static constexpr int kThreads = 10 * 32;
  static constexpr int kBoxes = 5;                        // 128-column boxes per chunk (576 -> 640)
  static constexpr int kBoxBytes = KC * 128;              // 64 tokens x 128 codes: 8 KB
  static constexpr int kChunkBytes = kBoxes * kBoxBytes;  // 40 KB
  static constexpr int kScaleBytes = KC * 4;              // 64 fp32 scales
  static constexpr int kOffRing = 0;
  static constexpr int kOffScale = kOffRing + NS * kChunkBytes;
  static constexpr int kOffQ = kOffScale + NS * 1024;     // 16 rows x 576 bf16, 9 blocks of 2 KB
  static constexpr int kOffP = kOffQ + kColBlocks * 16 * 128;   // 2 x [16 rows x 64 keys] f16
  static constexpr int kOffS = kOffP + 2 * 16 * 128;            // 2 x [4 warps][16][32] f32 partial S
  static constexpr int kOffAlpha = kOffS + 2 * 4 * 16 * 32 * 4; // alpha[2][16]
  static constexpr int kOffL = kOffAlpha + 2 * 16 * 4;          // l[2 segs][16]
  static constexpr int kOffM = kOffL + 2 * 16 * 4;              // m[2 segs][16]
  static constexpr int kOffT = kOffM + 2 * 16 * 4;              // 2^-t of a segment's last chunk [2]
  static constexpr int kOffBar = kOffT + 16;
  enum { FULL = 0, EMPTY = FULL + NS, QFULL = EMPTY + NS, QFREE = QFULL + 1, NBARS = QFREE + 1 };
  static constexpr int kOffAbort = kOffBar + NBARS * 8;
  static constexpr int kSmemBytes = kOffAbort + 16 + 1024;
  // named barriers (id, id + 1 for the two buffers): S tile full / empty, P tile full / empty
  static constexpr int kBarSFull = 1, kBarSEmpty = 3, kBarPFull = 5, kBarPEmpty = 7;
  static constexpr int kSPair = (kSWarps + 1) * 32, kPPair = (kPVWarps + 1) * 32;
  static_assert(kOffScale % 1024 == 0 && kOffQ % 1024 == 0, "TMA destinations need 1 KB alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ void fp8_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Four E4M3 codes (low byte first) -> two f16x2 (codes 0-1, codes 2-3), exact: every E4M3
// value is an f16 value.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t codes, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(codes));
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two bf16 (low half first) times the power of two s -> f16x2; exact while the products are
// f16 normal numbers.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t v, float s) {
  const __half2 h = __floats2half2_rn(__uint_as_float(v << 16) * s, __uint_as_float(v & 0xffff0000u) * s);
  return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ void ldsm_x4_b8(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t_b8(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Token range and page (chunk) count of sequence `seq` within part `pc` (part boundaries fall
// on page multiples).
__device__ __forceinline__ int fp8_chunk_range(const DecodeParams &p, const PartCursor &pc, int seq, int &L, int &t0,
                                               int &t1) {
  L = p.seqlens[seq];
  t0 = seq == pc.bi ? pc.bt : 0;
  t1 = seq == pc.ei ? pc.et : L;
  return t1 > t0 ? (t1 - t0 + Fp8x16::KC - 1) / Fp8x16::KC : 0;
}

__global__ void __launch_bounds__(Fp8x16::kThreads, 1)
    decode_fp8_kernel(const __grid_constant__ CUtensorMap k8_map, const __grid_constant__ CUtensorMap scale_map,
                      const __grid_constant__ CUtensorMap q_map, const DecodeParams p) {
  using T = Fp8x16;
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
  const float *scale_sm = reinterpret_cast<const float *>(smem + T::kOffScale);   // [NS][256 floats]
  float *sbuf = reinterpret_cast<float *>(smem + T::kOffS);
  float *alpha_sm = reinterpret_cast<float *>(smem + T::kOffAlpha);
  float *l_sm = reinterpret_cast<float *>(smem + T::kOffL);
  float *m_sm = reinterpret_cast<float *>(smem + T::kOffM);
  float *t_sm = reinterpret_cast<float *>(smem + T::kOffT);
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

  if (warp == T::kProducer) {
    // ------------------------- producer: query tiles and code chunks -------------------------
    if (lane == 0) {
      prefetch_tensormap(&k8_map);
      prefetch_tensormap(&scale_map);
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
      const int nch = fp8_chunk_range(p, pc, seq, L, t0, t1);
      if (nch == 0) continue;
      int good = 1;
      if (lane == 0) {
        if (!mbar_wait(bar(T::QFREE), (qs & 1) ^ 1, abort, p.status, lim_ns)) {
          good = 0;
        } else {
          mbar_arrive_expect_tx(bar(T::QFULL), uint32_t(kColBlocks * p.R * 128));
#pragma unroll
          for (int c = 0; c < kColBlocks; ++c)
            tma_load_4d(sQ + c * 16 * 128, &q_map, bar(T::QFULL), c * 64, kvh * p.g, 0, seq);
          last_q = qs;
        }
      }
      ok = __shfl_sync(0xffffffffu, good, 0) != 0;
      ++qs;
      const int32_t *bt_row = p.block_table + (int64_t)seq * p.bt_stride + t0 / kPage;
      for (int base = 0; ok && base < nch; base += 32) {
        const int mine = base + lane < nch ? bt_row[base + lane] : 0;
        const int cnt = min(32, nch - base);
        for (int i = 0; ok && i < cnt; ++i, ++it) {
          const int phys = __shfl_sync(0xffffffffu, mine, i);
          const int s = it % T::NS;
          int g2 = 1;
          if (lane == 0) {
            if (!mbar_wait(bar(T::EMPTY + s), ((it / T::NS) & 1) ^ 1, abort, p.status, lim_ns)) {
              g2 = 0;
            } else {
              mbar_arrive_expect_tx(bar(T::FULL + s), T::kChunkBytes + T::kScaleBytes);
              const uint32_t dst = sRing + s * T::kChunkBytes;
              const int row = phys * kPage;
#pragma unroll
              for (int c = 0; c < T::kBoxes; ++c)
                tma_load_3d_hint(dst + c * T::kBoxBytes, &k8_map, bar(T::FULL + s), c * 128, kvh, row, policy);
              tma_load_3d_hint(sbase + T::kOffScale + s * 1024, &scale_map, bar(T::FULL + s), 0, phys, kvh, policy);
              last_chunk[s] = it;
            }
          }
          ok = __shfl_sync(0xffffffffu, g2, 0) != 0;
        }
      }
    }
    if (lane == 0) {
      int never = 0;
      for (int s = 0; s < T::NS; ++s)
        if (last_chunk[s] >= 0)
          mbar_wait(bar(T::FULL + s), (last_chunk[s] / T::NS) & 1, &never, p.status, lim_ns);
      if (last_q >= 0) mbar_wait(bar(T::QFULL), last_q & 1, &never, p.status, lim_ns);
    }
    __syncwarp();
  } else if (warp < T::kSWarps) {
    // ------------------------- S warps: partial scores -------------------------
    // K step k covers code columns 16k..16k+15.  The thread's B fragment from ldmatrix holds
    // columns 16k + 4 c4 + {0, 1, 2, 3} of one key; in m16n8k16 those are the K positions
    // {2 c4, 2 c4 + 1, 2 c4 + 8, 2 c4 + 9}, so the A fragments take Q's columns in the same
    // order: a0/a1 = columns 4 c4, 4 c4 + 1 of rows g4, g4 + 8; a2/a3 = 4 c4 + 2, 4 c4 + 3.
    //
    // The score MMAs run in f16: the codes' f16 form is exact (one conversion per two codes),
    // and the query tile is carried in f16 after a power-of-two scale 2^e that puts its
    // largest |q| in [2^14, 2^15): every bf16 value of the tile within 2^28 of that maximum
    // is exact in f16, and smaller ones are rounded to f16 subnormals (an error below 2^-39 of
    // the largest product, far under the fp32 accumulation's rounding).  The partial scores
    // are multiplied back by 2^-e.
    const int kh = warp >> 1, kn = warp & 1;
    uint32_t qf[kD / 32][4];
    float qs_inv = 1.f;
    int it = 0, qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      int L, t0, t1;
      const int nch = fp8_chunk_range(p, pc, seq, L, t0, t1);
      if (nch == 0) continue;
      ok = ok && mbar_wait(bar(T::QFULL), qs & 1, abort, p.status, lim_ns);
      float q_scale = 1.f;
      if (ok) {
        // largest |q| over the tile's R rows (row r of a 16-row column block: bytes r*128..)
        uint32_t mx = 0;
        for (int i = lane; i < kColBlocks * p.R * 8; i += 32) {
          const int c = i / (p.R * 8), rem = i % (p.R * 8);
          uint32_t v0, v1, v2, v3;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3)
                       : "r"(sQ + c * 2048 + rem * 16));
          const uint32_t w[4] = {v0, v1, v2, v3};
#pragma unroll
          for (int k = 0; k < 4; ++k) mx = max(mx, max(w[k] & 0x7fffu, (w[k] >> 16) & 0x7fffu));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        // exponent of the largest |q| (bf16 field, bias 127); e = 14 - (exp - 127), kept
        // within the fp32 normal range
        const int ex = int(mx >> 7);
        const int e = mx == 0 ? 0 : max(-120, min(120, 141 - ex));
        q_scale = __uint_as_float(uint32_t(127 + e) << 23);
        qs_inv = __uint_as_float(uint32_t(127 - e) << 23);
      }
      if (ok) {
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk) {
          const int k = kh * (kD / 32) + kk;
          const int cb = k >> 2, ch = 2 * (k & 3) + (c4 >> 1), off = 8 * (c4 & 1);
          uint32_t lo0, hi0, lo1, hi1;
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(lo0), "=r"(hi0) : "r"(sQ + cb * 2048 + sw128(g4, ch) + off));
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(lo1), "=r"(hi1) : "r"(sQ + cb * 2048 + sw128(g4 + 8, ch) + off));
          qf[kk][0] = bf16x2_to_f16x2_scaled(lo0, q_scale);
          qf[kk][1] = bf16x2_to_f16x2_scaled(lo1, q_scale);
          qf[kk][2] = bf16x2_to_f16x2_scaled(hi0, q_scale);
          qf[kk][3] = bf16x2_to_f16x2_scaled(hi1, q_scale);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::QFREE));
      for (int n = 0; n < nch; ++n, ++it) {
        const int sb = it & 1;
        ok = ok && mbar_wait(bar(T::FULL + it % T::NS), (it / T::NS) & 1, abort, p.status, lim_ns);
        // this warp's 32 keys (kn * 32 ..) as four 8-key tiles: four independent accumulator
        // chains per K step
        float sc[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[t][e] = 0.f;
        if (ok) {
          const uint32_t chunk = sRing + (it % T::NS) * T::kChunkBytes;
          // matrix m of an x4 load: key tile 2 h + (m & 1) (keys kn*32 + 16 h + 8 (m & 1) ..),
          // K step k + (m >> 1)
          const int m = lane >> 3;
          auto kaddr = [&](int k, int h) {
            const int key = kn * 32 + h * 16 + (m & 1) * 8 + (lane & 7);
            const int kc = k + (m >> 1);
            return chunk + (kc >> 3) * T::kBoxBytes + sw128(key, kc & 7);
          };
#pragma unroll
          for (int kk = 0; kk < kD / 32; kk += 2) {
            const int k = kh * (kD / 32) + kk;
            uint32_t r[2][4];
            ldsm_x4_b8(kaddr(k, 0), r[0]);
            ldsm_x4_b8(kaddr(k, 1), r[1]);
#pragma unroll
            for (int dk = 0; dk < 2; ++dk)
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                  uint32_t b0, b1;
                  e4m3x4_to_f16x2x2(r[h][2 * dk + nt], b0, b1);
                  mma_f16_16816(sc[2 * h + nt], qf[kk + dk], b0, b1);
                }
          }
#pragma unroll
          for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[t][e] *= qs_inv;
        }
        if (it >= 2) named_bar_sync(T::kBarSEmpty + sb, T::kSPair);
        float *dst = sbuf + (sb * 4 + warp) * 16 * 32;
#pragma unroll
        for (int e = 0; e < 16; ++e) dst[e * 32 + lane] = sc[e >> 2][e & 3];
        fp8_bar_arrive(T::kBarSFull + sb, T::kSPair);
      }
      ++qs;
    }
    for (int c = max(it - 2, 0); c < it; ++c) named_bar_sync(T::kBarSEmpty + (c & 1), T::kSPair);
  } else if (warp == T::kSmWarp) {
    // ------------------------- softmax warp -------------------------
    int it = 0, qs = 0;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      int L, t0, t1;
      const int nch = fp8_chunk_range(p, pc, seq, L, t0, t1);
      if (nch == 0) continue;
      int lim[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = g4 + 8 * r;
        lim[r] = row < p.R ? min(t1, p.causal ? L - (p.s_q - 1 - row / p.g) : L) : -1;
      }
      float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
      int t_prev = 0;
      for (int n = 0; n < nch; ++n, ++it) {
        const int sb = it & 1, pb = it & 1;
        named_bar_sync(T::kBarSFull + sb, T::kSPair);
        // this thread's 32 scores: key halves kn = 0, 1; per half 4 key tiles x 4 values
        // (value e of tile e >> 2: row g4 + 8 ((e >> 1) & 1), key 8 (e >> 2) + 2 c4 + (e & 1))
        float sc[2][16];
        const float *src = sbuf + sb * 4 * 16 * 32;
#pragma unroll
        for (int kn = 0; kn < 2; ++kn)
#pragma unroll
          for (int e = 0; e < 16; ++e)
            sc[kn][e] = src[(kn * 16 + e) * 32 + lane] + src[((2 + kn) * 16 + e) * 32 + lane];
        fp8_bar_arrive(T::kBarSEmpty + sb, T::kSPair);
        // the chunk's token scales (landed with its codes; the S warps waited for them); the
        // slots past the piece's last token are not read, so that whatever the page holds
        // there enters neither the chunk's scale factor nor a product with a zero probability
        const float *ksc = scale_sm + (it % T::NS) * 256;
        float kscale[2][8];
#pragma unroll
        for (int kn = 0; kn < 2; ++kn)
#pragma unroll
          for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int kc = kn * 32 + t * 8 + c4 * 2 + u;
              kscale[kn][2 * t + u] = t0 + n * T::KC + kc < t1 ? ksc[kc] : 0.f;
            }
        // P V runs in f16: P times the key's scale times 2^t, with the power of two t of this
        // chunk chosen from its largest scale c so that every product (P <= 1) is below 2^15;
        // the accumulator carries the factor 2^t, changed between chunks through alpha
        float cmax = 0.f;
#pragma unroll
        for (int kn = 0; kn < 2; ++kn)
#pragma unroll
          for (int k = 0; k < 8; ++k) cmax = fmaxf(cmax, kscale[kn][k]);
        cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
        cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
        const int t_chunk = max(-120, min(120, 14 - (int((__float_as_uint(cmax) >> 23) & 0xff) - 127)));
        const float p_scale = __uint_as_float(uint32_t(127 + t_chunk) << 23);
        const int dt = max(-126, min(126, n == 0 ? 0 : t_chunk - t_prev));
        const float t_step = __uint_as_float(uint32_t(127 + dt) << 23);
        t_prev = t_chunk;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int kn = 0; kn < 2; ++kn)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int r = (e >> 1) & 1;
            const int kin = (e >> 2) * 2 + (e & 1);  // key tile * 2 + pair element
            const int key = t0 + n * T::KC + kn * 32 + (e >> 2) * 8 + c4 * 2 + (e & 1);
            const float v = key < lim[r] ? sc[kn][e] * kscale[kn][kin] * p.scale_log2 : -INFINITY;
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
          for (int t = 0; t < 4; ++t) {
            const float p0 = fast_exp2(sc[kn][t * 4 + 0] - base[0]), p1 = fast_exp2(sc[kn][t * 4 + 1] - base[0]);
            const float p2 = fast_exp2(sc[kn][t * 4 + 2] - base[1]), p3 = fast_exp2(sc[kn][t * 4 + 3] - base[1]);
            l[0] += p0 + p1;
            l[1] += p2 + p3;
            // the value row of a key is its scale times the codes: scale the probability
            const float s0 = kscale[kn][2 * t] * p_scale, s1 = kscale[kn][2 * t + 1] * p_scale;
            const int kl = kn * 32 + t * 8 + c4 * 2;
            const __half2 h01 = __floats2half2_rn(p0 * s0, p1 * s1), h23 = __floats2half2_rn(p2 * s0, p3 * s1);
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(ptile + sw128(g4, kl / 8) + (kl % 8) * 2),
                         "r"(*reinterpret_cast<const uint32_t *>(&h01)));
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(ptile + sw128(g4 + 8, kl / 8) + (kl % 8) * 2),
                         "r"(*reinterpret_cast<const uint32_t *>(&h23)));
          }
        if (c4 == 0) {
          alpha_sm[pb * 16 + g4] = alpha[0] * t_step;
          alpha_sm[pb * 16 + g4 + 8] = alpha[1] * t_step;
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
          if (lane == 0) t_sm[qs & 1] = __uint_as_float(uint32_t(127 - t_chunk) << 23);
        }
        fp8_bar_arrive(T::kBarPFull + pb, T::kPPair);
      }
      ++qs;
    }
    for (int c = max(it - 2, 0); c < it; ++c) named_bar_sync(T::kBarPEmpty + (c & 1), T::kPPair);
  } else {
    // ------------------------- PV warps -------------------------
    // Warp v: value columns 128 v .. 128 v + 127 = code box v.  For each 16-key step and
    // 16-column group j, ldmatrix.trans of the two 8-key x 16-column tiles gives the thread
    // keys 2 c4, 2 c4 + 1 (and + 8) of value columns 16 j + 2 g4, 16 j + 2 g4 + 1; the byte
    // permute 0x3120 splits them into the B fragments of the even and the odd columns.  Tile
    // 2 j holds the even columns, tile 2 j + 1 the odd ones, so the thread's accumulators
    // o[2j][0..1], o[2j+1][0..1] are value columns 16 j + 4 c4 + {0, 2, 1, 3} of row g4
    // (o[.][2..3] of row g4 + 8).
    const int v = warp - T::kPVWarp0;
    int it = 0, qs = 0;
    bool ok = true;
    for (int seq = pc.bi; part_has(pc, seq); ++seq) {
      int L, t0, t1;
      const int nch = fp8_chunk_range(p, pc, seq, L, t0, t1);
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
            p.lse[((int64_t)seq * p.h_q + kvh * p.g + tid % p.g) * p.s_q + tid / p.g] = -INFINITY;
          else
            p.lse_accum[acc_row0 + tid] = -INFINITY;
        }
        continue;
      }
      float o[16][4];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
      float lt[2] = {0.f, 0.f}, mr[2] = {-INFINITY, -INFINITY}, t_inv = 1.f;
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
          t_inv = t_sm[qs & 1];
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          o[j][0] *= a0;
          o[j][1] *= a0;
          o[j][2] *= a1;
          o[j][3] *= a1;
        }
        const uint32_t box = sRing + s * T::kChunkBytes + v * T::kBoxBytes;
        const uint32_t ptile = sP + pb * (16 * 128);
        ok = ok && !*abort;
        if (ok) {
#pragma unroll
          for (int ks = 0; ks < T::KC / 16; ++ks) {
            uint32_t a[4];
            ldsm_x4(ptile + sw128(lane & 15, ks * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
            // matrix m: keys 16 ks + 8 (m & 1) .., column group jp * 2 + (m >> 1)
            const int m = lane >> 3, key = ks * 16 + (m & 1) * 8 + (lane & 7);
#pragma unroll
            for (int jp = 0; jp < 4; ++jp) {
              uint32_t r[4];
              ldsm_x4_t_b8(box + sw128(key, jp * 2 + (m >> 1)), r);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int j = jp * 2 + h;
                const uint32_t lo = __byte_perm(r[2 * h], 0u, 0x3120), hi = __byte_perm(r[2 * h + 1], 0u, 0x3120);
                // even columns: low halves; odd columns: high halves
                uint32_t le, lod, he, hod;
                e4m3x4_to_f16x2x2(lo, le, lod);
                e4m3x4_to_f16x2x2(hi, he, hod);
                mma_f16_16816(o[2 * j], a, le, he);
                mma_f16_16816(o[2 * j + 1], a, lod, hod);
              }
            }
          }
        }
        fp8_bar_arrive(T::kBarPEmpty + pb, T::kPPair);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::EMPTY + s));
      }
      // ---- epilogue: O / l -> output (or fp32 split partial), natural-log LSE ----
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = g4 + 8 * r;
        if (row >= p.R || !ok) continue;
        // the accumulator carries 2^t of the sequence's last chunk
        const float inv = lt[r] > 0.f ? t_inv / lt[r] : 0.f;
        const int sq = row / p.g, h = kvh * p.g + row % p.g;
        const float lse_v = lt[r] > 0.f ? (mr[r] + fast_log2(lt[r])) * 0.69314718055994531f : -INFINITY;
        if (nsplit == 1) {
          __nv_bfloat16 *orow = p.out + (((int64_t)seq * p.s_q + sq) * p.h_q + h) * kDV + v * 128 + c4 * 4;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint2 *>(orow + j * 16) =
                make_uint2(pack_bf16x2(o[2 * j][2 * r] * inv, o[2 * j + 1][2 * r] * inv),
                           pack_bf16x2(o[2 * j][2 * r + 1] * inv, o[2 * j + 1][2 * r + 1] * inv));
          if (v == 0 && c4 == 0) p.lse[((int64_t)seq * p.h_q + h) * p.s_q + sq] = lse_v;
        } else {
          float *orow = p.o_accum + (acc_row0 + row) * kDV + v * 128 + c4 * 4;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4 *>(orow + j * 16) =
                make_float4(o[2 * j][2 * r] * inv, o[2 * j + 1][2 * r] * inv, o[2 * j][2 * r + 1] * inv,
                            o[2 * j + 1][2 * r + 1] * inv);
          if (v == 0 && c4 == 0) p.lse_accum[acc_row0 + row] = lse_v;
        }
      }
      ++qs;
    }
  }
  grid_launch_dependents();
  __syncthreads();
}

cudaError_t launch_decode_fp8(const CUtensorMap &k8_map, const CUtensorMap &scale_map, const CUtensorMap &q_map,
                              const DecodeParams &p, cudaStream_t stream) {
  using T = Fp8x16;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(decode_fp8_kernel), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_parts, 1, p.h_kv);
  return launch_early(decode_fp8_kernel, grid, dim3(T::kThreads), T::kSmemBytes, stream, k8_map, scale_map, q_map, p);
}

}  // namespace pagedmla
