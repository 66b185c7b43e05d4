// Absorption GEMMs around the latent decode ("DeepSeek FlashMLA ... practitioner notes",
// dpshk.com, section 2.1: with k_h = W^UK_h c the score q_h . k_h equals (W^UK_h^T q_h) . c,
// so the query is carried into latent space once and the cache is never expanded per head):
//   before the decode, per token t and head h:
//     q'[t, h, 0:512]   = sum_d q_nope[t, h, d] * W^UK[h, d, 0:512]      (K = 128)
//     q'[t, h, 512:576] = q_rope[t, h, 0:64]                             (passes through)
//   after the decode:
//     o[t, h, d] = sum_c o_lat[t, h, c] * W^UV[h, d, c]                  (K = 512)
// Both are per-head GEMMs C[M x N] = A[M x K] B[K x N] with M = tokens (batch x s_q).  At
// decode batch sizes they are bound by reading the weights (128 KB per head and product), so
// they run on warp MMA (mma.sync m16n8k16 bf16, fp32 accumulate): a CTA computes a 64-token x
// BN-column tile of one head (BN = 128 for q', 64 for the output), its four warps 16 tokens x
// BN columns each, over K chunks of 64 staged in shared memory by cp.async (three stages: two
// chunks load while one is multiplied; q' has only two chunks, so its launch gives the
// kernel two stages of shared memory and twice as many CTAs fit on an SM).  Tile rows are
// padded by 16 bytes, so the 8 rows of an ldmatrix fall in distinct banks.
//
// Both kernels are programmatic dependent launches: a CTA issues the copies of its weight
// tiles (model parameters, written long before) before it waits for the previous kernel in
// the stream, and the activation tiles after, so the weight reads overlap that kernel's
// tail.  The q' kernel's first column block also copies the rope columns of its tokens.
#include "launch.h"

namespace pagedmla {

constexpr int kAbBM = 64, kAbBK = 64, kAbWarps = 4, kAbStages = 3;

template <bool kKN, int BN>
struct AbsorbTile {
  static constexpr int kARow = kAbBK * 2 + 16;                       // A chunk [64 tokens][64 k]
  static constexpr int kABytes = kAbBM * kARow;
  // B chunk: [64 k][BN n] when B is given as [K][N], else [BN n][64 k]
  static constexpr int kBRow = kKN ? BN * 2 + 16 : kAbBK * 2 + 16;
  static constexpr int kBBytes = kKN ? kAbBK * kBRow : BN * kBRow;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kSmem = kAbStages * kStage;
  static_assert(!kKN || kAbWarps * 16 * (BN * 2 + 16) <= 2 * kStage, "q' output staging fits in two stages");
};

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// B given as [K][N] (W^UK: k = d, n = latent column) when kKN, else as [N][K] (W^UV: n = d,
// k = latent column).  M, N, K: tokens (any), columns (a multiple of BN), contraction (a
// multiple of 64).
// rope (q' only): q_rope, element (t, h, c) at t * r_row + h * r_head + c, copied into columns
// 512..575 of C's rows (blockIdx.x == 0 only); nullptr for the output product.
template <bool kKN, int BN>
__global__ void __launch_bounds__(kAbWarps * 32)
    absorb_gemm_kernel(const __nv_bfloat16 *__restrict__ A, int64_t a_row, int64_t a_head,
                       const __nv_bfloat16 *__restrict__ B, __nv_bfloat16 *__restrict__ C, int64_t c_row,
                       int64_t c_head, int M, int N, int K, const __nv_bfloat16 *__restrict__ rope, int64_t r_row,
                       int64_t r_head) {
  using T = AbsorbTile<kKN, BN>;
  extern __shared__ __align__(16) uint8_t absorb_smem[];
  const uint32_t sbase = smem_u32(absorb_smem);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int g4 = lane >> 2, c4 = lane & 3;
  const int n0 = blockIdx.x * BN, h = blockIdx.y, m0 = blockIdx.z * kAbBM;
  const __nv_bfloat16 *Ah = A + int64_t(h) * a_head;
  const __nv_bfloat16 *Bh = B + int64_t(h) * K * N;
  grid_launch_dependents();  // the next kernel may start its prologue

  auto load_a = [&](int st, int k0) {
    const uint32_t sa = sbase + st * T::kStage;
    for (int i = tid; i < kAbBM * (kAbBK / 8); i += kAbWarps * 32) {
      const int r = i / (kAbBK / 8), c = i % (kAbBK / 8), t = m0 + r;
      cp_async16_zfill(sa + r * T::kARow + c * 16, Ah + int64_t(min(t, M - 1)) * a_row + k0 + c * 8, t < M ? 16u : 0u);
    }
  };
  auto load_b = [&](int st, int k0) {
    const uint32_t sb = sbase + st * T::kStage + T::kABytes;
    if constexpr (kKN) {
      for (int i = tid; i < kAbBK * (BN / 8); i += kAbWarps * 32) {
        const int r = i / (BN / 8), c = i % (BN / 8);
        cp_async16_zfill(sb + r * T::kBRow + c * 16, Bh + int64_t(k0 + r) * N + n0 + c * 8, 16u);
      }
    } else {
      for (int i = tid; i < BN * (kAbBK / 8); i += kAbWarps * 32) {
        const int r = i / (kAbBK / 8), c = i % (kAbBK / 8);
        cp_async16_zfill(sb + r * T::kBRow + c * 16, Bh + int64_t(n0 + r) * K + k0 + c * 8, 16u);
      }
    }
  };

  float acc[BN / 8][4];
#pragma unroll
  for (int j = 0; j < BN / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  const int nk = K / kAbBK;
  // One commit group per chunk (empty past the end), so "all but the newest S - 2 groups
  // landed" means chunk kc has landed.  The prologue's weight copies are issued before the
  // dependency wait and fall into the first group, which is older than any of their chunks.
#pragma unroll
  for (int st = 0; st < kAbStages - 1; ++st)
    if (st < nk) load_b(st, st * kAbBK);
  grid_dependency_wait();  // the activations may come from the kernel just before
#pragma unroll
  for (int st = 0; st < kAbStages - 1; ++st) {
    if (st < nk) load_a(st, st * kAbBK);
    cp_async_commit();
  }
  if constexpr (kKN) {
    // the rope columns pass through: 64 tokens x 8 chunks of 16 bytes, while the copies fly
    if (blockIdx.x == 0)
      for (int i = tid; i < kAbBM * 8; i += kAbWarps * 32) {
        const int t = m0 + i / 8, c = i % 8;
        if (t < M)
          *reinterpret_cast<uint4 *>(C + int64_t(h) * c_head + int64_t(t) * c_row + 512 + 8 * c) =
              *reinterpret_cast<const uint4 *>(rope + t * r_row + h * r_head + 8 * c);
      }
  }
  for (int kc = 0; kc < nk; ++kc) {
    cp_async_wait<kAbStages - 2>();
    __syncthreads();  // chunk kc is visible to all warps; chunk kc - 1's stage is free
    const int kn = kc + kAbStages - 1;
    if (kn < nk) {
      load_a(kn % kAbStages, kn * kAbBK);
      load_b(kn % kAbStages, kn * kAbBK);
    }
    cp_async_commit();
    const uint32_t sa = sbase + (kc % kAbStages) * T::kStage, sb = sa + T::kABytes;
#pragma unroll
    for (int ks = 0; ks < kAbBK / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(sa + (warp * 16 + (lane & 15)) * T::kARow + (ks * 16 + (lane >> 4) * 8) * 2, a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int jp = 0; jp < BN / 16; ++jp) {
        uint32_t b[4];
        if constexpr (kKN)
          ldsm_x4_t(sb + (ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * T::kBRow + (jp * 16 + (lane >> 4) * 8) * 2,
                    b[0], b[1], b[2], b[3]);
        else
          ldsm_x4(sb + (jp * 16 + (lane & 7) + (lane >> 4) * 8) * T::kBRow + (ks * 16 + ((lane >> 3) & 1) * 8) * 2,
                  b[0], b[1], b[2], b[3]);
        mma_bf16_16816(acc[2 * jp], a, b[0], b[1]);
        mma_bf16_16816(acc[2 * jp + 1], a, b[2], b[3]);
      }
    }
  }
  if constexpr (kKN) {
    // q' (16-byte aligned): the warp's 16 x BN tile goes through shared memory (rows padded by
    // 16 bytes: the 8 rows of a fragment store fall in distinct banks) and leaves as 16-byte
    // stores, each warp instruction covering two whole 256-byte row segments
    constexpr int kORow = BN * 2 + 16, kChunks = BN / 8;
    __syncthreads();  // every warp has finished reading the ring
    const uint32_t so = sbase + warp * 16 * kORow;
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int j = 0; j < BN / 8; ++j)
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(so + (g4 + 8 * r) * kORow + (j * 8 + 2 * c4) * 2),
                     "r"(pack_bf16x2(acc[j][2 * r], acc[j][2 * r + 1])));
    __syncwarp();
#pragma unroll
    for (int q = lane; q < 16 * kChunks; q += 32) {
      const int row = q / kChunks, c = q % kChunks, t = m0 + warp * 16 + row;
      if (t >= M) continue;
      uint32_t v0, v1, v2, v3;
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3)
                   : "r"(so + row * kORow + c * 16));
      *reinterpret_cast<uint4 *>(C + int64_t(h) * c_head + int64_t(t) * c_row + n0 + 8 * c) = make_uint4(v0, v1, v2, v3);
    }
  } else {
    // the output (4-byte aligned): fragment stores straight from the accumulators
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int t = m0 + warp * 16 + g4 + 8 * r;
      if (t >= M) continue;
      __nv_bfloat16 *crow = C + int64_t(h) * c_head + int64_t(t) * c_row + n0 + 2 * c4;
#pragma unroll
      for (int j = 0; j < BN / 8; ++j)
        *reinterpret_cast<uint32_t *>(crow + 8 * j) = pack_bf16x2(acc[j][2 * r], acc[j][2 * r + 1]);
    }
  }
}

cudaError_t launch_absorb_q(const __nv_bfloat16 *q_nope, int64_t n_row, int64_t n_head, const __nv_bfloat16 *q_rope,
                            int64_t r_row, int64_t r_head, const __nv_bfloat16 *w_uk, __nv_bfloat16 *q_out, int T,
                            int H, cudaStream_t stream) {
  constexpr int kBN = 128;
  // K = 128: two chunks, stages 0 and 1 only (the third stage of the ring is never reached)
  constexpr int kSmem = 2 * AbsorbTile<true, kBN>::kStage;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(absorb_gemm_kernel<true, kBN>), kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(512 / kBN, H, (T + kAbBM - 1) / kAbBM);
  return launch_early(absorb_gemm_kernel<true, kBN>, grid, dim3(kAbWarps * 32), kSmem, stream, q_nope, n_row, n_head,
                      w_uk, q_out, int64_t(H) * kD, int64_t(kD), T, 512, 128, q_rope, r_row, r_head);
}

cudaError_t launch_absorb_out(const __nv_bfloat16 *o_lat, int64_t l_row, int64_t l_head, const __nv_bfloat16 *w_uv,
                              __nv_bfloat16 *out, int T, int H, cudaStream_t stream) {
  constexpr int kBN = 64;
  constexpr int kSmem = AbsorbTile<false, kBN>::kSmem;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(absorb_gemm_kernel<false, kBN>), kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(128 / kBN, H, (T + kAbBM - 1) / kAbBM);
  return launch_early(absorb_gemm_kernel<false, kBN>, grid, dim3(kAbWarps * 32), kSmem, stream, o_lat, l_row, l_head,
                      w_uv, out, int64_t(H) * 128, int64_t(128), T, 128, 512,
                      static_cast<const __nv_bfloat16 *>(nullptr), int64_t(0), int64_t(0));
}

}  // namespace pagedmla
