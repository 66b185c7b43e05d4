// Absorption GEMMs around the latent decode ("DeepSeek FlashMLA ... practitioner notes",
// dpshk.com, section 2.1: with k_h = W^UK_h c the score q_h . k_h equals (W^UK_h^T q_h) . c,
// so the query is carried into latent space once and the cache is never expanded per head):
//   before the decode, per token t and head h:
//     q'[t, h, 0:512]   = sum_d q_nope[t, h, d] * W^UK[h, d, 0:512]      (K = 128)
//     q'[t, h, 512:576] = q_rope[t, h, 0:64]                             (passes through)
//   after the decode:
//     o[t, h, d] = sum_c o_lat[t, h, c] * W^UV[h, d, c]                  (K = 512)
// Both are per-head GEMMs C[M x N] = A[M x K] B[K x N] with M = tokens (batch x s_q).  One
// warp computes 16 tokens x 64 columns with mma.sync m16n8k16 bf16 (fp32 accumulate),
// fragments loaded straight from global memory (the weights are read once per 64 tokens).
#include "launch.h"

namespace pagedmla {

constexpr int kAbsorbWarps = 4;  // 64 tokens per CTA

// B given as [K][N] (W^UK: k = d, n = latent column) when kKN, else as [N][K] (W^UV: n = d,
// k = latent column).
template <bool kKN>
__global__ void __launch_bounds__(kAbsorbWarps * 32)
    absorb_gemm_kernel(const __nv_bfloat16 *__restrict__ A, int64_t a_row, int64_t a_head, const __nv_bfloat16 *__restrict__ B,
                       __nv_bfloat16 *__restrict__ C, int64_t c_row, int64_t c_head, int M, int N, int K) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g4 = lane >> 2, c4 = lane & 3;
  const int n0 = blockIdx.x * 64, h = blockIdx.y, m0 = blockIdx.z * 64 + warp * 16;
  const __nv_bfloat16 *Ah = A + h * a_head;
  const __nv_bfloat16 *Bh = B + int64_t(h) * K * N;
  auto a_pair = [&](int m, int k) -> uint32_t {
    if (m >= M) return 0u;
    return __ldg(reinterpret_cast<const uint32_t *>(Ah + m * a_row + k));
  };
  auto b_pair = [&](int k, int n) -> uint32_t {
    if (kKN) {
      const uint16_t lo = __ldg(reinterpret_cast<const uint16_t *>(Bh + int64_t(k) * N + n));
      const uint16_t hi = __ldg(reinterpret_cast<const uint16_t *>(Bh + int64_t(k + 1) * N + n));
      return uint32_t(lo) | (uint32_t(hi) << 16);
    }
    return __ldg(reinterpret_cast<const uint32_t *>(Bh + int64_t(n) * K + k));
  };
  float acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  for (int k = 0; k < K; k += 16) {
    const int k0 = k + 2 * c4;
    const uint32_t a[4] = {a_pair(m0 + g4, k0), a_pair(m0 + g4 + 8, k0), a_pair(m0 + g4, k0 + 8),
                           a_pair(m0 + g4 + 8, k0 + 8)};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + 8 * j + g4;
      mma_bf16_16816(acc[j], a, b_pair(k0, n), b_pair(k0 + 8, n));
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int m = m0 + g4 + 8 * r;
    if (m >= M) continue;
    __nv_bfloat16 *crow = C + int64_t(h) * c_head + int64_t(m) * c_row + n0 + 2 * c4;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint32_t *>(crow + 8 * j) = pack_bf16x2(acc[j][2 * r], acc[j][2 * r + 1]);
  }
}

// Copies q_rope into columns 512-575 of q' (8 bf16 per thread).
__global__ void rope_copy_kernel(const __nv_bfloat16 *__restrict__ q_rope, int64_t r_row, int64_t r_head,
                                 __nv_bfloat16 *__restrict__ q_out, int T, int H) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;  // (t, h, 8-column chunk)
  if (i >= int64_t(T) * H * 8) return;
  const int c = int(i % 8), h = int((i / 8) % H), t = int(i / (8 * H));
  const uint4 v = *reinterpret_cast<const uint4 *>(q_rope + t * r_row + h * r_head + 8 * c);
  *reinterpret_cast<uint4 *>(q_out + (int64_t(t) * H + h) * kD + 512 + 8 * c) = v;
}

cudaError_t launch_absorb_q(const __nv_bfloat16 *q_nope, int64_t n_row, int64_t n_head, const __nv_bfloat16 *q_rope,
                            int64_t r_row, int64_t r_head, const __nv_bfloat16 *w_uk, __nv_bfloat16 *q_out, int T,
                            int H, cudaStream_t stream) {
  dim3 grid(512 / 64, H, (T + 63) / 64);
  absorb_gemm_kernel<true><<<grid, kAbsorbWarps * 32, 0, stream>>>(q_nope, n_row, n_head, w_uk, q_out,
                                                                   int64_t(H) * kD, kD, T, 512, 128);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = int64_t(T) * H * 8;
  rope_copy_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(q_rope, r_row, r_head, q_out, T, H);
  return cudaGetLastError();
}

cudaError_t launch_absorb_out(const __nv_bfloat16 *o_lat, int64_t l_row, int64_t l_head, const __nv_bfloat16 *w_uv,
                              __nv_bfloat16 *out, int T, int H, cudaStream_t stream) {
  dim3 grid(128 / 64, H, (T + 63) / 64);
  absorb_gemm_kernel<false><<<grid, kAbsorbWarps * 32, 0, stream>>>(o_lat, l_row, l_head, w_uv, out,
                                                                    int64_t(H) * 128, 128, T, 128, 512);
  return cudaGetLastError();
}

}  // namespace pagedmla
