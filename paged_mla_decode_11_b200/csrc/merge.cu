// Log-sum-exp merge of per-shard partial decodes of the same query rows: the merge step of a
// sequence whose keys are spread over several GPUs (each GPU decodes its shard of the pages
// and the shards' (out, lse) are gathered).  It is the same merge as the split-KV combine:
// lse = ln sum_k exp(lse_k), out = sum_k exp(lse_k - lse) out_k; shards with lse_k = -inf
// weigh nothing, and rows where every shard is -inf get out = 0, lse = -inf.
//
// One warp per (sequence, position, head) row: each lane owns 16 of the 512 value columns
// (two 16-byte bf16 loads per shard).
#include "launch.h"

namespace pagedmla {

constexpr int kMergeWarps = 4;

__global__ void __launch_bounds__(kMergeWarps * 32)
    merge_kernel(const __nv_bfloat16 *__restrict__ o_parts, const float *__restrict__ lse_parts, int n_parts,
                 int batch, int s_q, int h_q, __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = int64_t(blockIdx.x) * kMergeWarps + warp;   // (b, s, h) in output order
  const int64_t rows = int64_t(batch) * s_q * h_q;
  if (row >= rows) return;
  const int h = int(row % h_q), s = int((row / h_q) % s_q), b = int(row / (int64_t(h_q) * s_q));
  const int64_t lse_idx = (int64_t(b) * h_q + h) * s_q + s;        // [b][h_q][s_q]
  float mx = -INFINITY;
  for (int k = 0; k < n_parts; ++k) mx = fmaxf(mx, lse_parts[k * rows + lse_idx]);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float z = 0.f;
  if (mx != -INFINITY) {
    for (int k = 0; k < n_parts; ++k) {
      const float wk = __expf(lse_parts[k * rows + lse_idx] - mx);   // exp(-inf) = 0
      z += wk;
      const uint4 *src = reinterpret_cast<const uint4 *>(o_parts + (k * rows + row) * kDV) + lane * 2;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 u = src[i];
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[t]));
          acc[8 * i + 2 * t] += wk * f.x;
          acc[8 * i + 2 * t + 1] += wk * f.y;
        }
      }
    }
  }
  const float inv = z > 0.f ? 1.f / z : 0.f;
  uint4 *dst = reinterpret_cast<uint4 *>(out + row * kDV) + lane * 2;
#pragma unroll
  for (int i = 0; i < 2; ++i)
    dst[i] = make_uint4(pack_bf16x2(acc[8 * i] * inv, acc[8 * i + 1] * inv), pack_bf16x2(acc[8 * i + 2] * inv, acc[8 * i + 3] * inv),
                        pack_bf16x2(acc[8 * i + 4] * inv, acc[8 * i + 5] * inv), pack_bf16x2(acc[8 * i + 6] * inv, acc[8 * i + 7] * inv));
  if (lane == 0) lse[lse_idx] = z > 0.f ? mx + __logf(z) : -INFINITY;
}

cudaError_t launch_merge(const __nv_bfloat16 *o_parts, const float *lse_parts, int n_parts, int batch, int s_q,
                         int h_q, __nv_bfloat16 *out, float *lse, cudaStream_t stream) {
  const int64_t rows = int64_t(batch) * s_q * h_q;
  const dim3 grid(unsigned((rows + kMergeWarps - 1) / kMergeWarps));
  merge_kernel<<<grid, kMergeWarps * 32, 0, stream>>>(o_parts, lse_parts, n_parts, batch, s_q, h_q, out, lse);
  return cudaGetLastError();
}

}  // namespace pagedmla
