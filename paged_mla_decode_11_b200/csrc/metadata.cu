// Split-KV tile scheduler (the pages' get_mla_metadata: "OpenSourceWeek Day 1 -
// FlashMLA", section V.2, which shows only its call).  Plan, as specified in pagedmla.h:
// pages_b = ceil(L_b / 64); total = sum_b (pages_b + OVH); payload = ceil(total / parts)
// + OVH; each part, in order, finishes whole sequences while (pages left + OVH) fits in
// what remains of its payload and otherwise takes the next (remaining - OVH) pages of
// the current sequence, if that is positive.
//
// One CTA: the lengths are read in parallel into shared memory, one thread walks the
// plan there (integer arithmetic only, so the result is exact), then the split counts
// are turned into prefix sums.
#include "launch.h"
#include "pagedmla.h"

namespace pagedmla {

constexpr int kOvh = 5;
constexpr int kMetaThreads = 256;

__global__ void __launch_bounds__(kMetaThreads)
    metadata_kernel(const int32_t *__restrict__ seqlens, int batch, int num_parts,
                    int32_t *__restrict__ tile_md, int32_t *__restrict__ num_splits) {
  extern __shared__ int32_t sh[];
  int32_t *pages = sh;
  int32_t *touched = sh + batch;
  __shared__ long long warp_tot[kMetaThreads / 32];

  long long local = 0;
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    const int L = max(seqlens[b], 0);
    pages[b] = (L + kPage - 1) / kPage;
    touched[b] = 0;
    local += pages[b] + kOvh;
  }
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if (threadIdx.x % 32 == 0) warp_tot[threadIdx.x / 32] = local;
  __syncthreads();

  if (threadIdx.x == 0) {
    long long total = 0;
    for (int w = 0; w < kMetaThreads / 32; ++w) total += warp_tot[w];
    const long long payload = (total + num_parts - 1) / num_parts + kOvh;
    int i = 0;
    long long k = 0;
    for (int part = 0; part < num_parts; ++part) {
      const int begin_i = i;
      const long long begin_k = k;
      const int ord = i < batch ? touched[i] : 0;
      long long rem = payload;
      while (i < batch) {
        const long long left = pages[i] - k;
        if (left + kOvh <= rem) {
          rem -= left + kOvh;
          touched[i] += 1;
          ++i;
          k = 0;
        } else {
          if (rem - kOvh > 0) {
            k += rem - kOvh;
            touched[i] += 1;
          }
          break;
        }
      }
      int32_t *t = tile_md + part * 8;
      t[0] = begin_i;
      t[1] = static_cast<int32_t>(begin_k * kPage);
      t[2] = i;
      t[3] = static_cast<int32_t>(k * kPage);
      t[4] = ord;
      t[5] = 0;
      t[6] = 0;
      t[7] = 0;
    }
    int acc = 0;
    num_splits[0] = 0;
    for (int b = 0; b < batch; ++b) {
      acc += touched[b];
      num_splits[b + 1] = acc;
    }
  }
}

cudaError_t launch_metadata(const int32_t *seqlens, int batch, int num_parts, int32_t *tile_md,
                            int32_t *num_splits, cudaStream_t stream) {
  const size_t smem = size_t(batch) * 2 * sizeof(int32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(metadata_kernel),
                                  2 * MLA_MAX_BATCH * int(sizeof(int32_t)));
    if (e != cudaSuccess) return e;
  }
  metadata_kernel<<<1, kMetaThreads, smem, stream>>>(seqlens, batch, num_parts, tile_md, num_splits);
  return cudaGetLastError();
}

}  // namespace pagedmla
