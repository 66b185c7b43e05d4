// Split-KV tile scheduler (the pages' get_mla_metadata: "OpenSourceWeek Day 1 -
// FlashMLA", section V.2, which shows only its call).  Plan ("balanced cuts", specified
// in pagedmla.h): with OVH = max(1, ceil(R / 32)) pages per split, sequence b occupies
// OVH + ceil(L_b / 64) units of a cost axis (its OVH units first, then one unit per page); with T the axis length and
// payload = ceil(T / num_parts), part p covers [p * payload, (p + 1) * payload) clipped
// to T.  Position x maps to the cursor (i, max(0, x - start_i - OVH)) of the sequence i
// holding it, or (B, 0) at the end.
//
// Everything is a closed form of the prefix sums start_b, so one CTA computes the plan
// in parallel: a block scan of the costs, then one binary search per part cut and one
// closed-form split count per sequence, then a block scan of the split counts.
#include "launch.h"
#include "pagedmla.h"

namespace pagedmla {

constexpr int kMetaThreads = 512;

// Exclusive block-wide prefix sum of one value per thread; *total receives the sum.
__device__ long long block_exclusive_scan(long long v, long long *scratch, long long *total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  constexpr int kWarps = kMetaThreads / 32;
  long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < kWarps ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < kWarps) scratch[lane] = w;
  }
  __syncthreads();
  const long long before = warp > 0 ? scratch[warp - 1] : 0;
  *total = scratch[kWarps - 1];
  __syncthreads();
  return before + incl - v;
}

template <bool kOffsets>
__global__ void __launch_bounds__(kMetaThreads)
    metadata_kernel(const int32_t *__restrict__ seqlens, int batch, int ovh, int num_parts,
                    int32_t *__restrict__ tile_md, int32_t *__restrict__ num_splits) {
  // length of sequence b: an entry, or the difference of two offsets (a CSR row_ptr)
  auto len = [&](int b) { return kOffsets ? seqlens[b + 1] - seqlens[b] : seqlens[b]; };
  extern __shared__ long long start[];  // [batch + 1]
  __shared__ long long scratch[32];
  grid_launch_dependents();  // the decode kernel may start its prologue now
  const int per = (batch + kMetaThreads - 1) / kMetaThreads;
  const int lo = threadIdx.x * per, hi = min(batch, lo + per);

  // 1. start_b = exclusive prefix sum of (OVH + pages_b)
  long long mine = 0;
  for (int b = lo; b < hi; ++b) mine += ovh + (max(len(b), 0) + kPage - 1) / kPage;
  long long total;
  long long run = block_exclusive_scan(mine, scratch, &total);
  for (int b = lo; b < hi; ++b) {
    start[b] = run;
    run += ovh + (max(len(b), 0) + kPage - 1) / kPage;
  }
  if (threadIdx.x == 0) start[batch] = total;
  __syncthreads();
  const long long T = total;
  const long long payload = (T + num_parts - 1) / num_parts;

  // 2. one thread per part: both cuts -> cursors by binary search over start[]
  auto part_entry = [&](int p, int32_t (&t)[8]) {
    int ci[2];
    long long ck[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const long long x = min((long long)(p + e) * payload, T);
      if (x >= T) {
        ci[e] = batch;
        ck[e] = 0;
      } else {
        int a = 0, z = batch - 1;  // largest i with start[i] <= x
        while (a < z) {
          const int mid = (a + z + 1) / 2;
          if (start[mid] <= x) a = mid;
          else z = mid - 1;
        }
        ci[e] = a;
        ck[e] = max(0ll, x - start[a] - ovh);
      }
    }
    t[0] = ci[0];
    t[1] = int32_t(ck[0] * kPage);
    t[2] = ci[1];
    t[3] = int32_t(ck[1] * kPage);
    t[4] = ck[0] > 0 ? int(p - (start[ci[0]] + ovh) / payload) : 0;
    t[5] = t[6] = t[7] = 0;
  };
  int32_t held[8];
  const bool one_pass = num_parts <= kMetaThreads;
  if (one_pass && threadIdx.x < num_parts) part_entry(threadIdx.x, held);

  // 3. parts touching sequence b: 1 + cuts strictly inside its page units
  auto splits_of = [&](int b) { return 1 + max(0ll, (start[b + 1] - 1) / payload - (start[b] + ovh) / payload); };
  long long cnt = 0;
  for (int b = lo; b < hi; ++b) cnt += splits_of(b);
  long long all;
  run = block_exclusive_scan(cnt, scratch, &all);

  // The plan is complete; the kernel before this one in the stream may still read the
  // buffers it is written to (a previous step's plan), so wait for it before writing.  All
  // of the above, the length reads included, overlapped that kernel's tail.
  grid_dependency_wait();
  if (one_pass) {
    if (threadIdx.x < num_parts) {
#pragma unroll
      for (int k = 0; k < 8; ++k) tile_md[threadIdx.x * 8 + k] = held[k];
    }
  } else {
    for (int p = threadIdx.x; p < num_parts; p += kMetaThreads) {
      int32_t t[8];
      part_entry(p, t);
#pragma unroll
      for (int k = 0; k < 8; ++k) tile_md[p * 8 + k] = t[k];
    }
  }
  if (threadIdx.x == 0) num_splits[0] = 0;
  for (int b = lo; b < hi; ++b) {
    run += splits_of(b);
    num_splits[b + 1] = int32_t(run);
  }
}

cudaError_t launch_metadata(const int32_t *seqlens, int batch, int ovh, int num_parts, int32_t *tile_md,
                            int32_t *num_splits, cudaStream_t stream, bool lengths_are_offsets) {
  const size_t smem = size_t(batch + 1) * sizeof(long long);
  auto kern = lengths_are_offsets ? metadata_kernel<true> : metadata_kernel<false>;
  if (smem > 48 * 1024) {
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), int((MLA_MAX_BATCH + 1) * sizeof(long long)));
    if (e != cudaSuccess) return e;
  }
  // launched early: the plan is computed while the previous kernel finishes (see above)
  return launch_early(kern, dim3(1), dim3(kMetaThreads), smem, stream, seqlens, batch, ovh, num_parts, tile_md,
                      num_splits);
}

}  // namespace pagedmla
