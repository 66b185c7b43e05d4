// Log-sum-exp combine of split-KV partials (the method's merge of the partial results
// of one sequence's splits): lse = ln sum_k exp(lse_k), out = sum_k exp(lse_k - lse) o_k.
//
// One warp per (sequence, latent head, query row, half of the value columns); sequences
// with a single split are skipped (the decode kernel wrote them directly).  In its 256
// columns each lane owns 8 as two float4s strided 128 apart, so every warp-wide access
// covers 512 contiguous bytes.  CTAs are small (4 warps) so that many of them are resident
// as soon as the decode kernel's CTAs exit.
//
// Two instantiations: up to eight splits' rows in flight per warp at four CTAs per SM, and
// five splits at six CTAs per SM.  The second serves grids of more than two waves with 128 or
// more rows per latent head (the compute-bound shapes: a few dozen parts, so few splits per
// sequence, and many waves of CTAs each one or two round trips to L2 long, where more
// resident warps matter more); the first everything else: one-wave grids (fewer CTAs per SM
// spread them over more SMs) and shapes with a sequence split many ways, whose merge is a
// chain of batches on the step's critical path.  Measured in the whole step: compute-bound
// 218.4-219.4 against 220.1-221.8 us, causal (s_q = 2) 220.2-221.4 against 221.8-222.6 us;
// skewed (one sequence in 42 splits) 88.0-88.1 us with the first against 91.1-91.4 us.
//
// The kernel is launched early (programmatic dependent launch) and runs after the decode
// kernel's last CTA, so its latency is the tail of every decode call.  It therefore reads
// the plan before waiting for the decode kernel (the scheduler kernel wrote num_splits and
// had completed before any decode CTA passed its own dependency wait), and after the wait
// issues the split LSEs and the partial rows of the first kBatch splits in one round trip.
#include "launch.h"

namespace pagedmla {

constexpr int kCombineWarps = 4;           // two rows x two column halves

// kBatch: splits whose partial rows are loaded together; kCtas CTAs per SM bound the registers
// (128 per thread for 8 splits at 4 CTAs, 85 for 5 at 6).
template <int kBatch, int kCtas>
__global__ void __launch_bounds__(kCombineWarps * 32, kCtas)
    combine_kernel(const int32_t *__restrict__ num_splits, int s_q, int h_q, int h_kv, int R, int sq_fold,
                   const float *__restrict__ lse_accum, const float *__restrict__ o_accum,
                   __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
  // the next kernel may start its prologue; the scheduler kernel of a next step computes its
  // plan meanwhile and writes it only after this kernel has completed
  grid_launch_dependents();
  // row pairs of a sequence are the fastest grid index, so all rows of a long sequence (tens
  // of splits) are scheduled in the first wave rather than spread over the whole grid
  const int b = blockIdx.y, kvh = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = blockIdx.x * (kCombineWarps / 2) + warp / 2, half = warp % 2;
  // Everything this kernel reads comes from kernels that may still be running when it
  // starts (programmatic dependent launch), so it reads through L2 (ld.global.cg), never
  // through the non-coherent read-only path.
  const int ns0 = __ldcg(num_splits + b);
  const int n = __ldcg(num_splits + b + 1) - ns0;
  if (n <= 1 || row >= R) {
    // one CTA waits for the decode kernel even when nothing is split, so that this grid
    // never completes before its predecessor (the next kernel in the stream may write the
    // plan the decode kernel reads)
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) grid_dependency_wait();
    return;
  }
  const int g = h_q / h_kv;
  const int64_t stride = int64_t(h_kv) * R;  // between consecutive splits
  const int64_t base = (int64_t(ns0) * h_kv + kvh) * R + row;
  auto part_row = [&](int k) {
    return reinterpret_cast<const float4 *>(o_accum + (base + k * stride) * kDV + half * (kDV / 2));
  };
  auto lse_of = [&](int k) { return __ldcg(lse_accum + base + k * stride); };
  grid_dependency_wait();  // partials come from the decode kernel just before

  // one round trip: split `lane`'s LSE and the first kBatch splits' partial rows
  const float lk = lane < n ? lse_of(lane) : -INFINITY;
  float4 v[kBatch][2];
#pragma unroll
  for (int j = 0; j < kBatch; ++j)
    if (j < n)
#pragma unroll
      for (int i = 0; i < 2; ++i) v[j][i] = __ldcg(part_row(j) + lane + 32 * i);

  // merged LSE: max over splits, then ln sum exp
  float mx = lk;
  for (int k = lane + 32; k < n; k += 32) mx = fmaxf(mx, lse_of(k));
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  if (mx != -INFINITY) {
    sum = expf(lk - mx);
    for (int k = lane + 32; k < n; k += 32) sum += expf(lse_of(k) - mx);
  }
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float tot = mx == -INFINITY ? -INFINITY : mx + logf(sum);

  float4 acc[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = 0; k0 < n; k0 += 32) {
    // lane j holds the weight of split k0 + j
    const float l = k0 == 0 ? lk : (k0 + lane < n ? lse_of(k0 + lane) : -INFINITY);
    const float wl = tot != -INFINITY && k0 + lane < n ? expf(l - tot) : 0.f;
    const int kn = min(32, n - k0);
    for (int j0 = 0; j0 < kn; j0 += kBatch) {
      if (k0 + j0 > 0) {
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
          if (j0 + j < kn)
#pragma unroll
            for (int i = 0; i < 2; ++i) v[j][i] = __ldcg(part_row(k0 + j0 + j) + lane + 32 * i);
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        if (j0 + j >= kn) break;
        const float w = __shfl_sync(0xffffffffu, wl, j0 + j);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          acc[i].x += w * v[j][i].x;
          acc[i].y += w * v[j][i].y;
          acc[i].z += w * v[j][i].z;
          acc[i].w += w * v[j][i].w;
        }
      }
    }
  }
  const int s = row / g, h = kvh * g + row % g;
  __nv_bfloat16 *dst = out + ((int64_t(b) * s_q + s) * h_q + h) * kDV + half * (kDV / 2);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint2 u;
    u.x = pack_bf16x2(acc[i].x, acc[i].y);
    u.y = pack_bf16x2(acc[i].z, acc[i].w);
    *reinterpret_cast<uint2 *>(dst + 4 * (lane + 32 * i)) = u;
  }
  // sq_fold > 1 (sparse decode): "sequence" b is query token b % sq_fold of sequence b / sq_fold
  if (lane == 0 && half == 0)
    lse[(int64_t(b / sq_fold) * h_q + h) * (int64_t(s_q) * sq_fold) + int64_t(b % sq_fold) * s_q + s] = tot;
}

cudaError_t launch_combine(const int32_t *num_splits, int batch, int s_q, int h_q, int h_kv,
                           const float *lse_accum, const float *o_accum, __nv_bfloat16 *out,
                           float *lse, cudaStream_t stream, int sq_fold) {
  const int R = s_q * (h_q / h_kv);
  dim3 grid((R + kCombineWarps / 2 - 1) / (kCombineWarps / 2), batch, h_kv);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (R < 128 || int64_t(grid.x) * grid.y * grid.z <= int64_t(2) * 4 * sms)
    return launch_early(combine_kernel<8, 4>, grid, dim3(kCombineWarps * 32), 0, stream, num_splits, s_q, h_q, h_kv,
                        R, sq_fold, lse_accum, o_accum, out, lse);
  return launch_early(combine_kernel<5, 6>, grid, dim3(kCombineWarps * 32), 0, stream, num_splits, s_q, h_q, h_kv, R,
                      sq_fold, lse_accum, o_accum, out, lse);
}

// A CTA that waits on a barrier nothing completes, with the decode kernels' bounded
// wait; the wait gives up after timeout_ns, records the time-out and returns.
__global__ void watchdog_selftest_kernel(int *status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, status, timeout_ns);
  __syncthreads();
}

cudaError_t launch_watchdog_selftest(int *status, unsigned long long timeout_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace pagedmla
