// Shared device helpers for the paged MLA decode kernels (sm_100a only).
//
// Hand-written PTX wrappers: shared-memory mbarriers with bounded waits, TMA tensor
// loads, ldmatrix / warp MMA, named barriers, and the kernel parameter block.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pagedmla {

constexpr int kPage = 64;          // tokens per cache page
constexpr int kD = 576;            // latent row width (512 latent + 64 rope)
constexpr int kDV = 512;           // value width
constexpr int kColBlocks = kD / 64;               // 64-column (128-byte) blocks per row
constexpr int kPageBlockBytes = kPage * 128;      // one 64x64 bf16 block: 8 KB
constexpr int kPageBytes = kColBlocks * kPageBlockBytes;  // 73,728 B per page and head

// Status words at the start of the workspace.
constexpr int kStatusTimeout = 1;

struct DecodeParams {
  const __nv_bfloat16 *q;
  int64_t q_sb, q_ss, q_sh;        // element strides of q's batch, s_q, head dims
  int batch, s_q, h_q, h_kv, g, R; // g = h_q / h_kv, R = s_q * g rows per latent head
  const int32_t *block_table;
  int64_t bt_stride;
  const int32_t *seqlens;
  const int32_t *tile_md;
  int num_parts;
  const int32_t *num_splits;
  float scale_log2;                // softmax_scale * log2(e)
  int causal;
  __nv_bfloat16 *out;              // [batch, s_q, h_q, 512]
  float *lse;                      // [batch, h_q, s_q]
  float *lse_accum;                // [splits, h_kv, R]
  float *o_accum;                  // [splits, h_kv, R, 512]
  int *status;                     // workspace status block
  unsigned long long watchdog_ns;  // limit of every device-side wait
};

// ------------------------------------------------------------------------------------
// Timers and the watchdog.
// ------------------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report_timeout(int *status) {
  if (status) atomicOr(status, kStatusTimeout);
}

// ------------------------------------------------------------------------------------
// mbarriers (shared::cta).
// ------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity has completed.  Gives up after
// `limit_ns` (checked every 256 polls) or as soon as *abort is set by another thread;
// on giving up it records the time-out and raises *abort.  Returns true on success.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          int *status, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort) return false;
      if (global_ns() - t0 > limit_ns) {
        *abort = 1;
        report_timeout(status);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------------------------
// TMA: 3-D tiled tensor load into shared memory, completing on an mbarrier.
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------------------------
// Named barriers.
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------------------------
// 128-byte swizzle (the pattern TMA's SWIZZLE_128B writes): within each 1024-byte group
// of eight 128-byte rows, 16-byte chunk c of row r sits at chunk position c ^ (r & 7).
// ------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ------------------------------------------------------------------------------------
// Warp-level matrix ops (ldmatrix + mma.sync m16n8k16 bf16 -> fp32).
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ------------------------------------------------------------------------------------
// Scheduler tile decoding, shared by every decode kernel.
// ------------------------------------------------------------------------------------
struct PartCursor {
  int bi, bt, ei, et, bord;
};

__device__ __forceinline__ PartCursor load_part(const int32_t *tile_md, int part) {
  const int32_t *m = tile_md + part * 8;
  return PartCursor{m[0], m[1], m[2], m[3], m[4]};
}

__device__ __forceinline__ bool part_has(const PartCursor &c, int seq) {
  return seq < c.ei || (seq == c.ei && c.et > 0);
}

}  // namespace pagedmla
