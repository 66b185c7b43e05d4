// Internal launch entry points of the kernels behind the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace pagedmla {

// Records an error for mla_last_error_string() on this thread and returns `code`.
int record_error(int code, const char *msg);

// Raises a kernel's dynamic shared-memory limit once per (kernel, device), so that
// launches inside CUDA-graph capture make no attribute calls.
cudaError_t set_smem_once(const void *kernel, int bytes);

// lengths_are_offsets: seqlens holds batch + 1 offsets (a CSR row_ptr) and length b is
// seqlens[b + 1] - seqlens[b]
cudaError_t launch_metadata(const int32_t *seqlens, int batch, int ovh, int num_parts, int32_t *tile_md,
                            int32_t *num_splits, cudaStream_t stream, bool lengths_are_offsets = false);
cudaError_t launch_decode_mma(const CUtensorMap &map, const DecodeParams &p, cudaStream_t stream);
cudaError_t launch_decode_mma16(const CUtensorMap &kv_map, const CUtensorMap &q_map, const DecodeParams &p,
                                cudaStream_t stream);
// Token-level sparse decode, up to 16 query heads per latent head and query token (p.row_ptr,
// p.col_idx, p.sq_fold set; p.batch / p.s_q / p.R describe query tokens as sequences).
cudaError_t launch_decode_sparse16(const CUtensorMap &q_map, const DecodeParams &p, cudaStream_t stream);
// The 64-row tcgen05 kernel takes more than 16 rows per latent head.
bool wide_supported(int R, int g);
cudaError_t launch_decode_wide(const CUtensorMap &kv_map, const DecodeParams &p, cudaStream_t stream);
// The CTA-pair tcgen05 kernel takes whole 128-row blocks whose 64-row halves are (position,
// head) rectangles: g a multiple or a divisor of 64.
bool pair_supported(int R, int g);
cudaError_t launch_decode_pair(const CUtensorMap &kv_map, const CUtensorMap &q_map, const DecodeParams &p,
                               int q_box_heads, cudaStream_t stream);
cudaError_t launch_decode_tc_narrow(const CUtensorMap &kv_map, const CUtensorMap &q_map,
                                    const DecodeParams &p, cudaStream_t stream);
cudaError_t launch_decode_fp8(const CUtensorMap &k8_map, const CUtensorMap &scale_map, const CUtensorMap &q_map,
                              const DecodeParams &p, cudaStream_t stream);
cudaError_t launch_combine(const int32_t *num_splits, int batch, int s_q, int h_q, int h_kv,
                           const float *lse_accum, const float *o_accum, __nv_bfloat16 *out,
                           float *lse, cudaStream_t stream, int sq_fold = 1);
cudaError_t launch_merge(const __nv_bfloat16 *o_parts, const float *lse_parts, int n_parts, int batch, int s_q,
                         int h_q, __nv_bfloat16 *out, float *lse, cudaStream_t stream);
cudaError_t launch_absorb_q(const __nv_bfloat16 *q_nope, int64_t n_row, int64_t n_head, const __nv_bfloat16 *q_rope,
                            int64_t r_row, int64_t r_head, const __nv_bfloat16 *w_uk, __nv_bfloat16 *q_out, int T,
                            int H, cudaStream_t stream);
cudaError_t launch_absorb_out(const __nv_bfloat16 *o_lat, int64_t l_row, int64_t l_head, const __nv_bfloat16 *w_uv,
                              __nv_bfloat16 *out, int T, int H, cudaStream_t stream);
cudaError_t launch_watchdog_selftest(int *status, unsigned long long timeout_ns,
                                     cudaStream_t stream);

}  // namespace pagedmla
