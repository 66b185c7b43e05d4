// Decode for callers that cannot allocate device memory.
//
// Some callers of this library may not call cudaMalloc or any other allocator while they
// run: code executing inside another framework's memory budget, an inference server that
// reserves all device memory at start-up, or a real-time loop where an allocation could
// block or fail.  mla_decode_paged_static serves them: it is mla_decode_paged with the
// split-KV scratch (status block, fp32 partial outputs and LSEs) taken from one fixed,
// statically sized device array that the library module itself carries, instead of a
// caller-provided workspace.  The caller still provides every input and output buffer.
//
// In host code the array's name is only a host-side stand-in, never a device address: its
// device address is looked up with cudaGetSymbolAddress on every call, with the caller's
// device current (a cached address could outlive a reset or re-created primary context,
// which reloads the module and may move the array).  mla_query_status_static reads the
// array's status block, so a static call whose device-side waits gave up is reported.
#include <cuda_runtime.h>

#include <cstdio>

#include "launch.h"
#include "pagedmla.h"

namespace {

constexpr size_t kStaticScratchBytes = MLA_STATIC_SCRATCH_BYTES;  // held on every device that loads the library

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device (host-only lookup).
int static_scratch(void **out) {
  void *ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
  if (e != cudaSuccess || ptr == nullptr)
    return pagedmla::record_error(MLA_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
  *out = ptr;
  return MLA_OK;
}

}  // namespace

extern "C" MLA_API int mla_decode_paged_static(
    const void *q, const int64_t q_strides[3], int batch, int s_q, int h_q, int d, const void *k_cache,
    int64_t num_pages, int page_size, int h_kv, const int32_t *block_table, int64_t block_table_stride,
    const int32_t *cache_seqlens, int dv, const int32_t *tile_metadata, int num_parts,
    const int32_t *num_splits, float softmax_scale, int causal, void *out, float *lse, unsigned flags,
    mla_stream_t stream) {
  // The split partials stay in the library's private array, which the caller cannot name,
  // so leaving them unmerged for a later mla_combine is refused.
  if (flags & MLA_FLAG_SKIP_COMBINE)
    return pagedmla::record_error(MLA_ERR_ARG,
                                  "MLA_FLAG_SKIP_COMBINE is not accepted by mla_decode_paged_static: its split "
                                  "partials live in the library's static array, which mla_combine cannot be given");
  size_t need = 0;
  int rc = mla_workspace_size(batch, s_q, h_q, h_kv, num_parts, &need);
  if (rc) return rc;
  if (need > kStaticScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "this shape needs %zu bytes of split scratch; the static scratch holds %zu bytes "
             "(use mla_decode_paged with a caller-provided workspace)",
             need, kStaticScratchBytes);
    return pagedmla::record_error(MLA_ERR_WORKSPACE, msg);
  }
  void *ws = nullptr;
  rc = static_scratch(&ws);
  if (rc) return rc;
  // The status block must start at zero (a set word would report an earlier call's
  // time-out); the partial outputs are always written before they are read.
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return pagedmla::record_error(MLA_ERR_CUDA, "clearing the static scratch status block failed");
  return mla_decode_paged(q, q_strides, batch, s_q, h_q, d, k_cache, num_pages, page_size, h_kv, block_table,
                          block_table_stride, cache_seqlens, dv, tile_metadata, num_parts, num_splits,
                          softmax_scale, causal, out, lse, ws, kStaticScratchBytes, flags, stream);
}

extern "C" MLA_API int mla_query_status_static(mla_stream_t stream) {
  void *ws = nullptr;
  const int rc = static_scratch(&ws);
  if (rc) return rc;
  return mla_query_status(ws, stream);
}
