// C ABI of libpagedmla.so (declared in include/pagedmla.h): argument checks, the TMA
// tensor map of the page pool, workspace carving and kernel launches.  Nothing here
// allocates device memory or synchronises, except mla_query_status.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "launch.h"
#include "pagedmla.h"

using namespace pagedmla;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char *what) {
  return fail(MLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr unsigned long long kWatchdogNs = 2000000000ull;  // 2 s per device-side wait
constexpr size_t kStatusBytes = 256;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout: [status 256 B][lse_accum fp32 splits*h_kv*R][o_accum fp32 ...*512].
struct WorkspaceLayout {
  size_t lse_off, o_off, total;
};

WorkspaceLayout workspace_layout(int batch, int R, int h_kv, int num_parts) {
  const size_t splits = size_t(batch) + size_t(num_parts);
  WorkspaceLayout w;
  w.lse_off = kStatusBytes;
  w.o_off = align256(w.lse_off + splits * h_kv * R * sizeof(float));
  w.total = w.o_off + splits * h_kv * R * kDV * sizeof(float);
  return w;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The kernels are built for sm_100a only; refuse other devices up front.
int check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(MLA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100 (B200) only",
                dev, major, minor);
  return MLA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Page pool [num_pages * 64 tokens][h_kv][576] bf16 as a 3-D map (columns, latent head,
// token); one box = 64 columns (128 bytes, 128-byte swizzle) x 1 head x box_tokens tokens
// (64 = a page for the 64-row kernels, 32 = half a page for the 16-row kernels).
int encode_kv_map(CUtensorMap *map, const void *k_cache, int64_t num_pages, int h_kv, int box_tokens) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(h_kv), cuuint64_t(num_pages) * kPage};
  cuuint64_t strides[2] = {cuuint64_t(kD) * 2, cuuint64_t(h_kv) * kD * 2};
  cuuint32_t box[3] = {64, 1, cuuint32_t(box_tokens)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(k_cache), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return MLA_OK;
}

// Query [batch][s_q][h_q][576] bf16 with element strides (sb, ss, sh) as a 4-D map
// (columns, head, s_q, batch); one box = 64 columns (128-byte swizzle) x box_heads heads x
// box_s positions, i.e. box_heads * box_s query rows of a tile in row order s*g + h.
int encode_q_map(CUtensorMap *map, const void *q, int batch, int s_q, int h_q, int box_heads, int box_s,
                 const int64_t strides[3]) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[4] = {cuuint64_t(kD), cuuint64_t(h_q), cuuint64_t(s_q), cuuint64_t(batch)};
  cuuint64_t gstr[3] = {cuuint64_t(strides[2]) * 2, cuuint64_t(strides[1]) * 2, cuuint64_t(strides[0]) * 2};
  for (int i = 0; i < 3; ++i)
    if (gstr[i] == 0) gstr[i] = 16;  // a dimension of extent 1 may carry stride 0
  cuuint32_t box[4] = {64, cuuint32_t(box_heads), cuuint32_t(box_s), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q), dims, gstr, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled (query) failed (%d)", int(r));
  return MLA_OK;
}

// FP8 latent cache codes [num_pages * 64 tokens][h_kv][576] bytes as a 3-D map (columns, latent
// head, token); one box = 128 columns (128 bytes, 128-byte swizzle) x 1 head x 64 tokens.  A box
// at column 512 reaches past column 575; TMA fills those columns with zeros.
int encode_k8_map(CUtensorMap *map, const void *k8, int64_t num_pages, int h_kv) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(h_kv), cuuint64_t(num_pages) * kPage};
  cuuint64_t strides[2] = {cuuint64_t(kD), cuuint64_t(h_kv) * kD};
  cuuint32_t box[3] = {128, 1, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(k8), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled (fp8 cache) failed (%d)", int(r));
  return MLA_OK;
}

// Token scales [h_kv][num_pages][64] fp32 as a 3-D map (slot, page, latent head); one box =
// the 64 scales of a page.
int encode_scale_map(CUtensorMap *map, const float *k_scale, int64_t num_pages, int h_kv) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[3] = {cuuint64_t(kPage), cuuint64_t(num_pages), cuuint64_t(h_kv)};
  cuuint64_t strides[2] = {cuuint64_t(kPage) * 4, cuuint64_t(num_pages) * kPage * 4};
  cuuint32_t box[3] = {64, 1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(k_scale), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled (fp8 scales) failed (%d)", int(r));
  return MLA_OK;
}

int check_common(int batch, int s_q, int h_q, int h_kv, int dv) {
  if (batch < 1 || s_q < 1 || h_q < 1 || h_kv < 1)
    return fail(MLA_ERR_ARG, "batch, s_q, h_q and h_kv must be >= 1");
  if (h_q % h_kv != 0) return fail(MLA_ERR_ARG, "h_q (%d) must be a multiple of h_kv (%d)", h_q, h_kv);
  if (dv != kDV) return fail(MLA_ERR_UNSUPPORTED, "dv must be %d (got %d)", kDV, dv);
  const long long R = (long long)s_q * (h_q / h_kv);
  if (R > (1 << 20)) return fail(MLA_ERR_ARG, "s_q * h_q / h_kv too large");
  return MLA_OK;
}

}  // namespace

namespace pagedmla {

int record_error(int code, const char *msg) { return fail(code, "%s", msg); }

cudaError_t set_smem_once(const void *kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void *, int>> done;  // (kernel, device)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (auto &d : done)
    if (d.first == kernel && d.second == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.emplace_back(kernel, dev);
  return e;
}

}  // namespace pagedmla

extern "C" {

const char *mla_last_error_string(void) { return g_last_error.c_str(); }

int mla_device_sm_count(int device, int *num_sms) {
  if (!num_sms) return fail(MLA_ERR_ARG, "num_sms is null");
  cudaError_t e = cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(MultiProcessorCount)");
  return MLA_OK;
}

int mla_num_parts(int num_sms, int rows_per_kv_head, int h_kv, int *num_parts) {
  if (!num_parts) return fail(MLA_ERR_ARG, "num_parts is null");
  if (num_sms < 1 || rows_per_kv_head < 1 || h_kv < 1)
    return fail(MLA_ERR_ARG, "num_sms, rows_per_kv_head and h_kv must be >= 1");
  const long long m_blocks = (rows_per_kv_head + MLA_ROWS_PER_SM - 1) / MLA_ROWS_PER_SM;
  const long long parts = num_sms / (h_kv * m_blocks);
  *num_parts = parts < 1 ? 1 : int(parts);
  return MLA_OK;
}

int mla_metadata_size(int batch, int rows_per_kv_head, int h_kv, int *num_parts) {
  if (!num_parts) return fail(MLA_ERR_ARG, "num_parts is null");
  if (batch < 1 || batch > MLA_MAX_BATCH)
    return fail(MLA_ERR_ARG, "batch must be in [1, %d] (got %d)", MLA_MAX_BATCH, batch);
  if (rows_per_kv_head < 1 || rows_per_kv_head > (1 << 20))
    return fail(MLA_ERR_ARG, "rows_per_kv_head must be in [1, 2^20]");
  if (h_kv < 1) return fail(MLA_ERR_ARG, "h_kv must be >= 1");
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int sms = 0;
  const int rc = mla_device_sm_count(device, &sms);
  if (rc != MLA_OK) return rc;
  return mla_num_parts(sms, rows_per_kv_head, h_kv, num_parts);
}

int mla_get_metadata(const int32_t *cache_seqlens, int batch, int rows_per_kv_head, int num_parts,
                     int32_t *tile_metadata, int32_t *num_splits, mla_stream_t stream) {
  if (!cache_seqlens || !tile_metadata || !num_splits)
    return fail(MLA_ERR_ARG, "null pointer argument");
  if (batch < 1 || batch > MLA_MAX_BATCH)
    return fail(MLA_ERR_ARG, "batch must be in [1, %d] (got %d)", MLA_MAX_BATCH, batch);
  if (rows_per_kv_head < 1 || rows_per_kv_head > (1 << 20))
    return fail(MLA_ERR_ARG, "rows_per_kv_head must be in [1, 2^20]");
  if (num_parts < 1) return fail(MLA_ERR_ARG, "num_parts must be >= 1");
  const int ovh = std::max(1, (rows_per_kv_head + MLA_SPLIT_OVERHEAD_ROWS - 1) / MLA_SPLIT_OVERHEAD_ROWS);
  cudaError_t e = launch_metadata(cache_seqlens, batch, ovh, num_parts, tile_metadata, num_splits,
                                  reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "metadata kernel launch");
  return MLA_OK;
}

int mla_get_metadata_csr(const int32_t *row_ptr, int n_lists, int rows_per_kv_head, int num_parts,
                         int32_t *tile_metadata, int32_t *num_splits, mla_stream_t stream) {
  if (!row_ptr || !tile_metadata || !num_splits) return fail(MLA_ERR_ARG, "null pointer argument");
  if (n_lists < 1 || n_lists > MLA_MAX_BATCH)
    return fail(MLA_ERR_ARG, "n_lists must be in [1, %d] (got %d)", MLA_MAX_BATCH, n_lists);
  if (rows_per_kv_head < 1 || rows_per_kv_head > (1 << 20))
    return fail(MLA_ERR_ARG, "rows_per_kv_head must be in [1, 2^20]");
  if (num_parts < 1) return fail(MLA_ERR_ARG, "num_parts must be >= 1");
  const int ovh = std::max(1, (rows_per_kv_head + MLA_SPLIT_OVERHEAD_ROWS - 1) / MLA_SPLIT_OVERHEAD_ROWS);
  cudaError_t e = launch_metadata(row_ptr, n_lists, ovh, num_parts, tile_metadata, num_splits,
                                  reinterpret_cast<cudaStream_t>(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "metadata kernel launch");
  return MLA_OK;
}

int mla_workspace_size(int batch, int s_q, int h_q, int h_kv, int num_parts, size_t *bytes) {
  if (!bytes) return fail(MLA_ERR_ARG, "bytes is null");
  int rc = check_common(batch, s_q, h_q, h_kv, kDV);
  if (rc) return rc;
  if (num_parts < 1) return fail(MLA_ERR_ARG, "num_parts must be >= 1");
  *bytes = workspace_layout(batch, s_q * (h_q / h_kv), h_kv, num_parts).total;
  return MLA_OK;
}

int mla_decode_paged(const void *q, const int64_t q_strides[3], int batch, int s_q, int h_q,
                     int d, const void *k_cache, int64_t num_pages, int page_size, int h_kv,
                     const int32_t *block_table, int64_t block_table_stride,
                     const int32_t *cache_seqlens, int dv, const int32_t *tile_metadata,
                     int num_parts, const int32_t *num_splits, float softmax_scale,
                     int causal, void *out, float *lse, void *workspace,
                     size_t workspace_bytes, unsigned flags, mla_stream_t stream) {
  if (!q || !q_strides || !k_cache || !block_table || !cache_seqlens || !tile_metadata ||
      !num_splits || !out || !lse)
    return fail(MLA_ERR_ARG, "null pointer argument");
  int rc = check_common(batch, s_q, h_q, h_kv, dv);
  if (rc) return rc;
  if (d != kD) return fail(MLA_ERR_UNSUPPORTED, "d must be %d (got %d)", kD, d);
  if (page_size != kPage) return fail(MLA_ERR_UNSUPPORTED, "page_size must be %d (got %d)", kPage, page_size);
  if (num_pages < 1 || num_pages > (int64_t(1) << 25))
    return fail(MLA_ERR_ARG, "num_pages must be in [1, 2^25]");
  if (block_table_stride < 1) return fail(MLA_ERR_ARG, "block_table_stride must be >= 1");
  if (num_parts < 1) return fail(MLA_ERR_ARG, "num_parts must be >= 1");
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(MLA_ERR_ARG, "softmax_scale must be positive and finite");
  if (flags & ~(MLA_FLAG_SKIP_COMBINE | MLA_FLAG_WARP_MMA | MLA_FLAG_TCGEN05 | MLA_FLAG_ONE_SM))
    return fail(MLA_ERR_ARG, "unknown flags 0x%x", flags);
  if (__builtin_popcount(flags & (MLA_FLAG_WARP_MMA | MLA_FLAG_TCGEN05 | MLA_FLAG_ONE_SM)) > 1)
    return fail(MLA_ERR_ARG, "MLA_FLAG_WARP_MMA, MLA_FLAG_TCGEN05 and MLA_FLAG_ONE_SM are exclusive");
  for (int i = 0; i < 3; ++i)
    if (q_strides[i] < 0 || q_strides[i] % 8 != 0)
      return fail(MLA_ERR_ARG, "q strides must be non-negative multiples of 8 elements");
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return fail(MLA_ERR_ARG, "q, k_cache and out must be 16-byte aligned, lse 4-byte aligned");
  rc = check_device();
  if (rc) return rc;

  const int g = h_q / h_kv, R = s_q * g;
  const WorkspaceLayout wl = workspace_layout(batch, R, h_kv, num_parts);
  if (!workspace) return fail(MLA_ERR_WORKSPACE, "workspace is null");
  if (!aligned(workspace, 256)) return fail(MLA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (workspace_bytes < wl.total)
    return fail(MLA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, wl.total);

  // Kernel choice.  Measured on B200: a 1-SM tcgen05 MMA costs at least a 128x128x16 tile
  // (an M = 64 one as much as M = 128), so up to 16 query rows the 16-row warp-MMA tiles do
  // the same work in fewer tensor cycles; a CTA-pair MMA with 64 rows per SM and N = 256
  // runs at the full rate, so whole 128-row blocks go to the pair kernel; other shapes
  // above 16 rows to the 1-SM 64-row tcgen05 kernel.
  enum { kMma16, kMma64, kTc, kWide, kPair } kind;
  const bool pair_ok = pair_supported(R, g);
  if (flags & MLA_FLAG_WARP_MMA) {
    kind = R <= 16 ? kMma16 : kMma64;
  } else if (flags & MLA_FLAG_TCGEN05) {
    kind = R <= 16 ? kTc : (pair_ok ? kPair : kWide);
  } else if (flags & MLA_FLAG_ONE_SM) {
    kind = R <= 16 ? kMma16 : kWide;
  } else {
    kind = R <= 16 ? kMma16 : (pair_ok ? kPair : (wide_supported(R, g) ? kWide : kMma64));
  }
  CUtensorMap map;
  rc = encode_kv_map(&map, k_cache, num_pages, h_kv, kind == kMma64 || kind == kWide || kind == kPair ? kPage : 32);
  if (rc) return rc;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.q_sb = q_strides[0];
  p.q_ss = q_strides[1];
  p.q_sh = q_strides[2];
  p.batch = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.g = g;
  p.R = R;
  p.block_table = block_table;
  p.bt_stride = block_table_stride;
  p.kv_base = static_cast<const uint8_t *>(k_cache);
  p.kv_token_bytes = int64_t(h_kv) * kD * 2;
  p.seqlens = cache_seqlens;
  p.tile_md = tile_metadata;
  p.num_parts = num_parts;
  p.num_splits = num_splits;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.lse = lse;
  p.lse_accum = reinterpret_cast<float *>(ws + wl.lse_off);
  p.o_accum = reinterpret_cast<float *>(ws + wl.o_off);
  p.status = reinterpret_cast<int *>(ws);
  p.watchdog_ns = kWatchdogNs;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (kind == kMma64) {
    e = launch_decode_mma(map, p, st);
  } else if (kind == kWide) {
    e = launch_decode_wide(map, p, st);  // reads the query rows itself (any g)
  } else if (kind == kPair) {
    // each CTA's 64 query rows as one TMA box: 64 heads of one position (g a multiple of
    // 64), or all g heads of 64 / g positions (g a divisor of 64)
    const int box_heads = g % 64 == 0 ? 64 : g, box_s = g % 64 == 0 ? 1 : 64 / g;
    CUtensorMap qmap;
    rc = encode_q_map(&qmap, q, batch, s_q, h_q, box_heads, box_s, q_strides);
    if (rc) return rc;
    e = launch_decode_pair(map, qmap, p, box_heads, st);
  } else {
    CUtensorMap qmap;
    rc = encode_q_map(&qmap, q, batch, s_q, h_q, g, s_q, q_strides);
    if (rc) return rc;
    e = kind == kTc ? launch_decode_tc_narrow(map, qmap, p, st) : launch_decode_mma16(map, qmap, p, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  if (!(flags & MLA_FLAG_SKIP_COMBINE)) {
    e = launch_combine(num_splits, batch, s_q, h_q, h_kv, p.lse_accum, p.o_accum, p.out, lse, st);
    if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
  }
  return MLA_OK;
}

int mla_decode_paged_fp8(const void *q, const int64_t q_strides[3], int batch, int s_q, int h_q, int d,
                         const void *k8, const float *k_scale, int64_t num_pages, int page_size, int h_kv,
                         const int32_t *block_table, int64_t block_table_stride, const int32_t *cache_seqlens,
                         int dv, const int32_t *tile_metadata, int num_parts, const int32_t *num_splits,
                         float softmax_scale, int causal, void *out, float *lse, void *workspace,
                         size_t workspace_bytes, unsigned flags, mla_stream_t stream) {
  if (!q || !q_strides || !k8 || !k_scale || !block_table || !cache_seqlens || !tile_metadata || !num_splits ||
      !out || !lse)
    return fail(MLA_ERR_ARG, "null pointer argument");
  int rc = check_common(batch, s_q, h_q, h_kv, dv);
  if (rc) return rc;
  if (d != kD) return fail(MLA_ERR_UNSUPPORTED, "d must be %d (got %d)", kD, d);
  if (page_size != kPage) return fail(MLA_ERR_UNSUPPORTED, "page_size must be %d (got %d)", kPage, page_size);
  const int g = h_q / h_kv, R = s_q * g;
  if (R > 16)
    return fail(MLA_ERR_UNSUPPORTED,
                "the FP8 cache is decoded by the 16-row kernel: s_q * h_q / h_kv must be <= 16 (got %d)", R);
  if (num_pages < 1 || num_pages > (int64_t(1) << 25))
    return fail(MLA_ERR_ARG, "num_pages must be in [1, 2^25]");
  if (block_table_stride < 1) return fail(MLA_ERR_ARG, "block_table_stride must be >= 1");
  if (num_parts < 1) return fail(MLA_ERR_ARG, "num_parts must be >= 1");
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(MLA_ERR_ARG, "softmax_scale must be positive and finite");
  if (flags & ~MLA_FLAG_SKIP_COMBINE) return fail(MLA_ERR_ARG, "unknown flags 0x%x", flags);
  for (int i = 0; i < 3; ++i)
    if (q_strides[i] < 0 || q_strides[i] % 8 != 0)
      return fail(MLA_ERR_ARG, "q strides must be non-negative multiples of 8 elements");
  if (!aligned(q, 16) || !aligned(k8, 16) || !aligned(k_scale, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return fail(MLA_ERR_ARG, "q, k8, k_scale and out must be 16-byte aligned, lse 4-byte aligned");
  rc = check_device();
  if (rc) return rc;
  const WorkspaceLayout wl = workspace_layout(batch, R, h_kv, num_parts);
  if (!workspace) return fail(MLA_ERR_WORKSPACE, "workspace is null");
  if (!aligned(workspace, 256)) return fail(MLA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (workspace_bytes < wl.total)
    return fail(MLA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, wl.total);

  CUtensorMap k8_map, scale_map, qmap;
  rc = encode_k8_map(&k8_map, k8, num_pages, h_kv);
  if (rc) return rc;
  rc = encode_scale_map(&scale_map, k_scale, num_pages, h_kv);
  if (rc) return rc;
  rc = encode_q_map(&qmap, q, batch, s_q, h_q, g, s_q, q_strides);
  if (rc) return rc;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.q_sb = q_strides[0];
  p.q_ss = q_strides[1];
  p.q_sh = q_strides[2];
  p.batch = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.g = g;
  p.R = R;
  p.block_table = block_table;
  p.bt_stride = block_table_stride;
  p.kv_base = static_cast<const uint8_t *>(k8);
  p.kv_token_bytes = int64_t(h_kv) * kD;
  p.seqlens = cache_seqlens;
  p.tile_md = tile_metadata;
  p.num_parts = num_parts;
  p.num_splits = num_splits;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.lse = lse;
  p.lse_accum = reinterpret_cast<float *>(ws + wl.lse_off);
  p.o_accum = reinterpret_cast<float *>(ws + wl.o_off);
  p.status = reinterpret_cast<int *>(ws);
  p.watchdog_ns = kWatchdogNs;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_decode_fp8(k8_map, scale_map, qmap, p, st);
  if (e != cudaSuccess) return cuda_fail(e, "fp8 decode kernel launch");
  if (!(flags & MLA_FLAG_SKIP_COMBINE)) {
    e = launch_combine(num_splits, batch, s_q, h_q, h_kv, p.lse_accum, p.o_accum, p.out, lse, st);
    if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
  }
  return MLA_OK;
}

int mla_decode_sparse(const void *q, const int64_t q_strides[3], int batch, int s_q, int h_q, int d,
                      const void *k_cache, int64_t num_pages, int page_size, int h_kv, const int32_t *block_table,
                      int64_t block_table_stride, const int32_t *cache_seqlens, const int32_t *row_ptr,
                      const int32_t *col_idx, int dv, const int32_t *tile_metadata, int num_parts,
                      const int32_t *num_splits, float softmax_scale, int causal, void *out, float *lse,
                      void *workspace, size_t workspace_bytes, unsigned flags, mla_stream_t stream) {
  if (!q || !q_strides || !k_cache || !block_table || !cache_seqlens || !row_ptr || !col_idx || !tile_metadata ||
      !num_splits || !out || !lse)
    return fail(MLA_ERR_ARG, "null pointer argument");
  int rc = check_common(batch, s_q, h_q, h_kv, dv);
  if (rc) return rc;
  if (d != kD) return fail(MLA_ERR_UNSUPPORTED, "d must be %d (got %d)", kD, d);
  if (page_size != kPage) return fail(MLA_ERR_UNSUPPORTED, "page_size must be %d (got %d)", kPage, page_size);
  const int g = h_q / h_kv;
  if (g > 16)
    return fail(MLA_ERR_UNSUPPORTED, "the sparse decode takes up to 16 query heads per latent head (got %d)", g);
  if (int64_t(batch) * s_q > MLA_MAX_BATCH)
    return fail(MLA_ERR_ARG, "batch * s_q must be <= %d (got %lld)", MLA_MAX_BATCH, (long long)batch * s_q);
  if (num_pages < 1 || num_pages > (int64_t(1) << 25))
    return fail(MLA_ERR_ARG, "num_pages must be in [1, 2^25]");
  if (block_table_stride < 1) return fail(MLA_ERR_ARG, "block_table_stride must be >= 1");
  if (num_parts < 1) return fail(MLA_ERR_ARG, "num_parts must be >= 1");
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(MLA_ERR_ARG, "softmax_scale must be positive and finite");
  if (flags & ~MLA_FLAG_SKIP_COMBINE) return fail(MLA_ERR_ARG, "unknown flags 0x%x", flags);
  for (int i = 0; i < 3; ++i)
    if (q_strides[i] < 0 || q_strides[i] % 8 != 0)
      return fail(MLA_ERR_ARG, "q strides must be non-negative multiples of 8 elements");
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return fail(MLA_ERR_ARG, "q, k_cache and out must be 16-byte aligned, lse 4-byte aligned");
  rc = check_device();
  if (rc) return rc;
  const int n_tok = batch * s_q;
  const WorkspaceLayout wl = workspace_layout(n_tok, g, h_kv, num_parts);
  if (!workspace) return fail(MLA_ERR_WORKSPACE, "workspace is null");
  if (!aligned(workspace, 256)) return fail(MLA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (workspace_bytes < wl.total)
    return fail(MLA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, wl.total);

  // one query token per tile: all g heads of position s of sequence b
  CUtensorMap qmap;
  rc = encode_q_map(&qmap, q, batch, s_q, h_q, g, 1, q_strides);
  if (rc) return rc;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.q_sb = q_strides[0];
  p.q_ss = q_strides[1];
  p.q_sh = q_strides[2];
  p.batch = n_tok;  // query tokens are the tile "sequences"
  p.s_q = 1;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.g = g;
  p.R = g;
  p.block_table = block_table;
  p.bt_stride = block_table_stride;
  p.kv_base = static_cast<const uint8_t *>(k_cache);
  p.kv_token_bytes = int64_t(h_kv) * kD * 2;
  p.seqlens = cache_seqlens;
  p.tile_md = tile_metadata;
  p.num_parts = num_parts;
  p.num_splits = num_splits;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.lse = lse;
  p.lse_accum = reinterpret_cast<float *>(ws + wl.lse_off);
  p.o_accum = reinterpret_cast<float *>(ws + wl.o_off);
  p.status = reinterpret_cast<int *>(ws);
  p.watchdog_ns = kWatchdogNs;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.sq_fold = s_q;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_decode_sparse16(qmap, p, st);
  if (e != cudaSuccess) return cuda_fail(e, "sparse decode kernel launch");
  if (!(flags & MLA_FLAG_SKIP_COMBINE)) {
    e = launch_combine(num_splits, n_tok, 1, h_q, h_kv, p.lse_accum, p.o_accum, p.out, lse, st, s_q);
    if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
  }
  return MLA_OK;
}

int mla_combine(const int32_t *num_splits, int batch, int s_q, int h_q, int h_kv, int dv,
                int num_parts, const void *workspace, size_t workspace_bytes, void *out,
                float *lse, mla_stream_t stream) {
  if (!num_splits || !out || !lse) return fail(MLA_ERR_ARG, "null pointer argument");
  int rc = check_common(batch, s_q, h_q, h_kv, dv);
  if (rc) return rc;
  if (num_parts < 1) return fail(MLA_ERR_ARG, "num_parts must be >= 1");
  if (!aligned(out, 16) || !aligned(lse, 4)) return fail(MLA_ERR_ARG, "out must be 16-byte aligned");
  const int R = s_q * (h_q / h_kv);
  const WorkspaceLayout wl = workspace_layout(batch, R, h_kv, num_parts);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < wl.total)
    return fail(MLA_ERR_WORKSPACE, "workspace missing, misaligned or smaller than %zu bytes", wl.total);
  const uint8_t *ws = static_cast<const uint8_t *>(workspace);
  cudaError_t e = launch_combine(num_splits, batch, s_q, h_q, h_kv,
                                 reinterpret_cast<const float *>(ws + wl.lse_off),
                                 reinterpret_cast<const float *>(ws + wl.o_off),
                                 static_cast<__nv_bfloat16 *>(out), lse,
                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
  return MLA_OK;
}

int mla_merge_partials(const void *o_parts, const float *lse_parts, int n_parts, int batch, int s_q, int h_q,
                       int dv, void *out, float *lse, mla_stream_t stream) {
  if (!o_parts || !lse_parts || !out || !lse) return fail(MLA_ERR_ARG, "null pointer argument");
  if (n_parts < 1 || batch < 1 || s_q < 1 || h_q < 1)
    return fail(MLA_ERR_ARG, "n_parts, batch, s_q and h_q must be >= 1");
  if (dv != kDV) return fail(MLA_ERR_UNSUPPORTED, "dv must be %d (got %d)", kDV, dv);
  if (int64_t(batch) * s_q * h_q > (int64_t(1) << 31))
    return fail(MLA_ERR_ARG, "batch * s_q * h_q must be <= 2^31");
  if (!aligned(o_parts, 16) || !aligned(out, 16) || !aligned(lse_parts, 4) || !aligned(lse, 4))
    return fail(MLA_ERR_ARG, "o_parts and out must be 16-byte aligned, lse_parts and lse 4-byte aligned");
  cudaError_t e = launch_merge(static_cast<const __nv_bfloat16 *>(o_parts), lse_parts, n_parts, batch, s_q, h_q,
                               static_cast<__nv_bfloat16 *>(out), lse, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge kernel launch");
  return MLA_OK;
}

int mla_absorb_query(const void *q_nope, const int64_t nope_strides[2], const void *q_rope,
                     const int64_t rope_strides[2], const void *w_uk, int tokens, int heads, void *q_out,
                     mla_stream_t stream) {
  if (!q_nope || !nope_strides || !q_rope || !rope_strides || !w_uk || !q_out)
    return fail(MLA_ERR_ARG, "null pointer argument");
  if (tokens < 1 || heads < 1) return fail(MLA_ERR_ARG, "tokens and heads must be >= 1");
  if (int64_t(tokens + 63) / 64 > 65535 || heads > 65535) return fail(MLA_ERR_ARG, "too many tokens or heads");
  for (int i = 0; i < 2; ++i)
    if (nope_strides[i] < 0 || nope_strides[i] % 8 || rope_strides[i] < 0 || rope_strides[i] % 8)
      return fail(MLA_ERR_ARG, "strides must be non-negative multiples of 8 elements");
  if (!aligned(q_nope, 16) || !aligned(q_rope, 16) || !aligned(w_uk, 16) || !aligned(q_out, 16))
    return fail(MLA_ERR_ARG, "q_nope, q_rope, w_uk and q_out must be 16-byte aligned");
  cudaError_t e = launch_absorb_q(static_cast<const __nv_bfloat16 *>(q_nope), nope_strides[0], nope_strides[1],
                                  static_cast<const __nv_bfloat16 *>(q_rope), rope_strides[0], rope_strides[1],
                                  static_cast<const __nv_bfloat16 *>(w_uk), static_cast<__nv_bfloat16 *>(q_out), tokens,
                                  heads, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "query absorption launch");
  return MLA_OK;
}

int mla_absorb_output(const void *o_latent, const int64_t latent_strides[2], const void *w_uv, int tokens, int heads,
                      void *out, mla_stream_t stream) {
  if (!o_latent || !latent_strides || !w_uv || !out) return fail(MLA_ERR_ARG, "null pointer argument");
  if (tokens < 1 || heads < 1) return fail(MLA_ERR_ARG, "tokens and heads must be >= 1");
  if (int64_t(tokens + 63) / 64 > 65535 || heads > 65535) return fail(MLA_ERR_ARG, "too many tokens or heads");
  for (int i = 0; i < 2; ++i)
    if (latent_strides[i] < 0 || latent_strides[i] % 8)
      return fail(MLA_ERR_ARG, "strides must be non-negative multiples of 8 elements");
  if (!aligned(o_latent, 16) || !aligned(w_uv, 16) || !aligned(out, 4))
    return fail(MLA_ERR_ARG, "o_latent and w_uv must be 16-byte aligned, out 4-byte aligned");
  cudaError_t e = launch_absorb_out(static_cast<const __nv_bfloat16 *>(o_latent), latent_strides[0], latent_strides[1],
                                    static_cast<const __nv_bfloat16 *>(w_uv), static_cast<__nv_bfloat16 *>(out), tokens,
                                    heads, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "output absorption launch");
  return MLA_OK;
}

int mla_query_status(void *workspace, mla_stream_t stream) {
  if (!workspace) return fail(MLA_ERR_ARG, "workspace is null");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int status = 0;
  e = cudaMemcpy(&status, workspace, sizeof status, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the workspace status");
  if (status != 0) {
    e = cudaMemset(workspace, 0, sizeof status);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace status");
    if (status & kStatusTimeout)
      return fail(MLA_ERR_TIMEOUT, "a device-side wait timed out; results of that call are invalid");
  }
  return MLA_OK;
}

int mla_watchdog_selftest(void *workspace, uint64_t timeout_ns, mla_stream_t stream) {
  if (!workspace || !aligned(workspace, 256)) return fail(MLA_ERR_ARG, "workspace null or misaligned");
  if (timeout_ns == 0 || timeout_ns > 10ull * 1000000000ull)
    return fail(MLA_ERR_ARG, "timeout_ns must be in (0, 10 s]");
  cudaError_t e = launch_watchdog_selftest(static_cast<int *>(workspace), timeout_ns,
                                           reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "watchdog self-test launch");
  return MLA_OK;
}

}  // extern "C"
