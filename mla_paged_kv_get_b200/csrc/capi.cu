// capi.cu — the C ABI (include/mla_b200.h): argument checks, TMA tensor maps,
// kernel launches.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "../../include/mla_b200.h"
#include "decode.cuh"

namespace mla {
int metadata_max_batch();
int metadata_max_parts();
}

namespace {

constexpr unsigned long long kDefaultTimeoutNs = 4000000000ull;   // 4 s per device-side wait

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct DeviceInfo {
  int sms = -1;
  int major = 0;
  int minor = 0;
};

int device_info(DeviceInfo* out) {
  static DeviceInfo cache[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev].sms < 0) {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return MLA_ERR_CUDA;
    cache[dev] = d;
  }
  *out = cache[dev];
  return MLA_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int rows_per_block(int rows_per_kv) {
  if (rows_per_kv <= 16) return 16;
  if (rows_per_kv <= 32) return 32;
  return 64;
}

}  // namespace

extern "C" {

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported shape or device";
    case MLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_TIMEOUT: return "device-side wait timed out";
    case MLA_ERR_BAD_INPUT: return "device-side input check failed";
    default: return "unknown status";
  }
}

int mla_device_sm_count(void) {
  DeviceInfo d;
  const int st = device_info(&d);
  return st == MLA_OK ? d.sms : st;
}

int mla_rows_per_block(int rows_per_kv) {
  if (rows_per_kv < 1) return MLA_ERR_INVALID_ARG;
  return rows_per_block(rows_per_kv);
}

int mla_num_parts(int rows_per_kv, int h_kv, int num_sms) {
  if (rows_per_kv < 1 || h_kv < 1 || num_sms < 1) return MLA_ERR_INVALID_ARG;
  const int n = rows_per_block(rows_per_kv);
  const int t = (rows_per_kv + n - 1) / n;
  const int g = num_sms / (h_kv * t);
  return g > 1 ? g : 1;
}

int mla_get_metadata(const int32_t* cache_seqlens_d, int batch, int rows_per_kv, int h_kv, int num_sms,
                     int32_t* tile_md_d, int32_t* num_splits_d, int* num_parts_out, void* stream) {
  if (cache_seqlens_d == nullptr || tile_md_d == nullptr || num_splits_d == nullptr) return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > mla::metadata_max_batch() || rows_per_kv < 1 || h_kv < 1) return MLA_ERR_INVALID_ARG;
  if (num_sms <= 0) {
    DeviceInfo d;
    const int st = device_info(&d);
    if (st != MLA_OK) return st;
    num_sms = d.sms;
  }
  const int g = mla_num_parts(rows_per_kv, h_kv, num_sms);
  if (g < 1 || g > mla::metadata_max_parts()) return MLA_ERR_INVALID_ARG;
  if (mla::launch_metadata(cache_seqlens_d, batch, g, tile_md_d, num_splits_d,
                           static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (num_parts_out != nullptr) *num_parts_out = g;
  return MLA_OK;
}

size_t mla_workspace_bytes(int batch, int rows_per_kv, int h_kv, int dv, int num_parts) {
  if (batch < 1 || rows_per_kv < 1 || h_kv < 1 || dv < 1 || num_parts < 1) return 0;
  const size_t pieces = static_cast<size_t>(batch) + static_cast<size_t>(num_parts);
  const size_t bytes = pieces * h_kv * rows_per_kv * (static_cast<size_t>(dv) + 1) * sizeof(float);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

int mla_decode_paged_typed(int dtype, const void* q_d, const void* k_cache_d, int num_pages,
                           const int32_t* block_table_d, int max_pages_per_seq, const int32_t* cache_seqlens_d,
                           int batch, int s_q, int h_q, int h_kv, int d, int dv, const int32_t* tile_md_d,
                           const int32_t* num_splits_d, int num_parts, int causal, float softmax_scale,
                           void* workspace_d, size_t workspace_bytes, void* out_d, float* lse_d, int32_t* status_d,
                           int debug_flags, unsigned long long timeout_ns, void* stream) {
  if (dtype != MLA_DTYPE_BF16 && dtype != MLA_DTYPE_FP16) return MLA_ERR_INVALID_ARG;
  const CUtensorMapDataType tmap_type =
      dtype == MLA_DTYPE_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (q_d == nullptr || k_cache_d == nullptr || block_table_d == nullptr || cache_seqlens_d == nullptr ||
      tile_md_d == nullptr || num_splits_d == nullptr || out_d == nullptr || lse_d == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (d != MLA_HEAD_DIM || dv != MLA_VALUE_DIM) return MLA_ERR_UNSUPPORTED;
  if (batch < 1 || batch > mla::metadata_max_batch() || s_q < 1 || h_q < 1 || h_kv < 1 || h_q % h_kv != 0 || num_pages < 1 ||
      num_pages > (1 << 24) || max_pages_per_seq < 1 || max_pages_per_seq > (1 << 24) || num_parts < 1 ||
      num_parts > 65535)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(q_d, 16) || !aligned(k_cache_d, 16) || !aligned(out_d, 16) || !aligned(lse_d, 4) ||
      !aligned(block_table_d, 4) || !aligned(cache_seqlens_d, 4) || !aligned(tile_md_d, 4) ||
      !aligned(num_splits_d, 4))
    return MLA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return MLA_ERR_INVALID_ARG;
  const long long rows_ll = static_cast<long long>(s_q) * h_q / h_kv;
  if (rows_ll > 4096 || static_cast<long long>(batch) * s_q > (1ll << 30)) return MLA_ERR_INVALID_ARG;
  const int R = static_cast<int>(rows_ll);
  const int hg = h_q / h_kv;
  const int n = rows_per_block(R);
  if (!(hg % n == 0 || n % hg == 0)) return MLA_ERR_UNSUPPORTED;
  const size_t need = mla_workspace_bytes(batch, R, h_kv, dv, num_parts);
  if (workspace_d == nullptr || workspace_bytes < need || !aligned(workspace_d, 256)) return MLA_ERR_WORKSPACE;

  DeviceInfo dev;
  const int st = device_info(&dev);
  if (st != MLA_OK) return st;
  if (dev.major != 10) return MLA_ERR_UNSUPPORTED;
  EncodeTiledFn encode = encode_fn();
  if (encode == nullptr) return MLA_ERR_CUDA;

  const cuuint64_t tokens = static_cast<cuuint64_t>(num_pages) * MLA_PAGE_SIZE;
  const cuuint64_t token_bytes = static_cast<cuuint64_t>(h_kv) * MLA_HEAD_DIM * 2;   // one token, all heads
  // Cache pages as (64 cols, tokens, 9 chunks, heads): a box of `chunks` 64-column chunks of 64 tokens
  // lands in shared memory as [chunk][token][64 cols], the 128-byte swizzled K-major tile layout.
  auto page_map = [&](CUtensorMap* m, int chunks) -> bool {
    const cuuint64_t dims[4] = {64, tokens, 9, static_cast<cuuint64_t>(h_kv)};
    const cuuint64_t strides[3] = {token_bytes, 128, MLA_HEAD_DIM * 2ull};
    const cuuint32_t box[4] = {64, 64, static_cast<cuuint32_t>(chunks), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode(m, tmap_type, 4, const_cast<void*>(k_cache_d), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  // Q rows as (64 cols, hg, h_kv, batch*s_q, 9 chunks): a box of `rows` query rows and all nine chunks
  // lands as [chunk][row][64 cols].
  auto q_map = [&](CUtensorMap* m, int rows) -> bool {
    const int bh = hg < rows ? hg : rows;
    const int bs = rows / bh;
    const cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(hg), static_cast<cuuint64_t>(h_kv),
                                static_cast<cuuint64_t>(batch) * s_q, 9};
    const cuuint64_t strides[4] = {MLA_HEAD_DIM * 2ull, static_cast<cuuint64_t>(hg) * MLA_HEAD_DIM * 2ull,
                                   static_cast<cuuint64_t>(h_q) * MLA_HEAD_DIM * 2ull, 128};
    const cuuint32_t box[5] = {64, static_cast<cuuint32_t>(bh), 1, static_cast<cuuint32_t>(bs), 9};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return encode(m, tmap_type, 5, const_cast<void*>(q_d), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };

  mla::DecodeArgs a;
  a.k_cache = static_cast<const uint8_t*>(k_cache_d);
  a.block_table = block_table_d;
  a.seqlens = cache_seqlens_d;
  a.tile_md = tile_md_d;
  a.num_splits = num_splits_d;
  a.out = out_d;
  a.lse = lse_d;
  const size_t max_pieces = static_cast<size_t>(batch) + num_parts;
  a.o_part = static_cast<float*>(workspace_d);
  a.lse_part = a.o_part + max_pieces * h_kv * R * MLA_VALUE_DIM;
  a.status = status_d;
  a.batch = batch;
  a.s_q = s_q;
  a.h_q = h_q;
  a.h_kv = h_kv;
  a.hg = hg;
  a.R = R;
  a.max_pages = max_pages_per_seq;
  a.num_pages = num_pages;
  a.causal = causal ? 1 : 0;
  a.num_parts = num_parts;
  a.max_pieces = static_cast<int>(max_pieces);
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.debug_flags = debug_flags;
  a.timeout_ns = timeout_ns ? timeout_ns : kDefaultTimeoutNs;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int row_blocks = (R + n - 1) / n;
  // 65..128+ rows per KV head: CTA pairs with 2-SM MMAs; otherwise one CTA per row block
  const bool use_pair = R > 64 && !(debug_flags & 4);
  cudaError_t le;
  if (use_pair) {
    mla::PairMaps maps;
    if (!page_map(&maps.k, 3)) return MLA_ERR_CUDA;
    for (int rank = 0; rank < 2; ++rank) {
      // dv quarter of rank r: columns 256 h + 128 r + 64 sub + c -> (64 cols, tokens, 2 sub, 2 halves, heads);
      // a box is one dv half of one page: 64 tokens x 128 columns (16 KB)
      const cuuint64_t dims[5] = {64, tokens, 2, 2, static_cast<cuuint64_t>(h_kv)};
      const cuuint64_t strides[4] = {token_bytes, 128, 512, MLA_HEAD_DIM * 2ull};
      const cuuint32_t box[5] = {64, 64, 2, 1, 1};
      const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
      void* base = static_cast<char*>(const_cast<void*>(k_cache_d)) + 256 * rank;
      if (encode(&maps.v[rank], tmap_type, 5, base, dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MLA_ERR_CUDA;
    }
    if (!q_map(&maps.q, 64)) return MLA_ERR_CUDA;
    le = mla::launch_decode_pair(dtype, maps, a, row_blocks, s);
  } else {
    CUtensorMap tm_k, tm_q;
    if (!page_map(&tm_k, 1) || !q_map(&tm_q, n)) return MLA_ERR_CUDA;
    le = mla::launch_decode(n, dtype, tm_k, tm_q, a, row_blocks, s);
  }
  if (le != cudaSuccess) return MLA_ERR_CUDA;
  if (debug_flags & 2) return MLA_OK;
  if (mla::launch_combine(dtype, num_splits_d, a.o_part, a.lse_part, a.out, lse_d, batch, s_q, h_q, h_kv, R, dev.sms, s) !=
      cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

int mla_combine_typed(int dtype, const int32_t* num_splits_d, const void* workspace_d, size_t workspace_bytes,
                      int batch, int s_q, int h_q, int h_kv, int num_parts, void* out_d, float* lse_d,
                      void* stream) {
  if (dtype != MLA_DTYPE_BF16 && dtype != MLA_DTYPE_FP16) return MLA_ERR_INVALID_ARG;
  if (num_splits_d == nullptr || workspace_d == nullptr || out_d == nullptr || lse_d == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > mla::metadata_max_batch() || s_q < 1 || h_q < 1 || h_kv < 1 || h_q % h_kv != 0 ||
      num_parts < 1)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(out_d, 16) || !aligned(workspace_d, 256)) return MLA_ERR_INVALID_ARG;
  const int R = static_cast<int>(static_cast<long long>(s_q) * h_q / h_kv);
  if (workspace_bytes < mla_workspace_bytes(batch, R, h_kv, MLA_VALUE_DIM, num_parts)) return MLA_ERR_WORKSPACE;
  const size_t max_pieces = static_cast<size_t>(batch) + num_parts;
  const float* o_part = static_cast<const float*>(workspace_d);
  const float* lse_part = o_part + max_pieces * h_kv * R * MLA_VALUE_DIM;
  DeviceInfo dev;
  const int st = device_info(&dev);
  if (st != MLA_OK) return st;
  if (mla::launch_combine(dtype, num_splits_d, o_part, lse_part, out_d, lse_d, batch, s_q, h_q, h_kv, R, dev.sms,
                          static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

int mla_combine(const int32_t* num_splits_d, const void* workspace_d, size_t workspace_bytes, int batch, int s_q,
                int h_q, int h_kv, int num_parts, void* out_d, float* lse_d, void* stream) {
  return mla_combine_typed(MLA_DTYPE_BF16, num_splits_d, workspace_d, workspace_bytes, batch, s_q, h_q, h_kv,
                           num_parts, out_d, lse_d, stream);
}

int mla_decode_paged_ex(const void* q_d, const void* k_cache_d, int num_pages, const int32_t* block_table_d,
                        int max_pages_per_seq, const int32_t* cache_seqlens_d, int batch, int s_q, int h_q, int h_kv,
                        int d, int dv, const int32_t* tile_md_d, const int32_t* num_splits_d, int num_parts,
                        int causal, float softmax_scale, void* workspace_d, size_t workspace_bytes, void* out_d,
                        float* lse_d, int32_t* status_d, int debug_flags, unsigned long long timeout_ns,
                        void* stream) {
  return mla_decode_paged_typed(MLA_DTYPE_BF16, q_d, k_cache_d, num_pages, block_table_d, max_pages_per_seq,
                                cache_seqlens_d, batch, s_q, h_q, h_kv, d, dv, tile_md_d, num_splits_d, num_parts,
                                causal, softmax_scale, workspace_d, workspace_bytes, out_d, lse_d, status_d,
                                debug_flags, timeout_ns, stream);
}

int mla_decode_paged(const void* q_d, const void* k_cache_d, int num_pages, const int32_t* block_table_d,
                     int max_pages_per_seq, const int32_t* cache_seqlens_d, int batch, int s_q, int h_q, int h_kv,
                     int d, int dv, const int32_t* tile_md_d, const int32_t* num_splits_d, int num_parts, int causal,
                     float softmax_scale, void* workspace_d, size_t workspace_bytes, void* out_d, float* lse_d,
                     int32_t* status_d, void* stream) {
  return mla_decode_paged_ex(q_d, k_cache_d, num_pages, block_table_d, max_pages_per_seq, cache_seqlens_d, batch,
                             s_q, h_q, h_kv, d, dv, tile_md_d, num_splits_d, num_parts, causal, softmax_scale,
                             workspace_d, workspace_bytes, out_d, lse_d, status_d, 0, 0, stream);
}

}  // extern "C"
