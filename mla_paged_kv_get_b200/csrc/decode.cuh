// decode.cuh — launch interface of the decode, combine and metadata kernels
// (host side of the C ABI in capi.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace mla {

// Raise a kernel's dynamic shared-memory limit on the current device, once per device and process.
// `done` holds one bit per device (0..63) that has been configured; concurrent first calls may both
// set the attribute, which is idempotent.
template <typename Kernel>
inline cudaError_t set_smem_limit_once(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Launch with programmatic stream serialization: the kernel may begin (prologue up to its
// pdl_wait()) while the previous kernel of the stream is still running.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

struct DecodeArgs {
  const uint8_t* k_cache;       // [num_pages, 64, h_kv, 576] bf16 or fp16 (read through the tensor maps)
  const int32_t* block_table;   // [batch, max_pages]
  const int32_t* seqlens;       // [batch]
  const int32_t* tile_md;       // [num_parts, 8]
  const int32_t* num_splits;    // [batch + 1]
  void* out;                    // [batch, s_q, h_q, 512] bf16 or fp16
  float* lse;                   // [batch, s_q, h_q]
  float* o_part;                // [max_pieces, h_kv, R, 512]
  float* lse_part;              // [max_pieces, h_kv, R]
  int32_t* status;              // optional
  int batch, s_q, h_q, h_kv, hg, R;
  int max_pages, num_pages, causal, num_parts, max_pieces;
  float scale_log2;             // softmax_scale * log2(e)
  int debug_flags;
  unsigned long long timeout_ns;
};

int decode_smem_bytes(int rows_per_block);
// dtype: MLA_DTYPE_BF16 or MLA_DTYPE_FP16 (q, cache and out)
cudaError_t launch_decode(int rows_per_block, int dtype, const CUtensorMap& tm_k, const CUtensorMap& tm_q,
                          const DecodeArgs& a, int row_blocks, cudaStream_t stream);

// Tensor maps of the pair kernel: the score product's page chunks (24 KB boxes),
// each CTA rank's dv quarter of one dv half of a page (16 KB boxes) and the 64 Q rows (72 KB).
struct PairMaps {
  CUtensorMap k;
  CUtensorMap v[2];
  CUtensorMap q;
};

int decode_pair_smem_bytes();
cudaError_t launch_decode_pair(int dtype, const PairMaps& maps, const DecodeArgs& a, int row_blocks,
                               cudaStream_t stream);

cudaError_t launch_combine(int dtype, const int32_t* num_splits, const float* o_part, const float* lse_part,
                           void* out, float* lse, int batch, int s_q, int h_q, int h_kv, int R, int num_sms,
                           cudaStream_t stream);

cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int32_t* tile_md,
                            int32_t* num_splits, cudaStream_t stream);

}  // namespace mla
