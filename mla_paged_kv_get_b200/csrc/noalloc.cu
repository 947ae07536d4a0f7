// noalloc.cu — mla_decode_paged_noalloc: the decode entry point for callers
// that cannot allocate device memory.  The split partials live in a static
// device array owned by the library instead of a caller-supplied workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mla_b200.h"

namespace {

// Scratch for split partials, one copy per device that loads the library.
// Host code must not use this symbol as a pointer: on the host it is only a
// stand-in, and its device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_mla_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of the scratch array on the current device, looked up once
// per device with that device current.
int scratch_address(void** out) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_noalloc_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" int mla_decode_paged_noalloc(const void* q_d, const void* k_cache_d, int num_pages,
                                        const int32_t* block_table_d, int max_pages_per_seq,
                                        const int32_t* cache_seqlens_d, int batch, int s_q, int h_q, int h_kv,
                                        int d, int dv, const int32_t* tile_md_d, const int32_t* num_splits_d,
                                        int num_parts, int causal, float softmax_scale, void* out_d, float* lse_d,
                                        int32_t* status_d, void* stream) {
  if (batch < 1 || s_q < 1 || h_q < 1 || h_kv < 1 || h_q % h_kv != 0 || num_parts < 1) return MLA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(s_q) * h_q / h_kv;
  if (rows > 4096) return MLA_ERR_INVALID_ARG;
  const size_t need = mla_workspace_bytes(batch, static_cast<int>(rows), h_kv, dv, num_parts);
  if (need == 0 || need > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != MLA_OK) return st;
  return mla_decode_paged(q_d, k_cache_d, num_pages, block_table_d, max_pages_per_seq, cache_seqlens_d, batch, s_q,
                          h_q, h_kv, d, dv, tile_md_d, num_splits_d, num_parts, causal, softmax_scale, scratch,
                          MLA_NOALLOC_SCRATCH_BYTES, out_d, lse_d, status_d, stream);
}
