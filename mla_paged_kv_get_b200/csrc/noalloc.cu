// noalloc.cu — mla_decode_paged_noalloc: the decode entry point for callers
// that cannot allocate device memory.  The split partials live in a static
// device array owned by the library instead of a caller-supplied workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mla_b200.h"

namespace {

// Scratch for split partials, one copy per device that loads the library.
// Host code must not use this symbol as a pointer: on the host it is only a
// stand-in, and its device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_mla_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 = none yet).  Ids are
// never reused within a process, so a context destroyed and re-created (for
// example by cudaDeviceReset) gets a new one, unlike its handle, which may be.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  return ctx == nullptr || get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context of the current
// device.  Looked up once per device (cudaGetSymbolAddress with that device
// current) and again only when the device's context has changed since.
int scratch_address(void** out) {
  struct Entry {
    void* addr;
    unsigned long long ctx_id;
  };
  static Entry cache[kMaxDevices] = {};
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  unsigned long long ctx_id = 0;
  if (!current_context_id(&ctx_id)) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev].addr == nullptr || ctx_id == 0 || cache[dev].ctx_id != ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_noalloc_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    // the lookup makes the device's primary context current if no context was
    if (!current_context_id(&ctx_id) || ctx_id == 0) return MLA_ERR_CUDA;
    cache[dev] = Entry{p, ctx_id};
  }
  *out = cache[dev].addr;
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
