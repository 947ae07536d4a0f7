// metadata.cu — tile scheduler for variable-length decode (jsxs2.com "什麼是
// FlashMLA", §3.1 分塊調度與並行計算: the work is cut into blocks and scheduled
// over the GPU; cnblogs "DeepSeek 开源记-第1天-FlashMLA", §6.2: the metadata call
// takes the sequence lengths, s_q*h_q/h_kv and h_kv and returns the scheduler
// table and num_splits).
//
// The rule (integer-only, so the table is bit-exact and deterministic):
//   n_b = ceil(L_b / 64) pages, cost c_b = n_b + C (0 for an empty sequence),
//   C = 4 pages of per-piece overhead, capacity W = ceil(sum c_b / G) + C.
//   Parts 0..G-2 are filled in order from a (sequence, page) cursor: skip
//   empty sequences; take the rest of a sequence while rest + C <= remaining;
//   otherwise take remaining - C pages (if >= 1) and close the part.  The last
//   part takes everything left.  Entry p = (begin_b, begin_page, end_b,
//   end_page, first_piece, n_pieces, 0, 0), end exclusive; pieces are numbered
//   in sweep order and num_splits is the prefix sum of pieces per sequence.
//
// One CTA: all threads compute page counts and the total cost, one thread
// sweeps (G + batch steps out of shared memory), all threads scan the piece
// counts into num_splits.
#include "decode.cuh"

namespace mla {

namespace {

constexpr int kThreads = 1024;
constexpr int kOverheadPages = 4;

__global__ void __launch_bounds__(kThreads, 1)
mla_metadata_kernel(const int32_t* __restrict__ seqlens, int batch, int num_parts,
                    int32_t* __restrict__ tile_md, int32_t* __restrict__ num_splits) {
  extern __shared__ int smem_i[];
  int* n_s = smem_i;              // pages per sequence
  int* pieces = smem_i + batch;   // pieces per sequence
  __shared__ long long warp_tot[32];
  __shared__ int warp_scan[32];
  __shared__ long long total_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  long long local = 0;
  for (int b = tid; b < batch; b += kThreads) {
    const int L = __ldg(seqlens + b);
    const int nb = L > 0 ? (L + 63) / 64 : 0;
    n_s[b] = nb;
    pieces[b] = 0;
    if (nb > 0) local += nb + kOverheadPages;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if (lane == 0) warp_tot[warp] = local;
  __syncthreads();
  if (tid == 0) {
    long long t = 0;
    for (int w = 0; w < kThreads / 32; ++w) t += warp_tot[w];
    total_s = t;
  }
  __syncthreads();

  if (tid == 0) {
    const long long G = num_parts;
    const long long W = (total_s + G - 1) / G + kOverheadPages;
    int b = 0, page = 0, piece = 0;
    for (int p = 0; p < num_parts; ++p) {
      const int begin_b = b, begin_page = page, first_piece = piece;
      if (p == num_parts - 1) {
        while (b < batch) {
          if (n_s[b] > page) {
            ++pieces[b];
            ++piece;
          }
          ++b;
          page = 0;
        }
      } else {
        long long remaining = W;
        while (b < batch) {
          const int nb = n_s[b];
          if (nb == 0) {
            ++b;
            page = 0;
            continue;
          }
          const int rest = nb - page;
          if (rest + kOverheadPages <= remaining) {
            remaining -= rest + kOverheadPages;
            ++pieces[b];
            ++piece;
            ++b;
            page = 0;
          } else {
            const long long take = remaining - kOverheadPages;
            if (take >= 1) {
              page += static_cast<int>(take);
              ++pieces[b];
              ++piece;
            }
            break;
          }
        }
      }
      int32_t* row = tile_md + static_cast<size_t>(p) * 8;
      row[0] = begin_b;
      row[1] = begin_page;
      row[2] = b;
      row[3] = page;
      row[4] = first_piece;
      row[5] = piece - first_piece;
      row[6] = 0;
      row[7] = 0;
    }
  }
  __syncthreads();

  // exclusive scan of pieces -> num_splits[0..batch]
  const int per = (batch + kThreads - 1) / kThreads;
  const int start = min(tid * per, batch), end = min(start + per, batch);
  int mine = 0;
  for (int i = start; i < end; ++i) mine += pieces[i];
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = warp_scan[lane];
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    warp_scan[lane] = x - v;   // exclusive prefix over warps
  }
  __syncthreads();
  int run = warp_scan[warp] + incl - mine;
  for (int i = start; i < end; ++i) {
    num_splits[i] = run;
    run += pieces[i];
  }
  if (tid == kThreads - 1) num_splits[batch] = warp_scan[warp] + incl;
}

}  // namespace

int metadata_max_batch() { return 16384; }

cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int32_t* tile_md,
                            int32_t* num_splits, cudaStream_t stream) {
  const int smem = 2 * batch * static_cast<int>(sizeof(int));
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(mla_metadata_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         2 * metadata_max_batch() * static_cast<int>(sizeof(int)));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  mla_metadata_kernel<<<1, kThreads, smem, stream>>>(seqlens, batch, num_parts, tile_md, num_splits);
  return cudaGetLastError();
}

}  // namespace mla
