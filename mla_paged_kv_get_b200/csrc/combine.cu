// combine.cu — merge of split-KV partial results (cnblogs "DeepSeek 开源记-第1天-
// FlashMLA", §4.1 计算流程: 输出结果合并).
//
// For a row whose sequence was cut into n >= 2 pieces, each piece i left
// (O_i, lse_i) with O_i already normalised by its own denominator.  Then
//     lse = ln sum_i exp(lse_i),   O = sum_i exp(lse_i - lse) * O_i.
// Pieces with lse_i = -inf weigh nothing; if all are -inf the row is O = 0,
// lse = -inf.  Sequences with no piece (empty) get the same zero row.
// Sequences with exactly one piece were written by the decode kernel and are
// skipped here.
//
// A persistent grid (a few blocks per SM).  Each block first lists, in shared memory, the
// sequences the decode kernel did not finish (cut into n >= 2 pieces, or empty) with their first
// piece and piece count, from one block-wide scan over num_splits; the work items are then
// (listed sequence, KV head, row), one warp per row at a time, each lane owning 16 of its 512
// values.  A batch with nothing to merge costs one pass over num_splits.  The O loads of four
// pieces are issued together with the lse loads of up to 32, so a row of up to four pieces costs
// one memory latency and every further four pieces one more.
#include "ptx.cuh"
#include "decode.cuh"

namespace mla {

namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kThreads = 32 * kWarpsPerBlock;
constexpr int kBlocksPerSm = 2;
constexpr int kChunk = 4;          // pieces whose O loads are in flight together
constexpr int kMaxBatch = 8192;    // the metadata call's limit; the list takes 8 bytes per sequence

__device__ __forceinline__ int block_exclusive_scan_int(int v, int* warp_buf, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < kWarpsPerBlock ? warp_buf[lane] : 0;
    int x = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane < kWarpsPerBlock) warp_buf[lane] = x - w;
    if (lane == kWarpsPerBlock - 1) warp_buf[kWarpsPerBlock] = x;
  }
  __syncthreads();
  const int r = warp_buf[warp] + incl - v;
  *total = warp_buf[kWarpsPerBlock];
  __syncthreads();
  return r;
}

template <int T>
__global__ void __launch_bounds__(kThreads, kBlocksPerSm)
mla_combine_kernel(const int32_t* __restrict__ num_splits, const float* __restrict__ o_part,
                   const float* __restrict__ lse_part, uint16_t* __restrict__ out,
                   float* __restrict__ lse, int batch, int s_q, int h_q, int h_kv, int R) {
  pdl_trigger();   // the next kernel (a later step's metadata) may start launching; it waits for this grid
  pdl_wait();      // the partials and piece counts come from the decode kernel
  extern __shared__ int2 listed[];  // [batch]: (sequence | pieces << 16, first piece) of the sequences written here
  __shared__ int warp_buf[kWarpsPerBlock + 1];
  const int tid = threadIdx.x, lane = tid & 31;

  // ---- list the sequences with n != 1 pieces (contiguous chunk of sequences per thread)
  const int per = (batch + kThreads - 1) / kThreads;
  const int b0 = min(tid * per, batch), b1 = min(b0 + per, batch);
  int mine = 0;
  for (int b = b0; b < b1; ++b) mine += (__ldg(num_splits + b + 1) - __ldg(num_splits + b)) != 1;
  int count;
  int at = block_exclusive_scan_int(mine, warp_buf, &count);
  for (int b = b0; b < b1; ++b) {
    const int first = __ldg(num_splits + b), n = __ldg(num_splits + b + 1) - first;
    if (n != 1) listed[at++] = make_int2(b | (n << 16), first);
  }
  __syncthreads();
  if (count == 0) return;

  const int hg = h_q / h_kv;
  const size_t piece_stride = static_cast<size_t>(h_kv) * R;
  const size_t ostride4 = piece_stride * 512 / 4;   // float4 per piece
  const int items = count * h_kv * R;               // < 2^31: batch <= 8192, h_kv * R = s_q * h_q
  const int warps = gridDim.x * kWarpsPerBlock;
  for (int it = blockIdx.x * kWarpsPerBlock + (tid >> 5); it < items; it += warps) {
    const int r = it % R;
    const int g = (it / R) % h_kv;
    const int2 e = listed[it / (R * h_kv)];
    const int b = e.x & 0xffff, n = e.x >> 16, first = e.y;

    const int srow = r / hg, h = g * hg + r % hg;
    const size_t out_row = (static_cast<size_t>(b) * s_q + srow) * h_q + h;
    const size_t row0 = (static_cast<size_t>(first) * h_kv + g) * R + r;   // piece i: row0 + i * piece_stride
    const float4* obase = reinterpret_cast<const float4*>(o_part + row0 * 512) + lane;   // lane: float4 lane + 32 j
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    float top = -INFINITY, wsum = 0.f;
    float l32 = -INFINITY;   // lse of piece `lane` (the only lse registers: rows of up to 32 pieces)
    for (int base = 0; base < n; base += kChunk) {
      const int cnt = min(kChunk, n - base);
      float4 x[kChunk][4];
#pragma unroll
      for (int k = 0; k < kChunk; ++k) {
        if (k < cnt) {
#pragma unroll
          for (int j = 0; j < 4; ++j) x[k][j] = __ldg(obase + (base + k) * ostride4 + 32 * j);
        }
      }
      if (base == 0) {
        // the largest lse over all pieces while the O loads fly.  A piece with lse = -inf saw no
        // key, its O row holds zeros and weighs 0
        l32 = lane < n ? __ldg(lse_part + row0 + lane * piece_stride) : -INFINITY;
        top = l32;
        for (int i = lane + 32; i < n; i += 32) top = fmaxf(top, __ldg(lse_part + row0 + i * piece_stride));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
        if (top == -INFINITY) break;
      }
#pragma unroll
      for (int k = 0; k < kChunk; ++k) {
        if (k < cnt) {
          const int p = base + k;
          const float lp = n <= 32 ? __shfl_sync(0xffffffffu, l32, p)
                                   : __ldg(lse_part + row0 + static_cast<size_t>(p) * piece_stride);
          const float w = lp == -INFINITY ? 0.f : expf(lp - top);
          wsum += w;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[4 * j + 0] += w * x[k][j].x;
            acc[4 * j + 1] += w * x[k][j].y;
            acc[4 * j + 2] += w * x[k][j].z;
            acc[4 * j + 3] += w * x[k][j].w;
          }
        }
      }
    }
    float total_lse = -INFINITY;
    const float inv = top != -INFINITY ? 1.f / wsum : 0.f;
    if (top != -INFINITY) total_lse = top + logf(wsum);
    // lane owns values 4 lane + 128 j: write them as 8-byte pairs of bf16
    uint16_t* orow = out + out_row * 512;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint2*>(orow + 128 * j + 4 * lane) =
          make_uint2(pack2<T>(acc[4 * j] * inv, acc[4 * j + 1] * inv), pack2<T>(acc[4 * j + 2] * inv, acc[4 * j + 3] * inv));
    if (lane == 0) lse[out_row] = total_lse;
  }
}

}  // namespace

cudaError_t launch_combine(int dtype, const int32_t* num_splits, const float* o_part, const float* lse_part,
                           void* out, float* lse, int batch, int s_q, int h_q, int h_kv, int R, int num_sms,
                           cudaStream_t stream) {
  const long long items = static_cast<long long>(batch) * h_kv * R;
  if (batch > kMaxBatch || items >= (1ll << 31)) return cudaErrorInvalidValue;   // the kernel counts items in 32 bits
  const long long need = (items + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const long long cap = static_cast<long long>(num_sms) * kBlocksPerSm;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  const size_t smem = static_cast<size_t>(batch) * sizeof(int2);
  static std::atomic<uint64_t> configured_bf16{0}, configured_fp16{0};
  uint16_t* o = static_cast<uint16_t*>(out);
  if (dtype == kFP16) {
    const cudaError_t e = set_smem_limit_once(mla_combine_kernel<kFP16>, kMaxBatch * 8, configured_fp16);
    if (e != cudaSuccess) return e;
    return launch_pdl(mla_combine_kernel<kFP16>, dim3(blocks), dim3(kThreads), smem, stream, num_splits,
                      o_part, lse_part, o, lse, batch, s_q, h_q, h_kv, R);
  }
  const cudaError_t e = set_smem_limit_once(mla_combine_kernel<kBF16>, kMaxBatch * 8, configured_bf16);
  if (e != cudaSuccess) return e;
  return launch_pdl(mla_combine_kernel<kBF16>, dim3(blocks), dim3(kThreads), smem, stream, num_splits,
                    o_part, lse_part, o, lse, batch, s_q, h_q, h_kv, R);
}

}  // namespace mla
