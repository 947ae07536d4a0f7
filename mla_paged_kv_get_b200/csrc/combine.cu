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
// One warp per query row: each lane owns 16 of the 512 values, reads them with
// 16-byte loads per piece and writes 16 output values (two 16-byte stores), so a warp
// moves whole 2 KB partial rows and a 1 KB output row.  The lse values of all pieces
// are read in one round trip (one per lane) and four pieces' rows are in flight at
// once, so a row split n ways costs about 1 + n/4 memory latencies.
#include "ptx.cuh"
#include "decode.cuh"

namespace mla {

namespace {

constexpr int kRowsPerBlock = 4;
constexpr int kPiecesInFlight = 4;   // O rows of four pieces loaded before any is used

template <int T>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
mla_combine_kernel(const int32_t* __restrict__ num_splits, const float* __restrict__ o_part,
                   const float* __restrict__ lse_part, uint16_t* __restrict__ out,
                   float* __restrict__ lse, int batch, int s_q, int h_q, int h_kv, int R) {
  pdl_trigger();   // the next kernel (a later step's metadata) may start launching; it waits for this grid
  pdl_wait();      // the partials and piece counts come from the decode kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kRowsPerBlock + warp;
  const int g = blockIdx.y, b = blockIdx.z;
  if (r >= R) return;
  const int first = __ldg(num_splits + b);
  const int n = __ldg(num_splits + b + 1) - first;
  if (n == 1) return;

  const int hg = h_q / h_kv;
  const int srow = r / hg, h = g * hg + r % hg;
  const size_t out_row = (static_cast<size_t>(b) * s_q + srow) * h_q + h;

  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  const size_t row0 = (static_cast<size_t>(first) * h_kv + g) * R + r;   // piece i: row0 + i * h_kv * R
  const size_t piece_stride = static_cast<size_t>(h_kv) * R;
  // The lse of every piece at once, lane i holding pieces i, i + 32, ...: one memory round trip.
  float top = -INFINITY;
  for (int i = lane; i < n; i += 32) top = fmaxf(top, __ldg(lse_part + row0 + i * piece_stride));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
  float total_lse = -INFINITY;
  if (top != -INFINITY) {
    // Pieces 32 at a time: lane i holds the weight of piece base + i; their O rows are read four
    // pieces at a time, all four in flight before any is used.  A piece with lse = -inf saw no key;
    // its row holds zeros (the decode kernel wrote it) and weighs 0.
    float wpart = 0.f;
    for (int base = 0; base < n; base += 32) {
      const int mine = base + lane;
      const float li = mine < n ? __ldg(lse_part + row0 + mine * piece_stride) : -INFINITY;
      const float wi = li == -INFINITY ? 0.f : expf(li - top);
      wpart += wi;
      const int cnt = min(32, n - base);
      for (int j = 0; j < cnt; j += kPiecesInFlight) {
        float4 x[kPiecesInFlight][4];
#pragma unroll
        for (int k = 0; k < kPiecesInFlight; ++k) {
          if (j + k < cnt) {
            const float4* src =
                reinterpret_cast<const float4*>(o_part + (row0 + (base + j + k) * piece_stride) * 512) + lane * 4;
#pragma unroll
            for (int v = 0; v < 4; ++v) x[k][v] = __ldg(src + v);
          }
        }
#pragma unroll
        for (int k = 0; k < kPiecesInFlight; ++k) {
          const float w = __shfl_sync(0xffffffffu, wi, (j + k) & 31);
          if (j + k < cnt) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              acc[4 * v + 0] += w * x[k][v].x;
              acc[4 * v + 1] += w * x[k][v].y;
              acc[4 * v + 2] += w * x[k][v].z;
              acc[4 * v + 3] += w * x[k][v].w;
            }
          }
        }
      }
    }
    float wsum = wpart;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    const float inv = 1.f / wsum;
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] *= inv;
    total_lse = top + logf(wsum);
  }
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    packed[i] = pack2<T>(acc[2 * i], acc[2 * i + 1]);
  }
  uint4* dst = reinterpret_cast<uint4*>(out + out_row * 512) + lane * 2;
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  if (lane == 0) lse[out_row] = total_lse;
}

}  // namespace

cudaError_t launch_combine(int dtype, const int32_t* num_splits, const float* o_part, const float* lse_part,
                           void* out, float* lse, int batch, int s_q, int h_q, int h_kv, int R,
                           cudaStream_t stream) {
  const dim3 grid((R + kRowsPerBlock - 1) / kRowsPerBlock, h_kv, batch);
  uint16_t* o = static_cast<uint16_t*>(out);
  if (dtype == kFP16)
    return launch_pdl(mla_combine_kernel<kFP16>, grid, dim3(32 * kRowsPerBlock), 0, stream, num_splits, o_part,
                      lse_part, o, lse, batch, s_q, h_q, h_kv, R);
  return launch_pdl(mla_combine_kernel<kBF16>, grid, dim3(32 * kRowsPerBlock), 0, stream, num_splits, o_part,
                    lse_part, o, lse, batch, s_q, h_q, h_kv, R);
}

}  // namespace mla
