// metadata.cu — tile scheduler for variable-length decode (jsxs2.com "什麼是
// FlashMLA", §3.1 分塊調度與並行計算: the work is cut into blocks and scheduled
// over the GPU; cnblogs "DeepSeek 开源记-第1天-FlashMLA", §6.2: the metadata call
// takes the sequence lengths, s_q*h_q/h_kv and h_kv and returns the scheduler
// table and num_splits).
//
// The rule (integer-only, so the table is bit-exact and deterministic) is a
// partition of a cost line:
//   sequence b with n_b = ceil(L_b / 64) pages occupies c_b = C + n_b units
//   (0 if empty): C = 4 overhead units, then one unit per page.  P_b is the
//   prefix sum of c_b.  Of the G_max table entries (the launch grid), G are
//   used: with W(G) = max(1, ceil(total / G)), G in [ceil(G_max/2), G_max]
//   minimises W(G) + S (S = 12 pages, the price of a merge pass) if some
//   sequence's first and last page fall in different parts, else W(G); the
//   largest G on ties; G = G_max when B * (number of candidates) > 32768 or
//   total >= 2^31.
//   W = W(G); part p < G owns units [p*W, (p+1)*W) (part G-1 everything after
//   (G-1)*W), parts G .. G_max-1 are empty, and page j of sequence b goes to
//   the part that owns unit P_b + C + j.
//   pos(U) = first (sequence, page) whose unit is >= U, or (B, 0).  Entry p is
//   (pos(p*W), pos((p+1)*W) or (B,0) for part G-1, first_piece, n_pieces, 0,
//   0), (B, 0, B, 0, total pieces, 0, 0, 0) for an empty part; a piece is a
//   (part, sequence) pair with >= 1 page, numbered part by part; num_splits is
//   the prefix sum of pieces per sequence.
//
// Every part and every sequence is independent given the prefix sums, so one
// CTA does it with two block scans (cost, then pieces) and one binary search
// per part boundary: no sequential sweep.  Because a sequence's pieces lie in
// consecutive parts, numbering pieces part by part is the same as numbering
// them sequence by sequence, so a part's first piece follows from num_splits
// in closed form.
#include "decode.cuh"

namespace mla {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
static_assert(kWarps == 32, "per-warp partials are reduced by one warp, one per lane");
constexpr int kOverhead = 4;
constexpr int kSplitPenalty = 12;
constexpr int kSearchBudget = 32768;   // (sequences x candidate part counts) examined at most
constexpr int kMaxBatch = 8192;
constexpr int kMaxParts = 4096;

// Exclusive prefix of `v` over the CTA (thread order); `*total` gets the sum.
__device__ long long block_exclusive_scan(long long v, long long* warp_buf, long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const long long w = warp_buf[lane];
    long long x = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    warp_buf[lane] = x - w;
    if (lane == 31) warp_buf[32] = x;
  }
  __syncthreads();
  const long long r = warp_buf[warp] + incl - v;
  *total = warp_buf[32];
  __syncthreads();
  return r;
}

struct Pos {
  int b, page;
};

__global__ void __launch_bounds__(kThreads, 1)
mla_metadata_kernel(const int32_t* __restrict__ seqlens, int batch, int num_parts,
                    int32_t* __restrict__ tile_md, int32_t* __restrict__ num_splits) {
  // The decode kernel, launched with programmatic serialization after this one, may start its
  // prologue now; it reads tile_md and num_splits only after this grid has completed.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // This grid may itself start before the previous kernel of the stream has finished (the combine
  // of an earlier step still reads num_splits).  Everything up to the first write of an output
  // reads only the lengths, which no kernel of this library writes, so it overlaps that kernel;
  // griddepcontrol.wait comes just before the outputs are written.
  extern __shared__ long long smem_ll[];
  long long* p_incl = smem_ll;                                        // [batch]  P_{b+1}
  int* n_s = reinterpret_cast<int*>(p_incl + batch);                  // [batch]  pages
  int* ns_s = n_s + batch;                                            // [batch+1] num_splits
  __shared__ long long warp_buf[33];
  const int tid = threadIdx.x;

  // ---- prefix sums of cost (contiguous chunk of sequences per thread)
  const int per = (batch + kThreads - 1) / kThreads;
  const int b0 = min(tid * per, batch), b1 = min(b0 + per, batch);
  long long my_cost = 0;
  int my_max_n = 0;
  for (int b = b0; b < b1; ++b) {
    const int L = __ldg(seqlens + b);
    const int nb = L > 0 ? (L + 63) / 64 : 0;
    n_s[b] = nb;
    my_cost += nb > 0 ? nb + kOverhead : 0;
    my_max_n = max(my_max_n, nb);
  }
  __shared__ int max_n_w[kWarps];   // longest sequence (pages) per warp; published by the scan's barriers
  {
    int m = my_max_n;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) max_n_w[tid >> 5] = m;
  }
  long long total_cost;
  long long run = block_exclusive_scan(my_cost, warp_buf, &total_cost);
  for (int b = b0; b < b1; ++b) {
    const int nb = n_s[b];
    run += nb > 0 ? nb + kOverhead : 0;
    p_incl[b] = run;
  }
  __syncthreads();

  // ---- number of parts in use
  __shared__ unsigned long long best_key[kWarps];
  const int lane = tid & 31;
  int max_n = max_n_w[lane];   // kWarps == 32: one warp entry per lane
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) max_n = max(max_n, __shfl_xor_sync(0xffffffffu, max_n, o));
  const int g_lo = max(1, (num_parts + 1) / 2);
  const int ncand = num_parts - g_lo + 1;
  const long long w_max = total_cost > 0 ? (total_cost + num_parts - 1) / num_parts : 1;
  int g_use = num_parts;
  // Skipped when G_max must win anyway: a candidate that splits costs >= W(G_max) + S, one that does
  // not must hold the longest sequence in one part (no part exceeds W units), so costs >= max_n; if
  // max_n >= W(G_max) + S no candidate beats G_max, which wins the ties.  Otherwise only a G with
  // max_n <= W(G) < W(G_max) + S can cost less than G_max, so only those (and G_max) are tested, one
  // warp per candidate, in 32-bit integers (the cost line fits).
  if (static_cast<long long>(batch) * ncand <= kSearchBudget && max_n < w_max + kSplitPenalty &&
      total_cost < (1ll << 31)) {
    const unsigned int total32 = static_cast<unsigned int>(total_cost);
    const int warp = tid >> 5;
    unsigned long long key = ~0ull;   // smallest cost, then largest G: (cost << 32) | (~G & 0xffffffff)
    for (int i = warp; i < ncand; i += kWarps) {
      const unsigned int Gc = static_cast<unsigned int>(g_lo + i);
      const unsigned int Wc = total32 > 0 ? (total32 + Gc - 1) / Gc : 1u;
      const bool tested = static_cast<int>(Gc) == num_parts ||
                          (Wc >= static_cast<unsigned int>(max_n) && Wc < static_cast<unsigned int>(w_max + kSplitPenalty));
      if (!tested) continue;
      bool split = false;
      for (int b = lane; b < batch; b += 32) {
        const int nb = n_s[b];
        if (nb == 0) continue;
        const unsigned int first = static_cast<unsigned int>((b > 0 ? p_incl[b - 1] : 0) + kOverhead);
        const unsigned int pf = min(first / Wc, Gc - 1), pl = min((first + nb - 1) / Wc, Gc - 1);
        split |= pf != pl;
      }
      split = __any_sync(0xffffffffu, split);
      const unsigned long long cost = static_cast<unsigned long long>(Wc) + (split ? kSplitPenalty : 0);
      const unsigned long long k2 = (cost << 32) | (0xffffffffull - static_cast<unsigned long long>(Gc));
      key = k2 < key ? k2 : key;
    }
    if (lane == 0) best_key[warp] = key;
    __syncthreads();
    unsigned long long best = best_key[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
      best = y < best ? y : best;
    }
    g_use = static_cast<int>(0xffffffffull - (best & 0xffffffffull));
  }
  // Quotients on the cost line in 32 bits whenever it fits (the usual case): a 64-bit division is
  // a long software sequence on the GPU.
  const bool line32 = total_cost < (1ll << 31);
  auto udiv = [line32](long long n, long long d) -> long long {
    return line32 ? static_cast<long long>(static_cast<unsigned int>(n) / static_cast<unsigned int>(d)) : n / d;
  };
  const long long G = g_use;
  const long long W = total_cost > 0 ? udiv(total_cost + G - 1, G) : 1;

  auto pos = [&](long long U) -> Pos {
    if (U >= total_cost) return Pos{batch, 0};
    int lo = 0, hi = batch - 1;            // first b with p_incl[b] > U
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (p_incl[mid] > U) hi = mid; else lo = mid + 1;
    }
    const long long start = lo > 0 ? p_incl[lo - 1] : 0;
    const long long pg = U - start - kOverhead;
    return Pos{lo, pg > 0 ? static_cast<int>(pg) : 0};
  };
  auto part_of = [&](long long unit) -> int {
    const long long p = udiv(unit, W);
    return static_cast<int>(p < G - 1 ? p : G - 1);
  };
  auto first_unit = [&](int b) -> long long { return (b > 0 ? p_incl[b - 1] : 0) + kOverhead; };

  // ---- pieces per sequence -> num_splits (a sequence's pieces sit in consecutive parts)
  long long my_pieces = 0;
  for (int b = b0; b < b1; ++b) {
    const int nb = n_s[b];
    if (nb > 0) my_pieces += part_of(first_unit(b) + nb - 1) - part_of(first_unit(b)) + 1;
  }
  long long total_pieces;
  long long run_p = block_exclusive_scan(my_pieces, warp_buf, &total_pieces);
  for (int b = b0; b < b1; ++b) {
    ns_s[b] = static_cast<int>(run_p);
    const int nb = n_s[b];
    if (nb > 0) run_p += part_of(first_unit(b) + nb - 1) - part_of(first_unit(b)) + 1;
  }
  if (tid == 0) ns_s[batch] = static_cast<int>(total_pieces);
  __syncthreads();

  // ---- outputs, once the previous kernel of the stream has finished with them
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int b = tid; b <= batch; b += kThreads) num_splits[b] = static_cast<int32_t>(ns_s[b]);

  // ---- parts.  Pieces are numbered part by part, which along the cost line is also sequence by
  // sequence, so the pieces before the part that begins at `be` are those of the sequences before
  // be.b plus, when be cuts sequence be.b, one per part from the one holding its page 0 to this one.
  auto pieces_before = [&](int p, Pos be) -> int {
    return ns_s[be.b] + (be.page > 0 ? p - part_of(first_unit(be.b)) : 0);
  };
  for (int p = tid; p < num_parts; p += kThreads) {
    const Pos be = p < G ? pos(static_cast<long long>(p) * W) : Pos{batch, 0};
    const Pos en = p < G - 1 ? pos(static_cast<long long>(p + 1) * W) : Pos{batch, 0};
    const int first = pieces_before(p, be);
    const int next = p < G - 1 ? pieces_before(p + 1, en) : ns_s[batch];
    int32_t* row = tile_md + static_cast<size_t>(p) * 8;
    row[0] = be.b;
    row[1] = be.page;
    row[2] = en.b;
    row[3] = en.page;
    row[4] = first;
    row[5] = next - first;
    row[6] = 0;
    row[7] = 0;
  }
}

}  // namespace

int metadata_max_batch() { return kMaxBatch; }
int metadata_max_parts() { return kMaxParts; }

cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int32_t* tile_md,
                            int32_t* num_splits, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(batch) * sizeof(long long) + (2 * batch + 1) * sizeof(int);
  constexpr int kMaxSmem = kMaxBatch * static_cast<int>(sizeof(long long)) +
                           (2 * kMaxBatch + 1) * static_cast<int>(sizeof(int));
  static std::atomic<uint64_t> configured{0};
  const cudaError_t e = set_smem_limit_once(mla_metadata_kernel, kMaxSmem, configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(mla_metadata_kernel, dim3(1), dim3(kThreads), smem, stream, seqlens, batch, num_parts, tile_md,
                    num_splits);
}

}  // namespace mla
