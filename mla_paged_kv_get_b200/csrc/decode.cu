// decode.cu — split-KV MLA decode kernel for B200 (sm_100a).
//
// What it computes (cnblogs "DeepSeek 开源记-第1天-FlashMLA", §2 关键特性, §4.1
// 计算流程, §6.2 基本使用): for every query row of a (sequence, KV head), the
// softmax-weighted sum of the first 512 dims of the cached 576-wide rows, and
// the log-sum-exp of the scores, over a 64-token paged cache.
//
// Design (B200-first; the pages' Hopper design is prior art only):
//   * One CTA per (row block of N query rows, KV head, scheduler part).  A part
//     is a page-granular range of (sequence, page) pairs produced by the
//     metadata kernel; it can span several sequences ("segments").
//   * Tiles of 128 keys = two 64-token pages.  The score product is computed
//     transposed, S^T[key, row] = K[key, :] . Q[row, :], so the 128 keys fill
//     the M = 128 datapath of one tcgen05.mma and the N query rows (16/32/64)
//     are the MMA's N; the output is also transposed, O^T[dv, row] +=
//     V^T[dv, key] . P^T[key, row], four M = 128 slices of dv.  TMEM holds
//     O^T (4N columns) and two S^T buffers (2N columns).
//   * Warp roles: warps 0-3 own TMEM lanes 0-127 (one key per thread for S,
//     one dv value per thread for O) and do masking, the online softmax and
//     the epilogue; the next warps issue TMA loads; one thread of the last
//     warp but one issues the score MMAs, one of the last warp the value MMAs.
//   * The cache is read through the page table by TMA (128-byte swizzle,
//     64 x 64 boxes, two per 16 KB ring slot) on mbarriers.  A tile is
//     streamed twice: nine slots for the score product (one 64-column chunk
//     of both pages each) and eight for the value product (128 dv columns of
//     one page each; the second read is an L2 hit).  This keeps the ring
//     independent of the tile size, which does not fit in shared memory next
//     to Q.
//   * Online softmax in log2 units with a lazy rescale: the running max moves
//     only when a score exceeds it by more than TAU = 8 (a factor 256); the
//     final normalisation uses the same running max, so the result is exact
//     up to rounding.  P is rounded to bf16 for the MMA and the denominator
//     sums those rounded values.
//   * Epilogue: O / l is staged through shared memory and written with 16-byte
//     stores, to `out` (bf16) when the sequence is not split, else to fp32
//     partials merged by the combine kernel.
//   * Every wait is bounded; an expired wait records MLA_ERR_TIMEOUT and the
//     CTA unwinds (drains its own TMA loads and MMAs, frees TMEM, returns).
#include <float.h>

#include "ptx.cuh"
#include "decode.cuh"
#include "segments.cuh"

namespace mla {

namespace {

constexpr int kKeys = 128;          // keys per tile (two pages)
constexpr int kSlotBytes = 16384;   // one ring slot: two 64 x 64 boxes
constexpr int kBoxBytes = 8192;     // one TMA box: 64 tokens x 64 bf16 columns
constexpr int kSoftmaxWarps = 4;
constexpr float kTau = 8.0f;        // lazy-rescale threshold (log2 units)
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kSoftmaxBar = 1;      // named barrier of warps 0-3

template <int N>
struct Cfg {
  // TMA issue is the bottleneck of 8 KB boxes (one warp moves ~28 GB/s): several producer
  // warps issue interleaved loads.  N = 64 keeps two so that 256 threads keep 255 registers.
  static constexpr int kProducers = N == 64 ? 2 : 4;
  static constexpr int kThreads = 32 * (kSoftmaxWarps + kProducers + 2);
  static constexpr int kMmaWarp = kSoftmaxWarps + kProducers;   // score-product issuer; owns TMEM
  static constexpr int kPvWarp = kMmaWarp + 1;                   // value-product issuer
  // Two rings, one per MMA issuer: score-product chunks (from HBM) and value-product chunks (the
  // same pages again, L2 hits).  A phase-parity wait is only sound when the waiter is at most
  // one phase ahead, so each ring has one consumer that takes it in order, and each slot one
  // producer warp (ring index modulo the producer count, ring sizes multiples of it).
  // 16-row blocks (measured): the score ring streams from HBM and is held by how fast its loads
  // are issued, so it gets three producer warps and six slots; the value ring's loads hit L2 and
  // one warp keeps up, but it needs six slots (four cost 30 %).  The rings are disjoint, so a full
  // one never holds up the other's loads.
  static constexpr int kSlotsQk = N == 16 ? 6 : 4;
  static constexpr int kSlotsPv = N == 16 ? 6 : 4;
  static constexpr int kQkProducers = N == 16 ? 3 : kProducers;
  static constexpr int kPvProducers = N == 16 ? 1 : kProducers;
  static constexpr int kSlots = kSlotsQk + kSlotsPv;
  static_assert(kSlotsQk % kQkProducers == 0 && kSlotsPv % kPvProducers == 0, "slot ownership");
  static constexpr int kPBuf = N == 64 ? 1 : 2;        // P^T buffers (one for N = 64: smem goes to the ring)
  static constexpr int kQBytes = N * 128 * 9;          // 9 chunks of [N rows][64 cols]
  static constexpr int kPBytes = kKeys * N * 2;        // P^T: [128 keys][N rows] bf16
  static constexpr int kTmemCols = N == 64 ? 512 : (N == 32 ? 256 : 128);
  static constexpr int kOffQ = kSlots * kSlotBytes;
  static constexpr int kOffP = kOffQ + kQBytes;
  static constexpr int kOffCtrl = kOffP + kPBuf * kPBytes;
  static constexpr int kCtrlBytes = 4096;
  static constexpr int kSmemBytes = kOffCtrl + kCtrlBytes + 1024;   // + base alignment slack
  static constexpr uint32_t kPSwizzle = N == 64 ? 2u : (N == 32 ? 4u : 6u);   // 128/64/32 B
  static constexpr uint32_t kPSwizzleMask = N == 64 ? 7u : (N == 32 ? 3u : 1u);
};

struct Ctrl {
  uint64_t full[16];
  uint64_t empty[16];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], p_free[2];
  uint64_t o_free, never, drain[2];
  uint32_t tmem_base;
  int abort_flag;         // any role gave up
  int softmax_abort;      // written only by warps 0-3, read after their barrier
  int pad;
  float m_run[64];        // running max per row, log2 units
  float alpha[64];        // rescale factor per row
  float inv_l[64];
  float lse_row[64];
  int kmax[64];           // keys < kmax[row] are visible in the current segment
  float red[4][64];       // cross-warp reduction scratch
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------------ producers (warps 4 ..)
// The slot-load sequence of a segment is fixed: Q, QK(0), then QK(t), PV(t-1) for t >= 1, then
// PV(T-1); QK(t) is nine loads (one 64-column chunk of both pages), PV(t) eight (128 dv columns of
// one page).  QK loads go to the score ring, PV loads to the value ring.  Each ring has its set of
// producer warps (all of them, or two per ring for 16-row blocks); a producer issues the loads whose
// index in the ring is its own modulo the set's size, so it owns fixed slots and waits only for the
// consumption of its own earlier loads.
template <int N>
__device__ void producer_role(const CUtensorMap* tm_k, const CUtensorMap* tm_q, const DecodeArgs& a,
                              Ctrl& ct, uint8_t* slots, uint8_t* qs, const Ctl& ctl, int rb, int g,
                              const int32_t* md, int pw) {
  using C = Cfg<N>;
  const int lane = threadIdx.x & 31;
  const int hg = a.hg;
  // Q box coordinates of this row block (host guarantees hg % N == 0 or N % hg == 0).
  const int r0 = rb * N;
  const int q_h0 = hg >= N ? r0 % hg : 0;
  const int q_s0 = r0 / hg;
  const int oob_page = a.num_pages;   // page coordinate past the cache: zero-filled box

  uint32_t qk_idx = 0, pv_idx = 0;
  uint32_t mine = 0, mine_parity = 0;   // slots holding a load of this warp, and its phase parity
  int qloads = 0;
  bool alive = true;
  SegIter it;
  it.init(md);
  Seg s;

  // lane 0 waits, the decision is broadcast so the warp stays converged
  auto wait_uniform = [&](uint64_t* bar, uint32_t parity) -> bool {
    int ok = 1;
    if (lane == 0) ok = wait_phase(bar, parity, ctl) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };

  while (alive && it.next(a, s)) {
    if (s.ntiles == 0) continue;
    if (pw == 0) {
      if (qloads > 0 && !wait_uniform(&ct.q_empty, (qloads - 1) & 1)) { alive = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(&ct.q_full, C::kQBytes);
        tma_load_5d(qs, tm_q, &ct.q_full, 0, q_h0, g, s.b * a.s_q + q_s0, 0);
      }
    }
    ++qloads;

    // page ids through a 32-entry window held one per lane
    const int32_t* bt_row = a.block_table + static_cast<size_t>(s.b) * a.max_pages;
    int win_base = -1, win_val = 0;
    auto page_id = [&](int pg) -> int {
      const int base = pg & ~31;
      if (base != win_base) {
        win_base = base;
        const int idx = base + lane;
        win_val = idx < s.hi ? __ldg(bt_row + idx) : oob_page;
      }
      int v = __shfl_sync(0xffffffffu, win_val, pg & 31);
      if (pg >= s.hi) return oob_page;          // absent second page of an odd tail
      if (v < 0 || v >= a.num_pages) {          // corrupt page id: never read out of bounds
        if (lane == 0) record_status(a.status, MLA_ERR_BAD_INPUT);
        v = oob_page;
      }
      return v;
    };

    // one slot: two 8 KB boxes; returns false when the CTA is aborting
    auto issue = [&](bool pv, int chunk0, int chunk1, int pid0, int pid1) -> bool {
      const uint32_t ridx = pv ? pv_idx++ : qk_idx++;
      const int owner = pv ? C::kProducers - C::kPvProducers + static_cast<int>(ridx % C::kPvProducers)
                           : static_cast<int>(ridx % C::kQkProducers);
      if (owner != pw) return true;
      const uint32_t n = pv ? C::kSlotsPv : C::kSlotsQk;
      const uint32_t slot = (pv ? C::kSlotsQk : 0) + ridx % n;
      if (ridx >= n && !wait_uniform(&ct.empty[slot], ((ridx / n) - 1) & 1)) return false;
      mine |= 1u << slot;
      mine_parity = (mine_parity & ~(1u << slot)) | (((ridx / n) & 1u) << slot);
      if (lane == 0) {
        uint8_t* dst = slots + slot * kSlotBytes;
        mbar_arrive_expect_tx(&ct.full[slot], 2 * kBoxBytes);
        tma_load_4d(dst, tm_k, &ct.full[slot], 0, 64 * pid0, chunk0, g);
        tma_load_4d(dst + kBoxBytes, tm_k, &ct.full[slot], 0, 64 * pid1, chunk1, g);
      }
      return true;
    };
    auto issue_qk = [&](int t) -> bool {
      // [page][64 tokens][64 cols]: the 128 keys of the tile contiguous, one column chunk
      const int pid0 = page_id(s.lo + 2 * t), pid1 = page_id(s.lo + 2 * t + 1);
      for (int c = 0; c < 9; ++c)
        if (!issue(false, c, c, pid0, pid1)) return false;
      return true;
    };
    auto issue_pv = [&](int t) -> bool {
      // [chunk j][64 tokens][64 cols] of one page: 128 dv columns of 64 keys
      const int pid0 = page_id(s.lo + 2 * t), pid1 = page_id(s.lo + 2 * t + 1);
      for (int u = 0; u < 8; ++u) {
        const int pid = (u & 1) ? pid1 : pid0;
        const int c = 2 * (u >> 1);
        if (!issue(true, c, c + 1, pid, pid)) return false;
      }
      return true;
    };

    if (!issue_qk(0)) { alive = false; break; }
#pragma unroll 1
    for (int t = 1; t < s.ntiles && alive; ++t) {
      if (!issue_qk(t) || !issue_pv(t - 1)) alive = false;
    }
    if (alive && !issue_pv(s.ntiles - 1)) alive = false;
  }

  if (!alive && lane == 0) {
    // unwind: let every TMA load this warp issued land before the CTA exits (the latest load of
    // each of its slots; earlier ones were consumed before the slot was refilled)
    for (int slot = 0; slot < C::kSlots; ++slot)
      if (mine & (1u << slot)) drain_phase(&ct.full[slot], (mine_parity >> slot) & 1u, 1000000000ull);
    if (pw == 0 && qloads > 0) drain_phase(&ct.q_full, (qloads - 1) & 1, 1000000000ull);
  }
  __syncwarp();
}

// ------------------------------------------------------------------ MMA issuers
// Two threads issue MMAs: lane 0 of kMmaWarp the score products, lane 0 of kPvWarp the value
// products.  Each commit and barrier test of an issuing thread stalls its MMA stream for a few
// hundred cycles; two issuers hide those stalls behind each other's MMAs.  Each consumes its own
// ring in order.  Called by lane 0 only.
template <int N, int T>
__device__ void mma_role(const DecodeArgs& a, Ctrl& ct, uint8_t* slots, uint8_t* qs, uint8_t* ps,
                         uint32_t tmem, const Ctl& ctl, const int32_t* md, const bool pv_role) {
  using C = Cfg<N>;
  const uint32_t idesc_qk = idesc_f32<T>(128, N, false, false);   // K-major A (keys), K-major B (rows)
  const uint32_t idesc_pv = idesc_f32<T>(128, N, true, true);     // MN-major A (dv), MN-major B (rows)
  const uint32_t slots_addr = smem_addr(slots);
  const uint32_t q_addr = smem_addr(qs);
  const uint32_t p_addr = smem_addr(ps);

  uint32_t ridx = 0;   // loads of this issuer's ring consumed so far
  int tg = 0, qloads = 0, seg_i = 0;   // seg_i: segments with tiles issued so far
  bool alive = true;
  SegIter it;
  it.init(md);
  Seg s;

  while (alive && it.next(a, s)) {
    const int tg0 = tg;
    if (s.ntiles == 0) continue;   // nothing to issue; its epilogue does not touch O in TMEM
    if (!pv_role) {
      if (!wait_phase_lean(&ct.q_full, qloads & 1, ctl)) { alive = false; break; }
      ++qloads;
      tc_fence_after();
    }

    auto do_qk = [&](int t) -> bool {
      if (pv_role) return true;
      const int tgl = tg0 + t, sb = tgl & 1;
      if (tgl >= 2 && !wait_phase_lean(&ct.s_free[sb], ((tgl >> 1) - 1) & 1, ctl)) return false;
      tc_fence_after();
      const uint32_t d_tmem = tmem + 4 * N + sb * N;
#pragma unroll 1
      for (int c = 0; c < 9; ++c) {
        const uint32_t slot = ridx % C::kSlotsQk;
        if (!wait_phase_lean(&ct.full[slot], (ridx / C::kSlotsQk) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t base = slots_addr + slot * kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // A = K: 128 keys x 16 columns, K-major; B = Q chunk c: N rows x 16 columns, K-major
          const uint64_t ad = smem_desc(base + kk * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(q_addr + c * N * 128 + kk * 32, 16, 1024, 2);
          umma_bf16(d_tmem, ad, bd, idesc_qk, (c | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&ct.empty[slot]);
        ++ridx;
      }
      umma_commit(&ct.s_full[sb]);
      if (t == s.ntiles - 1) umma_commit(&ct.q_empty);
      return true;
    };

    auto do_pv = [&](int t) -> bool {
      if (!pv_role) return true;
      const int tgl = tg0 + t, pb = tgl & 1;
      // O in TMEM is overwritten from the first value product of a segment on: wait until the softmax
      // has read out the previous segment that had tiles (one o_free phase per such segment)
      if (t == 0 && seg_i > 0 && !wait_phase_lean(&ct.o_free, (seg_i - 1) & 1, ctl)) return false;
      if (!wait_phase_lean(&ct.p_full[pb], (tgl >> 1) & 1, ctl)) return false;
      tc_fence_after();
      const uint32_t pbase = p_addr + (tgl % C::kPBuf) * C::kPBytes;
#pragma unroll 1
      for (int u = 0; u < 8; ++u) {
        const uint32_t slot = C::kSlotsQk + ridx % C::kSlotsPv;
        if (!wait_phase_lean(&ct.full[slot], (ridx / C::kSlotsPv) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t base = slots_addr + slot * kSlotBytes;
        const int q = u & 1;   // page of the tile: keys 64q .. 64q+63
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // A = V^T: 128 dv (two 64-column boxes 8 KB apart) x 16 keys, MN-major
          const uint64_t ad = smem_desc(base + kk * 2048, kBoxBytes, 1024, 2);
          // B = P^T: 16 keys x N rows, MN-major (rows contiguous)
          const uint64_t bd = smem_desc(pbase + (4 * q + kk) * 16 * 2 * N, C::kPBytes, 16 * N, C::kPSwizzle);
          umma_bf16(tmem + (u >> 1) * N, ad, bd, idesc_pv, (t > 0 || q > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&ct.empty[slot]);
        ++ridx;
      }
      umma_commit(&ct.p_free[pb]);
      return true;
    };

    if (!do_qk(0)) { alive = false; break; }
#pragma unroll 1
    for (int t = 1; t < s.ntiles && alive; ++t) {
      if (!do_qk(t) || !do_pv(t - 1)) alive = false;
    }
    if (alive && !do_pv(s.ntiles - 1)) alive = false;
    tg += s.ntiles;
    ++seg_i;
  }

  // every MMA this thread issued has finished, and its commits have landed, before TMEM is
  // freed and the CTA exits (on the normal path the softmax has waited for them already, but
  // not after an abort)
  uint64_t* drain = &ct.drain[pv_role ? 1 : 0];
  umma_commit(drain);
  drain_phase(drain, 0, 1000000000ull);
}

// ------------------------------------------------------------------ softmax + epilogue
template <int N, int T>
__device__ void softmax_role(const DecodeArgs& a, Ctrl& ct, uint8_t* ps, uint32_t tmem, const Ctl& ctl,
                             int rb, int g, const int32_t* md) {
  using C = Cfg<N>;
  const int tid = threadIdx.x;        // 0..127: TMEM lane (key of a tile / dv of an O slice)
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
  const int rows_here = min(N, a.R - rb * N);
  const int hg = a.hg;

  float lsum[N];
#pragma unroll
  for (int c = 0; c < N; ++c) lsum[c] = 0.f;

  // All 128 threads take every exit together: a failed wait is published in
  // softmax_abort and read back after the next barrier of the group.
  auto uniform_ok = [&](bool ok) -> bool {
    if (!ok) ct.softmax_abort = 1;
    named_sync(kSoftmaxBar, 128);
    return ct.softmax_abort == 0;
  };

  if (a.debug_flags & 1) {
    // fault-detection test: wait on a barrier nothing signals
    if (!uniform_ok(wait_phase(&ct.never, 0, ctl))) return;
  }

  int tg = 0;
  SegIter it;
  it.init(md);
  Seg s;
  while (it.next(a, s)) {
    if (tid < N) {
      int kmax = 0;
      if (tid < rows_here && s.ok) {
        const int srow = (rb * N + tid) / hg;
        const int seg_end = min(s.hi * 64, s.L);
        const int lim = a.causal ? s.L - (a.s_q - 1 - srow) : s.L;
        kmax = min(seg_end, lim);
      }
      ct.kmax[tid] = kmax;
      ct.m_run[tid] = -INFINITY;
    }
    if (!s.ok && tid == 0) record_status(a.status, MLA_ERR_BAD_INPUT);
    named_sync(kSoftmaxBar, 128);

#pragma unroll 1
    for (int t = 0; t < s.ntiles; ++t, ++tg) {
      const int sb = tg & 1;
      bool ok = wait_phase(&ct.s_full[sb], (tg >> 1) & 1, ctl);
      // the P buffer of this tile is free once the value product that last read it has finished
      if (ok && tg >= C::kPBuf)
        ok = wait_phase(&ct.p_free[(tg - C::kPBuf) & 1], ((tg - C::kPBuf) >> 1) & 1, ctl);
      float x[N];
      bool need = false;
      if (ok) {
        tc_fence_after();
        uint32_t sv[N];
#pragma unroll
        for (int c16 = 0; c16 < N / 16; ++c16) {
          uint32_t r[16];
          tmem_ld16(tmem + lane_base + 4 * N + sb * N + 16 * c16, r);
#pragma unroll
          for (int i = 0; i < 16; ++i) sv[16 * c16 + i] = r[i];
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&ct.s_free[sb]);
        const int key = (s.lo + 2 * t) * 64 + tid;
#pragma unroll
        for (int c = 0; c < N; ++c) {
          const bool vis = key < ct.kmax[c];
          x[c] = vis ? __uint_as_float(sv[c]) * a.scale_log2 : -INFINITY;
          need |= x[c] > ct.m_run[c] + kTau;
        }
      }
      if (!ok) ct.softmax_abort = 1;
      need = named_sync_or(kSoftmaxBar, 128, need);
      if (ct.softmax_abort) return;

      if (need) {
        // exact column maxima over the 128 keys of the tile
#pragma unroll
        for (int c = 0; c < N; ++c) {
          const float v = warp_max(x[c]);
          if (lane == 0) ct.red[warp][c] = v;
        }
        named_sync(kSoftmaxBar, 128);
        if (tid < N) {
          const float mt = fmaxf(fmaxf(ct.red[0][tid], ct.red[1][tid]), fmaxf(ct.red[2][tid], ct.red[3][tid]));
          const float mo = ct.m_run[tid];
          const float mn = fmaxf(mo, mt);
          ct.alpha[tid] = (mo == -INFINITY) ? (mn == -INFINITY ? 1.f : 0.f) : ex2(mo - mn);
          ct.m_run[tid] = mn;
        }
        named_sync(kSoftmaxBar, 128);
#pragma unroll
        for (int c = 0; c < N; ++c) lsum[c] *= ct.alpha[c];
        if (t > 0) {
          // O^T holds tiles < t: wait for the value product of tile tg-1, rescale in TMEM
          const bool okr = wait_phase(&ct.p_free[(tg - 1) & 1], ((tg - 1) >> 1) & 1, ctl);
          if (!uniform_ok(okr)) return;
          tc_fence_after();
#pragma unroll 1
          for (int d = 0; d < 4; ++d) {
#pragma unroll
            for (int c16 = 0; c16 < N / 16; ++c16) {
              uint32_t r[16];
              const uint32_t ta = tmem + lane_base + d * N + 16 * c16;
              tmem_ld16(ta, r);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * ct.alpha[16 * c16 + i]);
              tmem_st16(ta, r);
            }
          }
          tmem_wait_st();
        }
      }

      // P^T row of this key: N bf16 values, swizzled 16-byte chunks
      uint8_t* pbuf = ps + (tg % C::kPBuf) * C::kPBytes;
#pragma unroll
      for (int c8 = 0; c8 < N / 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = 8 * c8 + 2 * i;
          const float p0 = x[c] == -INFINITY ? 0.f : ex2(x[c] - ct.m_run[c]);
          const float p1 = x[c + 1] == -INFINITY ? 0.f : ex2(x[c + 1] - ct.m_run[c + 1]);
          w[i] = pack2<T>(p0, p1);
          lsum[c] += unpack_lo<T>(w[i]);
          lsum[c + 1] += unpack_hi<T>(w[i]);
        }
        const uint32_t off = static_cast<uint32_t>(tid * 2 * N + c8 * 16);
        const uint32_t phys = off ^ (((off >> 7) & C::kPSwizzleMask) << 4);
        *reinterpret_cast<uint4*>(pbuf + phys) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(&ct.p_full[sb]);
    }

    // ---------------- epilogue of the segment
    if (s.ntiles > 0) {
      const int tl = tg - 1;
      const bool okw = wait_phase(&ct.p_free[tl & 1], (tl >> 1) & 1, ctl);
      if (!uniform_ok(okw)) return;
      tc_fence_after();
    }
#pragma unroll
    for (int c = 0; c < N; ++c) {
      const float v = warp_sum(lsum[c]);
      if (lane == 0) ct.red[warp][c] = v;
      lsum[c] = 0.f;
    }
    named_sync(kSoftmaxBar, 128);
    if (tid < N) {
      const float l = (ct.red[0][tid] + ct.red[1][tid]) + (ct.red[2][tid] + ct.red[3][tid]);
      const bool any = l > 0.f;
      ct.inv_l[tid] = any ? 1.f / l : 0.f;
      ct.lse_row[tid] = any ? (ct.m_run[tid] + log2f(l)) * kLn2 : -INFINITY;
    }
    named_sync(kSoftmaxBar, 128);

    const int npieces = __ldg(a.num_splits + s.b + 1) - __ldg(a.num_splits + s.b);
    const bool final_out = npieces == 1;
    const bool can_write = final_out || s.piece < a.max_pieces;
    if (!can_write && tid == 0) record_status(a.status, MLA_ERR_BAD_INPUT);
    uint16_t* stage_h = reinterpret_cast<uint16_t*>(ps);

#pragma unroll 1
    for (int d = 0; d < 4; ++d) {
      float v[N];
      if (s.ntiles > 0) {
#pragma unroll
        for (int c16 = 0; c16 < N / 16; ++c16) {
          uint32_t r[16];
          tmem_ld16(tmem + lane_base + d * N + 16 * c16, r);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[16 * c16 + i] = __uint_as_float(r[i]);
        }
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < N; ++c) v[c] = 0.f;
      }
      if (final_out) {
        // stage [row][128 dv] bf16 (one P buffer) so each output row slice leaves as 16-byte vectors
#pragma unroll
        for (int c = 0; c < N; ++c) stage_h[c * 128 + tid] = to_bits<T>(v[c] * ct.inv_l[c]);
        named_sync(kSoftmaxBar, 128);
        if (can_write) {
          for (int i = tid; i < rows_here * 16; i += 128) {
            const int c = i >> 4, vv = i & 15;
            const int r = rb * N + c;
            const int srow = r / hg, h = g * hg + r % hg;
            const uint4 val = reinterpret_cast<const uint4*>(ps)[c * 16 + vv];
            uint16_t* dst = static_cast<uint16_t*>(a.out) + ((static_cast<size_t>(s.b) * a.s_q + srow) * a.h_q + h) * 512 + d * 128;
            reinterpret_cast<uint4*>(dst)[vv] = val;
          }
        }
        named_sync(kSoftmaxBar, 128);
      } else if (can_write) {
        // fp32 partials: a warp writes 32 consecutive floats (128 bytes) per row
        float* dst = a.o_part + ((static_cast<size_t>(s.piece) * a.h_kv + g) * a.R + rb * N) * 512 + d * 128 + tid;
#pragma unroll
        for (int c = 0; c < N; ++c) {
          if (c < rows_here) dst[static_cast<size_t>(c) * 512] = v[c] * ct.inv_l[c];
        }
      }
    }
    if (tid < rows_here && can_write) {
      const int r = rb * N + tid;
      if (final_out) {
        const int srow = r / hg, h = g * hg + r % hg;
        a.lse[(static_cast<size_t>(s.b) * a.s_q + srow) * a.h_q + h] = ct.lse_row[tid];
      } else {
        a.lse_part[(static_cast<size_t>(s.piece) * a.h_kv + g) * a.R + r] = ct.lse_row[tid];
      }
    }
    // O may be overwritten again: signalled only after segments that had tiles, the ones whose O came
    // from TMEM, so the value issuer (which waits once per such segment) can never be lapped
    if (s.ntiles > 0) {
      tc_fence_before();
      mbar_arrive(&ct.o_free);
    }
  }
}

template <int N, int T>
__global__ void __launch_bounds__(Cfg<N>::kThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const DecodeArgs a) {
  using C = Cfg<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* slots = smem;
  uint8_t* qs = smem + C::kOffQ;
  uint8_t* ps = smem + C::kOffP;
  Ctrl& ct = *reinterpret_cast<Ctrl*>(smem + C::kOffCtrl);

  const int warp = threadIdx.x >> 5;
  const int rb = blockIdx.x, g = blockIdx.y, part = blockIdx.z;
  const int32_t* md = a.tile_md + static_cast<size_t>(part) * MLA_MD_WORDS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(&ct.full[i], 1);
      mbar_init(&ct.empty[i], 1);
    }
    mbar_init(&ct.q_full, 1);
    mbar_init(&ct.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ct.s_full[i], 1);
      mbar_init(&ct.s_free[i], 128);
      mbar_init(&ct.p_full[i], 128);
      mbar_init(&ct.p_free[i], 1);
    }
    mbar_init(&ct.o_free, 128);
    mbar_init(&ct.never, 1);
    mbar_init(&ct.drain[0], 1);
    mbar_init(&ct.drain[1], 1);
    ct.abort_flag = 0;
    ct.softmax_abort = 0;
    fence_barrier_init();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(&ct.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kSoftmaxWarps && (threadIdx.x & 31) == 0) {
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();   // the combine may start launching; it waits for this grid to finish
  pdl_wait();      // the part table and piece counts come from the metadata kernel
  const uint32_t tmem = ct.tmem_base;
  const Ctl ctl{&ct.abort_flag, a.status, a.timeout_ns};

  if (warp < kSoftmaxWarps) {
    softmax_role<N, T>(a, ct, ps, tmem, ctl, rb, g, md);
  } else if (warp < C::kMmaWarp) {
    producer_role<N>(&tm_k, &tm_q, a, ct, slots, qs, ctl, rb, g, md, warp - kSoftmaxWarps);
  } else {
    if ((threadIdx.x & 31) == 0) mma_role<N, T>(a, ct, slots, qs, ps, tmem, ctl, md, warp == C::kPvWarp);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace

int decode_smem_bytes(int n) {
  switch (n) {
    case 16: return Cfg<16>::kSmemBytes;
    case 32: return Cfg<32>::kSmemBytes;
    case 64: return Cfg<64>::kSmemBytes;
    default: return -1;
  }
}

template <int N, int T>
static cudaError_t launch_n(const CUtensorMap& tm_k, const CUtensorMap& tm_q, const DecodeArgs& a, dim3 grid,
                            cudaStream_t stream) {
  static std::atomic<uint64_t> configured{0};
  const cudaError_t e = set_smem_limit_once(mla_decode_kernel<N, T>, Cfg<N>::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(mla_decode_kernel<N, T>, grid, dim3(Cfg<N>::kThreads), Cfg<N>::kSmemBytes, stream, tm_k, tm_q, a);
}

template <int T>
static cudaError_t launch_t(int n, const CUtensorMap& tm_k, const CUtensorMap& tm_q, const DecodeArgs& a, dim3 grid,
                            cudaStream_t stream) {
  switch (n) {
    case 16: return launch_n<16, T>(tm_k, tm_q, a, grid, stream);
    case 32: return launch_n<32, T>(tm_k, tm_q, a, grid, stream);
    case 64: return launch_n<64, T>(tm_k, tm_q, a, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode(int n, int dtype, const CUtensorMap& tm_k, const CUtensorMap& tm_q, const DecodeArgs& a,
                          int row_blocks, cudaStream_t stream) {
  const dim3 grid(row_blocks, a.h_kv, a.num_parts);
  if (dtype == kFP16) return launch_t<kFP16>(n, tm_k, tm_q, a, grid, stream);
  return launch_t<kBF16>(n, tm_k, tm_q, a, grid, stream);
}

}  // namespace mla
