// decode_pair.cu — split-KV MLA decode for 65..128 query rows per KV head, run
// by CTA pairs (cluster of 2, tcgen05 cta_group::2) on B200.
//
// What it computes is the same as decode.cu (cnblogs "DeepSeek 开源记-第1天-
// FlashMLA", §2 关键特性, §4.1 计算流程, §6.2 基本使用).  How:
//   * A pair of CTAs (one per SM) drives one 2-SM MMA.  Each CTA keeps 64 query
//     rows (72 KB) in shared memory: S = Q.K^T is one M = 128 x N = 128 x 576
//     product per 128-key tile, the 128 keys being two 64-token pages of which
//     each CTA loads one.  So every cache byte of the score product crosses
//     L2 -> SM exactly once, and each SM reads only half of the B operand.
//   * O = P.V in two M = 128 x N = 256 products (dv halves); each CTA supplies
//     128 dv columns of each half for both pages (a second, L2-hit read of a
//     quarter of the latent columns per page) and the P of its own 64 rows.
//   * Three MMA-issuing threads on the leader CTA.  A pair MMA of 64 rows per SM
//     is only 32 cycles of tensor work, less than one thread needs to issue it
//     with its barrier tests and commits, so the 36 score MMAs of a tile are
//     split between two issuers (the first and second 288 latent columns), each
//     accumulating its own partial S in TMEM; the softmax adds the two.  The
//     third issuer runs the value products.
//   * Two P buffers: the softmax of tile t+1 writes its P while the value
//     product of tile t still reads the other one.
//   * Loads are few and large: a TMA instruction costs about the same whether
//     it moves 8 KB or 24 KB, so the score product's page arrives as three
//     24 KB boxes (three 64-column chunks each, one 4-D tensor map), a dv half
//     of the value quarter of a page as one 16 KB box (5-D map per CTA rank)
//     and Q as one 72 KB box per sequence.
//   * TMEM per CTA: O (2 x 128 columns: 64 rows x 512 dv in the pair layout
//     that puts the second half of N in lanes 64..127) and two S buffers of
//     two partial sums each (4 x 64 columns).  Thread t of warps 0-3 owns TMEM
//     lane t: row t % 64 and key half (or dv quarter) t / 64, so the softmax of
//     a row is split between two threads and needs no shuffles.
//   * Separate load rings for the score product (24 KB slots) and for the
//     value product (16 KB slots), each with its own producer warp, so value
//     loads for tile t overlap the score product of tile t+1.
//   * The peer's TMA loads complete on the leader's barriers (cta_group::2
//     loads, no multicast), MMA completions are committed to both CTAs, and
//     the peer's softmax warps arrive on the leader's barriers through cluster
//     shared memory.
//   * Online softmax in log2 units with the lazy rescale of decode.cu (TAU = 8),
//     every wait bounded; an expired wait records MLA_ERR_TIMEOUT and the pair
//     unwinds.
#include <float.h>

#include "ptx.cuh"
#include "decode.cuh"
#include "segments.cuh"

namespace mla {

namespace {

constexpr int kRows = 64;              // query rows per CTA
constexpr int kBox = 8192;             // one 64-column chunk of 64 tokens (or rows), bf16
constexpr int kKSlots = 3;             // score ring: three chunks of this CTA's page per slot
constexpr int kKSlotBytes = 3 * kBox;
constexpr int kVSlots = 3;             // value ring: [2 chunks] of one dv half of one page per slot
constexpr int kVSlotBytes = 2 * kBox;
constexpr int kThreads = 288;          // warps 0-3 softmax, 4 score loads, 5 value loads, 6-8 MMA issuers
constexpr int kQBytes = 9 * kBox;      // 64 rows x 576: [chunk][row][64 cols]
constexpr int kPBytes = 2 * kBox;      // one P buffer: [key half][64 rows][64 keys] bf16
constexpr int kPBufs = 2;
constexpr int kOffP = kQBytes;
constexpr int kOffK = kOffP + kPBufs * kPBytes;
constexpr int kOffV = kOffK + kKSlots * kKSlotBytes;
constexpr int kOffCtrl = kOffV + kVSlots * kVSlotBytes;
constexpr int kCtrlBytes = 1024;
constexpr int kSmemBytes = kOffCtrl + kCtrlBytes + 1024;   // + base alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr uint32_t kTmemCols = 512;
constexpr int kColO = 0;               // O half h at column 128 h
constexpr int kColS = 256;             // partial S p (0, 1) of buffer b at column 256 + 128 p + 64 b
// The 36 K steps (16 latent columns each) of a tile's score product, by issuer: the first 18
// (slot 0 and half of slot 1) and the last 18.  Slot 1 is read by both.
constexpr int kKStepsPerIssuer = 18;
constexpr float kTau = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kSoftmaxBar = 1;

struct Ctrl {
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t v_full[kVSlots], v_empty[kVSlots];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], p_free[2];    // by tile parity, whatever the number of P buffers
  uint64_t o_free, never, drain[3];
  uint32_t tmem_base;
  int abort_flag;
  int softmax_abort;
  int pad;
  float red[2][kRows];    // [key half][row] scratch shared by the two threads of a row
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void settle_ns(uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < ns) {
  }
}

// Page ids of the current sequence, 32 at a time, one per lane of the warp.
struct PageWindow {
  const int32_t* row;
  int hi, base, val, num_pages;
  int32_t* status;

  __device__ void reset(const int32_t* r, int h, int np, int32_t* st) {
    row = r;
    hi = h;
    base = -1;
    val = 0;
    num_pages = np;
    status = st;
  }
  // All 32 lanes call this with the same `pg`.
  __device__ int get(int pg) {
    const int lane = threadIdx.x & 31;
    const int b = pg & ~31;
    if (b != base) {
      base = b;
      const int idx = b + lane;
      val = idx < hi ? __ldg(row + idx) : num_pages;
    }
    int v = __shfl_sync(0xffffffffu, val, pg & 31);
    if (pg >= hi) return num_pages;               // absent second page: zero-filled box
    if (v < 0 || v >= num_pages) {                // corrupt id: never read out of bounds
      if (lane == 0) record_status(status, MLA_ERR_BAD_INPUT);
      v = num_pages;
    }
    return v;
  }
};

// ------------------------------------------------------------------ loads
// Warp 4: Q at each segment start, then the nine 64-column boxes of this CTA's
// page of every tile, for the score product.
__device__ void score_loads(const PairMaps& maps, const DecodeArgs& a, Ctrl& ct,
                            uint8_t* qs, uint8_t* ks, const Ctl& ctl, uint32_t rank, int rb, int g,
                            const int32_t* md, uint32_t leader_q_full, uint32_t leader_k_full0) {
  const int lane = threadIdx.x & 31;
  const int hg = a.hg;
  const int r0 = rb * kRows;
  const int q_h0 = hg >= kRows ? r0 % hg : 0;
  const int q_s0 = r0 / hg;
  const bool leader = rank == 0;
  uint32_t kidx = 0;
  int qloads = 0;
  bool alive = true;
  auto wait_uniform = [&](uint64_t* bar, uint32_t parity) -> bool {
    int ok = 1;
    if (lane == 0) ok = wait_phase(bar, parity, ctl) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };
  SegIter it;
  it.init(md);
  Seg s;
  PageWindow win;
  while (alive && it.next(a, s)) {
    if (s.ntiles == 0) continue;
    if (qloads > 0 && !wait_uniform(&ct.q_empty, (qloads - 1) & 1)) { alive = false; break; }
    if (lane == 0) {
      if (leader) mbar_arrive_expect_tx(&ct.q_full, 2 * kQBytes);
      tma_load_5d_pair(qs, &maps.q, leader_q_full, 0, q_h0, g, s.b * a.s_q + q_s0, 0);
    }
    ++qloads;
    const int32_t* bt_row = a.block_table + static_cast<size_t>(s.b) * a.max_pages;
    win.reset(bt_row, s.hi, a.num_pages, a.status);
#pragma unroll 1
    for (int t = 0; t < s.ntiles && alive; ++t) {
      const int pid = win.get(s.lo + 2 * t + static_cast<int>(rank));
#pragma unroll 1
      for (int j = 0; j < 3; ++j) {
        const uint32_t slot = kidx % kKSlots;
        if (kidx >= static_cast<uint32_t>(kKSlots) && !wait_uniform(&ct.k_empty[slot], ((kidx / kKSlots) - 1) & 1)) {
          alive = false;
          break;
        }
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&ct.k_full[slot], 2 * kKSlotBytes);
          tma_load_4d_pair(ks + slot * kKSlotBytes, &maps.k, leader_k_full0 + slot * 8, 0, 64 * pid, 3 * j, g);
        }
        ++kidx;
      }
    }
  }
  __syncwarp();
}

// Warp 5: for the value product of every tile, this CTA's 128 dv columns of each
// dv half, page by page and half by half: one 16 KB slot [chunk][64 tokens][64 cols].
__device__ void value_loads(const PairMaps& maps, const DecodeArgs& a, Ctrl& ct, uint8_t* vs, const Ctl& ctl,
                            uint32_t rank, int g, const int32_t* md, uint32_t leader_v_full0) {
  const int lane = threadIdx.x & 31;
  const bool leader = rank == 0;
  uint32_t vidx = 0;
  bool alive = true;
  auto wait_uniform = [&](uint64_t* bar, uint32_t parity) -> bool {
    int ok = 1;
    if (lane == 0) ok = wait_phase(bar, parity, ctl) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };
  SegIter it;
  it.init(md);
  Seg s;
  PageWindow win;
  while (alive && it.next(a, s)) {
    if (s.ntiles == 0) continue;
    win.reset(a.block_table + static_cast<size_t>(s.b) * a.max_pages, s.hi, a.num_pages, a.status);
#pragma unroll 1
    for (int t = 0; t < s.ntiles && alive; ++t) {
      const int pid0 = win.get(s.lo + 2 * t), pid1 = win.get(s.lo + 2 * t + 1);
#pragma unroll 1
      for (int u = 0; u < 4; ++u) {     // page u / 2 of the tile, dv half u % 2
        const uint32_t slot = vidx % kVSlots;
        if (vidx >= static_cast<uint32_t>(kVSlots) && !wait_uniform(&ct.v_empty[slot], ((vidx / kVSlots) - 1) & 1)) {
          alive = false;
          break;
        }
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&ct.v_full[slot], 2 * kVSlotBytes);
          tma_load_5d_pair(vs + slot * kVSlotBytes, &maps.v[rank], leader_v_full0 + slot * 8, 0,
                           64 * ((u >> 1) ? pid1 : pid0), 0, u & 1, g);
        }
        ++vidx;
      }
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------------ MMA (leader CTA, three threads)
// Lane 0 of warps 6 and 7 issue the score products: ROLE 0 the first 18 K steps of every tile into
// partial S 0, ROLE 1 the last 18 into partial S 1.  Lane 0 of warp 8 (ROLE 2) issues the value
// products.  The commit and barrier stalls of one issuer are hidden behind the others' MMAs, and
// each issuer alone is fast enough for its share of the tile.
template <int T, int ROLE>
__device__ bool mma_issue(const DecodeArgs& a, Ctrl& ct, uint8_t* qs, uint8_t* ps, uint8_t* ks, uint8_t* vs,
                          uint32_t tmem, const Ctl& ctl, const int32_t* md) {
  constexpr bool kValue = ROLE == 2;
  const uint32_t idesc_qk = idesc_f32<T>(128, 128, false, false);   // A = Q (K-major), B = K (K-major)
  const uint32_t idesc_pv = idesc_f32<T>(128, 256, false, true);    // A = P (K-major), B = V (MN-major)
  const uint32_t q_addr = smem_addr(qs), p_addr = smem_addr(ps), k_addr = smem_addr(ks), v_addr = smem_addr(vs);
  uint32_t vidx = 0;
  int tg = 0, qloads = 0, seg_i = 0;   // seg_i: segments with tiles issued so far
  SegIter it;
  it.init(md);
  Seg s;
  while (it.next(a, s)) {
    const int tg0 = tg;
    if (s.ntiles == 0) continue;   // nothing to issue; its epilogue does not touch O in TMEM
    if constexpr (!kValue) {
      if (!wait_phase_lean(&ct.q_full, qloads & 1, ctl)) return false;
      ++qloads;
      tc_fence_after();
#pragma unroll 1
      for (int t = 0; t < s.ntiles; ++t) {
        const int tgl = tg0 + t, sb = tgl & 1;
        if (tgl >= 2 && !wait_phase_lean(&ct.s_free[sb], ((tgl >> 1) - 1) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + kColS + 128 * ROLE + 64 * sb;
        constexpr int k0 = ROLE * kKStepsPerIssuer;
#pragma unroll
        for (int j = k0 / 12; j <= (k0 + kKStepsPerIssuer - 1) / 12; ++j) {
          // slot j holds latent chunks 3j .. 3j+2 of this CTA's page (every slot is loaded once a tile)
          if (!wait_phase_lean(&ct.k_full[j], tgl & 1, ctl)) return false;
          tc_fence_after();
#pragma unroll
          for (int k = (k0 > 12 * j ? k0 : 12 * j); k < (k0 + kKStepsPerIssuer < 12 * j + 12 ? k0 + kKStepsPerIssuer : 12 * j + 12); ++k) {
            const int c = k >> 2, kk = k & 3;      // latent chunk (0..8) and its 16-column step
            const uint64_t ad = smem_desc(q_addr + c * kBox + kk * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(k_addr + j * kKSlotBytes + (c - 3 * j) * kBox + kk * 32, 16, 1024, 2);
            umma_bf16_pair(d_tmem, ad, bd, idesc_qk, k != k0 ? 1u : 0u);
          }
          umma_commit_pair(&ct.k_empty[j]);
        }
        umma_commit_pair(&ct.s_full[sb]);
        if (t == s.ntiles - 1) umma_commit_pair(&ct.q_empty);
      }
    } else {
#pragma unroll 1
      for (int t = 0; t < s.ntiles; ++t) {
        const int tgl = tg0 + t, pb = tgl & 1;
        // O in TMEM is overwritten from the first value product of a segment on: wait until the
        // softmax has read out the previous segment that had tiles (one o_free phase per such segment)
        if (t == 0 && seg_i > 0 && !wait_phase_lean(&ct.o_free, (seg_i - 1) & 1, ctl)) return false;
        if (!wait_phase_lean(&ct.p_full[pb], (tgl >> 1) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t pbase = p_addr + (tgl % kPBufs) * kPBytes;
#pragma unroll 1
        for (int u = 0; u < 4; ++u) {       // page q = u / 2 of the tile, dv half h = u % 2
          const int q = u >> 1, h = u & 1;
          const uint32_t slot = vidx % kVSlots;
          if (!wait_phase_lean(&ct.v_full[slot], (vidx / kVSlots) & 1, ctl)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // A = P: 128 rows (64 per CTA) x 16 keys of page q, K-major
            const uint64_t ad = smem_desc(pbase + q * kBox + kk * 32, 16, 1024, 2);
            // B = V: 16 keys x 256 dv (128 per CTA: two chunks 8 KB apart), MN-major
            const uint64_t bd = smem_desc(v_addr + slot * kVSlotBytes + kk * 2048, kBox, 1024, 2);
            umma_bf16_pair(tmem + kColO + 128 * h, ad, bd, idesc_pv, (t > 0 || q > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit_pair(&ct.v_empty[slot]);
          ++vidx;
        }
        umma_commit_pair(&ct.p_free[pb]);
      }
    }
    tg += s.ntiles;
    ++seg_i;
  }
  return true;
}

// ------------------------------------------------------------------ softmax + epilogue (warps 0-3)
template <int T>
__device__ void softmax_rows(const DecodeArgs& a, Ctrl& ct, uint8_t* ps, uint32_t tmem, const Ctl& ctl,
                             uint32_t rank, int rb, int g, const int32_t* md, uint32_t leader_s_free0,
                             uint32_t leader_p_full0, uint32_t leader_o_free) {
  const int tid = threadIdx.x;                 // TMEM lane
  const int warp = tid >> 5, lane = tid & 31;
  const int r = tid & 63, kh = tid >> 6;       // row of this CTA, key half / dv quarter
  const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
  const int rr = rb * kRows + r;               // row within the KV head group
  const bool row_valid = rr < a.R;
  const int hg = a.hg;
  const int srow = row_valid ? rr / hg : 0;
  const int head = g * hg + (row_valid ? rr % hg : 0);

  auto uniform_ok = [&](bool ok) -> bool {
    if (!ok) ct.softmax_abort = 1;
    named_sync(kSoftmaxBar, 128);
    return ct.softmax_abort == 0;
  };
  if (a.debug_flags & 1) {
    if (!uniform_ok(wait_phase(&ct.never, 0, ctl))) return;
  }

  int tg = 0;
  SegIter it;
  it.init(md);
  Seg s;
  while (it.next(a, s)) {
    int kmax = 0;
    if (row_valid && s.ok) {
      const int seg_end = min(s.hi * 64, s.L);
      const int lim = a.causal ? s.L - (a.s_q - 1 - srow) : s.L;
      kmax = min(seg_end, lim);
    }
    if (!s.ok && tid == 0) record_status(a.status, MLA_ERR_BAD_INPUT);
    float m_run = -INFINITY, lsum = 0.f;

#pragma unroll 1
    for (int t = 0; t < s.ntiles; ++t, ++tg) {
      const int sb = tg & 1;
      bool ok = wait_phase(&ct.s_full[sb], (tg >> 1) & 1, ctl);
      float x[64];
      bool need = false;
      float mloc = -INFINITY;
      if (ok) {
        tc_fence_after();
        // S = partial 0 + partial 1 (the two score issuers' halves of the 576 columns)
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tmem + lane_base + kColS + 64 * sb + 16 * c16, v0);
          tmem_ld16(tmem + lane_base + kColS + 128 + 64 * sb + 16 * c16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) x[16 * c16 + i] = __uint_as_float(v0[i]) + __uint_as_float(v1[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(leader_s_free0 + sb * 8);
        const int nvis = kmax - ((s.lo + 2 * t) * 64 + 64 * kh);   // visible keys of this half
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (nvis >= 64) {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            x[j] *= a.scale_log2;
            m4[j & 3] = fmaxf(m4[j & 3], x[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            x[j] = j < nvis ? x[j] * a.scale_log2 : -INFINITY;
            m4[j & 3] = fmaxf(m4[j & 3], x[j]);
          }
        }
        mloc = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        need = mloc > m_run + kTau;
      }
      if (!ok) ct.softmax_abort = 1;
      need = named_sync_or(kSoftmaxBar, 128, need);
      if (ct.softmax_abort) return;

      if (need) {
        ct.red[kh][r] = mloc;
        named_sync(kSoftmaxBar, 128);
        const float mt = fmaxf(ct.red[0][r], ct.red[1][r]);
        const float mn = fmaxf(m_run, mt);
        const float alpha = m_run == -INFINITY ? (mn == -INFINITY ? 1.f : 0.f) : ex2(m_run - mn);
        m_run = mn;
        lsum *= alpha;
        if (t > 0) {
          // O holds tiles < t: wait for the value product of tile tg-1, then rescale O in TMEM
          const bool okr = wait_phase(&ct.p_free[(tg - 1) & 1], ((tg - 1) >> 1) & 1, ctl);
          if (!uniform_ok(okr)) return;
          tc_fence_after();
#pragma unroll 1
          for (int c16 = 0; c16 < 16; ++c16) {     // this lane's 256 O columns (both dv halves)
            uint32_t v[16];
            const uint32_t ta = tmem + lane_base + kColO + 16 * c16;
            tmem_ld16(ta, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
            tmem_st16(ta, v);
          }
          tmem_wait_st();
        }
        named_sync(kSoftmaxBar, 128);              // red[] is reused by the next tile
      }

      // P row slice: 64 keys of this thread's half, 128 bytes, 128-byte swizzle.
      // exp2(-inf - m) = 0 for masked keys; m_run is finite once a key was seen.
      const float mneg = m_run == -INFINITY ? 0.f : -m_run;
      uint32_t w[32];
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        w[i] = pack2<T>(ex2(x[2 * i] + mneg), ex2(x[2 * i + 1] + mneg));
        l4[i & 3] += unpack_lo<T>(w[i]) + unpack_hi<T>(w[i]);
      }
      lsum += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      // this tile's P buffer is free once the value product of tile tg - kPBufs has finished with it
      if (tg >= kPBufs &&
          !uniform_ok(wait_phase(&ct.p_free[(tg - kPBufs) & 1], ((tg - kPBufs) >> 1) & 1, ctl)))
        return;
      uint8_t* prow = ps + (tg % kPBufs) * kPBytes + kh * kBox + r * 128;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8)
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (r & 7)) << 4)) =
            make_uint4(w[4 * c8], w[4 * c8 + 1], w[4 * c8 + 2], w[4 * c8 + 3]);
      fence_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_p_full0 + (tg & 1) * 8);
    }

    // ---------------- epilogue of the segment
    if (s.ntiles > 0) {
      const int tl = tg - 1;
      const bool okw = wait_phase(&ct.p_free[tl & 1], (tl >> 1) & 1, ctl);
      if (!uniform_ok(okw)) return;
      tc_fence_after();
    }
    ct.red[kh][r] = lsum;
    named_sync(kSoftmaxBar, 128);
    const float l = ct.red[0][r] + ct.red[1][r];
    const bool any = l > 0.f;
    const float inv = any ? 1.f / l : 0.f;
    const float lse = any ? (m_run + log2f(l)) * kLn2 : -INFINITY;
    named_sync(kSoftmaxBar, 128);

    const int npieces = __ldg(a.num_splits + s.b + 1) - __ldg(a.num_splits + s.b);
    const bool final_out = npieces == 1;
    const bool can_write = row_valid && (final_out || s.piece < a.max_pieces);
    if (!final_out && s.piece >= a.max_pieces && tid == 0) record_status(a.status, MLA_ERR_BAD_INPUT);
#pragma unroll 1
    for (int c32 = 0; c32 < 8; ++c32) {      // 32 O columns at a time: dv half c32 / 4
      float v[32];
      if (s.ntiles > 0) {
        uint32_t u0[16], u1[16];
        tmem_ld16(tmem + lane_base + kColO + 32 * c32, u0);
        tmem_ld16(tmem + lane_base + kColO + 32 * c32 + 16, u1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          v[i] = __uint_as_float(u0[i]) * inv;
          v[16 + i] = __uint_as_float(u1[i]) * inv;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (can_write) {
        // this thread's dv columns: 128 contiguous values of its row in each dv half
        const int dv0 = 256 * (c32 >> 2) + 128 * kh + 32 * (c32 & 3);
        if (final_out) {
          uint4* dst = reinterpret_cast<uint4*>(
              static_cast<uint16_t*>(a.out) + ((static_cast<size_t>(s.b) * a.s_q + srow) * a.h_q + head) * 512 + dv0);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(pack2<T>(v[8 * k], v[8 * k + 1]), pack2<T>(v[8 * k + 2], v[8 * k + 3]),
                                pack2<T>(v[8 * k + 4], v[8 * k + 5]), pack2<T>(v[8 * k + 6], v[8 * k + 7]));
        } else {
          float4* dst = reinterpret_cast<float4*>(
              a.o_part + ((static_cast<size_t>(s.piece) * a.h_kv + g) * a.R + rr) * 512 + dv0);
#pragma unroll
          for (int k = 0; k < 8; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        }
      }
    }
    if (kh == 0 && can_write) {
      if (final_out)
        a.lse[(static_cast<size_t>(s.b) * a.s_q + srow) * a.h_q + head] = lse;
      else
        a.lse_part[(static_cast<size_t>(s.piece) * a.h_kv + g) * a.R + rr] = lse;
    }
    // O may be overwritten again: signalled only after segments that had tiles, the ones whose O came
    // from TMEM, so the value issuer (which waits once per such segment) can never be lapped
    if (s.ntiles > 0) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_o_free);
    }
  }
}

template <int T>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mla_decode_pair_kernel(const __grid_constant__ PairMaps maps, const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* qs = smem;
  uint8_t* ps = smem + kOffP;
  uint8_t* ks = smem + kOffK;
  uint8_t* vs = smem + kOffV;
  Ctrl& ct = *reinterpret_cast<Ctrl*>(smem + kOffCtrl);

  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_ctarank();
  const int rb = blockIdx.x;                    // row block of 64 rows; the pair is (2i, 2i+1)
  const int g = blockIdx.y, part = blockIdx.z;
  const int32_t* md = a.tile_md + static_cast<size_t>(part) * MLA_MD_WORDS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKSlots; ++i) {
      mbar_init(&ct.k_full[i], 1);
      // slot 1 is read by both score issuers, slots 0 and 2 by one each
      mbar_init(&ct.k_empty[i], (12 * i < kKStepsPerIssuer && 12 * i + 12 > kKStepsPerIssuer) ? 2 : 1);
    }
    for (int i = 0; i < kVSlots; ++i) {
      mbar_init(&ct.v_full[i], 1);
      mbar_init(&ct.v_empty[i], 1);
    }
    mbar_init(&ct.q_full, 1);
    mbar_init(&ct.q_empty, 2);        // both score issuers read Q
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ct.s_full[i], 2);    // both partial sums
      mbar_init(&ct.s_free[i], 8);    // one arrival per softmax warp of both CTAs
      mbar_init(&ct.p_full[i], 8);
      mbar_init(&ct.p_free[i], 1);
    }
    mbar_init(&ct.o_free, 8);
    mbar_init(&ct.never, 1);
    for (int i = 0; i < 3; ++i) mbar_init(&ct.drain[i], 1);
    ct.abort_flag = 0;
    ct.softmax_abort = 0;
    fence_barrier_init();
  }
  if (warp == 6) {
    tmem_alloc_pair(&ct.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 4 && (threadIdx.x & 31) == 0) {
    tma_prefetch_map(&maps.k);
    tma_prefetch_map(&maps.q);
    tma_prefetch_map(&maps.v[0]);
    tma_prefetch_map(&maps.v[1]);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();           // barriers of both CTAs initialised before any remote arrive or load
  tc_fence_after();
  pdl_trigger();            // the combine may start launching; it waits for this grid to finish
  pdl_wait();               // the part table and piece counts come from the metadata kernel
  const uint32_t tmem = ct.tmem_base;
  const Ctl ctl{&ct.abort_flag, a.status, a.timeout_ns};
  // barriers of the leader CTA, in the cluster shared window
  const uint32_t L_q_full = mapa_shared(smem_addr(&ct.q_full), 0);
  const uint32_t L_k_full0 = mapa_shared(smem_addr(&ct.k_full[0]), 0);
  const uint32_t L_v_full0 = mapa_shared(smem_addr(&ct.v_full[0]), 0);
  const uint32_t L_s_free0 = mapa_shared(smem_addr(&ct.s_free[0]), 0);
  const uint32_t L_p_full0 = mapa_shared(smem_addr(&ct.p_full[0]), 0);
  const uint32_t L_o_free = mapa_shared(smem_addr(&ct.o_free), 0);

  if (warp < 4) {
    softmax_rows<T>(a, ct, ps, tmem, ctl, rank, rb, g, md, L_s_free0, L_p_full0, L_o_free);
  } else if (warp == 4) {
    score_loads(maps, a, ct, qs, ks, ctl, rank, rb, g, md, L_q_full, L_k_full0);
  } else if (warp == 5) {
    value_loads(maps, a, ct, vs, ctl, rank, g, md, L_v_full0);
  } else {
    if (rank == 0 && (threadIdx.x & 31) == 0) {
      const int role = warp - 6;
      if (role == 0) (void)mma_issue<T, 0>(a, ct, qs, ps, ks, vs, tmem, ctl, md);
      else if (role == 1) (void)mma_issue<T, 1>(a, ct, qs, ps, ks, vs, tmem, ctl, md);
      else (void)mma_issue<T, 2>(a, ct, qs, ps, ks, vs, tmem, ctl, md);
      // every MMA this thread issued has finished, and its commits have landed, before TMEM is
      // freed and the pair exits (the softmax has waited for them unless the pair is aborting)
      umma_commit_pair_leader(&ct.drain[role]);
      drain_phase(&ct.drain[role], 0, 1000000000ull);
    }
    __syncwarp();
  }
  __syncthreads();
  if (ct.abort_flag) settle_ns(200000);   // let loads already issued land before the pair exits
  tc_fence_before();
  cluster_sync();
  if (warp == 6) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

int decode_pair_smem_bytes() { return kSmemBytes; }

template <int T>
static cudaError_t launch_pair_t(const PairMaps& maps, const DecodeArgs& a, int row_blocks, cudaStream_t stream) {
  static std::atomic<uint64_t> configured{0};
  const cudaError_t e = set_smem_limit_once(mla_decode_pair_kernel<T>, kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  const int pairs = (row_blocks + 1) / 2;
  const dim3 grid(2 * pairs, a.h_kv, a.num_parts);
  return launch_pdl(mla_decode_pair_kernel<T>, grid, dim3(kThreads), kSmemBytes, stream, maps, a);
}

cudaError_t launch_decode_pair(int dtype, const PairMaps& maps, const DecodeArgs& a, int row_blocks,
                               cudaStream_t stream) {
  if (dtype == kFP16) return launch_pair_t<kFP16>(maps, a, row_blocks, stream);
  return launch_pair_t<kBF16>(maps, a, row_blocks, stream);
}

}  // namespace mla
