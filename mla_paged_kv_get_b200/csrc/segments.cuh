// segments.cuh — how every role of a decode CTA walks its scheduler part.
//
// A part (one tile-scheduler entry) is a page range in (sequence, page) order;
// it is cut into segments, one per sequence it touches.  Each segment is one
// "piece" of that sequence: piece ids are consecutive from the entry's
// first_piece.  All roles (loads, MMA, softmax) enumerate exactly the same
// segments from the same data, so their pipelines stay in step.
#pragma once

#include "decode.cuh"

namespace mla {

// One (sequence, page range) piece of a part, as every role enumerates it.
struct Seg {
  int b, lo, hi, L, ntiles, piece;
  bool ok;
};

struct SegIter {
  int b, begin_b, begin_page, end_b, end_page, piece;

  __device__ void init(const int32_t* md) {
    begin_b = __ldg(md + 0);
    begin_page = __ldg(md + 1);
    end_b = __ldg(md + 2);
    end_page = __ldg(md + 3);
    piece = __ldg(md + 4);
    b = begin_b;
  }

  __device__ bool next(const DecodeArgs& a, Seg& s) {
    while (b < a.batch && (b < end_b || (b == end_b && end_page > 0))) {
      const int cur = b++;
      const int L = __ldg(a.seqlens + cur);
      const int nb = L > 0 ? (L + 63) / 64 : 0;
      const int lo = cur == begin_b ? begin_page : 0;
      const int hi = cur == end_b ? end_page : nb;
      if (hi <= lo) continue;
      s.b = cur;
      s.lo = lo;
      s.L = L;
      s.piece = piece++;
      s.ok = L <= a.max_pages * 64 && hi <= nb;
      s.hi = s.ok ? hi : lo;
      s.ntiles = s.ok ? (hi - lo + 1) / 2 : 0;
      return true;
    }
    return false;
  }
};

}  // namespace mla
