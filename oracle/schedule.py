"""Integer restatement of the tile scheduler (metadata) for bit-exact checks.

TEST INFRASTRUCTURE ONLY: the CUDA library implements the same rule on the
GPU from its prose statement; the two share no code.

The pages name the idea only: work is cut into blocks and scheduled over the
GPU in parallel (jsxs2.com "什麼是FlashMLA", §3.1 分塊調度與並行計算), and
the metadata call takes the per-sequence lengths plus ``s_q*h_q//h_kv`` and
``h_kv`` and returns ``tile_scheduler_metadata, num_splits`` (cnblogs
"DeepSeek 开源记-第1天-FlashMLA", §6.2 基本使用).  The concrete rule below is
this project's reading of them:

* rows per KV head ``R = s_q*h_q/h_kv`` are cut into row blocks of
  ``N = 16`` (R <= 16), ``32`` (R <= 32) or ``64`` rows; ``T = ceil(R/N)``;
* ``G_max = max(1, num_sms // (h_kv*T))`` parts at most (the launch grid);
* the cost line: sequence ``b`` with ``n_b = ceil(L_b/64)`` pages occupies
  ``c_b = C + n_b`` units (0 if empty), ``C = 4`` units of per-sequence
  overhead first, then one unit per page; ``P_b`` is the prefix sum of the
  ``c_b`` and ``total = P_B``;
* the number of parts in use ``G`` is chosen among ``[ceil(G_max/2), G_max]``:
  with ``W(G) = max(1, ceil(total / G))``, sequence ``b`` is *split* by ``G``
  when its first and last page fall in different parts
  (``min(unit // W, G-1)`` differs for ``P_b + C`` and ``P_b + C + n_b - 1``);
  ``cost(G) = W(G) + S`` if any sequence is split, else ``W(G)``, with
  ``S = 12`` pages (a split costs the merge pass); ``G`` minimises the cost,
  the largest ``G`` on ties.  When ``B * (number of candidates)`` exceeds
  32768, or ``total >= 2**31``, the search is skipped and ``G = G_max``;
* ``W = W(G)``; part ``p < G`` owns units ``[p*W, (p+1)*W)``, part ``G-1``
  everything from ``(G-1)*W`` on, and parts ``G .. G_max-1`` are empty;
* page ``j`` of sequence ``b`` goes to the part owning unit ``P_b + C + j``;
* ``pos(U)``: the first (sequence, page) whose unit is ``>= U`` (``(B, 0)``
  past the end); ``tile_md[p] = (begin_b, begin_page, end_b, end_page,
  first_piece, n_pieces, 0, 0)`` with ``begin = pos(p*W)`` and
  ``end = pos((p+1)*W)`` (``(B, 0)`` for part ``G-1``), end exclusive; an
  empty part ``p >= G`` is ``(B, 0, B, 0, total pieces, 0, 0, 0)``;
* a piece is a (part, sequence) pair with at least one page; pieces are
  numbered part by part, sequences in order within a part; ``first_piece``
  is the number of pieces in earlier parts; ``num_splits`` is the prefix sum
  (length ``B + 1``) of the number of pieces of each sequence.

No floating point anywhere.
"""

from __future__ import annotations

SPLIT_OVERHEAD_PAGES = 4   # C
SPLIT_PENALTY_PAGES = 12   # S
SEARCH_BUDGET = 32768      # (sequences x candidate part counts) examined at most
PAGE = 64
MD_WORDS = 8


def rows_per_block(rows_per_kv: int) -> int:
    if rows_per_kv <= 16:
        return 16
    if rows_per_kv <= 32:
        return 32
    return 64


def num_row_blocks(rows_per_kv: int) -> int:
    n = rows_per_block(rows_per_kv)
    return (rows_per_kv + n - 1) // n


def num_parts(rows_per_kv: int, h_kv: int, num_sms: int) -> int:
    return max(1, num_sms // (h_kv * num_row_blocks(rows_per_kv)))


def _pages(seqlens):
    return [(int(L) + PAGE - 1) // PAGE if int(L) > 0 else 0 for L in seqlens]


def parts_in_use(n, start, total, G_max: int) -> int:
    """The number of parts G the rule picks (see the module docstring)."""
    C, S = SPLIT_OVERHEAD_PAGES, SPLIT_PENALTY_PAGES
    lo = max(1, (G_max + 1) // 2)
    if len(n) * (G_max - lo + 1) > SEARCH_BUDGET or total >= 1 << 31:
        return G_max
    best_cost, best_G = None, G_max
    for G in range(lo, G_max + 1):
        W = max(1, (total + G - 1) // G)
        split = False
        for b in range(len(n)):
            if n[b] > 0:
                first = start[b] + C
                last = first + n[b] - 1
                if min(first // W, G - 1) != min(last // W, G - 1):
                    split = True
                    break
        cost = W + (S if split else 0)
        if best_cost is None or cost <= best_cost:
            best_cost, best_G = cost, G
    return best_G


def get_metadata(seqlens, rows_per_kv: int, h_kv: int, num_sms: int):
    """Return ``(tile_md, num_splits)`` as lists of Python ints."""
    C = SPLIT_OVERHEAD_PAGES
    n = _pages(seqlens)
    B = len(n)
    G_max = num_parts(rows_per_kv, h_kv, num_sms)
    start = []          # P_b
    acc = 0
    for nb in n:
        start.append(acc)
        acc += nb + C if nb > 0 else 0
    total = acc
    G = parts_in_use(n, start, total, G_max)
    W = max(1, (total + G - 1) // G)

    def part_of(unit):
        return min(unit // W, G - 1)

    # every page, in order, to its part
    owner = {}
    for b in range(B):
        for j in range(n[b]):
            owner[(b, j)] = part_of(start[b] + C + j)

    def pos(U):
        for b in range(B):
            if n[b] > 0 and start[b] + n[b] + C > U:
                return (b, max(0, U - start[b] - C))
        return (B, 0)

    tile_md = []
    first = 0
    for p in range(G):
        begin = pos(p * W)
        end = pos((p + 1) * W) if p < G - 1 else (B, 0)
        pieces = sorted({b for (b, j), q in owner.items() if q == p})
        tile_md.append([begin[0], begin[1], end[0], end[1], first, len(pieces), 0, 0])
        first += len(pieces)
    for p in range(G, G_max):
        tile_md.append([B, 0, B, 0, first, 0, 0, 0])

    num_splits = [0]
    for b in range(B):
        parts = {owner[(b, j)] for j in range(n[b])}
        num_splits.append(num_splits[-1] + len(parts))
    return tile_md, num_splits


def part_segments(md_row, seqlens):
    """The (sequence, page_lo, page_hi) pieces a part covers, in order."""
    begin_b, begin_page, end_b, end_page = md_row[:4]
    n = _pages(seqlens)
    out = []
    b = begin_b
    while b < len(n) and (b < end_b or (b == end_b and end_page > 0)):
        lo = begin_page if b == begin_b else 0
        hi = end_page if b == end_b else n[b]
        if hi > lo:
            out.append((b, lo, hi))
        b += 1
    return out
