"""Integer restatement of the tile scheduler (metadata) for bit-exact checks.

TEST INFRASTRUCTURE ONLY: the CUDA library implements the same rule on the
GPU from its prose statement; the two share no code.

The pages name the idea only: work is cut into blocks and scheduled over the
GPU in parallel (jsxs2.com "什麼是FlashMLA", §3.1 分塊調度與並行計算), and
the metadata call takes the per-sequence lengths plus ``s_q*h_q//h_kv`` and
``h_kv`` and returns ``tile_scheduler_metadata, num_splits`` (cnblogs
"DeepSeek 开源记-第1天-FlashMLA", §6.2 基本使用).  The concrete rule below is
this project's reading, stated in full in DESIGN.md ("Scheduler rule"):

* rows per KV head ``R = s_q*h_q/h_kv`` are cut into row blocks of
  ``N = 16`` (R <= 16), ``32`` (R <= 32) or ``64`` rows; ``T = ceil(R/N)``;
* ``G = max(1, num_sms // (h_kv*T))`` parts; each part is one CTA per
  (row block, KV head);
* sequence ``b`` has ``n_b = ceil(L_b/64)`` pages and costs
  ``c_b = n_b + C`` (0 if empty), ``C = 4`` pages of per-piece overhead;
* capacity ``W = ceil(sum_b c_b / G) + C``;
* parts ``0..G-2`` are filled in order: whole sequences while
  ``rest + C <= remaining``; otherwise ``remaining - C`` pages of the
  current sequence (if that is at least 1) and the part closes;
* the last part takes everything left;
* ``tile_md[p] = (begin_b, begin_page, end_b, end_page, first_piece,
  n_pieces, 0, 0)`` with the end exclusive in (sequence, page) order;
* pieces are numbered in sweep order; ``num_splits`` is the prefix sum of the
  number of pieces per sequence (length ``B + 1``).

No floating point anywhere.
"""

from __future__ import annotations

SPLIT_OVERHEAD_PAGES = 4   # C
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


def get_metadata(seqlens, rows_per_kv: int, h_kv: int, num_sms: int):
    """Return ``(tile_md, num_splits)`` as lists of Python ints.

    ``tile_md`` has ``G`` rows of 8 words; ``num_splits`` has ``B + 1``
    entries.
    """
    C = SPLIT_OVERHEAD_PAGES
    lens = [int(x) for x in seqlens]
    B = len(lens)
    G = num_parts(rows_per_kv, h_kv, num_sms)
    n = [(L + PAGE - 1) // PAGE if L > 0 else 0 for L in lens]
    total = sum(nb + C for nb in n if nb > 0)
    W = (total + G - 1) // G + C

    tile_md = []
    pieces_of = [0] * B
    b, page, piece = 0, 0, 0
    for p in range(G):
        begin_b, begin_page, first_piece = b, page, piece
        if p == G - 1:
            while b < B:
                if n[b] > page:
                    pieces_of[b] += 1
                    piece += 1
                b, page = b + 1, 0
        else:
            remaining = W
            while b < B:
                if n[b] == 0:
                    b, page = b + 1, 0
                    continue
                rest = n[b] - page
                if rest + C <= remaining:
                    remaining -= rest + C
                    pieces_of[b] += 1
                    piece += 1
                    b, page = b + 1, 0
                else:
                    take = remaining - C
                    if take >= 1:
                        page += take
                        pieces_of[b] += 1
                        piece += 1
                    break
        tile_md.append([begin_b, begin_page, b, page, first_piece, piece - first_piece, 0, 0])

    num_splits = [0]
    for b in range(B):
        num_splits.append(num_splits[-1] + pieces_of[b])
    return tile_md, num_splits


def part_segments(md_row, seqlens):
    """The (sequence, page_lo, page_hi) pieces a part covers, in order."""
    begin_b, begin_page, end_b, end_page = md_row[:4]
    out = []
    b = begin_b
    while b < len(seqlens) and (b < end_b or (b == end_b and end_page > 0)):
        L = int(seqlens[b])
        nb = (L + PAGE - 1) // PAGE if L > 0 else 0
        lo = begin_page if b == begin_b else 0
        hi = end_page if b == end_b else nb
        if hi > lo:
            out.append((b, lo, hi))
        b += 1
    return out
