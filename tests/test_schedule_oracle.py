"""Pins of the integer scheduler restatement: hand-worked cases and invariants."""

import json
import os
import random

import pytest

from oracle import schedule as sch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_worked_cases():
    cases = json.load(open(os.path.join(GOLDEN, "schedule_hand_cases.json")))["cases"]
    for c in cases:
        md, ns = sch.get_metadata(c["seqlens"], c["rows_per_kv"], c["h_kv"], c["num_sms"])
        assert md == c["tile_md"], c["derivation"]
        assert ns == c["num_splits"], c["derivation"]


def check_invariants(seqlens, rows_per_kv, h_kv, num_sms):
    md, ns = sch.get_metadata(seqlens, rows_per_kv, h_kv, num_sms)
    G_max = sch.num_parts(rows_per_kv, h_kv, num_sms)
    B = len(seqlens)
    C = sch.SPLIT_OVERHEAD_PAGES
    n = [(L + 63) // 64 for L in seqlens]
    total = sum(x + C for x in n if x > 0)
    # the parts in use (the choice itself is pinned by the hand cases and the equal-length case)
    starts = []
    acc = 0
    for x in n:
        starts.append(acc)
        acc += x + C if x > 0 else 0
    G = sch.parts_in_use(n, starts, total, G_max)
    assert (G_max + 1) // 2 <= G <= G_max
    assert all(md[p] == [B, 0, B, 0, md[p][4], 0, 0, 0] for p in range(G, G_max))
    W = max(1, (total + G - 1) // G)
    assert len(md) == G_max and len(ns) == B + 1 and ns[0] == 0
    covered = {}
    pieces_seen = [0] * B
    prev_end = (0, 0)
    piece = 0
    for p, row in enumerate(md):
        if p > 0:
            assert (row[0], row[1]) == prev_end        # contiguous, ordered
        assert (row[2], row[3]) >= (row[0], row[1])
        prev_end = (row[2], row[3])
        assert row[4] == piece
        segs = sch.part_segments(row, seqlens)
        assert row[5] == len(segs)
        pages = 0
        for (b, lo, hi) in segs:
            assert 0 <= lo < hi <= n[b]
            for pg in range(lo, hi):
                assert (b, pg) not in covered
                covered[(b, pg)] = p
            pieces_seen[b] += 1
            pages += hi - lo
        assert pages <= W                                # no part holds more than its units
        piece += len(segs)
    assert prev_end == (B, 0)
    assert set(covered) == {(b, pg) for b in range(B) for pg in range(n[b])}
    for b in range(B):
        assert ns[b + 1] - ns[b] == pieces_seen[b]
    assert ns[B] == piece
    return md, ns


@pytest.mark.parametrize("seed", range(40))
def test_invariants_random(seed):
    rng = random.Random(seed)
    B = rng.choice([1, 2, 3, 7, 64, 128, 132, 300])
    mode = rng.randrange(4)
    if mode == 0:
        lens = [rng.randint(0, 8192) for _ in range(B)]
    elif mode == 1:
        lens = [rng.choice([0, 1, 63, 64, 65, 127, 128]) for _ in range(B)]
    elif mode == 2:
        lens = [rng.randint(32768, 65536) for _ in range(B)]
    else:
        lens = [4096] * B
    rows = rng.choice([1, 16, 17, 32, 64, 128, 256])
    h_kv = rng.choice([1, 1, 2])
    sms = rng.choice([1, 7, 148])
    check_invariants(lens, rows, h_kv, sms)


def test_all_empty_and_single_token():
    md, ns = check_invariants([0, 0, 0], 16, 1, 148)
    assert ns == [0, 0, 0, 0]
    md, ns = check_invariants([1], 128, 1, 148)
    assert ns == [0, 1]


def test_equal_lengths_take_one_part_each():
    """64 sequences of 64 pages (68 units each) and at most 74 parts: 64 parts of 68 units
    hold one whole sequence each (cost 68), while any 65..74 parts are narrower than a
    sequence's 64 pages at some boundary and split one (cost >= 60 + 12); so 64 parts are
    used, each sequence is one piece, and parts 64..73 are empty."""
    lens = [4096] * 64
    md, ns = check_invariants(lens, 128, 1, 148)
    assert ns == list(range(65))
    assert all(md[p][:6] == [p, 0, p + 1, 0, p, 1] for p in range(64))
    assert all(md[p] == [64, 0, 64, 0, 64, 0, 0, 0] for p in range(64, 74))


def test_long_sequences_get_split():
    lens = [65536] * 8
    md, ns = check_invariants(lens, 128, 1, 148)
    G = sch.num_parts(128, 1, 148)
    assert G == 74
    assert ns[-1] > 8                     # most sequences must be cut
    C = sch.SPLIT_OVERHEAD_PAGES
    W = (sum(1024 + C for _ in lens) + G - 1) // G
    pages = [sum(hi - lo for (_, lo, hi) in sch.part_segments(r, lens)) for r in md]
    # every part but the last owns W units, of which at most C are overhead
    for p in range(G - 1):
        assert W - C <= pages[p] <= W


def test_row_block_rule():
    assert [sch.rows_per_block(r) for r in (1, 16, 17, 32, 33, 64, 128)] == [16, 16, 32, 32, 64, 64, 64]
    assert sch.num_row_blocks(128) == 2 and sch.num_row_blocks(16) == 1
    assert sch.num_parts(128, 1, 148) == 74 and sch.num_parts(16, 1, 148) == 148
