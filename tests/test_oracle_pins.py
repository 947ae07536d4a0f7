"""Pins of the fp64 oracle against facts fixed by the definition and the pages.

None of these tests re-types the oracle's formula: each checks a closed form,
an invariant, a special case that reduces to a textbook/library routine, or a
brute-force restatement on tiny inputs written with plain Python loops.
Several mutants of the oracle (planted mistakes, on the CPU) are shown to be
caught.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from mla_paged_kv_get_b200 import inputs
from oracle import mla_oracle as mo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np(w):
    return (w.q.float().double().numpy(), w.k_cache.float().double().numpy(),
            w.block_table.numpy().astype(np.int64), w.seqlens.numpy().astype(np.int64))


def _keys_by_loop(k_cache, bt_row, L, g):
    """Independent gather: token by token through the page table."""
    rows = []
    for j in range(L):
        page = int(bt_row[j // 64])
        rows.append(k_cache[page, j % 64, g, :])
    return np.array(rows).reshape(L, 576)


def test_closed_form_fixture():
    fx = json.load(open(os.path.join(GOLDEN, "decode_closed_form.json")))
    q = np.zeros((1, 1, 1, 576))
    q[0, 0, 0, 0] = 1.0
    k = np.zeros((2, 64, 1, 576))
    k[0, 0, 0, 0] = 1.0
    k[0, 0, 0, 1] = 2.0                        # token 0
    bt = np.array([[0, 1]])
    out, lse = mo.decode_dense(q, k, bt, np.array([fx["seqlen"]]), 1, False, math.log(3.0))
    assert abs(lse[0, 0, 0] - math.log(4.0)) < 1e-14
    expect = np.zeros(512)
    for i, v in fx["expected_out_nonzero"].items():
        expect[int(i)] = v
    assert np.abs(out[0, 0, 0] - expect).max() < 1e-14


def test_single_token_gives_v_and_score():
    w = inputs.build("one", [1, 1], s_q=1, h_q=16, seed=11)
    q, k, bt, sl = _np(w)
    out, lse = mo.decode_dense(q, k, bt, sl, 1, False, w.scale)
    for b in range(2):
        k0 = k[bt[b, 0], 0, 0]
        assert np.array_equal(out[b, 0], np.broadcast_to(k0[:512], (16, 512)))
        for h in range(16):
            x0 = w.scale * math.fsum(float(a) * float(c) for a, c in zip(q[b, 0, h], k0))
            assert abs(lse[b, 0, h] - x0) < 1e-12


def test_zero_query_gives_mean_and_log_n():
    w = inputs.build("zeroq", [37, 130], s_q=1, h_q=16, seed=12)
    q, k, bt, sl = _np(w)
    q[:] = 0.0
    out, lse = mo.decode_dense(q, k, bt, sl, 1, False, w.scale)
    for b, L in enumerate(sl):
        K = _keys_by_loop(k, bt[b], int(L), 0)
        mean = K[:, :512].sum(axis=0) / L
        assert np.abs(out[b, 0] - mean).max() < 1e-12
        assert np.abs(lse[b, 0] - math.log(L)).max() < 1e-12


def test_zero_scale_gives_mean():
    w = inputs.build("zeroscale", [70], s_q=1, h_q=16, seed=13)
    q, k, bt, sl = _np(w)
    out, lse = mo.decode_dense(q, k, bt, sl, 1, False, 0.0)
    K = _keys_by_loop(k, bt[0], 70, 0)
    assert np.abs(out[0, 0] - K[:, :512].mean(axis=0)).max() < 1e-12
    assert np.abs(lse[0, 0] - math.log(70)).max() < 1e-12


def test_identical_keys_give_v0_and_shifted_lse():
    w = inputs.build("same", [150], s_q=1, h_q=16, seed=14)
    q, k, bt, sl = _np(w)
    row = k[bt[0, 0], 0, 0].copy()
    for j in range(150):
        k[bt[0, j // 64], j % 64, 0] = row
    out, lse = mo.decode_dense(q, k, bt, sl, 1, False, w.scale)
    assert np.abs(out[0, 0] - row[:512]).max() < 1e-12
    for h in range(16):
        x0 = w.scale * math.fsum(float(a) * float(c) for a, c in zip(q[0, 0, h], row))
        assert abs(lse[0, 0, h] - (x0 + math.log(150))) < 1e-12


def test_weights_are_a_distribution():
    w = inputs.build("wts", [257], s_q=1, h_q=16, seed=15)
    q, k, bt, sl = _np(w)
    K = _keys_by_loop(k, bt[0], 257, 0)
    for h in range(16):
        p = mo.attention_weights(q[0, 0, h], K, w.scale)
        assert p.min() >= 0.0
        assert abs(p.sum() - 1.0) < 1e-12
    # a block of rows gives one distribution per row, each equal to its single-row form
    pb = mo.attention_weights(q[0, 0], K, w.scale)
    assert pb.shape == (16, 257)
    assert np.all(np.abs(pb.sum(axis=1) - 1.0) < 1e-12)
    for h in range(16):
        assert np.array_equal(pb[h], mo.attention_weights(q[0, 0, h], K, w.scale))
    # closed forms: a zero query weighs every key 1/n; a single key weighs 1
    assert np.allclose(mo.attention_weights(np.zeros((3, 576)), K, w.scale), 1.0 / 257, rtol=0, atol=1e-15)
    assert mo.attention_weights(q[0, 0, :2], K[:1], w.scale).tolist() == [[1.0], [1.0]]


def test_page_permutation_is_bit_identical():
    w = inputs.build("perm", [200, 64, 1], s_q=2, h_q=32, causal=True, seed=16)
    q, k, bt, sl = _np(w)
    out0, lse0 = mo.decode_dense(q, k, bt, sl, 1, True, w.scale)
    rng = np.random.default_rng(5)
    perm = rng.permutation(k.shape[0])          # new physical position of each page
    k2 = np.empty_like(k)
    k2[perm] = k
    bt2 = perm[bt]
    out1, lse1 = mo.decode_dense(q, k2, bt2, sl, 1, True, w.scale)
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)


@pytest.mark.parametrize("causal", [False, True])
def test_split_then_merge_equals_unsplit(causal):
    w = inputs.build("split", [300, 64, 65, 5], s_q=2, h_q=16, causal=causal, seed=17)
    q, k, bt, sl = _np(w)
    out0, lse0 = mo.decode_dense(q, k, bt, sl, 1, causal, w.scale)
    rng = np.random.default_rng(9)

    def cuts(b):
        n = (int(sl[b]) + 63) // 64
        return sorted(rng.choice(np.arange(1, max(n, 2)), size=min(2, max(n - 1, 0)), replace=False).tolist()) if n > 1 else []

    out1, lse1 = mo.decode_streaming(q, k, bt, sl, 1, causal, w.scale, split_pages=cuts)
    assert np.abs(out0 - out1).max() < 1e-12
    assert np.abs(lse0 - lse1).max() < 1e-12


def test_causal_row_equals_shorter_noncausal_call():
    w = inputs.build("causal", [90, 129], s_q=2, h_q=16, causal=True, seed=18)
    q, k, bt, sl = _np(w)
    out, lse = mo.decode_dense(q, k, bt, sl, 1, True, w.scale)
    for s in range(2):
        sl2 = sl - 2 + 1 + s
        o2, l2 = mo.decode_dense(q[:, s:s + 1], k, bt, sl2, 1, False, w.scale)
        assert np.array_equal(out[:, s], o2[:, 0]) and np.array_equal(lse[:, s], l2[:, 0])


def test_hard_max_limit_picks_argmax_row():
    w = inputs.build("hardmax", [190], s_q=1, h_q=16, seed=19)
    q, k, bt, sl = _np(w)
    K = _keys_by_loop(k, bt[0], 190, 0)
    out, _ = mo.decode_dense(q, k, bt, sl, 1, False, w.scale * 1e3)
    checked = 0
    for h in range(16):
        scores = [math.fsum(float(a) * float(c) for a, c in zip(q[0, 0, h], K[j])) for j in range(190)]
        top = max(range(190), key=lambda j: scores[j])
        # |O - V_top| <= sum_{j != top} w_j |V_j - V_top| with w_j <= exp(-(s_top - s_j) * scale)
        bound = sum(math.exp(-(scores[top] - scores[j]) * w.scale * 1e3) for j in range(190) if j != top)
        bound *= 2.0 * np.abs(K[:, :512]).max()
        err = np.abs(out[0, 0, h] - K[top, :512]).max()
        assert err <= bound + 1e-12
        if bound < 1e-3:
            checked += 1
    assert checked >= 4


def _brute(q, k, bt, sl, h_kv, causal, scale):
    B, s_q, h_q, _ = q.shape
    hg = h_q // h_kv
    out = np.zeros((B, s_q, h_q, 512))
    lse = np.zeros((B, s_q, h_q))
    for b in range(B):
        L = int(sl[b])
        for s in range(s_q):
            n = L - (s_q - 1 - s) if causal else L
            n = max(0, min(n, L))
            for h in range(h_q):
                g = h // hg
                xs = []
                for j in range(n):
                    krow = k[int(bt[b, j // 64]), j % 64, g]
                    xs.append(scale * math.fsum(float(a) * float(c) for a, c in zip(q[b, s, h], krow)))
                if n == 0:
                    lse[b, s, h] = -math.inf
                    continue
                m = max(xs)
                es = [math.exp(x - m) for x in xs]
                tot = math.fsum(es)
                lse[b, s, h] = m + math.log(tot)
                for c in range(512):
                    out[b, s, h, c] = math.fsum(es[j] * float(k[int(bt[b, j // 64]), j % 64, g, c])
                                                for j in range(n)) / tot
    return out, lse


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_brute_force_tiny(seed):
    g = torch.Generator().manual_seed(seed)
    B = int(torch.randint(1, 4, (1,), generator=g))
    lens = torch.randint(0, 131, (B,), generator=g).tolist()
    causal = seed % 2 == 1
    h_kv = 2 if seed == 3 else 1
    w = inputs.build("brute", lens, s_q=2, h_q=4, h_kv=h_kv, causal=causal, seed=seed + 20)
    q, k, bt, sl = _np(w)
    o1, l1 = mo.decode_dense(q, k, bt, sl, h_kv, causal, w.scale)
    o2, l2 = _brute(q, k, bt, sl, h_kv, causal, w.scale)
    fin = np.isfinite(l2)
    assert np.array_equal(np.isfinite(l1), fin)
    assert np.abs(l1[fin] - l2[fin]).max(initial=0) < 1e-12
    assert np.abs(o1 - o2).max() < 1e-12


def test_against_torch_sdpa_fp64():
    w = inputs.build("sdpa", [333, 64, 1], s_q=1, h_q=16, seed=21)
    q, k, bt, sl = _np(w)
    out, lse = mo.decode_dense(q, k, bt, sl, 1, False, w.scale)
    for b, L in enumerate(sl):
        K = torch.from_numpy(_keys_by_loop(k, bt[b], int(L), 0))[None, None]   # [1,1,L,576]
        Q = torch.from_numpy(q[b, 0])[None, :, None]                            # [1,16,1,576]
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, K.expand(1, 16, -1, -1), K[..., :512].expand(1, 16, -1, -1), scale=w.scale)
        assert (ref[0, :, 0].numpy() - out[b, 0]).__abs__().max() < 1e-12
        x = w.scale * (torch.from_numpy(q[b, 0]) @ K[0, 0].T)
        assert np.abs(torch.logsumexp(x, dim=-1).numpy() - lse[b, 0]).max() < 1e-12


def test_empty_sequence_and_merge_of_empty_parts():
    w = inputs.build("empty", [0, 3], s_q=2, h_q=16, causal=True, seed=22)
    q, k, bt, sl = _np(w)
    out, lse = mo.decode_dense(q, k, bt, sl, 1, True, w.scale)
    assert np.all(out[0] == 0.0) and np.all(np.isneginf(lse[0]))
    ls, o = mo.merge_partials([-np.inf, -np.inf], [np.ones(4), np.ones(4)])
    assert np.isneginf(ls) and np.all(o == 0.0)
    ls, o = mo.merge_partials([-np.inf, 0.5], [np.full(4, 7.0), np.full(4, 2.0)])
    assert ls == 0.5 and np.all(o == 2.0)


# ---- planted mistakes: each must be caught by one of the pins above --------

def _with_mutant(monkeypatch, name, fn):
    monkeypatch.setattr(mo, name, fn)


def test_mutant_gather_swapped_page_and_slot_is_caught(monkeypatch):
    def bad_gather(k_cache, block_table_row, L, g):
        j = np.arange(L)
        return k_cache[block_table_row[j % 64 % len(block_table_row)], j // 64, g, :]
    _with_mutant(monkeypatch, "gather_keys", bad_gather)
    with pytest.raises(AssertionError):
        test_zero_query_gives_mean_and_log_n()


def test_mutant_causal_off_by_one_is_caught(monkeypatch):
    def bad_visible(L, s, s_q, causal):
        n = L - (s_q - s) if causal else L
        return max(0, min(n, L))
    _with_mutant(monkeypatch, "visible_keys", bad_visible)
    with pytest.raises(AssertionError):
        test_brute_force_tiny(1)
