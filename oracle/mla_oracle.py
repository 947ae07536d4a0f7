"""fp64 CPU oracle: MLA decode attention over a paged, shared latent KV cache.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this module, and this module never imports the CUDA library.

What is computed (cnblogs "DeepSeek 开源记-第1天-FlashMLA", §2 核心功能 /
关键特性 and §6.2 基本使用; m.ygpos.cn "DeepSeek代碼開源第一彈Flash MLA",
release list "BF16, 分頁kvcache 塊大小64"):

* the cache holds one 576-wide row per token and KV head (512 latent dims
  followed by 64 rotary dims); every query head of a group shares it
  ("Shared KV 模式");
* the cache is paged: token j of sequence b lives in page
  ``block_table[b, j // 64]`` at slot ``j % 64``;
* for each query row, ``x_j = scale * <q, K_j>`` over the 576 dims,
  ``lse = ln sum_j exp(x_j)`` and ``O = sum_j exp(x_j - lse) * V_j`` where
  ``V_j`` is the first ``dv = 512`` dims of the same cached row;
* the call returns ``(out, lse)`` (cnblogs §6.2: ``output, lse =
  flash_mla_with_kvcache(...)``).

Readings where the pages are silent (this project's choices):

* ``lse`` is the natural logarithm, shape ``[B, s_q, h_q]``.
* causal: the ``s_q`` query tokens are the last ``s_q`` positions of the
  sequence, so query token ``s`` sees keys ``j < L - (s_q - 1 - s)``.
* a row that sees no key returns ``O = 0`` and ``lse = -inf``.
* query head ``h`` reads KV head ``h // (h_q // h_kv)``.

All arithmetic is float64 on inputs that are bf16 values widened exactly.
Matrix products use numpy's ``@`` (a library primitive); nothing here is
blocked, fused or reordered beyond the definition, except in
``decode_streaming``, which follows the pages' stated compute flow (cnblogs
§4.1 计算流程: load, blockwise scores, softmax, merge of the outputs) on
purpose so that it can be checked against ``decode_dense``.
"""

from __future__ import annotations

import math

import numpy as np

D_QK = 576   # cached row width: 512 latent + 64 rotary (cnblogs §2 关键特性)
D_V = 512    # value width, the first 512 dims of the same row (cnblogs §2)
PAGE = 64    # tokens per KV page (m.ygpos.cn release list; cnblogs tweet)


def as_f64(x) -> np.ndarray:
    """Widen any array-like (numpy or a CPU torch tensor) to float64."""
    if hasattr(x, "detach"):  # torch tensor: widen through float32, exact for bf16
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def as_i64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.asarray(x, dtype=np.int64)


def gather_keys(k_cache: np.ndarray, block_table_row: np.ndarray, L: int, g: int) -> np.ndarray:
    """Rows ``K_j`` for ``j < L`` of KV head ``g``, read through the page table.

    ``k_cache`` is ``[num_pages, 64, h_kv, 576]``.  Returns ``[L, 576]``.
    """
    j = np.arange(L, dtype=np.int64)
    pages = block_table_row[j // PAGE]
    return k_cache[pages, j % PAGE, g, :]


def visible_keys(L: int, s: int, s_q: int, causal: bool) -> int:
    """Number of keys query token ``s`` attends to (causal reading above)."""
    n = L - (s_q - 1 - s) if causal else L
    return max(0, min(n, L))


def decode_dense(q, k_cache, block_table, seqlens, h_kv: int, causal: bool, scale: float,
                 dv: int = D_V, batches=None):
    """Dense two-pass form: gather all keys, all scores, max, sum, output.

    q: ``[B, s_q, h_q, 576]``; k_cache: ``[P, 64, h_kv, 576]``;
    block_table: ``[B, max_pages]``; seqlens: ``[B]``.
    Returns ``out [B, s_q, h_q, dv]`` and ``lse [B, s_q, h_q]`` in float64.
    ``batches`` restricts the work to a subset of sequence indices (the other
    rows are left as NaN) so that large inputs can be sampled.
    """
    q = as_f64(q)
    k_cache = as_f64(k_cache)
    block_table = as_i64(block_table)
    seqlens = as_i64(seqlens)
    B, s_q, h_q, d = q.shape
    assert d == D_QK and k_cache.shape[-1] == D_QK and h_q % h_kv == 0
    hg = h_q // h_kv
    out = np.full((B, s_q, h_q, dv), np.nan)
    lse = np.full((B, s_q, h_q), np.nan)
    for b in (range(B) if batches is None else batches):
        L = int(seqlens[b])
        for g in range(h_kv):
            K = gather_keys(k_cache, block_table[b], L, g)
            V = K[:, :dv]
            heads = slice(g * hg, (g + 1) * hg)
            for s in range(s_q):
                n = visible_keys(L, s, s_q, causal)
                if n == 0:
                    out[b, s, heads] = 0.0
                    lse[b, s, heads] = -np.inf
                    continue
                x = scale * (q[b, s, heads] @ K[:n].T)          # [hg, n]
                m = x.max(axis=1, keepdims=True)
                e = np.exp(x - m)
                l = e.sum(axis=1)
                lse[b, s, heads] = m[:, 0] + np.log(l)
                out[b, s, heads] = (e @ V[:n]) / l[:, None]
    return out, lse


def attention_weights(q_rows, K: np.ndarray, scale: float) -> np.ndarray:
    """Softmax weights ``exp(x_j - lse)`` of query rows over keys ``K``.

    ``q_rows`` is one row ``[576]`` (result ``[n]``) or several ``[r, 576]``
    (result ``[r, n]``, one distribution per row).
    """
    x = scale * (as_f64(q_rows) @ as_f64(K).T)
    m = x.max(axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=-1, keepdims=True)


def merge_partials(lse_parts, o_parts):
    """Merge per-split results (cnblogs §4.1 计算流程, 输出结果合并).

    ``lse = ln sum_i exp(lse_i)`` and ``O = sum_i exp(lse_i - lse) * O_i``.
    Splits with ``lse_i = -inf`` carry no weight; if every split is empty the
    result is ``O = 0``, ``lse = -inf``.
    """
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    o_parts = np.asarray(o_parts, dtype=np.float64)
    top = lse_parts.max(axis=0)
    finite = np.isfinite(top)
    safe_top = np.where(finite, top, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - safe_top), 0.0)
    tot = w.sum(axis=0)
    lse = np.where(finite, safe_top + np.log(np.where(finite, tot, 1.0)), -np.inf)
    coef = np.where(finite, w / np.where(finite, tot, 1.0), 0.0)
    o = (coef[..., None] * o_parts).sum(axis=0)
    return lse, o


def decode_streaming(q, k_cache, block_table, seqlens, h_kv: int, causal: bool, scale: float,
                     dv: int = D_V, split_pages=None):
    """Streaming form: page-by-page online softmax, optional splits, merge.

    Follows the pages' flow (cnblogs §4.1): load the query, score one 64-token
    page at a time, keep a running max ``m``, running sum ``l`` and running
    weighted sum ``acc`` (rescaled by ``exp(m_old - m_new)`` when the max
    grows), and at the end of each split emit ``(acc / l, m + ln l)``; the
    splits are then merged by ``merge_partials``.

    ``split_pages(b)`` returns the sorted page indices where new splits start
    for sequence ``b`` (default: none, one split per sequence).
    """
    q = as_f64(q)
    k_cache = as_f64(k_cache)
    block_table = as_i64(block_table)
    seqlens = as_i64(seqlens)
    B, s_q, h_q, _ = q.shape
    hg = h_q // h_kv
    out = np.zeros((B, s_q, h_q, dv))
    lse = np.full((B, s_q, h_q), -np.inf)
    for b in range(B):
        L = int(seqlens[b])
        n_pages = (L + PAGE - 1) // PAGE
        cuts = sorted(set([0] + list(split_pages(b) if split_pages else []) + [n_pages]))
        cuts = [c for c in cuts if 0 <= c <= n_pages]
        for g in range(h_kv):
            for s in range(s_q):
                n = visible_keys(L, s, s_q, causal)
                for h in range(g * hg, (g + 1) * hg):
                    qv = q[b, s, h]
                    lse_parts, o_parts = [], []
                    for c0, c1 in zip(cuts[:-1], cuts[1:]):
                        m, l, acc = -np.inf, 0.0, np.zeros(dv)
                        for p in range(c0, c1):
                            j0, j1 = p * PAGE, min((p + 1) * PAGE, n)
                            if j1 <= j0:
                                continue
                            page = k_cache[block_table[b, p], : j1 - j0, g, :]
                            x = scale * (page @ qv)
                            m_new = max(m, float(x.max()))
                            alpha = math.exp(m - m_new) if m != -np.inf else 0.0
                            e = np.exp(x - m_new)
                            l = l * alpha + e.sum()
                            acc = acc * alpha + e @ page[:, :dv]
                            m = m_new
                        if l > 0.0:
                            lse_parts.append(m + math.log(l))
                            o_parts.append(acc / l)
                        else:
                            lse_parts.append(-np.inf)
                            o_parts.append(np.zeros(dv))
                    if lse_parts:
                        ls, o = merge_partials(lse_parts, o_parts)
                        lse[b, s, h] = ls
                        out[b, s, h] = o
    return out, lse
