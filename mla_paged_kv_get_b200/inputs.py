"""Seeded synthetic decode workloads (shared by the tests, the bench and the oracle legs).

This module only draws random numbers and lays them out; it contains none of
the attention arithmetic.  Every tensor is created on the CPU with a
``torch.Generator`` so that the CUDA path and the fp64 oracle see the same
bytes.

Recipe (shapes follow the decode setting of the pages: bf16 paged latent
cache, 64-token pages, one shared KV head of width 576, variable lengths):

* ``q`` and the cache are float32 ``randn`` rounded to bf16 (round to
  nearest even), or to fp16 for the fp16 path;
* the used pages are ``randperm`` over all pages and dealt out in order to the
  page-table rows, so physical placement is shuffled;
* one extra *poison page* filled with finite values of magnitude 30 sits in
  every unused page-table slot, and the tokens beyond ``L`` in each sequence's
  last page hold the same poison: a kernel that reads past a sequence end or
  through an unused slot changes the output visibly.
"""

from __future__ import annotations

import dataclasses
import math

import torch

D_QK = 576
D_V = 512
PAGE = 64
POISON = 30.0


@dataclasses.dataclass
class Workload:
    name: str
    q: torch.Tensor            # [B, s_q, h_q, 576] bf16
    k_cache: torch.Tensor      # [num_pages, 64, h_kv, 576] bf16
    block_table: torch.Tensor  # [B, max_pages] int32
    seqlens: torch.Tensor      # [B] int32
    s_q: int
    h_q: int
    h_kv: int
    causal: bool
    scale: float
    seed: int

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def rows_per_kv(self) -> int:
        return self.s_q * self.h_q // self.h_kv

    def describe(self) -> dict:
        return {
            "workload": self.name, "batch": self.batch, "s_q": self.s_q, "h_q": self.h_q,
            "h_kv": self.h_kv, "d": D_QK, "dv": D_V, "page": PAGE, "causal": self.causal,
            "softmax_scale": self.scale, "seed": self.seed,
            "mean_seqlen": float(self.seqlens.float().mean()),
            "total_tokens": int(self.seqlens.long().sum()),
        }


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def build(name: str, seqlens, s_q: int, h_q: int, h_kv: int = 1, causal: bool = False,
          scale: float | None = None, seed: int = 0, shuffle: bool = True,
          spare_slots: int = 1, poison: float = POISON, dtype: torch.dtype = torch.bfloat16) -> Workload:
    """Lay out one workload with the recipe in the module docstring (q and cache in `dtype`:
    bf16, or fp16 for the fp16 path)."""
    g = _gen(seed)
    seqlens = torch.as_tensor(list(seqlens), dtype=torch.int32)
    B = seqlens.numel()
    n_pages = [(int(L) + PAGE - 1) // PAGE for L in seqlens.tolist()]
    used = sum(n_pages)
    max_pages = max(max(n_pages) if n_pages else 0, 0) + spare_slots
    max_pages = max(max_pages, 1)
    poison_page = used                       # the last physical page
    num_pages = used + 1

    q = torch.randn((B, s_q, h_q, D_QK), generator=g, dtype=torch.float32).to(dtype)
    k = torch.randn((num_pages, PAGE, h_kv, D_QK), generator=g, dtype=torch.float32)
    sign = torch.randint(0, 2, (PAGE, h_kv, D_QK), generator=g, dtype=torch.int32) * 2 - 1
    k[poison_page] = poison * sign.float()

    order = torch.randperm(used, generator=g) if shuffle else torch.arange(used)
    block_table = torch.full((B, max_pages), poison_page, dtype=torch.int32)
    cursor = 0
    for b in range(B):
        nb = n_pages[b]
        block_table[b, :nb] = order[cursor:cursor + nb].to(torch.int32)
        cursor += nb
        L = int(seqlens[b])
        tail = nb * PAGE - L
        if tail > 0:
            last = int(block_table[b, nb - 1])
            k[last, PAGE - tail:] = poison * sign[PAGE - tail:].float()
    k_cache = k.to(dtype)
    if scale is None:
        scale = D_QK ** -0.5
    return Workload(name, q, k_cache, block_table, seqlens, s_q, h_q, h_kv, causal,
                    float(scale), seed)


# The five decode configurations the measurements are quoted on.
CONFIG_NAMES = {
    1: "tiny",
    2: "compute_bound",
    3: "varlen_memory_bound",
    4: "mtp_causal",
    5: "long_context_split_kv",
}


def config_seqlens(index: int) -> list[int]:
    g = _gen(1000 + index)
    if index == 1:
        return [100, 64]
    if index == 2:
        return [4096] * 64
    if index == 3:
        return torch.randint(1, 8193, (128,), generator=g).tolist()
    if index == 4:
        x = torch.normal(4096.0, 1024.0, (132,), generator=g)
        return x.round().clamp(64, 8192).to(torch.int64).tolist()
    if index == 5:
        return torch.randint(32768, 65537, (8,), generator=g).tolist()
    raise ValueError(f"unknown config {index}")


def config(index: int, seqlens=None) -> Workload:
    """Workload ``index`` (1..5); ``seqlens`` overrides the drawn lengths."""
    lens = config_seqlens(index) if seqlens is None else list(seqlens)
    seed = 2000 + index
    if index == 1:
        return build(CONFIG_NAMES[1], lens, s_q=1, h_q=16, seed=seed)
    if index == 2:
        return build(CONFIG_NAMES[2], lens, s_q=1, h_q=128, seed=seed)
    if index == 3:
        return build(CONFIG_NAMES[3], lens, s_q=1, h_q=16, seed=seed)
    if index == 4:
        return build(CONFIG_NAMES[4], lens, s_q=2, h_q=64, causal=True, seed=seed)
    if index == 5:
        return build(CONFIG_NAMES[5], lens, s_q=1, h_q=128, seed=seed)
    raise ValueError(f"unknown config {index}")


def random_case(seed: int, max_batch: int = 4, max_len: int = 300, h_q_choices=(16, 32, 64, 128),
                s_q_choices=(1, 2), h_kv_choices=(1,), allow_empty: bool = True) -> Workload:
    """A small random case for sweeps (ragged lengths, both causal modes)."""
    g = _gen(seed)
    B = int(torch.randint(1, max_batch + 1, (1,), generator=g))
    lo = 0 if allow_empty else 1
    lens = torch.randint(lo, max_len + 1, (B,), generator=g).tolist()
    h_q = h_q_choices[int(torch.randint(0, len(h_q_choices), (1,), generator=g))]
    s_q = s_q_choices[int(torch.randint(0, len(s_q_choices), (1,), generator=g))]
    h_kv = h_kv_choices[int(torch.randint(0, len(h_kv_choices), (1,), generator=g))]
    causal = bool(torch.randint(0, 2, (1,), generator=g))
    return build(f"random_{seed}", lens, s_q=s_q, h_q=h_q, h_kv=h_kv, causal=causal,
                 seed=seed + 7)


def human_bytes(n: int) -> str:
    return f"{n / 1e6:.1f} MB" if n < 1e9 else f"{n / 1e9:.2f} GB"


def pages_needed(seqlens) -> int:
    return sum(math.ceil(int(L) / PAGE) for L in seqlens)
