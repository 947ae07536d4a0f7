"""GPU parity: metadata bit-exact, decode within the stated tolerances, through the C ABI."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from mla_paged_kv_get_b200 import binding, inputs
from oracle import mla_oracle as mo
from oracle import schedule as sch

from gpu_util import compare, to_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    binding.load_library()


def run_gpu(w, num_sms=None, **kw):
    q, k, bt, sl = to_gpu(w)
    tile_md, num_splits = binding.get_metadata(sl, w.rows_per_kv, w.h_kv, num_sms)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = binding.decode_paged(q, k, bt, sl, 512, tile_md, num_splits, causal=w.causal,
                                    softmax_scale=w.scale, status=status, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, binding.status_string(int(status.item()))
    return out, lse, tile_md, num_splits


def oracle(w, batches=None):
    return mo.decode_dense(w.q, w.k_cache, w.block_table, w.seqlens, w.h_kv, w.causal, w.scale,
                           batches=batches)


# ---------------------------------------------------------------- metadata

@pytest.mark.parametrize("seed", range(12))
def test_metadata_bit_exact(seed):
    g = torch.Generator().manual_seed(seed)
    B = [1, 2, 7, 64, 128, 132, 300, 1000][seed % 8]
    mode = seed % 4
    if mode == 0:
        lens = torch.randint(0, 8193, (B,), generator=g)
    elif mode == 1:
        lens = torch.tensor([[0, 1, 63, 64, 65, 127, 128][i % 7] for i in range(B)])
    elif mode == 2:
        lens = torch.randint(32768, 65537, (B,), generator=g)
    else:
        lens = torch.full((B,), 4096)
    for rows, h_kv, sms in [(16, 1, 148), (128, 1, 148), (128, 1, 7), (32, 2, 148), (16, 1, 1), (256, 1, 148)]:
        md, ns = binding.get_metadata(lens.to(torch.int32).cuda(), rows, h_kv, sms)
        md_ref, ns_ref = sch.get_metadata(lens.tolist(), rows, h_kv, sms)
        assert md.cpu().tolist() == md_ref
        assert ns.cpu().tolist() == ns_ref



@pytest.mark.parametrize("rows,sms", [(128, 148), (16, 148), (128, 20)])
def test_metadata_part_count_search_bit_exact(rows, sms):
    """Near-equal batches around the part limit, where the part-count search
    runs and sometimes leaves trailing parts empty."""
    g = torch.Generator().manual_seed(rows * 1000 + sms)
    G_max = sch.num_parts(rows, 1, sms)
    fewer = 0
    for B in [G_max // 2, G_max // 2 + 1, G_max - 1, G_max, G_max + 1, 2 * G_max - 3, 3 * G_max]:
        for jitter in [0, 64, 700]:
            lens = 4096 + torch.randint(0, jitter + 1, (B,), generator=g)
            md, ns = binding.get_metadata(lens.to(torch.int32).cuda(), rows, 1, sms)
            md_ref, ns_ref = sch.get_metadata(lens.tolist(), rows, 1, sms)
            assert md.cpu().tolist() == md_ref, (B, jitter)
            assert ns.cpu().tolist() == ns_ref, (B, jitter)
            fewer += md_ref[-1][:4] == [B, 0, B, 0]
    assert fewer > 0   # the cases do reach a part count below the limit



def test_metadata_max_batch_bit_exact():
    """The largest batch the metadata call accepts (8192 sequences: the kernel's shared-memory
    tables are at their largest), with empty sequences mixed in; one more is rejected."""
    g = torch.Generator().manual_seed(8192)
    B = 8192
    lens = torch.randint(0, 2049, (B,), generator=g)
    lens[::7] = 0
    for rows, sms in [(16, 148), (128, 148)]:
        md, ns = binding.get_metadata(lens.to(torch.int32).cuda(), rows, 1, sms)
        md_ref, ns_ref = sch.get_metadata(lens.tolist(), rows, 1, sms)
        assert md.cpu().tolist() == md_ref
        assert ns.cpu().tolist() == ns_ref
    with pytest.raises(binding.MLAError):
        binding.get_metadata(torch.ones(B + 1, dtype=torch.int32, device="cuda"), 16, 1, 148)


# ---------------------------------------------------------------- decode parity

def test_tiny_config():
    w = inputs.config(1)
    out, lse, _, _ = run_gpu(w)
    o_ref, l_ref = oracle(w)
    compare(w, out, lse, o_ref, l_ref, what="tiny")


@pytest.mark.parametrize("seed", range(16))
def test_random_small_cases(seed):
    w = inputs.random_case(100 + seed, max_batch=5, max_len=700, h_q_choices=(16, 32, 64, 128),
                           s_q_choices=(1, 2), h_kv_choices=(1, 2) if seed % 3 == 0 else (1,))
    sms = [148, 7, 3, 1][seed % 4]
    out, lse, _, _ = run_gpu(w, num_sms=sms)
    o_ref, l_ref = oracle(w)
    compare(w, out, lse, o_ref, l_ref, what=f"random {seed}")


@pytest.mark.parametrize("rows", [(1, 16), (1, 32), (2, 16), (1, 64), (1, 128), (2, 64), (4, 32), (1, 8), (3, 16)])
def test_row_shapes(rows):
    s_q, h_q = rows
    w = inputs.build(f"rows{s_q}x{h_q}", [1, 63, 64, 65, 129, 300], s_q=s_q, h_q=h_q, causal=s_q > 1, seed=77)
    out, lse, _, _ = run_gpu(w, num_sms=5)
    o_ref, l_ref = oracle(w)
    compare(w, out, lse, o_ref, l_ref, what=f"s_q={s_q} h_q={h_q}")


def test_edge_lengths_and_empty_rows():
    # empty sequence, single token, exact page, page + 1, causal rows that see nothing
    w = inputs.build("edges", [0, 1, 64, 65, 2, 128], s_q=2, h_q=16, causal=True, seed=5)
    out, lse, _, ns = run_gpu(w, num_sms=4)
    o_ref, l_ref = oracle(w)
    compare(w, out, lse, o_ref, l_ref, what="edges")
    o = out.float().cpu()
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0].cpu()))
    # seqlen 1, causal s_q=2: token 0 sees nothing, token 1 sees key 0 -> O = V_0
    assert torch.all(o[1, 0] == 0)
    v0 = w.k_cache[w.block_table[1, 0], 0, 0, :512].float()
    assert (o[1, 1] - v0).abs().max() <= 2 ** -8 * v0.abs().max()


def test_page_permutation_bit_identical():
    w = inputs.build("perm", [700, 333, 64], s_q=1, h_q=128, seed=6)
    out0, lse0, _, _ = run_gpu(w)
    perm = torch.randperm(w.k_cache.shape[0], generator=torch.Generator().manual_seed(1))
    k2 = torch.empty_like(w.k_cache)
    k2[perm] = w.k_cache
    w.k_cache = k2
    w.block_table = perm[w.block_table.long()].to(torch.int32)
    out1, lse1, _, _ = run_gpu(w)
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)


def test_poison_does_not_leak():
    w = inputs.build("poison", [100, 64, 129], s_q=2, h_q=16, causal=True, seed=8)
    out0, lse0, _, _ = run_gpu(w, num_sms=3)
    w2 = inputs.build("poison", [100, 64, 129], s_q=2, h_q=16, causal=True, seed=8, poison=-7.5)
    out1, lse1, _, _ = run_gpu(w2, num_sms=3)
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)


def test_forced_part_counts_agree():
    w = inputs.build("parts", [5000, 3000, 64, 1], s_q=1, h_q=128, seed=9)
    o_ref, l_ref = oracle(w)
    for sms in (1, 2, 9, 148):
        out, lse, _, _ = run_gpu(w, num_sms=sms)
        compare(w, out, lse, o_ref, l_ref, what=f"num_sms={sms}")


@pytest.mark.parametrize("index", [2, 3, 4, 5])
def test_full_size_configs_every_sequence(index):
    """The full workloads in the launch configuration the bench uses: every sequence
    of the batch against the oracle, and the metadata of the whole batch bit-exact."""
    w = inputs.config(index)
    out, lse, md, ns = run_gpu(w)
    o_ref, l_ref = oracle(w)
    compare(w, out, lse, o_ref, l_ref, what=f"config {index}")
    md_ref, ns_ref = sch.get_metadata(w.seqlens.tolist(), w.rows_per_kv, w.h_kv, torch.cuda.get_device_properties(0).multi_processor_count)
    assert md.cpu().tolist() == md_ref and ns.cpu().tolist() == ns_ref
    # every row is finite and every lse finite (all sequences are non-empty)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("h_q,sms", [(16, 148), (16, 2), (128, 148), (128, 2)])
def test_sequence_longer_than_its_block_table_row(h_q, sms):
    """cache_seqlens[b] > 64 * max_pages_per_seq is a caller error the kernels detect on the
    device: the status word reads MLA_ERR_BAD_INPUT, that sequence's rows are zero with
    lse = -inf, nothing past its block-table row is read, and the other sequences are
    still right.  With two SMs the long sequence is cut into several pieces (merge path)."""
    w = inputs.build(f"overlong{h_q}", [300, 200, 500, 64], s_q=1, h_q=h_q, seed=12)
    max_pages = w.block_table.shape[1]
    bad = w.seqlens.clone()
    bad[1] = 64 * max_pages + 5                  # one page more than its row can name
    q, k, bt, _ = to_gpu(w)
    sl = bad.cuda()
    md, ns = binding.get_metadata(sl, w.rows_per_kv, w.h_kv, num_sms=sms)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = binding.decode_paged(q, k, bt, sl, 512, md, ns, softmax_scale=w.scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == binding.MLA_ERR_BAD_INPUT
    assert torch.all(out[1].float() == 0) and torch.all(torch.isneginf(lse[1]))
    good = [0, 2, 3]
    o_ref, l_ref = oracle(w, batches=good)
    compare(w, out, lse, o_ref, l_ref, batches=good, what=f"overlong h_q={h_q} sms={sms}")


@pytest.mark.gpu
@pytest.mark.parametrize("h_q,sms", [(16, 2), (16, 148), (128, 2), (128, 148)])
def test_runs_of_overlong_sequences(h_q, sms):
    """Runs of over-long sequences between valid ones: each is a segment without tiles in the
    part that holds it (with two SMs, one part holds them all, back to back).  Every launch
    reports MLA_ERR_BAD_INPUT with zero rows and lse = -inf for them, and the valid sequences
    match the oracle, bit for bit from launch to launch.  The value-product issuer counts the
    softmax's O hand-offs; had it lost count over the empty segments, it would wait out its
    limit and abort the part, and the valid sequences after the run would come out wrong."""
    w = inputs.build(f"overlong_run{h_q}", [300, 100, 100, 100, 200, 100, 100, 500, 64], s_q=1, h_q=h_q,
                     seed=13)
    max_pages = w.block_table.shape[1]
    bad_rows, good = [1, 2, 3, 5, 6], [0, 4, 7, 8]
    lens = w.seqlens.clone()
    lens[bad_rows] = 64 * max_pages + 5
    q, k, bt, _ = to_gpu(w)
    sl = lens.cuda()
    md, ns = binding.get_metadata(sl, w.rows_per_kv, w.h_kv, num_sms=sms)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_ref, l_ref = oracle(w, batches=good)
    out0 = lse0 = None
    for i in range(20):
        status.zero_()
        out, lse = binding.decode_paged(q, k, bt, sl, 512, md, ns, softmax_scale=w.scale, status=status,
                                        timeout_ns=200_000_000)
        torch.cuda.synchronize()
        assert int(status.item()) == binding.MLA_ERR_BAD_INPUT, binding.status_string(int(status.item()))
        assert torch.all(out[bad_rows].float() == 0) and torch.all(torch.isneginf(lse[bad_rows]))
        if i == 0:
            compare(w, out, lse, o_ref, l_ref, batches=good, what=f"overlong run h_q={h_q} sms={sms}")
            out0, lse0 = out.clone(), lse.clone()
        else:
            assert torch.equal(out[good].view(torch.int16), out0[good].view(torch.int16))
            assert torch.equal(lse[good].view(torch.int32), lse0[good].view(torch.int32))


@pytest.mark.parametrize("rows", [16, 32, 64, 128])
def test_repeated_launches_are_bit_identical(rows):
    """Hundreds of back-to-back launches on the varlen lengths of the memory-bound
    workload, with short wait limits: every launch finishes without a timeout and
    reproduces the first bit for bit.  Pipeline races between the roles of a CTA
    (a barrier phase taken for the wrong load) show up here as timeouts or as
    launches that differ."""
    w = inputs.build(f"repeat{rows}", inputs.config_seqlens(3), s_q=1, h_q=rows, seed=90 + rows)
    q, k, bt, sl = to_gpu(w)
    md, ns = binding.get_metadata(sl, w.rows_per_kv, w.h_kv)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(binding.workspace_bytes(w.batch, w.rows_per_kv, w.h_kv, md.shape[0]),
                     dtype=torch.uint8, device="cuda")
    out0, lse0 = binding.decode_paged(q, k, bt, sl, 512, md, ns, softmax_scale=w.scale, workspace=ws,
                                      status=status, timeout_ns=200_000_000)
    out0, lse0 = out0.clone(), lse0.clone()
    out, lse = torch.empty_like(out0), torch.empty_like(lse0)
    bad = torch.zeros((), dtype=torch.int64, device="cuda")
    for _ in range(300):
        binding.decode_paged(q, k, bt, sl, 512, md, ns, softmax_scale=w.scale, workspace=ws, out=out, lse=lse,
                             status=status, timeout_ns=200_000_000)
        bad += (out.view(torch.int16) != out0.view(torch.int16)).any() | (lse.view(torch.int32) != lse0.view(torch.int32)).any()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, binding.status_string(int(status.item()))
    assert int(bad.item()) == 0
    o_ref, l_ref = oracle(w)
    compare(w, out0, lse0, o_ref, l_ref, what=f"repeat rows={rows}")


def test_step_replays_from_a_cuda_graph():
    """Metadata, decode and combine are stream-ordered with no host synchronisation,
    so one decode step captures into a CUDA graph; replays on new cache lengths and
    contents give what eager calls give, bit for bit."""
    w = inputs.config(3)
    q, k, bt, sl = to_gpu(w)
    G = binding.num_parts(w.rows_per_kv, w.h_kv)
    ws = torch.empty(binding.workspace_bytes(w.batch, w.rows_per_kv, w.h_kv, G), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.batch, w.s_q, w.h_q, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.batch, w.s_q, w.h_q), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        md, ns = binding.get_metadata(sl, w.rows_per_kv, w.h_kv)
        binding.decode_paged(q, k, bt, sl, 512, md, ns, softmax_scale=w.scale, workspace=ws, out=out, lse=lse,
                             status=status)

    step()                                   # first call sets the kernels' shared-memory attributes
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for trial in range(3):
        # new lengths (same page table capacity) and new cache values, written in place
        g = torch.Generator().manual_seed(500 + trial)
        new_len = torch.randint(1, 64 * bt.shape[1] + 1, (w.batch,), generator=g, dtype=torch.int32)
        sl.copy_(new_len.cuda())
        k.copy_((torch.randn(k.shape, generator=g) * 0.5).to(torch.bfloat16).cuda())
        graph.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got_out, got_lse = out.clone(), lse.clone()
        step()
        torch.cuda.synchronize()
        assert torch.equal(got_out.view(torch.int16), out.view(torch.int16))
        assert torch.equal(got_lse.view(torch.int32), lse.view(torch.int32))
    del graph


@pytest.mark.parametrize("shape", [(1, 16, False), (1, 32, False), (1, 64, False), (1, 128, False), (2, 64, True)])
def test_fp16_inputs_match_oracle(shape):
    """The fp16 path (same kernels, fp16 MMAs, P and out in fp16) against the oracle
    on the fp16 inputs, split sequences included so the fp16 combine runs too."""
    s_q, h_q, causal = shape
    w = inputs.build(f"fp16_{s_q}x{h_q}", [1, 63, 64, 65, 200, 777, 2048], s_q=s_q, h_q=h_q, causal=causal,
                     seed=61 + h_q, dtype=torch.float16)
    o_ref, l_ref = oracle(w)
    for sms in (148, 5):
        out, lse, _, _ = run_gpu(w, num_sms=sms)
        assert out.dtype == torch.float16
        compare(w, out, lse, o_ref, l_ref, what=f"fp16 s_q={s_q} h_q={h_q} sms={sms}")


# ---------------------------------------------------------------- failure paths

def test_bounded_wait_reports_timeout_and_context_survives():
    w = inputs.config(1)
    q, k, bt, sl = to_gpu(w)
    md, ns = binding.get_metadata(sl, w.rows_per_kv, w.h_kv)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.decode_paged(q, k, bt, sl, 512, md, ns, softmax_scale=w.scale, status=status,
                         debug_flags=1, timeout_ns=20_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) == binding.MLA_ERR_TIMEOUT
    out, lse, _, _ = run_gpu(w)           # the context is still usable
    o_ref, l_ref = oracle(w)
    compare(w, out, lse, o_ref, l_ref, what="after timeout")


def test_corrupt_page_id_is_reported_not_read():
    w = inputs.build("corrupt", [200, 100], s_q=1, h_q=16, seed=10)
    w.block_table[0, 1] = 10 ** 6          # beyond the cache
    q, k, bt, sl = to_gpu(w)
    md, ns = binding.get_metadata(sl, w.rows_per_kv, w.h_kv)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = binding.decode_paged(q, k, bt, sl, 512, md, ns, softmax_scale=w.scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == binding.MLA_ERR_BAD_INPUT
    o_ref, l_ref = oracle(w, batches=[1])  # the untouched sequence is still right
    compare(w, out, lse, o_ref, l_ref, batches=[1], what="corrupt")


def test_host_side_argument_errors():
    w = inputs.config(1)
    q, k, bt, sl = to_gpu(w)
    md, ns = binding.get_metadata(sl, w.rows_per_kv, w.h_kv)
    with pytest.raises(binding.MLAError):     # dv must be 512
        binding.decode_paged(q, k, bt, sl, 256, md, ns)
    with pytest.raises(binding.MLAError):     # workspace too small
        binding.decode_paged(q, k, bt, sl, 512, md, ns,
                             workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(ValueError):           # wrong dtype is caught before the library
        binding.decode_paged(q.float(), k, bt, sl, 512, md, ns)


# ---------------------------------------------------------------- the two decode kernels

@pytest.mark.parametrize("shape", [(1, 128, False), (2, 64, True), (1, 256, False), (3, 32, True)])
def test_pair_and_single_cta_kernels_both_match_oracle(shape):
    """More than 64 rows per KV head run on CTA pairs (2-SM MMAs); debug flag 4
    forces one CTA per 64-row block.  Both must match the oracle."""
    s_q, h_q, causal = shape
    w = inputs.build(f"pair{s_q}x{h_q}", [1, 63, 64, 65, 129, 640, 1000], s_q=s_q, h_q=h_q, causal=causal, seed=41)
    o_ref, l_ref = oracle(w)
    for flags in (0, 4):
        for sms in (148, 6):
            out, lse, _, _ = run_gpu(w, num_sms=sms, debug_flags=flags)
            compare(w, out, lse, o_ref, l_ref, what=f"s_q={s_q} h_q={h_q} flags={flags} sms={sms}")
