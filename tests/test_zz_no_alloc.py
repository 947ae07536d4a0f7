"""The allocation-free decode entry point agrees with the workspace entry point.

mla_decode_paged_noalloc exists for callers that cannot call cudaMalloc (for
example an operator running inside a host framework that owns the device
memory pool, or a runtime that forbids allocation after start-up).  It keeps
the split partials in a scratch array that the library holds in device memory.

The test calls it through the C ABI three times in a row: first on a
different workload with more split pieces (which fills the scratch array with
its partials), then twice on the target workload.  A call that read a partial
it did not write would pick up the earlier call's leftovers.  Every result is
compared with the ordinary (workspace) entry point on the same inputs, within
the tolerances of the other parity tests (the two entry points run the same
kernels, so they are bit-identical too), and with the fp64 oracle.

The file name sorts last so that a run stopping at the first failure has run
every other test before this one.
"""

import ctypes

import pytest
import torch

from mla_paged_kv_get_b200 import binding, inputs
from oracle import mla_oracle as mo

from gpu_util import compare

pytestmark = pytest.mark.gpu


def _declare(lib):
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.mla_decode_paged_noalloc.argtypes = [vp, vp, ci, vp, ci, vp, ci, ci, ci, ci, ci, ci, vp, vp, ci, ci, cf,
                                             vp, vp, vp, vp]
    lib.mla_decode_paged_noalloc.restype = ci


def _noalloc_call(lib, w, q, k, bt, sl, tile_md, num_splits, like_out, like_lse):
    P = binding._ptr
    out = torch.full_like(like_out, float("nan"))
    lse = torch.full_like(like_lse, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.mla_decode_paged_noalloc(P(q), P(k), k.shape[0], P(bt), bt.shape[1], P(sl), w.batch, w.s_q,
                                      w.h_q, w.h_kv, 576, 512, P(tile_md), P(num_splits), tile_md.shape[0],
                                      int(w.causal), w.scale, P(out), P(lse), P(status), ctypes.c_void_p(stream))
    assert rc == 0, binding.status_string(rc)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, lse


def _case(w, num_sms):
    q, k, bt, sl = (w.q.cuda(), w.k_cache.cuda(), w.block_table.cuda(), w.seqlens.cuda())
    tile_md, num_splits = binding.get_metadata(sl, w.rows_per_kv, w.h_kv, num_sms=num_sms)
    assert int(num_splits[-1]) > w.batch       # some sequence is split: partials go through scratch
    ws_out, ws_lse = binding.decode_paged(q, k, bt, sl, 512, tile_md, num_splits, causal=w.causal,
                                          softmax_scale=w.scale)
    torch.cuda.synchronize()
    o_ref, l_ref = mo.decode_dense(w.q, w.k_cache, w.block_table, w.seqlens, w.h_kv, w.causal, w.scale)
    return (q, k, bt, sl, tile_md, num_splits), (ws_out, ws_lse), (o_ref, l_ref)


def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    lib = binding.load_library()
    _declare(lib)
    # a different workload first: more pieces, other rows, other lengths
    first = inputs.build("noalloc_first", [5000, 64, 2500, 1, 4100, 777, 3000], s_q=1, h_q=128, seed=77)
    target = inputs.build("noalloc", [3000, 700, 64, 5, 1900], s_q=2, h_q=64, causal=True, seed=31)
    for tag, w, sms, calls in (("first", first, 40, 1), ("target", target, 16, 2)):
        dev_args, (ws_out, ws_lse), (o_ref, l_ref) = _case(w, sms)
        for call in range(calls):
            out, lse = _noalloc_call(lib, w, *dev_args, ws_out, ws_lse)
            what = f"noalloc {tag} call {call}"
            compare(w, out, lse, ws_out.float().cpu().numpy(), ws_lse.cpu().numpy(), what=what + " vs workspace")
            assert torch.equal(out.view(torch.int16), ws_out.view(torch.int16))
            assert torch.equal(lse.view(torch.int32), ws_lse.view(torch.int32))
            compare(w, out, lse, o_ref, l_ref, what=what + " vs oracle")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    lib = binding.load_library()
    _declare(lib)
    # 2000 sequences x 128 rows of partials need far more than the fixed scratch
    null = ctypes.c_void_p(0)
    one = torch.zeros(16, dtype=torch.int32, device="cuda")
    rc = lib.mla_decode_paged_noalloc(binding._ptr(one), binding._ptr(one), 1, binding._ptr(one), 1,
                                      binding._ptr(one), 2000, 1, 128, 1, 576, 512, binding._ptr(one),
                                      binding._ptr(one), 74, 0, 0.04, binding._ptr(one), binding._ptr(one),
                                      null, null)
    assert rc == -3     # MLA_ERR_WORKSPACE
