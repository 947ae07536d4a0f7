"""The allocation-free decode entry point agrees with the workspace entry point.

mla_decode_paged_noalloc exists for callers that cannot call cudaMalloc (for
example an operator running inside a host framework that owns the device
memory pool, or a runtime that forbids allocation after start-up).  It keeps
the split partials in a scratch array that the library holds in device memory.
This test calls it through the C ABI twice in a row on a workload whose
sequences are split (so the scratch array is really used, and the second call
starts from the first call's leftovers) and compares each result with the
ordinary entry point, within the tolerances of the other parity tests.

The file name sorts last so that a run stopping at the first failure has run
every other test before this one.
"""

import ctypes

import pytest
import torch

from mla_paged_kv_get_b200 import binding, inputs

from gpu_util import compare

pytestmark = pytest.mark.gpu


def _declare(lib):
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.mla_decode_paged_noalloc.argtypes = [vp, vp, ci, vp, ci, vp, ci, ci, ci, ci, ci, ci, vp, vp, ci, ci, cf,
                                             vp, vp, vp, vp]
    lib.mla_decode_paged_noalloc.restype = ci


def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    lib = binding.load_library()
    _declare(lib)
    w = inputs.build("noalloc", [3000, 700, 64, 5, 1900], s_q=2, h_q=64, causal=True, seed=31)
    q, k, bt, sl = (w.q.cuda(), w.k_cache.cuda(), w.block_table.cuda(), w.seqlens.cuda())
    tile_md, num_splits = binding.get_metadata(sl, w.rows_per_kv, w.h_kv, num_sms=16)
    assert int(num_splits[-1]) > w.batch       # some sequence is split: partials go through scratch
    out_ref, lse_ref = binding.decode_paged(q, k, bt, sl, 512, tile_md, num_splits, causal=True,
                                            softmax_scale=w.scale)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    P = binding._ptr
    for call in range(2):
        out = torch.full_like(out_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = lib.mla_decode_paged_noalloc(P(q), P(k), k.shape[0], P(bt), bt.shape[1], P(sl), w.batch, w.s_q,
                                          w.h_q, w.h_kv, 576, 512, P(tile_md), P(num_splits), tile_md.shape[0],
                                          1, w.scale, P(out), P(lse), P(status), ctypes.c_void_p(stream))
        assert rc == 0, binding.status_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        compare(w, out, lse, out_ref.float().cpu().numpy(), lse_ref.cpu().numpy(), what=f"noalloc call {call}")


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
