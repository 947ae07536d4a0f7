"""The C-ABI library loads on a machine without a GPU and exports every symbol
that include/mla_b200.h declares; host-only calls answer without a device."""

import ctypes
import os
import re

import pytest

from mla_paged_kv_get_b200 import binding, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "mla_b200.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("mla_get_metadata", "mla_decode_paged", "mla_num_parts", "mla_workspace_bytes",
                 "mla_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_host_only_calls(lib):
    assert lib.mla_num_parts(128, 1, 148) == 74
    assert lib.mla_num_parts(16, 1, 148) == 148
    assert lib.mla_num_parts(16, 2, 8) == 4
    assert lib.mla_num_parts(0, 1, 148) < 0
    assert [lib.mla_rows_per_block(r) for r in (1, 16, 17, 32, 33, 128)] == [16, 16, 32, 32, 64, 64]
    ws = lib.mla_workspace_bytes(8, 128, 1, 512, 74)
    assert ws == ((8 + 74) * 128 * 513 * 4 + 255) // 256 * 256
    assert lib.mla_workspace_bytes(0, 128, 1, 512, 74) == 0
    assert lib.mla_status_string(0) == b"ok"
    assert b"timed out" in lib.mla_status_string(-5)


def test_scheduler_part_count_matches_oracle(lib):
    from oracle import schedule
    for rows in (1, 16, 17, 32, 64, 96, 128, 256):
        for h_kv in (1, 2):
            for sms in (1, 7, 148):
                assert lib.mla_num_parts(rows, h_kv, sms) == schedule.num_parts(rows, h_kv, sms)


def test_decode_rejects_bad_arguments_without_a_gpu(lib):
    # argument checks happen before any device call: null pointers, bad dims
    rc = lib.mla_decode_paged(None, None, 1, None, 1, None, 1, 1, 16, 1, 576, 512, None, None, 1, 0,
                              ctypes.c_float(0.04), None, 0, None, None, None, None)
    assert rc == -1


def test_traffic_records_name_existing_decode_sources():
    """The stored ncu traffic is reported only while the decode kernels' sources hash to the recorded
    value: every file in that hash must exist, and each record must name a hash of the same form."""
    import json
    import bench
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    csrc = os.path.join(root, "mla_paged_kv_get_b200", "csrc")
    for name in bench.DECODE_SOURCES:
        assert os.path.isfile(os.path.join(csrc, name)), name
    sha = bench.source_sha()
    assert re.fullmatch(r"[0-9a-f]{16}", sha)
    for rec in ("decode_compute_bound_traffic.json", "decode_varlen_memory_bound_traffic.json"):
        with open(os.path.join(root, "profiles", rec)) as f:
            d = json.load(f)
        assert re.fullmatch(r"[0-9a-f]{16}", d["kernel_source_sha"]) and d["dram_bytes_per_launch"] > 0
