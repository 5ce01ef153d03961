"""The C-ABI library builds, loads without a GPU, and exports every declared entry point."""

import ctypes
import os

import generative_recommender_sequence_b200 as hstu
from generative_recommender_sequence_b200 import build as build_mod


def test_library_exports_every_declared_symbol():
    build_mod.build()
    lib = hstu.load()
    names = hstu.declared_symbols()
    assert len(names) >= 16
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.hstu_version() == 100
    assert lib.hstu_status_string(2) == b"out of KV pages"


def test_binding_signatures_cover_the_header():
    from generative_recommender_sequence_b200 import _lib
    assert sorted(_lib._SIGNATURES) == hstu.declared_symbols()


def test_host_argument_checks_need_no_gpu():
    lib = hstu.load()
    # null / negative arguments are rejected on the host before any CUDA call
    assert lib.hstu_attn_fwd(None, None, None, None, -1, 0, 0, 4, 128, 128, 1, None, 1.0, None, None) == 1
    assert lib.hstu_attn_fwd(None, None, None, None, 0, 0, 0, 4, 96, 96, 1, None, 1.0, None, None) == 4
    out = ctypes.c_void_p()
    assert lib.hstu_kv_table_create(16, 16, 4, 128, 1, 8, 8, None, ctypes.byref(out)) == 1  # page size
    bad_perm = (ctypes.c_int32 * 4)(0, 1, 1, 3)
    assert lib.hstu_kv_table_create(4, 32, 4, 128, 1, 8, 8, ctypes.cast(bad_perm, ctypes.c_void_p),
                                    ctypes.byref(out)) == 1
    assert lib.hstu_block_fwd(None, None, 1, 1, 1, 1, 512, 4, 64, None, None, None, 1.0, 1e-5,
                              None, 0, None) == 4
    # the bounded-wait self test refuses limits outside 1 us .. 2 s before any launch
    assert lib.hstu_wait_timeout_selftest(0, None) == 1
    assert lib.hstu_wait_timeout_selftest(2000001, None) == 1
    # the one-call KV step: no table, a negative batch or bound, missing offsets
    assert lib.hstu_kv_step(None, None, None, None, None, 1, 1, None, None, 0, None) == 1
    assert lib.hstu_kv_step(None, None, None, None, None, -1, 1, None, None, 0, None) == 1
    assert lib.hstu_kv_step(None, None, None, None, None, 1, -1, None, None, 0, None) == 1


def test_oracle_is_not_imported_by_the_product_package():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "generative_recommender_sequence_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "hstu_oracle" not in text, f
