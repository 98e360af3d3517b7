"""CPU-only checks of the C ABI: the library builds, loads without a GPU, exports every function
include/gsparse.h declares, and its host-only helpers agree with the oracle. No kernel runs."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gsparse.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(gsparse_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def gs():
    from compressed_sgd_b200 import build
    build.build()
    import compressed_sgd_b200
    return compressed_sgd_b200


def test_every_declared_symbol_is_exported(gs):
    lib = gs.lib()
    names = declared_functions()
    assert len(names) >= 16
    for name in names:
        assert hasattr(lib, name), name
    # the binding knows every declared entry point, with nothing extra
    assert sorted(gs.exported_symbols()) == names


def test_library_is_in_tree_sm100a_build(gs):
    assert os.path.dirname(gs.LIB_PATH).startswith(os.path.join(ROOT, "compressed_sgd_b200"))
    assert b"sm_100a" in gs.lib().gsparse_version()


def test_host_helpers_match_oracle(gs):
    for n in [0, 1, 99, 100, 101, 1 << 20, 1863690, (1 << 31) - 1]:
        for keep in [(0, 1), (1, 100), (1, 10), (1, 1000), (3, 7), (1, 1)]:
            assert gs.k_for(n, keep) == oracle.k_for(n, *keep)
    for p in [0.1, 0.01, 0.001, 0.5, 1e-6]:
        assert gs.golomb_b_star(p) == oracle.golomb_b_star(p)
    assert gs.k_for(10, (2, 1)) == -1 and gs.golomb_b_star(1.0) == -1
    for T in [0, 1, 4, 10]:
        for t in range(T + 2):
            for start, end in [(0.25, 0.001), (0.5, 0.01), (1.0, 1.0)]:
                assert gs.warmup_keep(t, T, start, end) == oracle.warmup_keep(t, T, start, end)


def test_workspace_queries(gs):
    lib = gs.lib()
    a = lib.gsparse_residual_topk_workspace_size(1 << 30, 1, 1, 100)
    b = lib.gsparse_residual_topk_workspace_min(1 << 30, 1)
    assert 0 < b < a < (1 << 30)            # well under 1 B per entry at a 99% drop
    assert lib.gsparse_residual_topk_workspace_size(-1, 1, 1, 100) == 0
    assert lib.gsparse_binarize_workspace_size(1000, 3, 1, 1000) > lib.gsparse_binarize_workspace_min(1000, 3, 1, 1000) - 1
    assert lib.gsparse_quantize_workspace_size(10 ** 6) > 0
    assert 0 < lib.gsparse_golomb_encode_workspace_size(10 ** 6) < 10 ** 5     # block totals only
    assert lib.gsparse_scatter_accumulate_workspace_size(4, 1 << 20) > 0
    for s in range(6):
        assert lib.gsparse_status_string(s)


def test_golomb_chunk_hint(gs):
    # the largest power of two in [4, 64] leaving at least 16384 chunks
    assert gs.golomb_chunk_hint(0) == 4 and gs.golomb_chunk_hint(25_558) == 4
    assert gs.golomb_chunk_hint(16384 * 64) == 64 and gs.golomb_chunk_hint(16384 * 64 - 1) == 32
    assert gs.golomb_chunk_hint(16384 * 8) == 8 and gs.golomb_chunk_hint(10_737_419) == 64
    for cap in [1, 1000, 10 ** 5, 10 ** 6, 10 ** 8]:
        c = gs.golomb_chunk_hint(cap)
        assert c in (4, 8, 16, 32, 64)
        assert c == 4 or cap // c >= 16384
        assert c == 64 or cap // (2 * c) < 16384
