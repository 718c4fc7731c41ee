"""The C-ABI library on a machine without a GPU: it loads, exports every symbol that
include/dllm.h declares, and rejects invalid arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from mask_only_logits_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dllm.h")


@pytest.fixture(scope="module")
def lib():
    build.build()                       # no-op when libdllm.so is up to date
    return _abi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)          # drop comments
    return sorted(set(re.findall(r"\b(dllm_[a-z_0-9]+)\s*\(", text)))


def test_header_and_bindings_agree():
    assert declared_functions() == sorted(_abi.PROTOTYPES)


def test_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # and nothing but C symbols: the names are not mangled
    nm = os.popen(f"nm -D --defined-only {_abi.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (dllm_\w+)", nm))
    assert set(declared_functions()) <= exported


def test_version_and_status_strings(lib):
    assert lib.dllm_version() == 10200
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9, -10, -11):
        assert lib.dllm_status_string(code)
    assert lib.dllm_status_string(-99) == b"unknown status"


def test_workspace_bytes(lib):
    ws = lib.dllm_workspace_bytes
    assert ws(1, 256, 256, 4096) > 256 * 256 * 2
    # grows with B*L*d (the gathered rows dominate), never shrinks with more rows
    assert ws(1, 4096, 4096, 126464) >= 4096 * 4096 * 2
    assert ws(1, 131072, 4096, 126464) >= 131072 * 4096 * 2
    assert ws(8, 8192, 2048, 151936) >= 8 * 8192 * 2048 * 2
    # invalid shapes -> 0
    assert ws(0, 10, 64, 10) == 0
    assert ws(1, 0, 64, 10) == 0
    assert ws(1, 10, 100, 10) == 0           # d not a multiple of 64
    assert ws(1, 10, 64, 0) == 0
    assert ws(1 << 16, 1 << 15, 64, 10) == 0  # B*L >= 2^31


def test_workspace_rows_arithmetic(lib):
    """A workspace sized for max_rows masked rows: at least the gathered rows, growing with
    max_rows, equal to the upper bound at B*L; the capacity of a workspace is the largest
    row count whose size fits, so sizing for r rows gives a capacity of at least r."""
    rows_b, cap = lib.dllm_workspace_bytes_rows, lib.dllm_workspace_rows
    for B, L, d, V in [(1, 131072, 4096, 126464), (8, 8192, 2048, 151936), (1, 256, 256, 4096),
                       (3, 97, 192, 777)]:
        n = B * L
        full = lib.dllm_workspace_bytes(B, L, d, V)
        assert rows_b(B, L, d, V, n) == full and rows_b(B, L, d, V, 10 * n) == full
        prev = 0
        for r in sorted({1, 2, 127, 128, 129, 4096, n // 10, n // 2, (9 * n) // 10, n - 1, n}):
            if r < 1 or r > n:
                continue
            b = rows_b(B, L, d, V, r)
            assert b >= 2 * d * r and b >= prev and b <= full, (B, L, d, V, r)
            prev = b
            c = cap(B, L, d, V, b)
            assert r <= c <= n and rows_b(B, L, d, V, c) <= b, (r, c)
            if c < n:
                assert rows_b(B, L, d, V, c + 1) > b                     # the largest that fits
            assert cap(B, L, d, V, b - 1) < r or rows_b(B, L, d, V, r) <= b - 1
        assert cap(B, L, d, V, full) == n and cap(B, L, d, V, 1 << 62) == n
        assert cap(B, L, d, V, rows_b(B, L, d, V, 1) - 1) == 0
    # the cfg3 sweep: the workspace of a step follows its masked count
    B, L, d, V = 1, 131072, 4096, 126464
    for r_m in (0.1, 0.5, 0.9):
        m = int(r_m * L)
        assert rows_b(B, L, d, V, m) < lib.dllm_workspace_bytes(B, L, d, V) * (r_m + 0.02)
    assert rows_b(B, L, d, V, 0) == 0 and rows_b(0, L, d, V, 5) == 0
    assert cap(B, L, 100, V, 1 << 30) == 0


def test_arena_validates_on_host(lib):
    out = ctypes.c_void_p()
    assert lib.dllm_arena_create(1 << 20, 0, None) == -1
    assert lib.dllm_arena_create(0, 0, ctypes.byref(out)) == -3
    assert lib.dllm_arena_map(None, 10) == -1
    assert lib.dllm_arena_ptr(None) is None
    assert lib.dllm_arena_mapped(None) == 0 and lib.dllm_arena_reserved(None) == 0
    assert lib.dllm_arena_chunk(None) == 0
    assert lib.dllm_arena_destroy(None) == 0


def _p(x):
    return ctypes.c_void_p(x)


def test_host_validation_without_gpu(lib):
    """Every rejection happens before any CUDA call, so it works on a CPU-only machine."""
    a = 1 << 20                                    # a 16-byte aligned fake address
    nul = _p(None)
    # mask_compact
    assert lib.dllm_mask_compact(nul, 1, 8, _p(a), _p(a), _p(a), _p(a), 1 << 20, nul) == -1
    assert lib.dllm_mask_compact(_p(a), 0, 8, _p(a), _p(a), _p(a), _p(a), 1 << 20, nul) == -3
    assert lib.dllm_mask_compact(_p(a + 1), 1, 8, _p(a), _p(a), _p(a), _p(a), 1 << 20, nul) == -2
    assert lib.dllm_mask_compact(_p(a), 1, 8, _p(a), _p(a), _p(a), _p(a), 0, nul) == -4
    # masked_logits
    args = [_p(a), _p(a), _p(a), 1, 256, 256, 4096, _p(a), _p(a), _p(a), _p(a), _p(a), _p(a)]
    assert lib.dllm_masked_logits(*args, _p(a), 10, nul) == -4             # workspace too small
    bad_d = list(args)
    bad_d[5] = 100
    assert lib.dllm_masked_logits(*bad_d, _p(a), 1 << 30, nul) == -3
    bad_al = list(args)
    bad_al[2] = _p(a + 8)
    assert lib.dllm_masked_logits(*bad_al, _p(a), 1 << 30, nul) == -2
    null_tok = list(args)
    null_tok[7] = nul
    assert lib.dllm_masked_logits(*null_tok, _p(a), 1 << 30, nul) == -1
    # select_unmask
    sel = [_p(a), _p(a), _p(a), 1, 16]
    assert lib.dllm_select_unmask(*sel, 0, nul, nul, nul, _p(a), _p(a), nul, nul, nul) == -3
    assert lib.dllm_select_unmask(*sel, 1025, nul, nul, nul, _p(a), _p(a), nul, nul, nul) == -3
    assert lib.dllm_select_unmask(*sel, 4, _p(a), nul, nul, _p(a), _p(a), nul, nul, nul) == -1
    assert lib.dllm_select_unmask(*sel, 4, nul, nul, nul, _p(a), _p(a), _p(a), nul, nul) == -1
    assert lib.dllm_select_unmask(*sel, 4, nul, nul, nul, _p(a + 4), _p(a), nul, nul, nul) == -2
    # decode_step checks the selection arguments before launching anything
    step = [_p(a), _p(a), _p(a), 1, 256, 256, 4096]
    assert lib.dllm_decode_step(*step, 0, nul, nul, *[_p(a)] * 6, _p(a), _p(a), nul, nul,
                                _p(a), 1 << 30, nul) == -3
    # merge hook
    assert lib.dllm_debug_lse_merge(nul, _p(a), _p(a), 4, 2, _p(a), _p(a), _p(a), nul) == -1
    assert lib.dllm_debug_lse_merge(_p(a), _p(a), _p(a), 0, 2, _p(a), _p(a), _p(a), nul) == -3


def test_window_entry_points_validate_on_host(lib):
    a = 1 << 20
    nul = _p(None)
    # compaction: exactly one window pointer given, or a misaligned one
    assert lib.dllm_mask_compact_window(_p(a), 1, 8, _p(a), nul, _p(a), _p(a), _p(a), _p(a),
                                        1 << 20, nul) == -1
    assert lib.dllm_mask_compact_window(_p(a), 1, 8, _p(a), _p(a + 4), _p(a), _p(a), _p(a), _p(a),
                                        1 << 20, nul) == -2
    assert lib.dllm_mask_compact_window(_p(a), 0, 8, _p(a), _p(a), _p(a), _p(a), _p(a), _p(a),
                                        1 << 20, nul) == -3
    # current-block-only logits: windows are required
    ins = [_p(a), _p(a), _p(a), 1, 256, 256, 4096]
    outs = [_p(a), _p(a), _p(a), nul, nul, _p(a), _p(a), _p(a), _p(a), 1 << 30, nul]
    assert lib.dllm_masked_logits_window(*ins, nul, nul, 0, *outs) == -1
    assert lib.dllm_masked_logits_window(*ins, _p(a), nul, 0, *outs) == -1
    assert lib.dllm_masked_logits_window(*ins, _p(a), _p(a), 4, *outs) == -3      # unknown stat
    small_ws = outs[:-2] + [10, nul]
    assert lib.dllm_masked_logits_window(*ins, _p(a), _p(a), 0, *small_ws) == -4
    # block step: windows required, k checked before any launch
    assert lib.dllm_decode_block_step(*ins, 4, nul, nul, *[_p(a)] * 6, _p(a), _p(a), nul, nul,
                                      _p(a), 1 << 30, nul) == -1
    assert lib.dllm_decode_block_step(*ins, 0, _p(a), _p(a), *[_p(a)] * 6, _p(a), _p(a), nul, nul,
                                      _p(a), 1 << 30, nul) == -3


def test_graft_entry_build_accepts_this_library(lib, monkeypatch):
    """__graft_entry__.build() imports the package and checks the ABI version; run it here
    with the (already built) library so that a version bump cannot break it unnoticed."""
    import importlib
    import sys
    monkeypatch.syspath_prepend(ROOT)
    entry = importlib.import_module("__graft_entry__")
    monkeypatch.setattr(build, "build", lambda *a, **k: _abi.LIB_PATH)
    entry.build()
    assert "mask_only_logits_b200" in sys.modules
