"""The C-ABI library on the CPU: it loads, exports every symbol include/ic.h declares,
and its host-side argument checks answer with status codes before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

from sparse_attention_indexer_sum_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ic.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ic_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(ic_\w+)$", out, flags=re.M))
    for name in _declared():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # nothing else leaks out with the C prefix
    assert exported == set(_declared())


def test_debug_bounds_library_exports_the_same_symbols():
    # the -DIC_DEBUG_BOUNDS build of the same sources (device-side index checks)
    path = build.build(debug_bounds=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    assert set(re.findall(r"\s[TW]\s+(ic_\w+)$", out, flags=re.M)) == set(_declared())
    assert ctypes.CDLL(path).ic_version() == binding.lib().ic_version()


def test_version_and_empty_error(lib):
    assert binding.ic_version() == 102
    assert isinstance(binding.ic_last_error(), str)


def _stack_call(lib, pattern, nlayers, desc=None):
    desc = desc or binding.make_desc(L=16, k=4, H=4, D=32, idx_dtype=binding.IC_F32, heads=4,
                                     dk=64, dv=64, attn_dtype=binding.IC_F32, scale=0.125)
    arr = (binding.ic_layer_io * max(nlayers, 1))()
    return lib.ic_layer_stack(pattern.encode() if pattern is not None else None,
                              ctypes.byref(desc), arr, nlayers, None, None, 0, None)


@pytest.mark.parametrize("pattern", ["", "S,F", "F,X", "f,s", " , "])
def test_stack_rejects_bad_patterns(lib, pattern):
    assert _stack_call(lib, pattern, 2) == binding.IC_ERR_INVALID_ARG
    assert "pattern" in binding.ic_last_error() or "first layer" in binding.ic_last_error()


def test_stack_rejects_layer_count_mismatch_and_null_inputs(lib):
    assert _stack_call(lib, "F,S,S", 2) == binding.IC_ERR_INVALID_ARG
    assert "layers" in binding.ic_last_error()
    # right count, but the layer inputs are NULL: caught before any launch
    assert _stack_call(lib, "F,S", 2) == binding.IC_ERR_INVALID_ARG
    assert "NULL" in binding.ic_last_error()


def test_stack_rejects_decode_flag_mismatch(lib):
    desc = binding.make_desc(L=16, k=4, H=4, D=32, idx_dtype=binding.IC_F32, heads=4, dk=64, dv=64,
                             attn_dtype=binding.IC_F32, scale=0.125, decode=True, batch=2)
    assert _stack_call(lib, "F", 1, desc) == binding.IC_ERR_INVALID_ARG
    assert "decode" in binding.ic_last_error()


def test_entry_points_reject_null_and_bad_sizes(lib):
    P = ctypes.c_void_p
    fake = P(256)  # never dereferenced: the checks fail first
    assert lib.ic_topk(None, 4, 10, 10, -1, 2, None, None) == binding.IC_ERR_INVALID_ARG
    assert lib.ic_topk(fake, 4, 10, 10, -1, 4096, fake, None) == binding.IC_ERR_INVALID_ARG
    assert lib.ic_topk(fake, 4, 10, 5, -1, 2, fake, None) == binding.IC_ERR_INVALID_ARG
    assert lib.ic_indexer_scores(fake, None, fake, None, fake, binding.IC_BF16, 1, 32, 128, 4, 8, 0,
                                 fake, 8, None) == binding.IC_ERR_UNSUPPORTED
    assert lib.ic_indexer_scores(fake, None, fake, None, fake, binding.IC_E4M3, 1, 64, 128, 4, 8, 0,
                                 fake, 8, None) == binding.IC_ERR_INVALID_ARG  # scales missing
    assert lib.ic_indexer_scores(fake, None, fake, None, fake, binding.IC_BF16, 1, 64, 128, 4, 8, -1,
                                 fake, 8, None) == binding.IC_ERR_INVALID_ARG  # pos0 < 0
    assert lib.ic_sparse_attn(fake, fake, 576, None, fake, binding.IC_BF16, 1, 4, 8, 576, 512, 16,
                              8, 1.0, fake, None, None, 0, None) == binding.IC_ERR_UNSUPPORTED
    assert lib.ic_quant_e4m3_rows(fake, binding.IC_BF16, 4, 100, fake, fake,
                                  None) == binding.IC_ERR_INVALID_ARG


def test_workspace_sizes(lib):
    d = binding.make_desc(L=200000, k=2048, H=64, D=128, idx_dtype=binding.IC_BF16, heads=16,
                          dk=576, dv=512, attn_dtype=binding.IC_BF16, scale=576 ** -0.5)
    assert binding.ic_stack_workspace_size(d) == 4096 * 200000 * 4
    assert binding.ic_attn_workspace_size(1, 200000, 16, 512, 2048) == 0  # no split at prefill


def test_row_range_stack_rejects_rows_outside_the_sequence(lib):
    desc = binding.make_desc(L=16, k=4, H=4, D=32, idx_dtype=binding.IC_F32, heads=4, dk=64, dv=64,
                             attn_dtype=binding.IC_F32, scale=0.125)
    arr = (binding.ic_layer_io * 1)()
    for row0, rows in ((10, 7), (-1, 4), (0, -2)):
        assert lib.ic_layer_stack_rows(b"F", ctypes.byref(desc), arr, 1, row0, rows, None, None, 0,
                                       None) == binding.IC_ERR_INVALID_ARG
        assert "outside" in binding.ic_last_error()
    # a valid range gets as far as the NULL layer inputs
    assert lib.ic_layer_stack_rows(b"F", ctypes.byref(desc), arr, 1, 4, 8, None, None, 0,
                                   None) == binding.IC_ERR_INVALID_ARG
    assert "NULL" in binding.ic_last_error()


def test_varlen_stack_rejects_bad_sequence_offsets(lib):
    desc = binding.make_desc(L=16, k=4, H=4, D=32, idx_dtype=binding.IC_F32, heads=4, dk=64, dv=64,
                             attn_dtype=binding.IC_F32, scale=0.125)
    arr = (binding.ic_layer_io * 1)()
    for cu in ([1, 4], [0, 8, 4], [0, 17]):
        c = (ctypes.c_long * len(cu))(*cu)
        assert lib.ic_layer_stack_varlen(b"F", ctypes.byref(desc), arr, 1, c, len(cu) - 1, None,
                                         None, 0, None) == binding.IC_ERR_INVALID_ARG
        assert "varlen" in binding.ic_last_error()


def test_indexer_topk_rejects_before_launch(lib):
    fake = ctypes.c_void_p(256)  # never dereferenced: the checks fail first
    # fp32 has no fused path
    st = lib.ic_indexer_topk(fake, None, fake, None, fake, binding.IC_F32, 2, 4, 32, 100, 99, 8,
                             fake, fake, 1 << 20, None)
    assert st == binding.IC_ERR_UNSUPPORTED
    # k outside [1, 2048]
    st = lib.ic_indexer_topk(fake, None, fake, None, fake, binding.IC_BF16, 2, 64, 128, 100, 99,
                             4096, fake, fake, 1 << 20, None)
    assert st == binding.IC_ERR_INVALID_ARG
    # e4m3 without scales
    st = lib.ic_indexer_topk(fake, None, fake, None, fake, binding.IC_E4M3, 2, 64, 128, 100, 99,
                             16, fake, fake, 1 << 20, None)
    assert st == binding.IC_ERR_INVALID_ARG
    assert binding.ic_indexer_topk_workspace_size(0, 100, 99) == 0


def test_topk_varlen_rejects_before_launch(lib):
    fake = ctypes.c_void_p(256)
    assert lib.ic_topk_varlen(fake, 4, 100, 100, None, 8, fake, None) == binding.IC_ERR_INVALID_ARG
    assert lib.ic_topk_varlen(fake, 4, 100, 50, fake, 8, fake, None) == binding.IC_ERR_INVALID_ARG


def test_pack_kv_and_fp8_attention_reject_before_launch(lib):
    fake = ctypes.c_void_p(256)
    assert lib.ic_pack_kv_e4m3(fake, 4, 570, fake, 656, None) == binding.IC_ERR_INVALID_ARG
    assert lib.ic_pack_kv_e4m3(fake, 4, 576, fake, 650, None) == binding.IC_ERR_INVALID_ARG
    # an fp8 cache needs rows of at least 656 bytes, a multiple of 16
    st = lib.ic_sparse_attn(fake, fake, 576, None, fake, binding.IC_E4M3, 1, 4, 16, 576, 512, 100,
                            64, 1.0, fake, None, None, 0, None)
    assert st == binding.IC_ERR_INVALID_ARG
