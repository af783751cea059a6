"""The C-ABI library loads and exports every entry point of include/lb.h (CPU only).

Only argument-validation paths are called here: they return before any CUDA call.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "lb.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lb_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lb():
    from binary_rank_linear_lb_b200 import build
    build.build()
    import binary_rank_linear_lb_b200 as m
    return m


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("lb_pack_signs", "lb_linear_forward", "lb_stack_forward"):
        assert must in names


def test_every_declared_symbol_is_exported(lb):
    L = ctypes.CDLL(lb.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert set(lb.EXPORTS) <= set(declared_functions())


def test_status_strings(lb):
    L = lb.lib()
    assert L.lb_status_string(0) == b"LB_OK"
    assert L.lb_status_string(5) == b"LB_ERR_TIMEOUT"
    assert L.lb_status_string(99) == b"LB_ERR_UNKNOWN"
    assert L.lb_version() >= 100


def test_argument_errors_return_before_any_launch(lb):
    L = lb.lib()
    assert L.lb_pack_signs(None, 4, 4, 4, 0, None, 1, None) == lb.LB_ERR_INVALID_ARG
    assert L.lb_pack_signs(16, 4, 4, 4, 2, 16, 1, None) == lb.LB_ERR_INVALID_ARG
    assert L.lb_pack_signs(16, 4, 40, 40, 1, 16, 1, None) == lb.LB_ERR_INVALID_ARG
    assert L.lb_pack_signs(18, 4, 4, 4, 1, 16, 1, None) == lb.LB_ERR_ALIGNMENT
    br = (lb.lb_branch * 2)(lb.lb_branch(16, 16, 16, 16, 16), lb.lb_branch(16, 16, 16, 16, 16))
    a = ctypes.addressof(br)
    assert L.lb_linear_forward(None, 0, 1, 64, 64, 32, a, 2, 16, 16, 1 << 20, None) == \
        lb.LB_ERR_INVALID_ARG
    assert L.lb_linear_forward(16, 0, 1, 64, 64, 0, a, 2, 16, 16, 1 << 20, None) == \
        lb.LB_ERR_INVALID_ARG
    assert L.lb_linear_forward(16, 0, 1, 64, 64, 32, a, 3, 16, 16, 1 << 20, None) == \
        lb.LB_ERR_INVALID_ARG
    assert L.lb_linear_forward(16, 7, 1, 64, 64, 32, a, 2, 16, 16, 1 << 20, None) == \
        lb.LB_ERR_INVALID_ARG
    assert L.lb_linear_forward(24, 0, 1, 64, 64, 32, a, 2, 16, 16, 1 << 20, None) == \
        lb.LB_ERR_ALIGNMENT
    assert L.lb_linear_forward(16, 0, 1, 64, 64, 32, a, 2, 16, 16, 8, None) == \
        lb.LB_ERR_WORKSPACE
    assert L.lb_linear_workspace_size(1, 64, 64, 32, 2) >= 256 + 2 * 32 * 4
    assert L.lb_linear_workspace_size(1, 64, 64, 0, 2) == 0


def test_stack_workspace_size_is_host_only(lb):
    L = lb.lib()
    nl, nb = 2, 2
    brs = (lb.lb_branch * (nl * 7 * nb))(*[lb.lb_branch(256, 256, 256, 256, 256)
                                          for _ in range(nl * 7 * nb)])
    ranks = (ctypes.c_int64 * (nl * 7))(*([64] * (nl * 7)))
    d = lb.lb_stack_desc(nl, 256, 512, 4, 2, 64, nb, 0, ctypes.addressof(brs),
                         ctypes.addressof(ranks))
    size = L.lb_stack_workspace_size(ctypes.byref(d))
    assert size > 0 and size % 256 == 0
    bad = lb.lb_stack_desc(nl, 256, 512, 4, 3, 64, nb, 0, ctypes.addressof(brs),
                           ctypes.addressof(ranks))
    assert L.lb_stack_workspace_size(ctypes.byref(bad)) == 0
    assert L.lb_stack_forward(ctypes.byref(bad), 256, size, 256, 256, None) == \
        lb.LB_ERR_INVALID_ARG


def test_sliced_layout_sizes_and_argument_errors(lb):
    L = lb.lib()
    S, R = lb.LB_LAYOUT_SLICES, lb.LB_LAYOUT_ROWS
    # n rows of k signs: full 16-word slices, then the last slice's words rounded up to 4
    for n, k, words in ((1, 1, 4), (3, 512, 48), (2, 513, 2 * (16 + 4)), (5, 3136, 5 * (96 + 4)),
                        (7, 1100, 7 * (32 + 4)), (4, 8192, 4 * 256)):
        assert L.lb_packed_words(n, k, S, 0) == words
    assert L.lb_packed_words(3, 100, R, 0) == 3 * 4
    assert L.lb_packed_words(3, 100, R, 9) == 27
    assert L.lb_packed_words(3, 100, R, 2) == 0          # pitch below ceil(k/32)
    assert L.lb_packed_words(3, 100, 7, 0) == 0          # no such layout
    assert L.lb_packed_words(0, 100, S, 0) == 0
    assert L.lb_pack_signs_sliced(None, 4, 4, 4, 0, 16, None) == lb.LB_ERR_INVALID_ARG
    assert L.lb_pack_signs_sliced(16, 4, 4, 4, 2, 16, None) == lb.LB_ERR_INVALID_ARG
    assert L.lb_pack_signs_sliced(16, 4, 4, 4, 1, 24, None) == lb.LB_ERR_ALIGNMENT
    # a sliced branch takes no row pitch, and the layout must be known
    for ld_v, layout in ((4, S), (0, 9)):
        br = (lb.lb_branch * 1)(lb.lb_branch(16, 16, 16, 16, 16, ld_v, 0, layout, 0))
        assert L.lb_linear_forward(16, 0, 1, 64, 64, 32, ctypes.addressof(br), 1, 16, 16,
                                   1 << 20, None) == lb.LB_ERR_INVALID_ARG
