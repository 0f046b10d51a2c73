"""libep.so loads without a GPU, exports every entry point include/ep.h
declares, and its host-only calls behave as the header says."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ep.h")


@pytest.fixture(scope="module")
def lib():
    from combine_topk_idx_rank_b200 import build
    return C.CDLL(build.build())


def declared_functions(header=HEADER):
    src = open(header).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(ep_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("ep_get_dispatch_layout", "ep_dispatch", "ep_combine", "ep_read_error",
              "ep_workspace_bytes", "ep_recv_capacity_bound", "ep_copy_recv_counts",
              "ep_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_testing_header_symbols_are_exported(lib):
    names = declared_functions(os.path.join(ROOT, "include", "ep_testing.h"))
    assert names == ["ep_testing_dispatch_stalled", "ep_testing_get_dispatch_layout_stalled"]
    for n in names:
        assert hasattr(lib, n), n


def test_no_environment_switch_in_the_library():
    # the bounded-wait tests reach the stalled routing through ep_testing.h only
    for f in os.listdir(os.path.join(ROOT, "combine_topk_idx_rank_b200", "csrc")):
        src = open(os.path.join(ROOT, "combine_topk_idx_rank_b200", "csrc", f)).read()
        assert "getenv" not in src, f


def test_binding_exports_match_header():
    from combine_topk_idx_rank_b200 import ep
    assert sorted(ep.EXPORTED) == declared_functions()


def test_host_helpers(lib):
    lib.ep_recv_capacity_bound.restype = C.c_int64
    lib.ep_workspace_bytes.restype = C.c_size_t
    lib.ep_status_string.restype = C.c_char_p
    assert lib.ep_recv_capacity_bound(32768, 8, 256, 128) == 32768 * 8 + 256 * 127
    assert lib.ep_recv_capacity_bound(10, 2, 4, 1) == 20
    ws = lib.ep_workspace_bytes(32768, 8, 256, 8)
    assert ws % 256 == 0 and ws >= 128 * 256 * 4       # histogram of 128 chunks (256 tokens) x 256 experts
    assert lib.ep_workspace_bytes(100, 8, 256, 8) == 0  # T % R != 0 -> rejected
    assert lib.ep_workspace_bytes(64, 17, 256, 8) == 0  # K > 16
    assert lib.ep_status_string(3) == b"receive capacity too small"


def test_invalid_arguments_return_before_any_launch(lib):
    # every call below fails validation on the host, so no CUDA call is made
    p = C.c_void_p
    lib.ep_dispatch.restype = C.c_int
    lib.ep_combine.restype = C.c_int
    lib.ep_get_dispatch_layout.restype = C.c_int
    lib.ep_read_error.restype = C.c_int
    args = [p(None), 64, 512, p(None), p(None), 2, 16, 8, p(None), p(None), p(None), p(None), p(None),
            C.c_int64(0), p(None), p(None), p(None), p(None), p(None), C.c_size_t(0), p(None)]
    assert lib.ep_dispatch(*args) == 1                  # opts == NULL
    assert lib.ep_combine(p(None), p(None), p(None), p(None), p(None)) == 1
    assert lib.ep_get_dispatch_layout(p(None), 64, 2, 16, 3, p(None), p(None), p(None), p(None),
                                      p(None), C.c_size_t(0), p(None)) == 1   # E % R != 0
    assert lib.ep_read_error(p(None), p(None), p(None)) == 1
