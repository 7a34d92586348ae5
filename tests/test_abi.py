"""CPU checks of the C ABI: the library loads, exports every function its header
declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def L():
    from sparse_attention_04_b200 import build
    build.build()
    from sparse_attention_04_b200 import _lib
    return _lib


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    fns = declared_functions()
    for f in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla", "dsa_decode_step"):
        assert f in fns


def test_every_declared_function_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dsa_\w+)", out))
    for f in declared_functions():
        assert f in exported, f
        assert hasattr(L.lib, f)
    assert set(L.EXPORTS) == set(declared_functions())


def test_status_strings_and_version(L):
    for code, name in L.STATUS.items():
        assert L.status_string(code).startswith(name)
    assert L.status_string(99) == "DSA_ERR_UNKNOWN"
    assert L.lib.dsa_version() == 100


P = lambda x: ctypes.c_void_p(x)
A = 4096  # a 16-byte-aligned fake device address: validation must fail before any use


def test_topk_argument_validation(L):
    f = L.lib.dsa_topk
    assert f(P(A), 64, P(A), 1, 1, 0, P(A), None, None) == 1          # k = 0
    assert f(P(A), 64, P(A), 1, 1, 2049, P(A), None, None) == 1       # k > 2048
    assert f(None, 64, P(A), 1, 1, 8, P(A), None, None) == 1          # NULL scores
    assert f(P(A), 63, P(A), 1, 1, 8, P(A), None, None) == 1          # ld not a multiple of 4
    assert f(P(A), 64, P(A), 0, 1, 8, P(A), None, None) == 1          # B = 0
    assert f(P(A + 4), 64, P(A), 1, 1, 8, P(A), None, None) == 1      # misaligned


def test_indexer_argument_validation(L):
    f = L.lib.dsa_indexer_scores
    ok = [P(A), P(A), P(A), None, 0, P(A), 1, 1, 1024, P(A), 1024, None, None]
    bad_dtype = list(ok); bad_dtype[4] = 7
    assert f(*bad_dtype) == 1
    e4m3_no_scale = list(ok); e4m3_no_scale[4] = 1
    assert f(*e4m3_no_scale) == 1
    bad_ld = list(ok); bad_ld[10] = 1022
    assert f(*bad_ld) == 1
    no_q = list(ok); no_q[0] = None
    assert f(*no_q) == 1


def test_sparse_mla_argument_validation(L):
    f = L.lib.dsa_sparse_mla
    base = [P(A), P(A), P(A), P(A), 1, 1, 128, 2048, 0.07, 4096, P(A), 0, None, None, 0, None, None]
    too_many_heads = list(base); too_many_heads[6] = 129
    assert f(*too_many_heads) == 2
    bad_out = list(base); bad_out[11] = 1
    assert f(*bad_out) == 1
    need = L.sparse_mla_workspace_size(1, 1, 128, 2048)
    assert need > 0                                               # B=1 decode splits the keys
    assert f(*base) == 3                                          # workspace missing
    small = list(base); small[13] = P(A); small[14] = need - 16
    assert f(*small) == 3
    nan_scale = list(base); nan_scale[8] = float("nan")
    assert f(*nan_scale) == 1


def test_host_copy_validation(L):
    h2d, d2h = L.lib.dsa_copy_host_to_device, L.lib.dsa_copy_device_to_host
    assert h2d(P(A), P(A), 0, None) == 0                          # nothing to copy
    assert h2d(P(A), P(A), 24, None) == 1                         # not a multiple of 16
    assert h2d(None, P(A), 32, None) == 1 and d2h(P(A), None, 32, None) == 1
    assert d2h(P(A + 8), P(A), 32, None) == 1                     # misaligned


def test_workspace_sizes(L):
    s_off, ld, i_off, m_off = L.decode_step_workspace_layout(32, 131072, 2048, 128)
    assert s_off == 0 and ld == 131072 and i_off >= 32 * ld * 4 and m_off >= i_off + 32 * 2048 * 4
    assert i_off % 256 == 0 and m_off % 256 == 0
    assert L.decode_step_workspace_size(1, 32768, 2048, 128) >= m_off * 0
    assert L.decode_step_workspace_size(0, 10, 10, 10) == 0
    assert L.sparse_mla_workspace_size(4096, 1, 128, 2048) == 0     # prefill: one split per row
    f = L.lib.dsa_decode_step
    args = [P(A), P(A), P(A), None, 0, P(A), P(A), P(A), 1, 32768, 32768, 2048, 128, 0.07, P(A), 0,
            None, P(A), 1024, None, None]
    assert f(*args) == 3


def test_stall_hook_rejects_bad_limits(L):
    """The timeout test hook checks its arguments on the host."""
    f = L.lib.dsa_debug_stall_attention
    assert f(1, 10) == 1                # limit below 1 ms
    assert f(1, 5 * 10 ** 9) == 1       # above 1 s
    assert f(-1, 5_000_000) == 1        # negative count
    assert f(0, 0) == 0                 # cancel
