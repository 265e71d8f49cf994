"""The C ABI library loads, exports every symbol include/attn.h declares, and validates arguments on
the host before launching anything (CPU only: no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

import online_softmax_attention_fwd_b200 as attn
from online_softmax_attention_fwd_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return attn.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported_and_bound(L):
    names = declared_functions()
    assert len(names) >= 13
    bound = {n for n, _, _ in attn.SIGNATURES}
    for n in names:
        assert hasattr(L, n), f"{n} not exported"
        assert n in bound, f"{n} has no ctypes signature in the binding"


def test_status_strings(L):
    for code in range(7):
        assert attn.status_string(code)
    assert "timed out" in attn.status_string(6)


@pytest.mark.parametrize("L_,expect", [(0, 4), (1, 4), (256, 4), (1024, 4), (1025, 5), (2048, 8),
                                       (4096, 16), (4097, 16), (100000, 16)])
def test_default_split_rule(L, L_, expect):
    assert attn.default_splits(L_, 16) == expect
    assert attn.default_splits(L_, 3) == min(3, expect)


def test_workspace_sizes(L):
    ws = attn.decode_workspace_size(48, 32, 128, 16)
    assert ws >= 48 * 32 * 16 * (128 + 2) * 4 and ws % 256 == 0
    assert attn.bwd_workspace_size(1, 32, 8, 4096, 4096, 128) >= 32 * 4096 * 4
    assert attn.decode_workspace_size(0, 32, 128, 16) == 0


A = ctypes.c_void_p(0x100000)     # a 16-byte aligned, never dereferenced stand-in address
U = ctypes.c_void_p(0x100004)     # misaligned


def fwd_call(L, q=A, o=A, B=1, Hq=2, Hkv=2, Sq=8, Sk=8, D=64, causal=0):
    return L.attn_fwd(q, A, A, o, A, B, Hq, Hkv, Sq, Sk, D, causal, 0.125, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(B=0), 1), (dict(Sq=-1), 1), (dict(Hq=3, Hkv=2), 1),
    (dict(causal=2), 1), (dict(q=U), 3), (dict(D=96), 2), (dict(D=256), 2)])
def test_forward_argument_errors(L, kw, code):
    assert fwd_call(L, **kw) == code


def test_backward_workspace_errors(L):
    need = L.attn_bwd_workspace_size(1, 2, 2, 8, 8, 64)
    args = [A] * 9
    assert L.attn_bwd(*args, None, need, 1, 2, 2, 8, 8, 64, 0, 0.1, None) == 4
    assert L.attn_bwd(*args, A, need - 1, 1, 2, 2, 8, 8, 64, 0, 0.1, None) == 4
    assert L.attn_bwd(*args, ctypes.c_void_p(0x100010), need, 1, 2, 2, 8, 8, 64, 0, 0.1, None) == 3


def test_decode_argument_errors(L):
    ws = L.attn_decode_workspace_size(4, 8, 128, 16)
    base = dict(max_splits=16, N=4, Hq=8, Hkv=2, D=128, ws=A, wsb=ws)

    def call(**kw):
        a = {**base, **kw}
        return L.attn_decode_splitkv(A, A, A, A, None, a["max_splits"], A, A, a["N"], a["Hq"], a["Hkv"],
                                     a["D"], 0.1, a["ws"], a["wsb"], None)
    assert call(N=0) == 1
    assert call(Hq=6, Hkv=4) == 1
    assert call(max_splits=0) == 1
    assert call(max_splits=65) == 1
    assert call(D=80) == 2
    assert call(wsb=ws - 1) == 4
    assert call(ws=None) == 4


def test_paged_decode_argument_errors(L):
    ws = L.attn_decode_workspace_size(4, 8, 128, 16)
    base = dict(bt=A, max_pages=8, lens=A, page_size=64, num_pages=100, max_splits=16, N=4, Hq=8, Hkv=2,
                D=128, ws=A, wsb=ws)

    def call(**kw):
        a = {**base, **kw}
        return L.attn_decode_paged(A, A, A, a["bt"], a["max_pages"], a["lens"], a["page_size"], a["num_pages"],
                                   None, a["max_splits"], A, A, a["N"], a["Hq"], a["Hkv"], a["D"], 0.1, a["ws"],
                                   a["wsb"], None)
    assert call(page_size=8) == 1          # below one 16-key block
    assert call(page_size=24) == 1         # not a multiple of 16
    assert call(num_pages=0) == 1
    assert call(max_pages=0) == 1
    assert call(num_pages=1 << 26, page_size=64) == 1   # pool rows past 2^31
    assert call(lens=None) == 1
    assert call(bt=None) == 1
    assert call(bt=U) == 3
    assert call(lens=U) == 3
    assert call(Hq=6, Hkv=4) == 1
    assert call(D=80) == 2
    assert call(wsb=ws - 1) == 4


def test_launch_counter_and_last_path_without_gpu(L):
    assert attn.launch_count() >= 0
    assert isinstance(attn.last_path(0), str)
    assert attn.last_path(7) == "none"


def test_fault_injection_switch_only_in_the_test_build(L):
    # libattn.so never exports the test-only switch; the fault-injection build does
    import subprocess
    shipped = subprocess.run(["nm", "-D", "--defined-only", build_mod.LIB_PATH], capture_output=True, text=True).stdout
    test_build = subprocess.run(["nm", "-D", "--defined-only", build_mod.FAULT_LIB_PATH], capture_output=True,
                                text=True).stdout
    assert "attn_fault_inject" not in shipped
    assert "attn_fault_inject" in test_build
