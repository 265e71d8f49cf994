"""The kernels' timeout path, run on purpose in the test-only fault-injection build.

Every on-chip wait in the library's kernels is bounded; when a bound is hit the kernel records
ATTN_ERR_TIMEOUT in the device status word, lets its own copies and tensor-core operations land,
frees its tensor memory and returns. libattn_faultinject.so is the same source built with
ATTN_FAULT_INJECT: waits give up after 20 ms, and ``attn_fault_inject(family, block)`` makes the
producer warp of CTA 0 skip one copy, so that the consumer waiting for it runs out of time. Each
test then checks (1) the status word says ATTN_ERR_TIMEOUT, (2) reading it cleared it, and (3) the
same process runs the same call correctly once injection is off -- the GPU context survived.
Nothing here traps, faults or spins without a bound.
"""
import ctypes

import numpy as np
import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
import oracle
from online_softmax_attention_fwd_b200 import _binding
from online_softmax_attention_fwd_b200 import build as build_mod
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_grad_bf16, assert_lse, assert_o_bf16, np64

pytestmark = pytest.mark.gpu

TIMEOUT = 6


@pytest.fixture(scope="module")
def faultlib():
    L = ctypes.CDLL(build_mod.FAULT_LIB_PATH)
    for name, res, args in _binding.SIGNATURES:
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    L.attn_fault_inject.restype = None
    L.attn_fault_inject.argtypes = [ctypes.c_int, ctypes.c_int]
    return L


@pytest.fixture()
def through(faultlib):
    """Routes the binding's calls to the fault-injection library for the duration of a test."""
    saved = _binding._lib
    _binding._lib = faultlib
    try:
        yield faultlib
    finally:
        faultlib.attn_fault_inject(-1, -1)
        _binding._lib = saved


def _status(L):
    return int(L.attn_get_device_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))


def test_forward_wait_runs_out_then_recovers(through):
    L = through
    w = W.random_prefill(1, 512, 512, 4, 2, 128, True, seed=51)
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (w.q, w.k, w.v))
    L.attn_fault_inject(0, 2)            # CTA 0 never loads its third K block
    attn.fwd(q, k, v, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == TIMEOUT
    assert _status(L) == 0               # reading the word cleared it
    L.attn_fault_inject(-1, -1)
    o, lse = attn.fwd(q, k, v, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == 0
    o_ref, lse_ref = oracle.attention_fwd(np64(w.q), np64(w.k), np64(w.v), True, w.scale)
    assert_o_bf16(np64(o), o_ref)
    assert_lse(np64(lse), lse_ref)


def test_backward_wait_runs_out_then_recovers(through):
    L = through
    w = W.random_prefill(1, 512, 512, 4, 2, 128, True, seed=52)
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (w.q, w.k, w.v, w.do))
    o, lse = attn.fwd(q, k, v, causal=True, scale=w.scale)
    L.attn_fault_inject(1, 5)            # CTA 0 never loads its sixth Q / dO tile
    attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == TIMEOUT
    assert _status(L) == 0
    L.attn_fault_inject(-1, -1)
    dq, dk, dv = attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == 0
    refs = oracle.attention_bwd(np64(w.q), np64(w.k), np64(w.v), np64(w.do), True, w.scale)
    for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        assert_grad_bf16(np64(g), r, name)


def test_decode_wait_runs_out_then_recovers(through):
    L = through
    w = W.random_decode(4, 8, 2, 128, [1000, 1000, 1000, 1000], seed=53)
    dev = torch.device("cuda")
    q, k, v, off = (t.to(dev) for t in (w.q, w.k, w.v, w.offsets))
    L.attn_fault_inject(2, 5)            # CTA 0 never fills its sixth ring block
    attn.decode(q, k, v, off, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == TIMEOUT
    assert _status(L) == 0
    L.attn_fault_inject(-1, -1)
    o, lse = attn.decode(q, k, v, off, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == 0
    o_ref, lse_ref = oracle.decode_attention(np64(w.q), np64(w.k), np64(w.v), w.offsets.numpy(), w.scale)
    assert_o_bf16(np64(o), o_ref)
    assert_lse(np64(lse), lse_ref)


def test_packed_forward_wait_runs_out_then_recovers(through):
    # the packed forward (item list built in shared memory) takes the same unwind path
    L = through
    w = W.packed_prefill([300, 0, 700, 129], [300, 0, 700, 129], 4, 2, 128, True, seed=54)
    dev = torch.device("cuda")
    q, k, v, cq, ck = (t.to(dev) for t in (w.q, w.k, w.v, w.cu_q, w.cu_k))
    L.attn_fault_inject(0, 2)
    attn.fwd_varlen(q, k, v, cq, ck, 700, 700, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == TIMEOUT
    assert _status(L) == 0
    L.attn_fault_inject(-1, -1)
    o, lse = attn.fwd_varlen(q, k, v, cq, ck, 700, 700, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == 0
    o_ref, lse_ref = oracle.attention_fwd_varlen(np64(w.q), np64(w.k), np64(w.v), w.cu_q.numpy(), w.cu_k.numpy(),
                                                 True, w.scale)
    assert_o_bf16(np64(o), o_ref)
    assert_lse(np64(lse), lse_ref)


def test_sequence_order_backward_wait_runs_out_then_recovers(through):
    # a batch large enough for the backward's sequence-by-sequence CTA order
    L = through
    w = W.random_prefill(3, 2048, 2048, 16, 4, 128, True, seed=55)
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (w.q, w.k, w.v, w.do))
    o, lse = attn.fwd(q, k, v, causal=True, scale=w.scale)
    L.attn_fault_inject(1, 5)
    attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == TIMEOUT
    assert _status(L) == 0
    L.attn_fault_inject(-1, -1)
    dq, dk, dv = attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _status(L) == 0
    refs = oracle.attention_bwd(np64(w.q), np64(w.k), np64(w.v), np64(w.do), True, w.scale)
    for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        assert_grad_bf16(np64(g), r, name)
