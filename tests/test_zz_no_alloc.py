"""The split-KV decode entry point that allocates nothing: attn_decode_splitkv_static.

It exists for callers of this library that cannot give it device scratch memory -- a host framework
that owns all device memory through its own pool and hands plugins no workspace, or a latency-bound
serving loop that may not call cudaMalloc on its hot path. Its partial (m, l, o) triples live in a
fixed 16 MiB array inside the library instead of a caller workspace, so its results must equal
those of attn_decode_splitkv, and they must stay right when the array is reused by the next call.

This file is collected last on purpose, so that a run stopping at the first failure has already
run every other test; it passes both alone and after the rest of the suite.
"""
import ctypes

import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_lse, assert_o_bf16, np64

A = ctypes.c_void_p(0x100000)  # aligned stand-in address; never dereferenced by the host checks


def _static_decode(q, k, v, offsets, max_splits=16):
    N, Hq, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((N, Hq), dtype=torch.float32, device=q.device)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    status = attn.lib().attn_decode_splitkv_static(
        p(q), p(k), p(v), p(offsets), None, max_splits, p(o), p(lse), N, Hq, k.shape[1], D,
        1.0 / D ** 0.5, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return status, o, lse


@pytest.mark.gpu
def test_static_decode_matches_workspace_decode_on_two_calls_in_a_row():
    dev = torch.device("cuda")
    batches = [W.decode48(),
               W.random_decode(7, 32, 8, 128, [1, 4096, 0, 777, 2048, 3000, 5], seed=3)]
    inputs, refs = [], []
    for w in batches:
        q, k, v, off = (t.to(dev) for t in (w.q, w.k, w.v, w.offsets))
        inputs.append((q, k, v, off))
        refs.append(attn.decode(q, k, v, off, max_splits=16, scale=w.scale))  # caller-workspace entry
    torch.cuda.synchronize()
    # two calls in a row: the second reuses the array the first one left its partial triples in
    outs = [_static_decode(*x) for x in inputs]
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    for (status, o, lse), (o_ref, lse_ref) in zip(outs, refs):
        assert status == 0, attn.status_string(status)
        assert_o_bf16(np64(o), np64(o_ref))
        assert_lse(np64(lse), np64(lse_ref))


def test_static_decode_rejects_problems_beyond_its_scratch():
    # 48 streams x 64 heads x 64 splits at D = 128 need about 102 MB of partial triples > 16 MiB:
    # refused with ATTN_ERR_WORKSPACE on the host, before any launch (runs without a GPU).
    L = attn.lib()
    assert L.attn_decode_splitkv_static(A, A, A, A, None, 64, A, A, 48, 64, 8, 128, 0.1, None) == 4
    assert L.attn_decode_splitkv_static(A, A, A, A, None, 0, A, A, 48, 32, 8, 128, 0.1, None) == 1
