"""The split-KV decode entry point that allocates nothing: attn_decode_splitkv_static.

It exists for callers of this library that cannot give it device scratch memory -- a host framework
that owns all device memory through its own pool and hands plugins no workspace, or a latency-bound
serving loop that may not call cudaMalloc on its hot path. Its partial (m, l, o) triples live in a
fixed 16 MiB array inside the library instead of a caller workspace, so its results must match the
fp64 oracle and those of attn_decode_splitkv, and they must stay right when the array is reused by
the next call.

This file is collected last on purpose, so that a run stopping at the first failure has already
run every other test; it passes both alone and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
import oracle
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_lse, assert_o_bf16, np64

A = ctypes.c_void_p(0x100000)  # aligned stand-in address; never dereferenced by the host checks


def _static_decode(q, k, v, offsets, num_splits=None, max_splits=16, scale=None):
    N, Hq, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((N, Hq), dtype=torch.float32, device=q.device)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    scale = 1.0 / D ** 0.5 if scale is None else scale
    status = attn.lib().attn_decode_splitkv_static(
        p(q), p(k), p(v), p(offsets), p(num_splits), max_splits, p(o), p(lse), N, Hq, k.shape[1], D,
        scale, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return status, o, lse


def _sparse_batch():
    # 300 streams: above the 256-stream limit of the dense item numbering, so the split kernel walks
    # the sparse slot space and skips slots past each stream's split count -- the path most likely
    # to leave a stale triple of the previous call behind if a slot were read but not written.
    g = np.random.default_rng(5)
    lengths = g.integers(0, 300, 300)
    lengths[::37] = 0
    w = W.random_decode(300, 8, 2, 64, lengths.tolist(), seed=21)
    splits = torch.as_tensor(g.integers(1, 17, 300), dtype=torch.int32)
    return w, splits


@pytest.mark.gpu
def test_static_decode_matches_oracle_and_workspace_decode_on_calls_in_a_row():
    dev = torch.device("cuda")
    sparse, sparse_splits = _sparse_batch()
    batches = [(W.decode48(), None),
               (W.random_decode(7, 32, 8, 128, [1, 4096, 0, 777, 2048, 3000, 5], seed=3), None),
               (sparse, sparse_splits)]
    inputs, oracle_refs, ws_refs = [], [], []
    for w, ns in batches:
        q, k, v, off = (t.to(dev) for t in (w.q, w.k, w.v, w.offsets))
        nsd = None if ns is None else ns.to(dev)
        inputs.append((q, k, v, off, nsd, w.scale))
        oracle_refs.append(oracle.decode_attention(np64(w.q), np64(w.k), np64(w.v), w.offsets.numpy(), w.scale))
        ws_refs.append(attn.decode(q, k, v, off, num_splits=nsd, max_splits=16, scale=w.scale))
    torch.cuda.synchronize()
    # calls in a row: each reuses the array the previous one left its partial triples in (the
    # largest first, then a smaller one, then the sparse slot walk)
    outs = [_static_decode(q, k, v, off, num_splits=ns, scale=sc) for q, k, v, off, ns, sc in inputs]
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    assert attn.last_path(2) == "decode_splitkv_static_mma16816"
    for (status, o, lse), (o_ref, lse_ref), (o_ws, lse_ws) in zip(outs, oracle_refs, ws_refs):
        assert status == 0, attn.status_string(status)
        assert_o_bf16(np64(o), o_ref)
        assert_lse(np64(lse), lse_ref)
        assert_o_bf16(np64(o), np64(o_ws), "O vs the workspace entry point")


def test_static_decode_rejects_problems_beyond_its_scratch():
    # 48 streams x 64 heads x 64 splits at D = 128 need about 102 MB of partial triples > 16 MiB:
    # refused with ATTN_ERR_WORKSPACE on the host, before any launch (runs without a GPU).
    L = attn.lib()
    assert L.attn_decode_splitkv_static(A, A, A, A, None, 64, A, A, 48, 64, 8, 128, 0.1, None) == 4
    assert L.attn_decode_splitkv_static(A, A, A, A, None, 0, A, A, 48, 32, 8, 128, 0.1, None) == 1
    # the same argument checks as attn_decode_splitkv: a misaligned pointer is refused
    bad = ctypes.c_void_p(0x100008)
    assert L.attn_decode_splitkv_static(A, A, A, A, None, 16, bad, A, 4, 8, 2, 128, 0.1, None) == 3
