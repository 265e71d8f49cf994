"""Seeded random shapes through every bf16 entry point, each checked against the fp64 oracle: prefill
forward and backward (dense and packed), split-KV decode with one or several query tokens (packed
and paged caches, default and explicit split counts). The shapes are drawn once from a fixed
seed, so a failure names a reproducible case; sizes stay small enough for the oracle."""
import numpy as np
import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
import oracle
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_grad_bf16, assert_lse, assert_o_bf16, np64

pytestmark = pytest.mark.gpu

_rng = np.random.default_rng(20261203)


def _group():
    Hkv = int(_rng.choice([1, 2, 4]))
    G = int(_rng.choice([1, 2, 3, 4, 8]))
    return Hkv * G, Hkv


PREFILL = []
for _ in range(14):
    Hq, Hkv = _group()
    PREFILL.append((int(_rng.integers(1, 4)), int(_rng.integers(1, 700)), int(_rng.integers(1, 700)), Hq, Hkv,
                    int(_rng.choice([64, 128])), bool(_rng.integers(0, 2)), int(_rng.integers(1 << 30))))

DECODE = []
for _ in range(12):
    Hq, Hkv = _group()
    N = int(_rng.integers(1, 40))
    q_len = int(_rng.choice([1, 1, 2, 3, 5]))
    lengths = [int(x) for x in _rng.integers(q_len, 3000, N)]
    DECODE.append((N, Hq, Hkv, int(_rng.choice([64, 128])), q_len, lengths, bool(_rng.integers(0, 2)),
                   int(_rng.choice([16, 32, 64])), int(_rng.integers(1 << 30))))

PACKED = []
for _ in range(6):
    Hq, Hkv = _group()
    nseq = int(_rng.integers(1, 9))
    lq = [int(x) for x in _rng.integers(0, 900, nseq)]
    lq[0] = max(lq[0], 1)  # at least one token in the batch
    PACKED.append((lq, Hq, Hkv, int(_rng.choice([64, 128])), bool(_rng.integers(0, 2)), int(_rng.integers(1 << 30))))


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal,seed", PREFILL)
def test_prefill_random_shapes(B, Sq, Sk, Hq, Hkv, D, causal, seed):
    w = W.random_prefill(B, Sq, Sk, Hq, Hkv, D, causal, seed=seed)
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (w.q, w.k, w.v, w.do))
    o, lse = attn.fwd(q, k, v, causal=causal, scale=w.scale)
    grads = attn.bwd(q, k, v, o, lse, do, causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    args = (np64(w.q), np64(w.k), np64(w.v))
    o_ref, lse_ref = oracle.attention_fwd(*args, causal, w.scale)
    assert_o_bf16(np64(o), o_ref)
    assert_lse(np64(lse), lse_ref)
    refs = oracle.attention_bwd(*args, np64(w.do), causal, w.scale)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, refs):
        assert_grad_bf16(np64(g), r, name)


@pytest.mark.parametrize("N,Hq,Hkv,D,q_len,lengths,explicit,page,seed", DECODE)
def test_decode_random_shapes(N, Hq, Hkv, D, q_len, lengths, explicit, page, seed):
    w = W.random_decode(N, Hq, Hkv, D, lengths, seed=seed, q_len=None if q_len == 1 else q_len)
    dev = torch.device("cuda")
    q, k, v, off = (t.to(dev) for t in (w.q, w.k, w.v, w.offsets))
    splits = None
    if explicit:
        splits = torch.tensor([int(x) for x in np.random.default_rng(seed).integers(1, 17, N)], dtype=torch.int32,
                              device=dev)
    o, lse = attn.decode(q, k, v, off, num_splits=splits, scale=w.scale)
    pc = W.paged_from_packed(w, page, seed=seed % 1000)
    kp, vp, bt, sl = (t.to(dev) for t in (pc.k_pages, pc.v_pages, pc.block_table, pc.seq_lens))
    op, lsep = attn.decode_paged(q, kp, vp, bt, sl, num_splits=splits, scale=w.scale)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    if q_len == 1:
        o_ref, lse_ref = oracle.decode_attention(np64(w.q), np64(w.k), np64(w.v), w.offsets.numpy(), w.scale)
    else:
        o_ref, lse_ref = oracle.decode_attention_qlen(np64(w.q), np64(w.k), np64(w.v), w.offsets.numpy(), w.scale)
    for oo, ll in ((o, lse), (op, lsep)):
        assert_o_bf16(np64(oo), o_ref)
        assert_lse(np64(ll), lse_ref)


@pytest.mark.parametrize("lq,Hq,Hkv,D,causal,seed", PACKED)
def test_packed_random_lengths(lq, Hq, Hkv, D, causal, seed):
    w = W.packed_prefill(lq, lq, Hq, Hkv, D, causal, seed=seed)
    dev = torch.device("cuda")
    q, k, v, do, cq, ck = (t.to(dev) for t in (w.q, w.k, w.v, w.do, w.cu_q, w.cu_k))
    m = max(1, max(lq))
    o, lse = attn.fwd_varlen(q, k, v, cq, ck, m, m, causal=causal, scale=w.scale)
    grads = attn.bwd_varlen(q, k, v, o, lse, do, cq, ck, m, m, causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    args = (np64(w.q), np64(w.k), np64(w.v))
    o_ref, lse_ref = oracle.attention_fwd_varlen(*args, w.cu_q.numpy(), w.cu_k.numpy(), causal, w.scale)
    assert_o_bf16(np64(o), o_ref)
    assert_lse(np64(lse), lse_ref)
    refs = oracle.attention_bwd_varlen(*args, np64(w.do), w.cu_q.numpy(), w.cu_k.numpy(), causal, w.scale)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, refs):
        assert_grad_bf16(np64(g), r, name)
