"""GPU parity of the packed variable-length prefill (attn_fwd_varlen / attn_bwd_varlen) against the
fp64 oracle: each sequence attends only to its own keys."""
import numpy as np
import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
import oracle
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_grad_bf16, assert_grad_tiles, assert_lse, assert_o_bf16, np64

pytestmark = pytest.mark.gpu


def run(w, backward=True, max_q=None, max_k=None):
    dev = torch.device("cuda")
    q, k, v, do, cq, ck = (t.to(dev) for t in (w.q, w.k, w.v, w.do, w.cu_q, w.cu_k))
    mq = int(w.meta["lengths_q"].max()) if max_q is None else max_q
    mk = int(w.meta["lengths_k"].max()) if max_k is None else max_k
    o, lse = attn.fwd_varlen(q, k, v, cq, ck, mq, mk, causal=w.causal, scale=w.scale)
    grads = None
    if backward:
        grads = attn.bwd_varlen(q, k, v, o, lse, do, cq, ck, mq, mk, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    return o, lse, grads


def check(w, backward=True):
    o, lse, grads = run(w, backward)
    assert attn.device_status() == 0
    assert attn.last_path(0) == "fwd_sm100_tcgen05_varlen"
    args = (np64(w.q), np64(w.k), np64(w.v))
    o_ref, lse_ref = oracle.attention_fwd_varlen(*args, w.cu_q.numpy(), w.cu_k.numpy(), w.causal, w.scale)
    assert_o_bf16(np64(o), o_ref)
    assert_lse(np64(lse), lse_ref)
    if backward:
        assert attn.last_path(1) == "bwd_sm100_tcgen05_varlen"
        refs = oracle.attention_bwd_varlen(*args, np64(w.do), w.cu_q.numpy(), w.cu_k.numpy(), w.causal, w.scale)
        for name, g, r in zip(("dQ", "dK", "dV"), grads, refs):
            assert_grad_bf16(np64(g), r, name)
            assert_grad_tiles(np64(g)[None], r[None], name)


@pytest.mark.parametrize("lq,lk,Hq,Hkv,D,causal", [
    ([300, 1, 129, 700], [300, 1, 129, 700], 4, 2, 128, True),    # ragged, a one-token prompt
    ([200, 333, 64], [200, 333, 64], 3, 1, 64, True),              # odd group size (row pairs)
    ([100, 250, 0, 400], [500, 250, 7, 400], 8, 2, 128, True),     # Sq < Sk (chunked prefill), an empty one
    ([256, 128, 90], [256, 300, 90], 2, 2, 64, False),
    ([50, 80], [0, 80], 4, 4, 128, True),                          # a sequence with no key: O = 0, lse = -inf
])
def test_varlen_matches_oracle(lq, lk, Hq, Hkv, D, causal):
    check(W.packed_prefill(lq, lk, Hq, Hkv, D, causal, seed=sum(lq) + sum(lk) + D))


@pytest.mark.parametrize("lq,Hq,Hkv,D", [
    ([700, 5, 300, 0, 256, 255, 129, 1, 640], 3, 1, 64),     # single-head items, ranks of many sizes
    ([1000, 3, 0, 517, 129, 128, 127, 1], 8, 2, 128),        # head pairs
])
def test_varlen_item_list_skips_missing_ranks(lq, Hq, Hkv, D):
    # the forward deals only the (sequence, rank) items that exist, longest first: every sequence's
    # rows still come out, whatever the spread of lengths
    check(W.packed_prefill(lq, lq, Hq, Hkv, D, True, seed=sum(lq) + Hq))


def test_varlen_more_sequences_than_the_item_tables():
    # 1100 short sequences (more than the forward's shared-memory item tables hold): every
    # (sequence, rank) pair stays an item and the empty ones are skipped
    rng = np.random.default_rng(11)
    lq = [int(x) for x in rng.integers(0, 7, 1100)]
    check(W.packed_prefill(lq, lq, 2, 1, 64, True, seed=11))


def test_varlen_equal_lengths_equal_dense_call():
    # the same batch packed and dense gives bit-identical forward results and gradients
    wd = W.random_prefill(3, 384, 384, 8, 2, 128, True, seed=5)
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (wd.q, wd.k, wd.v, wd.do))
    o, lse = attn.fwd(q, k, v, causal=True, scale=wd.scale)
    g = attn.bwd(q, k, v, o, lse, do, causal=True, scale=wd.scale)
    cu = torch.arange(4, dtype=torch.int32, device=dev) * 384
    flat = lambda t: t.reshape(-1, t.shape[2], t.shape[3])
    ov, lv = attn.fwd_varlen(flat(q), flat(k), flat(v), cu, cu, 384, 384, causal=True, scale=wd.scale)
    gv = attn.bwd_varlen(flat(q), flat(k), flat(v), ov, lv, flat(do), cu, cu, 384, 384, causal=True,
                         scale=wd.scale)
    torch.cuda.synchronize()
    assert torch.equal(flat(o), ov)
    assert torch.equal(lse.permute(1, 0, 2).reshape(8, -1), lv)
    # dK and dV are reduced in tensor memory in a fixed order; dQ by floating-point atomics, whose
    # order (and so the last bit) may differ between two runs
    assert torch.equal(flat(g[1]), gv[1]) and torch.equal(flat(g[2]), gv[2])
    a, b = np64(flat(g[0])), np64(gv[0])
    assert np.linalg.norm(a - b) <= 1e-3 * np.linalg.norm(a)


def test_varlen_prefill_8x():
    w = W.varlen_prefill_8x()
    o, lse, grads = run(w)
    assert attn.device_status() == 0
    # sampled rows of every sequence against the oracle's per-sequence forward
    rng = np.random.default_rng(0)
    cq = w.cu_q.numpy()
    qn, kn, vn = np64(w.q), np64(w.k), np64(w.v)
    for b in range(len(cq) - 1):
        L = cq[b + 1] - cq[b]
        rows = np.unique(np.concatenate([np.arange(4), np.arange(L - 4, L), rng.integers(0, L, 24)]))
        for h in (0, 13, 31):
            ro, rl = oracle.attention_fwd_rows(qn[None, cq[b]:cq[b + 1]], kn[None, cq[b]:cq[b + 1]],
                                               vn[None, cq[b]:cq[b + 1]], True, w.scale, 0, h, rows)
            assert_o_bf16(np64(o)[cq[b] + rows, h], ro)
            assert_lse(np64(lse)[h, cq[b] + rows], rl)
    # gradient invariants per sequence: sum_j dK_j = 0 and sum_j dV_j = sum over the group's rows of dO
    dq, dk, dv = (np64(t) for t in grads)
    do = np64(w.do)
    for b in range(len(cq) - 1):
        s = slice(cq[b], cq[b + 1])
        want = do[s].reshape(-1, 8, 4, 128).sum(axis=(0, 2))
        assert np.max(np.abs(dv[s].sum(axis=0) - want)) <= 2e-2 * np.abs(want).max() + 0.5
        assert np.max(np.abs(dk[s].sum(axis=0))) <= 2e-2 * np.abs(dk[s]).sum(axis=0).max()


def test_varlen_bad_offsets_are_reported_not_followed():
    # offsets past the packed rows: that sequence is skipped and the status says invalid argument;
    # the other sequences are right
    w = W.packed_prefill([100, 60, 80], [100, 60, 80], 4, 2, 128, True, seed=3)
    dev = torch.device("cuda")
    bad_q = w.cu_q.clone()
    bad_k = w.cu_k.clone()
    bad_q[2] = 10_000_000
    bad_k[2] = 10_000_000
    q, k, v, cq, ck = (t.to(dev) for t in (w.q, w.k, w.v, bad_q, bad_k))
    o = torch.zeros_like(q)
    lse = torch.zeros(4, q.shape[0], dtype=torch.float32, device=dev)
    attn.fwd_varlen(q, k, v, cq, ck, 100, 100, causal=True, scale=w.scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert attn.device_status() == 1
    assert attn.device_status() == 0
    o_ref, lse_ref = oracle.attention_fwd_varlen(np64(w.q), np64(w.k), np64(w.v), w.cu_q.numpy(), w.cu_k.numpy(),
                                                 True, w.scale)
    assert_o_bf16(np64(o)[:100], o_ref[:100])
    assert_lse(np64(lse)[:, :100], lse_ref[:, :100])
