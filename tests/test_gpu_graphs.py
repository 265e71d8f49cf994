"""The library's calls inside CUDA graphs: a decode step (split + combine), a paged decode step and a
prefill forward + backward are captured once and replayed with new inputs written into the same
device buffers; every replay is checked against the fp64 oracle. The calls make no host
synchronisation and no allocation of their own when their outputs and workspace are passed in,
so a captured step replays without the host."""
import numpy as np
import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
import oracle
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_grad_bf16, assert_lse, assert_o_bf16, np64

pytestmark = pytest.mark.gpu


def capture(fn):
    """fn once outside (lazy set-up), then captured into a graph."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def test_decode_step_replays_in_a_graph():
    dev = torch.device("cuda")
    lengths = [700, 33, 1500, 1]
    w0 = W.random_decode(4, 8, 2, 128, lengths, seed=61)
    q, k, v, off = (t.to(dev) for t in (w0.q, w0.k, w0.v, w0.offsets))
    o = torch.empty_like(q)
    lse = torch.empty(4, 8, dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_size(4, 8, 128, 16), dtype=torch.uint8, device=dev)
    g = capture(lambda: attn.decode(q, k, v, off, scale=w0.scale, out=o, lse=lse, workspace=ws))
    for seed in (62, 63):
        w = W.random_decode(4, 8, 2, 128, lengths, seed=seed)
        q.copy_(w.q.to(dev))
        k.copy_(w.k.to(dev))
        v.copy_(w.v.to(dev))
        g.replay()
        torch.cuda.synchronize()
        assert attn.device_status() == 0
        o_ref, lse_ref = oracle.decode_attention(np64(w.q), np64(w.k), np64(w.v), w.offsets.numpy(), w.scale)
        assert_o_bf16(np64(o), o_ref)
        assert_lse(np64(lse), lse_ref)


def test_paged_decode_step_replays_in_a_graph():
    dev = torch.device("cuda")
    lengths = [300, 64, 1000]
    w0 = W.random_decode(3, 4, 1, 64, lengths, seed=71)
    pc0 = W.paged_from_packed(w0, 32, seed=1)
    q = w0.q.to(dev)
    kp, vp, bt, sl = (t.to(dev) for t in (pc0.k_pages, pc0.v_pages, pc0.block_table, pc0.seq_lens))
    o = torch.empty_like(q)
    lse = torch.empty(3, 4, dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_size(3, 4, 64, 16), dtype=torch.uint8, device=dev)
    g = capture(lambda: attn.decode_paged(q, kp, vp, bt, sl, scale=w0.scale, out=o, lse=lse, workspace=ws))
    for seed in (72, 73):
        w = W.random_decode(3, 4, 1, 64, lengths, seed=seed)
        pc = W.paged_from_packed(w, 32, seed=1)  # same page layout, new contents
        assert torch.equal(pc.block_table, pc0.block_table)
        q.copy_(w.q.to(dev))
        kp.copy_(pc.k_pages.to(dev))
        vp.copy_(pc.v_pages.to(dev))
        g.replay()
        torch.cuda.synchronize()
        assert attn.device_status() == 0
        o_ref, lse_ref = oracle.decode_attention(np64(w.q), np64(w.k), np64(w.v), w.offsets.numpy(), w.scale)
        assert_o_bf16(np64(o), o_ref)
        assert_lse(np64(lse), lse_ref)


def test_prefill_forward_backward_replay_in_a_graph():
    dev = torch.device("cuda")
    shape = (1, 384, 384, 4, 2, 128, True)
    w0 = W.random_prefill(*shape, seed=81)
    q, k, v, do = (t.to(dev) for t in (w0.q, w0.k, w0.v, w0.do))
    o = torch.empty_like(q)
    lse = torch.empty(1, 4, 384, dtype=torch.float32, device=dev)
    grads = tuple(torch.empty_like(t) for t in (q, k, v))
    ws = torch.empty(attn.bwd_workspace_size(1, 4, 2, 384, 384, 128), dtype=torch.uint8, device=dev)

    def step():
        attn.fwd(q, k, v, causal=True, scale=w0.scale, out=o, lse=lse)
        attn.bwd(q, k, v, o, lse, do, causal=True, scale=w0.scale, workspace=ws, out=grads)

    g = capture(step)
    for seed in (82, 83):
        w = W.random_prefill(*shape, seed=seed)
        for dst, src in zip((q, k, v, do), (w.q, w.k, w.v, w.do)):
            dst.copy_(src.to(dev))
        g.replay()
        torch.cuda.synchronize()
        assert attn.device_status() == 0
        o_ref, lse_ref = oracle.attention_fwd(np64(w.q), np64(w.k), np64(w.v), True, w.scale)
        assert_o_bf16(np64(o), o_ref)
        assert_lse(np64(lse), lse_ref)
        refs = oracle.attention_bwd(np64(w.q), np64(w.k), np64(w.v), np64(w.do), True, w.scale)
        for name, gr, r in zip(("dQ", "dK", "dV"), grads, refs):
            assert_grad_bf16(np64(gr), r, name)
