"""Context-parallel ring forward: its schedule on CPU ranks (gloo), and its kernels on one GPU.

The ring spreads one sequence over W ranks (zigzag shards) and merges the partial attentions of
each key/value shard with the online-softmax monoid ("Não escreva kernels, derive-os",
"Aprofundamento", first paragraph). On CPU the per-step attention and merge are the oracle's
(two-pass attention, and the monoid's merge on (lse, 1, O) triples), so these tests check the
schedule, the shard exchange and the bookkeeping against the full-sequence oracle; the GPU test
runs the library's kernels through the same schedule on one device.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from online_softmax_attention_fwd_b200 import ring


def oracle_attend(q, k, v, causal, scale):
    o, lse = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, scale)
    return torch.from_numpy(o), torch.from_numpy(lse)


def oracle_fold(o_acc, lse_acc, o_part, lse_part, o_out):
    # (O, lse) is the triple (m = lse, l = 1, o = O); merge with the oracle's monoid, finalise
    B, S, H, D = o_acc.shape
    for b in range(B):
        for i in range(S):
            for h in range(H):
                t = oracle.monoid_merge((float(lse_acc[b, h, i]), 1.0, o_acc[b, i, h].numpy()),
                                        (float(lse_part[b, h, i]), 1.0, o_part[b, i, h].numpy()))
                o, lse = oracle.monoid_finalize(t)
                o_acc[b, i, h] = torch.from_numpy(np.asarray(o))
                lse_acc[b, h, i] = lse
    if o_out is not None:
        o_out.copy_(o_acc)


def _inputs(B, S, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, S, Hq, D, generator=g, dtype=torch.float64),
            torch.randn(B, S, Hkv, D, generator=g, dtype=torch.float64),
            torch.randn(B, S, Hkv, D, generator=g, dtype=torch.float64))


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_schedule_covers_every_visible_pair_once(world):
    # over all ranks and steps, each (query chunk, key chunk) pair with key <= query appears exactly
    # once (causal on the diagonal), and every rank attends the same number of chunk pairs
    seen = {}
    work = []
    for r in range(world):
        qc = ring.zigzag_chunks(r, world)
        n = 0
        for s, (src, pairs) in enumerate(ring.ring_schedule(r, world, True)):
            assert src == (r - s) % world
            kc = ring.zigzag_chunks(src, world)
            for qi, ki, causal in pairs:
                key = (qc[qi], kc[ki])
                assert key not in seen
                seen[key] = causal
                assert causal == (kc[ki] == qc[qi])
                n += 1 if not causal else 0.5
        work.append(n)
    C = 2 * world
    assert set(seen) == {(a, b) for a in range(C) for b in range(a + 1)}
    assert len(set(work)) == 1


def test_zigzag_shards_round_trip():
    x = torch.arange(2 * 3 * 12 * 5, dtype=torch.float64).reshape(2, 12, 3, 5)
    shards = [ring.zigzag_shard(x, r, 3) for r in range(3)]
    assert torch.equal(ring.zigzag_unshard(shards), x)


@pytest.mark.parametrize("world,causal,Hq,Hkv", [(2, True, 4, 2), (3, True, 2, 1), (2, False, 2, 2)])
def test_local_ring_equals_full_attention_oracle(world, causal, Hq, Hkv):
    q, k, v = _inputs(1, 4 * world, Hq, Hkv, 3, seed=world)
    o, lse = ring.ring_attention_fwd_local(q, k, v, world, causal, 0.6, attend=oracle_attend, fold=oracle_fold)
    o_ref, lse_ref = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, 0.6)
    np.testing.assert_allclose(o.numpy(), o_ref, atol=1e-12)
    np.testing.assert_allclose(lse.numpy(), lse_ref, atol=1e-12)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _ring_worker(rank, world, port, causal, q_out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _inputs(2, 4 * world, 4, 2, 3, seed=7)
        o, lse = ring.ring_attention_fwd(ring.zigzag_shard(q, rank, world), ring.zigzag_shard(k, rank, world),
                                         ring.zigzag_shard(v, rank, world), causal, 0.45,
                                         attend=oracle_attend, fold=oracle_fold)
        q_out.put((rank, o.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (2, False)])
def test_ring_over_gloo_ranks_equals_full_attention_oracle(world, causal):
    ctx = mp.get_context("spawn")
    qo = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ring_worker, args=(r, world, port, causal, qo)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qo.get(timeout=240) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v = _inputs(2, 4 * world, 4, 2, 3, seed=7)
    o_ref, lse_ref = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, 0.45)
    o = ring.zigzag_unshard([torch.from_numpy(r[1]) for r in res], dim=1).numpy()
    lse = ring.zigzag_unshard([torch.from_numpy(r[2]) for r in res], dim=2).numpy()
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# On the GPU: the library's forward and merge kernels through the same schedule.
# ---------------------------------------------------------------------------------------------

@pytest.mark.gpu
def test_merge_kernel_joins_two_key_halves():
    import online_softmax_attention_fwd_b200 as attn
    from online_softmax_attention_fwd_b200 import workloads as W
    from tests._util import assert_lse, assert_o_bf16, np64
    w = W.random_prefill(2, 300, 700, 8, 2, 128, False, seed=41)
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (w.q, w.k, w.v))
    o1, l1 = attn.fwd(q, k[:, :256].contiguous(), v[:, :256].contiguous(), scale=w.scale)
    o2, l2 = attn.fwd(q, k[:, 256:].contiguous(), v[:, 256:].contiguous(), scale=w.scale)
    o_acc = torch.empty(q.shape, dtype=torch.float32, device=dev)
    l_acc = torch.full(l1.shape, float("-inf"), dtype=torch.float32, device=dev)
    o_out = torch.empty_like(q)
    attn.merge(o_acc, l_acc, o1, l1)
    attn.merge(o_acc, l_acc, o2, l2, o_out)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    o_ref, lse_ref = oracle.attention_fwd(np64(w.q), np64(w.k), np64(w.v), False, w.scale)
    assert_o_bf16(np64(o_out), o_ref)
    assert_o_bf16(np64(o_acc), o_ref)
    assert_lse(np64(l_acc), lse_ref)
    # the identity: a partial whose lse is -inf everywhere leaves the running result unchanged
    before_o, before_l = o_acc.clone(), l_acc.clone()
    attn.merge(o_acc, l_acc, torch.full_like(o1, float("nan")), torch.full_like(l1, float("-inf")))
    torch.cuda.synchronize()
    assert torch.equal(o_acc, before_o) and torch.equal(l_acc, before_l)


@pytest.mark.gpu
@pytest.mark.parametrize("world,S,Hq,Hkv,D,causal", [
    (2, 1024, 8, 2, 128, True), (4, 2048, 4, 4, 64, True), (3, 768, 4, 1, 128, False)])
def test_ring_on_one_gpu_equals_full_attention(world, S, Hq, Hkv, D, causal):
    import online_softmax_attention_fwd_b200 as attn
    from online_softmax_attention_fwd_b200 import workloads as W
    from tests._util import assert_lse, assert_o_bf16, np64
    w = W.random_prefill(1, S, S, Hq, Hkv, D, causal, seed=S + world)
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (w.q, w.k, w.v))
    o, lse = ring.ring_attention_fwd_local(q, k, v, world, causal, w.scale)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    o_ref, lse_ref = oracle.attention_fwd(np64(w.q), np64(w.k), np64(w.v), causal, w.scale)
    assert_o_bf16(np64(o), o_ref)
    assert_lse(np64(lse), lse_ref)
