"""GPU backward parity: libattn.so (through its C ABI) vs the fp64 oracle's closed-form backward."""
import numpy as np
import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
import oracle
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_f32, assert_grad_bf16, assert_grad_tiles, np64

pytestmark = pytest.mark.gpu


def run_fwd_bwd(w, f32=False):
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (w.q, w.k, w.v, w.do))
    if f32:
        o, lse = attn.fwd_f32(q, k, v, causal=w.causal, scale=w.scale)
        dq, dk, dv = attn.bwd_f32(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)
    else:
        o, lse = attn.fwd(q, k, v, causal=w.causal, scale=w.scale)
        dq, dk, dv = attn.bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    return np64(dq), np64(dk), np64(dv)


def refs(w):
    return oracle.attention_bwd(np64(w.q), np64(w.k), np64(w.v), np64(w.do), w.causal, w.scale)


def check_bwd(w):
    dq, dk, dv = run_fwd_bwd(w)
    rq, rk, rv = refs(w)
    assert_grad_bf16(dq, rq, "dQ")
    assert_grad_bf16(dk, rk, "dK")
    assert_grad_bf16(dv, rv, "dV")
    assert_grad_tiles(dq, rq, "dQ")
    assert_grad_tiles(dk, rk, "dK")
    assert_grad_tiles(dv, rv, "dV")


def test_tiny_causal_fp32():
    w = W.tiny_causal(torch.float32)
    dq, dk, dv = run_fwd_bwd(w, f32=True)
    rq, rk, rv = refs(w)
    assert_f32(dq, rq, "dQ")
    assert_f32(dk, rk, "dK")
    assert_f32(dv, rv, "dV")


def test_tiny_causal_bf16():
    check_bwd(W.tiny_causal(torch.bfloat16))


@pytest.mark.parametrize("causal", [False, True])
def test_block512(causal):
    check_bwd(W.block512(causal))


@pytest.mark.parametrize("reading", ["A", "B"])
def test_gqa_prefill_4k(reading):
    check_bwd(W.gqa_prefill_4k(reading))


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal", [
    (1, 200, 200, 2, 1, 128, True), (2, 333, 333, 4, 2, 64, False), (1, 130, 517, 8, 2, 128, True),
    (1, 300, 100, 4, 4, 64, True), (1, 1, 257, 8, 1, 128, False), (3, 64, 64, 8, 8, 128, True)])
def test_odd_shapes(B, Sq, Sk, Hq, Hkv, D, causal):
    check_bwd(W.random_prefill(B, Sq, Sk, Hq, Hkv, D, causal, seed=B * 1000 + Sq + Sk + D))


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal", [
    (3, 2048, 2048, 16, 4, 128, True), (5, 2048, 2048, 16, 16, 64, False)])
def test_large_batches_run_sequence_by_sequence(B, Sq, Sk, Hq, Hkv, D, causal):
    # batches whose Q, dO and dQ accumulator rows exceed half of L2 take the sequence-by-sequence
    # CTA order (a second instantiation of the backward kernel)
    assert B * Hq * D * (4 * Sq + 4 * ((Sq + 127) // 128 * 128)) > 64 * 1024 * 1024
    check_bwd(W.random_prefill(B, Sq, Sk, Hq, Hkv, D, causal, seed=B + Sq + D))


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal", [
    (1, 77, 77, 3, 1, 40, True), (2, 50, 90, 2, 2, 256, False), (1, 33, 20, 4, 2, 64, True)])
def test_fp32_any_head_dim(B, Sq, Sk, Hq, Hkv, D, causal):
    w = W.random_prefill(B, Sq, Sk, Hq, Hkv, D, causal, dtype=torch.float32, seed=9)
    dq, dk, dv = run_fwd_bwd(w, f32=True)
    rq, rk, rv = refs(w)
    assert_f32(dq, rq, "dQ")
    assert_f32(dk, rk, "dK")
    assert_f32(dv, rv, "dV")


def test_gradient_invariants_full_size():
    # sum_j dK_j = 0 and sum_j dV_j = sum over the group's rows of dO, at the 4k GQA size
    w = W.gqa_prefill_4k("A")
    dq, dk, dv = run_fwd_bwd(w)
    do = np64(w.do)
    G = w.q.shape[2] // w.k.shape[2]
    want_dv = do.reshape(1, 4096, 8, G, 128).sum(axis=(1, 3))
    scale_dv = np.abs(want_dv).max()
    assert np.max(np.abs(dv.sum(axis=1) - want_dv)) <= 2e-2 * scale_dv + 0.5
    assert np.max(np.abs(dk.sum(axis=1))) <= 2e-2 * np.abs(dk).sum(axis=1).max()


# dQ bound for the rising-key inputs. Their keys share a large component (a ramp up to ~120 in one
# dimension), and dQ_i = scale sum_j dS_ij K_j sums to a small vector out of large terms (the dS_ij
# of a row sum to 0), so the bf16 rounding of dS (and of P and O before it) is amplified there.
# An fp64 evaluation of the backward with exactly those roundings (P, O and dS rounded to bf16, all
# else exact) gives dQ rel-L2 1.4e-2, 2.0e-2 and 2.8e-2 on the three cases below, and up to 3.6e-2
# per 64-row tile; dK and dV stay near 2.5e-3. Bound: twice the worst of those.
RISING_DQ_REL_L2 = 7e-2


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal", [
    (1, 640, 640, 4, 2, 128, True), (1, 600, 600, 3, 1, 64, True), (2, 384, 700, 2, 2, 128, False)])
def test_rising_keys(B, Sq, Sk, Hq, Hkv, D, causal):
    # peaky rows (most of the mass on the newest keys) through the whole forward + backward
    from tests._util import rel_l2, tile_rel_l2
    w = W.rising_prefill(B, Sq, Sk, Hq, Hkv, D, causal, seed=Sq + Sk + D)
    dq, dk, dv = run_fwd_bwd(w)
    rq, rk, rv = refs(w)
    assert_grad_bf16(dk, rk, "dK")
    assert_grad_bf16(dv, rv, "dV")
    assert_grad_tiles(dk, rk, "dK")
    assert_grad_tiles(dv, rv, "dV")
    assert rel_l2(dq, rq) <= RISING_DQ_REL_L2 and tile_rel_l2(dq, rq).max() <= RISING_DQ_REL_L2
