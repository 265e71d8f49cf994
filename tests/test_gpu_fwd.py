"""GPU forward parity: libattn.so (through its C ABI) vs the fp64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
import oracle
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_f32, assert_lse, assert_o_bf16, assert_o_fp8, np64, running_max_moves

pytestmark = pytest.mark.gpu


def run_fwd(w, f32=False):
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (w.q, w.k, w.v))
    fn = attn.fwd_f32 if f32 else attn.fwd
    o, lse = fn(q, k, v, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    return np64(o), np64(lse)


def check_fwd(w):
    o, lse = run_fwd(w)
    assert attn.last_path(0) == "fwd_sm100_tcgen05"
    o_ref, lse_ref = oracle.attention_fwd(np64(w.q), np64(w.k), np64(w.v), w.causal, w.scale)
    assert_o_bf16(o, o_ref)
    assert_lse(lse, lse_ref)


def test_tiny_causal_fp32():
    w = W.tiny_causal(torch.float32)
    o, lse = run_fwd(w, f32=True)
    assert attn.last_path(0) == "fwd_simt_f32"
    o_ref, lse_ref = oracle.attention_fwd(np64(w.q), np64(w.k), np64(w.v), True, w.scale)
    assert_f32(o, o_ref, "O")
    assert_f32(lse, lse_ref, "lse")


def test_tiny_causal_bf16():
    check_fwd(W.tiny_causal(torch.bfloat16))


@pytest.mark.parametrize("causal", [False, True])
def test_block512(causal):
    check_fwd(W.block512(causal))


@pytest.mark.parametrize("reading", ["A", "B"])
def test_gqa_prefill_4k(reading):
    check_fwd(W.gqa_prefill_4k(reading))


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal", [
    (1, 200, 200, 2, 1, 128, True),      # ragged tail, several tiles
    (2, 333, 333, 4, 2, 64, False),
    (1, 130, 517, 8, 2, 128, True),      # Sq < Sk, bottom-right causal
    (1, 300, 100, 4, 4, 64, True),       # Sq > Sk: first rows see no key
    (1, 1, 257, 8, 1, 128, False),       # one query row
    (1, 129, 1, 2, 2, 64, False),        # one key
    (3, 64, 64, 8, 8, 128, True),
    (1, 256, 384, 16, 2, 64, True),
])
def test_odd_shapes(B, Sq, Sk, Hq, Hkv, D, causal):
    check_fwd(W.random_prefill(B, Sq, Sk, Hq, Hkv, D, causal, seed=B * 1000 + Sq + Sk + D))


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 4, 128), (4, 2, 128), (8, 2, 64), (8, 1, 64)])
def test_gqa_ratios(Hq, Hkv, D):
    check_fwd(W.random_prefill(2, 257, 257, Hq, Hkv, D, True, seed=Hq * 10 + Hkv))


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal", [
    (1, 77, 77, 3, 1, 40, True), (2, 50, 90, 2, 2, 256, False), (1, 33, 20, 4, 2, 64, True)])
def test_fp32_any_head_dim(B, Sq, Sk, Hq, Hkv, D, causal):
    w = W.random_prefill(B, Sq, Sk, Hq, Hkv, D, causal, dtype=torch.float32, seed=7)
    o, lse = run_fwd(w, f32=True)
    o_ref, lse_ref = oracle.attention_fwd(np64(w.q), np64(w.k), np64(w.v), causal, w.scale)
    assert_f32(o, o_ref, "O")
    assert_f32(lse, lse_ref, "lse")


def test_constant_scores_gpu():
    # Q = 0 gives the mean of the visible V rows; exact closed form at full tile size.
    w = W.random_prefill(1, 256, 256, 2, 2, 128, True, seed=3)
    w.q.zero_()
    o, lse = run_fwd(w)
    vv = np64(w.v)[0]                       # [Sk, H, D]
    cums = np.cumsum(vv, axis=0) / np.arange(1, 257)[:, None, None]
    assert np.max(np.abs(o[0] - cums)) < 2e-2
    np.testing.assert_allclose(lse[0], np.log(np.arange(1, 257))[None, :].repeat(2, 0), atol=1e-4)


def _sample_rows(w, rng):
    S = w.q.shape[1]
    rows_per_head = []
    for h in range(w.q.shape[2]):
        g = h // (w.q.shape[2] // w.k.shape[2])
        peaks = w.meta["peaks"][g].numpy()
        pk = rng.choice(peaks, size=min(32, len(peaks)), replace=False)
        extra = np.concatenate([pk, np.minimum(pk + 1, S - 1)])
        rows = np.concatenate([np.arange(64), np.arange(S - 64, S), rng.integers(0, S, 128), extra])
        rows_per_head.append(np.unique(rows))
    return rows_per_head


def test_long_prefill_44k_sampled_rows():
    w = W.long_prefill_44k()
    o, lse = run_fwd(w)
    rng = np.random.default_rng(0)
    rows_per_head = _sample_rows(w, rng)
    qn, kn, vn = np64(w.q), np64(w.k), np64(w.v)
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for h, rows in enumerate(rows_per_head):
        ro, rl = oracle.attention_fwd_rows(qn, kn, vn, True, w.scale, 0, h, rows)
        ref_o.append(ro)
        ref_l.append(rl)
        got_o.append(o[0, rows, h])
        got_l.append(lse[0, h, rows])
    assert_o_bf16(np.concatenate(got_o), np.concatenate(ref_o), "O (sampled rows)")
    assert_lse(np.concatenate(got_l), np.concatenate(ref_l))
    # property at full size: every row is a convex combination of V rows, so |O| <= max |V|
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal", [
    (1, 640, 640, 4, 2, 128, True),      # head pairs, five key blocks
    (1, 600, 600, 3, 1, 64, True),       # row pairs (odd group size), ragged tail
    (2, 384, 700, 2, 2, 128, False),     # Sq < Sk, ragged last block
    (1, 512, 512, 8, 1, 64, False),
    (1, 300, 900, 4, 1, 128, True),      # bottom-right causal with Sq < Sk
])
def test_running_output_rescaled(B, Sq, Sk, Hq, Hkv, D, causal):
    # Keys that grow along the sequence make later key blocks raise many rows' maximum score by more
    # than 8 (base 2) over every earlier block's, which is when the kernel multiplies the running
    # output O in tensor memory by 2^(m_old - m_new): the monoid's rescale step. Counted here on
    # the oracle's scores: a large share of rows must move their maximum after the first block.
    w = W.rising_prefill(B, Sq, Sk, Hq, Hkv, D, causal, seed=Sq + Sk + D)
    x = oracle.attention_scores(np64(w.q), np64(w.k), causal, w.scale)
    moves = running_max_moves(x, 128)
    assert (moves > 0).mean() > 0.25 and (moves == 0).mean() > 0.05, (moves > 0).mean()
    check_fwd(w)


# ---------------------------------------------------------------------------------------------
# FP8 (e4m3) inputs with per-tensor scales (attn_fwd_fp8)
# ---------------------------------------------------------------------------------------------

def run_fp8(w):
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (w.q, w.k, w.v))
    o, lse = attn.fwd_fp8(q, k, v, w.q_scale, w.k_scale, w.v_scale, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    assert attn.last_path(0) == "fwd_sm100_tcgen05_fp8"
    return np64(o), np64(lse)


def check_fp8(w):
    o, lse = run_fp8(w)
    o_ref, lse_ref = oracle.attention_fwd_fp8(w.q.numpy(), w.k.numpy(), w.v.numpy(), w.q_scale, w.k_scale,
                                              w.v_scale, w.causal, w.scale)
    assert_o_fp8(o, o_ref)
    assert_lse(lse, lse_ref)


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,causal", [
    (1, 512, 512, 4, 2, True),       # head pairs
    (2, 300, 300, 8, 8, False),      # ragged tail
    (1, 1000, 1000, 3, 1, True),     # odd group size (row pairs)
    (1, 130, 517, 8, 2, True),       # Sq < Sk
    (1, 4096, 4096, 32, 8, True),    # the 4k GQA prefill's shape
])
def test_fp8_forward(B, Sq, Sk, Hq, Hkv, causal):
    check_fp8(W.fp8_prefill(B, Sq, Sk, Hq, Hkv, 128, causal, seed=Sq + Sk))


def test_fp8_forward_rescales_running_output():
    w = W.fp8_prefill(1, 640, 640, 4, 2, 128, True, seed=5, rising=True)
    x = oracle.attention_scores(w.q_scale * oracle.e4m3_to_float(w.q.numpy()),
                                w.k_scale * oracle.e4m3_to_float(w.k.numpy()), True, w.scale)
    assert (running_max_moves(x, 128) > 0).mean() > 0.25
    check_fp8(w)
