"""Pins for the fp64 oracle, against things other than the oracle itself (CPU only).

Each pin is written as a check that takes the implementation under test as an argument, so that
``test_oracle_mutations.py`` can plant plausible mistakes in the oracle and show a pin fails.
Sources: the attention definition and the online-softmax monoid named in "Não escreva kernels,
derive-os" ("Aprofundamento", first paragraph), the backward of its "Perguntas frequentes", and the
causal forward passes of the aibriefing page ("Details"). Values below are hand-worked closed forms,
library routines (torch's fp64 scaled_dot_product_attention, scipy's logsumexp/softmax), invariants
and finite differences.
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp, softmax

import oracle

RNG = np.random.default_rng(1234)


def _rand(*shape, rng=None):
    return (rng or RNG).standard_normal(shape)


# ---------------------------------------------------------------------------------------------
# Reusable pins: each takes a forward `fwd(q,k,v,causal,scale) -> (o, lse)` or a backward
# `bwd(q,k,v,do,causal,scale) -> (dq,dk,dv)` and raises AssertionError when it is wrong.
# ---------------------------------------------------------------------------------------------

def pin_two_by_two_fwd(fwd):
    # Q = K = I2, V = [[1,2],[3,4]], scale 1. Row 0 scores (1, 0) -> P = (a, b), a = sigma(1).
    a = 1.0 / (1.0 + math.exp(-1.0))
    b = 1.0 - a
    q = np.eye(2).reshape(1, 2, 1, 2)
    k = np.eye(2).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 2, 1, 2)
    o, lse = fwd(q, k, v, False, 1.0)
    want = np.array([[a + 3 * b, 2 * a + 4 * b], [b + 3 * a, 2 * b + 4 * a]])
    np.testing.assert_allclose(o[0, :, 0, :], want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], [math.log(1 + math.e)] * 2, rtol=0, atol=1e-12)
    # printed to ten places in the hand derivation: 1.5378828428 / 2.4621171572 / 1.3132616875
    assert abs(o[0, 0, 0, 0] - 1.5378828428) < 1e-9 and abs(o[0, 1, 0, 0] - 2.4621171572) < 1e-9
    o, lse = fwd(q, k, v, True, 1.0)
    np.testing.assert_allclose(o[0, 0, 0, :], [1.0, 2.0], atol=1e-12)
    assert abs(lse[0, 0, 0] - 1.0) < 1e-12
    np.testing.assert_allclose(o[0, 1, 0, :], want[1], atol=1e-12)


def pin_two_by_two_bwd(bwd):
    a = 1.0 / (1.0 + math.exp(-1.0))
    b = 1.0 - a
    t = 2 * a * b                       # = 2e / (1+e)^2
    assert abs(t - 0.3932238665) < 1e-9
    q = np.eye(2).reshape(1, 2, 1, 2)
    k = np.eye(2).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 2, 1, 2)
    do = np.array([[1.0, 0.0], [0.0, 0.0]]).reshape(1, 2, 1, 2)
    dq, dk, dv = bwd(q, k, v, do, False, 1.0)
    np.testing.assert_allclose(dq[0, :, 0, :], [[-t, t], [0, 0]], atol=1e-12)
    np.testing.assert_allclose(dk[0, :, 0, :], [[-t, 0], [t, 0]], atol=1e-12)
    np.testing.assert_allclose(dv[0, :, 0, :], [[a, 0], [b, 0]], atol=1e-12)


def pin_single_key(fwd):
    # One query over one key returns that key's value, and lse is the scaled score itself.
    q, k, v = _rand(2, 1, 3, 5), _rand(2, 1, 3, 5), _rand(2, 1, 3, 5)
    s = 0.37
    o, lse = fwd(q, k, v, False, s)
    np.testing.assert_allclose(o, v, atol=1e-12)
    np.testing.assert_allclose(lse, s * np.einsum("bshd,bshd->bhs", q, k), atol=1e-12)


def pin_constant_scores(fwd, Sq, Sk, causal):
    # Q = 0 makes every visible score 0: O is the plain mean of the visible V rows and
    # lse = ln(#visible). Causal is bottom-right aligned: row i sees keys 0 .. i + Sk - Sq.
    B, H, D = 2, 3, 4
    q = np.zeros((B, Sq, H, D))
    k, v = _rand(B, Sk, H, D), _rand(B, Sk, H, D)
    o, lse = fwd(q, k, v, causal, 0.9)
    for i in range(Sq):
        n = (min(Sk, i + Sk - Sq + 1) if causal else Sk)
        if n <= 0:
            np.testing.assert_array_equal(o[:, i], 0.0)
            assert np.all(np.isneginf(lse[:, :, i]))
            continue
        np.testing.assert_allclose(o[:, i], v[:, :n].mean(axis=1), atol=1e-12)
        np.testing.assert_allclose(lse[:, :, i], math.log(n), atol=1e-12)


def pin_tiny_scale(fwd):
    # scale -> 0 gives the mean of V whatever Q and K are.
    q, k, v = _rand(1, 5, 2, 4), _rand(1, 7, 2, 4), _rand(1, 7, 2, 4)
    o, _ = fwd(q, k, v, False, 1e-13)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape), atol=1e-11)


def pin_kv_permutation(fwd):
    # Non-causal output does not depend on the order of the (key, value) pairs.
    q, k, v = _rand(2, 6, 4, 8), _rand(2, 9, 2, 8), _rand(2, 9, 2, 8)
    o1, l1 = fwd(q, k, v, False, 0.5)
    perm = RNG.permutation(9)
    o2, l2 = fwd(q, k[:, perm], v[:, perm], False, 0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def _torch_sdpa(q, k, v, causal, scale):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=causal, scale=scale,
                                       enable_gqa=q.shape[2] != k.shape[2])
    return o.permute(0, 2, 1, 3).numpy()


def pin_library_sdpa(fwd, B, S, Sk, Hq, Hkv, D, causal, scale):
    # torch's fp64 CPU attention (a library routine) must agree; for causal only Sq == Sk, where
    # its top-left convention coincides with the bottom-right one.
    q, k, v = _rand(B, S, Hq, D), _rand(B, Sk, Hkv, D), _rand(B, Sk, Hkv, D)
    o, _ = fwd(q, k, v, causal, scale)
    np.testing.assert_allclose(o, _torch_sdpa(q, k, v, causal, scale), rtol=1e-11, atol=1e-12)


def pin_lse_library(fwd, causal):
    # lse against scipy's logsumexp of the scores built with numpy's einsum; with V = I the
    # library attention returns P itself, which must equal exp(x - lse).
    B, S, Hq, Hkv = 1, 6, 4, 2
    q, k = _rand(B, S, Hq, 3), _rand(B, S, Hkv, 3)
    v = np.broadcast_to(np.eye(S)[None, :, None, :], (B, S, Hkv, S)).copy()
    s = 0.7
    o, lse = fwd(q, k, v, causal, s)
    Pt = _torch_sdpa(q, k, v, causal, s)          # [B, S(i), Hq, S(j)] = P
    np.testing.assert_allclose(o, Pt, atol=1e-12)
    kk = np.repeat(k, Hq // Hkv, axis=2)
    x = s * np.einsum("bihd,bjhd->bhij", q, kk)
    if causal:
        x = np.where(np.tril(np.ones((S, S), bool))[None, None], x, -np.inf)
    np.testing.assert_allclose(lse, logsumexp(x, axis=-1), atol=1e-12)


def pin_fd_backward(fwd, bwd, B, Sq, Sk, Hq, Hkv, D, causal, scale, rtol=1e-6):
    # Central finite differences of L = sum(O * W) (so dL/dO = W) in fp64.
    rng = np.random.default_rng(7)
    q, k, v = rng.standard_normal((B, Sq, Hq, D)), rng.standard_normal((B, Sk, Hkv, D)), \
        rng.standard_normal((B, Sk, Hkv, D))
    W = rng.standard_normal((B, Sq, Hq, D))
    dq, dk, dv = bwd(q, k, v, W, causal, scale)
    h = 1e-6

    def loss(q_, k_, v_):
        return float(np.sum(fwd(q_, k_, v_, causal, scale)[0] * W))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in itertools.product(*[range(n) for n in x.shape]):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.max(np.abs(fd - g)) / max(np.max(np.abs(fd)), 1e-30)
        assert err < rtol, f"d{name}: finite-difference mismatch {err:.2e}"


def pin_brute_jacobian(bwd):
    # dS from the full Jacobian matrix J = diag(p) - p p^T applied to dP, row by row, vs the
    # closed form inside the backward (read off via dV, dQ on a one-head case).
    rng = np.random.default_rng(3)
    Sq, Sk, D = 4, 5, 3
    q, k, v = rng.standard_normal((1, Sq, 1, D)), rng.standard_normal((1, Sk, 1, D)), \
        rng.standard_normal((1, Sk, 1, D))
    do = rng.standard_normal((1, Sq, 1, D))
    s = 0.8
    x = s * q[0, :, 0] @ k[0, :, 0].T
    dQ = np.zeros((Sq, D))
    dK = np.zeros((Sk, D))
    dV = np.zeros((Sk, D))
    for i in range(Sq):
        p = softmax(x[i])                         # scipy
        J = np.diag(p) - np.outer(p, p)
        dp = v[0, :, 0] @ do[0, i, 0]             # dL/dP_j = dO_i . V_j
        dx = J.T @ dp
        dQ[i] = s * dx @ k[0, :, 0]
        dK += s * np.outer(dx, q[0, i, 0])
        dV += np.outer(p, do[0, i, 0])
    dq, dk, dv = bwd(q, k, v, do, False, s)
    np.testing.assert_allclose(dq[0, :, 0], dQ, atol=1e-12)
    np.testing.assert_allclose(dk[0, :, 0], dK, atol=1e-12)
    np.testing.assert_allclose(dv[0, :, 0], dV, atol=1e-12)


def pin_bwd_invariants(bwd, causal):
    # sum_j dS_ij = 0 per row, hence sum_j dK_j = 0 per key/value head, and
    # sum_j dV_j = sum over the group's query heads and rows of dO (P rows sum to 1).
    B, S, Hq, Hkv, D = 2, 7, 4, 2, 5
    q, k, v, do = _rand(B, S, Hq, D), _rand(B, S, Hkv, D), _rand(B, S, Hkv, D), _rand(B, S, Hq, D)
    dq, dk, dv = bwd(q, k, v, do, causal, 0.6)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    G = Hq // Hkv
    want = do.reshape(B, S, Hkv, G, D).sum(axis=(1, 3))
    np.testing.assert_allclose(dv.sum(axis=1), want, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# The pins applied to the oracle.
# ---------------------------------------------------------------------------------------------

FWD = oracle.attention_fwd
BWD = oracle.attention_bwd


def test_two_by_two_forward():
    pin_two_by_two_fwd(FWD)


def test_two_by_two_backward():
    pin_two_by_two_bwd(BWD)


def test_single_key_returns_v():
    pin_single_key(FWD)


@pytest.mark.parametrize("Sq,Sk,causal", [(6, 6, False), (6, 6, True), (4, 9, True), (9, 4, True),
                                          (1, 5, True), (5, 1, False)])
def test_constant_scores_give_mean_of_v(Sq, Sk, causal):
    pin_constant_scores(FWD, Sq, Sk, causal)


def test_tiny_scale_gives_mean():
    pin_tiny_scale(FWD)


def test_kv_permutation_invariance():
    pin_kv_permutation(FWD)


@pytest.mark.parametrize("B,S,Sk,Hq,Hkv,D,causal,scale", [
    (1, 8, 8, 2, 2, 4, False, 0.5), (2, 9, 9, 4, 2, 8, True, 0.3), (1, 5, 11, 8, 1, 3, False, 1.1),
    (1, 16, 16, 4, 4, 16, True, 0.25), (1, 1, 7, 4, 2, 8, False, 0.4)])
def test_against_library_attention(B, S, Sk, Hq, Hkv, D, causal, scale):
    pin_library_sdpa(FWD, B, S, Sk, Hq, Hkv, D, causal, scale)


@pytest.mark.parametrize("causal", [False, True])
def test_lse_against_library(causal):
    pin_lse_library(FWD, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one_and_lse_bounds(causal):
    q, k, v = _rand(2, 6, 4, 3), _rand(2, 8, 2, 3), _rand(2, 8, 2, 3)
    P = oracle.attention_probs(q, k, causal, 0.9)
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-12)
    x = oracle.attention_scores(q, k, causal, 0.9)
    _, lse = FWD(q, k, v, causal, 0.9)
    nvis = np.isfinite(x).sum(-1)
    xmax = x.max(-1)
    assert np.all(lse >= xmax - 1e-12) and np.all(lse <= xmax + np.log(nvis) + 1e-12)
    # P equals exp(x - lse) on visible keys and 0 elsewhere.
    with np.errstate(invalid="ignore"):
        want = np.where(np.isfinite(x), np.exp(x - lse[..., None]), 0.0)
    np.testing.assert_allclose(P, want, atol=1e-12)


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,D,causal", [
    (1, 3, 3, 2, 2, 2, False), (1, 3, 3, 2, 2, 2, True), (1, 3, 3, 2, 1, 2, True),
    (1, 2, 4, 2, 1, 2, True)])
def test_backward_matches_finite_differences(B, Sq, Sk, Hq, Hkv, D, causal):
    pin_fd_backward(FWD, BWD, B, Sq, Sk, Hq, Hkv, D, causal, 0.7)


def test_backward_matches_brute_force_jacobian():
    pin_brute_jacobian(BWD)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    pin_bwd_invariants(BWD, causal)


def test_fully_masked_rows_have_zero_gradient():
    # Sq > Sk with causal: the first Sq - Sk rows see nothing; their dQ is 0.
    q, k, v, do = _rand(1, 6, 2, 3), _rand(1, 3, 2, 3), _rand(1, 3, 2, 3), _rand(1, 6, 2, 3)
    dq, _, _ = BWD(q, k, v, do, True, 0.5)
    np.testing.assert_array_equal(dq[:, :3], 0.0)


def test_rows_oracle_matches_full_oracle():
    q, k, v = _rand(1, 40, 4, 8), _rand(1, 40, 2, 8), _rand(1, 40, 2, 8)
    o, lse = FWD(q, k, v, True, 0.35)
    rows = [0, 1, 17, 38, 39]
    for h in range(4):
        orow, lrow = oracle.attention_fwd_rows(q, k, v, True, 0.35, 0, h, rows)
        np.testing.assert_allclose(orow, o[0, rows, h], atol=1e-12)
        np.testing.assert_allclose(lrow, lse[0, h, rows], atol=1e-12)


def test_decode_matches_forward_with_one_query():
    rng = np.random.default_rng(5)
    lengths = [5, 1, 0, 12]
    off = np.concatenate([[0], np.cumsum(lengths)])
    N, Hq, Hkv, D = len(lengths), 4, 2, 6
    q = rng.standard_normal((N, Hq, D))
    k = rng.standard_normal((off[-1], Hkv, D))
    v = rng.standard_normal((off[-1], Hkv, D))
    o, lse = oracle.decode_attention(q, k, v, off, 0.45)
    for n in range(N):
        s, e = off[n], off[n + 1]
        if e == s:
            np.testing.assert_array_equal(o[n], 0.0)
            assert np.all(np.isneginf(lse[n]))
            continue
        o1 = _torch_sdpa(q[n][None, None], k[None, s:e], v[None, s:e], False, 0.45)
        np.testing.assert_allclose(o[n], o1[0, 0], atol=1e-12)
        of, lf = FWD(q[n][None, None], k[None, s:e], v[None, s:e], False, 0.45)
        np.testing.assert_allclose(lse[n], lf[0, :, 0], atol=1e-12)


def check_paged_rows(paged_rows):
    # pages of 2 rows; stream 0 owns pages 3 then 0 and has 3 keys, stream 1 owns page 1, 1 key,
    # stream 2 has none (its table row is never read, so it may hold anything)
    table = np.array([[3, 0], [1, 99], [-7, 42]])
    idx = paged_rows(table, [3, 1, 0], 2)
    np.testing.assert_array_equal(idx[0][0], [3, 3, 0])
    np.testing.assert_array_equal(idx[0][1], [0, 1, 0])
    np.testing.assert_array_equal(idx[1][0], [1])
    np.testing.assert_array_equal(idx[1][1], [0])
    assert len(idx[2][0]) == 0


def test_paged_rows_by_hand():
    check_paged_rows(oracle.paged_rows)


def check_paged_decode(decode_paged):
    # keys written into a shuffled pool by hand (a scatter, the inverse of the oracle's gather);
    # every pool row that holds no key is NaN and must not reach the result
    rng = np.random.default_rng(9)
    P, Hq, Hkv, D = 4, 6, 2, 5
    lengths = [7, 4, 0, 1, 9]
    q = rng.standard_normal((len(lengths), Hq, D))
    keys = [rng.standard_normal((L, Hkv, D)) for L in lengths]
    vals = [rng.standard_normal((L, Hkv, D)) for L in lengths]
    need = [(L + P - 1) // P for L in lengths]
    order = rng.permutation(sum(need) + 2)          # two spare pages
    kp = np.full((len(order), P, Hkv, D), np.nan)
    vp = np.full((len(order), P, Hkv, D), np.nan)
    table = np.full((len(lengths), max(need)), -1)
    used = 0
    for n, L in enumerate(lengths):
        for t in range(L):
            if t % P == 0:
                table[n, t // P] = order[used]
                used += 1
            kp[table[n, t // P], t % P] = keys[n][t]
            vp[table[n, t // P], t % P] = vals[n][t]
    o, lse = decode_paged(q, kp, vp, table, lengths, 0.4)
    assert np.all(np.isfinite(o))
    for n, L in enumerate(lengths):
        if L == 0:
            np.testing.assert_array_equal(o[n], 0.0)
            assert np.all(np.isneginf(lse[n]))
            continue
        o1 = _torch_sdpa(q[n][None, None], keys[n][None], vals[n][None], False, 0.4)
        np.testing.assert_allclose(o[n], o1[0, 0], atol=1e-12)
        for h in range(Hq):
            x = 0.4 * keys[n][:, h // (Hq // Hkv), :] @ q[n, h]
            assert abs(lse[n, h] - logsumexp(x)) < 1e-12


def test_paged_decode_matches_sdpa_per_stream():
    check_paged_decode(oracle.decode_attention_paged)


def check_decode_qlen(decode_qlen):
    # Several query tokens per stream: token t of a stream with L keys sees keys 0 .. L - q_len + t.
    # Written here from that definition with scipy's softmax / logsumexp per (stream, token, head),
    # plus torch's SDPA with the same mask as a boolean tensor.
    rng = np.random.default_rng(21)
    ql, Hq, Hkv, D = 3, 4, 2, 5
    lengths = [6, 3, 2, 0, 9, 1]              # L < q_len: the first tokens see no key
    off = np.concatenate([[0], np.cumsum(lengths)])
    q = rng.standard_normal((len(lengths), ql, Hq, D))
    k = rng.standard_normal((off[-1], Hkv, D))
    v = rng.standard_normal((off[-1], Hkv, D))
    o, lse = decode_qlen(q, k, v, off, 0.6)
    assert o.shape == (len(lengths), ql, Hq, D) and lse.shape == (len(lengths), Hq, ql)
    for n, L in enumerate(lengths):
        s = off[n]
        for t in range(ql):
            vis = L - ql + t + 1                  # number of keys token t sees
            for h in range(Hq):
                g = h // (Hq // Hkv)
                if vis <= 0:
                    np.testing.assert_array_equal(o[n, t, h], 0.0)
                    assert np.isneginf(lse[n, h, t])
                    continue
                x = 0.6 * k[s:s + vis, g] @ q[n, t, h]
                np.testing.assert_allclose(o[n, t, h], softmax(x) @ v[s:s + vis, g], atol=1e-12)
                assert abs(lse[n, h, t] - logsumexp(x)) < 1e-12
        if L >= ql:
            mask = torch.as_tensor(np.arange(L)[None, :] <= (np.arange(ql)[:, None] + L - ql))
            qt = torch.as_tensor(q[n]).permute(1, 0, 2)[None]                      # [1, Hq, ql, D]
            kt = torch.as_tensor(k[s:s + L]).repeat_interleave(Hq // Hkv, 1).permute(1, 0, 2)[None]
            vt = torch.as_tensor(v[s:s + L]).repeat_interleave(Hq // Hkv, 1).permute(1, 0, 2)[None]
            ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.6)[0].permute(1, 0, 2)
            np.testing.assert_allclose(o[n], ref.numpy(), atol=1e-12)


def test_decode_qlen_by_definition():
    check_decode_qlen(oracle.decode_attention_qlen)


def test_decode_qlen_one_token_is_decode():
    rng = np.random.default_rng(22)
    lengths = [4, 0, 7]
    off = np.concatenate([[0], np.cumsum(lengths)])
    q = rng.standard_normal((3, 4, 6))
    k = rng.standard_normal((off[-1], 2, 6))
    v = rng.standard_normal((off[-1], 2, 6))
    o1, l1 = oracle.decode_attention(q, k, v, off, 0.3)
    o2, l2 = oracle.decode_attention_qlen(q[:, None], k, v, off, 0.3)
    np.testing.assert_allclose(o2[:, 0], o1, atol=1e-14)
    np.testing.assert_array_equal(np.isneginf(l2[..., 0]), np.isneginf(l1))
    np.testing.assert_allclose(np.where(np.isneginf(l1), 0, l2[..., 0]), np.where(np.isneginf(l1), 0, l1), atol=1e-14)


def check_paged_decode_qlen(decode_paged_qlen):
    # the same pool-by-scatter as check_paged_decode, with two query tokens per stream
    rng = np.random.default_rng(23)
    P, Hq, Hkv, D, ql = 4, 4, 2, 5, 2
    lengths = [7, 1, 0, 9]
    q = rng.standard_normal((len(lengths), ql, Hq, D))
    keys = [rng.standard_normal((L, Hkv, D)) for L in lengths]
    vals = [rng.standard_normal((L, Hkv, D)) for L in lengths]
    need = [(L + P - 1) // P for L in lengths]
    order = rng.permutation(sum(need) + 1)
    kp = np.full((len(order), P, Hkv, D), np.nan)
    vp = np.full((len(order), P, Hkv, D), np.nan)
    table = np.full((len(lengths), max(need)), -1)
    used = 0
    for n, L in enumerate(lengths):
        for t in range(L):
            if t % P == 0:
                table[n, t // P] = order[used]
                used += 1
            kp[table[n, t // P], t % P] = keys[n][t]
            vp[table[n, t // P], t % P] = vals[n][t]
    o, lse = decode_paged_qlen(q, kp, vp, table, lengths, 0.4)
    assert np.all(np.isfinite(o))
    for n, L in enumerate(lengths):
        for t in range(ql):
            vis = L - ql + t + 1
            for h in range(Hq):
                if vis <= 0:
                    assert np.all(o[n, t, h] == 0) and np.isneginf(lse[n, h, t])
                    continue
                x = 0.4 * keys[n][:vis, h // (Hq // Hkv)] @ q[n, t, h]
                np.testing.assert_allclose(o[n, t, h], softmax(x) @ vals[n][:vis, h // (Hq // Hkv)], atol=1e-12)
                assert abs(lse[n, h, t] - logsumexp(x)) < 1e-12


def test_paged_decode_qlen_by_definition():
    check_paged_decode_qlen(oracle.decode_attention_paged_qlen)


def check_varlen(fwd_varlen, bwd_varlen):
    # Packed sequences of different lengths. Pins: (1) a batch of equal lengths equals the padded
    # batch's torch SDPA (bottom-right causal, GQA by repeating kv heads); (2) every sequence equals
    # torch SDPA on its own slices, so no sequence sees another's keys; (3) a sequence with no key
    # or no query row contributes nothing and its rows get O = 0, lse = -inf; (4) the gradients
    # match central finite differences of the packed forward on a tiny case.
    rng = np.random.default_rng(31)
    Hq, Hkv, D = 4, 2, 3
    lq = [3, 0, 5, 2, 4]
    lk = [5, 2, 5, 0, 4]
    cq = np.concatenate([[0], np.cumsum(lq)])
    ck = np.concatenate([[0], np.cumsum(lk)])
    q = rng.standard_normal((cq[-1], Hq, D))
    k = rng.standard_normal((ck[-1], Hkv, D))
    v = rng.standard_normal((ck[-1], Hkv, D))
    do = rng.standard_normal((cq[-1], Hq, D))
    for causal in (False, True):
        o, lse = fwd_varlen(q, k, v, cq, ck, causal, 0.7)
        assert o.shape == q.shape and lse.shape == (Hq, cq[-1])
        for b in range(len(lq)):
            rows = slice(cq[b], cq[b + 1])
            if lq[b] == 0:
                continue
            if lk[b] == 0:
                assert np.all(o[rows] == 0) and np.all(np.isneginf(lse[:, rows]))
                continue
            # torch's is_causal is top-left aligned; the bottom-right mask goes in as a boolean tensor
            mask = torch.as_tensor(np.arange(lk[b])[None] <= np.arange(lq[b])[:, None] + lk[b] - lq[b]) \
                if causal else None
            t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).permute(1, 0, 2)[None]
            ref = F.scaled_dot_product_attention(t(q[rows]), t(k[ck[b]:ck[b + 1]]), t(v[ck[b]:ck[b + 1]]),
                                                 attn_mask=mask, scale=0.7, enable_gqa=True)
            np.testing.assert_allclose(o[rows], ref[0].permute(1, 0, 2).numpy(), atol=1e-12)
            for h in range(Hq):
                x = 0.7 * q[rows, h] @ k[ck[b]:ck[b + 1], h // 2].T
                if causal:
                    x = np.where(np.arange(lk[b])[None] <= np.arange(lq[b])[:, None] + lk[b] - lq[b], x, -np.inf)
                with np.errstate(divide="ignore"):
                    want = logsumexp(x, axis=1)
                np.testing.assert_allclose(lse[h, rows], want, atol=1e-12)
    # finite differences of sum(O * dO) on the packed batch
    causal = True
    dq, dk, dv = bwd_varlen(q, k, v, do, cq, ck, causal, 0.7)
    f = lambda qq, kk, vv: float(np.sum(fwd_varlen(qq, kk, vv, cq, ck, causal, 0.7)[0] * do))
    eps = 1e-6
    for arr, grad in ((q, dq), (k, dk), (v, dv)):
        for idx in [(0, 0, 0), (arr.shape[0] - 1, 1, 2), (arr.shape[0] // 2, arr.shape[1] - 1, 1)]:
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += eps
            a2[idx] -= eps
            args1 = [a1 if arr is x else x for x in (q, k, v)]
            args2 = [a2 if arr is x else x for x in (q, k, v)]
            fd = (f(*args1) - f(*args2)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-6 * max(1.0, abs(fd)), (idx, fd, grad[idx])


def test_varlen_by_definition():
    check_varlen(oracle.attention_fwd_varlen, oracle.attention_bwd_varlen)


def test_varlen_equal_lengths_is_the_dense_batch():
    rng = np.random.default_rng(32)
    B, S, Hq, Hkv, D = 3, 6, 4, 2, 4
    q, k, v, do = (rng.standard_normal((B, S, H, D)) for H in (Hq, Hkv, Hkv, Hq))
    cu = np.arange(B + 1) * S
    for causal in (False, True):
        o, lse = oracle.attention_fwd_varlen(q.reshape(-1, Hq, D), k.reshape(-1, Hkv, D), v.reshape(-1, Hkv, D),
                                             cu, cu, causal, 0.5)
        od, ld = oracle.attention_fwd(q, k, v, causal, 0.5)
        np.testing.assert_allclose(o, od.reshape(-1, Hq, D), atol=1e-14)
        np.testing.assert_allclose(lse, ld.transpose(1, 0, 2).reshape(Hq, -1), atol=1e-14)
        g = oracle.attention_bwd_varlen(q.reshape(-1, Hq, D), k.reshape(-1, Hkv, D), v.reshape(-1, Hkv, D),
                                        do.reshape(-1, Hq, D), cu, cu, causal, 0.5)
        gd = oracle.attention_bwd(q, k, v, do, causal, 0.5)
        for a, b in zip(g, gd):
            np.testing.assert_allclose(a, b.reshape(a.shape), atol=1e-14)


def check_e4m3(decode):
    # hand-worked codes, then every code against torch's float8_e4m3fn conversion (a library routine)
    assert decode(0x38) == 1.0                      # e = 7, m = 0
    assert decode(0x7E) == 448.0                    # largest finite: 2^8 * 1.75
    assert decode(0x01) == 2.0 ** -9                # smallest subnormal: 2^-6 * 1/8
    assert decode(0x08) == 2.0 ** -6                # smallest normal
    assert decode(0xB8) == -1.0 and decode(0x3C) == 1.5 and decode(0x44) == 3.0
    assert np.isnan(decode(0x7F)) and np.isnan(decode(0xFF))
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    np.testing.assert_array_equal(got[~np.isnan(ref)], ref[~np.isnan(ref)])


def test_e4m3_decoder():
    check_e4m3(oracle.e4m3_to_float)


def check_fp8_attention(fwd8):
    # the per-tensor scales enter as the real inputs: q_scale and k_scale only through their
    # product in the scores, v_scale as a factor of O (lse does not depend on it)
    rng = np.random.default_rng(33)
    vals = torch.from_numpy(rng.standard_normal((3, 1, 20, 2, 8)))
    q8, k8, v8 = (x.to(torch.float8_e4m3fn).view(torch.uint8).numpy() for x in vals)
    dq, dk, dv = (torch.from_numpy(x).view(torch.float8_e4m3fn).to(torch.float64).numpy() for x in (q8, k8, v8))
    for causal in (False, True):
        o, lse = fwd8(q8, k8, v8, 0.5, 3.0, 2.0, causal, 0.3)
        o_ref, lse_ref = oracle.attention_fwd(0.5 * dq, 3.0 * dk, 2.0 * dv, causal, 0.3)
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-12)
        o2, lse2 = fwd8(q8, k8, v8, 1.5, 1.0, 1.0, causal, 0.3)   # same score scale product
        np.testing.assert_allclose(o2 * 2.0, o, atol=1e-12)
        np.testing.assert_allclose(lse2, lse, atol=1e-12)


def test_fp8_attention_scales():
    check_fp8_attention(oracle.attention_fwd_fp8)


# ---------------------------------------------------------------------------------------------
# Monoid algebra.
# ---------------------------------------------------------------------------------------------

def _rand_triple(D, rng):
    m = rng.standard_normal() * 3
    return (m, rng.uniform(0.5, 4.0), rng.standard_normal(D))


def _close(a, b, tol=1e-12):
    assert (a[0] == b[0]) or abs(a[0] - b[0]) < tol
    assert abs(a[1] - b[1]) <= tol * max(1.0, abs(a[1]))
    np.testing.assert_allclose(a[2], b[2], rtol=tol, atol=tol)


def test_monoid_associative_and_commutative():
    rng = np.random.default_rng(11)
    for _ in range(200):
        a, b, c = (_rand_triple(5, rng) for _ in range(3))
        M = oracle.monoid_merge
        _close(M(M(a, b), c), M(a, M(b, c)))
        _close(M(a, b), M(b, a))


def test_monoid_identity():
    rng = np.random.default_rng(12)
    e = oracle.monoid_identity(5)
    for _ in range(20):
        a = _rand_triple(5, rng)
        _close(oracle.monoid_merge(a, e), a)
        _close(oracle.monoid_merge(e, a), a)
    ee = oracle.monoid_merge(e, e)
    assert ee[0] == -np.inf and ee[1] == 0.0 and not np.any(np.isnan(ee[2]))
    o, lse = oracle.monoid_finalize(ee)
    assert np.all(o == 0) and lse == -np.inf


def test_monoid_any_partition_and_tree_equals_two_pass():
    rng = np.random.default_rng(13)
    n, D, s = 37, 6, 0.8
    q = rng.standard_normal(D)
    k = rng.standard_normal((n, D))
    v = rng.standard_normal((n, D))
    x = s * k @ q
    leaves = [oracle.monoid_leaf(x[j], v[j]) for j in range(n)]
    o_ref, lse_ref = FWD(q[None, None, None], k[None, :, None], v[None, :, None], False, s)
    o_ref, lse_ref = o_ref[0, 0, 0], lse_ref[0, 0, 0]
    for trial in range(30):
        # a random partition into chunks, an empty chunk thrown in, merged in a random tree order
        cuts = np.sort(rng.choice(np.arange(1, n), size=rng.integers(0, 8), replace=False))
        chunks = np.split(np.arange(n), cuts)
        parts = []
        for ch in chunks:
            t = oracle.monoid_identity(D)
            for j in ch:
                t = oracle.monoid_merge(t, leaves[j])
            parts.append(t)
        parts.append(oracle.monoid_identity(D))
        while len(parts) > 1:
            i = rng.integers(0, len(parts) - 1)
            parts[i:i + 2] = [oracle.monoid_merge(parts[i], parts[i + 1])]
        o, lse = oracle.monoid_finalize(parts[0])
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        assert abs(lse - lse_ref) < 1e-12


def test_monoid_chunk_with_minus_inf_max():
    rng = np.random.default_rng(14)
    a = _rand_triple(4, rng)
    neg = (-np.inf, 0.0, np.zeros(4))
    _close(oracle.monoid_merge(neg, a), a)
    _close(oracle.monoid_merge(a, neg), a)
