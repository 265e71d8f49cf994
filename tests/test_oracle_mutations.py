"""Planted mistakes: each plausible error in the oracle must make at least one pin fail (CPU only).

The broken variants below are built on the CPU from the oracle (wrappers that misuse it, or a copy
of the closed-form backward with one deliberate slip). A pin that passed on a broken oracle would
be no pin at all.
"""
import math

import numpy as np
import pytest

import oracle
from tests import test_oracle as T

FWD = oracle.attention_fwd


def fwd_dropped_scale(q, k, v, causal, scale):
    return FWD(q, k, v, causal, 1.0)


def fwd_top_left_causal(q, k, v, causal, scale):
    # Causal aligned to the top-left corner (query i sees keys j <= i) instead of bottom-right.
    Sq, Sk = q.shape[1], k.shape[1]
    if not causal or Sq >= Sk:
        return FWD(q, k, v, causal, scale)
    pad = np.zeros((q.shape[0], Sk - Sq) + q.shape[2:])
    o, lse = FWD(np.concatenate([q, pad], axis=1), k, v, causal, scale)
    return o[:, :Sq], lse[..., :Sq]


def fwd_gqa_modulo(q, k, v, causal, scale):
    # Query head h read from key/value head h % Hkv instead of h // (Hq / Hkv).
    Hq, Hkv = q.shape[2], k.shape[2]
    outs, lses = [], []
    for h in range(Hq):
        g = h % Hkv
        o, l = FWD(q[:, :, h:h + 1], k[:, :, g:g + 1], v[:, :, g:g + 1], causal, scale)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs, axis=2), np.concatenate(lses, axis=1)


def fwd_log2_lse(q, k, v, causal, scale):
    o, lse = FWD(q, k, v, causal, scale)
    return o, lse / math.log(2.0)


def make_bwd(mistake):
    def bwd(q, k, v, do, causal, scale):
        q, k, v, do = (np.asarray(t, np.float64) for t in (q, k, v, do))
        B, Sq, Hq, D = q.shape
        Sk, Hkv = k.shape[1], k.shape[2]
        G = Hq // Hkv
        vis = oracle.visible_mask(Sq, Sk, causal)
        P_all = oracle.attention_probs(q, k, causal, scale)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for b in range(B):
            for h in range(Hq):
                g = h // G
                P = P_all[b, h]
                O = P @ v[b, :, g]
                dP = do[b, :, h] @ v[b, :, g].T
                delta = np.sum(do[b, :, h] * O, axis=1)
                if mistake == "delta_sign":
                    dS = P * (dP + delta[:, None])
                elif mistake == "no_delta":
                    dS = P * dP
                else:
                    dS = P * (dP - delta[:, None])
                dq[b, :, h] = (1.0 if mistake == "dq_no_scale" else scale) * (dS @ k[b, :, g])
                if mistake == "dk_transposed":
                    dk[b, :, g] += scale * (dS @ q[b, :, h])
                else:
                    dk[b, :, g] += scale * (dS.T @ q[b, :, h])
                if mistake == "dv_uses_dS":
                    dv[b, :, g] += dS.T @ do[b, :, h]
                elif mistake == "dv_no_group_sum":
                    dv[b, :, g] = P.T @ do[b, :, h]
                else:
                    dv[b, :, g] += P.T @ do[b, :, h]
        return dq, dk, dv
    return bwd


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_control_unbroken_backward_copy_passes_the_pins():
    good = make_bwd(None)
    assert not _fails(T.pin_two_by_two_bwd, good)
    assert not _fails(T.pin_fd_backward, FWD, good, 1, 3, 3, 2, 1, 2, True, 0.7)


@pytest.mark.parametrize("bad,pins", [
    (fwd_dropped_scale, [(T.pin_single_key,), (T.pin_library_sdpa, 1, 8, 8, 2, 2, 4, False, 0.5)]),
    (fwd_top_left_causal, [(T.pin_constant_scores, 4, 9, True)]),
    (fwd_gqa_modulo, [(T.pin_library_sdpa, 2, 9, 9, 4, 2, 8, True, 0.3), (T.pin_lse_library, True)]),
    (fwd_log2_lse, [(T.pin_two_by_two_fwd,), (T.pin_constant_scores, 6, 6, True)]),
])
def test_forward_mistakes_are_caught(bad, pins):
    for pin, *args in pins:
        assert _fails(pin, bad, *args), f"{pin.__name__} missed {bad.__name__}"


@pytest.mark.parametrize("mistake", ["delta_sign", "no_delta", "dq_no_scale", "dk_transposed",
                                     "dv_uses_dS", "dv_no_group_sum"])
def test_backward_mistakes_are_caught(mistake):
    bad = make_bwd(mistake)
    caught = (_fails(T.pin_fd_backward, FWD, bad, 1, 3, 3, 2, 1, 2, True, 0.7)
              or _fails(T.pin_two_by_two_bwd, bad))
    assert caught, f"no pin caught backward mistake {mistake}"


def test_monoid_merge_without_rescale_is_caught():
    def bad_merge(a, b):
        M = max(a[0], b[0])
        return (M, a[1] + b[1], a[2] + b[2])

    rng = np.random.default_rng(0)
    D, s = 4, 0.9
    q, k, v = rng.standard_normal(D), rng.standard_normal((9, D)), rng.standard_normal((9, D))
    x = s * k @ q
    t = oracle.monoid_identity(D)
    for j in range(9):
        t = bad_merge(t, oracle.monoid_leaf(x[j], v[j]))
    o, _ = oracle.monoid_finalize(t)
    o_ref, _ = FWD(q[None, None, None], k[None, :, None], v[None, :, None], False, s)
    assert not np.allclose(o, o_ref[0, 0, 0], atol=1e-6)


# ---------------------------------------------------------------------------------------------
# Paged decode: the gather of a stream's keys from its pages.
# ---------------------------------------------------------------------------------------------

def paged_rows_swapped(block_table, seq_lens, page_size):
    # page and row index exchanged: page from t % page_size, row from t // page_size
    bt = np.asarray(block_table, dtype=np.int64)
    out = []
    for n, L in enumerate(np.asarray(seq_lens, dtype=np.int64)):
        t = np.arange(int(L), dtype=np.int64)
        out.append((bt[n, np.minimum(t % page_size, bt.shape[1] - 1)], t // page_size))
    return out


def paged_rows_first_page_only(block_table, seq_lens, page_size):
    # every key read from the stream's first page
    bt = np.asarray(block_table, dtype=np.int64)
    return [(np.full(int(L), bt[n, 0]), np.arange(int(L)) % page_size)
            for n, L in enumerate(np.asarray(seq_lens, dtype=np.int64))]


def paged_decode_with(rows_fn):
    def decode(q, k_pages, v_pages, block_table, seq_lens, scale):
        k_pages, v_pages = np.asarray(k_pages, np.float64), np.asarray(v_pages, np.float64)
        idx = rows_fn(block_table, seq_lens, k_pages.shape[1])
        k = np.concatenate([k_pages[p, r] for p, r in idx], axis=0)
        v = np.concatenate([v_pages[p, r] for p, r in idx], axis=0)
        off = np.concatenate([[0], np.cumsum([len(p) for p, _ in idx])])
        return oracle.decode_attention(q, k, v, off, scale)
    return decode


@pytest.mark.parametrize("rows_fn", [paged_rows_swapped, paged_rows_first_page_only])
def test_paged_pins_catch_gather_mistakes(rows_fn):
    with pytest.raises(AssertionError):
        T.check_paged_rows(rows_fn)
    with pytest.raises(AssertionError):
        T.check_paged_decode(paged_decode_with(rows_fn))


def decode_qlen_top_left(q, k, v, offsets, scale):
    # Several tokens per stream with the mask aligned to the top-left corner (token t sees keys
    # 0 .. t) instead of the newest positions.
    off = np.asarray(offsets)
    N, ql, Hq, D = q.shape
    o = np.zeros((N, ql, Hq, D))
    lse = np.full((N, Hq, ql), -np.inf)
    for n in range(N):
        s, e = off[n], off[n + 1]
        if e <= s:
            continue
        L = e - s
        qq = np.concatenate([q[n], np.zeros((max(0, L - ql), Hq, D))], axis=0)[None] if L > ql else q[n][None]
        on, ln = oracle.attention_fwd(qq, k[None, s:e], v[None, s:e], True, scale)
        o[n], lse[n] = on[0, :ql], ln[0, :, :ql]
    return o, lse


def decode_qlen_last_token_for_all(q, k, v, offsets, scale):
    # every token sees the whole cache (the causal mask among the new tokens forgotten)
    off = np.asarray(offsets)
    N, ql, Hq, D = q.shape
    o = np.zeros((N, ql, Hq, D))
    lse = np.full((N, Hq, ql), -np.inf)
    for t in range(ql):
        ot, lt = oracle.decode_attention(q[:, t], k, v, off, scale)
        o[:, t], lse[:, :, t] = ot, lt
    return o, lse


@pytest.mark.parametrize("bad", [decode_qlen_top_left, decode_qlen_last_token_for_all])
def test_decode_qlen_mistakes_are_caught(bad):
    with pytest.raises(AssertionError):
        T.check_decode_qlen(bad)


def varlen_one_sequence(q, k, v, cq, ck, causal, scale):
    # the packed rows treated as one long sequence: sequences see each other's keys
    o, lse = oracle.attention_fwd(q[None], k[None], v[None], causal, scale)
    return o[0], lse[0]


def varlen_bwd_one_sequence(q, k, v, do, cq, ck, causal, scale):
    g = oracle.attention_bwd(q[None], k[None], v[None], do[None], causal, scale)
    return tuple(x[0] for x in g)


def varlen_bwd_without_dv(q, k, v, do, cq, ck, causal, scale):
    dq, dk, dv = oracle.attention_bwd_varlen(q, k, v, do, cq, ck, causal, scale)
    return dq, dk, np.zeros_like(dv)


@pytest.mark.parametrize("fwd,bwd", [
    (varlen_one_sequence, oracle.attention_bwd_varlen),
    (oracle.attention_fwd_varlen, varlen_bwd_one_sequence),
    (oracle.attention_fwd_varlen, varlen_bwd_without_dv),
])
def test_varlen_mistakes_are_caught(fwd, bwd):
    with pytest.raises(AssertionError):
        T.check_varlen(fwd, bwd)


def e4m3_bias_8(codes):
    return oracle.e4m3_to_float(codes) / 2.0


def e4m3_no_subnormals(codes):
    c = np.asarray(codes, dtype=np.int64) & 0xFF
    v = oracle.e4m3_to_float(codes)
    return np.where(((c >> 3) & 0xF) == 0, 0.0 * v, v)


@pytest.mark.parametrize("bad", [e4m3_bias_8, e4m3_no_subnormals])
def test_e4m3_decoder_mistakes_are_caught(bad):
    with pytest.raises(AssertionError):
        T.check_e4m3(bad)


def fp8_v_scale_on_scores(q8, k8, v8, qs, ks, vs, causal, scale):
    return oracle.attention_fwd_fp8(q8, k8, v8, qs * vs, ks, 1.0, causal, scale)


def test_fp8_scale_mistake_is_caught():
    with pytest.raises(AssertionError):
        T.check_fp8_attention(fp8_v_scale_on_scores)
