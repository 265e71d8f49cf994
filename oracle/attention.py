"""fp64 NumPy oracle: scaled-dot-product attention written as its plain definition.

TEST INFRASTRUCTURE ONLY (see the package docstring for who may import it).

Sources. The pages state the method only in words:
  * "Não escreva kernels, derive-os" (ceviu.com.br), section "Aprofundamento", first paragraph:
    flash attention is what falls out once the online softmax is recognised as a monoid, and a
    comprehension is a reduction under a monoid whose body is a graph of scalar expressions.
  * Same page, section "Perguntas frequentes", "O que o Tang propõe de diferente?": the backward
    pass also comes out of rewrites of the same graph.
  * "Tang Project Derives GPU Kernels via IR ..." (aibriefing.imbch.dev), section "Details", fourth
    bullet: the workload includes causal forward passes.
No formula is printed on any page. Readings taken where the pages are silent:
  * attention is softmax(scale * Q K^T + mask) V, per query head h over key/value head
    g = h // (Hq / Hkv) (grouped-query heads, contiguous groups);
  * the causal mask is bottom-right aligned: query i sees key j iff j <= i + (Sk - Sq);
  * a query row that sees no key has O = 0 and lse = -inf;
  * lse is the natural log of sum_j exp(x_j) over the visible scaled scores x_j;
  * the backward differentiates O only (not lse), using the softmax Jacobian diag(P) - P P^T;
  * the monoid is the textbook online-softmax triple (m, l, o) with o unnormalised and the merge
    (m,l,o) (+) (m',l',o') = (M, l e^{m-M} + l' e^{m'-M}, o e^{m-M} + o' e^{m'-M}), M = max(m, m'),
    identity (-inf, 0, 0), and e^{-inf - M} taken as 0 so no inf - inf is ever formed.

Layouts (row-major): Q, O, dO, dQ are [B, Sq, Hq, D]; K, V, dK, dV are [B, Sk, Hkv, D]; lse is
[B, Hq, Sq]. Decode: q [N, Hq, D], packed k, v [T, Hkv, D], offsets [N + 1]; or a paged cache:
pools [num_pages, page_size, Hkv, D], block_table [N, max_pages], seq_lens [N].

The attention functions use the explicit two-pass softmax (pass 1: the row max; pass 2: the
exponentials, their sum and the weighted sum of V). The monoid functions exist for the algebra
tests only; the attention oracle does not use them.
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _dims(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be 4-D [B, S, H, D]")
    B, Sq, Hq, D = q.shape
    Bk, Sk, Hkv, Dk = k.shape
    if Bk != B or Dk != D or v.shape[:3] != k.shape[:3]:
        raise ValueError(f"shape mismatch q{q.shape} k{k.shape} v{v.shape}")
    if Hkv <= 0 or Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return B, Sq, Sk, Hq, Hkv, D, Hq // Hkv


def visible_mask(Sq: int, Sk: int, causal: bool) -> np.ndarray:
    """bool [Sq, Sk]: True where query i may attend to key j.

    Causal masking (the "causal forward passes" of the aibriefing page, "Details") is read as
    bottom-right aligned: j <= i + (Sk - Sq). With Sq == Sk this is the usual j <= i.
    """
    if not causal:
        return np.ones((Sq, Sk), dtype=bool)
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    return j <= i + (Sk - Sq)


def attention_scores(q, k, causal: bool, scale: float) -> np.ndarray:
    """Scaled scores x[b, h, i, j] = scale * sum_d Q[b,i,h,d] K[b,j,h//G,d]; masked entries -inf.

    The body of the attention comprehension ("Não escreva kernels, derive-os", "Aprofundamento",
    first paragraph). Returns fp64 [B, Hq, Sq, Sk]; meant for small shapes.
    """
    q, k = _f64(q), _f64(k)
    B, Sq, Sk, Hq, Hkv, D, G = _dims(q, k, k)
    vis = visible_mask(Sq, Sk, causal)
    x = np.empty((B, Hq, Sq, Sk), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            xh = scale * (q[b, :, h, :] @ k[b, :, g, :].T)
            x[b, h] = np.where(vis, xh, NEG_INF)
    return x


def _two_pass_softmax(x: np.ndarray, vis: np.ndarray):
    """Explicit two-pass softmax of one head's score matrix x [Sq, Sk] under mask vis.

    Pass 1 takes the row max M; pass 2 forms e^{x - M}, its sum Z and P = e / Z. Rows with no
    visible key give P = 0, M = -inf, Z = 0. Returns (P, M, Z).
    """
    x = np.where(vis, x, NEG_INF)
    has_key = vis.any(axis=1)
    M = np.where(has_key, x.max(axis=1, initial=NEG_INF), NEG_INF)      # pass 1
    M_safe = np.where(has_key, M, 0.0)
    e = np.where(vis, np.exp(x - M_safe[:, None]), 0.0)                 # pass 2
    Z = e.sum(axis=1)
    Z_safe = np.where(Z > 0, Z, 1.0)
    P = e / Z_safe[:, None]
    return P, M, Z


def attention_probs(q, k, causal: bool, scale: float) -> np.ndarray:
    """Softmax probabilities P[b, h, i, j] (fp64), rows over visible keys; for invariant tests."""
    q, k = _f64(q), _f64(k)
    B, Sq, Sk, Hq, Hkv, D, G = _dims(q, k, k)
    vis = visible_mask(Sq, Sk, causal)
    x = attention_scores(q, k, causal, scale)
    P = np.empty_like(x)
    for b in range(B):
        for h in range(Hq):
            P[b, h] = _two_pass_softmax(x[b, h], vis)[0]
    return P


def attention_fwd(q, k, v, causal: bool, scale: float):
    """Forward attention O = softmax(scale * Q K^T + mask) V and lse = M + ln Z, in fp64.

    The plain definition that the flash form reaches up to rounding ("Não escreva kernels,
    derive-os", "Aprofundamento", first paragraph). Returns (O [B,Sq,Hq,D], lse [B,Hq,Sq]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, Sk, Hq, Hkv, D, G = _dims(q, k, v)
    vis = visible_mask(Sq, Sk, causal)
    o = np.zeros((B, Sq, Hq, v.shape[3]), dtype=np.float64)
    lse = np.full((B, Hq, Sq), NEG_INF, dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            x = scale * (q[b, :, h, :] @ k[b, :, g, :].T)
            P, M, Z = _two_pass_softmax(x, vis)
            o[b, :, h, :] = P @ v[b, :, g, :]
            with np.errstate(divide="ignore"):
                lse[b, h] = np.where(Z > 0, M + np.log(np.where(Z > 0, Z, 1.0)), NEG_INF)
    return o, lse


def attention_fwd_rows(q, k, v, causal: bool, scale: float, b: int, h: int, rows):
    """Forward attention for selected query rows of one (batch, head): exact over all visible keys.

    Same definition as ``attention_fwd``; used where the full output is too large for the oracle
    (the 44k-token causal prefill of "Não escreva kernels, derive-os", "Aprofundamento", third
    paragraph). Returns (O [len(rows), D], lse [len(rows)]).
    """
    rows = np.asarray(rows, dtype=np.int64)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    g = h // G
    kg = _f64(k[b, :, g, :])
    vg = _f64(v[b, :, g, :])
    qr = _f64(q[b, rows, h, :])
    x = scale * (qr @ kg.T)                                     # [R, Sk]
    if causal:
        vis = np.arange(Sk)[None, :] <= (rows[:, None] + (Sk - Sq))
    else:
        vis = np.ones_like(x, dtype=bool)
    P, M, Z = _two_pass_softmax(x, vis)
    o = P @ vg
    with np.errstate(divide="ignore"):
        lse = np.where(Z > 0, M + np.log(np.where(Z > 0, Z, 1.0)), NEG_INF)
    return o, lse


def attention_bwd(q, k, v, do, causal: bool, scale: float):
    """Backward of O = softmax(x) V with x = scale * Q K^T + mask, from the softmax Jacobian.

    With P the softmax rows, dP = dO V^T and Delta_i = sum_d dO_i O_i = sum_j P_ij dP_ij, the
    Jacobian diag(P) - P P^T gives dS_ij = P_ij (dP_ij - Delta_i); then
    dQ = scale dS K, dK = scale dS^T Q and dV = P^T dO, dK and dV summed over the query heads that
    share a key/value head. The backward "comes out of rewrites" of the same graph
    ("Não escreva kernels, derive-os", "Perguntas frequentes", "O que o Tang propõe de diferente?").
    O is recomputed here from the definition; lse is not differentiated.
    Returns (dQ [B,Sq,Hq,D], dK [B,Sk,Hkv,D], dV [B,Sk,Hkv,D]).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Sq, Sk, Hq, Hkv, D, G = _dims(q, k, v)
    if do.shape != q.shape:
        raise ValueError("dO must have the shape of Q")
    vis = visible_mask(Sq, Sk, causal)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            x = scale * (q[b, :, h, :] @ k[b, :, g, :].T)
            P, _, _ = _two_pass_softmax(x, vis)
            O = P @ v[b, :, g, :]
            dP = do[b, :, h, :] @ v[b, :, g, :].T
            delta = np.sum(do[b, :, h, :] * O, axis=1)
            dS = P * (dP - delta[:, None])
            dq[b, :, h, :] = scale * (dS @ k[b, :, g, :])
            dk[b, :, g, :] += scale * (dS.T @ q[b, :, h, :])
            dv[b, :, g, :] += P.T @ do[b, :, h, :]
    return dq, dk, dv


def attention_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, causal: bool, scale: float):
    """Forward attention over a packed batch of sequences of different lengths (the multi-stream
    prefill behind the 44k-token time to first token of "Não escreva kernels, derive-os",
    "Aprofundamento", third paragraph): sequence b owns query rows cu_q[b] .. cu_q[b+1] - 1 and
    key/value rows cu_k[b] .. cu_k[b+1] - 1, and attends only to its own keys (causal: bottom-right
    aligned within the sequence). Each sequence is ``attention_fwd`` with B = 1 on its slices.
    q [Tq, Hq, D]; k, v [Tk, Hkv, D]. Returns (O [Tq, Hq, D], lse [Hq, Tq])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    Tq, Hq, D = q.shape
    o = np.zeros((Tq, Hq, v.shape[2]), dtype=np.float64)
    lse = np.full((Hq, Tq), NEG_INF, dtype=np.float64)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if q1 <= q0 or k1 <= k0:
            continue                      # no query rows, or no key: O = 0, lse = -inf
        ob, lb = attention_fwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], causal, scale)
        o[q0:q1] = ob[0]
        lse[:, q0:q1] = lb[0]
    return o, lse


def attention_bwd_varlen(q, k, v, do, cu_seqlens_q, cu_seqlens_k, causal: bool, scale: float):
    """Backward of ``attention_fwd_varlen``: ``attention_bwd`` on each sequence's slices; keys of
    a sequence that no query row sees get dK = dV = 0. Returns (dQ [Tq,Hq,D], dK, dV [Tk,Hkv,D])."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if q1 <= q0 or k1 <= k0:
            continue
        gq, gk, gv = attention_bwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], do[None, q0:q1], causal, scale)
        dq[q0:q1], dk[k0:k1], dv[k0:k1] = gq[0], gk[0], gv[0]
    return dq, dk, dv


def e4m3_to_float(codes) -> np.ndarray:
    """Values of 8-bit E4M3 codes (the OCP 8-bit floating-point format with 4 exponent bits, bias 7,
    and 3 mantissa bits; no infinities, S.1111.111 is NaN): exponent field 0 is subnormal,
    (-1)^s 2^-6 m/8; otherwise (-1)^s 2^(e-7) (1 + m/8). Largest finite value 448."""
    c = np.asarray(codes, dtype=np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def attention_fwd_fp8(q8, k8, v8, q_scale: float, k_scale: float, v_scale: float, causal: bool, scale: float):
    """Forward attention on 8-bit E4M3 inputs with per-tensor scales (the FP8 checkpoint the third
    paragraph of "Aprofundamento" credits with a much shorter time to first token): the real inputs
    are Q = q_scale q8, K = k_scale k8, V = v_scale v8, and the result is ``attention_fwd`` of them.
    q8 [B, Sq, Hq, D], k8 / v8 [B, Sk, Hkv, D] hold the codes (uint8). Returns (O, lse) in fp64."""
    q = q_scale * e4m3_to_float(q8)
    k = k_scale * e4m3_to_float(k8)
    v = v_scale * e4m3_to_float(v8)
    return attention_fwd(q, k, v, causal, scale)


def decode_attention(q, k, v, offsets, scale: float):
    """Decode attention: stream n's single query attends all L_n = off[n+1] - off[n] of its keys.

    The decode streams of "Não escreva kernels, derive-os" ("Aprofundamento", third paragraph: 16 to
    48 concurrent streams). The newest position sees every cached key, so there is no mask; this is
    the forward with Sq = 1 and Sk = L_n. Splitting the keys and merging partial triples changes
    only rounding, so the oracle does not split. A stream with no key gives O = 0, lse = -inf.
    q [N, Hq, D]; packed k, v [T, Hkv, D]; offsets [N + 1]. Returns (O [N,Hq,D], lse [N,Hq]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    off = np.asarray(offsets, dtype=np.int64)
    N, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    o = np.zeros((N, Hq, D), dtype=np.float64)
    lse = np.full((N, Hq), NEG_INF, dtype=np.float64)
    for n in range(N):
        s, e = int(off[n]), int(off[n + 1])
        if e <= s:
            continue
        for h in range(Hq):
            g = h // G
            x = scale * (k[s:e, g, :] @ q[n, h, :])           # [L]
            M = x.max()                                       # pass 1
            w = np.exp(x - M)                                 # pass 2
            Z = w.sum()
            o[n, h, :] = (w / Z) @ v[s:e, g, :]
            lse[n, h] = M + math.log(Z)
    return o, lse


def paged_rows(block_table, seq_lens, page_size: int):
    """The pool (page, row) of every key of every stream of a paged cache, by its definition: key t
    of stream n is row t % page_size of page block_table[n, t // page_size]. Returns one pair of
    index arrays (pages [L_n], rows [L_n]) per stream; only the table entries of pages that hold
    keys are read."""
    bt = np.asarray(block_table, dtype=np.int64)
    out = []
    for n, L in enumerate(np.asarray(seq_lens, dtype=np.int64)):
        t = np.arange(int(L), dtype=np.int64)
        out.append((bt[n, t // page_size], t % page_size))
    return out


def decode_attention_paged(q, k_pages, v_pages, block_table, seq_lens, scale: float):
    """Decode attention over a paged cache: the keys and values of each stream are gathered from
    the pool [num_pages, page_size, Hkv, D] in key order (``paged_rows``), and the result is
    ``decode_attention`` of that packed cache. Pool rows that hold no key are never read."""
    k_pages, v_pages = _f64(k_pages), _f64(v_pages)
    idx = paged_rows(block_table, seq_lens, k_pages.shape[1])
    ks = [k_pages[p, r] for p, r in idx]
    vs = [v_pages[p, r] for p, r in idx]
    Hkv, D = k_pages.shape[2], k_pages.shape[3]
    k = np.concatenate(ks, axis=0) if ks else np.zeros((0, Hkv, D))
    v = np.concatenate(vs, axis=0) if vs else np.zeros((0, Hkv, D))
    off = np.zeros(len(idx) + 1, dtype=np.int64)
    off[1:] = np.cumsum([len(p) for p, _ in idx])
    return decode_attention(q, k, v, off, scale)


def decode_attention_qlen(q, k, v, offsets, scale: float):
    """Decode with several query tokens per stream (a speculative or chunked step): stream n brings
    q_len new query tokens whose keys are already the newest q_len rows of its L_n cached keys, so
    token t sits at position L_n - q_len + t and sees keys 0 .. L_n - q_len + t. That is the causal
    forward with Sq = q_len and Sk = L_n under the bottom-right alignment (``visible_mask``), done
    stream by stream with ``attention_fwd``. Tokens that see no key (L_n < q_len) get O = 0 and
    lse = -inf. The decode steps are the 16-48-stream steps of "Não escreva kernels, derive-os"
    ("Aprofundamento", third paragraph); a step with more than one token per stream is this
    library's reading of the same step for speculative decoding.
    q [N, q_len, Hq, D]; packed k, v [T, Hkv, D]; offsets [N + 1].
    Returns (O [N, q_len, Hq, D], lse [N, Hq, q_len])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    off = np.asarray(offsets, dtype=np.int64)
    N, ql, Hq, D = q.shape
    o = np.zeros((N, ql, Hq, D), dtype=np.float64)
    lse = np.full((N, Hq, ql), NEG_INF, dtype=np.float64)
    for n in range(N):
        s, e = int(off[n]), int(off[n + 1])
        if e <= s:
            continue
        on, ln = attention_fwd(q[n][None], k[s:e][None], v[s:e][None], True, scale)
        o[n], lse[n] = on[0], ln[0]
    return o, lse


def decode_attention_paged_qlen(q, k_pages, v_pages, block_table, seq_lens, scale: float):
    """``decode_attention_qlen`` over a paged cache: each stream's keys and values are gathered from
    the pool in key order (``paged_rows``) first."""
    k_pages, v_pages = _f64(k_pages), _f64(v_pages)
    idx = paged_rows(block_table, seq_lens, k_pages.shape[1])
    Hkv, D = k_pages.shape[2], k_pages.shape[3]
    ks = [k_pages[p, r] for p, r in idx]
    vs = [v_pages[p, r] for p, r in idx]
    k = np.concatenate(ks, axis=0) if ks else np.zeros((0, Hkv, D))
    v = np.concatenate(vs, axis=0) if vs else np.zeros((0, Hkv, D))
    off = np.zeros(len(idx) + 1, dtype=np.int64)
    off[1:] = np.cumsum([len(p) for p, _ in idx])
    return decode_attention_qlen(q, k, v, off, scale)


# ---------------------------------------------------------------------------------------------
# The online-softmax monoid, written out for the algebra tests ("Não escreva kernels, derive-os",
# "Aprofundamento", first paragraph: the online softmax recognised as a monoid). A triple is
# (m, l, o): running max, running sum of e^{x - m}, and the unnormalised accumulator sum e^{x-m} v.
# ---------------------------------------------------------------------------------------------

def monoid_identity(D: int):
    """Identity triple (-inf, 0, 0)."""
    return (NEG_INF, 0.0, np.zeros(D, dtype=np.float64))


def monoid_leaf(x: float, v) -> tuple:
    """Triple of one key with scaled score x and value row v: (x, 1, v)."""
    return (float(x), 1.0, _f64(v).copy())


def _weight(m: float, M: float) -> float:
    # e^{m - M}, with e^{-inf - M} := 0 (also when M = -inf), so no inf - inf is formed.
    if m == NEG_INF:
        return 0.0
    return math.exp(m - M)


def monoid_merge(a: tuple, b: tuple) -> tuple:
    """(m,l,o) (+) (m',l',o') = (M, l e^{m-M} + l' e^{m'-M}, o e^{m-M} + o' e^{m'-M}), M = max."""
    m1, l1, o1 = a
    m2, l2, o2 = b
    M = max(m1, m2)
    w1 = _weight(m1, M)
    w2 = _weight(m2, M)
    return (M, l1 * w1 + l2 * w2, _f64(o1) * w1 + _f64(o2) * w2)


def monoid_finalize(t: tuple):
    """Finalise a triple to (O = o / l, lse = m + ln l); the identity gives (0, -inf)."""
    m, l, o = t
    if l == 0.0:
        return np.zeros_like(_f64(o)), NEG_INF
    return _f64(o) / l, m + math.log(l)
