"""Seeded synthetic inputs for the attention library's tests and benchmark.

This module holds no attention arithmetic: it only draws random tensors (torch CPU generator,
fp32 normal samples, then a cast), so that the CUDA path and the fp64 oracle are fed the very same
values. Each workload is named for what it is and its sizes, after the workloads the pages measure:

* ``tiny_causal``: B=1, Hq=Hkv=2, Sq=Sk=128, D=64, causal, scale 1/8, fp32 (+ the same values in bf16).
* ``block512``: one transformer block's attention at sequence 512 (B=4, H=16, D=64), the block the
  "Não escreva kernels, derive-os" page times on an RTX 3090 ("Aprofundamento", second paragraph).
* ``gqa_prefill_4k``: GQA causal prefill shaped like an 8B decoder (B=1, Hq=32, Hkv=8, S=4096,
  D=128), standing in for the Qwen3-8B decode graph of the same paragraph.
* ``decode48``: 48 decode streams (Hq=32, Hkv=8, D=128), per-stream cache lengths uniform in
  [1024, 4096], packed, the 48-stream decode step of the third paragraph.
* ``paged_from_packed``: a decode batch's caches laid out in fixed-size pages of a shuffled pool with
  a block table (a serving engine's paged cache); unused pool rows hold NaN.
* ``rising_prefill`` / ``rising_decode``: N(0,1) inputs whose keys grow along the sequence in one
  dimension (a ramp added to K[..., 0]) while each query row draws its own weight on that dimension,
  so that later key blocks raise a row's maximum score far above the earlier blocks' for some rows
  and not for others: the inputs that make an online softmax rescale its running output.
* ``packed_prefill`` / ``varlen_prefill_8x``: several sequences of different lengths packed back
  to back (cu_seqlens offsets), the multi-prompt prefill of a serving engine behind the 44k-token
  time to first token of the third paragraph; ``varlen_prefill_8x`` is 8 prompts with lengths
  uniform in [512, 4096], Hq=32, Hkv=8, D=128, causal.
* ``fp8_prefill``: the same draws quantised to E4M3 codes with one scale per tensor (amax / 448),
  the FP8 checkpoint of the third paragraph.
* ``long_prefill_44k``: one 44032-token causal prefill (Hq=32, Hkv=8, D=128) with 1 % of keys given
  a +4.0 shift on one random dimension per key, the 44k-token time-to-first-token case of the third
  paragraph. No dataset or trained weight is used anywhere.

Draw order inside one workload is fixed: Q, K, V, dO, then any structural draws (shift positions);
the decode workload draws its lengths first, because the packed K/V size depends on them. Each
workload uses its own generator seeded with 0 unless a seed is given.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass
class Prefill:
    name: str
    q: torch.Tensor          # [B, Sq, Hq, D]
    k: torch.Tensor          # [B, Sk, Hkv, D]
    v: torch.Tensor          # [B, Sk, Hkv, D]
    do: Optional[torch.Tensor]  # [B, Sq, Hq, D] or None (forward-only workload)
    causal: bool
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def dims(self):
        B, Sq, Hq, D = self.q.shape
        return dict(B=B, Hq=Hq, Hkv=self.k.shape[2], Sq=Sq, Sk=self.k.shape[1], D=D)


@dataclass
class Decode:
    name: str
    q: torch.Tensor          # [N, Hq, D]
    k: torch.Tensor          # [T, Hkv, D] packed
    v: torch.Tensor          # [T, Hkv, D] packed
    offsets: torch.Tensor    # [N + 1] int32, offsets[0] = 0
    scale: float
    meta: dict = field(default_factory=dict)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _randn(g: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def random_prefill(B, Sq, Sk, Hq, Hkv, D, causal, dtype=torch.bfloat16, seed=0, scale=None,
                   with_do=True, name=None) -> Prefill:
    """i.i.d. N(0,1) Q, K, V (and dO) of the given shape, cast to ``dtype``."""
    g = _gen(seed)
    q = _randn(g, B, Sq, Hq, D)
    k = _randn(g, B, Sk, Hkv, D)
    v = _randn(g, B, Sk, Hkv, D)
    do = _randn(g, B, Sq, Hq, D) if with_do else None
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    return Prefill(name or f"random_b{B}_sq{Sq}_sk{Sk}_hq{Hq}_hkv{Hkv}_d{D}",
                   q.to(dtype), k.to(dtype), v.to(dtype),
                   None if do is None else do.to(dtype), causal, scale)


def rising_prefill(B, Sq, Sk, Hq, Hkv, D, causal, rise_per_128=24.0, seed=0) -> Prefill:
    """N(0,1) Q, K, V, dO (bf16), then K[b, j, g, 0] += rise_per_128 * j / 128 and
    Q[b, i, h, 0] = a uniform draw in [0, 3] per row and head, before the cast.

    With scale 1/sqrt(D), a row's score for key j then grows by about a * rise_per_128 / sqrt(D) per
    128 keys: for a near 3 and the default rise that is more than 8 in base 2 (5.5 nats) per block
    at D = 128, so the row's running maximum moves at nearly every key block; rows with a near 0 keep
    their first maximum. Draw order: Q, K, V, dO, then the per-row weights.
    """
    g = _gen(seed)
    q = _randn(g, B, Sq, Hq, D)
    k = _randn(g, B, Sk, Hkv, D)
    v = _randn(g, B, Sk, Hkv, D)
    do = _randn(g, B, Sq, Hq, D)
    a = torch.rand(B, Sq, Hq, generator=g) * 3.0
    q[..., 0] = a
    k[..., 0] += rise_per_128 * torch.arange(Sk, dtype=torch.float32)[None, :, None] / 128.0
    bf = torch.bfloat16
    return Prefill(f"rising_b{B}_sq{Sq}_sk{Sk}_hq{Hq}_hkv{Hkv}_d{D}", q.to(bf), k.to(bf), v.to(bf),
                   do.to(bf), causal, 1.0 / math.sqrt(D), meta=dict(rise_per_128=rise_per_128))


@dataclass
class Packed:
    name: str
    q: torch.Tensor          # [Tq, Hq, D]
    k: torch.Tensor          # [Tk, Hkv, D]
    v: torch.Tensor          # [Tk, Hkv, D]
    do: torch.Tensor         # [Tq, Hq, D]
    cu_q: torch.Tensor       # [B + 1] int32
    cu_k: torch.Tensor       # [B + 1] int32
    causal: bool
    scale: float
    meta: dict = field(default_factory=dict)


def packed_prefill(lengths_q, lengths_k, Hq, Hkv, D, causal, seed=0, dtype=torch.bfloat16, name=None) -> Packed:
    """Sequences of the given lengths packed back to back: i.i.d. N(0,1) Q [Tq, Hq, D], K, V
    [Tk, Hkv, D] and dO (draw order Q, K, V, dO), with int32 offsets cu_q / cu_k."""
    lq = torch.as_tensor(lengths_q, dtype=torch.int64)
    lk = torch.as_tensor(lengths_k, dtype=torch.int64)
    cu_q = torch.zeros(lq.numel() + 1, dtype=torch.int64)
    cu_k = torch.zeros(lk.numel() + 1, dtype=torch.int64)
    cu_q[1:] = torch.cumsum(lq, 0)
    cu_k[1:] = torch.cumsum(lk, 0)
    g = _gen(seed)
    q = _randn(g, int(cu_q[-1]), Hq, D)
    k = _randn(g, int(cu_k[-1]), Hkv, D)
    v = _randn(g, int(cu_k[-1]), Hkv, D)
    do = _randn(g, int(cu_q[-1]), Hq, D)
    return Packed(name or f"packed_b{lq.numel()}_hq{Hq}_hkv{Hkv}_d{D}", q.to(dtype), k.to(dtype), v.to(dtype),
                  do.to(dtype), cu_q.to(torch.int32), cu_k.to(torch.int32), causal, 1.0 / math.sqrt(D),
                  meta=dict(lengths_q=lq, lengths_k=lk))


def varlen_prefill_8x(lo: int = 512, hi: int = 4096) -> Packed:
    """8 causal prompts with lengths uniform in [512, 4096] (drawn first, seed 0), packed; Hq=32,
    Hkv=8, D=128, bf16, forward and backward."""
    g = _gen(0)
    lengths = torch.randint(lo, hi + 1, (8,), generator=g)
    w = packed_prefill(lengths.tolist(), lengths.tolist(), 32, 8, 128, True, seed=1)
    w.name = f"varlen_prefill_b8_len{lo}-{hi}_hq32_hkv8_d128_causal"
    return w


@dataclass
class Fp8Prefill:
    name: str
    q: torch.Tensor          # [B, Sq, Hq, D] uint8 E4M3 codes
    k: torch.Tensor          # [B, Sk, Hkv, D] uint8
    v: torch.Tensor          # [B, Sk, Hkv, D] uint8
    q_scale: float
    k_scale: float
    v_scale: float
    causal: bool
    scale: float


def _to_e4m3(x: torch.Tensor):
    s = float(x.abs().max()) / 448.0
    s = s if s > 0 else 1.0
    return (x / s).to(torch.float8_e4m3fn).view(torch.uint8), s


def fp8_prefill(B, Sq, Sk, Hq, Hkv, D, causal, seed=0, rising=False) -> Fp8Prefill:
    """``random_prefill``'s draws (or ``rising_prefill``'s, with ``rising``) quantised to E4M3 codes,
    one scale per tensor (its largest magnitude / 448, the largest E4M3 value)."""
    w = rising_prefill(B, Sq, Sk, Hq, Hkv, D, causal, seed=seed) if rising else \
        random_prefill(B, Sq, Sk, Hq, Hkv, D, causal, dtype=torch.float32, seed=seed)
    (q, qs), (k, ks), (v, vs) = (_to_e4m3(t.float()) for t in (w.q, w.k, w.v))
    return Fp8Prefill(f"fp8_b{B}_sq{Sq}_sk{Sk}_hq{Hq}_hkv{Hkv}_d{D}", q, k, v, qs, ks, vs, causal, w.scale)


def tiny_causal(dtype=torch.float32) -> Prefill:
    """B=1, Hq=Hkv=2, Sq=Sk=128, D=64, causal, scale 1/sqrt(64); fp32 draws from seed 0."""
    w = random_prefill(1, 128, 128, 2, 2, 64, True, dtype=dtype, seed=0, scale=1.0 / 8.0)
    w.name = "tiny_causal_b1_h2_s128_d64"
    return w


def block512(causal: bool) -> Prefill:
    """Transformer-block attention: B=4, Hq=Hkv=16, S=512, D=64, bf16, forward and backward."""
    w = random_prefill(4, 512, 512, 16, 16, 64, causal, seed=0)
    w.name = f"block_b4_h16_s512_d64_{'causal' if causal else 'full'}"
    return w


def gqa_prefill_4k(reading: str = "A") -> Prefill:
    """GQA causal prefill: B=1, Hq=32, Hkv=8, S=4096, D=128, bf16, forward and backward.

    Q and K are i.i.d. N(0,1) "scaled by 1/sqrt(128)". Reading A (default): the tensors themselves
    are multiplied by 128^-1/2 after sampling and the softmax scale is still 1/sqrt(D). Reading B:
    the tensors stay N(0,1) and only the softmax scale is 1/sqrt(128).
    """
    g = _gen(0)
    B, S, Hq, Hkv, D = 1, 4096, 32, 8, 128
    q = _randn(g, B, S, Hq, D)
    k = _randn(g, B, S, Hkv, D)
    v = _randn(g, B, S, Hkv, D)
    do = _randn(g, B, S, Hq, D)
    if reading == "A":
        q = q * (1.0 / math.sqrt(128.0))
        k = k * (1.0 / math.sqrt(128.0))
    elif reading != "B":
        raise ValueError("reading must be 'A' or 'B'")
    bf = torch.bfloat16
    return Prefill(f"gqa_prefill_b1_hq32_hkv8_s4096_d128_causal_{reading}", q.to(bf), k.to(bf),
                   v.to(bf), do.to(bf), True, 1.0 / math.sqrt(D), meta=dict(reading=reading))


def long_prefill_44k(S: int = 44032, shift_fraction: float = 0.01, shift: float = 4.0) -> Prefill:
    """Long causal prefill, forward only: B=1, Sq=Sk=S (44032), Hq=32, Hkv=8, D=128, bf16.

    For each key/value head independently, round(0.01 * S) key positions are drawn without
    replacement and each gets +4.0 on one dimension drawn uniformly in [0, 128), before the bf16
    cast (4.0 is exact in bf16). The shifted positions are returned in ``meta['peaks']`` as
    a list, one int64 tensor of positions per key/value head.
    """
    g = _gen(0)
    B, Hq, Hkv, D = 1, 32, 8, 128
    q = _randn(g, B, S, Hq, D)
    k = _randn(g, B, S, Hkv, D)
    v = _randn(g, B, S, Hkv, D)
    n_peak = int(round(shift_fraction * S))
    peaks = []
    for h in range(Hkv):
        pos = torch.randperm(S, generator=g)[:n_peak]
        dim = torch.randint(0, D, (n_peak,), generator=g)
        k[0, pos, h, dim] += shift
        peaks.append(torch.sort(pos).values)
    bf = torch.bfloat16
    return Prefill(f"long_prefill_b1_s{S}_hq32_hkv8_d128_causal", q.to(bf), k.to(bf), v.to(bf),
                   None, True, 1.0 / math.sqrt(D), meta=dict(peaks=peaks))


def random_decode(N, Hq, Hkv, D, lengths, seed=0, dtype=torch.bfloat16, name=None, q_len=None) -> Decode:
    """Decode batch with the given per-stream cache lengths; K/V packed [T, Hkv, D]. Queries are
    [N, Hq, D] (one token per stream), or [N, q_len, Hq, D] when ``q_len`` is given (the newest
    q_len positions of each cache; q_len = 1 draws the same values as the 3-D form)."""
    g = _gen(seed)
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    offsets = torch.zeros(N + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(lengths, 0)
    T = int(offsets[-1])
    q = _randn(g, N, Hq, D) if q_len is None else _randn(g, N, q_len, Hq, D)
    k = _randn(g, T, Hkv, D)
    v = _randn(g, T, Hkv, D)
    return Decode(name or f"decode_n{N}_hq{Hq}_hkv{Hkv}_d{D}", q.to(dtype), k.to(dtype),
                  v.to(dtype), offsets.to(torch.int32), 1.0 / math.sqrt(D),
                  meta=dict(lengths=lengths))


def rising_decode(N, Hq, Hkv, D, lengths, rise_per_128=24.0, seed=0, q_len=None) -> Decode:
    """``random_decode`` whose cached keys grow along each stream in dimension 0
    (K[t, g, 0] += rise_per_128 * t / 128 for the stream's t-th key) and whose query rows draw their
    weight on that dimension uniformly in [0, 3]: later key blocks raise the maximum score of some
    heads far above the earlier blocks' (see ``rising_prefill``)."""
    w = random_decode(N, Hq, Hkv, D, lengths, seed=seed, dtype=torch.float32, q_len=q_len)
    g = _gen(seed + 1)
    off = w.offsets.to(torch.int64)
    k = w.k.clone()
    for n in range(N):
        s0, s1 = int(off[n]), int(off[n + 1])
        k[s0:s1, :, 0] += rise_per_128 * torch.arange(s1 - s0, dtype=torch.float32)[:, None] / 128.0
    q = w.q.clone()
    q[..., 0] = torch.rand(q.shape[:-1], generator=g) * 3.0
    bf = torch.bfloat16
    return Decode(f"rising_decode_n{N}_hq{Hq}_hkv{Hkv}_d{D}", q.to(bf), k.to(bf), w.v.to(bf), w.offsets,
                  w.scale, meta=dict(lengths=w.meta["lengths"], rise_per_128=rise_per_128))


@dataclass
class PagedCache:
    k_pages: torch.Tensor      # [num_pages, page_size, Hkv, D]
    v_pages: torch.Tensor      # [num_pages, page_size, Hkv, D]
    block_table: torch.Tensor  # [N, max_pages] int32 page ids (-1 where a stream has no page)
    seq_lens: torch.Tensor     # [N] int32


def paged_from_packed(w: Decode, page_size: int, seed: int = 0, spare_pages: int = 3,
                      fill: float = float("nan")) -> PagedCache:
    """The same caches as ``w`` laid out in pages of ``page_size`` rows in a shuffled pool.

    Stream n's key t goes to row t % page_size of its (t // page_size)-th page; the pages of all
    streams, plus ``spare_pages`` unused ones, take a random order in the pool (seeded). Pool rows
    that hold no key (the rest of a stream's last page, and the spare pages) are set to ``fill``
    (NaN by default), so that reading one shows up in the result.
    """
    g = _gen(seed)
    off = w.offsets.to(torch.int64)
    N = off.numel() - 1
    lens = off[1:] - off[:-1]
    npg = (lens + page_size - 1) // page_size
    total = int(npg.sum()) + spare_pages
    perm = torch.randperm(total, generator=g)
    Hkv, D = w.k.shape[1], w.k.shape[2]
    kp = torch.full((total, page_size, Hkv, D), fill, dtype=w.k.dtype)
    vp = torch.full((total, page_size, Hkv, D), fill, dtype=w.v.dtype)
    max_pages = max(1, int(npg.max()) if N > 0 else 1)
    table = torch.full((N, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for n in range(N):
        s0 = int(off[n])
        for i in range(int(npg[n])):
            page = int(perm[nxt])
            nxt += 1
            table[n, i] = page
            r0 = i * page_size
            r1 = min(int(lens[n]), r0 + page_size)
            kp[page, : r1 - r0] = w.k[s0 + r0: s0 + r1]
            vp[page, : r1 - r0] = w.v[s0 + r0: s0 + r1]
    return PagedCache(kp, vp, table, lens.to(torch.int32))


def decode48(N: int = 48, lo: int = 1024, hi: int = 4096) -> Decode:
    """48 decode streams, Hq=32, Hkv=8, D=128, bf16; lengths uniform in [1024, 4096] (seed 0).

    The lengths are drawn first from the workload's generator, then Q, K, V.
    """
    g = _gen(0)
    lengths = torch.randint(lo, hi + 1, (N,), generator=g)
    offsets = torch.zeros(N + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(lengths, 0)
    T = int(offsets[-1])
    Hq, Hkv, D = 32, 8, 128
    q = _randn(g, N, Hq, D)
    k = _randn(g, T, Hkv, D)
    v = _randn(g, T, Hkv, D)
    bf = torch.bfloat16
    return Decode(f"decode_n{N}_hq32_hkv8_d128_len{lo}-{hi}", q.to(bf), k.to(bf), v.to(bf),
                  offsets.to(torch.int32), 1.0 / math.sqrt(D), meta=dict(lengths=lengths))
