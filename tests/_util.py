"""Shared helpers for the parity tests: tolerances and tensor conversion.

Tolerances (written here once, used by every parity test):
  fp32 path: max-abs <= 1e-5 on O, lse, dQ, dK, dV.
  bf16 path: O rel-L2 <= 1e-2 and max-abs <= 2e-2; dQ, dK, dV rel-L2 <= 2e-2; lse max-abs <= 1e-3.
rel-L2 = ||x - y||_2 / ||y||_2 over the whole tensor, y the fp64 oracle.

Gradients are also checked tile by tile (``assert_grad_tiles``): rel-L2 <= 2e-2 for every
(batch, head, 64-row tile), so that one wrong tile cannot hide in a whole-tensor norm. A tile whose
reference norm is below 5 % of the root-mean-square tile norm is measured against that 5 % floor
instead of its own norm (its relative error is rounding on a near-zero tile, not a wrong result).
"""
import numpy as np
import torch

F32_MAX_ABS = 1e-5
BF16_O_REL_L2 = 1e-2
BF16_O_MAX_ABS = 2e-2
BF16_GRAD_REL_L2 = 2e-2
LSE_MAX_ABS = 1e-3
# FP8 (e4m3) forward: P is rounded to e4m3 before P V. e4m3 keeps 3 mantissa bits, so a rounded P
# is off by up to 2^-4 of itself (about 3.6 % rms); O is a P-weighted mean of V rows and inherits
# errors of that relative size, averaged over the keys: about 2 % rel-L2 on N(0,1) inputs (fp64
# simulation of the rounding at S = 512 and 4096). Bound: twice that.
FP8_O_REL_L2 = 4e-2
FP8_O_MAX_ABS = 1e-1


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(x: np.ndarray, y: np.ndarray) -> float:
    den = float(np.linalg.norm(y))
    return float(np.linalg.norm(x - y)) / (den if den > 0 else 1.0)


def max_abs(x: np.ndarray, y: np.ndarray) -> float:
    # equal infinities (lse of a row that sees no key) count as exact
    both_inf = np.isinf(x) & np.isinf(y) & (np.sign(x) == np.sign(y))
    d = np.where(both_inf, 0.0, np.abs(x - y))
    return float(np.max(d)) if d.size else 0.0


def assert_o_bf16(o, o_ref, what="O"):
    r, m = rel_l2(o, o_ref), max_abs(o, o_ref)
    assert r <= BF16_O_REL_L2 and m <= BF16_O_MAX_ABS, f"{what}: rel-L2 {r:.3e}, max-abs {m:.3e}"


def assert_o_fp8(o, o_ref, what="O"):
    r, m = rel_l2(o, o_ref), max_abs(o, o_ref)
    assert r <= FP8_O_REL_L2 and m <= FP8_O_MAX_ABS, f"{what}: rel-L2 {r:.3e}, max-abs {m:.3e}"


def assert_lse(lse, lse_ref, tol=LSE_MAX_ABS):
    m = max_abs(lse, lse_ref)
    assert m <= tol, f"lse: max-abs {m:.3e}"


def assert_grad_bf16(g, g_ref, what):
    r = rel_l2(g, g_ref)
    assert r <= BF16_GRAD_REL_L2, f"{what}: rel-L2 {r:.3e}"


def assert_f32(x, ref, what):
    m = max_abs(x, ref)
    assert m <= F32_MAX_ABS, f"{what}: max-abs {m:.3e}"


TILE_FLOOR = 0.05


def tile_rel_l2(x: np.ndarray, y: np.ndarray, tile: int = 64) -> np.ndarray:
    """rel-L2 per (batch, 64-row tile, head) of [B, S, H, D] tensors, with the floor above."""
    B, S, H, D = y.shape
    nt = (S + tile - 1) // tile
    pad = nt * tile - S
    xp = np.pad(x, ((0, 0), (0, pad), (0, 0), (0, 0))).reshape(B, nt, tile, H, D)
    yp = np.pad(y, ((0, 0), (0, pad), (0, 0), (0, 0))).reshape(B, nt, tile, H, D)
    err = np.sqrt(((xp - yp) ** 2).sum(axis=(2, 4)))
    nrm = np.sqrt((yp ** 2).sum(axis=(2, 4)))
    floor = TILE_FLOOR * float(np.sqrt(np.mean(nrm ** 2)))
    return err / np.maximum(nrm, floor if floor > 0 else 1.0)


def assert_grad_tiles(g, g_ref, what, tile: int = 64):
    r = tile_rel_l2(g, g_ref, tile)
    b, t, h = np.unravel_index(int(np.argmax(r)), r.shape)
    assert float(r.max()) <= BF16_GRAD_REL_L2, \
        f"{what}: tile (batch {b}, rows {t * tile}..{t * tile + tile - 1}, head {h}) rel-L2 {float(r.max()):.3e}"


LOG2E = 1.4426950408889634


def running_max_moves(x: np.ndarray, block: int) -> np.ndarray:
    """For scaled scores x [..., Sk] (masked entries -inf), how often an online softmax that keeps
    its reference maximum until a key block's maximum exceeds it by more than 8 in base 2 has to
    move it (and rescale its running output) after the row's first key block. Counted per row."""
    xb = x * LOG2E
    Sk = xb.shape[-1]
    nb = (Sk + block - 1) // block
    pad = nb * block - Sk
    xb = np.pad(xb, [(0, 0)] * (xb.ndim - 1) + [(0, pad)], constant_values=-np.inf)
    bmax = xb.reshape(xb.shape[:-1] + (nb, block)).max(axis=-1)
    m = np.full(bmax.shape[:-1], -np.inf)
    moves = np.zeros(bmax.shape[:-1], dtype=np.int64)
    for j in range(nb):
        mx = bmax[..., j]
        move = (mx > m + 8.0) & np.isfinite(mx)
        moves += (move & np.isfinite(m)).astype(np.int64)
        m = np.where(move, mx, m)
    return moves
