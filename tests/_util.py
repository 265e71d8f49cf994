"""Shared helpers for the parity tests: tolerances and tensor conversion.

Tolerances (written here once, used by every parity test):
  fp32 path: max-abs <= 1e-5 on O, lse, dQ, dK, dV.
  bf16 path: O rel-L2 <= 1e-2 and max-abs <= 2e-2; dQ, dK, dV rel-L2 <= 2e-2; lse max-abs <= 1e-3.
rel-L2 = ||x - y||_2 / ||y||_2 over the whole tensor, y the fp64 oracle.
"""
import numpy as np
import torch

F32_MAX_ABS = 1e-5
BF16_O_REL_L2 = 1e-2
BF16_O_MAX_ABS = 2e-2
BF16_GRAD_REL_L2 = 2e-2
LSE_MAX_ABS = 1e-3


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


def assert_lse(lse, lse_ref, tol=LSE_MAX_ABS):
    m = max_abs(lse, lse_ref)
    assert m <= tol, f"lse: max-abs {m:.3e}"


def assert_grad_bf16(g, g_ref, what):
    r = rel_l2(g, g_ref)
    assert r <= BF16_GRAD_REL_L2, f"{what}: rel-L2 {r:.3e}"


def assert_f32(x, ref, what):
    m = max_abs(x, ref)
    assert m <= F32_MAX_ABS, f"{what}: max-abs {m:.3e}"
