"""The oracle against stored values: tests/golden/two_by_two_attention.txt holds a hand-worked case
(two queries over two keys, its closed forms and their values, with the passages they follow)."""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    vals = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    return vals


def test_two_by_two_golden():
    g = _read("two_by_two_attention.txt")
    q = np.eye(2).reshape(1, 2, 1, 2)
    k = np.eye(2).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 2, 1, 2)
    do = np.array([[1.0, 0.0], [0.0, 0.0]]).reshape(1, 2, 1, 2)
    for causal, tag in ((False, "full"), (True, "causal")):
        o, lse = oracle.attention_fwd(q, k, v, causal, 1.0)
        np.testing.assert_allclose(o[0, :, 0, :].ravel(), g[f"o_{tag}"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[0, 0], g[f"lse_{tag}"], rtol=0, atol=1e-14)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, False, 1.0)
    np.testing.assert_allclose(dq[0, :, 0, :].ravel(), g["dq_full"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk[0, :, 0, :].ravel(), g["dk_full"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv[0, :, 0, :].ravel(), g["dv_full"], rtol=0, atol=1e-14)
    # the stored values agree with their own closed forms
    a, b, t = g["a"][0], g["b"][0], g["t"][0]
    assert abs(a + b - 1.0) < 1e-15 and abs(t - 2 * a * b) < 1e-15
