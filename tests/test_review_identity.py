"""The review prefix's end state as one weighted sum over pooled cells.

The tensor-core path computes h_init without a recurrence: scanning the prefix
[R, flip(R)] (cell r of R at positions r and 2Np-1-r) from a zero state leaves
sum_r W_r x_r B_r^T with W_r = d_r (exp(A P_r) + exp(A (2D - P_r - d_r))),
P_r the sum of d over the cells before r and D over all cells. This checks that
identity against the sequential scan, in fp64, on random cells.
"""
import numpy as np
import pytest


def _scan(d, x, Bm, A):
    h = np.zeros((x.shape[1], Bm.shape[1]))
    seq = list(range(len(d))) + list(range(len(d) - 1, -1, -1))
    for r in seq:
        h = np.exp(d[r] * A) * h + d[r] * np.outer(x[r], Bm[r])
    return h


def _weighted(d, x, Bm, A):
    P = np.concatenate([[0.0], np.cumsum(d)[:-1]])
    D = d.sum()
    W = d * (np.exp(A * P) + np.exp(A * (2 * D - P - d)))
    return np.einsum("r,rp,rn->pn", W, x, Bm)


@pytest.mark.parametrize("Np", [1, 2, 7, 64, 257])
def test_weighted_sum_equals_prefix_scan(Np):
    rng = np.random.default_rng(Np)
    d = np.log1p(np.exp(rng.standard_normal(Np) - 2.0))   # softplus: positive dt
    A = -np.exp(rng.uniform(0.0, np.log(16.0)))
    x = rng.standard_normal((Np, 5))
    Bm = rng.standard_normal((Np, 3))
    ref = _scan(d, x, Bm, A)
    got = _weighted(d, x, Bm, A)
    assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_weighted_sum_with_zero_decay_is_plain_sum():
    # A = 0: every weight is 2 d_r, the two visits of each cell
    rng = np.random.default_rng(3)
    d = rng.uniform(0.1, 1.0, 9)
    x = rng.standard_normal((9, 4))
    Bm = rng.standard_normal((9, 4))
    got = _weighted(d, x, Bm, 0.0)
    assert np.allclose(got, 2 * np.einsum("r,rp,rn->pn", d, x, Bm), rtol=1e-13, atol=0)
