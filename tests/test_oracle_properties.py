"""Property-based checks of the fp64 oracle on random tiny problems: the
invariants the definition of attention fixes (convex combination of value
rows, logsumexp bounds, invariance to a common shift of the keys, row sums of
the softmax Jacobian, linearity of the gradient in dO, homogeneity in V),
each over many shapes, scales and causal settings drawn by hypothesis."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

problems = st.tuples(
    st.integers(1, 2),          # B
    st.integers(1, 2),          # H
    st.integers(1, 9),          # N
    st.integers(1, 6),          # d
    st.booleans(),              # causal
    st.floats(0.05, 2.0),       # scale
    st.integers(0, 2 ** 31 - 1),  # data seed
)


def _data(B, H, N, d, seed, n=4):
    r = np.random.default_rng(seed)
    return [r.standard_normal((B, H, N, d)) for _ in range(n)]


def _visible(N, causal):
    """[i, j] True where key j is visible to query i."""
    m = np.ones((N, N), bool)
    return np.tril(m) if causal else m


@settings(max_examples=40, deadline=None)
@given(problems)
def test_output_is_a_convex_combination_and_lse_is_bounded(pb):
    B, H, N, d, causal, scale, seed = pb
    Q, K, V = _data(B, H, N, d, seed, 3)
    O, LSE = oracle.attention_forward(Q, K, V, scale, causal)
    vis = _visible(N, causal)
    S = scale * np.einsum("bhid,bhjd->bhij", Q, K)
    for i in range(N):
        Vi = V[:, :, vis[i], :]
        assert np.all(O[:, :, i, :] <= Vi.max(axis=2) + 1e-12)
        assert np.all(O[:, :, i, :] >= Vi.min(axis=2) - 1e-12)
        smax = S[:, :, i, vis[i]].max(axis=-1)
        assert np.all(LSE[:, :, i] >= smax - 1e-12)
        assert np.all(LSE[:, :, i] <= smax + np.log(vis[i].sum()) + 1e-12)


@settings(max_examples=40, deadline=None)
@given(problems)
def test_common_key_shift_moves_lse_only(pb):
    B, H, N, d, causal, scale, seed = pb
    Q, K, V = _data(B, H, N, d, seed, 3)
    u = np.random.default_rng(seed + 1).standard_normal(d)
    O1, L1 = oracle.attention_forward(Q, K, V, scale, causal)
    O2, L2 = oracle.attention_forward(Q, K + u, V, scale, causal)
    assert np.allclose(O1, O2, rtol=1e-9, atol=1e-11)
    assert np.allclose(L2 - L1, scale * np.einsum("bhid,d->bhi", Q, u), rtol=1e-9, atol=1e-10)


@settings(max_examples=40, deadline=None)
@given(problems)
def test_gradient_sums_and_linearity(pb):
    B, H, N, d, causal, scale, seed = pb
    Q, K, V, dO = _data(B, H, N, d, seed, 4)
    dO2 = np.random.default_rng(seed + 2).standard_normal(dO.shape)
    dQ, dK, dV = oracle.attention_backward(Q, K, V, dO, scale, causal)
    # Rows of P sum to one, rows of dS to zero.
    assert np.allclose(dV.sum(axis=2), dO.sum(axis=2), rtol=1e-9, atol=1e-10)
    assert np.allclose(dK.sum(axis=2), 0.0, atol=1e-10 * (1 + np.abs(dK).max()))
    # The gradient is linear in the upstream gradient dO.
    a = oracle.attention_backward(Q, K, V, dO + 2.5 * dO2, scale, causal)
    b = oracle.attention_backward(Q, K, V, dO2, scale, causal)
    for g0, gab, gb in zip((dQ, dK, dV), a, b):
        assert np.allclose(gab, g0 + 2.5 * gb, rtol=1e-9, atol=1e-10 * (1 + np.abs(gab).max()))


@settings(max_examples=30, deadline=None)
@given(problems, st.floats(-3.0, 3.0).filter(lambda c: abs(c) > 1e-3))
def test_output_and_value_gradient_are_homogeneous_in_v(pb, c):
    B, H, N, d, causal, scale, seed = pb
    Q, K, V, dO = _data(B, H, N, d, seed, 4)
    O1, L1 = oracle.attention_forward(Q, K, V, scale, causal)
    O2, L2 = oracle.attention_forward(Q, K, c * V, scale, causal)
    assert np.allclose(O2, c * O1, rtol=1e-9, atol=1e-11)
    assert np.allclose(L1, L2, rtol=0, atol=1e-12)
    _, _, dV1 = oracle.attention_backward(Q, K, V, dO, scale, causal)
    _, _, dV2 = oracle.attention_backward(Q, K, c * V, dO, scale, causal)
    assert np.allclose(dV1, dV2, rtol=1e-9, atol=1e-11)  # dV does not depend on V
