"""Pins for the fp64 oracle: closed forms, invariants, library special cases,
brute force and finite differences -- facts fixed by the pages and by
mathematics, not by the oracle itself.

Passages pinned (unite.ai, "Flash Attention: Revolutionizing Transformer
Efficiency"): the standard-attention definition; "The math behind Flash
Attention" item 1 (safe softmax) and item 2 (merge of partial softmaxes);
downcodes.com "triton transformer", usage section (the causal flag, read as
top-left aligned: query i sees keys j <= i).

Every pin is a function ``pin_*(lib)`` so that ``test_mutants_are_caught`` can
run the whole battery against deliberately broken copies of the oracle.
"""
import math
import os
import shutil
import tempfile

import numpy as np
import pytest
import scipy.special
import torch

import oracle

RTOL = 1e-11


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol=RTOL):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"max abs err {err:.3e} > {tol:.1e} * {scale:.3e}"


# ----------------------------------------------------------------------------
# Forward pins
# ----------------------------------------------------------------------------

def pin_single_key(lib):
    """N = 1: the only key gets weight 1, so O = V[0] and LSE = scale <q, k0>."""
    r = _rng(1)
    Q, K, V = (r.standard_normal((2, 3, 1, 5)) for _ in range(3))
    for causal in (False, True):
        O, LSE = oracle.attention_forward(Q, K, V, 0.37, causal, lib=lib)
        _close(O, V)
        _close(LSE, 0.37 * np.sum(Q * K, axis=-1))


def pin_causal_first_row(lib):
    """Causal row 0 sees key 0 only: O[0] = V[0], LSE[0] = scale <q0, k0>."""
    r = _rng(2)
    Q, K, V = (r.standard_normal((1, 2, 7, 4)) for _ in range(3))
    O, LSE = oracle.attention_forward(Q, K, V, 0.5, True, lib=lib)
    _close(O[:, :, 0], V[:, :, 0])
    _close(LSE[:, :, 0], 0.5 * np.sum(Q[:, :, 0] * K[:, :, 0], axis=-1))


def pin_identical_keys(lib):
    """All keys equal: uniform weights.  Non-causal O_i = mean_j V_j,
    LSE_i = scale <q_i, k> + ln N; causal O_i = mean_{j<=i} V_j,
    LSE_i = scale <q_i, k> + ln(i + 1)."""
    r = _rng(3)
    B, H, N, d = 1, 2, 9, 6
    Q = r.standard_normal((B, H, N, d))
    k = r.standard_normal((B, H, 1, d))
    K = np.repeat(k, N, axis=2)
    V = r.standard_normal((B, H, N, d))
    qk = 0.3 * np.sum(Q * k, axis=-1)
    O, LSE = oracle.attention_forward(Q, K, V, 0.3, False, lib=lib)
    _close(O, np.broadcast_to(V.mean(axis=2, keepdims=True), O.shape))
    _close(LSE, qk + math.log(N))
    O, LSE = oracle.attention_forward(Q, K, V, 0.3, True, lib=lib)
    counts = np.arange(1, N + 1, dtype=np.float64)
    _close(O, np.cumsum(V, axis=2) / counts[None, None, :, None])
    _close(LSE, qk + np.log(counts)[None, None, :])


def pin_one_hot_values_are_probabilities(lib):
    """With V = identity (N <= d) row i of O is the attention distribution:
    non-negative, summing to 1; causal rows put no weight on keys j > i."""
    r = _rng(4)
    N, d = 6, 8
    Q = r.standard_normal((1, 1, N, d)) * 2
    K = r.standard_normal((1, 1, N, d)) * 2
    V = np.zeros((1, 1, N, d))
    V[0, 0, np.arange(N), np.arange(N)] = 1.0
    for causal in (False, True):
        O, _ = oracle.attention_forward(Q, K, V, 0.8, causal, lib=lib)
        P = O[0, 0, :, :N]
        assert np.all(P >= 0)
        _close(P.sum(axis=1), np.ones(N))
        _close(O[0, 0, :, N:], np.zeros((N, d - N)))
        if causal:
            assert np.all(np.triu(P, k=1) == 0.0)
        else:
            assert np.all(P > 0)


def pin_convexity(lib):
    """O_i is a convex combination of value rows: min_j V <= O_i <= max_j V."""
    r = _rng(5)
    Q, K, V = (r.standard_normal((2, 2, 17, 3)) * 3 for _ in range(3))
    O, _ = oracle.attention_forward(Q, K, V, 1.0, False, lib=lib)
    lo = V.min(axis=2, keepdims=True) - 1e-12
    hi = V.max(axis=2, keepdims=True) + 1e-12
    assert np.all(O >= lo) and np.all(O <= hi)


def pin_vs_torch_sdpa(lib):
    """Library special case: torch's SDPA (CPU, fp64) and torch.logsumexp."""
    r = _rng(6)
    for (B, H, N, d, causal, scale) in [(2, 3, 13, 8, False, 0.35), (1, 2, 21, 16, True, 0.25),
                                        (1, 1, 3, 64, True, 0.125)]:
        Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
        O, LSE = oracle.attention_forward(Q, K, V, scale, causal, lib=lib)
        tq, tk, tv = (torch.from_numpy(x) for x in (Q, K, V))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                               scale=scale)
        s = scale * tq @ tk.transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        _close(O, ref.numpy())
        _close(LSE, torch.logsumexp(s, dim=-1).numpy())


def pin_bruteforce(lib):
    """Pure-Python loops over a tiny head, straight from the definition."""
    r = _rng(7)
    B, H, N, d = 1, 2, 5, 3
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    scale = 0.7
    for causal in (False, True):
        O, LSE = oracle.attention_forward(Q, K, V, scale, causal, lib=lib)
        for h in range(H):
            for i in range(N):
                keys = [j for j in range(N) if not (causal and j > i)]
                s = [scale * sum(Q[0, h, i, c] * K[0, h, j, c] for c in range(d)) for j in keys]
                z = sum(math.exp(x) for x in s)
                assert abs(LSE[0, h, i] - math.log(z)) < 1e-12
                for c in range(d):
                    o = sum(math.exp(x) / z * V[0, h, j, c] for x, j in zip(s, keys))
                    assert abs(O[0, h, i, c] - o) < 1e-12


def pin_shift_invariance(lib):
    """Adding u to every key leaves O unchanged and shifts LSE_i by scale <q_i, u>."""
    r = _rng(8)
    Q, K, V = (r.standard_normal((1, 2, 11, 4)) for _ in range(3))
    u = r.standard_normal((1, 2, 1, 4))
    for causal in (False, True):
        O0, L0 = oracle.attention_forward(Q, K, V, 0.6, causal, lib=lib)
        O1, L1 = oracle.attention_forward(Q, K + u, V, 0.6, causal, lib=lib)
        _close(O1, O0)
        _close(L1, L0 + 0.6 * np.sum(Q * u, axis=-1))


def pin_permutation_invariance(lib):
    """Non-causal: permuting key/value rows jointly changes nothing."""
    r = _rng(9)
    Q, K, V = (r.standard_normal((2, 1, 12, 5)) for _ in range(3))
    perm = r.permutation(12)
    O0, L0 = oracle.attention_forward(Q, K, V, 0.45, False, lib=lib)
    O1, L1 = oracle.attention_forward(Q, K[:, :, perm], V[:, :, perm], 0.45, False, lib=lib)
    _close(O1, O0)
    _close(L1, L0)


def pin_rows_match_full(lib):
    """The sampled-rows entry returns exactly the rows of the full forward."""
    r = _rng(10)
    B, H, N, d = 2, 2, 10, 4
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    rows = np.array([0, 9, 13, 27, 39, 21], np.int64)
    for causal in (False, True):
        O, L = oracle.attention_forward(Q, K, V, 0.5, causal, lib=lib)
        Or, Lr = oracle.attention_forward_rows(Q, K, V, 0.5, causal, rows, lib=lib)
        np.testing.assert_array_equal(Or, O.reshape(-1, d)[rows])
        np.testing.assert_array_equal(Lr, L.reshape(-1)[rows])


def pin_bf16_widening(lib):
    """bf16 bit patterns are widened exactly: same result as the fp64 path on
    the same (bf16-representable) values."""
    g = torch.Generator().manual_seed(11)
    t = [torch.randn(1, 2, 9, 8, generator=g).to(torch.bfloat16) for _ in range(3)]
    bits = [x.view(torch.int16).numpy().view(np.uint16) for x in t]
    f64 = [x.double().numpy() for x in t]
    for causal in (False, True):
        Ob, Lb = oracle.attention_forward(*bits, 0.3, causal, lib=lib)
        Of, Lf = oracle.attention_forward(*f64, 0.3, causal, lib=lib)
        np.testing.assert_array_equal(Ob, Of)
        np.testing.assert_array_equal(Lb, Lf)


# ----------------------------------------------------------------------------
# Merge (online softmax) pins
# ----------------------------------------------------------------------------

def _split_points(r, n, nblocks):
    cuts = np.sort(r.choice(np.arange(1, n), size=nblocks - 1, replace=False))
    return np.split(np.arange(n), cuts)


def pin_merge_equals_full_softmax(lib):
    """Splitting the keys into blocks and folding the partials with the merge
    rule gives the softmax over all keys (checked against scipy)."""
    r = _rng(12)
    n, d = 40, 6
    for trial in range(5):
        s = r.standard_normal(n) * (1 + 4 * trial)
        V = r.standard_normal((n, d))
        w = scipy.special.softmax(s)
        full_o, full_lse = w @ V, scipy.special.logsumexp(s)
        m, l, o = oracle.softmax_partial(s, V, lib=lib)
        _close(o, full_o)
        _close(m + math.log(l), full_lse)
        blocks = _split_points(r, n, 2 + trial)
        acc = oracle.softmax_partial(s[blocks[0]], V[blocks[0]], lib=lib)
        for b in blocks[1:]:
            acc = oracle.softmax_merge(acc, oracle.softmax_partial(s[b], V[b], lib=lib), lib=lib)
        _close(acc[2], full_o)
        _close(acc[0] + math.log(acc[1]), full_lse)


def pin_merge_is_symmetric(lib):
    """softmax(x U y) does not depend on which block comes first."""
    r = _rng(13)
    s, V = r.standard_normal(20) * 3, r.standard_normal((20, 4))
    px = oracle.softmax_partial(s[:7], V[:7], lib=lib)
    py = oracle.softmax_partial(s[7:], V[7:], lib=lib)
    a, b = oracle.softmax_merge(px, py, lib=lib), oracle.softmax_merge(py, px, lib=lib)
    _close(a[2], b[2])
    _close(a[0] + math.log(a[1]), b[0] + math.log(b[1]))


def pin_merge_extreme_ranges(lib):
    """Block maxima 1800 apart: the merge must rescale by exp(m_x - m) with
    m the larger maximum (item 1's reason for subtracting the max), else
    exp overflows."""
    r = _rng(19)
    s = np.concatenate([r.uniform(-905, -895, 10), r.uniform(895, 905, 10)])
    V = r.standard_normal((20, 3))
    for first, second in ((slice(0, 10), slice(10, 20)), (slice(10, 20), slice(0, 10))):
        acc = oracle.softmax_merge(oracle.softmax_partial(s[first], V[first], lib=lib),
                                   oracle.softmax_partial(s[second], V[second], lib=lib),
                                   lib=lib)
        assert np.all(np.isfinite(acc[2])) and math.isfinite(acc[0] + math.log(acc[1]))
        _close(acc[2], scipy.special.softmax(s) @ V)
        _close(acc[0] + math.log(acc[1]), scipy.special.logsumexp(s))


def pin_forward_extreme_scores(lib):
    """Scores of magnitude ~1e3 stay finite (safe softmax) and match torch."""
    r = _rng(20)
    Q, K, V = (r.standard_normal((1, 2, 10, 4)) for _ in range(3))
    for causal in (False, True):
        O, LSE = oracle.attention_forward(Q * 30, K * 30, V, 1.0, causal, lib=lib)
        tq, tk, tv = (torch.from_numpy(x) for x in (Q * 30, K * 30, V))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                               scale=1.0)
        s = tq @ tk.transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(10, 10, dtype=torch.bool).triu(1), float("-inf"))
        assert np.all(np.isfinite(O)) and np.all(np.isfinite(LSE))
        _close(O, ref.numpy())
        _close(LSE, torch.logsumexp(s, dim=-1).numpy())


def test_printed_blockwise_update_is_wrong_for_several_blocks():
    """The page's tiled listing divides an already-normalised O by the new
    row sum again.  That recurrence equals softmax only with one key block;
    with two or more it drifts -- which is why the oracle does not follow it."""
    r = _rng(14)
    n, d = 64, 4
    s, V = r.standard_normal(n) * 2, r.standard_normal((n, d))
    exact = scipy.special.softmax(s) @ V

    def printed(block):
        O, L, M = np.zeros(d), 0.0, -np.inf
        for j in range(0, n, block):
            sb, vb = s[j:j + block], V[j:j + block]
            m_new = max(M, sb.max())
            e, a = np.exp(sb - m_new), math.exp(M - m_new)
            L_new = a * L + e.sum()
            O = (a * O + e @ vb) / L_new
            L, M = L_new, m_new
        return O

    np.testing.assert_allclose(printed(n), exact, rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(printed(16) - exact)) > 1e-3


# ----------------------------------------------------------------------------
# Backward pins
# ----------------------------------------------------------------------------

def _fwd_obj(lib, Q, K, V, dO, scale, causal):
    O, _ = oracle.attention_forward(Q, K, V, scale, causal, lib=lib)
    return float(np.sum(O * dO))


def pin_backward_finite_differences(lib):
    """Central differences (h = 1e-6) of f = <O, dO> in every coordinate."""
    r = _rng(15)
    B, H, N, d, scale = 1, 2, 5, 3, 0.8
    Q, K, V, dO = (r.standard_normal((B, H, N, d)) for _ in range(4))
    h = 1e-6
    for causal in (False, True):
        grads = oracle.attention_backward(Q, K, V, dO, scale, causal, lib=lib)
        for which, g in enumerate(grads):
            num = np.zeros_like(g)
            for idx in np.ndindex(*g.shape):
                args = [Q.copy(), K.copy(), V.copy()]
                args[which][idx] += h
                fp = _fwd_obj(lib, *args, dO, scale, causal)
                args[which][idx] -= 2 * h
                fm = _fwd_obj(lib, *args, dO, scale, causal)
                num[idx] = (fp - fm) / (2 * h)
            np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7)


def pin_backward_vs_autograd(lib):
    """Library special case: torch.autograd (fp64) through the naive formula."""
    r = _rng(16)
    for (B, H, N, d, causal, scale) in [(1, 2, 9, 8, False, 0.3), (2, 1, 12, 4, True, 0.5)]:
        Q, K, V, dO = (r.standard_normal((B, H, N, d)) for _ in range(4))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
        s = scale * tq @ tk.transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        out = torch.softmax(s, dim=-1) @ tv
        out.backward(torch.from_numpy(dO))
        dQ, dK, dV = oracle.attention_backward(Q, K, V, dO, scale, causal, lib=lib)
        _close(dQ, tq.grad.numpy())
        _close(dK, tk.grad.numpy())
        _close(dV, tv.grad.numpy())


def pin_backward_invariants(lib):
    """Rows of dS sum to zero, so sum_j dK_j = 0; and sum_j dV_j = sum_i dO_i
    because every row of P sums to one."""
    r = _rng(17)
    Q, K, V, dO = (r.standard_normal((2, 2, 15, 6)) for _ in range(4))
    for causal in (False, True):
        dQ, dK, dV = oracle.attention_backward(Q, K, V, dO, 0.4, causal, lib=lib)
        _close(dK.sum(axis=2), np.zeros((2, 2, 6)), tol=1e-11)
        _close(dV.sum(axis=2), dO.sum(axis=2))


def pin_backward_single_key(lib):
    """N = 1: O = V, so dV = dO and dQ = dK = 0."""
    r = _rng(18)
    Q, K, V, dO = (r.standard_normal((1, 2, 1, 4)) for _ in range(4))
    dQ, dK, dV = oracle.attention_backward(Q, K, V, dO, 0.5, True, lib=lib)
    _close(dV, dO)
    _close(dQ, np.zeros_like(dQ))
    _close(dK, np.zeros_like(dK))


# ----------------------------------------------------------------------------
# Grouped-query attention pins (unite.ai page, "FlashAttention-2" item 3)
# ----------------------------------------------------------------------------

def pin_gqa_forward_vs_torch(lib):
    """Library special case: torch SDPA (fp64) with enable_gqa; and Hkv = H is
    plain multi-head attention."""
    r = _rng(21)
    for (B, H, Hkv, N, d, causal) in [(2, 6, 2, 11, 8, False), (1, 4, 1, 9, 4, True),
                                      (1, 4, 4, 7, 4, True)]:
        Q = r.standard_normal((B, H, N, d))
        K, V = (r.standard_normal((B, Hkv, N, d)) for _ in range(2))
        O, LSE = oracle.attention_forward_gqa(Q, K, V, 0.4, causal, lib=lib)
        ref = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(x) for x in (Q, K, V)), is_causal=causal, scale=0.4,
            enable_gqa=True)
        _close(O, ref.numpy())
        Kr = np.repeat(K, H // Hkv, axis=1)
        s = 0.4 * torch.from_numpy(Q) @ torch.from_numpy(Kr).transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        _close(LSE, torch.logsumexp(s, dim=-1).numpy())


def pin_gqa_backward_vs_autograd(lib):
    """torch.autograd (fp64) through K/V repeated to every query head: the
    gradient of a shared K/V head sums over its group."""
    r = _rng(22)
    for (B, H, Hkv, N, d, causal) in [(1, 6, 2, 9, 4, True), (2, 4, 1, 7, 8, False)]:
        Q, dO = (r.standard_normal((B, H, N, d)) for _ in range(2))
        K, V = (r.standard_normal((B, Hkv, N, d)) for _ in range(2))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
        G = H // Hkv
        s = 0.5 * tq @ tk.repeat_interleave(G, dim=1).transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        (torch.softmax(s, dim=-1) @ tv.repeat_interleave(G, dim=1)).backward(torch.from_numpy(dO))
        dQ, dK, dV = oracle.attention_backward_gqa(Q, K, V, dO, 0.5, causal, lib=lib)
        _close(dQ, tq.grad.numpy())
        _close(dK, tk.grad.numpy())
        _close(dV, tv.grad.numpy())


# ----------------------------------------------------------------------------
# Padding pins (downcodes.com "triton transformer", BERT example: padding mask)
# ----------------------------------------------------------------------------

def _key_mask(seqlens, N, causal):
    """[B, 1, N, N] boolean: query i may attend key j."""
    B = len(seqlens)
    j = torch.arange(N)
    m = (j[None, :] < torch.tensor(seqlens)[:, None])[:, None, None, :].expand(B, 1, N, N)
    if causal:
        m = m & torch.ones(N, N, dtype=torch.bool).tril()
    return m


def pin_padding_forward_vs_torch(lib):
    """Real rows: torch SDPA (fp64) with a boolean key-padding mask; padding
    rows: O = 0, LSE = 0."""
    r = _rng(23)
    for (B, H, Hkv, N, d, causal, sl) in [(3, 2, 2, 9, 4, False, [9, 5, 1]),
                                          (2, 4, 2, 12, 8, True, [7, 12])]:
        Q = r.standard_normal((B, H, N, d))
        K, V = (r.standard_normal((B, Hkv, N, d)) for _ in range(2))
        O, LSE = oracle.attention_forward_varlen(Q, K, V, sl, 0.6, causal, lib=lib)
        G = H // Hkv
        tq = torch.from_numpy(Q)
        tk = torch.from_numpy(np.repeat(K, G, axis=1))
        tv = torch.from_numpy(np.repeat(V, G, axis=1))
        mask = _key_mask(sl, N, causal)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask,
                                                               scale=0.6)
        s = (0.6 * tq @ tk.transpose(-1, -2)).masked_fill(~mask, float("-inf"))
        for b, n in enumerate(sl):
            _close(O[b, :, :n], ref[b, :, :n].numpy())
            _close(LSE[b, :, :n], torch.logsumexp(s[b, :, :n], dim=-1).numpy())
            assert np.all(O[b, :, n:] == 0.0) and np.all(LSE[b, :, n:] == 0.0)


def pin_padding_backward_vs_autograd(lib):
    """torch.autograd (fp64) on real rows only: padding queries contribute
    nothing, padding tokens get zero gradients."""
    r = _rng(24)
    for (B, H, Hkv, N, d, causal, sl) in [(2, 2, 1, 10, 4, True, [6, 10]),
                                          (2, 2, 2, 8, 4, False, [3, 8])]:
        Q, dO = (r.standard_normal((B, H, N, d)) for _ in range(2))
        K, V = (r.standard_normal((B, Hkv, N, d)) for _ in range(2))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
        G = H // Hkv
        mask = _key_mask(sl, N, causal)
        s = (0.5 * tq @ tk.repeat_interleave(G, dim=1).transpose(-1, -2)).masked_fill(
            ~mask, float("-inf"))
        out = torch.softmax(s, dim=-1) @ tv.repeat_interleave(G, dim=1)
        real = (torch.arange(N)[None, :] < torch.tensor(sl)[:, None])[:, None, :, None]
        (out * torch.from_numpy(dO) * real).sum().backward()
        dQ, dK, dV = oracle.attention_backward_varlen(Q, K, V, dO, sl, 0.5, causal, lib=lib)
        _close(dQ, (tq.grad * real).numpy())
        _close(dK, tk.grad.numpy())
        _close(dV, tv.grad.numpy())


# ----------------------------------------------------------------------------
# Dropout pins (downcodes.com "triton transformer", usage section:
# attn_dropout).  The generator is Philox-4x32 (Salmon, Moraes, Dror, Shaw,
# "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) with 7 rounds.
# ----------------------------------------------------------------------------

# Known-answer vectors published with the generator (Random123 distribution,
# kat_vectors, philox4x32 with 10 rounds): (counter, key, output).
PHILOX_KAT = [
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


def _philox_py(ctr, key, rounds=10):
    """Philox-4x32 written out from the SC'11 definition (independent of the C)."""
    c, k = list(ctr), list(key)
    for _ in range(rounds):
        a, b = 0xD2511F53 * c[0], 0xCD9E8D57 * c[2]
        c = [((b >> 32) ^ c[1] ^ k[0]) & 0xFFFFFFFF, b & 0xFFFFFFFF,
             ((a >> 32) ^ c[3] ^ k[1]) & 0xFFFFFFFF, a & 0xFFFFFFFF]
        k = [(k[0] + 0x9E3779B9) & 0xFFFFFFFF, (k[1] + 0xBB67AE85) & 0xFFFFFFFF]
    return tuple(c)


def pin_philox_known_answers(lib):
    for ctr, key, want in PHILOX_KAT:
        assert _philox_py(ctr, key) == want
        assert tuple(int(x) for x in oracle.philox4x32_10(ctr, key, lib=lib)) == want


def pin_philox_seven_rounds(lib):
    """The dropout generator is the same round function stopped after 7
    rounds: the oracle's 7-round output equals the Python definition (pinned to
    the published 10-round vectors above) run for 7 rounds, on the vectors'
    counters and on random ones, and differs from the 10-round output."""
    r = np.random.default_rng(34)
    cases = [(c, k) for c, k, _ in PHILOX_KAT] + [
        (tuple(int(x) for x in r.integers(0, 2 ** 32, 4)), tuple(int(x) for x in r.integers(0, 2 ** 32, 2)))
        for _ in range(20)]
    for ctr, key in cases:
        got = tuple(int(x) for x in oracle.philox4x32_7(ctr, key, lib=lib))
        assert got == _philox_py(ctr, key, rounds=7)
        assert got != _philox_py(ctr, key, rounds=10)


def _keep_threshold(p):
    """t = floor((1 - p) 2^8 + 1/2): keys are kept with probability t / 2^8."""
    return math.floor((1.0 - p) * 2.0 ** 8 + 0.5)


def _keep_byte(words, j):
    """The 8-bit number of key j in a Philox output: word (j%16)//4, byte
    2 (j%2) + (j%4)//2 (keys 4w..4w+3 in bytes 0, 2, 1, 3 of word w)."""
    return (words[(j % 16) // 4] >> (8 * (2 * (j % 2) + (j % 4) // 2))) & 0xFF


def pin_dropout_mask_convention(lib):
    """Keep mask = the stated counter layout (j/16, i, b*H+h, offset), key =
    seed halves, 7 rounds, the stated byte of key j below t, evaluated
    independently."""
    assert _philox_py(*PHILOX_KAT[2][:2]) == PHILOX_KAT[2][2]
    B, H, N, p, seed, offset = 2, 3, 37, 0.3, 0x0123456789ABCDEF, 7
    m = oracle.dropout_keep_mask(B, H, N, p, seed, offset, lib=lib)
    t = _keep_threshold(p)
    key = (seed & 0xFFFFFFFF, seed >> 32)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                for j in range(N):
                    w = _philox_py((j // 16, i, b * H + h, offset), key, rounds=7)
                    assert m[b, h, i, j] == (_keep_byte(w, j) < t), (b, h, i, j)


def pin_dropout_keep_rate(lib):
    """Each element is kept with probability t / 2^8 (within 2^-9 of 1 - p):
    the kept fraction of 2^20 draws is within 6 standard deviations; p = 0
    and p < 2^-9 keep everything; p too close to 1 (t = 0) is rejected."""
    for p in (0.1, 0.5, 0.9, 0.123456):
        q = _keep_threshold(p) / 2.0 ** 8
        assert abs(q - (1 - p)) <= 2.0 ** -9
        m = oracle.dropout_keep_mask(1, 4, 512, p, 99, 3, lib=lib)
        n = m.size
        assert abs(m.mean() - q) <= 6 * math.sqrt(q * (1 - q) / n), (p, m.mean())
    assert oracle.dropout_keep_mask(1, 1, 64, 0.0, 5, lib=lib).all()
    assert oracle.dropout_keep_mask(1, 1, 64, 1e-3, 5, lib=lib).all()
    with pytest.raises(RuntimeError):
        oracle.dropout_keep_mask(1, 1, 8, 1.0 - 2.0 ** -10, 5, lib=lib)


def pin_dropout_zero_is_plain_attention(lib):
    r = _rng(31)
    Q, K, V = (r.standard_normal((2, 2, 9, 4)) for _ in range(3))
    O0, L0 = oracle.attention_forward(Q, K, V, 0.5, True, lib=lib)
    O, L = oracle.attention_forward_dropout(Q, K, V, 0.5, True, 0.0, 1234, lib=lib)
    assert np.array_equal(O, O0) and np.array_equal(L, L0)


def _dropout_torch(Q, K, V, z, p, scale, causal, seqlens):
    """(softmax(scale Q K^T, masked) * z / q) V in fp64 torch, with grads
    (q = t / 2^8, the keep probability)."""
    B, H, N, _ = Q.shape
    G = H // K.shape[1]
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    mask = _key_mask(seqlens if seqlens is not None else [N] * B, N, causal)
    s = (scale * tq @ tk.repeat_interleave(G, dim=1).transpose(-1, -2)).masked_fill(
        ~mask, float("-inf"))
    P = torch.softmax(s, dim=-1)
    q = _keep_threshold(p) / 2.0 ** 8
    out = (P * torch.from_numpy(z.astype(np.float64)) / q) @ tv.repeat_interleave(G, dim=1)
    return out, torch.logsumexp(s, dim=-1), (tq, tk, tv)


DROPOUT_CASES = [(2, 2, 1, 9, 4, True, [9, 6], 0.25), (1, 3, 3, 13, 8, False, None, 0.6),
                 (1, 4, 2, 10, 4, False, [7], 0.1)]


def pin_dropout_forward_vs_torch(lib):
    """O equals the explicit formula with the mask; LSE is the undropped one."""
    r = _rng(32)
    for (B, H, Hkv, N, d, causal, sl, p) in DROPOUT_CASES:
        Q = r.standard_normal((B, H, N, d))
        K, V = (r.standard_normal((B, Hkv, N, d)) for _ in range(2))
        seed, offset = 1000 + N, 5
        O, LSE = oracle.attention_forward_dropout(Q, K, V, 0.7, causal, p, seed, offset,
                                                  seqlens=sl, lib=lib)
        z = oracle.dropout_keep_mask(B, H, N, p, seed, offset, lib=lib)
        assert 0 < z.mean() < 1
        ref, lse, _ = _dropout_torch(Q, K, V, z, p, 0.7, causal, sl)
        for b in range(B):
            n = N if sl is None else sl[b]
            _close(O[b, :, :n], ref[b, :, :n].detach().numpy())
            _close(LSE[b, :, :n], lse[b, :, :n].detach().numpy())


def pin_dropout_backward_vs_autograd(lib):
    r = _rng(33)
    for (B, H, Hkv, N, d, causal, sl, p) in DROPOUT_CASES:
        Q, dO = (r.standard_normal((B, H, N, d)) for _ in range(2))
        K, V = (r.standard_normal((B, Hkv, N, d)) for _ in range(2))
        seed, offset = 77 + N, 2
        z = oracle.dropout_keep_mask(B, H, N, p, seed, offset, lib=lib)
        out, _, (tq, tk, tv) = _dropout_torch(Q, K, V, z, p, 0.7, causal, sl)
        lens = [N] * B if sl is None else sl
        real = (torch.arange(N)[None, :] < torch.tensor(lens)[:, None])[:, None, :, None]
        (out * torch.from_numpy(dO) * real).sum().backward()
        dQ, dK, dV = oracle.attention_backward_dropout(Q, K, V, dO, 0.7, causal, p, seed, offset,
                                                       seqlens=sl, lib=lib)
        _close(dQ, (tq.grad * real).numpy())
        _close(dK, tk.grad.numpy())
        _close(dV, tv.grad.numpy())


def pin_dropout_is_unbiased(lib):
    """Inverted dropout leaves O unchanged in expectation: the mean over 1500
    seeds is within 6 standard errors of the undropped O."""
    r = _rng(34)
    Q, K, V = (r.standard_normal((1, 1, 6, 3)) for _ in range(3))
    O0, _ = oracle.attention_forward(Q, K, V, 0.8, False, lib=lib)
    runs = np.stack([oracle.attention_forward_dropout(Q, K, V, 0.8, False, 0.4, sd, lib=lib)[0]
                     for sd in range(1500)])
    se = runs.std(axis=0) / math.sqrt(len(runs))
    assert np.all(np.abs(runs.mean(axis=0) - O0) <= 6 * se + 1e-12)


def pin_dropout_rows_and_heads_match_full(lib):
    """The sampled variants used at full sizes are bitwise the full oracle:
    dropout forward rows (GQA, causal) and the backward restricted to heads."""
    r = _rng(35)
    B, H, Hkv, N, d = 2, 4, 2, 11, 4
    Q = r.standard_normal((B, H, N, d))
    K, V = (r.standard_normal((B, Hkv, N, d)) for _ in range(2))
    for p_drop in (0.3, 0.0):
        O, L = oracle.attention_forward_dropout(Q, K, V, 0.6, True, p_drop, 42, 3, lib=lib)
        rows = np.array([0, 5, N - 1, N + 2, 3 * N + 7, B * H * N - 1])
        Or, Lr = oracle.attention_forward_dropout_rows(Q, K, V, 0.6, True, p_drop, 42, 3, rows,
                                                       lib=lib)
        assert np.array_equal(Or, O.reshape(-1, d)[rows]) and np.array_equal(Lr, L.reshape(-1)[rows])
    Q, dO, K, V = (r.standard_normal((B, H, N, d)) for _ in range(4))
    dQ, dK, dV = oracle.attention_backward_dropout(Q, K, V, dO, 0.6, False, 0.25, 7, 1, lib=lib)
    heads = [5, 2]
    hq, hk, hv = oracle.attention_backward_dropout_heads(Q, K, V, dO, 0.6, False, 0.25, 7, 1, heads,
                                                         lib=lib)
    for t, f in ((hq, dQ), (hk, dK), (hv, dV)):
        t2, f2 = t.reshape(B * H, N, d), f.reshape(B * H, N, d)
        for bh in range(B * H):
            if bh in heads:
                assert np.array_equal(t2[bh], f2[bh]), bh
            else:
                assert not t2[bh].any(), bh
    with pytest.raises(RuntimeError):
        oracle.attention_backward_dropout_heads(Q, K, V, dO, 0.6, False, 0.25, 7, 1, [2, 2], lib=lib)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle.load())


def test_bad_arguments_are_rejected():
    lib = oracle.load()
    z = np.zeros((1, 1, 0, 4))
    with pytest.raises(RuntimeError):
        oracle.attention_forward(z, z, z, 1.0, False, lib=lib)
    Q = np.zeros((1, 1, 3, 4))
    with pytest.raises(RuntimeError):
        oracle.attention_forward_rows(Q, Q, Q, 1.0, False, np.array([3]), lib=lib)
    for p in (1.0, -0.1, float("nan")):
        with pytest.raises(RuntimeError):
            oracle.attention_forward_dropout(Q, Q, Q, 1.0, False, p, 1, lib=lib)
        with pytest.raises(RuntimeError):
            oracle.dropout_keep_mask(1, 1, 3, p, 1, lib=lib)


def test_golden_regression():
    """Values written by tests/golden/make_golden.py (which calls only the
    oracle): guards against accidental edits, not a pin to the pages."""
    import json
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_small.json")
    with open(path) as f:
        gold = json.load(f)
    for case in gold["cases"]:
        from io_aware_exact_31_b200.workloads import make_inputs, bf16_bits
        x = make_inputs(case["B"], case["H"], case["N"], case["d"], seed=case["seed"],
                        with_dO=True)
        b = {k: bf16_bits(v) for k, v in x.items()}
        O, L = oracle.attention_forward(b["Q"], b["K"], b["V"], case["scale"], case["causal"])
        dQ, dK, dV = oracle.attention_backward(b["Q"], b["K"], b["V"], b["dO"], case["scale"],
                                               case["causal"])
        for name, val in (("O", O), ("LSE", L), ("dQ", dQ), ("dK", dK), ("dV", dV)):
            np.testing.assert_allclose(val.ravel(), np.array(case[name]), rtol=1e-12,
                                       atol=1e-13)


# ----------------------------------------------------------------------------
# Mutation check: each plausible mistake planted in a copy of the oracle
# source must make at least one pin fail.
# ----------------------------------------------------------------------------

MUTANTS = {
    "drop_scale_fwd": ("s[j] = scale * acc;", "s[j] = acc;", 0),
    "causal_off_by_one": ("if (causal && j > i)", "if (causal && j >= i)", 0),
    "causal_flipped": ("if (causal && j > i)", "if (causal && j < i)", 0),
    "lse_missing_max": ("*lse = m + log(sum);", "*lse = log(sum);", 0),
    "no_normalisation": ("double p = s[j] / sum;", "double p = s[j];", 0),
    "wrong_value_row": ("o_row[c] += p * ld(V, kv_base + j * d + c, dtype);",
                        "o_row[c] += p * ld(V, kv_base + i * d + c, dtype);", 0),
    "gqa_interleaved_heads": ("return (bh / H) * Hkv + (bh % H) / (H / Hkv);",
                              "return (bh / H) * Hkv + (bh % H) % Hkv;", 0),
    "gqa_dK_overwrites": ("dK[kv_base + j * d + c] += scale * acc_k;",
                          "dK[kv_base + j * d + c] = scale * acc_k;", 0),
    "pad_keys_not_masked": ("attention_row(Q, K, V, dtype, len, d,",
                            "attention_row(Q, K, V, dtype, N, d,", 0),
    "pad_query_off_by_one": ("if (i >= len) { /* padding query row */",
                             "if (i > len) { /* padding query row */", 0),
    "pad_bwd_uses_full_length": ("const int64_t N = seq_len(seqlens, bh / H, N_full);",
                                 "const int64_t N = N_full;", 0),
    "exp_sign": ("s[j] = exp(s[j] - m); /* exp(-inf)", "s[j] = exp(m - s[j]); /* exp(-inf)", 0),
    "bwd_drop_scale_in_scores": ("s[j] = scale * acc;", "s[j] = acc;", 1),
    "bwd_drop_D": ("ds[j] = P[i * N + j] * (ds[j] - D);", "ds[j] = P[i * N + j] * ds[j];", 0),
    "bwd_dV_uses_dS": ("acc_v += pd * ld(dO", "acc_v += dS[i * N + j] * ld(dO", 0),
    "bwd_dQ_no_scale": ("dQ[base + i * d + c] = scale * acc;", "dQ[base + i * d + c] = acc;", 0),
    "bwd_dK_transposed_dS": ("acc_k += dS[i * N + j]", "acc_k += dS[j * N + i]", 0),
    "bwd_causal_off_by_one": ("if (causal && j > i)", "if (causal && j >= i)", 1),
    "merge_unweighted": ("o[c] = (a * o_x[c] + b * o_y[c]) / ll;",
                         "o[c] = (exp(m_x - mm) * o_x[c] + exp(m_y - mm) * o_y[c]) / ll;", 0),
    "merge_max_wrong": ("const double mm = fmax(m_x, m_y);", "const double mm = m_x;", 0),
    "philox_round_count": ("for (int r = 0; r < rounds; ++r) {", "for (int r = 0; r < rounds - 1; ++r) {", 0),
    "drop_ten_rounds": ("#define DROP_ROUNDS 7", "#define DROP_ROUNDS 10", 0),
    "philox_hi_lo_swapped": ("c1 = (uint32_t)p1;", "c1 = (uint32_t)(p1 >> 32);", 0),
    "drop_counter_transposed": ("{(uint32_t)(j / 16), (uint32_t)i,", "{(uint32_t)(i / 16), (uint32_t)j,", 0),
    "drop_counter_8_keys": ("{(uint32_t)(j / 16), (uint32_t)i,", "{(uint32_t)(j / 8), (uint32_t)i,", 0),
    "drop_word_index": ("w[(j % 16) / 4]", "w[(i % 16) / 4]", 0),
    "drop_byte_order": ("(8 * (2 * (j % 2) + (j % 4) / 2))", "(8 * (j % 4))", 0),
    "drop_7_bit_uniform": (") & 0xFFu;", ") & 0x7Fu;", 0),
    "drop_keep_inverted": ("return u < dr->threshold;", "return u >= dr->threshold;", 0),
    "drop_scale_one_minus_p": ("dr->keep_scale = 256.0 / t;", "dr->keep_scale = 1.0 / (1.0 - p);", 0),
    "drop_seed_halves_swapped": ("dr->key[0] = (uint32_t)seed;", "dr->key[0] = (uint32_t)(seed >> 32);", 0),
    "drop_no_keep_scale": ("? p * dr->keep_scale : 0.0;", "? p : 0.0;", 0),
    "drop_fwd_kv_head": ("scale, causal, dr, bh, s,", "scale, causal, dr, kv_head(bh, H, Hkv), s,", 0),
    "drop_bwd_dP_unmasked": ("ds[j] = dr ? acc * Z[i * N + j] : acc;", "ds[j] = acc;", 0),
    "drop_bwd_dV_undropped": ("const double pd = dr ? P[i * N + j] * Z[i * N + j] : P[i * N + j];",
                              "const double pd = P[i * N + j];", 0),
    "drop_rows_query_head_for_kv": ("kv_head(bh, H, Hkv) * N * d, i, scale,\n                          causal, dr, bh",
                                    "bh * N * d, i, scale,\n                          causal, dr, bh", 0),
    "drop_bwd_kv_head": ("Z[i * N + j] = dropout_keep(dr, bh, i, j)",
                         "Z[i * N + j] = dropout_keep(dr, kv_head(bh, H, Hkv), i, j)", 0),
}


def _mutate(src, old, new, occurrence):
    idx = -1
    for _ in range(occurrence + 1):
        idx = src.find(old, idx + 1)
        assert idx >= 0, f"mutation anchor not found: {old!r} #{occurrence}"
    return src[:idx] + new + src[idx + len(old):]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name):
    old, new, occ = MUTANTS[name]
    with open(oracle._SRC) as f:
        src = f.read()
    mutated = _mutate(src, old, new, occ)
    assert mutated != src
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        c_path = os.path.join(tmp, "m.c")
        so_path = os.path.join(tmp, "libm.so")
        with open(c_path, "w") as f:
            f.write(mutated)
        oracle.build(force=True, src=c_path, out=so_path)
        lib = oracle.load(so_path)
        caught = []
        for pin in PINS:
            try:
                pin(lib)
            except (AssertionError, RuntimeError, ValueError, FloatingPointError):
                caught.append(pin.__name__)
        assert caught, f"mutant {name} passed every pin"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def test_bf16_rounding_allowance_is_the_format_half_ulp():
    """The O band is applied beyond |bf16(O_ref) - O_ref|; that distance is at
    most half a bf16 ulp (1/32 for |x| in [8, 16), 1/512 for [1, 2))."""
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from _parity import bf16_rounding_distance
    x = np.array([8.09199975993264, 1.0 + 2 ** -9, 1.0, -3.3, 12.0 + 2 ** -5])
    dist = bf16_rounding_distance(x)
    assert abs(dist[0] - 0.029499759932640757) < 1e-12
    assert dist[1] == 2 ** -9 and dist[2] == 0.0 and dist[4] == 2 ** -5
    assert np.all(dist <= np.exp2(np.floor(np.log2(np.abs(x))) - 8) + 1e-15)
