"""Pins of the oracle's prefill backward (gradients of Eq. (10) of the Kwai
Summary Attention Technical Report under the KSA mask of section 2.2):
central finite differences of the loss sum(do * o), the causal-attention
special case (window covering the whole sequence) against autograd of
PyTorch's fp64 scaled_dot_product_attention, and two exact identities of
softmax attention (the key gradients of a kv head sum to zero; the value
gradients sum to the output gradients of its q heads)."""
import numpy as np
import pytest
import torch

import oracle


def _inputs(n, k, Hq, Hkv, d, seed):
    L = n + n // k
    rng = np.random.default_rng(seed)
    f = lambda H: rng.standard_normal((L, H, d))
    return f(Hq), f(Hkv), f(Hkv), f(Hq)


@pytest.mark.parametrize("n,k,C,Hq,Hkv,d", [(11, 3, 1, 4, 2, 8), (9, 4, 0, 2, 1, 8), (7, 1, 2, 2, 2, 4),
                                            (17, 4, 1, 2, 1, 6)])
def test_bwd_matches_finite_differences(n, k, C, Hq, Hkv, d):
    q, kk, v, do = _inputs(n, k, Hq, Hkv, d, seed=n + 10 * k + C)
    dq, dk, dv, o, _ = oracle.ksa_attention_bwd(n, k, C, q, kk, v, do)

    def loss(q_, k_, v_):
        return float((oracle.ksa_attention_bwd(n, k, C, q_, k_, v_, do)[3] * do).sum())

    eps = 1e-6
    rng = np.random.default_rng(1)
    for which, arr, grad in (("q", q, dq), ("k", kk, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            args = {"q": q, "k": kk, "v": v}
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            lp = loss(*(plus if nm == which else args[nm] for nm in ("q", "k", "v")))
            lm = loss(*(minus if nm == which else args[nm] for nm in ("q", "k", "v")))
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


@pytest.mark.parametrize("n,k,Hq,Hkv,d", [(24, 4, 4, 2, 16), (13, 3, 2, 1, 8)])
def test_bwd_full_window_equals_causal_sdpa_autograd(n, k, Hq, Hkv, d):
    """With the window covering the whole sequence (C >= n/k) text rows attend
    causally to all text and see no summary; with zero output gradient on the
    summary rows the text gradients are those of causal attention."""
    C = n // k + 1
    q, kk, v, do = _inputs(n, k, Hq, Hkv, d, seed=3)
    idx = oracle.aug_index(n, k)
    L = len(idx)
    text = np.array([a for a in range(L) if not (a < (n // k) * (k + 1) and a % (k + 1) == k)])
    summ = np.setdiff1d(np.arange(L), text)
    do[summ] = 0
    dq, dk, dv, _, _ = oracle.ksa_attention_bwd(n, k, C, q, kk, v, do)
    G = Hq // Hkv
    tq = torch.tensor(q[text], dtype=torch.float64).transpose(0, 1).requires_grad_(True)   # [Hq, n, d]
    tk = torch.tensor(kk[text], dtype=torch.float64).transpose(0, 1).requires_grad_(True)
    tv = torch.tensor(v[text], dtype=torch.float64).transpose(0, 1).requires_grad_(True)
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(G, dim=0), tv.repeat_interleave(G, dim=0), is_causal=True)
    (out * torch.tensor(do[text], dtype=torch.float64).transpose(0, 1)).sum().backward()
    np.testing.assert_allclose(dq[text], tq.grad.transpose(0, 1).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk[text], tk.grad.transpose(0, 1).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv[text], tv.grad.transpose(0, 1).numpy(), rtol=1e-10, atol=1e-12)
    # summaries are invisible to text queries, and the summary rows' own
    # output gradient is zero: nothing flows into them
    assert np.abs(dk[summ]).max() == 0 and np.abs(dv[summ]).max() == 0 and np.abs(dq[summ]).max() == 0


@pytest.mark.parametrize("n,k,C", [(40, 4, 2), (33, 8, 1), (64, 8, 0)])
def test_bwd_identities(n, k, C):
    Hq, Hkv, d = 4, 2, 16
    q, kk, v, do = _inputs(n, k, Hq, Hkv, d, seed=7)
    dq, dk, dv, _, _ = oracle.ksa_attention_bwd(n, k, C, q, kk, v, do)
    L = q.shape[0]
    G = Hq // Hkv
    assert np.abs(dk.sum(axis=0)).max() < 1e-11
    want = do.reshape(L, Hkv, G, d).sum(axis=(0, 2))
    np.testing.assert_allclose(dv.sum(axis=0), want, rtol=1e-12, atol=1e-11)


def test_bwd_padded_layout():
    """The packed, padded augmented layout of the library: each sequence's
    rows map to its own gradients; padding rows stay zero."""
    seqlens, k, C, Hq, Hkv, d = [10, 8, 3], 4, 1, 2, 1, 8
    rows = sum(((n + k - 1) // k) * (k + 1) for n in seqlens)
    rng = np.random.default_rng(5)
    qa, ka, va, doa = (rng.standard_normal((rows, H, d)) for H in (Hq, Hkv, Hkv, Hq))
    dq, dk, dv = oracle.ksa_prefill_bwd_aug(seqlens, k, C, qa, ka, va, doa)
    base = 0
    live = np.zeros(rows, bool)
    for n in seqlens:
        r = base + oracle.aug_index(n, k)
        live[r] = True
        g = oracle.ksa_attention_bwd(n, k, C, qa[r], ka[r], va[r], doa[r])
        np.testing.assert_array_equal(dq[r], g[0])
        np.testing.assert_array_equal(dk[r], g[1])
        base += ((n + k - 1) // k) * (k + 1)
    assert np.abs(dq[~live]).max() == 0 and np.abs(dk[~live]).max() == 0 and np.abs(dv[~live]).max() == 0


@pytest.mark.parametrize("n,k,C", [(40, 4, 2), (35, 8, 1), (13, 1, 0)])
def test_bwd_dq_rows_match_dense(n, k, C):
    """The per-row form (closed-form visible set) equals the dense backward,
    and the visible sets equal the rows of the dense mask."""
    Hq, Hkv, d = 4, 2, 8
    q, kk, v, do = _inputs(n, k, Hq, Hkv, d, seed=9)
    dq = oracle.ksa_attention_bwd(n, k, C, q, kk, v, do)[0]
    M = oracle.dense_mask(n, k, C)
    rows = np.arange(q.shape[0])
    for a in rows:
        np.testing.assert_array_equal(np.sort(oracle.visible_keys(n, k, C, int(a))), np.nonzero(M[a])[0])
    np.testing.assert_allclose(oracle.ksa_attention_bwd_dq_rows(n, k, C, q, kk, v, do, rows), dq, rtol=1e-12,
                               atol=1e-12)


@pytest.mark.parametrize("n,k,C", [(40, 4, 2), (35, 8, 1), (13, 1, 0), (30, 3, 0)])
def test_bwd_dkv_keys_match_dense(n, k, C):
    """The per-key form (queries from the key's side of the rules) equals the
    dense backward's dk and dv, and each key's seeing queries equal the
    column of the dense mask."""
    Hq, Hkv, d = 4, 2, 8
    q, kk, v, do = _inputs(n, k, Hq, Hkv, d, seed=19)
    _, dk, dv, _, _ = oracle.ksa_attention_bwd(n, k, C, q, kk, v, do)
    M = oracle.dense_mask(n, k, C)
    for a in range(q.shape[0]):
        np.testing.assert_array_equal(np.sort(oracle.seeing_queries(n, k, C, a)), np.nonzero(M[:, a])[0])
    keys = np.arange(q.shape[0])[::-1]   # any order
    gk, gv = oracle.ksa_attention_bwd_dkv_keys(n, k, C, q, kk, v, do, keys)
    np.testing.assert_allclose(gk, dk[keys], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gv, dv[keys], rtol=1e-12, atol=1e-12)
    sub = keys[::5]   # a subset: rows that see no requested key add nothing
    gk, gv = oracle.ksa_attention_bwd_dkv_keys(n, k, C, q, kk, v, do, sub)
    np.testing.assert_allclose(gk, dk[sub], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gv, dv[sub], rtol=1e-12, atol=1e-12)


def test_rope_transpose_and_inverse():
    """RoPE is a rotation: rotating by -pos undoes it, and it is its own
    transpose's inverse (<R x, g> = <x, R^T g>)."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((50, 3, 16))
    g = rng.standard_normal((50, 3, 16))
    pos = rng.integers(0, 100000, 50)
    rx = oracle.rope(x, pos, 1e6)
    np.testing.assert_allclose(oracle.rope(rx, -pos, 1e6), x, rtol=1e-12, atol=1e-12)
    assert abs((rx * g).sum() - (x * oracle.rope(g, -pos, 1e6)).sum()) < 1e-9


def test_interleave_rope_bwd_is_the_transpose():
    """<interleave_rope(inputs), G> = <inputs, interleave_rope_bwd(G)> for the
    augmented gradients G (the definition of the backward of a linear map)."""
    seqlens, k, Hq, Hkv, d, theta = [11, 8, 5], 4, 2, 1, 8, 1e6
    rng = np.random.default_rng(12)
    nt, ns = sum(seqlens), sum(n // k for n in seqlens)
    qt, kt, vt = (rng.standard_normal((nt, H, d)) for H in (Hq, Hkv, Hkv))
    qs, ks, vs = (rng.standard_normal((ns, H, d)) for H in (Hq, Hkv, Hkv))
    rows = sum(((n + k - 1) // k) * (k + 1) for n in seqlens)
    qa, ka, va = np.zeros((rows, Hq, d)), np.zeros((rows, Hkv, d)), np.zeros((rows, Hkv, d))
    base = t0 = s0 = 0
    for n in seqlens:
        m = n // k
        i = np.arange(n)
        tr = base + (i // k) * (k + 1) + i % k
        sr = base + np.arange(m) * (k + 1) + k
        pt, ps = oracle.text_positions(n), oracle.summary_positions(n, k)
        qa[tr], ka[tr], va[tr] = oracle.rope(qt[t0:t0 + n], pt, theta), oracle.rope(kt[t0:t0 + n], pt, theta), vt[t0:t0 + n]
        if m:
            qa[sr], ka[sr], va[sr] = oracle.rope(qs[s0:s0 + m], ps, theta), oracle.rope(ks[s0:s0 + m], ps, theta), vs[s0:s0 + m]
        base += ((n + k - 1) // k) * (k + 1)
        t0 += n
        s0 += m
    G = [rng.standard_normal(a.shape) for a in (qa, ka, va)]
    back = oracle.interleave_rope_bwd(seqlens, k, theta, *G)
    lhs = sum((a * g).sum() for a, g in zip((qa, ka, va), G))
    rhs = sum((a * b).sum() for a, b in zip((qt, kt, vt, qs, ks, vs), back))
    assert abs(lhs - rhs) < 1e-8 * max(1.0, abs(lhs))
