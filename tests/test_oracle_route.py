"""Pins of the oracle's router (A1) and permutation (A3).

Router: top-k experts by softmax probability (the TPU7x MoE page, section on where the
sparsity lies: 512 experts, top-10 by softmax probability), weights renormalised over the k.
Permutation: contiguous per-expert groups ordered by the packed (expert, token) key (the
InferenceX page, section on MoE routing and expert kernels).
"""
import math

import numpy as np
import pytest


def _brute_topk(L, k):
    """Full sort of one row by (logit desc, index asc)."""
    order = sorted(range(len(L)), key=lambda e: (-float(L[e]), e))
    return order[:k]


@pytest.mark.parametrize("T,E,k", [(7, 8, 2), (33, 64, 6), (5, 512, 10), (4, 3, 3), (9, 16, 1)])
def test_route_matches_full_sort(orc, T, E, k):
    rng = np.random.default_rng(T * 1000 + E)
    L = rng.standard_normal((T, E)).astype(np.float32)
    idx, w = orc.route(L, k)
    for t in range(T):
        sel = _brute_topk(L[t], k)
        assert list(idx[t]) == sel
        lv = np.array([float(L[t, e]) for e in sel])
        p = np.exp(lv - lv.max())
        p /= p.sum()
        assert np.allclose(w[t], p, rtol=0, atol=1e-15)
        assert abs(w[t].sum() - 1.0) < 1e-15


def test_route_ties_lower_index_wins(orc):
    L = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, 0.0]], np.float32)
    idx, w = orc.route(L, 3)
    assert list(idx[0]) == [1, 2, 4]
    assert np.allclose(w[0], [1 / 3] * 3, atol=1e-15)
    idx, w = orc.route(L, 4)
    assert list(idx[0]) == [1, 2, 4, 3]
    L = np.zeros((1, 8), np.float32)
    idx, _ = orc.route(L, 5)
    assert list(idx[0]) == [0, 1, 2, 3, 4]


def test_route_two_experts_closed_form(orc):
    L = np.array([[0.25, -1.5], [2.0, 2.5]], np.float32)
    idx, w = orc.route(L, 2)
    assert list(idx[0]) == [0, 1] and list(idx[1]) == [1, 0]
    assert abs(w[0, 0] - 1 / (1 + math.exp(-1.5 - 0.25))) < 1e-15
    assert abs(w[1, 0] - 1 / (1 + math.exp(2.0 - 2.5))) < 1e-15


def test_route_k_equals_E_is_full_softmax(orc):
    rng = np.random.default_rng(3)
    L = rng.standard_normal((6, 12)).astype(np.float32)
    idx, w = orc.route(L, 12)
    for t in range(6):
        p = np.exp(L[t].astype(np.float64) - L[t].max())
        p /= p.sum()
        assert np.allclose(w[t], p[idx[t]], atol=1e-15)
        assert sorted(idx[t]) == list(range(12))


def test_route_k1_is_argmax_weight_one(orc):
    rng = np.random.default_rng(4)
    L = rng.standard_normal((50, 40)).astype(np.float32)
    idx, w = orc.route(L, 1)
    assert np.array_equal(idx[:, 0], np.argmax(L, axis=1))
    assert np.all(w == 1.0)


def test_route_rejects_bad_k(orc):
    with pytest.raises(ValueError):
        orc.route(np.zeros((2, 4), np.float32), 5)


@pytest.mark.parametrize("T,E,k", [(16, 8, 2), (100, 32, 4), (3, 512, 10), (0, 4, 2), (1, 1, 1)])
def test_permute_invariants(orc, T, E, k):
    rng = np.random.default_rng(T + E + k)
    L = rng.standard_normal((T, E)).astype(np.float32)
    idx, _ = orc.route(L, k)
    counts, offsets, perm, pos = orc.permute(idx, E)
    assert counts.sum() == T * k
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets) == counts)
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)  # tokens strictly increasing inside a group
        assert counts[e] == int((idx == e).sum())
    # pos is the inverse of perm; every (t, j) lands exactly once
    rows = pos.reshape(-1)
    assert sorted(rows.tolist()) == list(range(T * k))
    for t in range(T):
        for j in range(k):
            r = pos[t, j]
            assert perm[r] == t
            e = idx[t, j]
            assert offsets[e] <= r < offsets[e + 1]


def test_permute_matches_lexsort(orc):
    rng = np.random.default_rng(9)
    T, E, k = 300, 64, 6
    idx, _ = orc.route(rng.standard_normal((T, E)).astype(np.float32), k)
    counts, offsets, perm, pos = orc.permute(idx, E)
    e_flat = idx.reshape(-1)
    t_flat = np.repeat(np.arange(T), k)
    order = np.lexsort((t_flat, e_flat))  # primary key expert, then token
    assert np.array_equal(perm, t_flat[order])
    assert np.array_equal(np.bincount(e_flat, minlength=E), counts)


def test_router_logits_against_exact_sums(orc):
    """bf16 x bf16 products are exact in fp64; the oracle's logits equal an exact-rational sum."""
    import torch
    from fractions import Fraction
    g = torch.Generator().manual_seed(11)
    x = torch.randn(3, 64, generator=g).to(torch.bfloat16)
    w = torch.randn(5, 64, generator=g).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    lg, bd = orc.router_logits(xb, wb)
    xf, wf = x.double().numpy(), w.double().numpy()
    for t in range(3):
        for e in range(5):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[t], wf[e]))
            assert abs(Fraction(lg[t, e]) - exact) <= Fraction(1, 2 ** 40) * (1 + abs(exact))
            assert bd[t, e] == np.abs(xf[t] * wf[e]).sum()
