"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a library routine, a closed form, an
invariant, a printed example or brute force, so that a dropped term, a wrong
sign or index or a transposed operand fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(20261202)


# ------------------------------------------------------------------ meanpool

def test_meanpool_matches_numpy_mean():
    K = rng.standard_normal((96, 16))
    got = oracle.meanpool(K, 4)
    want = K.reshape(24, 4, 16).mean(axis=1)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)


def test_meanpool_ragged_last_block_uses_true_count():
    K = rng.standard_normal((300, 8))
    got = oracle.meanpool(K, 128)
    want = np.stack([K[0:128].mean(0), K[128:256].mean(0), K[256:300].mean(0)])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)


def test_meanpool_matches_torch_avg_pool():
    K = torch.randn(64, 32, dtype=torch.float64)
    want = torch.nn.functional.avg_pool1d(K.T[None], 8, 8)[0].T.numpy()
    np.testing.assert_allclose(oracle.meanpool(K.numpy(), 8), want, atol=1e-15)


# ------------------------------------------------------------------ k-means

def _planted(shares, d=32, sep=50.0, noise=0.0, seed=0):
    """Queries grouped in contiguous runs so that the deterministic init row
    floor(c*M/8) falls inside run c."""
    g = np.random.default_rng(seed)
    centers = g.standard_normal((len(shares), d)) * sep
    rows = []
    for c, n in enumerate(shares):
        rows.append(centers[c] + noise * g.standard_normal((n, d)))
    return np.concatenate(rows), centers


def test_kmeans_recovers_planted_clusters_and_shares():
    # run c covers rows [16c - 3, ...) so that row 16c lies in it
    shares = [13, 16, 16, 16, 16, 16, 16, 19]
    Qb, centers = _planted(shares, noise=0.1)
    C, w, lab = oracle.kmeans(Qb, 8, 10)
    np.testing.assert_allclose(w, np.array(shares) / 128.0, atol=0)
    want_lab = np.repeat(np.arange(8), shares)
    np.testing.assert_array_equal(lab, want_lab)
    for c in range(8):
        np.testing.assert_allclose(C[c], Qb[want_lab == c].mean(0), atol=1e-12)


def test_kmeans_identical_queries_single_cluster():
    q = rng.standard_normal(64)
    Qb = np.tile(q, (128, 1))
    C, w, lab = oracle.kmeans(Qb, 8, 10)
    assert w[0] == 1.0 and np.all(w[1:] == 0.0)
    assert np.all(lab == 0)
    np.testing.assert_allclose(C[0], q, atol=0)


def test_kmeans_matches_sklearn_lloyd():
    from sklearn.cluster import KMeans
    agree = 0
    for seed in range(6):
        g = np.random.default_rng(100 + seed)
        Qb = g.standard_normal((128, 64)) + 0.8 * np.sin(np.arange(128)[:, None] / 9.0 + np.arange(64))
        init = Qb[[(c * 128) // 8 for c in range(8)]].copy()
        C, w, lab = oracle.kmeans(Qb, 8, 10)
        if np.any(w == 0):  # sklearn relocates empty clusters; not comparable
            continue
        km = KMeans(n_clusters=8, init=init, n_init=1, max_iter=10, algorithm="lloyd", tol=0.0)
        km.fit(Qb)
        np.testing.assert_allclose(C, km.cluster_centers_, rtol=1e-9, atol=1e-9)
        agree += 1
    assert agree >= 3


def test_kmeans_fixed_point_invariant():
    Qb = rng.standard_normal((128, 32))
    C, w, lab = oracle.kmeans(Qb, 8, 200)  # converged
    d2 = ((Qb[:, None, :] - C[None, :, :]) ** 2).sum(-1)
    best = d2.min(1)
    assert np.all(d2[np.arange(128), lab] <= best + 1e-12)
    for c in range(8):
        if w[c] > 0:
            np.testing.assert_allclose(C[c], Qb[lab == c].mean(0), atol=1e-12)
    assert abs(w.sum() - 1.0) < 1e-15


def test_kmeans_ragged_block_fewer_rows():
    Qb = rng.standard_normal((16, 8))
    C, w, lab = oracle.kmeans(Qb, 8, 10)
    assert abs(w.sum() - 1.0) < 1e-15
    assert lab.min() >= 0 and lab.max() < 8


# ------------------------------------------------------------------ scores

def test_scores_one_cluster_is_block_mean_softmax():
    """With one cluster the selector reduces to the block-mean baseline:
    softmax over KV blocks of mean(q) . kbar / sqrt(d)."""
    Qb = torch.randn(128, 64, dtype=torch.float64)
    K = torch.randn(512, 64, dtype=torch.float64)
    C, w, _ = oracle.kmeans(Qb.numpy(), 1, 10)
    np.testing.assert_allclose(C[0], Qb.mean(0).numpy(), atol=1e-14)
    Kbar = oracle.meanpool(K.numpy(), 4)
    s = oracle.scores(C, w, Kbar, 1 / 8.0)
    want = torch.softmax(Qb.mean(0) @ torch.from_numpy(Kbar).T / 8.0, dim=0).numpy()
    np.testing.assert_allclose(s, want, rtol=1e-12, atol=1e-18)


def test_scores_planted_clusters_weighted_softmax():
    shares = [13, 16, 16, 16, 16, 16, 16, 19]
    Qb, centers = _planted(shares, d=32, sep=1.0)
    C, w, _ = oracle.kmeans(Qb, 8, 10)
    Kbar = torch.randn(200, 32, dtype=torch.float64)
    scale = 0.3
    s = oracle.scores(C, w, Kbar.numpy(), scale)
    P = torch.softmax(torch.from_numpy(centers) @ Kbar.T * scale, dim=1)
    want = (torch.tensor(shares, dtype=torch.float64)[:, None] / 128 * P).sum(0).numpy()
    np.testing.assert_allclose(s, want, rtol=1e-12)
    assert abs(s.sum() - 1) < 1e-13


def test_scores_equivariant_under_block_permutation():
    C = rng.standard_normal((8, 16))
    w = rng.dirichlet(np.ones(8))
    Kbar = rng.standard_normal((50, 16))
    perm = rng.permutation(50)
    s = oracle.scores(C, w, Kbar, 0.25)
    sp = oracle.scores(C, w, Kbar[perm], 0.25)
    np.testing.assert_allclose(sp, s[perm], rtol=1e-13)


# ------------------------------------------------------------------ water-fill

def _bisect_pi(s, Bblk):
    lo, hi = 0.0, 1.0
    while np.minimum(1.0, hi * s).sum() < Bblk:
        hi *= 2
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if np.minimum(1.0, mid * s).sum() < Bblk:
            lo = mid
        else:
            hi = mid
    return np.minimum(1.0, hi * s)


@pytest.mark.parametrize("n,Bblk", [(1000, 100.0), (1024, 128.0), (18900, 1512.0), (50, 49.5)])
def test_waterfill_invariants_and_bisection(n, Bblk):
    s = rng.pareto(1.2, n) + 1e-6  # heavy tail -> several capping rounds
    s /= s.sum()
    pi, lam, rounds = oracle.waterfill(s, Bblk)
    assert abs(pi.sum() - Bblk) <= 1e-12 * Bblk
    assert np.all(pi >= 0) and np.all(pi <= 1)
    unc = pi < 1
    np.testing.assert_allclose(pi[unc], lam * s[unc], rtol=1e-15)
    assert np.all(lam * s[~unc] >= 1 - 1e-15)
    order = np.argsort(s)
    assert np.all(np.diff(pi[order]) >= -1e-15)
    np.testing.assert_allclose(pi, _bisect_pi(s, Bblk), rtol=1e-12, atol=1e-15)
    assert rounds >= 1


def test_waterfill_uniform_scores_closed_form():
    s = np.full(800, 1 / 800)
    pi, lam, _ = oracle.waterfill(s, 80.0)
    np.testing.assert_allclose(pi, 0.1, rtol=1e-13)


def test_waterfill_full_budget_takes_every_positive_block():
    s = np.array([0.5, 0.0, 0.25, 0.25])
    pi, _, rounds = oracle.waterfill(s, 4.0)
    np.testing.assert_array_equal(pi, [1, 0, 1, 1])
    assert rounds == 0


def test_waterfill_dominant_block_always_taken():
    """The most important blocks are always taken (SIP paragraph)."""
    s = np.array([0.9] + [0.1 / 99] * 99)
    pi, lam, _ = oracle.waterfill(s, 10.0)
    assert pi[0] == 1.0
    np.testing.assert_allclose(pi[1:], 9.0 / 99, rtol=1e-13)


# ------------------------------------------------------------------ RNG

@pytest.mark.parametrize("key,ctr", [
    ((0, 0), (0, 0, 0, 0)),
    ((2**64 - 1, 2**64 - 1), (2**64 - 2, 2**64 - 1, 2**64 - 1, 2**64 - 1)),
    ((0x243F6A8885A308D3, 0x13198A2E03707344), (0xA4093822299F31D0, 0x082EFA98EC4E6C89,
                                                0x452821E638D01377, 0xBE5466CF34E90C6C)),
    ((12345, 0), (7, 3, 2, 0)),
])
def test_philox_matches_numpy_bit_generator(key, ctr):
    """numpy's Philox (4x64, 10 rounds) advances its counter by one before
    each block, so its first block for counter c is Philox(c + 1)."""
    bg = np.random.Philox(key=np.array(key, dtype=np.uint64),
                          counter=np.array(ctr, dtype=np.uint64))
    np.testing.assert_array_equal(bg.state["state"]["counter"], np.array(ctr, dtype=np.uint64))
    want = bg.random_raw(4)
    c1 = list(ctr)
    c1[0] = (c1[0] + 1) % 2**64
    if c1[0] == 0:  # carry, as numpy does
        c1[1] = (c1[1] + 1) % 2**64
    got = oracle.philox4x64_10(c1, key)
    np.testing.assert_array_equal(got, want)


def test_uniform_uses_halves_of_counter_block_words():
    seed, b, h, qb = 77, 0, 3, 5
    for j in [0, 1, 2, 3, 4, 7, 8, 9, 1001]:
        words = oracle.philox4x64_10([j // 8, qb, h, b], [seed, 0])
        w = int(words[(j // 2) % 4])
        half = (w & 0xFFFFFFFF) if j % 2 else (w >> 32)
        assert oracle.uniform(seed, b, h, qb, j) == float(half >> 8) * 2.0**-24


def test_uniform_statistics():
    u = np.array([oracle.uniform(9, 0, 1, 2, j) for j in range(200000)])
    assert u.min() >= 0 and u.max() < 1
    assert abs(u.mean() - 0.5) < 5 * math.sqrt(1 / 12 / u.size)
    hist, _ = np.histogram(u, bins=256, range=(0, 1))
    exp = u.size / 256
    chi2 = ((hist - exp) ** 2 / exp).sum()
    assert chi2 < 255 + 6 * math.sqrt(2 * 255)
    r = np.corrcoef(u[:-1], u[1:])[0, 1]
    assert abs(r) < 5 / math.sqrt(u.size)


# ------------------------------------------------------------------ sampling

def test_sample_deterministic_ends_and_order():
    pi = np.array([1.0, 0.0, 0.5, 1.0, 0.0, 0.3] * 50, dtype=np.float32)
    idx, ps, n = oracle.sample(pi, 3, 0, 0, 0)
    assert n == idx.size
    assert np.all(np.diff(idx) > 0)
    assert set(np.flatnonzero(pi == 1.0)) <= set(idx.tolist())
    assert not set(np.flatnonzero(pi == 0.0)) & set(idx.tolist())
    np.testing.assert_array_equal(ps, pi[idx])


def test_sample_inclusion_frequency_matches_pi():
    pi = np.linspace(0.02, 0.98, 40).astype(np.float32)
    S = 4000
    hits = np.zeros(40)
    for seed in range(S):
        idx, _, _ = oracle.sample(pi, seed, 0, 1, 2)
        hits[idx] += 1
    z = (hits / S - pi) / np.sqrt(pi * (1 - pi) / S)
    assert np.max(np.abs(z)) < 5


def test_sample_capacity_reports_true_count():
    pi = np.ones(100, dtype=np.float32)
    idx, ps, n = oracle.sample(pi, 1, 0, 0, 0, cap=10)
    assert n == 100 and idx.size == 10
    np.testing.assert_array_equal(idx, np.arange(10))


def test_plan_capacity_formula():
    assert oracle.plan_capacity(18900, 0.08) == min(18900, math.ceil(1512 + 8 * math.sqrt(1512) + 32))
    assert oracle.plan_capacity(1024, 1.0) == 1024


# ------------------------------------------------------------------ top-k

def test_topk_matches_numpy_lexsort():
    s = np.round(rng.random(500), 2)  # many ties
    for k in [0, 1, 37, 250, 500]:
        order = np.lexsort((np.arange(500), -s))[:k]
        np.testing.assert_array_equal(oracle.topk(s, k), np.sort(order))


# ------------------------------------------------------------------ attention

def test_dense_matches_torch_sdpa():
    q = torch.randn(1, 1, 70, 32, dtype=torch.float64)
    k = torch.randn(1, 1, 90, 32, dtype=torch.float64)
    v = torch.randn(1, 1, 90, 32, dtype=torch.float64)
    want = torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0].numpy()
    O, lse = oracle.dense(q[0, 0], k[0, 0], v[0, 0], 1 / math.sqrt(32))
    np.testing.assert_allclose(O, want, atol=1e-13)
    want_lse = torch.logsumexp(q[0, 0] @ k[0, 0].T / math.sqrt(32), dim=1).numpy()
    np.testing.assert_allclose(lse, want_lse, atol=1e-13)


@pytest.mark.parametrize("kb,N", [(4, 256), (128, 300), (8, 96)])
def test_sparse_block_matches_sdpa_with_log_inverse_pi_mask(kb, N):
    """The HT estimator as a logit shift: an SDPA with an additive mask equal
    to ln(1/pi_j) on the selected blocks' keys and -inf elsewhere."""
    d, M = 16, 40
    Q = torch.randn(M, d, dtype=torch.float64)
    K = torch.randn(N, d, dtype=torch.float64)
    V = torch.randn(N, d, dtype=torch.float64)
    nkvb = -(-N // kb)
    sel = np.sort(rng.choice(nkvb, size=max(1, nkvb // 2), replace=False)).astype(np.int32)
    if nkvb - 1 not in sel:
        sel = np.append(sel, nkvb - 1).astype(np.int32)  # ragged block included
    pis = rng.uniform(0.05, 1.0, sel.size).astype(np.float32)
    mask = torch.full((M, N), -math.inf, dtype=torch.float64)
    for j, p in zip(sel, pis):
        mask[:, j * kb:min(N, (j + 1) * kb)] = math.log(1.0 / float(p))
    scale = 0.21
    want = torch.nn.functional.scaled_dot_product_attention(
        Q[None, None], K[None, None], V[None, None], attn_mask=mask[None, None], scale=scale)[0, 0]
    O, lse = oracle.sparse_block(Q, K, V, kb, sel, pis, scale)
    np.testing.assert_allclose(O, want.numpy(), atol=1e-13)
    np.testing.assert_allclose(lse, torch.logsumexp(Q @ K.T * scale + mask, 1).numpy(), atol=1e-12)


def test_ht_weight_example_from_the_page():
    """SIP paragraph: a block chosen with probability 25% counts as four."""
    with open(os.path.join(GOLDEN, "ht_weight.json")) as f:
        g = json.load(f)
    d = 8
    Q = rng.standard_normal((1, d))
    K = np.repeat(rng.standard_normal((2, d)), 4, axis=0)  # two 4-token blocks
    V = rng.standard_normal((8, d))
    O, lse = oracle.sparse_block(Q, K, V, 4, [0, 1], [1.0, g["pi"]], 1.0)
    a = np.exp(Q @ K.T)[0]
    w = np.array([1.0] * 4 + [g["counts_as_blocks"]] * 4)
    np.testing.assert_allclose(O[0], (w * a) @ V / (w * a).sum(), atol=1e-13)


def test_full_budget_sparse_equals_dense():
    d, N = 32, 256
    Q = rng.standard_normal((128, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    O, lse = oracle.sparse_block(Q, K, V, 4, np.arange(N // 4), np.ones(N // 4), 0.2)
    Od, lsed = oracle.dense(Q, K, V, 0.2)
    np.testing.assert_allclose(O, Od, atol=1e-12)
    np.testing.assert_allclose(lse, lsed, atol=1e-12)


def test_empty_selection_gives_zero_output():
    O, lse = oracle.sparse_block(rng.standard_normal((4, 8)), rng.standard_normal((16, 8)),
                                 rng.standard_normal((16, 8)), 4, [], [], 1.0)
    assert np.all(O == 0) and np.all(np.isneginf(lse))


def test_ht_unbiased_exact_enumeration():
    """E over Poisson samples of the HT numerator and normaliser equals the
    dense ones, computed by enumerating every subset of a tiny row."""
    nkvb, kb, d = 8, 4, 8
    N = nkvb * kb
    Q = rng.standard_normal((3, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    pi = np.array([1.0, 0.5, 0.25, 0.8, 0.1, 0.6, 0.3, 0.9], dtype=np.float32)
    scale = 0.4
    Od, lsed = oracle.dense(Q, K, V, scale)
    Dd = np.exp(lsed)
    Nd = Od * Dd[:, None]
    EN = np.zeros_like(Nd)
    ED = np.zeros_like(Dd)
    for mask in itertools.product([0, 1], repeat=nkvb):
        sel = np.flatnonzero(mask)
        pd = pi.astype(np.float64)  # the exact fp32 values, arithmetic in double
        p = np.prod([pd[j] if m else 1.0 - pd[j] for j, m in enumerate(mask)])
        if p == 0:
            continue
        O, lse = oracle.sparse_block(Q, K, V, kb, sel, pi[sel], scale)
        D = np.exp(lse)
        EN += p * O * D[:, None]
        ED += p * D
    np.testing.assert_allclose(ED, Dd, rtol=1e-12)
    np.testing.assert_allclose(EN, Nd, rtol=1e-11, atol=1e-12)


def test_ht_unbiased_monte_carlo_z():
    nkvb, kb, d = 64, 4, 8
    N = nkvb * kb
    Q = rng.standard_normal((2, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    s = rng.random(nkvb) ** 3 + 1e-3
    s /= s.sum()
    pi = oracle.waterfill(s, 12.0)[0].astype(np.float32)
    scale = 0.5
    a = np.exp(Q @ K.T * scale)                          # [2, N]
    ab = a.reshape(2, nkvb, kb).sum(-1)                   # per-block normaliser terms
    D_true = ab.sum(1)
    pid = pi.astype(np.float64)
    var = ((1 - pid) / pid * ab ** 2).sum(1)
    S = 3000
    Dhat = np.zeros((S, 2))
    for seed in range(S):
        idx, ps, _ = oracle.sample(pi, seed, 0, 0, 0)
        O, lse = oracle.sparse_block(Q, K, V, kb, idx, ps, scale)
        Dhat[seed] = np.exp(lse)
    z = (Dhat.mean(0) - D_true) / np.sqrt(var / S)
    assert np.all(np.abs(z) < 5), z
