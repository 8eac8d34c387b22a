"""Whole-method checks of the oracle on the tiny workload (CPU only).

* the batched drivers agree with the per-row functions (indexing);
* a full budget reproduces dense attention;
* the Horvitz-Thompson sampled forward is closer to dense attention than
  top-k truncation at the same block budget (the claim of the SIP paragraph
  of the AB-Attention news page and of the "where earlier sparse schemes
  fail" section).
"""
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_12_b200 import inputs

W = inputs.TINY


@pytest.fixture(scope="module")
def tiny():
    Q, K, V = inputs.make_qkv(W)
    scale = 1 / math.sqrt(W.d)
    sel = oracle.selector_all(Q, K, W.q_block, W.kv_block, W.n_clusters, W.kmeans_iters, scale)
    Od, lsed = [], []
    Qd, Kd, Vd = oracle.f64(Q), oracle.f64(K), oracle.f64(V)
    for h in range(W.H):
        o, l = oracle.dense(Qd[0, h], Kd[0, h], Vd[0, h], scale)
        Od.append(o)
        lsed.append(l)
    return dict(Q=Qd, K=Kd, V=Vd, scale=scale, sel=sel, Od=np.stack(Od)[None], lsed=np.stack(lsed)[None])


def test_selector_all_matches_per_row(tiny):
    sel, Q, K = tiny["sel"], tiny["Q"], tiny["K"]
    h, qb = 1, 7
    Kbar = oracle.meanpool(K[0, h], W.kv_block)
    np.testing.assert_array_equal(sel["Kbar"][0, h], Kbar)
    C, w, lab = oracle.kmeans(Q[0, h, qb * 128:(qb + 1) * 128], 8, 10)
    np.testing.assert_array_equal(sel["C"][0, h, qb], C)
    np.testing.assert_array_equal(sel["w"][0, h, qb], w)
    s = oracle.scores(C, w, Kbar, tiny["scale"])
    np.testing.assert_array_equal(sel["S"][0, h, qb], s)
    np.testing.assert_allclose(sel["S"].sum(-1), 1.0, rtol=1e-12)


def test_plan_all_matches_per_row(tiny):
    S = tiny["sel"]["S"]
    plan = oracle.plan_all(S, W.budget, 0, 11, want_pi=True)
    h, qb = 0, 31
    nkvb = S.shape[-1]
    pi, _, _ = oracle.waterfill(S[0, h, qb], W.budget * nkvb)
    np.testing.assert_array_equal(plan["pi"][0, h, qb], pi.astype(np.float32))
    idx, ps, n = oracle.sample(pi.astype(np.float32), 11, 0, h, qb, plan["cap"])
    assert plan["counts"][0, h, qb] == n
    np.testing.assert_array_equal(plan["idx"][0, h, qb, :n], idx)
    np.testing.assert_array_equal(plan["pi_sel"][0, h, qb, :n], ps)
    # expected count per row is the budget
    assert abs(plan["counts"].mean() - W.budget * nkvb) < 5 * math.sqrt(W.budget * nkvb / plan["counts"].size)


def test_batched_full_budget_equals_dense(tiny):
    nqb, nkvb = W.N // 128, W.N // 4
    rows = W.H * nqb
    counts = np.full(rows, nkvb)
    idx = np.tile(np.arange(nkvb, dtype=np.int32), (rows, 1))
    ps = np.ones((rows, nkvb), dtype=np.float32)
    O, lse = oracle.forward_rows(tiny["Q"], tiny["K"], tiny["V"], 128, 4, counts, idx, ps, tiny["scale"])
    np.testing.assert_allclose(O, tiny["Od"], atol=1e-12)
    np.testing.assert_allclose(lse, tiny["lsed"], atol=1e-12)


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_sampling_beats_topk_truncation(tiny):
    S = tiny["sel"]["S"]
    errs = []
    for seed in range(16):
        p = oracle.plan_all(S, W.budget, 0, seed)
        O, _ = oracle.forward_rows(tiny["Q"], tiny["K"], tiny["V"], 128, 4, p["counts"], p["idx"],
                                   p["pi_sel"], tiny["scale"])
        errs.append(_rel_l2(O, tiny["Od"]))
    p = oracle.plan_all(S, W.budget, 1, 0)
    O, _ = oracle.forward_rows(tiny["Q"], tiny["K"], tiny["V"], 128, 4, p["counts"], p["idx"],
                               p["pi_sel"], tiny["scale"])
    e_topk = _rel_l2(O, tiny["Od"])
    e_sip = float(np.mean(errs))
    print(f"rel-L2 vs dense: SIP mean {e_sip:.4f} (16 seeds), top-k {e_topk:.4f}, "
          f"SIP/top-k = {e_sip / e_topk:.3f}")
    assert e_sip < e_topk
