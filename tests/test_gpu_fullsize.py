"""GPU path vs the CPU oracle at the workloads' full sizes, in the launch
configuration the benchmark times (abattn_plan + abattn_forward over whole
layers), checked on a seeded sample of (head, q-block) rows that the
oracle computes one by one; the ragged last q-block of a head is always in
the sample.

Per sampled row:
  * the plan of abattn_plan equals the plan of the staged entry points
    (meanpool -> kmeans -> score -> plan_from_scores);
  * k-means labels agree with the oracle (>= 99% of queries);
  * scores from the GPU's own centroids and weights match the oracle's
    within 1e-3 relative (entries >= 1e-6 of the row max);
  * the water-filled pi of the GPU's fp32 score row matches the oracle's
    within 1e-5 relative, and the sampled plan equals the oracle's sample of
    the GPU's pi bit for bit;
  * the forward output matches the oracle's forward on the GPU's plan within
    max-abs 2e-2 and relative-L2 5e-3.  The max-abs bound is stated for
    unit-scale values and applied per element through the error model of
    the kernel's P.V product: P is rounded to bf16 (relative error <= 2^-9)
    before it multiplies V, so the error of output element (i, c) is bounded
    by 2^-9 * A_ic with A_ic = sum_t p_it |v_tc|, the same softmax weights
    applied to |V| (the oracle's forward with |V| in place of V).  The bound
    is |error_ic| <= 2e-2 * max(1, A_ic): the plain absolute 2e-2 wherever
    A <= 1, scaled only where the row draws on large values (the 14B-like
    layer's x8 outlier tokens).  The layers without outliers are also held
    to the plain bound on |error| / max(1, |O|).  The relative-L2 bound is
    scale-free and applies unchanged.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_12_b200 import abi, inputs

pytestmark = pytest.mark.gpu

WORKLOADS = [inputs.WAN_1_3B, inputs.WAN_14B, inputs.HUNYUAN]


def check_forward(w, Og, Oo, Ao, what):
    """Max-abs 2e-2 per element on |error| / max(1, A) with A the oracle's
    forward on |V| (the bf16-P error model), the plain |error| / max(1, |O|)
    on layers without outlier tokens, and relative-L2 5e-3.  Prints the
    unscaled error so each layer's margin is on record."""
    e = np.abs(Og - Oo)
    err_a = (e / np.maximum(1.0, Ao)).max()
    err_o = (e / np.maximum(1.0, np.abs(Oo))).max()
    rel = np.linalg.norm(Og - Oo) / np.linalg.norm(Oo)
    print(f"{w.name} {what}: max|err| {e.max():.3e} (max A {Ao.max():.2f}), "
          f"err/max(1,A) {err_a:.3e}, err/max(1,|O|) {err_o:.3e}, rel-L2 {rel:.3e}")
    assert err_a <= 2e-2 and rel <= 5e-3, (what, err_a, rel)
    if w.outlier_frac == 0:
        assert err_o <= 2e-2, (what, err_o)


def _cfg(w, **kw):
    c = abi.Config(kv_block=w.kv_block, budget=w.budget, n_clusters=w.n_clusters,
                   kmeans_iters=w.kmeans_iters, seed=w.seed)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.fixture(scope="module", params=WORKLOADS, ids=[w.name for w in WORKLOADS])
def layer(request):
    w = request.param
    Qc, Kc, Vc = inputs.make_qkv(w)
    Q, K, V = Qc.cuda(), Kc.cuda(), Vc.cuda()
    shape = tuple(Q.shape)
    cfg = _cfg(w)
    plan = abi.Planner(shape, cfg)(Q, K)
    outs = []
    for _ in range(w.forwards_per_plan):
        O, lse = abi.forward(Q, K, V, plan, cfg)
        outs.append(O)
    # staged stages, same kernels
    Kb = abi.meanpool(K, w.kv_block)
    C, wt, lab = abi.kmeans(Q, cfg)
    S = abi.score(C, wt, Kb, shape, cfg)
    splan, pi = abi.plan_from_scores(S, shape, cfg, want_pi=True)
    abi.check()
    rows = inputs.row_sample(w, 6, seed=99)
    heads = sorted({h for _, h, _ in rows})
    data = {h: tuple(oracle.f64(t[0, h]) for t in (Qc, Kc, Vc)) for h in heads}
    yield dict(w=w, cfg=cfg, Q=Q, K=K, V=V, plan=plan, outs=outs, lse=lse, C=C, wt=wt, lab=lab, S=S,
               splan=splan, pi=pi, rows=rows, data=data)
    del Q, K, V
    torch.cuda.empty_cache()


def test_plan_call_equals_staged_stages(layer):
    p, q = layer["plan"], layer["splan"]
    assert torch.equal(p.counts, q.counts)
    n = p.counts.cpu().numpy()
    pi_, qi = p.idx.cpu().numpy(), q.idx.cpu().numpy()
    ps, qs = p.pi_sel.cpu().numpy(), q.pi_sel.cpu().numpy()
    for r in np.ndindex(n.shape):
        np.testing.assert_array_equal(pi_[r][:n[r]], qi[r][:n[r]])
        np.testing.assert_array_equal(ps[r][:n[r]], qs[r][:n[r]])


def test_repeated_forwards_on_one_plan_are_identical(layer):
    outs = layer["outs"]
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_sampled_rows_against_oracle(layer):
    w, rows, data = layer["w"], layer["rows"], layer["data"]
    scale = 1 / math.sqrt(w.d)
    nkvb = -(-w.N // w.kv_block)
    lab = layer["lab"].cpu().numpy()
    C = layer["C"].cpu().numpy()
    wt = layer["wt"].cpu().numpy()
    S = layer["S"]
    pi = layer["pi"]
    plan = layer["plan"]
    O = layer["outs"][0]
    for b, h, qb in rows:
        q, k, v = data[h]
        q0 = qb * 128
        M = min(128, w.N - q0)
        Kbar = oracle.meanpool(k, w.kv_block)
        # k-means labels
        _, _, lo = oracle.kmeans(q[q0:q0 + M], w.n_clusters, w.kmeans_iters)
        agree = np.mean(lab[b, h, qb, :M] == lo)
        assert agree >= 0.99, (h, qb, agree)
        # scores from the GPU's centroids / weights
        so = oracle.scores(C[b, h, qb].astype(np.float64), wt[b, h, qb].astype(np.float64), Kbar, scale)
        sg = S[b, h, qb].cpu().numpy().astype(np.float64)
        big = so >= 1e-6 * so.max()
        assert np.max(np.abs(sg - so)[big] / so[big]) <= 1e-3
        assert np.max(np.abs(sg - so)[~big], initial=0) <= 1e-9
        # water-fill of the GPU's fp32 scores and the plan sampled from the GPU's pi
        po, _, _ = oracle.waterfill(sg, w.budget * nkvb)
        pg = pi[b, h, qb].cpu().numpy()
        assert np.max(np.abs(pg - po) / np.maximum(po, 1e-30)) <= 1e-5
        idx_o, ps_o, n_o = oracle.sample(pg, w.seed, b, h, qb, plan.cap)
        n = int(plan.counts[b, h, qb])
        assert n == min(n_o, plan.cap)
        np.testing.assert_array_equal(plan.idx[b, h, qb, :n].cpu().numpy(), idx_o)
        np.testing.assert_array_equal(plan.pi_sel[b, h, qb, :n].cpu().numpy(), ps_o)
        # forward on the GPU's plan
        Oo, lo_ = oracle.sparse_block(q[q0:q0 + M], k, v, w.kv_block, idx_o, ps_o, scale)
        Ao, _ = oracle.sparse_block(q[q0:q0 + M], k, np.abs(v), w.kv_block, idx_o, ps_o, scale)
        Og = O[b, h, q0:q0 + M].float().cpu().numpy().astype(np.float64)
        check_forward(w, Og, Oo, Ao, f"sparse row (h {h}, qb {qb})")
        np.testing.assert_allclose(layer["lse"][b, h, q0:q0 + M].cpu().numpy(), lo_, atol=2e-3, rtol=1e-4)


def test_topk_rows_bit_exact_from_fp32_scores(layer):
    w = layer["w"]
    shape = tuple(layer["Q"].shape)
    cfg = _cfg(w, mode=abi.MODE_TOPK)
    p = abi.plan_from_scores(layer["S"], shape, cfg)
    abi.check()
    nkvb = -(-w.N // w.kv_block)
    k = int(math.floor(w.budget * nkvb + 0.5))
    for b, h, qb in layer["rows"]:
        s = layer["S"][b, h, qb].cpu().numpy().astype(np.float64)
        idx = oracle.topk(s, k)
        assert int(p.counts[b, h, qb]) == k
        np.testing.assert_array_equal(p.idx[b, h, qb, :k].cpu().numpy(), idx)


def test_dense_rows_against_oracle(layer):
    w = layer["w"]
    if w is not inputs.WAN_14B:
        pytest.skip("dense checked on the 14B-like layer")
    h = layer["rows"][0][1]
    Q, K, V = (t[:, h:h + 1].contiguous() for t in (layer["Q"], layer["K"], layer["V"]))
    O, lse = abi.dense_forward(Q, K, V)
    abi.check()
    q, k, v = layer["data"][h]
    for q0 in (0, 128 * 300, w.N - 16):
        Oo, lo = oracle.dense(q[q0:q0 + 16], k, v, 1 / math.sqrt(w.d))
        Ao, _ = oracle.dense(q[q0:q0 + 16], k, np.abs(v), 1 / math.sqrt(w.d))
        Og = O[0, 0, q0:q0 + 16].float().cpu().numpy().astype(np.float64)
        check_forward(w, Og, Oo, Ao, f"dense rows {q0}..{q0 + 15} (h {h})")
        np.testing.assert_allclose(lse[0, 0, q0:q0 + 16].cpu().numpy(), lo, atol=2e-3, rtol=1e-4)


def test_e4m3_forward_rows_against_oracle(layer):
    """The E4M3 forward on the layer's plan, for the sampled rows: against the
    oracle on the dequantised Q and K (same bound as the bf16 forward), and its
    rel-L2 against the oracle on the bf16 inputs printed."""
    w, plan, cfg = layer["w"], layer["plan"], layer["cfg"]
    if w.d != 128:
        pytest.skip("the E4M3 forward takes d = 128")
    Q8, qs = abi.quantize_e4m3(layer["Q"], 128)
    K8, ks = abi.quantize_e4m3(layer["K"], w.kv_block)
    O8, lse8 = abi.forward_e4m3(Q8, qs, K8, ks, layer["V"], plan, cfg)
    abi.check()
    scale = 1 / math.sqrt(w.d)
    for b, h, qb in layer["rows"][:3]:
        _, _, v = layer["data"][h]
        q0 = qb * 128
        M = min(128, w.N - q0)
        qd = oracle.dequantize_e4m3_rows(Q8[b, h].cpu().numpy(), qs[b, h].cpu().numpy(), 128)[q0:q0 + M]
        kd = oracle.dequantize_e4m3_rows(K8[b, h].cpu().numpy(), ks[b, h].cpu().numpy(), w.kv_block)
        n = int(plan.counts[b, h, qb])
        idx = plan.idx[b, h, qb, :n].cpu().numpy()
        ps = plan.pi_sel[b, h, qb, :n].cpu().numpy()
        Oo, lo_ = oracle.sparse_block(qd, kd, v, w.kv_block, idx, ps, scale)
        Ao, _ = oracle.sparse_block(qd, kd, np.abs(v), w.kv_block, idx, ps, scale)
        Og = O8[b, h, q0:q0 + M].float().cpu().numpy().astype(np.float64)
        check_forward(w, Og, Oo, Ao, f"E4M3 row (h {h}, qb {qb})")
        np.testing.assert_allclose(lse8[b, h, q0:q0 + M].cpu().numpy(), lo_, atol=2e-3, rtol=1e-4)
        q, k, _ = layer["data"][h]
        Ox, _ = oracle.sparse_block(q[q0:q0 + M], k, v, w.kv_block, idx, ps, scale)
        print(f"{w.name} E4M3 row (h {h}, qb {qb}) vs the bf16 inputs: rel-L2 "
              f"{np.linalg.norm(Og - Ox) / np.linalg.norm(Ox):.3e}")
