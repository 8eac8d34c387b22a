"""GPU path vs the CPU oracle, through the C ABI (tiny and small shapes).

Tolerances: plan bit-exact when fed the oracle's float32 pi; scores within
1e-3 relative (entries >= 1e-6 of the row max; smaller ones 1e-9 absolute);
pi from the GPU water-fill within 1e-5 relative; forward within max-abs 2e-2
and relative-L2 5e-3 of the oracle on the same plan (bf16 inputs, fp32
accumulation).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_12_b200 import abi, inputs

pytestmark = pytest.mark.gpu

W = inputs.TINY
SCALE = 1 / math.sqrt(W.d)


def cfg_of(w, **kw):
    c = abi.Config(kv_block=w.kv_block, budget=w.budget, n_clusters=w.n_clusters,
                   kmeans_iters=w.kmeans_iters, seed=w.seed)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def assert_forward_close(Og, Oo, what=""):
    """max-abs 2e-2 on |error| / max(1, |O|) (absolute at unit scale; bf16
    outputs above 4 are themselves rounded by more than 2e-2) and
    relative-L2 5e-3."""
    Og = np.asarray(Og, dtype=np.float64)
    err = (np.abs(Og - Oo) / np.maximum(1.0, np.abs(Oo))).max()
    rel = np.linalg.norm(Og - Oo) / max(np.linalg.norm(Oo), 1e-30)
    assert err <= 2e-2 and rel <= 5e-3, f"{what}: max-abs {err:.3e}, rel-L2 {rel:.3e}"
    return err, rel


def assert_scores_close(Sg, So):
    Sg = np.asarray(Sg, dtype=np.float64)
    mx = So.max(axis=-1, keepdims=True)
    big = So >= 1e-6 * mx
    rel = np.abs(Sg - So) / np.maximum(So, 1e-300)
    assert rel[big].max() <= 1e-3, rel[big].max()
    assert np.abs(Sg - So)[~big].max(initial=0) <= 1e-9


@pytest.fixture(scope="module")
def tiny():
    Qc, Kc, Vc = inputs.make_qkv(W)
    sel = oracle.selector_all(Qc, Kc, 128, W.kv_block, W.n_clusters, W.kmeans_iters, SCALE)
    return dict(Qc=Qc, Kc=Kc, Vc=Vc, Q=Qc.cuda(), K=Kc.cuda(), V=Vc.cuda(), sel=sel)


# ------------------------------------------------------------------ selector

def test_library_loads_and_reports_version():
    assert "sm_100a" in abi.version()


def test_meanpool_parity(tiny):
    Kb = abi.meanpool(tiny["K"], W.kv_block)
    abi.check()
    np.testing.assert_allclose(Kb.cpu().numpy(), tiny["sel"]["Kbar"], rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("kb,N", [(128, 300), (8, 4096), (4, 1000)])
def test_meanpool_ragged(kb, N):
    K = torch.randn(1, 3, N, 64, generator=torch.Generator().manual_seed(N)).to(torch.bfloat16)
    Kb = abi.meanpool(K.cuda(), kb)
    abi.check()
    for h in range(3):
        np.testing.assert_allclose(Kb[0, h].cpu().numpy(), oracle.meanpool(K[0, h], kb), rtol=1e-6, atol=1e-6)


def test_kmeans_parity(tiny):
    cfg = cfg_of(W)
    C, w, lab = abi.kmeans(tiny["Q"], cfg)
    abi.check()
    C, w, lab = C.cpu().numpy(), w.cpu().numpy(), lab.cpu().numpy()
    So = tiny["sel"]
    agree_rows, agree_lab = 0, 0
    nrows = lab.shape[2] * lab.shape[1]
    for h in range(W.H):
        for qb in range(lab.shape[2]):
            lo = So["labels"][0, h, qb]
            lg = lab[0, h, qb]
            agree_lab += (lo == lg).sum()
            if np.array_equal(lo, lg):
                agree_rows += 1
                np.testing.assert_allclose(C[0, h, qb], So["C"][0, h, qb], rtol=1e-5, atol=1e-5)
                np.testing.assert_array_equal(w[0, h, qb], So["w"][0, h, qb].astype(np.float32))
    print(f"k-means: {agree_rows}/{nrows} rows identical, label agreement {agree_lab / (nrows * 128):.5f}")
    assert agree_lab / (nrows * 128) >= 0.99
    assert agree_rows >= 0.9 * nrows


@pytest.mark.parametrize("d", [64, 128])
def test_kmeans_ragged_block_and_few_clusters(d):
    N = 1000
    Q = torch.randn(1, 2, N, d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    cfg = abi.Config(n_clusters=5, kmeans_iters=7)
    C, w, lab = abi.kmeans(Q.cuda(), cfg)
    abi.check()
    qb = N // 128  # ragged block, 104 rows
    Co, wo, lo = oracle.kmeans(Q[0, 1, qb * 128:], 5, 7)
    lg = lab[0, 1, qb].cpu().numpy()
    assert np.all(lg[N - qb * 128:] == -1)
    np.testing.assert_array_equal(lg[:N - qb * 128], lo)
    np.testing.assert_allclose(C[0, 1, qb].cpu().numpy(), Co, rtol=1e-5, atol=1e-5)
    np.testing.assert_array_equal(w[0, 1, qb].cpu().numpy(), wo.astype(np.float32))


def test_kmeans_degenerate_cases():
    """No iterations (the initial centroids, equal weights) and a block of
    identical queries (every distance ties, so every query joins cluster 0)."""
    N, d = 256, 64
    g = torch.Generator().manual_seed(9)
    Q = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    Q[0, 0, 128:] = Q[0, 0, 128]
    C0, w0, lab0 = abi.kmeans(Q.cuda(), abi.Config(kmeans_iters=0))
    C, w, lab = abi.kmeans(Q.cuda(), abi.Config(kmeans_iters=10))
    abi.check()
    for qb in range(2):
        Co, wo, lo = oracle.kmeans(Q[0, 0, qb * 128:(qb + 1) * 128], 8, 0)
        np.testing.assert_array_equal(C0[0, 0, qb].cpu().numpy(), Co.astype(np.float32))
        np.testing.assert_array_equal(w0[0, 0, qb].cpu().numpy(), wo.astype(np.float32))
        np.testing.assert_array_equal(lab0[0, 0, qb].cpu().numpy(), lo)  # -1: no query assigned
    Co, wo, lo = oracle.kmeans(Q[0, 0, 128:], 8, 10)
    np.testing.assert_array_equal(lab[0, 0, 1].cpu().numpy(), lo)
    assert np.all(lo == 0) and wo[0] == 1.0
    np.testing.assert_array_equal(w[0, 0, 1].cpu().numpy(), wo.astype(np.float32))
    np.testing.assert_allclose(C[0, 0, 1].cpu().numpy(), Co, rtol=1e-6, atol=1e-6)


def test_score_parity_fed_inputs(tiny):
    """Scores from the oracle's own centroids, weights and mean keys (rounded
    to float32, the kernel's input type), against the oracle on the same
    rounded inputs."""
    So = tiny["sel"]
    C32 = torch.from_numpy(So["C"]).float()
    w32 = torch.from_numpy(So["w"]).float()
    K32 = torch.from_numpy(So["Kbar"]).float()
    Sg = abi.score(C32.cuda(), w32.cuda(), K32.cuda(), tuple(tiny["Q"].shape), cfg_of(W))
    abi.check()
    Sg = Sg.cpu().numpy()
    for h in range(W.H):
        for qb in range(0, Sg.shape[2], 3):
            so = oracle.scores(C32[0, h, qb].double(), w32[0, h, qb].double(), K32[0, h].double(), SCALE)
            assert_scores_close(Sg[0, h, qb], so)
            assert abs(Sg[0, h, qb].sum() - 1) < 1e-4


def test_score_parity_end_to_end(tiny):
    cfg = cfg_of(W)
    shape = tuple(tiny["Q"].shape)
    Kb = abi.meanpool(tiny["K"], W.kv_block)
    C, w, lab = abi.kmeans(tiny["Q"], cfg)
    Sg = abi.score(C, w, Kb, shape, cfg)
    abi.check()
    Sg, lab = Sg.cpu().numpy(), lab.cpu().numpy()
    So = tiny["sel"]
    checked = 0
    for h in range(W.H):
        for qb in range(Sg.shape[2]):
            if np.array_equal(lab[0, h, qb], So["labels"][0, h, qb]):
                assert_scores_close(Sg[0, h, qb], So["S"][0, h, qb])
                checked += 1
    assert checked >= 0.9 * W.H * Sg.shape[2]


# ------------------------------------------------------------------ planner

def test_plan_from_pi_bit_exact(tiny):
    cfg = cfg_of(W)
    shape = tuple(tiny["Q"].shape)
    po = oracle.plan_all(tiny["sel"]["S"], W.budget, 0, W.seed, want_pi=True)
    pi = torch.from_numpy(po["pi"])
    pg = abi.plan_from_pi(pi.cuda(), shape, cfg)
    abi.check()
    assert pg.cap == po["cap"]
    cg = pg.counts.cpu().numpy()
    np.testing.assert_array_equal(cg, po["counts"])
    ig, sg = pg.idx.cpu().numpy(), pg.pi_sel.cpu().numpy()
    for r in np.ndindex(cg.shape):
        n = cg[r]
        np.testing.assert_array_equal(ig[r][:n], po["idx"][r][:n])
        np.testing.assert_array_equal(sg[r][:n], po["pi_sel"][r][:n])


@pytest.mark.parametrize("seed", [0, 1, 2**40 + 7])
def test_plan_from_pi_bit_exact_random_pi(seed):
    B, H, N, d = 2, 3, 2000, 64
    nqb, nkvb = -(-N // 128), N // 4
    g = np.random.default_rng(seed % 1000)
    pi = g.random((B, H, nqb, nkvb)).astype(np.float32) ** 3
    pi[..., ::17] = 1.0
    pi[..., 5::23] = 0.0
    cfg = abi.Config(kv_block=4, budget=0.3, seed=seed)
    pg = abi.plan_from_pi(torch.from_numpy(pi).cuda(), (B, H, N, d), cfg)
    abi.check()
    cg, ig, sg = pg.counts.cpu().numpy(), pg.idx.cpu().numpy(), pg.pi_sel.cpu().numpy()
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                idx, ps, n = oracle.sample(pi[b, h, qb], seed, b, h, qb, pg.cap)
                assert cg[b, h, qb] == min(n, pg.cap)
                np.testing.assert_array_equal(ig[b, h, qb, :cg[b, h, qb]], idx)
                np.testing.assert_array_equal(sg[b, h, qb, :cg[b, h, qb]], ps)


def test_waterfill_pi_parity(tiny):
    cfg = cfg_of(W)
    shape = tuple(tiny["Q"].shape)
    S32 = torch.from_numpy(tiny["sel"]["S"]).float()
    pg, pig = abi.plan_from_scores(S32.cuda(), shape, cfg, want_pi=True)
    abi.check()
    pig = pig.cpu().numpy()
    S64 = S32.double().numpy()
    po = oracle.plan_all(S64, W.budget, 0, W.seed, want_pi=True)
    rel = np.abs(pig - po["pi"]) / np.maximum(po["pi"], 1e-30)
    assert rel.max() <= 1e-5
    exact = np.mean(pig == po["pi"])
    print(f"water-fill: {exact:.6f} of pi bit-identical, max rel {rel.max():.2e}")
    # when every pi agrees bit for bit, so must the sampled plan
    if exact == 1.0:
        np.testing.assert_array_equal(pg.counts.cpu().numpy(), po["counts"])


def _fallback_rows(n, rng):
    """Score rows for the water-fill's fallback paths (n = 4096 blocks, 8%
    budget; the kernel lists as capping candidates the blocks within a factor
    32 of the first threshold): (a) lambda grows past 32 times its first
    value, so the rounds after the first scan the whole row (and cap 100 more
    blocks); (b) more than 2048 blocks qualify as candidates, so the list
    overflows and the later rounds scan the row; (c) an ordinary heavy-tailed
    row;
    (d) the same row normalised to sum 1, as scores are, whose candidates are
    listed while the row loads; (e) row (d) times 1/4, whose sum is below 1/2,
    so the first round scans the row instead."""
    a = np.concatenate([np.full(60, 1e6), np.full(100, 40.0), np.full(n - 160, 1.0)])
    b = np.concatenate([np.full(60, 2000.0), np.full(200, 500.0), np.full(2100, 40.0), np.full(n - 2360, 0.1)])
    c = np.exp(rng.standard_normal(n) * 2.0)
    d = np.exp(rng.standard_normal(n) * 3.0)
    d = d / d.sum()
    for r in (a, b):
        rng.shuffle(r)
    return [a, b, c, d, d * 0.25]


def test_waterfill_fallback_paths():
    B, H, N, d = 1, 1, 16384, 64
    cfg = abi.Config(kv_block=4, budget=0.08, seed=11)
    n = N // 4
    Bblk = cfg.budget * n
    rng = np.random.default_rng(5)
    rows = _fallback_rows(n, rng)
    # the rows take the paths they are built for
    lam0 = [Bblk / r.sum() for r in rows]
    pis = [oracle.waterfill(r, Bblk) for r in rows]
    assert pis[0][1] / lam0[0] > 32
    assert ((rows[1] * 32 * lam0[1] >= 1) & (rows[1] * lam0[1] < 1)).sum() > 2048
    assert (pis[0][0] >= 1).sum() == 160 and (pis[1][0] >= 1).sum() == 60
    S = np.tile(rows[2], (N // 128, 1))
    S[:2] = rows[0], rows[1]
    S[3:5] = rows[3], rows[4]
    S32 = torch.from_numpy(S.astype(np.float32)).reshape(B, H, N // 128, n)
    pg, pig = abi.plan_from_scores(S32.cuda(), (B, H, N, d), cfg, want_pi=True)
    abi.check()
    pig = pig.cpu().numpy()[0, 0]
    counts, idx, ps = (t.cpu().numpy()[0, 0] for t in (pg.counts, pg.idx, pg.pi_sel))
    for qb in (0, 1, 2, 3, 4, N // 128 - 1):
        po, _, _ = oracle.waterfill(S32[0, 0, qb].double().numpy(), Bblk)
        assert np.max(np.abs(pig[qb] - po) / np.maximum(po, 1e-30)) <= 1e-5, qb
        idx_o, ps_o, n_o = oracle.sample(pig[qb], cfg.seed, 0, 0, qb, pg.cap)
        assert counts[qb] == min(n_o, pg.cap)
        np.testing.assert_array_equal(idx[qb, :counts[qb]], idx_o)
        np.testing.assert_array_equal(ps[qb, :counts[qb]], ps_o)


def test_head_offset_slices_equal_whole_layer(tiny):
    """A rank holding a slice of the heads plans it with head_offset = the
    slice's first global head: its plan and output equal those rows of the
    whole layer's (bit for bit), its plan is the oracle's sample of its own pi
    with the global head index, its forward matches the oracle's, and without
    the offset the plan differs."""
    cfg = cfg_of(W)
    full = abi.plan(tiny["Q"], tiny["K"], cfg)
    Of, lf = abi.forward(tiny["Q"], tiny["K"], tiny["V"], full, cfg)
    n_full = full.counts.cpu().numpy()
    for lo in range(W.H):
        Qs, Ks, Vs = (t[:, lo:lo + 1].contiguous() for t in (tiny["Q"], tiny["K"], tiny["V"]))
        cs = cfg_of(W, head_offset=lo)
        ps = abi.plan(Qs, Ks, cs)
        Os, ls = abi.forward(Qs, Ks, Vs, ps, cs)
        abi.check()
        n = ps.counts.cpu().numpy()
        np.testing.assert_array_equal(n[0, 0], n_full[0, lo])
        for qb in range(n.shape[2]):
            c = n[0, 0, qb]
            assert torch.equal(ps.idx[0, 0, qb, :c], full.idx[0, lo, qb, :c])
            assert torch.equal(ps.pi_sel[0, 0, qb, :c], full.pi_sel[0, lo, qb, :c])
        assert torch.equal(Os[0, 0], Of[0, lo]) and torch.equal(ls[0, 0], lf[0, lo])
    # the oracle draws with the global head index: the last head's slice,
    # planned alone with its head_offset, samples exactly the oracle's plan of
    # the slice's own pi, and its forward on that plan matches the oracle's
    lo = W.H - 1
    Qs, Ks, Vs = (t[:, lo:lo + 1].contiguous() for t in (tiny["Q"], tiny["K"], tiny["V"]))
    cs = cfg_of(W, head_offset=lo)
    shape_s = tuple(Qs.shape)
    Kb = abi.meanpool(Ks, W.kv_block)
    C, wt, _ = abi.kmeans(Qs, cs)
    S = abi.score(C, wt, Kb, shape_s, cs)
    pl, pi = abi.plan_from_scores(S, shape_s, cs, want_pi=True)
    abi.check()
    pi_np = pi.cpu().numpy()
    cnt, idx, pss = pl.counts.cpu().numpy(), pl.idx.cpu().numpy(), pl.pi_sel.cpu().numpy()
    for qb in range(cnt.shape[2]):
        idx_o, ps_o, n_o = oracle.sample(pi_np[0, 0, qb], W.seed, 0, lo, qb, pl.cap)
        assert cnt[0, 0, qb] == min(n_o, pl.cap)
        np.testing.assert_array_equal(idx[0, 0, qb, :cnt[0, 0, qb]], idx_o)
        np.testing.assert_array_equal(pss[0, 0, qb, :cnt[0, 0, qb]], ps_o)
    Os, _ = abi.forward(Qs, Ks, Vs, pl, cs)
    abi.check()
    Oo, _ = oracle.forward_rows(Qs.cpu(), Ks.cpu(), Vs.cpu(), 128, W.kv_block, cnt, idx, pss, SCALE)
    assert_forward_close(Os.float().cpu().numpy(), Oo, "head slice")
    # head 1 planned as if it were head 0 draws other uniforms
    p0 = abi.plan(tiny["Q"][:, 1:2].contiguous(), tiny["K"][:, 1:2].contiguous(), cfg_of(W))
    abi.check()
    differs = any(not torch.equal(p0.idx[0, 0, qb, :int(p0.counts[0, 0, qb])],
                                  full.idx[0, 1, qb, :int(full.counts[0, 1, qb])])
                  for qb in range(p0.counts.shape[2]))
    assert differs


def test_topk_bit_exact_from_fp32_scores(tiny):
    cfg = cfg_of(W, mode=abi.MODE_TOPK)
    shape = tuple(tiny["Q"].shape)
    S32 = torch.from_numpy(tiny["sel"]["S"]).float()
    S32[0, 0, 0, 10:40] = S32[0, 0, 0, 10]  # ties across the threshold
    pg = abi.plan_from_scores(S32.cuda(), shape, cfg)
    abi.check()
    po = oracle.plan_all(S32.double().numpy(), W.budget, 1, 0)
    np.testing.assert_array_equal(pg.counts.cpu().numpy(), po["counts"])
    k = int(po["counts"].reshape(-1)[0])
    np.testing.assert_array_equal(pg.idx.cpu().numpy()[..., :k], po["idx"][..., :k])
    assert np.all(pg.pi_sel.cpu().numpy()[..., :k] == 1.0)


def test_plan_overflow_is_reported():
    B, H, N, d = 1, 1, 1024, 64
    nkvb = N // 4
    cfg = abi.Config(kv_block=4, budget=0.05)
    cap = abi.capacity((B, H, N, d), cfg)
    pi = torch.ones(B, H, N // 128, nkvb, dtype=torch.float32, device="cuda")
    pg = abi.plan_from_pi(pi, (B, H, N, d), cfg)
    with pytest.raises(abi.AbattnError) as e:
        abi.check()
    assert e.value.code == abi.ERR_PLAN_OVERFLOW
    assert np.all(pg.counts.cpu().numpy() == cap)
    abi.check()  # the error word was cleared


# ------------------------------------------------------------------ forward

def _oracle_forward(Q, K, V, plan, kb, rows=None, scale=None):
    return oracle.forward_rows(Q, K, V, 128, kb, plan.counts.cpu().numpy(), plan.idx.cpu().numpy(),
                               plan.pi_sel.cpu().numpy(), scale if scale else 1 / math.sqrt(Q.shape[-1]),
                               rows=rows)


def test_sparse_forward_parity_tiny(tiny):
    cfg = cfg_of(W)
    plan = abi.plan(tiny["Q"], tiny["K"], cfg)
    O, lse = abi.forward(tiny["Q"], tiny["K"], tiny["V"], plan, cfg)
    abi.check()
    Oo, lo = _oracle_forward(tiny["Qc"], tiny["Kc"], tiny["Vc"], plan, W.kv_block)
    assert_forward_close(O.float().cpu().numpy(), Oo, "sparse tiny")
    np.testing.assert_allclose(lse.cpu().numpy(), lo, atol=2e-3, rtol=1e-4)


def test_dense_forward_parity_tiny(tiny):
    O, lse = abi.dense_forward(tiny["Q"], tiny["K"], tiny["V"])
    abi.check()
    Qd, Kd, Vd = (oracle.f64(t) for t in (tiny["Qc"], tiny["Kc"], tiny["Vc"]))
    for h in range(W.H):
        Oo, lo = oracle.dense(Qd[0, h], Kd[0, h], Vd[0, h], SCALE)
        assert_forward_close(O[0, h].float().cpu().numpy(), Oo, f"dense h{h}")
        np.testing.assert_allclose(lse[0, h].cpu().numpy(), lo, atol=2e-3, rtol=1e-4)


def test_full_plan_equals_dense(tiny):
    shape = tuple(tiny["Q"].shape)
    plan = abi.full_plan(shape, 4)
    Os, ls = abi.forward(tiny["Q"], tiny["K"], tiny["V"], plan, abi.Config(kv_block=4))
    Od, ld = abi.dense_forward(tiny["Q"], tiny["K"], tiny["V"])
    abi.check()
    assert_forward_close(Os.float().cpu().numpy(), Od.float().cpu().numpy().astype(np.float64), "full vs dense")
    np.testing.assert_allclose(ls.cpu().numpy(), ld.cpu().numpy(), atol=1e-3)


def test_batch_of_two_indexes_rows_by_batch():
    """B = 2 (every workload above has B = 1): each stage indexes its rows as
    (b, h, qb) and the plan's Philox counter carries b.  Mean keys, k-means and
    scores (fed the oracle's inputs) against the oracle; the plan bit for bit
    from the oracle's pi; the forward against the oracle on the GPU's plan."""
    B, H, N, d, kb = 2, 2, 1000, 128, 4
    g = torch.Generator().manual_seed(11)
    Qc, Kc, Vc = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    cfg = abi.Config(kv_block=kb, budget=0.2, seed=5)
    Q, K, V = Qc.cuda(), Kc.cuda(), Vc.cuda()
    shape, scale = (B, H, N, d), 1 / math.sqrt(d)
    sel = oracle.selector_all(Qc, Kc, 128, kb, cfg.n_clusters, cfg.kmeans_iters, scale)
    Kb = abi.meanpool(K, kb)
    C, w, lab = abi.kmeans(Q, cfg)
    abi.check()
    np.testing.assert_allclose(Kb.cpu().numpy(), sel["Kbar"], rtol=1e-6, atol=1e-6)
    assert (lab.cpu().numpy() == sel["labels"]).mean() >= 0.99
    C32, w32, K32 = (torch.from_numpy(sel[k]).float() for k in ("C", "w", "Kbar"))
    Sg = abi.score(C32.cuda(), w32.cuda(), K32.cuda(), shape, cfg).cpu().numpy()
    abi.check()
    for b, h, qb in np.ndindex(B, H, 8):
        so = oracle.scores(C32[b, h, qb].double(), w32[b, h, qb].double(), K32[b, h].double(), scale)
        assert_scores_close(Sg[b, h, qb], so)
    po = oracle.plan_all(sel["S"], cfg.budget, 0, cfg.seed, want_pi=True)
    pg = abi.plan_from_pi(torch.from_numpy(po["pi"]).cuda(), shape, cfg)
    abi.check()
    cg, ig, sg = pg.counts.cpu().numpy(), pg.idx.cpu().numpy(), pg.pi_sel.cpu().numpy()
    np.testing.assert_array_equal(cg, po["counts"])
    for r in np.ndindex(cg.shape):
        np.testing.assert_array_equal(ig[r][:cg[r]], po["idx"][r][:cg[r]])
        np.testing.assert_array_equal(sg[r][:cg[r]], po["pi_sel"][r][:cg[r]])
    plan = abi.plan(Q, K, cfg)
    O, lse = abi.forward(Q, K, V, plan, cfg)
    abi.check()
    Oo, lo = _oracle_forward(Qc, Kc, Vc, plan, kb)
    assert_forward_close(O.float().cpu().numpy(), Oo, "B = 2")
    np.testing.assert_allclose(lse.cpu().numpy(), lo, atol=2e-3, rtol=1e-4)


def _climbing_logits(N, d, step_log2=40.0, seed=0):
    """Q, K, V in bf16 whose scaled logits (log2 units) climb by about
    step_log2 per 128-key tile for the first 64 queries of every q-block: each
    tile raises those rows' running max by more than the forward's lazy
    rescale threshold (a factor 2^32), so their O is rescaled at every tile.
    The other 64 queries see logits of a few units and never rescale, so one
    warpgroup holds warps on both paths."""
    g = torch.Generator().manual_seed(seed)
    Q = 0.05 * torch.randn(1, 1, N, d, generator=g)
    K = 0.5 * torch.randn(1, 1, N, d, generator=g)
    V = torch.randn(1, 1, N, d, generator=g)
    Q[0, 0, (torch.arange(N) % 128) < 64, 0] = 8.0
    tile = (torch.arange(N) // 128).double()
    K[0, 0, :, 0] = (step_log2 * tile * math.sqrt(d) / (8.0 * math.log2(math.e))
                     + 0.5 * torch.randn(N, generator=g, dtype=torch.float64)).float()
    return tuple(t.to(torch.bfloat16) for t in (Q, K, V))


# N % 4 == 0: per-group bias path of the sparse kernel; otherwise per key
@pytest.mark.parametrize("d,N", [(128, 1024), (64, 1000), (128, 1001)])
def test_lazy_rescale_on_climbing_logits(d, N):
    Qc, Kc, Vc = _climbing_logits(N, d)
    Q, K, V = Qc.cuda(), Kc.cuda(), Vc.cuda()
    Oo, lo = oracle.dense(Qc[0, 0], Kc[0, 0], Vc[0, 0], 1 / math.sqrt(d))
    assert lo[:64].max() > 100.0  # the climbing rows reach logits far past the threshold
    Od, ld = abi.dense_forward(Q, K, V)
    plan = abi.full_plan(tuple(Q.shape), 4)
    Os, ls = abi.forward(Q, K, V, plan, abi.Config(kv_block=4))
    abi.check()
    for O, lse, what in ((Od, ld, "dense"), (Os, ls, "sparse, full plan")):
        assert_forward_close(O[0, 0].float().cpu().numpy(), Oo, f"{what} d{d} N{N}")
        np.testing.assert_allclose(lse[0, 0].cpu().numpy(), lo, atol=2e-3, rtol=1e-4, err_msg=what)


# N % 4 == 0 takes the kernel's per-group bias path, the rest its per-key path
@pytest.mark.parametrize("d,N,kb,budget", [(128, 1000, 4, 0.2), (128, 300, 128, 0.5), (64, 777, 128, 1.0),
                                           (128, 640, 16, 0.3), (64, 2048, 8, 0.1), (128, 1234, 4, 0.25),
                                           (64, 1003, 32, 0.4),
                                           # degenerate: one query and one block, a few keys, one tile + 2
                                           (64, 1, 4, 1.0), (128, 5, 4, 0.5), (128, 130, 4, 0.3)])
def test_sparse_forward_ragged_shapes(d, N, kb, budget):
    g = torch.Generator().manual_seed(N + kb)
    Qc, Kc, Vc = (torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    cfg = abi.Config(kv_block=kb, budget=budget, seed=3)
    Q, K, V = Qc.cuda(), Kc.cuda(), Vc.cuda()
    plan = abi.plan(Q, K, cfg)
    O, lse = abi.forward(Q, K, V, plan, cfg)
    abi.check()
    Oo, lo = _oracle_forward(Qc, Kc, Vc, plan, kb)
    assert_forward_close(O.float().cpu().numpy(), Oo, f"d{d} N{N} kb{kb}")
    np.testing.assert_allclose(lse.cpu().numpy(), lo, atol=2e-3, rtol=1e-4)
    if N % 128:
        Od, _ = abi.dense_forward(Q, K, V)
        abi.check()
        Oo_d, _ = oracle.dense(Qc[0, 1], Kc[0, 1], Vc[0, 1], 1 / math.sqrt(d))
        assert_forward_close(Od[0, 1].float().cpu().numpy(), Oo_d, "dense ragged")


def test_empty_and_custom_plans():
    B, H, N, d = 1, 1, 512, 128
    g = torch.Generator().manual_seed(9)
    Qc, Kc, Vc = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    nqb = N // 128
    cap = 40
    counts = torch.tensor([[[0, 1, 33, 40]]], dtype=torch.int32)
    idx = torch.zeros(B, H, nqb, cap, dtype=torch.int32)
    ps = torch.zeros(B, H, nqb, cap, dtype=torch.float32)
    rng = np.random.default_rng(1)
    for qb in range(nqb):
        n = int(counts[0, 0, qb])
        sel = np.sort(rng.choice(N // 4, n, replace=False))
        idx[0, 0, qb, :n] = torch.from_numpy(sel.astype(np.int32))
        ps[0, 0, qb, :n] = torch.from_numpy(rng.uniform(0.01, 1, n).astype(np.float32))
    plan = abi.Plan(counts.cuda(), idx.cuda(), ps.cuda(), cap, 4)
    O, lse = abi.forward(Qc.cuda(), Kc.cuda(), Vc.cuda(), plan, abi.Config(kv_block=4))
    abi.check()
    Oo, lo = _oracle_forward(Qc, Kc, Vc, plan, 4)
    Og = O.float().cpu().numpy()
    assert np.all(Og[0, 0, :128] == 0) and np.all(np.isneginf(lse[0, 0, :128].cpu().numpy()))
    assert_forward_close(Og[0, 0, 128:], Oo[0, 0, 128:], "custom plan")


def test_bad_plan_index_is_skipped_and_reported():
    B, H, N, d = 1, 1, 256, 64
    Q = torch.randn(B, H, N, d, device="cuda").to(torch.bfloat16)
    counts = torch.tensor([[[2, 1]]], dtype=torch.int32, device="cuda")
    idx = torch.tensor([[[[3, 10**6], [-5, 0]]]], dtype=torch.int32, device="cuda")
    ps = torch.ones(1, 1, 2, 2, device="cuda")
    O, lse = abi.forward(Q, Q, Q, abi.Plan(counts, idx, ps, 2, 4), abi.Config(kv_block=4))
    with pytest.raises(abi.AbattnError) as e:
        abi.check()
    assert e.value.code == abi.ERR_BOUNDS
    assert torch.isfinite(O[0, 0, :128].float()).all()


def test_sip_beats_topk_on_gpu(tiny):
    """The HT-sampled forward is closer to dense than top-k truncation."""
    shape = tuple(tiny["Q"].shape)
    Od, _ = abi.dense_forward(tiny["Q"], tiny["K"], tiny["V"])
    errs = []
    for seed in range(8):
        cfg = cfg_of(W, seed=seed)
        plan = abi.plan(tiny["Q"], tiny["K"], cfg)
        O, _ = abi.forward(tiny["Q"], tiny["K"], tiny["V"], plan, cfg)
        errs.append(((O.float() - Od.float()).norm() / Od.float().norm()).item())
    cfg = cfg_of(W, mode=abi.MODE_TOPK)
    plan = abi.plan(tiny["Q"], tiny["K"], cfg)
    O, _ = abi.forward(tiny["Q"], tiny["K"], tiny["V"], plan, cfg)
    abi.check()
    e_top = ((O.float() - Od.float()).norm() / Od.float().norm()).item()
    print(f"GPU rel-L2 vs dense: SIP {np.mean(errs):.4f}, top-k {e_top:.4f}")
    assert np.mean(errs) < e_top
