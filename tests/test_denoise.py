"""Denoising-loop harness: the policy's schedule (CPU) and, on the GPU, that
every attention call the harness makes equals the same library call made
directly (dense steps, plan steps, reused plans), and that a sparse step on a
reused plan matches the CPU oracle's forward on that plan."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle

from block_sparse_attention_12_b200 import denoise, inputs
from block_sparse_attention_12_b200.denoise import DENSE, PLAN_SPARSE, SPARSE, Policy, schedule


def test_schedule_default_policy():
    p = Policy()
    s = schedule(p, 40)
    assert len(s) == 50 and all(len(r) == 40 for r in s)
    assert all(a == DENSE for r in s[:10] for a in r)       # dense warm-up steps
    assert all(r[0] == DENSE for r in s)                     # the first block stays dense
    flat = [a for r in s[10:] for a in r[1:]]
    assert flat.count(PLAN_SPARSE) == 39 * 10                # steps 10, 14, ..., 46
    assert flat.count(SPARSE) == 39 * 30
    assert [t for t in range(50) if s[t][1] == PLAN_SPARSE] == list(range(10, 50, 4))


@pytest.mark.parametrize("steps,dense_steps,every,dense_layers,layers", [
    (7, 2, 3, 1, 2), (5, 0, 1, 0, 3), (4, 9, 2, 1, 2), (9, 1, 4, 2, 3)])
def test_schedule_rules(steps, dense_steps, every, dense_layers, layers):
    s = schedule(Policy(steps, dense_steps, every, dense_layers), layers)
    last_plan = [None] * layers
    for t, row in enumerate(s):
        for i, a in enumerate(row):
            if t < dense_steps or i < dense_layers:
                assert a == DENSE
            else:
                assert a in (PLAN_SPARSE, SPARSE)
                if a == PLAN_SPARSE:
                    last_plan[i] = t
                assert last_plan[i] is not None and t - last_plan[i] < every  # a plan exists and is recent


def test_schedule_rejects_bad_policy():
    with pytest.raises(ValueError):
        schedule(Policy(plan_every=0), 2)


def _same_plan(p, q):
    """Equal counts and equal entries up to each row's count (the slots past
    a row's count are not written by the planner)."""
    if not torch.equal(p.counts, q.counts):
        return False
    n = p.counts.flatten().tolist()
    pi, qi = p.idx.flatten(0, 2), q.idx.flatten(0, 2)
    ps, qs = p.pi_sel.flatten(0, 2), q.pi_sel.flatten(0, 2)
    return all(torch.equal(pi[r, :c], qi[r, :c]) and torch.equal(ps[r, :c], qs[r, :c]) for r, c in enumerate(n))


@pytest.mark.gpu
def test_harness_calls_equal_direct_calls():
    from block_sparse_attention_12_b200 import abi
    w = dataclasses.replace(inputs.TINY, H=1)
    pol = Policy(steps=7, dense_steps=2, plan_every=3, dense_layers=1)
    res = denoise.run(w, pol, layers=2, keep_outputs=True)
    assert res["counts"] == {DENSE: 2 * 2 + 5, PLAN_SPARSE: 2, SPARSE: 3}
    L, cfg = res["layers"], res["cfg"]
    sched = schedule(pol, 2)
    last = [None, None]
    anchored = False
    for t, row in enumerate(sched):
        for lay in L:
            lay.set_step(t)
        for i, a in enumerate(row):
            O, lse, plan = res["record"][(t, i)]
            lay = L[i]
            if a == DENSE:
                Od, ld = abi.dense_forward(lay.Q, lay.K, lay.V)
                assert torch.equal(O, Od) and torch.equal(lse, ld)
                continue
            if a == PLAN_SPARSE:
                assert _same_plan(plan, abi.plan(lay.Q, lay.K, cfg))  # the plan on this step's activations
                last[i] = plan
            else:  # a reused plan is the one made at the layer's last plan step
                assert _same_plan(plan, last[i])
            Os, ls = abi.forward(lay.Q, lay.K, lay.V, plan, cfg)
            assert torch.equal(O, Os) and torch.equal(lse, ls)
            if a == SPARSE and not anchored:
                # the oracle's forward on the plan the harness reused, with this
                # step's activations: max-abs 2e-2 on |err| / max(1, |O|), rel-L2 5e-3
                Oo, lo = oracle.forward_rows(lay.Q.cpu(), lay.K.cpu(), lay.V.cpu(), 128, w.kv_block,
                                             plan.counts.cpu().numpy(), plan.idx.cpu().numpy(),
                                             plan.pi_sel.cpu().numpy(), 1 / math.sqrt(w.d))
                Og = O.float().cpu().numpy().astype(np.float64)
                assert (np.abs(Og - Oo) / np.maximum(1.0, np.abs(Oo))).max() <= 2e-2
                assert np.linalg.norm(Og - Oo) / np.linalg.norm(Oo) <= 5e-3
                anchored = True
    assert anchored
    abi.check()
    # (per-call times solved from these tiny, launch-bound steps mean little;
    # the bench reports them on the full-size layers)
    assert all(math.isfinite(x) for x in denoise.per_call_ms(pol, res, 2))
