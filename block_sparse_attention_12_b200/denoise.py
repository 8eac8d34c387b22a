"""Synthetic denoising-loop harness for the AB-Attention hot path.

The AB-Attention news page (hamidun, Arabic), section "how it was measured":
the first 10 of 50 denoising steps and the first transformer block run dense
attention; the other steps and blocks run AB-Attention. Section "three
techniques", fine-grained kernel paragraph: the plan (selector + SIP) is
recomputed once every 4 steps and reused in between.

This module drives that policy over synthetic layers whose activations drift
from step to step, through the C-ABI binding (`abi`). Every attention call is
one of the library's entry points; the harness only decides which one runs,
keeps each layer's latest plan, and times the attention calls with CUDA
events on the launching stream. The activation update between steps is not
timed.
"""
from __future__ import annotations

import dataclasses
import math

import torch

from . import abi, inputs

DENSE, PLAN_SPARSE, SPARSE = "dense", "plan+sparse", "sparse"


@dataclasses.dataclass
class Policy:
    steps: int = 50        # denoising steps
    dense_steps: int = 10  # the first steps run dense attention in every layer
    plan_every: int = 4    # a layer re-plans every this many sparse steps
    dense_layers: int = 1  # the first layers (transformer blocks) always run dense


def schedule(policy: Policy, layers: int) -> list[list[str]]:
    """The action of every (step, layer): DENSE, PLAN_SPARSE (plan on this
    step's activations, then the sparse forward) or SPARSE (the layer's last
    plan reused)."""
    if policy.steps < 0 or policy.dense_steps < 0 or policy.plan_every < 1 or policy.dense_layers < 0:
        raise ValueError(f"bad policy {policy}")
    out = []
    for t in range(policy.steps):
        row = []
        for layer in range(layers):
            if t < policy.dense_steps or layer < policy.dense_layers:
                row.append(DENSE)
            elif (t - policy.dense_steps) % policy.plan_every == 0:
                row.append(PLAN_SPARSE)
            else:
                row.append(SPARSE)
        out.append(row)
    return out


class Layer:
    """One attention layer: seeded base activations plus a seeded drift
    direction; the activations of step t are base + drift * t * step_scale."""

    def __init__(self, w: inputs.Workload, layer: int, device="cuda", drift=0.3, steps=50):
        seed = w.seed + 7919 * (layer + 1)
        self.Q0, self.K0, self.V0 = inputs.make_qkv(w, device=device, seed=seed)
        g = torch.Generator(device=device).manual_seed(seed)
        self.dQ, self.dK, self.dV = (torch.randn(self.Q0.shape, generator=g, device=device).to(torch.bfloat16)
                                     for _ in range(3))
        self.Q, self.K, self.V = (torch.empty_like(self.Q0) for _ in range(3))
        self.step_scale = drift / max(1, steps)

    def set_step(self, t: int) -> None:
        a = self.step_scale * t
        torch.add(self.Q0, self.dQ, alpha=a, out=self.Q)
        torch.add(self.K0, self.dK, alpha=a, out=self.K)
        torch.add(self.V0, self.dV, alpha=a, out=self.V)


def run(w: inputs.Workload, policy: Policy, layers: int = 2, device="cuda", keep_outputs=False, drift=0.3):
    """Runs the policy; returns per-step attention ms (CUDA events around the
    attention calls only), counts of each action and, with keep_outputs, the
    (step, layer) -> (O, plan used) record."""
    cfg = abi.Config(kv_block=w.kv_block, budget=w.budget, n_clusters=w.n_clusters,
                     kmeans_iters=w.kmeans_iters, seed=w.seed)
    L = [Layer(w, i, device, drift, policy.steps) for i in range(layers)]
    shape = tuple(L[0].Q0.shape)
    planners = [abi.Planner(shape, cfg) for _ in range(layers)]
    O = torch.empty_like(L[0].Q0)
    lse = torch.empty(shape[:3], dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    plan_of = [None] * layers
    sched = schedule(policy, layers)
    step_ms, counts, record = [], {DENSE: 0, PLAN_SPARSE: 0, SPARSE: 0}, {}
    for t, row in enumerate(sched):
        for layer in L:
            layer.set_step(t)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i, act in enumerate(row):
            lay = L[i]
            if act == DENSE:
                abi.dense_forward(lay.Q, lay.K, lay.V, O=O, lse=lse)
            else:
                if act == PLAN_SPARSE:
                    # each layer owns its planner, whose buffers change only when
                    # that layer plans again
                    plan_of[i] = planners[i](lay.Q, lay.K)
                abi.forward(lay.Q, lay.K, lay.V, plan_of[i], cfg, O=O, lse=lse)
            counts[act] += 1
            if keep_outputs:  # (tests only: copies inside the timed region)
                pl = plan_of[i]
                kept = None if act == DENSE else abi.Plan(pl.counts.clone(), pl.idx.clone(), pl.pi_sel.clone(),
                                                         pl.cap, pl.kv_block)
                record[(t, i)] = (O.clone(), lse.clone(), kept)
        e1.record(stream)
        torch.cuda.synchronize()
        step_ms.append(e0.elapsed_time(e1))
    abi.check()
    return {"step_ms": step_ms, "counts": counts, "record": record, "cfg": cfg, "layers": L}


def per_call_ms(policy: Policy, res: dict, layers: int):
    """Dense, sparse-forward and plan times per call, solved from the step
    timings: dense-warm-up steps run only dense calls; later steps run
    `dense_layers` dense calls plus one sparse forward (and on re-plan steps
    one plan) per other layer."""
    sched = schedule(policy, layers)
    ms = res["step_ms"]
    dl = min(policy.dense_layers, layers)
    warm = [m for t, m in enumerate(ms) if t < policy.dense_steps]
    dense = sum(warm) / len(warm) / layers if warm else float("nan")
    rest = layers - dl
    sp = [m for t, m in enumerate(ms) if t >= policy.dense_steps and SPARSE in sched[t]]
    pl = [m for t, m in enumerate(ms) if t >= policy.dense_steps and PLAN_SPARSE in sched[t]]
    sparse = (sum(sp) / len(sp) - dl * dense) / rest if sp and rest else float("nan")
    plan = (sum(pl) / len(pl) - dl * dense) / rest - sparse if pl and rest else float("nan")
    return dense, sparse, plan


def summary(w: inputs.Workload, policy: Policy, res: dict, layers: int, dense_ms: float, sparse_ms: float,
            plan_ms: float, model_layers: int) -> dict:
    """Amortised attention time per step for the measured layers, and for a
    model of `model_layers` blocks built from the measured per-call times
    (dense, sparse forward, plan) under the same policy."""
    steps = policy.steps
    measured = sum(res["step_ms"]) / steps
    sched = schedule(policy, model_layers)
    flat = [a for row in sched for a in row]
    model = (flat.count(DENSE) * dense_ms + flat.count(PLAN_SPARSE) * (plan_ms + sparse_ms)
             + flat.count(SPARSE) * sparse_ms) / steps
    all_dense = model_layers * dense_ms
    return {
        "denoise": w.name,
        "policy": dataclasses.asdict(policy),
        "measured_layers": layers,
        "attention_ms_per_step_measured": measured,
        "calls": res["counts"],
        "per_call_ms": {"dense": dense_ms, "sparse_forward": sparse_ms, "plan": plan_ms},
        "model_layers": model_layers,
        "model_attention_ms_per_step": model,
        "model_all_dense_ms_per_step": all_dense,
        "model_attention_speedup": all_dense / model if model > 0 else math.inf,
    }
