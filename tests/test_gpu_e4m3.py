"""The E4M3 forward (QK^T in 8-bit floats, the VC-Attention pages' 8-bit
attention on B200) against the CPU oracle, through the C ABI.

The quantiser is compared bit for bit with the oracle's (codes and scales).
The forward is compared with the oracle evaluated on the dequantised Q and K
(code value x block scale, in fp64) and the bf16 V on the same plan, at the
bf16 forward's tolerances (max-abs 2e-2 on |error| / max(1, |O|), relative-L2
5e-3): what remains is the kernel's own rounding, with the quantisation
itself fixed by the codes.  The error of the whole 8-bit path against the
oracle on the unquantised inputs is printed, not asserted (its own bar is in
the design notes).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_12_b200 import abi, inputs

pytestmark = pytest.mark.gpu


def _bf16_inputs(B, H, N, seed, outlier_rows=0, zero_rows=0):
    """N(0,1) rows; outlier_rows rows of Q and K scaled by 8 (they set their
    blocks' scales); V stays N(0,1), so |O| < 1 and the plain bound applies
    (the full-size test covers x8 V rows with the per-element bound)."""
    g = torch.Generator().manual_seed(seed)
    Q, K, V = (torch.randn(B, H, N, 128, generator=g) for _ in range(3))
    if outlier_rows:
        sel = torch.randperm(N, generator=g)[:outlier_rows]
        for t in (Q, K):
            t[:, :, sel] *= 8.0
    if zero_rows:
        Q[:, :, :zero_rows] = 0.0
        K[:, :, :zero_rows] = 0.0
    return tuple(t.to(torch.bfloat16) for t in (Q, K, V))


@pytest.mark.parametrize("N,rpb", [(1000, 4), (4096, 128), (1000, 128), (777 * 4, 8), (130, 32)])
def test_quantize_e4m3_bit_exact(N, rpb):
    X, _, _ = _bf16_inputs(1, 2, N, seed=N + rpb, outlier_rows=N // 100 + 1, zero_rows=min(rpb, 8))
    codes, scales = abi.quantize_e4m3(X.cuda(), rpb)
    abi.check()
    oc, osc = oracle.quantize_e4m3_rows(X.float().numpy(), rpb)
    assert np.array_equal(scales.cpu().numpy(), osc)
    got = codes.cpu().numpy()
    # +0 and -0 are the same value: compare decoded values, then codes
    assert np.array_equal(oracle.e4m3_decode(got), oracle.e4m3_decode(oc))
    nz = oracle.e4m3_decode(oc) != 0
    assert np.array_equal(got[nz], oc[nz])


def _check_forward(Qc, Kc, Vc, kb, budget, what):
    cfg = abi.Config(kv_block=kb, budget=budget, seed=5)
    Q, K, V = Qc.cuda(), Kc.cuda(), Vc.cuda()
    plan = abi.plan(Q, K, cfg)
    Q8, qs = abi.quantize_e4m3(Q, 128)
    K8, ks = abi.quantize_e4m3(K, kb)
    O, lse = abi.forward_e4m3(Q8, qs, K8, ks, V, plan, cfg)
    abi.check()
    Qd = oracle.dequantize_e4m3_rows(Q8.cpu().numpy(), qs.cpu().numpy(), 128)
    Kd = oracle.dequantize_e4m3_rows(K8.cpu().numpy(), ks.cpu().numpy(), kb)
    args = (128, kb, plan.counts.cpu().numpy(), plan.idx.cpu().numpy(), plan.pi_sel.cpu().numpy(),
            1 / math.sqrt(128))
    Oo, lo = oracle.forward_rows(Qd, Kd, Vc, *args)
    Og = O.float().cpu().numpy()
    err = (np.abs(Og - Oo) / np.maximum(1.0, np.abs(Oo))).max()
    rel = np.linalg.norm(Og - Oo) / np.linalg.norm(Oo)
    Ox, _ = oracle.forward_rows(Qc, Kc, Vc, *args)
    rel_x = np.linalg.norm(Og - Ox) / np.linalg.norm(Ox)
    print(f"{what}: vs oracle on dequantised Q, K: max-abs {err:.3e} rel-L2 {rel:.3e}; "
          f"vs oracle on the bf16 inputs: rel-L2 {rel_x:.3e}")
    assert err <= 2e-2 and rel <= 5e-3, (what, err, rel)
    np.testing.assert_allclose(lse.cpu().numpy(), lo, atol=2e-3, rtol=1e-4)
    return rel_x


@pytest.mark.parametrize("N,kb,budget", [(4096, 4, 0.125), (1000, 4, 0.3), (1236, 8, 0.25), (2048, 128, 0.5),
                                         (132, 4, 1.0)])
def test_forward_e4m3_against_oracle_on_dequantised_inputs(N, kb, budget):
    Qc, Kc, Vc = _bf16_inputs(1, 2, N, seed=N + kb, outlier_rows=N // 100)
    _check_forward(Qc, Kc, Vc, kb, budget, f"N{N} kb{kb}")


def test_forward_e4m3_on_the_tiny_workload():
    w = inputs.TINY
    # the tiny workload has d = 64; the same recipe at d = 128
    import dataclasses
    w = dataclasses.replace(w, d=128)
    Qc, Kc, Vc = inputs.make_qkv(w)
    rel_x = _check_forward(Qc, Kc, Vc, w.kv_block, w.budget, "tiny recipe at d 128")
    assert rel_x < 0.1  # the 8-bit path stays close to the exact one


def test_forward_e4m3_rejects_unsupported_shapes():
    X = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(abi.AbattnError) as e:
        abi.quantize_e4m3(X, 128)
    assert e.value.code == abi.ERR_SHAPE
    X = torch.zeros(1, 1, 256, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(abi.AbattnError) as e:
        abi.quantize_e4m3(X, 3)
    assert e.value.code == abi.ERR_PARAM
