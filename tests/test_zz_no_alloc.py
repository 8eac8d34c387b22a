"""abattn_plan_noalloc: the plan for callers that cannot allocate device
memory (e.g. a host whose runtime owns every device allocation through its
own pool, or code that must not allocate while it runs).  Its scratch is a
fixed array inside the library, so its results must match abattn_plan with
a caller workspace, call after call, and problems too large for that array
must be refused before anything runs.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_12_b200 import abi, inputs


def test_noalloc_rejects_problems_larger_than_its_scratch():
    shape = (1, 40, 75600, 128)
    cfg = abi.Config(kv_block=4, budget=0.08)
    # the binding's limit is read from the header the library is built from
    assert abi.NOALLOC_SCRATCH_BYTES == abi._header_define("ABATTN_NOALLOC_SCRATCH_BYTES") == 32 << 20
    assert abi.plan_workspace_bytes(shape, cfg) > abi.NOALLOC_SCRATCH_BYTES
    # NULL tensors: whichever check comes first, nothing can be launched on them
    rc = abi.lib().abattn_plan_noalloc(None, None, ctypes.byref(abi.Dims(*shape)), ctypes.byref(cfg.params()),
                                       None, None, None, abi.capacity(shape, cfg), None)
    assert rc == abi.ERR_WORKSPACE
    # a problem that fits gets past the size check and stops at the NULL pointers
    small = (1, 2, 4096, 64)
    assert abi.plan_workspace_bytes(small, cfg) <= abi.NOALLOC_SCRATCH_BYTES
    rc = abi.lib().abattn_plan_noalloc(None, None, ctypes.byref(abi.Dims(*small)), ctypes.byref(cfg.params()),
                                       None, None, None, abi.capacity(small, cfg), None)
    assert rc == abi.ERR_NULL


@pytest.mark.gpu
def test_noalloc_plan_matches_workspace_plan_twice():
    w = inputs.TINY
    Q, K, _ = (t.cuda() for t in inputs.make_qkv(w))
    shape = tuple(Q.shape)
    for seed, mode in ((w.seed, abi.MODE_SIP), (7, abi.MODE_SIP), (0, abi.MODE_TOPK)):
        cfg = abi.Config(kv_block=w.kv_block, budget=w.budget, seed=seed, mode=mode)
        assert abi.plan_workspace_bytes(shape, cfg) <= abi.NOALLOC_SCRATCH_BYTES
        ref = abi.plan(Q, K, cfg)
        abi.check()
        for _ in range(2):  # two calls in a row reuse the library's scratch array
            got = abi.plan_noalloc(Q, K, cfg, plan=abi.empty_plan(shape, cfg))
            abi.check()
            np.testing.assert_array_equal(got.counts.cpu().numpy(), ref.counts.cpu().numpy())
            n = got.counts.cpu().numpy()
            gi, ri = got.idx.cpu().numpy(), ref.idx.cpu().numpy()
            gp, rp = got.pi_sel.cpu().numpy(), ref.pi_sel.cpu().numpy()
            for r in np.ndindex(n.shape):
                np.testing.assert_array_equal(gi[r][:n[r]], ri[r][:n[r]])
                np.testing.assert_array_equal(gp[r][:n[r]], rp[r][:n[r]])
    # a second shape after the first: the array keeps the last call's contents
    Q2 = torch.randn(1, 3, 1000, 128, device="cuda").to(torch.bfloat16)
    K2 = torch.randn(1, 3, 1000, 128, device="cuda").to(torch.bfloat16)
    cfg = abi.Config(kv_block=4, budget=0.2, seed=5)
    ref = abi.plan(Q2, K2, cfg)
    got = abi.plan_noalloc(Q2, K2, cfg)
    abi.check()
    np.testing.assert_array_equal(got.counts.cpu().numpy(), ref.counts.cpu().numpy())
    assert torch.equal(got.idx, ref.idx) or all(
        torch.equal(got.idx[0, h, q, :c], ref.idx[0, h, q, :c])
        for h in range(3) for q, c in enumerate(ref.counts[0, h].tolist()))
