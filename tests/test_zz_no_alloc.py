"""The allocation-free backward entry point (attn_bwd_noalloc).

It serves callers that cannot allocate device memory at call time (a plugin
host that gives its kernels no workspace, or an application whose device
memory is fixed in advance by its own pool): it runs the backward pass on a
fixed block the library holds instead of on a caller workspace.  These tests
call it through the C ABI and check its gradients against attn_bwd on the
same inputs and against the fp64 oracle, on two calls in a row, since every
call reuses the same block.
This file is collected last so that a failure here leaves every other test
already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_common import GRAD_REL_L2, Case, host_f64, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    return m


def _call_noalloc(ta, c, out, lse, mask, dq, dk, dv):
    P = ctypes.c_void_p
    mp = c.dev_params.c()
    rc = ta.LIB.attn_bwd_noalloc(P(c.q.data_ptr()), P(c.k.data_ptr()), P(c.v.data_ptr()), P(out.data_ptr()),
                                 P(lse.data_ptr()), P(c.dout.data_ptr()), P(dq.data_ptr()), P(dk.data_ptr()),
                                 P(dv.data_ptr()), c.B, c.Hq, c.Hkv, c.Sq, c.Skv, c.D, c.scale, c.mod,
                                 ctypes.byref(mp), ctypes.byref(mask.c),
                                 P(torch.cuda.current_stream().cuda_stream))
    return rc


@pytest.mark.parametrize("mod", [oracle.MOD_NONE, oracle.MOD_CAUSAL])
@pytest.mark.parametrize("D", [64, 128])
def test_noalloc_matches_workspace_backward_twice(ta, mod, D):
    c = Case(41, 2, 4, 2, 700, 700, D, mod)
    assert ta.attn_bwd_workspace_size(c.B, c.Hq, c.Sq, c.D) <= ta.attn_bwd_noalloc_max_workspace()
    mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv)
    out = torch.empty_like(c.q)
    lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
    ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params, block_mask=mask)
    ref = [torch.empty_like(c.q), torch.empty_like(c.k), torch.empty_like(c.v)]
    ws = ta.new_bwd_workspace(c.B, c.Hq, c.Sq, c.D)
    ta.attn_bwd(c.q, c.k, c.v, out, lse, c.dout, *ref, ws, scale=c.scale, mod_kind=c.mod,
                mod_params=c.dev_params, block_mask=mask)
    exact = c.oracle_bwd()
    for _ in range(2):  # the second call reuses the block the first one left behind
        got = [torch.full_like(c.q, float("nan")), torch.full_like(c.k, float("nan")),
               torch.full_like(c.v, float("nan"))]
        assert _call_noalloc(ta, c, out, lse, mask, *got) == 0
        torch.cuda.synchronize()
        assert ta.attn_get_status() == 0
        for g, r, x in zip(got, ref, exact):
            assert rel_l2(host_f64(g), host_f64(r)) <= GRAD_REL_L2
            # and against the fp64 oracle on the same inputs
            assert rel_l2(host_f64(g), x) <= GRAD_REL_L2
        # dK and dV have a fixed summation order: identical to the workspace call
        assert torch.equal(got[1].view(torch.int16), ref[1].view(torch.int16))
        assert torch.equal(got[2].view(torch.int16), ref[2].view(torch.int16))


def test_noalloc_rejects_problems_beyond_its_block(ta):
    # 8 x 16 heads of 8192 rows at D = 128 need far more than the fixed block
    B, Hq, S, D = 8, 16, 8192, 128
    assert ta.attn_bwd_workspace_size(B, Hq, S, D) > ta.attn_bwd_noalloc_max_workspace()
    P = ctypes.c_void_p
    fake = P(1 << 32)  # never dereferenced: the size check comes first
    rc = ta.LIB.attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, B, Hq, Hq, S, S, D,
                                 D ** -0.5, 0, None, None, P(torch.cuda.current_stream().cuda_stream))
    assert rc == -4  # ATTN_ERR_WORKSPACE
