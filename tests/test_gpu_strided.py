"""Strided inputs and outputs: [B][S][H][D] storage seen as [B][H][S][D]
views gives results bit-identical to contiguous tensors (the tiles, their
order and the arithmetic do not depend on the layout)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case, check_lse, check_o, host_f64
from test_gpu_backward import check_grads, small_params

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    return m


def bshd(t):
    """The same values in [B][S][H][D] storage, as a [B][H][S][D] view."""
    return t.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)


@pytest.mark.parametrize("mod", [oracle.MOD_NONE, oracle.MOD_CAUSAL, oracle.MOD_ALIBI])
@pytest.mark.parametrize("D", [64, 128])
def test_bshd_views_match_contiguous_bitwise(ta, mod, D):
    S = 300
    c = Case(120 + mod + D, 2, 4, 2, S, S, D, mod, small_params(mod, S))
    mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv)
    kw = dict(scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params, block_mask=mask)
    out = torch.empty_like(c.q)
    lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
    ta.attn_fwd(c.q, c.k, c.v, out, lse, **kw)
    ws = ta.new_bwd_workspace(c.B, c.Hq, c.Sq, c.D)
    dq, dk, dv = torch.empty_like(c.q), torch.empty_like(c.k), torch.empty_like(c.v)
    ta.attn_bwd(c.q, c.k, c.v, out, lse, c.dout, dq, dk, dv, ws, **kw)

    q2, k2, v2, do2 = bshd(c.q), bshd(c.k), bshd(c.v), bshd(c.dout)
    out2, dq2, dk2, dv2 = bshd(torch.empty_like(c.q)), bshd(torch.empty_like(c.q)), bshd(torch.empty_like(c.k)), \
        bshd(torch.empty_like(c.v))
    lse2 = torch.empty_like(lse)
    ta.attn_fwd_strided(q2, k2, v2, out2, lse2, **kw)
    ta.attn_bwd_strided(q2, k2, v2, out2, lse2, do2, dq2, dk2, dv2, ws, **kw)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    assert torch.equal(out.view(torch.int16), out2.contiguous().view(torch.int16))
    assert torch.equal(lse, lse2)
    for a, b in ((dk, dk2), (dv, dv2)):
        assert torch.equal(a.view(torch.int16), b.contiguous().view(torch.int16))
    # dQ goes through L2 reductions in any order: close, not bitwise
    assert torch.allclose(dq.float(), dq2.float(), atol=2e-3, rtol=2e-2)
    # and the strided results against the fp64 oracle
    O, L = c.oracle_fwd()
    check_o(host_f64(out2), O, f"strided mod {mod} D {D}")
    check_lse(lse2.cpu().double().numpy(), L, f"strided mod {mod} D {D}")
    check_grads([host_f64(t) for t in (dq2, dk2, dv2)], c.oracle_bwd(), f"strided mod {mod} D {D}")


def test_bad_strides_are_refused(ta):
    c = Case(130, 1, 2, 2, 128, 128, 64, oracle.MOD_NONE)
    odd = torch.empty(1, 2, 128, 68, dtype=torch.bfloat16, device="cuda")[..., :64]  # row stride 68
    out = torch.empty_like(c.q)
    with pytest.raises(ta.AttnError):
        ta.attn_fwd_strided(odd, c.k, c.v, out)


def padded(t, pad=8):
    """The same values in rows of D + pad elements: every other row then
    starts 16 bytes past a 32-byte boundary (the epilogues' narrow stores)."""
    B, H, S, D = t.shape
    buf = torch.zeros(B, H, S, D + pad, dtype=t.dtype, device=t.device)
    buf[..., :D] = t
    return buf[..., :D]


@pytest.mark.parametrize("D", [64, 128])
def test_padded_rows_match_contiguous_bitwise(ta, D):
    """Rows of D + 8 elements: O, dK and dV rows alternate between 32-byte
    aligned starts (32-byte stores) and 16-byte aligned ones (16-byte stores);
    both give the contiguous call's bits."""
    S = 257
    c = Case(140 + D, 2, 4, 2, S, S, D, oracle.MOD_CAUSAL, small_params(oracle.MOD_CAUSAL, S))
    mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv)
    kw = dict(scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params, block_mask=mask)
    out = torch.empty_like(c.q)
    lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
    ta.attn_fwd(c.q, c.k, c.v, out, lse, **kw)
    ws = ta.new_bwd_workspace(c.B, c.Hq, c.Sq, c.D)
    dq, dk, dv = torch.empty_like(c.q), torch.empty_like(c.k), torch.empty_like(c.v)
    ta.attn_bwd(c.q, c.k, c.v, out, lse, c.dout, dq, dk, dv, ws, **kw)

    q2, k2, v2, do2 = padded(c.q), padded(c.k), padded(c.v), padded(c.dout)
    out2, dq2, dk2, dv2 = (padded(torch.zeros_like(t)) for t in (c.q, c.q, c.k, c.v))
    lse2 = torch.empty_like(lse)
    ta.attn_fwd_strided(q2, k2, v2, out2, lse2, **kw)
    ta.attn_bwd_strided(q2, k2, v2, out2, lse2, do2, dq2, dk2, dv2, ws, **kw)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    assert out2.stride(2) == D + 8
    assert torch.equal(out.view(torch.int16), out2.contiguous().view(torch.int16))
    assert torch.equal(lse, lse2)
    for a, b in ((dk, dk2), (dv, dv2)):
        assert torch.equal(a.view(torch.int16), b.contiguous().view(torch.int16))
    assert torch.allclose(dq.float(), dq2.float(), atol=2e-3, rtol=2e-2)
    O, L = c.oracle_fwd()
    check_o(host_f64(out2), O, f"padded D {D}")
    check_grads([host_f64(t) for t in (dq2, dk2, dv2)], c.oracle_bwd(), f"padded D {D}")
