"""Packed sequences with their own query and key lengths (MASK_VARLEN) on the
sm_100a kernels against the fp64 oracle: forward and backward, with and
without a block mask, Sq != Skv, empty sequences, score mods."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case, check_lse, check_o, host_f64
from oracle import MASK_VARLEN, MOD_ALIBI, MOD_NONE, MOD_SOFTCAP
from synth_inputs import ModParams
from test_gpu_backward import check_grads, run_fwd_bwd
from test_gpu_block_mask import compare as compare_mask  # noqa: F401
from test_gpu_forward import run_fwd

pytestmark = pytest.mark.gpu

QO = [[0, 90, 90, 300, 301, 520], [0, 520, 520, 520, 520, 520]]
KO = [[0, 200, 330, 331, 600, 700], [0, 700, 700, 700, 700, 700]]


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    return m


@pytest.mark.parametrize("mod", [MOD_NONE | MASK_VARLEN, MOD_SOFTCAP | MASK_VARLEN, MOD_ALIBI | MASK_VARLEN])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("use_mask", [False, True])
def test_varlen_forward_and_backward(ta, mod, D, use_mask):
    p = ModParams(softcap=20.0, q_offsets=QO, k_offsets=KO)
    c = Case(160 + (mod & 0xFF) + D, 2, 4, 2, 520, 700, D, mod, p)
    out, lse = run_fwd(ta, c, use_mask=use_mask)
    O, L = c.oracle_fwd()
    check_o(host_f64(out), O, f"varlen {mod:#x} D {D}")
    check_lse(lse.cpu().double().numpy(), L, f"varlen {mod:#x} D {D}")
    got = [host_f64(t) for t in run_fwd_bwd(ta, c, use_mask)]
    check_grads(got, c.oracle_bwd(), f"varlen {mod:#x} D {D}")


def test_varlen_block_mask_is_exact(ta):
    from synth_inputs import pad_offsets
    p = ModParams(q_offsets=QO, k_offsets=KO)
    dp = ta.ModParams(q_offsets=torch.from_numpy(pad_offsets(QO)[0]).cuda(),
                      k_offsets=torch.from_numpy(pad_offsets(KO)[0]).cuda())
    mask = ta.new_block_mask(MOD_NONE | MASK_VARLEN, dp, 2, 520, 700)
    torch.cuda.synchronize()
    ref = oracle.block_mask(MOD_NONE | MASK_VARLEN, p, 2, 520, 700)
    for name, arr in ref.items():
        assert np.array_equal(mask.view(name).cpu().numpy(), arr), name
