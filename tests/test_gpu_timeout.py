"""The bounded-wait error path on the GPU.

A kernel wait that runs out records ATTN_ERR_TIMEOUT in the device status word
and returns, so that the CUDA context stays usable.  attn_check_wait_timeout
launches a kernel whose one wait is on a barrier that nothing arrives at, with
the library's bounded wait; the tests check that its status comes back as
ATTN_ERR_TIMEOUT after the limit, that reading it clears it, and that normal
calls afterwards are correct.  (The attention kernels' own exit after a wait
runs out, letting their copies and MMAs land, is modelled on the CPU in
test_abort_protocol.py.)"""
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case, check_lse, check_o, host_f64
from test_gpu_backward import check_grads, run_fwd_bwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    yield m
    m.attn_set_wait_limit_ms(4000)


def test_a_wait_that_runs_out_reports_timeout(ta):
    assert ta.attn_get_status() == 0
    ta.attn_set_wait_limit_ms(50)
    t0 = time.perf_counter()
    ta.attn_check_wait_timeout()
    assert ta.attn_get_status() == ta.ATTN_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.04 <= elapsed < 5.0
    assert ta.attn_get_status() == 0  # reading the status cleared it
    ta.attn_set_wait_limit_ms(4000)


def test_calls_after_a_timeout_are_correct(ta):
    ta.attn_set_wait_limit_ms(20)
    ta.attn_check_wait_timeout()
    assert ta.attn_get_status() == ta.ATTN_ERR_TIMEOUT
    ta.attn_set_wait_limit_ms(4000)
    c = Case(61, 2, 4, 2, 700, 700, 128, oracle.MOD_CAUSAL)
    got = [host_f64(t) for t in run_fwd_bwd(ta, c)]  # asserts a zero status itself
    check_grads(got, c.oracle_bwd(), "after a timeout")


def test_short_limits_do_not_fire_in_normal_calls(ta):
    """Every wait of the attention kernels is short in a normal call: with a
    20 ms limit the forward and backward still run and stay correct."""
    ta.attn_set_wait_limit_ms(20)
    try:
        c = Case(62, 2, 8, 2, 2048, 2048, 128, oracle.MOD_NONE)
        out = torch.empty_like(c.q)
        lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
        ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale)
        torch.cuda.synchronize()
        assert ta.attn_get_status() == 0
        rows = np.array([0, 5, 1000, 2047])
        O, L = c.oracle_fwd(heads=[(1, 7)], rows=rows)
        og = np.full(O.shape, np.nan)
        lg = np.full(L.shape, np.nan)
        og[1, 7, rows] = host_f64(out)[1, 7, rows]
        lg[1, 7, rows] = lse.cpu().double().numpy()[1, 7, rows]
        check_o(og, O)
        check_lse(lg, L)
    finally:
        ta.attn_set_wait_limit_ms(4000)
