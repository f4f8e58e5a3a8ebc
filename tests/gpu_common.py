"""Helpers shared by the GPU parity tests: seeded inputs on the device, the
oracle on the same inputs, and the tolerance checks."""
import numpy as np
import torch

import oracle
from synth_inputs import ModParams, bf16_bits_to_f64, draw_qkv, pack_bitmap, pad_offsets

# Tolerances for bf16 inputs with fp32 accumulation versus the fp64 oracle.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def to_dev(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def host_f64(t):
    return t.float().cpu().double().numpy()


class Case:
    """One seeded problem: bf16 inputs (host bits, device tensors, fp64 copies)."""

    def __init__(self, seed, B, Hq, Hkv, Sq, Skv, D, mod, mod_params=None, scale=None):
        import tiled_attention_25_b200 as ta
        self.B, self.Hq, self.Hkv, self.Sq, self.Skv, self.D = B, Hq, Hkv, Sq, Skv, D
        self.mod = mod
        self.scale = D ** -0.5 if scale is None else scale
        self.p = mod_params or ModParams()
        bits = draw_qkv(seed, B, Hq, Hkv, Sq, Skv, D)
        self.bits = bits
        self.q, self.k, self.v, self.dout = (to_dev(bits[n]) for n in ("q", "k", "v", "dout"))
        self.qf, self.kf, self.vf, self.doutf = (bf16_bits_to_f64(bits[n]) for n in ("q", "k", "v", "dout"))
        doc_t = None
        if oracle.has_document(mod):
            arr, _ = pad_offsets(self.p.doc_offsets)
            doc_t = torch.from_numpy(arr).cuda()
        vq_t = vk_t = None
        if int(mod) & oracle.MASK_VARLEN:
            vq_t = torch.from_numpy(pad_offsets(self.p.q_offsets)[0]).cuda()
            vk_t = torch.from_numpy(pad_offsets(self.p.k_offsets)[0]).cuda()
        bm_t = None
        if oracle.has_bitmap(mod):
            bm_t = torch.from_numpy(pack_bitmap(self.p.bitmap)).cuda()
        self.dev_params = ta.ModParams(softcap=self.p.softcap, window=self.p.window, boost=self.p.boost,
                                       boost_radius=self.p.boost_radius, doc_offsets=doc_t, bitmap=bm_t,
                                       q_offsets=vq_t, k_offsets=vk_t)

    def oracle_fwd(self, heads=None, rows=None):
        return oracle.attention_forward(self.qf, self.kf, self.vf, self.scale, self.mod, self.p,
                                        heads=heads, rows=rows)

    def oracle_bwd(self, groups=None, q_rows=None, kv_rows=None, contrib_rows=None):
        return oracle.attention_backward(self.qf, self.kf, self.vf, self.doutf, self.scale, self.mod,
                                         self.p, groups=groups, q_rows=q_rows, kv_rows=kv_rows,
                                         contrib_rows=contrib_rows)


def check_o(o_gpu, o_ref, what=""):
    sel = ~np.isnan(o_ref)
    err = np.abs(o_gpu[sel] - o_ref[sel])
    assert err.size > 0
    assert err.max() <= O_MAX_ABS, f"{what} O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{what} O mean-abs {err.mean():.3e}"


def check_lse(l_gpu, l_ref, what=""):
    sel = ~np.isnan(l_ref)
    a, b = l_gpu[sel], l_ref[sel]
    both_inf = np.isneginf(a) & np.isneginf(b)
    err = np.abs(np.where(both_inf, 0.0, a - b))
    assert np.isfinite(err).all(), f"{what} LSE non-finite mismatch"
    assert err.max() <= LSE_ABS, f"{what} LSE abs {err.max():.3e}"


def rel_l2(x, ref):
    sel = ~np.isnan(ref)
    return float(np.linalg.norm(x[sel] - ref[sel]) / max(np.linalg.norm(ref[sel]), 1e-30))


def sample_rows(S, n, seed, extra=()):
    """Sorted sample of rows: both ends, tile edges near the tail, plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in rng.choice(S, size=min(n, S), replace=False))
    for r in (0, 1, 127, 128, S - 129, S - 128, S - 2, S - 1, *extra):
        if 0 <= r < S:
            rows.add(int(r))
    return np.array(sorted(rows), dtype=np.int64)
