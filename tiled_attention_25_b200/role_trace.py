"""Per-role cycle breakdown of the forward and backward kernels.

Runs one forward and one backward call of a workload through the profiling
build (libattn25_trace.so, built by `python tiled_attention_25_b200/build.py
--trace`), whose kernels add the clock64 time of each wait and compute phase
of every warp role into a device buffer, and prints a markdown table of the
per-CTA averages per unit of work (a 128-key tile step forward, a 64-query
step backward) plus the share of each role's time spent in the softmax
exponentials.

    python tiled_attention_25_b200/role_trace.py [workload:mod ...]

The default workload is dense:none (4 x 8 x 4096 x 128, non-causal).
"""
from __future__ import annotations

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
os.environ.setdefault("ATTN25_LIBRARY", os.path.join(HERE, "libattn25_trace.so"))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import tiled_attention_25_b200 as ta  # noqa: E402
from synth_inputs import MOD_NAMES, WORKLOADS, draw_workload, mod_params_for, pad_offsets  # noqa: E402

# Counter words of each role (forward at 0, backward at 128) and their meaning.
FWD_ROLES = {
    "softmax tile 0 (per warp)": (0, 4, ["total", "wait S", "scores, max, rescale", "exp2 and P store",
                                         "wait last PV", "epilogue", "rescales", "tiles"]),
    "softmax tile 1 (per warp)": (16, 4, ["total", "wait S", "scores, max, rescale", "exp2 and P store",
                                          "wait last PV", "epilogue", "rescales", "tiles"]),
    "MMA warp": (32, 1, ["total", "wait Q", "wait K", "wait V", "wait P0", "wait P1"]),
    "TMA warp": (48, 1, ["total", "wait Q free", "wait K/V slot free"]),
}
BWD_ROLES = {
    "P warps (per warp)": (128, 4, ["total", "wait Q", "wait S^T", "P total", "TMEM load", "exp2 math",
                                    "TMEM store", "wait accumulators", "dV epilogue"]),
    "dS warps (per warp)": (192, 4, ["total", "wait Q", "wait P^T", "TMEM load", "wait dP^T",
                                     "wait dS buffer", "dS math and store", "wait accumulators",
                                     "dK epilogue"]),
    "dQ drain (per warp)": (144, 4, ["total", "wait dQ^T", "L2 reductions"]),
    "MMA warp": (160, 1, ["total", "wait K/V", "wait accumulators free", "wait Q", "wait P^T",
                          "wait dS^T", "-", "steps", "wait dP^T read"]),
    "TMA warp": (176, 1, ["total", "wait K/V free", "wait Q stage free"]),
}


def _problem(spec):
    name, _, mod_name = spec.partition(":")
    w = WORKLOADS[name]
    mod_name = mod_name or w.mods[0]
    mod = MOD_NAMES[mod_name]
    p = mod_params_for(w, mod_name)
    bits = draw_workload(w)
    dev = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v, do = (dev(bits[n]) for n in ("q", "k", "v", "dout"))
    doc = torch.from_numpy(pad_offsets(p.doc_offsets)[0]).cuda() if p.doc_offsets else None
    dp = ta.ModParams(softcap=p.softcap, window=p.window, boost=p.boost, boost_radius=p.boost_radius,
                      doc_offsets=doc)
    return w, mod, dp, q, k, v, do


def _table(counters, roles, grid, units):
    rows = []
    for role, (base, warps, labels) in roles.items():
        vals = [counters[base + i] / (warps * grid) for i in range(len(labels))]
        for lab, val in zip(labels, vals):
            if lab == "-":
                continue
            if lab in ("steps", "rescales", "tiles"):
                rows.append((role, lab, val, None))
            else:
                rows.append((role, lab, val / units, val / vals[0] if vals[0] else 0.0))
    return rows


def trace(spec):
    w, mod, dp, q, k, v, do = _problem(spec)
    mask = ta.new_block_mask(mod, dp, w.B, w.Sq, w.Skv)
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.Hq, w.Sq, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = ta.new_bwd_workspace(w.B, w.Hq, w.Sq, w.D)
    for _ in range(3):
        ta.attn_fwd(q, k, v, out, lse, mod_kind=mod, mod_params=dp, block_mask=mask)
        ta.attn_bwd(q, k, v, out, lse, do, dq, dk, dv, ws, mod_kind=mod, mod_params=dp, block_mask=mask)
    torch.cuda.synchronize()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ta.abi.attn_trace_reset()
    ta.attn_fwd(q, k, v, out, lse, mod_kind=mod, mod_params=dp, block_mask=mask)
    ta.attn_bwd(q, k, v, out, lse, do, dq, dk, dv, ws, mod_kind=mod, mod_params=dp, block_mask=mask)
    c = ta.abi.attn_trace_read(256)
    if ta.attn_get_status() != 0:
        raise RuntimeError("kernel status")
    mask_view = mask.view("tile_class").cpu().numpy()
    nq, nk = mask_view.shape[1], mask_view.shape[2]
    n_tiles = int((mask_view != 0).sum()) * w.Hq       # forward: (query tile, key tile) pairs
    n_steps = int((mask_view != 0).sum()) * 2 * w.Hq   # backward: 64-query steps
    grid_f = min(sms, w.B * ((nq + 1) // 2) * w.Hq)
    grid_b = min(sms, w.B * nk * w.Hkv)
    # per CTA, per unit of work: the softmax warps of one tile handle half of the pairs
    fwd = _table(c, FWD_ROLES, grid_f, n_tiles / grid_f / 2)
    bwd = _table(c, BWD_ROLES, grid_b, n_steps / grid_b)
    return {"workload": spec, "sms": sms, "fwd_tiles_per_cta": n_tiles / grid_f,
            "bwd_steps_per_cta": n_steps / grid_b, "forward": fwd, "backward": bwd}


def markdown(res):
    out = [f"### {res['workload']}", "",
           f"Forward: {res['fwd_tiles_per_cta']:.1f} (query tile, key tile) pairs per CTA; "
           f"backward: {res['bwd_steps_per_cta']:.1f} 64-query steps per CTA.", "",
           "| kernel | role | phase | clk per unit | share of role time |", "|---|---|---|---|---|"]
    for kern in ("forward", "backward"):
        for role, lab, val, share in res[kern]:
            s = "" if share is None else f"{100 * share:.0f}%"
            unit = f"{val:.1f}" if share is not None else f"{val:.0f} (count)"
            out.append(f"| {kern} | {role} | {lab} | {unit} | {s} |")
    return "\n".join(out)


if __name__ == "__main__":
    specs = [a for a in sys.argv[1:] if not a.startswith("--")] or ["dense:none"]
    for s in specs:
        r = trace(s)
        print(markdown(r))
        print()
        print(json.dumps(r))
