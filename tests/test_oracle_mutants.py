"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

Each mutant rewrites one expression of an oracle function from its source,
installs it for the duration of one test, and runs a pin from test_oracle.py
or test_oracle_block_mask.py that must then fail.
"""
import inspect
import textwrap

import pytest

import oracle
import oracle.attention as oa
import oracle.block_sparsity as ob
import oracle.fp8 as ofp8
import test_oracle as pins
import test_oracle_block_mask as bm_pins
import test_oracle_bitmap as bitmap_pins
import test_oracle_compose as comp_pins
import test_oracle_fp8 as fp8_pins
import test_oracle_varlen as varlen_pins


def _install(module, func_name, old, new, monkeypatch):
    src = textwrap.dedent(inspect.getsource(getattr(module, func_name)))
    assert old in src, (func_name, old)
    src = src.replace(old, new, 1)
    ns = dict(module.__dict__)
    exec(compile(src, f"<mutant {func_name}>", "exec"), ns)
    original = getattr(module, func_name)
    monkeypatch.setattr(module, func_name, ns[func_name])
    # the package re-exports some functions: patch those names too
    if getattr(oracle, func_name, None) is original:
        monkeypatch.setattr(oracle, func_name, ns[func_name])


MUTANTS = [
    # (module, function, original text, planted mistake, pin that must fail)
    (oa, "attention_forward", "s = scale * (q[b, h, r] @ k[b, hk].T)", "s = (q[b, h, r] @ k[b, hk].T)",
     lambda: pins.test_matches_torch_sdpa_float64(False)),
    (oa, "_single_mod", "s_mod = s - slope * np.abs(qi - kj)", "s_mod = s + slope * np.abs(qi - kj)",
     pins.test_zero_queries_alibi_geometric_sums),
    (oa, "alibi_slope", "(h + 1)", "h", pins.test_zero_queries_alibi_geometric_sums),
    (oa, "_single_mod", "keep = kj <= qi", "keep = kj < qi", pins.test_causal_first_query_attends_key0),
    (oa, "_single_mod", "keep = kj <= qi", "keep = kj >= qi", pins.test_causal_first_query_attends_key0),
    (oa, "_single_mod", "keep = (diff >= 0) & (diff < params.window)", "keep = (diff >= 0) & (diff <= params.window)",
     pins.test_window_one_attends_only_self),
    (oa, "_single_mod", "inside = np.abs(qi - kj) < params.boost_radius", "inside = np.abs(qi - kj) <= params.boost_radius",
     lambda: pins.test_single_key_gives_v0(oa.MOD_LOCAL_BOOST)),
    (oa, "_kv_head", "return h // (Hq // Hkv)", "return h % Hkv", pins.test_gqa_equals_mha_with_repeated_kv),
    (oa, "_row_softmax", "e = np.exp(x - m_safe[:, None])", "e = np.exp(x)",
     lambda: pins.test_single_key_gives_v0(oa.MOD_NONE)),
    (oa, "_row_softmax", "m_safe + np.log(", "m_safe + np.log2(", pins.test_zero_queries_mean_of_values),
    (oa, "attention_backward", "dS = P * (dP - Di[:, None]) * dmod", "dS = P * dP * dmod",
     lambda: pins.test_gradients_match_central_differences(oa.MOD_NONE)),
    (oa, "_single_mod", "dmod = 1.0 - t * t", "dmod = 1.0 - t",
     lambda: pins.test_gradients_match_central_differences(oa.MOD_SOFTCAP)),
    (oa, "attention_backward", "dv_acc += P[:, kv_sel].T @ dout[b, h, r]", "dv_acc += P[:, kv_sel].T @ dout[b, hk, r]",
     pins.test_gqa_equals_mha_with_repeated_kv),
    (oa, "attention_backward", "dq[b, h, r] = scale * (dS @ k[b, hk])", "dq[b, h, r] = (dS @ k[b, hk])",
     lambda: pins.test_gradients_match_central_differences(oa.MOD_NONE)),
    (oa, "online_forward", "l = l * alpha + p.sum(axis=1)", "l = l + p.sum(axis=1)",
     lambda: pins.test_online_softmax_matches_two_pass(oa.MOD_NONE)),
    (oa, "score_mod", "keep = keep & keep_m", "keep = keep | keep_m",
     lambda: comp_pins.test_composed_probs_are_restricted_softmax(oa.MOD_ALIBI | oa.MASK_CAUSAL)),
    (oa, "score_mod", "for kind in masks:", "for kind in masks[:1]:",
     comp_pins.test_zero_queries_window_and_documents_count_keys),
    (oa, "score_mod", "_single_mod(s, base, params", "_single_mod(s, masks[0] if masks else base, params",
     comp_pins.test_zero_queries_causal_alibi_geometric_sums),
    (ofp8, "quantize_e4m3", "q = np.round(a / quantum) * quantum", "q = np.floor(a / quantum + 0.5) * quantum",
     fp8_pins.test_ties_round_to_even_like_torch),
    (ofp8, "hadamard", "H = np.block([[H, H], [H, -H]])", "H = np.block([[H, H], [H, H]])",
     lambda: fp8_pins.test_hadamard_properties(8)),
    (ofp8, "quantize_per_head", "amax / E4M3_MAX", "amax", fp8_pins.test_on_grid_inputs_give_exact_attention),
    (ofp8, "attention_forward_fp8", "q, k = q @ R, k @ R", "q, k = q @ R, k",
     fp8_pins.test_rotation_lowers_the_fp8_error_on_outliers),
    (oa, "_single_mod", "seq_k[ko[d]:ko[d + 1]] = d", "seq_k[qo[d]:qo[d + 1]] = d",
     lambda: varlen_pins.test_sequences_are_independent_problems(oa.MOD_NONE | oa.MASK_VARLEN)),
    (ob, "classify_tiles", "elif min(counts) == blocks[0].size:", "elif min(counts) == tile * tile:",
     bm_pins.test_single_row_tail_tile_is_full),
    (ob, "classify_tiles", "if max(counts) == 0:", "if min(counts) == 0:",
     bitmap_pins.test_per_head_bitmap_classes_hold_for_every_head),
    (oa, "_single_mod", "[qi, kj]", "[kj, qi]",
     lambda: bitmap_pins.test_random_bitmap_is_restricted_softmax(oa.MOD_NONE | oa.MASK_BITMAP)),
    (oa, "_single_mod", "h if bm.shape[1] > 1 else 0", "0", bitmap_pins.test_per_head_bitmap_equals_separate_heads),
    (ob, "block_mask", "key=lambda u: (-pair_cost[u], u)", "key=lambda u: (pair_cost[u], u)", bm_pins.test_orders_are_lpt_permutations),
]


@pytest.mark.parametrize("i", range(len(MUTANTS)))
def test_planted_mistake_is_caught(i, monkeypatch):
    module, fn, old, new, pin = MUTANTS[i]
    _install(module, fn, old, new, monkeypatch)
    with pytest.raises(AssertionError):
        pin()
