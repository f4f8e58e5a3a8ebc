"""The library's host-side useful-element counts (used for throughput) against
the oracle's element-by-element count, for single and composed mods."""
import pytest

import oracle
from oracle import (MASK_CAUSAL, MASK_DOCUMENT, MASK_SLIDING_WINDOW, MOD_ALIBI, MOD_CAUSAL,
                    MOD_DOCUMENT, MOD_LOCAL_BOOST, MOD_NONE, MOD_SLIDING_WINDOW, MOD_SOFTCAP)
from synth_inputs import ModParams

MODS = [MOD_NONE, MOD_CAUSAL, MOD_ALIBI, MOD_SOFTCAP, MOD_SLIDING_WINDOW, MOD_LOCAL_BOOST,
        MOD_DOCUMENT, MOD_ALIBI | MASK_CAUSAL, MOD_SOFTCAP | MASK_SLIDING_WINDOW,
        MOD_LOCAL_BOOST | MASK_DOCUMENT, MOD_SLIDING_WINDOW | MASK_DOCUMENT,
        MOD_NONE | MASK_CAUSAL | MASK_SLIDING_WINDOW | MASK_DOCUMENT]


@pytest.mark.parametrize("mod", MODS)
def test_counts_match_oracle(mod):
    from tiled_attention_25_b200.counts import useful_elements
    S = 700
    docs = [[0, 130, 300, 301, 555, S], [0, S]]
    p = ModParams(window=37, doc_offsets=docs)
    assert useful_elements(mod, 2, 3, S, S, window=37, doc_offsets=docs) == \
        oracle.useful_elements(mod, p, 2, 3, S, S)


@pytest.mark.parametrize("Sq,Skv", [(300, 900), (900, 300)])
def test_counts_unequal_lengths(Sq, Skv):
    from tiled_attention_25_b200.counts import useful_elements
    for mod in (MOD_CAUSAL, MOD_SLIDING_WINDOW, MOD_ALIBI | MASK_SLIDING_WINDOW):
        assert useful_elements(mod, 1, 2, Sq, Skv, window=100) == \
            oracle.useful_elements(mod, ModParams(window=100), 1, 2, Sq, Skv)


@pytest.mark.parametrize("mod_name", ["alibi+causal", "softcap+sliding_window", "sliding_window+document", "bitmap"])
def test_bench_counts_of_composed_workloads(mod_name):
    # the bench's useful-element count for the composed and bitmap workloads,
    # on a reduced shape, against the oracle's element-by-element count
    import dataclasses
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import tiled_attention_25_b200 as ta
    from synth_inputs import MOD_NAMES, WORKLOADS, mod_params_for
    w = dataclasses.replace(WORKLOADS["composed"], B=2, Hq=2, Hkv=2, Sq=700, Skv=700)
    p = mod_params_for(w, mod_name)
    if p.doc_offsets is not None:
        p.doc_offsets = [[0, 130, 300, 301, 555, 700], [0, 700]]
    p.window = 200
    n, _, _ = bench.useful_counts(ta, w, mod_name, p)
    assert n == oracle.useful_elements(MOD_NAMES[mod_name], p, w.B, w.Hq, w.Sq, w.Skv)
