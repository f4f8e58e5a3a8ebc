"""build_block_mask on the GPU, byte for byte against the brute-force oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case  # noqa: F401  (imports the shared test path setup)
from synth_inputs import ModParams, WORKLOADS, doc_offsets_for, pad_offsets

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    return m


def compare(ta, mod, p, B, Sq, Skv):
    doc_t = None
    if oracle.has_document(mod):
        doc_t = torch.from_numpy(pad_offsets(p.doc_offsets)[0]).cuda()
    dp = ta.ModParams(window=p.window, doc_offsets=doc_t)
    mask = ta.new_block_mask(mod, dp, B, Sq, Skv)
    torch.cuda.synchronize()
    ref = oracle.block_mask(mod, p, B, Sq, Skv)
    for name, arr in ref.items():
        got = mask.view(name).cpu().numpy()
        assert got.dtype == arr.dtype and got.shape == arr.shape, name
        assert np.array_equal(got, arr), f"{name} differs (mod {mod}, {B}x{Sq}x{Skv})"


@pytest.mark.parametrize("S", [1, 127, 128, 129, 300, 1000, 4096])
@pytest.mark.parametrize("mod", [oracle.MOD_NONE, oracle.MOD_CAUSAL, oracle.MOD_SLIDING_WINDOW, oracle.MOD_DOCUMENT])
def test_block_mask_shapes(ta, S, mod):
    p = ModParams(window=max(1, S // 3))
    if oracle.has_document(mod):
        p.doc_offsets = [[0, S], sorted(set([0, S // 4, S // 4 + 1, S // 2, S]))]
    compare(ta, mod, p, 2, S, S)


@pytest.mark.parametrize("Sq,Skv", [(200, 900), (900, 200)])
def test_block_mask_unequal(ta, Sq, Skv):
    for mod in (oracle.MOD_CAUSAL, oracle.MOD_SLIDING_WINDOW):
        compare(ta, mod, ModParams(window=150), 1, Sq, Skv)


def test_block_mask_single_token_documents(ta):
    S = 700
    offs = [0, 1, 2, 3, 130, 131, 256, 257, 699, 700]
    compare(ta, oracle.MOD_DOCUMENT, ModParams(doc_offsets=[offs]), 1, S, S)


@pytest.mark.parametrize("name,mod", [("dense", oracle.MOD_CAUSAL), ("score_mods", oracle.MOD_SLIDING_WINDOW),
                                      ("documents", oracle.MOD_DOCUMENT), ("gqa_long", oracle.MOD_CAUSAL)])
def test_block_mask_workloads(ta, name, mod):
    w = WORKLOADS[name]
    p = ModParams()
    if oracle.has_document(mod):
        p.doc_offsets = doc_offsets_for(w)
    compare(ta, mod, p, w.B, w.Sq, w.Skv)
