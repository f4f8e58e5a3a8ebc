"""Pins of the FP8 / incoherent-processing oracle.

The e4m3 rounding is checked against torch's float8_e4m3fn cast (a library
routine, independent of the oracle) and the format's own grid; the rotation
against the defining properties of a Hadamard matrix; the FP8 attention
against exact attention where quantisation is a no-op; and the method against
the pages' claim ("FlashAttention-3 …", FlashAttention-3의 기술적 혁신, item
3): rotating Q and K before quantising lowers the FP8 attention error.
"""
import numpy as np
import pytest
import torch

import oracle


def e4m3_grid():
    """All finite e4m3 values, decoded by torch from the 256 codes."""
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    return np.unique(codes[np.isfinite(codes)])


def test_grid_values_are_fixed_points():
    g = e4m3_grid()
    assert g.max() == 448.0 and g.min() == -448.0 and len(g) == 253  # 254 finite codes, +-0 merge
    assert np.array_equal(oracle.quantize_e4m3(g), g)


def test_rounding_matches_torch_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(oracle.quantize_e4m3(x), ref)


def test_ties_round_to_even_like_torch():
    g = e4m3_grid()
    mids = (g[:-1] + g[1:]) / 2
    ref = torch.from_numpy(mids).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(oracle.quantize_e4m3(mids), ref)
    # and a tie goes to the neighbour whose 3-bit mantissa is even
    q = oracle.quantize_e4m3(np.array([1.0625, 1.1875, 2.0 ** -10]))
    assert np.array_equal(q, [1.0, 1.25, 0.0])


def test_saturates_at_448():
    x = np.array([448.0, 450.0, 463.9, 464.0, 1e6, -1e6])
    assert np.array_equal(oracle.quantize_e4m3(x), [448, 448, 448, 448, 448, -448])


@pytest.mark.parametrize("D", [1, 2, 8, 64, 128])
def test_hadamard_properties(D):
    H = oracle.hadamard(D)
    assert set(np.unique(H)) <= {-1.0, 1.0}
    assert np.array_equal(H @ H.T, D * np.eye(D))
    assert np.array_equal(H, H.T) and np.all(H[0] == 1)
    signs = np.where(np.random.default_rng(D).random(D) < 0.5, -1.0, 1.0)
    R = oracle.rotation(D, signs)
    assert np.allclose(R @ R.T, np.eye(D), atol=1e-14)


def test_hadamard_rejects_other_orders():
    for D in (0, 3, 96):
        with pytest.raises(ValueError):
            oracle.hadamard(D)


def test_rotation_cancels_in_the_scores():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal((5, 128)), rng.standard_normal((7, 128))
    R = oracle.rotation(128, np.where(rng.random(128) < 0.5, -1.0, 1.0))
    assert np.allclose((q @ R) @ (k @ R).T, q @ k.T, atol=1e-12)


def test_on_grid_inputs_give_exact_attention():
    # values already on the e4m3 grid with a head maximum of 448: the per-head
    # scale is 1 and quantisation changes nothing
    rng = np.random.default_rng(3)
    B, H, S, D = 2, 2, 24, 16
    g = e4m3_grid()

    def on_grid(shape):
        x = rng.choice(g[np.abs(g) <= 64], size=shape)
        x[..., 0, 0] = 448.0
        return x

    q, k = on_grid((B, H, S, D)), on_grid((B, H, S, D))
    v = rng.standard_normal((B, H, S, D))
    O8, L8 = oracle.attention_forward_fp8(q, k, v, 1e-3, signs=None, mod=oracle.MOD_CAUSAL)
    O, L = oracle.attention_forward(q, k, v, 1e-3, oracle.MOD_CAUSAL)
    assert np.array_equal(O8, O) and np.array_equal(L8, L)


def outlier_inputs(seed, B=1, H=4, S=256, D=128, n_out=4, mag=20.0):
    """N(0, 1) queries and keys whose first n_out channels are scaled by mag
    (outlier features), and N(0, 1) values."""
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, H, S, D)) for _ in range(3))
    q[..., :n_out] *= mag
    k[..., :n_out] *= mag
    return q, k, v


def test_rotation_lowers_the_fp8_error_on_outliers():
    # the pages report about 2.6 times lower error with the rotation; on
    # these outlier inputs the oracle must show a clear gain
    q, k, v = outlier_inputs(4)
    scale = 128 ** -0.5 / 4
    O, _ = oracle.attention_forward(q, k, v, scale)
    signs = np.where(np.random.default_rng(5).random(128) < 0.5, -1.0, 1.0)
    O_plain, _ = oracle.attention_forward_fp8(q, k, v, scale, signs=None)
    O_rot, _ = oracle.attention_forward_fp8(q, k, v, scale, signs=signs)
    err_plain = np.sqrt(np.mean((O_plain - O) ** 2))
    err_rot = np.sqrt(np.mean((O_rot - O) ** 2))
    assert err_plain / err_rot > 1.5, (err_plain, err_rot)


def test_rotation_changes_little_without_outliers():
    # Gaussian features have no outliers to spread: both errors are of one size
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((1, 2, 128, 64)) for _ in range(3))
    scale = 64 ** -0.5
    O, _ = oracle.attention_forward(q, k, v, scale)
    signs = np.where(rng.random(64) < 0.5, -1.0, 1.0)
    e_plain = np.sqrt(np.mean((oracle.attention_forward_fp8(q, k, v, scale)[0] - O) ** 2))
    e_rot = np.sqrt(np.mean((oracle.attention_forward_fp8(q, k, v, scale, signs=signs)[0] - O) ** 2))
    assert 0.5 < e_plain / e_rot < 2.0


def test_outlier_recipe_reproduces_the_printed_gain():
    # The pages report about 2.6 times lower FP8 attention error with the
    # rotation, on inputs they do not describe.  With 8 of 128 channels at 5
    # times the scale (the recipe of the FP8 workload), the oracle's gain lies
    # around that figure.
    ratios = []
    for seed in range(3):
        q, k, v = outlier_inputs(10 + seed, n_out=8, mag=5.0)
        scale = 128 ** -0.5
        O, _ = oracle.attention_forward(q, k, v, scale)
        signs = np.where(np.random.default_rng(50 + seed).random(128) < 0.5, -1.0, 1.0)
        e_plain = np.sqrt(np.mean((oracle.attention_forward_fp8(q, k, v, scale)[0] - O) ** 2))
        e_rot = np.sqrt(np.mean((oracle.attention_forward_fp8(q, k, v, scale, signs=signs)[0] - O) ** 2))
        ratios.append(e_plain / e_rot)
    assert 2.0 < np.mean(ratios) < 3.5, ratios


@pytest.mark.parametrize("D", [2, 16, 128])
def test_fwht_is_the_hadamard_product(D):
    # integer inputs: both sides are exact in fp64
    x = np.random.default_rng(D).integers(-50, 50, size=(3, D)).astype(np.float64)
    assert np.array_equal(oracle.fwht(x), x @ oracle.hadamard(D))
    # and fp32 butterflies stay within rounding of the exact product
    xf = np.random.default_rng(D + 1).standard_normal((3, D)).astype(np.float32)
    assert np.allclose(oracle.fwht(xf), xf.astype(np.float64) @ oracle.hadamard(D), rtol=0, atol=1e-5 * D)


def test_fp32_prep_agrees_with_the_definition():
    # the fp32 step sequence quantises to the same codes as the fp64 rotation
    # except where an fp32 rounding moves a value across a tie
    q, _, _ = outlier_inputs(20, H=2, S=128)
    signs = np.where(np.random.default_rng(21).random(128) < 0.5, -1.0, 1.0)
    codes32, s32 = oracle.prep_fp32(q, signs)
    codes64, s64 = oracle.quantize_per_head(q @ oracle.rotation(128, signs))
    assert np.allclose(s32, s64, rtol=1e-6)
    differ = codes32 != codes64
    assert differ.mean() < 1e-3
    # where they differ, they are neighbours on the grid
    g = e4m3_grid()
    idx32 = np.searchsorted(g, codes32[differ])
    idx64 = np.searchsorted(g, codes64[differ])
    assert np.all(np.abs(idx32 - idx64) == 1)
