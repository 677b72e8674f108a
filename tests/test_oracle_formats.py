"""Pins for the oracle's number formats and quantizer (CPU only).

Each test checks the oracle against something other than itself: torch's own FP8 cast,
the bit-field definition of E2M1, numpy's round-half-to-even, values printed on the pages,
or values derived by hand from the format definition.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import fp4kv_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _all_finite_bf16_nonneg():
    bits = np.arange(0, 0x7F80, dtype=np.uint16)  # +0 .. largest finite
    return bits, O.bf16_bits_to_f64(bits)


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256)
    ours = O.e4m3_decode(codes)
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert len(O.E4M3_POS_VALUES) == 127 and np.all(np.diff(O.E4M3_POS_VALUES) > 0)


def test_bf16_bits_to_f64_matches_torch_all_patterns():
    """Every one of the 65,536 bf16 bit patterns decodes to torch's own bfloat16 -> float64
    value (NaN patterns to NaN), so a wrong shift or width fails here."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):  # the NaN patterns
        ours = O.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))  # -0 stays -0
    assert nan.sum() == 2 * 127  # exponent all ones, mantissa non-zero, either sign


def test_e2m1_values_from_bitfields():
    # E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal.
    vals = []
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = (m * 0.5) if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
        vals.append(-mag if s else mag)
    assert np.array_equal(O.e2m1_decode(np.arange(16)), np.array(vals))


def test_format_max_is_the_pages_2688():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    assert O.E4M3_MAX == facts["e4m3_max"]["value"]
    assert O.E2M1_MAX == facts["e2m1_max"]["value"]
    assert O.E4M3_MAX * O.E2M1_MAX == facts["fp4_format_max"]["value"]
    assert O.GROUP == facts["channels_per_scale"]["value"]


def test_e4m3_rounding_matches_torch_cast():
    # every non-negative finite bf16 value up to 448, plus every E4M3 midpoint and its
    # float32 neighbours (torch casts through float32, so inputs must be fp32 values)
    _, v = _all_finite_bf16_nonneg()
    v = v[v <= 448]
    T = O.E4M3_POS_VALUES
    mids = ((T[:-1] + T[1:]) / 2).astype(np.float32)
    extra = np.concatenate([mids, np.nextafter(mids, np.float32(0)),
                            np.nextafter(mids, np.float32(1e9))]).astype(np.float64)
    x = np.concatenate([v, extra, np.linspace(0, 448, 100001)])
    ours = O.e4m3_round_sat(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
    assert np.array_equal(ours, ref)


def test_e4m3_saturates_above_448():
    x = np.array([448.0, 460.0, 464.0, 500.0, 2688.0, 1e30])
    assert np.all(O.e4m3_round_sat(x) == 0x7E)


def _e2m1_round_half_even_per_binade(r):
    """Independent E2M1 rounding: in each binade the grid is uniform, so round r/step
    half-to-even with numpy and saturate at 6."""
    r = np.asarray(r, dtype=np.float64)
    step = np.where(r < 2, 0.5, np.where(r < 4, 1.0, 2.0))
    v = np.minimum(np.round(r / step) * step, 6.0)
    return np.searchsorted(O.E2M1_POS_VALUES, v)  # value -> magnitude code


def test_e2m1_rounding_vs_half_even_per_binade():
    G = O.E2M1_POS_VALUES
    mids = (G[:-1] + G[1:]) / 2
    r = np.concatenate([
        G, mids, np.nextafter(mids, 0), np.nextafter(mids, 10),
        np.linspace(0, 8, 200001), [6.0, 6.5, 7.0, 100.0, 1e30]])
    assert np.array_equal(O.e2m1_mag_round_sat(r), _e2m1_round_half_even_per_binade(r))


def test_scale_exhaustive_over_bf16_amax():
    # S = E4M3_RNE_sat(amax / 6) for every non-negative finite bf16 amax, checked
    # against torch's cast (round-to-nearest-even) plus explicit saturation at 448.
    _, amax = _all_finite_bf16_nonneg()
    q = amax / 6.0
    ref = torch.from_numpy(np.minimum(q, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8)
    ours = O.e4m3_round_sat(q)
    assert np.array_equal(ours, ref.numpy().astype(np.int64))
    assert np.all(ours[amax >= 2688] == 0x7E)  # the format's largest scale


@pytest.mark.slow
def test_codes_exhaustive_bf16_x_all_scales():
    # every finite bf16 |x| against every positive E4M3 scale
    _, v = _all_finite_bf16_nonneg()
    S = O.E4M3_POS_VALUES[1:]
    for s in S:
        r = v / s
        assert np.array_equal(O.e2m1_mag_round_sat(r), _e2m1_round_half_even_per_binade(r)), s


def test_golden_hand_derived_example():
    g = json.load(open(os.path.join(GOLDEN, "quant_example.json")))
    x = np.array(g["rows"], dtype=np.float64)
    x[0, 7] = -0.0
    x[1, 3] = -0.0
    packed, scales = O.kv_quant_fp4(x)
    assert scales.tolist() == g["scales"]
    assert [bytes(r).hex().upper() for r in packed] == g["packed_hex"]
    codes = np.empty_like(x, dtype=np.int64)
    codes[:, 0::2] = packed & 15
    codes[:, 1::2] = packed >> 4
    assert codes.tolist() == g["codes"]


def test_quant_error_bound_and_saturation():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((512, 512)) * np.exp(rng.uniform(-20, 8, (512, 1)))
    x = O.bf16_bits_to_f64((x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))
    packed, scales = O.kv_quant_fp4(x)
    xh = O.kv_dequant_fp4(packed, scales)
    S = np.repeat(O.e4m3_decode(scales), 16, axis=1)
    inside = np.abs(x) <= 6 * S
    # inside the representable range the error is at most half the widest grid step (2S)
    assert np.all(np.abs(x - xh)[inside] <= S[inside])
    # outside it the value saturates to +-6S with the sign kept
    assert np.all(xh[~inside] == np.sign(x[~inside]) * 6 * S[~inside])
    assert np.all(np.abs(xh) <= 2688)
    assert np.array_equal(np.signbit(xh) | (xh == 0), np.signbit(x) | (xh == 0))


def test_requantize_is_identity_when_group_max_code_is_6():
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 16, (64, 512))
    codes[:, ::16] = rng.choice([7, 15], (64, 32))  # every group holds +-6
    s = rng.integers(1, 127, (64, 32))
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    xh = O.kv_dequant_fp4(packed, s.astype(np.uint8))
    p2, s2 = O.kv_quant_fp4(xh)
    # -0 codes (8) come back as 8, +0 as 0: the sign bit is preserved exactly
    assert np.array_equal(s2, s) and np.array_equal(p2, packed)


def test_rows_within_the_pages_norm_bound_never_clamp_the_scale():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    d = facts["kv_latent_channels"]["value"]
    rng = np.random.default_rng(2)
    x = rng.standard_normal((256, d))
    x *= np.sqrt(d) / np.linalg.norm(x, axis=1, keepdims=True)  # L2 norm sqrt(512)
    x[0] = 0
    x[0, 5] = np.sqrt(d)  # all mass on one channel: |x| = 22.6
    assert np.abs(x).max() <= facts["per_channel_bound"]["value"] + 0.03
    _, scales = O.kv_quant_fp4(x)
    assert scales.max() < 0x7E  # the scale never reaches 448


def test_packed_row_size_and_890_bytes_per_token():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    assert O.packed_row_bytes(512) == 256 + 32 == 288
    # One decomposition of the pages' 890 B/token (our arithmetic, not the pages'):
    # 2.5 cached entries per token, each a 288 B FP4 row plus a 68 B indexer key
    # (64 B of 4-bit codes for 128 dims and one 4 B scale).
    assert O.global_kv_bytes_per_token(2.5, 512, 68) == facts["global_kv_bytes_per_token"]["value"]


def test_swa_fp8_golden_codes():
    """Hand-derived E4M3 codes of the sliding-window KV's FP8 storage (tests/golden)."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "swa_fp8_example.json")))
    for c in g["cases"]:
        assert int(O.swa_quant_fp8(np.float64(c["x"]))) == c["code"], c["why"]
