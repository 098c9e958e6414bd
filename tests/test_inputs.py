"""Pins of the seeded input generators (CPU only)."""
import os

import numpy as np
import pytest
import torch

from moe_inputs import CONFIGS, config, gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kat_rows():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                v = [int(t, 16) for t in line.split()]
                rows.append((v[0:4], v[4:6], tuple(v[6:10])))
    return rows


@pytest.mark.parametrize("ctr,key,expect", _kat_rows())
def test_philox_known_answers(ctr, key, expect):
    assert gen.philox4x32_10(ctr, key) == expect


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    a = np.concatenate([rng.standard_normal(200000).astype(np.float32) * 3,
                        # exact ties between two bf16 values, both parities
                        (np.arange(1, 4000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
                        np.array([0.0, -0.0, 1e-40, -3.4e38, 65504.0], dtype=np.float32)])
    ours = gen.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(gen.bf16_bits_to_f32(ours),
                                  torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_e4m3_encode_decode_match_torch():
    rng = np.random.default_rng(2)
    vals = [rng.standard_normal(100000).astype(np.float32) * 50,
            rng.uniform(-0.02, 0.02, 100000).astype(np.float32),
            np.array([0.0, -0.0, 448.0, -448.0, 2 ** -9, 2 ** -10, 3 * 2 ** -11, 2 ** -6,
                      1.0625, 1.1875, 240.0, 256.0, 272.0, 288.0], dtype=np.float32)]
    # midpoints between adjacent e4m3 values exercise round-half-even
    finite = np.sort(np.unique(gen.E4M3_VALUES[np.isfinite(gen.E4M3_VALUES)]))
    vals.append(((finite[1:] + finite[:-1]) / 2).astype(np.float32))
    a = np.concatenate(vals)
    a = np.clip(a, -448, 448)
    ours = gen.f32_to_e4m3_bits(a)
    ref = torch.from_numpy(a).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)
    codes = np.arange(256, dtype=np.uint8)
    tv = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    ok = np.isfinite(tv)
    np.testing.assert_array_equal(gen.E4M3_VALUES[ok], tv[ok])
    assert np.isnan(gen.E4M3_VALUES[~ok]).all()


def test_irwin_hall_shape():
    c = config(2)
    e = gen.expert_host(c, 0, 3)
    v = gen.bf16_bits_to_f32(e.gu).astype(np.float64).ravel()
    n = v.size
    assert abs(v.mean()) < 5 * c.w_sigma / np.sqrt(n)
    assert abs(v.std() / c.w_sigma - 1) < 2e-3
    # support of the 8-uniform sum: (262140 / sqrt(2863311530)) sd = 4.899 sd
    assert np.abs(v).max() <= 4.9 * c.w_sigma * (1 + 2 ** -8)
    # excess kurtosis of an Irwin-Hall sum of 8 uniforms is -1.2/8
    k = ((v - v.mean()) ** 4).mean() / v.var() ** 2 - 3
    assert abs(k + 0.15) < 0.02


def test_expert_keys_distinct_and_deterministic():
    c = config(1)
    a = gen.expert_host(c, 0, 1)
    b = gen.expert_host(c, 0, 1)
    d = gen.expert_host(c, 0, 2)
    np.testing.assert_array_equal(a.gu, b.gu)
    assert (a.gu != d.gu).mean() > 0.9
    n = a.down.size
    assert (a.gu.reshape(-1)[:n] != a.down.reshape(-1)).mean() > 0.9
    keys = {gen.weight_key(c, l, e, t) for l in range(2) for e in range(9) for t in range(2)}
    assert len(keys) == 2 * 9 * 2


def test_e4m3_block_scales():
    c = config(5).with_(H=256, I=128)
    e = gen.expert_host(c, 0, 0)
    assert e.gu.dtype == np.uint8 and e.gu_scale.shape == (2, 2)
    # the largest code of every block is the saturation value 448 (0x7E) in magnitude
    for br in range(2):
        for bc in range(2):
            blk = e.gu[br * 128:(br + 1) * 128, bc * 128:(bc + 1) * 128]
            assert (blk & 0x7F).max() == 0x7E
    w = e.gu_f64()
    assert abs(w.std() / c.w_sigma - 1) < 0.05


def test_sequence_lengths_cv():
    c = config(4)
    L = np.array(gen.seq_lengths(c), dtype=np.float64)
    assert L.sum() == c.T and len(L) == c.seq_count and (L > 0).all()
    assert abs(L.std() / L.mean() - c.seq_cv) < 1e-3


def test_zipf_bias_ranks():
    c = config(4)
    b = gen.gen_bias(c)
    s = np.sort(b)[::-1].astype(np.float64)
    r = np.arange(1, c.E + 1, dtype=np.float64)
    np.testing.assert_allclose(s, c.zipf_amp * r ** -c.zipf_s, rtol=1e-6)
    hot = np.argsort(-b)[:8]
    assert (hot < c.local_count).any() and (hot >= c.local_count).any()


def test_layer_inputs_shapes():
    for cid, c in CONFIGS.items():
        if c.T * c.H > 2 ** 24:
            continue
        li = gen.layer_inputs(c)
        assert li.x.shape == (c.T, c.H) and li.wg.shape == (c.E, c.H)
        if c.x_dtype == "bf16":
            np.testing.assert_array_equal(gen.bf16_bits_to_f32(li.x_bits), li.x)
