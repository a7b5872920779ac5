"""Pins for the oracle's low-bit KV cache (brentwoodlivery.com 5.3.18:
affine quantization s = (r_max - r_min)/(2^b - 1), z = round(-r_min/s),
q = round(r/s) + z, r_hat = s (q - z)).  An exact-rational restatement of
those formulas reproduces the page's worked example and is the yardstick for
the oracle's fp32 quantizer; the int8 decode is pinned to library attention
on the dequantized rows."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_481_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def exact_affine(values, bits):
    """The page's formulas in exact rational arithmetic (round half to even)."""
    vals = [Fraction(v) for v in values]
    qmax = 2 ** bits - 1
    s = (max(vals) - min(vals)) / qmax
    z = round(-min(vals) / s)
    q = [min(max(round(v / s) + z, 0), qmax) for v in vals]
    return s, z, q


def test_page_worked_example_exactly():
    g = json.load(open(os.path.join(GOLDEN, "quant_example.json")))
    s, z, q = exact_affine([Fraction(g["r_min"]), Fraction(g["r_max"]), Fraction(g["r"])],
                           g["bits"])
    assert s == Fraction(g["s"]) and z == g["z"] and q[2] == g["q"]
    r_hat = s * (q[2] - z)
    assert r_hat == Fraction(g["r_hat"])
    assert abs(r_hat - Fraction(g["r"])) == Fraction(g["error"]) == s / 2


def test_oracle_4bit_on_the_example_values():
    # fp16 rounds 0.35 up to 0.3501, away from the tie: the page's code 10
    x = np.array([[-0.6, 0.9, 0.35]], np.float16)
    codes, params = oracle.quantize_rows(x, bits=4)
    assert codes.tolist() == [[0, 15, 10]]
    assert abs(params[0, 0] - 0.1) < 1e-6 and params[0, 1] == 6


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fp32_quantizer_agrees_with_exact_rationals(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((300, 128)) * rng.uniform(0.01, 20, (300, 1))
         + rng.uniform(-5, 5, (300, 1))).astype(np.float16)
    codes, params = oracle.quantize_rows(x, bits=8)
    mismatched = 0
    for row, c, (s32, z32) in zip(x, codes, params):
        s, z, q = exact_affine([float(v) for v in row], 8)
        assert abs(float(s32) - float(s)) <= 2 ** -23 * float(s)      # one fp32 rounding
        assert int(z32) == z or abs(float(-Fraction(float(row.min())) / s) % 1 - Fraction(1, 2)) < 1e-4
        for v, got, want in zip(row, c, q):
            if got != want:
                mismatched += 1
                # only where r/s sits on a rounding tie, within fp32 error
                frac = (Fraction(float(v)) / s) % 1
                assert abs(frac - Fraction(1, 2)) < Fraction(1, 10**4)
    assert mismatched <= 3


def test_reconstruction_error_is_half_a_step():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((400, 128)) * 3).astype(np.float16)
    codes, params = oracle.quantize_rows(x)
    assert codes.min() >= 0 and codes.max() <= 255
    err = np.abs(oracle.dequantize(codes, params) - x.astype(np.float64))
    step = params[:, :1].astype(np.float64)
    # half a step, except the clamped extremes of a row (at most 1.5 steps)
    assert (err <= 1.5 * step + 1e-9).all()
    assert (err <= 0.5 * step * (1 + 1e-5) + 1e-12).mean() > 0.99


def test_constant_and_zero_rows_reconstruct_exactly():
    x = np.array([[0.75] * 64, [-3.5] * 64, [0.0] * 64], np.float16)
    codes, params = oracle.quantize_rows(x)
    assert np.array_equal(oracle.dequantize(codes, params), x.astype(np.float64))


def _int8_pool(wl):
    """Quantize every context token into an int8 pool with the oracle."""
    nb, h, bs, d = wl.k_cache.shape
    kc = np.zeros((nb, h, bs, d), np.uint8)
    vc = np.zeros_like(kc)
    kp = np.zeros((nb, h, bs, 2), np.float32)
    vp = np.zeros_like(kp)
    for b, length in enumerate(wl.context_lens):
        pos = np.arange(length)
        slots = wl.block_tables[b, pos // bs].astype(np.int64) * bs + pos % bs
        k = wl.logical_k[b].permute(1, 0, 2).contiguous().numpy()
        v = wl.logical_v[b].permute(1, 0, 2).contiguous().numpy()
        kc, vc, kp, vp = oracle.reshape_and_cache_int8(k, v, kc, vc, kp, vp, slots, bs)
    return kc, vc, kp, vp


@pytest.mark.parametrize("seed,d,bs,lens", [(1, 128, 16, [1, 17, 100]), (2, 64, 8, [9, 64, 33])])
def test_int8_decode_equals_library_attention_on_dequantized_rows(seed, d, bs, lens):
    wl = workloads.make_random(seed, lens, num_heads=3, head_dim=d, block_size=bs, pool_factor=2.0)
    kc, vc, kp, vp = _int8_pool(wl)
    out = oracle.paged_decode_int8(wl.q.numpy(), kc, vc, kp, vp, wl.block_tables,
                                   wl.context_lens, wl.scale)
    for b, length in enumerate(wl.context_lens):
        codes_k, par_k = oracle.quantize_rows(wl.logical_k[b].reshape(-1, d).numpy())
        codes_v, par_v = oracle.quantize_rows(wl.logical_v[b].reshape(-1, d).numpy())
        kh = torch.from_numpy(oracle.dequantize(codes_k, par_k)).view(3, length, d)
        vh = torch.from_numpy(oracle.dequantize(codes_v, par_v)).view(3, length, d)
        for h in range(3):
            qv = wl.q[b, h].double().view(1, 1, 1, d)
            ref = F.scaled_dot_product_attention(qv, kh[h].view(1, 1, length, d),
                                                 vh[h].view(1, 1, length, d),
                                                 scale=wl.scale).view(-1).numpy()
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-11, atol=1e-12)


def test_int8_cache_write_places_rows_at_their_slots():
    wl = workloads.make_random(3, [20, 5], num_heads=2, head_dim=64, block_size=16,
                               pool_factor=2.0)
    kc, vc, kp, vp = _int8_pool(wl)
    for b, length in enumerate(wl.context_lens):
        t = int(length) - 1
        p = wl.block_tables[b, t // 16]
        codes, par = oracle.quantize_rows(wl.logical_k[b][:, t].numpy())
        assert np.array_equal(kc[p, :, t % 16], codes)
        assert np.array_equal(kp[p, :, t % 16], par)
