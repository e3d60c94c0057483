"""Pins of the oracle's int8 KV pieces against things other than themselves.

The row quantizer follows the quantizer that "Gemma 4 Technical Report",
Quantization and Efficiency, states (scale = (2^b - 1) / (max - min),
code = round((x - min) * scale), dequantized min + code / scale), read with
b = 8 and one (min, step) pair per cached row. The page's own worked example
(int2/int4 codes of two channels) is not self-consistent (its scales do not
follow from its formula), so the pins here are hand-derived rows, exact
arithmetic, and invariants. The dense attention over given keys is pinned
against the oracle's bf16 attention, an independent route to the same
definition.
"""
import numpy as np
import pytest
import torch

import oracle


def bf16_bits(x):
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b):
    return torch.from_numpy(np.asarray(b, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def rand_bits(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    t = (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_hand_derived_row():
    # min -1, max 3: scale = 255 / 4 = 63.75; (x + 1) * 63.75 = 0, 63.75, 95.625, 255
    codes, lo, step = oracle.quantize_rows_u8(bf16_bits([[-1.0, 0.0, 0.5, 3.0]]))
    assert codes.tolist() == [[0, 64, 96, 255]]
    assert lo.tolist() == [-1.0]
    assert step[0] == np.float32(4.0) / np.float32(255.0)


def test_ties_round_to_even():
    # min 0, max 255: scale = 1, so 2.5 and 3.5 are exact ties
    codes, lo, step = oracle.quantize_rows_u8(bf16_bits([[0.0, 255.0, 2.5, 3.5, 4.5]]))
    assert codes.tolist() == [[0, 255, 2, 4, 4]]
    assert lo[0] == 0.0 and step[0] == 1.0


def test_constant_row():
    codes, lo, step = oracle.quantize_rows_u8(bf16_bits([[1.5] * 8, [-2.0] * 8]))
    assert (codes == 0).all()
    assert lo.tolist() == [1.5, -2.0] and (step == 0).all()
    assert (oracle.dequantize_rows_u8(codes, lo, step) == np.array([[1.5] * 8, [-2.0] * 8])).all()


def test_codes_against_exact_rounding():
    """Away from ties, the code is the nearest integer to (x - min) / (max - min) * 255
    computed exactly (fp64); the fp32 decision may differ only within fp32
    rounding of a tie."""
    x = rand_bits((64, 256), seed=5, scale=3.0)
    codes, lo, step = oracle.quantize_rows_u8(x)
    xv = bits_to_f64(x)
    mn, mx = xv.min(axis=1, keepdims=True), xv.max(axis=1, keepdims=True)
    t = (xv - mn) / (mx - mn) * 255.0
    exact = np.rint(t)
    near_tie = np.abs(np.abs(t - np.floor(t)) - 0.5) < 1e-4
    assert (codes[~near_tie] == exact[~near_tie]).all()
    assert (np.abs(codes.astype(np.int64) - exact) <= 1).all()
    assert (codes.min(axis=1) == 0).all() and (codes.max(axis=1) == 255).all()
    assert (lo == mn[:, 0]).all()


def test_round_trip_error_bound_and_monotone():
    x = rand_bits((32, 512), seed=6, scale=0.7)
    codes, lo, step = oracle.quantize_rows_u8(x)
    xv = bits_to_f64(x)
    xh = oracle.dequantize_rows_u8(codes, lo, step)
    # half a step, plus the fp32 rounding of the scale and of the stored step
    bound = 0.5 * step.astype(np.float64)[:, None] * (1 + 1e-5) + 1e-6 * np.abs(xv).max()
    assert (np.abs(xh - xv) <= bound).all()
    for r in range(x.shape[0]):
        order = np.argsort(xv[r], kind="stable")
        assert (np.diff(codes[r][order].astype(np.int64)) >= 0).all()


def test_dense_attention_matches_bf16_oracle():
    """attend_rows over bf16-valued keys equals hlg_attention on the same
    values (keys arrive rotated: rot_from beyond every key; the query is
    rotated at its position by both routes)."""
    B, T, Hq, Hkv, D = 2, 37, 4, 2, 64
    q = rand_bits((B, 1, Hq, D), seed=7)
    k = rand_bits((B, T, Hkv, D), seed=8)
    v = rand_bits((B, T, Hkv, D), seed=9)
    lens = [37, 20]
    scale = 0.125
    ref, ref_lse = oracle.attention(q, k, v, q_pos0=[L - 1 for L in lens], n_keys=lens, rot_from=[10 ** 9] * B,
                                    window=0, rope_frac=1.0, theta=1e4, scale=scale)
    G = Hq // Hkv
    rows_q, begin, count = [], [], []
    keys = bits_to_f64(k).transpose(0, 2, 1, 3).reshape(B * Hkv * T, D)
    vals = bits_to_f64(v).transpose(0, 2, 1, 3).reshape(B * Hkv * T, D)
    for b in range(B):
        for h in range(Hq):
            rows_q.append(oracle.rope_bf16(q[b, 0, h], lens[b] - 1, 1.0, 1e4))
            begin.append((b * Hkv + h // G) * T)
            count.append(lens[b])
    out, lse = oracle.attend_rows(np.array(rows_q), keys, vals, begin, count, scale)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
    assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_dense_attention_closed_forms():
    rng = np.random.default_rng(3)
    k = rng.standard_normal((9, 16))
    v_const = np.tile(rng.standard_normal(16), (9, 1))
    q = rng.standard_normal((2, 16))
    out, _ = oracle.attend_rows(q, k, v_const, [0, 4], [9, 5], 0.3)
    assert np.allclose(out, v_const[:2], atol=1e-13)           # constant V gives that constant
    v = rng.standard_normal((9, 16))
    out, lse = oracle.attend_rows(np.zeros((1, 16)), k, v, [2], [4], 1.0)
    assert np.allclose(out[0], v[2:6].mean(axis=0), atol=1e-13)  # Q = 0: mean of the visible V
    assert np.isclose(lse[0], np.log(4.0))
    out, _ = oracle.attend_rows(q[:1], k, v, [6], [1], 1.0)
    assert np.allclose(out[0], v[6], atol=1e-15)                # one key: its value


def test_rejects_out_of_range_keys():
    with pytest.raises(ValueError):
        oracle.attend_rows(np.zeros((1, 4)), np.zeros((3, 4)), np.zeros((3, 4)), [2], [2], 1.0)
