"""Pins of the fp64 oracle against things other than itself: hand-derived
closed forms on tiny inputs, hand-listed visible sets, library routines on
special cases (torch SDPA in fp64, numpy complex rotation), invariants, and
the figures the pages print (tests/golden/page_figures.json).

Each pin is chosen so that a plausible mistake (dropped term, wrong sign or
index, transposed operand, off-by-one window) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def bf16_bits(x):
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b):
    return torch.from_numpy(np.asarray(b, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def rand_bits(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    t = (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def complex_rope(x, pos, frac, theta):
    """Independent route: rotate pairs as complex numbers (numpy)."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    n_rot = int(math.floor(frac * (D // 2)))
    z = x[..., 0::2] + 1j * x[..., 1::2]
    i = np.arange(D // 2)
    ang = np.where(i < n_rot, pos * theta ** (-2.0 * i / D), 0.0)
    z = z * np.exp(1j * ang)
    y = np.empty_like(x)
    y[..., 0::2] = z.real
    y[..., 1::2] = z.imag
    return y


# --------------------------------------------------------------------------- tiny hand examples
def test_hand_example_window2_nope(oracle):
    """D=2, NoPE, window 2 (key j visible iff i-2 < j <= i), scale 1.
    q0=(1,0) q1=(0,1) q2=(1,1); k0=(1,0) k1=(0,2) k2=(1,-1); v0=(1,0) v1=(0,1) v2=(2,2).
    Row0 sees {0}: s=1 -> o=v0, lse=1.
    Row1 sees {0,1}: s=(0,2) -> o=(1,e^2)/(1+e^2), lse=log(1+e^2).
    Row2 sees {1,2}: s=(2,0) -> o=(2, e^2+2)/(1+e^2), lse=log(1+e^2)."""
    q = bf16_bits([[1, 0], [0, 1], [1, 1]]).reshape(1, 3, 1, 2)
    k = bf16_bits([[1, 0], [0, 2], [1, -1]]).reshape(1, 3, 1, 2)
    v = bf16_bits([[1, 0], [0, 1], [2, 2]]).reshape(1, 3, 1, 2)
    out, lse = oracle.attention(q, k, v, q_pos0=0, n_keys=3, rot_from=0, window=2,
                                rope_frac=0.0, theta=1e4, scale=1.0)
    e2 = math.exp(2.0)
    exp_out = np.array([[1, 0], [1 / (1 + e2), e2 / (1 + e2)], [2 / (1 + e2), (e2 + 2) / (1 + e2)]])
    exp_lse = np.array([1.0, math.log(1 + e2), math.log(1 + e2)])
    np.testing.assert_allclose(out, exp_out, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, exp_lse, rtol=0, atol=1e-15)


def test_hand_example_global_row2(oracle):
    """Same inputs, global (window 0): row 2 sees {0,1,2} with s=(1,2,0)."""
    q = bf16_bits([[1, 0], [0, 1], [1, 1]]).reshape(1, 3, 1, 2)
    k = bf16_bits([[1, 0], [0, 2], [1, -1]]).reshape(1, 3, 1, 2)
    v = bf16_bits([[1, 0], [0, 1], [2, 2]]).reshape(1, 3, 1, 2)
    out, lse = oracle.attention(q, k, v, q_pos0=0, n_keys=3, rot_from=0, window=0,
                                rope_frac=0.0, theta=1e4, scale=1.0, rows=[[0, 0, 2]])
    e, e2 = math.e, math.exp(2.0)
    z = e + e2 + 1
    np.testing.assert_allclose(out[0], [(e + 2) / z, (e2 + 2) / z], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], math.log(z), rtol=0, atol=1e-15)


def test_hand_example_rope_sign(oracle):
    """D=2, full RoPE: pair 0 turns by the position (theta^0 = 1). With q=(1,0)
    and k=(0,1): <R_p q, R_j k> = sin(p - j); a flipped rotation sign gives
    sin(j - p). Query at position 2, keys 0..2, v = (1,0), (0,1), (1,1)."""
    q = bf16_bits([[0, 0], [0, 0], [1, 0]]).reshape(1, 3, 1, 2)
    k = bf16_bits([[0, 1], [0, 1], [0, 1]]).reshape(1, 3, 1, 2)
    v = bf16_bits([[1, 0], [0, 1], [1, 1]]).reshape(1, 3, 1, 2)
    out, lse = oracle.attention(q, k, v, q_pos0=0, n_keys=3, rot_from=0, window=0,
                                rope_frac=1.0, theta=1e4, scale=1.0, rows=[[0, 0, 2]])
    s = np.array([math.sin(2.0), math.sin(1.0), 0.0])
    w = np.exp(s) / np.exp(s).sum()
    np.testing.assert_allclose(out[0], [w[0] + w[2], w[1] + w[2]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0], math.log(np.exp(s).sum()), rtol=0, atol=1e-14)


def test_rope_frequency_uses_full_head_dim(oracle):
    """D=4, theta=100: pair 1 turns at 100^(-2/4) = 0.1 rad per position.
    rope_frac=0.5 rotates only pair 0 (floor(0.5*2) = 1 pair)."""
    x = np.array([0.0, 0.0, 1.0, 0.0])
    y = oracle.rope(x, pos=7, rope_frac=1.0, theta=100.0)
    np.testing.assert_allclose(y, [0, 0, math.cos(0.7), math.sin(0.7)], rtol=0, atol=1e-15)
    y = oracle.rope(x, pos=7, rope_frac=0.5, theta=100.0)
    np.testing.assert_array_equal(y, x)
    x0 = np.array([1.0, 0.0, 0.0, 0.0])
    y = oracle.rope(x0, pos=7, rope_frac=0.5, theta=100.0)
    np.testing.assert_allclose(y, [math.cos(7), math.sin(7), 0, 0], rtol=0, atol=1e-15)


# --------------------------------------------------------------------------- p-RoPE
def test_p_rope_quarter_of_pairs(oracle):
    """rope_frac 0.25 at D=512: 64 pairs (dims 0..127) rotate, theta=1e6;
    dims 128..511 equal the input bit for bit; agrees with complex rotation."""
    figs = json.load(open(GOLDEN))["p_rope"]
    assert oracle.rope_n_rotated_pairs(512, figs["p"]) == 64
    assert oracle.rope_n_rotated_pairs(256, 1.0) == 128
    assert oracle.rope_n_rotated_pairs(512, 0.0) == 0
    x = bits_to_f64(rand_bits((512,), 11))
    for pos in (0, 1, 4095, 262143):
        y = oracle.rope(x, pos, figs["p"], figs["theta"])
        np.testing.assert_array_equal(y[128:], x[128:])
        np.testing.assert_allclose(y, complex_rope(x, pos, figs["p"], figs["theta"]), rtol=0, atol=1e-9)
        if pos:
            assert not np.allclose(y[:2], x[:2])


def test_rope_identities(oracle):
    """Norm preservation; relative position: <R_m q, R_n k> = <R_(m-n) q, k>;
    rope_frac = 0 is the identity (NoPE)."""
    q = bits_to_f64(rand_bits((256,), 1))
    k = bits_to_f64(rand_bits((256,), 2))
    for frac, theta in ((1.0, 1e4), (0.25, 1e6)):
        for m, n in ((5, 3), (1000, 17), (262143, 131072)):
            qm = oracle.rope(q, m, frac, theta)
            kn = oracle.rope(k, n, frac, theta)
            assert abs(np.linalg.norm(qm) - np.linalg.norm(q)) < 1e-12 * np.linalg.norm(q)
            rel = oracle.rope(q, m - n, frac, theta)
            assert abs(qm @ kn - rel @ k) < 1e-8 * (np.abs(q).sum() * np.abs(k).max())
    np.testing.assert_array_equal(oracle.rope(q, 12345, 0.0, 1e4), q)


# --------------------------------------------------------------------------- masks
def test_visible_sets_hand_listed(oracle):
    """Window 3, positions 0..5: the window holds 3 keys including the query."""
    listed = [[0], [0, 1], [0, 1, 2], [1, 2, 3], [2, 3, 4], [3, 4, 5]]
    for p, want in enumerate(listed):
        lo, hi, cnt = oracle.visible_range(p, 3, 6)
        assert list(range(lo, hi + 1)) == want and cnt == len(want)
    # global: everything up to and including the query
    for p in range(6):
        assert oracle.visible_range(p, 0, 6) == (0, p, p + 1)
    # a decode query sees its whole context (n_keys bound)
    assert oracle.visible_range(99, 0, 100) == (0, 99, 100)
    assert oracle.visible_range(99, 16, 100) == (84, 99, 16)


def test_visible_count_formula(oracle):
    """Sum over queries of min(i+1, W) -- the local-layer work count."""
    S, W = 1000, 512
    tot = sum(oracle.visible_range(i, W, S)[2] for i in range(S))
    assert tot == sum(min(i + 1, W) for i in range(S))
    assert sum(oracle.visible_range(i, 0, S)[2] for i in range(S)) == S * (S + 1) // 2


def test_cache_slots(oracle):
    assert [oracle.cache_slot(p, 4) for p in range(10)] == [0, 1, 2, 3, 0, 1, 2, 3, 0, 1]
    assert [oracle.cache_slot(p, 0) for p in (0, 5, 262143)] == [0, 5, 262143]


def _small(seed, B=1, S=9, T=None, Hq=4, Hkv=2, D=8):
    T = T or S
    return (rand_bits((B, S, Hq, D), seed), rand_bits((B, T, Hkv, D), seed + 1),
            rand_bits((B, T, Hkv, D), seed + 2))


def test_window_at_least_s_equals_global(oracle):
    q, k, v = _small(3, S=12)
    kw = dict(q_pos0=0, n_keys=12, rot_from=0, rope_frac=1.0, theta=1e4, scale=0.3)
    a, la = oracle.attention(q, k, v, window=0, **kw)
    for W in (12, 16, 4096):
        b, lb = oracle.attention(q, k, v, window=W, **kw)
        np.testing.assert_array_equal(a, b)
        np.testing.assert_array_equal(la, lb)
    c, _ = oracle.attention(q, k, v, window=4, **kw)
    assert not np.allclose(a, c)


# --------------------------------------------------------------------------- library routines
def _sdpa(q, k, v, mask, scale):
    """torch SDPA in fp64 on [B,H,S,D] tensors with an explicit boolean mask."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=torch.from_numpy(mask), scale=scale).numpy()


@pytest.mark.parametrize("window", [0, 5])
def test_nope_matches_sdpa(oracle, window):
    """rope_frac = 0: the oracle equals fp64 SDPA with a causal (windowed) mask
    and the KV heads repeated for GQA."""
    B, S, Hq, Hkv, D = 2, 17, 4, 2, 16
    q, k, v = _small(5, B=B, S=S, Hq=Hq, Hkv=Hkv, D=D)
    out, _ = oracle.attention(q, k, v, q_pos0=0, n_keys=S, rot_from=0, window=window,
                              rope_frac=0.0, theta=1e4, scale=0.25)
    qf = bits_to_f64(q).transpose(0, 2, 1, 3)
    kf = np.repeat(bits_to_f64(k).transpose(0, 2, 1, 3), Hq // Hkv, axis=1)
    vf = np.repeat(bits_to_f64(v).transpose(0, 2, 1, 3), Hq // Hkv, axis=1)
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    mask = (j <= i) & ((j > i - window) if window else True)
    ref = _sdpa(qf, kf, vf, mask, 0.25).reshape(-1, D)  # rows in (b, h, i) order
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_rope_attention_matches_sdpa_on_rotated_inputs(oracle):
    """Full and partial RoPE inside attention, with a chunk offset (queries at
    positions P..P+S-1 against keys 0..P+S-1): equals SDPA on inputs rotated by
    numpy complex multiplication at their own positions."""
    B, S, P, Hq, Hkv, D = 1, 6, 10, 2, 1, 16
    for frac, theta in ((1.0, 1e4), (0.25, 1e6)):
        q = rand_bits((B, S, Hq, D), 21)
        k = rand_bits((B, P + S, Hkv, D), 22)
        v = rand_bits((B, P + S, Hkv, D), 23)
        out, _ = oracle.attention(q, k, v, q_pos0=P, n_keys=P + S, rot_from=0, window=0,
                                  rope_frac=frac, theta=theta, scale=0.5)
        qf = bits_to_f64(q)
        kf = bits_to_f64(k)
        qr = np.stack([complex_rope(qf[0, i], P + i, frac, theta) for i in range(S)])[None]
        kr = np.stack([complex_rope(kf[0, j], j, frac, theta) for j in range(P + S)])[None]
        qt = qr.transpose(0, 2, 1, 3)
        kt = np.repeat(kr.transpose(0, 2, 1, 3), Hq // Hkv, axis=1)
        vt = np.repeat(bits_to_f64(v).transpose(0, 2, 1, 3), Hq // Hkv, axis=1)
        i = np.arange(S)[:, None] + P
        j = np.arange(P + S)[None, :]
        ref = _sdpa(qt, kt, vt, j <= i, 0.5).reshape(-1, D)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)


def test_prerotated_keys_are_used_as_given(oracle):
    """Keys below rot_from arrive rotated (a filled cache): rotating them outside
    and passing rot_from = T equals letting the oracle rotate them."""
    B, S, T, Hq, Hkv, D = 1, 3, 20, 2, 1, 16
    q = rand_bits((B, S, Hq, D), 31)
    k = rand_bits((B, T, Hkv, D), 32)
    v = rand_bits((B, T, Hkv, D), 33)
    kw = dict(q_pos0=T - S, n_keys=T, window=0, rope_frac=0.25, theta=1e6, scale=0.3)
    a, _ = oracle.attention(q, k, v, rot_from=0, **kw)
    kf = bits_to_f64(k)
    krot = np.stack([oracle.rope(kf[0, j, 0], j, 0.25, 1e6) for j in range(T)])
    krot_bits = bf16_bits(krot).reshape(B, T, Hkv, D)
    # bf16 re-rounding of the rotated keys changes the answer slightly
    b, _ = oracle.attention(q, krot_bits, v, rot_from=T, **kw)
    np.testing.assert_allclose(a, b, rtol=0, atol=2e-2)
    c, _ = oracle.attention(q, krot_bits, v, rot_from=0, **kw)
    assert np.abs(a - c).max() > np.abs(a - b).max()


# --------------------------------------------------------------------------- invariants
def test_gqa_equals_mha_with_repeated_kv(oracle):
    B, S, Hq, Hkv, D = 1, 10, 8, 2, 16
    q, k, v = _small(41, B=B, S=S, Hq=Hq, Hkv=Hkv, D=D)
    kw = dict(q_pos0=0, n_keys=S, rot_from=0, window=4, rope_frac=1.0, theta=1e4, scale=0.25)
    a, la = oracle.attention(q, k, v, **kw)
    rep = Hq // Hkv
    k2 = np.repeat(k, rep, axis=2)
    v2 = np.repeat(v, rep, axis=2)
    b, lb = oracle.attention(q, k2, v2, **kw)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)
    # and head h must read KV head h // rep, not h % Hkv
    k3 = np.tile(k, (1, 1, rep, 1))
    v3 = np.tile(v, (1, 1, rep, 1))
    c, _ = oracle.attention(q, k3, v3, **kw)
    assert not np.allclose(a, c)


def test_constant_values_and_zero_query(oracle):
    """Softmax rows sum to 1: constant V returns that constant; Q = 0 gives
    uniform weights, i.e. the mean of the visible V rows and lse = log(count)."""
    B, S, Hq, Hkv, D, W = 1, 12, 2, 1, 8, 5
    q, k, _ = _small(51, B=B, S=S, Hq=Hq, Hkv=Hkv, D=D)
    c = bf16_bits(np.linspace(-2, 2, D))
    v = np.tile(c, (B, S, Hkv, 1))
    out, _ = oracle.attention(q, k, v, q_pos0=0, n_keys=S, rot_from=0, window=W,
                              rope_frac=1.0, theta=1e4, scale=0.7)
    np.testing.assert_allclose(out, np.tile(bits_to_f64(c), (B * S * Hq, 1)), rtol=0, atol=1e-14)
    qz = np.zeros_like(q)
    _, _, vr = _small(52, B=B, S=S, Hq=Hq, Hkv=Hkv, D=D)
    out, lse = oracle.attention(qz, k, vr, q_pos0=0, n_keys=S, rot_from=0, window=W,
                                rope_frac=1.0, theta=1e4, scale=0.7,
                                rows=[[0, 0, i] for i in range(S)])
    vf = bits_to_f64(vr)[0, :, 0]
    for i in range(S):
        lo = max(0, i - W + 1)
        np.testing.assert_allclose(out[i], vf[lo:i + 1].mean(axis=0), rtol=0, atol=1e-14)
        assert abs(lse[i] - math.log(i + 1 - lo)) < 1e-14


def test_brute_force_tiny_against_explicit_sum(oracle):
    """Brute force over S<=4, D=4, every (window, offset): softmax written as
    explicit exponentials over the hand rule's visible set."""
    rng = np.random.default_rng(7)
    for S in range(1, 5):
        for W in (0, 1, 2, 3):
            x = rng.integers(-3, 4, size=(3, S, 4)).astype(np.float64) / 2
            q, k, v = (bf16_bits(x[i]).reshape(1, S, 1, 4) for i in range(3))
            out, lse = oracle.attention(q, k, v, q_pos0=0, n_keys=S, rot_from=0, window=W,
                                        rope_frac=0.0, theta=1e4, scale=1.0)
            for i in range(S):
                vis = [j for j in range(S) if j <= i and (W == 0 or j > i - W)]
                s = np.array([x[0, i] @ x[1, j] for j in vis])
                e = np.exp(s)
                np.testing.assert_allclose(out[i], (e[:, None] * x[2, vis]).sum(0) / e.sum(),
                                           rtol=0, atol=1e-13)
                assert abs(lse[i] - math.log(e.sum())) < 1e-13


# --------------------------------------------------------------------------- schedule / sharing / bytes
def test_interleave_rule_matches_page_figures(oracle):
    figs = json.load(open(GOLDEN))
    assert figs["final_layer_global"]["value"] is True
    for row in figs["layer_counts"]:
        n, r = row["n_layers"], row["local_per_global"]
        sched = oracle.layer_schedule(n, r)
        assert sched[-1], row["model"]
        # r local layers then one global, throughout
        for l in range(n - 1):
            assert sched[l] == ((l + 1) % (r + 1) == 0)
    assert sum(oracle.layer_schedule(35, 4)) == 7
    assert sum(oracle.layer_schedule(42, 5)) == 7
    assert sum(oracle.layer_schedule(60, 5)) == 10
    # 42 layers at 4:1 would end on a local layer: the last one is forced global
    s = oracle.layer_schedule(42, 4)
    assert s[-1] and not ((41 + 1) % 5 == 0) and sum(s) == 9
    # E2B-shaped block: 4 local + global; 31B-shaped: 5 local + global
    assert oracle.layer_schedule(5, 4) == [False] * 4 + [True]
    assert oracle.layer_schedule(6, 5) == [False] * 5 + [True]


def test_share_resolution(oracle):
    """Shared layers read the latest non-shared earlier layer of their type."""
    assert [oracle.share_source(6, 5, 2, l) for l in range(6)] == [0, 1, 2, 3, 3, -1]
    src12 = [oracle.share_source(12, 5, 2, l) for l in range(12)]
    assert src12[:10] == list(range(10)) and src12[10] == 9 and src12[11] == 5
    assert oracle.share_source(8, 0, 3, 7) == 4  # all-global stack


def test_byte_counter_page_figures(oracle):
    figs = json.load(open(GOLDEN))
    ex = figs["k_equals_v_example"]
    one = oracle.layer_cache_bytes(1, 1, ex["tokens"], ex["dims"], elem_bytes=1, k_equals_v=True)
    two = oracle.layer_cache_bytes(1, 1, ex["tokens"], ex["dims"], elem_bytes=1, k_equals_v=False)
    assert one == ex["cached_with_k_eq_v"] and 100 * (two - one) // two == ex["reduction_percent"]
    # 8 global layers, the last 3 sharing: 37.5 % fewer global KV bytes
    kw = dict(local_kv_heads=16, local_head_dim=256, local_capacity=1024, global_kv_heads=4,
              global_head_dim=512, global_capacity=4096, which="global")
    full = oracle.stack_cache_bytes(8, 0, 0, 1, **kw)
    shared = oracle.stack_cache_bytes(8, 0, 3, 1, **kw)
    assert 100.0 * (full - shared) / full == figs["global_kv_reduction_up_to_percent"]["value"]
    # 31B-shaped decode block, 6 layers with the last 2 shared: only layer 4
    # (local, source 3) has a source, so one local cache disappears
    kw["which"] = "all"
    a = oracle.stack_cache_bytes(6, 5, 0, 64, **kw)
    b = oracle.stack_cache_bytes(6, 5, 2, 64, **kw)
    assert a - b == oracle.layer_cache_bytes(64, 16, 1024, 256)


# --------------------------------------------------------------------------- K = V
@pytest.mark.parametrize("frac,theta", [(1.0, 1e4), (0.25, 1e6)])
def test_k_equals_v_matches_sdpa_with_rotated_keys_as_values(oracle, frac, theta):
    """K = V (v = None): the values are the keys as the cache holds them, i.e.
    rotated. Equals fp64 SDPA whose keys and values are both the keys rotated
    by numpy complex multiplication at their own positions (chunk offset P,
    GQA 4:2)."""
    B, S, P, Hq, Hkv, D = 1, 5, 7, 4, 2, 16
    q = rand_bits((B, S, Hq, D), 61)
    k = rand_bits((B, P + S, Hkv, D), 62)
    out, lse = oracle.attention(q, k, None, q_pos0=P, n_keys=P + S, rot_from=0, window=0,
                                rope_frac=frac, theta=theta, scale=0.4)
    qf, kf = bits_to_f64(q), bits_to_f64(k)
    qr = np.stack([complex_rope(qf[0, i], P + i, frac, theta) for i in range(S)])[None]
    kr = np.stack([complex_rope(kf[0, j], j, frac, theta) for j in range(P + S)])[None]
    qt = qr.transpose(0, 2, 1, 3)
    kt = np.repeat(kr.transpose(0, 2, 1, 3), Hq // Hkv, axis=1)
    i = np.arange(S)[:, None] + P
    j = np.arange(P + S)[None, :]
    ref = _sdpa(qt, kt, kt, j <= i, 0.4).reshape(-1, D)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)
    # the values differ from the unrotated keys wherever a pair turns
    plain, _ = oracle.attention(q, k, k, q_pos0=P, n_keys=P + S, rot_from=0, window=0,
                                rope_frac=frac, theta=theta, scale=0.4)
    assert np.abs(out - plain).max() > 1e-3


def test_k_equals_v_worked_example_and_cached_keys(oracle):
    """The page's worked example (4 tokens, 8 dims, values set equal to the
    keys): the output equals the standard computation given V = K explicitly.
    Keys that arrive rotated (a filled cache, rot_from = T) serve as values
    exactly as given."""
    figs = json.load(open(GOLDEN))["k_equals_v_example"]
    T, D = figs["tokens"], figs["dims"]
    q = rand_bits((1, T, 1, D), 71)
    k = rand_bits((1, T, 1, D), 72)
    kw = dict(q_pos0=0, n_keys=T, window=0, theta=1e4, scale=1 / math.sqrt(D))
    a, la = oracle.attention(q, k, None, rot_from=0, rope_frac=0.0, **kw)
    b, lb = oracle.attention(q, k, k, rot_from=0, rope_frac=0.0, **kw)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)
    c, _ = oracle.attention(q, k, None, rot_from=T, rope_frac=1.0, **kw)
    d, _ = oracle.attention(q, k, k, rot_from=T, rope_frac=1.0, **kw)
    np.testing.assert_array_equal(c, d)


@pytest.mark.parametrize("window", [0, 6])
def test_new_token_chunk_equals_one_token_steps(oracle, window):
    """Multi-token decode (the target's pass over a drafter's proposals): T
    new tokens after L - T cached ones, each seeing the cache and the earlier
    new tokens (window-limited on a local layer), give row for row what T
    single-token steps at lengths L - T + 1 .. L give."""
    B, T, L, Hq, Hkv, D = 1, 4, 19, 4, 2, 16
    q = rand_bits((B, T, Hq, D), 71)
    k = rand_bits((B, L, Hkv, D), 72)
    v = rand_bits((B, L, Hkv, D), 73)
    kw = dict(rot_from=L - T, window=window, rope_frac=0.25, theta=1e6, scale=0.3)
    chunk, lse = oracle.attention(q, k, v, q_pos0=L - T, n_keys=L, **kw)
    chunk = chunk.reshape(B, Hq, T, D)
    lse = lse.reshape(B, Hq, T)
    for t in range(T):
        n = L - T + t + 1
        one, lse1 = oracle.attention(np.ascontiguousarray(q[:, t:t + 1]), np.ascontiguousarray(k[:, :n]),
                                     np.ascontiguousarray(v[:, :n]), q_pos0=n - 1, n_keys=n, **kw)
        np.testing.assert_allclose(chunk[:, :, t].reshape(-1, D), one, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, t].reshape(-1), lse1, rtol=0, atol=1e-13)
