"""Pins for the CPU oracle: each oracle function is checked against something
other than itself -- format definitions, a library routine (torch's
float8_e4m3fn cast, torch SDPA in fp64), closed forms, hand-worked cases,
invariants and brute force on tiny inputs.  A plausible mistake anywhere
(a dropped term, a wrong sign or index, a transposed operand) fails one.

CPU only (no gpu marker)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ E4M3
def test_e4m3_decode_matches_torch_float8_e4m3fn_all_codes():
    """Library routine: torch's float8_e4m3fn reinterpretation of all 256 codes."""
    ours = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    nan_o, nan_r = np.isnan(ours), np.isnan(ref)
    assert (nan_o == nan_r).all()
    assert nan_o.sum() == 2  # S.1111.111 only
    np.testing.assert_array_equal(ours[~nan_o], ref[~nan_r])


def test_e4m3_closed_forms():
    c = golden("constants.json")
    t = oracle.e4m3_table()
    assert t[0x7E] == c["e4m3_max"]["value"] == 448.0
    assert np.nanmax(np.abs(t)) == 448.0
    assert t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    assert len(set(t[~np.isnan(t)].tolist())) == 253  # 254 finite codes, +0 == -0


def test_e4m3_encode_matches_torch_cast_dense_and_midpoints():
    """Dense sample + every midpoint between representable values (+/- 1 ulp):
    our RNE encoder agrees with torch's .to(float8_e4m3fn) within [-448, 448]."""
    t = oracle.e4m3_table()
    pos = np.unique(t[(~np.isnan(t)) & (t >= 0)])
    mids = (pos[:-1] + pos[1:]) / 2
    mids = mids.astype(np.float32)
    probes = np.concatenate([
        mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
        pos.astype(np.float32),
        np.random.default_rng(0).uniform(-448, 448, 20000).astype(np.float32),
        (np.random.default_rng(1).standard_normal(20000) * 0.01).astype(np.float32),
    ])
    probes = np.concatenate([probes, -probes])
    probes = probes[np.abs(probes) <= 448]
    ours = oracle.e4m3_encode(probes)
    ref = torch.from_numpy(probes).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # -0.0 vs +0.0 both decode to zero; compare decoded values, then codes of non-zeros
    np.testing.assert_array_equal(t[ours], t[ref])


def test_e4m3_encode_brute_force_nearest_ties_to_even():
    t = oracle.e4m3_table()
    fin = ~np.isnan(t)
    vals = t[fin]
    codes = np.arange(256)[fin]
    rng = np.random.default_rng(2)
    xs = np.concatenate([rng.uniform(-450, 450, 3000), rng.standard_normal(3000) * 1e-2]).astype(np.float32)
    enc = oracle.e4m3_encode(xs)
    for x, c in zip(xs, enc):
        if abs(x) >= 448:
            assert t[c] == math.copysign(448.0, x)
            continue
        err = np.abs(vals.astype(np.float64) - float(x))
        best = err.min()
        assert abs(t[c] - float(x)) == best
        ties = codes[err == best]
        if len(set(vals[err == best].tolist())) > 1:  # a true tie between two values
            assert (c & 1) == 0 or t[c] == 0.0


def test_e4m3_saturates():
    enc = oracle.e4m3_encode(np.array([448.0, 460.0, 1e6, np.inf, -1e6], np.float32))
    assert list(oracle.e4m3_table()[enc]) == [448.0, 448.0, 448.0, 448.0, -448.0]


# ------------------------------------------------------------------ E2M1
def test_e2m1_decode_grid_and_15_distinct_values():
    c = golden("constants.json")
    t = oracle.e2m1_table()
    assert sorted(set(np.abs(t).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert len(set(t.tolist())) == c["fp4_distinct_values"]["value"] == 15
    assert t.max() == c["e2m1_max"]["value"] == 6.0


@pytest.mark.parametrize("x,expect", [
    (0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),
    (0.26, 0.5), (2.6, 3.0), (7.0, 6.0), (100.0, 6.0), (-0.75, -1.0), (-5.0, -4.0), (5.01, 6.0),
])
def test_e2m1_encode_hand_cases(x, expect):
    """Ties go to the even mantissa: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4."""
    assert oracle.e2m1_table()[oracle.e2m1_encode(np.array([x], np.float32))[0]] == expect


def test_e2m1_brute_force_nearest():
    t = oracle.e2m1_table()
    xs = np.random.default_rng(3).uniform(-7, 7, 5000).astype(np.float32)
    enc = oracle.e2m1_encode(xs)
    for x, c in zip(xs, enc):
        target = min(max(float(x), -6.0), 6.0)
        assert abs(t[c] - target) == np.abs(t.astype(np.float64) - target).min()


# ------------------------------------------------------------------ means / smoothing
def test_mean_exact_closed_form():
    X = np.array([[1, 3], [3, 5], [2, 7]], np.float32)
    np.testing.assert_array_equal(oracle.mean_rows(X), np.array([2, 5], np.float32))
    # a value whose fp32 mean needs one rounding of an exact fp64 sum
    X = np.array([[1.0], [2.0], [2.0]], np.float32)
    assert oracle.mean_rows(X)[0] == np.float32(5.0 / 3.0)


def test_block_means_ragged_tail_uses_valid_rows_only():
    X = np.arange(10, dtype=np.float32).reshape(5, 2)  # rows (0,1),(2,3),(4,5),(6,7),(8,9)
    m = oracle.block_means(X, 2)
    np.testing.assert_array_equal(m, np.array([[1, 2], [5, 6], [8, 9]], np.float32))


# ------------------------------------------------------------------ INT8
def test_int8_hand_worked_smooth_k():
    """K rows (1,3),(3,5): km = (2,4), gamma = (-1,-1),(1,1), s = 1/127, K^ = -+127."""
    K = np.array([[1, 3], [3, 5]], np.float32)
    km = oracle.mean_rows(K)
    np.testing.assert_array_equal(km, [2, 4])
    k8, s = oracle.quant_int8(K, 64, km)
    assert s[0] == np.float32(1.0) / np.float32(127.0)
    np.testing.assert_array_equal(k8, [[-127, -127], [127, 127]])


def test_int8_properties_random_blocks():
    rng = np.random.default_rng(4)
    X = (rng.standard_normal((300, 64)) * 3).astype(np.float32)
    q8, s = oracle.quant_int8(X, 64)
    assert len(s) == 5
    for i in range(5):
        blk = X[i * 64:(i + 1) * 64]
        codes = q8[i * 64:(i + 1) * 64].astype(np.int32)
        amax = np.abs(blk).max()
        assert np.abs(codes).max() == 127
        # the amax element maps to +-127
        r, c = np.unravel_index(np.abs(blk).argmax(), blk.shape)
        assert abs(codes[r, c]) == 127
        # reconstruction error within half a step (plus fp32 slop)
        err = np.abs(blk - codes * np.float64(s[i]))
        assert err.max() <= 0.5 * s[i] * (1 + 1e-5)
        assert abs(float(s[i]) * 127 - amax) <= 1e-6 * amax


def test_int8_zero_block_and_round_half_even():
    X = np.zeros((64, 4), np.float32)
    q8, s = oracle.quant_int8(X, 64)
    assert s[0] == 0 and (q8 == 0).all()
    # amax = 127 -> scale 1.0 exactly; 2.5 -> 2, 3.5 -> 4, -2.5 -> -2 (half to even)
    X = np.zeros((64, 4), np.float32)
    X[0, :] = [127.0, 2.5, 3.5, -2.5]
    q8, s = oracle.quant_int8(X, 64)
    assert s[0] == 1.0
    assert list(q8[0]) == [127, 2, 4, -2]


def test_int8_per_block_mean_subtraction_index():
    """Block i subtracts mean row i (a wrong block index would leave a bias)."""
    X = np.concatenate([np.full((4, 2), 10, np.float32), np.full((4, 2), -10, np.float32)])
    X[0, 0] += 1
    X[4, 1] -= 1
    means = oracle.block_means(X, 4)
    q8, s = oracle.quant_int8(X, 4, means, True)
    assert q8[0, 0] == 127 and q8[4, 1] == -127


# ------------------------------------------------------------------ FP8 V
def test_fp8_per_channel_v():
    V = np.array([[1.0, -2.0], [0.5, 4.0], [-3.0, 1.0]], np.float32)
    v8, sv = oracle.quant_fp8_per_channel(V)
    np.testing.assert_array_equal(sv, np.array([3.0, 4.0], np.float32) / np.float32(448))
    t = oracle.e4m3_table()
    # the per-channel amax element lands exactly on 448
    assert t[v8[2, 0]] == -448.0 and t[v8[1, 1]] == 448.0
    # decode * scale reproduces V within E4M3's half step (relative 2^-4)
    rec = t[v8] * sv
    assert np.all(np.abs(rec - V) <= np.abs(V) * 2.0 ** -4 + 1e-12)


# ------------------------------------------------------------------ delta_S
def test_delta_s_hand_and_zero_sum_invariant():
    K = np.array([[1, 3], [3, 5]], np.float32)       # gamma(K) = (-1,-1), (1,1)
    qbar = np.array([[2, 1], [0.5, -4]], np.float32)
    dS = oracle.delta_s(qbar, K, oracle.mean_rows(K))
    np.testing.assert_array_equal(dS, np.array([[-3, 3], [3.5, -3.5]], np.float32))
    # sum over all tokens of gamma(K) is zero, so every delta_S row sums to ~0
    rng = np.random.default_rng(5)
    K = (rng.standard_normal((257, 16)) + 5).astype(np.float32)
    qbar = rng.standard_normal((3, 16)).astype(np.float32)
    dS = oracle.delta_s(qbar, K, oracle.mean_rows(K))
    assert np.abs(dS.astype(np.float64).sum(axis=1)).max() < 1e-3


# ------------------------------------------------------------------ attention
def _rand_qkv(B, Hq, Hkv, N, d, seed, kbias=0.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, N, d, generator=g)
    k = torch.randn(B, Hkv, N, d, generator=g) + torch.randn(1, Hkv, 1, d, generator=g) * kbias
    v = torch.randn(B, Hkv, N, d, generator=g)
    return q, k, v


@pytest.mark.parametrize("causal", [False, True])
def test_naive_f64_matches_torch_sdpa_f64(causal):
    """Library routine: torch's scaled_dot_product_attention in float64."""
    q, k, v = _rand_qkv(1, 1, 1, 37, 16, 6)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), is_causal=causal, scale=0.3)[0, 0].numpy()
    out = oracle.attention_exact_head(q, k, v, 0, 0, 0, 37, causal=causal, sm_scale=0.3)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_naive_closed_forms():
    N, d = 9, 4
    rng = np.random.default_rng(7)
    v = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    q = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    k = np.zeros((1, 1, N, d), np.float32)
    # K = 0 -> uniform weights -> mean of V (causal: mean of V[0..r])
    out = oracle.attention_exact_head(q, k, v, 0, 0, 0, N, causal=False, sm_scale=1.0)
    np.testing.assert_allclose(out, np.tile(v[0, 0].astype(np.float64).mean(0), (N, 1)), atol=1e-12)
    out = oracle.attention_exact_head(q, k, v, 0, 0, 0, N, causal=True, sm_scale=1.0)
    for r in range(N):
        np.testing.assert_allclose(out[r], v[0, 0, :r + 1].astype(np.float64).mean(0), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tile", [16, 32, 128])
def test_blocked_online_softmax_equals_naive_in_f64(causal, tile):
    """Special case: identity codecs, fp64 -> the blocked two-level online softmax
    must equal textbook softmax(QK^T s)V (pins m/l/alpha updates, the fresh
    per-tile O_t, the rescale of O and the final normalisation)."""
    q, k, v = _rand_qkv(1, 1, 1, 203, 32, 8, kbias=2.0)
    ref = oracle.attention_exact_head(q, k, v, 0, 0, 0, 203, causal=causal, sm_scale=0.4)
    out = oracle.attention_blocked_f64_head(q, k, v, 0, 0, 0, 203, causal=causal, sm_scale=0.4, tile=tile)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def _naive_f64(Q, K, V, causal, sm):
    Q, K, V = (np.ascontiguousarray(x, np.float64) for x in (Q, K, V))
    N, d = Q.shape
    out = np.empty((N, d), np.float64)
    rc = oracle.lib().or_attn_naive_f64(Q.ctypes.data, K.ctypes.data, V.ctypes.data, N, d, int(causal),
                                        float(sm), 0, N, out.ctypes.data)
    assert rc == 0
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_smooth_k_shift_invariance_exact(causal):
    """Smooth K is exact: attention on K and on K - mean(K) agree in fp64."""
    q, k, v = _rand_qkv(1, 1, 1, 150, 32, 9, kbias=3.0)
    Q, K, V = (x[0, 0].double().numpy() for x in (q, k, v))
    km = oracle.mean_rows(k[0, 0]).astype(np.float64)
    a = _naive_f64(Q, K, V, causal, 0.2)
    b = _naive_f64(Q, K - km, V, causal, 0.2)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_smooth_q_delta_s_compensation_exact_in_f64(causal):
    """Smooth Q + delta_S: with (Q - q_i) and gamma(K), adding delta_S = q_i . gamma(K)^T
    and dropping the row-constant term reproduces exact attention (fp64, identity
    codecs).  A wrong sign or block index of delta_S fails this."""
    N, d, bq = 200, 32, 64
    q, k, v = _rand_qkv(1, 1, 1, N, d, 10, kbias=2.0)
    q = q + torch.randn(1, 1, 1, d, generator=torch.Generator().manual_seed(11)) * 2
    ref = oracle.attention_exact_head(q, k, v, 0, 0, 0, N, causal=causal, sm_scale=0.3)
    Q = q[0, 0].numpy().astype(np.float32)
    K = k[0, 0].numpy().astype(np.float32)
    V = v[0, 0].numpy().astype(np.float64)
    km = oracle.mean_rows(K)
    qbar = oracle.block_means(Q, bq)
    dS = oracle.delta_s(qbar, K, km)
    Qs = (Q - np.repeat(qbar, bq, axis=0)[:N]).astype(np.float64)
    Ks = (K - km).astype(np.float64)
    out = oracle._attn_core(np.ascontiguousarray(Qs), np.ascontiguousarray(Ks), np.ascontiguousarray(V),
                            None, None, dS, bq, None, N, d, causal, 0.3, 0, 0, 0, N, tile=64)
    # delta_S itself is rounded to fp32, hence 1e-6 rather than 1e-12
    np.testing.assert_allclose(out, ref, atol=2e-6)


def test_e4m3_p_path_hand_worked_2x2():
    """Hand-worked: S row = [1, 0] -> P~ = [1, e^-1]; x448 -> [448, 164.8];
    E4M3 -> [448, 160]; l = 1 + e^-1; V^ = [1, 2] (codes 0x38, 0x40), s_v = 0.5:
    out = (448*1 + 160*2) / l / 448 * 0.5."""
    Qv = np.array([[127.0], [127.0]])
    Kv = np.array([[127.0], [0.0]])
    Vv = np.array([[1.0], [2.0]])
    s = 1.0 / 127.0
    out = oracle._attn_core(Qv, Kv, Vv, np.array([s, s]), np.array([s, s]), None, 64,
                            np.array([0.5]), 2, 1, False, 1.0, 1, 1, 0, 1)
    l = 1.0 + math.exp(-1.0)
    expect = (448.0 * 1 + 160.0 * 2) / l / 448.0 * 0.5
    assert abs(out[0, 0] - expect) < 1e-6


def test_nvfp4_two_level_p_hand_worked():
    """SA3 two-level P: P~ = [1, e^-1] -> s_P1 = 1/2688; P2 = [2688, 988.9];
    s_P2 = E4M3(2688/6 = 448) = 448; P2/448 = [6, 2.207] -> E2M1 [6, 2];
    P^ s_P2 s_P1 = [1, 1/3]; V = [1, 2]: out = (1*1 + 2/3) / (1 + e^-1)."""
    Qv = np.array([[1.0], [1.0]])
    Kv = np.array([[1.0], [0.0]])
    Vv = np.array([[1.0], [2.0]])
    out = oracle._attn_core(Qv, Kv, Vv, None, None, None, 64, None, 2, 1, False, 1.0, 2, 1, 0, 1, tile=16)
    expect = (1.0 + 2.0 / 3.0) / (1.0 + math.exp(-1.0))
    assert abs(out[0, 0] - expect) < 1e-6


def test_e4m3_p_path_hand_worked_4x4_causal_growing_max():
    """Hand-worked 4x4 causal case, K tile = 2 keys, so the online softmax of rows
    2 and 3 spans two tiles and their max grows in the second one.
    d = 1; s_q = s_k = 1, sm_scale = 1, so S[r, c] = Q^[r] K^[c].
    Q^ = [1, 1, 1, 2], K^ = [-1, -2, 0, -3], V = [1, 2, 0.5, 4], s_v = 0.25.
      row 0: key 0: S = [-1]; P~ = [1]; l = 1; P^ = [448]; O = 448
             out = 448 / 1 / 448 * 0.25 = 0.25
      row 1: keys 0, 1: S = [-1, -2], m = -1; P~ = [1, e^-1], l = 1 + e^-1;
             448 e^-1 = 164.8 -> E4M3 160 (grid step 16 in [128, 256));
             O = 448 * 1 + 160 * 2 = 768
      row 2: tile 0 as row 1 (m = -1, l0 = 1 + e^-1, O0 = 768); tile 1 holds
             key 2 only (key 3 is causally masked): S = [0], m grows -1 -> 0,
             alpha = e^-1; P~ = [1] -> 448; O_t = 448 * 0.5 = 224
             l = e^-1 l0 + 1, O = e^-1 * 768 + 224
      row 3: tile 0: S = [-2, -4], m = -2; P~ = [1, e^-2]; 448 e^-2 = 60.63 ->
             E4M3 60 (step 4 in [32, 64)); O0 = 448 + 60 * 2 = 568, l0 = 1 + e^-2
             tile 1: S = [0, -6], m grows -2 -> 0, alpha = e^-2;
             P~ = [1, e^-6]; 448 e^-6 = 1.1105 -> E4M3 1.125 (step 1/8 in
             [1, 2)); O_t = 448 * 0.5 + 1.125 * 4 = 228.5
             l = e^-2 l0 + 1 + e^-6, O = e^-2 * 568 + 228.5
    out = O / l / 448 * 0.25 in every row."""
    Qv = np.array([[1.0], [1.0], [1.0], [2.0]])
    Kv = np.array([[-1.0], [-2.0], [0.0], [-3.0]])
    Vv = np.array([[1.0], [2.0], [0.5], [4.0]])
    one = np.ones(4)
    out = oracle._attn_core(Qv, Kv, Vv, one, one, None, 64, np.array([0.25]), 4, 1, True, 1.0, 1, 1, 0, 4,
                            tile=2)
    e = math.exp
    l2 = e(-1) * (1 + e(-1)) + 1
    l3 = e(-2) * (1 + e(-2)) + 1 + e(-6)
    expect = np.array([
        448.0 / 1.0,
        768.0 / (1 + e(-1)),
        (e(-1) * 768.0 + 224.0) / l2,
        (e(-2) * 568.0 + 228.5) / l3,
    ]) / 448.0 * 0.25
    np.testing.assert_allclose(out[:, 0], expect, rtol=2e-6)


def test_nvfp4_two_level_p_per_16_groups_hand_worked():
    """SA3 two-level P quantisation of one 64-key tile whose four 16-key groups
    have different maxima, so one s_P2 per 16 keys, per 32 or per tile give
    different outputs.  d = 1, Q = 1, sm_scale = 1, so S = K; the row max is key 0
    (S = 0), hence P~ = e^S and s_P1 = 1 / 2688, P2 = 2688 P~.
      group 0: P~ = [1, 15 x e^-30]: amax 2688 -> s_P2 = E4M3(448) = 448;
               P2 / s_P2 = [6, ~0] -> E2M1 [6, 0]: P^ s_P2 s_P1 = [1, 0...]
      group 1: 16 x P~ = 0.1: P2 = 268.8, s_P2 = E4M3(44.8) = 44 (step 4 in
               [32, 64)); 268.8 / 44 = 6.11 -> 6: each 6 * 44 / 2688 = 264 / 2688
      group 2: P~ = [0.25, 15 x 0.05]: P2 = [672, 134.4], s_P2 = E4M3(112) = 112;
               [6, 1.2] -> E2M1 [6, 1]: [0.25, 15 x 112 / 2688]
      group 3: 16 x P~ = 0.02: P2 = 53.76, s_P2 = E4M3(8.96) = 9;
               5.97 -> E2M1 6: each 54 / 2688
    V = 1, 2, 4, 8 on groups 0..3; l = 1 + 1.6 + 1 + 0.32 = 3.92 (fp32 P~, before
    quantisation).  One s_P2 per 32 keys gives 0.9035 (V = 1) instead of
    0.9612; one per tile gives 0.9779."""
    K = np.concatenate([[0.0], np.full(15, -30.0), np.full(16, math.log(0.1)), [math.log(0.25)],
                        np.full(15, math.log(0.05)), np.full(16, math.log(0.02))])[:, None]
    Q = np.ones((64, 1))
    V = np.repeat([1.0, 2.0, 4.0, 8.0], 16)[:, None]
    g = np.array([1.0,
                  16 * 264 / 2688,
                  0.25 + 15 * 112 / 2688,
                  16 * 54 / 2688])
    l = 1 + 16 * 0.1 + 0.25 + 15 * 0.05 + 16 * 0.02
    out = oracle._attn_core(Q, K, V, None, None, None, 64, None, 64, 1, False, 1.0, 2, 1, 0, 1, tile=64)
    assert abs(out[0, 0] - (g @ np.array([1.0, 2.0, 4.0, 8.0])) / l) < 2e-6 * out[0, 0]
    ones = np.ones((64, 1))
    out1 = oracle._attn_core(Q, K, ones, None, None, None, 64, None, 64, 1, False, 1.0, 2, 1, 0, 1, tile=64)
    assert abs(out1[0, 0] - g.sum() / l) < 2e-6


def test_oracle_int8_fp8_cosine_vs_exact_small_workloads():
    """Whole oracle vs fp64 exact: cosine >= 0.998 on each INT8/FP8 recipe at a
    size of a few tiles with a ragged tail (full-size versions run on the GPU machine)."""
    from quantized_attention_block_b200 import workloads as W
    for name in ("tiny", "prefill", "video", "gqa"):
        w = W.get(name)
        ws = W.small_variant(w, N=333 if name != "tiny" else w.N)
        q, k, v = W.make_qkv(ws)
        quant = oracle.quantize_sage(q, k, v, bq=ws.bq, bk=ws.bk, smooth_k=ws.smooth_k, smooth_q=ws.smooth_q)
        outs, refs = [], []
        for h in range(ws.Hq):
            outs.append(oracle.attention_sage_head(quant, 0, h, 0, ws.N, bq=ws.bq, bk=ws.bk,
                                                   causal=ws.causal, sm_scale=ws.sm_scale))
            refs.append(oracle.attention_exact_head(q, k, v, 0, h, 0, ws.N, causal=ws.causal,
                                                    sm_scale=ws.sm_scale))
        m = oracle.metrics(np.stack(refs), np.stack(outs))
        assert m["cos"] >= 0.998, (name, m)


def test_oracle_nvfp4_cosine_vs_exact_small():
    from quantized_attention_block_b200 import workloads as W
    ws = W.small_variant(W.get("nvfp4"), N=300)
    q, k, v = W.make_qkv(ws)
    quant = oracle.quantize_nvfp4(q, k, v, bq=ws.bq)
    outs, refs = [], []
    for h in range(ws.Hq):
        outs.append(oracle.attention_nvfp4_head(quant, 0, h, 0, ws.N, bq=ws.bq, causal=False,
                                                sm_scale=ws.sm_scale))
        refs.append(oracle.attention_exact_head(q, k, v, 0, h, 0, ws.N, causal=False, sm_scale=ws.sm_scale))
    m = oracle.metrics(np.stack(refs), np.stack(outs))
    assert m["cos"] >= 0.99, m


def test_nvfp4_quant_properties():
    rng = np.random.default_rng(12)
    X = (rng.standard_normal((5, 32)) * 2).astype(np.float32)
    codes, sf = oracle.quant_nvfp4_rows(X, 128)
    t4, t8 = oracle.e2m1_table(), oracle.e4m3_table()
    for r in range(5):
        for g in range(2):
            blk = X[r, g * 16:(g + 1) * 16]
            s = t8[sf[r, g]]
            # scale is E4M3 of amax/6 (within E4M3's relative half step)
            assert abs(s - np.abs(blk).max() / 6) <= np.abs(blk).max() / 6 * 2.0 ** -4
            rec = t4[codes[r, g * 16:(g + 1) * 16]] * s
            # each element within half an E2M1 step of its (saturated) value
            x = np.clip(blk / s, -6, 6)
            assert np.all(np.abs(rec / s - x) <= np.maximum(0.25, np.abs(x) * 0.25) + 1e-6)
    V = (rng.standard_normal((37, 16))).astype(np.float32)
    codes, sf = oracle.quant_nvfp4_cols(V)
    assert sf.shape == (3, 16)
    # groups run along tokens: group 2 covers rows 32..36 only
    assert t8[sf[2, 0]] == t8[oracle.e4m3_encode(np.array([np.abs(V[32:, 0]).max() / 6], np.float32))[0]]


# ---------------------------------------------------------------- log-sum-exp
def _lse_textbook(Q, K, sm_scale, causal):
    """fp64 log-sum-exp of each row of sm_scale Q K^T (causal: keys <= row), via
    scipy's logsumexp -- an independent routine."""
    from scipy.special import logsumexp
    S = (Q.astype(np.float64) @ K.astype(np.float64).T) * sm_scale
    if causal:
        S = np.where(np.tril(np.ones_like(S, dtype=bool)), S, -np.inf)
    return logsumexp(S, axis=1)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tile", [16, 32, 128])
def test_oracle_lse_identity_codecs_equals_logsumexp(causal, tile):
    """The blocked online softmax's m + ln l (identity codecs, fp64) is the
    row log-sum-exp: pins the running-max / running-sum bookkeeping."""
    g = torch.Generator().manual_seed(11)
    N, d = 77, 64
    q = torch.randn(1, 1, N, d, generator=g) * 2
    k = torch.randn(1, 1, N, d, generator=g) * 2
    v = torch.randn(1, 1, N, d, generator=g)
    _, lse = oracle.attention_blocked_f64_head(q, k, v, 0, 0, 0, N, causal=causal, sm_scale=0.125,
                                               tile=tile, with_lse=True)
    ref = _lse_textbook(q[0, 0].numpy(), k[0, 0].numpy(), 0.125, causal)
    np.testing.assert_allclose(lse, ref, rtol=1e-12, atol=1e-12)


def test_oracle_lse_zero_keys_is_log_of_visible_keys():
    N, d = 40, 64
    q = torch.randn(1, 1, N, d, generator=torch.Generator().manual_seed(3))
    k = torch.zeros(1, 1, N, d)
    v = torch.ones(1, 1, N, d)
    for causal in (False, True):
        _, lse = oracle.attention_blocked_f64_head(q, k, v, 0, 0, 0, N, causal=causal, sm_scale=0.3,
                                                   tile=16, with_lse=True)
        visible = np.arange(1, N + 1) if causal else np.full(N, N)
        np.testing.assert_allclose(lse, np.log(visible), rtol=0, atol=1e-13)


def test_oracle_lse_smooth_k_shift_identity():
    """Shifting every key by a constant vector km shifts row i's scores by
    sm_scale (Q_i . km): lse(K + km) = lse(K) + sm_scale Q km.  Inputs are small
    dyadic values so that K + km is exact in fp32."""
    g = torch.Generator().manual_seed(5)
    N, d = 50, 64
    q = torch.randint(-16, 17, (1, 1, N, d), generator=g).float() / 8
    k = torch.randint(-16, 17, (1, 1, N, d), generator=g).float() / 8
    km = torch.randint(-8, 9, (d,), generator=g).float() / 4
    v = torch.randn(1, 1, N, d, generator=g)
    sm = 0.125
    _, lse_k = oracle.attention_blocked_f64_head(q, k, v, 0, 0, 0, N, causal=True, sm_scale=sm, with_lse=True)
    _, lse_shift = oracle.attention_blocked_f64_head(q, k + km, v, 0, 0, 0, N, causal=True, sm_scale=sm,
                                                     with_lse=True)
    corr = sm * (q[0, 0].double().numpy() @ km.double().numpy())
    np.testing.assert_allclose(lse_shift, lse_k + corr, rtol=1e-12, atol=1e-10)


def test_oracle_sage_lse_with_correction_tracks_exact():
    """The quantised pipeline's log-sum-exp (smoothed K) plus the smooth-K
    correction lands on the exact fp64 log-sum-exp of the original scores; a
    dropped or sign-flipped correction would be off by |sm_scale Q km|, which
    the K bias of the prefill recipe makes several units large."""
    from quantized_attention_block_b200 import workloads as W
    ws = W.small_variant(W.get("prefill"), N=200, B=1, Hq=1, Hkv=1)
    q, k, v = W.make_qkv(ws)
    quant = oracle.quantize_sage(q, k, v, bq=ws.bq, bk=ws.bk, smooth_k=True, smooth_q=False)
    _, lse = oracle.attention_sage_head(quant, 0, 0, 0, ws.N, bq=ws.bq, bk=ws.bk, causal=ws.causal,
                                        sm_scale=ws.sm_scale, with_lse=True)
    corr = oracle.lse_smooth_k_correction(q, quant, 0, 0, 0, ws.N, sm_scale=ws.sm_scale)
    ref = _lse_textbook(q[0, 0].float().numpy(), k[0, 0].float().numpy(), ws.sm_scale, ws.causal)
    err_with = np.abs(lse + corr - ref).max()      # the INT8 score quantisation error (K outliers)
    err_without = np.abs(lse - ref).max()
    err_flipped = np.abs(lse - corr - ref).max()
    assert np.abs(corr).max() > 1.0  # the correction matters on this recipe
    assert err_with < 0.5 and err_with < 0.05 * err_without and err_with < 0.05 * err_flipped
