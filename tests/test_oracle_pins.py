"""Pins for the CPU oracle, each against something other than the oracle itself:
hand-derived values, closed forms, exact rational arithmetic, invariants of the
method, and library routines for the special cases that reduce to them.

Sources: "Bitnet.cpp: Efficient Edge Inference for Ternary LLMs" reading notes
(section 1.1 ternary weights; section 2.3 I2_S, int8 activations, 2.0 bpw;
section 4.1 lossless conditions), FairyFuse article ("ternary quantisation
scheme": the +-0.5 alpha thresholds; "fused kernel design": add/subtract only),
and the bitnet.cpp CPU tutorial section 1.2 (multiplication degenerates to
addition or subtraction).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from ternary_weight_bit_bitlinear_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_round(fr: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 of a non-negative rational."""
    if fr == 0:
        return np.float32(0.0)
    E = fr.numerator.bit_length() - fr.denominator.bit_length()
    while Fraction(2) ** E > fr:
        E -= 1
    while Fraction(2) ** (E + 1) <= fr:
        E += 1
    ulp = max(E - 23, -149)
    scaled = fr / Fraction(2) ** ulp
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return np.float32(n * 2.0 ** ulp)


def exact_mean_abs(w) -> Fraction:
    w = np.asarray(w, dtype=np.float32).ravel()
    return sum((Fraction(abs(float(v))) for v in w), Fraction(0)) / w.size


def rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- alpha

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_alpha_is_correctly_rounded_mean(seed):
    r = rng(seed)
    w = (r.standard_normal(3000) * 0.02).astype(np.float32)
    assert oracle.absmean(w) == f32_round(exact_mean_abs(w))


def test_alpha_wide_dynamic_range_and_subnormals():
    r = rng(7)
    mant = r.uniform(1, 2, 2000)
    expo = r.integers(-149, 100, 2000)
    w = (mant * np.exp2(expo.astype(np.float64))).astype(np.float32)
    w[::3] *= -1
    w[:20] = np.float32(1e-45) * np.arange(1, 21, dtype=np.float32)   # subnormals
    assert oracle.absmean(w) == f32_round(exact_mean_abs(w))
    sub = (np.arange(1, 50, dtype=np.float32) * np.float32(1.4e-45))
    assert oracle.absmean(sub) == f32_round(exact_mean_abs(sub))


def test_alpha_closed_forms():
    # W = +-c  =>  alpha = c exactly
    for c in [0.02, 1.0, 3.0e-30, 7.5e20]:
        w = np.full(1000, c, dtype=np.float32)
        w[::2] *= -1
        assert oracle.absmean(w) == np.float32(c)
    # integer-valued: mean of 1..n is (n+1)/2
    w = np.arange(1, 102, dtype=np.float32)
    assert oracle.absmean(w) == np.float32(51.0)
    # all zero => alpha = 0 and every code is 0
    z = np.zeros((4, 32), dtype=np.float32)
    assert oracle.absmean(z) == 0.0
    assert not oracle.ternarize(z, 0.0).any()


def test_alpha_order_independent():
    r = rng(3)
    w = (r.standard_normal(5000) * 0.02).astype(np.float32)
    a = oracle.absmean(w)
    for s in range(3):
        assert oracle.absmean(rng(100 + s).permutation(w)) == a


def test_alpha_rejects_non_finite():
    w = np.ones(64, dtype=np.float32)
    w[5] = np.inf
    with pytest.raises(ValueError):
        oracle.absmean(w)
    w[5] = np.nan
    with pytest.raises(ValueError):
        oracle.absmean(w)


def test_bins_match_exact_sum():
    r = rng(11)
    w = (r.standard_normal(777) * 3).astype(np.float32)
    bins, st = oracle.abs_bins(w)
    assert st == 0
    total = sum(Fraction(int(b)) * Fraction(2) ** (e - 150) for e, b in enumerate(bins))
    assert total == sum(Fraction(abs(float(v))) for v in w)


# ----------------------------------------------------------------------------- ternarise

def test_codes_are_ternary_and_gaussian_zero_fraction():
    w = inputs.latent_weights(512, 1024, seed=5).numpy()
    a = oracle.absmean(w)
    c = oracle.ternarize(w, a)
    assert set(np.unique(c).tolist()) <= {-1, 0, 1}
    # For W ~ N(0, s^2), alpha = s*sqrt(2/pi); code 0 iff |w| <= alpha/2:
    # P = 2*Phi(sqrt(2/pi)/2) - 1 = erf(sqrt(2/pi)/2/sqrt(2)).
    p0 = math.erf(math.sqrt(2 / math.pi) / 2 / math.sqrt(2))
    assert abs(p0 - 0.3101) < 1e-3
    assert abs((c == 0).mean() - p0) < 0.01


def test_ternarize_matches_threshold_rule_away_from_ties():
    r = rng(4)
    w = (r.standard_normal(20000) * 0.02).astype(np.float32)
    a = oracle.absmean(w)
    c = oracle.ternarize(w, a)
    ratio = w / a                                       # IEEE fp32 division
    away = np.abs(ratio) != np.float32(0.5)
    thr = np.where(w.astype(np.float64) > 0.5 * float(a), 1,
                   np.where(w.astype(np.float64) < -0.5 * float(a), -1, 0))
    assert np.array_equal(c[away], thr[away])


def test_ternarize_exact_ties_round_to_even():
    a = np.float32(0.25)
    w = np.array([0.125, -0.125, 0.375, -0.375, 0.0, 0.5, -7.0, 0.12499999],
                 dtype=np.float32)
    # w/a = 0.5 -> 0 ; -0.5 -> 0 ; 1.5 -> 2 -> clamp 1 ; -1.5 -> -1 ; 0 ; 2 -> 1 ; -28 -> -1
    assert oracle.ternarize(w, a).tolist() == [0, 0, 1, -1, 0, 1, -1, 0]


def test_ternarize_sign_and_power_of_two_invariance():
    w = inputs.latent_weights(64, 256, seed=9).numpy()
    a = oracle.absmean(w)
    c = oracle.ternarize(w, a)
    assert np.array_equal(oracle.ternarize(-w, oracle.absmean(-w)), -c)
    for j in (-3, 5):
        w2 = (w * np.float32(2.0 ** j)).astype(np.float32)
        a2 = oracle.absmean(w2)
        assert a2 == np.float32(a * np.float32(2.0 ** j))
        assert np.array_equal(oracle.ternarize(w2, a2), c)


# ----------------------------------------------------------------------------- pack

def test_pack_layout_hand_derived_words():
    zero = np.zeros((1, 16), dtype=np.int8)
    assert oracle.pack(zero)[0, 0] == 0x55555555           # every field = code 0+1 = 01
    cases = {(1, +1): 0x55555655,    # k=1 -> bit 8, field 10
             (4, +1): 0x55555559,    # k=4 -> bit 2
             (15, +1): 0x95555555,   # k=15 -> bit 30
             (5, -1): 0x55555155,    # k=5 -> bit 10, field 00
             (0, -1): 0x55555554}    # k=0 -> bit 0
    for (k, v), word in cases.items():
        c = zero.copy()
        c[0, k] = v
        assert oracle.pack(c)[0, 0] == word, (k, v)
    # second word of a row holds k = 16..31
    c = np.zeros((2, 32), dtype=np.int8)
    c[1, 16] = 1
    p = oracle.pack(c)
    assert p.shape == (2, 4) and p[1, 1] == 0x55555556 and p[1, 0] == 0x55555555
    assert (p[:, 2:] == 0x55555555).all()    # row padded to 16 bytes with code 0


def test_pack_roundtrip_size_and_byte_lanes():
    r = rng(12)
    M, K = 24, 128
    c = r.integers(-1, 2, size=(M, K)).astype(np.int8)
    p = oracle.pack(c)
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    assert p.nbytes * 8 / (M * K) == facts["i2s_bits_per_weight"]["value"]
    assert np.array_equal(oracle.unpack(p, M, K), c)
    # no 2-bit field ever holds 3
    fields = np.stack([(p >> np.uint32(2 * i)) & np.uint32(3) for i in range(16)])
    assert not (fields == 3).any()
    # (word >> 2j) & 0x03030303 yields the codes+1 of weights 16w+4j .. 16w+4j+3,
    # one per byte lane, in k order
    for j in range(4):
        lanes = ((p >> np.uint32(2 * j)) & np.uint32(0x03030303)).view(np.uint8)
        lanes = lanes.reshape(M, K // 16, 4).astype(np.int16) - 1
        assert np.array_equal(lanes, c.reshape(M, K // 16, 4, 4)[:, :, j, :])


@pytest.mark.parametrize("K", [16, 48, 80, 96, 1008])
def test_pack_ragged_rows_padded_with_code_zero(K):
    # rows whose K is not a multiple of 64 are padded to a 16-byte boundary;
    # padding fields hold 01 (code 0), so a padded row weighs exactly what the
    # unpadded one does
    r = rng(K)
    M = 5
    c = r.integers(-1, 2, size=(M, K)).astype(np.int8)
    p = oracle.pack(c)
    wpr = -(-K // 64) * 4
    assert oracle.packed_row_words(K) == wpr and p.shape == (M, wpr)
    assert p.nbytes % (16 * M) == 0
    assert np.array_equal(oracle.unpack(p, M, K), c)
    # the first K/16 words are the unpadded layout, word by word
    for m in range(M):
        for w in range(K // 16):
            word = 0
            for i in range(16):
                k = 16 * w + i
                word |= (int(c[m, k]) + 1) << (8 * (k % 4) + 2 * ((k % 16) // 4))
            assert p[m, w] == word
    assert (p[:, K // 16:] == 0x55555555).all()
    # a padding field that is not code 0 is rejected
    if K % 64:
        bad = p.copy()
        bad[0, -1] ^= np.uint32(1)
        with pytest.raises(ValueError):
            oracle.unpack(bad, M, K)
    # the padding changes no product: acc over the padded row equals acc over K
    q = r.integers(-128, 128, size=(3, K)).astype(np.int8)
    assert np.array_equal(oracle.matmul_i32(oracle.unpack(p, M, K), q),
                          oracle.matmul_addsub(c, q))


def test_packed_rows_are_unpadded_when_k_is_a_multiple_of_64():
    for K in (64, 128, 2560, 6912, 11008, 28672):
        assert oracle.packed_row_words(K) == K // 16


def test_pack_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.pack(np.full((1, 16), 2, dtype=np.int8))
    bad = np.full((1, 1), 0xFFFFFFFF, dtype=np.uint32)
    with pytest.raises(ValueError):
        oracle.unpack(bad, 1, 16)


# ----------------------------------------------------------------------------- activations

def test_quant_act_half_even_hand_values():
    # amax = 127 makes s = 127/127 = 1 exactly, so q = rint(x) with ties to even
    x = np.array([[0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.49, 127.0, -126.5]], np.float32)
    q, amax, qsum = oracle.quant_act(x)
    assert amax[0] == 127.0
    assert q[0].tolist() == [0, 2, 2, 0, -2, -2, 3, 127, -126]
    assert qsum[0] == sum([0, 2, 2, 0, -2, -2, 3, 127, -126])


def test_quant_act_zero_token_and_bounds():
    x = np.zeros((3, 64), np.float32)
    x[1] = inputs.activations(1, 64, seed=3).numpy()
    q, amax, qsum = oracle.quant_act(x)
    assert amax[0] == 0 and not q[0].any() and qsum[0] == 0
    assert np.abs(q[1].astype(int)).max() == 127
    assert q[1][np.argmax(np.abs(x[1]))] in (127, -127)
    assert (q[1].astype(int) >= -127).all()


def test_quant_act_symmetry_and_power_of_two():
    x = inputs.activations(4, 512, seed=8, outlier_count=4).numpy()
    q, amax, _ = oracle.quant_act(x)
    qn, amaxn, _ = oracle.quant_act(-x)
    assert np.array_equal(qn, -q) and np.array_equal(amaxn, amax)
    for j in (-4, 6):
        q2, amax2, _ = oracle.quant_act(x * np.float32(2.0 ** j))
        assert np.array_equal(q2, q)
        assert np.array_equal(amax2, amax * np.float32(2.0 ** j))


def test_quant_act_overflowing_scale():
    # amax so small that 127/amax overflows fp32: s = inf, x*s = +-inf -> clamp, 0*inf -> 0
    tiny = np.float32(1e-44)
    x = np.array([[tiny, -tiny, 0.0, tiny / 2]], np.float32)
    q, amax, _ = oracle.quant_act(x)
    with np.errstate(over="ignore"):
        assert np.isinf(np.float32(127.0) / amax[0])
    assert q[0].tolist() == [127, -128, 0, 127]


def test_quant_act_rounding_within_half_step():
    x = inputs.activations(8, 1024, seed=21, outlier_frac=0.01).numpy()
    q, amax, _ = oracle.quant_act(x)
    step = amax.astype(np.float64)[:, None] / 127
    err = np.abs(x - q * step)
    assert (err <= step * (0.5 + 1e-4)).all()   # s and x*s each round once


def test_per_tensor_quant_pins():
    x = inputs.activations(5, 256, seed=44, outlier_count=3).numpy()
    q, amax, qsum = oracle.quant_act_per_tensor(x)
    # one scale: every amax entry is max|x| over the tensor
    assert (amax == np.abs(x).max()).all()
    # a single token is the per-token rule
    for n in range(5):
        q1, a1, s1 = oracle.quant_act(x[n:n + 1])
        qt, at, st = oracle.quant_act_per_tensor(x[n:n + 1])
        assert np.array_equal(q1, qt) and a1[0] == at[0] and s1[0] == st[0]
    # the token holding the tensor maximum quantises as it would per token
    top = np.argmax(np.abs(x).max(axis=1))
    assert np.array_equal(q[top], oracle.quant_act(x[top:top + 1])[0][0])
    # hand values: amax = 127 gives s = 1, so q = rint(x) with ties to even
    y = np.array([[0.5, 2.5, -1.5, 3.0], [127.0, -0.5, 1.5, 0.0]], np.float32)
    qy, ay, sy = oracle.quant_act_per_tensor(y)
    assert qy.tolist() == [[0, 2, -2, 3], [127, 0, 2, 0]] and sy.tolist() == [3, 129]
    # all zero
    qz, az, sz = oracle.quant_act_per_tensor(np.zeros((3, 128), np.float32))
    assert not qz.any() and not az.any() and not sz.any()


# ----------------------------------------------------------------------------- matmul

@pytest.mark.parametrize("M,K,N", [(1, 16, 1), (5, 16, 3), (16, 16, 2), (7, 32, 3)])
def test_addsub_brute_force_equals_mad(M, K, N):
    r = rng(M * 100 + K + N)
    c = r.integers(-1, 2, size=(M, K)).astype(np.int8)
    q = r.integers(-128, 128, size=(N, K)).astype(np.int8)
    a1 = oracle.matmul_i32(c, q)
    a2 = oracle.matmul_addsub(c, q)
    a3 = q.astype(np.int64) @ c.astype(np.int64).T          # library matmul
    assert np.array_equal(a1, a2) and np.array_equal(a1, a3)


def test_matmul_library_agreement_larger():
    r = rng(31)
    c = r.integers(-1, 2, size=(96, 512)).astype(np.int8)
    q = r.integers(-128, 128, size=(5, 512)).astype(np.int8)
    assert np.array_equal(oracle.matmul_i32(c, q), q.astype(np.int64) @ c.astype(np.int64).T)


def test_all_plus_one_and_minus_one_give_row_sums():
    x = inputs.activations(3, 256, seed=2).numpy()
    for sign in (1, -1):
        W = np.full((8, 256), sign * 0.013, np.float32)
        out = oracle.bitlinear(W, x)
        assert out["alpha"] == np.float32(0.013)
        assert (out["codes"] == sign).all()
        assert np.array_equal(out["acc"], sign * np.repeat(out["qsum"][:, None], 8, 1))
        assert np.array_equal(out["qsum"], out["q"].astype(np.int64).sum(1))


def test_one_hot_activation_selects_a_code_column():
    W = inputs.latent_weights(16, 64, seed=13).numpy()
    x = np.zeros((1, 64), np.float32)
    x[0, 37] = 3.0
    out = oracle.bitlinear(W, x)
    assert out["q"][0, 37] == 127 and np.count_nonzero(out["q"]) == 1
    assert np.array_equal(out["acc"][0], 127 * out["codes"][:, 37].astype(np.int32))


def test_negated_activation_negates_acc():
    W = inputs.latent_weights(32, 128, seed=14).numpy()
    x = inputs.activations(2, 128, seed=15).numpy()
    a = oracle.bitlinear(W, x)
    b = oracle.bitlinear(W, -x)
    assert np.array_equal(b["acc"], -a["acc"]) and np.array_equal(b["y"], -a["y"])


def test_accumulator_bound():
    K = 28672
    c = np.ones((1, K), np.int8)
    q = np.full((1, K), 127, np.int8)
    acc = oracle.matmul_i32(c, q)
    assert acc[0, 0] == 127 * K and 127 * K < 2 ** 24


# ----------------------------------------------------------------------------- rescale / layer

def test_rescale_within_three_roundings_of_exact():
    r = rng(41)
    acc = r.integers(-3_000_000, 3_000_000, size=(3, 50)).astype(np.int32)
    amax = np.array([0.7, 12.5, 3.3e-3], np.float32)
    alpha = np.float32(0.0151)
    y = oracle.rescale(acc, alpha, amax)
    for n in range(3):
        for m in range(50):
            exact = Fraction(int(acc[n, m])) * Fraction(float(alpha)) * Fraction(float(amax[n])) / 127
            if exact == 0:
                assert y[n, m] == 0
                continue
            rel = abs((Fraction(float(y[n, m])) - exact) / exact)
            assert rel <= 3 * Fraction(1, 2 ** 24)


def test_unquantised_agreement_bound():
    W = inputs.latent_weights(64, 512, seed=16).numpy()
    x = inputs.activations(3, 512, seed=17, outlier_count=4).numpy()
    out = oracle.bitlinear(W, x)
    Wt = out["alpha"].astype(np.float64) * out["codes"].astype(np.float64)   # dequantised
    ref = x.astype(np.float64) @ Wt.T
    nnz = np.count_nonzero(out["codes"], axis=1)
    bound = (float(out["alpha"]) * out["amax"].astype(np.float64)[:, None] / 254 * nnz[None, :])
    slack = 4e-7 * np.abs(ref) + 1e-30      # fp32 rounding of y, s and x*s
    assert (np.abs(out["y"] - ref) <= bound * (1 + 1e-4) + slack).all()


def test_pages_facts_fixture():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    assert abs(math.log2(3) - facts["ternary_bits_per_weight"]["value"]) < 0.005
    assert facts["tl2_bits_per_weight"]["value"] == pytest.approx(5 / 3, abs=0.005)
    assert facts["ternary_values"]["value"] == [-1, 0, 1]
    assert facts["fairyfuse_threshold_fraction"]["value"] == 0.5
    # the threshold rule is the ternariser away from ties
    a = np.float32(1.0)
    t = facts["fairyfuse_threshold_fraction"]["value"]
    w = np.array([t + 1e-3, -(t + 1e-3), t - 1e-3, 0.0], np.float32)
    assert oracle.ternarize(w, a).tolist() == [1, -1, 0, 0]


def test_seeded_regression_fixture():
    path = os.path.join(GOLDEN, "oracle_small_case.json")
    g = json.load(open(path))
    W = np.array(g["W"], np.float32).reshape(g["M"], g["K"])
    x = np.array(g["x"], np.float32).reshape(g["N"], g["K"])
    out = oracle.bitlinear(W, x)
    assert float(out["alpha"]) == g["alpha"]
    assert out["packed"].ravel().tolist() == g["packed"]
    assert out["q"].ravel().tolist() == g["q"]
    assert out["acc"].ravel().tolist() == g["acc"]
    assert out["y"].ravel().tolist() == g["y"]


# ----------------------------------------------------------------------------- TL2-style storage

def _tl2_group(c0, c1, c2):
    """(sign, index) of a group of three codes at the front of a 96-wide row."""
    codes = np.zeros((1, 96), dtype=np.int8)
    codes[0, :3] = (c0, c1, c2)
    row = oracle.tl2_encode(codes)[0]
    return int(row[16] & 1), int(row[0] & 15)      # sign plane starts after 16 index bytes


def test_tl2_mirror_consolidation_and_sign_index_split():
    # 27 combinations of three ternary weights fold onto 14 indices (4 bits) and
    # a sign bit: negating every code of a group flips its sign and nothing else
    import itertools
    seen = {}
    for combo in itertools.product((-1, 0, 1), repeat=3):
        s, i = _tl2_group(*combo)
        assert 0 <= i <= 13
        seen[(s, i)] = combo
        ns, ni = _tl2_group(*[-c for c in combo])
        if any(combo):
            assert ni == i and ns == 1 - s, combo
        else:
            assert (s, i) == (0, 0) and (ns, ni) == (0, 0)
    assert len(seen) == 27                                  # one code per combination
    assert len({i for _, i in seen}) == 14


@pytest.mark.parametrize("K", [16, 96, 112, 384, 2560, 6912, 4096, 176])
def test_tl2_roundtrip_size_and_remainder(K):
    r = rng(K + 3)
    M = 4
    c = r.integers(-1, 2, size=(M, K)).astype(np.int8)
    t = oracle.tl2_encode(c)
    nb, k2 = K // 96, K % 96
    assert t.shape == (M, 16 * nb + 16 * (-(-nb // 4)) + 16 * (-(-k2 // 64)))
    assert t.shape[1] % 16 == 0
    assert np.array_equal(oracle.tl2_decode(t, M, K), c)
    # the remainder (the last K % 96 weights) is the 2-bit layout of oracle.pack
    if k2:
        tail = t[:, t.shape[1] - 16 * (-(-k2 // 64)):].copy().view(np.uint32)
        assert np.array_equal(tail, oracle.pack(c[:, 96 * nb:]))


def test_tl2_bits_per_weight_from_the_pages():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    K = 384                        # four whole blocks of 96: no remainder, no padding
    assert oracle.tl2_row_bytes(K) * 8 / K == pytest.approx(5 / 3, abs=1e-12)
    assert oracle.tl2_row_bytes(K) * 8 / K == pytest.approx(
        facts["tl2_bits_per_weight"]["value"], abs=0.005)
    # the shapes of the 2B model: 6912 = 72 blocks exactly; 2560 keeps a 64-weight remainder
    assert oracle.tl2_row_bytes(6912) == 6912 * 5 // 3 // 8
    assert oracle.tl2_row_bytes(2560) == 26 * 16 + 112 + 16


def test_tl2_rejects_invalid_rows():
    c = np.zeros((1, 96), dtype=np.int8)
    t = oracle.tl2_encode(c)
    assert not t.any()                           # all-zero codes: index 0, sign 0 everywhere
    bad = t.copy()
    bad[0, 0] = 14                               # index above 13
    with pytest.raises(ValueError):
        oracle.tl2_decode(bad, 1, 96)
    bad = t.copy()
    bad[0, 16] = 1                               # sign on the zero group (negative zero)
    with pytest.raises(ValueError):
        oracle.tl2_decode(bad, 1, 96)
    bad = t.copy()
    bad[0, 20] = 1                               # sign-plane padding
    with pytest.raises(ValueError):
        oracle.tl2_decode(bad, 1, 96)
