"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: the
textbook definition softmax(Q K^T * scale) V evaluated by torch in float64,
closed forms on hand-built inputs whose skip set is known, invariants of the
method, numpy's least-squares fit, and constants printed on the pages
(tests/golden/page_constants.txt). A plausible slip in the oracle (a dropped
column, a wrong running-max rule, a sign or index error in the vote, log2 vs
natural log) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.golden import first

T = oracle.TILE


def as_bf16(x):
    return synth.f32_to_bf16(np.asarray(x, dtype=np.float32))


def textbook(q, k, v, cu, H, D, scale, col_mask=None):
    """softmax(Q K^T * scale) V per (sequence, head) in float64 via torch.
    col_mask(b, h) -> bool [S] of the key columns that take part (all if None)."""
    qf, kf, vf = (torch.from_numpy(synth.bf16_to_f32(a).astype(np.float64)) for a in (q, k, v))
    out = {}
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        for h in range(H):
            logits = (qf[s0:s1, h] @ kf[s0:s1, h].T) * scale
            if col_mask is not None:
                m = torch.from_numpy(col_mask(b, h))
                logits[:, ~m] = -math.inf
            out[(b, h)] = torch.softmax(logits, dim=-1) @ vf[s0:s1, h]
    return out


def unit_rows(res, i, cu, units):
    b, h, qb = units[i]
    S = int(cu[b + 1] - cu[b])
    n = min(T, S - qb * T)
    return res["out"][i, :n]


def varlen_random(lengths, H, D, seed, amp=3.0):
    w = synth.Workload("t", [(1, 1, s) for s in lengths], H=H, D=D, seed=seed, amp=amp)
    q, k, v = synth.generate(w, nthreads=4)
    return w, q, k, v


# ---------------------------------------------------------------- dense path


@pytest.mark.parametrize("D", [64, 128])
def test_dense_walk_equals_textbook_softmax(D):
    """tsf = 0 (lambda -> 0): the tiled online walk reproduces softmax attention
    on ragged lengths (1, short, exactly one tile, one tile + 1, several tiles)."""
    lengths = [1, 5, 127, 128, 129, 300]
    H = 2
    w, q, k, v = varlen_random(lengths, H, D, seed=3)
    cu = w.cu_seqlens
    res = oracle.walk(q, k, v, cu, H, D, tsf=0.0)
    ref = textbook(q, k, v, cu, H, D, 1.0 / math.sqrt(D))
    units = res["units"]
    assert res["skips"].sum() == 0
    vmax = np.abs(synth.bf16_to_f32(v)).max()
    for i, (b, h, qb) in enumerate(units):
        got = unit_rows(res, i, cu, units)
        exp = ref[(b, h)][qb * T: qb * T + got.shape[0]].numpy()
        # scores are rounded to fp32 in the log2 domain: ~1e-6 relative weight error
        np.testing.assert_allclose(got, exp, rtol=0, atol=2e-5 * vmax)
        # fp32 output of a double accumulation: nothing coarser than that
        assert np.all(np.isfinite(got))


def test_dense_walk_exact_on_integer_scores():
    """Integer Q, K and a scale whose log2-domain factor is exactly 0.25 make
    every score exact in fp32, so the walk must equal the textbook softmax to
    double rounding: pins score scaling (log2 e factor) and column coverage."""
    D, H = 64, 1
    lengths = [300, 131]
    rng = np.random.default_rng(11)
    n = sum(lengths)
    q = as_bf16(rng.integers(-2, 3, size=(n, H, D)))
    k = as_bf16(rng.integers(-2, 3, size=(n, H, D)))
    v = as_bf16(rng.standard_normal((n, H, D)))
    cu = np.array([0, lengths[0], n], dtype=np.int32)
    scale = 0.25 / math.log2(math.e)
    assert oracle.score_scale(scale, D) == 0.25
    res = oracle.walk(q, k, v, cu, H, D, softmax_scale=scale, tsf=0.0)
    ref = textbook(q, k, v, cu, H, D, scale)
    for i, (b, h, qb) in enumerate(res["units"]):
        got = unit_rows(res, i, cu, res["units"])
        exp = ref[(b, h)][qb * T: qb * T + got.shape[0]].numpy()
        np.testing.assert_allclose(got, exp, rtol=1e-6, atol=1e-7)


# ------------------------------------------------------ hand-built skip sets


def constant_score_inputs(S, D=64, seed=0):
    rng = np.random.default_rng(seed)
    q = as_bf16(np.zeros((S, 1, D)))
    k = as_bf16(rng.standard_normal((S, 1, D)))
    v = as_bf16(rng.standard_normal((S, 1, D)))
    return q, k, v, np.array([0, S], dtype=np.int32)


@pytest.mark.parametrize("S", [1000, 640])
def test_constant_scores(S):
    """Q = 0 gives all-zero scores: every d is 0 after tile 0. lambda <= 1
    (including lambda = 1 exactly, strict <) skips nothing and gives the mean
    of all V rows; lambda > 1 skips every tile but the first and gives the
    mean of the first tile's V rows."""
    q, k, v, cu = constant_score_inputs(S)
    vf = synth.bf16_to_f32(v)[:, 0].astype(np.float64)
    nt = (S + T - 1) // T
    for tsf, expect_skips, rows in [(0.3 * S, 0, S), (1.0 * S, 0, S), (2.0 * S, nt - 1, T)]:
        res = oracle.walk(q, k, v, cu, 1, 64, tsf=tsf)
        assert np.all(res["skips"] == expect_skips), tsf
        exp = vf[:rows].mean(axis=0)
        for i in range(res["out"].shape[0]):
            n = min(T, S - i * T)
            np.testing.assert_allclose(res["out"][i, :n], np.broadcast_to(exp, (n, 64)), rtol=0, atol=1e-6)
        d = res["dstat"][:, 1:nt]
        assert np.all(d == 0.0) and np.all(np.isinf(res["dstat"][:, 0]))


def dominant_tile_inputs(S, jstar, D=64):
    """Every Q row is u = 16 e0; K rows of tile jstar are 16 e0, all other K rows
    are 0. Scores: 256/sqrt(D) on tile jstar, 0 elsewhere."""
    rng = np.random.default_rng(5)
    q = np.zeros((S, 1, D), dtype=np.float32)
    q[:, 0, 0] = 16.0
    k = np.zeros((S, 1, D), dtype=np.float32)
    k[jstar * T: min(S, (jstar + 1) * T), 0, 0] = 16.0
    v = rng.standard_normal((S, 1, D)).astype(np.float32)
    return as_bf16(q), as_bf16(k), as_bf16(v), np.array([0, S], dtype=np.int32)


@pytest.mark.parametrize("S,jstar", [(1024, 3), (1000, 7), (700, 0)])
def test_dominant_tile_known_skip_set(S, jstar):
    """lambda <= 1: tiles 0..j* are kept, every later tile is skipped.
    lambda > 1: tile 0 and tile j* are kept, everything else is skipped; with
    a running max taken AFTER the tile, j* would be skipped too, so this pins
    the before-the-tile rule. Outputs equal softmax over the kept columns."""
    D = 64
    q, k, v, cu = dominant_tile_inputs(S, jstar, D)
    nt = (S + T - 1) // T
    scale = 1.0 / math.sqrt(D)
    for lam in [1e-3, 0.5, 4.0]:
        res = oracle.walk(q, k, v, cu, 1, D, tsf=lam * S)
        if lam <= 1:
            kept = set(range(0, jstar + 1))
        else:
            kept = {0, jstar}
        expect = np.array([0 if j in kept else 1 for j in range(nt)], dtype=np.uint8)
        for i in range(nt):
            np.testing.assert_array_equal(res["decision"][i, :nt], expect, err_msg=f"lam={lam} qb={i}")
        cols = np.zeros(S, dtype=bool)
        for j in kept:
            cols[j * T: min(S, (j + 1) * T)] = True
        ref = textbook(q, k, v, cu, 1, D, scale, col_mask=lambda b, h: cols)[(0, 0)].numpy()
        for i in range(nt):
            n = min(T, S - i * T)
            np.testing.assert_allclose(res["out"][i, :n], ref[i * T: i * T + n], rtol=1e-6, atol=1e-6)


# --------------------------------------------------------------- invariants


def test_skip_sets_nested_in_lambda():
    """For lambda <= 1 a skipped tile never raises the running max, so the
    trajectory does not depend on lambda and skip sets grow with lambda."""
    w, q, k, v = varlen_random([1000, 777], 2, 64, seed=9)
    cu = w.cu_seqlens
    lams = [1e-6, 1e-4, 1e-3, 1e-2, 0.1, 0.5, 1.0]
    prev = None
    total = []
    for lam in lams:
        L = [oracle.lambda_log2(lam)] * 2
        res = oracle.walk(q, k, v, cu, 2, 64, L_seq=L)
        dec = res["decision"].astype(bool)
        if prev is not None:
            assert np.all(dec[prev]), f"a tile skipped at a smaller lambda is kept at {lam}"
        prev = dec
        total.append(int(dec.sum()))
    assert total == sorted(total) and total[-1] > total[0]


def test_skip_error_bound():
    """For lambda <= 1 every skipped probability is below lambda relative to
    the final max (the kept max has weight 1), so per row
    |O_skip - O_dense| <= 2 * n_skipped_tiles * 128 * lambda * max|V|."""
    w, q, k, v = varlen_random([1500], 2, 128, seed=4)
    cu = w.cu_seqlens
    dense = oracle.walk(q, k, v, cu, 2, 128, tsf=0.0)
    vmax = np.abs(synth.bf16_to_f32(v)).max()
    for lam in [1e-4, 1e-2, 0.2]:
        res = oracle.walk(q, k, v, cu, 2, 128, L_seq=[oracle.lambda_log2(lam)])
        for i in range(res["out"].shape[0]):
            bound = 2 * res["skips"][i] * T * lam * vmax
            err = np.abs(res["out"][i] - dense["out"][i]).max()
            assert err <= bound + 1e-6, (lam, i, err, bound)
    assert res["skips"].sum() > 0


def test_calibration_counts_equal_forward_skips():
    """Calibration never skips (its output is the dense one, bit for bit) and
    for every lambda_k <= 1 its count equals the forward pass's skip count."""
    lams = [1e-5, 1e-3, 1e-2, 0.1, 0.7, 1.0]
    w, q, k, v = varlen_random([900, 1300], 2, 64, seed=2)
    cu = w.cu_seqlens
    cal = oracle.walk(q, k, v, cu, 2, 64, cal_lambdas=lams)
    dense = oracle.walk(q, k, v, cu, 2, 64, tsf=0.0)
    np.testing.assert_array_equal(cal["out"], dense["out"])
    for kk, lam in enumerate(lams):
        fw = oracle.walk(q, k, v, cu, 2, 64, L_seq=[oracle.lambda_log2(lam)] * 2)
        np.testing.assert_array_equal(cal["counts"][:, kk], fw["skips"])


def test_forced_decisions_replay():
    """Forcing the oracle's own decisions reproduces it; forcing a keep on a
    skipped tile changes the skip count by one."""
    w, q, k, v = varlen_random([1000], 1, 64, seed=6)
    cu = w.cu_seqlens
    L = [oracle.threshold_log2(5000.0, 1000)]
    base = oracle.walk(q, k, v, cu, 1, 64, L_seq=L)
    rep = oracle.walk(q, k, v, cu, 1, 64, L_seq=L, forced=base["decision"].astype(np.int8))
    np.testing.assert_array_equal(rep["out"], base["out"])
    forced = -np.ones_like(base["decision"], dtype=np.int8)
    i, j = np.argwhere(base["decision"] == 1)[0]
    forced[i, j] = 0
    alt = oracle.walk(q, k, v, cu, 1, 64, L_seq=L, forced=forced)
    assert alt["skips"][i] == base["skips"][i] - 1 or alt["skips"][i] < base["skips"][i]


def test_sampled_units_match_full_walk():
    """A unit's result does not depend on which other units are walked."""
    w, q, k, v = varlen_random([700, 260], 3, 64, seed=1)
    cu = w.cu_seqlens
    full = oracle.walk(q, k, v, cu, 3, 64, tsf=300.0)
    units = oracle.sample_units(cu, 3, 5, seed=3)
    part = oracle.walk(q, k, v, cu, 3, 64, tsf=300.0, units=units, max_tiles=full["max_tiles"])
    index = {tuple(u): i for i, u in enumerate(full["units"])}
    for i, u in enumerate(units):
        np.testing.assert_array_equal(part["out"][i], full["out"][index[tuple(u)]])
        np.testing.assert_array_equal(part["decision"][i], full["decision"][index[tuple(u)]])


# ----------------------------------------------------- threshold conversion


def test_threshold_conversion_page_pin():
    """The pages replaced a raw log2 threshold of -0.7 by lambda = 0.61557,
    so L = log2(lambda) without a softmax-scale factor; lambda is
    threshold_scale_factor / S_kv; tsf = 0 disables skipping."""
    (lam, raw), = first("page_constants.txt", "lambda_log2")
    for S in [1024, 75600]:
        assert oracle.threshold_log2(lam * S, S) == pytest.approx(raw, abs=1e-4)
    assert oracle.threshold_log2(0.0, 1024) == -math.inf
    assert oracle.threshold_log2(1024.0, 1024) == 0.0
    assert oracle.threshold_log2(5000.0, 75600) == pytest.approx(math.log2(5000 / 75600), abs=1e-6)
    assert oracle.score_scale(0.0, 128) == pytest.approx(1 / math.sqrt(128) / math.log(2), rel=1e-7)


def test_raw_lambda_conversion_pins():
    """The calibration trials are raw lambda values compared as log2(lambda):
    the page constant (lambda 0.61557 replacing log2-space -0.7) holds for the
    raw conversion too; exact powers of two map to their exponents (a natural
    log or a missing fp32 rounding would not); 2**L gives lambda back to fp32
    precision for every printed trial; and the raw conversion agrees with the
    scale-factor one, lambda = tsf / S_kv, where tsf / S_kv is exact."""
    (lam, raw), = first("page_constants.txt", "lambda_log2")
    assert oracle.lambda_log2(lam) == pytest.approx(raw, abs=1e-4)
    for e in range(-24, 4):
        assert oracle.lambda_log2(2.0 ** e) == float(e)
    (trials,) = first("page_constants.txt", "trials")
    for x in trials:
        L = oracle.lambda_log2(x)
        assert np.float32(L) == L  # an fp32 value
        assert 2.0 ** L == pytest.approx(x, rel=3e-7 * max(1.0, abs(L)))
        for S in [1024, 65536]:  # powers of two: x * S / S is exact in double
            assert oracle.lambda_log2(x) == oracle.threshold_log2(x * S, S)
    assert oracle.lambda_log2(0.0) == -math.inf and oracle.lambda_log2(-1.0) == -math.inf
    assert oracle.lambda_log2(1.0) == 0.0


# ------------------------------------------------------------ fit / resolve


def test_fit_recovers_page_coefficients():
    """Points drawn from each printed (a, b) pair are fitted back exactly;
    points at s = 0 or 1 carry no information and are ignored."""
    s = np.linspace(0.1, 0.9, 9)
    for a, b in first("page_constants.txt", "formula"):
        sf = np.array([oracle.resolve(a, b, x) for x in s])
        assert oracle.resolve(a, b, 0.0) == a
        fa, fb, smin, smax = oracle.fit_logspace(s, sf)
        assert fa == pytest.approx(a, rel=1e-12) and fb == pytest.approx(b, rel=1e-12)
        assert (smin, smax) == (pytest.approx(0.1), pytest.approx(0.9))
        junk_s = np.concatenate([s, [0.0, 1.0, 0.5]])
        junk_sf = np.concatenate([sf, [123.0, 456.0, -1.0]])
        assert oracle.fit_logspace(junk_s, junk_sf)[:2] == pytest.approx((fa, fb), rel=1e-12)


def test_fit_matches_numpy_polyfit_on_noisy_points():
    rng = np.random.default_rng(0)
    s = rng.uniform(0.05, 0.95, 40)
    sf = 7.93 * np.exp(8.61 * s) * np.exp(rng.normal(0, 0.3, 40))
    b, ln_a = np.polyfit(s, np.log(sf), 1)
    fa, fb, _, _ = oracle.fit_logspace(s, sf)
    assert fb == pytest.approx(b, rel=1e-10) and fa == pytest.approx(math.exp(ln_a), rel=1e-10)


def test_fit_and_resolve_reject_degenerate_input():
    with pytest.raises(ValueError):
        oracle.fit_logspace([0.5, 0.5], [1.0, 2.0])
    with pytest.raises(ValueError):
        oracle.fit_logspace([0.0, 1.0], [1.0, 2.0])
    assert math.isnan(oracle.resolve(-1.0, 2.0, 0.5))
    assert math.isnan(oracle.resolve(1.0, 2.0, 1.5))


# ------------------------------------------------------ 8-bit P.V reading


def e4m3_values():
    """Every non-negative finite E4M3 value, built from the bit fields (4
    exponent bits, bias 7, 3 mantissa bits, exponent field 0 subnormal, the
    all-ones pattern S.1111.111 not a number)."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            vals.append(m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(sorted(vals))


def test_e4m3_nearest_is_the_brute_force_nearest_value():
    """The oracle's rounding equals the nearest value of the enumerated E4M3
    set, ties to the value with an even mantissa, saturating at 448; and it
    agrees with the input quantiser's independent implementation."""
    vals = e4m3_values()
    assert len(vals) == 127 and vals[-1] == 448.0 and vals[1] == 2.0 ** -9
    rng = np.random.default_rng(3)
    xs = np.concatenate([vals, (vals[1:] + vals[:-1]) / 2,  # every midpoint: a tie
                         rng.uniform(0, 460, 3000), np.exp2(rng.uniform(-14, 9, 3000)), [460.0, 1e6]])
    codes = {v: i for i, v in enumerate(vals)}
    for x in xs:
        got = oracle.e4m3_nearest(float(x))
        if x >= 448.0:
            assert got == 448.0
            continue
        d = np.abs(vals - x)
        best = vals[d == d.min()]
        if len(best) == 2:  # tie: the even code (mantissa LSB 0) wins
            best = [b for b in best if codes[b] % 2 == 0]
        assert got == best[0], (x, got, best)
    q = synth.f32_to_e4m3(np.asarray(xs[xs < 448], dtype=np.float32))
    np.testing.assert_array_equal(synth.e4m3_to_f32(q).astype(np.float64),
                                  [oracle.e4m3_nearest(float(np.float32(x))) for x in xs[xs < 448]])


def _integer_score_case(S, D=16, seed=0, spread=5):
    """Q, K with small integers so that every score q.k is an integer, and a
    softmax scale whose log2-domain factor is exactly 1: s2 = q.k."""
    rng = np.random.default_rng(seed)
    q = np.zeros((S, 1, D), np.float32)
    q[:, 0, :3] = rng.integers(0, 2, (S, 3))  # rows differ in which of three score terms they see
    k = rng.integers(-1, 2, (S, 1, D)).astype(np.float32)
    k[:, 0, :3] = rng.integers(0, spread, (S, 3))  # scores q.k in [0, 3 (spread - 1)]
    v = rng.standard_normal((S, 1, D)).astype(np.float32)
    scale = math.log(2.0)
    assert oracle.score_scale(scale, D) == 1.0
    return as_bf16(q), as_bf16(k), as_bf16(v), np.array([0, S], np.int32), scale


def test_e4m3_pv_is_exact_when_every_probability_is_a_power_of_two():
    """Integer scores (window of a few units): against the integer reference
    every P = 2^(s - r + 8) is a power of two inside the E4M3 range, so the
    8-bit P.V walk must give the exact walk's output; rescales are powers of
    two as well. (A wrong reference or shift would push P out of range.)"""
    q, k, v, cu, scale = _integer_score_case(300)
    exact = oracle.walk(q, k, v, cu, 1, 16, softmax_scale=scale, tsf=0.0)
    pv8 = oracle.walk(q, k, v, cu, 1, 16, softmax_scale=scale, tsf=0.0, p_e4m3=True)
    np.testing.assert_allclose(pv8["out"], exact["out"], rtol=1e-6, atol=1e-7)
    # a shift that would push P over 448 saturates, and then the outputs differ
    sat = oracle.walk(q, k, v, cu, 1, 16, softmax_scale=scale, tsf=0.0, p_e4m3=True, p_shift=10.0)
    assert np.abs(sat["out"] - exact["out"]).max() > 1e-3


def test_e4m3_pv_single_tile_by_hand():
    """One row, one tile: P_c = 2^(s_c - ceil(max s) + 8), O = sum(round(P_c) v_c) / sum(P_c)
    with round() the brute-force nearest E4M3 value; V one-hot per column so
    each output coordinate isolates one rounded probability."""
    S, D = 9, 16
    s = np.array([0.3, -1.7, 2.2, 2.45, -5.1, 0.0, 1.15, -0.6, 2.4])  # log2-domain scores
    q = np.zeros((S, 1, D), np.float32)
    k = np.zeros((S, 1, D), np.float32)
    q[:, 0, 0] = 1.0
    k[:, 0, 0] = s  # q.k = s for the first query row (other rows: same)
    v = np.zeros((S, 1, D), np.float32)
    for c in range(S):
        v[c, 0, c] = 1.0
    qb, kb, vb = as_bf16(q), as_bf16(k), as_bf16(v)
    s_bf = synth.bf16_to_f32(kb[:, 0, 0]).astype(np.float64)  # the scores after bf16 rounding of k
    res = oracle.walk(qb, kb, vb, np.array([0, S], np.int32), 1, D, softmax_scale=math.log(2.0), tsf=0.0,
                      p_e4m3=True)
    vals = e4m3_values()
    r = math.ceil(s_bf.max())
    P = 2.0 ** (s_bf - r + 8)
    Pq = np.array([vals[np.argmin(np.abs(vals - p))] for p in P])  # no ties among these values
    expect = Pq / P.sum()
    np.testing.assert_allclose(res["out"][0, 0, :S], expect, rtol=1e-6)


def test_e4m3_pv_error_bound_against_the_exact_walk():
    """Rounding P to E4M3 moves each product by at most 2^-4 of it, and the
    flushed values are below 2^-10 against a row maximum above 2^7, so
    |O_8bit - O_exact| <= (2^-4 + S * 2^-17) * max|V| per row."""
    w, q, k, v = varlen_random([1000, 333], 2, 64, seed=8)
    cu = w.cu_seqlens
    exact = oracle.walk(q, k, v, cu, 2, 64, tsf=0.0)
    pv8 = oracle.walk(q, k, v, cu, 2, 64, tsf=0.0, p_e4m3=True)
    vmax = np.abs(synth.bf16_to_f32(v)).max()
    err = np.abs(pv8["out"] - exact["out"]).max()
    assert err <= (2.0 ** -4 + 1000 * 2.0 ** -17) * vmax
    assert err > 0  # the rounding is really applied
    sk = oracle.walk(q, k, v, cu, 2, 64, tsf=500.0, p_e4m3=True)  # the skip rule does not change
    assert np.array_equal(sk["decision"], oracle.walk(q, k, v, cu, 2, 64, tsf=500.0)["decision"])
