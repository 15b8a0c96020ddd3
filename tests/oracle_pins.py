"""Pins of the CPU oracle to things other than itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with a closed form, an invariant, a textbook routine or an
independent brute-force formulation.  ``test_oracle_pins.py`` runs them on
the real oracle; ``test_oracle_mutations.py`` runs them on copies of the
oracle with planted mistakes and checks that every mistake is caught.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import qsa_inputs as Q

SQRT_D = math.sqrt(128.0)


def _bf(x):
    """bf16 bits of values that are exactly representable."""
    b = Q.f32_to_bf16(np.asarray(x, dtype=np.float32))
    assert np.array_equal(Q.bf16_to_f32(b), np.asarray(x, dtype=np.float32)), "not bf16-exact"
    return b


def _rope_complex(x: np.ndarray, pos: int, theta=1e7, rope_dim=64) -> np.ndarray:
    """RoPE as complex multiplication: z_i = x_i + i x_{i+32} times e^{i pos theta^(-i/32)}."""
    half = rope_dim // 2
    y = np.array(x, dtype=np.float64, copy=True)
    z = x[..., :half] + 1j * x[..., half:rope_dim]
    f = theta ** (-np.arange(half) / half)
    z = z * np.exp(1j * pos * f)
    y[..., :half] = z.real
    y[..., half:rope_dim] = z.imag
    return y


# --------------------------------------------------------------------- RoPE
def pin_rope_identity_at_zero(O):
    x = np.random.default_rng(1).standard_normal(256)
    assert np.array_equal(O.rope(x, 0), x)


def pin_rope_norm_and_tail(O):
    x = np.random.default_rng(2).standard_normal(256)
    for pos in (1, 7, 4095, 262143, 1048575):
        y = O.rope(x, pos)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)
        assert np.array_equal(y[64:], x[64:]), "dims beyond rope_dim must be untouched"
        # each (i, i+32) pair keeps its own length
        assert np.allclose(np.hypot(y[:32], y[32:64]), np.hypot(x[:32], x[32:64]), rtol=1e-13)


def pin_rope_complex_form(O):
    """Rotate-half pairs, frequency theta^(-2i/64), theta = 1e7: as complex rotations."""
    rng = np.random.default_rng(3)
    for pos in (1, 3, 1000, 262144, 1048575):
        x = rng.standard_normal(256)
        assert np.allclose(O.rope(x, pos), _rope_complex(x, pos), rtol=0, atol=1e-9), pos


def pin_rope_relative(O):
    """(R_m q).(R_n k) depends only on m - n."""
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(256), rng.standard_normal(256)
    for m, n in ((5, 2), (1000, 10), (700000, 699990)):
        a = O.rope(q, m) @ O.rope(k, n)
        b = O.rope(q, m - n) @ k
        assert abs(a - b) < 1e-8 * (abs(b) + 1), (m, n, a, b)


# ------------------------------------------------------------------- scores
def pin_token_score_closed_form(O):
    """q_h = a_h e_0, k = b e_0: s = sum_h w_h max(0, a_h b) / sqrt(128)."""
    a = np.array([2.0, -3.0, 0.5, 4.0])
    b = 1.5
    w = np.array([0.25, 0.5, 0.125, 0.125])
    q = np.zeros((4, 128)); q[:, 0] = a
    k = np.zeros(128); k[0] = b
    want = sum(w[h] * max(0.0, a[h] * b) for h in range(4)) / SQRT_D
    got = O.token_score(_bf(q), _bf(w), _bf(k))
    assert abs(got - want) < 1e-15, (got, want)
    # the key element other than dim 0 matters too (no dropped dims)
    k2 = k.copy(); k2[127] = 2.0
    q2 = q.copy(); q2[3, 127] = 1.0
    want2 = sum(w[h] * max(0.0, a[h] * b + (2.0 if h == 3 else 0.0)) for h in range(4)) / SQRT_D
    got2 = O.token_score(_bf(q2), _bf(w), _bf(k2))
    assert abs(got2 - want2) < 1e-15, (got2, want2)


def _matrix_scores(q_idx, w, k_idx, r=4):
    """Brute force in matrix form: all token pairs at once, then block max."""
    T = q_idx.shape[0]
    qf, wf, kf = Q.bf16_to_f64(q_idx), Q.bf16_to_f64(w), Q.bf16_to_f64(k_idx)
    dots = np.einsum("thc,jc->thj", qf, kf)                    # [T][4][T]
    s = (wf[:, :, None] * np.maximum(dots, 0.0)).sum(1) / SQRT_D  # [T][T]
    causal = np.tril(np.ones((T, T), dtype=bool))
    s = np.where(causal, s, -np.inf)
    nb = (T + r - 1) // r
    pad = np.full((nb * r, nb * r), -np.inf)
    pad[:T, :T] = s
    S = pad.reshape(nb, r, nb, r).max(axis=(1, 3))
    S[np.triu(np.ones((nb, nb), dtype=bool), 1)] = np.nan
    return S


def pin_block_scores_brute(O):
    for T, seed in ((1, 0), (5, 1), (13, 2), (64, 3), (67, 4)):
        P = Q.PrefillProblem(T=T, seed=seed, n_plant=2)
        q_idx, w, k_idx = P.q_idx(), P.w(), P.k_idx()
        want = _matrix_scores(q_idx, w, k_idx)
        got = O.index_scores(T, q_idx, w, k_idx)
        m = ~np.isnan(want)
        assert np.array_equal(m, ~np.isnan(got)), T
        assert np.allclose(got[m], want[m], rtol=1e-12, atol=1e-14), T


def pin_block_scores_page_formula(O):
    """Block size 1 and constant head weight c: S * sqrt(128) / c is the
    indexer score I_ib = sum_h ReLU(<q_i^h, k_b>) with the block key = the key."""
    import oracle as OR
    P1 = OR.params(block=1, budget=O.P.budget)
    O1 = type(O)(P1, O.L)
    T = 23
    P = Q.PrefillProblem(T=T, seed=5)
    q_idx, k_idx = P.q_idx(), P.k_idx()
    c = 8.0
    w = _bf(np.full((T, 4), c))
    S = O1.index_scores(T, q_idx, w, k_idx)
    qf, kf = Q.bf16_to_f64(q_idx), Q.bf16_to_f64(k_idx)
    I = np.maximum(np.einsum("thc,jc->thj", qf, kf), 0.0).sum(1)   # [T][T]
    for i in range(T):
        for b in range(i + 1):
            assert abs(S[i, b] * SQRT_D / c - I[i, b]) < 1e-10 * (1 + abs(I[i, b])), (i, b)


def pin_identical_keys_block(O):
    """A key block of four identical keys scores the max over query tokens of
    the score against that one key; a block after the query is never scored."""
    T = 16
    P = Q.PrefillProblem(T=T, seed=6)
    q_idx, w, k_idx = P.q_idx(), P.w(), P.k_idx().copy()
    k_idx[4:8] = k_idx[5]
    S = O.index_scores(T, q_idx, w, k_idx)
    for qb in (1, 2, 3):
        want = max(O.token_score(q_idx[t], w[t], k_idx[5]) for t in range(4 * qb, 4 * qb + 4))
        assert abs(S[qb, 1] - want) < 1e-14 * (1 + want)
    # own block: token 4qb sees only key 4qb
    for qb in range(4):
        t0 = 4 * qb
        want = max(O.token_score(q_idx[t], w[t], k_idx[j]) for t in range(t0, t0 + 4) for j in range(t0, t + 1))
        assert abs(S[qb, qb] - want) < 1e-14 * (1 + want)


# ------------------------------------------------------------- YaRN (f4)
def _yarn_oracle(O, factor=4.0):
    import oracle as OR
    return type(O)(OR.params(budget=O.P.budget, yarn_factor=factor), O.L)


def _pair_angles(Oy, pos):
    """Rotation angle of every pair (i, i + 32) at position pos, and the
    radius, read off the image of the unit vectors e_i."""
    ang, rad = np.zeros(32), np.zeros(32)
    for i in range(32):
        x = np.zeros(256)
        x[i] = 1.0
        y = Oy.rope(x, pos)
        ang[i] = math.atan2(y[i + 32], y[i])
        rad[i] = math.hypot(y[i], y[i + 32])
    return ang, rad


def pin_yarn_attention_factor_and_tail(O):
    """The rotated dims are scaled by 0.1 ln s + 1 (s = 4: 1.13863), the other
    192 dims are untouched, for any position."""
    Oy = _yarn_oracle(O)
    m = 0.1 * math.log(4.0) + 1.0
    rng = np.random.default_rng(1)
    for pos in (0, 7, 262143, 1048575):
        x = rng.standard_normal(256)
        y = Oy.rope(x, pos)
        assert abs(np.linalg.norm(y[:64]) - m * np.linalg.norm(x[:64])) < 1e-12 * np.linalg.norm(x[:64])
        assert np.array_equal(y[64:], x[64:])


def pin_yarn_relative_positions(O):
    """<R(x, a), R(y, b)> depends on a - b only, as for plain RoPE."""
    Oy = _yarn_oracle(O)
    rng = np.random.default_rng(2)
    x, y = rng.standard_normal(256), rng.standard_normal(256)
    for a, b, shift in ((5, 3, 1000), (300000, 299000, 700000), (17, 900000, 12345)):
        d0 = Oy.rope(x, a) @ Oy.rope(y, b)
        d1 = Oy.rope(x, a + shift) @ Oy.rope(y, b + shift)
        assert abs(d0 - d1) < 1e-9 * (1 + abs(d0)), (a, b)


def pin_yarn_frequency_regimes(O):
    """Pair 0 (wavelength 2 pi, far shorter than the 262144-token original
    context) keeps its frequency 1; pair 31 (wavelength ~1.3e7 tokens, longer
    than the context) is interpolated to theta^(-31/32) / 4; every pair's
    frequency lies between f_i / 4 and f_i, and its ratio to f_i does not
    increase with i; factor 1 is plain RoPE."""
    Oy = _yarn_oracle(O)
    ang, rad = _pair_angles(Oy, 1)
    f = 1e7 ** (-np.arange(32) / 32.0)
    assert abs(ang[0] - 1.0) < 1e-12
    assert abs(ang[31] - f[31] / 4.0) < 1e-15
    ratio = ang / f
    assert np.all(ratio <= 1.0 + 1e-12) and np.all(ratio >= 0.25 - 1e-12)
    assert np.all(np.diff(ratio) <= 1e-12)
    assert np.any(np.abs(ratio - 1.0) < 1e-12) and np.any(np.abs(ratio - 0.25) < 1e-12)
    O1 = _yarn_oracle(O, factor=1.0)
    x = np.random.default_rng(3).standard_normal(256)
    assert np.array_equal(O1.rope(x, 123456), O.rope(x, 123456))


# ------------------------------------------------ mean-pooled block keys (f2)
def _bf16_rne_exact(x) -> float:
    """Round a rational to the nearest bf16 value (ties to even), by integer
    arithmetic on its exact value (fractions), independent of any float path."""
    from fractions import Fraction
    x = Fraction(x)
    if x == 0:
        return 0.0
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()   # 2^e <= a < 2^(e+2)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    unit = max(e - 7, -133)                 # 8 significant bits; bf16 subnormals below 2^-126
    q = a / Fraction(2) ** unit
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * float(Fraction(n) * Fraction(2) ** unit)


def _mean_pool_scores(q_idx, w, k_idx, r=4):
    """S(qb, kb) with mean-pooled block keys, all in numpy / exact rationals:
    kbar = bf16 of the mean of the block's present keys (mean: exact sum, one
    fp64 division), score = max over the block's tokens."""
    from fractions import Fraction
    T = q_idx.shape[0]
    nb = (T + r - 1) // r
    kf = Q.bf16_to_f64(k_idx)
    kbar = np.zeros((nb, kf.shape[1]))
    for b in range(nb):
        rows = kf[b * r: min(b * r + r, T)]
        n = rows.shape[0]
        for c in range(kf.shape[1]):
            exact_sum = sum(Fraction(float(v)) for v in rows[:, c])
            mean64 = float(exact_sum) / n          # the sum is exact in fp64; one division
            kbar[b, c] = _bf16_rne_exact(mean64)
    qf, wf = Q.bf16_to_f64(q_idx), Q.bf16_to_f64(w)
    dots = np.einsum("thc,bc->thb", qf, kbar)
    s = (wf[:, :, None] * np.maximum(dots, 0.0)).sum(1) / SQRT_D   # [T][nb]
    S = np.full((nb, nb), np.nan)
    for qb in range(nb):
        S[qb, :qb + 1] = s[qb * r: min(qb * r + r, T), :qb + 1].max(axis=0)
    return S


def _mean_pool_oracle(O):
    import oracle as OR
    return type(O)(OR.params(budget=O.P.budget, aggregation=OR.AGG_MEAN_POOL), O.L)


def pin_mean_pool_brute(O):
    """Mean-pooled scores equal an independent brute force (exact rational
    rounding of the block means, numpy dot products), ragged tails included."""
    Om = _mean_pool_oracle(O)
    for T, seed in ((1, 0), (6, 1), (29, 2), (67, 3)):
        P = Q.PrefillProblem(T=T, seed=40 + seed, n_plant=2)
        q_idx, w, k_idx = P.q_idx(), P.w(), P.k_idx()
        want = _mean_pool_scores(q_idx, w, k_idx)
        got = Om.index_scores(T, q_idx, w, k_idx)
        m = ~np.isnan(want)
        assert np.allclose(got[m], want[m], rtol=1e-12, atol=1e-14), T


def pin_mean_pool_relations(O):
    """Closed forms: a block of four identical keys has that key as its mean,
    so its mean-pool score is the token-pair score; keys k, -k, k, -k average
    to 0 and score 0; keys 1, 2, 3, 4 times k average to 2.5 k."""
    Om = _mean_pool_oracle(O)
    T = 24
    P = Q.PrefillProblem(T=T, seed=9)
    q_idx, w, k_idx = P.q_idx(), P.w(), P.k_idx().copy()
    k_idx[4:8] = k_idx[6]
    base = _bf(np.full(128, 0.5, np.float32))
    k_idx[8:12] = np.stack([base, _bf(-Q.bf16_to_f32(base)), base, _bf(-Q.bf16_to_f32(base))])
    unit = _bf(np.full(128, 0.25, np.float32))
    k_idx[12:16] = np.stack([_bf(Q.bf16_to_f32(unit) * m) for m in (1, 2, 3, 4)])
    Sm = Om.index_scores(T, q_idx, w, k_idx)
    Sp = O.index_scores(T, q_idx, w, k_idx)
    for qb in (2, 3, 4, 5):
        assert abs(Sm[qb, 1] - Sp[qb, 1]) < 1e-13 * (1 + Sp[qb, 1]), qb
        assert Sm[qb, 2] == 0.0, qb
        qf, wf = Q.bf16_to_f64(q_idx), Q.bf16_to_f64(w)
        if qb >= 3:
            kb3 = np.full(128, 0.625)
            want = max((wf[t] * np.maximum(qf[t] @ kb3, 0.0)).sum() / SQRT_D for t in range(4 * qb, 4 * qb + 4))
            assert abs(Sm[qb, 3] - want) < 1e-12 * (1 + want), qb


def pin_bf16_rounding_of_means(O):
    """The block mean is rounded to bf16 once, to nearest even: a mean exactly
    half-way between two bf16 values goes to the even one, and one just above
    half-way goes up."""
    Om = _mean_pool_oracle(O)
    T = 8
    P = Q.PrefillProblem(T=T, seed=12)
    q_idx, w = P.q_idx(), P.w()
    q_idx[4:8] = 0
    q_idx[4:8, 0, 0] = _bf(np.float32(1.0))       # score = w0 * ReLU(kbar[0]) / sqrt(128)
    k_idx = np.zeros((T, 128), np.uint16)
    # 1 + 2^-8 is half-way between 1 and 1 + 2^-7: keys 1, 1, 1 + 2^-7, 1 + 2^-7 -> ties to even = 1
    a, b = np.float32(1.0), np.float32(1.0 + 2 ** -7)
    k_idx[0:4, 0] = _bf(np.array([a, a, b, b]))
    S = Om.index_scores(T, q_idx, w, k_idx)
    wf = Q.bf16_to_f64(w)
    assert abs(S[1, 0] - max(wf[t, 0] for t in range(4, 8)) * 1.0 / SQRT_D) < 1e-15
    # keys 1, 1, 1 + 2^-7, 1 + 2^-6: mean 1 + 3 * 2^-9 (above half-way) -> 1 + 2^-7
    k_idx[3, 0] = _bf(np.float32(1.0 + 2 ** -6))
    S = Om.index_scores(T, q_idx, w, k_idx)
    assert abs(S[1, 0] - max(wf[t, 0] for t in range(4, 8)) * (1.0 + 2 ** -7) / SQRT_D) < 1e-15


def _rope_exact_rounded(x, pos, exact):
    """Complex-form RoPE of a 128-dim indexer vector at pos (dims 0..63),
    rounded to bf16 by exact rationals unless exact."""
    y = _rope_complex(x, pos)
    return y if exact else np.array([_bf16_rne_exact(v) for v in y])


def _mean_pool_rope_scores(q_idx, w, k_idx, pos0, exact, r=4):
    """Brute force of the block-start-position reading: block means (rounded
    to bf16 unless exact) rotated at 4b + pos0 and queries rotated at t + pos0
    (each rounded to bf16 unless exact), numpy dot products."""
    from fractions import Fraction
    T = q_idx.shape[0]
    nb = (T + r - 1) // r
    kf = Q.bf16_to_f64(k_idx)
    kbar = np.zeros((nb, kf.shape[1]))
    for b in range(nb):
        rows = kf[b * r: min(b * r + r, T)]
        mean = np.array([float(sum(Fraction(float(v)) for v in rows[:, c])) / rows.shape[0]
                         for c in range(kf.shape[1])])
        if not exact:
            mean = np.array([_bf16_rne_exact(v) for v in mean])
        kbar[b] = _rope_exact_rounded(mean, pos0 + r * b, exact)
    qf = Q.bf16_to_f64(q_idx)
    qr = np.stack([[_rope_exact_rounded(qf[t, h], pos0 + t, exact) for h in range(qf.shape[1])] for t in range(T)])
    wf = Q.bf16_to_f64(w)
    dots = np.einsum("thc,bc->thb", qr, kbar)
    s = (wf[:, :, None] * np.maximum(dots, 0.0)).sum(1) / SQRT_D
    S = np.full((nb, nb), np.nan)
    for qb in range(nb):
        S[qb, :qb + 1] = s[qb * r: min(qb * r + r, T), :qb + 1].max(axis=0)
    return S


def _idx_rope_oracle(O, exact=0, pos0=0):
    import oracle as OR
    return type(O)(OR.params(budget=O.P.budget, aggregation=OR.AGG_MEAN_POOL, idx_rope=1, idx_exact=exact,
                             idx_pos0=pos0), O.L)


def pin_idx_rope_brute(O):
    """Mean pooling with the block-start position ([PT] §QSA): scores equal a
    brute force on complex-form RoPE (key of block b at 4b, query of token t
    at t, both offset by pos0), with and without the bf16 rounding of the
    operands, ragged tails included."""
    for T, seed, pos0 in ((7, 0, 0), (29, 1, 0), (41, 2, 1000), (13, 3, 262140)):
        P = Q.PrefillProblem(T=T, seed=60 + seed, n_plant=2)
        q_idx, w, k_idx = P.q_idx(), P.w(), P.k_idx()
        for exact in (0, 1):
            want = _mean_pool_rope_scores(q_idx, w, k_idx, pos0, exact)
            got = _idx_rope_oracle(O, exact, pos0).index_scores(T, q_idx, w, k_idx)
            m = ~np.isnan(want)
            assert np.allclose(got[m], want[m], rtol=1e-9, atol=1e-12), (T, exact)


def pin_idx_rope_relative_positions(O):
    """With exact operands the scores depend on positions only through the
    distance between the query token and the key block's start: a common
    offset of every position leaves them unchanged, while the rotation itself
    changes them (a key block scored at distance 0 and at distance 40 differ)."""
    T = 48
    P = Q.PrefillProblem(T=T, seed=71, n_plant=3)
    q_idx, w, k_idx = P.q_idx(), P.w(), P.k_idx()
    S0 = _idx_rope_oracle(O, 1, 0).index_scores(T, q_idx, w, k_idx)
    S1 = _idx_rope_oracle(O, 1, 123457).index_scores(T, q_idx, w, k_idx)
    m = ~np.isnan(S0)
    assert np.allclose(S0[m], S1[m], rtol=1e-8, atol=1e-12)
    Sp = _mean_pool_oracle(O).index_scores(T, q_idx, w, k_idx)
    assert not np.allclose(S0[m], Sp[m], rtol=1e-3), "the rotation must change the scores"


# ---------------------------------------------------------------- selection
def _select_lexsort(S_row, qb, budget):
    if qb + 1 <= budget:
        return np.arange(qb + 1)
    cand = np.arange(qb - 1)
    order = np.lexsort((cand, -S_row[:qb - 1]))      # score desc, index asc
    top = cand[order[:budget - 2]]
    return np.sort(np.concatenate([top, [qb - 1, qb]]))


def pin_select_vs_lexsort(O):
    rng = np.random.default_rng(7)
    B = O.P.budget
    for qb in (0, 1, B - 2, B - 1, B, B + 1, B + 5, 3 * B + 7):
        S = rng.random(qb + 1).round(2)            # many ties
        sel, cnt = O.select(qb, S)
        want = _select_lexsort(S, qb, B)
        assert cnt == len(want), (qb, cnt)
        assert np.array_equal(sel[:cnt], want), qb
        assert (sel[cnt:] == -1).all()


def pin_select_invariants(O):
    rng = np.random.default_rng(8)
    B = O.P.budget
    for qb in (B - 1, B, 2 * B + 3):
        S = rng.random(qb + 1)
        sel, cnt = O.select(qb, S)
        s = sel[:cnt]
        assert cnt == min(B, qb + 1)
        assert np.all(np.diff(s) > 0)
        assert qb in s and (qb - 1 in s or qb == 0)
        if qb + 1 > B:
            free_sel = [b for b in s if b < qb - 1]
            unsel = np.setdiff1d(np.arange(qb - 1), s)
            assert min(S[free_sel]) >= max(S[unsel])
    # all scores equal: the lowest indices win
    qb = 3 * B
    sel, cnt = O.select(qb, np.zeros(qb + 1))
    assert np.array_equal(sel[:cnt], np.concatenate([np.arange(B - 2), [qb - 1, qb]]))


# ---------------------------------------------------------------- attention
def _dense_causal_sdpa(q, k, v, pos0=0):
    """Dense causal GQA attention via torch's SDPA in fp64 on complex-form RoPE."""
    T = q.shape[0]
    qf = np.stack([_rope_complex(Q.bf16_to_f64(q[t]), pos0 + t) for t in range(T)])   # [T][24][256]
    kf = np.stack([_rope_complex(Q.bf16_to_f64(k[t]), pos0 + t) for t in range(T)])   # [T][2][256]
    vf = Q.bf16_to_f64(v)
    qt = torch.from_numpy(qf).permute(1, 0, 2)[None]
    kt = torch.from_numpy(kf).permute(1, 0, 2).repeat_interleave(12, dim=0)[None]
    vt = torch.from_numpy(vf).permute(1, 0, 2).repeat_interleave(12, dim=0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    logits = torch.einsum("bhtc,bhjc->bhtj", qt, kt) / 16.0
    logits = logits.masked_fill(~torch.tril(torch.ones(T, T, dtype=torch.bool)), float("-inf"))
    lse = torch.logsumexp(logits, dim=-1)
    return o[0].permute(1, 0, 2).numpy(), lse[0].permute(1, 0).numpy()


def pin_attention_dense_when_budget_covers(O):
    """Budget >= number of blocks: QSA is dense causal attention."""
    import oracle as OR
    for T, pos0 in ((37, 0), (64, 0), (21, 1000)):
        Ob = type(O)(OR.params(budget=64), O.L)
        P = Q.PrefillProblem(T=T, seed=9, n_plant=3)
        h = P.host()
        sel, cnt, out, lse = Ob.prefill_blocks(T, h["q"], h["k"], h["v"], h["q_idx"], h["w"], h["k_idx"], pos0=pos0)
        want_o, want_l = _dense_causal_sdpa(h["q"], h["k"], h["v"], pos0)
        assert np.allclose(out[:T], want_o, rtol=1e-10, atol=1e-12), T
        assert np.allclose(lse[:T], want_l, rtol=1e-10, atol=1e-12), T


def pin_attend_gathered_dense(O):
    """The explicit-key-list entry: every token of a short sequence over all
    its keys (given in shuffled order, later keys included so that the causal
    skip matters) equals dense causal GQA attention (torch SDPA, fp64)."""
    T = 23
    P = Q.PrefillProblem(T=T, seed=41, n_plant=0)
    h = P.host()
    want, want_lse = _dense_causal_sdpa(h["q"], h["k"], h["v"])
    perm = np.random.default_rng(5).permutation(T)
    for t in (0, 1, 7, 22):
        out, lse = O.attend_gathered(t, h["q"][t], perm, h["k"][perm], h["v"][perm])
        assert np.abs(out - want[t]).max() < 1e-10, t
        assert np.abs(lse - want_lse[t]).max() < 1e-10, t


def pin_attention_constant_v_and_single_key(O):
    T = 12
    P = Q.PrefillProblem(T=T, seed=10)
    q, k = P.q(), P.k()
    vv = np.zeros((T, 2, 256), dtype=np.float32)
    vv[:, 0, :] = 0.75
    vv[:, 1, :] = np.linspace(-2, 2, 256, dtype=np.float32).round(2)
    v = Q.f32_to_bf16(vv)
    sel = np.tile(np.arange(O.P.budget, dtype=np.int32), (3, 1))
    sel[:, 3:] = -1
    cnt = np.full(3, 3, np.int32)
    out, lse = O.attend_blocks(T, q, k, v, np.arange(3), sel, cnt)
    vf = Q.bf16_to_f64(v)
    assert np.allclose(out[:, :12, :], vf[0, 0], atol=1e-12)
    assert np.allclose(out[:, 12:, :], vf[0, 1], atol=1e-12)
    # token 0 has a single key: out = v_0, lse = its logit
    vr = P.v()
    out, lse = O.attend_blocks(T, q, k, vr, np.arange(1), sel[:1], cnt[:1])
    vf = Q.bf16_to_f64(vr)
    for h in range(24):
        assert np.allclose(out[0, h], vf[0, h // 12], atol=1e-13)
        logit = (Q.bf16_to_f64(q[0, h]) @ Q.bf16_to_f64(k[0, h // 12])) / 16.0   # RoPE is the identity at 0
        assert abs(lse[0, h] - logit) < 1e-12


def pin_attention_respects_selection(O):
    """Keys outside the selected blocks do not influence the output."""
    T = 32
    P = Q.PrefillProblem(T=T, seed=11)
    q, k, v = P.q(), P.k(), P.v()
    qb = 7
    sel = np.full((1, O.P.budget), -1, np.int32)
    sel[0, :3] = [1, 4, 7]
    cnt = np.array([3], np.int32)
    out1, _ = O.attend_blocks(T, q, k, v, [qb], sel, cnt)
    k2, v2 = k.copy(), v.copy()
    for b in (0, 2, 3, 5, 6):
        k2[4 * b: 4 * b + 4] = 0x3F80
        v2[4 * b: 4 * b + 4] = 0x4000
    out2, _ = O.attend_blocks(T, q, k2, v2, [qb], sel, cnt)
    assert np.array_equal(out1, out2)
    # and the keys that are selected do
    v3 = v.copy(); v3[4 * 4] = 0x4000
    out3, _ = O.attend_blocks(T, q, k, v3, [qb], sel, cnt)
    assert not np.array_equal(out1, out3)


# ------------------------------------------------------------------- decode
def pin_decode_equals_prefill_last(O):
    """Decode of token L over caches (keys rotated then rounded to bf16) gives
    prefill's token-L output, up to that rounding; the selection is exact."""
    import oracle as OR
    for L in (40, 41, 43, 70):
        Ob = type(O)(OR.params(budget=8), O.L)
        T = L + 1
        P = Q.PrefillProblem(T=T, seed=12 + L, n_plant=2)
        h = P.host()
        qb = L // 4
        sel, cnt, out, lse = Ob.prefill_blocks(T, h["q"], h["k"], h["v"], h["q_idx"], h["w"], h["k_idx"], [qb])
        kf = np.stack([_rope_complex(Q.bf16_to_f64(h["k"][t]), t) for t in range(L)])
        k_cache = Q.f32_to_bf16(kf.astype(np.float32))
        t0 = qb * 4
        dsel, dcnt, dout, dlse = Ob.decode(L, k_cache, h["v"][:L], h["k_idx"][:L], h["q_idx"][t0:L], h["w"][t0:L],
                                           h["q"][L], h["k"][L], h["v"][L], h["q_idx"][L], h["k_idx"][L], h["w"][L])
        assert dcnt == cnt[0] and np.array_equal(dsel, sel[0]), L
        i = L - t0
        assert np.abs(dout - out[i]).max() < 2e-2
        assert np.linalg.norm(dout - out[i]) < 5e-3 * np.linalg.norm(out[i])



# ---------------------------------------------------------------- top-k reuse
def pin_reuse_selection_examples(O):
    """The reused row joined with the token's forced blocks, worked by hand
    from the rule (qb - 1 and qb always attended, the rest kept as given)."""
    cases = [(5, [0, 2, 3], [0, 2, 3, 4, 5]),          # row of block 3 reused in block 5
             (5, [1, 4, 5], [1, 4, 5]),                # own row: unchanged
             (4, [0, 2, 3, 4], [0, 2, 3, 4]),
             (4, [1, 2, 3], [1, 2, 3, 4]),             # row of block 3 reused in block 4
             (0, [], [0]),
             (0, [0], [0]),
             (1, [0], [0, 1]),
             (7, [0, 1, 2, 3], [0, 1, 2, 3, 6, 7]),
             (9, [8], [8, 9])]
    for qb, row, want in cases:
        got, n = O.reuse_selection(qb, np.array(row, np.int32), len(row))
        assert n == len(want) and list(got) == want, (qb, row, list(got))
    for qb, row in ((3, [0, 4]), (2, [-1, 2])):
        try:
            O.reuse_selection(qb, np.array(row, np.int32), len(row))
        except ValueError:
            continue
        raise AssertionError(f"non-causal row accepted: qb={qb} {row}")


def pin_reuse_same_block_is_plain_decode(O):
    """Reusing the row that the decode itself selects, at the same token or a
    later token of the same query block (stage 2 already forced qb - 1, qb),
    attends the same blocks: identical outputs at the same token."""
    import oracle as OR
    Ob = type(O)(OR.params(budget=6), O.L)
    for L in (41, 44, 70):
        P = Q.PrefillProblem(T=L + 1, seed=30 + L, n_plant=2)
        h = P.host()
        qb = L // 4
        kf = np.stack([_rope_complex(Q.bf16_to_f64(h["k"][t]), t) for t in range(L)])
        k_cache = Q.f32_to_bf16(kf.astype(np.float32))
        t0 = 4 * qb
        args = (L, k_cache, h["v"][:L], h["k_idx"][:L], h["q_idx"][t0:L], h["w"][t0:L], h["q"][L], h["k"][L],
                h["v"][L], h["q_idx"][L], h["k_idx"][L], h["w"][L])
        sel, cnt, out, lse = Ob.decode(*args)
        rsel, rn, rout, rlse = Ob.decode_reuse(*args, sel_in=sel, cnt_in=cnt)
        assert rn == cnt and np.array_equal(rsel, sel[:cnt]), L
        assert np.array_equal(rout, out) and np.array_equal(rlse, lse), L
        if L % 4 < 3:
            again, n2 = Ob.reuse_selection((L + 1) // 4, sel, cnt)
            assert n2 == cnt and np.array_equal(again, sel[:cnt])


def pin_reuse_decode_brute(O):
    """A draft token one block past the reused row: numpy softmax over exactly
    the keys of the row's blocks and of qb - 1, qb up to the token."""
    import oracle as OR
    Ob = type(O)(OR.params(budget=4), O.L)
    L = 50                                  # qb = 12
    P = Q.PrefillProblem(T=L + 1, seed=77, n_plant=1)
    h = P.host()
    qb = L // 4
    kf = np.stack([_rope_complex(Q.bf16_to_f64(h["k"][t]), t) for t in range(L)])
    k_cache = Q.f32_to_bf16(kf.astype(np.float32))
    row = np.array([2, 7, 10, 11], np.int32)   # a budget-4 row of block 11
    t0 = 4 * qb
    _, n, out, lse = Ob.decode_reuse(L, k_cache, h["v"][:L], h["k_idx"][:L], h["q_idx"][t0:L], h["w"][t0:L],
                                     h["q"][L], h["k"][L], h["v"][L], h["q_idx"][L], h["k_idx"][L], h["w"][L],
                                     sel_in=row, cnt_in=4)
    assert n == 5
    js = [j for b in (2, 7, 10, 11, 12) for j in range(4 * b, 4 * b + 4) if j <= L]
    keys = np.concatenate([Q.bf16_to_f64(k_cache), _rope_complex(Q.bf16_to_f64(h["k"][L]), L)[None]])
    vals = Q.bf16_to_f64(h["v"][:L + 1])
    for hh in range(24):
        g = hh // 12
        q = _rope_complex(Q.bf16_to_f64(h["q"][L, hh]), L)
        lg = np.array([q @ keys[j, g] for j in js]) / 16.0
        m = lg.max()
        e = np.exp(lg - m)
        want = (e[:, None] * np.stack([vals[j, g] for j in js])).sum(0) / e.sum()
        assert np.allclose(out[hh], want, rtol=1e-11, atol=1e-12), hh
        assert abs(lse[hh] - (m + np.log(e.sum()))) < 1e-11


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
