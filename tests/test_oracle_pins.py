"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test names the passage it pins.  None of them re-derives a result with the oracle's own
formula: they use hand-derived values, closed forms, an independent textbook Babai
(Gram-Schmidt on a tall basis), brute-force enumeration, or invariants, chosen so that a dropped
term, a wrong sign or index, or a transposed operand in the oracle fails one of them.
"""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import gptq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(T, n, m, seed, decay=0.8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, n)) * (np.arange(1, n + 1) ** -decay)
    x = x @ np.linalg.qr(rng.standard_normal((n, n)))[0].T
    w = 0.02 * rng.standard_normal((m, n))
    return w, x


# --------------------------------------------------------------------------------------------
# hand-derived two-column example (tests/golden/gptq_two_column_hand.json)
# --------------------------------------------------------------------------------------------

def test_golden_two_column_forward_reverse_bound():
    g = json.load(open(os.path.join(GOLDEN, "gptq_two_column_hand.json")))
    hd = np.array(g["Hd"])
    w = np.array([g["w"]])
    s, z = O.minmax_grid(w, g["bits"])
    assert s[0] == pytest.approx(g["grid"]["scale"], rel=1e-15)
    assert z[0] == g["grid"]["zero"]
    U = O.hinv_upper_factor(hd)
    np.testing.assert_allclose(U, np.array(g["U"]), rtol=1e-13, atol=1e-15)
    f = O.gptq_columns(w, U, g["bits"])
    assert f["codes"][0].tolist() == g["forward_codes"]
    np.testing.assert_allclose(f["Q"][0], g["forward_Q"], rtol=1e-13)
    assert O.quadratic_loss(w, f["Q"], hd) == pytest.approx(g["forward_loss_damped"], rel=1e-12)
    assert float(np.sum(f["e"] ** 2)) == pytest.approx(g["forward_loss_damped"], rel=1e-12)
    L = np.linalg.cholesky(hd)
    np.testing.assert_allclose(L, np.array(g["L"]), rtol=1e-13, atol=1e-15)
    r = O.babai_sic_reverse(w, L, g["bits"], clip=False)
    assert r["codes"][0].tolist() == g["reverse_codes"]
    assert O.quadratic_loss(w, r["Q"], hd) == pytest.approx(g["reverse_loss_damped"], rel=1e-12)
    bound = O.babai_bound(np.full((1, 2), g["grid"]["scale"]), np.diag(L) ** 2)
    assert bound == pytest.approx(g["reverse_bound"], rel=1e-12)


def test_golden_brute_force_minimum():
    g = json.load(open(os.path.join(GOLDEN, "gptq_two_column_hand.json")))
    hd = np.array(g["Hd"])
    w = np.array([g["w"]])
    best = min(O.quadratic_loss(w, np.array([[0.15 * a, 0.15 * b]]), hd)
               for a in range(4) for b in range(4))
    assert best == pytest.approx(g["brute_force_min_loss"], rel=1e-12)


# --------------------------------------------------------------------------------------------
# Hessian, dead features, damping, factor
# --------------------------------------------------------------------------------------------

def test_loss_identity_pins_hessian_convention():
    """||(W-Q) X^T||^2 = tr(D (X^T X) D^T) = tr(D H D^T)/2 (GEOM 2.1; H = 2 X^T X).

    X is T x n with T != n, so a transposed X, a missing factor 2 or a D^T H D slip fails."""
    w, x = _rand_problem(T=37, n=9, m=5, seed=1)
    q = w + 0.01 * np.random.default_rng(2).standard_normal(w.shape)
    direct = sum(float(np.dot(w[r] - q[r], x[t]) ** 2) for r in range(5) for t in range(37))
    assert O.proxy_loss(w, q, x) == pytest.approx(direct, rel=1e-12)
    H = O.hessian(x)
    assert H.shape == (9, 9)
    assert 0.5 * O.quadratic_loss(w, q, H) == pytest.approx(direct, rel=1e-12)


def test_dead_features_then_damping_hand_values():
    """Dead feature erasure (WaterSIC, additional techniques) before relative damping."""
    H = np.array([[0.0, 0.0, 0.0], [0.0, 2.0, 0.5], [0.0, 0.5, 4.0]])
    W = np.array([[1.0, 2.0, 3.0], [-1.0, -2.0, -3.0]])
    h, w, dead = O.fix_dead_features(H, W)
    assert dead.tolist() == [True, False, False]
    assert h[0, 0] == 1.0 and h[1, 2] == 0.5
    assert w[:, 0].tolist() == [0.0, 0.0] and w[:, 1:].tolist() == [[2.0, 3.0], [-2.0, -3.0]]
    hd, delta = O.dampen(h, 0.01)
    assert delta == pytest.approx(0.01 * 7.0 / 3.0, rel=1e-15)
    np.testing.assert_allclose(np.diag(hd), [1.0 + 0.07 / 3, 2.0 + 0.07 / 3, 4.0 + 0.07 / 3])
    assert hd[1, 2] == 0.5 and hd[2, 1] == 0.5


def test_hinv_factor_closed_form():
    """U upper, positive diagonal, U^T U H_d = I (the defining property of GPTQ's factor)."""
    _, x = _rand_problem(T=40, n=24, m=1, seed=3)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    U = O.hinv_upper_factor(hd)
    assert np.all(np.tril(U, -1) == 0.0)
    assert np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ hd, np.eye(24), atol=1e-9)


def test_hinv_factor_rejects_indefinite():
    with pytest.raises(np.linalg.LinAlgError):
        O.hinv_upper_factor(np.array([[1.0, 2.0], [2.0, 1.0]]))


# --------------------------------------------------------------------------------------------
# grid
# --------------------------------------------------------------------------------------------

def test_minmax_grid_hand_values():
    w = np.array([[-0.3, 0.6], [0.2, 0.5], [0.0, 0.0], [-0.4, -0.1]])
    s, z = O.minmax_grid(w, 2)
    np.testing.assert_allclose(s, [0.3, 0.5 / 3, 2.0 / 3, 0.4 / 3], rtol=1e-15)
    # -lo/s: 1; 0; 1.5 -> 2 (half to even); 3
    assert z.tolist() == [1.0, 0.0, 2.0, 3.0]


def test_clipfree_grid_reduces_to_minmax_at_alpha_one_and_widens():
    rng = np.random.default_rng(4)
    w = rng.standard_normal((50, 16)) * 0.02
    s1, z1 = O.minmax_grid(w, 3)
    s2, z2 = O.clipfree_grid(w, 3, np.ones(50))
    np.testing.assert_allclose(s2, s1, rtol=1e-14)
    assert np.array_equal(z1, z2)
    s3, z3 = O.clipfree_grid(w, 3, np.full(50, 2.0))
    np.testing.assert_allclose(s3, 2 * s1, rtol=1e-14)
    # the widened range still maps [lo, hi] inside the code range
    lo = np.minimum(w.min(1), 0)
    hi = np.maximum(w.max(1), 0)
    assert np.all(np.rint(lo / s3) + z3 >= 0) and np.all(np.rint(hi / s3) + z3 <= 7)


def test_clipfree_grid_centred_zero_point_hand_values():
    """The clip-free grid centres the row's range [lo, hi] on the code range: with the widened
    step s = alpha (hi - lo) / (2^b - 1), z = rint((2^b - 1)/2 - (hi + lo)/(2 s)) ("The Geometry
    of LLM Quantization", section 2.3, no-clipping setting: one uniform grid per row, wide
    enough that nothing clips).  Rows a, b and e are chosen so that the uncentred zero point
    rint(-lo / s) differs from the centred one."""
    w2 = np.array([[0.25, 1.0],     # a: lo 0,  hi 1
                   [-1.0, -0.5],    # b: lo -1, hi 0
                   [-0.3, 0.5],     # c: lo -0.3, hi 0.5
                   [0.0, 0.0]])     # d: flat row -> [lo, hi] = [-1, 1]
    alpha = np.array([2.0, 1.25, 2.0, 1.25])
    s, z = O.clipfree_grid(w2, 2, alpha)
    # a: s = 2 * 1 / 3;       z = rint(1.5 - 1 / (4/3))       = rint(0.75)   = 1  (rint(-lo/s) = 0)
    # b: s = 1.25 * 1 / 3;    z = rint(1.5 + 1 / (2.5/3))     = rint(2.7)    = 3  (rint(2.4) = 2)
    # c: s = 2 * 0.8 / 3;     z = rint(1.5 - 0.2 / (3.2/3))   = rint(1.3125) = 1
    # d: s = 1.25 * 2 / 3;    z = rint(1.5 - 0)               = 2 (half to even)
    np.testing.assert_allclose(s, [2.0 / 3, 1.25 / 3, 1.6 / 3, 2.5 / 3], rtol=1e-15)
    assert z.tolist() == [1.0, 3.0, 1.0, 2.0]
    # e: 3 bits, lo 0, hi 0.7, alpha 2: s = 1.4 / 7 = 0.2; z = rint(3.5 - 0.7 / 0.4) = rint(1.75) = 2
    s3, z3 = O.clipfree_grid(np.array([[0.1, 0.7]]), 3, np.array([2.0]))
    np.testing.assert_allclose(s3, [0.2], rtol=1e-15)
    assert z3.tolist() == [2.0]


# --------------------------------------------------------------------------------------------
# column loop: special cases, independent Babai, brute force, invariants
# --------------------------------------------------------------------------------------------

def _rtn(w, s, z, maxq):
    return np.clip(np.rint(w / s[:, None]) + z[:, None], 0, maxq)


@pytest.mark.parametrize("group", [0, 4])
def test_diagonal_hessian_gptq_equals_rtn(group):
    """No cross-column coupling => no feedback => GPTQ = round-to-nearest (GEOM 4 baseline)."""
    rng = np.random.default_rng(5)
    w = 0.02 * rng.standard_normal((30, 16))
    hd = np.diag(rng.uniform(0.5, 3.0, 16))
    U = O.hinv_upper_factor(hd)
    res = O.gptq_columns(w, U, 3, group=group)
    if group == 0:
        s, z = O.minmax_grid(w, 3)
        expect = _rtn(w, s, z, 7)
    else:
        expect = np.concatenate([_rtn(w[:, k:k + 4], *O.minmax_grid(w[:, k:k + 4], 3), 7)
                                 for k in range(0, 16, 4)], axis=1)
    assert np.array_equal(res["codes"], expect.astype(np.int64))


def _babai_gram_schmidt(Bm, t):
    """Textbook nearest plane: Gram-Schmidt of the basis columns, last basis vector first."""
    d = Bm.shape[1]
    gs = np.zeros_like(Bm)
    for i in range(d):
        v = Bm[:, i].copy()
        for k in range(i):
            v -= (v @ gs[:, k]) / (gs[:, k] @ gs[:, k]) * gs[:, k]
        gs[:, i] = v
    r = t.copy()
    u = np.zeros(d)
    for i in range(d - 1, -1, -1):
        c = np.rint((r @ gs[:, i]) / (gs[:, i] @ gs[:, i]))
        u[i] = c
        r = r - c * Bm[:, i]
    return u


@pytest.mark.parametrize("seed", range(4))
def test_gptq_is_babai_on_tall_factor(seed):
    """GEOM 2.2 Theorem 4 with 2.1 Theorem 1: the oracle's GPTQ (forward, unclamped) equals
    textbook Babai on the basis [sqrt2 X; sqrt(delta) I] diag(s) with basis order reversed; the
    last-to-first SIC form equals Babai in the natural order."""
    n, T, m = 12, 40, 60
    w, x = _rand_problem(T, n, m, seed=10 + seed)
    hd, delta = O.dampen(O.hessian(x), 0.01)
    F = np.vstack([np.sqrt(2.0) * x, np.sqrt(delta) * np.eye(n)])
    U = O.hinv_upper_factor(hd)
    L = np.linalg.cholesky(hd)
    fwd = O.gptq_columns(w, U, 3, clip=False)
    rev = O.babai_sic_reverse(w, L, 3, clip=False)
    s = fwd["scales"][:, 0]
    for r in range(m):
        tgt = F @ w[r]
        u_f = _babai_gram_schmidt((F * s[r])[:, ::-1], tgt)[::-1]
        u_r = _babai_gram_schmidt(F * s[r], tgt)
        assert np.array_equal(fwd["codes"][r] - fwd["zeros"][r, 0], u_f.astype(np.int64))
        assert np.array_equal(rev["codes"][r] - rev["zeros"][r, 0], u_r.astype(np.int64))


def test_extra_propagation_after_projection_changes_nothing():
    """GEOM 2.2: a further GPTQ pass over the Babai result, on the same lattice (grid), leaves
    it unchanged: the result is a lattice point, every error is zero and nothing propagates."""
    w, x = _rand_problem(64, 16, 40, seed=20)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    U = O.hinv_upper_factor(hd)
    first = O.gptq_columns(w, U, 4)
    s, z = first["scales"][:, 0], first["zeros"][:, 0]
    again = O.gptq_columns(first["Q"], U, 4, grid=(s, z))
    assert np.array_equal(again["codes"], first["codes"])
    np.testing.assert_allclose(again["e"], 0.0, atol=1e-15)
    assert np.array_equal(again["zeros"][:, 0], z) and np.allclose(again["scales"][:, 0], s)


@pytest.mark.parametrize("bits,d", [(2, 6), (3, 5), (4, 4)])
def test_brute_force_cvp_lower_bounds_gptq(bits, d):
    """The exact CVP over the clamped code box is <= GPTQ's loss (NP-hard problem, greedy
    heuristic), and GPTQ is never worse than round-to-nearest on these instances' average."""
    w, x = _rand_problem(3 * d, d, 25, seed=30 + bits)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    U = O.hinv_upper_factor(hd)
    res = O.gptq_columns(w, U, bits)
    s, z = res["scales"][:, 0], res["zeros"][:, 0]
    maxq = 2 ** bits - 1
    grid = np.array(list(itertools.product(range(maxq + 1), repeat=d)), dtype=np.float64)
    tot_g = tot_r = 0.0
    for r in range(w.shape[0]):
        qs = s[r] * (grid - z[r])
        dd = w[r][None, :] - qs
        best = np.min(np.einsum("ki,ij,kj->k", dd, hd, dd))
        dg = w[r] - res["Q"][r]
        lg = dg @ hd @ dg
        assert best <= lg * (1 + 1e-12)
        qr = s[r] * (_rtn(w[r:r + 1], s[r:r + 1], z[r:r + 1], maxq)[0] - z[r])
        tot_g += lg
        tot_r += (w[r] - qr) @ hd @ (w[r] - qr)
    assert tot_g <= tot_r


def _gptq_blocked(w, U, bits, group, B):
    w = w.copy()
    m, n = w.shape
    maxq = 2 ** bits - 1
    codes = np.zeros((m, n), dtype=np.int64)
    if group == 0:
        s, z = O.minmax_grid(w, bits)
    for b0 in range(0, n, B):
        b1 = min(b0 + B, n)
        blk = w[:, b0:b1].copy()
        E = np.zeros((m, b1 - b0))
        for jj in range(b1 - b0):
            j = b0 + jj
            if group and j % group == 0:
                s, z = O.minmax_grid(blk[:, jj:jj + group], bits)
            c = np.clip(np.rint(blk[:, jj] / s) + z, 0, maxq)
            e = (blk[:, jj] - s * (c - z)) / U[j, j]
            blk[:, jj + 1:] -= np.outer(e, U[j, j + 1:b1])
            E[:, jj] = e
            codes[:, j] = c
        w[:, b1:] -= E @ U[b0:b1, b1:]
    return codes


@pytest.mark.parametrize("group,B", [(0, 8), (8, 16), (4, 8)])
def test_lazy_block_update_is_exact_reassociation(group, B):
    """Deferring the trailing update to block ends changes no code (exact re-association)."""
    w, x = _rand_problem(96, 40, 50, seed=40 + B)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    U = O.hinv_upper_factor(hd)
    ref = O.gptq_columns(w, U, 3, group=group)["codes"]
    assert np.array_equal(_gptq_blocked(w, U, 3, group, B), ref)


def test_sum_of_scaled_errors_equals_damped_loss():
    """sum_j e_j^2 = tr(D H_d D^T), since D = U^T E."""
    w, x = _rand_problem(80, 32, 30, seed=50)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    U = O.hinv_upper_factor(hd)
    res = O.gptq_columns(w, U, 3, group=8)
    assert float(np.sum(res["e"] ** 2)) == pytest.approx(O.quadratic_loss(w, res["Q"], hd),
                                                         rel=1e-10)


def test_scale_invariance_and_order_reversal():
    """Codes do not change under H -> cH (c > 0, damping is relative); the last-to-first SIC
    form equals the forward GPTQ form run on column-reversed W and J H J."""
    w, x = _rand_problem(70, 24, 40, seed=60)
    h = O.hessian(x)
    hd, _ = O.dampen(h, 0.01)
    hd7, _ = O.dampen(7.0 * h, 0.01)
    a = O.gptq_columns(w, O.hinv_upper_factor(hd), 4, group=8)["codes"]
    b = O.gptq_columns(w, O.hinv_upper_factor(hd7), 4, group=8)["codes"]
    assert np.array_equal(a, b)
    for clip in (True, False):
        sic = O.babai_sic_reverse(w, np.linalg.cholesky(hd), 3, clip=clip)
        fw = O.gptq_columns(w[:, ::-1], O.hinv_upper_factor(hd[::-1, ::-1]), 3, clip=clip)
        assert np.array_equal(sic["codes"], fw["codes"][:, ::-1])
        np.testing.assert_allclose(sic["Q"], fw["Q"][:, ::-1], rtol=0, atol=1e-15)


@pytest.mark.parametrize("reverse", [False, True])
def test_clipfree_loss_within_babai_bound(reverse):
    """GEOM 2.3 Theorem 5: without clipping the damped loss of every row is at most
    (1/4) sum_p s^2 D_pp, D the LDL pivots in the processing order."""
    w, x = _rand_problem(200, 48, 64, seed=70)
    h = O.hessian(x)
    hd, _ = O.dampen(h, 0.01)
    if reverse:
        L = np.linalg.cholesky(hd)
        res = O.babai_sic_reverse(w, L, 3, clip=False)
        piv = np.diag(L) ** 2
    else:
        U = O.hinv_upper_factor(hd)
        res = O.gptq_columns(w, U, 3, clip=False)
        piv = 1.0 / np.diag(U) ** 2
    # pivots must be those of the processing order: LDL of the permuted Hessian
    P = np.arange(48)[::-1] if reverse else np.arange(48)
    hp = hd[np.ix_(P, P)]
    # UDU^T of the permuted matrix (last pivot first): Cholesky of J hp J, read backwards
    Lr = np.linalg.cholesky(hp[::-1, ::-1])
    piv_ldl = (np.diag(Lr) ** 2)[::-1][np.argsort(P)]
    np.testing.assert_allclose(piv, piv_ldl, rtol=1e-10)
    s = res["scales"][:, 0]
    for r in range(64):
        d = w[r] - res["Q"][r]
        assert d @ hd @ d <= 0.25 * s[r] ** 2 * piv.sum() * (1 + 1e-12)


# --------------------------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------------------------

def test_pack_codes_hand_values_and_roundtrip():
    codes = np.array([[1, 2, 3, 15, 0, 7, 8, 9, 10]])
    p = O.pack_codes(codes, 4)
    assert p.shape == (1, 2)
    assert int(p[0, 0]) == (1 | 2 << 4 | 3 << 8 | 15 << 12 | 0 << 16 | 7 << 20 | 8 << 24 | 9 << 28)
    assert int(p[0, 1]) == 10
    # 3-bit codes straddle word boundaries: code 10 sits at bits [30, 33)
    rng = np.random.default_rng(80)
    c3 = rng.integers(0, 8, size=(5, 77))
    p3 = O.pack_codes(c3, 3)
    assert p3.shape == (5, -(-77 * 3 // 32))
    bits = np.unpackbits(p3.view(np.uint8).reshape(5, -1), axis=1, bitorder="little")
    back = np.stack([bits[:, 3 * k] + 2 * bits[:, 3 * k + 1] + 4 * bits[:, 3 * k + 2]
                     for k in range(77)], axis=1)
    assert np.array_equal(back, c3)
    assert bits[:, 3 * 77:].sum() == 0


# --------------------------------------------------------------------------------------------
# the whole layer
# --------------------------------------------------------------------------------------------

def test_quantize_layer_clipfree_ladder_fits_every_row():
    w, x = _rand_problem(300, 32, 80, seed=90)
    out = O.quantize_layer(w, x, bits=2, reverse=True, clip=False)
    assert out["codes"].min() >= 0 and out["codes"].max() <= 3
    assert out["ladder_rounds"] >= 1          # 2-bit unclamped rounding overflows at alpha = 1
    assert np.all(out["alpha"] >= 1.0)
    assert out["loss_damped"] <= out["bound"]


def test_quantize_layer_clipfree_ladder_hand_trace():
    """The scale ladder of the clip-free variant, traced by hand (reading of "per-row step s set
    so that no entry needs clipping", with the scale search of "The Geometry of LLM
    Quantization", section 3, SSQR, as the mechanism): only the rows whose codes leave
    [0, 2^b - 1] are rerun, each time with alpha multiplied by 1.25; a row that fits keeps
    alpha = 1.

    H = [[5, 2], [2, 1]] (det 1, no damping) gives H^-1 = [[1, -2], [-2, 5]] and the upper
    factor U = [[1, -2], [0, 1]]: column 1 receives w1 - e0 U01 = w1 + 2 e0.  2 bits, maxq 3.

    row 0, w = [0.45, 1.0], lo 0, hi 1:
      alpha 1:    s = 1/3,  z = rint(1.5 - 1.5) = 0; c0 = rint(1.35) = 1, e0 = 0.45 - 1/3
                  = 0.11667; w1' = 1.23333, 3.7 -> c1 = 4 > 3: overflow
      alpha 1.25: s = 5/12, z = rint(1.5 - 1.2) = 0; c0 = rint(1.08) = 1, e0 = 0.03333;
                  w1' = 1.06667, 2.56 -> c1 = 3: fits
    row 1, w = [-0.3, 0.1], lo -0.3, hi 0.1:
      alpha 1:    s = 0.4/3, z = rint(1.5 + 0.75) = 2; c0 = rint(-2.25) + 2 = 0, e0 = -0.03333;
                  w1' = 0.03333, 0.25 -> c1 = 0 + 2 = 2: fits
    row 2, w = [-0.35, 1.0], lo -0.35, hi 1, range 1.35:
      alpha 1:      s = 0.45,     z = rint(1.5 - 0.72222) = 1; c0 = rint(-0.77778) + 1 = 0,
                    e0 = 0.1;   w1' = 1.2,   rint(2.66667) + 1 = 4: overflow
      alpha 1.25:   s = 0.5625,   z = rint(1.5 - 0.57778) = 1; c0 = rint(-0.62222) + 1 = 0,
                    e0 = 0.2125; w1' = 1.425, rint(2.53333) + 1 = 4: overflow
      alpha 1.5625: s = 0.703125, z = rint(1.5 - 0.46222) = 1; c0 = rint(-0.49778) + 1 = 1,
                    q0 = 0, e0 = -0.35; w1' = 0.3, rint(0.42667) + 1 = 1: fits
    """
    H = np.array([[5.0, 2.0], [2.0, 1.0]])
    W = np.array([[0.45, 1.0], [-0.3, 0.1], [-0.35, 1.0]])
    np.testing.assert_allclose(O.hinv_upper_factor(H), [[1.0, -2.0], [0.0, 1.0]], atol=1e-14)
    out = O.quantize_layer(W, None, bits=2, clip=False, damp=0.0, H=H)
    np.testing.assert_allclose(out["alpha"], [1.25, 1.0, 1.5625], rtol=1e-15)
    assert out["ladder_rounds"] == 2
    assert out["codes"].tolist() == [[1, 3], [0, 2], [1, 1]]
    assert out["zeros"][:, 0].tolist() == [0.0, 2.0, 1.0]
    np.testing.assert_allclose(out["scales"][:, 0], [1.25 / 3, 0.4 / 3, 0.703125], rtol=1e-14)


def test_quantize_layer_dead_feature_and_loss_bookkeeping():
    w, x = _rand_problem(120, 20, 16, seed=91)
    x[:, 5] = 0.0
    out = O.quantize_layer(w, x, bits=4, group=8)
    assert out["dead"][5] and out["dead"].sum() == 1
    # the dead column quantizes a zeroed weight: q = 0 exactly
    assert np.all(out["Q"][:, 5] == 0.0)
    assert out["loss_proxy"] == pytest.approx(out["loss_proxy_h"], rel=1e-10)
    assert out["sum_e2"] == pytest.approx(out["loss_damped"], rel=1e-10)
    # damped = undamped + delta ||D||^2 (what the GPU reports without X)
    d = (w - out["Q"])
    d[:, 5] = 0.0
    assert out["loss_damped"] == pytest.approx(2 * out["loss_proxy"] + out["delta"] * np.sum(d * d),
                                               rel=1e-10)


def test_quantize_layer_sampled_rows_match_full():
    w, x = _rand_problem(90, 24, 40, seed=92)
    full = O.quantize_layer(w, x, bits=3, group=8)
    rows = [3, 17, 39]
    part = O.quantize_layer(w, x, bits=3, group=8, rows=rows)
    assert np.array_equal(part["codes"], full["codes"][rows])
    np.testing.assert_allclose(part["scales"], full["scales"][rows])


# --------------------------------------------------------------------------------------------
# quantization order (GEOM 2.3: the bound depends on the order; min-pivot and act-order)
# --------------------------------------------------------------------------------------------

def test_act_order_hand_values_and_dead_fix():
    """act-order = descending Hessian diagonal; equal values keep column order; a dead column
    counts with its fixed diagonal 1."""
    assert O.act_order(np.diag([2.0, 5.0, 5.0, 1.0])).tolist() == [1, 2, 0, 3]
    h = np.diag([0.0, 3.0, 1.0, 0.5])
    hf, _, dead = O.fix_dead_features(h, np.zeros((1, 4)))
    assert dead.tolist() == [True, False, False, False]
    assert O.act_order(hf).tolist() == [1, 0, 2, 3]
    res = O.quantize_layer(np.ones((1, 4)) * 0.1, None, 4, H=h, order="act")
    assert res["perm"].tolist() == [1, 0, 2, 3]


def test_min_pivot_two_by_two_closed_form():
    """H = [[a, b], [b, c]], a < c: eliminating column 0 first gives D = (a, c - b^2/a), whose
    sum is below the other order's a + c - b^2/c; column 0 is then decided last, and in the
    processing order (1, 0) the pivots are var(x1 | x0) = c - b^2/a and a."""
    a, b, c = 2.0, 1.5, 5.0
    h = np.array([[a, b], [b, c]])
    perm = O.min_pivot_order(h)
    assert perm.tolist() == [1, 0]
    U = O.hinv_upper_factor(h[np.ix_(perm, perm)])
    np.testing.assert_allclose(1.0 / np.diag(U) ** 2, [c - b * b / a, a], rtol=1e-14)
    assert (c - b * b / a) + a < (a - b * b / c) + c


def test_min_pivot_greedy_by_conditional_variances():
    """Each elimination step takes the remaining column of smallest variance given the columns
    eliminated before it, computed here from inverses of principal submatrices (no Schur
    updates); the factor of the permuted Hessian has exactly those pivots, last first."""
    w, x = _rand_problem(30, 7, 1, seed=91)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    perm = O.min_pivot_order(hd)
    elim = perm[::-1].tolist()
    chosen = []
    for k in range(7):
        E = elim[:k]
        var = {}
        for i in range(7):
            if i in E:
                continue
            idx = E + [i]
            var[i] = 1.0 / np.linalg.inv(hd[np.ix_(idx, idx)])[-1, -1]
        best = min(var, key=lambda i: (var[i], i))
        assert elim[k] == best
        chosen.append(var[best])
    U = O.hinv_upper_factor(hd[np.ix_(perm, perm)])
    np.testing.assert_allclose(1.0 / np.diag(U) ** 2, chosen[::-1], rtol=1e-10)
    # the pivots' product is det(H_d) in every order
    np.testing.assert_allclose(np.sum(np.log(chosen)), np.linalg.slogdet(hd)[1], rtol=1e-12)


@pytest.mark.parametrize("kind", ["act", "min_pivot", "random"])
def test_ordered_gptq_is_babai_in_that_order(kind):
    """GEOM 2.2 Theorem 4 with an order T: GPTQ over the columns in processing order equals
    textbook Babai on the tall basis [sqrt2 X; sqrt(delta) I] diag(s) with the basis columns in
    the reverse of that order; codes come back in the original column positions."""
    n, T, m = 10, 40, 40
    w, x = _rand_problem(T, n, m, seed=95)
    order = np.random.default_rng(3).permutation(n) if kind == "random" else kind
    res = O.quantize_layer(w, x, 3, clip=False, order=order)
    perm = res["perm"]
    if kind != "random":
        assert sorted(perm.tolist()) != perm.tolist() or kind == "act"
    F = np.vstack([np.sqrt(2.0) * x, np.sqrt(res["delta"]) * np.eye(n)])
    for r in range(m):
        s = res["scales"][r, 0]
        u = _babai_gram_schmidt((F * s)[:, perm[::-1]], F @ w[r])
        expect = np.empty(n, dtype=np.int64)
        expect[perm[::-1]] = u.astype(np.int64)
        assert np.array_equal(res["codes"][r] - int(res["zeros"][r, 0]), expect)


def test_ordered_groups_cover_processing_order_on_diagonal_hessian():
    """Diagonal H: no feedback, so GPTQ in any order is round-to-nearest; with groups the grid
    of group g comes from the original weights of the columns processed g-th (reading: groups
    follow the processing order)."""
    rng = np.random.default_rng(97)
    n, m, g = 12, 9, 4
    d = rng.uniform(0.5, 3.0, n)
    w = 0.02 * rng.standard_normal((m, n))
    res = O.quantize_layer(w, None, 3, group=g, H=np.diag(d), order="act")
    perm = np.argsort(-d, kind="stable")
    assert np.array_equal(res["perm"], perm)
    for k in range(n // g):
        cols = perm[k * g:(k + 1) * g]
        lo = np.minimum(w[:, cols].min(axis=1), 0.0)
        hi = np.maximum(w[:, cols].max(axis=1), 0.0)
        s = (hi - lo) / 7.0
        z = np.rint(-lo / s)
        np.testing.assert_array_equal(res["scales"][:, k], s)
        code = np.clip(np.rint(w[:, cols] / s[:, None]) + z[:, None], 0, 7)
        np.testing.assert_array_equal(res["codes"][:, cols], code)


@pytest.mark.parametrize("order", ["act", "min_pivot"])
def test_clipfree_bound_holds_in_every_order(order):
    """GEOM 2.3 Theorem 5 for the permuted Hessian: the clip-free damped loss of the whole layer
    stays below (1/4) sum s^2 D in that order's pivots."""
    w, x = _rand_problem(200, 32, 48, seed=99)
    res = O.quantize_layer(w, x, 3, clip=False, order=order)
    assert res["loss_damped"] <= res["bound"] * (1 + 1e-12)


def test_identity_and_reversal_orders_match_the_flags():
    """order = identity is the forward path; order = reversed columns (per-row grid) gives the
    codes of the last-to-first SIC form."""
    w, x = _rand_problem(80, 16, 20, seed=101)
    nat = O.quantize_layer(w, x, 4, group=8)
    idn = O.quantize_layer(w, x, 4, group=8, order=np.arange(16))
    assert np.array_equal(nat["codes"], idn["codes"])
    rev = O.quantize_layer(w, x, 3, reverse=True)
    prm = O.quantize_layer(w, x, 3, order=np.arange(16)[::-1])
    assert np.array_equal(rev["codes"], prm["codes"])


# --------------------------------------------------------------------------------------------
# ZSIC per-column spacing (WaterSIC section 2: alpha_i proportional to 1 / |l_ii|)
# --------------------------------------------------------------------------------------------

def test_zsic_spacing_hand_values():
    """pivots (1, 4, 16): |l| = (1, 2, 4), geometric mean 2, so kappa = (2, 1, 1/2)."""
    np.testing.assert_allclose(O.zsic_spacing([1.0, 4.0, 16.0]), [2.0, 1.0, 0.5], rtol=1e-15)


def test_zsic_on_diagonal_hessian_is_rtn_with_column_steps():
    """Diagonal H: no feedback; column j is rounded on the step s sqrt(g2 / H_d,jj) with g2 the
    geometric mean of the damped diagonal (closed form of alpha_j proportional to 1/|l_jj|)."""
    rng = np.random.default_rng(111)
    n, m = 10, 7
    d = rng.uniform(0.5, 4.0, n)
    w = 0.02 * rng.standard_normal((m, n))
    res = O.quantize_layer(w, None, 4, H=np.diag(d), spacing="zsic")
    dd = d + 0.01 * d.mean()
    kap = np.sqrt(np.exp(np.mean(np.log(dd))) / dd)
    s, z = res["scales"][:, 0], res["zeros"][:, 0]
    code = np.clip(np.rint(w / (s[:, None] * kap[None, :])) + z[:, None], 0, 15)
    np.testing.assert_array_equal(res["codes"], code)


@pytest.mark.parametrize("seed", range(3))
def test_zsic_is_babai_on_column_scaled_basis(seed):
    """Clip-free ZSIC = textbook Babai on the tall basis [sqrt2 X; sqrt(delta) I] diag(s kappa)
    with the basis order reversed."""
    n, T, m = 10, 40, 30
    w, x = _rand_problem(T, n, m, seed=113 + seed)
    res = O.quantize_layer(w, x, 3, clip=False, spacing="zsic")
    F = np.vstack([np.sqrt(2.0) * x, np.sqrt(res["delta"]) * np.eye(n)])
    kap = res["col_scale"]
    for r in range(m):
        s = res["scales"][r, 0]
        u = _babai_gram_schmidt((F * (s * kap))[:, ::-1], F @ w[r])[::-1]
        assert np.array_equal(res["codes"][r] - int(res["zeros"][r, 0]), u.astype(np.int64))


def test_zsic_bound_and_am_gm_against_uniform():
    """Theorem 5 with per-column steps: the clip-free damped loss of each row is at most
    (1/4) sum_j (s kappa_j)^2 D_jj = (n/4) s^2 g^2; and at the same row step this is at most the
    uniform grid's (1/4) s^2 sum_j D_jj (arithmetic vs geometric mean of the pivots)."""
    w, x = _rand_problem(200, 32, 40, seed=117)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    U = O.hinv_upper_factor(hd)
    D = 1.0 / np.diag(U) ** 2
    kap = O.zsic_spacing(D)
    s, z = O.clipfree_grid(w, 3, np.ones(40))
    zs = O.gptq_columns(w, U, 3, clip=False, grid=(s, z), col_scale=kap)
    g2 = np.exp(np.mean(np.log(D)))
    for r in range(40):
        d = w[r] - zs["Q"][r]
        b_z = 0.25 * s[r] ** 2 * np.sum(kap ** 2 * D)
        np.testing.assert_allclose(b_z, 0.25 * 32 * s[r] ** 2 * g2, rtol=1e-12)
        assert d @ hd @ d <= b_z * (1 + 1e-12)
        assert b_z <= 0.25 * s[r] ** 2 * D.sum()


# --------------------------------------------------------------------------------------------
# Huffman coding of unconstrained integer codes (GEOM section 3, HPTQ)
# --------------------------------------------------------------------------------------------

def test_huffman_textbook_example():
    """The classic six-symbol example (counts 45, 13, 12, 16, 9, 5): optimal total length 224,
    lengths (1, 3, 3, 3, 4, 4)."""
    ln = O.huffman_lengths([45, 13, 12, 16, 9, 5])
    assert int(np.dot(ln, [45, 13, 12, 16, 9, 5])) == 224
    assert sorted(ln.tolist()) == [1, 3, 3, 3, 4, 4]


@pytest.mark.parametrize("seed", range(3))
def test_huffman_kraft_entropy_and_roundtrip(seed):
    """Kraft equality sum 2^-l = 1 (a full prefix code), N H <= total < N (H + 1), the canonical
    codewords are prefix-free, and decoding the stream gives the symbols back."""
    rng = np.random.default_rng(200 + seed)
    sym = np.clip(np.rint(rng.standard_t(3, 3000) * 3).astype(np.int64) + 40, 0, 80)
    counts = np.bincount(sym, minlength=81)
    ln = O.huffman_lengths(counts)
    used = counts > 0
    assert abs(np.sum(2.0 ** -ln[used]) - 1.0) < 1e-12
    p = counts[used] / counts.sum()
    H = -np.sum(p * np.log2(p))
    total = int(np.dot(counts, ln))
    assert sym.size * H <= total < sym.size * (H + 1)
    cw = O.canonical_codewords(ln)
    words = [format(int(cw[i]), f"0{ln[i]}b") for i in np.nonzero(used)[0]]
    for a in words:
        for b in words:
            assert a == b or not b.startswith(a)
    stream, nbits = O.huffman_encode(sym, ln)
    assert nbits == total
    assert np.array_equal(O.huffman_decode(stream, nbits, ln, sym.size), sym)


def test_unbounded_lattice_on_diagonal_hessian_is_rounding():
    """Unconstrained lattice, diagonal H: no feedback, codes = rint(w / s) with zero point 0 and
    s the min-max step of the row (values far outside the b-bit range stay unclamped)."""
    rng = np.random.default_rng(211)
    w = 0.02 * rng.standard_normal((6, 12))
    w[0, 3] = 0.5  # an outlier
    res = O.quantize_layer(w, None, 3, H=np.diag(rng.uniform(1, 2, 12)), clip="unbounded")
    s = (np.maximum(w.max(1), 0) - np.minimum(w.min(1), 0)) / 7.0
    np.testing.assert_array_equal(res["codes"], np.rint(w / s[:, None]))
    assert (res["zeros"] == 0).all()
    assert res["rate"] > 0


# --------------------------------------------------------------------------------------------
# SSQR: full-precision outliers and the scale search (GEOM section 3)
# --------------------------------------------------------------------------------------------

def test_ssqr_outliers_are_exact_and_feed_nothing_forward():
    """An outlier keeps its error-fed value exactly (e = 0); the normals' codes are in range and
    their dequantized values lie on the row grid; with a tiny alpha almost every entry is an
    outlier and Q equals W (no error anywhere)."""
    w, x = _rand_problem(80, 16, 12, seed=221)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    U = O.hinv_upper_factor(hd)
    r = O.ssqr_columns(w, U, 3, np.full(12, 0.3))
    assert r["outlier"].any() and (~r["outlier"]).any()
    assert np.all(r["e"][r["outlier"]] == 0.0)
    c = r["codes"]
    assert c[~r["outlier"]].min() >= 0 and c[~r["outlier"]].max() <= 7
    s, z = r["scales"][:, 0], r["zeros"][:, 0]
    grid = s[:, None] * (c - z[:, None])
    np.testing.assert_allclose(r["Q"][~r["outlier"]], grid[~r["outlier"]], rtol=0, atol=1e-15)
    tiny = O.ssqr_columns(w, U, 3, np.full(12, 1e-9))
    assert tiny["outlier"].all() and np.array_equal(tiny["Q"], w)


@pytest.mark.parametrize("density", [0.0, 0.05, 0.2])
def test_ssqr_search_is_a_bisection_of_feasibility(density):
    """The chosen alpha is feasible (at most density * n outliers per row) and the last
    infeasible probe lies within the bisection resolution below it, so no finer grid within
    that resolution meets the density; with density 0 no row has an outlier."""
    w, x = _rand_problem(100, 20, 10, seed=223)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    U = O.hinv_upper_factor(hd)
    steps = 16
    r, alpha, lo = O.ssqr_search(w, U, 3, density, steps=steps)
    limit = np.floor(density * 20 + 1e-9)
    assert np.all(r["outlier"].sum(axis=1) <= limit)
    hi = np.log2(alpha)
    assert np.all(hi - lo <= 9.0 / 2 ** steps + 1e-12)
    probe = O.ssqr_columns(w, U, 3, 2.0 ** lo)["outlier"].sum(axis=1)
    assert np.all(probe > limit)
    if density == 0.0:
        assert not r["outlier"].any()


# ---------------------------------------------------------------------------------------------
# The follow harness of gptq_columns: near-ties taken over, everything else counted
# ---------------------------------------------------------------------------------------------

def test_follow_own_decisions_changes_nothing():
    rng = np.random.default_rng(5)
    W = rng.standard_normal((6, 40))
    X = rng.standard_normal((200, 40))
    plain = O.quantize_layer(W, X, bits=3, group=8)
    fol = O.quantize_layer(W, X, bits=3, group=8,
                           follow=dict(codes=plain["codes"], zeros=plain["zeros"]))
    assert fol["followed"] == 0 and fol["disagree"] == 0
    assert np.array_equal(fol["codes"], plain["codes"])
    assert np.array_equal(fol["Q"], plain["Q"])


def test_follow_takes_a_tie_and_counts_a_real_difference():
    """U = I (nothing fed forward), 2-bit, row [0, 1.75, 3.5]: s = 7/6, z = 0, so column 1 sits
    on the boundary between codes 1 and 2 (own choice 2, round half to even) and column 2 is
    3 with no tie."""
    U = np.eye(3)
    w = np.array([[0.0, 1.75, 3.5]])
    own = O.gptq_columns(w, U, 2)
    assert own["codes"].tolist() == [[0, 2, 3]]
    tie = O.gptq_columns(w, U, 2, follow=dict(codes=[[0, 1, 3]]))
    assert tie["codes"].tolist() == [[0, 1, 3]] and (tie["followed"], tie["disagree"]) == (1, 0)
    far = O.gptq_columns(w, U, 2, follow=dict(codes=[[0, 2, 1]]))
    assert far["codes"].tolist() == [[0, 2, 3]] and (far["followed"], far["disagree"]) == (0, 1)
    off_by_one = O.gptq_columns(w, U, 2, follow=dict(codes=[[1, 2, 3]]))  # t = 0: no tie
    assert off_by_one["codes"].tolist() == [[0, 2, 3]] and off_by_one["disagree"] == 1


def test_follow_carries_on_from_the_followed_code():
    """U = [[1, 1], [0, 1]], 2-bit, row [0.75, 1.5]: s = 0.5, z = 0.  Own: t0 = 1.5 -> 2,
    e0 = -0.25, w1 = 1.75, t1 = 3.5 -> 4 -> clamp 3.  Followed code 1: e0 = 0.25, w1 = 1.25,
    t1 = 2.5 -> 2 (half to even)."""
    U = np.array([[1.0, 1.0], [0.0, 1.0]])
    w = np.array([[0.75, 1.5]])
    assert O.gptq_columns(w, U, 2)["codes"].tolist() == [[2, 3]]
    r = O.gptq_columns(w, U, 2, follow=dict(codes=[[1, 2]]))
    assert r["codes"].tolist() == [[1, 2]] and (r["followed"], r["disagree"]) == (1, 0)
    np.testing.assert_allclose(r["e"], [[0.25, 1.25 - 1.0]])


def test_follow_takes_a_tied_zero_point():
    """group 2, 2-bit, row [-0.75, 0.75]: s = 0.5, -lo/s = 1.5, own zero 2 (half to even);
    followed zero 1.  Codes: rint(-1.5) + 1 = -1 -> 0 and rint(1.5) + 1 = 3."""
    U = np.eye(2)
    w = np.array([[-0.75, 0.75]])
    own = O.gptq_columns(w, U, 2, group=2)
    assert own["zeros"].tolist() == [[2.0]] and own["codes"].tolist() == [[0, 3]]
    r = O.gptq_columns(w, U, 2, group=2, follow=dict(codes=[[0, 3]], zeros=[[1]]))
    assert r["zeros"].tolist() == [[1.0]] and r["codes"].tolist() == [[0, 3]]
    assert (r["followed"], r["disagree"]) == (1, 0)
    np.testing.assert_allclose(r["Q"], [[-0.5, 1.0]])


def test_follow_is_refused_where_it_has_no_meaning():
    rng = np.random.default_rng(1)
    W = rng.standard_normal((2, 8))
    X = rng.standard_normal((40, 8))
    f = dict(codes=np.zeros((2, 8), dtype=np.int64))
    with pytest.raises(ValueError):
        O.quantize_layer(W, X, bits=3, reverse=True, follow=f)
    with pytest.raises(ValueError):
        O.quantize_layer(W, X, bits=3, clip=False, follow=f)


# ---------------------------------------------------------------------------------------------
# HPTQ rate control: the coded size of the integers and the search for a budget
# ---------------------------------------------------------------------------------------------

def test_hptq_rate_hand_values():
    # two symbols, equal counts: one bit each
    assert O.hptq_rate([[0, 0, 1, 1]]) == 1.0
    # counts 5, 2, 1, 1: merges 1+1, 2+2, 4+5 give lengths 1, 2, 3, 3 -> 5 + 4 + 3 + 3 = 15 bits
    codes = np.array([0] * 5 + [1] * 2 + [2, 3])
    assert O.hptq_rate(codes) == 15 / 9
    # only the differences between codes matter
    assert O.hptq_rate(codes - 7) == 15 / 9
    # one symbol still costs one bit per weight
    assert O.hptq_rate(np.zeros(6, dtype=np.int64)) == 1.0


def test_hptq_search_hand_trace():
    """U = I (nothing fed forward), one row [0, 1, 2, 3], 2-bit min-max step s = 1, lattice
    alpha s Z.  Coded sizes: alpha 1 -> [0,1,2,3], 8 bits; alpha 2 -> [0,0,1,2] (half to even),
    6 bits; alpha 2^0.5 -> [0,1,1,2], 6 bits; alpha 2^0.25 -> [0,1,2,3], 8 bits.  Budget 1.5
    bits/weight (6 bits): t = 0 does not fit, t = 1 does; bisection: t = 0.5 fits, t = 0.25
    does not."""
    U = np.eye(4)
    w = np.array([[0.0, 1.0, 2.0, 3.0]])
    r, alpha, bits, lo = O.hptq_search(w, U, 2, 1.5, steps=2, max_doublings=4)
    assert alpha == 2.0 ** 0.5 and bits == 6 and lo == 0.25
    assert r["codes"].tolist() == [[0, 1, 1, 2]]
    np.testing.assert_allclose(r["scales"][:, 0], [2.0 ** 0.5])
    # alpha = 1 already fits a 2-bit budget: the bracket starts at t = -8, and t = -4 fits too
    r, alpha, bits, lo = O.hptq_search(w, U, 2, 2.0, steps=1)
    assert alpha == 2.0 ** -4 and lo == -8.0
    assert r["codes"].tolist() == [[0, 16, 32, 48]] and bits == 8
    # below one bit per weight nothing fits
    with pytest.raises(ValueError):
        O.hptq_search(w, U, 2, 0.5, steps=2, max_doublings=3)


@pytest.mark.parametrize("budget", [2.5, 3.5])
def test_hptq_search_brackets_the_budget(budget):
    """On a random layer the result fits, the last value that did not fit does not, and the
    bracket has the width the bisection leaves."""
    rng = np.random.default_rng(3)
    W = rng.standard_normal((6, 48))
    X = rng.standard_normal((300, 48))
    H = O.hessian(X)
    hd, _ = O.dampen(H, 0.01)
    U = O.hinv_upper_factor(hd)
    steps = 6
    r, alpha, bits, lo = O.hptq_search(W, U, 4, budget, steps=steps)
    t = np.log2(alpha)
    assert bits <= budget * W.size
    assert O.hptq_rate(r["codes"]) * W.size == bits
    if lo > -8.0:
        assert t - lo == 2.0 ** -steps
        r_lo = O.gptq_columns(W, U, 4, clip="unbounded", alpha=np.full(6, 2.0 ** lo))
        assert O.hptq_rate(r_lo["codes"]) > budget


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_hptq_rate_lies_within_one_bit_of_the_entropy(seed):
    """Shannon's bound for a Huffman code: H <= rate < H + 1 bits per symbol, H the empirical
    entropy of the codes; equal to H when every probability is a power of two."""
    rng = np.random.default_rng(seed)
    codes = np.rint(rng.standard_normal(5000) * (1.0 + seed)).astype(np.int64)
    _, counts = np.unique(codes, return_counts=True)
    p = counts / counts.sum()
    H = float(-(p * np.log2(p)).sum())
    r = O.hptq_rate(codes)
    assert H - 1e-12 <= r < H + 1.0
    dyadic = np.repeat([0, 1, 2, 3], [8, 4, 2, 2])           # p = 1/2, 1/4, 1/8, 1/8
    assert O.hptq_rate(dyadic) == pytest.approx(1.75)
