"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every test runs on both implementations of the oracle: the C++ reference (oracle/bq_ref.cpp,
through oracle/cref.py) and the numpy one (oracle/bq_oracle.py), through the fixture ``O``.
Each test checks the oracle against something other than itself: values
worked by hand from a page's formula (tests/golden, with citations), closed
forms, brute force over tiny inputs, invariants and special cases. A planted
mistake in the oracle (dropped term, wrong sign, transposed operand, wrong
rounding mode) fails at least one of these.
"""
import math

import numpy as np
import pytest

import bq_inputs as I


@pytest.fixture(params=["cpp", "numpy"])
def O(request):
    """The oracle implementation under test: the C++ reference or the numpy one."""
    if request.param == "cpp":
        from oracle import cref
        return cref
    from oracle import bq_oracle
    return bq_oracle


# --------------------------------------------------------------------- sign
def test_sign_zero_is_plus_one(O, golden):
    g = golden("sign_zero.json")
    got = O.sign_pm1(np.array(g["inputs"], dtype=np.float32))
    assert got.tolist() == g["expect"]


# ------------------------------------------------------- activation int8
def test_act_int8_hand_values(O, golden):
    g = golden("act_int8_handpicked.json")
    q, gamma = O.quantize_act_int8(np.array(g["x"], dtype=np.float32))
    assert q.tolist() == g["q"]
    assert gamma.tolist() == g["gamma"]


def test_act_int8_endpoints_and_range(O):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((16, 300)) * rng.uniform(0.1, 50, (16, 1))).astype(np.float32)
    q, gamma = O.quantize_act_int8(x)
    assert q.min() >= -127 and q.max() <= 127
    for m in range(16):
        kmax = int(np.argmax(np.abs(x[m])))
        assert abs(int(q[m, kmax])) == 127          # the absmax element maps to +-127
        assert np.sign(q[m, kmax]) == np.sign(x[m, kmax])
    # dequantized error is within half a step
    xh = O.dequant_act_int8(q, gamma)
    step = gamma.astype(np.float64) / 127.0
    assert np.all(np.abs(xh - x) <= 0.5 * step[:, None] * (1 + 1e-6))


# -------------------------------------------------------------------- RaBiT
def test_rabit_recursion_hand_example(O, golden):
    g = golden("rabit_recursion.json")
    p = O.rabit_pack(np.array(g["W"], np.float32), np.array(g["h2"], np.float32))
    assert p["B1"].tolist() == g["B1"]
    assert p["B2"].tolist() == g["B2"]
    assert p["g1"].tolist() == g["g1"]
    assert p["g2"].tolist() == g["g2"]
    assert O.rabit_weight(p).tolist() == g["W_hat"]


def test_rabit_constant_magnitude_rows_reconstruct_exactly(O):
    # |W[n,k]| = c_n for all k -> g1 = c_n, R1 == 0, B2 = sign(0) = +1, g2 = 0, W_hat = W
    rng = np.random.default_rng(1)
    c = np.array([0.5, 0.25, 0.125, 2.0], np.float32)
    s = np.where(rng.random((4, 64)) < 0.5, -1.0, 1.0).astype(np.float32)
    W = (c[:, None] * s).astype(np.float32)
    p = O.rabit_pack(W, np.ones(64, np.float32))
    assert np.all(p["g1"] == c)
    assert np.all(p["B2"] == 1)
    assert np.all(p["g2"] == 0)
    assert np.array_equal(O.rabit_weight(p), W.astype(np.float64))


def test_rabit_layer_is_sum_of_two_sign_paths(O):
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((8, 96)) * 0.02).astype(np.float32)
    h2 = rng.uniform(0.5, 1.5, 96).astype(np.float32)
    x = rng.standard_normal((3, 96)).astype(np.float32)
    p = O.rabit_pack(W, h2)
    r = O.rabit_layer(p, x)
    # dense W_hat x equals g1*acc1 + g2*acc2 with acc_p = sum_k B_p h_p x, computed per element
    for m in range(3):
        for n in range(8):
            a1 = sum(float(p["B1"][n, k]) * float(x[m, k]) for k in range(96))
            a2 = sum(float(p["B2"][n, k]) * float(h2[k]) * float(x[m, k]) for k in range(96))
            ref = float(p["g1"][n]) * a1 + float(p["g2"][n]) * a2
            assert abs(r["y"][m, n] - ref) <= 1e-12 * (1 + abs(ref))
    # the residual path reduces the reconstruction error of a single path
    e1 = np.mean((W - p["g1"][:, None] * p["B1"]) ** 2)
    e2 = np.mean((W - O.rabit_weight(dict(p, h2=np.ones(96, np.float32)))) ** 2)
    assert e2 < e1


# ------------------------------------------------------------------- BitNet
def test_bitnet_alpha_is_mean_abs(O):
    W = np.array([[0.5, -0.25], [-1.0, 0.25]], np.float32)
    p = O.bitnet_pack(W)
    assert p["alpha"] == np.float32(0.5)
    assert p["B"].tolist() == [[1, -1], [-1, 1]]


def test_xnor_popcount_identity_all_pairs(O):
    # BitNet §2.3 binary product: for +-1 vectors, sum a*b = 2*popc(xnor(a,b)) - K
    K = 8
    vals = [[1 if (v >> j) & 1 else -1 for j in range(K)] for v in range(1 << K)]
    for a in vals[::3]:
        for b in vals:
            assert O.xnor_popcount_dot(a, b) == sum(x * y for x, y in zip(a, b))


def test_w1a8_plane_identity_all_int8_codes(O):
    # sum_k B_k q_k = sum q - 2 * sum_c omega_c popc(NEG & X_c) for every int8 code value
    rng = np.random.default_rng(3)
    codes = np.arange(-127, 128)
    for rep in range(4):
        q = rng.permutation(codes)[:32]
        neg = (rng.random(32) < 0.5).astype(np.int64)
        B = 1 - 2 * neg
        direct = int(np.dot(B, q))
        via_planes = int(q.sum()) - 2 * O.bitplane_dot(neg, 1, False, q, 8, True)
        assert direct == via_planes
    # and the per-code plane decomposition itself
    for v in codes:
        pl = O.planes_of([v], 8)
        assert sum(w * int(p[0]) for w, p in zip(O.plane_weights(8, True), pl)) == v


def test_bitnet_layer_integer_and_float_routes_agree(O):
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((24, 128)) * 0.02).astype(np.float32)
    x = rng.standard_normal((2, 128)).astype(np.float32)
    p = O.bitnet_pack(W)
    r = O.bitnet_layer(p, x)
    y_int = float(p["alpha"]) * (r["gamma"].astype(np.float64)[:, None] / 127.0) * r["acc"]
    assert np.allclose(r["y"], y_int, rtol=1e-12, atol=1e-15)
    # acc against an element loop over the +-1 weights
    for n in range(0, 24, 5):
        assert r["acc"][1, n] == sum(int(p["B"][n, k]) * int(r["q"][1, k]) for k in range(128))


# ------------------------------------------------------------------ ternary
def test_ternary_hand_examples(O, golden):
    for c in golden("ternary_handpicked.json")["cases"]:
        p = O.ternary_pack(np.array(c["W"], np.float32))
        assert float(p["gamma_w"]) == c["gamma"]
        assert p["T"].tolist() == c["T"]


def test_ternary_zero_fraction_of_gaussian(O):
    # threshold 0.5*gamma with gamma = sigma*sqrt(2/pi): P(|Z| < 0.5 sqrt(2/pi)) = erf(0.5/sqrt(pi))
    W = (np.random.default_rng(6).standard_normal((1024, 1024)) * 0.02).astype(np.float32)
    p = O.ternary_pack(W)
    frac = float(np.mean(p["T"] == 0))
    assert abs(frac - math.erf(0.5 / math.sqrt(math.pi))) < 0.003
    assert abs(float(np.mean(p["T"] == 1)) - float(np.mean(p["T"] == -1))) < 0.003


def test_ternary_int_route_equals_dequant_route(O):
    # HGF §1.2: Y = Y_int * gamma_x gamma_W / 127
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((16, 64)) * 0.02).astype(np.float32)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    p = O.ternary_pack(W)
    r = O.ternary_layer(p, x)
    y_int = r["acc"] * (float(p["gamma_w"]) * r["gamma"].astype(np.float64)[:, None] / 127.0)
    assert np.allclose(r["y_ternary"], y_int, rtol=1e-12, atol=1e-15)


def test_lora_correction_closed_form(O):
    # tanh(ln 2) = 3/5 and SiLU(ln 3) = ln 3 * sigmoid(ln 3) = 0.75 ln 3
    A = np.array([[math.log(3.0)]])
    B = np.array([[1.0, -2.0, 0.5]])
    x = np.array([[1.0]], np.float32)
    got = O.lora_correction(x, A, B, math.log(2.0))
    # lora_alpha passes through float32 first; use its exact tanh bound
    a32 = float(np.float32(math.log(2.0)))
    scale = (math.exp(2 * a32) - 1) / (math.exp(2 * a32) + 1)
    assert abs(scale - 0.6) < 1e-7
    want = 0.6 * 0.75 * math.log(3.0) * np.array([1.0, -2.0, 0.5])
    assert np.allclose(got[0], want, rtol=1e-6)
    # x A = 0 -> SiLU(0) = 0 -> no correction
    assert np.all(O.lora_correction(np.zeros((1, 1), np.float32), A, B, 0.1) == 0)


# ---------------------------------------------------------------------- ABQ
def test_abq_hand_examples(O, golden):
    for c in golden("abq_handpicked.json")["cases"]:
        q, d, z = O.quantize_rows_asym(np.array([c["row"]], np.float32), c["bits"])
        assert q[0].tolist() == c["q"]
        assert float(d[0]) == c["delta"]
        assert int(z[0]) == c["z"]


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
def test_abq_grid_round_trip(O, bits):
    # values already on a binary-exact grid lo + Delta*i dequantize exactly
    L = 1 << bits
    delta = 2.0 ** -6
    lo = -delta * (L // 2)
    row = (lo + delta * np.arange(L)).astype(np.float32)
    q, d, z = O.quantize_rows_asym(row[None], bits)
    assert q[0].tolist() == list(range(L))
    assert np.array_equal(d[0] * (q[0] - z[0]).astype(np.float64), row.astype(np.float64))


@pytest.mark.parametrize("w,a", [(w, a) for w in (2, 4, 6, 8) for a in (2, 4, 6, 8)])
def test_abq_bitplane_identity_brute_force(O, w, a):
    # sum_b sum_c 2^(b+c) popc(W_b & X_c) == sum q_w q_x for unsigned codes
    rng = np.random.default_rng(w * 10 + a)
    for _ in range(3):
        qw = rng.integers(0, 1 << w, 16)
        qx = rng.integers(0, 1 << a, 16)
        assert O.bitplane_dot(qw, w, False, qx, a, False) == int(np.dot(qw, qx))


def test_abq_zero_point_expansion_and_bounds(O):
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((12, 256)) * 0.02).astype(np.float32)
    x = (rng.standard_normal((3, 256)) * 3).astype(np.float32)
    for wb, ab in [(2, 8), (4, 4), (6, 6), (8, 8)]:
        p = O.abq_pack(W, wb)
        assert p["Q"].min() >= 0 and p["Q"].max() <= (1 << wb) - 1
        r = O.abq_layer(p, x, ab)
        assert r["Qx"].min() >= 0 and r["Qx"].max() <= (1 << ab) - 1
        K = W.shape[1]
        P = r["Qx"].astype(np.int64) @ p["Q"].astype(np.int64).T
        Sw, Sx = p["Q"].sum(1).astype(np.int64), r["Qx"].sum(1).astype(np.int64)
        zw, zx = p["z"].astype(np.int64), r["z_x"].astype(np.int64)
        I2 = P - zx[:, None] * Sw[None] - zw[None] * Sx[:, None] + K * zx[:, None] * zw[None]
        assert np.array_equal(r["I"], I2)
        assert np.abs(P).max() <= ((1 << wb) - 1) * ((1 << ab) - 1) * K
        y_int = r["delta_x"].astype(np.float64)[:, None] * p["delta"].astype(np.float64)[None] * r["I"]
        assert np.allclose(r["y"], y_int, rtol=1e-12, atol=1e-15)


# --------------------------------------------------------------------- BVSR
def test_nearest_rank_quantile(O):
    v = np.arange(16.0)
    assert [O.nearest_rank(v, 2 * a + 1, 16) for a in range(8)] == [2.0 * a for a in range(8)]
    v = np.arange(10.0)  # ceil(1*10/16) = 1 -> v[0]; ceil(15*10/16) = 10 -> v[9]
    assert O.nearest_rank(v, 1, 16) == 0.0 and O.nearest_rank(v, 15, 16) == 9.0


def test_bvsr_ratio2_sets_are_the_uniform_rtn_grid(O):
    # r = 2: subset sums of {1,2,4,8}/15 scaled to [lo, hi] are lo + (hi-lo) i/15, i = 0..15
    W = (np.random.default_rng(9).standard_normal((32, 256)) * 0.02).astype(np.float32)
    tab = O.bvsr_set_table(W)
    P = O.bvsr_points(tab)
    for s in range(64, 128):
        lo, span = float(tab[s, 4]), float(tab[s, 0]) * 15
        want = lo + span * np.arange(16) / 15
        assert np.allclose(P[s], want, rtol=0, atol=1e-7 * (abs(lo) + abs(span)))
        assert np.all(np.diff(P[s]) > 0)


def test_bvsr_encoding_matches_rtn_for_uniform_set(O):
    # a table whose only set is the uniform grid on [lo, hi]: codes are round((w-lo)/Delta) clamped
    lo, hi = -0.06, 0.09
    span = hi - lo
    row = np.array([span * 2 ** i / 15 for i in range(4)] + [lo], np.float32)
    tab = np.tile(row, (256, 1))
    rng = np.random.default_rng(10)
    w = rng.uniform(-0.08, 0.11, (64, 32)).astype(np.float32)
    codes, sets = O.bvsr_encode_vectors(w, tab)
    P = O.bvsr_points(tab)[0]
    delta = (P[15] - P[0]) / 15
    rtn = np.clip(np.rint((w.astype(np.float64) - P[0]) / delta), 0, 15)
    far = np.abs((w - P[0]) / delta - np.floor((w - P[0]) / delta) - 0.5) > 1e-3
    assert np.array_equal(codes[far], rtn[far].astype(np.uint8))
    assert np.all(sets == 0)            # equal errors everywhere: lowest set index


def test_bvsr_exact_integer_table(O):
    # c = {1,2,4,8}, o = 0 makes the 16 points the integers 0..15: integer weights encode exactly
    tab = np.zeros((256, 5), np.float32)
    tab[:, :4] = [50.0, 60.0, 70.0, 80.0]
    tab[:, 4] = 1000.0
    tab[7] = [1.0, 2.0, 4.0, 8.0, 0.0]
    w = np.random.default_rng(11).integers(0, 16, (20, 32)).astype(np.float32)
    codes, sets = O.bvsr_encode_vectors(w, tab)
    assert np.all(sets == 7)
    assert np.array_equal(codes, w.astype(np.uint8))


def test_bvsr_search_is_exhaustive_optimum(O):
    # no other set, and no single-element code change, gives a smaller squared error
    W = (np.random.default_rng(12).standard_normal((4, 64)) * 0.02).astype(np.float32)
    tab = O.bvsr_set_table(W)
    P = O.bvsr_points(tab)
    vecs = W.reshape(-1, 32)
    codes, sets = O.bvsr_encode_vectors(vecs, tab)
    for v in range(vecs.shape[0]):
        w = vecs[v].astype(np.float64)
        errs = []
        for s in range(256):
            e = 0.0
            for x in w:
                e += min((x - p) ** 2 for p in P[s])
            errs.append(e)
        best = float(np.sum((w - P[sets[v], codes[v]]) ** 2))
        assert best <= min(errs) * (1 + 1e-12) + 1e-18
        for e_i in range(32):
            for c in range(16):
                assert (w[e_i] - P[sets[v], c]) ** 2 >= (w[e_i] - P[sets[v], codes[v, e_i]]) ** 2 - 1e-18


def test_bvsr_layer_routes_agree(O):
    rng = np.random.default_rng(13)
    W = (rng.standard_normal((6, 128)) * 0.02).astype(np.float32)
    x = rng.standard_normal((2, 128)).astype(np.float32)
    p = O.bvsr_pack(W)
    r = O.bvsr_layer(p["codes"], p["sets"], p["table"], x)
    # y as sum over vectors of sum_i c_i T_i + o S (integer plane sums per vector)
    tab = p["table"].astype(np.float64)
    for m in range(2):
        for n in range(6):
            tot = 0.0
            for v in range(4):
                s = int(p["sets"][n, v])
                qv = r["q"][m, 32 * v:32 * v + 32].astype(np.int64)
                cv = p["codes"][n, 32 * v:32 * v + 32].astype(np.int64)
                T = [int(np.dot((cv >> i) & 1, qv)) for i in range(4)]
                tot += sum(tab[s, i] * T[i] for i in range(4)) + tab[s, 4] * int(qv.sum())
            ref = tot * float(r["gamma"][m]) / 127.0
            assert abs(r["y"][m, n] - ref) <= 1e-12 * (1 + abs(ref))


# ---------------------------------------------------------- size / memory wall
def test_memory_wall_and_sizes(O, golden):
    g = golden("memory_wall.json")
    w = g["wall"]
    tps = O.decode_tokens_per_s(w["bandwidth_Bps"], w["params"], w["bits"])
    assert abs(tps - w["tokens_per_s_printed"]) <= w["tol"]
    assert O.weight_bits_per_param("bitnet") * 7e9 / 8 == g["size_1bit_bytes"]
    assert 16 * 7e9 / 8 == g["size_fp16_bytes"]
    assert O.weight_bits_per_param("ternary") == g["ternary_bits"]
    assert O.weight_bits_per_param("bvsr") == 4.25
    assert O.weight_bits_per_param("abq", 6) == 6.0


def test_tolerance_helper(O):
    y_ref = np.array([1.0, -2.0, 0.5])
    assert O.tolerance_ok(y_ref + 1.9e-3, y_ref)
    assert not O.tolerance_ok(y_ref + 2.1e-3, y_ref)


def test_bvsr_table_construction_hand_built(O):
    # 16 vectors whose minima are -(v+1)/1000 and maxima (v+1)/500, every other element 0.
    # Nearest-rank (2a+1)/16 quantile of 16 values is the (2a+1)-th smallest: lo_a = -(16-2a)/1000,
    # hi_b = (2b+1)/500. Set 64j + 8a + b: o = lo_a, c_i = (hi_b - lo_a) r_j^i / sum_i' r_j^i'.
    V = 16
    W = np.zeros((1, 32 * V), np.float32)
    for v in range(V):
        W[0, 32 * v + 3] = -(v + 1) / 1000.0
        W[0, 32 * v + 17] = (v + 1) / 500.0
    tab = O.bvsr_set_table(W)
    mins = sorted(np.float32(-(v + 1) / 1000.0) for v in range(V))
    maxs = sorted(np.float32((v + 1) / 500.0) for v in range(V))
    for j, r in enumerate((1.5, 2.0, 2.5, 3.0)):
        for a in range(8):
            for b in range(8):
                s = 64 * j + 8 * a + b
                lo, hi = float(mins[2 * a]), float(maxs[2 * b])
                assert tab[s, 4] == np.float32(lo)
                tot = sum(r ** i for i in range(4))
                for i in range(4):
                    assert tab[s, i] == np.float32((hi - lo) * r ** i / tot)
    assert tab[0, 4] == np.float32(-0.016) and tab[64 + 7, 0] * 15 == pytest.approx(0.030 + 0.016, rel=1e-6)


# ------------------------------------------------------------------ RaBiT iterative residual SVID
def test_svid_exact_signed_rank1(O):
    """W = s * (a b^T) with power-of-two a, b: one round recovers W up to float32 rounding of
    g and h (the rank-1 fit is exact in real arithmetic), and path 2 carries only that rounding."""
    rng = np.random.default_rng(5)
    a = 2.0 ** rng.integers(-6, -2, 16)
    b = 2.0 ** rng.integers(-2, 2, 64)
    s = np.where(rng.random((16, 64)) < 0.5, -1.0, 1.0)
    W = (s * np.outer(a, b)).astype(np.float32)
    p = O.rabit_pack_svid(W, rounds=1)
    assert np.array_equal(p["B1"], O.sign_pm1(W))
    w2 = float(np.sum(W.astype(np.float64) ** 2))
    assert O.rabit_recon_error(p, W) <= 1e-12 * w2
    p1 = dict(p, g2=np.zeros_like(p["g2"]))               # path 1 alone
    assert O.rabit_recon_error(p1, W) <= 1e-12 * w2
    assert np.all(np.abs(p["g2"]) <= 1e-6 * np.abs(p["g1"]).max())


def test_svid_first_step_is_mean_abs_and_error_never_grows(O):
    W = I.weights(24, 256, seed=9)
    base = O.rabit_pack(W, np.ones(256, np.float32))
    p1 = O.rabit_pack_svid(W, rounds=1)
    # the first g-step from h = 1 is the mean |W| of each row, as in rabit_pack
    g_first = np.array([O.mean_abs_f32(W[n]) for n in range(24)], dtype=np.float32)
    assert np.array_equal(base["g1"], g_first)
    errs = [O.rabit_recon_error(O.rabit_pack_svid(W, rounds=r), W) for r in (1, 2, 5, 20)]
    for e0, e1 in zip(errs, errs[1:]):
        assert e1 <= e0 * (1 + 1e-6)
    assert errs[-1] < O.rabit_recon_error(base, W)


def test_svid_g_step_is_least_squares(O):
    """For fixed h, g from the SVID step solves min_g ||A - g h^T||^2 row by row (checked with
    numpy's least squares on the first round's target A = |W|)."""
    W = I.weights(8, 128, seed=3)
    A = np.abs(W.astype(np.float64))
    h = np.linspace(0.5, 1.5, 128)
    g_ls = np.array([np.linalg.lstsq(h[:, None], A[i], rcond=None)[0][0] for i in range(8)])
    g_step = (A * h[None, :]).sum(1) / (h * h).sum()
    assert np.allclose(g_ls, g_step, rtol=1e-12)
    p = O.rabit_pack_svid(W, rounds=1)
    g_formula = (A.sum(1) / 128).astype(np.float32)      # h = 1 in the first step
    assert np.allclose(p["g1"], g_formula, rtol=1e-6)


# ------------------------------------------------------------------ ABQ bit balance (W2*)
def test_bit_balance_symmetric_levels(O):
    W = I.weights(12, 256, seed=21)
    p = O.abq_pack_balanced(W)
    pn = O.abq_pack_balanced(-W)
    assert set(np.unique(p["Q"])) <= {0, 1, 2, 3, 4} and np.all(p["z"] == 2)
    assert np.array_equal(pn["delta"], p["delta"])
    assert np.array_equal(pn["Q"], 4 - p["Q"])            # rn is odd, the grid is symmetric
    # the row extremes map to the outermost levels
    assert np.all(p["Q"][np.arange(12), np.abs(W).argmax(1)] % 4 == 0)


def test_bit_balance_grid_round_trip(O):
    d = np.float32(0.0625)
    levels = np.array([-2, -1, 0, 1, 2], np.float32) * d
    rng = np.random.default_rng(2)
    W = rng.choice(levels, size=(6, 128)).astype(np.float32)
    W[:, 0], W[:, 1] = 2 * d, -2 * d                      # each row spans the full range
    p = O.abq_pack_balanced(W)
    assert np.all(p["delta"] == d)
    deq = (p["Q"] - p["z"][:, None]).astype(np.float64) * p["delta"][:, None]
    assert np.array_equal(deq, W.astype(np.float64))


def test_bf16_round_hand_values(O):
    """Round to nearest bf16, ties to even (hand-worked bit patterns)."""
    vals = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -20, -2.5], np.float32)
    # 1 + 2^-8 is half-way between 1 and 1 + 2^-7: ties to the even mantissa (1.0);
    # 1 + 3*2^-8 is half-way between 1 + 2^-7 and 1 + 2^-6: ties to 1 + 2^-6;
    # just above half-way rounds up; -2.5 is exact
    want = np.array([1.0, 1.0, 1.0 + 2.0 ** -6, 1.0 + 2.0 ** -7, -2.5], np.float32)
    assert np.array_equal(O.bf16_round(vals), want)


def test_svid_first_round_path2_g_is_mean_abs_of_residual(O):
    """In the first Gauss-Seidel round, path 2's g-step starts from h = 1, so g2 is the row mean of |W - W_1|
    (W_1 from the returned path-1 state): pins the split of the magnitude between g and h."""
    W = I.weights(10, 256, seed=13)
    p = O.rabit_pack_svid(W, rounds=1)
    w1 = (p["g1"].astype(np.float64)[:, None] * p["h1"].astype(np.float64)[None, :]) * p["B1"]
    g2 = np.abs(W.astype(np.float64) - w1).mean(1)
    assert np.allclose(p["g2"], g2, rtol=1e-6)


# ------------------------------------------------------------------ RaBiT with P paths (groundwork)
def test_rabit_paths_two_equals_rabit_pack(O):
    W = I.weights(9, 256, seed=17)
    h2 = I.uniform(256, 0.5, 1.5, seed=2, tid=3)
    a = O.rabit_pack(W, h2)
    b = O.rabit_pack_paths(W, [np.ones(256, np.float32), h2])
    assert np.array_equal(b["B"][0], a["B1"]) and np.array_equal(b["B"][1], a["B2"])
    assert np.array_equal(b["g"][0], a["g1"]) and np.array_equal(b["g"][1], a["g2"])
    assert np.array_equal(O.rabit_weight_paths(b), O.rabit_weight(a))


def test_rabit_third_path_lowers_error_by_k_g_squared(O):
    """With h = 1: ||R - g sign(R)||^2 = ||R||^2 - K g^2 per row when g = mean|R|."""
    W = I.weights(7, 512, seed=23)
    ones = np.ones(512, np.float32)
    p2 = O.rabit_pack_paths(W, [ones, ones])
    p3 = O.rabit_pack_paths(W, [ones, ones, ones])
    e2 = ((W.astype(np.float64) - O.rabit_weight_paths(p2)) ** 2).sum(1)
    e3 = ((W.astype(np.float64) - O.rabit_weight_paths(p3)) ** 2).sum(1)
    g3 = p3["g"][2].astype(np.float64)
    assert np.allclose(e2 - e3, 512 * g3 ** 2, rtol=1e-5)
    assert np.all(e3 < e2)


def test_rabit_three_paths_hand_example(O):
    """Three paths with non-unit h (every value dyadic, so exact), worked by hand:
    W = [.75, -.25, .5, -1]: B1 = [+ - + -], g1 = 2.5/4 = .625, R1 = [.125, .375, -.125, -.375];
    B2 = [+ + - -], g2 = 1/4 = .25, R2 = R1 - .25 B2 h2 with h2 = [1, 2, 1, .5]
       = [-.125, -.125, .125, -.25]; B3 = [- - + -], g3 = .625/4 = .15625;
    W_hat = sum_p g_p B_p h_p with h3 = [2, 1, .5, 1] = [.5625, -.28125, .453125, -.90625]."""
    W = np.array([[0.75, -0.25, 0.5, -1.0]], np.float32)
    hs = [np.ones(4, np.float32), np.array([1, 2, 1, 0.5], np.float32), np.array([2, 1, 0.5, 1], np.float32)]
    p = O.rabit_pack_paths(W, hs)
    assert p["B"][:, 0].tolist() == [[1, -1, 1, -1], [1, 1, -1, -1], [-1, -1, 1, -1]]
    assert p["g"][:, 0].tolist() == [0.625, 0.25, 0.15625]
    assert O.rabit_weight_paths(p)[0].tolist() == [0.5625, -0.28125, 0.453125, -0.90625]


# ---------------------------------------------------------------------------
# ABQ distribution compensation ([ABQ] §3.2 eq.(3), gamma = 1)
# ---------------------------------------------------------------------------
# Dyadic data: every product a[n] b[k] and every sum below is exact in float32.
_COMP_A = np.array([1.0, -2.0, 0.5], np.float32)                                    # per output row
_COMP_B = np.array([0.25, -0.125, 0.0625, 0.0, 0.5, -0.25, 0.125, 1.0], np.float32) / 8  # per column
_COMP_Q0 = np.array([[0, 1, 2, 3, 3, 2, 1, 0],     # 2-bit grid codes; every row reaches 0 and 3
                     [3, 0, 0, 1, 2, 3, 1, 2],
                     [1, 3, 2, 0, 0, 1, 3, 2]], np.int32)


def test_abq_compensation_closed_form(O):
    """W = G - a b^T with G on the 2-bit grid Delta = 1/16, z = 1: the compensated codes
    are the grid codes, Delta and z come back exactly; without compensation they do not."""
    G = ((_COMP_Q0 - 1) * 0.0625).astype(np.float32)
    W = (G - np.outer(_COMP_A, _COMP_B)).astype(np.float32)
    assert np.array_equal((W + np.outer(_COMP_A, _COMP_B)).astype(np.float32), G)   # exact data
    p = O.abq_pack_compensated(W, _COMP_A, _COMP_B, 2)
    assert np.array_equal(p["Q"], _COMP_Q0)
    assert np.all(p["delta"] == np.float32(0.0625)) and np.all(p["z"] == 1)
    assert not np.array_equal(O.abq_pack(W, 2)["Q"], _COMP_Q0)
    # swapping the roles of a and b cannot even be formed: W is 3 x 8
    with pytest.raises(AssertionError):
        O.abq_pack_compensated(W, _COMP_B, _COMP_A, 2)


def test_abq_compensation_exact_cancellation_is_the_degenerate_row(O):
    """W = -a b^T: W' = 0 exactly, every row is constant, so the 1e-5 range floor applies,
    z = 0 and every code is 0 at any width."""
    W = (-np.outer(_COMP_A, _COMP_B)).astype(np.float32)
    for w in (1, 2, 4, 8):
        p = O.abq_pack_compensated(W, _COMP_A, _COMP_B, w)
        assert np.all(p["Q"] == 0) and np.all(p["z"] == 0)
        assert np.all(p["delta"] > 0) and np.all(p["delta"] <= np.float32(1e-5))   # = at w = 1


def test_abq_compensation_off_is_the_plain_pack(O):
    """a = 0 (or b = 0): W + 0 = W, so the codes, Delta and z are the plain pack's."""
    W = I.weights(37, 256, seed=5, outlier_frac=0.01)
    a, b = I.compensation_vectors(37, 256, seed=5)
    for w in (2, 5, 8):
        ref = O.abq_pack(W, w)
        for aa, bb in ((np.zeros_like(a), b), (a, np.zeros_like(b))):
            p = O.abq_pack_compensated(W, aa, bb, w)
            assert all(np.array_equal(p[k], ref[k]) for k in ("Q", "delta", "z"))
    assert not np.array_equal(O.abq_pack_compensated(W, a, b, 8)["Q"], O.abq_pack(W, 8)["Q"])


def test_abq_compensation_rounds_the_product_first(O):
    """The product is rounded before the sum: (1 + 2^-12)^2 = 1 + 2^-11 + 2^-24 rounds (a tie,
    to even) to 1 + 2^-11, so W = -(1 + 2^-11) compensates to exactly 0 (a fused
    multiply-add would leave 2^-24)."""
    u = np.float32(1 + 2.0 ** -12)
    W = np.array([[-(1 + 2.0 ** -11), 1.0]], np.float32)
    Wc = O.abq_compensated_weights(W, np.array([u]), np.array([u, 0.0], np.float32))
    assert Wc[0, 0] == 0.0 and Wc[0, 1] == 1.0


def test_abq_compensation_balanced_antisymmetry(O):
    """W2* on W' : (W, a) -> (-W, -a) negates W' exactly, so q -> 4 - q with the same Delta."""
    W = I.weights(29, 512, seed=7)
    a, b = I.compensation_vectors(29, 512, seed=7)
    p = O.abq_pack_compensated(W, a, b, 3, balanced=True)
    m = O.abq_pack_compensated(-W, -a, b, 3, balanced=True)
    assert np.array_equal(m["Q"], 4 - p["Q"]) and np.array_equal(m["delta"], p["delta"])
    assert p["Q"].min() == 0 and p["Q"].max() == 4
    assert not np.array_equal(p["Q"], O.abq_pack_balanced(W)["Q"])


def test_every_public_oracle_function_states_its_pins(O):
    """Each public function of the oracle and its layout readers says what pins it (or that its
    parity is unpinned), so an unpinned addition cannot slip in silently."""
    import inspect
    from oracle import layout as Lay
    missing = [f"{m.__name__}.{n}" for m in (O, Lay) for n, f in inspect.getmembers(m, inspect.isfunction)
               if not n.startswith("_") and f.__module__ == m.__name__
               and "Pinned" not in (f.__doc__ or "") and "parity unpinned" not in (f.__doc__ or "").lower()]
    assert not missing, missing


# --------------------------------------------------------------------- BVSR coefficient cache (clustering)
def test_bvsr_cluster_zero_rounds_is_the_quantile_table(O):
    """Without a k-means round the centroids are the quantile grid, so the table is the grid
    reading's table bit for bit."""
    W = I.weights(32, 512, seed=21)
    assert np.array_equal(O.bvsr_cluster_table(W, 0)["table"], O.bvsr_set_table(W))


def test_bvsr_cluster_objective_never_grows(O):
    """Lloyd rounds: each assignment and each exact mean can only lower the sum of squared
    distances of the vectors' (min, max) to their centroid."""
    W = I.weights(48, 1024, seed=22)
    v = W.reshape(-1, 32)
    pts = np.stack([v.min(1), v.max(1)], 1).astype(np.float64)
    J = []
    for r in range(1, 7):
        c = O.bvsr_cluster_table(W, r)
        cen = c["centroids"][c["family"].astype(int), c["assign"].astype(int)]
        J.append(float(((pts - cen) ** 2).sum()))
    assert all(b <= a * (1 + 1e-12) for a, b in zip(J, J[1:])), J
    assert J[-1] < J[0]


def test_bvsr_cluster_family_is_the_best_of_the_vectors_own_sets(O):
    """A vector's family is the ratio whose set on its own range fits it best: the exhaustive
    encoder, given a table whose sets 0..3 are the vector's own four sets (taken from the
    quantile table of the vector alone, where every grid point is its min and max), picks set
    index == family."""
    W = I.weights(8, 256, seed=23)
    c = O.bvsr_cluster_table(W, 2)
    vecs = W.reshape(-1, 32)
    for vi in range(0, vecs.shape[0], 7):
        own = O.bvsr_set_table(vecs[vi:vi + 1])
        tab = np.repeat(own[[192]], 256, axis=0)
        tab[:4] = own[[0, 64, 128, 192]]
        _, sets = O.bvsr_encode_vectors(vecs[vi:vi + 1], tab)
        assert int(sets[0]) == int(c["family"][vi])


def test_bvsr_cluster_exact_grid_vectors():
    """Hand case: every vector holds -1/2 + k/16 for k = 0..15 (each twice). The ratio-2 set on
    its range [-1/2, 7/16] has exactly those points (c = 1/16, 2/16, 4/16, 8/16), so the family is
    1 (ratio 2, error 0); all vectors share one range, so after a round their centroid is that
    range exactly, and the cluster's set is (1/16, 1/8, 1/4, 1/2, -1/2)."""
    from oracle import bq_oracle as Nmp, cref as Cpp
    row = (-0.5 + np.arange(16) / 16.0).astype(np.float32)
    W = np.tile(np.concatenate([row, row[::-1]]), (4, 2)).astype(np.float32)  # 4 rows x 64: 8 vectors
    for O in (Cpp, Nmp):
        c = O.bvsr_cluster_table(W, 1)
        assert np.all(c["family"] == 1)
        cl = int(c["assign"][0])
        assert np.all(c["assign"] == cl)
        assert c["centroids"][1, cl].tolist() == [-0.5, 0.4375]
        assert c["table"][64 + cl].tolist() == [0.0625, 0.125, 0.25, 0.5, -0.5]
        codes, sets = O.bvsr_encode_vectors(W.reshape(-1, 32), c["table"])
        assert np.all(sets == 64 + cl) and codes[0].tolist() == list(range(16)) + list(range(15, -1, -1))
