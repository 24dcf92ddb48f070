"""The two oracle implementations against each other, on seeded inputs of the workloads' shapes.

oracle/bq_ref.cpp (C++, plain loops, through oracle/cref.py) and oracle/bq_oracle.py (numpy)
are written independently from the same passages. Every integer result (codes, set indices,
zero points, accumulators) and every float32 scale must agree bit for bit, and the float64
layer outputs to within a few float64 roundings (the two sum in different orders). Both are
also held to the same pins (tests/test_oracle_pins.py runs each pin on both).
"""
import numpy as np
import pytest

import bq_inputs as I
from oracle import bq_oracle as N
from oracle import cref as C


def _same(a, b, what):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    assert np.array_equal(a, b), f"{what}: {int(np.sum(a != b))} of {a.size} differ"


def _close64(a, b, what, rel=1e-13):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape
    bound = rel * (float(np.max(np.abs(b))) + 1e-300)
    assert float(np.max(np.abs(a - b))) <= bound, what


@pytest.mark.parametrize("N_,K,M", [(97, 640, 5), (16, 256, 1), (33, 2048, 9)])
def test_activation_quantizers_agree(N_, K, M):
    x = I.activations(M, K, seed=N_ + K)
    for a, b, w in zip(N.quantize_act_int8(x), C.quantize_act_int8(x), ("q", "gamma")):
        _same(a, b, f"act {w}")
    for bits in (1, 2, 3, 4, 6, 8):
        for a, b, w in zip(N.quantize_rows_asym(x, bits), C.quantize_rows_asym(x, bits), "qdz"):
            _same(a, b, f"asym{bits} {w}")


@pytest.mark.parametrize("N_,K,M", [(97, 640, 3), (256, 512, 1)])
def test_sign_formats_agree(N_, K, M):
    inp = I.layer_inputs("ternary", N_, K, M, seed=N_, lora_rank=32)
    W, x = inp["W"], inp["x"]
    a, b = N.bitnet_pack(W), C.bitnet_pack(W)
    _same(a["B"], b["B"], "bitnet B")
    _same(a["alpha"], b["alpha"], "alpha")
    ra, rb = N.bitnet_layer(a, x), C.bitnet_layer(b, x)
    _same(ra["acc"], rb["acc"], "bitnet acc")
    _close64(ra["y"], rb["y"], "bitnet y")
    a = N.ternary_pack(W, inp["lora_A"], inp["lora_B"], 0.1)
    b = C.ternary_pack(W, inp["lora_A"], inp["lora_B"], 0.1)
    for k in ("T", "gamma_w", "A", "B"):
        _same(a[k], b[k], f"ternary {k}")
    ra, rb = N.ternary_layer(a, x), C.ternary_layer(b, x)
    _same(ra["acc"], rb["acc"], "ternary acc")
    for k in ("y", "y_ternary", "y_lora"):
        _close64(ra[k], rb[k], f"ternary {k}")


@pytest.mark.parametrize("P", [2, 3])
def test_rabit_agrees(P):
    inp = I.layer_inputs("rabit3", 256, 512, 2, seed=P)
    W, x = inp["W"], inp["x"]
    hs = [np.ones(512, np.float32), inp["h2"], inp["h3"]][:P]
    a, b = N.rabit_pack_paths(W, hs), C.rabit_pack_paths(W, hs)
    for k in ("B", "g", "h"):
        _same(a[k], b[k], f"paths {k}")
    _close64(N.rabit_weight_paths(a), C.rabit_weight_paths(b), "W_hat", rel=1e-15)
    if P == 2:
        a2, b2 = N.rabit_pack(W, hs[1]), C.rabit_pack(W, hs[1])
        for k in a2:
            _same(a2[k], b2[k], f"rabit {k}")
        ra, rb = N.rabit_layer(a2, x), C.rabit_layer(b2, x)
        for k in ("y", "acc1", "acc2"):
            _close64(ra[k], rb[k], f"rabit {k}")


@pytest.mark.parametrize("rounds", [1, 3, 20])
def test_rabit_svid_agrees(rounds):
    W = I.weights(40, 384, seed=rounds)
    a, b = N.rabit_pack_svid(W, rounds), C.rabit_pack_svid(W, rounds)
    for k in a:
        _same(a[k], b[k], f"svid {k}")
    assert N.rabit_recon_error(a, W) == pytest.approx(C.rabit_recon_error(b, W), rel=1e-12)


@pytest.mark.parametrize("w,a", [(2, 8), (4, 4), (6, 6), (8, 8), (1, 1), (3, 5)])
def test_abq_agrees(w, a):
    inp = I.layer_inputs("abq", 97, 640, 9, seed=w * 10 + a)
    W, x = inp["W"], inp["x"]
    pa, pb = N.abq_pack(W, w), C.abq_pack(W, w)
    for k in ("Q", "delta", "z"):
        _same(pa[k], pb[k], f"abq {k}")
    ra, rb = N.abq_layer(pa, x, a), C.abq_layer(pb, x, a)
    for k in ("Qx", "delta_x", "z_x", "I"):
        _same(ra[k], rb[k], f"abq layer {k}")
    _close64(ra["y"], rb["y"], "abq y")


def test_abq_balanced_and_compensated_agree():
    inp = I.layer_inputs("abq", 97, 640, 1, seed=3)
    W = inp["W"]
    ca, cb = I.compensation_vectors(97, 640, seed=3)
    for k in ("Q", "delta", "z"):
        _same(N.abq_pack_balanced(W)[k], C.abq_pack_balanced(W)[k], f"W2* {k}")
    _same(N.abq_compensated_weights(W, ca, cb), C.abq_compensated_weights(W, ca, cb), "W + a b^T")
    for w, bal in ((2, False), (8, False), (3, True)):
        a, b = N.abq_pack_compensated(W, ca, cb, w, bal), C.abq_pack_compensated(W, ca, cb, w, bal)
        for k in ("Q", "delta", "z"):
            _same(a[k], b[k], f"compensated w{w} {k}")


def test_bvsr_agrees():
    inp = I.layer_inputs("bvsr", 64, 512, 3, seed=5)
    W, x = inp["W"], inp["x"]
    ta, tb = N.bvsr_set_table(W), C.bvsr_set_table(W)
    _same(ta, tb, "table")
    _same(N.bvsr_points(ta), C.bvsr_points(tb), "points")
    rows = np.array([0, 1, 17, 63])
    a, b = N.bvsr_pack(W, rows=rows), C.bvsr_pack(W, rows=rows)
    _same(a["codes"], b["codes"], "codes")
    _same(a["sets"], b["sets"], "sets")
    ra, rb = N.bvsr_layer(a["codes"], a["sets"], a["table"], x), C.bvsr_layer(b["codes"], b["sets"], b["table"], x)
    _same(ra["acc"], rb["acc"], "bvsr acc")
    _close64(ra["y"], rb["y"], "bvsr y")


def test_bitplane_identities_agree():
    rng = np.random.default_rng(0)
    for w, a in ((1, 8), (2, 8), (4, 4), (8, 8)):
        qw = rng.integers(0, 1 << w, 100)
        qx = rng.integers(-(1 << (a - 1)), 1 << (a - 1), 100)
        assert N.bitplane_dot(qw, w, False, qx, a, True) == C.bitplane_dot(qw, w, False, qx, a, True)
    s1, s2 = rng.choice([-1, 1], 77), rng.choice([-1, 1], 77)
    assert N.xnor_popcount_dot(s1, s2) == C.xnor_popcount_dot(s1, s2)


def test_cpp_reference_runs_on_several_threads_with_the_same_results():
    """OpenMP splits rows between threads; every row's arithmetic is the same on any count."""
    inp = I.layer_inputs("bvsr", 64, 512, 3, seed=8)
    n0 = C.threads()
    try:
        C.set_threads(1)
        one = C.bvsr_pack(inp["W"], rows=np.arange(16))
        y1 = C.bitnet_layer(C.bitnet_pack(inp["W"]), inp["x"])["y"]
        C.set_threads(max(2, n0))
        many = C.bvsr_pack(inp["W"], rows=np.arange(16))
        ym = C.bitnet_layer(C.bitnet_pack(inp["W"]), inp["x"])["y"]
    finally:
        C.set_threads(n0)
    _same(one["codes"], many["codes"], "codes")
    _same(one["sets"], many["sets"], "sets")
    _same(y1, ym, "y")


@pytest.mark.parametrize("rounds", [0, 1, 4])
def test_bvsr_cluster_table_agrees(rounds):
    W = I.weights(48, 1024, seed=30 + rounds)
    a, b = N.bvsr_cluster_table(W, rounds), C.bvsr_cluster_table(W, rounds)
    for k in ("table", "family", "assign", "centroids"):
        _same(a[k], b[k], f"cluster {k}")
    pa, pb = N.bvsr_pack(W, rows=np.array([0, 47]), cluster_rounds=rounds), C.bvsr_pack(W, rows=np.array([0, 47]), cluster_rounds=rounds)
    _same(pa["codes"], pb["codes"], "codes")
    _same(pa["sets"], pb["sets"], "sets")
