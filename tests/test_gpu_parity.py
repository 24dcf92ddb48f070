"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Small cases span several 16-row blocks and 256-k tiles with ragged tails
(N not a multiple of 16, K not a multiple of 256) and several token groups;
the oracle checks every output. Integer accumulators must be bit-exact;
y must satisfy max|y - y_ref| <= 1e-3 (||y_ref||_inf + 1e-6).
"""
import numpy as np
import pytest

import bq_inputs as I
from oracle import cref as O
from tests.parity_util import (GpuLayer, assert_codes_near_tie, assert_y_close, check_act, oracle_layer,
                               oracle_pack, rabit_near, ternary_near, to_dev_bf16, to_dev_f32, torch_mods,
                               ulp_diff)

pytestmark = pytest.mark.gpu

# ragged N and K; (40, 2560) leaves some warps without k-tiles, (24, 6144) streams in chunks
SMALL = [(16, 256), (50, 384), (97, 640), (33, 128), (40, 2560), (24, 6144)]
ABQ_WA = [(2, 8), (4, 4), (6, 6), (8, 8), (1, 3), (3, 5), (5, 2), (7, 7), (1, 1), (8, 1)]


def _paths_of(d):
    """(B [P,N,K], g [P,N], h [P,K]) of a two-path dict (B1, B2, ...) or a P-path one (B, g, h)."""
    if "B1" in d:
        return (np.stack([d["B1"], d["B2"]]), np.stack([d["g1"], d["g2"]]), np.stack([d["h1"], d["h2"]]))
    return np.asarray(d["B"]), np.asarray(d["g"]), np.asarray(d["h"])


def _rabit_parity(p, ref, W, what):
    """Signs, g and h of a RaBiT pack against the oracle, with the near-tie rule: every sign is
    compared; path 1 (sign(W)) must match exactly; a later path's sign may differ only where
    its residual is within a few ulps of 0 or where the previous path's sign already differed.
    g_p is within 1 ulp where the row's earlier scales agree exactly and within 2 where one of
    them differs (the difference reaches g_p through the residual). Then the GPU's signs must be
    exactly the recursion applied to the GPU's own scales."""
    Bg, gg, hg = _paths_of(p)
    Br, gr, hr = _paths_of(ref)
    P = Br.shape[0]
    assert np.all(hg[0] == 1) and np.array_equal(hg[1:], hr[1:])
    assert np.array_equal(Bg[0], Br[0]), f"{what}: sign(W) differs"
    same = np.ones(Bg.shape[1], bool)
    for q in range(P):
        assert np.all(ulp_diff(gg[q], gr[q]) <= np.where(same, 1, 2)), f"{what}: g{q + 1}"
        same &= gg[q] == gr[q]
    near = rabit_near(W, Br, gr, hr)
    prev = np.zeros(Bg.shape[1:], bool)
    for q in range(1, P):
        assert_codes_near_tie(Bg[q], Br[q], near[q - 1] | prev, f"{what} B{q + 1}")
        prev |= Bg[q] != Br[q]
    R = np.asarray(W, np.float64).copy()
    for q in range(P):
        assert np.array_equal(Bg[q], np.where(R >= 0, 1, -1)), f"{what}: B{q + 1} is not sign of the GPU's residual"
        R = R - (gg[q].astype(np.float64)[:, None] * Bg[q]) * hg[q].astype(np.float64)[None, :]


def _ternary_parity(p, ref, W, what):
    """gamma_W within 1 ulp; every code compared under the near-tie rule (W / gamma at +-0.5);
    and the GPU's codes are exactly clamp(rn(W / gamma_gpu), -1, 1) of its own gamma."""
    assert ulp_diff(p["gamma_w"], ref["gamma_w"]) <= 1
    assert_codes_near_tie(p["T"], ref["T"], ternary_near(W, ref["gamma_w"]), what)
    own = np.clip(np.rint((np.asarray(W, np.float32) / np.float32(p["gamma_w"])).astype(np.float32)), -1, 1)
    assert np.array_equal(p["T"], own.astype(p["T"].dtype)), f"{what}: codes are not those of the GPU's gamma"


def _pack_parity(gl: GpuLayer, fmt, w_bits=0):
    p = gl.read()
    ref = oracle_pack(fmt, gl.inp, w_bits)
    W = gl.inp["W"]
    if fmt in ("rabit", "rabit3"):
        _rabit_parity(p, ref, W, fmt)
    elif fmt == "bitnet":
        assert np.array_equal(p["B"], ref["B"])
        assert ulp_diff(p["alpha"], ref["alpha"]) <= 1
    elif fmt == "ternary":
        _ternary_parity(p, ref, W, "ternary T")
        assert p["field_max"] <= 2
        assert np.array_equal(p["A"], ref["A"]) and np.array_equal(p["B"], ref["B"])
        assert p["lora_alpha"] == np.float32(0.1)
    elif fmt == "abq":
        assert np.array_equal(p["delta"], ref["delta"])
        assert np.array_equal(p["z"], ref["z"])
        assert np.array_equal(p["Q"], ref["Q"])
        assert np.array_equal(p["S_w"], ref["Q"].sum(1))
    elif fmt == "bvsr":
        assert np.array_equal(p["table"], ref["table"])
        assert np.array_equal(p["sets"], ref["sets"])
        assert np.array_equal(p["codes"], ref["codes"])
    return p


def _layer_parity(gl: GpuLayer, p, fmt, a_bits=0):
    r = oracle_layer(fmt, p, gl.inp["x"], a_bits)
    if gl.acc_h is not None:
        assert np.array_equal(gl.acc_h, r["acc"]), "integer accumulator differs"
    assert_y_close(gl.y_h, r["y"], fmt)


@pytest.mark.parametrize("N,K", SMALL)
@pytest.mark.parametrize("fmt", ["bitnet", "ternary", "bvsr", "rabit"])
@pytest.mark.parametrize("M", [1, 3, 9])
def test_small_parity(fmt, N, K, M):
    if fmt == "rabit" and M > 3:
        M = 2
    gl = GpuLayer(fmt, N, K, M, seed=N + K + M)
    p = _pack_parity(gl, fmt)
    check_act(gl)
    _layer_parity(gl, p, fmt)


@pytest.mark.parametrize("wa", ABQ_WA)
@pytest.mark.parametrize("N,K,M", [(50, 384, 1), (97, 640, 9), (16, 256, 8), (64, 6400, 2)])
def test_small_parity_abq(wa, N, K, M):
    w, a = wa
    gl = GpuLayer("abq", N, K, M, seed=w * 10 + a, w_bits=w, a_bits=a)
    p = _pack_parity(gl, "abq", w)
    check_act(gl)
    _layer_parity(gl, p, "abq", a)


@pytest.mark.parametrize("fmt", ["bitnet", "ternary", "bvsr"])
@pytest.mark.parametrize("N,K", [(97, 640), (40, 2560)])
def test_max_tokens(fmt, N, K):
    """M = 64, the largest batch: eight token groups of eight, ragged N and K; act + gemm and
    the fused call agree bit for bit (checked in GpuLayer) and match the oracle."""
    gl = GpuLayer(fmt, N, K, 64, seed=N + K)
    p = _pack_parity(gl, fmt)
    check_act(gl)
    _layer_parity(gl, p, fmt)


@pytest.mark.parametrize("N,K,M", [(97, 640, 12), (50, 2560, 16), (40, 5120, 13), (33, 128, 16)])
def test_bvsr_two_token_groups(N, K, M):
    """BVSR from an act buffer holds up to 16 tokens a CTA as two 8-token MMA groups on each
    decoded weight fragment: second groups partly and fully filled, ragged N. Below 16 tokens
    the fused call (at most 8 tokens a CTA) equals act + gemm (two groups) bit for bit, which
    GpuLayer checks; both match the oracle."""
    torch, bq = torch_mods()
    gl = GpuLayer("bvsr", N, K, M, seed=N + K + M)
    assert bq.bq_linear_plan(gl.ql.layer, M, False)["tokens_per_cta"] == M
    p = _pack_parity(gl, "bvsr")
    check_act(gl)
    _layer_parity(gl, p, "bvsr")


@pytest.mark.parametrize("N,K", SMALL)
@pytest.mark.parametrize("M", [1, 3])
def test_small_parity_rabit3(N, K, M):
    """Three residual paths: pack (signs, g, h), act (h_p x) and layer (fused and not)."""
    gl = GpuLayer("rabit3", N, K, M, seed=N + K + M)
    p = _pack_parity(gl, "rabit3")
    check_act(gl)
    _layer_parity(gl, p, "rabit3")


def test_full_rabit3():
    gl = GpuLayer("rabit3", 256, 512, 1)
    p = _pack_parity(gl, "rabit3")
    check_act(gl)
    _layer_parity(gl, p, "rabit3")


def test_rabit3_constant_magnitude_rows():
    """|W| = c on a row: R_1 = 0 exactly, so paths 2 and 3 get sign +1 and g = 0, and the
    layer is W x itself."""
    inp = I.layer_inputs("rabit3", 40, 384, 2, seed=9)
    c = np.float32(0.03125)
    inp["W"] = np.where(inp["W"] >= 0, c, -c).astype(np.float32)
    gl = GpuLayer("rabit3", 40, 384, 2, inputs=inp)
    p = gl.read()
    assert np.all(p["g"][0] == c) and np.all(p["g"][1:] == 0) and np.all(p["B"][1:] == 1)
    assert_y_close(gl.y_h, inp["x"].astype(np.float64) @ inp["W"].astype(np.float64).T, "rabit3 |W| = c")


@pytest.mark.parametrize("fmt", ["bitnet", "ternary", "bvsr", "rabit", "rabit3", "abq"])
def test_zero_activations(fmt):
    gl = GpuLayer(fmt, 40, 256, 2, w_bits=4, a_bits=4, nullify_x=True)
    check_act(gl)
    if fmt == "ternary":
        assert np.all(gl.y_h == 0)   # SiLU(0) = 0, gamma_x = 0
    elif fmt == "abq":
        p = gl.read()
        _layer_parity(gl, p, "abq", 4)
    else:
        assert np.all(gl.y_h == 0)


def test_ternary_m_values_and_lora():
    for M in (1, 4, 16):
        gl = GpuLayer("ternary", 2048, 2048, M, seed=M)
        p = _pack_parity(gl, "ternary")
        check_act(gl)
        _layer_parity(gl, p, "ternary")


@pytest.mark.parametrize("rank", [8, 64])
@pytest.mark.parametrize("N,K,M", [(97, 640, 1), (40, 2560, 9)])
def test_ternary_lora_ranks(rank, N, K, M):
    """The smallest and the largest correction rank (steps of 8 up to 64), ragged shapes."""
    gl = GpuLayer("ternary", N, K, M, seed=rank + N, lora_rank=rank)
    p = _pack_parity(gl, "ternary")
    assert p["A"].shape == (K, rank) and p["B"].shape == (rank, N)
    check_act(gl)
    _layer_parity(gl, p, "ternary")


def test_outlier_heavy_activations():
    inp = I.layer_inputs("bitnet", 64, 512, 3, seed=4)
    inp["x"] = I.bf16_round(inp["x"] * np.where(np.arange(512) % 37 == 0, 300.0, 1.0)[None, :])
    gl = GpuLayer("bitnet", 64, 512, 3, inputs=inp)
    check_act(gl)
    _layer_parity(gl, gl.read(), "bitnet")


def test_n_equals_one_and_min_k():
    for fmt in ("bitnet", "ternary", "bvsr", "abq", "rabit", "rabit3"):
        gl = GpuLayer(fmt, 1, 128, 1, w_bits=2, a_bits=8)
        p = _pack_parity(gl, fmt, 2)
        _layer_parity(gl, p, fmt, 8)


def test_exact_zero_weights_are_plus_one():
    inp = I.layer_inputs("bitnet", 16, 256, 1, seed=3)
    inp["W"][:, ::5] = 0.0
    inp["W"][3, ::7] = -0.0
    gl = GpuLayer("bitnet", 16, 256, 1, inputs=inp)
    p = gl.read()
    assert np.all(p["B"][:, ::5][inp["W"][:, ::5] == 0] == 1)
    _layer_parity(gl, p, "bitnet")


# ------------------------------------------------------------------ full sizes
def _sample_blocks(N, n=6, seed=0):
    RB = (N + 15) // 16
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, RB - 1], rng.choice(RB, size=min(n, RB), replace=False)]))


def _full_size(fmt, N, K, M, w_bits=0, a_bits=0):
    gl = GpuLayer(fmt, N, K, M, w_bits=w_bits, a_bits=a_bits)
    rbs = _sample_blocks(N)
    p = gl.read(rbs)
    rows = p["rows"]
    keep = rows < N
    rows = rows[keep]
    for key in ("B", "T", "Q", "codes", "sets", "delta", "z", "S_w"):
        if key in p:
            p[key] = p[key][keep]
    if "B" in p and fmt == "ternary":
        p["B"] = p["B"][:, keep]
    ref = oracle_pack(fmt, gl.inp, w_bits, rows=rows)
    if fmt == "bitnet":
        assert np.array_equal(p["B"], ref["B"]) and ulp_diff(p["alpha"], ref["alpha"]) <= 1
    elif fmt == "ternary":
        _ternary_parity(p, ref, gl.inp["W"][rows], f"ternary T {N}x{K} (sampled rows)")
    elif fmt == "abq":
        assert np.array_equal(p["Q"], ref["Q"]) and np.array_equal(p["delta"], ref["delta"])
        assert np.array_equal(p["z"], ref["z"])
    elif fmt == "bvsr":
        assert np.array_equal(p["table"], ref["table"])
        assert np.array_equal(p["sets"], ref["sets"]) and np.array_equal(p["codes"], ref["codes"])
    check_act(gl)
    r = oracle_layer(fmt, p, gl.inp["x"], a_bits)
    if gl.acc_h is not None:
        assert np.array_equal(gl.acc_h[:, rows], r["acc"])
    assert_y_close(gl.y_h[:, rows], r["y"], f"{fmt} {N}x{K}")
    assert np.all(np.isfinite(gl.y_h))


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_full_bitnet(N, K):
    _full_size("bitnet", N, K, 1)


@pytest.mark.parametrize("N,K", [(5120, 5120), (13824, 5120), (5120, 13824)])
def test_full_bvsr(N, K):
    _full_size("bvsr", N, K, 1)


@pytest.mark.parametrize("wa", [(2, 8), (4, 4), (6, 6), (8, 8)])
@pytest.mark.parametrize("N", [4096, 11008])
@pytest.mark.parametrize("M", [1, 8, 64])
def test_full_abq(wa, N, M):
    _full_size("abq", N, 4096, M, wa[0], wa[1])


def test_full_rabit():
    gl = GpuLayer("rabit", 256, 512, 1)
    p = _pack_parity(gl, "rabit")
    check_act(gl)
    _layer_parity(gl, p, "rabit")


# ------------------------------------------------------------------ device checks
def test_act_buffer_mismatch_is_reported():
    """An act buffer quantized for M=2 used with M=1: the kernel sees the header
    mismatch, writes nothing and raises the device error word."""
    from tests.parity_util import torch_mods
    torch, bq = torch_mods()
    gl = GpuLayer("bitnet", 32, 256, 2)
    y = torch.full((1, 32), 7.0, device="cuda")
    bq.bq_gemv(gl.ql.layer, gl.ql.act_buffer(2), y)
    with pytest.raises(bq.BQError) as e:
        bq.bq_device_check()
    assert e.value.status == bq.BQ_ERR_DEVICE_CHECK
    assert torch.all(y == 7.0)
    bq.bq_device_check()   # the word was cleared


@pytest.mark.parametrize("fmt,kw_act,kw_layer", [("ternary", dict(lora_rank=8), dict(lora_rank=32)),
                                                  ("abq", dict(w_bits=4, a_bits=4), dict(w_bits=4, a_bits=8))])
def test_act_buffer_of_another_layer_config_is_refused(fmt, kw_act, kw_layer):
    """An act buffer quantized for a layer of the same format, N, K and M but another correction
    rank (its sections are smaller) or activation width: the kernel reads only its header,
    writes nothing and raises the device error word."""
    from tests.parity_util import torch_mods
    torch, bq = torch_mods()
    src = GpuLayer(fmt, 32, 256, 1, **kw_act)
    dst = GpuLayer(fmt, 32, 256, 1, **kw_layer)
    y = torch.full((1, 32), 7.0, device="cuda")
    bq.bq_gemv(dst.ql.layer, src.ql.act_buffer(1), y)
    with pytest.raises(bq.BQError) as e:
        bq.bq_device_check()
    assert e.value.status == bq.BQ_ERR_DEVICE_CHECK
    assert torch.all(y == 7.0)
    bq.bq_device_check()


@pytest.mark.parametrize("M_act,a_act", [(17, 8), (20, 4), (64, 8)])
def test_tensor_core_gemm_refuses_a_mismatched_act_buffer(M_act, a_act):
    """The tensor-core GEMM (ABQ, 20 tokens) given an act buffer made for fewer or more tokens
    or another activation width: it reads nothing past the header (no code copy, no token
    words), writes nothing and raises the device error word; the next good call is exact."""
    from tests.parity_util import torch_mods
    torch, bq = torch_mods()
    src = GpuLayer("abq", 200, 512, M_act, seed=3, w_bits=8, a_bits=a_act)
    dst = GpuLayer("abq", 200, 512, 20, seed=4, w_bits=8, a_bits=8)
    y = torch.full((20, 200), 7.0, device="cuda")
    bq.bq_gemm(dst.ql.layer, src.ql.act_buffer(M_act), 20, y)
    with pytest.raises(bq.BQError) as e:
        bq.bq_device_check()
    assert e.value.status == bq.BQ_ERR_DEVICE_CHECK
    assert torch.all(y == 7.0)
    bq.bq_gemm(dst.ql.layer, dst.ql.act_buffer(20), 20, y)
    torch.cuda.synchronize()
    bq.bq_device_check()
    assert np.array_equal(y.cpu().numpy(), dst.y_h)


# ------------------------------------------------------------------ grouped layers sharing x
@pytest.mark.parametrize("fmt,Ns,K,M,wa", [("bitnet", (64, 97, 40), 512, 1, (1, 8)),
                                           ("bitnet", (4096, 4096, 4096), 4096, 1, (1, 8)),
                                           ("bitnet", (33, 16), 1280, 9, (1, 8)),
                                           ("abq", (50, 33), 384, 9, (4, 4)),
                                           ("abq", (11008, 11008), 4096, 1, (2, 8)),
                                           ("ternary", (48, 80, 16, 31), 640, 3, (2, 8))])
def test_linear_group_equals_separate_calls(fmt, Ns, K, M, wa):
    """One grouped launch gives, bit for bit, what separate bq_linear calls give (each of
    which the other tests hold to the oracle); the first member is also checked against the
    oracle directly."""
    from tests.parity_util import torch_mods
    torch, bq = torch_mods()
    w, a = wa
    x = to_dev_bf16(I.activations(M, K, seed=11))
    qls, inps = [], []
    for i, N in enumerate(Ns):
        inp = I.layer_inputs(fmt, N, K, M, seed=20 + i, lora_rank=0)
        kw = dict(w_bits=w, a_bits=a) if fmt == "abq" else {}
        qls.append(bq.QuantLinear(fmt, to_dev_f32(inp["W"]), **kw))
        inps.append(inp)
    ys = [torch.full((M, N), float("nan"), device="cuda") for N in Ns]
    accs = [torch.full((M, N), -(1 << 62), dtype=torch.int64, device="cuda") for N in Ns]
    bq.bq_linear_group([q.layer for q in qls], x, M, ys, accs)
    for q, y, acc, N in zip(qls, ys, accs, Ns):
        y1 = torch.full((M, N), float("nan"), device="cuda")
        a1 = torch.full((M, N), -(1 << 62), dtype=torch.int64, device="cuda")
        q.linear(x, y1, a1)
        torch.cuda.synchronize()
        assert torch.equal(acc, a1)
        assert torch.equal(y, y1)
    bq.bq_device_check()
    from tests.parity_util import L as layout
    p = layout.read_packed(qls[0].packed.cpu().numpy().tobytes())
    xh = I.activations(M, K, seed=11)
    r = oracle_layer(fmt, p, xh, a)
    assert np.array_equal(accs[0].cpu().numpy(), r["acc"])
    assert_y_close(ys[0].cpu().numpy(), r["y"], f"{fmt} group member 0")


# ------------------------------------------------------------------ long rows (K up to the limit)
@pytest.mark.parametrize("fmt,N,K,M,wa", [("bitnet", 32, 65536, 1, (1, 8)), ("bitnet", 20, 40960, 3, (1, 8)),
                                           ("abq", 24, 33024, 2, (4, 4)), ("bvsr", 16, 33024, 1, (4, 8)),
                                           ("ternary", 16, 36864, 2, (2, 8))])
def test_long_rows(fmt, N, K, M, wa):
    """K past what the fused staging holds in registers (32768 for one token): the fused call
    re-reads x and must still equal the unfused path and the oracle."""
    w, a = wa
    gl = GpuLayer(fmt, N, K, M, seed=K % 97, w_bits=w, a_bits=a)
    p = _pack_parity(gl, fmt, w)
    check_act(gl)
    _layer_parity(gl, p, fmt, a)


# ------------------------------------------------------------------ RaBiT SVID initialisation
@pytest.mark.parametrize("N,K,rounds", [(40, 384, 1), (40, 384, 20), (256, 512, 20), (17, 256, 3)])
def test_rabit_svid_pack_and_layer(N, K, rounds):
    """The pack's iterative residual SVID gives the oracle's signs, g and h bit for bit (same
    float64 operations in the same order); the layer on them matches the oracle's layer."""
    from tests.parity_util import L as layout, torch_mods
    torch, bq = torch_mods()
    W = I.weights(N, K, seed=N + rounds)
    x = I.activations(2, K, seed=5)
    ql = bq.QuantLinear("rabit", to_dev_f32(W), rabit_svid_rounds=rounds)
    p = layout.read_packed(ql.packed.cpu().numpy().tobytes())
    ref = O.rabit_pack_svid(W, rounds)
    for key in ("B1", "B2"):
        assert np.array_equal(p[key], ref[key]), key
    for key in ("g1", "g2", "h1", "h2"):
        assert np.array_equal(p[key], ref[key]), key
    xd = to_dev_bf16(x)
    y = torch.full((2, N), float("nan"), device="cuda")
    ql.linear(xd, y)
    y2 = torch.full((2, N), float("nan"), device="cuda")
    ql.forward(xd, y2)
    torch.cuda.synchronize()
    bq.bq_device_check()
    r = O.rabit_layer(ref, x)
    assert_y_close(y.cpu().numpy(), r["y"], "rabit svid fused")
    assert_y_close(y2.cpu().numpy(), r["y"], "rabit svid act+gemv")
    assert O.rabit_recon_error(ref, W) <= O.rabit_recon_error(O.rabit_pack(W, np.ones(K, np.float32)), W)


# ------------------------------------------------------------------ maximum N
def test_max_rows_abq():
    """N = 2^20 rows (the limit), K = 128, M = 2: ABQ's per-row codes let sampled rows be
    checked against the oracle. W is drawn on the device; only the sampled rows come back."""
    from tests.parity_util import L as layout, torch_mods
    torch, bq = torch_mods()
    N, K, M = 1 << 20, 128, 2
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    W = torch.randn(N, K, device="cuda", generator=g) * 0.02
    ql = bq.QuantLinear("abq", W, w_bits=2, a_bits=8)
    x = I.activations(M, K, seed=4)
    y = torch.full((M, N), float("nan"), device="cuda")
    acc = torch.full((M, N), -(1 << 62), dtype=torch.int64, device="cuda")
    ql.linear(to_dev_bf16(x), y, acc)
    torch.cuda.synchronize()
    bq.bq_device_check()
    rbs = np.array([0, 1, 777, 40000, (N // 16) - 1])
    p = layout.read_packed(ql.packed.cpu().numpy().tobytes(), rbs)
    rows = p["rows"]
    Wh = W[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    ref = O.abq_pack(Wh, 2)
    assert np.array_equal(p["Q"], ref["Q"]) and np.array_equal(p["delta"], ref["delta"])
    r = O.abq_layer(p, x, 8)
    assert np.array_equal(acc.cpu().numpy()[:, rows], r["I"])
    assert_y_close(y.cpu().numpy()[:, rows], r["y"], "abq N = 2^20")
    assert bool(torch.isfinite(y).all())


# ------------------------------------------------------------------ ABQ bit balance (W2*)
@pytest.mark.parametrize("N,K,M", [(50, 384, 1), (97, 640, 9), (4096, 4096, 1)])
def test_abq_bit_balance(N, K, M):
    """W2*: the pack's symmetric five-level codes, Delta and z equal the oracle's; the layer (the
    ABQ w = 3 kernels) matches the oracle's integer accumulator exactly and y within tolerance."""
    from tests.parity_util import L as layout, torch_mods
    torch, bq = torch_mods()
    inp = I.layer_inputs("abq", N, K, M, seed=N + K)
    W, x = inp["W"], inp["x"]
    ql = bq.QuantLinear("abq", to_dev_f32(W), w_bits=3, a_bits=8, abq_bit_balance=1)
    p = layout.read_packed(ql.packed.cpu().numpy().tobytes())
    ref = O.abq_pack_balanced(W)
    assert np.array_equal(p["Q"], ref["Q"]) and np.array_equal(p["delta"], ref["delta"])
    assert np.array_equal(p["z"], ref["z"]) and np.array_equal(p["S_w"], ref["Q"].sum(1))
    xd = to_dev_bf16(x)
    for run in (ql.linear, ql.forward):
        y = torch.full((M, N), float("nan"), device="cuda")
        acc = torch.full((M, N), -(1 << 62), dtype=torch.int64, device="cuda")
        run(xd, y, acc)
        torch.cuda.synchronize()
        r = O.abq_layer(p, x, 8)
        assert np.array_equal(acc.cpu().numpy(), r["I"])
        assert_y_close(y.cpu().numpy(), r["y"], "abq W2*")
    bq.bq_device_check()


# ------------------------------------------------------------------ ABQ distribution compensation
@pytest.mark.parametrize("w,a,balanced", [(2, 8, False), (4, 4, False), (8, 8, False), (3, 8, True)])
@pytest.mark.parametrize("N,K,M", [(50, 384, 1), (97, 640, 9), (4096, 4096, 1)])
def test_abq_compensation(w, a, balanced, N, K, M):
    """W + a b^T quantized in the pack: codes, Delta, z and S_w equal the oracle's bit for bit;
    the unchanged ABQ layer then matches the oracle's integer accumulator exactly."""
    from tests.parity_util import L as layout, torch_mods
    torch, bq = torch_mods()
    inp = I.layer_inputs("abq", N, K, M, seed=N + w)
    W, x = inp["W"], inp["x"]
    ca, cb = I.compensation_vectors(N, K, seed=N + w)
    ql = bq.QuantLinear("abq", to_dev_f32(W), w_bits=w, a_bits=a, abq_bit_balance=int(balanced),
                        abq_comp_a=to_dev_f32(ca), abq_comp_b=to_dev_f32(cb))
    p = layout.read_packed(ql.packed.cpu().numpy().tobytes())
    ref = O.abq_pack_compensated(W, ca, cb, w, balanced)
    assert np.array_equal(p["delta"], ref["delta"]) and np.array_equal(p["z"], ref["z"])
    assert np.array_equal(p["Q"], ref["Q"]) and np.array_equal(p["S_w"], ref["Q"].sum(1))
    xd = to_dev_bf16(x)
    y = torch.full((M, N), float("nan"), device="cuda")
    acc = torch.full((M, N), -(1 << 62), dtype=torch.int64, device="cuda")
    ql.linear(xd, y, acc)
    torch.cuda.synchronize()
    r = O.abq_layer(p, x, a)
    assert np.array_equal(acc.cpu().numpy(), r["I"])
    assert_y_close(y.cpu().numpy(), r["y"], "abq compensated")
    bq.bq_device_check()


# ------------------------------------------------------------------ BVSR coefficient cache by clustering
@pytest.mark.parametrize("N,K,M,rounds", [(50, 384, 1, 1), (97, 640, 3, 4), (256, 2048, 1, 8), (5120, 5120, 1, 8)])
def test_bvsr_cluster_pack_and_layer(N, K, M, rounds):
    """The clustering reading of the coefficient cache: the pack's per-vector families, k-means
    centroids (exact integer sums, so the GPU's atomic order does not matter) and resulting
    table equal the C++ oracle's bit for bit, and so do the searched sets and codes (sampled row
    blocks at the full size); the layer on them matches the oracle."""
    from tests.parity_util import L as layout, torch_mods
    torch, bq = torch_mods()
    inp = I.layer_inputs("bvsr", N, K, M, seed=N + rounds)
    W, x = inp["W"], inp["x"]
    ql = bq.QuantLinear("bvsr", to_dev_f32(W), bvsr_cluster_rounds=rounds)
    rbs = None if N <= 256 else _sample_blocks(N, n=4, seed=rounds)
    p = layout.read_packed(ql.packed.cpu().numpy().tobytes(), rbs)
    rows = p["rows"][p["rows"] < N]
    ref = O.bvsr_pack(W, rows=rows, cluster_rounds=rounds)
    assert np.array_equal(p["table"], ref["table"])
    assert np.array_equal(p["sets"][:len(rows)], ref["sets"]) and np.array_equal(p["codes"][:len(rows)], ref["codes"])
    xd = to_dev_bf16(x)
    y = torch.full((M, N), float("nan"), device="cuda")
    acc = torch.full((M, N), -(1 << 62), dtype=torch.int64, device="cuda")
    ql.linear(xd, y, acc)
    torch.cuda.synchronize()
    bq.bq_device_check()
    r = O.bvsr_layer(ref["codes"], ref["sets"], ref["table"], x)
    assert np.array_equal(acc.cpu().numpy()[:, rows], r["acc"])
    assert_y_close(y.cpu().numpy()[:, rows], r["y"], f"bvsr clustered {N}x{K}")


# ------------------------------------------------------------------ ABQ on the tcgen05 tensor cores
@pytest.mark.parametrize("N,K,M,w,a", [(50, 384, 16, 8, 8), (128, 256, 17, 8, 8), (200, 640, 33, 8, 4),
                                       (300, 4096, 64, 8, 8), (16, 1280, 64, 8, 1), (97, 640, 48, 8, 6),
                                       (1000, 2048, 32, 8, 8), (97, 640, 16, 1, 8), (200, 384, 24, 2, 8),
                                       (50, 1280, 64, 3, 5), (130, 640, 40, 4, 4), (97, 256, 64, 5, 2),
                                       (300, 2048, 33, 6, 6), (64, 640, 17, 7, 7),
                                       (640, 2816, 64, 2, 8), (2560, 1792, 40, 4, 4),
                                       (64, 256, 16, 4, 4), (130, 20480, 20, 8, 8), (48, 16384, 32, 3, 6),
                                       (100, 1536, 24, 5, 5), (60, 1792, 48, 6, 4)])
def test_abq_tensor_cores(N, K, M, w, a):
    """ABQ with 16..64 tokens runs as a tcgen05 kind::i8 GEMM (the weight code bytes assembled
    from their bit-field streams while the operands are re-laid into canonical shared-memory
    layouts, accumulators in tensor memory), for every weight width 1..8: ragged row counts (a
    partial 128-row CTA), token counts rounded up to the MMA's N, several activation widths,
    k-tiles split over clusters of 1..8 CTAs (evenly and raggedly) whose partial products
    meet in distributed shared memory, one k-tile, and rows at and past the 16 K elements the
    act kernel keeps in shared memory.
    act + gemm and the fused call both take it and agree bit for bit (GpuLayer); the integer
    accumulators equal the oracle's, y within tolerance."""
    gl = GpuLayer("abq", N, K, M, seed=N + M + a, w_bits=w, a_bits=a)
    p = _pack_parity(gl, "abq", w)
    check_act(gl)
    _layer_parity(gl, p, "abq", a)
