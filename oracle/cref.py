"""The C++ reference (``oracle/bq_ref.cpp``) behind the same Python API as ``bq_oracle``.

Test infrastructure, like the rest of ``oracle/``: only the tests, the smoke check and the
bench's CPU legs import it. Every quantizer, search, sum and product runs in the C++ library;
this module only moves numpy arrays in and out and assembles the same dictionaries
``bq_oracle`` returns, so the pins and the parity tests can run against either implementation.
The library is built on first import if it is missing or older than its source.
"""
from __future__ import annotations

import ctypes

import numpy as np

from oracle import build_ref

_lib = ctypes.CDLL(build_ref.build())
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_F = ctypes.c_float
_D = ctypes.c_double

_SIGS = {
    "bqref_threads": (_I, []),
    "bqref_set_threads": (None, [_I]),
    "bqref_sign": (_I, [_P, _I64, _P]),
    "bqref_mean_abs": (_I, [_P, _I64, _P]),
    "bqref_bf16_round": (_I, [_P, _I64, _P]),
    "bqref_quantize_act_int8": (_I, [_P, _I64, _I64, _P, _P]),
    "bqref_dequant_act_int8": (_I, [_P, _P, _I64, _I64, _P]),
    "bqref_quantize_rows_asym": (_I, [_P, _I64, _I64, _I, _P, _P, _P]),
    "bqref_rabit_pack_paths": (_I, [_P, _I64, _I64, _I, _P, _P, _P]),
    "bqref_rabit_weight": (_I, [_P, _P, _P, _I, _I64, _I64, _P]),
    "bqref_rabit_recon_error": (_I, [_P, _P, _P, _P, _I, _I64, _I64, _P]),
    "bqref_rabit_pack_svid": (_I, [_P, _I64, _I64, _I, _P, _P, _P]),
    "bqref_rabit_layer": (_I, [_P, _P, _P, _I, _I64, _I64, _P, _I64, _P, _P]),
    "bqref_bitnet_pack": (_I, [_P, _I64, _I64, _P, _P]),
    "bqref_ternary_pack": (_I, [_P, _I64, _I64, _P, _P]),
    "bqref_bitnet_layer": (_I, [_P, _F, _I64, _I64, _P, _I64, _P, _P, _P, _P]),
    "bqref_lora_correction": (_I, [_P, _I64, _I64, _P, _P, _I, _I64, _F, _P]),
    "bqref_ternary_layer": (_I, [_P, _F, _P, _P, _I, _F, _I64, _I64, _P, _I64, _P, _P, _P, _P, _P, _P]),
    "bqref_abq_pack_balanced": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "bqref_abq_compensate": (_I, [_P, _P, _P, _I64, _I64, _P]),
    "bqref_abq_layer": (_I, [_P, _P, _P, _I64, _I64, _P, _I64, _I, _P, _P, _P, _P, _P]),
    "bqref_planes_of": (_I, [_P, _I64, _I, _P]),
    "bqref_plane_weights": (_I, [_I, _I, _P]),
    "bqref_bitplane_dot": (_I, [_P, _I, _I, _P, _I, _I, _I64, _P]),
    "bqref_xnor_popcount_dot": (_I, [_P, _P, _I64, _P]),
    "bqref_nearest_rank": (_I, [_P, _I64, _I64, _I64, _P]),
    "bqref_bvsr_set_table": (_I, [_P, _I64, _I64, _P]),
    "bqref_bvsr_points": (_I, [_P, _I, _P]),
    "bqref_bvsr_encode": (_I, [_P, _I64, _P, _P, _P]),
    "bqref_bvsr_layer": (_I, [_P, _P, _P, _I64, _I64, _P, _I64, _P, _P, _P, _P]),
    "bqref_bvsr_cluster_table": (_I, [_P, _I64, _I64, _I, _P, _P, _P, _P]),
    "bqref_decode_tokens_per_s": (_D, [_D, _D, _D]),
    "bqref_weight_bits_per_param": (_D, [_I, _I]),
    "bqref_silu": (_I, [_P, _I64, _P]),
    "bqref_tolerance_ok": (_I, [_P, _I64, _P, _I64, _D]),
}
for _n, (_r, _a) in _SIGS.items():
    _f = getattr(_lib, _n)
    _f.restype, _f.argtypes = _r, _a

BVSR_VEC = 32
BVSR_PLANES = 4
BVSR_RATIOS = (1.5, 2.0, 2.5, 3.0)
BVSR_GRID = 8
_FMT = {"rabit": 1, "bitnet": 2, "ternary": 3, "abq": 4, "bvsr": 5}


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a) -> int:
    return a.ctypes.data


def _ok(rc):
    if rc != 0:
        raise ValueError("the C++ reference refused its arguments")


def threads() -> int:
    """OpenMP threads the C++ reference uses. A run setting, not oracle arithmetic:
    parity unpinned, nothing to pin."""
    return _lib.bqref_threads()


def set_threads(n: int) -> None:
    """Set the OpenMP threads of the C++ reference (the bench times one core and all cores). A run
    setting: parity unpinned, nothing to pin."""
    _lib.bqref_set_threads(int(n))


# ------------------------------------------------------------------ helpers
def bf16_round(a) -> np.ndarray:
    """Nearest bfloat16, ties to even, as float32 ([HGF] §2.1 correction matrices stored in bf16).
    Pinned by tests (hand values: exact, tie to even down and up, above half)."""
    f = _c(a, np.float32)
    out = np.empty_like(f)
    _ok(_lib.bqref_bf16_round(_p(f), f.size, _p(out)))
    return out


def sign_pm1(v) -> np.ndarray:
    """sign(v) = +1 if v >= 0 else -1 ([BitNet] §2.1); sign(-0.0) = +1. Pinned by tests (zero,
    negative zero, tiny values)."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.int8)
    _ok(_lib.bqref_sign(_p(v), v.size, _p(out)))
    return out


def mean_abs_f32(a) -> np.float32:
    """mean |a|, float64 sum in index order, stored float32. Pinned by tests (BitNet alpha hand
    check; the SVID first g-step equals it)."""
    a = _c(a, np.float32)
    out = np.zeros(1, np.float32)
    _ok(_lib.bqref_mean_abs(_p(a), a.size, _p(out)))
    return out[0]


# ------------------------------------------------------------------ activations
def quantize_act_int8(x):
    """Per-token absmax int8 ([HGF] §1.2): gamma = max|x|, q = clamp(rn(x * (127 / gamma)), -127,
    127) in float32 ops; gamma = 0 gives q = 0. Returns (q, gamma). Pinned by tests (scale endpoints
    map to +-127, ties, zero rows)."""
    x = _c(x, np.float32)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    g = np.empty(M, np.float32)
    _ok(_lib.bqref_quantize_act_int8(_p(x), M, K, _p(q), _p(g)))
    return q, g


def dequant_act_int8(q, gamma) -> np.ndarray:
    """x_hat = q gamma / 127 in float64 ([HGF] §1.2). Pinned by tests (act endpoints and range)."""
    q, gamma = _c(q, np.int8), _c(gamma, np.float32)
    out = np.empty(q.shape, np.float64)
    _ok(_lib.bqref_dequant_act_int8(_p(q), _p(gamma), q.shape[0], q.shape[1], _p(out)))
    return out


def quantize_rows_asym(V, bits: int):
    """Per-row asymmetric uniform codes ([ABQ] §3.2 eq.(3), compensation off, no clipping): Delta =
    max(hi - lo, 1e-5) / (2^bits - 1), z = rn(-lo / Delta), q = clamp(rn(v / Delta) + z, 0, 2^bits -
    1), float32 ops. Returns (q, Delta, z). Pinned by tests (a hand example with a rounding tie,
    grid round trip)."""
    V = _c(V, np.float32)
    R, L = V.shape
    q = np.empty((R, L), np.int32)
    d = np.empty(R, np.float32)
    z = np.empty(R, np.int32)
    _ok(_lib.bqref_quantize_rows_asym(_p(V), R, L, int(bits), _p(q), _p(d), _p(z)))
    return q, d, z


# ------------------------------------------------------------------ RaBiT
def rabit_pack_paths(W, hs) -> dict:
    """Residual recursion with P paths ([RaBiT] §2.1-2.2; §6 read as a third path): B_p =
    sign(R_{p-1}), g_p = mean_k |R_{p-1}|, R_p = R_{p-1} - g_p B_p h_p. Returns B [P,N,K], g [P,N],
    h [P,K]. Pinned by tests (P = 2 equals rabit_pack bit for bit; each added path lowers the error
    by K g^2 per row; three-path hand example)."""
    W = _c(W, np.float32)
    N, K = W.shape
    h = _c(np.stack([np.asarray(v, np.float32) for v in hs]), np.float32)
    P = h.shape[0]
    B = np.empty((P, N, K), np.int8)
    g = np.empty((P, N), np.float32)
    _ok(_lib.bqref_rabit_pack_paths(_p(W), N, K, P, _p(h), _p(B), _p(g)))
    return dict(B=B, g=g, h=h)


def rabit_pack(W, h2) -> dict:
    """Two-path residual binarization ([RaBiT] §2.2): rabit_pack_paths with h1 = 1 and the given h2.
    Pinned by tests (recursion-order hand example, constant-magnitude rows)."""
    K = np.asarray(W).shape[1]
    r = rabit_pack_paths(W, [np.ones(K, np.float32), h2])
    return dict(B1=r["B"][0], B2=r["B"][1], g1=r["g"][0], g2=r["g"][1], h1=r["h"][0], h2=r["h"][1])


def _paths(p):
    if "B" in p and np.asarray(p["B"]).ndim == 3:
        return _c(p["B"], np.int8), _c(p["g"], np.float32), _c(p["h"], np.float32)
    return (_c(np.stack([p["B1"], p["B2"]]), np.int8), _c(np.stack([p["g1"], p["g2"]]), np.float32),
            _c(np.stack([p["h1"], p["h2"]]), np.float32))


def rabit_weight_paths(p) -> np.ndarray:
    """W_hat = sum_p g_p B_p h_p in float64 ([RaBiT] §2.1). Pinned by tests (P = 2 equals
    rabit_weight; the hand recursion's W_hat)."""
    B, g, h = _paths(p)
    P, N, K = B.shape
    out = np.empty((N, K), np.float64)
    _ok(_lib.bqref_rabit_weight(_p(B), _p(g), _p(h), P, N, K, _p(out)))
    return out


def rabit_weight(p) -> np.ndarray:
    """W_hat = g1 B1 h1 + g2 B2 h2 in float64 ([RaBiT] §2.1). Pinned by tests (RaBiT hand
    recursion, constant-magnitude rows reconstruct exactly)."""
    return rabit_weight_paths(p)


def rabit_recon_error(p, W) -> float:
    """||W - W_hat||^2 in float64. Pinned by tests (zero error on the exact signed rank-1 input to
    rounding)."""
    B, g, h = _paths(p)
    W = _c(W, np.float32)
    out = np.zeros(1, np.float64)
    _ok(_lib.bqref_rabit_recon_error(_p(W), _p(B), _p(g), _p(h), B.shape[0], B.shape[1], B.shape[2], _p(out)))
    return float(out[0])


def rabit_pack_svid(W, rounds: int = 20) -> dict:
    """[RaBiT] §2.3 iterative residual SVID, two paths, Gauss-Seidel (see the C++ source for the
    reading). Pinned by tests (exact signed rank-1 case, monotone error, least-squares step)."""
    W = _c(W, np.float32)
    N, K = W.shape
    B = np.empty((2, N, K), np.int8)
    g = np.empty((2, N), np.float32)
    h = np.empty((2, K), np.float32)
    _ok(_lib.bqref_rabit_pack_svid(_p(W), N, K, int(rounds), _p(B), _p(g), _p(h)))
    return dict(B1=B[0], B2=B[1], g1=g[0], g2=g[1], h1=h[0], h2=h[1])


def rabit_layer(p, x) -> dict:
    """y = W_hat x in float64 with x unquantized ([RaBiT] §3.2 applies signs to the input), and
    acc_p = sum_k B_p h_p x per path. Pinned by tests (the layer equals the sum of the two sign
    paths)."""
    B, g, h = _paths(p)
    x = _c(x, np.float32)
    P, N, K = B.shape
    M = x.shape[0]
    y = np.empty((M, N), np.float64)
    acc = np.empty((P, M, N), np.float64)
    _ok(_lib.bqref_rabit_layer(_p(B), _p(g), _p(h), P, N, K, _p(x), M, _p(y), _p(acc)))
    out = dict(y=y, acc=acc)
    for q in range(P):
        out[f"acc{q + 1}"] = acc[q]
    return out


# ------------------------------------------------------------------ BitNet, ternary
def bitnet_pack(W) -> dict:
    """W ~ alpha sign(W), alpha = mean|W| per tensor ([BitNet] §2.2). Pinned by tests (alpha =
    mean|W| hand check, sign(0) = +1)."""
    W = _c(W, np.float32)
    B = np.empty(W.shape, np.int8)
    a = np.zeros(1, np.float32)
    _ok(_lib.bqref_bitnet_pack(_p(W), W.shape[0], W.shape[1], _p(B), _p(a)))
    return dict(B=B, alpha=a[0])


def bitnet_layer(p, x) -> dict:
    """acc = sum_k B q (int64); y = sum_k (alpha B)(q gamma / 127) in float64 ([BitNet] §2.3, [HGF]
    §1.2). Pinned by tests (integer and dequantized routes agree; the W1A8 plane identity)."""
    B = _c(p["B"], np.int8)
    x = _c(x, np.float32)
    N, K = B.shape
    M = x.shape[0]
    q = np.empty((M, K), np.int8)
    gam = np.empty(M, np.float32)
    acc = np.empty((M, N), np.int64)
    y = np.empty((M, N), np.float64)
    _ok(_lib.bqref_bitnet_layer(_p(B), float(p["alpha"]), N, K, _p(x), M, _p(q), _p(gam), _p(acc), _p(y)))
    return dict(q=q, gamma=gam, acc=acc, y=y)


def ternary_pack(W, lora_A=None, lora_B=None, lora_alpha: float = 0.1) -> dict:
    """gamma = mean|W|, T = clamp(rn(W / gamma), -1, 1) with a float32 divide, ties to even ([HGF]
    §1.2); LoRA A and B rounded to bf16 ([HGF] §2.1). Pinned by tests (hand examples with +-0.5
    ties, zero fraction of a Gaussian matrix)."""
    W = _c(W, np.float32)
    T = np.empty(W.shape, np.int8)
    g = np.zeros(1, np.float32)
    _ok(_lib.bqref_ternary_pack(_p(W), W.shape[0], W.shape[1], _p(T), _p(g)))
    out = dict(T=T, gamma_w=g[0], lora_alpha=np.float32(lora_alpha))
    if lora_A is not None:
        out["A"] = bf16_round(lora_A)
        out["B"] = bf16_round(lora_B)
    return out


def silu(z):
    """SiLU(z) = z / (1 + exp(-z)) in float64 ([HGF] §2.1). Pinned through lora_correction's closed
    form (rank 1)."""
    z = _c(z, np.float64)
    out = np.empty_like(z)
    _ok(_lib.bqref_silu(_p(z), z.size, _p(out)))
    return out


def lora_correction(x, A, B, alpha) -> np.ndarray:
    """tanh(alpha) SiLU(x A) B in float64 with x unquantized ([HGF] §2.1). Pinned by tests (closed
    form with rank 1)."""
    x, A, B = _c(x, np.float32), _c(A, np.float32), _c(B, np.float32)
    M, K = x.shape
    r, N = B.shape
    out = np.empty((M, N), np.float64)
    _ok(_lib.bqref_lora_correction(_p(x), M, K, _p(A), _p(B), r, N, float(np.float32(alpha)), _p(out)))
    return out


def ternary_layer(p, x) -> dict:
    """acc = sum_k T q (int64); y = (gamma_w T)(q gamma_x / 127) in float64 plus the gated
    correction ([HGF] §1.2, §2.1). Pinned by tests (integer route equals the dequantized route)."""
    T = _c(p["T"], np.int8)
    x = _c(x, np.float32)
    N, K = T.shape
    M = x.shape[0]
    if "A" in p:
        A, Bl = _c(p["A"], np.float32), _c(p["B"], np.float32)
        r = A.shape[1]
    else:
        A = Bl = np.zeros(1, np.float32)
        r = 0
    q = np.empty((M, K), np.int8)
    gam = np.empty(M, np.float32)
    acc = np.empty((M, N), np.int64)
    y, yt, yl = (np.empty((M, N), np.float64) for _ in range(3))
    _ok(_lib.bqref_ternary_layer(_p(T), float(p["gamma_w"]), _p(A), _p(Bl), r, float(p.get("lora_alpha", 0.1)), N, K,
                                 _p(x), M, _p(q), _p(gam), _p(acc), _p(y), _p(yt), _p(yl)))
    return dict(q=q, gamma=gam, acc=acc, y=y, y_ternary=yt, y_lora=yl)


# ------------------------------------------------------------------ ABQ
def abq_pack(W, w_bits: int) -> dict:
    """Per-output-row asymmetric weight codes (quantize_rows_asym). Pinned by tests (hand examples
    with a rounding tie, grid round trip)."""
    Q, d, z = quantize_rows_asym(W, w_bits)
    return dict(Q=Q, delta=d, z=z, w_bits=w_bits)


def abq_pack_balanced(W) -> dict:
    """[ABQ] §3.3 bit balance W2*: hi = max|W|, Delta = max(2 hi, 1e-5) / 4, z = 2, q = clamp(rn(W /
    Delta) + 2, 0, 4). Pinned by tests (exact antisymmetry q(-W) = 4 - q(W), grid round trip,
    levels)."""
    W = _c(W, np.float32)
    N, K = W.shape
    Q = np.empty((N, K), np.int32)
    d = np.empty(N, np.float32)
    z = np.empty(N, np.int32)
    _ok(_lib.bqref_abq_pack_balanced(_p(W), N, K, _p(Q), _p(d), _p(z)))
    return dict(Q=Q, delta=d, z=z, w_bits=3)


def abq_compensated_weights(W, a, b) -> np.ndarray:
    """[ABQ] §3.2 eq.(3) with gamma = 1: W + a b^T in float32, the product rounded before the sum.
    Pinned by tests (a = 0 leaves W unchanged; dyadic closed forms exact in float32; the product is
    rounded first)."""
    W, a, b = _c(W, np.float32), _c(a, np.float32), _c(b, np.float32)
    assert a.shape == (W.shape[0],) and b.shape == (W.shape[1],)
    out = np.empty_like(W)
    _ok(_lib.bqref_abq_compensate(_p(W), _p(a), _p(b), W.shape[0], W.shape[1], _p(out)))
    return out


def abq_pack_compensated(W, a, b, w_bits: int, balanced: bool = False) -> dict:
    """The codes of W + a b^T ([ABQ] §3.2 eq.(3), gamma = 1), plain or W2*. Pinned by tests
    (closed-form grid codes, exact cancellation to the degenerate row, W2* antisymmetry)."""
    Wc = abq_compensated_weights(W, a, b)
    if balanced:
        assert w_bits == 3
        return abq_pack_balanced(Wc)
    return abq_pack(Wc, w_bits)


def abq_layer(p, x, a_bits: int) -> dict:
    """Activation codes per token with a bits; I = sum_k (qw - zw)(qx - zx) (int64), y = sum_k (Dw
    cw)(Dx cx) in float64 ([ABQ] §3.2). Pinned by tests (zero-point expansion equals the centred
    product; |I| bounds)."""
    Q, d, z = _c(p["Q"], np.int32), _c(p["delta"], np.float32), _c(p["z"], np.int32)
    x = _c(x, np.float32)
    N, K = Q.shape
    M = x.shape[0]
    Qx = np.empty((M, K), np.int32)
    dx = np.empty(M, np.float32)
    zx = np.empty(M, np.int32)
    I = np.empty((M, N), np.int64)
    y = np.empty((M, N), np.float64)
    _ok(_lib.bqref_abq_layer(_p(Q), _p(d), _p(z), N, K, _p(x), M, int(a_bits), _p(Qx), _p(dx), _p(zx), _p(I), _p(y)))
    return dict(Qx=Qx, delta_x=dx, z_x=zx, I=I, y=y)


# ------------------------------------------------------------------ bit-plane identities
def planes_of(codes, bits: int) -> list:
    """Bit-plane b of each code (bit b modulo 2^bits). Pinned by tests (the W1A8 plane identity over
    all int8 codes)."""
    c = _c(np.asarray(codes).ravel(), np.int64)
    out = np.empty((bits, c.size), np.uint8)
    _ok(_lib.bqref_planes_of(_p(c), c.size, int(bits), _p(out)))
    return [out[b] for b in range(bits)]


def plane_weights(bits: int, signed: bool) -> list:
    """Plane weights 2^b, the top plane -2^(bits-1) when signed. Pinned by tests (the W1A8 plane
    identity: plane 7 weighs -128)."""
    out = np.empty(bits, np.int64)
    _ok(_lib.bqref_plane_weights(int(bits), int(bool(signed)), _p(out)))
    return [int(v) for v in out]


def bitplane_dot(wc, w_bits, w_signed, xc, x_bits, x_signed) -> int:
    """sum_b sum_c w_b w_c popc(W_b AND X_c) over one vector pair ([ABQ] abstract: binary
    tensor-core equivalent operations), with popcounts of packed words. Pinned by tests (brute
    force: equals the integer dot product for every bit pair)."""
    w, x = _c(np.asarray(wc).ravel(), np.int64), _c(np.asarray(xc).ravel(), np.int64)
    assert w.size == x.size
    out = np.zeros(1, np.int64)
    _ok(_lib.bqref_bitplane_dot(_p(w), int(w_bits), int(bool(w_signed)), _p(x), int(x_bits), int(bool(x_signed)),
                                w.size, _p(out)))
    return int(out[0])


def xnor_popcount_dot(a_pm1, b_pm1) -> int:
    """[BitNet] §2.3: 2 popc(xnor(a, b)) - K for +-1 vectors. Pinned by tests (brute force over all
    +-1 pairs)."""
    a, b = _c(a_pm1, np.int8), _c(b_pm1, np.int8)
    out = np.zeros(1, np.int64)
    _ok(_lib.bqref_xnor_popcount_dot(_p(a), _p(b), a.size, _p(out)))
    return int(out[0])


# ------------------------------------------------------------------ BVSR
def nearest_rank(sorted_vals, num: int, den: int):
    """Nearest-rank quantile num/den of an ascending array: element ceil(num V / den) - 1. Pinned by
    tests (hand quantiles)."""
    v = _c(sorted_vals, np.float64)
    out = np.zeros(1, np.float64)
    _ok(_lib.bqref_nearest_rank(_p(v), v.size, int(num), int(den), _p(out)))
    return out[0]


def bvsr_set_table(W) -> np.ndarray:
    """The 256 cached coefficient sets of a matrix ([BVSR] Introduction; the construction is a
    reading: ratio family x quantile grid of vector minima and maxima). Parity unpinned as a
    reading; pinned by the r = 2 uniform-grid case and a hand-built table."""
    W = _c(W, np.float32)
    t = np.empty((256, 5), np.float32)
    _ok(_lib.bqref_bvsr_set_table(_p(W), W.shape[0], W.shape[1], _p(t)))
    return t


def bvsr_cluster_table(W, rounds: int) -> dict:
    """[BVSR] Introduction, coefficient cache, clustering reading: per-vector best ratio family
    on its own range, then per family Lloyd k-means of the vectors' (min, max) into 64 centroids
    from the quantile grid, with exact fixed-point centroid sums; set 64 j + c spans centroid c.
    Returns table [256,5], family [V], assign [V], centroids [4,64,2]. Parity unpinned as a
    reading; pinned by tests (rounds = 0 is bvsr_set_table, the k-means objective never grows,
    brute-force family choice, a hand case of exact clusters)."""
    W = _c(W, np.float32)
    N, K = W.shape
    V = N * (K // BVSR_VEC)
    t = np.empty((256, 5), np.float32)
    fam = np.empty(V, np.uint8)
    asg = np.empty(V, np.uint8)
    cen = np.empty((4, 64, 2), np.float64)
    _ok(_lib.bqref_bvsr_cluster_table(_p(W), N, K, int(rounds), _p(t), _p(fam), _p(asg), _p(cen)))
    return dict(table=t, family=fam, assign=asg, centroids=cen)


def bvsr_points(table) -> np.ndarray:
    """P[s, code] = o + sum of the c_i selected by the bits of code, added in i order in float64.
    Pinned by tests (ratio-2 sets are the uniform RTN grid)."""
    t = _c(table, np.float32)
    S = t.shape[0]
    P = np.empty((S, 16), np.float64)
    _ok(_lib.bqref_bvsr_points(_p(t), S, _p(P)))
    return P


def bvsr_encode_vectors(vecs, table):
    """Exhaustive search ([BVSR] Introduction): nearest of 16 points per element (lowest code on a
    tie), least squared error per vector over the 256 sets (lowest set on a tie). Returns (codes,
    sets). Pinned by tests (matches RTN for the uniform set; exhaustive optimum on tiny inputs)."""
    v = _c(vecs, np.float32)
    t = _c(table, np.float32)
    assert t.shape == (256, 5)
    V = v.shape[0]
    codes = np.empty((V, BVSR_VEC), np.uint8)
    sets = np.empty(V, np.uint8)
    _ok(_lib.bqref_bvsr_encode(_p(v), V, _p(t), _p(codes), _p(sets)))
    return codes, sets


def bvsr_pack(W, table=None, rows=None, cluster_rounds: int = 0) -> dict:
    """BVSR 4-bit pack of W (rows optionally restricted): table, codes and set indices. Pinned by
    tests (layer routes agree); the set construction itself is a reading: parity unpinned."""
    W = _c(W, np.float32)
    N, K = W.shape
    if table is None:
        table = bvsr_cluster_table(W, cluster_rounds)["table"] if cluster_rounds > 0 else bvsr_set_table(W)
    sel = np.arange(N) if rows is None else np.asarray(rows)
    codes, sets = bvsr_encode_vectors(W[sel].reshape(-1, BVSR_VEC), table)
    return dict(codes=codes.reshape(len(sel), K), sets=sets.reshape(len(sel), K // BVSR_VEC), table=table, rows=sel)


def bvsr_weight(codes, sets, table) -> np.ndarray:
    """W_hat[n,k] = P[set(n, k / 32), code(n,k)] in float64. Pinned by tests (the dequantized route
    of bvsr_layer equals its integer route)."""
    P = bvsr_points(table)
    s_full = np.repeat(np.asarray(sets, np.int64), BVSR_VEC, axis=1)
    return P[s_full, np.asarray(codes, np.int64)]


def bvsr_layer(codes, sets, table, x) -> dict:
    """acc = sum_k code q (int64); y = sum_k W_hat x_hat in float64 with per-token absmax int8
    activations ([BVSR] Introduction). Pinned by tests (integer and dequantized routes agree; exact
    integer table case)."""
    c, s, t = _c(codes, np.uint8), _c(sets, np.uint8), _c(table, np.float32)
    x = _c(x, np.float32)
    N, K = c.shape
    M = x.shape[0]
    q = np.empty((M, K), np.int8)
    gam = np.empty(M, np.float32)
    acc = np.empty((M, N), np.int64)
    y = np.empty((M, N), np.float64)
    _ok(_lib.bqref_bvsr_layer(_p(c), _p(s), _p(t), N, K, _p(x), M, _p(q), _p(gam), _p(acc), _p(y)))
    return dict(q=q, gamma=gam, acc=acc, y=y)


# ------------------------------------------------------------------ sizes, tolerance
def decode_tokens_per_s(bandwidth_bytes_s: float, params: float, bits: float) -> float:
    """Memory-wall bound B / (P b / 8) tokens per second ([HGF] §1.1). Pinned by tests (the HGF
    page's printed 35 tokens/s at FP16)."""
    return float(_lib.bqref_decode_tokens_per_s(float(bandwidth_bytes_s), float(params), float(bits)))


def weight_bits_per_param(fmt: str, w_bits: int = 0) -> float:
    """Storage bits per weight of the packed planes or bitvectors (BVSR counts its set byte per 32
    weights). Pinned by tests (2 bits for ternary, 4.25 for BVSR, 1 for BitNet)."""
    return float(_lib.bqref_weight_bits_per_param(_FMT[fmt], int(w_bits)))


def tolerance_ok(y, y_ref, rel: float = 1e-3) -> bool:
    """max|y - y_ref| <= rel (||y_ref||_inf + 1e-6). Pinned by tests (hand cases on both sides of
    the bound)."""
    y, r = _c(y, np.float64).ravel(), _c(y_ref, np.float64).ravel()
    if r.size and y.size != r.size:
        raise ValueError("shape mismatch")
    return bool(_lib.bqref_tolerance_ok(_p(y), y.size, _p(r), r.size, float(rel)))
