"""Reference quantizers and layers (float64 / int64), CPU only — test infrastructure.

Conventions
-----------
* W [N,K] float32 weights, x [M,K] bf16-exact float32 activations, y [M,N].
* "rn" = IEEE round-to-nearest-even (numpy ``rint``).
* Decisions that turn floating point into an integer code (sign, rounding,
  nearest point) are taken in float32 where the stored operands are float32,
  exactly as written below, so the CUDA path can reach the same codes
  bit-for-bit; every sum, mean and layer product is float64 / int64.
* Integer accumulators are direct code products (textbook loops via int64
  matmul): no bit-planes and no popcount, so they are independent of the
  bit-plane arithmetic they check.

Page keys ([RaBiT], [HGF], [ABQ], [BVSR], [BitNet]) are listed in the package
docstring.
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# shared helpers
# ---------------------------------------------------------------------------


def _f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float32)


def bf16_round(a) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), returned as float32.

    Used where a format stores a tensor in bf16 (the LoRA matrices of [HGF]
    §2.1 are an fp16/bf16 correction path).
    Pinned by tests (hand values: exact, tie to even down and up, above half)."""
    f = np.ascontiguousarray(_f32(a))
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(f.shape)


def sign_pm1(v) -> np.ndarray:
    """sign(v) = +1 if v >= 0 else -1 ([BitNet] §2.1). -0.0 >= 0 holds, so
    sign(-0.0) = +1. Pinned by tests (zero, negative zero, tiny values)."""
    v = np.asarray(v)
    return np.where(v >= 0, 1, -1).astype(np.int8)


def mean_abs_f32(a) -> np.float32:
    """mean(|a|) summed in float64, stored as float32.
    Pinned by tests (BitNet alpha hand check; the SVID first g-step equals it)."""
    a64 = np.abs(np.asarray(a, dtype=np.float64))
    if a64.size == 0:
        return np.float32(0.0)
    return np.float32(a64.sum() / a64.size)


# ---------------------------------------------------------------------------
# activation quantization
# ---------------------------------------------------------------------------


def quantize_act_int8(x) -> tuple[np.ndarray, np.ndarray]:
    """Per-token absmax int8 quantization ([HGF] §1.2: activations to 8-bit
    integers, dequantized by gamma_x/127; [BVSR] Introduction: lightweight
    online quantization of the input).

    gamma[m] = max_k |x[m,k]|;  s = 127 / gamma (float32);
    q = clamp(rn(x * s), -127, 127) with x*s a float32 product.
    gamma == 0 gives q == 0. Returns (q int8 [M,K], gamma float32 [M]).
    Pinned by tests (scale endpoints map to +-127, ties, zero rows)."""
    x = _f32(x)
    M, K = x.shape
    gamma = np.abs(x).max(axis=1) if K > 0 else np.zeros(M, np.float32)
    gamma = gamma.astype(np.float32)
    q = np.zeros((M, K), dtype=np.int8)
    for m in range(M):
        if gamma[m] > 0:
            s = np.float32(127.0) / gamma[m]
            v = (x[m] * s).astype(np.float32)
            q[m] = np.clip(np.rint(v), -127, 127).astype(np.int8)
    return q, gamma


def dequant_act_int8(q, gamma) -> np.ndarray:
    """x_hat = q * gamma / 127 in float64 ([HGF] §1.2 dequantization).
    Pinned by tests (act endpoints and range: q gamma / 127 recovers the row extremes)."""
    return q.astype(np.float64) * (gamma.astype(np.float64)[:, None] / 127.0)


def quantize_rows_asym(V, bits: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Uniform asymmetric quantizer per row ([ABQ] §3.2 eq.(3) with the
    compensation term off, gamma=0, and no learned clipping, alpha=beta=1 of
    §3.1 eq.(1)):

      lo = min(row), hi = max(row)                       (float32, exact)
      Delta = max(hi - lo, 1e-5) / (2^bits - 1)          (float32 ops)
      z = rn(-lo / Delta)                                (integer, not clamped)
      q = clamp(rn(v / Delta) + z, 0, 2^bits - 1)

    Returns (q int32 [R,L], Delta float32 [R], z int32 [R]).
    Pinned by tests (a hand example with a rounding tie, grid round-trip)."""
    V = _f32(V)
    R, L = V.shape
    qmax = (1 << bits) - 1
    lo = V.min(axis=1).astype(np.float32)
    hi = V.max(axis=1).astype(np.float32)
    rng_ = np.maximum((hi - lo).astype(np.float32), np.float32(1e-5)).astype(np.float32)
    delta = (rng_ / np.float32(qmax)).astype(np.float32)
    z = np.rint((-lo / delta).astype(np.float32)).astype(np.int64)
    q = np.rint((V / delta[:, None]).astype(np.float32)).astype(np.int64) + z[:, None]
    q = np.clip(q, 0, qmax)
    return q.astype(np.int32), delta, z.astype(np.int32)


# ---------------------------------------------------------------------------
# RaBiT: two residual binary paths ([RaBiT] §2.1, §2.2)
# ---------------------------------------------------------------------------


def rabit_pack(W, h2) -> dict:
    """W_hat = g1*B1*h1 + g2*B2*h2 built by the residual recursion of [RaBiT]
    §2.2: B1 = sign(W); W1 = g1 B1 h1; R1 = W - W1; B2 = sign(R1); W2 = g2 B2 h2.

    The pages learn g and h; here g_p[n] = mean_k |.| of the binarized matrix
    row (W for path 1, R1 for path 2), h1 = 1, h2 given.
    R1 is formed from the stored float32 g1, and sign(R1) is the sign of the
    exact difference W - g1*B1 (a float32 subtraction keeps that sign).
    Pinned by tests (recursion-order hand example, constant-magnitude rows)."""
    W = _f32(W)
    N, K = W.shape
    B1 = sign_pm1(W)
    g1 = np.array([mean_abs_f32(W[n]) for n in range(N)], dtype=np.float32)
    h1 = np.ones(K, dtype=np.float32)
    R1 = W.astype(np.float64) - g1.astype(np.float64)[:, None] * B1 * h1.astype(np.float64)
    B2 = sign_pm1(R1)
    g2 = np.array([mean_abs_f32(R1[n]) for n in range(N)], dtype=np.float32)
    return dict(B1=B1, B2=B2, g1=g1, g2=g2, h1=h1, h2=_f32(h2).copy())


def _seq_sum(a, axis) -> np.ndarray:
    """float64 sum in index order (left to right) along `axis`."""
    a = np.asarray(a, dtype=np.float64)
    if a.shape[axis] == 0:
        return np.zeros(np.delete(a.shape, axis), dtype=np.float64)
    return np.take(np.add.accumulate(a, axis=axis), -1, axis=axis)


def rabit_pack_svid(W, rounds: int = 20) -> dict:
    """[RaBiT] §2.3 "function-aware initialization", stage 1: iterative residual SVID,
    Gauss-Seidel alternation over the two paths (default 20 iterations, §5). Stage 2 (channel
    importance from calibration data) is out of scope.

    Reading (the page gives no formulas): path p approximates its target T_p = W - W_other by
    sign(T_p) * (g_p h_p^T), g_p per row, h_p per column (SVID: signs times a rank-1
    magnitude). Each round updates path 1 then path 2; a path update sets B_p = sign(T_p),
    then one alternating least-squares step of |T_p| ~ g_p h_p^T: g first, then h.
      g_p[i] = sum_j |T_ij| h_p[j] / sum_j h_p[j]^2        (0 if the denominator is 0)
      h_p[j] = sum_i |T_ij| g_p[i] / sum_i g_p[i]^2        (unchanged if the denominator is 0)
    Start: g = 0, h = 1 for both paths. Arithmetic: float64 with sums in index order;
    g and h are rounded to float32 after every update (their storage);
    W_p[i,j] = (g_p[i] * h_p[j]) * B_p[i,j]; sign(0) = +1.
    Every step minimizes ||W - W_1 - W_2||^2 over its own block, so the error is non-increasing.
    The first g-step is exactly the mean-|W| scale of rabit_pack.
    Pinned by tests (exact signed rank-1 input, monotone error, least-squares step)."""
    W64 = _f32(W).astype(np.float64)
    N, K = W64.shape
    g = [np.zeros(N, np.float32), np.zeros(N, np.float32)]
    h = [np.ones(K, np.float32), np.ones(K, np.float32)]
    B = [sign_pm1(W64), np.ones((N, K), np.int8)]

    def path_weight(q):
        return (g[q].astype(np.float64)[:, None] * h[q].astype(np.float64)[None, :]) * B[q]

    for _ in range(rounds):
        for q in (0, 1):
            T = W64 - path_weight(1 - q)
            B[q] = sign_pm1(T)
            A = np.abs(T)
            hq = h[q].astype(np.float64)
            hh = _seq_sum(hq * hq, 0)
            g[q] = (_seq_sum(A * hq[None, :], 1) / hh).astype(np.float32) if hh > 0 else np.zeros(N, np.float32)
            gq = g[q].astype(np.float64)
            gg = _seq_sum(gq * gq, 0)
            if gg > 0:
                h[q] = (_seq_sum(A * gq[:, None], 0) / gg).astype(np.float32)
    return dict(B1=B[0], B2=B[1], g1=g[0], g2=g[1], h1=h[0], h2=h[1])


def rabit_recon_error(p, W) -> float:
    """||W - W_hat||^2 in float64.
    Pinned by tests (zero error on the exact signed rank-1 input to rounding)."""
    d = _f32(W).astype(np.float64) - rabit_weight(p)
    return float(np.sum(d * d))


def rabit_pack_paths(W, hs) -> dict:
    """The residual recursion of rabit_pack with P = len(hs) paths ([RaBiT] §2.1-2.2; §6 lists
    a 3-bit extension, read as a third path): R_0 = W; path p takes B_p = sign(R_{p-1}),
    g_p[n] = mean_k |R_{p-1}[n,:]| (float64 sum, stored float32) and the given h_p, then
    R_p = R_{p-1} - g_p B_p h_p in float64 from the stored g_p and h_p.
    hs: P float32 vectors [K] (hs[0] is 1 in the two-path reading). Returns B [P,N,K] int8,
    g [P,N] float32, h [P,K] float32. With P = 2 and hs = (1, h2) it is rabit_pack.
    Pinned by tests (P = 2 equals rabit_pack bit for bit; with h = 1 each added path lowers
    ||W - W_hat||^2 by K g_p^2 per row)."""
    W = _f32(W)
    N, K = W.shape
    P = len(hs)
    R = W.astype(np.float64)
    B = np.zeros((P, N, K), np.int8)
    g = np.zeros((P, N), np.float32)
    h = np.stack([_f32(v) for v in hs]).astype(np.float32)
    for p in range(P):
        B[p] = sign_pm1(R)
        g[p] = np.array([mean_abs_f32(R[n]) for n in range(N)], dtype=np.float32)
        R = R - g[p].astype(np.float64)[:, None] * B[p] * h[p].astype(np.float64)[None, :]
    return dict(B=B, g=g, h=h)


def rabit_weight_paths(p) -> np.ndarray:
    """W_hat [N,K] float64 = sum_p g_p B_p h_p for a rabit_pack_paths result.
    Pinned by tests (P = 2 equals rabit_weight)."""
    return sum(p["g"][q].astype(np.float64)[:, None] * p["B"][q] * p["h"][q].astype(np.float64)[None, :]
               for q in range(p["B"].shape[0]))


def rabit_weight(p) -> np.ndarray:
    """W_hat [N,K] float64 = g1*B1*h1 + g2*B2*h2 ([RaBiT] §2.1).
    Pinned by tests (RaBiT hand recursion, constant-magnitude rows reconstruct exactly)."""
    g1, g2 = p["g1"].astype(np.float64), p["g2"].astype(np.float64)
    h1, h2 = p["h1"].astype(np.float64), p["h2"].astype(np.float64)
    return g1[:, None] * p["B1"] * h1[None, :] + g2[:, None] * p["B2"] * h2[None, :]


def rabit_layer(p, x) -> dict:
    """y = W_hat x in float64 with x the unquantized bf16 activations (the
    RaBiT kernel of [RaBiT] §3.2 applies signs to the input, no activation
    quantization). Also returns the per-path sums acc_p = sum_k B_p h_p x.
    Pinned by tests (the layer equals the sum of the two sign paths, dense vs per path)."""
    x64 = _f32(x).astype(np.float64)
    y = x64 @ rabit_weight(p).T
    acc1 = x64 @ (p["B1"] * p["h1"].astype(np.float64)[None, :]).T
    acc2 = x64 @ (p["B2"] * p["h2"].astype(np.float64)[None, :]).T
    return dict(y=y, acc1=acc1, acc2=acc2)


# ---------------------------------------------------------------------------
# BitNet W1A8 ([BitNet] §2.1-2.3)
# ---------------------------------------------------------------------------


def bitnet_pack(W) -> dict:
    """W ~= alpha * sign(W) with one alpha per matrix ([BitNet] §2.2); the page
    learns alpha, here alpha = mean|W| over the whole tensor.
    Pinned by tests (alpha = mean|W| hand check, sign(0) = +1)."""
    W = _f32(W)
    return dict(B=sign_pm1(W), alpha=mean_abs_f32(W))


def bitnet_layer(p, x) -> dict:
    """acc = sum_k B[n,k] q[m,k] (int64); y = sum_k (alpha B)(q gamma/127) in
    float64 ([BitNet] §2.3 binary product scaled by alpha; activation scale of
    [HGF] §1.2).
    Pinned by tests (integer and dequantized-float routes agree; the W1A8 plane identity over all int8 codes)."""
    q, gamma = quantize_act_int8(x)
    acc = q.astype(np.int64) @ p["B"].astype(np.int64).T
    w_hat = np.float64(p["alpha"]) * p["B"].astype(np.float64)
    y = dequant_act_int8(q, gamma) @ w_hat.T
    return dict(q=q, gamma=gamma, acc=acc, y=y)


# ---------------------------------------------------------------------------
# Ternary W1.58A8 with gated low-rank correction ([HGF] §1.2, §2.1, §4.1)
# ---------------------------------------------------------------------------


def ternary_pack(W, lora_A=None, lora_B=None, lora_alpha: float = 0.1) -> dict:
    """gamma = mean|W| (the code of [HGF] §1.2 uses the mean although the prose
    says absmax); T = clamp(rn(W / gamma), -1, 1) with W/gamma a float32
    division and rn ties-to-even (torch.round). gamma == 0 gives T == 0.
    LoRA A [K,r], B [r,N] are stored in bf16 ([HGF] §2.1 fp16 correction path).
    Pinned by tests (hand examples with +-0.5 ties, zero fraction of a
    Gaussian matrix)."""
    W = _f32(W)
    gamma = mean_abs_f32(W)
    if gamma > 0:
        T = np.clip(np.rint((W / gamma).astype(np.float32)), -1, 1).astype(np.int8)
    else:
        T = np.zeros(W.shape, dtype=np.int8)
    out = dict(T=T, gamma_w=gamma, lora_alpha=np.float32(lora_alpha))
    if lora_A is not None:
        out["A"] = bf16_round(lora_A)
        out["B"] = bf16_round(lora_B)
    return out


def silu(z):
    """SiLU(z) = z / (1 + exp(-z)) ([HGF] §2.1 gate nonlinearity).
    Pinned through lora_correction's closed form (rank 1)."""
    return z / (1.0 + np.exp(-z))


def lora_correction(x, A, B, alpha) -> np.ndarray:
    """tanh(alpha) * (SiLU(x @ A) @ B) in float64 ([HGF] §2.1), x unquantized.
    Pinned by tests (closed form with rank 1)."""
    x64 = _f32(x).astype(np.float64)
    u = silu(x64 @ A.astype(np.float64))
    return math.tanh(float(np.float32(alpha))) * (u @ B.astype(np.float64))


def ternary_layer(p, x) -> dict:
    """acc = sum_k T q (int64); y = gamma_w*gamma_x/127 * acc + LoRA term,
    the ternary part computed as a float64 product of dequantized operands
    ([HGF] §1.2 int8 product with Y_int * gamma_x gamma_W / 127).
    Pinned by tests (integer route equals the dequantized route)."""
    q, gamma = quantize_act_int8(x)
    acc = q.astype(np.int64) @ p["T"].astype(np.int64).T
    w_hat = np.float64(p["gamma_w"]) * p["T"].astype(np.float64)
    y_t = dequant_act_int8(q, gamma) @ w_hat.T
    y_l = lora_correction(x, p["A"], p["B"], p["lora_alpha"]) if "A" in p else 0.0 * y_t
    return dict(q=q, gamma=gamma, acc=acc, y=y_t + y_l, y_ternary=y_t, y_lora=y_l)


# ---------------------------------------------------------------------------
# ABQ-style arbitrary-bit WxAy ([ABQ] §3.1-3.2, abstract)
# ---------------------------------------------------------------------------


def abq_pack_balanced(W) -> dict:
    """[ABQ] §3.3 bit-balance strategy (W2*): INT2's four levels are asymmetric, so the
    code space is widened to the symmetric {-2, -1, 0, 1, 2}. Reading: per row,
    hi = max|W|, lo = -hi, Delta = max(hi - lo, 1e-5) / 4 (float32 ops, as quantize_rows_asym
    with 4 intervals), z = 2, q = clamp(rn(W / Delta) + 2, 0, 4): a 3-bit code, so the packed
    buffer is an ABQ w = 3 buffer whose codes take 5 values.
    Pinned by tests (exact antisymmetry q(-W) = 4 - q(W), grid round trip, levels)."""
    W = _f32(W)
    hi = np.abs(W).max(axis=1).astype(np.float32)
    rng_ = np.maximum((hi - (-hi)).astype(np.float32), np.float32(1e-5)).astype(np.float32)
    delta = (rng_ / np.float32(4)).astype(np.float32)
    q = np.rint((W / delta[:, None]).astype(np.float32)).astype(np.int64) + 2
    q = np.clip(q, 0, 4)
    return dict(Q=q.astype(np.int32), delta=delta, z=np.full(W.shape[0], 2, np.int32), w_bits=3)


def abq_compensated_weights(W, a, b) -> np.ndarray:
    """[ABQ] §3.2 eq.(3) distribution compensation: the matrix that is quantized is
    W + gamma a b^T, gamma = 1 (compensation on) or 0 (off). Readings: a has one entry
    per output row n and b one per input column k, so that a b^T has the shape of W;
    a and b are given (the page fits them by calibration); the sum is formed in float32,
    the product a[n] b[k] rounded first, then the sum (two roundings, no fused multiply-add).
    Pinned by tests (a = 0 leaves W unchanged; dyadic closed forms exact in float32)."""
    W, a, b = _f32(W), _f32(a), _f32(b)
    assert a.shape == (W.shape[0],) and b.shape == (W.shape[1],)
    prod = (a[:, None] * b[None, :]).astype(np.float32)
    return (W + prod).astype(np.float32)


def abq_pack_compensated(W, a, b, w_bits: int, balanced: bool = False) -> dict:
    """[ABQ] §3.2 eq.(3) with gamma = 1: the codes of W' = W + a b^T
    (abq_compensated_weights). Reading: the step Delta and zero point z are those of the
    quantizer applied to W' itself (the row range of W'), so eq.(3)'s clamp to
    0..2^n - 1 cuts nothing but rounding overshoot; with balanced, W' gets the W2*
    codes of abq_pack_balanced (w_bits = 3). The layer then computes y = W'_hat x with
    the ordinary ABQ layer.
    Pinned by tests (closed-form grid codes, exact cancellation to the degenerate row,
    W2* antisymmetry under (W, a) -> (-W, -a))."""
    Wc = abq_compensated_weights(W, a, b)
    if balanced:
        assert w_bits == 3
        return abq_pack_balanced(Wc)
    return abq_pack(Wc, w_bits)


def abq_pack(W, w_bits: int) -> dict:
    """Per-output-row asymmetric weight codes (quantize_rows_asym).
    Pinned by tests (hand examples with a rounding tie, grid round trip)."""
    Q, delta, z = quantize_rows_asym(W, w_bits)
    return dict(Q=Q, delta=delta, z=z, w_bits=w_bits)


def abq_layer(p, x, a_bits: int) -> dict:
    """Per-token asymmetric activation codes, then
    I = sum_k (qw - zw)(qx - zx) (int64) and y = Dw*Dx*I as the float64 product
    of the dequantized operands.
    Pinned by tests (zero-point expansion equals the centred product; |I| bounds)."""
    Qx, dx, zx = quantize_rows_asym(x, a_bits)
    cw = p["Q"].astype(np.int64) - p["z"].astype(np.int64)[:, None]
    cx = Qx.astype(np.int64) - zx.astype(np.int64)[:, None]
    I = cx @ cw.T
    w_hat = p["delta"].astype(np.float64)[:, None] * cw
    x_hat = dx.astype(np.float64)[:, None] * cx
    y = x_hat @ w_hat.T
    return dict(Qx=Qx, delta_x=dx, z_x=zx, I=I, y=y)


# ---------------------------------------------------------------------------
# Bit-plane identities (what the binary AND+popcount kernels compute)
# ---------------------------------------------------------------------------


def popcount(v) -> np.ndarray:
    """Number of set bits of each unsigned 64-bit word, counted bit by bit.
    Pinned through the XNOR and bit-plane identities (brute force over all pairs)."""
    v = np.asarray(v, dtype=np.uint64)
    c = np.zeros(v.shape, dtype=np.int64)
    for b in range(64):
        c += ((v >> np.uint64(b)) & np.uint64(1)).astype(np.int64)
    return c


def planes_of(codes, bits: int) -> list:
    """Bit-plane b of non-negative or two's-complement codes: a 0/1 array.
    Pinned by tests (the W1A8 plane identity over all int8 codes)."""
    c = np.asarray(codes, dtype=np.int64) & ((1 << bits) - 1)
    return [((c >> b) & 1).astype(np.uint8) for b in range(bits)]


def plane_weights(bits: int, signed: bool) -> list:
    """omega_b = 2^b; for two's complement the top plane weighs -2^(bits-1).
    Pinned by tests (the W1A8 plane identity: plane 7 weighs -128)."""
    w = [1 << b for b in range(bits)]
    if signed:
        w[-1] = -w[-1]
    return w


def pack_bits(bitvec) -> int:
    """A 0/1 vector as one integer word, element j at bit j (LSB first).
    Pinned through the XNOR and bit-plane identities (brute force over all pairs)."""
    out = 0
    for j, b in enumerate(np.asarray(bitvec).tolist()):
        out |= int(b) << j
    return out


def bitplane_dot(wc, w_bits, w_signed, xc, x_bits, x_signed) -> int:
    """sum_b sum_c omega_b omega_c popc(W_b AND X_c) over one vector pair, the
    arbitrary-bit product of [ABQ] (abstract: binary tensor-core equivalent
    operations), computed literally with popcounts of packed words.
    Pinned by tests (brute force: equals the integer dot product for every bit pair)."""
    wp, xp = planes_of(wc, w_bits), planes_of(xc, x_bits)
    ww, xw = plane_weights(w_bits, w_signed), plane_weights(x_bits, x_signed)
    tot = 0
    for b in range(w_bits):
        Wb = pack_bits(wp[b])
        for c in range(x_bits):
            Xc = pack_bits(xp[c])
            tot += ww[b] * xw[c] * bin(Wb & Xc).count("1")
    return tot


def xnor_popcount_dot(a_pm1, b_pm1) -> int:
    """[BitNet] §2.3: popcount(xnor(a, b)) for +-1 vectors coded as bit 1 <=> +1.
    Returns 2*popc(xnor) - K, the +-1 inner product (the page's formula without
    the affine correction is the count of agreeing positions).
    Pinned by tests (brute force over all +-1 pairs: 2 popc(xnor) - K)."""
    a = pack_bits(np.asarray(a_pm1) > 0)
    b = pack_bits(np.asarray(b_pm1) > 0)
    K = len(a_pm1)
    xnor = ~(a ^ b) & ((1 << K) - 1)
    return 2 * bin(xnor).count("1") - K


# ---------------------------------------------------------------------------
# BVSR: bitvector-sum weights with cached coefficient sets ([BVSR] Introduction)
# ---------------------------------------------------------------------------

BVSR_VEC = 32
BVSR_RATIOS = (1.5, 2.0, 2.5, 3.0)
BVSR_GRID = 8          # lo/hi grid points per side: 4 ratios x 8 x 8 = 256 sets
BVSR_PLANES = 4


def nearest_rank(sorted_vals: np.ndarray, num: int, den: int):
    """Nearest-rank quantile num/den of an ascending array: element
    ceil(num*V/den) - 1 (integer arithmetic).
    Pinned by tests (hand quantiles)."""
    V = len(sorted_vals)
    rank = (num * V + den - 1) // den
    return sorted_vals[max(rank - 1, 0)]


def bvsr_set_table(W) -> np.ndarray:
    """The cached coefficient sets shared by all vectors of a matrix.

    [BVSR] Introduction: geometric-series subset sums scaled and shifted by
    data-dependent terms; geometric coefficient sets paired with an auxiliary
    grid aligned to the data range; 256 sets (4 ratios x 8 x 8).
    Reading (the page gives no formula): set s = 64*j + 8*a + b has ratio
    r_j in {1.5, 2, 2.5, 3}, template t_i = r^i / sum_{i'<4} r^{i'},
    lo_a = the (2a+1)/16 nearest-rank quantile of the per-vector minima,
    hi_b = the (2b+1)/16 quantile of the per-vector maxima,
    c_i = (hi_b - lo_a) * t_i and o = lo_a (float64, stored float32).
    Returns table float32 [256, 5] = (c0, c1, c2, c3, o). Parity unpinned as a
    reading; pinned by the r=2 uniform-grid case and size arithmetic."""
    W = _f32(W)
    N, K = W.shape
    vecs = W.reshape(N, K // BVSR_VEC, BVSR_VEC)
    smin = np.sort(vecs.min(axis=2).ravel())
    smax = np.sort(vecs.max(axis=2).ravel())
    los = [np.float64(nearest_rank(smin, 2 * a + 1, 16)) for a in range(BVSR_GRID)]
    his = [np.float64(nearest_rank(smax, 2 * b + 1, 16)) for b in range(BVSR_GRID)]
    table = np.zeros((len(BVSR_RATIOS) * BVSR_GRID * BVSR_GRID, 5), dtype=np.float32)
    for j, r in enumerate(BVSR_RATIOS):
        pw = [r ** i for i in range(BVSR_PLANES)]
        tsum = sum(pw)
        t = [pw[i] / tsum for i in range(BVSR_PLANES)]
        for a in range(BVSR_GRID):
            for b in range(BVSR_GRID):
                s = 64 * j + 8 * a + b
                span = his[b] - los[a]
                for i in range(BVSR_PLANES):
                    table[s, i] = np.float32(span * t[i])
                table[s, 4] = np.float32(los[a])
    return table


def bvsr_cluster_table(W, rounds: int) -> dict:
    """[BVSR] Introduction: the coefficient sets are shared across weight vectors by a selection
    step the page calls the coefficient cache. Clustering reading (the page gives no procedure):
      1. every vector takes lo = min, hi = max and the ratio family j whose set on its own range
         (c = (hi - lo) t_j, o = lo, float32) gives it the least squared error (lowest j on a tie);
      2. per family, Lloyd's k-means of the vectors' (lo, hi) into 64 centroids, started from the
         8 x 8 quantile grid of bvsr_set_table (centroid 8a + b = (lo_a, hi_b)): each round assigns
         every point to the nearest centroid (squared distance, float64, lowest index on a tie) and
         moves each centroid with points to their mean, sum(rn(v 2^40)) / count / 2^40 with the
         sum in int64 (exact, order-free); a centroid without points stays;
      3. set 64 j + c: c_i = (hi_c - lo_c) t_{j,i}, o = lo_c, float32. rounds = 0 is bvsr_set_table.
    Returns table [256,5], family [V], assign [V] (0 without rounds), centroids [4,64,2].
    Parity unpinned as a reading; pinned by tests (rounds = 0 is bvsr_set_table, the k-means
    objective never grows, brute-force family choice, a hand case of exact clusters)."""
    W = _f32(W)
    N, K = W.shape
    vecs = W.reshape(-1, BVSR_VEC)
    V = vecs.shape[0]
    lo, hi = vecs.min(axis=1), vecs.max(axis=1)
    smin, smax = np.sort(lo.astype(np.float64)), np.sort(hi.astype(np.float64))
    los = [np.float64(nearest_rank(smin, 2 * a + 1, 16)) for a in range(BVSR_GRID)]
    his = [np.float64(nearest_rank(smax, 2 * b + 1, 16)) for b in range(BVSR_GRID)]
    temps = []
    for r in BVSR_RATIOS:
        pw = [r ** i for i in range(BVSR_PLANES)]
        temps.append([pw[i] / sum(pw) for i in range(BVSR_PLANES)])
    span = hi.astype(np.float64) - lo.astype(np.float64)
    errs = np.zeros((len(BVSR_RATIOS), V))
    for j, t in enumerate(temps):
        sets = np.zeros((V, 5), np.float32)
        for i in range(BVSR_PLANES):
            sets[:, i] = (span * t[i]).astype(np.float32)
        sets[:, 4] = lo
        P = bvsr_points(sets)                                          # [V,16]
        w = vecs.astype(np.float64)
        best = np.argmin(np.abs(w[:, :, None] - P[:, None, :]), axis=2)  # [V,32]
        pb = np.take_along_axis(P, best, axis=1)
        e = np.zeros(V)
        for k in range(BVSR_VEC):
            d = w[:, k] - pb[:, k]
            e = e + d * d
        errs[j] = e
    fam = np.argmin(errs, axis=0).astype(np.uint8)
    cen = np.zeros((4, 64, 2))
    for a in range(BVSR_GRID):
        for b in range(BVSR_GRID):
            cen[:, 8 * a + b] = (los[a], his[b])
    asg = np.zeros(V, np.uint8)
    fx = lambda v: np.rint(np.ldexp(v.astype(np.float64), 40)).astype(np.int64)
    flo, fhi = fx(lo), fx(hi)
    for _ in range(rounds):
        c = cen[fam]                                                   # [V,64,2]
        d = (lo.astype(np.float64)[:, None] - c[:, :, 0]) ** 2 + (hi.astype(np.float64)[:, None] - c[:, :, 1]) ** 2
        asg = np.argmin(d, axis=1).astype(np.uint8)
        idx = fam.astype(np.int64) * 64 + asg
        sl = np.zeros(256, np.int64); sh = np.zeros(256, np.int64); cnt = np.zeros(256, np.int64)
        np.add.at(sl, idx, flo); np.add.at(sh, idx, fhi); np.add.at(cnt, idx, 1)
        has = cnt > 0
        flat = cen.reshape(256, 2)
        flat[has, 0] = np.ldexp(sl[has].astype(np.float64) / cnt[has], -40)
        flat[has, 1] = np.ldexp(sh[has].astype(np.float64) / cnt[has], -40)
        cen = flat.reshape(4, 64, 2)
    table = np.zeros((256, 5), np.float32)
    for j, t in enumerate(temps):
        for c in range(64):
            s = 64 * j + c
            sp = cen[j, c, 1] - cen[j, c, 0]
            for i in range(BVSR_PLANES):
                table[s, i] = np.float32(sp * t[i])
            table[s, 4] = np.float32(cen[j, c, 0])
    return dict(table=table, family=fam, assign=asg, centroids=cen)


def bvsr_points(table) -> np.ndarray:
    """P[s, code] = o + c0 b0 + c1 b1 + c2 b2 + c3 b3 (b_i = bit i of code),
    summed left to right in float64 from the float32 coefficients.
    Pinned by tests (ratio-2 sets are the uniform RTN grid)."""
    t = np.asarray(table, dtype=np.float32).astype(np.float64)
    S = t.shape[0]
    P = np.zeros((S, 16), dtype=np.float64)
    for code in range(16):
        acc = t[:, 4].copy()
        for i in range(BVSR_PLANES):
            if (code >> i) & 1:
                acc = acc + t[:, i]
        P[:, code] = acc
    return P


def bvsr_encode_vectors(vecs, table) -> tuple[np.ndarray, np.ndarray]:
    """Exhaustive search ([BVSR] Introduction): for every vector and every set,
    each element takes the nearest of the set's 16 points (smallest |w - p|,
    lowest code on a tie), the set's error is sum_e (w_e - p)^2 accumulated in
    element order in float64, and the vector takes the set with the smallest
    error (lowest set index on a tie).
    vecs float32 [V, 32] -> (codes uint8 [V, 32], set index uint8 [V]).
    Pinned by tests (matches RTN for the uniform set; exhaustive optimum on tiny inputs)."""
    vecs = _f32(vecs)
    V = vecs.shape[0]
    P = bvsr_points(table)                      # [S,16]
    codes_out = np.zeros((V, BVSR_VEC), dtype=np.uint8)
    sets_out = np.zeros(V, dtype=np.uint8)
    chunk = 32
    for v0 in range(0, V, chunk):
        w = vecs[v0:v0 + chunk].astype(np.float64)              # [c,32]
        d = np.abs(w[:, None, :, None] - P[None, :, None, :])   # [c,S,32,16]
        best = np.argmin(d, axis=3)                             # [c,S,32]
        pbest = P[np.arange(P.shape[0])[None, :, None], best]   # [c,S,32]
        err = np.zeros(best.shape[:2], dtype=np.float64)
        for e in range(BVSR_VEC):
            de = w[:, None, e] - pbest[:, :, e]
            err = err + de * de
        s = np.argmin(err, axis=1)
        sets_out[v0:v0 + chunk] = s
        codes_out[v0:v0 + chunk] = best[np.arange(w.shape[0]), s]
    return codes_out, sets_out


def bvsr_pack(W, table=None, rows=None, cluster_rounds: int = 0) -> dict:
    """BVSR 4-bit pack of W [N,K] (K % 32 == 0). ``rows`` restricts the
    encoding to a subset of rows (the table still comes from the whole W).
    Returns codes uint8 [R,K], set index uint8 [R,K/32], table [256,5].
    Pinned by tests (layer routes agree); the set construction itself is a reading: parity unpinned."""
    W = _f32(W)
    N, K = W.shape
    if table is None:
        table = bvsr_cluster_table(W, cluster_rounds)["table"] if cluster_rounds > 0 else bvsr_set_table(W)
    sel = np.arange(N) if rows is None else np.asarray(rows)
    sub = W[sel]
    codes, sets = bvsr_encode_vectors(sub.reshape(-1, BVSR_VEC), table)
    return dict(codes=codes.reshape(len(sel), K), sets=sets.reshape(len(sel), K // BVSR_VEC),
                table=table, rows=sel)


def bvsr_weight(codes, sets, table) -> np.ndarray:
    """W_hat[n,k] = P[set(n, k/32), code(n,k)] in float64.
    Pinned by tests (the dequantized route of bvsr_layer equals its integer route)."""
    P = bvsr_points(table)
    R, K = codes.shape
    s_full = np.repeat(sets.astype(np.int64), BVSR_VEC, axis=1)
    return P[s_full, codes.astype(np.int64)]


def bvsr_layer(codes, sets, table, x) -> dict:
    """acc = sum_k code q (int64, code = sum_i 2^i b_i); y = sum_k W_hat x_hat in
    float64, x_hat the per-token absmax int8 activations ([BVSR] Introduction:
    activations quantized online, product without weight dequantization).
    Pinned by tests (integer and dequantized routes agree; exact integer table case)."""
    q, gamma = quantize_act_int8(x)
    acc = q.astype(np.int64) @ codes.astype(np.int64).T
    y = dequant_act_int8(q, gamma) @ bvsr_weight(codes, sets, table).T
    return dict(q=q, gamma=gamma, acc=acc, y=y)


# ---------------------------------------------------------------------------
# size and bandwidth arithmetic
# ---------------------------------------------------------------------------


def decode_tokens_per_s(bandwidth_bytes_s: float, params: float, bits: float) -> float:
    """Memory-wall bound T_max <= B_mem / (P * b / 8) ([HGF] §1.1).
    Pinned by tests (the HGF page's printed 35 tokens/s at FP16)."""
    return bandwidth_bytes_s / (params * bits / 8.0)


def weight_bits_per_param(fmt: str, w_bits: int = 0) -> float:
    """Storage bits per weight of the packed planes/bitvectors (scales excluded;
    BVSR counts its 1-byte set index per 32-element vector).
    Pinned by tests (2 bits for ternary, 4.25 for BVSR, 1 for BitNet)."""
    return {"rabit": 2.0, "bitnet": 1.0, "ternary": 2.0, "abq": float(w_bits),
            "bvsr": BVSR_PLANES + 8.0 / BVSR_VEC}[fmt]


def tolerance_ok(y, y_ref, rel: float = 1e-3) -> bool:
    """max|y - y_ref| <= rel * (||y_ref||_inf + 1e-6).
    Pinned by tests (hand cases on both sides of the bound)."""
    y, y_ref = np.asarray(y, np.float64), np.asarray(y_ref, np.float64)
    if y_ref.size == 0:
        return y.size == 0
    return float(np.max(np.abs(y - y_ref))) <= rel * (float(np.max(np.abs(y_ref))) + 1e-6)
