"""Helpers for GPU parity tests: run the CUDA path through the C ABI, read its
buffers back with the oracle's independent readers, and compare with the
oracle (the C++ reference, oracle/bq_ref.cpp through oracle/cref.py). Test
infrastructure only."""
from __future__ import annotations

import numpy as np

import bq_inputs as I
from oracle import cref as O
from oracle import layout as L

RTOL = 1e-3  # max|y - y_ref| <= 1e-3 (||y_ref||_inf + 1e-6)


def torch_mods():
    import torch
    from bit_weight_quantization_b200 import bq
    return torch, bq


def to_dev_f32(a):
    torch, _ = torch_mods()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def to_dev_bf16(x):
    torch, _ = torch_mods()
    bits = I.bf16_bits(x).view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(bits)).cuda().view(torch.bfloat16)


def ulp_diff(a, b) -> np.ndarray:
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)


NEAR_TIE_ULPS = 4          # a code may differ only this close (float32 ulps) to its boundary
NEAR_TIE_LOG: list = []    # (what, codes compared, codes that differ, near-tie codes)


def assert_codes_near_tie(got, ref, near, what):
    """Pack parity where several results are correct: every code is compared, and a code may
    differ from the oracle's only where ``near`` marks the quantity that decides it within
    NEAR_TIE_ULPS float32 ulps of its rounding or selection boundary (the GPU reduces the scale
    that feeds the decision in another order than the oracle). Every differing code is counted
    and reported; the count is returned."""
    got, ref, near = np.asarray(got), np.asarray(ref), np.asarray(near, bool)
    assert got.shape == ref.shape == near.shape, (got.shape, ref.shape, near.shape)
    diff = got != ref
    n_diff, n_far = int(diff.sum()), int((diff & ~near).sum())
    NEAR_TIE_LOG.append((what, int(got.size), n_diff, int(near.sum())))
    if n_diff:
        print(f"[near-tie] {what}: {n_diff} of {got.size} codes differ from the oracle "
              f"({n_diff - n_far} within {NEAR_TIE_ULPS} ulps of a boundary)")
    assert n_far == 0, f"{what}: {n_far} codes differ from the oracle away from any decision boundary"
    return n_diff


def ulps_of(v) -> np.ndarray:
    """float32 spacing at |v| (one ulp)."""
    return np.spacing(np.abs(np.asarray(v, np.float32))).astype(np.float64)


def ternary_near(W, gamma_ref) -> np.ndarray:
    """Ternary codes are decided by W / gamma (float32) against the rounding boundaries +-0.5."""
    d = (np.asarray(W, np.float32) / np.float32(gamma_ref)).astype(np.float32).astype(np.float64)
    return np.abs(np.abs(d) - 0.5) <= NEAR_TIE_ULPS * float(np.spacing(np.float32(0.5)))


def rabit_near(W, B, g, h) -> list:
    """RaBiT path p (p >= 1) signs are decided by the residual R_{p-1} = W - sum_{q<p} g_q B_q h_q
    (float64) against 0; its inputs move by about one ulp of each g_q h_q when the GPU's g_q
    differs from the oracle's by one ulp. Masks for paths 1.. (path 0, sign(W), has no scale)."""
    W64 = np.asarray(W, np.float64)
    R = W64.copy()
    tol = np.zeros(W64.shape[0])
    out = []
    for q in range(len(B) - 1):
        R = R - (g[q].astype(np.float64)[:, None] * B[q]) * h[q].astype(np.float64)[None, :]
        tol = tol + ulps_of(g[q]) * float(np.max(np.abs(h[q])))
        out.append(np.abs(R) <= NEAR_TIE_ULPS * tol[:, None])
    return out


def assert_y_close(y, y_ref, what=""):
    y, y_ref = np.asarray(y, np.float64), np.asarray(y_ref, np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = float(np.max(np.abs(y - y_ref))) if y.size else 0.0
    bound = RTOL * ((float(np.max(np.abs(y_ref))) if y_ref.size else 0.0) + 1e-6)
    assert err <= bound, f"{what}: max|y-y_ref| = {err:.3e} > {bound:.3e}"


class GpuLayer:
    """One layer packed and run by the library, plus host copies of its buffers."""

    def __init__(self, fmt, N, K, M, seed=0, w_bits=0, a_bits=0, lora_rank=32, lora_alpha=0.1,
                 inputs=None, nullify_x=False):
        torch, bq = torch_mods()
        self.fmt, self.N, self.K, self.M = fmt, N, K, M
        self.w_bits, self.a_bits = w_bits, a_bits
        inp = inputs if inputs is not None else I.layer_inputs(fmt, N, K, M, seed, lora_rank)
        if nullify_x:
            inp["x"] = np.zeros_like(inp["x"])
        self.inp = inp
        self.W = to_dev_f32(inp["W"])
        kw = {}
        if fmt in ("rabit", "rabit3"):
            kw["h2"] = to_dev_f32(inp["h2"])
        if fmt == "rabit3":
            kw["h3"] = to_dev_f32(inp["h3"])
        if fmt == "ternary":
            kw.update(lora_rank=lora_rank, lora_alpha=lora_alpha,
                      lora_A=to_dev_f32(inp["lora_A"]), lora_B=to_dev_f32(inp["lora_B"]))
        if fmt == "abq":
            kw.update(w_bits=w_bits, a_bits=a_bits)
        self.ql = bq.QuantLinear(fmt, self.W, **kw)
        self.x = to_dev_bf16(inp["x"])
        self.y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        self.acc = None
        if fmt not in ("rabit", "rabit3"):
            self.acc = torch.full((M, N), -(1 << 62), dtype=torch.int64, device="cuda")
        self.ql.forward(self.x, self.y, self.acc)
        # the fused path (bq_linear) on the same inputs
        self.y_f = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        self.acc_f = None if self.acc is None else torch.full((M, N), -(1 << 62), dtype=torch.int64, device="cuda")
        self.ql.linear(self.x, self.y_f, self.acc_f)
        torch.cuda.synchronize()
        bq.bq_device_check()
        self.packed = self.ql.packed.cpu().numpy().tobytes()
        self.act = self.ql.act_buffer(M).cpu().numpy().tobytes()
        self.y_h = self.y.cpu().numpy()
        self.acc_h = self.acc.cpu().numpy() if self.acc is not None else None
        self.yf_h = self.y_f.cpu().numpy()
        self.accf_h = self.acc_f.cpu().numpy() if self.acc_f is not None else None
        # the fused kernel runs the same arithmetic as bq_quantize_act + bq_gemm
        assert np.array_equal(self.yf_h, self.y_h, equal_nan=False), f"{fmt}: fused y differs from act+gemm"
        if self.acc_h is not None:
            assert np.array_equal(self.accf_h, self.acc_h), f"{fmt}: fused acc differs"

    def read(self, row_blocks=None):
        return L.read_packed(self.packed, row_blocks)


def oracle_pack(fmt, inp, w_bits=0, lora_alpha=0.1, rows=None):
    W = inp["W"]
    if fmt == "rabit":
        return O.rabit_pack(W, inp["h2"])
    if fmt == "rabit3":
        return O.rabit_pack_paths(W, [np.ones(W.shape[1], np.float32), inp["h2"], inp["h3"]])
    if fmt == "bitnet":
        p = O.bitnet_pack(W)
        if rows is not None:
            p["B"] = p["B"][rows]
        return p
    if fmt == "ternary":
        p = O.ternary_pack(W, inp.get("lora_A"), inp.get("lora_B"), lora_alpha)
        if rows is not None:
            p["T"] = p["T"][rows]
        return p
    if fmt == "abq":
        sub = W if rows is None else W[rows]
        return O.abq_pack(sub, w_bits)
    if fmt == "bvsr":
        return O.bvsr_pack(W, rows=rows)
    raise ValueError(fmt)


def oracle_layer(fmt, p, x, a_bits=0):
    """Reference layer on the library's own decoded codes (dict from the reader)."""
    if fmt == "rabit":
        return O.rabit_layer(p, x)
    if fmt == "rabit3":
        return O.rabit_layer(p, x)
    if fmt == "bitnet":
        return O.bitnet_layer(p, x)
    if fmt == "ternary":
        return O.ternary_layer(p, x)
    if fmt == "abq":
        r = O.abq_layer(p, x, a_bits)
        r["acc"] = r["I"]
        return r
    if fmt == "bvsr":
        return O.bvsr_layer(p["codes"], p["sets"], p["table"], x)
    raise ValueError(fmt)


def check_act(gl: GpuLayer):
    """Activation buffer against the oracle's activation quantizer (bit-exact)."""
    a = L.read_act(gl.act)
    x = gl.inp["x"]
    assert a["M"] == gl.M and a["K"] == gl.K
    if gl.fmt in ("rabit", "rabit3"):
        hs = [gl.inp["h2"]] + ([gl.inp["h3"]] if gl.fmt == "rabit3" else [])
        assert a["xt"].shape[0] == 1 + len(hs)
        assert np.array_equal(a["xt"][0], x.astype(np.float32))
        for p, h in enumerate(hs, start=1):
            assert np.array_equal(a["xt"][p], (h[None, :] * x).astype(np.float32))
        assert np.all(a["xt_pad"] == 0)
        return
    if gl.fmt == "abq":
        Qx, dx, zx = O.quantize_rows_asym(x, gl.a_bits)
        assert np.array_equal(a["codes"].astype(np.int32), Qx)
        if 16 <= gl.M <= 64:   # the copy in the operand layout the tensor-core layer reads
            assert np.array_equal(a["codes_t"].astype(np.int32), Qx)
            assert not a["codes_t_pad"].any() and not a["codes_t_pad_tokens"].any()
        else:
            assert "codes_t" not in a
        assert np.array_equal(a["scale"], dx) and np.array_equal(a["zero"], zx)
        assert np.array_equal(a["sum"], Qx.sum(1).astype(np.int32))
    else:
        q, gamma = O.quantize_act_int8(x)
        assert np.array_equal(a["codes"], q)
        assert np.array_equal(a["scale"], gamma)
        assert np.array_equal(a["sum"], q.astype(np.int64).sum(1))
        if gl.fmt == "bvsr":
            gs = q.astype(np.int64).reshape(gl.M, -1, 32).sum(2)
            assert np.array_equal(a["gsum"], gs)
        if gl.fmt == "ternary":
            z_ref = x.astype(np.float64) @ L.read_packed(gl.packed)["A"].astype(np.float64)
            z = a["u_part"].astype(np.float64).sum(0)
            assert np.allclose(z, z_ref, rtol=1e-4, atol=1e-4 * (np.abs(z_ref).max() + 1e-6))
    assert np.all(a["codes_pad"] == 0)
