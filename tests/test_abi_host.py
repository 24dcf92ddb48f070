"""The C-ABI library on the host (no GPU): it loads, exports every declared
call, sizes buffers per the documented layout, and rejects bad arguments with
the documented status before anything is enqueued."""
import ctypes
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

from bit_weight_quantization_b200 import bq
from oracle import layout as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "bq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bq_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", bq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(bq.EXPORTED) == set(names)


def test_status_strings_and_version():
    assert bq.bq_version() == bq.BQ_ABI_VERSION == 4
    hdr = open(os.path.join(ROOT, "include", "bq.h")).read()
    assert re.search(r"#define BQ_ABI_VERSION (\d+)", hdr).group(1) == str(bq.BQ_ABI_VERSION)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_binding_structs_match_the_c_header(tmp_path):
    """Every field offset and the size of each ctypes struct equal what a C compiler makes of
    include/bq.h."""
    structs = {"bq_pack_desc": bq.bq_pack_desc, "bq_layer": bq.bq_layer, "bq_plan_info": bq.bq_plan_info}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "bq.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for f, _ in cls._fields_:
            lines.append(f'  printf("{name} {f} %zu\\n", offsetof({name}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "offsets.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "offsets"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    got = dict(l.rsplit(" ", 1) for l in subprocess.run([str(exe)], check=True, capture_output=True,
                                                       text=True).stdout.splitlines())
    for name, cls in structs.items():
        assert int(got[f"{name} size"]) == ctypes.sizeof(cls), name
        for f, _ in cls._fields_:
            assert int(got[f"{name} {f}"]) == getattr(cls, f).offset, (name, f)
    assert bq.bq_status_str(0) == "ok"
    assert "device" in bq.bq_status_str(6)


@pytest.mark.parametrize("fmt,kw,N,K,expect", [
    ("bitnet", {}, 4096, 4096, 256 + 4096 * 4096 // 8),
    ("bitnet", {}, 50, 384, 256 + 64 * 512 // 8),
    ("ternary", dict(lora_rank=32), 2048, 2048, 256 + 2048 * 2048 // 4 + 2048 * 32 * 2 * 2),
    ("abq", dict(w_bits=6, a_bits=6), 4096, 4096, 256 + 4096 * 4096 * 6 // 8 + 3 * 4096 * 4),
    ("bvsr", {}, 5120, 5120, 256 + 5120 * 5120 // 2 + 256 * 8 * 4 + 10240 + 5120 * 5120 // 32),
    # RaBiT: P sign planes, g [P][N], h [P][K] f32
    ("rabit", {}, 256, 512, 256 + 2 * 256 * 512 // 8 + 2 * 256 * 4 + 2 * 512 * 4),
    ("rabit3", {}, 256, 512, 256 + 3 * 256 * 512 // 8 + 3 * 256 * 4 + 3 * 512 * 4),
])
def test_packed_bytes_match_layout(fmt, kw, N, K, expect):
    d = bq.make_desc(fmt, **kw)
    assert bq.bq_packed_bytes(d, N, K) == expect


def test_packed_bits_per_weight():
    # 2 bits/weight ternary packing, 1 bit BitNet, w bits ABQ, 4 + 8/32 BVSR (planes + set index)
    N = K = 4096
    for fmt, kw, bits in [("bitnet", {}, 1), ("ternary", {}, 2), ("abq", dict(w_bits=2, a_bits=8), 2),
                          ("abq", dict(w_bits=8, a_bits=8), 8)]:
        tot = bq.bq_packed_bytes(bq.make_desc(fmt, **kw), N, K)
        assert tot - 256 - (3 * N * 4 if fmt == "abq" else 0) == N * K * bits // 8
    tot = bq.bq_packed_bytes(bq.make_desc("bvsr"), N, K)
    assert tot - 256 - 256 * 8 * 4 - 10240 == N * K * 4.25 / 8   # table, then 10 KB of pack scratch


@pytest.mark.parametrize("N,K,status", [(0, 256, 3), (16, 0, 3), (16, 200, 3), (16, 64, 3),
                                        ((1 << 20) + 1, 256, 3), (16, (1 << 16) + 128, 3)])
def test_packed_bytes_rejects_sizes(N, K, status):
    d = bq.make_desc("bitnet")
    out = ctypes.c_size_t()
    assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), N, K, ctypes.byref(out)) == status


def test_bad_descriptors():
    out = ctypes.c_size_t()
    for d, st in [(bq.make_desc(9), 1), (bq.make_desc("abq", 0, 8), 1), (bq.make_desc("abq", 8, 9), 1),
                  (bq.make_desc("ternary", lora_rank=65, lora_A=16, lora_B=16), 1),
                  (bq.make_desc("ternary", lora_rank=8), 0), (bq.make_desc("rabit"), 0)]:
        assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 256, ctypes.byref(out)) == st
    # the pack call itself needs the device pointers the format reads
    layer = bq.bq_layer()
    fake = 1 << 40
    for d in (bq.make_desc("rabit"), bq.make_desc("ternary", lora_rank=8)):
        assert bq.raw_status("bq_pack_weights", ctypes.byref(d), fake, 64, 256, fake, 1 << 30, None,
                             ctypes.byref(layer)) == 1
    # (2^8-1)^2 * K must stay below 2^31 for exact int32 plane sums
    d = bq.make_desc("abq", 8, 8)
    assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 33024, ctypes.byref(out)) == 0
    assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 33152, ctypes.byref(out)) == 3
    assert bq.raw_status("bq_packed_bytes", None, 64, 256, ctypes.byref(out)) == 1


def test_pack_rejects_before_launch():
    d = bq.make_desc("bitnet")
    layer = bq.bq_layer()
    nbytes = bq.bq_packed_bytes(d, 64, 256)
    fake = 1 << 40   # never dereferenced: validation fails first
    args = lambda W, P, n: (ctypes.byref(d), W, 64, 256, P, n, None, ctypes.byref(layer))
    assert bq.raw_status("bq_pack_weights", *args(None, fake, nbytes)) == 1      # null W
    assert bq.raw_status("bq_pack_weights", *args(fake + 4, fake, nbytes)) == 1  # W not 16-aligned
    assert bq.raw_status("bq_pack_weights", *args(fake, fake + 16, nbytes)) == 1  # packed not 256-aligned
    assert bq.raw_status("bq_pack_weights", *args(fake, fake, nbytes - 1)) == 3  # buffer too small
    assert bq.raw_status("bq_pack_weights", ctypes.byref(d), fake, 64, 257, fake, nbytes, None,
                         ctypes.byref(layer)) == 3                                    # K % 128 != 0


def _host_header(fmt, N, K, **kw):
    """A packed header written by the oracle side from the documented layout."""
    d = bq.make_desc(fmt, **kw)
    total = bq.bq_packed_bytes(d, N, K)
    N_pad, K_pad = -(-N // 16) * 16, -(-K // 256) * 256
    h = np.zeros(64, "<u4")
    h[0], h[1], h[2], h[3], h[4], h[5], h[6] = L.PK_MAGIC, 1, bq.FORMATS[fmt], N, K, N_pad, K_pad
    # BVSR: one stream of 4-bit codes in the nibble order of its tiles
    fields = {"bitnet": [1], "ternary": [2], "bvsr": [4], "rabit": [1, 1], "rabit3": [1, 1, 1]}.get(fmt)
    P = len(fields) if fmt.startswith("rabit") else 0
    if fmt == "abq":
        w = kw["w_bits"]
        fields, rem = [], w
        while rem:
            f = 8 if rem >= 8 else 4 if rem >= 4 else 2 if rem >= 2 else 1
            fields.append(f)
            rem -= f
    h[7] = {"bitnet": 1, "ternary": 2, "bvsr": 4, "rabit": 2, "rabit3": 3}.get(fmt, kw.get("w_bits", 0))
    h[8] = 16 if P else kw.get("a_bits", 8)
    h[9] = len(fields)
    sh = 0
    for i, f in enumerate(fields):
        h[10 + i], h[14 + i] = f, (i if P else sh)
        sh += f
    h[18] = 0 if P else 512 * sum(fields) + (128 if fmt == "bvsr" else 0)
    h[19] = kw.get("lora_rank", 0)
    tiles = P * N_pad * K_pad // 8 if P else (N_pad // 16) * (K_pad // 256) * h[18]
    rows = 3 * N_pad * 4 if fmt == "abq" else P * N_pad * 4
    a256 = lambda v: (v + 255) // 256 * 256
    off_rows = a256(256 + tiles)
    aux = K_pad * 4 if P else {"ternary": K_pad * h[19] * 2, "bvsr": 256 * 8 * 4 + 10240}.get(fmt, 0)
    aux2 = (P - 1) * K_pad * 4 if P else {"ternary": N_pad * h[19] * 2}.get(fmt, 0)
    off_aux = a256(off_rows + rows)
    off_aux2 = a256(off_aux + aux)
    for word, v in [(22, total), (24, 256), (26, off_rows), (28, off_aux), (30, off_aux2)]:
        h[word], h[word + 1] = v & 0xFFFFFFFF, v >> 32
    assert a256(off_aux2 + aux2) == total
    return h


@pytest.mark.parametrize("fmt,kw", [("bitnet", {}), ("ternary", dict(lora_rank=32)),
                                    ("abq", dict(w_bits=6, a_bits=6)), ("bvsr", {})])
def test_packed_validate_host_header(fmt, kw):
    h = _host_header(fmt, 300, 1024, **kw)
    layer = bq.bq_packed_validate(h.tobytes(), 1 << 20)
    assert (layer.fmt, layer.N, layer.K, layer.N_pad, layer.K_pad) == (bq.FORMATS[fmt], 300, 1024, 304, 1024)
    assert bq.bq_act_bytes(layer, 1) > 256
    bad = h.copy()
    bad[26] += 256                              # wrong section offset
    with pytest.raises(bq.BQError) as e:
        bq.bq_packed_validate(bad.tobytes(), 1 << 20)
    assert e.value.status == bq.BQ_ERR_BAD_PACKED
    bad = h.copy()
    bad[0] ^= 1                                 # wrong magic
    with pytest.raises(bq.BQError):
        bq.bq_packed_validate(bad.tobytes(), 1 << 20)


def test_act_and_gemv_reject_before_launch():
    h = _host_header("bitnet", 64, 256)
    layer = bq.bq_packed_validate(h.tobytes(), 1 << 20)
    nact = bq.bq_act_bytes(layer, 2)
    assert nact == 256 + 512 + 256   # header, codes 2 x 256, token params padded to 256
    L_ = ctypes.byref(layer)
    fake = 1 << 40
    assert bq.raw_status("bq_quantize_act", L_, fake, 65, fake, nact, None) == 3       # M > 64
    assert bq.raw_status("bq_quantize_act", L_, fake + 2, 2, fake, nact, None) == 1    # x unaligned
    assert bq.raw_status("bq_quantize_act", L_, fake, 2, fake, nact - 1, None) == 3    # act too small
    assert bq.raw_status("bq_quantize_act", L_, fake, 0, fake, 0, None) == 0           # M = 0: no-op
    assert bq.raw_status("bq_gemm", L_, fake + 128, 2, fake, None, None) == 1          # act unaligned
    assert bq.raw_status("bq_gemm", L_, fake, 2, None, None, None) == 1                # null y
    assert bq.raw_status("bq_gemm", L_, fake, 0, fake, None, None) == 0                # M = 0: no-op
    assert bq.raw_status("bq_gemm", None, fake, 1, fake, None, None) == 1


def test_static_scratch_rejects_before_launch():
    """Null layer / bad sizes are refused on the host, before any device work."""
    assert bq.raw_status("bq_linear_static_scratch", None, None, 1, None, None, None) == bq.BQ_ERR_INVALID_ARG


def test_linear_group_rejects_before_launch():
    """Grouped layers: sizes, mismatches and unsupported formats are refused on the host."""
    def layer(fmt, N, K, **kw):
        return bq.bq_packed_validate(_host_header(fmt, N, K, **kw).tobytes(), 1 << 20)
    fake = 1 << 40
    a, b = layer("bitnet", 64, 256), layer("bitnet", 32, 256)
    ys = [fake, fake]

    def st(layers, M=1, x=fake, y=ys):
        arr = (bq.bq_layer * len(layers))(*layers)
        yp = (ctypes.c_void_p * len(y))(*y)
        return bq.raw_status("bq_linear_group", arr, len(layers), x, M, yp, None, None)
    assert st([a, b], M=0) == bq.BQ_OK                                  # nothing to do
    assert st([a, b], M=65) == bq.BQ_ERR_SIZE
    assert st([a, b], x=fake + 2) == bq.BQ_ERR_INVALID_ARG               # x unaligned
    assert st([a, b], y=[fake, 0]) == bq.BQ_ERR_INVALID_ARG              # null y
    assert st([a, layer("bitnet", 32, 512)]) == bq.BQ_ERR_INVALID_ARG    # K differs
    assert st([a, layer("abq", 32, 256, w_bits=4, a_bits=4)]) == bq.BQ_ERR_INVALID_ARG
    assert st([layer("bvsr", 32, 256)] * 2) == bq.BQ_ERR_UNSUPPORTED
    assert st([layer("ternary", 32, 256, lora_rank=32)] * 2) == bq.BQ_ERR_UNSUPPORTED
    arr = (bq.bq_layer * 5)(*([a] * 5))
    yp = (ctypes.c_void_p * 5)(*([fake] * 5))
    assert bq.raw_status("bq_linear_group", arr, 5, fake, 1, yp, None, None) == bq.BQ_ERR_INVALID_ARG
    assert bq.raw_status("bq_linear_group", arr, 0, fake, 1, yp, None, None) == bq.BQ_ERR_INVALID_ARG


def test_svid_descriptor_checks():
    out = ctypes.c_size_t(0)
    for fmt, rounds, st in [("rabit", -1, bq.BQ_ERR_INVALID_ARG), ("rabit", 1001, bq.BQ_ERR_INVALID_ARG),
                            ("rabit", 20, bq.BQ_OK), ("bitnet", 5, bq.BQ_ERR_INVALID_ARG)]:
        d = bq.make_desc(fmt, rabit_svid_rounds=rounds)
        assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 256, ctypes.byref(out)) == st
    # the SVID pack fits h2 itself (no h2 pointer needed); the plain recursion needs one
    d = bq.make_desc("rabit", rabit_svid_rounds=0)
    fake = 1 << 40
    assert bq.raw_status("bq_pack_weights", ctypes.byref(d), fake, 64, 256, fake, 1 << 30, None,
                         ctypes.byref(bq.bq_layer())) == bq.BQ_ERR_INVALID_ARG


def test_bit_balance_descriptor_checks():
    out = ctypes.c_size_t(0)
    for fmt, w, bal, st in [("abq", 3, 1, bq.BQ_OK), ("abq", 2, 1, bq.BQ_ERR_INVALID_ARG),
                            ("abq", 3, 2, bq.BQ_ERR_INVALID_ARG), ("bitnet", 0, 1, bq.BQ_ERR_INVALID_ARG)]:
        d = bq.make_desc(fmt, w_bits=w, a_bits=8, abq_bit_balance=bal)
        assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 256, ctypes.byref(out)) == st


def test_compensation_descriptor_checks():
    """a and b: both or neither, ABQ only, 4-byte aligned; refused before anything runs."""
    out = ctypes.c_size_t(0)
    fake = 1 << 40
    d = bq.make_desc("bitnet", abq_comp_a=fake, abq_comp_b=fake)
    assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 256, ctypes.byref(out)) == bq.BQ_ERR_INVALID_ARG
    d = bq.make_desc("abq", w_bits=4, a_bits=4, abq_comp_a=fake, abq_comp_b=fake)
    assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 256, ctypes.byref(out)) == bq.BQ_OK
    plain = bq.make_desc("abq", w_bits=4, a_bits=4)
    assert bq.bq_packed_bytes(d, 64, 256) == bq.bq_packed_bytes(plain, 64, 256)   # same buffer
    for a, b in [(fake, None), (None, fake), (fake + 2, fake), (fake, fake + 1)]:
        d = bq.make_desc("abq", w_bits=4, a_bits=4, abq_comp_a=a, abq_comp_b=b)
        assert bq.raw_status("bq_pack_weights", ctypes.byref(d), fake, 64, 256, fake, 1 << 30, None,
                             ctypes.byref(bq.bq_layer())) == bq.BQ_ERR_INVALID_ARG


@pytest.mark.parametrize("fmt", ["rabit", "rabit3"])
def test_rabit_host_header_and_act_bytes(fmt):
    """The documented RaBiT layout validates; the act buffer holds P x M x K_pad f32 (h_p x);
    the layer kernel of the tiled formats has no plan for it."""
    P = 2 if fmt == "rabit" else 3
    layer = bq.bq_packed_validate(_host_header(fmt, 300, 640).tobytes(), 1 << 20)
    assert (layer.fmt, layer.N_pad, layer.K_pad, layer.w_bits) == (bq.FORMATS[fmt], 304, 768, P)
    assert bq.bq_act_bytes(layer, 5) == 256 + 256 + P * 5 * 768 * 4   # header, token words, xt
    with pytest.raises(bq.BQError) as e:
        bq.bq_linear_plan(layer, 1)
    assert e.value.status == bq.BQ_ERR_UNSUPPORTED


def test_rabit3_descriptor_checks():
    out = ctypes.c_size_t(0)
    fake = 1 << 40
    for d, st in [(bq.make_desc("rabit3"), bq.BQ_OK),
                  (bq.make_desc("rabit3", rabit_svid_rounds=20), bq.BQ_ERR_INVALID_ARG),   # recursion only
                  (bq.make_desc("rabit", h3=fake), bq.BQ_ERR_INVALID_ARG),                 # h3: format 6 only
                  (bq.make_desc("bitnet", h3=fake), bq.BQ_ERR_INVALID_ARG)]:
        assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 256, ctypes.byref(out)) == st
    for h2, h3 in [(fake, None), (None, fake), (fake, fake + 2)]:
        d = bq.make_desc("rabit3", h2=h2, h3=h3)
        assert bq.raw_status("bq_pack_weights", ctypes.byref(d), fake, 64, 256, fake, 1 << 30, None,
                             ctypes.byref(bq.bq_layer())) == bq.BQ_ERR_INVALID_ARG


def _plan_cases():
    return [("bitnet", 4096, 4096, {}), ("bitnet", 11008, 4096, {}), ("bitnet", 4096, 11008, {}),
            ("bitnet", 300, 40960, {}), ("ternary", 2048, 2048, dict(lora_rank=32)),
            ("abq", 4096, 4096, dict(w_bits=2, a_bits=8)), ("abq", 11008, 4096, dict(w_bits=8, a_bits=8)),
            ("bvsr", 5120, 13824, {}), ("bvsr", 64, 256, {})]


def fused_call(fmt, M, fused):
    """Whether bq_linear runs the fused kernel (ABQ from 2 tokens and BVSR from 16 go through
    an act buffer), or fused is False (bq_gemm)."""
    return fused and not ((fmt == "abq" and M >= 2) or (fmt == "bvsr" and M >= 16))


@pytest.mark.parametrize("fmt,N,K,kw", _plan_cases())
@pytest.mark.parametrize("M", [1, 3, 8, 9, 64])
@pytest.mark.parametrize("fused", [True, False])
def test_linear_plan_invariants(fmt, N, K, kw, M, fused):
    """The launch plan covers every token, k tile and row block, and fits the SM (host only)."""
    h = _host_header(fmt, N, K, **kw)
    p = bq.bq_linear_plan(bq.bq_packed_validate(h.tobytes(), 1 << 30), M, fused)
    K_pad, N_pad, tile_bytes = int(h[6]), int(h[5]), int(h[18])
    KT, RB, npad = K_pad // 256, N_pad // 16, K_pad // 8
    pow2 = lambda t: 1 << (t - 1).bit_length()
    chunks = lambda t: -(-npad // (256 // pow2(t)))
    tpc, J = p["tokens_per_cta"], p["x_chunks_per_thread"]
    tmax = 16 if fmt == "bvsr" and not fused_call(fmt, M, fused) else 8   # BVSR from an act buffer: two MMA groups
    assert 1 <= tpc <= min(tmax, M) and p["token_groups"] == -(-M // tpc)
    if (fmt == "abq" and M >= 2) or (fmt == "bvsr" and M >= 16):   # bq_linear quantizes once
        fused = False                                                # into an act buffer, then the layer
    if fused:   # the most tokens whose x fits 16 chunks per thread; else one token read twice
        fits = [t for t in range(1, min(8, M) + 1) if chunks(t) <= 16]
        assert tpc == (max(fits) if fits else 1)
        assert J == (chunks(tpc) if fits else 0)
    else:       # the most tokens whose int8 codes fit 96 KB
        cstride = KT * 256 + 16
        assert J == 0 and tpc == max([t for t in range(1, min(tmax, M) + 1) if t * cstride <= 96 * 1024] + [1])
    cps = 2 if fmt == "bvsr" and tpc == 1 and fused else 1   # CTAs of one launch per SM (148 SMs when no device)
    CPG = p["ctas_per_group"]
    assert CPG == max(1, min(RB, -(-cps * 148 // p["token_groups"])))
    wpr, T = p["warps_per_row_block"], p["tiles_per_warp"]
    assert wpr in (1, 2, 4, 8) and T == -(-KT // wpr)
    assert fmt != "bvsr" or wpr >= 4   # a BVSR tile is a long chain: at least 4 warps a row block
    S, C = p["ring_stages"], p["tiles_per_stage"]
    ipc = -(-RB // CPG)
    active = min(8 // wpr, ipc) * wpr   # warps that hold row blocks share the ring
    big = ipc * KT * tile_bytes > 128 * 1024 and cps == 1   # a large slab takes the SM's whole ring
    assert 2 <= S <= 4 and 1 <= C <= T and active * S * C * tile_bytes <= (220 if big else 96) * 1024
    assert p["shared_bytes"] % 128 == 0 and active * S * C * tile_bytes < p["shared_bytes"] <= 227 * 1024


def test_linear_plan_of_the_measured_llama7b_layers():
    """The decode plans of the Llama-7B BitNet layers whose timings and DRAM traffic were
    measured; a change here means those measurements are of another plan."""
    want = {(4096, 4096): (4, 4, 4, 2), (11008, 4096): (1, 4, 9, 2), (4096, 11008): (4, 4, 6, 6)}
    for (N, K), (wpr, S, C, J) in want.items():
        p = bq.bq_linear_plan(bq.bq_packed_validate(_host_header("bitnet", N, K).tobytes(), 1 << 30), 1)
        got = (p["warps_per_row_block"], p["ring_stages"], p["tiles_per_stage"], p["x_chunks_per_thread"])
        assert got == (wpr, S, C, J), (N, K, got)


def test_linear_plan_rejects():
    layer = bq.bq_packed_validate(_host_header("bitnet", 64, 256).tobytes(), 1 << 20)
    info = bq.bq_plan_info()
    for M, st in [(0, bq.BQ_ERR_SIZE), (65, bq.BQ_ERR_SIZE), (1, bq.BQ_OK)]:
        assert bq.raw_status("bq_linear_plan", ctypes.byref(layer), M, 1, ctypes.byref(info)) == st
    assert bq.raw_status("bq_linear_plan", ctypes.byref(layer), 1, 1, None) == bq.BQ_ERR_INVALID_ARG
    assert bq.raw_status("bq_linear_plan", None, 1, 1, ctypes.byref(info)) == bq.BQ_ERR_INVALID_ARG


def test_rabit3_size_matches_the_hand_fixture():
    """The library's buffer size for the hand-derived three-path fixture's shape is the fixture's."""
    import json
    c = json.load(open(os.path.join(ROOT, "tests", "golden", "layout_bits.json")))["rabit3_one_bit"]
    assert bq.bq_packed_bytes(bq.make_desc("rabit3"), c["N"], c["K"]) == c["sizes"]["total"]


def test_product_path_never_imports_the_oracle():
    """The package (binding, build, CUDA sources) never touches oracle/ or tests/; bench.py
    imports the oracle only inside oracle_sample (its CPU-baseline and reference legs)."""
    import ast
    pkg = os.path.join(ROOT, "bit_weight_quantization_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn), encoding="utf-8").read()
                assert not re.search(r"\b(import|from)\s+(oracle|tests)\b|#include\s+\"[^\"]*oracle", src), fn
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    parent = {c: n for n in ast.walk(tree) for c in ast.iter_child_nodes(n)}
    found = 0
    for node in ast.walk(tree):
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [node.module or ""] if isinstance(node, ast.ImportFrom) else [a.name for a in node.names]
            if any(n.split(".")[0] == "oracle" for n in names):
                fn = parent.get(node)
                while fn is not None and not isinstance(fn, ast.FunctionDef):
                    fn = parent.get(fn)
                assert fn is not None and fn.name == "oracle_sample", ast.dump(node)
                found += 1
    assert found >= 1


def test_packed_validate_refuses_every_inconsistent_word():
    """A header must be exactly what the pack writes: each single-word corruption below is
    BQ_ERR_BAD_PACKED, including a ternary rank that is not a multiple of 8 (the kernels load
    the correction rows 16 bytes at a time)."""
    def bad(fmt, kw, word, value, N=64, K=256):
        h = _host_header(fmt, N, K, **kw)
        h[word] = value
        with pytest.raises(bq.BQError) as e:
            bq.bq_packed_validate(h.tobytes(), 1 << 20)
        assert e.value.status == bq.BQ_ERR_BAD_PACKED, (fmt, word, value)
    f32 = lambda v: int(np.array([v], "<f4").view("<u4")[0])
    bad("bitnet", {}, 7, 2)                                  # w_bits
    bad("bitnet", {}, 8, 4)                                  # a_bits
    bad("bvsr", {}, 10, 2)                                   # a field width
    bad("abq", dict(w_bits=6, a_bits=6), 15, 3)              # a stream shift
    bad("bitnet", {}, 19, 8)                                 # a correction rank on BitNet
    bad("ternary", dict(lora_rank=32), 19, 28)               # rank changed: sizes disagree
    bad("ternary", dict(lora_rank=32), 20, f32(np.nan))      # gate alpha
    bad("bitnet", {}, 20, f32(0.1))                          # alpha on a format without a correction
    bad("bitnet", {}, 21, f32(-1.0))                         # negative tensor scale
    bad("ternary", {}, 21, f32(np.inf))
    bad("abq", dict(w_bits=4, a_bits=4), 21, f32(1.0))       # a tensor scale where none is used
    bad("rabit3", {}, 40, 1)                                 # a reserved word
    # the documented values themselves pass
    h = _host_header("ternary", 64, 256, lora_rank=32)
    h[20], h[21] = f32(0.1), f32(0.02)
    bq.bq_packed_validate(h.tobytes(), 1 << 20)


def test_packed_validate_refuses_a_rank_not_a_multiple_of_8():
    """Ternary rank 12 with sections sized consistently for it (N 64, K 256, by hand: tiles
    4 x 1024 at 256, A bf16 [256][12] at 4352, B^T bf16 [64][12] at align256(4352 + 6144) =
    10496, total align256(10496 + 1536) = 12032): only the rank rule can refuse it."""
    h = _host_header("ternary", 64, 256, lora_rank=32)
    h[19] = 12
    for word, v in [(22, 12032), (26, 4352), (28, 4352), (30, 10496)]:
        h[word], h[word + 1] = v, 0
    with pytest.raises(bq.BQError) as e:
        bq.bq_packed_validate(h.tobytes(), 1 << 20)
    assert e.value.status == bq.BQ_ERR_BAD_PACKED
    h[19] = 16   # a multiple of 8 with sizes for 16 passes
    for word, v in [(22, 256 + 4096 + 256 * 16 * 2 + 64 * 16 * 2), (26, 4352), (28, 4352), (30, 4352 + 8192)]:
        h[word], h[word + 1] = v, 0
    assert bq.bq_packed_validate(h.tobytes(), 1 << 20).lora_rank == 16


def test_pack_refuses_a_non_finite_gate():
    out = ctypes.c_size_t(0)
    for alpha in (float("inf"), float("nan")):
        d = bq.make_desc("ternary", lora_rank=8, lora_alpha=alpha)
        assert bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 256, ctypes.byref(out)) == bq.BQ_ERR_INVALID_ARG


def test_hand_made_layer_descriptors_follow_the_pack_rules():
    """A bq_layer built or edited by hand meets the pack's rules in every call: ternary rank a
    multiple of 8 within 0..64, no rank for other formats, ABQ within the int32 bound."""
    def status(layer):
        out = ctypes.c_size_t(0)
        return bq.raw_status("bq_act_bytes", ctypes.byref(layer), 1, ctypes.byref(out))
    t = bq.bq_packed_validate(_host_header("ternary", 64, 256, lora_rank=32).tobytes(), 1 << 20)
    assert status(t) == bq.BQ_OK
    for r in (12, -8, 72):
        t.lora_rank = r
        assert status(t) == bq.BQ_ERR_INVALID_ARG, r
    b = bq.bq_packed_validate(_host_header("bitnet", 64, 256).tobytes(), 1 << 20)
    b.lora_rank = 8
    assert status(b) == bq.BQ_ERR_INVALID_ARG
    a = bq.bq_packed_validate(_host_header("abq", 64, 65536, w_bits=8, a_bits=7).tobytes(), 1 << 30)
    assert status(a) == bq.BQ_OK                     # 255 * 127 * 65536 = 2,122,383,360 < 2^31
    a.a_bits = 8
    assert status(a) == bq.BQ_ERR_INVALID_ARG        # 255 * 255 * 65536 = 4,261,478,400 >= 2^31


def _rand_int(rng):
    return rng.choice([rng.randint(-3, 10), rng.randint(-100, 70000), rng.getrandbits(31), -rng.getrandbits(31)])


def test_host_queries_under_random_arguments():
    """Seeded fuzz of the host-only calls: random descriptors, sizes and hand-edited layer
    descriptors always get a status back, and whatever is accepted has sane sizes (256-byte
    multiples, a plan that fits the SM)."""
    import random
    rng = random.Random(1234)
    layers = [("bitnet", {}), ("ternary", dict(lora_rank=32)), ("abq", dict(w_bits=4, a_bits=4)),
              ("bvsr", {}), ("rabit", {}), ("rabit3", {})]
    for _ in range(1500):
        d = bq.bq_pack_desc(rng.randint(-1, 8), _rand_int(rng), _rand_int(rng), _rand_int(rng),
                            rng.choice([0.1, float("nan"), float("inf")]), None, None, None,
                            _rand_int(rng) if rng.random() < 0.3 else 0, _rand_int(rng) if rng.random() < 0.3 else 0,
                            None, None, None)
        out = ctypes.c_size_t(0)
        K = rng.choice([_rand_int(rng), 128 * rng.randint(1, 600)])
        if bq.raw_status("bq_packed_bytes", ctypes.byref(d), _rand_int(rng), K, ctypes.byref(out)) == bq.BQ_OK:
            assert out.value >= 256 and out.value % 256 == 0
        fmt, kw = rng.choice(layers)
        L_ = bq.bq_packed_validate(_host_header(fmt, rng.randint(1, 3000), 128 * rng.randint(1, 64), **kw).tobytes(),
                                   1 << 30)
        for f in rng.sample(["fmt", "N", "K", "N_pad", "K_pad", "w_bits", "a_bits", "lora_rank"], rng.randint(0, 2)):
            setattr(L_, f, _rand_int(rng))
        o = ctypes.c_size_t(0)
        if bq.raw_status("bq_act_bytes", ctypes.byref(L_), rng.choice([0, 1, 64, 65]), ctypes.byref(o)) == bq.BQ_OK:
            assert o.value % 256 == 0
        info = bq.bq_plan_info()
        if bq.raw_status("bq_linear_plan", ctypes.byref(L_), rng.choice([1, 8, 64]), 1, ctypes.byref(info)) == bq.BQ_OK:
            assert 0 < info.shared_bytes <= 227 * 1024 and info.ring_stages >= 2


def test_packed_validate_under_mutated_headers():
    """Seeded fuzz: valid headers with one to three words overwritten are either refused with
    BQ_ERR_BAD_PACKED or describe a layer the host queries accept."""
    import random
    rng = random.Random(99)
    layers = [("bitnet", {}), ("ternary", dict(lora_rank=32)), ("abq", dict(w_bits=3, a_bits=5)), ("bvsr", {}),
              ("rabit", {}), ("rabit3", {})]
    for _ in range(1500):
        fmt, kw = rng.choice(layers)
        h = _host_header(fmt, rng.randint(1, 5000), 128 * rng.randint(1, 100), **kw)
        for _ in range(rng.randint(1, 3)):
            w = rng.randint(1, 63)
            h[w] = rng.choice([0, 1, 0xFFFFFFFF, rng.getrandbits(32), (int(h[w]) + rng.choice([-256, -1, 1, 256])) & 0xFFFFFFFF])
        try:
            layer = bq.bq_packed_validate(h.tobytes(), 1 << 20)
        except bq.BQError as e:
            assert e.status == bq.BQ_ERR_BAD_PACKED
            continue
        assert bq.bq_act_bytes(layer, 1) % 256 == 0


def test_pack_refuses_unaligned_or_missing_correction_matrices():
    fake = 1 << 40
    for A, B in [(None, fake), (fake, None), (fake + 2, fake), (fake, fake + 1)]:
        d = bq.make_desc("ternary", lora_rank=8, lora_A=A, lora_B=B)
        assert bq.raw_status("bq_pack_weights", ctypes.byref(d), fake, 64, 256, fake, 1 << 30, None,
                             ctypes.byref(bq.bq_layer())) == bq.BQ_ERR_INVALID_ARG


def test_bvsr_cluster_rounds_are_checked():
    """bvsr_cluster_rounds: 0..100 for BVSR, 0 for every other format (host only)."""
    fake = 1 << 40
    layer = bq.bq_layer()
    for fmt, r, ok in [("bvsr", 0, True), ("bvsr", 8, True), ("bvsr", 100, True), ("bvsr", 101, False),
                       ("bvsr", -1, False), ("bitnet", 1, False), ("abq", 2, False)]:
        kw = dict(w_bits=4, a_bits=4) if fmt == "abq" else {}
        d = bq.make_desc(fmt, bvsr_cluster_rounds=r, **kw)
        st = bq.raw_status("bq_packed_bytes", ctypes.byref(d), 64, 256, ctypes.byref(ctypes.c_size_t()))
        assert (st == bq.BQ_OK) == ok, (fmt, r, st)
    assert layer is not None and fake


@pytest.mark.parametrize("M", [1, 4, 15, 16, 17, 64])
def test_bvsr_linear_workspace_is_the_act_buffer_from_16_tokens(M):
    """bq_linear on BVSR runs fused (no workspace) below 16 tokens and through an act buffer
    (its workspace) from 16 on."""
    layer = bq.bq_packed_validate(_host_header("bvsr", 512, 1280).tobytes(), 1 << 30)
    ws = bq.bq_linear_workspace_bytes(layer, M)
    if M < 16:
        assert ws == 0
    else:
        assert ws == bq.bq_act_bytes(layer, M) > 0


@pytest.mark.parametrize("M", [2, 15, 16, 17, 33, 64])
def test_abq_act_bytes_and_workspace_follow_the_documented_sections(M):
    """The ABQ act buffer per include/bq.h: header 256, codes M x KT x 256, token words M x 16
    (padded to 256), and for 16 <= M <= 64 the tensor-core copy Mp x KT x 256 (Mp = M rounded up
    to 16); bq_linear's workspace for M >= 2 is that act buffer."""
    h = _host_header("abq", 300, 1280, w_bits=8, a_bits=8)
    layer = bq.bq_packed_validate(h.tobytes(), 1 << 30)
    KT = 1280 // 256
    up = lambda n: (n + 255) // 256 * 256
    want = 256 + up(M * KT * 256) + up(M * 16)
    if 16 <= M <= 64:
        want += up(((M + 15) // 16 * 16) * KT * 256)
    assert bq.bq_act_bytes(layer, M) == want
    assert bq.bq_linear_workspace_bytes(layer, M) == want
