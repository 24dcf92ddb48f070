"""Independent readers of the library's byte formats — test infrastructure only.

These decode a host copy of a packed-weight buffer or an activation buffer,
following the documented byte layout (declared in ``include/bq.h``), back
into plain codes and scales that the reference layers of ``bq_oracle`` take.
Nothing here is shared with the CUDA path; a reader bug and a writer bug
would have to agree on the same wrong index to go unnoticed, and the golden
fixtures in ``tests/golden`` pin single-bit positions by hand.

Packed weight buffer: 256-byte header of little-endian 32-bit words, then
sections at the header's offsets.

  word  field                      word  field
  0     magic 0x4B505142 'BQPK'    18    tile_bytes
  1     version (1)                19    lora_rank
  2     format (1..6)              20    lora_alpha (f32)
  3     N                          21    tensor_scale (f32): BitNet alpha, ternary gamma_W
  4     K                          22-23 total_bytes (u64)
  5     N_pad (multiple of 16)     24-25 off_tiles (u64)
  6     K_pad (multiple of 256)    26-27 off_rows  (u64)
  7     w_bits                     28-29 off_aux   (u64)
  8     a_bits                     30-31 off_aux2  (u64)
  9     n_streams
  10-13 stream field width f_s (bits per weight per stream)
  14-17 stream shift (bit offset of the stream inside the code / plane index)

Tiled weights (formats 2-5): tile (rb, kt) covers rows 16*rb .. +15 and
k = 256*kt .. +255 and sits at off_tiles + (rb*KT + kt)*tile_bytes, with the
streams one after another, stream s taking 512*f_s bytes laid out as
[u < f_s][lane < 32][4 words]. In word r (0..3) of uint4 u of lane = 4g+t,
the f-bit field j (bits f*j .. f*j+f-1) of byte b holds the weight at

  row = 16*rb + g + 8*(r & 1)
  k   = 32*(8*kt + u*(8/f) + j) + 16*(r >> 1) + 4*t + b.

BVSR tiles (one stream, n_streams = 1, field width 4) hold 4-bit codes in their own
nibble order, not the generic field order above: the first 2048 bytes are 4 blocks
i < 4 of [lane < 32][4 words]; word 2*v + h of lane 4g+t in block i holds, for vector
j = 2i + v of the tile, nibble b (bits 4b..4b+3) of its low half the code of
row 16*rb + g and of its high half the code of row 16*rb + g + 8, at
k = 256*kt + 32*j + 16*h + 4*t + b. The tile ends with 128 bytes of set indices:
byte 2048 + 8*g + j holds the set of row 16*rb + g (g < 16 here), vector 8*kt + j
(32 elements each).

RaBiT (format 1: P = 2 paths; format 6: P = 3) is not tiled: plane p (0..P-1)
word w of row n is the uint32 at off_tiles + 4*((p*N_pad + n)*(K_pad/32) + w),
bit j <-> k = 32w + j; a set bit means sign -1. Rows hold g_p as f32 [P][N_pad];
h_1 sits at off_aux and h_2 (.. h_P) at off_aux2, K_pad f32 each, one after another.
"""
from __future__ import annotations

import numpy as np

PK_MAGIC = 0x4B505142
ACT_MAGIC = 0x43415142
FMT_RABIT, FMT_BITNET, FMT_TERNARY, FMT_ABQ, FMT_BVSR, FMT_RABIT3 = 1, 2, 3, 4, 5, 6
FMT_NAMES = {1: "rabit", 2: "bitnet", 3: "ternary", 4: "abq", 5: "bvsr", 6: "rabit3"}


def _u32(buf: bytes, word: int) -> int:
    return int(np.frombuffer(buf, dtype="<u4", count=1, offset=4 * word)[0])


def _u64(buf: bytes, word: int) -> int:
    return int(np.frombuffer(buf, dtype="<u8", count=1, offset=4 * word)[0])


def _f32(buf: bytes, word: int) -> np.float32:
    return np.frombuffer(buf, dtype="<f4", count=1, offset=4 * word)[0]


def read_header(buf: bytes) -> dict:
    """The packed buffer's 64-word header as a dict (documented word layout).
    Pinned by tests (host header fixtures; every GPU pack round trip)."""
    if _u32(buf, 0) != PK_MAGIC:
        raise ValueError("bad packed magic")
    h = dict(version=_u32(buf, 1), fmt=_u32(buf, 2), N=_u32(buf, 3), K=_u32(buf, 4),
             N_pad=_u32(buf, 5), K_pad=_u32(buf, 6), w_bits=_u32(buf, 7), a_bits=_u32(buf, 8),
             n_streams=_u32(buf, 9), tile_bytes=_u32(buf, 18), lora_rank=_u32(buf, 19),
             lora_alpha=_f32(buf, 20), tensor_scale=_f32(buf, 21), total_bytes=_u64(buf, 22),
             off_tiles=_u64(buf, 24), off_rows=_u64(buf, 26), off_aux=_u64(buf, 28),
             off_aux2=_u64(buf, 30))
    h["fields"] = [_u32(buf, 10 + s) for s in range(h["n_streams"])]
    h["shifts"] = [_u32(buf, 14 + s) for s in range(h["n_streams"])]
    return h


def tiled_field_index(N_pad: int, K_pad: int, f: int):
    """For one stream of field width f, the (row, k) that each field of a tile
    holds, as arrays over [u, lane, r, b, j] (the documented formula).
    Pinned by tests (single-bit layout fixtures, tests/golden/layout_bits.json)."""
    u = np.arange(f)[:, None, None, None, None]
    lane = np.arange(32)[None, :, None, None, None]
    r = np.arange(4)[None, None, :, None, None]
    b = np.arange(4)[None, None, None, :, None]
    j = np.arange(8 // f)[None, None, None, None, :]
    g, t = lane // 4, lane % 4
    row = g + 8 * (r & 1) + 0 * (u + b + j)
    kk = 32 * (u * (8 // f) + j) + 16 * (r >> 1) + 4 * t + b
    return row, kk


def read_stream_codes(buf: bytes, h: dict, s: int, row_blocks=None) -> np.ndarray:
    """Stream s of a tiled buffer as unsigned field values (uint8): [N, K], or
    [16*len(row_blocks), K] for a subset of 16-row blocks.
    Pinned by tests (single-bit layout fixtures; GPU pack round trips)."""
    f = h["fields"][s]
    N, K, N_pad, K_pad = h["N"], h["K"], h["N_pad"], h["K_pad"]
    RB, KT, tb = N_pad // 16, K_pad // 256, h["tile_bytes"]
    s_off = sum(512 * h["fields"][i] for i in range(s))
    rbs = np.arange(RB) if row_blocks is None else np.asarray(row_blocks)
    raw = np.frombuffer(buf, dtype=np.uint8, count=RB * KT * tb, offset=h["off_tiles"]).reshape(RB, KT, tb)
    tiles = raw[rbs][:, :, s_off:s_off + 512 * f].reshape(len(rbs), KT, f, 32, 4, 4)
    row_i, k_i = tiled_field_index(N_pad, K_pad, f)
    nj = 8 // f
    mask = (1 << f) - 1
    vals = (tiles[..., None] >> (f * np.arange(nj))) & mask       # [R, KT, f, 32, 4, 4, nj]
    out = np.zeros((16 * len(rbs), K_pad), dtype=np.uint8)
    rb = np.arange(len(rbs))[:, None, None, None, None, None, None]
    kt = np.arange(KT)[None, :, None, None, None, None, None]
    rows, ks = np.broadcast_arrays(16 * rb + row_i[None, None], 256 * kt + k_i[None, None])
    out[rows, ks] = vals
    if row_blocks is None:
        return out[:N, :K]
    return out[:, :K]


def read_bvsr_codes(buf: bytes, h: dict, row_blocks=None) -> np.ndarray:
    """The 4-bit codes of a BVSR buffer (nibble order of its tiles): uint8 [N, K], or
    [16*len(row_blocks), K] for a subset of 16-row blocks.
    Pinned by tests (a hand-derived nibble fixture; GPU pack round trips)."""
    N, K, N_pad, K_pad = h["N"], h["K"], h["N_pad"], h["K_pad"]
    RB, KT, tb = N_pad // 16, K_pad // 256, h["tile_bytes"]
    rbs = np.arange(RB) if row_blocks is None else np.asarray(row_blocks)
    raw = np.frombuffer(buf, dtype=np.uint8, count=RB * KT * tb, offset=h["off_tiles"]).reshape(RB, KT, tb)
    words = np.ascontiguousarray(raw[rbs][:, :, :2048]).view("<u4")
    w = words.reshape(len(rbs), KT, 4, 8, 4, 2, 2)               # [rb][kt][i][g][t][v][h]
    shift = 16 * np.arange(2)[:, None] + 4 * np.arange(4)[None, :]  # [rbit][b]
    nib = (w[..., None, None] >> shift.astype(np.uint32)) & 0xF     # [rb][kt][i][g][t][v][h][rbit][b]
    # row = 16 rb + 8 rbit + g, k = 256 kt + 32 (2i + v) + 16 h + 4 t + b
    arr = nib.transpose(0, 7, 3, 1, 2, 5, 6, 4, 8).reshape(16 * len(rbs), K_pad).astype(np.uint8)
    if row_blocks is None:
        return arr[:N, :K]
    return arr[:, :K]


def read_packed(buf: bytes, row_blocks=None) -> dict:
    """Decode a packed buffer into the dict shape that bq_oracle's layers take.
    ``row_blocks`` (tiled formats) restricts the per-row arrays to those 16-row
    blocks (rows 16*rb .. 16*rb+15, padding rows included); ``rows`` lists them.
    Pinned by tests (single-bit layout fixtures; GPU pack round trips of every format)."""
    h = read_header(buf)
    fmt, N, K, N_pad, K_pad = h["fmt"], h["N"], h["K"], h["N_pad"], h["K_pad"]
    out = dict(header=h)
    rb = row_blocks
    if rb is not None:
        sel = (16 * np.asarray(rb)[:, None] + np.arange(16)[None, :]).ravel()
    else:
        sel = np.arange(N)
    out["rows"] = sel
    if fmt == FMT_RABIT:
        W32 = K_pad // 32
        raw = np.frombuffer(buf, dtype="<u4", count=2 * N_pad * W32, offset=h["off_tiles"])
        planes = raw.reshape(2, N_pad, W32)
        bits = ((planes[..., None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(2, N_pad, K_pad)
        out["B1"] = np.where(bits[0, :N, :K] == 1, -1, 1).astype(np.int8)
        out["B2"] = np.where(bits[1, :N, :K] == 1, -1, 1).astype(np.int8)
        g = np.frombuffer(buf, dtype="<f4", count=2 * N_pad, offset=h["off_rows"])
        out["g1"], out["g2"] = g[:N].copy(), g[N_pad:N_pad + N].copy()
        out["h1"] = np.frombuffer(buf, dtype="<f4", count=K, offset=h["off_aux"]).copy()
        out["h2"] = np.frombuffer(buf, dtype="<f4", count=K, offset=h["off_aux2"]).copy()
    elif fmt == FMT_RABIT3:   # the rabit_pack_paths shape: B [P,N,K], g [P,N], h [P,K]
        P, W32 = 3, K_pad // 32
        raw = np.frombuffer(buf, dtype="<u4", count=P * N_pad * W32, offset=h["off_tiles"])
        bits = ((raw.reshape(P, N_pad, W32)[..., None] >> np.arange(32, dtype=np.uint32)) & 1)
        out["B"] = np.where(bits.reshape(P, N_pad, K_pad)[:, :N, :K] == 1, -1, 1).astype(np.int8)
        g = np.frombuffer(buf, dtype="<f4", count=P * N_pad, offset=h["off_rows"]).reshape(P, N_pad)
        out["g"] = g[:, :N].copy()
        h1 = np.frombuffer(buf, dtype="<f4", count=K, offset=h["off_aux"])
        h23 = np.frombuffer(buf, dtype="<f4", count=(P - 1) * K_pad, offset=h["off_aux2"]).reshape(P - 1, K_pad)
        out["h"] = np.concatenate([h1[None, :], h23[:, :K]]).copy()
    elif fmt == FMT_BITNET:
        neg = read_stream_codes(buf, h, 0, rb)
        out["B"] = np.where(neg == 1, -1, 1).astype(np.int8)
        out["alpha"] = h["tensor_scale"]
    elif fmt == FMT_TERNARY:
        u = read_stream_codes(buf, h, 0, rb).astype(np.int16)
        out["T"] = (u - 1).astype(np.int8)
        out["field_max"] = int(u.max()) if u.size else 0
        out["gamma_w"] = h["tensor_scale"]
        out["lora_alpha"] = h["lora_alpha"]
        r = h["lora_rank"]
        if r > 0:
            A = np.frombuffer(buf, dtype="<u2", count=K_pad * r, offset=h["off_aux"]).reshape(K_pad, r)
            Bt = np.frombuffer(buf, dtype="<u2", count=N_pad * r, offset=h["off_aux2"]).reshape(N_pad, r)
            out["A"] = _bf16_to_f32(A[:K])
            out["B"] = _bf16_to_f32(Bt[sel]).T.copy()
    elif fmt == FMT_ABQ:
        Q = np.zeros((len(sel), K), dtype=np.int32)
        for s in range(h["n_streams"]):
            Q += read_stream_codes(buf, h, s, rb).astype(np.int32) << h["shifts"][s]
        out["Q"] = Q
        rowsec = np.frombuffer(buf, dtype="<u4", count=3 * N_pad, offset=h["off_rows"])
        out["delta"] = rowsec[:N_pad][sel].view("<f4").copy()
        out["z"] = rowsec[N_pad:2 * N_pad][sel].view("<i4").copy()
        out["S_w"] = rowsec[2 * N_pad:3 * N_pad][sel].view("<i4").copy()
        out["w_bits"] = h["w_bits"]
        out["a_bits"] = h["a_bits"]
    elif fmt == FMT_BVSR:
        out["codes"] = read_bvsr_codes(buf, h, rb)
        tab = np.frombuffer(buf, dtype="<f4", count=256 * 8, offset=h["off_aux"]).reshape(256, 8)
        out["table"] = tab[:, :5].copy()
        out["table_derived"] = tab[:, 5:].copy()
        # set index of (row g of the tile, vector j of the tile) at byte 2048 + 8 g + j of the tile
        RB, KT, tb = N_pad // 16, K_pad // 256, h["tile_bytes"]
        raw = np.frombuffer(buf, dtype=np.uint8, count=RB * KT * tb, offset=h["off_tiles"]).reshape(RB, KT, tb)
        rbs = np.arange(RB) if rb is None else np.asarray(rb)
        idx = raw[rbs][:, :, 2048:2048 + 128].reshape(len(rbs), KT, 16, 8)
        sets = idx.transpose(0, 2, 1, 3).reshape(16 * len(rbs), K_pad // 32)
        out["sets"] = (sets[:N] if rb is None else sets)[:, :K // 32].copy()
    else:
        raise ValueError(f"unknown format {fmt}")
    return out


def _bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# activation buffer
# ---------------------------------------------------------------------------
#
# 256-byte header of 32-bit words:
#   0 magic 0x43415142 'BQAC'   1 version   2 format   3 M   4 K   5 K_pad
#   6 a_bits   7 lora_rank   8-9 total_bytes   10-11 off_codes   12-13 off_tok
#   14-15 off_gsum   16-17 off_u   18-19 off_xt   20-21 off_ct (0 when absent)
# codes (formats 2-5): per token m and k-tile kt, 256 bytes; byte
#   (m*KT + kt)*256 + 64*t + 8*mu + 4*h + b  holds the code of
#   k = 32*(8*kt + mu) + 16*h + 4*t + b   (int8 for A8 formats, uint8 for ABQ).
# tok: [M][4] words: A8 {gamma_x f32, sum_q i32, 0, 0}; ABQ {Delta_x f32, z_x i32, S_x i32, 0}
# gsum (BVSR): int32 [M][K_pad/32] sums of q over each 32-element vector
# u (ternary): float32 [KT][M][lora_rank] partial dot products of x and A over each
#   256-k tile; the layer's LoRA input is SiLU(sum over tiles)
# xt (RaBiT): float32 [2][M][K_pad] = h_p * x
# ct (ABQ, 16 <= M <= 64): uint8 [KT][16 k-units][Mp/8][8 tokens][16 bytes], Mp = M rounded
#   up to 16; k-unit 2i + p//16, byte p%16 holds the code of k = 256*kt + 32*i + k' with
#   p = 8*((k'%16)//4) + 4*(k'//16) + k'%4; tokens M .. Mp-1 hold 0


def read_act(buf: bytes) -> dict:
    """An activation buffer decoded into codes, token parameters, vector sums and LoRA
    partials. Pinned by tests (single activation-code fixture; every GPU act round trip)."""
    if _u32(buf, 0) != ACT_MAGIC:
        raise ValueError("bad act magic")
    fmt, M, K, K_pad = _u32(buf, 2), _u32(buf, 3), _u32(buf, 4), _u32(buf, 5)
    a = dict(fmt=fmt, M=M, K=K, K_pad=K_pad, a_bits=_u32(buf, 6), lora_rank=_u32(buf, 7),
             total_bytes=_u64(buf, 8), off_codes=_u64(buf, 10), off_tok=_u64(buf, 12),
             off_gsum=_u64(buf, 14), off_u=_u64(buf, 16), off_xt=_u64(buf, 18), off_ct=_u64(buf, 20))
    KT = K_pad // 256
    if fmt in (FMT_RABIT, FMT_RABIT3):
        P = 2 if fmt == FMT_RABIT else 3
        xt = np.frombuffer(buf, dtype="<f4", count=P * M * K_pad, offset=a["off_xt"])
        a["xt"] = xt.reshape(P, M, K_pad)[:, :, :K].copy()
        a["xt_pad"] = xt.reshape(P, M, K_pad)[:, :, K:].copy()
        return a
    dt = np.uint8 if fmt == FMT_ABQ else np.int8
    raw = np.frombuffer(buf, dtype=dt, count=M * KT * 256, offset=a["off_codes"]).reshape(M, KT, 4, 8, 2, 4)
    t = np.arange(4)[:, None, None, None]
    mu = np.arange(8)[None, :, None, None]
    hh = np.arange(2)[None, None, :, None]
    b = np.arange(4)[None, None, None, :]
    kin = 32 * mu + 16 * hh + 4 * t + b                      # [4,8,2,4]
    codes = np.zeros((M, K_pad), dtype=dt)
    for kt in range(KT):
        codes[:, 256 * kt + kin.ravel()] = raw[:, kt].reshape(M, -1)
    a["codes"] = codes[:, :K]
    a["codes_pad"] = codes[:, K:]
    if a["off_ct"]:  # the tensor-core copy (ABQ with 16..64 tokens)
        Mp = (M + 15) // 16 * 16
        rt = np.frombuffer(buf, dtype=dt, count=KT * Mp * 256, offset=a["off_ct"]).reshape(KT, 16, Mp // 8, 8, 16)
        pos = rt.transpose(2, 3, 0, 1, 4).reshape(Mp, KT, 256)   # [n, kt, 16*unit + byte]
        u, byte = np.arange(256) // 16, np.arange(256) % 16
        p = 16 * (u % 2) + byte                                  # position within the 32-k chunk
        kk = 32 * (u // 2) + 16 * ((p >> 2) & 1) + 4 * (p >> 3) + (p & 3)
        ct = np.zeros((Mp, KT, 256), dtype=dt)
        ct[:, :, kk] = pos
        ct = ct.reshape(Mp, KT * 256)
        a["codes_t"] = ct[:M, :K].copy()
        a["codes_t_pad"] = ct[:M, K:].copy()
        a["codes_t_pad_tokens"] = ct[M:].copy()
    tok = np.frombuffer(buf, dtype="<u4", count=4 * M, offset=a["off_tok"]).reshape(M, 4)
    a["scale"] = tok[:, 0].view("<f4").copy()
    a["zero"] = tok[:, 1].view("<i4").copy()
    a["sum"] = tok[:, 2].view("<i4").copy() if fmt == FMT_ABQ else tok[:, 1].view("<i4").copy()
    if fmt == FMT_BVSR:
        a["gsum"] = np.frombuffer(buf, dtype="<i4", count=M * (K_pad // 32),
                                  offset=a["off_gsum"]).reshape(M, K_pad // 32)[:, :K // 32].copy()
    if fmt == FMT_TERNARY and a["lora_rank"] > 0:
        r = a["lora_rank"]
        a["u_part"] = np.frombuffer(buf, dtype="<f4", count=KT * M * r, offset=a["off_u"]).reshape(KT, M, r).copy()
    return a
