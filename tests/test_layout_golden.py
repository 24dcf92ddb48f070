"""The oracle's byte-format readers against hand-derived single-field positions."""
import numpy as np

from oracle import layout as L


def _packed(fmt, N, K, fields, tile_bytes, body, tensor_scale=1.0):
    N_pad, K_pad = -(-N // 16) * 16, -(-K // 256) * 256
    hdr = np.zeros(64, dtype="<u4")
    hdr[0], hdr[1], hdr[2], hdr[3], hdr[4], hdr[5], hdr[6] = L.PK_MAGIC, 1, fmt, N, K, N_pad, K_pad
    hdr[9] = len(fields)
    for s, f in enumerate(fields):
        hdr[10 + s] = f
    hdr[18] = tile_bytes
    hdr[21] = np.array([tensor_scale], "<f4").view("<u4")[0]
    total = 256 + len(body)
    hdr[22], hdr[24] = total, 256
    return hdr.tobytes() + bytes(body)


def test_bitnet_single_negative(golden):
    g = golden("layout_bits.json")
    for key in ("bitnet_one_negative", "bitnet_second"):
        c = g[key]
        tiles = (c["N"] // 16) * (c["K"] // 256)
        body = bytearray(tiles * c["tile_bytes"])
        body[c["byte"]] = c["value"]
        p = L.read_packed(_packed(L.FMT_BITNET, c["N"], c["K"], [1], c["tile_bytes"], body))
        neg = np.argwhere(p["B"] == -1).tolist()
        assert neg == c["neg"]


def test_ternary_single_plus(golden):
    c = golden("layout_bits.json")["ternary_one_plus"]
    body = bytearray([c["fill"]]) * c["tile_bytes"]
    body[c["byte"]] = c["value"]
    p = L.read_packed(_packed(L.FMT_TERNARY, c["N"], c["K"], [2], c["tile_bytes"], body))
    assert np.argwhere(p["T"] == 1).tolist() == c["plus"]
    assert np.count_nonzero(p["T"]) == 1


def test_act_single_code(golden):
    c = golden("layout_bits.json")["act_one_code"]
    hdr = np.zeros(64, dtype="<u4")
    hdr[0], hdr[1], hdr[2], hdr[3], hdr[4], hdr[5], hdr[6] = L.ACT_MAGIC, 1, L.FMT_BITNET, 1, 256, 256, 8
    hdr[10], hdr[12] = 256, 256 + 256
    body = bytearray(256 + 16)
    body[c["byte"]] = c["value"] & 0xFF
    a = L.read_act(hdr.tobytes() + bytes(body))
    nz = np.nonzero(a["codes"][0])[0].tolist()
    assert nz == [c["k"]] and int(a["codes"][0, c["k"]]) == c["value"]


def test_rabit3_single_bit_scale_and_h(golden):
    """Three-path RaBiT: one sign bit of path 3, one g3 and one h3 at hand-derived byte offsets."""
    c = golden("layout_bits.json")["rabit3_one_bit"]
    z = c["sizes"]
    N, K = c["N"], c["K"]
    hdr = np.zeros(64, dtype="<u4")
    hdr[0], hdr[1], hdr[2], hdr[3], hdr[4], hdr[5], hdr[6] = L.PK_MAGIC, 1, L.FMT_RABIT3, N, K, 32, 512
    hdr[7], hdr[8], hdr[9] = 3, 16, 3
    for word, v in [(22, z["total"]), (24, 256), (26, z["off_rows"]), (28, z["off_aux"]), (30, z["off_aux2"])]:
        hdr[word] = v
    buf = bytearray(z["total"])
    buf[:256] = hdr.tobytes()
    buf[c["sign_byte"]] = c["sign_value"]
    buf[c["g_byte"]:c["g_byte"] + 4] = np.array([c["g"]], "<f4").tobytes()
    buf[c["h_byte"]:c["h_byte"] + 4] = np.array([c["h"]], "<f4").tobytes()
    p = L.read_packed(bytes(buf))
    assert np.argwhere(p["B"] == -1).tolist() == [c["neg"]]
    assert np.argwhere(p["g"] != 0).tolist() == [c["neg"][:2]] and p["g"][2, 17] == c["g"]
    assert np.argwhere(p["h"] != 0).tolist() == [[2, c["neg"][2]]] and p["h"][2, 291] == c["h"]


def test_bvsr_single_nibble_and_set(golden):
    """BVSR: one 4-bit code and one set index at hand-derived byte offsets of the nibble order."""
    c = golden("layout_bits.json")["bvsr_one_nibble"]
    z = c["sizes"]
    N, K = c["N"], c["K"]
    hdr = np.zeros(64, dtype="<u4")
    hdr[0], hdr[1], hdr[2], hdr[3], hdr[4], hdr[5], hdr[6] = L.PK_MAGIC, 1, L.FMT_BVSR, N, K, 16, 256
    hdr[7], hdr[8], hdr[9], hdr[10], hdr[18] = 4, 8, 1, 4, c["tile_bytes"]
    for word, v in [(22, z["total"]), (24, 256), (26, z["off_aux"]), (28, z["off_aux"]), (30, z["total"])]:
        hdr[word] = v
    buf = bytearray(z["total"])
    buf[:256] = hdr.tobytes()
    buf[256 + c["byte"]] = c["value"]
    buf[256 + c["set_byte"]] = c["set"]
    p = L.read_packed(bytes(buf))
    assert np.argwhere(p["codes"] != 0).tolist() == [[c["row"], c["k"]]]
    assert int(p["codes"][c["row"], c["k"]]) == c["code"]
    assert np.argwhere(p["sets"] != 0).tolist() == [[c["row"], c["set_vector"]]]
    assert int(p["sets"][c["row"], c["set_vector"]]) == c["set"]
