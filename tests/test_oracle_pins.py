"""Pins of the CPU oracle to things other than itself (no GPU).

Each test ties one oracle step to a fact fixed outside the oracle: a hand-decoded block
(tests/golden/*.json), a pack/unpack round trip, an exact rational, a closed form, a library
routine (numpy float16, stable argsort, scipy softmax/expit, dense fp64 matmul) or brute force on
tiny inputs.  The choice is meant to make a dropped term, a wrong sign, a wrong index or a
transposed operand in the oracle fail at least one of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special

import oracle
from expert_ffn_token_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _h(hexstr):
    return bytes.fromhex(hexstr.replace(" ", ""))


def _kquant_block(g, size, qs_at, qh_at=None):
    b = bytearray(size)
    b[0:2] = _h(g["block"]["d"])[::-1]          # fixtures write fp16 big-endian (as a number)
    b[2:4] = _h(g["block"]["dmin"])[::-1]
    b[4:16] = _h(g["block"]["scales"])
    for i, v in g["block"].get("qh_nonzero", {}).items():
        b[qh_at + int(i)] = int(v, 16)
    for i, v in g["block"]["qs_nonzero"].items():
        b[qs_at + int(i)] = int(v, 16)
    return np.frombuffer(bytes(b), np.uint8)


# ------------------------------------------------------------------ O1 block decode


def test_q4k_hand_decoded_block():
    g = _load("q4k_e1.json")
    blk = _kquant_block(g, 144, 16)
    w64, w32 = oracle.dequant_row(oracle.FMT_Q4_K, blk)
    for n, v in g["expected"].items():
        assert w64[int(n)] == v and w32[int(n)] == np.float32(v), n
    # every element whose nibble is zero equals -dmin * m of its sub-block
    nz = {int(n) for n in ("0", "32", "128", "160", "255")}
    for n in range(256):
        if n in nz:
            continue
        j = 2 * (n // 64) + (1 if n % 64 >= 32 else 0)
        assert w64[n] == -0.5 * g["m"][j], n


def test_q5k_hand_decoded_block():
    g = _load("q5k_e3.json")
    blk = _kquant_block(g, 176, 48, qh_at=16)
    w64, w32 = oracle.dequant_row(oracle.FMT_Q5_K, blk)
    for n, v in g["expected"].items():
        assert w64[int(n)] == v and w32[int(n)] == np.float32(v), n


def test_q8_0_hand_decoded_block():
    g = _load("q8_0_e4.json")
    b = bytearray(34)
    b[0:2] = _h(g["block"]["d"])[::-1]
    for i, v in g["block"]["q_nonzero"].items():
        b[2 + int(i)] = int(v, 16)
    w64, w32 = oracle.dequant_row(oracle.FMT_Q8_0, np.frombuffer(bytes(b), np.uint8))
    for n, v in g["expected"].items():
        assert w64[int(n)] == v, n


def _q5_1_block(d16, m16, qh=0, qs=None):
    b = bytearray(24)
    b[0:2] = d16.to_bytes(2, "little")
    b[2:4] = m16.to_bytes(2, "little")
    b[4:8] = qh.to_bytes(4, "little")
    for i, v in (qs or {}).items():
        b[8 + i] = v
    return np.frombuffer(bytes(b), np.uint8)


def test_q5_1_hand_decoded_block():
    g = _load("q5_1_e5.json")
    blk = _q5_1_block(int(g["block"]["d"], 16), int(g["block"]["m"], 16), int(g["block"]["qh"], 16),
                      {int(i): int(v, 16) for i, v in g["block"]["qs_nonzero"].items()})
    w64, w32 = oracle.dequant_row(oracle.FMT_Q5_1, blk)
    for n, v in g["expected"].items():
        assert w64[int(n)] == v and w32[int(n)] == np.float32(v), n
    # every other element has q = 0 and equals the offset m
    for n in range(32):
        if str(n) not in g["expected"] and n not in (0, 1, 15, 16, 17, 31):
            assert w64[n] == -2.0, n


def test_q5_1_nibble_and_fifth_bit_every_element():
    # d = 1, m = 0: one nibble or one qh bit at a time lights exactly one element
    for byte in range(16):
        for hi in (0, 1):
            w, _ = oracle.dequant_row(oracle.FMT_Q5_1,
                                      _q5_1_block(0x3C00, 0, 0, {byte: 0x70 if hi else 0x07}))
            (nz,) = np.nonzero(w)
            assert list(nz) == [byte + 16 * hi] and w[byte + 16 * hi] == 7
    for bit in range(32):
        w, _ = oracle.dequant_row(oracle.FMT_Q5_1, _q5_1_block(0x3C00, 0, 1 << bit))
        (nz,) = np.nonzero(w)
        assert list(nz) == [bit] and w[bit] == 16


def test_q5_1_offset_rounds_once_in_fp32():
    # d = 1024, q = 31 (all bits set), m = 2^-14: the exact value 31744 + 2^-14 needs 29 bits,
    # so the fp32 weight is 31744 (one rounding) while the fp64 value keeps the offset
    w64, w32 = oracle.dequant_row(oracle.FMT_Q5_1,
                                  _q5_1_block(0x6400, 0x0400, 0xFFFFFFFF, {i: 0xFF for i in range(16)}))
    assert (w64 == 31744 + 2.0 ** -14).all() and (w32 == 31744.0).all()
    # negative offset with d = 0: the block is the constant m
    w64, _ = oracle.dequant_row(oracle.FMT_Q5_1, _q5_1_block(0, 0xBC00, 0x12345678, {3: 0x9A}))
    assert (w64 == -1.0).all()


def _q6_k_block(d16, scales, ql=None, qh=None):
    b = bytearray(210)
    for i, v in (ql or {}).items():
        b[i] = v
    for i, v in (qh or {}).items():
        b[128 + i] = v
    b[192:208] = np.array(scales, np.int8).tobytes()
    b[208:210] = d16.to_bytes(2, "little")
    return np.frombuffer(bytes(b), np.uint8)


def test_q6_k_hand_decoded_block():
    g = _load("q6_k_e6.json")
    blk = _q6_k_block(int(g["block"]["d"], 16), g["block"]["scales"],
                      {int(i): int(v, 16) for i, v in g["block"]["ql_nonzero"].items()},
                      {int(i): int(v, 16) for i, v in g["block"]["qh_nonzero"].items()})
    w64, w32 = oracle.dequant_row(oracle.FMT_Q6_K, blk)
    for n, v in g["expected"].items():
        assert w64[int(n)] == v and w32[int(n)] == np.float32(v), n


def test_q6_k_bit_positions_every_element():
    # d = 1, every scale 1: all quants are -32 until one low nibble or one pair of high bits
    # is set, which moves exactly one element
    base = _q6_k_block(0x3C00, [1] * 16)
    w0, _ = oracle.dequant_row(oracle.FMT_Q6_K, base)
    assert (w0 == -32).all()
    for byte in range(128):
        for hi in (0, 1):
            w, _ = oracle.dequant_row(oracle.FMT_Q6_K,
                                      _q6_k_block(0x3C00, [1] * 16, {byte: 0x30 if hi else 0x03}))
            (nz,) = np.nonzero(w != -32)
            h, rest = divmod(byte, 64)
            n = 128 * h + 32 * (2 * hi + rest // 32) + rest % 32
            assert list(nz) == [n] and w[n] == -29
    for byte in range(64):
        for g in range(4):
            w, _ = oracle.dequant_row(oracle.FMT_Q6_K,
                                      _q6_k_block(0x3C00, [1] * 16, qh={byte: 1 << (2 * g + 1)}))
            (nz,) = np.nonzero(w != -32)
            h, l = divmod(byte, 32)
            n = 128 * h + 32 * g + l
            assert list(nz) == [n] and w[n] == 0       # high bits 2 -> q = 32 - 32


def test_q6_k_scales_every_group_and_single_rounding():
    rng = np.random.default_rng(26)
    for _ in range(200):
        sc = rng.integers(-128, 128, size=16)
        raw = bytearray(rng.integers(0, 256, size=210, dtype=np.uint8).tobytes())
        raw[192:208] = np.array(sc, np.int8).tobytes()
        d = np.float16(rng.uniform(1e-3, 1e-2) * (1 if rng.random() < 0.8 else 1000))
        raw[208:210] = np.array([d]).view(np.uint8).tobytes()
        blk = np.frombuffer(bytes(raw), np.uint8)
        w64, w32 = oracle.dequant_row(oracle.FMT_Q6_K, blk)
        assert np.array_equal(w32, w64.astype(np.float32))
        dq = Fraction(float(d))
        for n in range(0, 256, 7):
            h, i = divmod(n, 128)
            g, l = divmod(i, 32)
            lo = raw[64 * h + l + 32 * (g & 1)]
            lo = lo & 15 if g < 2 else lo >> 4
            q = lo + 16 * ((raw[128 + 32 * h + l] >> (2 * g)) & 3) - 32
            assert Fraction(float(w64[n])) == dq * int(sc[8 * h + 2 * g + l // 16]) * q, n


def _pack_scales(sc, m):
    """Inverse of the 6-bit scale/min unpacking: 8 (sc, m) pairs -> 12 bytes."""
    S = [0] * 12
    for j in range(4):
        S[j] = (sc[j] & 63) | ((sc[j + 4] >> 4) << 6)
        S[j + 4] = (m[j] & 63) | ((m[j + 4] >> 4) << 6)
        S[j + 8] = (sc[j + 4] & 15) | ((m[j + 4] & 15) << 4)
    return bytes(S)


def test_kquant_scale_pack_unpack_round_trip_all_64x64():
    # block i puts (sc, m) = ((i//64 + 9j) % 64, (i%64 + 17j) % 64) at sub-block j: a bijection
    # of the 4096 pairs at every position.  With every nibble 1, d = 1, dmin = 0 the weights of
    # sub-block j equal sc_j; with nibbles 0, d = 0, dmin = 1 they equal -m_j.
    rows_sc, rows_m, want_sc, want_m = [], [], [], []
    for i in range(4096):
        sc = [(i // 64 + 9 * j) % 64 for j in range(8)]
        m = [(i % 64 + 17 * j) % 64 for j in range(8)]
        S = _pack_scales(sc, m)
        rows_sc.append(b"\x00\x3c\x00\x00" + S + b"\x11" * 128)
        rows_m.append(b"\x00\x00\x00\x3c" + S + b"\x00" * 128)
        want_sc.append(np.repeat(np.array(sc, np.float64)[[0, 1, 2, 3, 4, 5, 6, 7]], 32))
        want_m.append(np.repeat(-np.array(m, np.float64), 32))
    # element order: sub-blocks run 0,1 (n 0..63), 2,3 (64..127), ...: 32 elements each
    w_sc, _ = oracle.dequant_row(oracle.FMT_Q4_K, np.frombuffer(b"".join(rows_sc), np.uint8))
    w_m, _ = oracle.dequant_row(oracle.FMT_Q4_K, np.frombuffer(b"".join(rows_m), np.uint8))
    assert np.array_equal(w_sc, np.concatenate(want_sc))
    assert np.array_equal(w_m, np.concatenate(want_m))


def test_q5k_high_bit_plane_every_position():
    # one qh bit set at a time: element n gains exactly 16 * d * sc of its sub-block
    base = bytearray(176)
    base[0:2] = b"\x00\x3c"                  # d = 1
    base[4:16] = _pack_scales([1, 2, 3, 4, 5, 6, 7, 8], [0] * 8)
    w0, _ = oracle.dequant_row(oracle.FMT_Q5_K, np.frombuffer(bytes(base), np.uint8))
    assert not w0.any()
    for byte in range(32):
        for bit in range(8):
            b = bytearray(base)
            b[16 + byte] = 1 << bit
            w, _ = oracle.dequant_row(oracle.FMT_Q5_K, np.frombuffer(bytes(b), np.uint8))
            (nz,) = np.nonzero(w)
            # bit 2c of qh[r] -> element 64c + r ; bit 2c+1 -> element 64c + 32 + r
            n = 64 * (bit // 2) + 32 * (bit % 2) + byte
            assert list(nz) == [n]
            assert w[n] == 16 * (bit + 1)


def test_q4k_nibble_position_every_element():
    base = bytearray(144)
    base[0:2] = b"\x00\x3c"
    base[4:16] = _pack_scales([1, 2, 3, 4, 5, 6, 7, 8], [0] * 8)
    for byte in range(128):
        for hi in (0, 1):
            b = bytearray(base)
            b[16 + byte] = 0x10 if hi else 0x01
            w, _ = oracle.dequant_row(oracle.FMT_Q4_K, np.frombuffer(bytes(b), np.uint8))
            (nz,) = np.nonzero(w)
            c, r = byte // 32, byte % 32
            n = 64 * c + 32 * hi + r
            assert list(nz) == [n]
            assert w[n] == 2 * c + hi + 1


def _f16(bits):
    return Fraction(float(np.array([bits], np.uint16).view(np.float16)[0]))


def test_dequant_exact_rational_and_single_rounding():
    rng = np.random.default_rng(11)
    for fmt, bb in ((oracle.FMT_Q4_K, 144), (oracle.FMT_Q5_K, 176), (oracle.FMT_Q8_0, 34),
                    (oracle.FMT_Q5_1, 24)):
        raw = rng.integers(0, 256, size=bb * 64, dtype=np.uint8)
        # scales in the generator's range and a few extremes
        for i in range(64):
            d = np.float16(rng.uniform(1e-3, 1e-2)) if i % 8 else np.float16(rng.uniform(1, 100))
            raw[i * bb:i * bb + 2] = np.array([d]).view(np.uint8)
            if fmt == oracle.FMT_Q5_1:
                mm = np.float16(-rng.uniform(1e-3, 0.5))
                raw[i * bb + 2:i * bb + 4] = np.array([mm]).view(np.uint8)
            elif fmt != oracle.FMT_Q8_0:
                dm = np.float16(rng.uniform(1e-3, 1e-2))
                raw[i * bb + 2:i * bb + 4] = np.array([dm]).view(np.uint8)
        w64, w32 = oracle.dequant_row(fmt, raw)
        # fp32 weights are the exact values rounded once
        assert np.array_equal(w32, w64.astype(np.float32))
        # exact values are d*sc*q - dmin*m with integer sc, m, q in range: check as rationals
        for i in range(64):
            blk = raw[i * bb:(i + 1) * bb]
            d = _f16(int(blk[0]) | int(blk[1]) << 8)
            vals = [Fraction(float(v)) for v in w64[i * (32 if fmt >= 2 else 256):][:8]]
            if fmt == oracle.FMT_Q5_1:
                mm = _f16(int(blk[2]) | int(blk[3]) << 8)
                qh = int.from_bytes(bytes(blk[4:8]), "little")
                for n, v in enumerate(vals):
                    assert v == d * ((int(blk[8 + n]) & 15) | ((qh >> n) & 1) << 4) + mm
            elif fmt == oracle.FMT_Q8_0:
                for n, v in enumerate(vals):
                    assert v == d * int(np.int8(blk[2 + n]))
            else:
                dmin = _f16(int(blk[2]) | int(blk[3]) << 8)
                # sub-block 0, elements 0..7: (v + dmin*m)/(d*sc) must be an integer q in range
                m0 = int(blk[8]) & 63
                sc0 = int(blk[4]) & 63
                for v in vals:
                    if sc0 == 0:
                        assert v == -dmin * m0
                    else:
                        q = (v + dmin * m0) / (d * sc0)
                        assert q.denominator == 1 and 0 <= q <= (15 if fmt == 0 else 31)


def test_dequant_special_cases():
    # sc = m = 0 -> 0 ; dmin = 0 -> symmetric (no offset) ; Q8_0 with d = 1 -> w = q
    z = np.zeros(144, np.uint8)
    z[0:2] = [0x00, 0x3C]
    z[2:4] = [0x00, 0x3C]
    z[16:] = 0xFF
    assert not oracle.dequant_row(0, z)[0].any()
    b = np.zeros(34, np.uint8)
    b[0:2] = [0x00, 0x3C]
    b[2:] = np.arange(-16, 16).astype(np.int8).view(np.uint8)
    assert np.array_equal(oracle.dequant_row(2, b)[0], np.arange(-16, 16))


def test_half_conversions_match_numpy():
    rng = np.random.default_rng(5)
    vals = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-9, 6, 20000),
                           np.float32([0.0, -0.0, 65504.0, 65519.0, 65520.0, 1e9, 2.0 ** -24,
                                       2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, 1.0 + 2.0 ** -11,
                                       1.0 + 3 * 2.0 ** -11])])
    ours = np.array([oracle.float_to_half(float(v)) for v in vals], np.uint16)
    assert np.array_equal(ours, vals.astype(np.float16).view(np.uint16))
    bits = np.arange(0, 65536, dtype=np.uint16)
    finite = np.isfinite(bits.view(np.float16))
    mine = np.array([oracle.half_to_double(int(b)) for b in bits[finite]])
    assert np.array_equal(mine, bits[finite].view(np.float16).astype(np.float64))


# ------------------------------------------------------------------ O2 Q8_1


def test_q8_1_hand_block():
    g = _load("q8_1_e2.json")
    x = np.zeros(32, np.float32)
    for i, v in g["x_nonzero"].items():
        x[int(i)] = v
    q, d, s, bad = oracle.quantize_q8_1(x)
    want = np.zeros(32, np.int8)
    for i, v in g["q_nonzero"].items():
        want[int(i)] = v
    assert bad == 0 and np.array_equal(q, want)
    assert d[0] == int(g["d16"], 16) and s[0] == int(g["s16"], 16)


def test_q8_1_zero_nonfinite_and_invariants():
    q, d, s, bad = oracle.quantize_q8_1(np.zeros(64, np.float32))
    assert bad == 0 and not q.any() and not d.any() and not s.any()
    x = np.ones(64, np.float32)
    x[40] = np.nan
    q, d, s, bad = oracle.quantize_q8_1(x)
    assert bad == 1 and not q[32:].any() and d[1] == 0 and s[1] == 0 and q[:32].all()
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(32 * 500) * np.repeat(10.0 ** rng.uniform(-3, 3, 500), 32)
         ).astype(np.float32)
    q, d16, s16, _ = oracle.quantize_q8_1(x)
    xb = x.reshape(-1, 32).astype(np.float64)
    qb = q.reshape(-1, 32).astype(np.int64)
    dd32 = np.abs(x.reshape(-1, 32)).max(1) / np.float32(127)   # fp32 division, as defined
    dd = dd32.astype(np.float64)
    assert (np.abs(qb).max(1) == 127).all()
    err = np.abs(xb - qb * dd[:, None])
    assert (err <= dd[:, None] * (0.5 + 1e-5)).all()
    assert np.array_equal(d16, dd32.astype(np.float16).view(np.uint16))
    # s is d times the integer sum of q
    sums = qb.sum(1)
    assert np.array_equal(s16, (dd32 * sums.astype(np.float32)
                                ).astype(np.float16).view(np.uint16))


def test_q8_1_round_half_away_from_zero():
    # d = 1 exactly (amax 127): x = k + 0.5 rounds away from zero
    x = np.zeros(32, np.float32)
    x[0] = 127
    x[1:9] = [0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 126.5, -126.5]
    q, _, _, _ = oracle.quantize_q8_1(x)
    assert list(q[1:9]) == [1, -1, 2, -2, 3, -3, 127, -127]


# ------------------------------------------------------------------ O3 top-k


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(7)
    for trial in range(200):
        T, E = 3, int(rng.integers(2, 40))
        k = int(rng.integers(1, E + 1))
        L = rng.integers(-4, 4, size=(T, E)).astype(np.float32)   # many ties
        ids, w, bad = oracle.topk(L, k)
        assert bad == 0
        for t in range(T):
            want = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
            assert list(ids[t]) == want
            ref = scipy.special.softmax(L[t, want].astype(np.float64))
            assert np.abs(w[t] - ref).max() <= 1e-7
            assert abs(float(w[t].astype(np.float64).sum()) - 1.0) <= 1e-6


def test_topk_expert_relabelling_invariance():
    rng = np.random.default_rng(8)
    L = rng.standard_normal((16, 64)).astype(np.float32)
    p = rng.permutation(64)
    ids, w, _ = oracle.topk(L, 6)
    ids2, w2, _ = oracle.topk(L[:, p], 6)
    assert np.array_equal(p[ids2], ids) and np.array_equal(w, w2)


def test_topk_nonfinite_row_flagged():
    L = np.zeros((2, 8), np.float32)
    L[1, 3] = np.inf
    ids, w, bad = oracle.topk(L, 2)
    assert bad == 1 and list(ids[0]) == [0, 1]


# ------------------------------------------------------------------ O4 grouping


def test_grouping_against_stable_argsort():
    rng = np.random.default_rng(9)
    for _ in range(50):
        T, E = int(rng.integers(1, 60)), int(rng.integers(1, 20))
        k = int(rng.integers(1, E + 1))
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = oracle.group(ids, E)
        assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))
        assert offsets[0] == 0 and offsets[-1] == T * k and (np.diff(offsets) >= 0).all()
        assert np.array_equal(perm, np.argsort(ids.ravel(), kind="stable"))
        assert np.array_equal(np.sort(perm), np.arange(T * k))
        assert np.array_equal(inv[perm], np.arange(T * k))


# ------------------------------------------------------------------ O5-O9 the FFN


def _tiny(fmt_mix, H, F, E, k, T, shared, idx):
    mix = () if fmt_mix is None else fmt_mix
    return synth.Workload(f"pin{idx}", 100 + idx, H, F, E, k, T, shared, 1, "normal", sigma=1.5,
                          mix=mix)


def _dense(arena, lay, e, H, F):
    fmt = int(lay.fmts[e])
    bw = synth.BLOCK_WEIGHTS[fmt]
    Fp = -(-F // bw) * bw
    mats = []
    for t, (rows, width) in enumerate(((F, H), (F, H), (H, F))):
        nb = -(-width // bw)
        W, _ = oracle.dequant_matrix(fmt, arena[lay.offs[e, t]:], rows, int(lay.strides[e, t]), nb)
        mats.append(W)
    assert mats[2].shape == (H, Fp)
    return mats


def _q8_1_values(v):
    q, d16, _, _ = oracle.quantize_q8_1(v.astype(np.float32))
    return np.repeat(d16.view(np.float16).astype(np.float64), 32) * q


@pytest.mark.parametrize("case", [
    (0, None, 256, 256, 8, 2, 3, False),
    (1, None, 512, 384, 6, 3, 4, True),                       # down rows padded 384 -> 512
    (2, ((synth.Q8_0, 1.0),), 256, 160, 5, 2, 3, True),      # Q8_0, width 160
    (3, ((synth.Q4_K, 0.3), (synth.Q5_K, 0.7), (synth.Q8_0, 1.0)), 512, 640, 12, 4, 5, True),
    (4, ((synth.Q5_1, 1.0),), 256, 160, 5, 2, 3, True),      # Q5_1, width 160
    (5, ((synth.Q4_K, 0.25), (synth.Q5_K, 0.5), (synth.Q8_0, 0.75), (synth.Q5_1, 1.0)),
     512, 640, 12, 4, 5, True),
    (6, ((synth.Q6_K, 1.0),), 256, 160, 5, 2, 3, True),      # Q6_K, down rows padded
    (7, ((synth.Q4_K, 0.5), (synth.Q6_K, 1.0)), 512, 640, 8, 3, 4, True),
])
def test_forward_matches_dense_fp64(case):
    idx, mix, H, F, E, k, T, shared = case
    w = _tiny(mix, H, F, E, k, T, shared, idx)
    arena, lay = synth.host_arena(w, 0)
    x = synth.activations(w, 0)
    L = synth.router_logits(w, 0)
    ids, wt, _ = oracle.topk(L, k)
    ex = oracle.experts_table(lay.fmts, lay.offs, lay.strides)
    out, out64 = oracle.forward(arena, ex, lay.shared, H, F, x, ids, wt)
    for t in range(T):
        xh = _q8_1_values(x[t])
        acc = np.zeros(H)
        experts = [(int(e), float(wj)) for e, wj in zip(ids[t], wt[t])]
        if shared:
            experts.append((E, 1.0))
        for e, wj in experts:
            Wg, Wu, Wd = _dense(arena, lay, e, H, F)
            g = Wg @ xh
            u = Wu @ xh
            h = g * scipy.special.expit(g) * u
            hp = np.zeros(Wd.shape[1], np.float32)
            hp[:F] = h
            y = Wd @ _q8_1_values(hp)
            acc += wj * y
            if t == 0:
                r = oracle.expert_ffn(arena, ex[e], H, F, xh)
                assert np.allclose(r["g"], g, rtol=1e-12, atol=1e-12)
                assert np.allclose(r["u"], u, rtol=1e-12, atol=1e-12)
                assert np.allclose(r["y"], y, rtol=1e-12, atol=1e-9)
        assert np.allclose(out64[t], acc, rtol=1e-12, atol=1e-9)
        assert np.array_equal(out[t], out64[t].astype(np.float32))


def test_forward_identical_experts_ignore_routing():
    w = _tiny(None, 256, 256, 6, 3, 4, False, 41)
    arena, lay = synth.host_arena(w, 0)
    for e in range(1, lay.n):
        for t in range(3):
            n = int(lay.tensor_bytes[e, t])
            arena[lay.offs[e, t]:lay.offs[e, t] + n] = arena[lay.offs[0, t]:lay.offs[0, t] + n]
    x = synth.activations(w, 0)
    L = synth.router_logits(w, 0)
    ids, wt, _ = oracle.topk(L, 3)
    ex = oracle.experts_table(lay.fmts, lay.offs, lay.strides)
    _, out64 = oracle.forward(arena, ex, -1, 256, 256, x, ids, wt)
    for t in range(4):
        y = oracle.expert_ffn(arena, ex[0], 256, 256, _q8_1_values(x[t]))["y"]
        assert np.allclose(out64[t], y, rtol=1e-6, atol=1e-6 * np.abs(y).max())


def test_forward_k1_is_the_expert_and_zero_weights_give_zero():
    w = _tiny(None, 256, 256, 4, 1, 2, False, 42)
    arena, lay = synth.host_arena(w, 0)
    x = synth.activations(w, 0)
    ids, wt, _ = oracle.topk(synth.router_logits(w, 0), 1)
    assert (wt == 1.0).all()
    ex = oracle.experts_table(lay.fmts, lay.offs, lay.strides)
    _, out64 = oracle.forward(arena, ex, -1, 256, 256, x, ids, wt)
    for t in range(2):
        y = oracle.expert_ffn(arena, ex[ids[t, 0]], 256, 256, _q8_1_values(x[t]))["y"]
        assert np.array_equal(out64[t], y)
    z = arena.copy()
    for e in range(lay.n):
        for t in range(3):
            for r in range(lay.tensor_bytes[e, t] // lay.strides[e, t]):
                base = lay.offs[e, t] + r * lay.strides[e, t]
                for b in range(lay.strides[e, t] // 144):
                    z[base + 144 * b: base + 144 * b + 4] = 0      # d = dmin = 0
    _, o = oracle.forward(z, ex, -1, 256, 256, x, ids, wt)
    assert not o.any()


def test_q8_1_uses_ieee_fp32_division():
    # Blocks where d = amax/127 (one IEEE fp32 division, numpy's float32 '/') and the
    # reciprocal form amax * (1/127) give different q: the oracle must follow the division.
    rng = np.random.default_rng(21)
    cases = 0
    for _ in range(4000):
        amax = np.float32(rng.uniform(0.25, 8.0))
        d = amax / np.float32(127)
        d_alt = amax * (np.float32(1) / np.float32(127))
        x = np.zeros(32, np.float32)
        x[0] = amax
        # values whose quotient lands near a half-integer
        x[1:] = ((rng.integers(1, 126, 31) + 0.5) * np.float64(d)).astype(np.float32)
        r = x / d
        r_alt = x / d_alt
        q_ieee = np.sign(r) * np.floor(np.abs(r.astype(np.float64)) + 0.5)
        q_alt = np.sign(r_alt) * np.floor(np.abs(r_alt.astype(np.float64)) + 0.5)
        if np.array_equal(q_ieee, q_alt):
            continue
        q, _, _, _ = oracle.quantize_q8_1(x)
        assert np.array_equal(q, q_ieee.astype(np.int8))
        cases += 1
    assert cases >= 20


def test_generator_q5_1_blocks():
    # Q5_1 tensors: d from the scale draw, m = -16 * the dmin draw (both fp16), so every weight
    # lies in [m, m + 31 d] and the block's offset is negative
    w = _tiny(((synth.Q5_1, 1.0),), 256, 96, 3, 1, 2, False, 6)
    arena, lay = synth.host_arena(w, 0)
    assert (lay.fmts == synth.Q5_1).all() and lay.strides[0, 0] == 8 * 24 and lay.strides[0, 2] == 80
    for e in range(lay.n):
        for t in range(3):
            rows, width = synth.tensor_shape(w, t)
            nb = synth.row_blocks(synth.Q5_1, width)
            st = int(lay.strides[e, t])
            mat = arena[lay.offs[e, t]:lay.offs[e, t] + rows * st].reshape(rows, st)
            assert not mat[:, nb * 24:].any()
            blk = mat[:, :nb * 24].reshape(rows, nb, 24)
            d = blk[:, :, 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
            m = blk[:, :, 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
            assert (d >= 1e-3 * 0.999).all() and (d <= 1e-2 * 1.001).all()
            assert (m <= -16e-3 * 0.999).all() and (m >= -0.16 * 1.001).all()
            W, _ = oracle.dequant_matrix(synth.Q5_1, mat.ravel(), rows, st, nb)
            lo = np.repeat(m, 32, axis=1)
            assert (W >= lo).all() and (W <= lo + 31 * np.repeat(d, 32, axis=1)).all()


# ------------------------------------------------------------------ O10-O11 router and gate


def test_router_one_hot_rows_pick_the_inputs():
    rng = np.random.default_rng(21)
    T, H, E = 5, 64, 16
    x = rng.standard_normal((T, H)).astype(np.float32)
    pick = rng.permutation(H)[:E]
    Wr = np.zeros((E, H), np.float32)
    Wr[np.arange(E), pick] = 1.0
    l32, l64 = oracle.router(x, Wr)
    assert np.array_equal(l32, x[:, pick])            # one nonzero product per sum: exact
    l32q, _ = oracle.router(x, Wr * np.float32(0.25))
    assert np.array_equal(l32q, x[:, pick] * np.float32(0.25))


def test_router_matches_dense_fp64_matmul():
    rng = np.random.default_rng(22)
    T, H, E = 7, 2048, 64
    x = rng.standard_normal((T, H)).astype(np.float32)
    Wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    l32, l64 = oracle.router(x, Wr)
    ref = x.astype(np.float64) @ Wr.astype(np.float64).T
    # two fp64 summations of the same 2048 exact products differ by at most ~H ulp of sum|p|
    bound = 4e-13 * (np.abs(x).astype(np.float64) @ np.abs(Wr).astype(np.float64).T)
    assert (np.abs(l64 - ref) <= bound).all()
    assert np.array_equal(l32, l64.astype(np.float32))


def test_router_then_topk_follows_one_channel():
    # x one-hot at channel c: every logit is Wr[e][c] exactly, so the top-k are that column's
    # largest entries
    rng = np.random.default_rng(23)
    H, E, k = 32, 40, 6
    Wr = rng.permutation(E * H).reshape(E, H).astype(np.float32) / np.float32(64.0)
    for c in (0, 7, 31):
        x = np.zeros((1, H), np.float32)
        x[0, c] = 1.0
        l32, _ = oracle.router(x, Wr)
        ids, _, _ = oracle.topk(l32, k)
        assert list(ids[0]) == list(np.argsort(-Wr[:, c], kind="stable")[:k])


def test_shared_gate_closed_forms():
    rng = np.random.default_rng(24)
    T, H = 6, 256
    x = rng.standard_normal((T, H)).astype(np.float32)
    assert (oracle.shared_gate(x, np.zeros(H, np.float32)) == 0.5).all()
    wg = (rng.standard_normal(H) * 0.05).astype(np.float32)
    g = oracle.shared_gate(x, wg)
    ref = scipy.special.expit(x.astype(np.float64) @ wg.astype(np.float64))
    assert np.allclose(g, ref, rtol=1e-14, atol=0)
    big = oracle.shared_gate(x[:1], (x[0] * np.float32(1e4)).astype(np.float32))
    assert big[0] == 1.0                                # exp(-large) underflows: gate fully open


def test_gated_forward_is_routed_plus_gated_shared():
    w = _tiny(((synth.Q4_K, 0.5), (synth.Q5_1, 1.0)), 256, 160, 6, 2, 4, True, 7)
    arena, lay = synth.host_arena(w, 0)
    x = synth.activations(w, 0)
    ids, wt, _ = oracle.topk(synth.router_logits(w, 0), w.k)
    ex = oracle.experts_table(lay.fmts, lay.offs, lay.strides)
    rng = np.random.default_rng(25)
    g = oracle.shared_gate(x, (rng.standard_normal(w.hidden) * 0.1).astype(np.float32))
    assert (g > 0.05).all() and (g < 0.95).all()
    _, routed = oracle.forward(arena, ex, -1, w.hidden, w.ffn, x, ids, wt)
    _, gated = oracle.forward(arena, ex, lay.shared, w.hidden, w.ffn, x, ids, wt, gate=g)
    for t in range(w.tokens):
        y_s = oracle.expert_ffn(arena, ex[lay.shared], w.hidden, w.ffn, _q8_1_values(x[t]))["y"]
        assert np.allclose(gated[t], routed[t] + g[t] * y_s, rtol=1e-12, atol=1e-12)
    _, ungated = oracle.forward(arena, ex, lay.shared, w.hidden, w.ffn, x, ids, wt)
    _, ones = oracle.forward(arena, ex, lay.shared, w.hidden, w.ffn, x, ids, wt,
                             gate=np.ones(w.tokens))
    assert np.array_equal(ones, ungated)


# ------------------------------------------------------------------ O12 layer chain


def _chain_layer(w, layer, seed, zero=False, gate=False):
    arena, lay = synth.host_arena(w, layer)
    if zero:                       # every block's d and dmin 0: every expert outputs 0
        arena = arena.copy()
        for e in range(lay.n):
            for t in range(3):
                rows, width = synth.tensor_shape(w, t)
                fmt = int(lay.fmts[e])
                nb, bb = synth.row_blocks(fmt, width), synth.BLOCK_BYTES[fmt]
                st = int(lay.strides[e, t])
                m = arena[lay.offs[e, t]:lay.offs[e, t] + rows * st].reshape(rows, st)
                for b in range(nb):
                    m[:, b * bb:b * bb + (2 if fmt == synth.Q8_0 else 4)] = 0
    rng = np.random.default_rng(seed)
    return {"arena": arena, "experts": oracle.experts_table(lay.fmts, lay.offs, lay.strides),
            "shared": lay.shared, "hidden": w.hidden, "ffn": w.ffn,
            "router": (rng.standard_normal((w.n_experts, w.hidden)) * 0.05).astype(np.float32),
            "gate": (rng.standard_normal(w.hidden) * 0.05).astype(np.float32) if gate else None}


def test_chain_of_one_layer_is_the_layer_plus_residual():
    w = _tiny(None, 256, 256, 8, 2, 3, True, 8)
    L = _chain_layer(w, 0, 31, gate=True)
    x0 = synth.activations(w, 0)
    xL, ids = oracle.chain([L], x0, w.k)
    xn = oracle.rmsnorm(x0)
    logits, _ = oracle.router(xn, L["router"])
    rid, rw, _ = oracle.topk(logits, w.k)
    out, _ = oracle.forward(L["arena"], L["experts"], L["shared"], w.hidden, w.ffn, xn, rid, rw,
                            gate=oracle.shared_gate(xn, L["gate"]))
    assert np.array_equal(ids[0], rid)
    assert np.array_equal(xL, (x0 + out).astype(np.float32))


def test_rmsnorm_closed_forms():
    eps = oracle.RMS_EPS
    # a 3-4 row: mean square 12.5 (not the sum 25), so every value is divided by sqrt(12.5 + eps)
    got = oracle.rmsnorm(np.array([[3.0, 4.0], [0.0, 0.0]], np.float32))
    assert got[0, 0] == np.float32(3.0 / np.sqrt(12.5 + eps))
    assert got[0, 1] == np.float32(4.0 / np.sqrt(12.5 + eps))
    assert (got[1] == 0.0).all()                       # a zero row stays zero (eps > 0)
    # a constant row a: a / sqrt(a^2 + eps), the sign kept
    for a in (-7.0, 0.01, 2.0 ** 40):
        row = np.full((1, 64), a, np.float32)
        assert (oracle.rmsnorm(row) == np.float32(a / np.sqrt(a * a + eps))).all()
    # one spike among zeros of a row of n: the spike becomes sqrt(n) (eps negligible), the rest 0
    row = np.zeros((1, 256), np.float32)
    row[0, 17] = 1e3
    got = oracle.rmsnorm(row)
    assert abs(got[0, 17] - 16.0) < 1e-6 and np.count_nonzero(got) == 1
    # the norm weight scales each column after the division: [3, 4] with weight [2, 0.5]
    got = oracle.rmsnorm(np.array([[3.0, 4.0]], np.float32), np.array([2.0, 0.5], np.float32))
    assert got[0, 0] == np.float32(6.0 / np.sqrt(12.5 + eps))
    assert got[0, 1] == np.float32(2.0 / np.sqrt(12.5 + eps))
    # rows are independent, and the output's mean square is ms / (ms + eps)
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((3, 512)) * [[1e-2], [1.0], [1e3]]).astype(np.float32)
    got = oracle.rmsnorm(x).astype(np.float64)
    for i in range(3):
        assert np.array_equal(oracle.rmsnorm(x[i:i + 1])[0], got[i].astype(np.float32))
        ms = (x[i].astype(np.float64) ** 2).mean()
        assert abs((got[i] ** 2).mean() - ms / (ms + eps)) < 1e-6


def test_chain_of_silent_layers_keeps_the_residual():
    w = _tiny(None, 256, 256, 8, 2, 3, True, 9)
    layers = [_chain_layer(w, l, 40 + l, zero=True) for l in range(3)]
    x0 = synth.activations(w, 0)
    xL, ids = oracle.chain(layers, x0, w.k)
    assert np.array_equal(xL, x0) and len(ids) == 3


def test_chain_lookahead_with_identical_routers_predicts_from_the_previous_input():
    # layers that share one router: the early pick for layer l is the routing of x_{l-1}, which
    # is exactly what layer l-1 chose
    w = _tiny(None, 256, 256, 8, 2, 3, False, 10)
    base = _chain_layer(w, 0, 50)
    layers = [dict(base, arena=_chain_layer(w, l, 50)["arena"]) for l in range(3)]
    x0 = synth.activations(w, 0)
    _, ids, early = oracle.chain(layers, x0, w.k, lookahead=True)
    assert len(early) == 2
    for l in range(2):
        assert np.array_equal(early[l], ids[l])


def test_forward_q6_k_experts_match_dense_fp64():
    # a tiny layer of Q6_K experts built here (the generator does not draw Q6_K): random quants,
    # int8 scales in [-16, 16], d ~ U(1e-3, 1e-2); down rows of width 160 stored as one block
    rng = np.random.default_rng(27)
    H, F, E, k, T = 256, 160, 4, 2, 3
    n = E + 1
    shapes = ((F, H), (F, H), (H, F))
    offs = np.zeros((n, 3), np.int64)
    strides = np.zeros((n, 3), np.int64)
    chunks, pos = [], 0
    for e in range(n):
        for t, (rows, width) in enumerate(shapes):
            nb = -(-width // 256)
            st = -(-nb * 210 // 16) * 16
            m = rng.integers(0, 256, size=(rows, st), dtype=np.uint8)
            for b in range(nb):
                m[:, b * 210 + 192:b * 210 + 208] = rng.integers(-16, 17, size=(rows, 16)).astype(np.int8).view(np.uint8)
                d = rng.uniform(1e-3, 1e-2, size=rows).astype(np.float16)
                m[:, b * 210 + 208:b * 210 + 210] = d.view(np.uint8).reshape(rows, 2)
            m[:, nb * 210:] = 0
            pad = -pos % 256
            chunks.append(np.zeros(pad, np.uint8))
            pos += pad
            offs[e, t], strides[e, t] = pos, st
            chunks.append(m.ravel())
            pos += m.size
    arena = np.concatenate(chunks)
    ex = oracle.experts_table(np.full(n, oracle.FMT_Q6_K, np.int32), offs, strides)
    x = rng.standard_normal((T, H)).astype(np.float32)
    logits = (np.arange(E)[None, :] * 0.25 + rng.permutation(E * T).reshape(T, E)).astype(np.float32)
    ids, wt, _ = oracle.topk(logits, k)
    out, out64 = oracle.forward(arena, ex, E, H, F, x, ids, wt)
    dense = []
    for e in range(n):
        mats = []
        for t, (rows, width) in enumerate(shapes):
            nb = -(-width // 256)
            W, _ = oracle.dequant_matrix(oracle.FMT_Q6_K, arena[offs[e, t]:], rows, int(strides[e, t]), nb)
            mats.append(W)
        dense.append(mats)
    for t in range(T):
        xh = _q8_1_values(x[t])
        acc = np.zeros(H)
        for e, wj in [(int(a), float(b)) for a, b in zip(ids[t], wt[t])] + [(E, 1.0)]:
            Wg, Wu, Wd = dense[e]
            g = Wg @ xh
            u = Wu @ xh
            hp = np.zeros(Wd.shape[1], np.float32)
            hp[:F] = g * scipy.special.expit(g) * u
            acc += wj * (Wd @ _q8_1_values(hp))
        assert np.allclose(out64[t], acc, rtol=1e-12, atol=1e-9)
        assert np.array_equal(out[t], out64[t].astype(np.float32))


def test_generator_q6_k_blocks_and_padding():
    # Q6_K tensors: d from the scale draw at the end of each block; the down rows' weights past
    # the logical width 160 (groups 10-15 of the one block) are exactly 0
    w = _tiny(((synth.Q6_K, 1.0),), 256, 160, 3, 1, 2, False, 11)
    arena, lay = synth.host_arena(w, 0)
    assert (lay.fmts == synth.Q6_K).all() and lay.strides[0, 0] == 224
    for e in range(lay.n):
        for t in range(3):
            rows, width = synth.tensor_shape(w, t)
            st = int(lay.strides[e, t])
            mat = arena[lay.offs[e, t]:lay.offs[e, t] + rows * st].reshape(rows, st)
            assert not mat[:, 210:].any()
            d = mat[:, 208:210].copy().view(np.float16)[:, 0].astype(np.float64)
            assert (d >= 1e-3 * 0.999).all() and (d <= 1e-2 * 1.001).all()
            W, _ = oracle.dequant_matrix(synth.Q6_K, mat.ravel(), rows, st, 1)
            assert not W[:, width:].any() and W[:, :width].any()
    with pytest.raises(NotImplementedError):
        synth.device_fill_layer(w, 0, 0)


@pytest.mark.parametrize("case", [
    (61, None, 256, 256, 6, 2, 3, True),
    (62, ((synth.Q4_K, 0.25), (synth.Q5_K, 0.5), (synth.Q8_0, 0.75), (synth.Q5_1, 1.0)),
     512, 320, 8, 3, 4, True),
])
def test_down_combine_matches_dense_fp64(case):
    # O8-O9 from Q8_1(h) rows given from outside, against a dense fp64 matmul of the exact down
    # weights: random Q8_1 rows (int8 codes, positive fp16 scales), slots in a shuffled order
    idx, mix, H, F, E, k, T, shared = case
    w = _tiny(mix, H, F, E, k, T, shared, idx)
    arena, lay = synth.host_arena(w, 0)
    ex = oracle.experts_table(lay.fmts, lay.offs, lay.strides)
    rng = np.random.default_rng(idx)
    hpad = -(-F // 256) * 256
    n = 11
    slot_tok = rng.integers(0, T, n)
    slot_exp = rng.integers(0, lay.n, n)
    slot_w = rng.uniform(0.1, 1.0, n)
    hq = rng.integers(-127, 128, (n, hpad)).astype(np.int8)
    hd = np.float16(rng.uniform(1e-3, 10.0, (n, hpad // 32))).view(np.uint16)
    got = oracle.down_combine(arena, ex, H, F, hq, hd, slot_tok, slot_exp, slot_w, T)
    want = np.zeros((T, H))
    for s in range(n):
        _, _, Wd = _dense(arena, lay, int(slot_exp[s]), H, F)
        fp = Wd.shape[1]
        hh = hq[s, :fp].astype(np.float64) * np.repeat(hd[s].view(np.float16).astype(np.float64),
                                                       32)[:fp]
        want[slot_tok[s]] += slot_w[s] * (Wd @ hh)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-9 * np.abs(want).max())


def test_down_combine_of_the_oracles_own_h_is_the_forward():
    # with the Q8_1(h) of each (token, expert) as O5-O7 produce it, O8-O9 from outside give the
    # layer's output exactly as the whole forward does (the same sums in the same order)
    w = _tiny(None, 256, 256, 6, 2, 3, True, 63)
    arena, lay = synth.host_arena(w, 0)
    ex = oracle.experts_table(lay.fmts, lay.offs, lay.strides)
    x = synth.activations(w, 0)
    ids, wt, _ = oracle.topk(synth.router_logits(w, 0), 2)
    _, out64 = oracle.forward(arena, ex, lay.shared, 256, 256, x, ids, wt)
    rows_q, rows_d, st, se, sw = [], [], [], [], []
    for t in range(3):
        for e, wj in [(int(e), float(v)) for e, v in zip(ids[t], wt[t])] + [(6, 1.0)]:
            r = oracle.expert_ffn(arena, ex[e], 256, 256, _q8_1_values(x[t]))
            rows_q.append(r["hq"])
            rows_d.append(r["hd"])
            st.append(t)
            se.append(e)
            sw.append(wj)
    got = oracle.down_combine(arena, ex, 256, 256, np.stack(rows_q), np.stack(rows_d), st, se, sw, 3)
    assert np.array_equal(got, out64)
