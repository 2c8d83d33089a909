"""CPU oracle of the quantized MoE layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The CUDA library under ``expert_ffn_token_b200/`` never imports it, and this
package imports nothing from there: the two share no code, headers or constants.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64); this module only builds it with gcc
and marshals numpy arrays through ctypes.  Each wrapper names the oracle step it exposes
(O1-O9, written out at the top of ``moe_oracle.c``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "moe_oracle.c"
_LIB = _HERE / "liboracle.so"

FMT_Q4_K, FMT_Q5_K, FMT_Q8_0, FMT_Q5_1, FMT_Q6_K = 0, 1, 2, 3, 4

_lib = None


def build(force: bool = False) -> Path:
    """Compile moe_oracle.c with gcc (-O2, IEEE arithmetic: no fast-math, no FMA contraction)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.{os.getpid()}")
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-o", str(tmp), str(_SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(str(_LIB))
        P = ctypes.c_void_p
        L.oracle_dequant_row.argtypes = [ctypes.c_int, P, ctypes.c_int64, P, P]
        L.oracle_quantize_q8_1.argtypes = [P, ctypes.c_int64, P, P, P]
        L.oracle_quantize_q8_1.restype = ctypes.c_int64
        L.oracle_topk.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_group.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P]
        L.oracle_expert_ffn.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P]
        L.oracle_forward.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, P, P, P, ctypes.c_int, ctypes.c_int, P,
                                     ctypes.c_int, P, P]
        L.oracle_forward_gated.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, P, P, P, ctypes.c_int, ctypes.c_int, P,
                                           ctypes.c_int, P, P, P]
        L.oracle_router.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_down_combine.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P,
                                          ctypes.c_int, P, P, P, ctypes.c_int, ctypes.c_int, P]
        L.oracle_shared_gate.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P]
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_half_to_double.restype = ctypes.c_double
        L.oracle_float_to_half.argtypes = [ctypes.c_float]
        L.oracle_float_to_half.restype = ctypes.c_uint16
        L.oracle_block_weights.argtypes = [ctypes.c_int]
        L.oracle_block_bytes.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def block_weights(fmt: int) -> int:
    return lib().oracle_block_weights(fmt)


def block_bytes(fmt: int) -> int:
    return lib().oracle_block_bytes(fmt)


def half_to_double(bits: int) -> float:
    return lib().oracle_half_to_double(bits)


def float_to_half(x: float) -> int:
    return lib().oracle_float_to_half(x)


def dequant_row(fmt: int, row: np.ndarray):
    """O1: (exact fp64 weights, fp32 weights) of one packed row of whole blocks."""
    row = np.ascontiguousarray(row, dtype=np.uint8)
    bb, bw = block_bytes(fmt), block_weights(fmt)
    assert row.size % bb == 0
    nb = row.size // bb
    w64 = np.empty(nb * bw, np.float64)
    w32 = np.empty(nb * bw, np.float32)
    if lib().oracle_dequant_row(fmt, _p(row), nb, _p(w64), _p(w32)) != 0:
        raise ValueError("unknown format")
    return w64, w32


def dequant_matrix(fmt: int, buf: np.ndarray, rows: int, stride: int, nblocks: int):
    """O1 over `rows` packed rows of `nblocks` blocks, `stride` bytes apart."""
    bw = block_weights(fmt)
    w64 = np.empty((rows, nblocks * bw), np.float64)
    w32 = np.empty((rows, nblocks * bw), np.float32)
    bb = block_bytes(fmt)
    for r in range(rows):
        w64[r], w32[r] = dequant_row(fmt, buf[r * stride: r * stride + nblocks * bb])
    return w64, w32


def quantize_q8_1(x: np.ndarray):
    """O2: (q int8 [n], d16 uint16 [n/32], s16 uint16 [n/32], number of non-finite blocks)."""
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    assert x.size % 32 == 0
    nb = x.size // 32
    q = np.empty(x.size, np.int8)
    d = np.empty(nb, np.uint16)
    s = np.empty(nb, np.uint16)
    bad = lib().oracle_quantize_q8_1(_p(x), nb, _p(q), _p(d), _p(s))
    return q, d, s, int(bad)


def topk(logits: np.ndarray, k: int):
    """O3: (ids int32 [T][k], w fp32 [T][k], number of tokens with non-finite logits)."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    bad = lib().oracle_topk(_p(logits), T, E, k, _p(ids), _p(w))
    return ids, w, int(bad)


def group(ids: np.ndarray, E: int):
    """O4: (counts [E], offsets [E+1], perm [T*k], inv_perm [T*k])."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    if lib().oracle_group(_p(ids), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv)) != 0:
        raise ValueError("expert id out of range")
    return counts, offsets, perm, inv


EXPERT_DTYPE = np.dtype([("fmt", np.int32), ("reserved", np.int32), ("off", np.int64, 3),
                         ("stride", np.int64, 3)])


def experts_table(fmts, offs, strides) -> np.ndarray:
    """Pack per-expert (format, [gate, up, down] byte offsets, [gate, up, down] row strides)."""
    t = np.zeros(len(fmts), EXPERT_DTYPE)
    t["fmt"] = fmts
    t["off"] = offs
    t["stride"] = strides
    return t


def expert_ffn(arena: np.ndarray, expert: np.ndarray, hidden: int, ffn: int, xhat: np.ndarray):
    """O5-O8 for one token and one expert: dict of g, u, h, hq, hd, hs, y."""
    arena = np.ascontiguousarray(arena, dtype=np.uint8)
    ex = np.ascontiguousarray(expert, dtype=EXPERT_DTYPE).reshape(1)
    bw = block_weights(int(ex["fmt"][0]))
    fp = (ffn + bw - 1) // bw * bw
    xhat = np.ascontiguousarray(xhat, dtype=np.float64)
    out = dict(g=np.empty(ffn), u=np.empty(ffn), h=np.empty(ffn), hq=np.empty(fp, np.int8),
               hd=np.empty(fp // 32, np.uint16), hs=np.empty(fp // 32, np.uint16),
               y=np.empty(hidden))
    rc = lib().oracle_expert_ffn(_p(arena), _p(ex), hidden, ffn, _p(xhat), _p(out["g"]),
                                 _p(out["u"]), _p(out["h"]), _p(out["hq"]), _p(out["hd"]),
                                 _p(out["hs"]), _p(out["y"]))
    if rc != 0:
        raise ValueError("bad expert")
    return out


def down_combine(arena: np.ndarray, experts: np.ndarray, hidden: int, ffn: int, hq: np.ndarray,
                 hd: np.ndarray, slot_tok, slot_exp, slot_w, T: int) -> np.ndarray:
    """O8-O9 from given Q8_1(h) rows: out fp64 [T][hidden] = sum over slots s of
    slot_w[s] * W_down(slot_exp[s]) * dequant(hq[s], hd[s]), added to token slot_tok[s]."""
    arena = np.ascontiguousarray(arena, dtype=np.uint8)
    experts = np.ascontiguousarray(experts, dtype=EXPERT_DTYPE)
    hq = np.ascontiguousarray(hq, dtype=np.int8)
    hd = np.ascontiguousarray(hd, dtype=np.uint16)
    n, hpad = hq.shape
    assert hd.shape == (n, hpad // 32)
    st = np.ascontiguousarray(slot_tok, dtype=np.int32)
    se = np.ascontiguousarray(slot_exp, dtype=np.int32)
    sw = np.ascontiguousarray(slot_w, dtype=np.float64)
    out = np.empty((T, hidden), np.float64)
    if lib().oracle_down_combine(_p(arena), _p(experts), len(experts), hidden, ffn, _p(hq), _p(hd),
                                 hpad, _p(st), _p(se), _p(sw), n, T, _p(out)) != 0:
        raise ValueError("oracle_down_combine: bad arguments")
    return out


def router(x: np.ndarray, Wr: np.ndarray):
    """O10: router logits of x [T][H] and rows Wr [E][H]: (fp32 [T][E], fp64 sums [T][E])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    Wr = np.ascontiguousarray(Wr, dtype=np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    assert Wr.shape[1] == H
    l32 = np.empty((T, E), np.float32)
    l64 = np.empty((T, E), np.float64)
    if lib().oracle_router(_p(x), _p(Wr), T, H, E, _p(l32), _p(l64)) != 0:
        raise ValueError("oracle_router: bad arguments")
    return l32, l64


def shared_gate(x: np.ndarray, wg: np.ndarray) -> np.ndarray:
    """O11: the shared-expert gate sigmoid(x . wg) per token, fp64 [T]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    wg = np.ascontiguousarray(wg, dtype=np.float32)
    T, H = x.shape
    assert wg.shape == (H,)
    g = np.empty(T, np.float64)
    if lib().oracle_shared_gate(_p(x), _p(wg), T, H, _p(g)) != 0:
        raise ValueError("oracle_shared_gate: bad arguments")
    return g


def forward(arena: np.ndarray, experts: np.ndarray, shared: int, hidden: int, ffn: int,
            x: np.ndarray, ids: np.ndarray, w: np.ndarray, tokens=None, gate=None):
    """O1-O9: (out fp32, out fp64), one row per listed token (all tokens if `tokens` is None).
    With `gate` (fp64 [T], from shared_gate) the shared expert's output is scaled by it (O11)."""
    arena = np.ascontiguousarray(arena, dtype=np.uint8)
    experts = np.ascontiguousarray(experts, dtype=EXPERT_DTYPE)
    x = np.ascontiguousarray(x, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    T, k = ids.shape
    if tokens is None:
        n = T
        tp = None
    else:
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        n = tokens.size
        tp = _p(tokens)
    out = np.empty((n, hidden), np.float32)
    out64 = np.empty((n, hidden), np.float64)
    if gate is None:
        rc = lib().oracle_forward(_p(arena), _p(experts), len(experts), shared, hidden, ffn,
                                  _p(x), _p(ids), _p(w), T, k, tp, n, _p(out), _p(out64))
    else:
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        assert gate.shape == (T,)
        rc = lib().oracle_forward_gated(_p(arena), _p(experts), len(experts), shared, hidden,
                                        ffn, _p(x), _p(ids), _p(w), T, k, tp, n, _p(gate),
                                        _p(out), _p(out64))
    if rc != 0:
        raise ValueError("oracle_forward: bad arguments")
    return out, out64


RMS_EPS = 1e-6


def rmsnorm(x: np.ndarray, weight=None, eps: float = RMS_EPS) -> np.ndarray:
    """The input of a pre-norm decoder's MoE block: every row of fp32 x divided by the root of
    its mean square plus eps, times the fp32 norm weight [H] (all ones when None), in fp64
    (squares summed in fp64), rounded once to fp32."""
    x64 = np.ascontiguousarray(x, dtype=np.float32).astype(np.float64)
    ms = (x64 * x64).sum(axis=1, keepdims=True) / x64.shape[1]
    y = x64 / np.sqrt(ms + eps)
    if weight is not None:
        y = y * np.asarray(weight, dtype=np.float32).astype(np.float64)[None, :]
    return y.astype(np.float32)


def chain(layers, x0: np.ndarray, k: int, lookahead: bool = False):
    """O12: a chain of MoE layers on a residual stream, as in a pre-norm decoder: for each layer
    l, xn_l = rmsnorm(x_l, norm weight), logits = router(xn_l, Wr_l) (O10), top-k (O3), out_l =
    O1-O9 on xn_l (gated by O11 of xn_l when the layer has a gate row), and x_{l+1} =
    fp32(x_l + out_l).  `layers` is a sequence of dicts with keys arena, experts, shared, hidden,
    ffn, router (Wr [E][H]) and optionally gate (wg [H]) and norm (the RMSNorm weight [H]).

    Returns (x_L fp32 [T][H], per-layer ids).  With lookahead=True it also returns, for every
    layer l >= 1, the ids that layer l's router picks from xn_{l-1} (before layer l-1 has
    run): the experts a prefetch one layer ahead would fetch."""
    x = np.ascontiguousarray(x0, dtype=np.float32)
    all_ids, early = [], []
    for l, L in enumerate(layers):
        xn = rmsnorm(x, L.get("norm"))
        logits, _ = router(xn, L["router"])
        ids, w, _ = topk(logits, k)
        g = shared_gate(xn, L["gate"]) if L.get("gate") is not None else None
        out, _ = forward(L["arena"], L["experts"], L["shared"], L["hidden"], L["ffn"], xn, ids,
                         w, gate=g)
        if lookahead and l + 1 < len(layers):
            early.append(topk(router(xn, layers[l + 1]["router"])[0], k)[0])
        x = (x + out).astype(np.float32)
        all_ids.append(ids)
    return (x, all_ids, early) if lookahead else (x, all_ids)


def set_threads(n: int) -> int:
    """OpenMP threads for oracle_forward (0 keeps the default); returns the count in use."""
    return lib().oracle_set_threads(n)
