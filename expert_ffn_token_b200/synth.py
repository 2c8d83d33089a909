"""Seeded synthetic inputs for the quantized MoE layer (both the CUDA path and the oracle use them).

This module holds no step of the layer's arithmetic: it only draws random bytes, scales and
vectors with the shapes, value ranges and structure of the workloads below, and lays them out in
an expert arena.  The same draws are made on the GPU for the multi-GB arenas by
``csrc/synth_fill.cu`` (``libmoe_synth.so``), from the same published generator, so that the
host and the device produce identical bytes.

Generator (counter based, SplitMix64's mixing function, Steele, Lea & Flood, OOPSLA 2014):

    G        = 0x9E3779B97F4A7C15
    mix64(z) : z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
               z ^= z >> 31                                             (all mod 2^64)
    key(seed, i0, i1, ...) : k = mix64(seed + G); for each id: k = mix64(k ^ ((id + 1) * G))
    word(k, n)  = mix64(k + (n + 1) * G)
    uniform(k, n) = (word(k, n) >> 11) * 2^-53                        (in [0, 1))
    open_uniform(k, n) = ((word(k, n) >> 11) + 0.5) * 2^-53           (in (0, 1))

Weight tensors of expert e in layer l (tensor t: 0 gate, 1 up, 2 down), rows of whole blocks,
`stride` bytes apart:
    raw byte at p = row * stride + col (col < blocks * block_bytes):
        byte (p % 8) of word(key(seed, l, e, t, 0), p // 8)   (little endian)
    block i (= row * blocks + col // block_bytes):
        d    = fp16(fp32(1e-3 + 9e-3 * uniform(key(seed, l, e, t, 1), i)))   bytes 0-1
        dmin = fp16(fp32(1e-3 + 9e-3 * uniform(key(seed, l, e, t, 2), i)))   bytes 2-3 (K-quants)
        m    = -16 * dmin (exact in fp16)                                  bytes 2-3 (Q5_1)
    Q6_K blocks keep d at bytes 208-209 instead (the scale bytes 192-207 are raw int8 draws);
    their 16-weight groups past the row's logical width get scale 0.  Q6_K is drawn on the
    host only: the device fill refuses it.
    K-quant blocks that run past the row's logical width (down rows of width 640 stored as
    768) get scale and min 0 for the sub-blocks past the width, so those weights are exactly 0.
    Pad bytes after the last block of a row are 0.

Vectors (host only): x = N(0,1) by Box-Muller on (open_uniform(k, 2n), uniform(k, 2n+1)) with
k = key(seed, l, 100), optional outlier channels (key(seed, l, 101)) scaled by 20; router logits
N(0, sigma) (key(seed, l, 102, attempt)) or Zipf(s) popularity plus Gumbel noise (ranks from
key(seed, l, 103), noise from key(seed, l, 104, attempt)); a token's row is drawn again with
the next attempt until every adjacent gap among its k+1 largest fp32 logits is >= 1e-3.
Per-expert formats (mixed workload): uniform(key(seed, l, 105), e) < 0.60 Q4_K, < 0.85 Q5_K,
else Q8_0; a workload's `mix` can give other thresholds and Q5_1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

Q4_K, Q5_K, Q8_0, Q5_1, Q6_K = 0, 1, 2, 3, 4
FMT_NAMES = {Q4_K: "Q4_K", Q5_K: "Q5_K", Q8_0: "Q8_0", Q5_1: "Q5_1", Q6_K: "Q6_K"}
BLOCK_WEIGHTS = {Q4_K: 256, Q5_K: 256, Q8_0: 32, Q5_1: 32, Q6_K: 256}
BLOCK_BYTES = {Q4_K: 144, Q5_K: 176, Q8_0: 34, Q5_1: 24, Q6_K: 210}
TENSOR_ALIGN = 256

G = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def mix64(z):
    z = np.asarray(z, dtype=np.uint64).copy()
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def key(seed: int, *ids: int) -> int:
    with np.errstate(over="ignore"):
        k = mix64(np.array([seed], np.uint64) + G)
        for i in ids:
            k = mix64(k ^ (np.array([i + 1], np.uint64) * G))
    return int(k[0])


def words(k: int, n0: int, count: int) -> np.ndarray:
    n = np.arange(n0 + 1, n0 + 1 + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(k) + n * G)


def uniform(k: int, n0: int, count: int) -> np.ndarray:
    return (words(k, n0, count) >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def open_uniform(k: int, n0: int, count: int) -> np.ndarray:
    return ((words(k, n0, count) >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53


def normal(k: int, n0: int, count: int) -> np.ndarray:
    """Box-Muller, fp64, pairs (2n, 2n+1) of the stream -> one N(0,1) value n."""
    w = words(k, 2 * n0, 2 * count)
    u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53
    u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def scale_to_half(u: np.ndarray) -> np.ndarray:
    """fp16 bits of fp32(1e-3 + 9e-3 * u): the d / dmin draw."""
    v = (1e-3 + 9e-3 * u).astype(np.float32)
    return v.astype(np.float16).view(np.uint16)


# ------------------------------------------------------------------ workloads


@dataclass(frozen=True)
class Workload:
    name: str
    index: int              # seeds are 0x5EED0000 + index
    hidden: int
    ffn: int
    n_experts: int
    k: int
    tokens: int
    shared: bool
    layers: int
    logits: str             # "normal" or "zipf"
    sigma: float = 1.0
    zipf_s: float = 0.0
    outlier_frac: float = 0.0
    outlier_scale: float = 20.0
    mix: tuple = ()         # ((fmt, cumulative probability), ...) or () for all Q4_K
    note: str = ""

    @property
    def seed(self) -> int:
        return 0x5EED0000 + self.index


WORKLOADS = {
    "tiny": Workload("tiny", 1, 256, 256, 16, 2, 4, False, 1, "normal", sigma=1.0,
                     note="hidden 256, 16 experts, top-2, width 256, 4 tokens, Q4_K"),
    "decode": Workload("decode", 2, 2048, 512, 256, 8, 1, False, 48, "normal", sigma=2.0,
                       note="Qwen3.6-35B-A3B-shaped decode layer: hidden 2048, 256 experts, "
                            "top-8, width 512, 1 token, Q4_K, 48 independent layers"),
    "mtp_verify": Workload("mtp_verify", 3, 2560, 640, 512, 10, 3, True, 48, "zipf",
                           zipf_s=1.1,
                           note="Qwen3.8-Flash-Next-shaped MTP verify: hidden 2560, 512 experts,"
                                " top-10 + shared, width 640, 3 tokens, Q4_K, Zipf 1.1, 48 layers"),
    "prefill": Workload("prefill", 4, 2560, 640, 512, 10, 4096, True, 1, "normal", sigma=2.0,
                        outlier_frac=0.01,
                        note="prefill chunk: 4096 tokens, hidden 2560, 512 experts, top-10 + "
                             "shared, width 640, Q4_K, 1% outlier channels x20"),
    "mixed_prefill": Workload("mixed_prefill", 5, 2560, 640, 512, 10, 8192, True, 1, "zipf",
                              zipf_s=1.3, mix=((Q4_K, 0.60), (Q5_K, 0.85), (Q8_0, 1.0)),
                              note="mixed-format long prefill: 8192 tokens, 60% Q4_K / 25% Q5_K"
                                   " / 15% Q8_0 experts, Zipf 1.3"),
}


def with_tokens(w: Workload, tokens: int, layers: int | None = None) -> Workload:
    """The same layer recipe with another token count (edge and sampled parity cases)."""
    d = dict(w.__dict__)
    d["tokens"] = tokens
    if layers is not None:
        d["layers"] = layers
    return Workload(**d)


# ------------------------------------------------------------------ arena layout


def row_stride(fmt: int, width: int) -> int:
    """Bytes per packed row of `width` weights (whole blocks, rounded up to 16 bytes)."""
    nb = -(-width // BLOCK_WEIGHTS[fmt])
    return -(-nb * BLOCK_BYTES[fmt] // 16) * 16


def row_blocks(fmt: int, width: int) -> int:
    return -(-width // BLOCK_WEIGHTS[fmt])


@dataclass
class ArenaLayout:
    """Per layer: experts 0..E-1, then the shared expert (index E) if present; per expert the
    gate, up and down matrices, each starting on a 256-byte boundary."""
    hidden: int
    ffn: int
    fmts: np.ndarray                      # int32 [n]
    offs: np.ndarray                      # int64 [n][3]
    strides: np.ndarray                   # int64 [n][3]
    nbytes: int
    shared: int                           # index of the shared expert or -1
    tensor_bytes: np.ndarray = field(default=None)   # int64 [n][3]

    @property
    def n(self) -> int:
        return len(self.fmts)

    def expert_bytes(self, e: int) -> int:
        return int(self.tensor_bytes[e].sum())


def layer_formats(w: Workload, layer: int) -> np.ndarray:
    n = w.n_experts + (1 if w.shared else 0)
    if not w.mix:
        return np.full(n, Q4_K, np.int32)
    u = uniform(key(w.seed, layer, 105), 0, n)
    f = np.empty(n, np.int32)
    lo = 0.0
    for fmt, hi in w.mix:
        f[(u >= lo) & (u < hi)] = fmt
        lo = hi
    return f


def arena_layout(w: Workload, fmts: np.ndarray) -> ArenaLayout:
    n = len(fmts)
    offs = np.zeros((n, 3), np.int64)
    strides = np.zeros((n, 3), np.int64)
    tb = np.zeros((n, 3), np.int64)
    pos = 0
    for e in range(n):
        f = int(fmts[e])
        for t, (rows, width) in enumerate(((w.ffn, w.hidden), (w.ffn, w.hidden),
                                           (w.hidden, w.ffn))):
            pos = -(-pos // TENSOR_ALIGN) * TENSOR_ALIGN
            s = row_stride(f, width)
            offs[e, t] = pos
            strides[e, t] = s
            tb[e, t] = rows * s
            pos += rows * s
    pos = -(-pos // TENSOR_ALIGN) * TENSOR_ALIGN
    return ArenaLayout(w.hidden, w.ffn, fmts.astype(np.int32), offs, strides, pos,
                       w.n_experts if w.shared else -1, tb)


def tensor_shape(w: Workload, t: int):
    """(rows, logical width) of tensor t (0 gate, 1 up, 2 down)."""
    return (w.ffn, w.hidden) if t < 2 else (w.hidden, w.ffn)


def tensor_bytes(w: Workload, layer: int, e: int, t: int, fmt: int) -> np.ndarray:
    """Host bytes of one weight tensor, exactly as the device fill writes them."""
    rows, width = tensor_shape(w, t)
    stride = row_stride(fmt, width)
    nb = row_blocks(fmt, width)
    bb = BLOCK_BYTES[fmt]
    total = rows * stride
    raw = words(key(w.seed, layer, e, t, 0), 0, -(-total // 8)).view(np.uint8)[:total].copy()
    m = raw.reshape(rows, stride)
    m[:, nb * bb:] = 0
    blocks = m[:, :nb * bb].copy().reshape(rows, nb, bb)
    nblk = rows * nb
    d = scale_to_half(uniform(key(w.seed, layer, e, t, 1), 0, nblk)).reshape(rows, nb)
    blocks[:, :, 0] = (d & 0xFF).astype(np.uint8)
    blocks[:, :, 1] = (d >> 8).astype(np.uint8)
    if fmt == Q6_K:
        # d lives at the end of a Q6_K block; the first two bytes are quants like the rest
        raw_first = m[:, :nb * bb].reshape(rows, nb, bb)[:, :, 0:2].copy()
        blocks[:, :, 0:2] = raw_first
        blocks[:, :, 208] = (d & 0xFF).astype(np.uint8)
        blocks[:, :, 209] = (d >> 8).astype(np.uint8)
        valid = width - (nb - 1) * 256
        if valid < 256:
            blocks[:, nb - 1, 192 + valid // 16:208] = 0
    elif fmt == Q5_1:
        dm = scale_to_half(uniform(key(w.seed, layer, e, t, 2), 0, nblk)).reshape(rows, nb)
        mm = (dm + np.uint16(4 << 10)) | np.uint16(0x8000)      # -16 * dmin: exponent + 4, sign
        blocks[:, :, 2] = (mm & 0xFF).astype(np.uint8)
        blocks[:, :, 3] = (mm >> 8).astype(np.uint8)
    elif fmt != Q8_0:
        dm = scale_to_half(uniform(key(w.seed, layer, e, t, 2), 0, nblk)).reshape(rows, nb)
        blocks[:, :, 2] = (dm & 0xFF).astype(np.uint8)
        blocks[:, :, 3] = (dm >> 8).astype(np.uint8)
        valid = width - (nb - 1) * 256          # logical weights in the last block
        if valid < 256:
            kill_subblocks(blocks[:, nb - 1, 4:16], valid // 32)
    m[:, :nb * bb] = blocks.reshape(rows, nb * bb)
    return raw


def kill_subblocks(S: np.ndarray, n_valid: int) -> None:
    """Zero the 6-bit scale and min of sub-blocks n_valid..7 in packed K-quant scale bytes
    S[..., 12] (sub-block j < 4 keeps its scale/min in the low 6 bits of S[j] / S[j+4]; j >= 4
    in the nibbles of S[j+4] plus the top 2 bits of S[j-4] / S[j])."""
    for j in range(n_valid, 8):
        if j < 4:
            S[..., j] &= 0xC0
            S[..., j + 4] &= 0xC0
        else:
            S[..., j + 4] = 0
            S[..., j - 4] &= 0x3F
            S[..., j] &= 0x3F


def host_arena(w: Workload, layer: int, experts=None):
    """(arena bytes, layout) of one layer on the host.  With `experts` given, only those
    experts' tensors are filled (the rest stay zero) -- the oracle reads only what it needs."""
    fmts = layer_formats(w, layer)
    lay = arena_layout(w, fmts)
    buf = np.zeros(lay.nbytes, np.uint8)
    todo = range(lay.n) if experts is None else sorted(set(int(e) for e in experts))
    for e in todo:
        for t in range(3):
            b = tensor_bytes(w, layer, e, t, int(fmts[e]))
            buf[lay.offs[e, t]: lay.offs[e, t] + b.size] = b
    return buf, lay


def compact_arena(w: Workload, layer: int, experts):
    """Host arena holding only `experts` (packed back to back) and a layout whose offsets point
    into it; experts not listed get offset 0 and must not be read."""
    fmts = layer_formats(w, layer)
    full = arena_layout(w, fmts)
    offs = np.zeros_like(full.offs)
    chunks = []
    pos = 0
    for e in sorted(set(int(e) for e in experts)):
        for t in range(3):
            b = tensor_bytes(w, layer, e, t, int(fmts[e]))
            offs[e, t] = pos
            chunks.append(b)
            pad = -(-b.size // TENSOR_ALIGN) * TENSOR_ALIGN - b.size
            if pad:
                chunks.append(np.zeros(pad, np.uint8))
            pos += b.size + pad
    buf = np.concatenate(chunks) if chunks else np.zeros(0, np.uint8)
    lay = ArenaLayout(full.hidden, full.ffn, full.fmts, offs, full.strides, pos, full.shared,
                      full.tensor_bytes)
    return buf, lay


# ------------------------------------------------------------------ activations and logits


def activations(w: Workload, layer: int, tokens: int | None = None) -> np.ndarray:
    T = w.tokens if tokens is None else tokens
    x = normal(key(w.seed, layer, 100), 0, T * w.hidden).astype(np.float32).reshape(T, w.hidden)
    if w.outlier_frac > 0:
        n = math.ceil(w.outlier_frac * w.hidden)
        order = np.argsort(words(key(w.seed, layer, 101), 0, w.hidden), kind="stable")
        x[:, np.sort(order[:n])] *= np.float32(w.outlier_scale)
    return x


def _zipf_log_popularity(w: Workload, layer: int) -> np.ndarray:
    rank_of = np.empty(w.n_experts, np.int64)
    rank_of[np.argsort(words(key(w.seed, layer, 103), 0, w.n_experts), kind="stable")] = \
        np.arange(w.n_experts)
    r = (rank_of + 1).astype(np.float64)
    logp = -w.zipf_s * np.log(r)
    return logp - np.log(np.exp(logp).sum())


def _logit_rows(w: Workload, layer: int, attempt: int, rows: np.ndarray) -> np.ndarray:
    E = w.n_experts
    out = np.empty((rows.size, E), np.float32)
    for i, t in enumerate(rows):
        if w.logits == "zipf":
            u = open_uniform(key(w.seed, layer, 104, attempt), int(t) * E, E)
            out[i] = (_zipf_log_popularity(w, layer) - np.log(-np.log(u))).astype(np.float32)
        else:
            out[i] = (w.sigma * normal(key(w.seed, layer, 102, attempt), int(t) * E, E)
                      ).astype(np.float32)
    return out


def _gaps_ok(rows: np.ndarray, k: int) -> np.ndarray:
    top = -np.sort(-rows, axis=1)[:, :k + 1].astype(np.float64)
    return (np.diff(-top, axis=1) >= 1e-3).all(axis=1)


def router_logits(w: Workload, layer: int, tokens: int | None = None) -> np.ndarray:
    T = w.tokens if tokens is None else tokens
    E = w.n_experts
    if w.logits == "zipf":
        logp = _zipf_log_popularity(w, layer)
        u = open_uniform(key(w.seed, layer, 104, 0), 0, T * E).reshape(T, E)
        L = (logp[None, :] - np.log(-np.log(u))).astype(np.float32)
    else:
        L = (w.sigma * normal(key(w.seed, layer, 102, 0), 0, T * E)).astype(np.float32)
        L = L.reshape(T, E)
    bad = np.nonzero(~_gaps_ok(L, w.k))[0]
    attempt = 0
    while bad.size:
        attempt += 1
        L[bad] = _logit_rows(w, layer, attempt, bad)
        bad = bad[~_gaps_ok(L[bad], w.k)]
    return L


# ------------------------------------------------------------------ device fill (multi-GB arenas)

_synth_lib = None


def _synth():
    global _synth_lib
    if _synth_lib is None:
        import ctypes
        from pathlib import Path
        p = Path(__file__).resolve().parent / "libmoe_synth.so"
        if not p.exists():
            raise ImportError(f"{p} is not built: run `python -m expert_ffn_token_b200.build`")
        _synth_lib = ctypes.CDLL(str(p))
        _synth_lib.synth_fill_tensors.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                                  ctypes.c_void_p]
    return _synth_lib


def device_fill_layer(w: Workload, layer: int, d_base: int, stream=None) -> ArenaLayout:
    """Write layer `layer`'s arena at device address d_base (lay.nbytes bytes, 256-aligned):
    the same bytes as host_arena(w, layer), drawn on the GPU."""
    import ctypes

    class _T(ctypes.Structure):
        _fields_ = [("dst_off", ctypes.c_uint64), ("key_raw", ctypes.c_uint64),
                    ("key_d", ctypes.c_uint64), ("key_dmin", ctypes.c_uint64),
                    ("rows", ctypes.c_int32), ("stride", ctypes.c_int32),
                    ("nblocks", ctypes.c_int32), ("block_bytes", ctypes.c_int32),
                    ("kquant", ctypes.c_int32), ("valid_last", ctypes.c_int32)]

    fmts = layer_formats(w, layer)
    if (fmts == Q6_K).any():
        raise NotImplementedError("the device fill does not draw Q6_K blocks (host_arena does)")
    lay = arena_layout(w, fmts)
    tab = (_T * (lay.n * 3))()
    for e in range(lay.n):
        f = int(fmts[e])
        for t in range(3):
            rows, width = tensor_shape(w, t)
            nb = row_blocks(f, width)
            r = tab[e * 3 + t]
            r.dst_off = int(lay.offs[e, t])
            r.key_raw = key(w.seed, layer, e, t, 0)
            r.key_d = key(w.seed, layer, e, t, 1)
            r.key_dmin = key(w.seed, layer, e, t, 2)
            r.rows = rows
            r.stride = int(lay.strides[e, t])
            r.nblocks = nb
            r.block_bytes = BLOCK_BYTES[f]
            r.kquant = {Q8_0: 0, Q5_1: 2}.get(f, 1)
            r.valid_last = 8 if f in (Q8_0, Q5_1) else (width - (nb - 1) * 256) // 32
    rc = _synth().synth_fill_tensors(d_base, ctypes.cast(tab, ctypes.c_void_p), lay.n * 3, stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_tensors failed ({rc})")
    return lay


def layout_descs(lay: ArenaLayout):
    """(fmt, offsets, strides) per expert, the form moe.arena_create takes."""
    return [(int(lay.fmts[e]), tuple(int(v) for v in lay.offs[e]),
             tuple(int(v) for v in lay.strides[e])) for e in range(lay.n)]
