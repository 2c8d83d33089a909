"""ctypes binding of libmoe.so: the same entry points as include/moe.h, argument marshalling only.

Every step of the layer runs in the CUDA library; nothing here computes.  If the library is
missing this module raises on import -- there is no fallback of any kind.

Device pointers are passed as ints (``tensor.data_ptr()``); ``stream`` is a cudaStream_t as an
int (``torch.cuda.current_stream().cuda_stream``) or None for the default stream.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libmoe.so"

if not LIB_PATH.exists():
    raise ImportError(f"{LIB_PATH} is not built: run `python -m expert_ffn_token_b200.build`")

_lib = ctypes.CDLL(str(LIB_PATH))

OK = 0
ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_CUDA = 1, 2, 3, 4
ERR_NONFINITE, ERR_BOUNDS, ERR_TIMEOUT, ERR_WORKSPACE = 5, 6, 7, 8

FMT_Q4_K, FMT_Q5_K, FMT_Q8_0, FMT_Q5_1, FMT_Q6_K = 0, 1, 2, 3, 4

F_DETERMINISTIC = 1
F_FORCE_DECODE = 2
F_FORCE_PREFILL = 4
F_KEEP_H = 8
F_LOOKAHEAD = 16
F_TC_I8 = 32

EXPORTED = ["moe_arena_create", "moe_arena_destroy", "moe_workspace_size", "moe_quantize_act",
            "moe_route_workspace_size", "moe_route_topk", "moe_forward", "moe_ws_views",
            "moe_read_status", "moe_debug_dequant", "moe_status_string",
            "moe_kernels_enqueued", "moe_forward_noalloc", "moe_set_timing_events",
            "moe_router_logits", "moe_shared_gate", "moe_set_wait_limit",
            "moe_forward_routed", "moe_chain_workspace_size", "moe_chain_forward",
            "moe_chain_status"]


class ExpertDesc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("off", ctypes.c_uint64 * 3), ("stride", ctypes.c_uint64 * 3)]


class WsView(ctypes.Structure):
    _fields_ = [("status", ctypes.c_void_p), ("xq", ctypes.c_void_p), ("xd", ctypes.c_void_p),
                ("xs", ctypes.c_void_p), ("ids", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("perm", ctypes.c_void_p), ("inv_perm", ctypes.c_void_p),
                ("hq", ctypes.c_void_p), ("hd", ctypes.c_void_p), ("hs", ctypes.c_void_p),
                ("h", ctypes.c_void_p), ("slots", ctypes.c_int32), ("hpad", ctypes.c_int32),
                ("counters", ctypes.c_void_p)]


class ChainLayer(ctypes.Structure):
    _fields_ = [("arena", ctypes.c_void_p), ("d_router", ctypes.c_void_p),
                ("d_gate_row", ctypes.c_void_p), ("d_norm_weight", ctypes.c_void_p)]


class ChainTrace(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("xn", ctypes.c_void_p), ("logits", ctypes.c_void_p),
                ("ids", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("early", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_S = ctypes.c_size_t
_U = ctypes.c_uint32

_lib.moe_status_string.restype = ctypes.c_char_p
_lib.moe_status_string.argtypes = [_I]
_lib.moe_arena_create.argtypes = [_P, _S, _I, _I, _I, _I, _P, ctypes.POINTER(_P)]
_lib.moe_arena_destroy.argtypes = [_P]
_lib.moe_arena_destroy.restype = None
_lib.moe_workspace_size.argtypes = [_P, _I, _I, _U, ctypes.POINTER(_S)]
_lib.moe_quantize_act.argtypes = [_P, _I, _I, _P, _P, _P, _P, _P]
_lib.moe_route_workspace_size.argtypes = [_I, _I, _I, ctypes.POINTER(_S)]
_lib.moe_route_topk.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]
_lib.moe_forward.argtypes = [_P, _P, _P, _I, _I, _P, _P, _S, _U, _P]
_lib.moe_ws_views.argtypes = [_P, _P, _I, _I, _U, ctypes.POINTER(WsView)]
_lib.moe_read_status.argtypes = [_P, _P, _I, ctypes.POINTER(_I)]
_lib.moe_debug_dequant.argtypes = [_P, _I, _I, _P, _P]
_lib.moe_forward_noalloc.argtypes = [_P, _P, _P, _I, _I, _P, _P, _P]
_lib.moe_set_timing_events.argtypes = [_P, _P, _P, _P]
_lib.moe_router_logits.argtypes = [_P, _I, _I, _P, _I, _P, _P]
_lib.moe_shared_gate.argtypes = [_P, _I, _I, _P, _P, _P]
_lib.moe_set_wait_limit.argtypes = [_P, ctypes.c_uint64]
_lib.moe_forward_routed.argtypes = [_P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _S, _U, _P]
_lib.moe_chain_workspace_size.argtypes = [_P, _I, _I, _I, _U, ctypes.POINTER(_S)]
_lib.moe_chain_forward.argtypes = [_P, _I, _P, _I, _I, _P, _P, _S, _U, _P, _P]
_lib.moe_chain_status.argtypes = [_P, _I, _P, _I, _I, _U, ctypes.POINTER(_P)]
_lib.moe_kernels_enqueued.argtypes = []
_lib.moe_kernels_enqueued.restype = ctypes.c_uint64


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_string(code)} ({code})")
        self.code = code


def status_string(code: int) -> str:
    return _lib.moe_status_string(code).decode()


def _check(code: int, where: str) -> None:
    if code != OK:
        raise MoeError(code, where)


def library():
    """The loaded CDLL (for symbol checks)."""
    return _lib


def arena_create(d_arena: int, arena_bytes: int, hidden: int, ffn: int, n_experts: int,
                 shared_expert: int, descs) -> int:
    """descs: sequence of (fmt, (off_gate, off_up, off_down), (stride_gate, stride_up, stride_down))."""
    arr = (ExpertDesc * len(descs))()
    for i, (fmt, off, stride) in enumerate(descs):
        arr[i].fmt = int(fmt)
        arr[i].reserved = 0
        for t in range(3):
            arr[i].off[t] = int(off[t])
            arr[i].stride[t] = int(stride[t])
    h = _P()
    _check(_lib.moe_arena_create(d_arena, arena_bytes, hidden, ffn, n_experts, shared_expert,
                                 ctypes.cast(arr, _P), ctypes.byref(h)), "moe_arena_create")
    return h.value


def arena_destroy(arena: int) -> None:
    _lib.moe_arena_destroy(arena)


def workspace_size(arena: int, max_tokens: int, k: int, flags: int = 0) -> int:
    n = _S()
    _check(_lib.moe_workspace_size(arena, max_tokens, k, flags, ctypes.byref(n)),
           "moe_workspace_size")
    return n.value


def quantize_act(d_x: int, T: int, H: int, d_q: int, d_d: int, d_s: int, d_status=None,
                 stream=None) -> None:
    _check(_lib.moe_quantize_act(d_x, T, H, d_q, d_d, d_s, d_status, stream), "moe_quantize_act")


def route_workspace_size(T: int, E: int, k: int) -> int:
    n = _S()
    _check(_lib.moe_route_workspace_size(T, E, k, ctypes.byref(n)), "moe_route_workspace_size")
    return n.value


def router_logits(d_x: int, T: int, H: int, d_router: int, E: int, d_logits: int,
                  stream=None) -> None:
    _check(_lib.moe_router_logits(d_x, T, H, d_router, E, d_logits, stream), "moe_router_logits")


def router_logits_status(d_x, T, H, d_router, E, d_logits, stream=None) -> int:
    return _lib.moe_router_logits(d_x, T, H, d_router, E, d_logits, stream)


def shared_gate(d_x: int, T: int, H: int, d_gate_row: int, d_gate: int, stream=None) -> None:
    _check(_lib.moe_shared_gate(d_x, T, H, d_gate_row, d_gate, stream), "moe_shared_gate")


def route_topk(d_logits: int, T: int, E: int, k: int, d_ids: int, d_w: int, d_counts: int,
               d_offsets: int, d_perm: int, d_inv_perm, d_status, d_ws: int, ws_bytes: int,
               stream=None) -> None:
    _check(_lib.moe_route_topk(d_logits, T, E, k, d_ids, d_w, d_counts, d_offsets, d_perm,
                               d_inv_perm, d_status, d_ws, ws_bytes, stream), "moe_route_topk")


def forward(arena: int, d_x: int, d_logits: int, T: int, k: int, d_out: int, d_ws: int,
            ws_bytes: int, flags: int = 0, stream=None) -> None:
    _check(_lib.moe_forward(arena, d_x, d_logits, T, k, d_out, d_ws, ws_bytes, flags, stream),
           "moe_forward")


def forward_noalloc(arena: int, d_x: int, d_logits: int, T: int, k: int, d_out: int,
                    d_status=None, stream=None) -> None:
    """moe_forward_noalloc: the layer for 1..16 tokens using the library's fixed scratch."""
    _check(_lib.moe_forward_noalloc(arena, d_x, d_logits, T, k, d_out, d_status, stream),
           "moe_forward_noalloc")


def forward_noalloc_status(arena, d_x, d_logits, T, k, d_out, d_status=None, stream=None) -> int:
    """moe_forward_noalloc returning its status code instead of raising."""
    return _lib.moe_forward_noalloc(arena, d_x, d_logits, T, k, d_out, d_status, stream)


def forward_status(arena, d_x, d_logits, T, k, d_out, d_ws, ws_bytes, flags=0, stream=None) -> int:
    """moe_forward returning its status code instead of raising (for error-path tests)."""
    return _lib.moe_forward(arena, d_x, d_logits, T, k, d_out, d_ws, ws_bytes, flags, stream)


def forward_routed(arena: int, d_x: int, T: int, k: int, d_router: int, d_gate_row, d_logits: int,
                   d_gate, d_out: int, d_ws: int, ws_bytes: int, flags: int = 0,
                   stream=None) -> None:
    """moe_forward_routed: router (and optional shared gate) then the layer."""
    _check(forward_routed_status(arena, d_x, T, k, d_router, d_gate_row, d_logits, d_gate, d_out,
                                 d_ws, ws_bytes, flags, stream), "moe_forward_routed")


def forward_routed_status(arena, d_x, T, k, d_router, d_gate_row, d_logits, d_gate, d_out, d_ws,
                          ws_bytes, flags=0, stream=None) -> int:
    return _lib.moe_forward_routed(arena, d_x, T, k, d_router, d_gate_row, d_logits, d_gate, d_out,
                                   d_ws, ws_bytes, flags, stream)


def _chain_layers(layers):
    """layers: sequence of (arena handle, d_router, d_gate_row or None[, d_norm_weight or None])."""
    arr = (ChainLayer * len(layers))()
    for i, ly in enumerate(layers):
        arr[i].arena, arr[i].d_router, arr[i].d_gate_row = ly[0], ly[1], ly[2]
        arr[i].d_norm_weight = ly[3] if len(ly) > 3 else None
    return arr


def chain_workspace_size(layers, max_tokens: int, k: int, flags: int = 0) -> int:
    n = _S()
    _check(_lib.moe_chain_workspace_size(_chain_layers(layers), len(layers), max_tokens, k, flags,
                                         ctypes.byref(n)), "moe_chain_workspace_size")
    return n.value


def chain_forward_status(layers, d_x: int, T: int, k: int, d_x_out: int, d_ws: int,
                         ws_bytes: int, flags: int = 0, trace=None, stream=None) -> int:
    """moe_chain_forward returning its status; trace: dict of device pointers (ChainTrace
    field names) or None."""
    tr = None
    if trace is not None:
        tr = ChainTrace(**{k2: trace.get(k2) for k2, _ in ChainTrace._fields_})
    return _lib.moe_chain_forward(_chain_layers(layers), len(layers), d_x, T, k, d_x_out, d_ws,
                                  ws_bytes, flags, ctypes.byref(tr) if tr is not None else None,
                                  stream)


def chain_forward(layers, d_x: int, T: int, k: int, d_x_out: int, d_ws: int, ws_bytes: int,
                  flags: int = 0, trace=None, stream=None) -> None:
    _check(chain_forward_status(layers, d_x, T, k, d_x_out, d_ws, ws_bytes, flags, trace, stream),
           "moe_chain_forward")


def chain_status_word(layers, d_ws: int, T: int, k: int, flags: int = 0) -> int:
    p = _P()
    _check(_lib.moe_chain_status(_chain_layers(layers), len(layers), d_ws, T, k, flags,
                                 ctypes.byref(p)), "moe_chain_status")
    return p.value


def ws_views(arena: int, d_ws: int, T: int, k: int, flags: int = 0) -> dict:
    v = WsView()
    _check(_lib.moe_ws_views(arena, d_ws, T, k, flags, ctypes.byref(v)), "moe_ws_views")
    return {name: getattr(v, name) for name, _ in WsView._fields_}


def read_status(d_status: int, stream=None, clear: bool = True) -> int:
    s = _I()
    _check(_lib.moe_read_status(d_status, stream, 1 if clear else 0, ctypes.byref(s)),
           "moe_read_status")
    return s.value


def set_timing_events(arena: int, ev_begin=None, ev_mid=None, ev_end=None) -> None:
    """moe_set_timing_events: cudaEvent_t handles (ints) recorded around the tensor-core phases
    of later forwards on this arena, or None to stop."""
    _check(_lib.moe_set_timing_events(arena, ev_begin, ev_mid, ev_end), "moe_set_timing_events")


def set_wait_limit(arena: int, ns: int) -> None:
    """moe_set_wait_limit: limit of every bounded device wait of later calls on this arena."""
    _check(_lib.moe_set_wait_limit(arena, ns), "moe_set_wait_limit")


def kernels_enqueued() -> int:
    return int(_lib.moe_kernels_enqueued())


def debug_dequant(arena: int, expert: int, which: int, d_out: int, stream=None) -> None:
    _check(_lib.moe_debug_dequant(arena, expert, which, d_out, stream), "moe_debug_dequant")


# ------------------------------------------------------------------ torch convenience


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


class Layer:
    """One MoE layer over a device arena held in a torch uint8 tensor (marshalling only)."""

    def __init__(self, arena_tensor, hidden: int, ffn: int, n_experts: int, shared: bool,
                 descs, max_tokens: int, k: int, flags: int = 0):
        import torch
        self.arena_tensor = arena_tensor
        self.hidden, self.ffn, self.n_experts, self.k = hidden, ffn, n_experts, k
        self.flags = flags
        self.handle = arena_create(arena_tensor.data_ptr(), arena_tensor.numel(), hidden, ffn,
                                   n_experts, n_experts if shared else -1, descs)
        self.ws_bytes = workspace_size(self.handle, max_tokens, k, flags)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=arena_tensor.device)

    def forward(self, x, logits, out=None, flags=None):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        forward(self.handle, x.data_ptr(), logits.data_ptr(), T, self.k, out.data_ptr(),
                self.ws.data_ptr(), self.ws_bytes, self.flags if flags is None else flags,
                _stream())
        return out

    def views(self, T: int, flags=None) -> dict:
        return ws_views(self.handle, self.ws.data_ptr(), T, self.k,
                        self.flags if flags is None else flags)

    def status(self, clear: bool = True) -> int:
        return read_status(self.views(1)["status"], _stream(), clear)

    def close(self):
        if self.handle:
            arena_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
