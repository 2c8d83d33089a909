"""Host-side checks of the C ABI (no GPU): the library loads, exports every declared entry point,
and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def moe():
    from expert_ffn_token_b200 import build
    build.build()
    from expert_ffn_token_b200 import moe as m
    return m


def test_every_declared_symbol_is_exported(moe):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(moe.library(), n), n
    assert set(moe.EXPORTED) <= set(names)


def test_status_strings(moe):
    assert moe.status_string(0) == "ok"
    assert "workspace" in moe.status_string(moe.ERR_WORKSPACE)
    assert moe.status_string(99) == "unknown status"


FAKE = 0x7f0000000000        # 256-aligned, never dereferenced: validation fails first


def _desc(fmt=0, off=(0, 36864, 73728), stride=(144, 144, 144)):
    return [(fmt, off, stride)]


def test_arena_create_rejects_bad_arguments(moe):
    L = moe.library()
    h = ctypes.c_void_p()

    def create(ptr=FAKE, nbytes=1 << 20, H=256, F=256, E=1, shared=-1, descs=None):
        arr = (moe.ExpertDesc * 2)()
        for i, (fmt, off, stride) in enumerate(descs or _desc()):
            arr[i].fmt = fmt
            for t in range(3):
                arr[i].off[t] = off[t]
                arr[i].stride[t] = stride[t]
        return L.moe_arena_create(ptr, nbytes, H, F, E, shared, ctypes.cast(arr, ctypes.c_void_p),
                                  ctypes.byref(h))

    assert create(ptr=None) == moe.ERR_INVALID_ARG
    assert create(H=100) == moe.ERR_INVALID_ARG                 # not a multiple of 32
    assert create(F=0) == moe.ERR_INVALID_ARG
    assert create(ptr=FAKE + 16) == moe.ERR_ALIGNMENT             # arena not 256-aligned
    assert create(shared=3) == moe.ERR_INVALID_ARG                # shared must be E
    assert create(H=8192) == moe.ERR_UNSUPPORTED
    assert create(descs=_desc(fmt=7)) == moe.ERR_INVALID_ARG
    assert create(descs=_desc(fmt=4)) == moe.ERR_INVALID_ARG       # formats are 0..3
    assert create(descs=_desc(fmt=3, stride=(176, 176, 176))) == moe.ERR_INVALID_ARG  # Q5_1 row: 192 B
    assert create(descs=_desc(off=(8, 36864, 73728))) == moe.ERR_ALIGNMENT
    assert create(descs=_desc(stride=(128, 144, 144))) == moe.ERR_INVALID_ARG  # < packed row
    assert create(nbytes=100000) == moe.ERR_BOUNDS                # down matrix ends past it
    assert create(H=288, descs=_desc()) == moe.ERR_UNSUPPORTED    # K-quant rows need H % 256 == 0
    assert L.moe_arena_create(FAKE, 1, 256, 256, 1, -1, None, ctypes.byref(h)) == moe.ERR_INVALID_ARG


def test_router_and_gate_reject_bad_arguments(moe):
    L = moe.library()
    assert L.moe_router_logits(None, 1, 64, FAKE, 8, FAKE, None) == moe.ERR_INVALID_ARG
    assert L.moe_router_logits(FAKE, 0, 64, FAKE, 8, FAKE, None) == moe.ERR_INVALID_ARG
    assert L.moe_router_logits(FAKE, 1, 66, FAKE, 8, FAKE, None) == moe.ERR_INVALID_ARG  # H % 4
    assert L.moe_router_logits(FAKE + 4, 1, 64, FAKE, 8, FAKE, None) == moe.ERR_ALIGNMENT
    assert L.moe_router_logits(FAKE, 1, 64, FAKE, 8, FAKE + 2, None) == moe.ERR_ALIGNMENT
    assert L.moe_shared_gate(FAKE, 1, 64, None, FAKE, None) == moe.ERR_INVALID_ARG
    assert L.moe_shared_gate(FAKE, 1, 64, FAKE + 8, FAKE, None) == moe.ERR_ALIGNMENT


def test_entry_points_reject_null_arguments(moe):
    L = moe.library()
    n = ctypes.c_size_t()
    assert L.moe_workspace_size(None, 4, 2, 0, ctypes.byref(n)) == moe.ERR_INVALID_ARG
    assert L.moe_forward(None, FAKE, FAKE, 4, 2, FAKE, FAKE, 1 << 20, 0, None) == moe.ERR_INVALID_ARG
    assert L.moe_quantize_act(None, 4, 256, FAKE, FAKE, FAKE, None, None) == moe.ERR_INVALID_ARG
    assert L.moe_quantize_act(FAKE, 4, 100, FAKE, FAKE, FAKE, None, None) == moe.ERR_INVALID_ARG
    assert L.moe_quantize_act(FAKE + 4, 4, 256, FAKE, FAKE, FAKE, None, None) == moe.ERR_ALIGNMENT
    assert L.moe_route_workspace_size(4, 8, 9, ctypes.byref(n)) == moe.ERR_INVALID_ARG   # k > E
    assert L.moe_route_workspace_size(4, 8000, 9, ctypes.byref(n)) == moe.ERR_UNSUPPORTED
    assert L.moe_route_workspace_size(100, 512, 10, ctypes.byref(n)) == moe.OK and n.value > 0
    assert L.moe_route_topk(FAKE, 4, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 16,
                            None) == moe.ERR_WORKSPACE
    assert L.moe_route_topk(FAKE, 4, 8, 40, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1 << 20,
                            None) == moe.ERR_INVALID_ARG
    assert L.moe_debug_dequant(None, 0, 0, FAKE, None) == moe.ERR_INVALID_ARG
    v = moe.WsView()
    assert L.moe_ws_views(None, FAKE, 4, 2, 0, ctypes.byref(v)) == moe.ERR_INVALID_ARG
    s = ctypes.c_int()
    assert L.moe_read_status(None, None, 0, ctypes.byref(s)) == moe.ERR_INVALID_ARG


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "expert_ffn_token_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, f)) as fh:
                    text = fh.read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "moe_oracle" not in text and "liboracle" not in text, f


def _declared_arity():
    """Parameter count of every moe_* function declared in include/moe.h."""
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(moe_[a-z_]+)\s*\(([^)]*)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(moe):
    arity = _declared_arity()
    assert set(moe.EXPORTED) <= set(arity)
    for name in moe.EXPORTED:
        fn = getattr(moe.library(), name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == arity[name], (name, len(fn.argtypes), arity[name])


def test_header_constants_match_the_binding(moe):
    # every status code, expert format and forward flag the header defines has the same value
    # in the binding
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        hdr = f.read()
    consts = {}
    for name, val in re.findall(r"#define (MOE_F_[A-Z0-9_]+) (\d+)u", hdr):
        consts[name[len("MOE_"):]] = int(val)
    for name, val in re.findall(r"\b(MOE_(?:ERR_[A-Z_]+|OK|FMT_[A-Z0-9_]+))\s*=\s*(\d+)", hdr):
        consts[name[len("MOE_"):]] = int(val)
    assert {"F_TC_I8", "F_LOOKAHEAD", "ERR_TIMEOUT", "FMT_Q6_K", "OK"} <= set(consts)
    for name, val in consts.items():
        assert getattr(moe, name) == val, name
