"""moe_forward_noalloc, the allocation-free entry point, against moe_forward.

Callers that may not allocate device memory (graph capture, fixed-budget inference loops,
plug-ins inside a framework that owns allocation) use moe_forward_noalloc, which runs the same
layer on a scratch array built into the library.  This file checks, through the C ABI, that two
calls in a row give the same outputs as moe_forward on a caller workspace, within the parity
tolerance, and report a clean status.  It is named to be collected last.
"""
import numpy as np
import pytest

from expert_ffn_token_b200 import synth

pytestmark = pytest.mark.gpu

REL_TOL = 2e-3


def _rel(a, b):
    return (np.abs(a.astype(np.float64) - b).max(axis=1) / np.abs(b).max(axis=1)).max()


@pytest.mark.parametrize("name,T", [("decode", 1), ("mtp_verify", 3)])
def test_noalloc_matches_workspace_forward_twice(name, T):
    import torch
    assert torch.cuda.is_available()
    from expert_ffn_token_b200 import moe
    w = synth.with_tokens(synth.WORKLOADS[name], T, layers=1)
    lay = synth.arena_layout(w, synth.layer_formats(w, 0))
    arena = torch.empty(lay.nbytes, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    synth.device_fill_layer(w, 0, arena.data_ptr(), stream)
    layer = moe.Layer(arena, w.hidden, w.ffn, w.n_experts, w.shared, synth.layout_descs(lay), T, w.k)
    x = torch.from_numpy(synth.activations(w, 0)).cuda()
    logits = torch.from_numpy(synth.router_logits(w, 0)).cuda()
    ref = layer.forward(x, logits).cpu().numpy().astype(np.float64)
    assert layer.status() == 0
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        moe.forward_noalloc(layer.handle, x.data_ptr(), logits.data_ptr(), T, w.k, out.data_ptr(),
                            status.data_ptr(), stream)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        assert _rel(got, ref) <= REL_TOL
        assert int(status.item()) == 0
    layer.close()


def test_noalloc_rejects_large_batches():
    import torch
    from expert_ffn_token_b200 import moe
    w = synth.WORKLOADS["tiny"]
    lay = synth.arena_layout(w, synth.layer_formats(w, 0))
    arena = torch.empty(lay.nbytes, dtype=torch.uint8, device="cuda")
    synth.device_fill_layer(w, 0, arena.data_ptr(), torch.cuda.current_stream().cuda_stream)
    layer = moe.Layer(arena, w.hidden, w.ffn, w.n_experts, w.shared, synth.layout_descs(lay), 4, w.k)
    x = torch.zeros((17, w.hidden), device="cuda")
    lg = torch.zeros((17, w.n_experts), device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.forward_noalloc(layer.handle, x.data_ptr(), lg.data_ptr(), 17, w.k, x.data_ptr())
    assert e.value.code == moe.ERR_INVALID_ARG
    layer.close()
