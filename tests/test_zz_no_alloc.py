"""moe_forward_noalloc, the allocation-free entry point, against moe_forward and the oracle.

Some callers cannot allocate device memory at all: code running while a CUDA graph is being
captured (an allocation there breaks or serialises the capture), inference loops with a fixed
memory budget that must not reach an allocator in steady state, and plug-ins whose host
framework owns every allocation.  moe_forward_noalloc serves them: it runs the same layer on a
scratch array compiled into the library instead of a caller workspace.  This file checks,
through the C ABI, that two calls in a row give outputs bit for bit equal to moe_forward on a
caller workspace (the same deterministic decode kernel), that those outputs match the oracle,
that the status reads clean, and that shapes too large for the scratch are refused.  It is
named to be collected last.
"""
import numpy as np
import pytest

from expert_ffn_token_b200 import synth

from gpu_helpers import REL_TOL, oracle_layer, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T", [("decode", 1), ("mtp_verify", 3), ("mtp_verify", 16)])
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
    x_np, lg_np = synth.activations(w, 0), synth.router_logits(w, 0)
    x = torch.from_numpy(x_np).cuda()
    logits = torch.from_numpy(lg_np).cuda()
    ref = layer.forward(x, logits).cpu().numpy()
    assert layer.status() == 0
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        moe.forward_noalloc(layer.handle, x.data_ptr(), logits.data_ptr(), T, w.k, out.data_ptr(),
                            status.data_ptr(), stream)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.array_equal(got, ref)
        assert int(status.item()) == 0
    oref, _, _ = oracle_layer(w, 0, x_np, lg_np)
    assert rel_err(got, oref).max() <= REL_TOL
    layer.close()


def test_noalloc_rejects_shapes_beyond_the_scratch():
    import torch
    from expert_ffn_token_b200 import moe
    w = synth.WORKLOADS["tiny"]
    lay = synth.arena_layout(w, synth.layer_formats(w, 0))
    arena = torch.empty(lay.nbytes, dtype=torch.uint8, device="cuda")
    synth.device_fill_layer(w, 0, arena.data_ptr(), torch.cuda.current_stream().cuda_stream)
    layer = moe.Layer(arena, w.hidden, w.ffn, w.n_experts, w.shared, synth.layout_descs(lay), 4, w.k)
    x = torch.zeros((17, w.hidden), device="cuda")
    lg = torch.zeros((17, w.n_experts), device="cuda")
    with pytest.raises(moe.MoeError) as e:   # more tokens than the decode kernel takes
        moe.forward_noalloc(layer.handle, x.data_ptr(), lg.data_ptr(), 17, w.k, x.data_ptr())
    assert e.value.code == moe.ERR_INVALID_ARG
    layer.close()
    # a layer whose 16-token workspace exceeds the 4 MiB scratch: 4096 experts, top-32,
    # hidden 4096, width 4096 (descriptors over a small arena view are never read: refused first)
    row = synth.row_stride(synth.Q8_0, 4096)
    nbytes = 3 * 4096 * row
    arena2 = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    descs = [(synth.Q8_0, (0, 4096 * row, 2 * 4096 * row), (row, row, row))] * (4096 + 1)
    h = moe.arena_create(arena2.data_ptr(), nbytes, 4096, 4096, 4096, 4096, descs)
    ws = moe.workspace_size(h, 16, 32, 0)
    assert ws > 4 << 20
    x2 = torch.zeros((16, 4096), device="cuda")
    lg2 = torch.zeros((16, 4096), device="cuda")
    assert moe.forward_noalloc_status(h, x2.data_ptr(), lg2.data_ptr(), 16, 32,
                                      x2.data_ptr()) == moe.ERR_UNSUPPORTED
    moe.arena_destroy(h)
