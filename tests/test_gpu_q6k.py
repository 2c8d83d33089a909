"""GPU parity of Q6_K experts (the format real Q4_K_M model files mix into their FFN tensors).

Bit-exact: the decoded weights (moe_debug_dequant against O1).  Layers of mixed Q4_K / Q6_K /
Q8_0 / Q5_1 experts run on every path that takes Q6_K -- the fused decode kernel, the CUDA-core
grouped kernels (atomic and deterministic combine) and the dequant-GEMV kernels -- and are
checked like every other layer (gpu_helpers.check_layer).  The tensor-core path has no exact
operand form for Q6_K: such an arena has no tensor-core plan and MOE_F_FORCE_PREFILL returns
MOE_ERR_UNSUPPORTED.  The device fill draws no Q6_K blocks, so these arenas are drawn on the host
by the same seeded generator and copied to the device."""
import numpy as np
import pytest

import oracle
from expert_ffn_token_b200 import synth

from gpu_helpers import check_layer, torch_cuda

pytestmark = pytest.mark.gpu

# hidden 2560, 32 experts + shared, top-8, width 640 (the down rows' last super-block is half
# used), per expert 25% Q4_K / 50% Q6_K / 15% Q8_0 / 10% Q5_1
W6 = synth.Workload("q6k_mix", 16, 2560, 640, 32, 8, 40, True, 1, "normal", sigma=1.0,
                    mix=((synth.Q4_K, 0.25), (synth.Q6_K, 0.75), (synth.Q8_0, 0.90),
                         (synth.Q5_1, 1.0)),
                    note="mixed Q4_K/Q6_K/Q8_0/Q5_1 layer: hidden 2560, 32 experts + shared, "
                         "top-8, width 640")


@pytest.fixture(scope="module")
def torch():
    t = torch_cuda()
    from expert_ffn_token_b200 import moe  # noqa: F401  (fails loudly if the library is missing)
    return t


@pytest.fixture(scope="module")
def layer(torch):
    from expert_ffn_token_b200 import moe
    buf, lay = synth.host_arena(W6, 0)
    assert (lay.fmts == synth.Q6_K).sum() >= 8
    arena = torch.from_numpy(buf).cuda()
    L = moe.Layer(arena, W6.hidden, W6.ffn, W6.n_experts, W6.shared, synth.layout_descs(lay),
                  40, W6.k, moe.F_KEEP_H | moe.F_DETERMINISTIC)
    yield L, arena, buf, lay
    L.close()


def test_q6k_dequant_bit_exact(torch, layer):
    from expert_ffn_token_b200 import moe
    L, _, buf, lay = layer
    q6 = [int(e) for e in np.nonzero(lay.fmts == synth.Q6_K)[0][:3]]
    for e in q6:
        for t in range(3):
            rows, width = synth.tensor_shape(W6, t)
            nb = -(-width // 256)
            out = torch.empty((rows, nb * 256), dtype=torch.float32, device="cuda")
            moe.debug_dequant(L.handle, e, t, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
            _, ref32 = oracle.dequant_matrix(synth.Q6_K, buf[lay.offs[e, t]:], rows,
                                             int(lay.strides[e, t]), nb)
            assert np.array_equal(out.cpu().numpy().view(np.uint32), ref32.view(np.uint32)), (e, t)


@pytest.mark.parametrize("T,flags", [(3, 0),        # fused decode kernel
                                     (1, 0),
                                     (40, 0),       # CUDA-core grouped kernels, atomic combine
                                     (40, 1),       # deterministic combine
                                     (40, 2),       # dequant-GEMV kernels at T = 40
                                     (9, 2)])
def test_q6k_layer_paths(torch, layer, T, flags):
    L = layer[0]
    w = synth.with_tokens(W6, T)
    x = synth.activations(w, 0)
    logits = synth.router_logits(w, 0)
    ids, _, _ = oracle.topk(logits, w.k)
    fm = layer[3].fmts
    assert (fm[ids.ravel()] == synth.Q6_K).any()        # the batch reaches Q6_K experts
    check_layer(torch, w, 0, x, logits, flags=flags, L=L, name=f"q6k_mix T={T} flags={flags}")


def test_q6k_arena_has_no_tensor_core_plan(torch, layer):
    from expert_ffn_token_b200 import moe
    L = layer[0]
    x = torch.zeros((40, W6.hidden), dtype=torch.float32, device="cuda")
    lg = torch.zeros((40, W6.n_experts), dtype=torch.float32, device="cuda")
    out = torch.empty_like(x)
    before = moe.kernels_enqueued()
    st = moe.forward_status(L.handle, x.data_ptr(), lg.data_ptr(), 40, W6.k, out.data_ptr(),
                            L.ws.data_ptr(), L.ws_bytes, moe.F_FORCE_PREFILL,
                            torch.cuda.current_stream().cuda_stream)
    assert st == moe.ERR_UNSUPPORTED
    assert moe.kernels_enqueued() == before
