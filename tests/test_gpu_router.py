"""GPU checks of the router and the shared-expert gate against the oracle (O10, O11).

The GPU sums in fp32 (a fixed order per logit), the oracle in fp64: logits agree within the
fp32 summation bound, 1e-5 of sum |x[h] * Wr[e][h]|, far above the error of at most ~85
sequential fp32 additions per lane.  The top-k decision is checked on the GPU's own logits:
routing them on the GPU and in the oracle must choose the same experts in the same order."""
import numpy as np
import pytest

import oracle

from gpu_helpers import torch_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    t = torch_cuda()
    from expert_ffn_token_b200 import moe  # noqa: F401  (fails loudly if the library is missing)
    return t


def _stream(torch):
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("T,H,E,k", [(1, 2048, 256, 8), (3, 2560, 512, 10), (37, 256, 20, 4),
                                     (64, 2560, 512, 10)])
def test_router_logits_and_topk_against_oracle(torch, T, H, E, k):
    from expert_ffn_token_b200 import moe
    rng = np.random.default_rng(T * 131 + E)
    x = rng.standard_normal((T, H)).astype(np.float32)
    Wr = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    xd, wd = torch.from_numpy(x).cuda(), torch.from_numpy(Wr).cuda()
    ld = torch.empty((T, E), dtype=torch.float32, device="cuda")
    moe.router_logits(xd.data_ptr(), T, H, wd.data_ptr(), E, ld.data_ptr(), _stream(torch))
    gpu = ld.cpu().numpy()
    _, l64 = oracle.router(x, Wr)
    bound = 1e-5 * (np.abs(x).astype(np.float64) @ np.abs(Wr).astype(np.float64).T)
    assert (np.abs(gpu - l64) <= bound).all()
    # the same call repeats bit for bit
    ld2 = torch.empty_like(ld)
    moe.router_logits(xd.data_ptr(), T, H, wd.data_ptr(), E, ld2.data_ptr(), _stream(torch))
    assert torch.equal(ld, ld2)
    # routing the GPU's logits on the GPU equals the oracle's top-k of those logits
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    nws = moe.route_workspace_size(T, E, k)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    moe.route_topk(ld.data_ptr(), T, E, k, ids.data_ptr(), w.data_ptr(), counts.data_ptr(),
                   offs.data_ptr(), perm.data_ptr(), None, None, ws.data_ptr(), nws,
                   _stream(torch))
    rid, rw, _ = oracle.topk(gpu, k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.abs(w.cpu().numpy() - rw).max() <= 1e-6


@pytest.mark.parametrize("T,H", [(1, 2048), (3, 2560), (41, 256)])
def test_shared_gate_against_oracle(torch, T, H):
    from expert_ffn_token_b200 import moe
    rng = np.random.default_rng(T + H)
    x = rng.standard_normal((T, H)).astype(np.float32)
    wg = (rng.standard_normal(H) * 0.05).astype(np.float32)
    xd, wgd = torch.from_numpy(x).cuda(), torch.from_numpy(wg).cuda()   # kept alive
    gd = torch.empty(T, dtype=torch.float32, device="cuda")
    moe.shared_gate(xd.data_ptr(), T, H, wgd.data_ptr(), gd.data_ptr(), _stream(torch))
    g = oracle.shared_gate(x, wg)
    # sigmoid' <= 1/4 times the fp32 sum error, plus a few ulp of the fp32 sigmoid
    bound = 0.25e-5 * (np.abs(x).astype(np.float64) @ np.abs(wg).astype(np.float64)) + 1e-6
    assert (np.abs(gd.cpu().numpy() - g) <= bound).all()
