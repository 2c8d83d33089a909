"""Failure paths on the GPU: a bounded device wait that runs out.

The engine on the pages guards its decode loop with a stall watchdog that gives up after a
period without progress ("Strata - the details", "Troubleshooting").  Here every wait inside the
kernels is bounded by the arena's wait limit (moe_set_wait_limit).  With a limit far below what
the kernels' own hand-offs take (the grid-wide wait of the decode kernel, the mbarrier rings of
the tensor-core kernels), some wait runs out on purpose: the call must report MOE_ERR_TIMEOUT in
the status word, leave finite outputs, land the copies it had in flight before its CTAs leave,
and the next call with the default limit must be clean and correct.  No fault, trap or hang is
involved: every wait returns."""
import numpy as np
import pytest

from expert_ffn_token_b200 import synth

from gpu_helpers import REL_TOL, device_layer, inputs, oracle_layer, rel_err, run_forward, torch_cuda

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
SHORT_NS = 200            # far below any hand-off inside the kernels
DEFAULT_NS = 2_000_000_000


@pytest.fixture(scope="module")
def torch():
    t = torch_cuda()
    from expert_ffn_token_b200 import moe  # noqa: F401  (fails loudly if the library is missing)
    return t


def _timeout_then_recover(torch, w, layer, flags):
    from expert_ffn_token_b200 import moe
    T = w.tokens
    L, _, _ = device_layer(w, layer, max_tokens=T, flags=flags)
    x, logits = inputs(w, layer)
    moe.set_wait_limit(L.handle, SHORT_NS)
    xd = torch.from_numpy(x).cuda()
    ld = torch.from_numpy(logits).cuda()
    out = torch.zeros_like(xd)
    L.forward(xd, ld, out=out, flags=flags)
    torch.cuda.synchronize()
    assert L.status() == moe.ERR_TIMEOUT
    assert torch.isfinite(out).all()
    # the kernels left their counters at zero for the next call
    v = L.views(T, flags)
    off = v["counters"] - L.ws.data_ptr()
    assert (L.ws[off:off + 16] == 0).all()
    moe.set_wait_limit(L.handle, DEFAULT_NS)
    with pytest.raises(moe.MoeError):
        moe.set_wait_limit(L.handle, 0)
    gpu = run_forward(L, x, logits, flags=flags)
    assert L.status() == 0
    ref, _, _ = oracle_layer(w, layer, x, logits)
    assert rel_err(gpu, ref).max() <= REL_TOL
    L.close()


def test_decode_wait_times_out_and_next_call_is_clean(torch):
    # the fused decode kernel: the grid-wide wait (and the stage ring) give up
    _timeout_then_recover(torch, synth.with_tokens(W["decode"], 1, layers=1), 0, 0)


def test_tensor_core_wait_times_out_and_next_call_is_clean(torch):
    from expert_ffn_token_b200 import moe
    # the grouped tensor-core kernels: the mbarrier rings give up
    _timeout_then_recover(torch, W["tiny"], 0, moe.F_FORCE_PREFILL)


def test_tensor_core_i8_wait_times_out_and_next_call_is_clean(torch):
    from expert_ffn_token_b200 import moe
    # gate/up on kind::i8 products: its rings (operands, activations, row and column constants,
    # accumulator slots) give up the same way
    _timeout_then_recover(torch, W["tiny"], 0, moe.F_FORCE_PREFILL | moe.F_TC_I8)
