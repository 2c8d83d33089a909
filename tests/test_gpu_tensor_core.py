"""GPU checks of the tensor-core path for large batches, against the oracle on the same bytes.

The full-size prefill configs are covered in test_gpu_parity.py.  Here: a small layer that mixes
all three formats with a shared expert and rows whose super-block (or Q8_0 block) scale is zero,
so that the epilogue's per-row unit changes and its zero-scale branch are exercised; the
deterministic mode repeating bit for bit; and the timing-events hook."""
import numpy as np
import pytest

from expert_ffn_token_b200 import synth

from gpu_helpers import check_parity, torch_cuda

pytestmark = pytest.mark.gpu

# hidden 512 (two super-blocks), width 320 (down rows padded to 512), 24 experts, top-3 + shared,
# 150 tokens (jobs of a few dozen tokens, the shared job in 64-token slices), formats mixed
MIXED = synth.Workload("tc_mixed_small", 21, 512, 320, 24, 3, 150, True, 1, "normal", sigma=1.5,
                       mix=((synth.Q4_K, 0.34), (synth.Q5_K, 0.67), (synth.Q8_0, 1.0)),
                       note="small mixed-format layer for the tensor-core path")


@pytest.fixture(scope="module")
def torch():
    t = torch_cuda()
    from expert_ffn_token_b200 import moe  # noqa: F401  (fails loudly if the library is missing)
    return t


def _zero_some_scales(buf, lay, w, frac=0.1, seed=7):
    """Set the fp16 scale d of about `frac` of all blocks to zero (dmin kept)."""
    rng = np.random.default_rng(seed)
    n = lay.fmts.shape[0]
    for e in range(n):
        fmt = int(lay.fmts[e])
        bb = synth.BLOCK_BYTES[fmt]
        for t in range(3):
            rows = w.ffn if t < 2 else w.hidden
            width = w.hidden if t < 2 else w.ffn
            nb = synth.row_blocks(fmt, width)
            off, stride = int(lay.offs[e, t]), int(lay.strides[e, t])
            mat = buf[off: off + rows * stride].reshape(rows, stride)
            hit = rng.random((rows, nb)) < frac
            for b in range(nb):
                mat[hit[:, b], b * bb: b * bb + 2] = 0


def _layer(torch, w, flags):
    from expert_ffn_token_b200 import moe
    buf, lay = synth.host_arena(w, 0)
    _zero_some_scales(buf, lay, w)
    arena = torch.from_numpy(buf).cuda()
    L = moe.Layer(arena, w.hidden, w.ffn, w.n_experts, w.shared, synth.layout_descs(lay),
                  w.tokens, w.k, flags)
    return L, buf, lay


def _run(torch, L, x, logits, flags):
    xd = torch.from_numpy(x).cuda()
    ld = torch.from_numpy(logits).cuda()
    out = L.forward(xd, ld, flags=flags)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_mixed_formats_and_zero_scales(torch):
    from expert_ffn_token_b200 import moe
    w = MIXED
    fmts = synth.layer_formats(w, 0)
    assert len(set(int(f) for f in fmts)) == 3
    fl = moe.F_FORCE_PREFILL | moe.F_KEEP_H
    L, buf, lay = _layer(torch, w, fl)
    x, logits = synth.activations(w, 0), synth.router_logits(w, 0)
    gpu = _run(torch, L, x, logits, fl)
    assert L.status() == 0
    check_parity(L, w, 0, x, logits, gpu, fl, host=(buf, lay), name="tc: mixed formats, zero scales")
    L.close()


def test_deterministic_mode_repeats_bit_for_bit(torch):
    from expert_ffn_token_b200 import moe
    w = MIXED
    fl = moe.F_FORCE_PREFILL | moe.F_DETERMINISTIC | moe.F_KEEP_H
    L, buf, lay = _layer(torch, w, fl)
    x, logits = synth.activations(w, 0), synth.router_logits(w, 0)
    a = _run(torch, L, x, logits, fl)
    b = _run(torch, L, x, logits, fl)
    assert np.array_equal(a, b)
    check_parity(L, w, 0, x, logits, a, fl, host=(buf, lay), name="tc: deterministic mode")
    L.close()


def test_timing_events_bracket_the_grouped_gemm(torch):
    from expert_ffn_token_b200 import moe
    w = MIXED
    L, _, _ = _layer(torch, w, moe.F_FORCE_PREFILL)
    x, logits = synth.activations(w, 0), synth.router_logits(w, 0)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in ev:
        e.record()                      # creates the handles
    with pytest.raises(moe.MoeError):
        moe.set_timing_events(L.handle, ev[0].cuda_event, None, None)
    moe.set_timing_events(L.handle, *[e.cuda_event for e in ev])
    _run(torch, L, x, logits, moe.F_FORCE_PREFILL)
    assert ev[0].elapsed_time(ev[1]) > 0.0 and ev[1].elapsed_time(ev[2]) > 0.0
    moe.set_timing_events(L.handle)
    _run(torch, L, x, logits, moe.F_FORCE_PREFILL)
    assert L.status() == 0
    L.close()
