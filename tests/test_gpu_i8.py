"""The tensor-core gate/up phase on 8-bit integer products (MOE_F_TC_I8, k_gateup_i8) against the
oracle: the same layer checks as the exact kind::f16 kernel (intermediates bit for bit, Q8_1 of
the GPU's own h bit for bit, h and the outputs within the parity bars), on every format, on
ragged batches whose token slices leave partial tiles, and on the full-size prefill layers."""
import numpy as np
import pytest

import oracle
from expert_ffn_token_b200 import synth
from gpu_helpers import check_layer, device_layer, inputs, run_forward, torch_cuda

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
I8 = 32            # MOE_F_TC_I8
PREFILL = 4        # MOE_F_FORCE_PREFILL
DET = 1            # MOE_F_DETERMINISTIC

@pytest.fixture(scope="module")
def torch():
    return torch_cuda()


FOUR = synth.Workload("four_formats_i8", 24, 512, 320, 32, 4, 150, True, 1, "normal", sigma=1.5,
                      mix=((synth.Q4_K, 0.25), (synth.Q5_K, 0.5), (synth.Q8_0, 0.75),
                           (synth.Q5_1, 1.0)),
                      note="Q4_K, Q5_K, Q8_0 and Q5_1 experts in one layer")


@pytest.mark.parametrize("flags", [PREFILL | I8, PREFILL | DET | I8])
def test_i8_tiny(torch, flags):
    w = W["tiny"]
    x, logits = inputs(w, 0)
    check_layer(torch, w, 0, x, logits, flags=flags, name="i8 tiny")


@pytest.mark.parametrize("T", [17, 65, 100, 300])
def test_i8_ragged_batches(torch, T):
    # 3 tokens x top-10 of 512 experts + shared, reshaped to T tokens: most experts get 1-3
    # tokens (one 16-column MMA), the shared expert T (several 64-token slices and a tail)
    w = synth.with_tokens(W["mtp_verify"], T, layers=1)
    x, logits = inputs(w, 5)
    check_layer(torch, w, 5, x, logits, flags=I8, name=f"i8 ragged {T}")


@pytest.mark.parametrize("flags", [PREFILL | I8, PREFILL | DET | I8])
def test_i8_four_formats(torch, flags):
    w = FOUR
    x, logits = inputs(w, 0)
    check_layer(torch, w, 0, x, logits, flags=flags, name="i8 four formats")


def test_i8_repeats_and_agrees_with_f16(torch):
    # deterministic mode repeats bit for bit; both gate/up kernels pass the same oracle checks
    w = synth.with_tokens(W["mtp_verify"], 40, layers=1)
    x, logits = inputs(w, 3)
    fl = PREFILL | DET | 8
    L, _, _ = device_layer(w, 3, max_tokens=40, flags=fl)
    a = check_layer(torch, w, 3, x, logits, flags=PREFILL | DET | I8, L=L, name="i8")
    b = run_forward(L, x, logits, flags=fl | I8)
    assert np.array_equal(a, b)
    check_layer(torch, w, 3, x, logits, flags=PREFILL | DET, L=L, name="f16")
    L.close()


def _sample_tokens(T, ids, n, seed=0):
    """First, last, the last token of every expert that has any (its tail tile), random up to n."""
    rng = np.random.default_rng(seed)
    pick = {0, T - 1}
    for e in np.unique(ids):
        pick.add(int(np.nonzero((ids == e).any(axis=1))[0][-1]))
    rest = [t for t in rng.permutation(T) if int(t) not in pick]
    pick |= set(int(t) for t in rest[:max(0, n - len(pick))])
    return np.array(sorted(pick))


@pytest.mark.parametrize("name", ["prefill", "mixed_prefill"])
def test_i8_prefill_full_size_sampled(torch, name):
    w = W[name]
    x, logits = inputs(w, 0)
    ids, _, _ = oracle.topk(logits, w.k)
    check_layer(torch, w, 0, x, logits, flags=I8, tokens=_sample_tokens(w.tokens, ids, 512),
                name=f"i8 {name}")
