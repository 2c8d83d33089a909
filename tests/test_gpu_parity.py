"""GPU parity: the CUDA path (through the C ABI) against the oracle, on the same seeded inputs.

Bit-exact: dequantized weights, Q8_1 blocks, top-k ids, counts, offsets, permutation, and the
quantizer applied to the GPU's own h.  Tolerance: routing weights 1e-6; layer outputs
max|gpu - ref| / max|ref| <= 2e-3 per token (fp32 accumulation against fp64)."""
import numpy as np
import pytest

import oracle
from expert_ffn_token_b200 import synth

from gpu_helpers import W_TOL, check_layer, device_layer, inputs, run_forward, torch_cuda

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


@pytest.fixture(scope="module")
def torch():
    t = torch_cuda()
    from expert_ffn_token_b200 import moe  # noqa: F401  (fails loudly if the library is missing)
    return t


def _stream(torch):
    return torch.cuda.current_stream().cuda_stream


# ------------------------------------------------------------------ generator cross-check


def test_device_fill_matches_host_generator(torch):
    for name, layer, experts in (("tiny", 0, None), ("mixed_prefill", 0, [0, 7, 100, 511, 512]),
                                 ("decode", 47, [3, 255])):
        w = W[name]
        fmts = synth.layer_formats(w, layer)
        lay = synth.arena_layout(w, fmts)
        dev = torch.empty(lay.nbytes, dtype=torch.uint8, device="cuda")
        synth.device_fill_layer(w, layer, dev.data_ptr(), _stream(torch))
        host = dev.cpu().numpy()
        for e in (range(lay.n) if experts is None else experts):
            for t in range(3):
                ref = synth.tensor_bytes(w, layer, e, t, int(fmts[e]))
                got = host[lay.offs[e, t]:lay.offs[e, t] + ref.size]
                assert np.array_equal(got, ref), (name, e, t)
    # the mixed layer really mixes formats
    assert set(synth.layer_formats(W["mixed_prefill"], 0)) == {0, 1, 2}


# ------------------------------------------------------------------ O1 / a-side decoders


@pytest.mark.parametrize("name,layer,experts", [("tiny", 0, [0, 5]),
                                                ("mixed_prefill", 0, None),
                                                ("mtp_verify", 0, [512])])
def test_dequant_bit_exact(torch, name, layer, experts):
    from expert_ffn_token_b200 import moe
    w = W[name]
    L, arena, lay = device_layer(w, layer, max_tokens=1)
    if experts is None:   # one expert of each format
        experts = [int(np.nonzero(lay.fmts == f)[0][0]) for f in (0, 1, 2)]
    host = arena.cpu().numpy()
    for e in experts:
        fmt = int(lay.fmts[e])
        bw = synth.BLOCK_WEIGHTS[fmt]
        for t in range(3):
            rows, width = synth.tensor_shape(w, t)
            nb = -(-width // bw)
            out = torch.empty((rows, nb * bw), dtype=torch.float32, device="cuda")
            moe.debug_dequant(L.handle, e, t, out.data_ptr(), _stream(torch))
            _, ref32 = oracle.dequant_matrix(fmt, host[lay.offs[e, t]:], rows,
                                             int(lay.strides[e, t]), nb)
            got = out.cpu().numpy()
            assert np.array_equal(got.view(np.uint32), ref32.view(np.uint32)), (e, t)
    L.close()


# ------------------------------------------------------------------ a1 Q8_1


def test_quantize_bit_exact(torch):
    from expert_ffn_token_b200 import moe
    rng = np.random.default_rng(1)
    T, H = 37, 2560
    x = (rng.standard_normal((T, H)) * 10.0 ** rng.uniform(-4, 4, (T, 1))).astype(np.float32)
    x[3, :64] = 0.0                                    # all-zero blocks
    x[4, 5] = 1e30                                     # a huge value
    x[5, 40] = np.float32(2.0 ** -140)                 # subnormal amax
    x[6, :32] = [127, -63.5, 0.5] + [0] * 29           # worked example E2
    x[9, 70] = np.nan                                  # non-finite block 2 of row 9
    xd = torch.from_numpy(x).cuda()
    q = torch.empty((T, H), dtype=torch.int8, device="cuda")
    d = torch.empty((T, H // 32), dtype=torch.int16, device="cuda")
    s = torch.empty_like(d)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.quantize_act(xd.data_ptr(), T, H, q.data_ptr(), d.data_ptr(), s.data_ptr(), st.data_ptr(),
                     _stream(torch))
    rq, rd, rs, bad = oracle.quantize_q8_1(x)
    assert bad == 1
    assert np.array_equal(q.cpu().numpy().ravel(), rq)
    assert np.array_equal(d.cpu().numpy().view(np.uint16).ravel(), rd)
    assert np.array_equal(s.cpu().numpy().view(np.uint16).ravel(), rs)
    assert moe.read_status(st.data_ptr(), _stream(torch)) == moe.ERR_NONFINITE


# ------------------------------------------------------------------ a2 + a3 routing


@pytest.mark.parametrize("T,E,k,ties", [(1, 256, 8, False), (3, 512, 10, False), (4, 16, 2, True),
                                        (100, 64, 6, True), (4096, 512, 10, False),
                                        (8192, 512, 10, False), (65, 8, 8, True),
                                        (33, 4096, 32, False)])
def test_route_bit_exact(torch, T, E, k, ties):
    from expert_ffn_token_b200 import moe
    rng = np.random.default_rng(T * 7 + E)
    if ties:
        L = rng.integers(-3, 3, size=(T, E)).astype(np.float32)
    else:
        L = (2.0 * rng.standard_normal((T, E))).astype(np.float32)
    lg = torch.from_numpy(L).cuda()
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, k), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    nws = moe.route_workspace_size(T, E, k)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    moe.route_topk(lg.data_ptr(), T, E, k, ids.data_ptr(), wt.data_ptr(), counts.data_ptr(),
                   offs.data_ptr(), perm.data_ptr(), inv.data_ptr(), None, ws.data_ptr(), nws,
                   _stream(torch))
    rid, rw, _ = oracle.topk(L, k)
    rc, ro, rp, ri = oracle.group(rid, E)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.abs(wt.cpu().numpy() - rw).max() <= W_TOL
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offs.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)


# ------------------------------------------------------------------ a1-a7 the layer




@pytest.mark.parametrize("flags", [0, 2, 4, 5])     # auto, force decode, prefill, prefill+det
def test_layer_tiny_all_paths(torch, flags):
    w = W["tiny"]
    x, logits = inputs(w, 0)
    check_layer(torch, w, 0, x, logits, flags=flags)


@pytest.mark.parametrize("layer", [0, 23, 47])
def test_layer_decode_full_size(torch, layer):
    w = W["decode"]
    x, logits = inputs(w, layer)
    check_layer(torch, w, layer, x, logits)


@pytest.mark.parametrize("layer", [0, 47])
def test_layer_mtp_verify_full_size(torch, layer):
    w = W["mtp_verify"]
    x, logits = inputs(w, layer)
    check_layer(torch, w, layer, x, logits)


def _sample_tokens(T, ids, n=24, seed=0, every_expert=False):
    """First and last tokens, the hottest expert's first and last tokens, with every_expert the
    last token routed to each expert that has any (its tail tile on the grouped paths), and
    random tokens up to n."""
    rng = np.random.default_rng(seed)
    hot = np.bincount(ids.ravel()).argmax()
    hot_tokens = np.nonzero((ids == hot).any(axis=1))[0]
    pick = {0, T - 1, int(hot_tokens[0]), int(hot_tokens[-1])}
    if every_expert:
        for e in np.unique(ids):
            pick.add(int(np.nonzero((ids == e).any(axis=1))[0][-1]))
    rest = [t for t in rng.permutation(T) if int(t) not in pick]
    pick |= set(int(t) for t in rest[:max(0, n - len(pick))])
    return np.array(sorted(pick))


@pytest.mark.parametrize("name", ["prefill", "mixed_prefill"])
def test_layer_prefill_full_size_sampled(torch, name):
    w = W[name]
    x, logits = inputs(w, 0)
    ids, _, _ = oracle.topk(logits, w.k)
    counts = np.bincount(ids.ravel(), minlength=w.n_experts)
    if name == "mixed_prefill":
        # Zipf(1.3) popularity sampled k at a time without replacement (Gumbel top-k): a few
        # experts take > 1000 tokens, a long tail takes only a handful
        assert (counts > 1000).sum() >= 3 and (counts < 8).sum() >= 5 and (counts < 16).sum() >= 50
    # every token's integer outputs (views); the layer outputs of the last token of every expert
    # (each expert's tail tile) and random tokens, 512 or more in all
    check_layer(torch, w, 0, x, logits,
                tokens=_sample_tokens(w.tokens, ids, n=512, every_expert=True))


@pytest.mark.parametrize("T", [1, 2, 17, 65, 100, 300])
def test_layer_ragged_batches(torch, T):
    w = synth.with_tokens(W["mtp_verify"], T, layers=1)
    x, logits = inputs(w, 5)
    tokens = None
    if T > 64:
        ids, _, _ = oracle.topk(logits, w.k)
        tokens = _sample_tokens(T, ids, n=20, seed=T)
    check_layer(torch, w, 5, x, logits, tokens=tokens)


def test_decode_and_prefill_paths_agree(torch):
    # both paths against the oracle on the same 12 tokens; each path repeats bit for bit
    from expert_ffn_token_b200 import moe
    w = synth.with_tokens(W["mtp_verify"], 12, layers=1)
    x, logits = inputs(w, 2)
    fl = moe.F_FORCE_PREFILL | moe.F_DETERMINISTIC | moe.F_KEEP_H
    L, _, _ = device_layer(w, 2, max_tokens=12, flags=fl)
    a = check_layer(torch, w, 2, x, logits, flags=moe.F_FORCE_DECODE, L=L, name="paths: decode")
    b = check_layer(torch, w, 2, x, logits, flags=moe.F_FORCE_PREFILL | moe.F_DETERMINISTIC,
                     L=L, name="paths: tensor cores, deterministic")
    c = run_forward(L, x, logits, flags=fl)
    assert np.array_equal(b, c)                       # deterministic mode repeats bit for bit
    a2 = run_forward(L, x, logits, flags=moe.F_FORCE_DECODE | moe.F_KEEP_H)
    assert np.array_equal(a, a2)                      # decode path is deterministic
    L.close()


def test_edge_k1_and_k_equals_e(torch):
    for k, E in ((1, 16), (4, 4)):
        w = synth.Workload("edge", 60 + k, 256, 256, E, k, 5, True, 1, "normal")
        x, logits = inputs(w, 0)
        check_layer(torch, w, 0, x, logits)


def test_edge_one_expert_takes_every_token(torch):
    w = synth.with_tokens(W["tiny"], 300, layers=1)
    x, logits = inputs(w, 0)
    logits[:, 3] += 100.0
    check_layer(torch, w, 0, x, logits)


def test_nonfinite_activation_sets_status(torch):
    from expert_ffn_token_b200 import moe
    w = W["tiny"]
    x, logits = inputs(w, 0)
    x[1, 17] = np.inf
    L, _, _ = device_layer(w, 0, max_tokens=4)
    out = run_forward(L, x, logits)
    assert np.isfinite(out).all()
    assert L.status() == moe.ERR_NONFINITE
    assert L.status() == 0                             # read-and-clear
    L.close()


def test_host_errors_enqueue_nothing(torch):
    from expert_ffn_token_b200 import moe
    w = W["tiny"]
    L, _, _ = device_layer(w, 0, max_tokens=4)
    x = torch.zeros((4, 256), device="cuda")
    lg = torch.zeros((4, 16), device="cuda")
    out = torch.full((4, 256), 7.0, device="cuda")
    assert moe.forward_status(L.handle, x.data_ptr(), lg.data_ptr(), 5, 2, out.data_ptr(),
                              L.ws.data_ptr(), 1024, 0, None) == moe.ERR_WORKSPACE
    assert moe.forward_status(L.handle, x.data_ptr(), lg.data_ptr(), 4, 17, out.data_ptr(),
                              L.ws.data_ptr(), L.ws_bytes, 0, None) == moe.ERR_INVALID_ARG
    assert moe.forward_status(L.handle, x.data_ptr() + 4, lg.data_ptr(), 4, 2, out.data_ptr(),
                              L.ws.data_ptr(), L.ws_bytes, 0, None) == moe.ERR_ALIGNMENT
    # the tensor-core path needs a workspace sized for it: no silent switch to other kernels
    assert moe.forward_status(L.handle, x.data_ptr(), lg.data_ptr(), 4, 2, out.data_ptr(),
                              L.ws.data_ptr(), L.ws_bytes, moe.F_FORCE_PREFILL,
                              None) == moe.ERR_WORKSPACE
    assert moe.forward_status(L.handle, x.data_ptr(), lg.data_ptr(), 4, 2, out.data_ptr(),
                              L.ws.data_ptr(), L.ws_bytes,
                              moe.F_FORCE_PREFILL | moe.F_FORCE_DECODE, None) == moe.ERR_INVALID_ARG
    # the allocation-free entry point makes the same checks before it enqueues anything
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    n0 = moe.kernels_enqueued()
    for args, code in (((x.data_ptr() + 4, lg.data_ptr(), 4, 2, out.data_ptr()), moe.ERR_ALIGNMENT),
                       ((x.data_ptr(), lg.data_ptr(), 4, 17, out.data_ptr()), moe.ERR_INVALID_ARG),
                       ((x.data_ptr(), lg.data_ptr() + 2, 4, 2, out.data_ptr()), moe.ERR_ALIGNMENT),
                       ((x.data_ptr(), lg.data_ptr(), 4, 2, out.data_ptr() + 8), moe.ERR_ALIGNMENT)):
        assert moe.forward_noalloc_status(L.handle, *args, st.data_ptr(), None) == code
    assert moe.kernels_enqueued() == n0
    torch.cuda.synchronize()
    assert (out == 7.0).all()
    L.close()


def test_decode_large_expert_count_uses_grouped_kernels(torch):
    # 2048 experts exceed the fused decode kernel's plan: the three-kernel decode path runs
    w = synth.Workload("wideE", 70, 256, 256, 2048, 4, 3, True, 1, "normal", sigma=2.0)
    x, logits = inputs(w, 0)
    check_layer(torch, w, 0, x, logits)


# ------------------------------------------------------------------ Q5_1 experts

# hidden 512, width 320 (down rows padded to 512 on the tensor-core path), 32 experts, top-4
# + shared: every expert Q5_1, or the four formats mixed a quarter each
Q51 = synth.Workload("q5_1_layer", 23, 512, 320, 32, 4, 40, True, 1, "normal", sigma=1.5,
                     mix=((synth.Q5_1, 1.0),), note="Q5_1 experts")
FOUR = synth.Workload("four_formats", 24, 512, 320, 32, 4, 150, True, 1, "normal", sigma=1.5,
                      mix=((synth.Q4_K, 0.25), (synth.Q5_K, 0.5), (synth.Q8_0, 0.75),
                           (synth.Q5_1, 1.0)),
                      note="Q4_K, Q5_K, Q8_0 and Q5_1 experts in one layer")


def test_q5_1_device_fill_and_dequant_bit_exact(torch):
    from expert_ffn_token_b200 import moe
    w = FOUR
    fmts = synth.layer_formats(w, 0)
    assert set(int(f) for f in fmts) == {0, 1, 2, 3}
    L, arena, lay = device_layer(w, 0, max_tokens=1)
    host = arena.cpu().numpy()
    for e in range(lay.n):
        for t in range(3):
            ref = synth.tensor_bytes(w, 0, e, t, int(fmts[e]))
            assert np.array_equal(host[lay.offs[e, t]:lay.offs[e, t] + ref.size], ref), (e, t)
    for e in [int(np.nonzero(fmts == 3)[0][i]) for i in (0, 1)]:
        for t in range(3):
            rows, width = synth.tensor_shape(w, t)
            nb = -(-width // 32)
            out = torch.empty((rows, nb * 32), dtype=torch.float32, device="cuda")
            moe.debug_dequant(L.handle, e, t, out.data_ptr(), _stream(torch))
            _, ref32 = oracle.dequant_matrix(3, host[lay.offs[e, t]:], rows,
                                             int(lay.strides[e, t]), nb)
            assert np.array_equal(out.cpu().numpy().view(np.uint32), ref32.view(np.uint32)), (e, t)
    L.close()


@pytest.mark.parametrize("T,flags", [(1, 0), (3, 0), (16, 0), (40, 2), (40, 4), (40, 5)])
def test_q5_1_layer_every_path(torch, T, flags):
    # T <= 16: the fused decode kernel; 40 tokens forced to the CUDA-core grouped kernels (2),
    # or to the tensor cores (4), deterministic (5)
    w = synth.with_tokens(Q51, T)
    x, logits = inputs(w, 0)
    check_layer(torch, w, 0, x, logits, flags=flags)


@pytest.mark.parametrize("T,flags", [(2, 0), (12, 0), (150, 2), (150, 4), (150, 5)])
def test_four_formats_layer_every_path(torch, T, flags):
    w = synth.with_tokens(FOUR, T)
    x, logits = inputs(w, 0)
    check_layer(torch, w, 0, x, logits, flags=flags)


def test_q5_1_large_expert_count_grouped_decode(torch):
    w = synth.Workload("wideE_q51", 71, 256, 256, 2048, 4, 3, True, 1, "normal", sigma=2.0,
                       mix=((synth.Q5_1, 1.0),))
    x, logits = inputs(w, 0)
    check_layer(torch, w, 0, x, logits)
