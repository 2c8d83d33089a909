"""GPU parity of the router in front of the layer (moe_forward_routed) and of chained layers on a
residual stream (moe_chain_forward), against the oracle (O10, O11, O12 and O1-O9).

Checked in parts, each against the oracle on the GPU's own inputs of that step:
  - each layer's normalised input within 1e-5 (relative to the row's largest value) of the
    oracle's fp64 RMS normalisation of the GPU's x_l (fp32 sum of squares in a fixed order);
  - logits within the fp32 summation bound of the oracle's fp64 router sums (O10), the gate
    within the bound of O11;
  - the ids bit for bit equal to the oracle's top-k of the GPU's logits, the weights within 1e-6;
  - each layer's output against the oracle's layer (gated by the GPU's gate) on the GPU's x_l;
  - x_{l+1} = fp32(x_l + out_l) bit for bit;
  - the lookahead's predicted ids bit for bit equal to the top-k of layer l's router applied to
    xn_{l-1} on the GPU (the same fp32 sums), and equal to the oracle chain's early picks;
  - the whole chain against oracle.chain, ids equal in every layer and x_L within tolerance;
  - lookahead on or off, and a repeat, give bit-identical results."""
import numpy as np
import pytest

import oracle
from expert_ffn_token_b200 import synth

from gpu_helpers import (REL_TOL, RECORDS, W_TOL, check_parity, device_layer, rel_err, torch_cuda,
                         ws_array)

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


@pytest.fixture(scope="module")
def torch():
    t = torch_cuda()
    from expert_ffn_token_b200 import moe  # noqa: F401  (fails loudly if the library is missing)
    return t


def _stream(torch):
    return torch.cuda.current_stream().cuda_stream


def _rows(w, layer, gate):
    """Seeded router rows [E][H] (and a gate row [H]) for one layer: N(0, 0.05^2) fp32."""
    rng = np.random.default_rng(w.seed + 7919 * layer)
    Wr = (rng.standard_normal((w.n_experts, w.hidden)) * 0.05).astype(np.float32)
    wg = (rng.standard_normal(w.hidden) * 0.05).astype(np.float32) if gate else None
    return Wr, wg


def _logit_bound(x, Wr):
    return 1e-5 * (np.abs(x).astype(np.float64) @ np.abs(Wr).astype(np.float64).T)


def _gate_bound(x, wg):
    return 0.25e-5 * (np.abs(x).astype(np.float64) @ np.abs(wg).astype(np.float64)) + 1e-6


# ------------------------------------------------------------------ router + gate + layer


@pytest.mark.parametrize("name,T,flags", [("mtp_verify", 3, 0),          # decode kernel
                                          ("mtp_verify", 40, 0),         # tensor-core path
                                          ("mtp_verify", 40, 2),         # CUDA-core grouped path
                                          ("tiny", 4, 0)])               # no shared expert
def test_forward_routed_against_oracle(torch, name, T, flags):
    from expert_ffn_token_b200 import moe
    w = synth.with_tokens(W[name], T)
    fl = flags | moe.F_KEEP_H
    L, _, _ = device_layer(w, 0, max_tokens=T, flags=fl)
    x = synth.activations(w, 0)
    Wr, wg = _rows(w, 0, gate=w.shared)
    xd = torch.from_numpy(x).cuda()
    wrd = torch.from_numpy(Wr).cuda()
    wgd = torch.from_numpy(wg).cuda() if wg is not None else None
    lg = torch.empty((T, w.n_experts), dtype=torch.float32, device="cuda")
    gd = torch.empty(T, dtype=torch.float32, device="cuda")
    out = torch.empty_like(xd)
    moe.forward_routed(L.handle, xd.data_ptr(), T, w.k, wrd.data_ptr(),
                       wgd.data_ptr() if wgd is not None else None, lg.data_ptr(),
                       gd.data_ptr() if wgd is not None else None, out.data_ptr(),
                       L.ws.data_ptr(), L.ws_bytes, fl, _stream(torch))
    torch.cuda.synchronize()
    assert L.status() == 0
    logits = lg.cpu().numpy()
    _, l64 = oracle.router(x, Wr)
    assert (np.abs(logits - l64) <= _logit_bound(x, Wr)).all()
    gate = None
    if wg is not None:
        gate = gd.cpu().numpy()
        assert (np.abs(gate - oracle.shared_gate(x, wg)) <= _gate_bound(x, wg)).all()
    v = L.views(T, fl)
    rid, rw, _ = oracle.topk(logits, w.k)
    assert np.array_equal(ws_array(L, v["ids"], T * w.k, np.int32).reshape(T, w.k), rid)
    assert np.abs(ws_array(L, v["w"], T * w.k, np.float32).reshape(T, w.k) - rw).max() <= W_TOL
    check_parity(L, w, 0, x, logits, out.cpu().numpy(), fl, gate=gate,
                 name=f"routed {name} T={T} flags={flags}")
    # without a gate row the shared expert keeps weight 1: the plain layer on the same logits
    # gives the same bits (the batched paths add the slots atomically, in no fixed order)
    if wg is not None:
        out1 = torch.empty_like(xd)
        moe.forward_routed(L.handle, xd.data_ptr(), T, w.k, wrd.data_ptr(), None, lg.data_ptr(),
                           None, out1.data_ptr(), L.ws.data_ptr(), L.ws_bytes, fl, _stream(torch))
        out2 = L.forward(xd, lg, flags=fl)
        torch.cuda.synchronize()
        if T <= 16:
            assert torch.equal(out1, out2)
        else:
            assert ((out1 - out2).abs().amax(dim=1) <= 1e-6 * out2.abs().amax(dim=1)).all()
    L.close()


def test_forward_routed_host_errors(torch):
    from expert_ffn_token_b200 import moe
    w = W["tiny"]                  # no shared expert
    T = 2
    L, _, _ = device_layer(w, 0, max_tokens=T)
    xd = torch.zeros((T, w.hidden), dtype=torch.float32, device="cuda")
    wr = torch.zeros((w.n_experts, w.hidden), dtype=torch.float32, device="cuda")
    wg = torch.zeros(w.hidden, dtype=torch.float32, device="cuda")
    lg = torch.empty((T, w.n_experts), dtype=torch.float32, device="cuda")
    gd = torch.empty(T, dtype=torch.float32, device="cuda")
    out = torch.empty_like(xd)
    torch.cuda.synchronize()
    before = moe.kernels_enqueued()
    args = dict(arena=L.handle, d_x=xd.data_ptr(), T=T, k=w.k, d_router=wr.data_ptr(),
                d_gate_row=None, d_logits=lg.data_ptr(), d_gate=None, d_out=out.data_ptr(),
                d_ws=L.ws.data_ptr(), ws_bytes=L.ws_bytes, flags=0, stream=_stream(torch))
    # a gate row on an arena without a shared expert
    assert moe.forward_routed_status(**dict(args, d_gate_row=wg.data_ptr(),
                                            d_gate=gd.data_ptr())) == moe.ERR_INVALID_ARG
    assert moe.forward_routed_status(**dict(args, d_router=None)) == moe.ERR_INVALID_ARG
    assert moe.forward_routed_status(**dict(args, d_router=wr.data_ptr() + 4)) == moe.ERR_ALIGNMENT
    assert moe.forward_routed_status(**dict(args, ws_bytes=L.ws_bytes - 1)) == moe.ERR_WORKSPACE
    assert moe.forward_routed_status(**dict(args, k=w.n_experts + 1)) == moe.ERR_INVALID_ARG
    assert moe.kernels_enqueued() == before
    L.close()


# ------------------------------------------------------------------ chains


# RMSNorm weight of every chained layer.  The random experts are not zero-mean (their scale and
# min bytes are uniform draws), so a layer's output is close to a constant vector and the next
# layer's gate/up sums over a unit-RMS input reach ~3e3: h would pass 127 * 65504, beyond the
# fp16 scale of its Q8_1 blocks.  A weight of 1/32 keeps h in range; a trained model's norm
# weights and zero-mean experts do the same.
GAMMA = np.float32(2.0 ** -5)


def _chain_case(torch, name, T, n_layers, flags):
    """Device layers, router/gate rows, norm weights and x0 of a chain; the layers' arenas stay
    alive with the returned objects."""
    from expert_ffn_token_b200 import moe
    w = synth.with_tokens(W[name], T)
    fl = flags & ~moe.F_LOOKAHEAD
    gamma = np.full(w.hidden, GAMMA, np.float32)
    gd = torch.from_numpy(gamma).cuda()
    dev, rows = [], []
    for l in range(n_layers):
        L, _, _ = device_layer(w, l, max_tokens=T, flags=fl)
        Wr, wg = _rows(w, l, gate=w.shared)
        dev.append(L)
        rows.append((Wr, wg, torch.from_numpy(Wr).cuda(),
                     torch.from_numpy(wg).cuda() if wg is not None else None, gamma, gd))
    layers = [(L.handle, r[2].data_ptr(), r[3].data_ptr() if r[3] is not None else None,
               r[5].data_ptr()) for L, r in zip(dev, rows)]
    return w, dev, rows, layers


def _run_chain(torch, layers, x0, T, k, H, E, flags, trace=True):
    from expert_ffn_token_b200 import moe
    n = len(layers)
    nbytes = moe.chain_workspace_size(layers, T, k, flags)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    xd = torch.from_numpy(x0).cuda()
    xo = torch.empty_like(xd)
    tr = None
    bufs = {}
    if trace:
        bufs = {"x": torch.empty((n + 1, T, H), dtype=torch.float32, device="cuda"),
                "xn": torch.empty((n, T, H), dtype=torch.float32, device="cuda"),
                "logits": torch.empty((n, T, E), dtype=torch.float32, device="cuda"),
                "ids": torch.empty((n, T, k), dtype=torch.int32, device="cuda"),
                "w": torch.empty((n, T, k), dtype=torch.float32, device="cuda"),
                "gate": torch.zeros((n, T), dtype=torch.float32, device="cuda"),
                "out": torch.empty((n, T, H), dtype=torch.float32, device="cuda"),
                "early": torch.full((n, T, k), -1, dtype=torch.int32, device="cuda")}
        tr = {key: b.data_ptr() for key, b in bufs.items()}
    moe.chain_forward(layers, xd.data_ptr(), T, k, xo.data_ptr(), ws.data_ptr(), nbytes, flags,
                      tr, _stream(torch))
    torch.cuda.synchronize()
    st = moe.read_status(moe.chain_status_word(layers, ws.data_ptr(), T, k, flags), _stream(torch))
    assert st == 0
    return xo.cpu().numpy(), {key: b.cpu().numpy() for key, b in bufs.items()}


@pytest.mark.parametrize("name,T,n_layers,look", [("decode", 1, 4, True),
                                                  ("mtp_verify", 3, 3, True),
                                                  ("mtp_verify", 3, 2, False),
                                                  ("mtp_verify", 40, 2, False)])
def test_chain_against_oracle(torch, name, T, n_layers, look):
    from expert_ffn_token_b200 import moe
    # batches above 16 tokens combine deterministically, so that repeats compare bit for bit
    flags = (moe.F_LOOKAHEAD if look else 0) | (moe.F_DETERMINISTIC if T > 16 else 0)
    w, dev, rows, layers = _chain_case(torch, name, T, n_layers, flags)
    k, H, E = w.k, w.hidden, w.n_experts
    x0 = synth.activations(w, 0)
    xL, tr = _run_chain(torch, layers, x0, T, k, H, E, flags)
    assert np.array_equal(tr["x"][0], x0)
    assert np.array_equal(tr["x"][n_layers], xL)
    need = []
    for l in range(n_layers):
        xres = tr["x"][l]
        x = tr["xn"][l]
        ref_xn = oracle.rmsnorm(xres, rows[l][4])
        assert (np.abs(x - ref_xn).max(axis=1) <= 1e-5 * np.abs(ref_xn).max(axis=1)).all(), l
        Wr, wg = rows[l][0], rows[l][1]
        logits = tr["logits"][l]
        _, l64 = oracle.router(x, Wr)
        assert (np.abs(logits - l64) <= _logit_bound(x, Wr)).all(), l
        rid, rw, _ = oracle.topk(logits, k)
        assert np.array_equal(tr["ids"][l], rid), l
        assert np.abs(tr["w"][l] - rw).max() <= W_TOL
        gate = None
        if wg is not None:
            gate = tr["gate"][l]
            assert (np.abs(gate - oracle.shared_gate(x, wg)) <= _gate_bound(x, wg)).all(), l
        ids_l = set(int(e) for e in rid.ravel()) | ({E} if w.shared else set())
        need.append(ids_l)
        buf, lay = synth.compact_arena(w, l, ids_l)
        ex = oracle.experts_table(lay.fmts, lay.offs, lay.strides)
        ref, _ = oracle.forward(buf, ex, lay.shared, H, w.ffn, x, rid, rw,
                                gate=None if gate is None else gate.astype(np.float64))
        err = rel_err(tr["out"][l], ref.astype(np.float64))
        RECORDS.append({"check": f"chain {name} T={T} layer {l}", "tokens": T, "h_rel_err": 0.0,
                        "chain_rel_err": float(err.max()), "e2e_rel_err_clean": float(err.max()),
                        "e2e_rel_err_all": float(err.max()), "elementwise_clean": 0.0,
                        "flip_tokens": 0, "flips": 0})
        assert err.max() <= REL_TOL, (l, err.max())
        assert np.array_equal(tr["x"][l + 1], (xres + tr["out"][l]).astype(np.float32)), l
        if look and l >= 1:
            # the prediction is the top-k of layer l's router on xn_{l-1}, as the GPU sums it
            prev = torch.from_numpy(tr["xn"][l - 1]).cuda()
            lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
            moe.router_logits(prev.data_ptr(), T, H, rows[l][2].data_ptr(), E, lg.data_ptr(),
                              _stream(torch))
            pid, _, _ = oracle.topk(lg.cpu().numpy(), k)
            assert np.array_equal(tr["early"][l], pid), l
    if look:
        assert (tr["early"][0] == -1).all()
    # the oracle's chain from x0, on arenas holding the experts the GPU chose
    host_layers = []
    for l in range(n_layers):
        buf, lay = synth.compact_arena(w, l, need[l])
        host_layers.append({"arena": buf,
                            "experts": oracle.experts_table(lay.fmts, lay.offs, lay.strides),
                            "shared": lay.shared, "hidden": H, "ffn": w.ffn,
                            "router": rows[l][0], "gate": rows[l][1], "norm": rows[l][4]})
    res = oracle.chain(host_layers, x0, k, lookahead=look)
    for l in range(n_layers):
        assert np.array_equal(res[1][l], tr["ids"][l]), l
    if look:
        for l in range(1, n_layers):
            assert np.array_equal(res[2][l - 1], tr["early"][l]), l
    # x_L = x_0 + sum of the layers' outputs: each within REL_TOL of its own scale (a layer whose
    # gate/up sums are all far below zero outputs exactly 0: silu saturates and h underflows)
    scale = np.abs(x0).max(axis=1) + sum(np.abs(tr["out"][l]).max(axis=1) for l in range(n_layers))
    dev_err = np.abs(xL.astype(np.float64) - res[0]).max(axis=1) / scale
    assert dev_err.max() <= REL_TOL, dev_err.max()
    # the prediction only warms L2: lookahead off, and a repeat, give the same bits
    xL2, _ = _run_chain(torch, layers, x0, T, k, H, E, flags, trace=False)
    assert np.array_equal(xL2, xL)
    if look:
        xL3, _ = _run_chain(torch, layers, x0, T, k, H, E, flags & ~moe.F_LOOKAHEAD, trace=False)
        assert np.array_equal(xL3, xL)
    for L in dev:
        L.close()


def test_chain_host_errors(torch):
    from expert_ffn_token_b200 import moe
    w, dev, rows, layers = _chain_case(torch, "mtp_verify", 20, 2, 0)
    nbytes = moe.chain_workspace_size(layers, 20, w.k, 0)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    xd = torch.zeros((20, w.hidden), dtype=torch.float32, device="cuda")
    xo = torch.empty_like(xd)
    torch.cuda.synchronize()
    before = moe.kernels_enqueued()
    st = _stream(torch)
    run = moe.chain_forward_status
    # lookahead is for batches of <= 16 tokens
    assert run(layers, xd.data_ptr(), 20, w.k, xo.data_ptr(), ws.data_ptr(), nbytes,
               moe.F_LOOKAHEAD, None, st) == moe.ERR_INVALID_ARG
    assert run(layers, xd.data_ptr(), 20, w.k, xo.data_ptr(), ws.data_ptr(), nbytes - 1, 0, None,
               st) == moe.ERR_WORKSPACE
    assert run(layers, xd.data_ptr() + 4, 20, w.k, xo.data_ptr(), ws.data_ptr(), nbytes, 0, None,
               st) == moe.ERR_ALIGNMENT
    assert run([], xd.data_ptr(), 20, w.k, xo.data_ptr(), ws.data_ptr(), nbytes, 0, None,
               st) == moe.ERR_INVALID_ARG
    # layers of different hidden sizes
    t = W["tiny"]
    Lt, _, _ = device_layer(t, 0, max_tokens=20)
    wt = torch.zeros((t.n_experts, t.hidden), dtype=torch.float32, device="cuda")
    bad = [layers[0], (Lt.handle, wt.data_ptr(), None)]
    assert run(bad, xd.data_ptr(), 20, w.k, xo.data_ptr(), ws.data_ptr(), nbytes, 0, None,
               st) == moe.ERR_INVALID_ARG
    assert moe.kernels_enqueued() == before
    Lt.close()
    for L in dev:
        L.close()
