"""Chains of small-M forward calls in one persistent launch (mmf_bitlinear_chain),
through the C ABI: each call's y has the bits of the same call issued on its own
(group, GLU) and matches the oracle; calls that read earlier calls' outputs see
them complete; the launch is reusable and graph-capturable."""
import numpy as np
import pytest
import torch

from bitlinear_rmsnorm_quant_b200 import mmf
from bitlinear_rmsnorm_quant_b200 import inputs as I
from bitlinear_rmsnorm_quant_b200 import workloads as WL
from gpu_cases import Y_REL_TOL, bits_np, make_layer, y_rel_error

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
EPS = 1e-6
EPS_W = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bitlinear_rmsnorm_quant_b200 import build
    build.build()
    torch.cuda.set_device(0)
    yield
    mmf.check_async()


def _weights(seed, K, Ns, index0):
    """[(packed, scale, N, W)] for the given widths (N = 0 gives an empty entry)."""
    out = []
    for i, N in enumerate(Ns):
        W = make_layer(seed, 1, K, max(N, 1), index=index0 + i)[2][:N].contiguous()
        if N > 0:
            pk, sc = mmf.pack_ternary(W.to(DEV), EPS_W)
        else:
            pk, sc = torch.zeros(1, K // 16, dtype=torch.int32, device=DEV), torch.ones(1, device=DEV)
        out.append((pk, sc, N, W))
    return out


# (K, widths, GLU) of the calls of one chain: groups with empty and ragged
# projections, slabs of one or several stages, K from 128 to the limit
CALLS = [(2560, (2560, 100, 0, 333), False), (6912, (2560,), False), (1024, (300,), True),
         (128, (16, 3), False), (8192, (1000, 7), False), (2816, (1024,), True), (2560, (6912, 6912), False)]


@pytest.mark.parametrize("M", [1, 2, 3])
def test_chain_matches_single_calls_and_oracle(oracle, M):
    calls, expect = [], []
    for ci, (K, Ns, glu) in enumerate(CALLS):
        x, g, _ = make_layer(30 + ci, M, K, 1)
        u = I.activations(30 + ci, M, K, index=9) if glu else None
        ws = _weights(30 + ci, K, Ns, 1)
        xd, gd = x.to(DEV), g.to(DEV)
        ud = u.to(DEV) if glu else None
        ys = [torch.full((M, N), 7, dtype=torch.bfloat16, device=DEV) for (_, _, N, _) in ws]
        c = {"x": xd, "gamma": gd, "weights": [(pk, sc, y) for (pk, sc, _, _), y in zip(ws, ys)]}
        if glu:
            c["u"] = ud
            ref = [mmf.bitlinear_fwd_glu(xd, ud, gd, ws[0][0], ws[0][1], ws[0][2], EPS)]
        else:
            ref = mmf.bitlinear_fwd_group(xd, gd, [(pk, sc, N) for (pk, sc, N, _) in ws], EPS)
        calls.append(c)
        expect.append((x, u, g, ws, ys, ref))
    chain = mmf.Chain(calls, EPS)
    chain.run()
    torch.cuda.synchronize()
    assert mmf.check_async() is None
    for x, u, g, ws, ys, ref in expect:
        xin = bits_np(x) if u is None else oracle.glu_gate(bits_np(x), bits_np(u))
        for (pk, sc, N, W), y, r in zip(ws, ys, ref):
            assert y.shape == (M, N)
            if N == 0:
                continue
            assert torch.equal(y, r)
            y_ref, beta = oracle.bitlinear(xin, g.numpy(), EPS, W.numpy(), EPS_W)
            assert np.float32(sc.item()) == beta
            assert y_rel_error(bits_np(y), y_ref) <= Y_REL_TOL


@pytest.mark.parametrize("M", [1, 3])
def test_chain_of_dependent_calls(M):
    """Each call reads earlier calls' outputs (the previous y, and a GLU call
    reading two earlier ys); the chain gives the bits of issuing the calls one
    by one, launch after launch, and inside a CUDA graph."""
    K = 2048
    x, g, _ = make_layer(40, M, K, 1)
    gd = g.to(DEV)
    ws = _weights(40, K, (K,) * 12, 1)
    ys = [torch.empty(M, K, dtype=torch.bfloat16, device=DEV) for _ in ws]
    calls, cur = [], x.to(DEV)
    for i, (pk, sc, N, _) in enumerate(ws):
        if i == 6:
            calls.append({"x": ys[3], "u": ys[5], "gamma": gd, "weights": [(pk, sc, ys[i])]})
        else:
            calls.append({"x": cur, "gamma": gd, "weights": [(pk, sc, ys[i])]})
        cur = ys[i]
    # one by one
    ref, cur = [], x.to(DEV)
    for i, (pk, sc, N, _) in enumerate(ws):
        if i == 6:
            r = mmf.bitlinear_fwd_glu(ref[3], ref[5], gd, pk, sc, N, EPS)
        else:
            r = mmf.bitlinear_fwd_group(cur, gd, [(pk, sc, N)], EPS)[0]
        ref.append(r)
        cur = r
    chain = mmf.Chain(calls, EPS)
    for _ in range(3):
        for y in ys:
            y.fill_(0)
        chain.run()
        torch.cuda.synchronize()
        for y, r in zip(ys, ref):
            assert torch.equal(y, r)
    # captured in a graph, replayed
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        chain.run(s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        chain.run()
    for _ in range(2):
        for y in ys:
            y.fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        for y, r in zip(ys, ref):
            assert torch.equal(y, r)
    assert mmf.check_async() is None


def test_chain_decode_layer_sets(oracle):
    """Two layer sets of the 2.7B decode step (token-mixer gates, o, channel-mixer
    gate/up, down) at one token as one chain, against the same calls issued as
    groups; the down projection also against the oracle."""
    wl = WL.decode_2p7b(1)
    groups = {}
    for j, p in enumerate(wl.projections):
        groups.setdefault(p.input_index, []).append(j)
    calls, expect = [], []
    for l in range(2):
        for idx, js in sorted(groups.items()):
            K = wl.projections[js[0]].K
            x, g, _ = make_layer(50 + l, 1, K, 1, index=idx)
            ws = _weights(50 + l, K, [wl.projections[j].N for j in js], 10 * idx + 1)
            ys = [torch.empty(1, N, dtype=torch.bfloat16, device=DEV) for (_, _, N, _) in ws]
            calls.append({"x": x.to(DEV), "gamma": g.to(DEV),
                          "weights": [(pk, sc, y) for (pk, sc, _, _), y in zip(ws, ys)]})
            ref = mmf.bitlinear_fwd_group(calls[-1]["x"], calls[-1]["gamma"], [(pk, sc, N) for (pk, sc, N, _) in ws],
                                          EPS)
            expect.append((x, g, ws, ys, ref))
    chain = mmf.Chain(calls, EPS)
    chain.run()
    torch.cuda.synchronize()
    for x, g, ws, ys, ref in expect:
        for y, r in zip(ys, ref):
            assert torch.equal(y, r)
    x, g, ws, ys, _ = expect[-1]
    y_ref, _ = oracle.bitlinear(bits_np(x), g.numpy(), EPS, ws[0][3].numpy(), EPS_W)
    assert y_rel_error(bits_np(ys[0]), y_ref) <= Y_REL_TOL


def test_chain_edge_cases():
    """No tokens launches nothing; a chain whose calls have only empty
    projections runs; device-side argument errors."""
    K = 256
    x0 = torch.zeros(0, K, dtype=torch.bfloat16, device=DEV)
    g = torch.ones(K, device=DEV)
    pk, sc = mmf.pack_ternary(torch.randn(64, K, device=DEV))
    y0 = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    mmf.Chain([{"x": x0, "gamma": g, "weights": [(pk, sc, y0)]}]).run()
    x1 = torch.randn(1, K, device=DEV).to(torch.bfloat16)
    ye = torch.empty(1, 0, dtype=torch.bfloat16, device=DEV)
    y1 = torch.empty(1, 64, dtype=torch.bfloat16, device=DEV)
    ch = mmf.Chain([{"x": x1, "gamma": g, "weights": [(pk, sc, ye)]},
                    {"x": x1, "gamma": g, "weights": [(pk, sc, y1)]}])
    ch.run()
    torch.cuda.synchronize()
    assert torch.equal(y1, mmf.bitlinear_fwd(x1, g, pk, sc, 64, EPS))
    # a handle whose grid is not this device's SM count is refused
    bad = mmf.ChainHandle.from_buffer_copy(ch.handle)
    bad.grid = ch.handle.grid + 1
    import ctypes as C
    assert mmf.lib().mmf_bitlinear_chain(C.byref(bad), torch.cuda.current_stream().cuda_stream) == 1
    assert mmf.check_async() is None
