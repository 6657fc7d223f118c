"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: packed words, beta and int32 accumulators bit-exact; y within max
relative error 1e-2 (floored, see gpu_cases); at most 0.1% of int8 activation
codes differ, and then by one.  Sizes span several tiles with ragged tails on
all kernel paths (fused decode GEMV for M <= 3, the decode tensor-core kernel for
4 .. 32, the tcgen05 GEMM above), and the
full configuration sizes are checked on sampled tokens.
"""
import numpy as np
import pytest
import torch

from bitlinear_rmsnorm_quant_b200 import mmf
from bitlinear_rmsnorm_quant_b200 import inputs as I
from bitlinear_rmsnorm_quant_b200 import workloads as WL
from gpu_cases import (Q_MAX_DIFF_FRAC, Y_REL_TOL, bf16_to_f64, bits_np, make_layer, q_diff_stats,
                       y_rel_error)

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


def _pack(W):
    packed, scale = mmf.pack_ternary(W.to(DEV), EPS_W)
    return packed, scale


def _oracle_codes(oracle, W):
    wt, beta = oracle.absmean_ternary(W.numpy(), EPS_W)
    return wt, beta


# -- packer ------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(256, 256), (1, 128), (3, 384), (1000, 1024), (2816, 1024), (2560, 6912),
                                 (5632, 2048)])
def test_pack_bit_exact(oracle, N, K):
    _, _, W = make_layer(7, 1, K, N)
    packed, scale = _pack(W)
    torch.cuda.synchronize()
    wt, beta = _oracle_codes(oracle, W)
    assert np.float32(scale.item()) == beta
    ref = oracle.encode_packed(wt)
    got = packed.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, ref)


def test_pack_deterministic():
    _, _, W = make_layer(8, 1, 2560, 2560)
    Wd = W.to(DEV)
    p1, s1 = mmf.pack_ternary(Wd, EPS_W)
    p2, s2 = mmf.pack_ternary(Wd, EPS_W)
    torch.cuda.synchronize()
    assert torch.equal(p1, p2) and torch.equal(s1, s2)


def test_pack_special_matrices(oracle):
    # W = c*I gives the identity; a constant matrix gives all +1
    K = 256
    W = torch.eye(K, dtype=torch.float32) * 0.75
    packed, scale = _pack(W)
    wt, bad = oracle.decode_packed(packed.cpu().numpy().view(np.uint32), K)
    assert bad == 0 and np.array_equal(wt, np.eye(K, dtype=np.int8))
    packed, _ = _pack(torch.full((16, K), -0.3))
    wt, _ = oracle.decode_packed(packed.cpu().numpy().view(np.uint32), K)
    assert (wt == -1).all()


# -- RMSNorm + quantisation ------------------------------------------------------------

@pytest.mark.parametrize("M,K,outliers", [(16, 256, 0.0), (5, 128, 0.0), (300, 2048, 0.0), (37, 6912, 0.01),
                                          (64, 5632, 0.0),
                                          # large M: the persistent register kernel, one to four warps per
                                          # row (K <= 2048, 4096, 6912 (three warps of up to 9 chunks),
                                          # 8192), each lane holding as many 16-byte chunks as the width
                                          # needs (4 .. 9), ragged lanes at each width
                                          (4100, 1024, 0.0), (5000, 128, 0.0), (4096, 1280, 0.01),
                                          (4096, 2048, 0.01), (4099, 2560, 0.01), (4100, 3072, 0.0),
                                          (4096, 4096, 0.0), (4097, 5632, 0.0), (4096, 6144, 0.01),
                                          (4096, 6912, 0.01), (4100, 6272, 0.0), (4096, 7168, 0.01),
                                          (4097, 7296, 0.0),
                                          (4096, 8192, 0.0),
                                          # beyond its largest K, a CTA per row
                                          (4096, 8320, 0.0), (4096, 11392, 0.01)])
def test_quantize_act(oracle, M, K, outliers):
    x, g, _ = make_layer(9, M, K, 1, outlier_frac=outliers)
    q, a = mmf.quantize_act(x.to(DEV), g.to(DEV), EPS)
    torch.cuda.synchronize()
    q_ref, a_ref = oracle.rmsnorm_quant(bits_np(x), g.numpy(), EPS)
    frac, mx = q_diff_stats(q.cpu().numpy(), q_ref)
    assert mx <= 1 and frac <= Q_MAX_DIFF_FRAC
    assert np.allclose(a.cpu().numpy(), a_ref, rtol=2e-7, atol=0)


def test_quantize_special_rows(oracle):
    K = 512
    x = torch.zeros(4, K, dtype=torch.bfloat16)
    x[1] = 3.0
    x[2] = -0.5
    x[3, 7] = 1.0
    g = torch.ones(K)
    q, a = mmf.quantize_act(x.to(DEV), g.to(DEV), EPS)
    torch.cuda.synchronize()
    q = q.cpu()
    assert (q[0] == 0).all() and a[0].item() == np.float32(1e-5)
    assert (q[1] == 127).all() and (q[2] == -127).all()
    assert q[3, 7] == 127 and (q[3].abs().sum() == 127)


# -- ternary contraction: int32 bit-exact on the kernel's own q and packed W --------------

ACC_SHAPES = [
    # (M, K, N) CUDA-core decode kernel (1 .. 3 tokens): weight ring refilled many times per CTA
    (1, 128, 1), (1, 256, 256), (1, 6912, 20000),
    (2, 1024, 1000), (3, 2560, 333), (3, 6912, 2560), (2, 128, 8),
    # decode tensor-core kernel (4 .. 32 tokens): slabs of 256 rows per projection (ragged last
    # slab, slabs of fewer rows than 256), K split over clusters of 1 .. 8 CTAs (K = 128: one
    # chunk; K = 6912: 54 chunks; K = 8192), 16 and 32 operand rows, one slab to several waves
    (4, 4096, 9000), (5, 2816, 1024), (8, 6912, 2560), (9, 256, 300), (4, 128, 100),
    (16, 256, 256), (17, 384, 129), (32, 2560, 640), (32, 6912, 700), (24, 2560, 13824),
    (31, 8192, 40000), (12, 1024, 80000),
    # large-M tcgen05 path: several 128-row tiles, token tiles, K stages, ragged tails
    (33, 2048, 500), (100, 1024, 257), (256, 512, 384), (300, 384, 300), (513, 2048, 200),
]


@pytest.mark.parametrize("M,K,N", ACC_SHAPES)
def test_ternary_acc_bit_exact(oracle, M, K, N):
    x, g, W = make_layer(10, M, K, N)
    packed, _ = _pack(W)
    q, _ = mmf.quantize_act(x.to(DEV), g.to(DEV), EPS)
    acc = mmf.ternary_acc(q, packed, N)
    torch.cuda.synchronize()
    wt, bad = oracle.decode_packed(packed.cpu().numpy().view(np.uint32), K)
    assert bad == 0
    ref = oracle.ternary_acc(q.cpu().numpy(), wt)
    got = acc.cpu().numpy()
    assert np.array_equal(got, ref), f"{np.count_nonzero(got != ref)} of {got.size} differ"


def test_ternary_acc_extreme_codes(oracle):
    # every activation at +-127 and every weight at +-1: the largest |acc|
    M, K, N = 20, 6912, 256
    q = torch.full((M, K), 127, dtype=torch.int8)
    q[1::2] = -127
    W = torch.ones(N, K)
    W[N // 2:] = -1.0
    packed, _ = _pack(W)
    acc = mmf.ternary_acc(q.to(DEV), packed, N)
    acc1 = mmf.ternary_acc(q[:1].to(DEV), packed, N)
    torch.cuda.synchronize()
    wt, _ = oracle.decode_packed(packed.cpu().numpy().view(np.uint32), K)
    assert np.array_equal(acc.cpu().numpy(), oracle.ternary_acc(q.numpy(), wt))
    assert np.array_equal(acc1.cpu().numpy(), oracle.ternary_acc(q[:1].numpy(), wt))
    assert abs(int(acc[0, 0])) == 127 * K


# -- whole layer against the oracle ----------------------------------------------------------

def _layer_parity(oracle, x, g, W, sample_tokens=None):
    packed, scale = _pack(W)
    y = mmf.bitlinear_fwd(x.to(DEV), g.to(DEV), packed, scale, W.shape[0], EPS)
    torch.cuda.synchronize()
    xs = x if sample_tokens is None else x[sample_tokens]
    ys = y if sample_tokens is None else y[torch.as_tensor(sample_tokens, device=y.device)]
    y_ref, beta = oracle.bitlinear(bits_np(xs), g.numpy(), EPS, W.numpy(), EPS_W)
    assert np.float32(scale.item()) == beta
    err = y_rel_error(bits_np(ys), y_ref)
    assert err <= Y_REL_TOL, err
    return err


@pytest.mark.parametrize("M,K,N", [(1, 128, 16), (1, 1024, 2816), (4, 2560, 1000), (8, 6912, 2560), (1, 6912, 20000),
                                   (9, 256, 256), (16, 256, 256), (33, 2048, 500), (300, 384, 300),
                                   (1000, 1024, 384)])
def test_bitlinear_parity(oracle, M, K, N):
    x, g, W = make_layer(11, M, K, N)
    _layer_parity(oracle, x, g, W)


def test_smoke_config(oracle):
    w = WL.SMOKE
    p = w.projections[0]
    x, g, W = make_layer(w.seed, w.M, p.K, p.N)
    _layer_parity(oracle, x, g, W)


@pytest.mark.parametrize("wl", [WL.DECODE_370M, WL.decode_2p7b(1), WL.decode_2p7b(8), WL.decode_2p7b(32)],
                         ids=lambda w: w.name)
def test_decode_configs(oracle, wl):
    for j, p in enumerate(wl.projections):
        x, g, _ = make_layer(wl.seed, wl.M, p.K, 1, index=p.input_index, outlier_frac=wl.outlier_frac)
        W = I.latent_weights(wl.seed, p.N, p.K, index=16 + j)  # each projection its own matrix
        _layer_parity(oracle, x, g, W)


@pytest.mark.parametrize("wl", [WL.PREFILL_1P3B, WL.PREFILL_2P7B], ids=lambda w: w.name)
def test_prefill_config_sampled(oracle, wl):
    """Full prefill size (M=8192) on the GPU; the oracle checks 48 sampled tokens."""
    rng = np.random.default_rng(5)
    for p in wl.projections:
        x, g, W = make_layer(wl.seed, wl.M, p.K, p.N, index=p.input_index, outlier_frac=wl.outlier_frac)
        tokens = np.sort(rng.choice(wl.M, 48, replace=False))
        _layer_parity(oracle, x, g, W, sample_tokens=tokens)


def test_zero_and_degenerate_tokens(oracle):
    K, N = 1024, 512
    x, g, W = make_layer(12, 40, K, N)
    x[3] = 0.0
    x[7] = 2.5
    x[11, :] = 0.0
    x[11, 5] = -7.0
    _layer_parity(oracle, x, g, W)
    _layer_parity(oracle, x[:4], g, W)     # decode path with a zero token
    packed, scale = _pack(W)
    y = mmf.bitlinear_fwd(x.to(DEV), g.to(DEV), packed, scale, N, EPS)
    torch.cuda.synchronize()
    assert (y[3] == 0).all()


@pytest.mark.parametrize("case", ["random", "zero", "constant", "tie", "near_tie", "outlier", "negative_max"])
def test_single_token_matches_large_m_path(oracle, case):
    """M = 1 (decode kernel, which may take the absmax from the largest |x gamma|
    product) against the same token replicated to M = 16 (separate quantiser and
    tensor-core kernel, full absmax reduction): the same bits, and the oracle."""
    K, N = 2560, 512
    x, g, W = make_layer(21, 1, K, N)
    if case == "zero":
        x[:] = 0.0
    elif case == "constant":
        x[:] = 1.5
    elif case == "tie":
        x[0, 5] = 9.0
        x[0, 900] = -9.0
        g[5] = g[900] = 1.25
    elif case == "near_tie":
        x[0, 5] = 9.0
        x[0, 900] = 9.0
        g[5] = 1.0
        g[900] = float(np.nextafter(np.float32(1.0), np.float32(2.0)))
    elif case == "outlier":
        x[0, 17] = 100.0
    elif case == "negative_max":
        x[0, 33] = -50.0
        g[33] = 0.5
    packed, scale = _pack(W)
    xd, gd = x.to(DEV), g.to(DEV)
    y1 = mmf.bitlinear_fwd(xd, gd, packed, scale, N, EPS)
    y16 = mmf.bitlinear_fwd(xd.expand(16, K).contiguous(), gd, packed, scale, N, EPS)
    torch.cuda.synchronize()
    assert mmf.workspace_bytes(1, K, N) == 0 and mmf.workspace_bytes(16, K, N) > 0  # two different paths
    assert torch.equal(y1[0], y16[0]) and torch.equal(y16[0], y16[15])
    y_ref, _ = oracle.bitlinear(bits_np(x), g.numpy(), EPS, W.numpy(), EPS_W)
    assert y_rel_error(bits_np(y1), y_ref) <= Y_REL_TOL


@pytest.mark.parametrize("M", [2, 3, 5, 8, 13, 16, 17, 24, 32])
@pytest.mark.parametrize("K", [2560, 6912])
def test_decode_codes_match_large_m_path(oracle, M, K):
    """The decode paths never hand their codes out: the CUDA-core kernel (up to
    3 tokens) forms them in shared memory, the tensor-core one (4 .. 32 tokens)
    keeps them in the MMA's operand layout with zero rows up to 16 or 32
    tokens.  M tokens on it against the same tokens as the first rows of a
    64-token batch (codes in row-major order, which the quantiser test compares
    with the oracle, then the large-M tensor-core kernel): bit-equal y means
    equal codes, sums and absmax (a code off by one changes acc for every
    output row whose weight at that k is not 0).  Rows of the 2.7B decode
    workload, 1% outlier channels x20."""
    N = 512
    wl = WL.decode_2p7b(8)
    x, g, W = make_layer(wl.seed, 64, K, N, index=40 + M, outlier_frac=wl.outlier_frac)
    x[0, :] = x[0, :] * 0.0 + 1.5          # a constant token (every |r| ties)
    packed, scale = _pack(W)
    xd, gd = x.to(DEV), g.to(DEV)
    nt = 16 if M <= 16 else 32               # two different paths (codes in shared memory, or in the
    assert mmf.workspace_bytes(M, K, N) < nt * K + 1024 < mmf.workspace_bytes(64, K, N)   # operand layout)
    y_small = mmf.bitlinear_fwd(xd[:M].contiguous(), gd, packed, scale, N, EPS)
    y_big = mmf.bitlinear_fwd(xd, gd, packed, scale, N, EPS)
    torch.cuda.synchronize()
    assert torch.equal(y_small, y_big[:M])
    y_ref, _ = oracle.bitlinear(bits_np(x[:M]), g.numpy(), EPS, W.numpy(), EPS_W)
    assert y_rel_error(bits_np(y_small), y_ref) <= Y_REL_TOL


def test_training_batch_forward_sampled(oracle):
    """The training-batch forward's largest projection, 5632 -> 2048 at
    M = 2^8 * 2048 = 524288 tokens (its codes take M*K = 2.95e9 bytes, past
    2^31), full size on the GPU through the C ABI: the int8 codes and absmax of
    64 sampled tokens (half of them beyond row 2^31 / K) against the oracle,
    their int32 accumulators bit-exact on the kernel's own codes, and y within
    the layer bar.  x is drawn on the device; the oracle reads the sampled
    rows' bytes back from it."""
    wl = WL.TRAIN_FWD_1P3B
    p = [p for p in wl.projections if p.name == "down"][0]
    M, K, N = wl.M, p.K, p.N
    assert M * K > 2 ** 31
    rng = np.random.default_rng(11)
    edge = (2 ** 31) // K
    rows = np.sort(np.concatenate([rng.choice(edge, 32, replace=False),
                                   edge + rng.choice(M - edge, 31, replace=False), [M - 1]]))
    xd = I.activations(wl.seed, M, K, index=p.input_index, device=DEV)
    g = I.gamma(wl.seed, K, index=p.input_index)
    W = I.latent_weights(wl.seed, N, K, index=6)
    gd = g.to(DEV)
    packed, scale = _pack(W)
    ridx = torch.as_tensor(rows, device=DEV)
    x_rows = bits_np(xd[ridx])
    q, a = mmf.quantize_act(xd, gd, EPS)
    q_rows, a_rows = q[ridx].cpu().numpy(), a[ridx].cpu().numpy()
    acc = mmf.ternary_acc(q, packed, N)
    acc_rows = acc[ridx].cpu().numpy()
    del acc, q
    y = mmf.bitlinear_fwd(xd, gd, packed, scale, N, EPS)
    y_rows = bits_np(y[ridx])
    torch.cuda.synchronize()
    del y, xd
    q_ref, a_ref = oracle.rmsnorm_quant(x_rows, g.numpy(), EPS)
    frac, mx = q_diff_stats(q_rows, q_ref)
    assert mx <= 1 and frac <= Q_MAX_DIFF_FRAC
    assert np.allclose(a_rows, a_ref, rtol=2e-7, atol=0)
    wt, bad = oracle.decode_packed(packed.cpu().numpy().view(np.uint32), K)
    assert bad == 0
    assert np.array_equal(acc_rows, oracle.ternary_acc(q_rows, wt))
    y_ref, beta = oracle.bitlinear(x_rows, g.numpy(), EPS, W.numpy(), EPS_W)
    assert np.float32(scale.item()) == beta
    assert y_rel_error(y_rows, y_ref) <= Y_REL_TOL


# -- GLU channel mixer: down projection with SiLU(g) * u fused in -----------------------------

@pytest.mark.parametrize("M,K,N", [(1, 6912, 2560), (3, 2816, 1024), (8, 5632, 2048), (1, 128, 16),
                                   (16, 6912, 2560), (31, 2816, 1000),
                                   (64, 2816, 1024), (300, 6912, 640), (4100, 1024, 256)])
def test_glu_parity(oracle, M, K, N):
    """y of the fused GLU call against the oracle's gated product fed to its BitLinear."""
    g, gamma, W = make_layer(22, M, K, N)
    u = I.activations(22, M, K, index=5)
    packed, scale = _pack(W)
    y = mmf.bitlinear_fwd_glu(g.to(DEV), u.to(DEV), gamma.to(DEV), packed, scale, N, EPS)
    torch.cuda.synchronize()
    p_bits = oracle.glu_gate(bits_np(g), bits_np(u))
    y_ref, beta = oracle.bitlinear(p_bits, gamma.numpy(), EPS, W.numpy(), EPS_W)
    assert np.float32(scale.item()) == beta
    assert y_rel_error(bits_np(y), y_ref) <= Y_REL_TOL


def test_glu_paths_agree_and_match_plain_call():
    """One token on the decode kernel, the same token replicated on the large-M
    path, with and without PDL: identical bits.  And the fused call equals the
    plain call given the gated product the GPU forms (read back through the
    large-M path's own rounding: the same fp32 steps)."""
    K, N = 2816, 512
    g, gamma, W = make_layer(23, 1, K, N)
    u = I.activations(23, 1, K, index=6)
    packed, scale = _pack(W)
    gd, ud, gmd = g.to(DEV), u.to(DEV), gamma.to(DEV)
    y1 = mmf.bitlinear_fwd_glu(gd, ud, gmd, packed, scale, N, EPS)
    y1p = mmf.bitlinear_fwd_glu(gd, ud, gmd, packed, scale, N, EPS, flags=mmf.FWD_PDL)
    y16 = mmf.bitlinear_fwd_glu(gd.expand(16, K).contiguous(), ud.expand(16, K).contiguous(), gmd, packed, scale, N,
                                EPS)
    torch.cuda.synchronize()
    assert torch.equal(y1, y1p) and torch.equal(y1[0], y16[0]) and torch.equal(y16[0], y16[15])
    # the plain call on p computed on the host in the same fp32 steps agrees within the tolerance
    gf, uf = g.float(), u.float()
    p = (gf * (1.0 / (1.0 + torch.exp(-gf))) * uf).to(torch.bfloat16)
    y_plain = mmf.bitlinear_fwd(p.to(DEV), gmd, packed, scale, N, EPS)
    torch.cuda.synchronize()
    yv, yp = y1.float().cpu().numpy(), y_plain.float().cpu().numpy()
    assert np.abs(yv - yp).max() <= 1e-2 * max(np.abs(yp).max(), 1e-6)


# -- MLGRU token mixer recurrence -------------------------------------------------------------

@pytest.mark.parametrize("B,T,D", [
    # per-warp chunk kernel: few rows, D not a multiple of 8, no tokens
    (1, 1, 2560), (2, 37, 128), (3, 100, 66), (2, 5, 64), (1, 0, 64),
    # tensor-copy kernel: 128-token stages, ragged last stage (the next sequence's rows
    # read and ignored), channels past D in the last CTA, sequences shorter than a stage
    (4, 2048, 2048), (2, 300, 200), (1, 1000, 4104), (5, 70, 512), (3, 128, 64)])
@pytest.mark.parametrize("with_h0", [False, True])
def test_mlgru_scan_parity(oracle, B, T, D, with_h0):
    rng = np.random.default_rng(B * 1000 + T + D)
    mk = lambda: torch.from_numpy(rng.standard_normal((B, T, D)).astype(np.float32) * 2.0).to(torch.bfloat16)
    fp, cp, gp = mk(), mk(), mk()
    h0 = torch.from_numpy(rng.standard_normal((B, D)).astype(np.float32)) if with_h0 else None
    o, hl = mmf.mlgru_scan(fp.to(DEV), cp.to(DEV), gp.to(DEV), h0.to(DEV) if with_h0 else None)
    torch.cuda.synchronize()
    o_ref, hl_ref = oracle.mlgru_scan(bits_np(fp), bits_np(cp), bits_np(gp), h0.numpy() if with_h0 else None)
    ov, rv = bf16_to_f64(bits_np(o.cpu())), bf16_to_f64(o_ref)
    # chunked combination rounds differently from token-by-token: within fp32
    # rounding of the state, then at most one bf16 step of o
    h_tol = 1e-4 * (1.0 + np.abs(hl_ref))
    assert (np.abs(hl.cpu().numpy() - hl_ref) <= h_tol).all()
    assert (np.abs(ov - rv) <= np.abs(rv) * 2.0 ** -7 + 1e-6).all()
    if T > 0:
        assert (ov == rv).mean() > 0.99


@pytest.mark.parametrize("B,T,D", [(2, 300, 128), (1, 129, 66)])
def test_mlgru_scan_saturated_gates(oracle, B, T, D):
    """Pre-activations of +-60 mixed into normal ones: gates at 0 and 1 within
    fp32, the SiLU input large on both sides; the tensor-copy kernel (D = 128)
    and the per-warp-chunk one (D = 66).  The kernels clamp pre-activations at
    -28 before the exponential, so a gate of sigma(-60) = 9e-27 comes out as
    sigma(-28) = 7e-13: o then differs from the oracle's by far less than the
    absolute bound, though not bit for bit, so bit equality is counted over
    the outputs above 1e-6."""
    rng = np.random.default_rng(B * 7 + T + D)
    v = lambda: rng.standard_normal((B, T, D)).astype(np.float32) * 2.0
    fp, cp, gp = v(), v(), v()
    for a in (fp, cp, gp):
        a[rng.random(a.shape) < 0.1] = 60.0
        a[rng.random(a.shape) < 0.1] = -60.0
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    fb, cb, gb = bf(fp), bf(cp), bf(gp)
    o, hl = mmf.mlgru_scan(fb.to(DEV), cb.to(DEV), gb.to(DEV), None)
    torch.cuda.synchronize()
    o_ref, hl_ref = oracle.mlgru_scan(bits_np(fb), bits_np(cb), bits_np(gb), None)
    ov, rv = bf16_to_f64(bits_np(o.cpu())), bf16_to_f64(o_ref)
    assert np.isfinite(ov).all()
    assert (np.abs(hl.cpu().numpy() - hl_ref) <= 1e-4 * (1.0 + np.abs(hl_ref))).all()
    assert (np.abs(ov - rv) <= np.abs(rv) * 2.0 ** -7 + 1e-6).all()
    big = np.abs(rv) >= 1e-6
    assert big.mean() > 0.5 and (ov[big] == rv[big]).mean() > 0.99


def test_mlgru_scan_continues_across_calls():
    """Two calls over the halves of the tokens, the state carried, give the
    single call's output to fp32 rounding of the state."""
    B, T, D = 2, 300, 256
    rng = np.random.default_rng(7)
    mk = lambda: torch.from_numpy(rng.standard_normal((B, T, D)).astype(np.float32)).to(torch.bfloat16).to(DEV)
    fp, cp, gp = mk(), mk(), mk()
    o, hl = mmf.mlgru_scan(fp, cp, gp)
    o1, h1 = mmf.mlgru_scan(fp[:, :120].contiguous(), cp[:, :120].contiguous(), gp[:, :120].contiguous())
    o2, h2 = mmf.mlgru_scan(fp[:, 120:].contiguous(), cp[:, 120:].contiguous(), gp[:, 120:].contiguous(), h1)
    torch.cuda.synchronize()
    assert torch.allclose(hl, h2, rtol=1e-4, atol=1e-4)
    both = torch.cat([o1, o2], dim=1).float()
    assert ((both - o.float()).abs() <= o.float().abs() * 2.0 ** -7 + 1e-6).all()


# -- backward with the straight-through estimator --------------------------------------------

@pytest.mark.parametrize("M,K,N", [(1, 256, 128), (16, 512, 256), (64, 1024, 296), (300, 384, 1024),
                                   (1000, 2048, 512), (513, 256, 72), (257, 640, 1000)])
def test_bwd_parity(oracle, M, K, N):
    x, g, W = make_layer(24, M, K, N)
    dy = I.activations(24, M, N, index=7)
    packed, scale = _pack(W)
    dx, dg, dW = mmf.bitlinear_bwd(dy.to(DEV), x.to(DEV), g.to(DEV), packed, scale, EPS)
    torch.cuda.synchronize()
    wt, beta = oracle.absmean_ternary(W.numpy(), EPS_W)
    dx_ref, dg_ref, dW_ref = oracle.bitlinear_bwd(bits_np(dy), bits_np(x), g.numpy(), EPS, wt, beta)
    # tensor-core products with fp32 accumulation; x_q = q * absmax / 127 rounded
    # to bf16 for dW: errors well inside the layer's 1e-2 bar, relative to each
    # output's scale
    def rel(a, b):
        b = np.asarray(b, dtype=np.float64)
        return np.abs(np.asarray(a, dtype=np.float64) - b).max() / max(np.abs(b).max(), 1e-30)
    assert rel(bf16_to_f64(bits_np(dx.cpu())), bf16_to_f64(dx_ref)) <= 1e-2
    assert rel(dg.cpu().numpy(), dg_ref) <= 1e-3
    assert rel(dW.cpu().numpy(), dW_ref) <= 1e-2


def test_bwd_dr_exact_on_exact_inputs(oracle):
    """dy with few significant bits and ternary weights: every product and
    partial sum of dr = dy . w~ is exact in fp32, so dx matches the oracle's
    fp64 evaluation to its own bf16 rounding, whatever the order of the sums;
    and dW of one token is dy^T times the token's bf16 x_q exactly."""
    M, K, N = 1, 256, 192
    rng = np.random.default_rng(3)
    x, g, W = make_layer(25, M, K, N)
    dy = torch.from_numpy(rng.integers(-8, 9, size=(M, N)).astype(np.float32)).to(torch.bfloat16)
    packed, scale = _pack(W)
    dx, dg, dW = mmf.bitlinear_bwd(dy.to(DEV), x.to(DEV), g.to(DEV), packed, scale, EPS)
    torch.cuda.synchronize()
    wt, beta = oracle.absmean_ternary(W.numpy(), EPS_W)
    dx_ref, dg_ref, dW_ref = oracle.bitlinear_bwd(bits_np(dy), bits_np(x), g.numpy(), EPS, wt, beta)
    # dW[n][k] = dy[n] * bf16(q[k] * a / 127): one bf16 rounding of x_q, then an exact product
    q, a = oracle.rmsnorm_quant(bits_np(x), g.numpy(), EPS)
    xq = (q[0].astype(np.float32) * (np.float32(a[0]) / np.float32(127.0))).astype(np.float32)
    xq_b = bf16_to_f64(bits_np(torch.from_numpy(xq).to(torch.bfloat16)))
    assert np.array_equal(dW.cpu().numpy().astype(np.float64), np.outer(dy.float().numpy()[0], xq_b))
    # dx: exact dr, then the RMSNorm backward in fp64 (sums in another order): one bf16 step at most
    dxv, dxr = bf16_to_f64(bits_np(dx.cpu())), bf16_to_f64(dx_ref)
    assert (np.abs(dxv - dxr) <= np.abs(dxr) * 2.0 ** -8 + 1e-30).all()
    assert np.abs(dg.cpu().numpy() - dg_ref).max() <= 1e-5 * np.abs(dg_ref).max()


@pytest.mark.parametrize("M,N", [(0, 64), (16, 0)])
def test_bwd_empty_contractions(oracle, M, N):
    """An empty contraction gives zero products: M = 0 (no tokens) gives dW = 0
    and dgamma = 0; N = 0 (no outputs) gives dr = 0, so dx = 0."""
    K = 256
    x = torch.randn(M, K).to(torch.bfloat16).to(DEV)
    g = torch.ones(K, device=DEV)
    packed, scale = mmf.pack_ternary(torch.randn(max(N, 1), K, device=DEV))
    dy = torch.randn(M, N).to(torch.bfloat16).to(DEV)
    dx, dg, dW = mmf.bitlinear_bwd(dy, x, g, packed[:N] if N else packed[:0], scale, EPS)
    torch.cuda.synchronize()
    assert dW.shape == (N, K) and (dW == 0).all()
    assert (dg == 0).all()
    if M:
        assert (dx.float() == 0).all()


def test_bwd_rejects_unaligned_output_width():
    """dy rows are read by TMA: N must be a multiple of 8 (16-byte row pitch)."""
    L = mmf.lib()
    K, M, N = 256, 4, 300
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    p = buf.data_ptr()
    assert L.mmf_bitlinear_bwd(p, p, p, 1e-6, p, p, M, K, N, p, p, p, p, buf.numel(),
                               torch.cuda.current_stream().cuda_stream) == 2   # MMF_ERR_UNSUPPORTED_SHAPE
    mmf.check_async()


def test_empty_problems():
    K, N = 256, 64
    x = torch.zeros(0, K, dtype=torch.bfloat16, device=DEV)
    g = torch.ones(K, device=DEV)
    W = torch.randn(N, K, device=DEV)
    packed, scale = mmf.pack_ternary(W)
    y = mmf.bitlinear_fwd(x, g, packed, scale, N)
    assert y.shape == (0, N)
    y = mmf.bitlinear_fwd(torch.zeros(3, K, dtype=torch.bfloat16, device=DEV), g, packed, scale, 0)
    assert y.shape == (3, 0)
    torch.cuda.synchronize()


def test_fwd_deterministic():
    for M in (1, 64):
        x, g, W = make_layer(13, M, 2048, 1024)
        packed, scale = _pack(W)
        xd, gd = x.to(DEV), g.to(DEV)
        y1 = mmf.bitlinear_fwd(xd, gd, packed, scale, 1024)
        y2 = mmf.bitlinear_fwd(xd, gd, packed, scale, 1024)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2)


# -- grouped projections sharing x -------------------------------------------------------------

@pytest.mark.parametrize("M,K,Ns", [(1, 2560, (2560, 2560, 2560, 2560)), (1, 2560, (6912, 6912)),
                                    (3, 1024, (100, 0, 333, 64)), (8, 512, (128,) * 8),
                                    # decode tensor-core path: slabs of each projection's own, the last
                                    # one partial, an empty projection, K split over clusters or not
                                    (16, 2560, (2560, 100, 6912)), (5, 1024, (0, 257, 64)),
                                    (32, 6912, (2560, 300)), (24, 128, (1000, 3)),
                                    (64, 1024, (300, 129)), (300, 384, (256, 200, 17))])
@pytest.mark.parametrize("flags", [0, 1])
def test_group_matches_single_calls(oracle, M, K, Ns, flags):
    x, g, _ = make_layer(14, M, K, 1)
    xd, gd = x.to(DEV), g.to(DEV)
    weights, Ws = [], []
    for i, N in enumerate(Ns):
        W = make_layer(14, 1, K, max(N, 1), index=i + 1)[2][:N]
        Ws.append(W)
        packed, scale = _pack(W.contiguous()) if N > 0 else (torch.zeros(1, K // 16, dtype=torch.int32, device=DEV),
                                                             torch.ones(1, device=DEV))
        weights.append((packed, scale, N))
    ys = mmf.bitlinear_fwd_group(xd, gd, weights, EPS, flags=flags)
    singles = [mmf.bitlinear_fwd(xd, gd, pk, sc, N, EPS) if N > 0 else None for (pk, sc, N) in weights]
    torch.cuda.synchronize()
    for (pk, sc, N), y, y1, W in zip(weights, ys, singles, Ws):
        assert y.shape == (M, N)
        if N == 0:
            continue
        assert torch.equal(y, y1)
        y_ref, _ = oracle.bitlinear(bits_np(x), g.numpy(), EPS, W.contiguous().numpy(), EPS_W)
        assert y_rel_error(bits_np(y), y_ref) <= Y_REL_TOL


@pytest.mark.parametrize("M", [1, 16])
def test_group_pdl_chain_matches_plain(M):
    """A chain of PDL launches in one stream gives the same bits as plain launches
    (one token: the fused decode kernel; 16: quantiser and tensor-core kernel)."""
    K = 2048
    x, g, _ = make_layer(15, M, K, 1)
    xd, gd = x.to(DEV), g.to(DEV)
    weights = []
    for i in range(6):
        W = make_layer(15, 1, K, 1024, index=i + 1)[2]
        pk, sc = _pack(W)
        weights.append((pk, sc, 1024))
    plain = [mmf.bitlinear_fwd_group(xd, gd, [w], EPS)[0] for w in weights]
    chained = [mmf.bitlinear_fwd_group(xd, gd, [w], EPS, flags=mmf.FWD_PDL)[0] for w in weights]
    torch.cuda.synchronize()
    for a, b in zip(plain, chained):
        assert torch.equal(a, b)


@pytest.mark.parametrize("M", [1, 3, 8, 64])
def test_pdl_dependent_chain(M):
    """Each call's x is the previous call's y: under PDL the kernels fetch weights
    before the previous kernel ends but must read x only after it; the chain gives
    the same bits as ordinary launches."""
    K = 2048
    x, g, _ = make_layer(16, M, K, 1)
    weights = []
    for i in range(8):
        W = make_layer(16, 1, K, K, index=i + 1)[2]
        pk, sc = _pack(W)
        weights.append((pk, sc, K))
    gd = g.to(DEV)
    outs = {}
    for flags in (0, mmf.FWD_PDL):
        cur = x.to(DEV)
        trail = []
        for w in weights:
            cur = mmf.bitlinear_fwd_group(cur, gd, [w], EPS, flags=flags)[0]
            trail.append(cur)
        torch.cuda.synchronize()
        outs[flags] = trail
    for a, b in zip(outs[0], outs[mmf.FWD_PDL]):
        assert torch.equal(a, b)


# -- error paths on the device -----------------------------------------------------------------

def test_argument_errors_on_device():
    K, N = 256, 64
    x = torch.zeros(64, K, dtype=torch.bfloat16, device=DEV)
    g = torch.ones(K, device=DEV)
    packed, scale = mmf.pack_ternary(torch.randn(N, K, device=DEV))
    L = mmf.lib()
    s = torch.cuda.current_stream().cuda_stream
    y = torch.empty(64, N, dtype=torch.bfloat16, device=DEV)
    need = mmf.workspace_bytes(64, K, N)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    assert L.mmf_bitlinear_fwd(x.data_ptr(), g.data_ptr(), 1e-6, packed.data_ptr(), scale.data_ptr(), 64, K, N,
                               y.data_ptr(), ws.data_ptr(), need - 1, s) == 4
    assert L.mmf_bitlinear_fwd(x.data_ptr() + 2, g.data_ptr(), 1e-6, packed.data_ptr(), scale.data_ptr(), 64, K, N,
                               y.data_ptr(), ws.data_ptr(), need, s) == 3
    assert L.mmf_bitlinear_fwd(x.data_ptr(), g.data_ptr(), 1e-6, packed.data_ptr(), scale.data_ptr(), 64, 200, N,
                               y.data_ptr(), ws.data_ptr(), need, s) == 2
    assert L.mmf_bitlinear_fwd(x.data_ptr(), g.data_ptr(), 1e-6, packed.data_ptr(), scale.data_ptr(), 64, K, N,
                               y.data_ptr(), ws.data_ptr(), need, s) == 0
    mmf.check_async()


def test_timeout_is_reported_not_hung():
    """A bounded wait on a barrier nothing arrives at gives up, is reported by
    mmf_check_async as MMF_ERR_TIMEOUT, and leaves the context usable."""
    mmf.check_async()
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    mmf.selftest_timeout(20_000_000, flag)  # 20 ms
    with pytest.raises(mmf.MMFError) as e:
        mmf.check_async()
    assert e.value.status == 6
    assert int(flag[0]) == 1
    mmf.check_async()                        # cleared
    a = torch.arange(1024, dtype=torch.float32, device=DEV)
    b = torch.empty_like(a)
    mmf.hbm_copy(a, b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_hbm_copy():
    a = torch.randint(0, 1 << 30, (1 << 22,), dtype=torch.int32, device=DEV)
    b = torch.empty_like(a)
    mmf.hbm_copy(a, b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
