"""Checks that pin the CPU oracle to facts other than itself.

Each ``check_*`` function raises AssertionError when the oracle it is given is
wrong.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` plants a plausible mistake in a scratch copy of the
oracle source and shows that at least one check fails for it.

What pins what (no page prints a worked numeric example of BitLinear, so the
pins are closed forms, invariants, library routines on special cases, the
quantisers' error bounds and hand-worked tiny cases):
  bf16 rounding      torch's fp32->bf16 conversion (library routine), exact ties
  absmean codes      ties-to-even worked cases, scale homogeneity, sign symmetry,
                     W = c*I, library mean, Gaussian zero fraction 2*Phi(sqrt(2/pi)/2)-1
  packing            hand-placed words of the storage format, round trip
  rmsnorm + quant    hand-worked case, exact ties, constant rows, zero row,
                     homogeneity, torch rms_norm within the quantiser's half step
  ternary acc        numpy int64 matmul, exhaustive 3^4 weight rows, zero-weight
                     invariance, identity, all-ones
  rescale            exact powers of two, torch bf16 conversion within one ulp
  whole layer        fp64 dense product of the normalised activations with the
                     ternary weights, within the activation quantiser's bound
  GLU gated product  scipy's logistic function (fp64) within one bf16 rounding,
                     exact zeros, SiLU(v) - SiLU(-v) = v, saturation
  MLGRU recurrence   closed form for constant gates and inputs, forgetting and
                     keeping limits, continuation across calls, independence
  STE backward       central differences of the surrogate forward (dx, dgamma),
                     matmul with the quantised activations (dW), linearity in dy
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _bits_of(x_f32: np.ndarray) -> np.ndarray:
    """fp32 values that are exact in bf16 -> bf16 bit patterns."""
    x_f32 = np.ascontiguousarray(x_f32, dtype=np.float32)
    u = x_f32.view(np.uint32)
    assert ((u & 0xFFFF) == 0).all(), "value not exact in bf16"
    return (u >> 16).astype(np.uint16)


def _torch_bf16_bits(v_f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rand_bf16_x(rng, M, K, scale=1.0):
    x = (rng.standard_normal((M, K)) * scale).astype(np.float32)
    return _torch_bf16_bits(x)


# -- bf16 rounding ----------------------------------------------------------------

def check_bf16_rounding(orc):
    rng = np.random.default_rng(11)
    v = (rng.standard_normal(3000) * 10.0 ** rng.integers(-38, 37, 3000)).astype(np.float32)
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0xBF818000, 0x00008000,
                     0x00018000, 0x7F7F8000, 0x4B7F8000, 0x3F80C000, 0x3F804000],
                    dtype=np.uint32).view(np.float32)
    v = np.concatenate([v, ties, np.array([0.0, -0.0, 1e-45, -3e38], np.float32)])
    got = orc.f64_to_bf16_array(v.astype(np.float64))
    ref = _torch_bf16_bits(v)
    assert (got == ref).all(), f"bf16 rounding differs at {np.nonzero(got != ref)[0][:5]}"


# -- absmean ternarisation ----------------------------------------------------------

def check_absmean_worked_ties(orc):
    # mean|W| = 1 exactly and eps_w = 0, so the codes are rint(W) clipped:
    # 0.5 -> 0 and -0.5 -> 0 (ties to even), 1.5 -> 2 -> 1.
    wt, beta = orc.absmean_ternary(np.array([[0.5, -0.5, 1.5, 1.5]], np.float32), 0.0)
    assert beta == np.float32(1.0)
    assert wt.tolist() == [[0, 0, 1, 1]]
    # 0.25 -> 0, 0.75 -> 1, -0.75 -> -1, -2.25 -> -2 -> -1; mean|W| = 4/4 = 1
    wt, beta = orc.absmean_ternary(np.array([[0.25, 0.75, -0.75, -2.25]], np.float32), 0.0)
    assert beta == np.float32(1.0)
    assert wt.tolist() == [[0, 1, -1, -1]]
    # mean|W| = 0.5: W/beta = [0.4, 1.2, -0.2, -2.2] -> [0, 1, 0, -1]
    wt, beta = orc.absmean_ternary(np.array([[0.2, 0.6, -0.1, -1.1]], np.float32), 0.0)
    assert beta == np.float32(0.5)
    assert wt.tolist() == [[0, 1, 0, -1]]


def check_absmean_invariants(orc):
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((24, 64)) * 0.02).astype(np.float32)
    wt, beta = orc.absmean_ternary(W, 0.0)
    # library mean of |W| in fp64 (numpy's pairwise sum), rounded to fp32
    assert beta == np.float32(np.mean(np.abs(W.astype(np.float64))))
    # scale homogeneity for powers of two (exact in fp32)
    for c in (2.0 ** -3, 2.0 ** 5):
        wt2, beta2 = orc.absmean_ternary((W * np.float32(c)).astype(np.float32), 0.0)
        assert (wt2 == wt).all()
        assert beta2 == np.float32(beta * np.float32(c))
    # sign symmetry
    wt3, beta3 = orc.absmean_ternary(-W, 0.0)
    assert (wt3 == -wt).all() and beta3 == beta
    # W = c*I: beta = c/K, W/beta = K on the diagonal -> codes = I
    K = 32
    wt4, beta4 = orc.absmean_ternary((np.eye(K) * 0.75).astype(np.float32), 1e-5)
    assert (wt4 == np.eye(K, dtype=np.int8)).all()
    assert beta4 == np.float32(0.75 / K)
    # eps_w enters the divisor: with eps_w = beta the threshold doubles
    wt5, _ = orc.absmean_ternary(np.array([[0.25, 0.75, -0.75, -2.25]], np.float32), 1.0)
    assert wt5.tolist() == [[0, 0, 0, -1]]       # W/2 = [0.125, 0.375, -0.375, -1.125]


def check_absmean_gaussian_fraction(orc):
    # For Gaussian W, beta -> sigma*sqrt(2/pi) and a weight rounds to 0 when
    # |W| < beta/2, so P(0) = 2*Phi(sqrt(2/pi)/2) - 1 = erf(sqrt(2/pi)/(2*sqrt 2)).
    rng = np.random.default_rng(13)
    W = (rng.standard_normal((256, 256)) * 0.02).astype(np.float32)
    wt, beta = orc.absmean_ternary(W, 1e-5)
    p0 = math.erf(math.sqrt(2.0 / math.pi) / 2.0 / math.sqrt(2.0))
    n = wt.size
    tol = 5.0 * math.sqrt(p0 * (1 - p0) / n)
    assert abs(float((wt == 0).mean()) - p0) < tol, ((wt == 0).mean(), p0)
    for v in (1, -1):
        assert abs(float((wt == v).mean()) - (1 - p0) / 2) < tol
    assert abs(float(beta) - 0.02 * math.sqrt(2 / math.pi)) < 0.02 * 0.01


# -- packing ------------------------------------------------------------------------

def check_packing_words(orc):
    # Hand-placed words: every 2-bit field holds code = w + 1, so an all-zero
    # group of 16 is 0x55555555.  Weight i of a group sits at bit
    # 8*(i%4) + 2*(i//4): i=0 -> bit 0, i=1 -> bit 8, i=3 -> bit 24,
    # i=4 -> bit 2, i=15 -> bit 30.
    def word(vals):
        wt = np.zeros((1, 16), np.int8)
        for i, v in vals:
            wt[0, i] = v
        return int(orc.encode_packed(wt)[0, 0])

    assert word([]) == 0x55555555
    assert word([(0, 1)]) == 0x55555556
    assert word([(1, 1)]) == 0x55555655
    assert word([(3, 1)]) == 0x56555555
    assert word([(4, 1)]) == 0x55555559
    assert word([(15, 1)]) == 0x95555555
    assert word([(0, -1)]) == 0x55555554
    assert word([(15, -1)]) == 0x15555555
    assert word([(i, 1) for i in range(16)]) == 0xAAAAAAAA
    assert word([(i, -1) for i in range(16)]) == 0x00000000
    # round trip and row layout (word j of row n covers k = 16j .. 16j+15)
    rng = np.random.default_rng(14)
    wt = rng.integers(-1, 2, size=(5, 48)).astype(np.int8)
    p = orc.encode_packed(wt)
    assert p.shape == (5, 3)
    back, bad = orc.decode_packed(p, 48)
    assert bad == 0 and (back == wt).all()
    wt1 = np.zeros((2, 32), np.int8)
    wt1[1, 17] = 1                                  # row 1, word 1, i = 1
    p1 = orc.encode_packed(wt1)
    assert p1.tolist() == [[0x55555555, 0x55555555], [0x55555555, 0x55555655]]
    _, bad = orc.decode_packed(np.full((1, 1), 0xFFFFFFFF, np.uint32), 16)
    assert bad == 16


# -- RMSNorm + absmax int8 ------------------------------------------------------------

def check_quant_worked(orc):
    # x = [1, -2, 2, 4], gamma = 1, eps = 0: mean square 25/4 = 6.25, inv = 0.4,
    # r = [0.4, -0.8, 0.8, 1.6] (fp32), absmax 1.6, s = 127/1.6 = 79.375,
    # r*s = [31.75, -63.5, 63.5, 127] in fp32 -> q = [32, -64, 64, 127].
    x = _bits_of(np.array([[1, -2, 2, 4]], np.float32))
    q, a = orc.rmsnorm_quant(x, np.ones(4, np.float32), 0.0)
    assert q.tolist() == [[32, -64, 64, 127]]
    assert a[0] == np.float32(1.6)
    # Exact ties: x = 2 everywhere gives mean square 4 and inv = 0.5 exactly, so
    # r = gamma exactly; gamma[0] = 127 makes absmax 127 and s = 1, so
    # q = rint(gamma) with ties to even: 62.5 -> 62, 0.5 -> 0, 1.5 -> 2, -2.5 -> -2.
    g = np.array([127, 62.5, -62.5, 0.5, 1.5, -2.5, 3.5, 0.25], np.float32)
    x = _bits_of(np.full((1, 8), 2.0, np.float32))
    q, a = orc.rmsnorm_quant(x, g, 0.0)
    assert q.tolist() == [[127, 62, -62, 0, 2, -2, 4, 0]]
    assert a[0] == np.float32(127.0)


def check_quant_special_rows(orc):
    K = 128
    g = np.ones(K, np.float32)
    for c in (0.5, -3.0, 100.0):
        x = _bits_of(np.full((1, K), c, np.float32))
        q, _ = orc.rmsnorm_quant(x, g, 1e-6)
        assert (q == (127 if c > 0 else -127)).all()
    q, a = orc.rmsnorm_quant(np.zeros((2, K), np.uint16), g, 1e-6)
    assert (q == 0).all() and (a == np.float32(1e-5)).all()


def check_quant_homogeneity(orc):
    rng = np.random.default_rng(15)
    x = _rand_bf16_x(rng, 6, 256)
    g = (1.0 + 0.1 * rng.standard_normal(256)).astype(np.float32)
    q, a = orc.rmsnorm_quant(x, g, 0.0)
    xf = _bf16_bits_to_f64(x).astype(np.float32)
    for c in (2.0 ** -4, 2.0 ** 6):
        q2, a2 = orc.rmsnorm_quant(_bits_of(xf * np.float32(c)), g, 0.0)
        assert (q2 == q).all() and (a2 == a).all()
    # gamma scaled by a power of two scales absmax, not the codes
    q3, a3 = orc.rmsnorm_quant(x, g * np.float32(4.0), 0.0)
    assert (q3 == q).all() and (a3 == a * np.float32(4.0)).all()
    # every nonzero row reaches the full code range
    assert (np.abs(q).max(axis=1) == 127).all()


def check_quant_vs_rms_norm(orc):
    # torch's rms_norm in fp64 gives r; the quantiser must land within half a
    # step (absmax/254) of it, and absmax must match max|r|.
    rng = np.random.default_rng(16)
    for eps, scale in ((1e-6, 1.0), (0.5, 0.3)):
        x = _rand_bf16_x(rng, 5, 512, scale)
        g = (1.0 + 0.1 * rng.standard_normal(512)).astype(np.float32)
        q, a = orc.rmsnorm_quant(x, g, eps)
        xt = torch.from_numpy(_bf16_bits_to_f64(x))
        r = torch.nn.functional.rms_norm(xt, (512,), weight=torch.from_numpy(g.astype(np.float64)),
                                         eps=eps).numpy()
        amax = np.abs(r).max(axis=1)
        assert np.allclose(a, amax, rtol=1e-6, atol=0)
        err = np.abs(q.astype(np.float64) * (a[:, None] / 127.0) - r)
        # half a step, plus the fp32 rounding of r (a few ulp of absmax)
        assert (err <= a[:, None] * (1.0 / 254.0 + 1e-6)).all()


# -- ternary accumulation ------------------------------------------------------------

def check_acc_vs_matmul(orc):
    rng = np.random.default_rng(17)
    for M, K, N in ((3, 64, 5), (7, 256, 9), (1, 48, 2)):
        q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
        wt = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        acc = orc.ternary_acc(q, wt)
        ref = q.astype(np.int64) @ wt.astype(np.int64).T
        assert acc.shape == (M, N) and (acc == ref).all()


def check_acc_exhaustive_small(orc):
    # all 3^4 ternary rows against a few activation rows, by a products formula
    import itertools
    wt = np.array(list(itertools.product((-1, 0, 1), repeat=4)), np.int8)
    q = np.array([[127, -127, 1, 0], [-5, 7, -11, 13], [127, 127, 127, 127]], np.int8)
    acc = orc.ternary_acc(q, wt)
    for m in range(q.shape[0]):
        for n in range(wt.shape[0]):
            assert acc[m, n] == sum(int(wt[n, k]) * int(q[m, k]) for k in range(4))


def check_acc_invariants(orc):
    rng = np.random.default_rng(18)
    K = 128
    q = rng.integers(-127, 128, size=(4, K)).astype(np.int8)
    wt = rng.integers(-1, 2, size=(6, K)).astype(np.int8)
    acc = orc.ternary_acc(q, wt)
    # changing q where a row's weight is 0 leaves that row's result alone
    for n in range(6):
        q2 = q.copy()
        z = wt[n] == 0
        q2[:, z] = rng.integers(-127, 128, size=(4, int(z.sum()))).astype(np.int8)
        assert (orc.ternary_acc(q2, wt[n:n + 1])[:, 0] == acc[:, n]).all()
    eye = np.eye(K, dtype=np.int8)
    assert (orc.ternary_acc(q, eye) == q.astype(np.int32)).all()
    ones = np.ones((1, K), np.int8)
    assert (orc.ternary_acc(q, ones)[:, 0] == q.astype(np.int64).sum(axis=1)).all()
    assert (orc.ternary_acc(q, -ones)[:, 0] == -q.astype(np.int64).sum(axis=1)).all()


# -- rescale -------------------------------------------------------------------------

def check_rescale(orc):
    # absmax = 127 * 2^-3 and beta = 0.5 make the factor exactly 2^-4
    acc = np.array([[16, -32, 0, 1, 786432]], np.int32)
    y = orc.rescale(acc, np.array([127.0 / 8], np.float32), 0.5)
    assert y[0].tolist() == _bits_of(np.array([1.0, -2.0, 0.0, 0.0625, 49152.0], np.float32)).tolist()
    rng = np.random.default_rng(19)
    acc = rng.integers(-800000, 800000, size=(4, 64)).astype(np.int32)
    a = np.abs(rng.standard_normal(4)).astype(np.float32) + np.float32(0.1)
    beta = np.float32(0.0157)
    y = orc.rescale(acc, a, beta)
    exact = acc.astype(np.float64) * (a.astype(np.float64)[:, None] / 127.0) * float(beta)
    ref = _torch_bf16_bits(exact.astype(np.float32))    # exact -> fp32 -> bf16
    yv = _bf16_bits_to_f64(y)
    rv = _bf16_bits_to_f64(ref)
    ulp = np.abs(rv) * 2.0 ** -7
    assert (np.abs(yv - rv) <= ulp).all()
    assert (y == ref).mean() > 0.98
    assert (np.abs(yv - exact) <= np.abs(exact) * 2.0 ** -8 * (1 + 1e-9)).all()


# -- whole layer ---------------------------------------------------------------------

def check_layer_bound(orc):
    # |y - (r . W~^T) beta| <= nnz_n * (absmax/254) * beta + bf16 rounding,
    # with r from torch's fp64 rms_norm and the product by numpy.
    rng = np.random.default_rng(20)
    M, K, N = 6, 256, 40
    x = _rand_bf16_x(rng, M, K)
    g = (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    y, beta = orc.bitlinear(x, g, 1e-6, W, 1e-5)
    wt, beta2 = orc.absmean_ternary(W, 1e-5)
    assert beta2 == beta
    r = torch.nn.functional.rms_norm(torch.from_numpy(_bf16_bits_to_f64(x)), (K,),
                                     weight=torch.from_numpy(g.astype(np.float64)), eps=1e-6).numpy()
    ref = (r @ wt.astype(np.float64).T) * float(beta)
    amax = np.abs(r).max(axis=1)
    nnz = (wt != 0).sum(axis=1)
    bound = amax[:, None] * (1.0 / 254.0 + 1e-6) * nnz[None, :] * float(beta)
    yv = _bf16_bits_to_f64(y)
    assert (np.abs(yv - ref) <= bound + np.abs(yv) * 2.0 ** -8 + 1e-12).all()


def check_glu_gate(orc):
    """SiLU(g) * u against an independent SiLU (scipy's logistic function, in
    fp64) within one bf16 rounding; exact zeros; the odd-part identity
    SiLU(v) - SiLU(-v) = v; saturation for large |g|."""
    from scipy.special import expit

    rng = np.random.default_rng(31)
    g = _torch_bf16_bits(rng.standard_normal(4096).astype(np.float32) * 3.0)
    u = _torch_bf16_bits(rng.standard_normal(4096).astype(np.float32))
    p = _bf16_bits_to_f64(orc.glu_gate(g, u))
    gv, uv = _bf16_bits_to_f64(g), _bf16_bits_to_f64(u)
    ref = gv * expit(gv) * uv
    # one bf16 rounding (2^-8 relative) plus the fp32 steps before it
    assert (np.abs(p - ref) <= np.abs(ref) * (2.0 ** -8 + 2.0 ** -20) + 1e-30).all()
    # SiLU(0) = +0 * sigma(0) = +0, and +0 * u is a zero carrying the sign of u
    # (IEEE product sign rule): the exact bit pattern, not only the value
    z = np.zeros(64, dtype=np.uint16)
    want = np.where(np.signbit(_bf16_bits_to_f64(u[:64])), 0x8000, 0x0000).astype(np.uint16)
    assert np.array_equal(orc.glu_gate(z, u[:64]), want)
    # u = +0 gives a zero of g's sign (SiLU(g) has the sign of g)
    pz = orc.glu_gate(g[:64], np.zeros(64, dtype=np.uint16))
    assert (_bf16_bits_to_f64(pz) == 0).all()
    assert np.array_equal(np.signbit(_bf16_bits_to_f64(pz)), np.signbit(_bf16_bits_to_f64(g[:64])))
    # SiLU(v) - SiLU(-v) = v, with u = 1: within two bf16 roundings
    one = _bits_of(np.ones(256, dtype=np.float32))
    gp = _bits_of(np.linspace(-8, 8, 256).astype(np.float32).astype(np.float64).astype(np.float32)
                  .view(np.uint32).__and__(0xFFFF0000).view(np.float32))
    gn = _bits_of(-_bf16_bits_to_f64(gp).astype(np.float32))
    d = _bf16_bits_to_f64(orc.glu_gate(gp, one)) - _bf16_bits_to_f64(orc.glu_gate(gn, one))
    v = _bf16_bits_to_f64(gp)
    assert (np.abs(d - v) <= np.abs(v) * 2.0 ** -7 + 1e-30).all()
    # saturation: SiLU(30) = 30 to fp32 precision; SiLU(-30) is about -2.8e-12
    big = _bits_of(np.array([30.0, -30.0], dtype=np.float32))
    pb = _bf16_bits_to_f64(orc.glu_gate(big, _bits_of(np.array([2.0, 2.0], dtype=np.float32))))
    assert pb[0] == 60.0 and -1e-10 < pb[1] < 0.0


def check_mlgru_scan(orc):
    """The recurrence against closed forms: constant gates and inputs give
    h_t = c + f^t (h0 - c); f -> 0 forgets (h_t = SiLU(c_t)); f -> 1 keeps h0;
    the output gate at 0 pre-activation halves h; sequences and channels are
    independent; h_last continues the recurrence across calls."""
    B, T, D = 2, 40, 3

    def bits(v):
        return _bits_of(np.full((B, T, D), v, dtype=np.float32))

    sig = lambda v: 1.0 / (1.0 + math.exp(-v))
    # constant f_pre = 0.5, c_pre = 2.0, g_pre = 0: closed form
    h0 = np.array([[1.5, -2.0, 0.0], [4.0, 0.25, -1.0]], dtype=np.float32)
    o, hl = orc.mlgru_scan(bits(0.5), bits(2.0), bits(0.0), h0)
    f, c = sig(0.5), 2.0 * sig(2.0)
    for t in range(T):
        ref = c + f ** (t + 1) * (h0.astype(np.float64) - c)
        assert np.allclose(_bf16_bits_to_f64(o[:, t, :]), 0.5 * ref, rtol=2.0 ** -7, atol=1e-6)
    assert np.allclose(hl, c + f ** T * (h0.astype(np.float64) - c), rtol=1e-5, atol=1e-6)
    # f -> 0 (f_pre = -64): no memory, h_t = SiLU(c_t); f -> 1 (f_pre = 64): h stays h0
    rng = np.random.default_rng(41)
    cb = _torch_bf16_bits(rng.standard_normal((B, T, D)).astype(np.float32))
    o, hl = orc.mlgru_scan(bits(-64.0), cb, bits(64.0), h0)
    cv = _bf16_bits_to_f64(cb)
    assert np.allclose(_bf16_bits_to_f64(o), cv / (1.0 + np.exp(-cv)), rtol=2.0 ** -7, atol=1e-30)
    o, hl = orc.mlgru_scan(bits(64.0), cb, bits(64.0), h0)
    assert np.allclose(_bf16_bits_to_f64(o), np.broadcast_to(h0[:, None, :], (B, T, D)), rtol=2.0 ** -7)
    assert np.array_equal(hl, h0)
    # independence and continuation: two halves with h_last carried equal one call
    fb = _torch_bf16_bits(rng.standard_normal((B, T, D)).astype(np.float32))
    gb = _torch_bf16_bits(rng.standard_normal((B, T, D)).astype(np.float32))
    o_all, h_all = orc.mlgru_scan(fb, cb, gb, h0)
    o1, h1 = orc.mlgru_scan(fb[:, :17], cb[:, :17], gb[:, :17], h0)
    o2, h2 = orc.mlgru_scan(fb[:, 17:], cb[:, 17:], gb[:, 17:], h1)
    assert np.array_equal(o_all, np.concatenate([o1, o2], axis=1)) and np.array_equal(h_all, h2)
    o_b1, _ = orc.mlgru_scan(fb[1:], cb[1:], gb[1:], h0[1:])
    assert np.array_equal(o_all[1:], o_b1)


def check_bitlinear_bwd(orc):
    """The straight-through backward against central differences of the
    surrogate forward y = (RMSNorm(x) gamma) . W_q^T in fp64 (x and gamma
    perturbed, quantisers absent), dW against the matmul with the quantised
    activations, zeros for dy = 0 and exact doubling for 2 dy."""
    rng = np.random.default_rng(51)
    M, K, N, eps = 3, 16, 5, 1e-6
    xb = _torch_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    dyb = _torch_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    g = (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    wt = rng.integers(-1, 2, (N, K)).astype(np.int8)
    beta = np.float32(0.0175)
    dx, dg, dW = orc.bitlinear_bwd(dyb, xb, g, eps, wt, beta)
    xv, dy = _bf16_bits_to_f64(xb), _bf16_bits_to_f64(dyb)
    Wq = wt.astype(np.float64) * float(beta)

    def loss(x, gamma):
        inv = 1.0 / np.sqrt((x * x).mean(axis=1, keepdims=True) + eps)
        return float(((x * inv * gamma) @ Wq.T * dy).sum())

    h = 1e-6
    num_dx = np.zeros((M, K))
    num_dg = np.zeros(K)
    for m in range(M):
        for k in range(K):
            e = np.zeros((M, K))
            e[m, k] = h
            num_dx[m, k] = (loss(xv + e, g.astype(np.float64)) - loss(xv - e, g.astype(np.float64))) / (2 * h)
    for k in range(K):
        e = np.zeros(K)
        e[k] = h
        num_dg[k] = (loss(xv, g + e) - loss(xv, g - e)) / (2 * h)
    dxv = _bf16_bits_to_f64(dx)
    assert np.allclose(dxv, num_dx, rtol=2.0 ** -7, atol=1e-6)
    assert np.allclose(dg, num_dg, rtol=1e-5, atol=1e-6)
    q, a = orc.rmsnorm_quant(xb, g, eps)
    xq = q.astype(np.float64) * (a.astype(np.float64)[:, None] / 127.0)
    assert np.allclose(dW, dy.T @ xq, rtol=1e-6, atol=1e-9)
    zero = np.zeros_like(dyb)
    dx0, dg0, dW0 = orc.bitlinear_bwd(zero, xb, g, eps, wt, beta)
    assert (_bf16_bits_to_f64(dx0) == 0).all() and (dg0 == 0).all() and (dW0 == 0).all()
    dy2 = _bits_of(2.0 * _bf16_bits_to_f64(dyb).astype(np.float32))
    dx2, dg2, dW2 = orc.bitlinear_bwd(dy2, xb, g, eps, wt, beta)
    assert np.array_equal(_bf16_bits_to_f64(dx2), 2.0 * dxv) and np.array_equal(dg2, 2.0 * dg)
    assert np.array_equal(dW2, 2.0 * dW)


ALL_CHECKS = [
    check_bf16_rounding,
    check_absmean_worked_ties,
    check_absmean_invariants,
    check_absmean_gaussian_fraction,
    check_packing_words,
    check_quant_worked,
    check_quant_special_rows,
    check_quant_homogeneity,
    check_quant_vs_rms_norm,
    check_acc_vs_matmul,
    check_acc_exhaustive_small,
    check_acc_invariants,
    check_rescale,
    check_layer_bound,
    check_glu_gate,
    check_mlgru_scan,
    check_bitlinear_bwd,
]
