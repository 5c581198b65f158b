"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test compares the oracle to something it does not compute: figures the
pages print, exact rational arithmetic, closed forms, or a library routine
(torch / numpy) on tiny shapes. A dropped term, a wrong sign, a transposed
index or a wrong nibble order in the oracle fails at least one of them.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import fixtures
import oracle
from fixtures import gen

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# ---------------------------------------------------------------- helpers (independent of the oracle)
def bf16_exact(bits: int) -> Fraction:
    """Exact rational value of a bf16 bit pattern (finite, normal or subnormal)."""
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        return sign * Fraction(m, 1 << 7) * Fraction(1, 1 << 126)
    v = Fraction(128 + m, 128)
    return sign * (v * (Fraction(2) ** (e - 127)))


def codes_by_bitstring(words: np.ndarray, bits: int) -> np.ndarray:
    """Unpack one row of packed words by reading a binary string (LSB-first fields)."""
    out = []
    for w in words.tolist():
        s = format(int(w), "032b")[::-1]          # s[i] = bit i
        for f in range(32 // bits):
            field = s[f * bits:(f + 1) * bits][::-1]
            out.append(int(field, 2))
    return np.array(out, dtype=np.int64)


def dense_by_bitstring(q, s, b, K, G, bits):
    R = q.shape[0]
    W = np.empty((R, K))
    sf = gen.bf16_bits_to_f32(s).astype(np.float64)
    bf = gen.bf16_bits_to_f32(b).astype(np.float64)
    for r in range(R):
        c = codes_by_bitstring(q[r], bits)
        W[r] = c * np.repeat(sf[r], G) + np.repeat(bf[r], G)
    return W


def rand_mat(rng, R, K, G, bits, sigma=0.02, bias_mode="centred"):
    q = rng.integers(0, 2 ** 32, size=(R, K * bits // 32), dtype=np.uint64).astype(np.uint32)
    s = gen.f32_to_bf16_bits(np.abs(rng.normal(0, sigma, size=(R, K // G))).astype(np.float32))
    if bias_mode == "centred":
        b = gen.biases_from_scales(s, bits)
    else:
        b = gen.f32_to_bf16_bits(rng.normal(0, sigma, size=(R, K // G)).astype(np.float32))
    return q, s, b


def bf16_vec(rng, n, sigma=1.0):
    return gen.f32_to_bf16_bits(rng.normal(0, sigma, size=n).astype(np.float32))


# ---------------------------------------------------------------- storage layout vs the pages' byte counts
def test_expert_bytes_match_pages(golden_facts):
    cfg = fixtures.CONFIGS["layer_q4"]
    ex = fixtures.host_expert(cfg, 0, 3)
    nbytes = sum(a.nbytes for m in ex for a in m)
    # about 6.75 MB per active expert at 4 bits (SSD Expert Streaming)
    assert nbytes == 7_077_888
    assert nbytes / 2 ** 20 == golden_facts["expert_mb_4bit"]
    assert cfg.E == golden_facts["experts_per_layer"] and cfg.H == golden_facts["hidden"]
    assert cfg.k + 1 == golden_facts["active_per_token"]


def test_two_bit_bytes_match_table3(golden_facts):
    cfg = fixtures.CONFIGS["layer_q2"]
    ex = fixtures.host_expert(cfg, 0, 1)
    nbytes = sum(a.nbytes for m in ex for a in m)
    assert nbytes == 3_932_160
    per_token = nbytes * golden_facts["active_per_token"] * golden_facts["layers"]
    # 943 MB/token at K=4, quoted from the write-up's Table 3
    assert abs(per_token / 1e6 - golden_facts["io_mb_per_token_k4"]) < 1.0
    # and the SSD ceiling 17.5 GB/s / 943.7 MB ~ 18.5, printed as 18.6 tok/s
    ceiling = golden_facts["ssd_gbs"] * 1e9 / per_token
    assert abs(ceiling - golden_facts["theoretical_tok_s"]) / golden_facts["theoretical_tok_s"] < 0.01


# ---------------------------------------------------------------- dequant GEMV
@pytest.mark.parametrize("bits", [4, 2])
def test_fma_reordering_identity_exact(bits):
    """(q*s + b)*x summed over a group equals the reordered fma(q, s*x, b*x)
    (FMA-optimised dequant kernel) exactly in rational arithmetic; the oracle
    must agree with that exact value to fp64 rounding."""
    rng = np.random.default_rng(11 + bits)
    K, G = 128, 64
    q, s, b = rand_mat(rng, 3, K, G, bits, bias_mode="free")
    x = rng.normal(size=K)
    y = oracle.qgemv(q, s, b, x, K, G, bits)
    for r in range(3):
        codes = codes_by_bitstring(q[r], bits)
        exact_naive = Fraction(0)
        exact_fma = Fraction(0)
        for k in range(K):
            sv, bv, xv = bf16_exact(int(s[r, k // G])), bf16_exact(int(b[r, k // G])), Fraction(float(x[k]))
            exact_naive += (codes[k] * sv + bv) * xv
            exact_fma += codes[k] * (sv * xv) + bv * xv
        assert exact_naive == exact_fma
        bound = 1e-13 * sum(abs(float(c) * float(bf16_exact(int(s[r, k // G])))) * abs(x[k]) + abs(float(bf16_exact(int(b[r, k // G])))) * abs(x[k])
                            for k, c in enumerate(codes))
        assert abs(Fraction(float(y[r])) - exact_naive) <= Fraction(bound)


@pytest.mark.parametrize("bits", [4, 2])
def test_qgemv_vs_torch_float64(bits):
    rng = np.random.default_rng(3 + bits)
    R, K, G = 37, 256, 64
    q, s, b = rand_mat(rng, R, K, G, bits, bias_mode="free")
    x = rng.normal(size=K)
    W = dense_by_bitstring(q, s, b, K, G, bits)
    ref = (torch.from_numpy(W) @ torch.from_numpy(x)).numpy()
    y = oracle.qgemv(q, s, b, x, K, G, bits)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(oracle.dequant(q, s, b, K, G, bits), W)


@pytest.mark.parametrize("bits", [4, 2])
def test_one_hot_x_reads_one_column_lsb_first(bits):
    """A word whose fields count up 0,1,2,... LSB first; x = e_k must return code(k)*s + b."""
    per = 32 // bits
    word = 0
    for f in range(per):
        word |= (f % (1 << bits)) << (bits * f)
    R, K, G = 2, 64, 64
    q = np.full((R, K // per), word, dtype=np.uint32)
    s = gen.f32_to_bf16_bits(np.array([[0.5], [0.25]], dtype=np.float32))
    b = gen.f32_to_bf16_bits(np.array([[-1.0], [3.0]], dtype=np.float32))
    for k in (0, 1, per - 1, per, K - 1):
        x = np.zeros(K); x[k] = 1.0
        y = oracle.qgemv(q, s, b, x, K, G, bits)
        code = (k % per) % (1 << bits)
        assert y[0] == code * 0.5 - 1.0
        assert y[1] == code * 0.25 + 3.0


def test_scale_and_bias_index_by_row_and_group():
    R, K, G, bits = 3, 256, 64, 4
    q = np.full((R, K // 8), 0x11111111, dtype=np.uint32)       # every code = 1
    sv = np.arange(1, R * (K // G) + 1, dtype=np.float32).reshape(R, K // G)   # distinct per (r, g)
    s = gen.f32_to_bf16_bits(sv)
    b = gen.f32_to_bf16_bits(-sv / 4)
    for r in range(R):
        for g in range(K // G):
            x = np.zeros(K); x[g * G + 5] = 1.0
            y = oracle.qgemv(q, s, b, x, K, G, bits)
            assert y[r] == sv[r, g] - sv[r, g] / 4


def test_zero_scale_leaves_group_bias_times_group_sum():
    rng = np.random.default_rng(5)
    R, K, G, bits = 4, 192, 64, 4
    q, _, b = rand_mat(rng, R, K, G, bits, bias_mode="free")
    s = np.zeros((R, K // G), dtype=np.uint16)
    x = rng.normal(size=K)
    y = oracle.qgemv(q, s, b, x, K, G, bits)
    Xg = x.reshape(K // G, G).sum(axis=1)
    ref = gen.bf16_bits_to_f32(b).astype(np.float64) @ Xg
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


def test_qgemv_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.qgemv(np.zeros((1, 2), np.uint32), np.zeros((1, 1), np.uint16), np.zeros((1, 1), np.uint16),
                     np.zeros(16), 16, 64, 4)       # K not a multiple of G


# ---------------------------------------------------------------- SwiGLU, sigmoid
def test_silu_known_values_and_library():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(1.0) - 0.7310585786300049) < 1e-16
    assert abs(oracle.silu(-30.0)) < 1e-11
    assert oracle.sigmoid(0.0) == 0.5
    rng = np.random.default_rng(0)
    g, u = rng.normal(size=100) * 4, rng.normal(size=100)
    ref = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    np.testing.assert_allclose(oracle.swiglu(g, u), ref, rtol=1e-14, atol=1e-15)
    # gate and up are not interchangeable
    assert not np.allclose(oracle.swiglu(u, g), ref)


# ---------------------------------------------------------------- router
def test_router_logits_order_and_weights_vs_library():
    rng = np.random.default_rng(7)
    T, H, E, k = 5, 128, 24, 3
    x = bf16_vec(rng, T * H).reshape(T, H)
    Wr = bf16_vec(rng, E * H, 0.05).reshape(E, H)
    bias = rng.normal(size=E).astype(np.float32)
    gs = bf16_vec(rng, H, 0.05)
    idx, w, sg, logits = oracle.route(x, Wr, k, bias=bias, gs=gs, want_logits=True)
    xf = torch.from_numpy(gen.bf16_bits_to_f32(x).astype(np.float64))
    Wf = torch.from_numpy(gen.bf16_bits_to_f32(Wr).astype(np.float64))
    ref_logits = (xf @ Wf.T).numpy() + bias.astype(np.float64)
    np.testing.assert_allclose(logits, ref_logits, rtol=1e-13, atol=1e-13)
    p = torch.softmax(torch.from_numpy(ref_logits), dim=-1).numpy()
    for t in range(T):
        order = np.argsort(-ref_logits[t], kind="stable")[:k]
        np.testing.assert_array_equal(idx[t], order)
        np.testing.assert_allclose(w[t], p[t, order] / p[t, order].sum(), rtol=1e-13)
        assert abs(w[t].sum() - 1.0) < 1e-14
        assert np.all(np.diff(logits[t, idx[t]]) <= 0)
    gsf = torch.from_numpy(gen.bf16_bits_to_f32(gs).astype(np.float64))
    np.testing.assert_allclose(sg, torch.sigmoid(xf @ gsf).numpy(), rtol=1e-14)


def test_router_k_equals_E_gives_full_softmax():
    rng = np.random.default_rng(8)
    H, E = 64, 6
    x = bf16_vec(rng, H).reshape(1, H)
    Wr = bf16_vec(rng, E * H, 0.1).reshape(E, H)
    idx, w, _, logits = oracle.route(x, Wr, E, want_logits=True)
    full = torch.softmax(torch.from_numpy(logits[0]), dim=0).numpy()
    np.testing.assert_allclose(w[0], full[idx[0]], rtol=1e-14)
    assert sorted(idx[0].tolist()) == list(range(E))


def test_router_equal_logits_tie_break_lower_index():
    H, E, k = 64, 16, 3
    x = np.full((1, H), 0x3F80, dtype=np.uint16)        # x = 1
    Wr = np.zeros((E, H), dtype=np.uint16)                # all logits 0
    idx, w, _ = oracle.route(x, Wr, k)
    np.testing.assert_array_equal(idx[0], [0, 1, 2])
    np.testing.assert_allclose(w[0], [1 / 3] * 3, rtol=1e-15)
    # a bias on expert 9 makes it first; the rest keep index order
    bias = np.zeros(E, dtype=np.float32); bias[9] = 1.0
    idx, _, _ = oracle.route(x, Wr, k, bias=bias)
    np.testing.assert_array_equal(idx[0], [9, 0, 1])


# ---------------------------------------------------------------- combine + residual + RMSNorm
def test_combine_norm_vs_library():
    rng = np.random.default_rng(9)
    H, k = 96, 3
    y = rng.normal(size=(k, H)); w = np.array([0.5, 0.3, 0.2]); ys = rng.normal(size=H)
    h = rng.normal(size=H); gamma = bf16_vec(rng, H, 0.3) ; eps = 1e-6
    sg = 0.37
    h_out, x_out, xb = oracle.combine_norm(y, w, ys, sg, h, gamma, eps)
    h_ref = h + w @ y + sg * ys
    np.testing.assert_allclose(h_out, h_ref, rtol=1e-14, atol=1e-14)
    gf = torch.from_numpy(gen.bf16_bits_to_f32(gamma).astype(np.float64))
    x_ref = torch.nn.functional.rms_norm(torch.from_numpy(h_ref), (H,), weight=gf, eps=eps).numpy()
    np.testing.assert_allclose(x_out, x_ref, rtol=1e-13, atol=1e-14)
    # bf16 output is the round-to-nearest-even of the double result
    ref_b = np.array([_rne_bf16_exact(v) for v in x_out], dtype=np.uint16)
    np.testing.assert_array_equal(xb, ref_b)


def test_rmsnorm_closed_forms():
    H = 64
    gamma1 = np.full(H, 0x3F80, dtype=np.uint16)
    rng = np.random.default_rng(2)
    h = rng.normal(size=H)
    eps = 1e-3
    h_out, x_out, _ = oracle.combine_norm(np.zeros((1, H)), [0.0], None, 0.0, h, gamma1, eps)
    m = np.mean(h ** 2)
    assert abs(np.mean(x_out ** 2) - m / (m + eps)) < 1e-14
    c = -2.5
    _, x_out, _ = oracle.combine_norm(np.zeros((1, H)), [0.0], None, 0.0, np.full(H, c), gamma1, eps)
    np.testing.assert_allclose(x_out, np.sign(c) * np.sqrt(c * c / (c * c + eps)), rtol=1e-15)


def test_combine_one_hot_weight_and_shared_gate():
    H = 32
    y = np.stack([np.full(H, 1.0), np.full(H, 10.0)])
    h = np.zeros(H)
    gamma1 = np.full(H, 0x3F80, dtype=np.uint16)
    h_out, _, _ = oracle.combine_norm(y, [0.0, 1.0], np.full(H, 100.0), 0.5, h, gamma1, 1e-6)
    np.testing.assert_array_equal(h_out, np.full(H, 10.0 + 50.0))


# ---------------------------------------------------------------- bf16 rounding
def _rne_bf16_exact(v: float) -> int:
    """Reference RNE double -> bf16 by exact rational comparison of the two neighbours."""
    f = Fraction(v)
    if f == 0:
        return 0x8000 if np.signbit(v) else 0
    lo_bits = int(gen.f32_to_bf16_bits(np.array([v], dtype=np.float32))[0])
    cands = set()
    for d in (-2, -1, 0, 1, 2):
        bb = (lo_bits + d) & 0xFFFF
        if (bb & 0x7F80) != 0x7F80:
            cands.add(bb)
    best = min(cands, key=lambda bb: (abs(bf16_exact(bb) - f), bb & 1))
    return best


def test_double_to_bf16_rne_halfway_cases():
    vals = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -40, -(1.0 + 2 ** -8), 3.14159,
            1.0 + 2 ** -9, 0.0078125 * (1 + 2 ** -8), 65504.0, 1e-30]
    got = oracle.f64_to_bf16(vals)
    ref = [_rne_bf16_exact(v) for v in vals]
    np.testing.assert_array_equal(got, ref)
    assert got[0] == 0x3F80 and got[1] == 0x3F82     # ties to even, both directions


# ---------------------------------------------------------------- prefill grouping
def test_group_by_expert_vs_stable_argsort():
    rng = np.random.default_rng(4)
    T, k, E = 50, 3, 17
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm = oracle.group_by_expert(idx, E)
    flat = idx.ravel()
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))


# ---------------------------------------------------------------- expert and layer vs a torch composition
def _torch_expert(ex, x, H, I, G, bits):
    (gq, gs_, gb), (uq, us, ub), (dq, ds, db) = ex
    Wg = torch.from_numpy(dense_by_bitstring(gq, gs_, gb, H, G, bits))
    Wu = torch.from_numpy(dense_by_bitstring(uq, us, ub, H, G, bits))
    Wd = torch.from_numpy(dense_by_bitstring(dq, ds, db, I, G, bits))
    xt = torch.from_numpy(np.asarray(x, dtype=np.float64))
    a = torch.nn.functional.silu(Wg @ xt) * (Wu @ xt)
    return (Wd @ a).numpy(), a.numpy()


@pytest.mark.parametrize("bits", [4, 2])
def test_expert_vs_torch_composition(bits):
    cfg = fixtures.Config("t", H=128, E=4, k=2, I=64, bits=bits)
    ex = fixtures.host_expert(cfg, 0, 2)
    rng = np.random.default_rng(1)
    x = rng.normal(size=cfg.H)
    y, a = oracle.expert(ex, x, cfg.H, cfg.I, cfg.G, bits, want_a=True)
    y_ref, a_ref = _torch_expert(ex, x, cfg.H, cfg.I, cfg.G, bits)
    np.testing.assert_allclose(a, a_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("with_shared", [True, False])
def test_tiny_layer_vs_torch_composition(with_shared):
    cfg = fixtures.CONFIGS["tiny"]
    Wr, _, gsv, gamma = fixtures.layer_vectors(cfg, 0)
    experts = [fixtures.host_expert(cfg, 0, e) for e in range(cfg.E)]
    shared = fixtures.host_expert(cfg, 0, cfg.E) if with_shared else None
    x = gen.x_tokens(cfg, 0, T=2)
    h = gen.bf16_bits_to_f32(x).astype(np.float64)
    out = oracle.layer(x, h, Wr, gamma, experts, shared, I=cfg.I, k=cfg.k, G=cfg.G, bits=cfg.bits,
                       eps=cfg.rms_eps, gs=gsv if with_shared else None)
    xf = torch.from_numpy(h)
    logits = xf @ torch.from_numpy(gen.bf16_bits_to_f32(Wr).astype(np.float64)).T
    p = torch.softmax(logits, dim=-1)
    sgate = torch.sigmoid(xf @ torch.from_numpy(gen.bf16_bits_to_f32(gsv).astype(np.float64)))
    gf = torch.from_numpy(gen.bf16_bits_to_f32(gamma).astype(np.float64))
    for t in range(2):
        top = np.argsort(-logits[t].numpy(), kind="stable")[:cfg.k]
        np.testing.assert_array_equal(out["idx"][t], top)
        wt = p[t, top] / p[t, top].sum()
        moe = sum(float(wt[i]) * _torch_expert(experts[e], h[t], cfg.H, cfg.I, cfg.G, 4)[0] for i, e in enumerate(top))
        if with_shared:
            moe = moe + float(sgate[t]) * _torch_expert(shared, h[t], cfg.H, cfg.I, cfg.G, 4)[0]
        h_ref = h[t] + moe
        np.testing.assert_allclose(out["h_out"][t], h_ref, rtol=1e-11, atol=1e-11)
        x_ref = torch.nn.functional.rms_norm(torch.from_numpy(h_ref), (cfg.H,), weight=gf, eps=cfg.rms_eps).numpy()
        np.testing.assert_allclose(out["x_out"][t], x_ref, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- fixtures are deterministic
def test_fixture_streams_are_counter_based():
    key = gen.key_of(0, 3, gen.T_CODES, 7)
    a = gen.codes_words(key, 100)
    b = gen.codes_words(key, 40, start=60)
    np.testing.assert_array_equal(a[60:], b)
    z = gen.bf16_bits_to_f32(gen.normal_bf16(gen.key_of(0, 0, gen.T_X), 200_000, 1.0))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01


# ---------------------------------------------------------------- MXFP4 (third codec)
def _mx_table():
    """The MX encodings of tests/golden/mx_formats.txt: {code: Fraction}, {byte: Fraction or None}."""
    import os
    e2m1, e8m0, block = {}, {}, None
    with open(os.path.join(os.path.dirname(__file__), "golden", "mx_formats.txt")) as f:
        for line in f:
            t = line.split()
            if not t or t[0].startswith("#"):
                continue
            if t[0] == "block":
                block = int(t[1])
            elif t[0] == "e2m1":
                e2m1[int(t[1].replace(".", ""), 2)] = (t[2].startswith("-"), Fraction(t[2].lstrip("-")))
            elif t[0] == "e8m0":
                e8m0[int(t[1])] = None if t[2] == "nan" else Fraction(2) ** int(t[2].split("^")[1])
    return e2m1, e8m0, block


def test_mx_element_and_scale_values_match_the_format():
    """Every E2M1 code and the tabulated E8M0 bytes decode to the values of the MX format
    (signed zero included: code 1.00.0 is -0)."""
    e2m1, e8m0, block = _mx_table()
    assert block == 32 and len(e2m1) == 16
    for code, (neg, mag) in e2m1.items():
        v = oracle.e2m1(code)
        assert Fraction(abs(v)) == mag and np.signbit(v) == neg, code
    for byte, val in e8m0.items():
        v = oracle.e8m0(byte)
        assert (np.isnan(v) if val is None else Fraction(v) == val), byte
    for byte in range(255):   # every non-NaN byte: consecutive powers of two
        assert oracle.e8m0(byte + 1) == 2.0 * oracle.e8m0(byte) or byte == 254


def mx_dense_by_table(q, e, K):
    """MXFP4 matrix as exact Fractions from the format table and a bit-string unpacking."""
    e2m1, e8m0, block = _mx_table()
    R = q.shape[0]
    W = [[None] * K for _ in range(R)]
    for r in range(R):
        c = codes_by_bitstring(q[r], 4)
        for k in range(K):
            neg, mag = e2m1[int(c[k])]
            b = int(e[r][k // block])   # bytes between the tabulated ones: consecutive powers of two
            W[r][k] = (-mag if neg else mag) * e8m0[127] * Fraction(2) ** (b - 127)
    return W


def test_mx_dequant_and_gemv_brute_force():
    """A small random MXFP4 matrix (all 16 codes, scale bytes 100..140): the oracle's
    dequantised weights equal the table's exactly, and its mat-vec equals the exact
    rational dot products within one rounding per term."""
    rng = np.random.default_rng(11)
    R, K = 5, 96
    q = rng.integers(0, 2**32, size=(R, K // 8), dtype=np.uint64).astype(np.uint32)
    e = rng.integers(100, 141, size=(R, K // 32)).astype(np.uint8)
    Wt = mx_dense_by_table(q, e, K)
    Wo = oracle.mx_dequant(q, e, K)
    for r in range(R):
        for k in range(K):
            assert Fraction(Wo[r, k]) == Wt[r][k], (r, k)
    xb = gen.f32_to_bf16_bits(rng.standard_normal(K).astype(np.float32))
    x = [bf16_exact(int(b)) for b in xb]
    y = oracle.mx_gemv(q, e, gen.bf16_bits_to_f32(xb).astype(np.float64), K)
    for r in range(R):
        exact = sum(Wt[r][k] * x[k] for k in range(K))
        mag = sum(abs(Wt[r][k] * x[k]) for k in range(K))
        assert abs(Fraction(y[r]) - exact) <= mag * Fraction(K, 2**52), r


def test_mx_one_code_and_one_scale_land_where_the_layout_says():
    """A matrix with a single nonzero code (element k of row r) gives y[r] = value * x[k] and
    zero elsewhere; raising that block's scale byte by one doubles it. A wrong nibble order,
    word index or block index moves or loses the term."""
    R, K = 3, 128
    x = np.arange(1, K + 1, dtype=np.float64)
    for (r, k, code) in [(0, 0, 0x2), (1, 37, 0xF), (2, 127, 0x5), (1, 64, 0x9)]:
        q = np.zeros((R, K // 8), dtype=np.uint32)
        q[r, k // 8] = np.uint32(code << (4 * (k % 8)))
        e = np.full((R, K // 32), 127, dtype=np.uint8)
        y = oracle.mx_gemv(q, e, x, K)
        want = np.zeros(R)
        want[r] = oracle.e2m1(code) * x[k]
        np.testing.assert_array_equal(y, want)
        e[r, k // 32] += 1
        np.testing.assert_array_equal(oracle.mx_gemv(q, e, x, K), 2 * want)
        e[r, k // 32] -= 1
        e[r, (k // 32 + 1) % (K // 32)] += 5   # another block's scale: no effect
        np.testing.assert_array_equal(oracle.mx_gemv(q, e, x, K), want)


def test_mx_gemm_rows_are_the_gemv():
    """The batched form (dequantised matrix times the tokens by one library product) agrees with
    the index-order mat-vec on every token, to the rounding of two summation orders."""
    rng = np.random.default_rng(12)
    R, K, T = 16, 256, 5
    q = rng.integers(0, 2**32, size=(R, K // 8), dtype=np.uint64).astype(np.uint32)
    e = rng.integers(118, 126, size=(R, K // 32)).astype(np.uint8)
    xb = gen.f32_to_bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    Y = oracle.mx_gemm(q, e, xb, K)
    W = oracle.mx_dequant(q, e, K)
    for t in range(T):
        y = oracle.mx_gemv(q, e, gen.bf16_bits_to_f32(xb[t]).astype(np.float64), K)
        np.testing.assert_allclose(Y[t], y, rtol=0, atol=1e-13 * np.abs(W).sum(1).max() * 8)
