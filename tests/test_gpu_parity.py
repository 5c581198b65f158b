"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Index work (top-k ids, grouping permutation) must match bit for bit; floating
outputs within max relative error 2e-3 (max|gpu - oracle| / max|oracle|); bf16
outputs within 1 unit in the last place of the oracle's round-to-nearest-even.
"""
import numpy as np
import pytest
import torch

import fixtures
import fixtures.gpu as fxg
import oracle
import quantized_expert_decode_moe_b200 as qm
from fixtures import gen
from refs import bf16_ulp_diff, oracle_tokens, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3
# what the decode path's fixed-point operand tables reach (the bar above is the contract)
FIXED_POINT_BOUND = 2e-4


def _np16(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available()
    qm.lib()
    return torch.device("cuda")


def _rand_qmat(rng, R, K, bits, dev, sigma=0.02):
    q = rng.integers(0, 2 ** 32, size=(R, K * bits // 32), dtype=np.uint64).astype(np.uint32)
    s = gen.f32_to_bf16_bits(np.abs(rng.normal(0, sigma, size=(R, K // 64))).astype(np.float32))
    b = gen.f32_to_bf16_bits(rng.normal(0, sigma * 4, size=(R, K // 64)).astype(np.float32))
    W = qm.QMat(torch.from_numpy(q.view(np.int32)).to(dev), torch.from_numpy(s.view(np.int16)).to(dev),
                torch.from_numpy(b.view(np.int16)).to(dev))
    return (q, s, b), W


# ------------------------------------------------------------------ fixtures: device == host
@pytest.mark.parametrize("name", ["tiny", "layer_q2"])
def test_device_fixtures_match_host(dev, name):
    cfg = fixtures.CONFIGS[name]
    E = cfg.E if name == "tiny" else 8
    t = fxg.device_layer(cfg, 0, n_experts=E)
    for e in (0, E - 1):
        ex = fixtures.host_expert(cfg, 0, e)
        for m in range(3):
            np.testing.assert_array_equal(t["q"][m][e].cpu().numpy().view(np.uint32), ex[m][0])
            np.testing.assert_array_equal(_np16(t["s"][m][e]), ex[m][1])
            np.testing.assert_array_equal(_np16(t["b"][m][e]), ex[m][2])
    shared = fixtures.host_expert(cfg, 0, cfg.E)   # device index E is the shared expert's stream
    if name == "tiny":
        for m in range(3):
            np.testing.assert_array_equal(t["q"][m][E].cpu().numpy().view(np.uint32), shared[m][0])
    Wr, _, gs, gamma = fixtures.layer_vectors(cfg, 0)
    np.testing.assert_array_equal(_np16(t["router_w"]), Wr[:E])
    np.testing.assert_array_equal(_np16(t["gate_w"]), gs)
    np.testing.assert_array_equal(_np16(t["gamma"]), gamma)


def check_bf16_out(xb, xf, ref):
    """bf16 output = RNE of the fp32 output (bit exact), and each element within
    1 bf16 ulp of the oracle or within the normwise tolerance of it (elements
    near zero carry no relative precision at the 2e-3 normwise bar)."""
    np.testing.assert_array_equal(xb, gen.f32_to_bf16_bits(xf.astype(np.float32)))
    ref_b = oracle.f64_to_bf16(ref) if len(ref) <= 512 else gen.f32_to_bf16_bits(ref.astype(np.float32))
    ulp = np.abs(xb.astype(np.int32) - ref_b.astype(np.int32))
    close = np.abs(gen.bf16_bits_to_f32(xb).astype(np.float64) - ref) <= TOL * np.max(np.abs(ref))
    assert np.all((ulp <= 1) | close)


# ------------------------------------------------------------------ dequant GEMV
@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("R,K", [(304, 1024), (16, 128), (32, 256), (4096, 1024), (1024, 4096), (2048, 8192)])
def test_gemv_matches_oracle(dev, bits, R, K):
    rng = np.random.default_rng(R * 7 + K + bits)
    (q, s, b), W = _rand_qmat(rng, R, K, bits, dev)
    x = rng.normal(size=K).astype(np.float32)
    y = torch.empty(R, dtype=torch.float32, device=dev)
    fn = qm.moe_expert_gemv_q4 if bits == 4 else qm.moe_expert_gemv_q2
    fn(W, R, K, 64, torch.from_numpy(x).to(dev), y)
    ref = oracle.qgemv(q, s, b, x.astype(np.float64), K, 64, bits)
    err = rel_err(y.cpu().numpy(), ref)
    assert err <= TOL, err
    assert err <= 1e-5, f"precision regression {err}"


def test_gemv_zero_vector_and_scale_range(dev):
    rng = np.random.default_rng(1)
    (q, s, b), W = _rand_qmat(rng, 64, 512, 4, dev)
    y = torch.full((64,), 7.0, device=dev)
    qm.moe_expert_gemv_q4(W, 64, 512, 64, torch.zeros(512, device=dev), y)
    assert torch.all(y == 0)
    # tiny and huge activations keep their relative accuracy (per-vector power-of-two prescale)
    for mag in (1e-20, 1e20):
        x = (rng.normal(size=512) * mag).astype(np.float32)
        qm.moe_expert_gemv_q4(W, 64, 512, 64, torch.from_numpy(x).to(dev), y)
        ref = oracle.qgemv(q, s, b, x.astype(np.float64), 512, 64, 4)
        assert rel_err(y.cpu().numpy(), ref) <= 1e-5


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("name", ["tiny", "layer_q4", "stack_q4"])
def test_route_matches_oracle(dev, name):
    cfg = fixtures.CONFIGS[name]
    t = fxg.device_layer(cfg, 0, n_experts=cfg.E) if name == "tiny" else None
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    if t is None:   # router-only layer: experts are not touched by moe_route
        t = {"router_w": torch.from_numpy(Wr.view(np.int16)).to(dev),
             "router_bias": torch.from_numpy(rb).to(dev) if rb is not None else None,
             "gate_w": torch.from_numpy(gs.view(np.int16)).to(dev),
             "gamma": torch.from_numpy(gamma.view(np.int16)).to(dev)}
        dummy = torch.zeros(64, dtype=torch.int32, device=dev)
        ex = qm.Expert(*[qm.QMat(dummy, dummy, dummy)] * 3)
        layer = qm.Layer(hidden=cfg.H, inter=cfg.I, top_k=cfg.k, bits=cfg.bits, router_w=t["router_w"],
                         experts=[ex] * cfg.E, rms_gamma=t["gamma"], shared=ex, shared_gate_w=t["gate_w"],
                         router_bias=t["router_bias"])
    else:
        layer = qm.layer_from_tensors(cfg, t)
    T = 16
    x = gen.x_tokens(cfg, 3, T=T)
    ws = qm.new_workspace(layer, T)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    sg = torch.empty(T, dtype=torch.float32, device=dev)
    qm.moe_route(layer, torch.from_numpy(x.view(np.int16)).to(dev), idx, w, sg, ws=ws)
    ridx, rw, rsg = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(sg.cpu().numpy(), rsg, rtol=1e-6, atol=1e-7)


def test_route_logits_within_their_bound_of_the_fp64_definition(dev):
    """Many tokens (T > 8): a logit is computed in exact integer arithmetic on
    22-bit fixed-point forms of w and x (one power-of-two scale per router row
    and per token), so it differs from the plain index-order fp64 loop of the
    definition by at most the rounding of that fixed point and of the fp64
    sums; every logit must lie within the certified bound the library stores
    beside it, and the ranking must be the definition's. The shared-gate logit
    is an fp64 sum of exact products. moe_route leaves
    the logits in the workspace: double [T][E+1] at byte 256, column E the
    shared-gate logit; the bounds follow as float [T][E+1]."""
    cfg = fixtures.CONFIGS["stack_q4"]   # the biased router
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    dummy = torch.zeros(64, dtype=torch.int32, device=dev)
    ex = qm.Expert(*[qm.QMat(dummy, dummy, dummy)] * 3)
    layer = qm.Layer(hidden=cfg.H, inter=cfg.I, top_k=cfg.k, bits=cfg.bits,
                     router_w=torch.from_numpy(Wr.view(np.int16)).to(dev), experts=[ex] * cfg.E,
                     rms_gamma=torch.from_numpy(gamma.view(np.int16)).to(dev), shared=ex,
                     shared_gate_w=torch.from_numpy(gs.view(np.int16)).to(dev),
                     router_bias=torch.from_numpy(rb).to(dev))
    T = 40
    x = gen.x_tokens(cfg, 5, T=T)
    ws = qm.new_workspace(layer, T)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    qm.moe_route(layer, torch.from_numpy(x.view(np.int16)).to(dev), idx, w, ws=ws)
    torch.cuda.synchronize()
    got = ws[256:256 + 8 * T * (cfg.E + 1)].cpu().numpy().view(np.float64).reshape(T, cfg.E + 1)
    off = 256 + ((8 * T * (cfg.E + 1) + 255) // 256) * 256
    bnd = ws[off:off + 4 * T * (cfg.E + 1)].cpu().numpy().view(np.float32).reshape(T, cfg.E + 1)[:, :cfg.E]
    ridx, _, _, ref = oracle.route(x, Wr, cfg.k, bias=rb, want_logits=True)
    err = np.abs(got[:, :cfg.E] - ref)
    assert np.all(err <= bnd.astype(np.float64))
    # the bound is built from each row's own rounding residuals sum|v - v~| (most
    # bf16 values are exact in 22-bit fixed point) and the fp64 sums' rounding
    assert np.all(bnd < 1e-5)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    _, _, _, ref_g = oracle.route(x, gs[None, :], 1, want_logits=True)
    assert np.max(np.abs(got[:, cfg.E] - ref_g[:, 0])) <= 1e-9
    print(f"many-token router: largest |l - definition| {err.max():.2e}, largest bound {bnd.max():.2e}")


@pytest.mark.parametrize("E,k", [(512, 8), (4096, 8), (4096, 3), (100, 5)])
def test_route_wide_pools_and_top8(dev, E, k):
    """Random router, with exact duplicate rows 37 apart (equal logits that land
    in different warps), at one logit per thread and at eight per thread."""
    rng = np.random.default_rng(E * 10 + k)
    H, T = 512, 12
    Wr = gen.f32_to_bf16_bits(rng.normal(0, 0.02, size=(E, H)).astype(np.float32))
    for e in range(0, E - 37, 3):
        Wr[e + 37] = Wr[e]
    x = gen.f32_to_bf16_bits(rng.normal(0, 1, size=(T, H)).astype(np.float32))
    dummy = torch.zeros(64, dtype=torch.int32, device=dev)
    ex = qm.Expert(*[qm.QMat(dummy, dummy, dummy)] * 3)
    gamma = torch.zeros(H, dtype=torch.int16, device=dev)
    layer = qm.Layer(hidden=H, inter=128, top_k=k, bits=4, router_w=torch.from_numpy(Wr.view(np.int16)).to(dev),
                     experts=[ex] * E, rms_gamma=gamma)
    ws = qm.new_workspace(layer, T)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    qm.moe_route(layer, torch.from_numpy(x.view(np.int16)).to(dev), idx, w, ws=ws)
    ridx, rw, _ = oracle.route(x, Wr, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)


def test_route_ties_resolve_to_lower_index(dev):
    H, E, k = 256, 32, 3
    zero = torch.zeros((E, H), dtype=torch.int16, device=dev)
    dummy = torch.zeros(64, dtype=torch.int32, device=dev)
    ex = qm.Expert(*[qm.QMat(dummy, dummy, dummy)] * 3)
    gamma = torch.zeros(H, dtype=torch.int16, device=dev)
    layer = qm.Layer(hidden=H, inter=128, top_k=k, bits=4, router_w=zero, experts=[ex] * E, rms_gamma=gamma)
    ws = qm.new_workspace(layer, 2)
    x = torch.full((2, H), 0x3F80, dtype=torch.int16, device=dev)
    idx = torch.empty((2, k), dtype=torch.int32, device=dev)
    w = torch.empty((2, k), dtype=torch.float32, device=dev)
    qm.moe_route(layer, x, idx, w, ws=ws)
    assert idx.cpu().tolist() == [[0, 1, 2]] * 2
    np.testing.assert_allclose(w.cpu().numpy(), 1 / 3, rtol=1e-7)


# ------------------------------------------------------------------ combine + residual + RMSNorm
@pytest.mark.parametrize("T,H,k,shared", [(1, 4096, 3, True), (5, 256, 2, True), (3, 384, 1, False),
                                           (40, 4096, 3, True), (33, 8192, 8, False)])
def test_combine_norm_matches_oracle(dev, T, H, k, shared):
    """Up to 31 tokens the combine runs as clusters of eight CTAs per token, from 32 tokens up
    (16-byte aligned buffers) as one CTA per token."""
    rng = np.random.default_rng(T * H + k)
    y = rng.normal(size=(T, k, H)).astype(np.float32)
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    ys = rng.normal(size=(T, H)).astype(np.float32) if shared else None
    sg = rng.uniform(size=T).astype(np.float32) if shared else None
    h = rng.normal(size=(T, H)).astype(np.float32)
    gamma = gen.f32_to_bf16_bits((1 + 0.1 * rng.normal(size=H)).astype(np.float32))
    td = lambda a: None if a is None else torch.from_numpy(a).to(dev)
    hd = td(h.copy())
    xo = torch.empty((T, H), dtype=torch.int16, device=dev)
    xf = torch.empty((T, H), dtype=torch.float32, device=dev)
    qm.moe_combine_residual_norm(td(y), td(w), td(ys), td(sg), hd, torch.from_numpy(gamma.view(np.int16)).to(dev),
                                 1e-6, xo, xf)
    for t in range(T):
        h_ref, x_ref, xb_ref = oracle.combine_norm(y[t].astype(np.float64), w[t].astype(np.float64),
                                                   None if ys is None else ys[t].astype(np.float64),
                                                   float(sg[t]) if shared else 0.0, h[t].astype(np.float64), gamma, 1e-6)
        assert rel_err(hd[t].cpu().numpy(), h_ref) <= TOL
        assert rel_err(xf[t].cpu().numpy(), x_ref) <= TOL
        check_bf16_out(_np16(xo[t]), xf[t].cpu().numpy(), x_ref)


# ------------------------------------------------------------------ grouping by expert
@pytest.mark.parametrize("T,k,E", [(512, 3, 512), (7, 2, 16), (1, 3, 512), (300, 8, 64)])
def test_group_tokens_bit_exact(dev, T, k, E):
    rng = np.random.default_rng(T + k + E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    qm.moe_group_tokens(torch.from_numpy(idx).to(dev), E, counts, offsets, perm)
    rc, ro, rp = oracle.group_by_expert(idx, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
    np.testing.assert_array_equal(perm.cpu().numpy(), rp)


# ------------------------------------------------------------------ whole layer
def _layer_parity(cfg, t, layer, x_bits, dev, T_call):
    T = x_bits.shape[0]
    ws = qm.new_workspace(layer, T_call)
    xo = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
    xf = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    xd = torch.from_numpy(x_bits.view(np.int16)).to(dev)
    h0 = gen.bf16_bits_to_f32(x_bits).astype(np.float32)
    h = torch.from_numpy(h0.copy()).to(dev)
    for a in range(0, T, T_call):
        sl = slice(a, a + T_call)
        qm.moe_layer_forward(layer, xd[sl], h[sl], xo[sl], xf[sl], idx[sl], w[sl], ws=ws)
    assert qm.moe_poll_status(ws) == 0
    ref = oracle_tokens(cfg, 0, x_bits, h0.astype(np.float64))
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    np.testing.assert_allclose(w.cpu().numpy(), ref["w"], rtol=1e-6, atol=1e-7)
    errs = []
    for i in range(T):
        eh, ex = rel_err(h[i].cpu().numpy(), ref["h_out"][i]), rel_err(xf[i].cpu().numpy(), ref["x_out"][i])
        errs.append(max(eh, ex))
        assert eh <= TOL and ex <= TOL, (eh, ex)
        check_bf16_out(_np16(xo[i]), xf[i].cpu().numpy(), ref["x_out"][i])
    print(f"{cfg.name}: max rel err {max(errs):.3e}")
    return max(errs)


@pytest.mark.parametrize("T_call", [1, 3])
def test_layer_tiny_matches_oracle(dev, T_call):
    cfg = fixtures.CONFIGS["tiny"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    x = gen.x_tokens(cfg, 0, T=6)
    err = _layer_parity(cfg, t, layer, x, dev, T_call)
    # fixed point of the activation digits: 22 bits for the low code field,
    # 22 - BITS*q for field q (the field is used in place), so ~1e-5 per dot product
    assert err < FIXED_POINT_BOUND


@pytest.fixture(scope="module")
def big_q4(dev):
    cfg = fixtures.CONFIGS["layer_q4"]
    t = fxg.device_layer(cfg, 0)
    yield cfg, t, qm.layer_from_tensors(cfg, t)
    del t
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T_call", [1, 4])
def test_layer_q4_full_size_matches_oracle(dev, big_q4, T_call):
    cfg, t, layer = big_q4
    x = gen.x_tokens(cfg, 11, T=4)
    err = _layer_parity(cfg, t, layer, x, dev, T_call)
    assert err < FIXED_POINT_BOUND


def test_layer_q2_full_size_matches_oracle(dev):
    cfg = fixtures.CONFIGS["layer_q2"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    x = gen.x_tokens(cfg, 5, T=3)
    err = _layer_parity(cfg, t, layer, x, dev, 1)
    assert err < FIXED_POINT_BOUND
    del t, layer
    torch.cuda.empty_cache()


def test_layer_without_shared_expert(dev):
    cfg = fixtures.Config("noshared", H=512, E=24, k=3, I=256, bits=4, has_shared=False)
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    x = gen.x_tokens(cfg, 2, T=2)
    _layer_parity(cfg, t, layer, x, dev, 2)
