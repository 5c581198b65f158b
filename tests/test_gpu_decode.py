"""Decode path (T <= 8) on the GPU against the CPU oracle, through the C ABI.

The decode router sums each logit as compensated fp32 together with a
rigorous bound on its distance to the plain fp64 definition (exact bf16
products summed in index order, bias last). The top-k is certified against
that bound, and candidates closer than it are recomputed as the definition.
So the ids must equal the oracle's bit for bit:
  - on hundreds of tokens of the biased 512-expert router, one to eight
    tokens per call, with every logit inside its stated bound;
  - with exact duplicate router rows, at top-8 and with 4096 experts;
  - on constructed near ties: two rows equal but for one bf16 ulp of an
    element that meets a tiny activation (fp64 logits 2^-44 apart), and an
    exact tie. These must take the exact recheck, which the workspace header
    counts.
The same ids and layer outputs are checked through the decode layer (the
digit-block kernels by default; the four-kernel chain when
MOE_DECODE_KERNEL=chain, the fused kernel when MOE_DECODE_KERNEL=fused) and
the prefill path, and the decode paths run at the largest shapes they accept.
"""
import os

import numpy as np
import pytest
import torch

import fixtures
import fixtures.gpu as fxg
import oracle
import quantized_expert_decode_moe_b200 as qm
from fixtures import gen
from refs import rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available()
    qm.lib()
    return torch.device("cuda")


def _router_layer(Wr, rb, gs, gamma, H, k, dev, I=128):
    """A layer for moe_route only: the experts are never touched."""
    dummy = torch.zeros(64, dtype=torch.int32, device=dev)
    ex = qm.Expert(*[qm.QMat(dummy, dummy, dummy)] * 3)
    td = lambda a, dt: None if a is None else torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(dev)
    return qm.Layer(hidden=H, inter=I, top_k=k, bits=4, router_w=td(Wr, np.int16), experts=[ex] * Wr.shape[0],
                    rms_gamma=td(gamma, np.int16), shared=ex if gs is not None else None,
                    shared_gate_w=td(gs, np.int16), router_bias=td(rb, np.float32))


def _rechecks(ws):
    torch.cuda.synchronize()
    return int(ws[16:20].cpu().numpy().view(np.uint32)[0])


# ------------------------------------------------------------------ router: many tokens, logits within the bound
def test_decode_router_many_tokens_bit_exact_and_within_bound(dev):
    cfg = fixtures.CONFIGS["stack_q4"]   # 512 experts, hidden 4096, per-expert logit bias
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    layer = _router_layer(Wr, rb, gs, gamma, cfg.H, cfg.k, dev)
    N = 288
    x = gen.x_tokens(cfg, 77, T=N)
    ridx, rw, rsg, rlog = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs, want_logits=True)
    ws = qm.new_workspace(layer, 8)
    xd = torch.from_numpy(x.view(np.int16)).to(dev)
    idx = torch.empty((N, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((N, cfg.k), dtype=torch.float32, device=dev)
    sg = torch.empty(N, dtype=torch.float32, device=dev)
    a, T, worst = 0, 1, 0.0
    while a < N:                       # calls of 1, 2, ..., 8 tokens in turn
        T = min(T, N - a)
        qm.moe_route(layer, xd[a:a + T], idx[a:a + T], w[a:a + T], sg[a:a + T], ws=ws)
        torch.cuda.synchronize()
        got = ws[256:256 + 8 * T * (cfg.E + 1)].cpu().numpy().view(np.float64).reshape(T, cfg.E + 1)[:, :cfg.E]
        off = 256 + ((8 * T * (cfg.E + 1) + 255) // 256) * 256   # error bounds: float [T][E+1] after the logits
        bnd = ws[off:off + 4 * T * (cfg.E + 1)].cpu().numpy().view(np.float32).reshape(T, cfg.E + 1)[:, :cfg.E]
        err = np.abs(got - rlog[a:a + T])
        assert np.all(err <= bnd.astype(np.float64)), "a logit outside its certified bound"
        assert np.all(bnd < 1e-5), "bound far looser than the compensated sum"
        worst = max(worst, float(np.max(err / bnd)))
        a += T
        T = T % 8 + 1
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(sg.cpu().numpy(), rsg, rtol=1e-6, atol=1e-7)
    print(f"largest |fast - definition| / bound over {N} tokens: {worst:.2e}")


@pytest.mark.parametrize("T", [1, 5])
@pytest.mark.parametrize("E,k", [(512, 8), (4096, 8), (4096, 3), (100, 5)])
def test_decode_router_duplicate_rows_wide_pools(dev, E, k, T):
    """Exact duplicate rows 37 apart (equal logits that land in different
    warps), one logit per thread (E <= 512) and up to eight per thread."""
    rng = np.random.default_rng(E * 10 + k + T)
    H = 512
    Wr = gen.f32_to_bf16_bits(rng.normal(0, 0.02, size=(E, H)).astype(np.float32))
    for e in range(0, E - 37, 3):
        Wr[e + 37] = Wr[e]
    x = gen.f32_to_bf16_bits(rng.normal(0, 1, size=(T, H)).astype(np.float32))
    gamma = np.zeros(H, dtype=np.uint16)
    layer = _router_layer(Wr, None, None, gamma, H, k, dev)
    ws = qm.new_workspace(layer, T)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    qm.moe_route(layer, torch.from_numpy(x.view(np.int16)).to(dev), idx, w, ws=ws)
    ridx, rw, _ = oracle.route(x, Wr, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)


# ------------------------------------------------------------------ constructed near ties
NT = fixtures.Config("neartie", H=512, E=64, k=3, I=256, bits=4)


def _near_tie_router(seed):
    """Router rows for one token x: rows 10 and 20 equal (an exact tie at the
    top), rows 30 and 31 equal but for one bf16 ulp of element j, where x[j]
    = 2^-30, so their fp64 logits differ by 2^-44 (row 31 larger) while both
    sit at ranks 3 and 4: the definition keeps 31 and drops 30. Far below
    the compensated sum's certified bound, so only the exact recheck can
    decide. Returns (Wr, x bits [1][H])."""
    rng = np.random.default_rng(seed)
    H, E = NT.H, NT.E
    x = rng.normal(0, 1, size=H)
    j = 7
    x[j] = 2.0 ** -30
    xb = gen.f32_to_bf16_bits(x.astype(np.float32))
    xf = gen.bf16_bits_to_f32(xb).astype(np.float64)
    Wr = gen.f32_to_bf16_bits(rng.normal(0, 0.02, size=(E, H)).astype(np.float32))
    Wr[10] = Wr[20] = gen.f32_to_bf16_bits((0.004 * xf).astype(np.float32))
    r30 = gen.f32_to_bf16_bits((0.0035 * xf).astype(np.float32))
    r30[j] = gen.f32_to_bf16_bits(np.float32(0.01))
    r31 = r30.copy()
    r31[j] = r30[j] + 1                # next bf16 above a positive value
    Wr[30], Wr[31] = r30, r31
    return Wr, xb[None, :]


def test_near_ties_route_like_the_definition(dev):
    Wr, x = _near_tie_router(1)
    _, _, _, lg = oracle.route(x, Wr, 4, want_logits=True)
    assert lg[0, 31] > lg[0, 30] and lg[0, 31] - lg[0, 30] < 1e-12 and lg[0, 10] == lg[0, 20]
    ridx, rw, _ = oracle.route(x, Wr, NT.k)
    assert ridx.tolist() == [[10, 20, 31]]
    gamma = np.zeros(NT.H, dtype=np.uint16)
    layer = _router_layer(Wr, None, None, gamma, NT.H, NT.k, dev)
    for T in (1, 3, 12):   # the decode router (T <= 8) and the many-token router GEMM
        xs = np.repeat(x, T, axis=0)
        ws = qm.new_workspace(layer, T)
        idx = torch.empty((T, NT.k), dtype=torch.int32, device=dev)
        w = torch.empty((T, NT.k), dtype=torch.float32, device=dev)
        qm.moe_route(layer, torch.from_numpy(xs.view(np.int16)).to(dev), idx, w, ws=ws)
        assert idx.cpu().numpy().tolist() == ridx.tolist() * T
        np.testing.assert_allclose(w.cpu().numpy(), np.repeat(rw, T, axis=0), rtol=1e-6, atol=1e-7)
        assert _rechecks(ws) == T, "the near tie must be decided by the exact recheck"


@pytest.mark.parametrize("T", [1, 2, 9])
def test_near_ties_through_the_layer(dev, T):
    """The same near ties through moe_layer_forward: T = 1 and 2 take the
    decode kernels (T = 1 the fused kernel when MOE_DECODE_KERNEL=fused),
    T = 9 the prefill path; ids, weights and outputs against the oracle's
    layer with the same router."""
    Wr, x1 = _near_tie_router(2)
    t = fxg.device_layer(NT, 0)
    t["router_w"] = torch.from_numpy(Wr.view(np.int16)).to(dev)
    layer = qm.layer_from_tensors(NT, t)
    x = np.repeat(x1, T, axis=0)
    h0 = gen.bf16_bits_to_f32(x).astype(np.float32)
    ws = qm.new_workspace(layer, T)
    xd = torch.from_numpy(x.view(np.int16)).to(dev)
    h = torch.from_numpy(h0.copy()).to(dev)
    xo = torch.empty((T, NT.H), dtype=torch.int16, device=dev)
    xf = torch.empty((T, NT.H), dtype=torch.float32, device=dev)
    idx = torch.empty((T, NT.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, NT.k), dtype=torch.float32, device=dev)
    qm.moe_layer_forward(layer, xd, h, xo, xf, idx, w, ws=ws)
    assert qm.moe_poll_status(ws) == 0
    assert _rechecks(ws) == T
    _, _, gs, gamma = fixtures.layer_vectors(NT, 0)
    experts = [fixtures.host_expert(NT, 0, e) for e in range(NT.E)]
    ref = oracle.layer(x, h0.astype(np.float64), Wr, gamma, experts, fixtures.host_expert(NT, 0, NT.E), I=NT.I,
                       k=NT.k, G=NT.G, bits=NT.bits, eps=NT.rms_eps, gs=gs)
    assert ref["idx"].tolist() == [[10, 20, 31]] * T
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    np.testing.assert_allclose(w.cpu().numpy(), ref["w"], rtol=1e-6, atol=1e-7)
    for i in range(T):
        assert rel_err(h[i].cpu().numpy(), ref["h_out"][i]) <= TOL
        assert rel_err(xf[i].cpu().numpy(), ref["x_out"][i]) <= TOL


def test_fused_layer_routes_many_biased_tokens_like_the_oracle(dev):
    """256 single-token calls of the full 512-expert layer with the per-expert
    router bias; ids bit-exact against the oracle."""
    cfg = fixtures.CONFIGS["stack_q4"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    Wr, rb, gs, _ = fixtures.layer_vectors(cfg, 0)
    N = 256
    x = gen.x_tokens(cfg, 91, T=N)
    ridx, rw, _ = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
    ws = qm.new_workspace(layer, 1)
    xd = torch.from_numpy(x.view(np.int16)).to(dev)
    h = torch.from_numpy(gen.bf16_bits_to_f32(x).astype(np.float32)).to(dev)
    xo = torch.empty((N, cfg.H), dtype=torch.int16, device=dev)
    idx = torch.empty((N, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((N, cfg.k), dtype=torch.float32, device=dev)
    for i in range(N):
        qm.moe_layer_forward(layer, xd[i:i + 1], h[i:i + 1], xo[i:i + 1], None, idx[i:i + 1], w[i:i + 1], ws=ws)
    assert qm.moe_poll_status(ws) == 0
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)
    del t, layer
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ largest accepted shapes
def _layer_vs_oracle(cfg, T, dev, calls=2):
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    experts = [fixtures.host_expert(cfg, 0, e) for e in range(cfg.E)]
    shared = fixtures.host_expert(cfg, 0, cfg.E)
    ws = qm.new_workspace(layer, T)
    for c in range(calls):
        x = gen.x_tokens(cfg, 5 + c, T=T)
        h0 = gen.bf16_bits_to_f32(x).astype(np.float32)
        xd = torch.from_numpy(x.view(np.int16)).to(dev)
        h = torch.from_numpy(h0.copy()).to(dev)
        xo = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
        xf = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
        idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
        w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
        qm.moe_layer_forward(layer, xd, h, xo, xf, idx, w, ws=ws)
        assert qm.moe_poll_status(ws) == 0
        ref = oracle.layer(x, h0.astype(np.float64), Wr, gamma, experts, shared, I=cfg.I, k=cfg.k, G=cfg.G,
                           bits=cfg.bits, eps=cfg.rms_eps, gs=gs, router_bias=rb)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
        for i in range(T):
            eh, ex = rel_err(h[i].cpu().numpy(), ref["h_out"][i]), rel_err(xf[i].cpu().numpy(), ref["x_out"][i])
            assert eh <= TOL and ex <= TOL, (eh, ex)
            assert max(eh, ex) < 2e-4
    del t, layer
    torch.cuda.empty_cache()


@pytest.mark.parametrize("bits", [4, 2])
def test_fused_layer_at_its_largest_shape(dev, bits):
    """hidden 4096 and intermediate 1152 = 8 rows x 148 SMs (rounded to a span):
    the largest shape whose per-SM gate/up and down rows fit the fused kernel
    (which runs it when MOE_DECODE_KERNEL=fused; the decode path of the environment otherwise)."""
    cfg = fixtures.Config("fused_max", H=4096, E=16, k=3, I=1152, bits=bits,
                          scale_sigma=0.02 if bits == 4 else 0.05)
    _layer_vs_oracle(cfg, 1, dev)


def test_chain_at_its_largest_shape(dev):
    """hidden 7552 and intermediate 2688 at 4 bits, top-3 + shared: the largest
    staging of the four-kernel chain that fits one CTA; T = 1 (the fused kernel
    does not take hidden > 4096) and T = 2."""
    cfg = fixtures.Config("chain_max", H=7552, E=8, k=3, I=2688, bits=4)
    _layer_vs_oracle(cfg, 1, dev, calls=1)
    _layer_vs_oracle(cfg, 2, dev, calls=1)


@pytest.mark.parametrize("bits", [4, 2])
def test_odd_span_counts(dev, bits):
    """hidden 3968 (31 spans of 128) and intermediate 896 (7 spans): warps
    whose share of the spans starts on an odd span, and span pairs that cross
    a 16-byte chunk of scale words; T = 1 and T = 2."""
    cfg = fixtures.Config("odd_spans", H=3968, E=12, k=3, I=896, bits=bits,
                          scale_sigma=0.02 if bits == 4 else 0.05)
    _layer_vs_oracle(cfg, 1, dev, calls=1)
    _layer_vs_oracle(cfg, 2, dev, calls=1)


def test_decode_path_is_the_one_requested(dev):
    """Decode calls take the digit-block kernels, the four-kernel chain with
    MOE_DECODE_KERNEL=chain, the fused kernel (one token) with =fused."""
    t = fxg.device_layer(NT, 0)
    layer = qm.layer_from_tensors(NT, t)
    env = os.environ.get("MOE_DECODE_KERNEL")
    if env == "fused":
        assert qm.moe_layer_path(layer, 1) == ("fused", 2)
        assert qm.moe_layer_path(layer, 2) == ("chain", 5)
    else:
        want = "chain" if env == "chain" else "digit"
        assert qm.moe_layer_path(layer, 1) == (want, 5)
        assert qm.moe_layer_path(layer, 8) == (want, 5)
    assert qm.moe_layer_path(layer, 9) == ("prefill", 6)
