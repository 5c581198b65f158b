"""GPU parity of the prefill path (T > 8 tokens: grouping by expert into
chunks, grouped GEMMs of the packed codes against fixed-point activation
digits on the integer tensor cores, combine + residual + RMSNorm) against the
CPU oracle, through moe_layer_forward. The shared expert runs either on the
grouped integer kernels or as dense tcgen05 GEMMs on exact fp16 operands
(MOE_PREFILL_SHARED=mma / tc); the tests marked with `path` run both.

Routing ids bit-exact for every token; h and x_out within max relative error
2e-3 (max|gpu - oracle| / max|oracle|) per token; bf16 x_out within one ulp
of the oracle's rounding or the normwise bar.
"""
import numpy as np
import pytest
import torch

import fixtures
import fixtures.gpu as fxg
import oracle
import quantized_expert_decode_moe_b200 as qm
from fixtures import gen
from refs import oracle_tokens, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _np16(t):
    return t.cpu().numpy().view(np.uint16)


def _check_bf16(xb, ref, ref_b):
    ulp = np.abs(xb.astype(np.int32) - ref_b.astype(np.int32))
    close = np.abs(gen.bf16_bits_to_f32(xb).astype(np.float64) - ref) <= TOL * np.max(np.abs(ref))
    assert np.all((ulp <= 1) | close)


def _run(cfg, layer, x_bits, dev):
    T = x_bits.shape[0]
    ws = qm.new_workspace(layer, T)
    xo = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
    xf = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    h0 = gen.bf16_bits_to_f32(x_bits).astype(np.float32)
    h = torch.from_numpy(h0.copy()).to(dev)
    qm.moe_layer_forward(layer, torch.from_numpy(x_bits.view(np.int16)).to(dev), h, xo, xf, idx, w, ws=ws)
    assert qm.moe_poll_status(ws) == 0
    return h0, idx.cpu().numpy(), w.cpu().numpy(), h.cpu().numpy(), xf.cpu().numpy(), _np16(xo)


def _compare(cfg, x_bits, h0, idx, w, h, xf, xo, sample):
    ref = oracle_tokens(cfg, 0, x_bits[sample], h0[sample].astype(np.float64))
    np.testing.assert_array_equal(idx[sample], ref["idx"])
    np.testing.assert_allclose(w[sample], ref["w"], rtol=1e-6, atol=1e-7)
    worst = 0.0
    for n, i in enumerate(sample):
        eh, ex = rel_err(h[i], ref["h_out"][n]), rel_err(xf[i], ref["x_out"][n])
        assert eh <= TOL and ex <= TOL, (i, eh, ex)
        np.testing.assert_array_equal(xo[i], gen.f32_to_bf16_bits(xf[i]))
        _check_bf16(xo[i], ref["x_out"][n], ref["x_out_bf16"][n])
        worst = max(worst, eh, ex)
    print(f"{cfg.name} prefill T={x_bits.shape[0]}: max rel err {worst:.3e} over {len(sample)} tokens")
    return worst


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available()
    qm.lib()
    return torch.device("cuda")


@pytest.mark.parametrize("path", ["tc", "mma"])
@pytest.mark.parametrize("T", [9, 40])
def test_prefill_tiny_matches_oracle(dev, T, path, monkeypatch):
    monkeypatch.setenv("MOE_PREFILL_SHARED", path)
    cfg = fixtures.CONFIGS["tiny"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    x = gen.x_tokens(cfg, 21, T=T)
    out = _run(cfg, layer, x, dev)
    _compare(cfg, x, *out, sample=list(range(T)))


@pytest.mark.parametrize("bits,shared,path", [(2, True, "tc"), (2, True, "mma"), (4, True, "tc"), (4, False, "tc")])
def test_prefill_small_layers(dev, bits, shared, path, monkeypatch):
    monkeypatch.setenv("MOE_PREFILL_SHARED", path)
    cfg = fixtures.Config(f"pf{bits}{'s' if shared else 'n'}", H=512, E=24, k=3, I=256, bits=bits,
                          scale_sigma=0.05 if bits == 2 else 0.02, has_shared=shared)
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    x = gen.x_tokens(cfg, 4, T=33)
    out = _run(cfg, layer, x, dev)
    _compare(cfg, x, *out, sample=list(range(33)))


@pytest.mark.parametrize("path", ["tc", "mma"])
def test_prefill_wide_hidden(dev, path, monkeypatch):
    """Hidden 8192 (the widest layer the library takes): 4-token chunks and
    8 quantisation groups per warp in the gate/up kernel; 136 column stages
    (8192 data + 512 bias-term columns) in the tensor-core gate/up pass."""
    monkeypatch.setenv("MOE_PREFILL_SHARED", path)
    cfg = fixtures.Config("pfwide", H=8192, E=8, k=2, I=256, bits=4, has_shared=True)
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    x = gen.x_tokens(cfg, 7, T=12)
    out = _run(cfg, layer, x, dev)
    _compare(cfg, x, *out, sample=list(range(12)))


def test_prefill_full_size_512_tokens(dev):
    """The 512-token prefill of the 4-bit layer (hidden 4096, 512 experts,
    top-3 + shared): routing of all 512 tokens bit-exact, outputs of a
    sample of tokens (regenerating every expert the whole batch touches on
    the host is too slow for a test). At 512 tokens the shared expert takes
    the tcgen05 path by default: two 256-token blocks per weight tile and
    column splits whose partial sums the combine adds."""
    cfg = fixtures.CONFIGS["prefill_q4"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    x = gen.x_tokens(cfg, 0, T=cfg.T)
    h0, idx, w, h, xf, xo = _run(cfg, layer, x, dev)
    Wr, rb, gs, _ = fixtures.layer_vectors(cfg, 0)
    ridx, rw, _ = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=1e-6, atol=1e-7)
    assert len(np.unique(idx)) > 400   # the batch touches most of the 512 experts
    sample = [0, 1, 2, 63, 64, 200, 255, 256, 300, 447, 510, 511]
    _compare(cfg, x, h0, idx, w, h, xf, xo, sample=sample)
    del t, layer
    torch.cuda.empty_cache()


@pytest.mark.parametrize("path", ["tc", "mma"])
@pytest.mark.parametrize("where", ["x", "a"])
@pytest.mark.parametrize("name,T", [("tiny", 40), ("layer_q4", 16)])
def test_prefill_outlier_activations(dev, name, T, where, path, monkeypatch):
    """Activations as real models have them, one outlier per row: "x": every
    token's input carries one element 2^10 times the rest; "a": one
    intermediate row of the shared expert has its up-projection scales raised
    by 2^10, so every token's SwiGLU output a holds one value ~2^10 above the
    others. The prefill path writes activations as 16-bit fixed point with one
    exponent per 64-value group (each value within 2^-15 of its group's
    maximum), so an outlier costs only its own group bits. The experts'
    contribution h' - h must match the oracle's within the normwise bar; the
    routing bit for bit. On the tcgen05 path the shared expert's activations
    are fp16 with one exponent per token (a as hi + lo parts), exact for x."""
    monkeypatch.setenv("MOE_PREFILL_SHARED", path)
    cfg = fixtures.CONFIGS[name]
    n = None if name == "tiny" else 32
    c = cfg if n is None else fixtures.Config(cfg.name, H=cfg.H, E=n, k=cfg.k, I=cfg.I, bits=cfg.bits,
                                               scale_sigma=cfg.scale_sigma)
    t = fxg.device_layer(c, 0, n_experts=n)
    rng = np.random.default_rng(11)
    jstar = int(rng.integers(0, c.I))
    if where == "a":
        up_s = t["s"][1][c.E]                      # shared expert (stored at index E), up scales [I][H/64]
        boosted = up_s[jstar].cpu().numpy().view(np.uint16).astype(np.uint32) + (10 << 7)   # bf16 exponent + 10
        up_s[jstar] = torch.from_numpy(boosted.astype(np.uint16).view(np.int16)).to(dev)
    layer = qm.layer_from_tensors(c, t)
    x = gen.x_tokens(c, 23, T=T)
    if where == "x":
        xf = gen.bf16_bits_to_f32(x)
        for i in range(T):
            j = int(rng.integers(0, c.H))
            xf[i, j] = np.float32(1024.0) * np.sign(xf[i, j] if xf[i, j] != 0 else 1.0) * max(abs(xf[i]).max(), 1.0)
        x = gen.f32_to_bf16_bits(xf.astype(np.float32))
    h0, idx, w, h, xfo, xo = _run(c, layer, x, dev)
    Wr, rb, gs, gamma = fixtures.layer_vectors(c, 0)
    experts = [fixtures.host_expert(c, 0, e) for e in range(c.E)]
    shared = [list(m) for m in fixtures.host_expert(c, 0, c.E)]
    if where == "a":
        s_up = shared[1][1].copy()
        s_up[jstar] = (s_up[jstar].astype(np.uint32) + (10 << 7)).astype(np.uint16)
        shared[1][1] = s_up
    sample = list(range(0, T, max(1, T // 8)))
    ref = oracle.layer(x[sample], h0[sample].astype(np.float64), Wr, gamma, experts, [tuple(m) for m in shared],
                       I=c.I, k=c.k, G=c.G, bits=c.bits, eps=c.rms_eps, gs=gs, router_bias=rb)
    np.testing.assert_array_equal(idx[sample], ref["idx"])
    worst = 0.0
    for n_, i in enumerate(sample):
        d_gpu = h[i].astype(np.float64) - h0[i]
        d_ref = ref["h_out"][n_] - h0[i]
        e = float(np.max(np.abs(d_gpu - d_ref)) / np.max(np.abs(d_ref)))
        assert e <= TOL, (i, e)
        worst = max(worst, e)
    print(f"{name} outlier in {where}: max rel err of the experts' contribution {worst:.3e}")
