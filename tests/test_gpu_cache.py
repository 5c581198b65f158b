"""GPU: layers whose routed experts live in host memory, served through the
HBM expert cache (moe_layer_forward_cached). The kernels are the resident
path's, so the outputs must equal those of moe_layer_forward on the same layer
with every expert resident, bit for bit; the routing matches the oracle; the
cache counters add up."""
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


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available()
    qm.lib()
    return torch.device("cuda")


def host_experts(t, E):
    """Page-locked host copies of the routed experts of a device layer (index < E)."""
    hq = [t["q"][m][:E].cpu().pin_memory() for m in range(3)]
    hs = [t["s"][m][:E].cpu().pin_memory() for m in range(3)]
    hb = [t["b"][m][:E].cpu().pin_memory() for m in range(3)]
    return [qm.Expert(*[qm.QMat(hq[m][e], hs[m][e], hb[m][e]) for m in range(3)]) for e in range(E)]


def run(layer, x, h0, dev, cache=None, ws=None):
    T, H = x.shape
    k = layer.top_k
    h = torch.from_numpy(h0.copy()).to(dev)
    xo = torch.empty((T, H), dtype=torch.int16, device=dev)
    xf = torch.empty((T, H), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    xd = torch.from_numpy(x.view(np.int16)).to(dev)
    if cache is None:
        qm.moe_layer_forward(layer, xd, h, xo, xf, idx, w, ws=ws)
    else:
        qm.moe_layer_forward_cached(layer, cache, xd, h, xo, xf, idx, w, ws=ws)
    assert qm.moe_poll_status(ws) == 0
    return h.cpu().numpy(), xf.cpu().numpy(), xo.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def check_same(a, b):
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


@pytest.mark.parametrize("name,E,slots,calls", [("tiny", 16, 6, [1] * 10 + [3, 2]),
                                                 ("layer_q4", 32, 6, [1] * 6 + [2]),
                                                 ("tiny", 16, 16, [12, 20])])
def test_cached_layer_equals_resident(dev, name, E, slots, calls):
    """tiny: hidden 256, 16 experts, top-2, a 6-slot cache (decode, T up to 3: at most 6 distinct
    experts a call) and a 16-slot one (prefill, T = 12 and 20); layer_q4 shapes (hidden 4096,
    intermediate 1024, top-3 + shared) with 32 experts and a 6-slot cache."""
    base = fixtures.CONFIGS[name]
    cfg = base if E == base.E else fixtures.Config(base.name, H=base.H, E=E, k=base.k, I=base.I, bits=base.bits,
                                                   scale_sigma=base.scale_sigma)
    t = fxg.device_layer(cfg, 0, n_experts=E if E != base.E else None)
    layer = qm.layer_from_tensors(cfg, t)
    cache = qm.ExpertCache(layer, host_experts(t, E), slots)
    T_max = max(calls)
    ws_a, ws_b = qm.new_workspace(layer, T_max), qm.new_workspace(layer, T_max)
    distinct, seen = 0, set()
    for c, T in enumerate(calls):
        x = gen.x_tokens(cfg, 50 + c, T=T)
        h0 = gen.bf16_bits_to_f32(x).astype(np.float32)
        got = run(layer, x, h0, dev, cache=cache, ws=ws_a)
        ref = run(layer, x, h0, dev, ws=ws_b)
        check_same(got, ref)
        distinct += len(np.unique(got[3]))
        seen |= set(np.unique(got[3]).tolist())
        if c == 0:   # and the routing against the oracle
            Wr, rb, gs, _ = fixtures.layer_vectors(cfg, 0)
            ridx, _, _ = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
            np.testing.assert_array_equal(got[3], ridx)
    hits, misses, nbytes = qm.moe_cache_stats(cache)
    assert hits + misses == distinct
    per_expert = sum(t[a][m][0].numel() * t[a][m][0].element_size() for a in ("q", "s", "b") for m in range(3))
    assert nbytes == misses * per_expert
    assert len(seen) <= misses <= distinct   # every expert used is loaded at least once


def test_cached_layer_matches_oracle(dev):
    """One decode token of the tiny layer through the cache, against the fp64 oracle."""
    cfg = fixtures.CONFIGS["tiny"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    cache = qm.ExpertCache(layer, host_experts(t, cfg.E), 3)
    ws = qm.new_workspace(layer, 1)
    x = gen.x_tokens(cfg, 7, T=1)
    h0 = gen.bf16_bits_to_f32(x).astype(np.float32)
    h, xf, _, idx, _ = run(layer, x, h0, dev, cache=cache, ws=ws)
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    experts = [fixtures.host_expert(cfg, 0, e) for e in range(cfg.E)]
    shared = fixtures.host_expert(cfg, 0, cfg.E)
    ref = oracle.layer(x, h0.astype(np.float64), Wr, gamma, experts, shared, I=cfg.I, k=cfg.k, G=cfg.G,
                       bits=cfg.bits, eps=cfg.rms_eps, gs=gs, router_bias=rb)
    np.testing.assert_array_equal(idx, ref["idx"])
    assert rel_err(h[0], ref["h_out"][0]) <= 2e-3 and rel_err(xf[0], ref["x_out"][0]) <= 2e-3


def test_cache_too_small_for_a_call(dev):
    """A call that names more distinct experts than the cache has slots is refused (after routing,
    before any copy or layer kernel)."""
    cfg = fixtures.CONFIGS["tiny"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    cache = qm.ExpertCache(layer, host_experts(t, cfg.E), 1)
    ws = qm.new_workspace(layer, 1)
    x = gen.x_tokens(cfg, 3, T=1)
    h0 = gen.bf16_bits_to_f32(x).astype(np.float32)
    with pytest.raises(qm.MoeError) as e:
        run(layer, x, h0, dev, cache=cache, ws=ws)
    assert e.value.code == 2
    assert qm.moe_cache_stats(cache) == (0, 0, 0)
