"""Device-side failure path on the GPU, without a fault: a bounded wait runs
out (a barrier phase that nothing completes, or a grid-wide barrier round
that never fills), the kernel latches MOE_ERR_TIMEOUT in the workspace status
word and returns; the host reads it with moe_poll_status (which also clears
the grid-barrier counters left mid-round) and the same context and workspace
then serve a normal call that matches the oracle."""
import time

import numpy as np
import pytest
import torch

import fixtures
import fixtures.gpu as fxg
import oracle
import quantized_expert_decode_moe_b200 as qm
from fixtures import gen

pytestmark = pytest.mark.gpu
MOE_ERR_TIMEOUT = 5


def test_wait_timeout_is_latched_and_the_context_stays_usable():
    assert torch.cuda.is_available()
    dev = torch.device("cuda")
    cfg = fixtures.CONFIGS["tiny"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    ws = qm.new_workspace(layer, 1)
    t0 = time.perf_counter()
    qm.moe_selftest_wait_timeout(ws, 2_000_000)   # 2 ms
    assert qm.moe_poll_status(ws) == MOE_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0          # the wait ended by its bound
    assert qm.moe_poll_status(ws) == 0             # the poll cleared it
    # the same context and workspace serve a normal call afterwards
    T = 4
    x = gen.x_tokens(cfg, 11, T=T)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    ws4 = qm.new_workspace(layer, T)
    qm.moe_route(layer, torch.from_numpy(x.view(np.int16)).to(dev), idx, w, ws=ws4)
    assert qm.moe_poll_status(ws4) == 0
    Wr, rb, gs, _ = fixtures.layer_vectors(cfg, 0)
    ridx, rw, _ = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)


def test_grid_barrier_timeout_is_latched_and_the_workspace_recovers():
    """The fused decode kernel's grid-wide barrier: one CTA arrives at a round
    sized for two, its bounded wait runs out and leaves the arrival counter at
    1. After moe_poll_status the same workspace serves single-token layer
    calls whose routing and outputs match the oracle."""
    assert torch.cuda.is_available()
    dev = torch.device("cuda")
    cfg = fixtures.CONFIGS["tiny"]
    t = fxg.device_layer(cfg, 0)
    layer = qm.layer_from_tensors(cfg, t)
    ws = qm.new_workspace(layer, 1)
    t0 = time.perf_counter()
    qm.moe_selftest_grid_timeout(ws, 2_000_000)    # 2 ms
    assert qm.moe_poll_status(ws) == MOE_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert qm.moe_poll_status(ws) == 0
    torch.cuda.synchronize()
    assert int(ws[64:68].cpu().numpy().view(np.uint32)[0]) == 0   # the arrival counter was cleared
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    experts = [fixtures.host_expert(cfg, 0, e) for e in range(cfg.E)]
    shared = fixtures.host_expert(cfg, 0, cfg.E)
    for s in range(3):
        x = gen.x_tokens(cfg, 30 + s, T=1)
        h0 = gen.bf16_bits_to_f32(x).astype(np.float32)
        h = torch.from_numpy(h0.copy()).to(dev)
        xo = torch.empty((1, cfg.H), dtype=torch.int16, device=dev)
        xf = torch.empty((1, cfg.H), dtype=torch.float32, device=dev)
        idx = torch.empty((1, cfg.k), dtype=torch.int32, device=dev)
        qm.moe_layer_forward(layer, torch.from_numpy(x.view(np.int16)).to(dev), h, xo, xf, idx, ws=ws)
        assert qm.moe_poll_status(ws) == 0
        ref = oracle.layer(x, h0.astype(np.float64), Wr, gamma, experts, shared, I=cfg.I, k=cfg.k, G=cfg.G,
                           bits=cfg.bits, eps=cfg.rms_eps, gs=gs)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
        r = ref["x_out"][0]
        assert np.max(np.abs(xf[0].cpu().numpy() - r)) / np.max(np.abs(r)) <= 2e-3
