"""Device-side failure path on the GPU, without a fault: a bounded wait runs
out (a barrier phase that nothing completes), the kernel latches
MOE_ERR_TIMEOUT in the workspace status word and returns; the host reads it
with moe_poll_status and the same context and workspace then serve a normal
call that matches the oracle."""
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
