"""moe_layer_forward_noalloc: the layer forward for callers that cannot
allocate device memory themselves (a plug-in that only receives its input and
output buffers from a host application owning all device memory, or a
latency-critical loop that must not call cudaMalloc). Instead of a workspace
it uses one static scratch array inside the library.

Checked through the C ABI against moe_layer_forward with a caller-owned
workspace, within the parity tolerance, on two calls in a row (the second
call finds the first call's leftovers in the shared scratch). This file is
collected last so that a run stopping at the first failure has run every
other test already; it also passes on its own in a fresh process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import fixtures
import fixtures.gpu as fxg
import quantized_expert_decode_moe_b200 as qm
from fixtures import gen

pytestmark = pytest.mark.gpu
TOL = 2e-3


def rel_err(a, r):
    a, r = np.asarray(a, np.float64), np.asarray(r, np.float64)
    return float(np.max(np.abs(a - r)) / max(np.max(np.abs(r)), 1e-30))


def _run(fn, layer, cfg, x_bits, ws=None):
    T = x_bits.shape[0]
    dev = torch.device("cuda")
    xd = torch.from_numpy(x_bits.view(np.int16)).to(dev)
    h = torch.from_numpy(gen.bf16_bits_to_f32(x_bits).astype(np.float32)).to(dev)
    xo = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
    xf = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    if ws is None:
        fn(layer, xd, h, xo, xf, idx, w)
    else:
        fn(layer, xd, h, xo, xf, idx, w, ws=ws)
    torch.cuda.synchronize()
    return dict(h=h.cpu().numpy(), xf=xf.cpu().numpy(), xo=xo.cpu().numpy(), idx=idx.cpu().numpy(),
                w=w.cpu().numpy())


@pytest.mark.parametrize("name,T", [("tiny", 1), ("tiny", 3), ("layer_q4", 1), ("layer_q2", 2)])
def test_noalloc_forward_matches_workspace_forward(name, T):
    cfg = fixtures.CONFIGS[name]
    n = None if name == "tiny" else 32          # a 32-expert slice of the big layers keeps this quick
    t = fxg.device_layer(cfg, 0, n_experts=n)
    c = cfg if n is None else fixtures.Config(cfg.name, H=cfg.H, E=n, k=cfg.k, I=cfg.I, bits=cfg.bits,
                                               scale_sigma=cfg.scale_sigma)
    layer = qm.layer_from_tensors(c, t)
    ws = qm.new_workspace(layer, T)
    for call in range(2):
        x = gen.x_tokens(c, 40 + call, T=T)
        ref = _run(qm.moe_layer_forward, layer, c, x, ws=ws)
        got = _run(qm.moe_layer_forward_noalloc, layer, c, x)
        np.testing.assert_array_equal(got["idx"], ref["idx"])
        assert rel_err(got["w"], ref["w"]) <= TOL
        for i in range(T):
            assert rel_err(got["h"][i], ref["h"][i]) <= TOL
            assert rel_err(got["xf"][i], ref["xf"][i]) <= TOL
    assert qm.moe_noalloc_poll_status() == 0     # nothing latched in the static scratch


def test_noalloc_scratch_covers_largest_decode_shape():
    """Every decode shape the library accepts fits the static scratch, so the
    oversize rejection cannot trigger for a call that could otherwise run:
    the workspace for 8 tokens stays within MOE_NOALLOC_SCRATCH_BYTES at the
    largest hidden and intermediate sizes the decode kernels take (4 and 2
    bits, top-3 and top-8 with a shared expert, 4096 experts). A shape the
    decode kernels cannot run, and more than 8 tokens, are refused as
    unsupported before the scratch is touched."""
    L = qm.lib()
    p = 0x100000
    ex = qm._Expert(*[qm._QMat(p, p, p) for _ in range(3)])
    # the digit-block kernels take hidden and intermediate up to 8192 with top-3 + shared, and
    # intermediate up to 7296 with top-8 + shared (their down kernel's digit blocks of a)
    cases = [(4, 3, 8192, 8192), (4, 8, 8192, 7296), (2, 3, 8192, 8192), (2, 8, 8192, 7296)]
    for bits, k, H, I in cases:
        lay = qm._Layer(H, I, 4096, k, bits, 64, 1, 1e-6, p, None, p, ex, p, p)
        n = C.c_size_t(0)
        assert L.moe_workspace_size(C.byref(lay), 8, C.byref(n)) == 0, (bits, k, H, I)
        assert 0 < n.value <= qm.NOALLOC_SCRATCH_BYTES
        big = qm._Layer(H, I + 128, 4096, k, bits, 64, 1, 1e-6, p, None, p, ex, p, p)
        assert L.moe_workspace_size(C.byref(big), 8, C.byref(n)) == 2   # one span more: no longer fits
    pp = C.c_void_p(0x200000)
    lay = qm._Layer(4096, 1024, 512, 3, 4, 64, 1, 1e-6, p, None, p, ex, p, p)
    assert L.moe_layer_forward_noalloc(C.byref(lay), pp, pp, 9, pp, None, None, None, None) == 2   # MOE_ERR_UNSUPPORTED
    bad = qm._Layer(8192, 7424, 512, 8, 4, 64, 1, 1e-6, p, None, p, ex, p, p)
    assert L.moe_layer_forward_noalloc(C.byref(bad), pp, pp, 1, pp, None, None, None, None) == 2
