"""GPU: MXFP4 expert matrices (E2M1 codes, E8M0 scale per 32) against the oracle.

moe_expert_gemv_mxfp4 (decode mat-vec, fp32 block sums) and
moe_expert_gemm_mxfp4 (many tokens on tcgen05 kind::mxf4 with block scaling;
the bf16 activations as five E2M1 terms) are compared with the oracle's
double-precision products on the same seeded inputs, at sizes spanning
several tiles with ragged tails, the expert shapes of the 4-bit layer
(hidden 4096, intermediate 1024), the largest accepted K, and the degenerate
cases (zero activations, an outlier element, the NaN scale byte)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_decode_moe_b200 as qm
from fixtures import gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available()
    qm.lib()
    return torch.device("cuda")


def normwise(got, ref):
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300))


def mat(q, e, dev):
    return qm.MxMat(torch.from_numpy(q.view(np.int32)).to(dev), torch.from_numpy(e).to(dev))


def gemv(q, e, x, dev):
    W = mat(q, e, dev)
    xd = torch.from_numpy(x.astype(np.float32)).to(dev)
    y = torch.empty(q.shape[0], dtype=torch.float32, device=dev)
    qm.moe_expert_gemv_mxfp4(W, xd, y)
    return y.cpu().numpy()


def gemm(q, e, xb, dev):
    R, K = q.shape[0], q.shape[1] * 8
    W = mat(q, e, dev)
    ws = qm.new_mx_workspace(R, K, xb.shape[0])
    y = torch.full((xb.shape[0], R), float("nan"), dtype=torch.float32, device=dev)
    qm.moe_expert_gemm_mxfp4(W, torch.from_numpy(xb.view(np.int16)).to(dev), y, ws=ws)
    assert qm.moe_poll_status(ws) == 0
    return y.cpu().numpy()


# ------------------------------------------------------------------ mat-vec
@pytest.mark.parametrize("R,K", [(16, 64), (40, 96), (1024, 4096), (4096, 1024), (24, 8192), (3, 32)])
def test_gemv_matches_oracle(dev, R, K):
    q, e = gen.mx_matrix(R + K, R, K)
    x = gen.bf16_bits_to_f32(gen.mx_tokens(R, 1, K)[0]).astype(np.float64)
    got = gemv(q, e, x, dev)
    ref = oracle.mx_gemv(q, e, x, K)
    err = normwise(got, ref)
    # fp32 products and sums over at most 8192 terms: far inside the 2e-3 contract
    assert err <= 1e-5, err


def test_gemv_nan_scale_and_zero_codes(dev):
    """Scale byte 0xFF is NaN in the format: that row's output is NaN; an all-zero row is 0."""
    R, K = 8, 128
    q, e = gen.mx_matrix(5, R, K)
    q[2] = 0
    e[5, 1] = 0xFF
    x = np.linspace(-1, 1, K)
    got = gemv(q, e, x, dev)
    ref = oracle.mx_gemv(q, e, x, K)
    assert np.isnan(got[5]) and np.isnan(ref[5])
    assert got[2] == 0.0
    keep = [i for i in range(R) if i != 5]
    assert normwise(got[keep], ref[keep]) <= 1e-5


# ------------------------------------------------------------------ many tokens (tcgen05)
@pytest.mark.parametrize("R,K,T", [(128, 128, 1), (128, 256, 9), (256, 1024, 40), (384, 512, 130),
                                   (2048, 4096, 512), (4096, 1024, 64), (128, 8192, 33)])
def test_gemm_matches_oracle(dev, R, K, T):
    """One 128 x 128 tile up to the shared expert's gate/up (2048 x 4096, 512 tokens); ragged token
    tails (1, 9, 33, 40, 130); one 128-column stage up to 64 stages."""
    q, e = gen.mx_matrix(R * 7 + K, R, K)
    xb = gen.mx_tokens(T + K, T, K)
    got = gemm(q, e, xb, dev)
    ref = oracle.mx_gemm(q, e, xb, K)
    err = normwise(got, ref)
    # five E2M1 terms leave a residual below 4^-4/3 of each block's largest |x|; about 5e-5 normwise
    assert err <= 5e-4, err
    print(f"mxfp4 gemm R={R} K={K} T={T}: normwise error {err:.2e}")


def test_gemm_rows_equal_gemv_within_the_term_error(dev):
    """The tensor-core product of one token against the mat-vec of the same token (two
    independent kernels, different arithmetic), both against the oracle."""
    R, K = 1024, 4096
    q, e = gen.mx_matrix(77, R, K)
    xb = gen.mx_tokens(78, 1, K)
    x = gen.bf16_bits_to_f32(xb[0]).astype(np.float64)
    a = gemm(q, e, xb, dev)[0]
    b = gemv(q, e, x, dev)
    ref = oracle.mx_gemv(q, e, x, K)
    assert normwise(a, ref) <= 5e-4 and normwise(b, ref) <= 1e-5


def test_gemm_degenerate_activations(dev):
    """Zero tokens give exactly zero; a token whose one element is 2^10 times the rest costs only
    its own block; tokens of very different magnitudes in one tile keep their own scales."""
    R, K, T = 256, 1024, 6
    q, e = gen.mx_matrix(9, R, K)
    x = gen.bf16_bits_to_f32(gen.mx_tokens(10, T, K)).astype(np.float32)
    x[0] = 0.0
    x[1, 100] *= 1024.0
    x[2] *= 2.0 ** -40
    x[3] *= 2.0 ** 40
    x[4, ::2] = 0.0
    xb = gen.f32_to_bf16_bits(x)
    got = gemm(q, e, xb, dev)
    ref = oracle.mx_gemm(q, e, xb, K)
    assert np.all(got[0] == 0.0)
    for t in range(1, T):
        assert normwise(got[t], ref[t]) <= 5e-4, t


def test_gemm_rejects_bad_shapes_before_launch(dev):
    q, e = gen.mx_matrix(1, 256, 256)
    W = mat(q, e, dev)
    x = torch.zeros((4, 256), dtype=torch.int16, device=dev)
    y = torch.empty((4, 256), dtype=torch.float32, device=dev)
    ws = qm.new_mx_workspace(256, 256, 4)
    with pytest.raises(qm.MoeError) as ex:   # workspace for fewer tokens than the call has
        qm.moe_expert_gemm_mxfp4(W, torch.zeros((400, 256), dtype=torch.int16, device=dev),
                                 torch.empty((400, 256), dtype=torch.float32, device=dev), ws=ws)
    assert ex.value.code == 3
    with pytest.raises(qm.MoeError) as ex:   # R not a multiple of 128
        qm.moe_expert_gemm_mxfp4(qm.MxMat(W.q[:200], W.scales[:200]), x, y, ws=ws)
    assert ex.value.code == 2


# ------------------------------------------------------------------ a decode layer of MXFP4 experts
import fixtures  # noqa: E402


def mx_layer(name, E, dev, scale=(116, 120), k=None, shared=True):
    """The router, gamma and shared-gate vectors of a fixture layer with MXFP4 experts (seeded)."""
    base = fixtures.CONFIGS[name]
    k = base.k if k is None else k
    cfg = base if (E, k, shared) == (base.E, base.k, True) else fixtures.Config(
        base.name, H=base.H, E=E, k=k, I=base.I, bits=4, scale_sigma=base.scale_sigma, has_shared=shared)
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    H, I = cfg.H, cfg.I
    host = [gen.mx_expert(e, H, I, *scale) for e in range(E + 1)]

    def dev_expert(ex):
        return qm.Expert(*[qm.QMat(torch.from_numpy(q.view(np.int32)).to(dev), torch.from_numpy(e).to(dev), None)
                           for q, e in ex])

    def t16(a):
        return torch.from_numpy(a.view(np.int16)).to(dev)

    layer = qm.Layer(hidden=H, inter=I, top_k=cfg.k, bits=4, group=32, router_w=t16(Wr),
                     experts=[dev_expert(ex) for ex in host[:E]], rms_gamma=t16(gamma),
                     shared=dev_expert(host[E]) if shared else None, shared_gate_w=t16(gs) if shared else None,
                     router_bias=torch.from_numpy(rb).to(dev) if rb is not None else None, rms_eps=cfg.rms_eps)
    return cfg, layer, host, (Wr, rb, gs, gamma)


def run_mx_layer(cfg, layer, x, h0, dev):
    T, H = x.shape
    ws = qm.new_workspace(layer, T)
    h = torch.from_numpy(h0.astype(np.float32)).to(dev)
    xo = torch.empty((T, H), dtype=torch.int16, device=dev)
    xf = torch.empty((T, H), dtype=torch.float32, device=dev)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    qm.moe_layer_forward(layer, torch.from_numpy(x.view(np.int16)).to(dev), h, xo, xf, idx, w, ws=ws)
    assert qm.moe_poll_status(ws) == 0
    return h.cpu().numpy(), xf.cpu().numpy(), xo.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("name,E,T", [("tiny", 16, 1), ("tiny", 16, 3), ("tiny", 16, 8), ("layer_q4", 64, 1),
                                      ("layer_q4", 64, 4), ("tiny", 16, 40), ("layer_q4", 64, 130)])
def test_mx_layer_matches_oracle(dev, name, E, T):
    """Router, top-k, MXFP4 gate/up + SwiGLU, down + weighted combine + residual, RMSNorm: routing
    bit-exact, outputs within the layer tolerance of the oracle's composition of its own steps
    (hidden 256 / 16 experts, and hidden 4096 / intermediate 1024 / 64 experts, top-3 + shared);
    T = 40 and 130 take the many-token router (tcgen05) and run the experts per token."""
    cfg, layer, host, (Wr, rb, gs, gamma) = mx_layer(name, E, dev)
    x = gen.x_tokens(cfg, 31 + T, T=T)
    h0 = gen.bf16_bits_to_f32(x).astype(np.float64) * 0.5
    h, xf, xo, idx, w = run_mx_layer(cfg, layer, x, h0, dev)
    ref = oracle.mx_layer(x, h0, Wr, gamma, host[:E], host[E], k=cfg.k, eps=cfg.rms_eps, router_bias=rb, gs=gs)
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_allclose(w, ref["w"], rtol=1e-6, atol=1e-7)
    eh, ex_ = normwise(h, ref["h_out"]), normwise(xf, ref["x_out"])
    assert eh <= 2e-3 and ex_ <= 2e-3, (eh, ex_)
    assert eh <= 1e-4 and ex_ <= 1e-4, (eh, ex_)   # fp32 sums of exact products: far inside the bar
    assert np.array_equal(xo.view(np.uint16), gen.f32_to_bf16_bits(xf))   # x_out is the RNE of x_out_f32
    print(f"mxfp4 layer {name} E={E} T={T}: h' {eh:.2e}, x_out {ex_:.2e}")


@pytest.mark.parametrize("k,shared,T", [(1, False, 1), (5, True, 2), (8, True, 1), (8, True, 12)])
def test_mx_layer_slot_counts(dev, k, shared, T):
    """1 to 9 expert slots per token (top-1 without the shared expert, top-5 and top-8 with it): the
    down kernel holds up to 2, 6 or 9 slots in registers; routing bit-exact, outputs within the
    layer tolerance of the oracle."""
    cfg, layer, host, (Wr, rb, gs, gamma) = mx_layer("tiny", 16, dev, k=k, shared=shared)
    x = gen.x_tokens(cfg, 77 + k, T=T)
    h0 = gen.bf16_bits_to_f32(x).astype(np.float64) * 0.5
    h, xf, xo, idx, w = run_mx_layer(cfg, layer, x, h0, dev)
    ref = oracle.mx_layer(x, h0, Wr, gamma, host[:16], host[16] if shared else None, k=k, eps=cfg.rms_eps,
                          router_bias=rb, gs=gs if shared else None)
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_allclose(w, ref["w"], rtol=1e-6, atol=1e-7)
    eh, ex_ = normwise(h, ref["h_out"]), normwise(xf, ref["x_out"])
    assert eh <= 1e-4 and ex_ <= 1e-4, (eh, ex_)


def test_mx_layer_path_and_limits(dev):
    cfg, layer, _, _ = mx_layer("tiny", 16, dev)
    path, nev = C_int(), C_int()
    assert qm.lib().moe_layer_path(layer.cref(), 4, C.byref(path), C.byref(nev)) == 0
    assert (path.value, nev.value) == (4, 5)
    assert qm.lib().moe_layer_path(layer.cref(), 9, C.byref(path), C.byref(nev)) == 0   # many tokens too
    assert path.value == 4


def test_mx_stack_equals_layer_by_layer(dev):
    """Two MXFP4 layers through moe_stack_forward equal two moe_layer_forward calls, bit for bit."""
    cfg, l0, _, _ = mx_layer("tiny", 16, dev)
    _, l1, _, _ = mx_layer("tiny", 16, dev, scale=(115, 119))
    x = gen.x_tokens(cfg, 5, T=1)
    h0 = gen.bf16_bits_to_f32(x).astype(np.float32)
    ws = qm.new_workspace(l0, 1)
    h = torch.from_numpy(h0.copy()).to(dev)
    xo = torch.empty((1, cfg.H), dtype=torch.int16, device=dev)
    idx_all = torch.empty((2, cfg.k), dtype=torch.int32, device=dev)
    qm.moe_stack_forward([l0, l1], torch.from_numpy(x.view(np.int16)).to(dev), h, xo, idx_all, ws=ws)
    a = run_mx_layer(cfg, l0, x, h0, dev)
    b = run_mx_layer(cfg, l1, a[2].view(np.uint16), a[0], dev)
    np.testing.assert_array_equal(h.cpu().numpy(), b[0])
    np.testing.assert_array_equal(xo.cpu().numpy(), b[2])
    np.testing.assert_array_equal(idx_all.cpu().numpy(), np.stack([a[3][0], b[3][0]]))


import ctypes as C  # noqa: E402
C_int = C.c_int32
