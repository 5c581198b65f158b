"""Device-side generation of the same seeded inputs as ``fixtures.gen``.

Builds ``libmoe_fixtures.so`` from ``gen_gpu.cu`` and fills torch device
tensors in place. Bit-identical to the host generator (checked by a GPU test).
"""
from __future__ import annotations

import ctypes as C
import os
import shutil
import subprocess

import numpy as np

from . import gen

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen_gpu.cu")
_LIB = os.path.join(_HERE, "libmoe_fixtures.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc, "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
                               "-shared", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.fx_codes.argtypes = [C.c_void_p, C.c_void_p, C.c_uint64, C.c_uint64, C.c_void_p]
        _lib.fx_normal.argtypes = [C.c_void_p, C.c_void_p, C.c_uint64, C.c_uint64, C.c_void_p, C.c_int, C.c_void_p,
                                   C.c_int, C.c_void_p]
        _lib.fx_bias.argtypes = [C.c_void_p, C.c_void_p, C.c_uint64, C.c_int, C.c_void_p]
    return _lib


def _stream():
    import torch
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _keys(keys, device):
    import torch
    arr = np.array([k & ((1 << 64) - 1) for k in keys], dtype=np.uint64).view(np.int64)
    return torch.from_numpy(arr).to(device)


_tables = {}


def _table(sigma: float, device):
    import torch
    key = (sigma, str(device))
    if key not in _tables:
        t = gen.normal_table(sigma)
        thr = torch.from_numpy(t.thresholds.view(np.int32).copy()).to(device)
        vals = torch.from_numpy(t.values.view(np.int16).copy()).to(device)
        _tables[key] = (thr, vals, len(t.thresholds))
    return _tables[key]


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"fixture kernel launch failed (cuda error {rc})")


def fill_codes(out, keys, per: int):
    """out: int32 device tensor with len(keys)*per elements."""
    k = _keys(keys, out.device)
    _check(lib().fx_codes(C.c_void_p(out.data_ptr()), C.c_void_p(k.data_ptr()), per, out.numel(), _stream()))
    return k


def fill_normal(out, keys, per: int, sigma: float, signed: bool):
    """out: int16 device tensor (bf16 bit patterns) with len(keys)*per elements."""
    k = _keys(keys, out.device)
    thr, vals, n = _table(sigma, out.device)
    _check(lib().fx_normal(C.c_void_p(out.data_ptr()), C.c_void_p(k.data_ptr()), per, out.numel(),
                           C.c_void_p(thr.data_ptr()), n, C.c_void_p(vals.data_ptr()), int(signed), _stream()))
    return k


def fill_bias(out, scales, bits: int):
    _check(lib().fx_bias(C.c_void_p(out.data_ptr()), C.c_void_p(scales.data_ptr()), out.numel(), bits, _stream()))


def device_layer(cfg: gen.Config, layer: int, device="cuda", n_experts: int | None = None, expert_ids=None):
    """All tensors of one layer on the device, generated in place.

    Returns a dict: q[m], s[m], b[m] (m = 0 gate, 1 up, 2 down) of shape
    [E+1][R][...] (index E is the shared expert), router_w [E][H] (int16 bf16
    bits), router_bias [E] fp32 or None, gate_w [H], gamma [H].
    n_experts < E generates only the first n_experts routed experts (stream
    ids 0..n-1) plus the shared one (stream id E, stored at index n);
    expert_ids lists the stream ids to generate instead, stored in that order."""
    import torch
    E = cfg.E if n_experts is None else n_experts
    ids = list(range(E)) + [cfg.E] if expert_ids is None else list(expert_ids)
    nexp = len(ids)
    out = {"q": [], "s": [], "b": []}
    keep = []
    for m, shp in enumerate(gen.expert_mat_shapes(cfg.H, cfg.I)):
        wpr = shp.K * cfg.bits // 32
        q = torch.empty((nexp, shp.R, wpr), dtype=torch.int32, device=device)
        keep.append(fill_codes(q, [gen.key_of(cfg.seed, layer, gen.T_CODES + m, e) for e in ids], shp.R * wpr))
        s = torch.empty((nexp, shp.R, shp.K // cfg.G), dtype=torch.int16, device=device)
        keep.append(fill_normal(s, [gen.key_of(cfg.seed, layer, gen.T_SCALES + m, e) for e in ids],
                                shp.R * (shp.K // cfg.G), cfg.scale_sigma, signed=False))
        b = torch.empty_like(s)
        fill_bias(b, s, cfg.bits)
        out["q"].append(q); out["s"].append(s); out["b"].append(b)
    rw = torch.empty((cfg.E if expert_ids is not None else E, cfg.H), dtype=torch.int16, device=device)
    keep.append(fill_normal(rw, [gen.key_of(cfg.seed, layer, gen.T_ROUTER_W)], rw.numel(), cfg.router_sigma, True))
    out["router_w"] = rw
    rb = gen.router_bias_f32(cfg.seed, layer, cfg.E)[:E] if cfg.router_bias else None
    out["router_bias"] = torch.from_numpy(rb.copy()).to(device) if rb is not None else None
    gs = gen.normal_bf16(gen.key_of(cfg.seed, layer, gen.T_SHARED_GATE), cfg.H, cfg.gate_sigma)
    out["gate_w"] = torch.from_numpy(gs.view(np.int16).copy()).to(device)
    out["gamma"] = torch.from_numpy(gen.gamma_bf16(cfg.seed, layer, cfg.H).view(np.int16).copy()).to(device)
    torch.cuda.current_stream().synchronize()
    del keep
    return out

