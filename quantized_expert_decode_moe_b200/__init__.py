"""B200 (sm_100a) quantized MoE expert forward: thin Python binding.

Every function here has the name of the C-ABI entry point it wraps (see
``include/moe.h``) and only marshals arguments: torch device tensors become raw
pointers, the current torch stream becomes the cudaStream_t. All arithmetic
runs in the CUDA kernels of ``libmoe_b200.so``; there is no fallback path. If
the library is missing and cannot be built, importing any entry point raises.
"""
from __future__ import annotations

import ctypes as C
import os

__all__ = [
    "MoeError", "QMat", "Expert", "Layer", "lib", "build",
    "moe_abi_version", "moe_status_string", "moe_workspace_size", "moe_workspace_init", "moe_layer_path", "moe_route",
    "moe_expert_gemv_q4", "moe_expert_gemv_q2", "moe_combine_residual_norm", "moe_group_tokens",
    "moe_layer_forward", "moe_layer_forward_noalloc", "moe_layer_forward_timed", "moe_stack_forward", "moe_poll_status",
    "moe_selftest_wait_timeout", "moe_selftest_grid_timeout", "moe_noalloc_poll_status", "new_workspace",
    "MxMat", "moe_expert_gemv_mxfp4", "moe_mxfp4_workspace_size", "moe_expert_gemm_mxfp4", "new_mx_workspace",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")
_lib = None

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARGUMENT", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_DEVICE_FAULT"}


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({moe_status_string(code)})")


class _QMat(C.Structure):
    _fields_ = [("q", C.c_void_p), ("scales", C.c_void_p), ("biases", C.c_void_p)]


class _Expert(C.Structure):
    _fields_ = [("gate", _QMat), ("up", _QMat), ("down", _QMat)]


class _MxMat(C.Structure):
    _fields_ = [("q", C.c_void_p), ("scales", C.c_void_p)]


class _Layer(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("inter", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
                ("bits", C.c_int32), ("group", C.c_int32), ("has_shared", C.c_int32), ("rms_eps", C.c_float),
                ("router_w", C.c_void_p), ("router_bias", C.c_void_p), ("experts", C.c_void_p),
                ("shared", _Expert), ("shared_gate_w", C.c_void_p), ("rms_gamma", C.c_void_p)]


def build(force: bool = False) -> str:
    from . import buildlib
    return buildlib.build(force=force)


def lib():
    """The loaded CUDA library (built in-tree first if it is missing or stale)."""
    global _lib
    if _lib is None:
        try:
            path = build()
        except Exception as e:  # no nvcc: only a prebuilt library will do
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libmoe_b200.so is missing and could not be built: {e}") from e
            path = LIB_PATH
        L = C.CDLL(path)
        vp, i32, f32 = C.c_void_p, C.c_int32, C.c_float
        L.moe_abi_version.restype = i32
        L.moe_status_string.restype = C.c_char_p
        L.moe_status_string.argtypes = [C.c_int]
        L.moe_workspace_size.argtypes = [vp, i32, C.POINTER(C.c_size_t)]
        L.moe_workspace_init.argtypes = [vp, C.c_size_t, vp]
        L.moe_layer_path.argtypes = [vp, i32, C.POINTER(i32), C.POINTER(i32)]
        L.moe_route.argtypes = [vp, vp, i32, vp, vp, vp, vp, C.c_size_t, vp]
        L.moe_expert_gemv_q4.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.moe_expert_gemv_q2.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.moe_combine_residual_norm.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, f32, vp, vp, vp]
        L.moe_group_tokens.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, C.c_size_t, vp]
        L.moe_layer_forward.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, C.c_size_t, vp]
        L.moe_layer_forward_timed.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, C.c_size_t, vp, i32, vp]
        L.moe_layer_forward_noalloc.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp]
        L.moe_stack_forward.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, C.c_size_t, vp]
        L.moe_poll_status.argtypes = [vp, vp]
        L.moe_selftest_wait_timeout.argtypes = [vp, C.c_size_t, C.c_uint64, vp]
        L.moe_selftest_grid_timeout.argtypes = [vp, C.c_size_t, C.c_uint64, vp]
        L.moe_noalloc_poll_status.argtypes = [vp]
        sz = C.POINTER(C.c_size_t)
        u64 = C.POINTER(C.c_uint64)
        L.moe_cache_size.argtypes = [vp, i32, sz, sz]
        L.moe_cache_init.argtypes = [vp, vp, i32, vp, C.c_size_t, vp, C.c_size_t]
        L.moe_cache_admit.argtypes = [vp, vp, i32, vp, vp]
        L.moe_layer_forward_cached.argtypes = [vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, C.c_size_t, vp]
        L.moe_cache_stats.argtypes = [vp, u64, u64, u64]
        L.moe_expert_gemv_mxfp4.argtypes = [vp, i32, i32, vp, vp, vp]
        L.moe_mxfp4_workspace_size.argtypes = [i32, i32, i32, sz]
        L.moe_expert_gemm_mxfp4.argtypes = [vp, i32, i32, vp, i32, vp, vp, C.c_size_t, vp]
        _lib = L
    return _lib


# ------------------------------------------------------------------ marshalling helpers
def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ok(rc: int, where: str):
    if rc != 0:
        raise MoeError(rc, where)


class QMat:
    """One packed matrix: codes int32 [R][K*bits/32], scales/biases int16 (bf16 bits) [R][K/64].
    In a layer of MXFP4 experts (group 32): codes int32 [R][K/8], scales uint8 E8M0 [R][K/32], biases None."""

    def __init__(self, q, scales, biases):
        self.q, self.scales, self.biases = q, scales, biases

    def c(self) -> _QMat:
        return _QMat(self.q.data_ptr(), self.scales.data_ptr(), self.biases.data_ptr() if self.biases is not None else None)


class Expert:
    def __init__(self, gate: QMat, up: QMat, down: QMat):
        self.gate, self.up, self.down = gate, up, down

    def c(self) -> _Expert:
        return _Expert(self.gate.c(), self.up.c(), self.down.c())


class Layer:
    """Device tensors of one MoE layer and the moe_layer descriptor pointing at them.

    experts: list of E Expert (routed); shared: Expert or None."""

    def __init__(self, *, hidden, inter, top_k, bits, router_w, experts, rms_gamma, shared=None,
                 shared_gate_w=None, router_bias=None, rms_eps=1e-6, group=64):
        import torch
        self.hidden, self.inter, self.top_k, self.bits, self.group = hidden, inter, top_k, bits, group
        self.n_experts = len(experts)
        self.router_w, self.router_bias, self.rms_gamma = router_w, router_bias, rms_gamma
        self.shared, self.shared_gate_w, self.experts, self.rms_eps = shared, shared_gate_w, experts, rms_eps
        table = []
        for ex in experts:
            for m in (ex.gate, ex.up, ex.down):
                table += [m.q.data_ptr(), m.scales.data_ptr(), m.biases.data_ptr() if m.biases is not None else 0]
        self.expert_table = torch.tensor(table, dtype=torch.int64).to(router_w.device)
        self._c = _Layer(hidden, inter, self.n_experts, top_k, bits, group, 1 if shared is not None else 0,
                         float(rms_eps), router_w.data_ptr(), router_bias.data_ptr() if router_bias is not None else None,
                         self.expert_table.data_ptr(), shared.c() if shared is not None else _Expert(),
                         shared_gate_w.data_ptr() if shared_gate_w is not None else None, rms_gamma.data_ptr())

    def cref(self):
        return C.byref(self._c)


def layer_from_tensors(cfg, t: dict, n_experts: int | None = None) -> Layer:
    """Layer over the tensors of ``fixtures.gpu.device_layer`` (expert index E = shared)."""
    E = cfg.E if n_experts is None else n_experts

    def ex(e):
        return Expert(*[QMat(t["q"][m][e], t["s"][m][e], t["b"][m][e]) for m in range(3)])

    return Layer(hidden=cfg.H, inter=cfg.I, top_k=cfg.k, bits=cfg.bits, router_w=t["router_w"],
                 experts=[ex(e) for e in range(E)], rms_gamma=t["gamma"], shared=ex(E) if cfg.has_shared else None,
                 shared_gate_w=t["gate_w"] if cfg.has_shared else None, router_bias=t["router_bias"],
                 rms_eps=cfg.rms_eps, group=cfg.G)


# ------------------------------------------------------------------ entry points
def moe_abi_version() -> int:
    return lib().moe_abi_version()


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def moe_workspace_size(layer: Layer, max_tokens: int) -> int:
    n = C.c_size_t(0)
    _ok(lib().moe_workspace_size(layer.cref(), int(max_tokens), C.byref(n)), "moe_workspace_size")
    return n.value


PATHS = {1: "fused", 2: "chain", 3: "prefill", 4: "mxfp4", 5: "digit"}
NOALLOC_SCRATCH_BYTES = 8 << 20   # MOE_NOALLOC_SCRATCH_BYTES of include/moe.h


def moe_layer_path(layer: Layer, T: int):
    """(path name, events moe_layer_forward_timed records) for a call of T tokens on layer."""
    path, nev = C.c_int32(0), C.c_int32(0)
    _ok(lib().moe_layer_path(layer.cref(), int(T), C.byref(path), C.byref(nev)), "moe_layer_path")
    return PATHS[path.value], nev.value


def moe_workspace_init(ws, stream=None):
    _ok(lib().moe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_workspace_init")


def new_workspace(layer: Layer, max_tokens: int, device="cuda"):
    """A zero-initialised workspace tensor (caller-owned device memory)."""
    import torch
    ws = torch.zeros(moe_workspace_size(layer, max_tokens), dtype=torch.uint8, device=device)
    return ws


def moe_route(layer: Layer, x, topk_idx, topk_w, shared_gate=None, *, ws, stream=None):
    _ok(lib().moe_route(layer.cref(), _ptr(x), x.shape[0], _ptr(topk_idx), _ptr(topk_w), _ptr(shared_gate),
                        _ptr(ws), ws.numel(), _stream(stream)), "moe_route")


def moe_expert_gemv_q4(W: QMat, R: int, K: int, group: int, x, y, stream=None):
    w = W.c()
    _ok(lib().moe_expert_gemv_q4(C.byref(w), R, K, group, _ptr(x), _ptr(y), _stream(stream)), "moe_expert_gemv_q4")


def moe_expert_gemv_q2(W: QMat, R: int, K: int, group: int, x, y, stream=None):
    w = W.c()
    _ok(lib().moe_expert_gemv_q2(C.byref(w), R, K, group, _ptr(x), _ptr(y), _stream(stream)), "moe_expert_gemv_q2")


class MxMat:
    """One MXFP4 matrix: codes int32 [R][K/8] (E2M1 nibbles), scales uint8 [R][K/32] (E8M0)."""

    def __init__(self, q, scales):
        self.q, self.scales = q, scales

    def c(self) -> _MxMat:
        return _MxMat(self.q.data_ptr(), self.scales.data_ptr())


def moe_expert_gemv_mxfp4(W: MxMat, x, y, stream=None):
    """y = W x (fp32 [K] -> fp32 [R])."""
    w = W.c()
    R, K = W.scales.shape[0], W.scales.shape[1] * 32
    _ok(lib().moe_expert_gemv_mxfp4(C.byref(w), R, K, _ptr(x), _ptr(y), _stream(stream)), "moe_expert_gemv_mxfp4")


def moe_mxfp4_workspace_size(R: int, K: int, T: int) -> int:
    n = C.c_size_t(0)
    _ok(lib().moe_mxfp4_workspace_size(int(R), int(K), int(T), C.byref(n)), "moe_mxfp4_workspace_size")
    return n.value


def new_mx_workspace(R: int, K: int, T: int, device="cuda"):
    """A zero-initialised workspace for moe_expert_gemm_mxfp4 (caller-owned device memory)."""
    import torch
    return torch.zeros(moe_mxfp4_workspace_size(R, K, T), dtype=torch.uint8, device=device)


def moe_expert_gemm_mxfp4(W: MxMat, x, y, *, ws, stream=None):
    """Y[t] = W x[t]: x bf16 bits int16 [T][K], y fp32 [T][R]."""
    w = W.c()
    R, K = W.scales.shape[0], W.scales.shape[1] * 32
    _ok(lib().moe_expert_gemm_mxfp4(C.byref(w), R, K, _ptr(x), x.shape[0], _ptr(y), _ptr(ws), ws.numel(),
                                    _stream(stream)), "moe_expert_gemm_mxfp4")


def moe_combine_residual_norm(y_routed, topk_w, y_shared, shared_gate, h, gamma, eps: float, x_out, x_out_f32=None,
                              stream=None):
    T, H = h.shape
    k = y_routed.shape[1] if y_routed is not None else 0
    _ok(lib().moe_combine_residual_norm(T, H, k, _ptr(y_routed), _ptr(topk_w), _ptr(y_shared), _ptr(shared_gate),
                                        _ptr(h), _ptr(gamma), float(eps), _ptr(x_out), _ptr(x_out_f32),
                                        _stream(stream)), "moe_combine_residual_norm")


def moe_group_tokens(topk_idx, E: int, counts, offsets, perm, ws=None, stream=None):
    T, k = topk_idx.shape
    _ok(lib().moe_group_tokens(T, k, E, _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(ws),
                               0 if ws is None else ws.numel(), _stream(stream)), "moe_group_tokens")


def moe_layer_forward(layer: Layer, x_in, h, x_out, x_out_f32=None, topk_idx=None, topk_w=None, *, ws, stream=None):
    _ok(lib().moe_layer_forward(layer.cref(), _ptr(x_in), _ptr(h), x_in.shape[0], _ptr(x_out), _ptr(x_out_f32),
                                _ptr(topk_idx), _ptr(topk_w), _ptr(ws), ws.numel(), _stream(stream)),
        "moe_layer_forward")


def moe_layer_forward_noalloc(layer: Layer, x_in, h, x_out, x_out_f32=None, topk_idx=None, topk_w=None, stream=None):
    """moe_layer_forward with the library's own static scratch instead of a workspace, for callers that
    cannot allocate device memory (see include/moe.h). Decode only (1 <= T <= 8). Calls must not
    overlap on the GPU; a latched device status is read with moe_noalloc_poll_status."""
    _ok(lib().moe_layer_forward_noalloc(layer.cref(), _ptr(x_in), _ptr(h), x_in.shape[0], _ptr(x_out),
                                        _ptr(x_out_f32), _ptr(topk_idx), _ptr(topk_w), _stream(stream)),
        "moe_layer_forward_noalloc")


def moe_layer_forward_timed(layer: Layer, x_in, h, x_out, x_out_f32=None, topk_idx=None, topk_w=None, *, ws, events,
                            stream=None):
    """events: list of torch.cuda.Event(enable_timing=True), one more than the kernels of the path."""
    handles = (C.c_void_p * len(events))(*[e.cuda_event for e in events])
    _ok(lib().moe_layer_forward_timed(layer.cref(), _ptr(x_in), _ptr(h), x_in.shape[0], _ptr(x_out), _ptr(x_out_f32),
                                      _ptr(topk_idx), _ptr(topk_w), _ptr(ws), ws.numel(), handles, len(events),
                                      _stream(stream)), "moe_layer_forward_timed")


class _LayerArray:
    def __init__(self, layers):
        self.layers = list(layers)
        self.arr = (_Layer * len(self.layers))(*[l._c for l in self.layers])


def moe_stack_forward(layers, x_in, h, x_out, topk_idx_all=None, layer_inputs=None, layer_h=None, *, ws,
                      stream=None):
    arr = layers if isinstance(layers, _LayerArray) else _LayerArray(layers)
    _ok(lib().moe_stack_forward(arr.arr, len(arr.layers), _ptr(x_in), _ptr(h), _ptr(x_out), _ptr(topk_idx_all),
                                _ptr(layer_inputs), _ptr(layer_h), _ptr(ws), ws.numel(), _stream(stream)),
        "moe_stack_forward")


def stack_array(layers) -> _LayerArray:
    """Pre-built host array of layer descriptors for repeated moe_stack_forward calls."""
    return _LayerArray(layers)


def moe_poll_status(ws, stream=None) -> int:
    return lib().moe_poll_status(_ptr(ws), _stream(stream))


def moe_noalloc_poll_status(stream=None) -> int:
    """Status latched by earlier moe_layer_forward_noalloc calls on the current device (then cleared)."""
    return lib().moe_noalloc_poll_status(_stream(stream))


# ------------------------------------------------------------------ host-resident experts, HBM cache
def moe_cache_size(layer: Layer, slots: int):
    """(device bytes, host state bytes) of an expert cache with `slots` slots for `layer`."""
    d, h = C.c_size_t(0), C.c_size_t(0)
    _ok(lib().moe_cache_size(layer.cref(), int(slots), C.byref(d), C.byref(h)), "moe_cache_size")
    return d.value, h.value


class ExpertCache:
    """Caller-owned memory of an expert cache (see include/moe.h): the host experts' descriptor
    array, the device buffer (expert table + slots) and the host bookkeeping. host_experts: list of
    E Expert whose tensors are host (ideally pinned) memory; they must outlive the cache."""

    def __init__(self, layer: Layer, host_experts, slots: int, device="cuda"):
        import numpy as np
        import torch
        self.host_experts = host_experts
        self._host_c = (_Expert * len(host_experts))(*[e.c() for e in host_experts])
        dev_bytes, state_bytes = moe_cache_size(layer, slots)
        self.dev = torch.zeros(dev_bytes, dtype=torch.uint8, device=device)
        self.state = np.zeros((state_bytes + 7) // 8, dtype=np.uint64)
        self.slots = slots
        _ok(lib().moe_cache_init(layer.cref(), C.cast(self._host_c, C.c_void_p), int(slots), _ptr(self.dev),
                                 dev_bytes, C.c_void_p(self.state.ctypes.data), self.state.nbytes), "moe_cache_init")

    def state_ptr(self):
        return C.c_void_p(self.state.ctypes.data)


def moe_cache_admit(cache: ExpertCache, ids):
    """Host bookkeeping of one call: (slot per id, missed per id) as int32 numpy arrays."""
    import numpy as np
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    slot = np.empty_like(ids)
    missed = np.empty_like(ids)
    _ok(lib().moe_cache_admit(cache.state_ptr(), C.c_void_p(ids.ctypes.data), ids.size, C.c_void_p(slot.ctypes.data),
                              C.c_void_p(missed.ctypes.data)), "moe_cache_admit")
    return slot, missed


def moe_cache_stats(cache: ExpertCache):
    """(hits, misses, bytes copied) since the cache was set up."""
    h, m, b = C.c_uint64(0), C.c_uint64(0), C.c_uint64(0)
    _ok(lib().moe_cache_stats(cache.state_ptr(), C.byref(h), C.byref(m), C.byref(b)), "moe_cache_stats")
    return h.value, m.value, b.value


def moe_layer_forward_cached(layer: Layer, cache: ExpertCache, x_in, h, x_out, x_out_f32=None, topk_idx=None,
                             topk_w=None, *, ws, stream=None):
    _ok(lib().moe_layer_forward_cached(layer.cref(), cache.state_ptr(), _ptr(x_in), _ptr(h), x_in.shape[0],
                                       _ptr(x_out), _ptr(x_out_f32), _ptr(topk_idx), _ptr(topk_w), _ptr(ws),
                                       ws.numel(), _stream(stream)), "moe_layer_forward_cached")


def moe_selftest_grid_timeout(ws, bound_ns: int, stream=None):
    """A grid-barrier wait that runs out (see moe.h): latches MOE_ERR_TIMEOUT in ws."""
    _ok(lib().moe_selftest_grid_timeout(_ptr(ws), ws.numel() * ws.element_size(), int(bound_ns), _stream(stream)),
        "moe_selftest_grid_timeout")


def moe_selftest_wait_timeout(ws, bound_ns: int, stream=None):
    """A bounded device wait that runs out (see moe.h): latches MOE_ERR_TIMEOUT in ws."""
    _ok(lib().moe_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(), int(bound_ns), _stream(stream)),
        "moe_selftest_wait_timeout")
