"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point the header declares, its struct layouts match the header,
and argument errors are returned before anything is launched."""
import ctypes as C
import os
import re
import subprocess
import tempfile

import pytest

import quantized_expert_decode_moe_b200 as qm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_entry_point():
    L = qm.lib()
    names = header_functions()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert qm.moe_abi_version() == 1


def test_struct_layout_matches_header():
    src = r'''
#include <stdio.h>
#include <stddef.h>
#include "moe.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(moe_qmat), sizeof(moe_expert), sizeof(moe_layer),
         offsetof(moe_layer, rms_eps), offsetof(moe_layer, router_w), offsetof(moe_layer, experts),
         offsetof(moe_layer, shared), offsetof(moe_layer, rms_gamma));
  return 0;
}'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "a.c")
        open(c, "w").write(src)
        exe = os.path.join(d, "a")
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), "-o", exe, c])
        got = list(map(int, subprocess.check_output([exe]).split()))
    L = qm._Layer
    want = [C.sizeof(qm._QMat), C.sizeof(qm._Expert), C.sizeof(L), L.rms_eps.offset, L.router_w.offset,
            L.experts.offset, L.shared.offset, L.rms_gamma.offset]
    assert got == want


def test_status_strings():
    for code in range(7):
        assert qm.moe_status_string(code)
    assert qm.moe_status_string(99) == "unknown status"


def fake_layer(**kw):
    """A descriptor with fake (never dereferenced) aligned device pointers."""
    p = 0x100000
    ex = qm._Expert(*[qm._QMat(p, p, p) for _ in range(3)])
    f = dict(hidden=4096, inter=1024, n_experts=512, top_k=3, bits=4, group=64, has_shared=1, rms_eps=1e-6,
             router_w=p, router_bias=None, experts=p, shared=ex, shared_gate_w=p, rms_gamma=p)
    f.update(kw)
    return qm._Layer(**f)


def ws_size(layer, T=1):
    n = C.c_size_t(0)
    rc = qm.lib().moe_workspace_size(C.byref(layer), T, C.byref(n))
    return rc, n.value


def test_workspace_size_and_layer_validation():
    rc, n = ws_size(fake_layer())
    assert rc == 0 and n > 0
    rc4, n4 = ws_size(fake_layer(), T=4)
    assert rc4 == 0 and n4 > n
    assert ws_size(fake_layer(bits=3))[0] == 2            # unsupported bits
    assert ws_size(fake_layer(group=16))[0] == 2          # unsupported group
    assert ws_size(fake_layer(group=32, bits=2))[0] == 2  # group 32 is the MXFP4 codec: 4-bit only
    assert ws_size(fake_layer(group=32, bits=4))[0] == 0  # MXFP4 experts
    assert ws_size(fake_layer(top_k=9))[0] == 1           # k > 8
    assert ws_size(fake_layer(n_experts=2, top_k=3))[0] == 1   # k > E
    assert ws_size(fake_layer(hidden=4000))[0] == 1       # not a multiple of 128
    assert ws_size(fake_layer(inter=0))[0] == 1
    assert ws_size(fake_layer(rms_eps=0.0))[0] == 1
    assert ws_size(fake_layer(router_w=0x100008))[0] == 1  # misaligned
    assert ws_size(fake_layer(shared_gate_w=None))[0] == 1
    assert ws_size(fake_layer(shared_gate_w=None, has_shared=0))[0] == 0
    assert ws_size(fake_layer(experts=None))[0] == 1
    assert qm.lib().moe_workspace_size(None, 1, None) == 1


def test_prefill_workspace_holds_the_grouped_buffers():
    """Above 8 tokens the workspace also holds the prefill path's buffers: the
    expert outputs y [T(k+1)][H] fp32, the activation digit tables of x
    ([T][2H] bytes) and of the SwiGLU outputs ([T(k+1)][2I] bytes) and the fp64
    logits [T][E+1]; a call whose workspace was sized for fewer tokens is
    rejected before anything is launched."""
    lay = fake_layer()
    H, I, E, k = 4096, 1024, 512, 3
    _, n8 = ws_size(lay, T=8)
    _, n9 = ws_size(lay, T=9)
    _, n512 = ws_size(lay, T=512)
    T = 512
    need = T * (k + 1) * H * 4 + T * 2 * H + T * (k + 1) * 2 * I + T * (E + 1) * 8
    assert n512 >= need
    assert n9 - n8 >= 9 * (k + 1) * H * 4   # the prefill buffers appear at T = 9
    L = qm.lib()
    p = C.c_void_p(0x200000)
    ws = C.c_void_p(0x400000)
    assert L.moe_layer_forward(C.byref(lay), p, p, 9, p, None, None, None, ws, n8, None) == 3
    assert L.moe_route(C.byref(lay), p, 12, p, p, None, ws, n8, None) == 3


def test_entry_points_reject_bad_arguments_before_launch():
    L = qm.lib()
    lay = fake_layer()
    p = C.c_void_p(0x200000)
    _, n = ws_size(lay)
    ws = C.c_void_p(0x400000)
    # layer forward: null input, T = 0, workspace too small, misaligned h
    assert L.moe_layer_forward(C.byref(lay), None, p, 1, p, None, None, None, ws, n, None) == 1
    assert L.moe_layer_forward(C.byref(lay), p, p, 0, p, None, None, None, ws, n, None) == 1
    assert L.moe_layer_forward(C.byref(lay), p, p, 1, p, None, None, None, ws, n - 1, None) == 3
    assert L.moe_layer_forward(C.byref(lay), p, p, 1, p, None, None, None, None, n, None) == 3
    assert L.moe_layer_forward(C.byref(lay), p, C.c_void_p(0x200004), 1, p, None, None, None, ws, n, None) == 1
    assert L.moe_layer_forward(C.byref(lay), p, p, 1, p, None, None, None, C.c_void_p(0x400010), n, None) == 1
    # route: null outputs
    assert L.moe_route(C.byref(lay), p, 1, None, p, None, ws, n, None) == 1
    # gemv: bad group, K not a multiple of 128, R = 0, null matrix
    W = qm._QMat(0x100000, 0x100000, 0x100000)
    assert L.moe_expert_gemv_q4(C.byref(W), 16, 256, 32, p, p, None) == 2
    assert L.moe_expert_gemv_q4(C.byref(W), 16, 200, 64, p, p, None) == 1
    assert L.moe_expert_gemv_q2(C.byref(W), 0, 256, 64, p, p, None) == 1
    assert L.moe_expert_gemv_q4(C.byref(W), 300, 256, 64, p, p, None) == 1   # rows not a multiple of 16
    assert L.moe_expert_gemv_q2(None, 16, 256, 64, p, p, None) == 1
    # combine: eps <= 0, shared output without gate
    assert L.moe_combine_residual_norm(1, 256, 2, p, p, None, None, p, p, C.c_float(0.0), p, None, None) == 1
    assert L.moe_combine_residual_norm(1, 256, 2, p, p, p, None, p, p, C.c_float(1e-6), p, None, None) == 1
    # combine: H not a multiple of 8 or above 8192 is unsupported
    assert L.moe_combine_residual_norm(1, 100, 2, p, p, None, None, p, p, C.c_float(1e-6), p, None, None) == 2
    assert L.moe_combine_residual_norm(1, 16384, 2, p, p, None, None, p, p, C.c_float(1e-6), p, None, None) == 2
    # grouping: k > 8, E <= 0
    assert L.moe_group_tokens(4, 9, 16, p, p, p, p, None, 0, None) == 1
    assert L.moe_group_tokens(4, 2, 0, p, p, p, p, None, 0, None) == 1
    # stack: mismatched layers
    lays = (qm._Layer * 2)(fake_layer(), fake_layer(inter=2048))
    assert L.moe_stack_forward(lays, 2, p, p, p, None, None, None, ws, n, None) == 1
    assert L.moe_poll_status(None, None) == 3
    # failure-path diagnostics: no workspace, misaligned, bound out of range
    assert L.moe_selftest_wait_timeout(None, n, 1000, None) == 3
    assert L.moe_selftest_wait_timeout(C.c_void_p(0x400010), n, 1000, None) == 1
    assert L.moe_selftest_wait_timeout(ws, n, 0, None) == 1
    assert L.moe_selftest_wait_timeout(ws, n, 20 * 10 ** 9, None) == 1


def layer_path(layer, T):
    p, n = C.c_int32(), C.c_int32()
    rc = qm.lib().moe_layer_path(C.byref(layer), T, C.byref(p), C.byref(n))
    return rc, qm.PATHS.get(p.value) if rc == 0 else None


def test_unlaunchable_decode_shapes_are_rejected_before_launch(monkeypatch):
    """Hidden 8192, intermediate 8192, 4-bit, top-8 + shared: the digit-block
    down kernel would hold 9 slots x 256 digit blocks of 112 bytes, more than
    one CTA's shared memory, and the chain's and the fused kernel's staging
    does not fit either, so every decode entry point refuses the layer with
    MOE_ERR_UNSUPPORTED for every token count from 1 to 8. On a machine
    without a GPU any launch would fail with MOE_ERR_CUDA instead, so these
    codes also show that nothing was launched. The grouped prefill path
    (T > 8) still takes the layer, and the largest shapes each decode path
    accepts pass the checks."""
    monkeypatch.delenv("MOE_DECODE_KERNEL", raising=False)
    L = qm.lib()
    bad = fake_layer(hidden=8192, inter=8192, top_k=8)
    p = C.c_void_p(0x200000)
    ws = C.c_void_p(0x400000)
    for T in (1, 8):
        assert ws_size(bad, T)[0] == 2
    rc, n = ws_size(bad, 9)
    assert rc == 0 and n > 0
    ev = (C.c_void_p * 6)(*[0x1000] * 6)
    for T in range(1, 9):
        assert L.moe_layer_forward(C.byref(bad), p, p, T, p, None, None, None, ws, n, None) == 2
        assert L.moe_layer_forward_timed(C.byref(bad), p, p, T, p, None, None, None, ws, n, ev, 6, None) == 2
        assert L.moe_layer_forward_noalloc(C.byref(bad), p, p, T, p, None, None, None, None) == 2
    lays = (qm._Layer * 3)(bad, bad, bad)
    assert L.moe_stack_forward(lays, 3, p, p, p, None, None, None, ws, n, None) == 2
    # the digit-block kernels (default for decode): 9 slots up to intermediate 7296
    assert layer_path(fake_layer(hidden=8192, inter=7296, top_k=8), 8) == (0, "digit")
    assert layer_path(fake_layer(hidden=8192, inter=7424, top_k=8), 8)[0] == 2
    assert layer_path(fake_layer(), 1) == (0, "digit") and layer_path(fake_layer(), 9) == (0, "prefill")
    # a shape the grouped prefill cannot take runs the digit-block kernels token by token
    assert layer_path(fake_layer(hidden=4096, inter=2816), 9) == (0, "digit")
    # MOE_DECODE_KERNEL=chain: the chain up to hidden 7552 / inter 2688 (4-bit), else the digit kernels
    monkeypatch.setenv("MOE_DECODE_KERNEL", "chain")
    assert layer_path(fake_layer(hidden=7552, inter=2688), 1) == (0, "chain")
    assert layer_path(fake_layer(hidden=7552, inter=2688), 8) == (0, "chain")
    assert layer_path(fake_layer(hidden=7680, inter=1024), 8) == (0, "digit")
    assert layer_path(fake_layer(hidden=4096, inter=2816), 8) == (0, "digit")
    assert layer_path(fake_layer(hidden=8192, inter=2048, bits=2), 8) == (0, "chain")
    # MOE_DECODE_KERNEL=fused: the fused kernel (T = 1) up to hidden 4096 / inter 1152
    monkeypatch.setenv("MOE_DECODE_KERNEL", "fused")
    assert layer_path(fake_layer(hidden=4096, inter=1152), 1) == (0, "fused")
    assert layer_path(fake_layer(hidden=4096, inter=1152), 2) == (0, "chain")


def test_wait_bound_and_header_words_documented():
    """The header states the default bound of device-side waits and the
    workspace header words the tests read (status, recheck count, grid-barrier
    counters)."""
    text = open(HEADER).read()
    assert "100 ms" in text and "MOE_WAIT_TIMEOUT_NS" in text
    assert "byte offset 16" in text and "moe_noalloc_poll_status" in text


def test_mxfp4_entry_points_check_arguments_on_the_host():
    """The MXFP4 calls reject bad shapes, missing pointers and small workspaces before any CUDA
    call (so this runs without a GPU)."""
    L = qm.lib()
    n = C.c_size_t(0)
    assert L.moe_mxfp4_workspace_size(256, 4096, 512, C.byref(n)) == 0 and n.value > 256
    assert L.moe_mxfp4_workspace_size(200, 4096, 1, C.byref(n)) == 2      # R % 128
    assert L.moe_mxfp4_workspace_size(128, 4000, 1, C.byref(n)) == 2      # K % 128
    assert L.moe_mxfp4_workspace_size(128, 16384, 1, C.byref(n)) == 2     # K > 8192
    assert L.moe_mxfp4_workspace_size(128, 128, 0, C.byref(n)) == 1
    assert L.moe_mxfp4_workspace_size(128, 128, 1, None) == 1
    W = qm._MxMat(0x1000, 0x1000)
    assert L.moe_expert_gemv_mxfp4(None, 16, 64, C.c_void_p(0x1000), C.c_void_p(0x1000), None) == 1
    assert L.moe_expert_gemv_mxfp4(C.byref(W), 16, 48, C.c_void_p(0x1000), C.c_void_p(0x1000), None) == 1   # K % 32
    assert L.moe_expert_gemv_mxfp4(C.byref(W), 16, 16384, C.c_void_p(0x1000), C.c_void_p(0x1000), None) == 2
    assert L.moe_expert_gemv_mxfp4(C.byref(W), 16, 64, C.c_void_p(0x1008), C.c_void_p(0x1000), None) == 1   # x align
    L.moe_mxfp4_workspace_size(128, 128, 4, C.byref(n))
    need = n.value
    args = (C.c_void_p(0x1000), 4, C.c_void_p(0x1000), C.c_void_p(0x10000))
    assert L.moe_expert_gemm_mxfp4(C.byref(W), 128, 128, *args, need - 1, None) == 3
    assert L.moe_expert_gemm_mxfp4(C.byref(W), 100, 128, *args, need, None) == 2
    assert L.moe_expert_gemm_mxfp4(None, 128, 128, *args, need, None) == 1
    assert L.moe_expert_gemm_mxfp4(C.byref(W), 128, 128, C.c_void_p(0x1000), 4, C.c_void_p(0x1000),
                                   C.c_void_p(0x10010), need, None) == 1      # workspace not 256-byte aligned


def test_binding_constants_match_the_header():
    """The binding's copies of header constants: the no-alloc scratch size and the path codes."""
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")).read()
    m = re.search(r"#define MOE_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m and int(m.group(1)) << int(m.group(2)) == qm.NOALLOC_SCRATCH_BYTES
    codes = dict((int(v), k) for k, v in re.findall(r"MOE_PATH_(\w+) = (\d+)", hdr))
    assert {c: n.lower() for c, n in codes.items()} == {1: "fused", 2: "chain", 3: "prefill", 4: "mxfp4", 5: "digit"}
    assert qm.PATHS == {1: "fused", 2: "chain", 3: "prefill", 4: "mxfp4", 5: "digit"}
