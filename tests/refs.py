"""Oracle-side references for the parity tests.

Regenerates the experts a token touches on the host (fixtures.gen, bit-identical
to the device copies) and runs the CPU oracle on them. Test infrastructure only.
"""
from __future__ import annotations

from functools import lru_cache

import numpy as np

import fixtures
import oracle
from fixtures import gen


def rel_err(a, r) -> float:
    a = np.asarray(a, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    den = np.max(np.abs(r))
    return float(np.max(np.abs(a - r)) / (den if den > 0 else 1.0))


def bf16_ulp_diff(a_bits, b_bits) -> int:
    """Max distance in bf16 units in the last place (same-sign ordered ints)."""
    def ordered(b):
        b = np.asarray(b, dtype=np.uint16).astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return int(np.max(np.abs(ordered(a_bits) - ordered(b_bits)))) if np.size(a_bits) else 0


@lru_cache(maxsize=64)
def _expert_cached(cfg, layer, e):
    return fixtures.host_expert(cfg, layer, e)


@lru_cache(maxsize=32)
def layer_vectors(cfg, layer):
    return fixtures.layer_vectors(cfg, layer)


def oracle_tokens(cfg, layer, x_bits, h_in):
    """Oracle forward of one layer for tokens x_bits uint16 [T][H] with residual h_in float64 [T][H].
    Returns dict(idx, w, sg, h_out, x_out, x_out_bf16)."""
    Wr, rb, gs, gamma = layer_vectors(cfg, layer)
    x_bits = np.atleast_2d(np.asarray(x_bits, dtype=np.uint16))
    h_in = np.atleast_2d(np.asarray(h_in, dtype=np.float64))
    idx, w, sg = oracle.route(x_bits, Wr, cfg.k, bias=rb, gs=gs if cfg.has_shared else None)
    T = x_bits.shape[0]
    out = dict(idx=idx, w=w, sg=sg, h_out=np.empty((T, cfg.H)), x_out=np.empty((T, cfg.H)),
               x_out_bf16=np.empty((T, cfg.H), dtype=np.uint16))
    for t in range(T):
        xd = gen.bf16_bits_to_f32(x_bits[t]).astype(np.float64)
        ys = np.stack([oracle.expert(_expert_cached(cfg, layer, int(e)), xd, cfg.H, cfg.I, cfg.G, cfg.bits)
                       for e in idx[t]])
        y_sh = oracle.expert(_expert_cached(cfg, layer, cfg.E), xd, cfg.H, cfg.I, cfg.G, cfg.bits) \
            if cfg.has_shared else None
        h_out, x_out, xb = oracle.combine_norm(ys, w[t], y_sh, sg[t] if sg is not None else 0.0, h_in[t], gamma,
                                               cfg.rms_eps)
        out["h_out"][t], out["x_out"][t], out["x_out_bf16"][t] = h_out, x_out, xb
    return out
