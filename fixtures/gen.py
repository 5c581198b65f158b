"""Counter-based synthetic data for the quantized MoE expert forward.

Every value is a pure function of (seed, layer, tensor id, expert, index), so
any expert of any layer can be regenerated on its own, on the host (this
file, numpy) or on the device (``gen_gpu.cu``), bit for bit the same.

Generators
----------
* ``u64_stream``: SplitMix64 (Steele, Lea, Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): output i of a stream with key
  K is mix64(K + (i+1)*0x9E3779B97F4A7C15).
* Packed codes: one 32-bit word per output, the low 32 bits of the SplitMix64
  value. A uniform 32-bit word holds 8 uniform 4-bit codes (0..15) or 16
  uniform 2-bit codes (0..3).
* Normal bf16 values: exact inverse-CDF sampling of the bf16-rounded
  distribution. For sigma, the positive bf16 grid v_0 < v_1 < ... gets
  thresholds theta_j = floor(erf(m_j / (sigma*sqrt 2)) * 2^32) at the
  midpoints m_j = (v_j + v_{j+1})/2; a 32-bit uniform u selects v_j with j =
  #{theta <= u}. Integer comparisons only, so host and device agree exactly.
  Bit 63 of the same SplitMix64 output gives the sign of a signed normal.

Workload shapes follow the five configurations of the single-token and
prefill expert forward for a 512-expert, hidden-4096 layer (Flash-MoE
write-up, "Model architecture": 512 experts per layer, K=4 active including
one shared, hidden size 4096).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from functools import lru_cache

import numpy as np

M64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15

# tensor ids of the key derivation
T_X = 1
T_ROUTER_W = 2
T_ROUTER_BIAS = 3
T_SHARED_GATE = 4
T_GAMMA = 5
T_CODES = 16      # + matrix index (0 gate, 1 up, 2 down)
T_SCALES = 32     # + matrix index
T_MX_CODES = 48   # MXFP4 matrices
T_MX_SCALES = 49


def _mix64_int(z: int) -> int:
    z &= M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def key_of(seed: int, layer: int, tensor: int, expert: int = 0) -> int:
    """64-bit stream key of one tensor (a chain of SplitMix64 finalisers)."""
    k = _mix64_int(seed * GOLDEN + 0x1234567)
    for part in (layer, tensor, expert):
        k = _mix64_int(k ^ ((part + 1) * GOLDEN & M64))
    return k


def u64_stream(key: int, start: int, n: int) -> np.ndarray:
    """SplitMix64 outputs start .. start+n-1 of the stream with this key."""
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + i * np.uint64(GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def codes_words(key: int, n_words: int, start: int = 0) -> np.ndarray:
    return (u64_stream(key, start, n_words) & np.uint64(0xFFFFFFFF)).astype(np.uint32)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even float32 -> bf16 bit patterns (finite inputs)."""
    u = np.asarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


@dataclass(frozen=True)
class NormalTable:
    sigma: float
    thresholds: np.ndarray   # uint32 [n-1], nondecreasing
    values: np.ndarray       # uint16 [n], positive bf16 bit patterns, increasing


@lru_cache(maxsize=None)
def normal_table(sigma: float) -> NormalTable:
    """Thresholds for exact inverse-CDF sampling of |N(0, sigma^2)| on the bf16 grid."""
    bits = np.arange(1, 0x7F80, dtype=np.uint32).astype(np.uint16)   # positive finite bf16
    vals = bf16_bits_to_f32(bits).astype(np.float64)
    keep = (vals >= sigma * 2.0 ** -36) & (vals <= sigma * 9.0)
    bits, vals = bits[keep], vals[keep]
    mids = 0.5 * (vals[:-1] + vals[1:])
    s2 = sigma * math.sqrt(2.0)
    cdf = np.array([math.erf(m / s2) for m in mids], dtype=np.float64)
    th = np.floor(cdf * 4294967296.0)
    th = np.clip(th, 0.0, 4294967296.0).astype(np.uint64)
    # drop grid points that can never be drawn (zero-width cells at both ends)
    lo = int(np.searchsorted(th, 0, side="right"))            # th[:lo] == 0
    hi_idx = np.nonzero(th >= np.uint64(1 << 32))[0]
    hi = int(hi_idx[0]) if len(hi_idx) else len(th)          # th[hi] == 2^32
    values = bits[lo:hi + 1].copy()
    thresholds = th[lo:hi].astype(np.uint32)
    assert len(values) == len(thresholds) + 1 and len(values) < 8192
    return NormalTable(sigma, thresholds, values)


def _draw_magnitude(table: NormalTable, u32: np.ndarray) -> np.ndarray:
    j = np.searchsorted(table.thresholds, u32, side="right")
    return table.values[j]


def halfnormal_bf16(key: int, n: int, sigma: float, start: int = 0) -> np.ndarray:
    z = u64_stream(key, start, n)
    return _draw_magnitude(normal_table(sigma), (z & np.uint64(0xFFFFFFFF)).astype(np.uint32))


def normal_bf16(key: int, n: int, sigma: float, start: int = 0) -> np.ndarray:
    z = u64_stream(key, start, n)
    mag = _draw_magnitude(normal_table(sigma), (z & np.uint64(0xFFFFFFFF)).astype(np.uint32))
    sign = ((z >> np.uint64(63)).astype(np.uint16)) << np.uint16(15)
    return mag | sign


def biases_from_scales(scales: np.ndarray, bits: int) -> np.ndarray:
    """Group bias of the synthetic weights: -8*s for 4-bit codes (exact),
    bf16_rne(-1.5*s) for 2-bit codes, so that codes are centred on zero."""
    s = bf16_bits_to_f32(scales)
    if bits == 4:
        return f32_to_bf16_bits(np.float32(-8.0) * s)
    if bits == 2:
        return f32_to_bf16_bits(np.float32(-1.5) * s)
    raise ValueError(bits)


def gamma_bf16(seed: int, layer: int, H: int) -> np.ndarray:
    """RMSNorm weight 1 + 0.1*z, z ~ N(0,1) on the bf16 grid, rounded to bf16."""
    z = bf16_bits_to_f32(normal_bf16(key_of(seed, layer, T_GAMMA), H, 1.0)).astype(np.float64)
    return f32_to_bf16_bits((1.0 + 0.1 * z).astype(np.float32))


def router_bias_f32(seed: int, layer: int, E: int) -> np.ndarray:
    return bf16_bits_to_f32(normal_bf16(key_of(seed, layer, T_ROUTER_BIAS), E, 1.0))


@dataclass(frozen=True)
class MatShape:
    R: int
    K: int


def expert_mat_shapes(H: int, I: int):
    """gate [I][H], up [I][H], down [H][I] (rows = outputs, K = inputs)."""
    return (MatShape(I, H), MatShape(I, H), MatShape(H, I))


def mat_nbytes(R: int, K: int, bits: int, G: int) -> int:
    """Packed codes + bf16 scales + bf16 biases of one R x K matrix."""
    return R * K * bits // 8 + 2 * 2 * R * (K // G)


def expert_nbytes(H: int, I: int, bits: int, G: int) -> int:
    return sum(mat_nbytes(m.R, m.K, bits, G) for m in expert_mat_shapes(H, I))


@dataclass(frozen=True)
class Config:
    name: str
    H: int
    E: int
    k: int
    I: int
    bits: int
    G: int = 64
    T: int = 1
    layers: int = 1
    steps: int = 1
    scale_sigma: float = 0.02
    router_sigma: float = 0.02
    gate_sigma: float = 0.02
    router_bias: bool = False
    has_shared: bool = True
    rms_eps: float = 1e-6
    seed: int = 0
    note: str = field(default="", compare=False)

    @property
    def expert_bytes(self) -> int:
        return expert_nbytes(self.H, self.I, self.bits, self.G)

    @property
    def active_bytes_per_token(self) -> int:
        return (self.k + (1 if self.has_shared else 0)) * self.expert_bytes * self.layers


CONFIGS = {
    "tiny": Config("tiny", H=256, E=16, k=2, I=128, bits=4,
                   note="tiny MoE layer, 1 token, H256 E16+1 top-2 I128 4-bit"),
    "layer_q4": Config("layer_q4", H=4096, E=512, k=3, I=1024, bits=4,
                       note="one 512-expert hidden-4096 layer, decode batch 1, 4-bit"),
    "layer_q2": Config("layer_q2", H=4096, E=512, k=3, I=1024, bits=2, scale_sigma=0.05,
                       note="same layer, 2-bit experts"),
    "stack_q4": Config("stack_q4", H=4096, E=512, k=3, I=1024, bits=4, layers=24, steps=256,
                       router_bias=True, note="24 such 4-bit layers, 256 decode steps, biased router"),
    "prefill_q4": Config("prefill_q4", H=4096, E=512, k=3, I=1024, bits=4, T=512,
                         note="512-token prefill of the 4-bit layer"),
}


def layer_vectors(cfg: Config, layer: int):
    """Host copies of one layer's router weight, router bias, shared-gate vector and RMSNorm gamma."""
    seed = cfg.seed
    Wr = normal_bf16(key_of(seed, layer, T_ROUTER_W), cfg.E * cfg.H, cfg.router_sigma).reshape(cfg.E, cfg.H)
    rb = router_bias_f32(seed, layer, cfg.E) if cfg.router_bias else None
    gs = normal_bf16(key_of(seed, layer, T_SHARED_GATE), cfg.H, cfg.gate_sigma) if cfg.has_shared else None
    gamma = gamma_bf16(seed, layer, cfg.H)
    return Wr, rb, gs, gamma


def x_tokens(cfg: Config, step: int, T: int | None = None) -> np.ndarray:
    """Layer-0 input activations of one decode step (or the prefill batch): bf16 [T][H] ~ N(0,1)."""
    T = cfg.T if T is None else T
    return normal_bf16(key_of(cfg.seed, 1000 + step, T_X), T * cfg.H, 1.0).reshape(T, cfg.H)


def host_expert(cfg: Config, layer: int, expert: int):
    """(q, scales, biases) of gate, up, down of one expert (expert == E is the shared one)."""
    out = []
    for m, shp in enumerate(expert_mat_shapes(cfg.H, cfg.I)):
        nw = shp.R * shp.K * cfg.bits // 32
        q = codes_words(key_of(cfg.seed, layer, T_CODES + m, expert), nw).reshape(shp.R, shp.K * cfg.bits // 32)
        s = halfnormal_bf16(key_of(cfg.seed, layer, T_SCALES + m, expert), shp.R * (shp.K // cfg.G),
                            cfg.scale_sigma).reshape(shp.R, shp.K // cfg.G)
        b = biases_from_scales(s, cfg.bits)
        out.append((q, s, b))
    return tuple(out)


def mx_matrix(seed: int, R: int, K: int, scale_lo: int = 118, scale_hi: int = 124):
    """A synthetic MXFP4 matrix (no model weights): codes uint32 [R][K/8], one uniform 32-bit word
    per eight 4-bit codes (all sixteen E2M1 codes equally likely), and E8M0 scale bytes uint8
    [R][K/32] uniform in [scale_lo, scale_hi] (default 2^-9 .. 2^-3)."""
    q = codes_words(key_of(seed, 0, T_MX_CODES), R * K // 8).reshape(R, K // 8)
    u = u64_stream(key_of(seed, 0, T_MX_SCALES), 0, R * K // 32)
    e = (np.uint64(scale_lo) + u % np.uint64(scale_hi - scale_lo + 1)).astype(np.uint8).reshape(R, K // 32)
    return q, e


def mx_tokens(seed: int, T: int, K: int, sigma: float = 1.0) -> np.ndarray:
    """T rows of K normal bf16 activations (bit patterns, uint16 [T][K])."""
    return normal_bf16(key_of(seed, 0, T_X, 7), T * K, sigma).reshape(T, K)


def mx_expert(e: int, H: int, I: int, scale_lo: int = 116, scale_hi: int = 120):
    """Expert e of a synthetic MXFP4 layer: ((qg, eg), (qu, eu), (qd, ed)), gate and up [I][H],
    down [H][I] (scale bytes 116..120: 2^-11 .. 2^-7)."""
    return tuple(mx_matrix(1000 + 3 * e + m, *((I, H) if m < 2 else (H, I)), scale_lo, scale_hi) for m in range(3))
