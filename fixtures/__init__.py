"""Seeded synthetic inputs for the MoE expert-forward path.

This module is shared by the CPU oracle side and the CUDA side of the tests and
the bench. It holds no arithmetic of the method itself (no dequantisation, no
dot products, no routing): it only draws random numbers and lays them out in
the packed storage format that the pages' engine streams per expert
("SSD Expert Streaming": four active experts of about 6.75 MB each).
"""
from .gen import (  # noqa: F401
    Config, CONFIGS, MatShape, expert_mat_shapes, mat_nbytes, expert_nbytes,
    NormalTable, normal_table, key_of, u64_stream, codes_words, halfnormal_bf16,
    normal_bf16, biases_from_scales, gamma_bf16, router_bias_f32, layer_vectors,
    host_expert, bf16_bits_to_f32, f32_to_bf16_bits,
    T_X, T_ROUTER_W, T_ROUTER_BIAS, T_SHARED_GATE, T_GAMMA, T_CODES, T_SCALES,
)
