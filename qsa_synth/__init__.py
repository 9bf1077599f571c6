"""Seeded, counter-based synthetic inputs for the QSA layer forward.

This package only draws numbers: it holds none of the layer's arithmetic
(no pooling, scoring, selection or attention).  Both the CPU oracle's test
harness and the GPU tests/bench take their inputs from here, so the two sides
see bit-identical tensors.

Every value is a pure function of (seed, tensor id, logical coordinates), so a
harness can regenerate any row of a multi-GiB cache without materialising it.
"""

from .gen import (  # noqa: F401
    T_Q, T_K, T_V, T_IDXK, T_QIDX, T_W,
    splitmix64_at, uniform_int, unit_normal_bf16_bits,
    kv_coords, idxk_coords, qidx_coords, w_coords, q_coords,
    gen_q, gen_kv_rows, gen_idx_k, gen_q_idx, gen_w,
    bf16_bits_to_f32,
)
