"""Seeded synthetic inputs for MLA decode over a paged latent KV cache.

This module only draws numbers and lays them out in the buffers the decode step
consumes. It holds none of the attention arithmetic, so both the fp64 oracle
(``oracle/``) and the CUDA path (``head_latent_attention_06_b200``) can take
their inputs from it without sharing any of the method.

Shapes follow the latent-cache statement of MLA: every cached token carries one
d_c = 512 latent ``c_KV`` plus a decoupled 64-wide RoPE key (DeepSeek-V2 summary,
"Architecture"; snowgate thread 35, replies on the 512 + 64 latent record).
"""

from .workloads import (  # noqa: F401
    D_C, D_R, D_N, D_V, PAGE, ROW, SOFTMAX_SCALE,
    Workload, WorkloadSpec, PRESETS, preset, make_workload, bf16_bits, fp8_bits, int8_bits, f16_bits,
    row_bytes,
)
