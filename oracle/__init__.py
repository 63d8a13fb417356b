"""fp64 CPU oracle (test infrastructure only; see ``mla_oracle``).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs use this package.  It never imports the CUDA library.
"""

from .mla_oracle import (  # noqa: F401
    OracleInputs, bf16_to_f64, e4m3fn_to_f64, decode_nonabsorbed, decode_absorbed,
    absorb_q, up_proj_v, latent_attention, combine_splits,
)


def from_workload(w) -> OracleInputs:
    """Raw bits of a ``mla_inputs.Workload`` wrapped for the oracle."""
    from mla_inputs import bf16_bits, f16_bits, fp8_bits, int8_bits
    kind = w.spec.kv_dtype
    if kind == "bf16":
        kv, scale = bf16_bits(w.kv_cache), None
    elif kind == "q8_0":
        kv, scale = int8_bits(w.kv_cache), f16_bits(w.kv_scale)
    elif kind == "q4_0":
        kv, scale = w.kv_cache.contiguous().numpy(), f16_bits(w.kv_scale)
    else:
        kv, scale = fp8_bits(w.kv_cache), w.kv_scale.numpy()
    return OracleInputs(bf16_bits(w.q_nope), bf16_bits(w.q_pe), bf16_bits(w.w_uk),
                        bf16_bits(w.w_uv), kv, w.spec.kv_dtype, scale,
                        w.block_table.numpy(), w.seq_lens.numpy(), w.softmax_scale,
                        w.spec.causal)
