"""The cache-record arithmetic the pages print, against the byte formula the
roofline uses (``Workload.cache_bytes``): 512 + 64 values per token and layer,
576 B at fp8 and twice that at bf16; about 35 KB per token over the thread's 60
layers against about 240 KiB for its 8-head GQA example, a cut of about 7x."""

import json
import os

from mla_inputs import WorkloadSpec, make_workload, ROW

HERE = os.path.dirname(os.path.abspath(__file__))


def test_latent_record_bytes():
    g = json.load(open(os.path.join(HERE, "golden", "latent_record.json")))
    assert g["latent_width"] + g["rope_width"] == g["record_values"] == ROW
    for kv, want, extra in (("bf16", g["record_bytes_bf16"], 0), ("fp8", g["record_bytes_fp8"], 4)):
        w = make_workload(WorkloadSpec("g", B=2, H=1, s_q=1, lens=[3, 64], kv_dtype=kv, seed=1))
        # the fp8 cache also stores one fp32 scale per token
        assert w.cache_bytes() == 67 * (want + extra)
    stack = g["record_bytes_fp8"] * g["thread_layers"]
    assert abs(stack / 1000 - g["stack_bytes_per_token_approx_kb"]) < 1.0
    gqa = g["gqa_kv_heads"] * g["gqa_head_dim"] * 2 * g["gqa_bytes_per_element"] * g["thread_layers"]
    assert gqa / 1024 == g["gqa_stack_bytes_per_token_approx_kib"]
    assert round(gqa / stack) == g["traffic_ratio_approx"]
