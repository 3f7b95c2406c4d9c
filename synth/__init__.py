"""Seeded synthetic inputs for the gated local/full decode-attention path.

This package is the only code that both the CUDA path (tests, bench) and the
CPU oracle consume. It holds no arithmetic of the attention method itself:
only a counter-based random number generator, value lookup tables, the
workload recipes (shapes, context lengths, flag draws, paging, needle plants)
and bf16 rounding of generated values.
"""

from .gen import (  # noqa: F401
    KIND_HIDDEN, KIND_KV, KIND_NEEDLE, KIND_Q, KIND_VEC, KIND_W1,
    bf16_bits_to_f32, bf16_round_bits, f32_to_bf16_bits, fill_streams, mix64,
    mix64_int, normal_table, stream_key, table_values, uniform_table,
)
from .workloads import (  # noqa: F401
    MIXED_RATES, Needle, Workload, ctx128k, ctx16k, custom, mixed_batch, recall_step,
    tiny_fp32,
)
