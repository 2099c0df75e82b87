"""Float64 CPU oracle for FP8 paged decode attention (test infrastructure only).

Only tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package. It shares no code with the CUDA
library in ``fp8_paged_decode_split_b200``.
"""

from .fp8pd_oracle import (  # noqa: F401
    E4M3_MAX,
    E4M3_NAN_CODE,
    E4M3_TABLE,
    attended_range,
    combine_partials,
    e4m3_code_value,
    e4m3_decode,
    e4m3_encode,
    e4m3_round,
    e8m0_decode,
    fp8_compute_query,
    expand_groups,
    gather_tokens,
    group_scale,
    kv_append,
    mx_quantize,
    mx_scale_code,
    paged_decode_attention,
    paged_decode_partial,
    quantize,
    quantize_per_token,
    token_scale,
)
