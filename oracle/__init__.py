"""CPU oracle for the fused rotate + quantize operator (test infrastructure).

This package is test infrastructure only. It is imported by `tests/`, by
`__graft_entry__.smoke()` and by the `cpu_baseline` / `--impl reference` legs of
`bench.py`, and by nothing else. The product path (the CUDA library and its
Python binding) never imports, links or executes it, and the two share no code.

Source: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1
quantization fusion" (http://www.zwxr.cn/news/277566), sections "How it works",
"per-token mode", "per-group mode" cases 1-3, "Parameter quick reference" and
"Error code quick reference".

`consumer.py` restates the dequantization the page says the outputs are emitted for,
and the FP4 x FP4 contraction that would consume them (no kernel for it exists yet).

Parity unpinned: none. Every public function here is pinned against closed forms,
brute force, hand-worked values or textbook special cases, by
`tests/test_oracle_pins.py` (the operator) and `tests/test_oracle_consumer_pins.py`
(the consumers).
"""

from .flatquant import (  # noqa: F401
    E2M1_GRID,
    e2m1_encode,
    e2m1_decode,
    rotate,
    rotate_rounded,
    round_to_16bit,
    per_token_quantize,
    pack_nibbles,
    mx_group_view,
    mx_scale_exponent,
    mx_quantize,
    mx_scale_layout,
    flat_quant_per_token,
    flat_quant_mx,
)
from .consumer import (  # noqa: F401
    unpack_nibbles,
    int4_value,
    e2m1_value,
    group_bytes_from_layout,
    dequantize_per_token,
    dequantize_mx,
    mx_matmul,
)
