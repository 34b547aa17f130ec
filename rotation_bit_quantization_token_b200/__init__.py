"""Fused rotate + quantize (FlatQuantV2-style) for B200, sm_100a.

For each token of x[K, M, N]: x'' = P1 . (x . P2), quantized per token to INT4 or per
32-group to FP4 E2M1 with E8M0 scales, by hand-written CUDA kernels behind the C ABI of
include/fq.h (libfq.so, built in-tree). The Python layer marshals arguments only.
"""

from .api import (FlatQuant, HostPipeline, debug_rotate, quantize_mx,  # noqa: F401
                  quantize_mx_static, quantize_per_token)
from ._lib import FQError, load as load_library  # noqa: F401
