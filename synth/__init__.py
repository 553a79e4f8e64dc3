"""Seeded synthetic inputs for binary-weight decode GEMV workloads.

This package draws random numbers and lays them out in memory. It holds none of
the method's arithmetic: it never decodes a sign, reconstructs a weight or
forms a product. The same arrays feed the fp64 oracle (``oracle/``) and the
CUDA path (``binary_weight_decode_b200``), which share no code with each other.

Workload recipes (shapes, value distributions) follow the decode-time layers
named in the binary-weight papers: a Llama-7B-shaped attention projection
(4096x4096), the MLP projections (4096->11008, 11008->4096), a 5120x5120 layer
with a binary low-rank correction, and the full 32-layer decoder weight stream.
"""

from .layout import (  # noqa: F401
    ROW_TILE,
    COL_QUAD,
    packed_words,
    zero_padding_bits,
)
from .gen import (  # noqa: F401
    Layer,
    f32_to_bf16_bits,
    make_layer,
    make_activations,
    dense_signs,
)
from .configs import CONFIGS, config_layers  # noqa: F401
