"""fp64 CPU oracle for the binary-weight decode GEMV (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import or run anything in this package. It shares no code with
the CUDA library (``binary_weight_decode_b200``) and neither imports the other.
"""

from .bisco_oracle import (  # noqa: F401
    algorithmic_bytes,
    biloco_decompose,
    binary_correction_storage_bits,
    correction_z,
    decode_values,
    dense_correction_storage_bits,
    fluxbin_average_bit_width,
    fluxbin_sign_search,
    fluxbin_storage_bits,
    fp4_weight_bits,
    gemv,
    gemv_rows,
    pack_bit_matrix,
    reconstruct,
    unpack_bit_matrix,
    unpack_bit_rows,
)
