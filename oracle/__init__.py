"""CPU oracle of the compressed linear layer — test infrastructure only.

Imported by the tests, by the package smoke check and by the benchmark's
CPU-baseline leg; never by the product path.
"""
from .slim_oracle import (  # noqa: F401
    GROUP, QMAX, PAIRS, OracleRangeError,
    bf16_bits_to_f32, bf16_bits_to_f64,
    quantize, prune_2of4, mask_from_pairs, pack, pack_layer,
    unpack, effective_weight, forward, adapter_down,
    quantize_along_rows, quantize_adapters, dequantize_adapter, forward_quantized_adapters,
    QMAX8, quantize_activations, forward_w4a8,
    HYBRID_TILE, hybrid_effective_weight, forward_hybrid,
    errors, within_tolerance, canonical_bytes, REL_FRO_TOL, MAX_ABS_TOL,
)
