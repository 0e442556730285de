"""CPU fp64 oracle for HCA.  Test infrastructure only: the product path never
imports this package (see ``oracle.hca_oracle``)."""
from .hca_oracle import (  # noqa: F401
    BLOCK, HEADS, HEAD_DIM, WINDOW, attend, block_weights, cache_append, compress,
    decode_forward, decode_keys, dequantize_e4m3_rows, e4m3_decode, e4m3_encode,
    num_visible_blocks, prefill_backward, prefill_forward, quantize_e4m3_rows,
    round_bf16, sigmoid, vha_mix, visited_pairs, window_start,
)
