"""CPU oracle for the tiered mixed-precision MoE layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  It shares no code with the CUDA library.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import (BLOCK, QMAX, Shelf, bits_per_weight, bucketize,  # noqa: F401
                         build_shelf, combine, dequantize_f16, dequantize_f32,
                         expert_ffn, expert_ffn_f16_staged, round_f16, moe_layer, moe_stack, rms_norm, NORM_EPS, pack_rows, packed_row_bytes,
                         quantize_pack, quantize_rows, round_bf16, router_logits,
                         FP4_VALUES, quantize_rows_fp4, fp4_integers, pack_rows_fp4, unpack_rows_fp4,
                         dequantize_fp4_f32, quantize_pack_fp4,
                         select_topk, shelf_of, shelves_lookup, silu, topk_margin, unpack_rows)
