"""CPU oracle (test infrastructure only; never on the product path).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package. See ``oracle.oracle`` for the definitions and their sources.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import (bf16_to_f64, bf16_bits, bf16, f32, f16, dequant, dequant_int8_row,  # noqa: F401
                     dequant_int4_affine_g32, int4_codes, silu, gelu_tanh, sigmoid,
                     gated_activation, gate_up_act, ffn_hidden, residual_add, rms_norm,
                     ffn_dense, ffn_shared_expert, router_logits, topk_softmax,
                     expert_permutation, shared_seed, seeded_rank_sum, moe_layer,
                     dense_layer, layer)
