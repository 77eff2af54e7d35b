"""Seeded synthetic inputs (random draws only; none of the layer's arithmetic)."""
from .synth import (BF16_MAX, EXTREME_KINDS, extreme_token, extreme_tokens, HIDDEN, INTER, NUM_EXPERTS, TOP_K, GROUP, LayerWeights, layer_weights,
                    tokens, token_stream, zipf_router_bias, stack_token_seed, WORKLOADS,
                    VOCAB, lm_head_weights, LMHEAD_WORKLOADS, layer_weights_mxfp4)
