"""fp64 CPU oracle of the HSTU layer forward and backward and of Stochastic
Length sampling (test infrastructure only).

Imported only by the tests, the package smoke check and the benchmark's CPU
baseline leg; the CUDA library shares no code with it.
"""
from .hstu_oracle import (CAUSAL, MFALCON, OracleConfig, effective_n_norm, f1_split,
                          hstu_layer, hstu_stack, layer_norm, pointwise_attention,
                          position_bucket, silu, time_bucket, user_visibility,
                          visible_pairs)
from .hstu_backward import hstu_layer_backward, pointwise_attention_backward
from .stochastic_length import keep_whole, stochastic_length

__all__ = ["CAUSAL", "MFALCON", "OracleConfig", "effective_n_norm", "f1_split", "hstu_layer",
           "hstu_stack", "layer_norm", "pointwise_attention", "position_bucket", "silu",
           "time_bucket", "user_visibility", "visible_pairs", "keep_whole", "stochastic_length",
           "hstu_layer_backward", "pointwise_attention_backward"]
