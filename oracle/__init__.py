"""fp64 CPU oracle of the ReST ranking forward.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and
the benchmark's CPU-baseline leg. The library under
``shared_prefix_behavior_b200`` never imports it and shares no code with it.
"""
from .rest_oracle import (  # noqa: F401
    UnsortedTimestamps, rotation_index, frequencies, rotation_angles, rotate, sigmoid, silu,
    layer_norm, softmax_rows, causal_attention_probs, dga_sublayer, ffn_sublayer, srn,
    encoder, encoder_append, encoder_rows, attention_core, attention_core_backward, attention_core_dq_rows, cross_decode, score_head, rank_request,
)
