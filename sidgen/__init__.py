"""Seeded synthetic-input generators shared by the oracle and the CUDA path.

This module draws random numbers only. It holds none of the beam-search
arithmetic: no softmax, no trie walk, no selection. Both sides of a parity
test call it so that they see the same inputs:

* ``sidgen.host``   -- numpy twin (used by the oracle side and by catalog draws);
* ``sidgen.device`` -- CUDA twin in ``libsidgen.so`` (used by the GPU side to
  make logits on the device, keyed by each beam's prefix hash).

The two twins are bit-identical by construction: integer Philox4x32-10,
integer SplitMix64 hashing, an integer Irwin-Hall sum and exactly one
correctly rounded fp32 multiply per normal draw.
"""
from .host import (  # noqa: F401
    GOLDEN_GAMMA,
    PREFIX_HASH_SEED,
    STREAM_BEAM_LOGITS,
    STREAM_TABLE,
    STREAM_HIDDEN,
    STREAM_WEIGHT,
    bf16_bits_to_f32,
    child_hash,
    draw_catalog,
    f32_to_bf16_bits,
    k_sigma,
    normal_from_counters,
    philox4x32_10,
    prefix_hashes,
    request_roots,
    row_logits,
    table_logits,
    hidden_states,
    weight_matrix,
    root_hash,
    splitmix64_mix,
    splitmix64_stream,
)
