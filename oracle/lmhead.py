"""Oracle for the fused lm_head variant.

flashrec 0.1.0, Features > Decoding ("SID constraint"): lm_head is evaluated
over the SID token range only. The logits of a beam row are the dot products
of its hidden state with the SID-range rows of the lm_head weight; the step
then proceeds exactly as ``beam.beam_step``.

The bf16 operands are widened exactly to float64 and multiplied by numpy's
float64 matmul (a library primitive standing for the plain definition
logits[row, c] = sum_k h[row, k] * w[c, k]).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import numpy as np

from .beam import beam_step


def _bf16_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32) \
        .astype(np.float64)


def lmhead_logits(hidden_bf16_bits, weight_bf16_bits) -> np.ndarray:
    """hidden [rows, d], weight [V, d] (bf16 bit patterns) -> logits [rows, V] float64."""
    h = _bf16_to_f64(hidden_bf16_bits)
    w = _bf16_to_f64(weight_bf16_bits)
    return h @ w.T


def fused_lmhead_step(trie, step, hidden_bf16_bits, weight_bf16_bits, parent_scores,
                      parent_nodes, R, B_in, n):
    logits = lmhead_logits(hidden_bf16_bits, weight_bf16_bits)
    V = logits.shape[1]
    return beam_step(trie, step, logits, parent_scores, parent_nodes, R, B_in, n, V)
