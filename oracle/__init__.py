"""CPU oracle for the Llama-3 decoder forward pass.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline legs of bench.py, never by the CUDA library or its binding.
"""
from .llama_oracle import (Oracle, Params, SequenceCache, apply_rope, argmax, attention,  # noqa: F401
                           feed_forward, ffn_hidden_dim, rel_l2, rms_norm, rope_angles, rope_freqs,
                           silu, softmax_rows)
