"""Llama-3 decoder forward pass (prefill + KV-cache decode) on B200 (sm_100a).

The compute lives in libllama_b200.so (C ABI, include/llama_b200.h);
``llama_transformer_decoder_b200.binding`` is its ctypes binding, ``configs``
holds the model statements used by the tests and the benchmark and ``build``
compiles the library.
"""
from . import configs  # noqa: F401
