"""Model statements of the workloads (params.json fields of the Llama-3
walkthrough plus cache sizing). Plain data; building a model goes through
binding.llama_create."""
from __future__ import annotations

LLAMA3_8B = dict(dim=4096, n_layers=32, n_heads=32, n_kv_heads=8, vocab_size=128256, multiple_of=1024,
                 ffn_dim_multiplier=1.3, norm_eps=1e-5, rope_theta=500000.0)

TINY = dict(dim=256, n_layers=2, n_heads=8, n_kv_heads=2, vocab_size=1024, ffn_hidden=768, multiple_of=256,
            ffn_dim_multiplier=0.0, norm_eps=1e-5, rope_theta=500000.0)


def make_config(params: dict, *, dtype: int, max_batch: int, max_seq: int, max_tokens: int = 0, **over):
    """A binding.llama_config from a params dict (ffn_hidden 0 = derived)."""
    from .binding import llama_config
    p = dict(params)
    p.update(over)
    return llama_config(dim=p['dim'], n_layers=p['n_layers'], n_heads=p['n_heads'], n_kv_heads=p['n_kv_heads'],
                        vocab_size=p['vocab_size'], ffn_hidden=p.get('ffn_hidden', 0),
                        multiple_of=p.get('multiple_of', 256), ffn_dim_multiplier=p.get('ffn_dim_multiplier', 0.0),
                        norm_eps=p['norm_eps'], rope_theta=p['rope_theta'], max_batch=max_batch, max_seq=max_seq,
                        max_tokens=max_tokens, dtype=dtype, kv_page_size=p.get('kv_page_size', 0),
                        kv_pages=p.get('kv_pages', 0), act_dtype=p.get('act_dtype', 0))
