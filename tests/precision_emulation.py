"""Rounding-point emulation of the 16-bit GPU path on the CPU (test
infrastructure; calls only oracle/ and seeded_inputs/).

The oracle computes the pages' forward pass exactly (float64, no rounding of
intermediates). The 16-bit path rounds some intermediates to a 16-bit type
and keeps the rest in fp32: it rounds the normalised activations that enter
the Q/K/V and w1/w3 products, q, k and v, the softmax probabilities before
the product with V (as [W] 多头注意力 rounds softmax(...) to bf16), the
attention output that enters the Wo product, the SwiGLU product that enters
w2, and the final normalised row that enters the LM head; weights are the
exact bf16 draws; products accumulate in fp32; the residual stream and the
logits are fp32.

``forward_rounded`` replays exactly that in float32 with a chosen 16-bit
rounding (bf16 as the pages compute, or fp16 as the library's default
policy), so the logits' distance from the exact result can be measured
without a GPU: that distance is a property of where the rounding happens,
not of any kernel.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np

import seeded_inputs as si
from oracle import Params, apply_rope, rms_norm, silu


def round_bf16(x):
    return si.bf16_bits_to_f32(si.f32_to_bf16_bits(np.asarray(x, np.float32)))


def round_fp16(x):
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float32)


def no_round(x):
    return x


def layer_weights(seed: int, p: Params, i: int, std: float = 0.02) -> dict:
    """The bf16 draws of layer i (as float32), generated in parallel."""
    names = [f'layers.{i}.{k}.weight' for k in si.LAYER_KEYS]

    def one(name):
        shape = si.weight_shape(name, p.dim, p.n_heads, p.n_kv_heads, p.ffn_hidden, p.vocab_size)
        w = si.weight(seed, name, shape, p.n_layers, std, 'bf16')
        return name, (w if name.endswith('norm.weight') else si.bf16_bits_to_f32(w))

    with ThreadPoolExecutor(8) as ex:
        return dict(ex.map(one, names))


def embed_rows(seed: int, p: Params, tokens, std: float = 0.02) -> np.ndarray:
    stream = si.weight_stream('tok_embeddings.weight', p.n_layers)
    return np.stack([si.bf16_bits_to_f32(si.normal(seed, stream, p.dim, std, 'bf16', start=int(t) * p.dim))
                     for t in tokens])


def output_weight(seed: int, p: Params, std: float = 0.02) -> np.ndarray:
    stream = si.weight_stream('output.weight', p.n_layers)
    rows = p.vocab_size
    step = (rows + 7) // 8

    def part(a):
        b = min(rows, a + step)
        return si.bf16_bits_to_f32(si.normal(seed, stream, (b - a) * p.dim, std, 'bf16', start=a * p.dim))

    with ThreadPoolExecutor(8) as ex:
        return np.concatenate(list(ex.map(part, range(0, rows, step)))).reshape(rows, p.dim)


def _attention_rounded(q, k, v, rnd, dtype):
    """Causal GQA of one sequence (positions 0..S-1): p = exp(s - max) rounded
    before the value product, normalised by the sum of the unrounded p."""
    H, S, d = q.shape
    group = H // k.shape[0]
    mask = np.arange(S)[None, :] > np.arange(S)[:, None]
    out = np.empty((S, H * d), dtype)
    for h in range(H):
        s = (q[h] @ k[h // group].T) * (1.0 / np.sqrt(d))
        s = np.where(mask, -np.inf, s)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        out[:, h * d:(h + 1) * d] = (rnd(e) @ v[h // group]) / e.sum(axis=1, keepdims=True)
    return out


def layer_rounded(x, w, p: Params, i: int, rnd, dtype):
    """One decoder block in `dtype` arithmetic with 16-bit roundings `rnd`."""
    d, H, Hk = p.head_dim, p.n_heads, p.n_kv_heads
    S = x.shape[0]
    pre = f'layers.{i}.'
    W = {k: np.asarray(v, dtype) for k, v in w.items()}
    pos = np.arange(S)
    xn = rnd(rms_norm(x, W[pre + 'attention_norm.weight'], p.norm_eps))
    q = (xn @ W[pre + 'attention.wq.weight'].T).reshape(S, H, d).transpose(1, 0, 2)
    k = (xn @ W[pre + 'attention.wk.weight'].T).reshape(S, Hk, d).transpose(1, 0, 2)
    v = rnd((xn @ W[pre + 'attention.wv.weight'].T).reshape(S, Hk, d).transpose(1, 0, 2))
    q = rnd(apply_rope(q, pos, p.rope_theta).astype(dtype))
    k = rnd(apply_rope(k, pos, p.rope_theta).astype(dtype))
    o = rnd(_attention_rounded(q, k, v, rnd, dtype))
    h = x + o @ W[pre + 'attention.wo.weight'].T
    hn = rnd(rms_norm(h, W[pre + 'ffn_norm.weight'], p.norm_eps))
    g = rnd(silu(hn @ W[pre + 'feed_forward.w1.weight'].T) * (hn @ W[pre + 'feed_forward.w3.weight'].T))
    return (h + g @ W[pre + 'feed_forward.w2.weight'].T).astype(dtype)


def last_token_logits(seed: int, p: Params, tokens, variants: dict, std: float = 0.02) -> dict:
    """Last-token logits of every variant {name: (rnd, dtype)} over the same
    weights, each layer's weights generated once and shared by the variants."""
    x0 = embed_rows(seed, p, tokens, std)
    xs = {name: np.asarray(x0, dt) for name, (_, dt) in variants.items()}
    for i in range(p.n_layers):
        w = layer_weights(seed, p, i, std)
        for name, (rnd, dt) in variants.items():
            xs[name] = layer_rounded(xs[name], w, p, i, rnd, dt)
    out_w = output_weight(seed, p, std)
    res = {}
    for name, (rnd, dt) in variants.items():
        xf = rnd(rms_norm(xs[name][-1], np.ones(p.dim, dt), p.norm_eps))
        res[name] = np.asarray(xf, np.float64) @ np.asarray(out_w, np.float64).T
    return res


def _attention_rounded_at(q, k, v, q_pos, rnd, dtype):
    """_attention_rounded for queries at absolute positions q_pos over keys
    0 .. T-1 (key j visible to query i iff j <= q_pos[i])."""
    H, S, d = q.shape
    group = H // k.shape[0]
    mask = np.arange(k.shape[1])[None, :] > np.asarray(q_pos)[:, None]
    out = np.empty((S, H * d), dtype)
    for h in range(H):
        s = (q[h] @ k[h // group].T) * (1.0 / np.sqrt(d))
        s = np.where(mask, -np.inf, s)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        out[:, h * d:(h + 1) * d] = (rnd(e) @ v[h // group]) / e.sum(axis=1, keepdims=True)
    return out


def pass_after_cache_rounded(p: Params, w, cache_k, cache_v, tokens, rnd, dtype=np.float32):
    """Last-token logits of every row of one causal pass over `tokens` placed
    after a cache (cache_k[l], cache_v[l]: [Hk, c, d], exact values, taken as
    already rotated), with the 16-bit roundings `rnd` at the GPU path's
    rounding points (decode shapes: the normalised activations are rounded
    after the scale). Row i is the decode step that consumes tokens[i]."""
    d, H, Hk = p.head_dim, p.n_heads, p.n_kv_heads
    c = cache_k[0].shape[1]
    T = len(tokens)
    pos = c + np.arange(T)
    x = rnd(np.asarray(w['tok_embeddings.weight'][np.asarray(tokens)], dtype))
    for i in range(p.n_layers):
        pre = f'layers.{i}.'
        W = lambda n: np.asarray(w[pre + n], dtype)
        xn = rnd(rms_norm(x, W('attention_norm.weight'), p.norm_eps))
        q = (xn @ W('attention.wq.weight').T).reshape(T, H, d).transpose(1, 0, 2)
        k = (xn @ W('attention.wk.weight').T).reshape(T, Hk, d).transpose(1, 0, 2)
        v = rnd((xn @ W('attention.wv.weight').T).reshape(T, Hk, d).transpose(1, 0, 2))
        q = rnd(apply_rope(q, pos, p.rope_theta).astype(dtype))
        k = rnd(apply_rope(k, pos, p.rope_theta).astype(dtype))
        kall = np.concatenate([np.asarray(cache_k[i], dtype), k], axis=1)
        vall = np.concatenate([np.asarray(cache_v[i], dtype), v], axis=1)
        o = rnd(_attention_rounded_at(q, kall, vall, pos, rnd, dtype))
        h = x + o @ W('attention.wo.weight').T
        hn = rnd(rms_norm(h, W('ffn_norm.weight'), p.norm_eps))
        g = rnd(silu(hn @ W('feed_forward.w1.weight').T) * (hn @ W('feed_forward.w3.weight').T))
        x = (h + g @ W('feed_forward.w2.weight').T).astype(dtype)
    xf = rnd(rms_norm(x, np.asarray(w['norm.weight'], dtype), p.norm_eps))
    return np.asarray(xf, np.float64) @ np.asarray(w['output.weight'], np.float64).T
