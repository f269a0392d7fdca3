"""CPU oracle of the Llama-3 decoder forward pass (prefill and KV-cache decode).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or call this module.
The CUDA library never does, and this module never touches it: the two share
nothing but the seeded input generator (``seeded_inputs``).

It is the plain definition of what the pages compute, written with numpy in
float64 by default (``dtype=np.float32`` gives the single-precision variant
used as a timing baseline and as a rounding-noise probe). Matrix products use
numpy's ``@``; everything else is elementwise numpy in the order the pages
state it. No intermediate is rounded to bfloat16: bf16 inputs arrive as exact
float values and are used as such.

Sources (cited by page title and section):
  [W] "250行代码从头搭建Llama 3，GitHub一天4.6k星！Karpathy大赞" (ai02.cc walkthrough
      of llama3-from-scratch): sections 下载并读取模型权重 (weights, params),
      分词器与编码 (embedding), 构建Transformer层 (RMSNorm), 查询向量 / 位置编码 /
      键向量 / 查询和键相乘 / 掩码 / 值向量 / 注意力向量 / 多头注意力 (attention),
      相加与归一化 (residual), 前馈神经网络层 (SwiGLU), 预测下一个输出 (final norm,
      logits, argmax).
  [D] "Deepdive-llama3-from-scratch" (pitchhut.com): the rms_norm example and
      the KV-Cache chapter summary.
  [H] "Llama 3 implemented in pure NumPy | Hacker News Reader": cache
      pre-allocation by max_seq_len x max_batch_size; complex vs real rotary.

Readings where the pages are silent or garbled are stated at each function.
Every function is pinned by tests/test_oracle_pins.py except where its
docstring says "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Mapping

import numpy as np


# ---------------------------------------------------------------------------
# Model statement
@dataclass(frozen=True)
class Params:
    """Model hyper-parameters as printed in params.json ([W] 下载并读取模型权重)."""
    dim: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    vocab_size: int
    ffn_hidden: int
    norm_eps: float = 1e-5
    rope_theta: float = 500000.0

    @property
    def head_dim(self) -> int:
        # [W] 查询向量: head_dim = wq.shape[0] // n_heads (4096 // 32 = 128).
        return self.dim // self.n_heads


def ffn_hidden_dim(dim: int, multiple_of: int, ffn_dim_multiplier: float | None) -> int:
    """SwiGLU hidden width from (dim, multiple_of, ffn_dim_multiplier).

    The pages print only multiple_of = 1024 and ffn_dim_multiplier = 1.3
    ([W] 下载并读取模型权重) and no w1 shape. Reading: start from floor(8*dim/3)
    (two thirds of the classic 4*dim), scale by the multiplier (truncating), and
    round up to a multiple of multiple_of. For dim 4096 this is 14336.
    """
    hidden = (8 * dim) // 3
    if ffn_dim_multiplier is not None and ffn_dim_multiplier > 0:
        hidden = int(ffn_dim_multiplier * hidden)
    return multiple_of * ((hidden + multiple_of - 1) // multiple_of)


# ---------------------------------------------------------------------------
# Operations
def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x * rsqrt(mean(x**2 over the last axis) + eps) * g, per token.

    [W] 构建Transformer层 and [D] (rms_norm example): norm_eps guards a zero RMS.
    """
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return (x * (1.0 / np.sqrt(ms + eps))) * g


def rope_freqs(head_dim: int, theta: float) -> np.ndarray:
    """Inverse frequencies 1 / theta**(i / (head_dim/2)), i = 0 .. head_dim/2 - 1.

    [W] 位置编码: 64 parts of [0,1) for head_dim 128, freqs = 1/(rope_theta**t).
    Reading: no factor 2*pi (the printed table has none); computed in float64.
    """
    half = head_dim // 2
    return 1.0 / (float(theta) ** (np.arange(half, dtype=np.float64) / half))


def rope_angles(positions: np.ndarray, head_dim: int, theta: float) -> np.ndarray:
    """Angle m * freqs[i] for every absolute position m ([W] 位置编码, torch.outer)."""
    return np.outer(np.asarray(positions, dtype=np.float64), rope_freqs(head_dim, theta))


def apply_rope(u: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate adjacent pairs (u[2i], u[2i+1]) of the last axis as complex numbers.

    [W] 位置编码 / 键向量: the vector is viewed as [..., d/2, 2], each pair becomes
    the complex number u[2i] + i*u[2i+1] and is multiplied by
    exp(i * m * freqs[i]), then viewed back as reals. u has shape [..., S, d]
    and positions has shape [S] (absolute token index m, from 0).
    """
    d = u.shape[-1]
    ang = rope_angles(positions, d, theta)                      # [S, d/2]
    rot = np.exp(1j * ang)
    c = u[..., 0::2] + 1j * u[..., 1::2]
    c = c * rot
    out = np.empty_like(u)
    out[..., 0::2] = c.real
    out[..., 1::2] = c.imag
    return out


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax with -inf entries contributing zero ([W] 多头注意力, dim=1)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos: np.ndarray,
              return_probs: bool = False):
    """Causal grouped-query attention for one sequence.

    q: [H, S, d] (already rotated), k: [Hk, T, d] (rotated), v: [Hk, T, d];
    q_pos[s] is the absolute position of query s, and key j is visible to it
    iff j <= q_pos[s] ([W] 掩码: triu of -inf above the diagonal).
    Head h reads kv head h // (H // Hk) ([W] 多头注意力: head//4 for 32/8).
    Scores are q.k / sqrt(d) ([W] 查询和键相乘). Output [S, H*d], heads
    concatenated in order ([W] 多头注意力, torch.cat(dim=-1)).
    """
    H, S, d = q.shape
    Hk, T, _ = k.shape
    group = H // Hk
    scale = 1.0 / math.sqrt(d)
    keys = np.arange(T)
    mask = keys[None, :] > np.asarray(q_pos)[:, None]           # [S, T]
    out = np.empty((S, H * d), dtype=q.dtype)
    probs = []
    for h in range(H):
        g = h // group
        s = (q[h] @ k[g].T) * scale
        s = np.where(mask, -np.inf, s)
        p = softmax_rows(s)
        out[:, h * d:(h + 1) * d] = p @ v[g]
        if return_probs:
            probs.append(p)
    if return_probs:
        return out, np.stack(probs)
    return out


def silu(z: np.ndarray) -> np.ndarray:
    """z * sigmoid(z) = z / (1 + exp(-z)) (F.silu in [W] 前馈神经网络层)."""
    with np.errstate(over='ignore'):
        return z / (1.0 + np.exp(-z))


def feed_forward(xn: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """SwiGLU: (silu(xn w1^T) * (xn w3^T)) w2^T ([W] 前馈神经网络层)."""
    return (silu(xn @ w1.T) * (xn @ w3.T)) @ w2.T


# ---------------------------------------------------------------------------
# Decoder
@dataclass
class SequenceCache:
    """KV cache of one sequence: per layer post-RoPE K and raw V, [Hk, len, d].

    The pages describe a KV cache without code ([D] KV-Cache chapter); [H]
    adds that the cache is sized up front by max_seq_len and max_batch_size.
    Reading: store K after rotation (so decode never re-rotates) and V as is.
    """
    k: list = field(default_factory=list)
    v: list = field(default_factory=list)

    @property
    def length(self) -> int:
        return 0 if not self.k else self.k[0].shape[1]


class Oracle:
    """Plain forward pass over a weight mapping (names as in the checkpoint).

    ``weights[name]`` returns an array in the [out, in] convention of the
    checkpoint ([W] 多头注意力: y = x @ W.T). Values are cast to ``dtype``.
    """

    def __init__(self, params: Params, weights: Mapping[str, np.ndarray], dtype=np.float64):
        self.p = params
        self.w = weights
        self.dtype = dtype

    def W(self, name: str) -> np.ndarray:
        return np.asarray(self.w[name], dtype=self.dtype)

    def new_cache(self) -> SequenceCache:
        return SequenceCache()

    def layer(self, i: int, x: np.ndarray, cache: SequenceCache | None, pos0: int,
              rows: np.ndarray | None = None) -> np.ndarray:
        """One decoder block on x [S, dim] whose first token sits at position pos0.

        Steps ([W] 构建Transformer层 .. 相加与归一化 .. 前馈神经网络层):
        xn = rms_norm(x, attention_norm); q,k,v = xn wq^T, xn wk^T, xn wv^T split
        into heads of head_dim consecutive rows; rotate q and k; causal GQA over
        the cache plus the new keys; h = x + attn wo^T; out = h +
        SwiGLU(rms_norm(h, ffn_norm)). With ``rows`` only those query rows are
        produced (keys and values of every row are still computed).
        """
        p = self.p
        d, H, Hk = p.head_dim, p.n_heads, p.n_kv_heads
        S = x.shape[0]
        pre = f'layers.{i}.'
        x = np.asarray(x, dtype=self.dtype)
        xn = rms_norm(x, self.W(pre + 'attention_norm.weight'), p.norm_eps)
        pos = pos0 + np.arange(S)
        k = (xn @ self.W(pre + 'attention.wk.weight').T).reshape(S, Hk, d).transpose(1, 0, 2)
        v = (xn @ self.W(pre + 'attention.wv.weight').T).reshape(S, Hk, d).transpose(1, 0, 2)
        k = apply_rope(k, pos, p.rope_theta)
        if cache is not None:
            if len(cache.k) <= i:
                cache.k.append(k)
                cache.v.append(v)
            else:
                cache.k[i] = np.concatenate([cache.k[i], k], axis=1)
                cache.v[i] = np.concatenate([cache.v[i], v], axis=1)
            kall, vall = cache.k[i], cache.v[i]
        else:
            kall, vall = k, v
        sel = np.arange(S) if rows is None else np.asarray(rows)
        xs, xns = x[sel], xn[sel]
        q = (xns @ self.W(pre + 'attention.wq.weight').T).reshape(len(sel), H, d).transpose(1, 0, 2)
        q = apply_rope(q, pos[sel], p.rope_theta)
        o = attention(q, kall, vall, pos[sel])
        h = xs + o @ self.W(pre + 'attention.wo.weight').T
        hn = rms_norm(h, self.W(pre + 'ffn_norm.weight'), p.norm_eps)
        return h + feed_forward(hn, self.W(pre + 'feed_forward.w1.weight'),
                                self.W(pre + 'feed_forward.w3.weight'),
                                self.W(pre + 'feed_forward.w2.weight'))

    def embed(self, tokens: np.ndarray) -> np.ndarray:
        """Row gather of tok_embeddings ([W] 分词器与编码)."""
        return self.W('tok_embeddings.weight')[np.asarray(tokens)]

    def logits(self, x_last: np.ndarray) -> np.ndarray:
        """rms_norm(x, norm) then @ output^T on the last token ([W] 预测下一个输出).

        The page prints the final rms_norm line twice; the text describes one
        normalisation, so it is applied once.
        """
        xf = rms_norm(np.asarray(x_last, dtype=self.dtype), self.W('norm.weight'), self.p.norm_eps)
        return xf @ self.W('output.weight').T

    def forward(self, tokens: np.ndarray, cache: SequenceCache | None = None,
                return_hidden: bool = False):
        """Tokens [S] of one sequence, appended after the cache's current length.

        Returns the logits of the last token ([vocab]) and, if asked, the final
        hidden states before the last norm ([S, dim]). Without return_hidden the
        last layer evaluates only the last row (its keys and values are still
        computed for every row).
        """
        pos0 = 0 if cache is None else cache.length
        x = self.embed(tokens)
        S = x.shape[0]
        for i in range(self.p.n_layers):
            last_only = not return_hidden and i == self.p.n_layers - 1
            x = self.layer(i, x, cache, pos0, rows=np.array([S - 1]) if last_only else None)
        lg = self.logits(x[-1])
        return (lg, x) if return_hidden else lg

    def prefill(self, tokens: np.ndarray):
        """Batch prefill: tokens [B, S] -> (logits [B, vocab], caches)."""
        tokens = np.atleast_2d(tokens)
        caches = [self.new_cache() for _ in range(tokens.shape[0])]
        lg = np.stack([self.forward(t, c) for t, c in zip(tokens, caches)])
        return lg, caches

    def decode_step(self, tokens: np.ndarray, caches: list) -> np.ndarray:
        """One token per sequence at position len(cache): logits [B, vocab]."""
        return np.stack([self.forward(np.array([t]), c) for t, c in zip(np.ravel(tokens), caches)])


def argmax(logits: np.ndarray) -> np.ndarray:
    """Greedy next token ([W] 预测下一个输出: torch.argmax); ties -> lowest index."""
    return np.argmax(logits, axis=-1).astype(np.int32)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    """||a - b||_2 / ||b||_2 in float64 (the parity metric)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
