"""Shared test helpers: seeded host inputs for the oracle and device buffers
for the library. Host values come from seeded_inputs only; nothing here
reads a result of the CUDA path back into an oracle input."""
from __future__ import annotations

import numpy as np

import seeded_inputs as si
from oracle import Params

BF16, F32, F16 = 1, 0, 2


def params_from(cfg: dict, ffn_hidden: int) -> Params:
    return Params(dim=cfg['dim'], n_layers=cfg['n_layers'], n_heads=cfg['n_heads'], n_kv_heads=cfg['n_kv_heads'],
                  vocab_size=cfg['vocab_size'], ffn_hidden=ffn_hidden, norm_eps=cfg['norm_eps'],
                  rope_theta=cfg['rope_theta'])


class SeededWeights(dict):
    """Checkpoint-named weights of ``llama_init_weights(seed, std)``, generated on
    the host on first use (float32 values of the exact bf16, fp16 or fp32 draws)."""

    def __init__(self, p: Params, seed: int, std: float, dtype: int, cache: bool = True):
        super().__init__()
        self.p, self.seed, self.std, self.dtype, self.cache = p, seed, std, dtype, cache

    def __missing__(self, name):
        p = self.p
        shape = si.weight_shape(name, p.dim, p.n_heads, p.n_kv_heads, p.ffn_hidden, p.vocab_size)
        if name.endswith('norm.weight'):
            v = np.ones(shape, np.float32)
        elif self.dtype == F16:
            v = si.weight(self.seed, name, shape, p.n_layers, self.std, 'f32').astype(np.float16).astype(np.float32)
        else:
            raw = si.weight(self.seed, name, shape, p.n_layers, self.std, 'bf16' if self.dtype == BF16 else 'f32')
            v = si.bf16_bits_to_f32(raw) if self.dtype == BF16 else raw
        if self.cache:
            self[name] = v
        return v


def normal_values(seed: int, stream: int, shape, dtype: int, std: float = 1.0):
    """(host float32 values, raw array for upload: uint16 bf16 bits, float16 or
    float32). fp16 inputs are the fp32 draws rounded to nearest-even fp16."""
    n = int(np.prod(shape))
    if dtype == F16:
        raw = si.normal(seed, stream, n, std, 'f32').reshape(shape).astype(np.float16)
        return raw.astype(np.float32), raw
    raw = si.normal(seed, stream, n, std, 'bf16' if dtype == BF16 else 'f32').reshape(shape)
    vals = si.bf16_bits_to_f32(raw) if dtype == BF16 else raw
    return vals, raw


def torch_dtype(dtype: int):
    import torch
    return {BF16: torch.bfloat16, F16: torch.float16, F32: torch.float32}[dtype]


def to_device(raw: np.ndarray, dtype: int):
    import torch
    if dtype == BF16:
        t = torch.from_numpy(raw.view(np.int16).copy()).view(torch.bfloat16)
    elif dtype == F16:
        t = torch.from_numpy(np.ascontiguousarray(raw, dtype=np.float16))
    else:
        t = torch.from_numpy(np.ascontiguousarray(raw, dtype=np.float32))
    return t.cuda()


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


class Top1:
    """Greedy decisions of the GPU checked against the oracle's logits.

    ``add`` records one decision: the token the GPU chose, the oracle's logits
    for the same step (teacher-forced on the GPU's earlier tokens) and, when
    available, the GPU's logits. ``agree`` counts strict top-1 agreement
    (GPU token == oracle argmax). A disagreement is a near tie when the
    oracle's top-2 margin is below twice the largest |GPU - oracle| logit error
    of that row: both tokens are then correct within the logits' rounding.
    The near-tie count is reported, never used to pass a decision."""

    def __init__(self):
        self.total = 0
        self.agree = 0
        self.near_ties = 0
        self.small_margins = 0
        self.misses = []

    def add(self, gpu_token: int, oracle_logits, gpu_logits=None):
        ref = np.asarray(oracle_logits, np.float64)
        top2 = np.partition(ref, -2)[-2:]
        margin = float(top2[1] - top2[0])
        err = float(np.max(np.abs(np.asarray(gpu_logits, np.float64) - ref))) if gpu_logits is not None else None
        self.total += 1
        if err is not None and margin < 2 * err:
            self.small_margins += 1
        if int(gpu_token) == int(np.argmax(ref)):
            self.agree += 1
            return
        near = err is not None and margin < 2 * err
        self.near_ties += int(near)
        self.misses.append({'gpu': int(gpu_token), 'oracle': int(np.argmax(ref)), 'margin': margin,
                            'max_logit_err': err,
                            'gpu_token_deficit': float(ref.max() - ref[int(gpu_token)])})

    def fraction(self) -> float:
        return self.agree / max(self.total, 1)

    def summary(self) -> str:
        return (f'top-1 agreement {self.agree}/{self.total} = {self.fraction():.4f}; '
                f'oracle margins below 2x the logit error: {self.small_margins}; '
                f'disagreements that are such near ties: {self.near_ties}; misses: {self.misses[:8]}')


# Unit roundoff of the element type the attention kernels round P and the
# output to (bf16: 8 significant bits, fp16: 11). fp32 kernels: the relative
# error bound of the hardware exp2 approximation (a little under 2**-22).
ROUNDOFF = {BF16: 2.0 ** -8, F16: 2.0 ** -11, F32: 2.0 ** -21}


def attention_row_errors(got, q, k, v, q_pos, dtype):
    """Per (head, query row) check of an attention output against the oracle.

    got: [S, H*d] GPU output rows; q [H, S, d], k/v [Hk, T, d] exact values of
    the kernel's inputs; q_pos positions of the S rows. With unit roundoff u
    of the element type, the kernel rounds each probability p_j once (before
    the P V product) and each output element once, and accumulates in fp32:
    |o_gpu - o| <= u*|o| + u*sum_j p_j |v_j| + u*|o| (the row sum is taken
    over unrounded p). Returns (worst ratio of the row error to that bound
    over all heads and rows, rel-L2 over all rows); a ratio above 1 means a
    head or row is wrong beyond its rounding."""
    from oracle import attention
    H, S, d = q.shape
    Hk = k.shape[0]
    ref, probs = attention(q, k, v, q_pos, return_probs=True)          # [S, H*d], [H, S, T]
    got = np.asarray(got, np.float64).reshape(S, H, d)
    refh = ref.reshape(S, H, d)
    u = ROUNDOFF[dtype]
    worst = 0.0
    for h in range(H):
        g = h // (H // Hk)
        mix = probs[h] @ np.abs(v[g])                                   # [S, d]
        bound = u * (2 * np.linalg.norm(refh[:, h], axis=1) + np.linalg.norm(mix, axis=1))
        err = np.linalg.norm(got[:, h] - refh[:, h], axis=1)
        worst = max(worst, float(np.max(err / bound)))
    return worst, rel_l2(got.reshape(S, H * d), ref)
