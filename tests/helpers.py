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


def near_tie_ok(gpu_token: int, oracle_logits: np.ndarray, slack: float) -> bool:
    """The GPU's greedy token is the oracle's argmax, or within `slack` of its maximum
    (several tokens are then correct within the rounding of the bf16 path)."""
    return oracle_logits[gpu_token] >= oracle_logits.max() - slack
