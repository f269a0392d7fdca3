"""Seeded synthetic inputs shared by the CPU oracle, the tests and the bench.

This module holds no arithmetic of the decoder itself. It only draws the
numbers that stand in for trained weights, token ids, hidden states and KV
cache entries, which the pages take from Meta's checkpoint and tokenizer
(neither of which exists here).

Generator definition (the CUDA library implements the same definition in its
own device code; the two agree bit for bit):

* ``mix64`` is the SplitMix64 output function (Steele, Lea & Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014; constants as in
  Vigna's public-domain reference).
* A tensor is a *stream*: ``key = mix64(seed*G + stream*M1 + G)`` and its i-th
  64-bit draw is ``mix64(key + (i+1)*G)`` (all mod 2**64, G = golden gamma).
* Normal value i uses draws 2i and 2i+1: ``u1 = ((d0>>11)+1)*2**-53`` in (0,1],
  ``u2 = (d1>>11)*2**-53`` in [0,1), ``z = sqrt(-2*ln(u1)) * cos(2*pi*u2)``
  (Box & Muller 1958). ``ln`` and ``cos(2*pi*.)`` are evaluated with IEEE
  add/mul/div/sqrt only, in a fixed order (no fused multiply-add), so that any
  IEEE-754 machine reproduces the same bits:
  - ``ln``: ``u = m*2**e`` with m in [1/sqrt2, sqrt2), ``s=(m-1)/(m+1)``,
    ``ln m = 2*s*sum_k s**(2k)/(2k+1)`` (the atanh series), k = 0..10, Horner.
  - ``cos(2*pi*t)``: exact reductions by the symmetries t -> 1-t, t -> 1/2-t,
    t -> 1/4-t (t is a multiple of 2**-53, so they are exact), then the Taylor
    series of cos or sin on [0, pi/4], ten terms, Horner.
* ``value = float32(z * double(std))`` (round to nearest even); bf16 values are
  that float32 rounded to nearest even on the upper 16 bits.
* Token ids: ``((draw >> 32) * V) >> 32``.

Streams: weights use the key ordinal of the checkpoint listing on the pages
(tok_embeddings = 0; layer i: wq, wk, wv, wo, w1, w3, w2, attention_norm,
ffn_norm = 1+9i .. 9+9i; norm = 1+9L; output = 2+9L). Norm weights are 1.0.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

G = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB

_COS = [float.fromhex(h) for h in (
    '0x1.0000000000000p+0', '-0x1.0000000000000p-1', '0x1.5555555555555p-5',
    '-0x1.6c16c16c16c17p-10', '0x1.a01a01a01a01ap-16', '-0x1.27e4fb7789f5cp-22',
    '0x1.1eed8eff8d898p-29', '-0x1.93974a8c07c9dp-37', '0x1.ae7f3e733b81fp-45',
    '-0x1.6827863b97d97p-53')]
_SIN = [float.fromhex(h) for h in (
    '0x1.0000000000000p+0', '-0x1.5555555555555p-3', '0x1.1111111111111p-7',
    '-0x1.a01a01a01a01ap-13', '0x1.71de3a556c734p-19', '-0x1.ae64567f544e4p-26',
    '0x1.6124613a86d09p-33', '-0x1.ae7f3e733b81fp-41', '0x1.952c77030ad4ap-49',
    '-0x1.2f49b46814157p-57')]
_ATANH = [float.fromhex(h) for h in (
    '0x1.0000000000000p+0', '0x1.5555555555555p-2', '0x1.999999999999ap-3',
    '0x1.2492492492492p-3', '0x1.c71c71c71c71cp-4', '0x1.745d1745d1746p-4',
    '0x1.3b13b13b13b14p-4', '0x1.1111111111111p-4', '0x1.e1e1e1e1e1e1ep-5',
    '0x1.af286bca1af28p-5', '0x1.8618618618618p-5')]
LN2 = float.fromhex('0x1.62e42fefa39efp-1')
TWO_PI = float.fromhex('0x1.921fb54442d18p+2')
INV_SQRT2 = float.fromhex('0x1.6a09e667f3bcdp-1')

# Stream ordinals for non-weight inputs (kept far from the weight ordinals).
STREAM_TOKENS = 1 << 20
STREAM_HIDDEN = (1 << 20) + 1
STREAM_Q = (1 << 20) + 2
STREAM_LOGITS = (1 << 20) + 3
STREAM_KV_BASE = 1 << 21          # + 2*layer (+1 for V)
STREAM_K = (1 << 20) + 4
STREAM_V = (1 << 20) + 5

_U64 = np.uint64


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> _U64(30))) * _U64(M1)
    z = (z ^ (z >> _U64(27))) * _U64(M2)
    return z ^ (z >> _U64(31))


def stream_key(seed: int, stream: int) -> int:
    v = (seed * G + stream * M1 + G) & 0xFFFFFFFFFFFFFFFF
    return int(_mix64(np.array([v], dtype=np.uint64))[0])


def draws(seed: int, stream: int, index: np.ndarray) -> np.ndarray:
    """64-bit draws number ``index`` (uint64 array) of one stream."""
    key = _U64(stream_key(seed, stream))
    with np.errstate(over='ignore'):
        z = key + (index.astype(np.uint64) + _U64(1)) * _U64(G)
        return _mix64(z)


def det_log(u: np.ndarray) -> np.ndarray:
    """ln(u) for u in (0, 1] from IEEE basic operations (atanh series)."""
    m, e = np.frexp(u)                       # u = m * 2**e, m in [0.5, 1)
    small = m < INV_SQRT2
    m = np.where(small, m * 2.0, m)
    e = np.where(small, e - 1, e).astype(np.float64)
    s = (m - 1.0) / (m + 1.0)
    s2 = s * s
    p = np.full_like(s, _ATANH[-1])
    for c in reversed(_ATANH[:-1]):
        p = p * s2 + c
    return e * LN2 + (2.0 * s) * p


def det_cos2pi(t: np.ndarray) -> np.ndarray:
    """cos(2*pi*t) for t in [0, 1) from IEEE basic operations."""
    t = np.where(t > 0.5, 1.0 - t, t)
    neg = t > 0.25
    t = np.where(neg, 0.5 - t, t)
    use_sin = t > 0.125
    x = np.where(use_sin, 0.25 - t, t) * TWO_PI
    x2 = x * x
    pc = np.full_like(x, _COS[-1])
    for c in reversed(_COS[:-1]):
        pc = pc * x2 + c
    ps = np.full_like(x, _SIN[-1])
    for c in reversed(_SIN[:-1]):
        ps = ps * x2 + c
    r = np.where(use_sin, x * ps, pc)
    return np.where(neg, -r, r)


def normal_f64(seed: int, stream: int, index: np.ndarray) -> np.ndarray:
    """Standard normal draws (float64) for element indices ``index``."""
    index = np.asarray(index, dtype=np.uint64)
    d0 = draws(seed, stream, index * _U64(2))
    d1 = draws(seed, stream, index * _U64(2) + _U64(1))
    u1 = ((d0 >> _U64(11)) + _U64(1)).astype(np.float64) * 2.0 ** -53
    u2 = (d1 >> _U64(11)).astype(np.float64) * 2.0 ** -53
    return np.sqrt(-2.0 * det_log(u1)) * det_cos2pi(u2)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + _U64(0x7FFF) + ((b >> _U64(16)) & _U64(1))) >> _U64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# Optional C fast path (same definition, compiled with contraction disabled).
_lib = None
_lib_lock = threading.Lock()
_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, 'libseeded.so')


def build_c(force: bool = False) -> str:
    src = os.path.join(_HERE, 'seeded.c')
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(['gcc', '-O2', '-std=c11', '-fPIC', '-shared', '-fopenmp',
                               '-ffp-contract=off', '-fno-fast-math', src, '-o', _SO, '-lm'])
    return _SO


def _c():
    global _lib
    with _lib_lock:
        if _lib is None:
            try:
                build_c()
                lib = ctypes.CDLL(_SO)
            except Exception:          # no compiler: stay on numpy
                _lib = False
                return None
            lib.seeded_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_float, ctypes.c_int,
                                          ctypes.c_void_p]
            lib.seeded_normal.restype = None
            _lib = lib
    return _lib or None


def normal(seed: int, stream: int, count: int, std: float = 1.0, dtype: str = 'bf16',
           start: int = 0, use_c: bool = True) -> np.ndarray:
    """``count`` consecutive draws (from element ``start``) of N(0, std).

    dtype 'bf16' returns uint16 bit patterns, 'f32' float32 values.
    """
    std32 = float(np.float32(std))
    lib = _c() if use_c else None
    if lib is not None:
        out = np.empty(count, dtype=np.uint16 if dtype == 'bf16' else np.float32)
        lib.seeded_normal(seed & 0xFFFFFFFFFFFFFFFF, stream, start, count, std32,
                          1 if dtype == 'bf16' else 0, out.ctypes.data)
        return out
    out = np.empty(count, dtype=np.uint16 if dtype == 'bf16' else np.float32)
    step = 1 << 22
    for a in range(0, count, step):
        b = min(count, a + step)
        idx = np.arange(start + a, start + b, dtype=np.uint64)
        v = (normal_f64(seed, stream, idx) * std32).astype(np.float32)
        out[a:b] = f32_to_bf16_bits(v) if dtype == 'bf16' else v
    return out


def normal_at(seed: int, stream: int, index: np.ndarray, std: float = 1.0,
              dtype: str = 'bf16') -> np.ndarray:
    """Draws at arbitrary element indices (numpy path)."""
    std32 = float(np.float32(std))
    v = (normal_f64(seed, stream, np.asarray(index, dtype=np.uint64)) * std32).astype(np.float32)
    return f32_to_bf16_bits(v) if dtype == 'bf16' else v


def tokens(seed: int, count: int, vocab: int, stream: int = STREAM_TOKENS,
           start: int = 0) -> np.ndarray:
    """Token ids uniform in [0, vocab) (int32)."""
    d = draws(seed, stream, np.arange(start, start + count, dtype=np.uint64))
    with np.errstate(over='ignore'):
        return (((d >> _U64(32)) * _U64(vocab)) >> _U64(32)).astype(np.int32)


# Weight names in the checkpoint order printed on the pages.
LAYER_KEYS = ('attention.wq', 'attention.wk', 'attention.wv', 'attention.wo',
              'feed_forward.w1', 'feed_forward.w3', 'feed_forward.w2',
              'attention_norm', 'ffn_norm')


def weight_names(n_layers: int) -> list[str]:
    names = ['tok_embeddings.weight']
    for i in range(n_layers):
        names += [f'layers.{i}.{k}.weight' for k in LAYER_KEYS]
    return names + ['norm.weight', 'output.weight']


def weight_stream(name: str, n_layers: int) -> int:
    return weight_names(n_layers).index(name)


def weight_shape(name: str, dim: int, n_heads: int, n_kv_heads: int, ffn_hidden: int,
                 vocab: int) -> tuple[int, ...]:
    hd = dim // n_heads
    if name in ('tok_embeddings.weight', 'output.weight'):
        return (vocab, dim)
    if name == 'norm.weight' or name.endswith('_norm.weight'):
        return (dim,)
    leaf = name.split('.')[-2]
    return {'wq': (n_heads * hd, dim), 'wk': (n_kv_heads * hd, dim), 'wv': (n_kv_heads * hd, dim),
            'wo': (dim, n_heads * hd), 'w1': (ffn_hidden, dim), 'w3': (ffn_hidden, dim),
            'w2': (dim, ffn_hidden)}[leaf]


def weight(seed: int, name: str, shape: tuple[int, ...], n_layers: int, std: float,
           dtype: str = 'bf16') -> np.ndarray:
    """One weight tensor as generated by ``llama_init_weights`` (norms are 1.0)."""
    n = int(np.prod(shape))
    if name.endswith('norm.weight'):
        return np.ones(shape, dtype=np.float32)
    v = normal(seed, weight_stream(name, n_layers), n, std, dtype)
    return v.reshape(shape)
