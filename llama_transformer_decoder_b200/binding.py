"""ctypes binding of libllama_b200.so: argument marshalling only.

Every function has the name of the C entry point it calls. Tensor arguments
may be torch tensors (their data_ptr() is passed) or raw integer addresses;
streams may be torch.cuda.Stream objects, raw cudaStream_t integers or None
(the legacy default stream). A non-zero status raises LlamaError. There is no
other code path: if the library is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, 'libllama_b200.so')

LLAMA_OK = 0
LLAMA_ERR_INVALID_ARG = -1
LLAMA_ERR_SHAPE = -2
LLAMA_ERR_OOM = -3
LLAMA_ERR_CUDA = -4
LLAMA_ERR_DEVICE_TIMEOUT = -5
LLAMA_ERR_DEVICE_BOUNDS = -6
LLAMA_ERR_UNSUPPORTED = -7
LLAMA_ERR_RANGE = -8
LLAMA_F32 = 0
LLAMA_BF16 = 1
LLAMA_F16 = 2


class LlamaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f'{where}: {status_string(status)} ({status})')


class llama_config(ctypes.Structure):
    _fields_ = [('dim', ctypes.c_int32), ('n_layers', ctypes.c_int32), ('n_heads', ctypes.c_int32),
                ('n_kv_heads', ctypes.c_int32), ('vocab_size', ctypes.c_int32), ('ffn_hidden', ctypes.c_int32),
                ('multiple_of', ctypes.c_int32), ('ffn_dim_multiplier', ctypes.c_float),
                ('norm_eps', ctypes.c_float), ('rope_theta', ctypes.c_float), ('max_batch', ctypes.c_int32),
                ('max_seq', ctypes.c_int32), ('max_tokens', ctypes.c_int32), ('dtype', ctypes.c_int32),
                ('kv_page_size', ctypes.c_int32), ('kv_pages', ctypes.c_int32), ('act_dtype', ctypes.c_int32)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f'{LIB_PATH} is missing: build it with python -m llama_transformer_decoder_b200.build')
_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_U64 = ctypes.c_uint64
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_SIGS = {
    'llama_ffn_hidden': (_I32, [_I32, _I32, _F]),
    'llama_create': (ctypes.c_int, [ctypes.POINTER(llama_config), ctypes.POINTER(_P)]),
    'llama_destroy': (None, [_P]),
    'llama_get_config': (ctypes.c_int, [_P, ctypes.POINTER(llama_config)]),
    'llama_device_bytes': (_SZ, [_P]),
    'llama_init_weights': (ctypes.c_int, [_P, _U64, _F, _P]),
    'llama_set_weight': (ctypes.c_int, [_P, ctypes.c_char_p, _P, _SZ, ctypes.c_int, _P]),
    'llama_get_weight': (ctypes.c_int, [_P, ctypes.c_char_p, _P, _SZ, ctypes.c_int, _P]),
    'llama_prefill': (ctypes.c_int, [_P, _P, _I32, _I32, _P]),
    'llama_decode_step': (ctypes.c_int, [_P, _P, _I32, _P]),
    'llama_logits': (ctypes.c_int, [_P, _P, _P]),
    'llama_argmax': (ctypes.c_int, [_P, _P, _P]),
    'llama_generate': (ctypes.c_int, [_P, _P, _I32, _I32, _I32, _P, _P]),
    'llama_block_forward': (ctypes.c_int, [_P, _I32, _P, _P, _I32, _I32, _P]),
    'llama_fill_kv_random': (ctypes.c_int, [_P, _U64, _I32, _P]),
    'llama_set_kv': (ctypes.c_int, [_P, _I32, _P, _P, _I32, _I32, _P]),
    'llama_set_lengths': (ctypes.c_int, [_P, _P, _I32, _P]),
    'llama_get_lengths': (ctypes.c_int, [_P, _P, _I32]),
    'llama_get_block_table': (ctypes.c_int, [_P, _P, _I32]),
    'llama_reset': (ctypes.c_int, [_P, _P]),
    'llama_sync_status': (ctypes.c_int, [_P, _P]),
    'llama_status_string': (ctypes.c_char_p, [ctypes.c_int]),
    'llama_attention_prefill': (ctypes.c_int, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P]),
    'llama_attention_decode': (ctypes.c_int, [_P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P]),
    'llama_attention_decode_noalloc': (ctypes.c_int, [_P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32,
                                                      _P]),
    'llama_attention_prefill_paged': (ctypes.c_int, [_P, _P, _P, _P, _I32, _I32, _P, _P, _I32, _I32, _I32, _I32,
                                                     _I32, _I32, _P]),
    'llama_attention_decode_paged': (ctypes.c_int, [_P, _P, _P, _P, _I32, _I32, _P, _P, _I32, _I32, _I32, _I32,
                                                    _I32, _P]),
    'llama_linear': (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P]),
    'llama_rmsnorm': (ctypes.c_int, [_P, _P, _P, _I32, _I32, _F, _I32, _P]),
    'llama_argmax_rows': (ctypes.c_int, [_P, _P, _I32, _I32, _P]),
    'llama_fill_normal': (ctypes.c_int, [_P, _I64, _U64, _U64, _F, _I32, _P]),
    'llama_status': (ctypes.c_int, [_P]),
    'llama_wait_selftest': (ctypes.c_int, [_I32, _U64, _P]),
    'llama_profile': (ctypes.c_int, [_P, ctypes.c_int]),
    'llama_profile_read': (ctypes.c_int, [_P, _P, _P, ctypes.c_int]),
    'llama_profile_kind_name': (ctypes.c_char_p, [ctypes.c_int]),
    'llama_kernel_launches': (_U64, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def exported_symbols() -> list[str]:
    return list(_SIGS)


def status_string(status: int) -> str:
    return _lib.llama_status_string(status).decode()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, 'data_ptr'):
        return x.data_ptr()
    if hasattr(x, 'ctypes'):           # numpy array (host memory)
        return x.ctypes.data
    raise TypeError(f'cannot pass {type(x)} as a pointer')


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != LLAMA_OK:
        raise LlamaError(rc, where)


def llama_ffn_hidden(dim, multiple_of, ffn_dim_multiplier):
    return _lib.llama_ffn_hidden(dim, multiple_of, ffn_dim_multiplier)


def llama_create(cfg: llama_config) -> int:
    h = _P()
    _check(_lib.llama_create(ctypes.byref(cfg), ctypes.byref(h)), 'llama_create')
    return h.value


def llama_destroy(model) -> None:
    _lib.llama_destroy(model)


def llama_get_config(model) -> llama_config:
    c = llama_config()
    _check(_lib.llama_get_config(model, ctypes.byref(c)), 'llama_get_config')
    return c


def llama_device_bytes(model) -> int:
    return _lib.llama_device_bytes(model)


def llama_init_weights(model, seed, std, stream=None):
    _check(_lib.llama_init_weights(model, seed, std, _stream(stream)), 'llama_init_weights')


def llama_set_weight(model, name, src, nbytes, on_device, stream=None):
    _check(_lib.llama_set_weight(model, name.encode(), _ptr(src), nbytes, on_device, _stream(stream)),
           'llama_set_weight')


def llama_get_weight(model, name, dst, nbytes, on_device, stream=None):
    _check(_lib.llama_get_weight(model, name.encode(), _ptr(dst), nbytes, on_device, _stream(stream)),
           'llama_get_weight')


def llama_prefill(model, tokens, B, S, stream=None):
    _check(_lib.llama_prefill(model, _ptr(tokens), B, S, _stream(stream)), 'llama_prefill')


def llama_decode_step(model, tokens, B, stream=None):
    _check(_lib.llama_decode_step(model, _ptr(tokens), B, _stream(stream)), 'llama_decode_step')


def llama_logits(model, dst, stream=None):
    _check(_lib.llama_logits(model, _ptr(dst), _stream(stream)), 'llama_logits')


def llama_argmax(model, dst, stream=None):
    _check(_lib.llama_argmax(model, _ptr(dst), _stream(stream)), 'llama_argmax')


def llama_generate(model, host_tokens, B, S, n_new, host_out, stream=None):
    _check(_lib.llama_generate(model, _ptr(host_tokens), B, S, n_new, _ptr(host_out), _stream(stream)),
           'llama_generate')


def llama_block_forward(model, layer, x, y, B, S, stream=None):
    _check(_lib.llama_block_forward(model, layer, _ptr(x), _ptr(y), B, S, _stream(stream)), 'llama_block_forward')


def llama_fill_kv_random(model, seed, c, stream=None):
    _check(_lib.llama_fill_kv_random(model, seed, c, _stream(stream)), 'llama_fill_kv_random')


def llama_set_kv(model, layer, k, v, B, c, stream=None):
    _check(_lib.llama_set_kv(model, layer, _ptr(k), _ptr(v), B, c, _stream(stream)), 'llama_set_kv')


def llama_set_lengths(model, host_len, B, stream=None):
    _check(_lib.llama_set_lengths(model, _ptr(host_len), B, _stream(stream)), 'llama_set_lengths')


def llama_get_lengths(model, host_len, B):
    _check(_lib.llama_get_lengths(model, _ptr(host_len), B), 'llama_get_lengths')


def llama_get_block_table(model, host_table, B):
    _check(_lib.llama_get_block_table(model, _ptr(host_table), B), 'llama_get_block_table')


def llama_reset(model, stream=None):
    _check(_lib.llama_reset(model, _stream(stream)), 'llama_reset')


def llama_sync_status(model, stream=None) -> int:
    return _lib.llama_sync_status(model, _stream(stream))


def llama_attention_prefill(q, k, v, o, B, S, H, Hk, d, dtype, stream=None):
    _check(_lib.llama_attention_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, S, H, Hk, d, dtype, _stream(stream)),
           'llama_attention_prefill')


def llama_attention_decode(q, kc, vc, length, o, B, cmax, H, Hk, d, dtype, stream=None):
    _check(_lib.llama_attention_decode(_ptr(q), _ptr(kc), _ptr(vc), _ptr(length), _ptr(o), B, cmax, H, Hk, d, dtype,
                                       _stream(stream)), 'llama_attention_decode')


def llama_attention_prefill_paged(q, k_pages, v_pages, table, max_pages, n_pages, pos0, o, B, S, H, Hk, d, dtype,
                                  stream=None):
    _check(_lib.llama_attention_prefill_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(table), max_pages, n_pages,
                                              _ptr(pos0) if pos0 is not None else None, _ptr(o), B, S, H, Hk, d,
                                              dtype, _stream(stream)), 'llama_attention_prefill_paged')


def llama_attention_decode_paged(q, k_pages, v_pages, table, max_pages, n_pages, length, o, B, H, Hk, d, dtype,
                                 stream=None):
    _check(_lib.llama_attention_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(table), max_pages, n_pages,
                                             _ptr(length), _ptr(o), B, H, Hk, d, dtype, _stream(stream)),
           'llama_attention_decode_paged')


def llama_attention_decode_noalloc(q, kc, vc, length, o, B, cmax, H, Hk, d, dtype, stream=None):
    _check(_lib.llama_attention_decode_noalloc(_ptr(q), _ptr(kc), _ptr(vc), _ptr(length), _ptr(o), B, cmax, H, Hk,
                                               d, dtype, _stream(stream)), 'llama_attention_decode_noalloc')


def llama_linear(x, w, y, M, N, K, dtype, variant=0, stream=None):
    _check(_lib.llama_linear(_ptr(x), _ptr(w), _ptr(y), M, N, K, dtype, variant, _stream(stream)), 'llama_linear')


def llama_rmsnorm(x, g, y, M, D, eps, dtype, stream=None):
    _check(_lib.llama_rmsnorm(_ptr(x), _ptr(g), _ptr(y), M, D, eps, dtype, _stream(stream)), 'llama_rmsnorm')


def llama_argmax_rows(logits, out, B, V, stream=None):
    _check(_lib.llama_argmax_rows(_ptr(logits), _ptr(out), B, V, _stream(stream)), 'llama_argmax_rows')


def llama_fill_normal(dst, n, seed, stream_id, std, dtype, stream=None):
    _check(_lib.llama_fill_normal(_ptr(dst), n, seed, stream_id, std, dtype, _stream(stream)), 'llama_fill_normal')


def llama_status(stream=None) -> int:
    return _lib.llama_status(_stream(stream))


def llama_wait_selftest(kind, limit_ns, stream=None):
    _check(_lib.llama_wait_selftest(int(kind), int(limit_ns), _stream(stream)), 'llama_wait_selftest')


def llama_status_string(status: int) -> str:
    return status_string(status)


def llama_profile(model, enable):
    _check(_lib.llama_profile(model, int(enable)), 'llama_profile')


def llama_profile_read(model, n_kinds=16):
    """{kind name: (milliseconds, launches)} of the profiled launches since the last read."""
    ms = (ctypes.c_double * n_kinds)()
    ln = (ctypes.c_int64 * n_kinds)()
    n = _lib.llama_profile_read(model, ctypes.addressof(ms), ctypes.addressof(ln), n_kinds)
    if n < 0:
        raise LlamaError(n, 'llama_profile_read')
    return {llama_profile_kind_name(k): (ms[k], ln[k]) for k in range(n)}


def llama_profile_kind_name(kind):
    return _lib.llama_profile_kind_name(kind).decode()


def llama_kernel_launches():
    return _lib.llama_kernel_launches()
