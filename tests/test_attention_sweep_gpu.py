"""Causal GQA prefill attention at the sweep's large sizes (H = 32, Hk = 8,
d = 128), on sampled query rows.

The inputs are drawn on the device by the library's seeded generator (the
same definition as the host generator in seeded_inputs, bit for bit: see
test_device_generator_matches_host); the oracle takes the same draws from
the host generator, only for the rows it checks. Every query row is an
independent result, so checking sampled rows is exact for those rows: per
(sequence, head) 62 random rows plus rows 0 and S-1, every head, each row
within the rounding bound of the 16-bit kernel (tests.helpers.
attention_row_errors). The largest case holds more than 2**31 elements in q
and o, which exercises 64-bit offsets in the kernels.
"""
import numpy as np
import pytest

import seeded_inputs as si
from tests.helpers import BF16, F16, attention_row_errors, torch_dtype

pytestmark = pytest.mark.gpu

torch = pytest.importorskip('torch')
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip('needs a CUDA device', allow_module_level=True)

from llama_transformer_decoder_b200 import binding as L  # noqa: E402

H, HK, D = 32, 8, 128
SEED, SQ, SK, SV = 40, 1, 2, 3


def _device_normal(shape, stream, dtype):
    t = torch.empty(shape, dtype=torch_dtype(dtype), device='cuda')
    L.llama_fill_normal(t, t.numel(), SEED, stream, 1.0, dtype)
    return t


def _host_normal(stream, count, start, dtype):
    """The same draws as the device generator, as exact float64 values."""
    if dtype == BF16:
        return si.bf16_bits_to_f32(si.normal(SEED, stream, count, 1.0, 'bf16', start=start)).astype(np.float64)
    return si.normal(SEED, stream, count, 1.0, 'f32', start=start).astype(np.float16).astype(np.float64)


@pytest.mark.parametrize('dtype,B,S,check_b,n_rows', [
    (F16, 1, 8192, [0], 62),
    (F16, 1, 32768, [0], 62),
    (F16, 4, 32768, [0, 1, 2, 3], 62),
    (BF16, 16, 2048, list(range(16)), 62),
    (F16, 16, 32768, [0, 15], 14),            # q and o hold 2**31 elements
])
def test_attention_prefill_sampled_rows(dtype, B, S, check_b, n_rows):
    q = _device_normal((B, H, S, D), SQ, dtype)
    k = _device_normal((B, HK, S, D), SK, dtype)
    v = _device_normal((B, HK, S, D), SV, dtype)
    o = torch.empty((B, S, H * D), dtype=torch_dtype(dtype), device='cuda')
    L.llama_attention_prefill(q, k, v, o, B, S, H, HK, D, dtype)
    torch.cuda.synchronize()
    assert L.llama_status(None) == 0
    del q, k, v
    rng = np.random.RandomState(S + B)
    worst_all = 0.0
    for b in check_b:
        kb = _host_normal(SK, HK * S * D, b * HK * S * D, dtype).reshape(HK, S, D)
        vb = _host_normal(SV, HK * S * D, b * HK * S * D, dtype).reshape(HK, S, D)
        for h in range(H):
            rows = np.unique(np.r_[0, rng.choice(S, n_rows, replace=False), S - 1])
            qh = np.stack([_host_normal(SQ, D, ((b * H + h) * S + r) * D, dtype) for r in rows])[None]
            g = h // (H // HK)
            got = o[b, torch.from_numpy(rows).cuda(), h * D:(h + 1) * D].float().cpu().numpy()
            worst, err = attention_row_errors(got, qh, kb[g:g + 1], vb[g:g + 1], rows, dtype)
            worst_all = max(worst_all, worst)
            assert worst <= 1.0, (b, h, worst)
            assert err < (1e-2 if dtype == BF16 else 2e-3), (b, h, err)
    print(f'B={B} S={S}: worst row error / rounding bound = {worst_all:.3f}')
