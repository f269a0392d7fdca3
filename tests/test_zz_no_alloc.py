"""The decode-attention entry point that allocates no device memory.

Callers whose device memory is owned by their own allocator or pool, or who
cannot afford the device-wide synchronisation of cudaMalloc/cudaFree in a
hot loop, use llama_attention_decode_noalloc; it keeps its split partials in
a static device array. Here it must reproduce the allocating entry point,
within the bf16 tolerance of the decode tests, on two calls in a row (the
second call reuses the array the first one left behind). This file sorts last
so that it also runs after every other GPU test.
"""
import numpy as np
import pytest

from tests.helpers import BF16, normal_values, rel_l2, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip('torch')
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip('needs a CUDA device', allow_module_level=True)

from llama_transformer_decoder_b200 import binding as L  # noqa: E402


def _inputs(seed, B, H, Hk, d, cmax):
    _, qr = normal_values(seed, 1, (B, H, d), BF16)
    _, kr = normal_values(seed, 2, (B, Hk, cmax, d), BF16)
    _, vr = normal_values(seed, 3, (B, Hk, cmax, d), BF16)
    return to_device(qr, BF16), to_device(kr, BF16), to_device(vr, BF16)


def test_noalloc_decode_matches_allocating_entry_point():
    B, H, Hk, d, cmax = 4, 32, 8, 128, 4096
    for seed, lens in [(21, [1, 700, 4096, 2048]), (22, [4096, 3, 1500, 999])]:
        q, k, v = _inputs(seed, B, H, Hk, d, cmax)
        ln = torch.tensor(lens, dtype=torch.int32, device='cuda')
        ref = torch.empty((B, H * d), dtype=torch.bfloat16, device='cuda')
        got = torch.full((B, H * d), float('nan'), dtype=torch.bfloat16, device='cuda')
        L.llama_attention_decode(q, k, v, ln, ref, B, cmax, H, Hk, d, BF16)
        L.llama_attention_decode_noalloc(q, k, v, ln, got, B, cmax, H, Hk, d, BF16)
        torch.cuda.synchronize()
        a, b = got.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.all(np.isfinite(a))
        assert rel_l2(a, b) < 1e-2


def test_noalloc_decode_rejects_sizes_beyond_its_array():
    B, H, Hk, d, cmax = 256, 32, 8, 128, 64        # (256*8 + 4*148)*4*(128+2)*4 B > 4 MiB of partials
    q = torch.zeros((B, H, d), dtype=torch.bfloat16, device='cuda')
    k = torch.zeros((B, Hk, cmax, d), dtype=torch.bfloat16, device='cuda')
    ln = torch.ones(B, dtype=torch.int32, device='cuda')
    o = torch.empty((B, H * d), dtype=torch.bfloat16, device='cuda')
    with pytest.raises(L.LlamaError) as e:
        L.llama_attention_decode_noalloc(q, k, k, ln, o, B, cmax, H, Hk, d, BF16)
    assert e.value.status == L.LLAMA_ERR_SHAPE
