"""The decode-attention entry point that allocates no device memory.

Callers whose device memory is owned by their own allocator or pool, or who
cannot afford the device-wide synchronisation of cudaMalloc/cudaFree in a
hot loop, use llama_attention_decode_noalloc; it keeps its split partials in
a static device array. It runs the same kernels on the same inputs as the
allocating entry point, so its outputs must be bit-identical to that one's,
on two calls in a row (the second call reuses the array the first one left
behind), for every kernel family behind the call: the 16-bit head_dim-128
kernel, whose partials are sized by the SM count, and the split kernel
(fp32, and 16-bit with head_dim 64), whose partials are sized by the number
of key splits. This file sorts last so that it also runs after every other
GPU test.
"""
import numpy as np
import pytest

from tests.helpers import BF16, F16, F32, normal_values, to_device, torch_dtype

pytestmark = pytest.mark.gpu

torch = pytest.importorskip('torch')
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip('needs a CUDA device', allow_module_level=True)

from llama_transformer_decoder_b200 import binding as L  # noqa: E402


def _inputs(seed, B, H, Hk, d, cmax, dtype):
    _, qr = normal_values(seed, 1, (B, H, d), dtype)
    _, kr = normal_values(seed, 2, (B, Hk, cmax, d), dtype)
    _, vr = normal_values(seed, 3, (B, Hk, cmax, d), dtype)
    return to_device(qr, dtype), to_device(kr, dtype), to_device(vr, dtype)


CASES = [  # dtype, B, H, Hk, d, cmax, two sets of lengths (one per call)
    (BF16, 4, 32, 8, 128, 4096, [1, 700, 4096, 2048], [4096, 3, 1500, 999]),
    (F16, 8, 32, 8, 128, 65536, [65536, 60000, 65000, 40000, 65536, 50000, 1, 65535],   # claimed sub-chunks,
     [4096, 8000, 7000, 1, 8192, 8100, 7500, 6000]),                                     # then none
    (F16, 3, 8, 2, 64, 1000, [1000, 1, 517], [2, 999, 640]),
    (F32, 2, 8, 2, 32, 1000, [1000, 333], [17, 1000]),
    (F32, 2, 4, 4, 64, 900, [900, 1], [450, 899]),
]


@pytest.mark.parametrize('dtype,B,H,Hk,d,cmax,lens_a,lens_b', CASES)
def test_noalloc_decode_matches_allocating_entry_point(dtype, B, H, Hk, d, cmax, lens_a, lens_b):
    tdt = torch_dtype(dtype)
    for seed, lens in [(21, lens_a), (22, lens_b)]:
        q, k, v = _inputs(seed, B, H, Hk, d, cmax, dtype)
        ln = torch.tensor(lens, dtype=torch.int32, device='cuda')
        ref = torch.empty((B, H * d), dtype=tdt, device='cuda')
        got = torch.full((B, H * d), float('nan'), dtype=tdt, device='cuda')
        L.llama_attention_decode(q, k, v, ln, ref, B, cmax, H, Hk, d, dtype)
        L.llama_attention_decode_noalloc(q, k, v, ln, got, B, cmax, H, Hk, d, dtype)
        assert L.llama_status(None) == 0
        a, b = got.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.all(np.isfinite(a))
        assert np.array_equal(a, b), float(np.max(np.abs(a - b)))


@pytest.mark.parametrize('dtype,d', [(BF16, 128), (F32, 64)])
def test_noalloc_decode_reports_lengths_outside_the_cache(dtype, d):
    """A length above cmax (or below 1) gives a NaN row for that sequence only
    and latches LLAMA_ERR_DEVICE_BOUNDS in the call's own status word, which
    llama_status reads and clears; the other sequences are unaffected."""
    B, H, Hk, cmax = 3, 8, 2, 512
    q, k, v = _inputs(23, B, H, Hk, d, cmax, dtype)
    tdt = torch_dtype(dtype)
    good = torch.tensor([512, 100, 7], dtype=torch.int32, device='cuda')
    ref = torch.empty((B, H * d), dtype=tdt, device='cuda')
    L.llama_attention_decode_noalloc(q, k, v, good, ref, B, cmax, H, Hk, d, dtype)
    assert L.llama_status(None) == 0
    for bad_len in (cmax + 1, 0):
        bad = torch.tensor([512, bad_len, 7], dtype=torch.int32, device='cuda')
        got = torch.empty((B, H * d), dtype=tdt, device='cuda')
        L.llama_attention_decode_noalloc(q, k, v, bad, got, B, cmax, H, Hk, d, dtype)
        assert L.llama_status(None) == L.LLAMA_ERR_DEVICE_BOUNDS
        assert L.llama_status(None) == 0                 # cleared by the read
        g = got.float().cpu().numpy()
        assert np.all(np.isnan(g[1]))
        r = ref.float().cpu().numpy()
        assert np.array_equal(g[[0, 2]], r[[0, 2]])


def test_noalloc_decode_rejects_sizes_beyond_its_array():
    B, H, Hk, d, cmax = 512, 32, 8, 128, 64        # (512*8 + 4*148)*4*(128+2)*4 B > 8 MiB of partials
    q = torch.zeros((B, H, d), dtype=torch.bfloat16, device='cuda')
    k = torch.zeros((B, Hk, cmax, d), dtype=torch.bfloat16, device='cuda')
    ln = torch.ones(B, dtype=torch.int32, device='cuda')
    o = torch.empty((B, H * d), dtype=torch.bfloat16, device='cuda')
    with pytest.raises(L.LlamaError) as e:
        L.llama_attention_decode_noalloc(q, k, k, ln, o, B, cmax, H, Hk, d, BF16)
    assert e.value.status == L.LLAMA_ERR_SHAPE
