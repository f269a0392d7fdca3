"""Kernel parity on the GPU through the C ABI: generator, GEMMs (wide and
skinny tcgen05 paths, fp32 SIMT), RMSNorm, argmax, prefill and decode
attention, each against the CPU oracle on the same seeded inputs."""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import argmax, attention, rms_norm
from tests.helpers import BF16, F16, F32, attention_row_errors, normal_values, rel_l2, to_device, torch_dtype

pytestmark = pytest.mark.gpu

torch = pytest.importorskip('torch')
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip('needs a CUDA device', allow_module_level=True)

from llama_transformer_decoder_b200 import binding as L  # noqa: E402


def _sync_ok():
    assert L.llama_status(None) == 0


# ----------------------------------------------------------- generator
@pytest.mark.parametrize('dtype', [BF16, F16, F32])
def test_device_generator_matches_host(dtype):
    n = 3_000_017
    for seed, stream, std in [(0, 1, 0.02), (7, 123456, 1.0), (1, 2 ** 21 + 5, 1.0)]:
        t = torch.empty(n, dtype=torch_dtype(dtype), device='cuda')
        L.llama_fill_normal(t, n, seed, stream, std, dtype)
        torch.cuda.synchronize()
        if dtype == BF16:
            host = si.normal(seed, stream, n, std, 'bf16')
        elif dtype == F16:
            host = si.normal(seed, stream, n, std, 'f32').astype(np.float16).view(np.uint16)
        else:
            host = si.normal(seed, stream, n, std, 'f32').view(np.uint32)
        dev = t.view(torch.int16 if dtype != F32 else torch.int32).cpu().numpy()
        assert np.array_equal(dev.view(host.dtype), host)
    _sync_ok()


# -------------------------------------------------------------- GEMMs
GEMM_CASES = [
    # (M, N, K, variant)  variant 1 = wide persistent, 2 = skinny split-K
    (300, 520, 4104, 1),     # ragged M, N and K tails
    (128, 256, 64, 1),       # exactly one tile, one k-block
    (2048, 6144, 4096, 1),   # 8B QKV projection at S = 2048
    (17, 6144, 4096, 2),     # seq-17 block
    (32, 4096, 14336, 2),    # decode w2 (long K, split)
    (1, 1000, 4096, 2),      # one row, ragged N
    (200, 520, 4104, 2),     # ragged everything, NT = 256
    (100, 384, 256, 2),      # short K (one split)
    (64, 1024, 1024, 1),     # wide path with few rows
    (2100, 6000, 4104, 1),   # CTA-pair path with ragged M, N and K
    (4096, 4096, 1024, 1),   # CTA-pair path, several tiles per pair
]


@pytest.mark.parametrize('dtype', [BF16, F16])
@pytest.mark.parametrize('M,N,K,variant', GEMM_CASES)
def test_linear_16bit(M, N, K, variant, dtype):
    xv, xr = normal_values(11, 1, (M, K), dtype)
    wv, wr = normal_values(11, 2, (N, K), dtype, std=0.02)
    y = torch.full((M, N), float('nan'), device='cuda')
    L.llama_linear(to_device(xr, dtype), to_device(wr, dtype), y, M, N, K, dtype, variant)
    torch.cuda.synchronize()
    _sync_ok()
    ref = xv.astype(np.float64) @ wv.astype(np.float64).T
    got = y.cpu().numpy()
    assert np.all(np.isfinite(got))
    assert rel_l2(got, ref) < 1e-5
    # fp32 accumulation of exact 16-bit products: per element |err| << 1e-3 * |row scale|
    scale = np.sqrt((xv.astype(np.float64) ** 2).sum(1, keepdims=True) * (wv.astype(np.float64) ** 2).sum(1)[None, :])
    assert np.max(np.abs(got - ref) / scale) < 1e-5


@pytest.mark.parametrize('M,N,K,variant', [(32, 4096, 14336, 2), (2048, 4096, 4096, 1), (300, 520, 4104, 1)])
def test_linear_repeatable(M, N, K, variant):
    """Split tiles (skinny split-K, wide stream-K tail) are reduced in a fixed
    order: repeated calls agree bit for bit."""
    _, xr = normal_values(12, 1, (M, K), BF16)
    _, wr = normal_values(12, 2, (N, K), BF16, std=0.02)
    x, w = to_device(xr, BF16), to_device(wr, BF16)
    outs = []
    for _ in range(3):
        y = torch.empty((M, N), device='cuda')
        L.llama_linear(x, w, y, M, N, K, BF16, variant)
        outs.append(y.cpu())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


@pytest.mark.parametrize('M,N,K', [(17, 768, 256), (70, 130, 33), (1, 1024, 256)])
def test_linear_f32(M, N, K):
    xv, xr = normal_values(13, 1, (M, K), F32)
    wv, wr = normal_values(13, 2, (N, K), F32, std=0.02)
    y = torch.empty((M, N), device='cuda')
    L.llama_linear(to_device(xr, F32), to_device(wr, F32), y, M, N, K, F32, 0)
    ref = xv.astype(np.float64) @ wv.astype(np.float64).T
    assert rel_l2(y.cpu().numpy(), ref) < 1e-6
    _sync_ok()


# ------------------------------------------------------------ RMSNorm
@pytest.mark.parametrize('dtype', [BF16, F16, F32])
@pytest.mark.parametrize('M,D', [(1, 4096), (37, 4096), (2048, 4096), (5, 256), (3, 100), (2, 12288), (3, 8192)])
def test_rmsnorm(dtype, M, D):
    xv, xr = normal_values(14, 1, (M, D), F32)
    g = np.linspace(0.5, 1.5, D).astype(np.float32)
    y = torch.empty((M, D), dtype=torch_dtype(dtype), device='cuda')
    L.llama_rmsnorm(to_device(xr, F32), torch.from_numpy(g).cuda(), y, M, D, 1e-5, dtype)
    ref = rms_norm(xv.astype(np.float64), g.astype(np.float64), 1e-5)
    got = y.float().cpu().numpy()
    assert rel_l2(got, ref) < {BF16: 4e-3, F16: 5e-4, F32: 1e-6}[dtype]
    _sync_ok()


# ------------------------------------------------------------- argmax
def test_argmax_rows_exact_with_ties():
    B, V = 5, 128256
    lv, lr = normal_values(15, 3, (B, V), F32)
    lv = lv.copy()
    lv[1, 77] = lv[1, 1000] = lv[1].max() + 1.0        # tie: lowest index wins
    lv[2, :] = 0.5                                     # all equal -> 0
    lv[3, V - 1] = 100.0                               # last element
    out = torch.empty(B, dtype=torch.int32, device='cuda')
    L.llama_argmax_rows(torch.from_numpy(lv).cuda(), out, B, V)
    assert list(out.cpu().numpy()) == list(argmax(lv))
    assert list(out.cpu().numpy())[1:4] == [77, 0, V - 1]


# ----------------------------------------------------- prefill attention
# Even query heads per KV head run the two-heads-per-item kernel at every
# length; otherwise up to 4096 queries run the one-head persistent kernel and
# longer chunks the per-tile kernel (the group-1 and group-3 cases below).
PREFILL_CASES = [(BF16, 2, 200, 8, 2), (BF16, 1, 1, 4, 1), (BF16, 1, 64, 4, 4), (BF16, 1, 65, 8, 2),
                 (BF16, 1, 2048, 32, 8), (BF16, 2, 300, 32, 8), (BF16, 1, 4097, 8, 2), (BF16, 3, 129, 4, 1),
                 (F16, 2, 200, 8, 2), (F16, 1, 1, 4, 1), (F16, 1, 2048, 32, 8), (F16, 1, 4097, 8, 2),
                 (F16, 3, 129, 4, 1), (F16, 2, 300, 6, 2), (BF16, 1, 4200, 6, 2), (F16, 1, 4097, 3, 3),
                 (BF16, 1, 1000, 2, 2)]


@pytest.mark.parametrize('dtype,B,S,H,Hk', PREFILL_CASES)
def test_attention_prefill_16bit(dtype, B, S, H, Hk):
    d = 128
    qv, qr = normal_values(16, 1, (B, H, S, d), dtype)
    kv, kr = normal_values(16, 2, (B, Hk, S, d), dtype)
    vv, vr = normal_values(16, 3, (B, Hk, S, d), dtype)
    o = torch.empty((B, S, H * d), dtype=torch_dtype(dtype), device='cuda')
    L.llama_attention_prefill(to_device(qr, dtype), to_device(kr, dtype), to_device(vr, dtype), o, B, S, H, Hk, d,
                              dtype)
    torch.cuda.synchronize()
    _sync_ok()
    got = o.float().cpu().numpy()
    rows = np.arange(S) if S <= 512 else np.unique(np.r_[np.arange(0, S, 37), S - 1])
    for b in range(B):
        worst, err = attention_row_errors(got[b][rows], qv[b][:, rows].astype(np.float64), kv[b].astype(np.float64),
                                          vv[b].astype(np.float64), rows, dtype)
        assert worst <= 1.0, (b, worst)                   # every head and row within its rounding bound
        assert err < (1e-2 if dtype == BF16 else 2e-3)


@pytest.mark.parametrize('d', [32, 128])
def test_attention_prefill_f32(d):
    B, S, H, Hk = 2, 17, 8, 2
    qv, qr = normal_values(17, 1, (B, H, S, d), F32)
    kv, kr = normal_values(17, 2, (B, Hk, S, d), F32)
    vv, vr = normal_values(17, 3, (B, Hk, S, d), F32)
    o = torch.empty((B, S, H * d), device='cuda')
    L.llama_attention_prefill(to_device(qr, F32), to_device(kr, F32), to_device(vr, F32), o, B, S, H, Hk, d, F32)
    got = o.cpu().numpy()
    for b in range(B):
        worst, err = attention_row_errors(got[b], qv[b].astype(np.float64), kv[b].astype(np.float64),
                                          vv[b].astype(np.float64), np.arange(S), F32)
        assert worst <= 1.0, (b, worst)
        assert err < 1e-5
    _sync_ok()


# ------------------------------------------------------ decode attention
@pytest.mark.parametrize('dtype,d,B,H,Hk,cmax,lens', [
    (BF16, 128, 3, 32, 8, 1000, [1, 517, 1000]),
    (BF16, 128, 2, 8, 8, 4097, [4097, 130]),
    (BF16, 128, 2, 16, 2, 300, [300, 45]),                   # 8 query heads per kv head
    (BF16, 128, 32, 32, 8, 4224, [4097 + 4 * i for i in range(32)]),   # batch-32 decode shape
    (BF16, 128, 24, 32, 8, 8192, [1 + 341 * i for i in range(24)]),      # ragged lengths, 1 to 7844
    (BF16, 128, 1, 32, 8, 131072, [131072]),                 # longest cache of the sweep
    (BF16, 128, 64, 32, 8, 1024, [1 + 16 * i for i in range(64)]),
    (F16, 128, 1, 8, 1, 65536, [65536]),                   # one kv head: every decoding warp holds a piece of it
    (BF16, 128, 4, 32, 8, 2048, [2048, 1, 1500, 777]),       # ~20 pieces per head: two combine warps per head
    (F16, 128, 13, 12, 6, 700, [1 + 53 * i for i in range(13)]),   # 156 heads: a partial last combine block
    (F16, 128, 32, 32, 8, 16384, [16384 - 97 * i for i in range(32)]),   # claimed sub-chunks (>= 128 tiles per warp)
    (BF16, 128, 160, 8, 2, 8192, [8192 - 7 * i for i in range(160)]),   # claimed sub-chunks, B over the seek table
    (BF16, 64, 2, 8, 2, 300, [17, 300]),
    (F16, 128, 3, 32, 8, 1000, [1, 517, 1000]),
    (F16, 128, 32, 32, 8, 4224, [4097 + 4 * i for i in range(32)]),
    (F16, 128, 2, 16, 2, 300, [300, 45]),
    (F16, 64, 2, 8, 2, 300, [17, 300]),
    (F32, 32, 2, 8, 2, 300, [17, 300]),
    (F32, 128, 1, 4, 1, 64, [64]),
])
def test_attention_decode(dtype, d, B, H, Hk, cmax, lens):
    qv, qr = normal_values(18, 1, (B, H, d), dtype)
    kv, kr = normal_values(18, 2, (B, Hk, cmax, d), dtype)
    vv, vr = normal_values(18, 3, (B, Hk, cmax, d), dtype)
    ln = torch.tensor(lens, dtype=torch.int32, device='cuda')
    o = torch.empty((B, H * d), dtype=torch_dtype(dtype), device='cuda')
    L.llama_attention_decode(to_device(qr, dtype), to_device(kr, dtype), to_device(vr, dtype), ln, o, B, cmax, H, Hk,
                             d, dtype)
    torch.cuda.synchronize()
    _sync_ok()
    got = o.float().cpu().numpy()
    for b in (range(B) if B <= 32 else [0, 1, B // 2, B - 1]):
        n = lens[b]
        worst, err = attention_row_errors(got[b][None], qv[b][:, None, :].astype(np.float64),
                                          kv[b][:, :n].astype(np.float64), vv[b][:, :n].astype(np.float64),
                                          np.array([n - 1]), dtype)
        assert worst <= 1.0, (b, worst)                   # every head within its rounding bound
        assert err < {BF16: 1e-2, F16: 2e-3, F32: 1e-5}[dtype]


@pytest.mark.parametrize('B', [1, 5])
def test_attention_decode_bad_lengths_give_nan_rows(B):
    """A length outside [1, cmax] gives a NaN row for that sequence, latches
    LLAMA_ERR_DEVICE_BOUNDS, and leaves the other sequences' rows correct."""
    H, Hk, d, cmax = 32, 8, 128, 640
    lens = [0, 300, 641, 640, 17][:B] if B > 1 else [641]
    qv, qr = normal_values(19, 1, (B, H, d), BF16)
    kv, kr = normal_values(19, 2, (B, Hk, cmax, d), BF16)
    vv, vr = normal_values(19, 3, (B, Hk, cmax, d), BF16)
    o = torch.zeros((B, H * d), dtype=torch.bfloat16, device='cuda')
    L.llama_attention_decode(to_device(qr, BF16), to_device(kr, BF16), to_device(vr, BF16),
                             torch.tensor(lens, dtype=torch.int32, device='cuda'), o, B, cmax, H, Hk, d, BF16)
    assert L.llama_status(None) == L.LLAMA_ERR_DEVICE_BOUNDS
    assert L.llama_status(None) == 0                  # cleared
    got = o.float().cpu().numpy()
    for b, n in enumerate(lens):
        if not 1 <= n <= cmax:
            assert np.isnan(got[b]).all(), b
            continue
        worst, err = attention_row_errors(got[b][None], qv[b][:, None, :].astype(np.float64),
                                          kv[b][:, :n].astype(np.float64), vv[b][:, :n].astype(np.float64),
                                          np.array([n - 1]), BF16)
        assert worst <= 1.0, (b, worst)
        assert err < 1e-2


def test_attention_decode_few_tiles_after_many():
    """Fewer 32-key tiles than decoding warps, run right after a large call
    that filled the library's partial buffers: only the warps that own tiles
    may contribute to the merge."""
    big = dict(B=32, H=32, Hk=8, cmax=4224, lens=[4097 + 4 * i for i in range(32)])
    small = dict(B=2, H=4, Hk=2, cmax=256, lens=[101, 101])
    outs = []
    for i, c in enumerate((big, small)):
        B, H, Hk, cmax, lens = c['B'], c['H'], c['Hk'], c['cmax'], c['lens']
        qv, qr = normal_values(30 + i, 1, (B, H, 128), BF16)
        kv, kr = normal_values(30 + i, 2, (B, Hk, cmax, 128), BF16)
        vv, vr = normal_values(30 + i, 3, (B, Hk, cmax, 128), BF16)
        o = torch.empty((B, H * 128), dtype=torch.bfloat16, device='cuda')
        L.llama_attention_decode(to_device(qr, BF16), to_device(kr, BF16), to_device(vr, BF16),
                                 torch.tensor(lens, dtype=torch.int32, device='cuda'), o, B, cmax, H, Hk, 128, BF16)
        outs.append((o.float().cpu().numpy(), qv, kv, vv, lens))
    got, qv, kv, vv, lens = outs[1]
    for b in range(2):
        n = lens[b]
        ref = attention(qv[b][:, None, :].astype(np.float64), kv[b][:, :n].astype(np.float64),
                        vv[b][:, :n].astype(np.float64), np.array([n - 1]))[0]
        assert rel_l2(got[b], ref) < 1e-2
    _sync_ok()


# ------------------------------------------------------- paged KV cache
def _paginate(raw, n_pages, seed):
    """Scatter a logical cache [B][Hk][C][d] into pages [n_pages][Hk][128][d]
    under a random block table (distinct pages, unused slots -1)."""
    B, Hk, C, d = raw.shape
    max_pages = (C + 127) // 128
    rng = np.random.RandomState(seed)
    perm = rng.permutation(n_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    pages = np.zeros((n_pages, Hk, 128, d), raw.dtype)
    for b in range(B):
        for j in range(max_pages):
            rows = raw[b, :, j * 128:(j + 1) * 128]
            pages[perm[b, j], :, :rows.shape[1]] = rows
    return pages, perm, max_pages


@pytest.mark.parametrize('dtype', [F16, BF16])
def test_attention_decode_paged(dtype):
    B, H, Hk, d, C = 3, 32, 8, 128, 1000
    lens = [1, 300, 1000]
    qv, qr = normal_values(50, 1, (B, H, d), dtype)
    kv, kr = normal_values(50, 2, (B, Hk, C, d), dtype)
    vv, vr = normal_values(50, 3, (B, Hk, C, d), dtype)
    n_pages = 3 * 8 + 5
    kp, table, max_pages = _paginate(kr, n_pages, 1)
    vp, _, _ = _paginate(vr, n_pages, 1)
    o = torch.empty((B, H * d), dtype=torch_dtype(dtype), device='cuda')
    L.llama_attention_decode_paged(to_device(qr, dtype), to_device(kp, dtype), to_device(vp, dtype),
                                   torch.from_numpy(table).cuda(), max_pages, n_pages,
                                   torch.tensor(lens, dtype=torch.int32, device='cuda'), o, B, H, Hk, d, dtype)
    torch.cuda.synchronize()
    _sync_ok()
    got = o.float().cpu().numpy()
    for b in range(B):
        n = lens[b]
        worst, err = attention_row_errors(got[b][None], qv[b][:, None, :].astype(np.float64),
                                          kv[b][:, :n].astype(np.float64), vv[b][:, :n].astype(np.float64),
                                          np.array([n - 1]), dtype)
        assert worst <= 1.0, (b, worst)
        assert err < (1e-2 if dtype == BF16 else 2e-3)


def test_attention_decode_paged_claimed_sub_chunks():
    """A paged cache long enough (>= 128 tiles of 32 keys per decoding warp)
    for the claimed sub-chunks: claimed chunks start inside pages of other
    sequences' ranges; sampled sequences against the oracle."""
    dtype, B, H, Hk, d, C = F16, 24, 32, 8, 128, 14336
    lens = [C - 97 * i for i in range(B)]
    assert Hk * sum((n + 31) // 32 for n in lens) >= 128 * 148 * 4
    qv, qr = normal_values(52, 1, (B, H, d), dtype)
    kv, kr = normal_values(52, 2, (B, Hk, C, d), dtype)
    vv, vr = normal_values(52, 3, (B, Hk, C, d), dtype)
    n_pages = B * (C // 128) + 3
    kp, table, max_pages = _paginate(kr, n_pages, 3)
    vp, _, _ = _paginate(vr, n_pages, 3)
    del kr, vr
    o = torch.empty((B, H * d), dtype=torch.float16, device='cuda')
    L.llama_attention_decode_paged(to_device(qr, dtype), to_device(kp, dtype), to_device(vp, dtype),
                                   torch.from_numpy(table).cuda(), max_pages, n_pages,
                                   torch.tensor(lens, dtype=torch.int32, device='cuda'), o, B, H, Hk, d, dtype)
    torch.cuda.synchronize()
    _sync_ok()
    got = o.float().cpu().numpy()
    for b in (0, 1, B // 2, B - 1):
        n = lens[b]
        worst, err = attention_row_errors(got[b][None], qv[b][:, None, :].astype(np.float64),
                                          kv[b][:, :n].astype(np.float64), vv[b][:, :n].astype(np.float64),
                                          np.array([n - 1]), dtype)
        assert worst <= 1.0, (b, worst)
        assert err < 2e-3


def test_attention_prefill_paged_continues_a_cache():
    """Queries at positions pos0[b] .. pos0[b]+S-1 over a paged cache that
    already holds their keys (a prompt continued across page boundaries)."""
    dtype, B, S, H, Hk, d = F16, 2, 300, 32, 8, 128
    pos0 = [0, 200]
    C = max(pos0) + S
    qv, qr = normal_values(51, 1, (B, H, S, d), dtype)
    kv, kr = normal_values(51, 2, (B, Hk, C, d), dtype)
    vv, vr = normal_values(51, 3, (B, Hk, C, d), dtype)
    n_pages = 11
    kp, table, max_pages = _paginate(kr, n_pages, 2)
    vp, _, _ = _paginate(vr, n_pages, 2)
    o = torch.empty((B, S, H * d), dtype=torch.float16, device='cuda')
    L.llama_attention_prefill_paged(to_device(qr, dtype), to_device(kp, dtype), to_device(vp, dtype),
                                    torch.from_numpy(table).cuda(), max_pages, n_pages,
                                    torch.tensor(pos0, dtype=torch.int32, device='cuda'), o, B, S, H, Hk, d, dtype)
    torch.cuda.synchronize()
    _sync_ok()
    got = o.float().cpu().numpy()
    for b in range(B):
        n = pos0[b] + S
        worst, err = attention_row_errors(got[b], qv[b].astype(np.float64), kv[b][:, :n].astype(np.float64),
                                          vv[b][:, :n].astype(np.float64), pos0[b] + np.arange(S), dtype)
        assert worst <= 1.0, (b, worst)
        assert err < 2e-3


def test_attention_paged_rejects_bad_tables():
    B, H, Hk, d = 1, 8, 2, 128
    q = torch.zeros((B, H, d), dtype=torch.float16, device='cuda')
    pages = torch.zeros((2, Hk, 128, d), dtype=torch.float16, device='cuda')
    o = torch.empty((B, H * d), dtype=torch.float16, device='cuda')
    bad = torch.tensor([[0, 5]], dtype=torch.int32, device='cuda')      # page 5 of a 2-page pool
    with pytest.raises(L.LlamaError) as e:
        L.llama_attention_decode_paged(q, pages, pages, bad, 2, 2, torch.tensor([200], dtype=torch.int32,
                                                                                 device='cuda'), o, B, H, Hk, d, F16)
    assert e.value.status == L.LLAMA_ERR_SHAPE


# ------------------------------------------------- failure detection
@pytest.mark.parametrize('kind', [0, 1])
def test_bounded_wait_gives_up_and_context_stays_usable(kind):
    """A device wait that can never complete (kind 0: an mbarrier phase nobody
    arrives on; kind 1: a counter nobody increments) gives up after its limit
    (1 ms here, 2 s in the kernels), latches LLAMA_ERR_DEVICE_TIMEOUT and
    returns; the next kernels on the same context run normally."""
    import time
    t0 = time.perf_counter()
    L.llama_wait_selftest(kind, 1_000_000)
    assert L.llama_status(None) == L.LLAMA_ERR_DEVICE_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert L.llama_status(None) == 0                       # read and cleared
    xv, xr = normal_values(19, 1, (4, 256), F32)
    g = np.ones(256, np.float32)
    y = torch.empty((4, 256), device='cuda')
    L.llama_rmsnorm(to_device(xr, F32), torch.from_numpy(g).cuda(), y, 4, 256, 1e-5, F32)
    assert rel_l2(y.cpu().numpy(), rms_norm(xv.astype(np.float64), g.astype(np.float64), 1e-5)) < 1e-6
    _sync_ok()
