"""End-to-end parity of the model entry points (prefill, decode, block,
generate) against the CPU oracle on seeded weights and inputs."""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import Oracle, argmax
from tests.helpers import BF16, F32, SeededWeights, near_tie_ok, normal_values, params_from, rel_l2

pytestmark = pytest.mark.gpu

torch = pytest.importorskip('torch')
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip('needs a CUDA device', allow_module_level=True)

from llama_transformer_decoder_b200 import binding as L  # noqa: E402
from llama_transformer_decoder_b200.configs import LLAMA3_8B, TINY, make_config  # noqa: E402


class Model:
    def __init__(self, params, dtype, max_batch, max_seq, max_tokens=0):
        self.cfg = make_config(params, dtype=dtype, max_batch=max_batch, max_seq=max_seq, max_tokens=max_tokens)
        self.h = L.llama_create(self.cfg)
        self.rc = L.llama_get_config(self.h)
        self.params = dict(params)
        self.p = params_from(params, self.rc.ffn_hidden)

    def close(self):
        if self.h:
            L.llama_destroy(self.h)
            self.h = None

    def logits(self, B):
        out = torch.empty((B, self.rc.vocab_size), device='cuda')
        L.llama_logits(self.h, out)
        return out

    def argmax(self, B):
        out = torch.empty(B, dtype=torch.int32, device='cuda')
        L.llama_argmax(self.h, out)
        return out


@pytest.fixture
def tiny():
    m = Model(TINY, F32, max_batch=2, max_seq=64)
    L.llama_init_weights(m.h, 0, 0.02)
    yield m
    m.close()


def _check_status(m):
    assert L.llama_sync_status(m.h) == 0


def test_tiny_weights_match_host_generator(tiny):
    w = SeededWeights(tiny.p, 0, 0.02, F32, cache=False)
    for name in si.weight_names(tiny.p.n_layers):
        ref = w[name]
        buf = np.empty(ref.shape, np.float32)
        L.llama_get_weight(tiny.h, name, buf, buf.nbytes, 0)
        assert np.array_equal(buf.view(np.uint32), ref.view(np.uint32)), name


def test_tiny_fp32_prefill_and_greedy_decode(tiny):
    """Tiny fp32 configuration: 17 tokens, then 8 greedy decode steps; the oracle
    is teacher-forced with the GPU's tokens (rel-L2 <= 1e-3 on every logits row)."""
    toks = si.tokens(1, 17, 1024)
    L.llama_prefill(tiny.h, torch.from_numpy(toks).cuda(), 1, 17)
    orc = Oracle(tiny.p, SeededWeights(tiny.p, 0, 0.02, F32))
    ref, caches = orc.prefill(toks[None])
    got = tiny.logits(1).cpu().numpy()
    assert rel_l2(got, ref) < 1e-3
    agree = 0
    for step in range(8):
        nxt = tiny.argmax(1)
        t = int(nxt.cpu()[0])
        agree += int(t == int(argmax(ref)[0]))
        assert near_tie_ok(t, ref[0], 1e-4)
        L.llama_decode_step(tiny.h, nxt, 1)
        ref = orc.decode_step(np.array([t]), caches)
        got = tiny.logits(1).cpu().numpy()
        assert rel_l2(got, ref) < 1e-3, step
    assert agree >= 7
    lens = np.zeros(1, np.int32)
    L.llama_get_lengths(tiny.h, lens, 1)
    assert lens[0] == 25
    _check_status(tiny)


def test_tiny_generate_host_api(tiny):
    """llama_generate (host buffers in and out) gives the same tokens as the
    step-by-step calls."""
    toks = si.tokens(1, 2 * 9, 1024).reshape(2, 9)
    out = np.zeros((2, 5), np.int32)
    L.llama_generate(tiny.h, np.ascontiguousarray(toks), 2, 9, 4, out)
    L.llama_reset(tiny.h)
    L.llama_prefill(tiny.h, torch.from_numpy(toks).cuda(), 2, 9)
    seq = [tiny.argmax(2)]
    for _ in range(4):
        L.llama_decode_step(tiny.h, seq[-1], 2)
        seq.append(tiny.argmax(2))
    ref = torch.stack(seq, 1).cpu().numpy()
    assert np.array_equal(out, ref)
    _check_status(tiny)


def test_errors_leave_model_usable(tiny):
    with pytest.raises(L.LlamaError) as e:
        L.llama_prefill(tiny.h, torch.zeros(65, dtype=torch.int32, device='cuda'), 1, 65)
    assert e.value.status == L.LLAMA_ERR_SHAPE
    with pytest.raises(L.LlamaError) as e:
        L.llama_prefill(tiny.h, torch.zeros(3, dtype=torch.int32, device='cuda'), 3, 1)
    assert e.value.status == L.LLAMA_ERR_SHAPE
    with pytest.raises(L.LlamaError):
        L.llama_get_weight(tiny.h, 'layers.9.attention.wq.weight', np.zeros(4, np.float32), 16, 0)
    bad = torch.tensor([5, 4000, 7], dtype=torch.int32, device='cuda')   # 4000 >= vocab
    L.llama_prefill(tiny.h, bad, 1, 3)
    assert L.llama_sync_status(tiny.h) == L.LLAMA_ERR_DEVICE_BOUNDS
    assert L.llama_sync_status(tiny.h) == 0          # cleared
    L.llama_reset(tiny.h)
    L.llama_prefill(tiny.h, torch.tensor([1, 2, 3], dtype=torch.int32, device='cuda'), 1, 3)
    _check_status(tiny)


# ------------------------------------------------------------- bf16 block
BLOCK_8B = dict(LLAMA3_8B, n_layers=1, vocab_size=512)


@pytest.fixture(scope='module')
def block8b():
    m = Model(BLOCK_8B, BF16, max_batch=2, max_seq=2048, max_tokens=4096)
    L.llama_init_weights(m.h, 0, 0.02)
    w = SeededWeights(m.p, 0, 0.02, BF16)
    yield m, w
    m.close()


@pytest.mark.parametrize('B,S', [(1, 17), (1, 2048), (2, 300), (1, 1)])
def test_block_8b_bf16(block8b, B, S):
    """One 8B-shaped decoder block on N(0,1) hidden states (rel-L2 <= 2e-2)."""
    m, w = block8b
    assert m.rc.ffn_hidden == 14336
    L.llama_reset(m.h)
    xv, _ = normal_values(2, si.STREAM_HIDDEN, (B, S, 4096), BF16)
    x = torch.from_numpy(np.ascontiguousarray(xv)).cuda()
    y = torch.empty_like(x)
    L.llama_block_forward(m.h, 0, x, y, B, S)
    torch.cuda.synchronize()
    _check_status(m)
    got = y.cpu().numpy()
    orc = Oracle(m.p, w)
    rows = np.arange(S) if S <= 300 else np.unique(np.r_[np.arange(0, S, 97), S - 1])
    for b in range(B):
        ref = orc.layer(0, xv[b].astype(np.float64), None, 0, rows=rows)
        assert rel_l2(got[b][rows], ref) < 2e-2


# --------------------------------------------- bf16 multi-layer end to end
SMALL_BF16 = dict(dim=512, n_layers=3, n_heads=4, n_kv_heads=2, vocab_size=3000, ffn_hidden=1536,
                  norm_eps=1e-5, rope_theta=500000.0)


@pytest.mark.parametrize('B,S', [(3, 40), (2, 100)])
def test_small_bf16_model_prefill_decode(B, S):
    """3-layer bf16 model: prefill through the skinny (M <= 128) or wide GEMM
    path, then 6 decode steps (graph-replayed from the third); teacher-forced
    oracle, rel-L2 <= 2e-2 on every logits row."""
    m = Model(SMALL_BF16, BF16, max_batch=4, max_seq=256)
    try:
        L.llama_init_weights(m.h, 3, 0.02)
        orc = Oracle(m.p, SeededWeights(m.p, 3, 0.02, BF16))
        toks = si.tokens(1, B * S, 3000).reshape(B, S)
        L.llama_prefill(m.h, torch.from_numpy(toks).cuda(), B, S)
        ref, caches = orc.prefill(toks)
        got = m.logits(B).cpu().numpy()
        assert rel_l2(got, ref) < 2e-2
        for step in range(6):
            nxt = m.argmax(B)
            tn = nxt.cpu().numpy()
            slack = 4 * float(np.max(np.abs(got - ref))) + 1e-6
            for b in range(B):
                assert near_tie_ok(int(tn[b]), ref[b], slack)
            L.llama_decode_step(m.h, nxt, B)
            ref = orc.decode_step(tn, caches)
            got = m.logits(B).cpu().numpy()
            assert rel_l2(got, ref) < 2e-2, step
        _check_status(m)
    finally:
        m.close()


def test_chunked_prefill_continues_the_cache():
    """Two prefill calls on the same sequences (the second starts at the cached
    length) equal one oracle pass over the concatenated prompt: positions,
    RoPE angles and the causal mask follow the cache length."""
    m = Model(SMALL_BF16, BF16, max_batch=2, max_seq=512)
    try:
        L.llama_init_weights(m.h, 4, 0.02)
        orc = Oracle(m.p, SeededWeights(m.p, 4, 0.02, BF16))
        toks = si.tokens(7, 2 * 330, 3000).reshape(2, 330)
        L.llama_prefill(m.h, torch.from_numpy(np.ascontiguousarray(toks[:, :200])).cuda(), 2, 200)
        L.llama_prefill(m.h, torch.from_numpy(np.ascontiguousarray(toks[:, 200:])).cuda(), 2, 130)
        got = m.logits(2).cpu().numpy()
        ref = np.stack([orc.forward(toks[b]) for b in range(2)])
        assert rel_l2(got, ref) < 2e-2
        lens = np.zeros(2, np.int32)
        L.llama_get_lengths(m.h, lens, 2)
        assert list(lens) == [330, 330]
        _check_status(m)
    finally:
        m.close()
