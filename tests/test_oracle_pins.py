"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test names the passage of the pages (title + section) or the piece of
mathematics it checks. Brute-force cases re-derive results with plain Python
loops over scalars (math.exp, math.sqrt), independent of the numpy code.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import (Oracle, Params, apply_rope, argmax, attention, feed_forward, ffn_hidden_dim,
                    rel_l2, rms_norm, rope_freqs, silu, softmax_rows)

GOLDEN = os.path.join(os.path.dirname(__file__), 'golden')


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name), encoding='utf-8') as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith('#')]


# --------------------------------------------------------------------- config
def test_rope_freqs_match_printed_table():
    """[W] 位置编码 prints all 64 values of freqs for theta 500000, head_dim 128."""
    printed = np.array([float(v) for v in _golden_lines('rope_freqs_theta500000_d128.txt')])
    assert printed.shape == (64,)
    ours = rope_freqs(128, 500000.0)
    # 5 significant digits printed: half a unit in the 5th digit, relative.
    assert np.all(np.abs(ours - printed) <= 5.0001e-5 * np.abs(printed))
    # Closed form: at i = 32 the frequency is theta**-0.5.
    assert ours[32] == pytest.approx(500000.0 ** -0.5, rel=1e-15)


def test_ffn_hidden_from_params():
    """params.json ([W] 下载并读取模型权重) + the Llama-3-8B SwiGLU width 14336."""
    with open(os.path.join(GOLDEN, 'params_llama3_8b.json'), encoding='utf-8') as f:
        cfg = json.load(f)
    assert ffn_hidden_dim(cfg['dim'], cfg['multiple_of'], cfg['ffn_dim_multiplier']) == 14336
    # Tiny configuration: 768 = two thirds of 4*256 rounded up to 256.
    assert ffn_hidden_dim(256, 256, None) == 768
    p = Params(cfg['dim'], cfg['n_layers'], cfg['n_heads'], cfg['n_kv_heads'], cfg['vocab_size'],
               14336, cfg['norm_eps'], cfg['rope_theta'])
    assert p.head_dim == 128 and p.n_heads // p.n_kv_heads == 4


def test_checkpoint_key_order():
    """The seeded weight streams follow the key order printed in [W] 下载并读取模型权重."""
    import seeded_inputs as si
    printed = _golden_lines('checkpoint_key_order.txt')
    assert si.weight_names(32)[:20] == printed


def test_walkthrough_shapes():
    """Shapes printed for the 17-token prompt ([W], several sections)."""
    rows = [ln.split('|') for ln in _golden_lines('walkthrough_shapes.txt')]
    shapes = {r[0].strip(): tuple(int(v) for v in r[1].split(',')) for r in rows}
    p = Params(4096, 1, 32, 8, 128256, 14336)
    S = 17
    rng = np.random.default_rng(0)

    class ConstWeights(dict):
        def __missing__(self, name):
            if name.endswith('norm.weight'):
                return np.ones(p.dim, np.float32)
            shp = {'wq': (4096, 4096), 'wk': (1024, 4096), 'wv': (1024, 4096),
                   'wo': (4096, 4096), 'w1': (14336, 4096), 'w3': (14336, 4096),
                   'w2': (4096, 14336)}[name.split('.')[-2]]
            return np.broadcast_to(np.float32(1e-3), shp)

    orc = Oracle(p, ConstWeights(), dtype=np.float32)
    x = rng.standard_normal((S, p.dim)).astype(np.float32)
    assert x.shape == shapes['token_embeddings_unnormalized']
    assert rms_norm(x, np.ones(p.dim), p.norm_eps).shape == shapes['token_embeddings (after rms_norm)']
    assert orc.W('layers.0.attention.wq.weight').reshape(p.n_heads, p.head_dim, p.dim).shape == \
        shapes['wq viewed per head']
    assert orc.W('layers.0.attention.wk.weight').reshape(p.n_kv_heads, p.head_dim, p.dim).shape == \
        shapes['wk viewed per head']
    assert (S, p.head_dim // 2, 2) == shapes['q pairs']
    y = orc.layer(0, x, None, 0)
    assert y.shape == shapes['layer_0_embedding'] == shapes['stacked_qkv_attention']
    q = rng.standard_normal((p.n_heads, S, p.head_dim))
    k = rng.standard_normal((p.n_kv_heads, S, p.head_dim))
    o, pr = attention(q, k, k, np.arange(S), return_probs=True)
    assert o.shape == shapes['stacked_qkv_attention']
    assert pr.shape[1:] == shapes['qk_per_token']
    assert o[:, :p.head_dim].shape == shapes['qkv_attention (one head)']


# -------------------------------------------------------------------- RMSNorm
def test_rmsnorm_closed_forms():
    """[W] 构建Transformer层 / [D]: x * rsqrt(mean(x^2) + eps) * g."""
    eps = 1e-5
    assert np.allclose(rms_norm(np.ones(4), np.ones(4), eps), 1.0 / math.sqrt(1.0 + eps), rtol=0, atol=1e-15)
    x = np.array([3.0, 4.0])                      # mean square 12.5
    assert np.allclose(rms_norm(x, np.ones(2), eps), x / math.sqrt(12.5 + eps), rtol=1e-15)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 64)) * rng.uniform(0.001, 10, (7, 1))
    y = rms_norm(x, np.ones(64), eps)
    ms = np.mean(x * x, axis=1)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), np.sqrt(ms / (ms + eps)), rtol=1e-13)
    g = rng.standard_normal(64)
    assert np.allclose(rms_norm(x, g, eps), y * g, rtol=1e-14)
    # Without eps the norm is scale invariant.
    assert np.allclose(rms_norm(5.0 * x, np.ones(64), 0.0), rms_norm(x, np.ones(64), 0.0), rtol=1e-14)


# ----------------------------------------------------------------------- RoPE
def test_rope_pairing_and_direction():
    """[W] 位置编码: adjacent pairs are complex numbers multiplied by e^{i m f}."""
    theta = 10000.0
    f1 = theta ** -0.5                           # d = 4: freqs = [1, theta^-1/2]
    u = np.eye(4)
    r = apply_rope(u[:, None, :], np.array([1]), theta)[:, 0, :]
    c0, s0, c1, s1 = math.cos(1.0), math.sin(1.0), math.cos(f1), math.sin(f1)
    assert np.allclose(r[0], [c0, s0, 0, 0], atol=1e-15)      # 1 -> e^{i}
    assert np.allclose(r[1], [-s0, c0, 0, 0], atol=1e-15)     # i -> i e^{i}
    assert np.allclose(r[2], [0, 0, c1, s1], atol=1e-15)
    assert np.allclose(r[3], [0, 0, -s1, c1], atol=1e-15)


def test_rope_invariants():
    rng = np.random.default_rng(2)
    d, theta = 128, 500000.0
    u = rng.standard_normal((3, 9, d))
    pos = rng.integers(0, 40000, 9)
    # identity at position 0
    assert np.array_equal(apply_rope(u, np.zeros(9, int), theta), u)
    # each pair keeps its length
    r = apply_rope(u, pos, theta)
    assert np.allclose(np.hypot(r[..., 0::2], r[..., 1::2]), np.hypot(u[..., 0::2], u[..., 1::2]), rtol=1e-13)
    # q(m).k(n) depends on m - n only
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    for m, n, s in [(5, 2, 7), (100, 3, 1000), (0, 31, 4096)]:
        a = apply_rope(q[None], np.array([m]), theta)[0] @ apply_rope(k[None], np.array([n]), theta)[0]
        b = apply_rope(q[None], np.array([m + s]), theta)[0] @ apply_rope(k[None], np.array([n + s]), theta)[0]
        assert a == pytest.approx(b, rel=1e-9, abs=1e-9)
    # rotations compose
    a = apply_rope(apply_rope(u, pos, theta), pos + 3, theta)
    assert np.allclose(a, apply_rope(u, 2 * pos + 3, theta), atol=1e-9)


# ------------------------------------------------------------------ attention
def _brute_attention(q, k, v, q_pos):
    """Scalar loops: scores, causal mask, softmax, weighted sum, head concat."""
    H, S, d = q.shape
    Hk, T, _ = k.shape
    out = [[0.0] * (H * d) for _ in range(S)]
    for h in range(H):
        g = (h * Hk) // H
        for i in range(S):
            sc = []
            for j in range(int(q_pos[i]) + 1):
                sc.append(sum(q[h, i, t] * k[g, j, t] for t in range(d)) / math.sqrt(d))
            mx = max(sc)
            e = [math.exp(s - mx) for s in sc]
            z = sum(e)
            for t in range(d):
                out[i][h * d + t] = sum(e[j] / z * v[g, j, t] for j in range(len(e)))
    return np.array(out)


def test_attention_brute_force():
    """[W] 查询和键相乘 / 掩码 / 多头注意力 on tiny inputs, with a cache offset."""
    rng = np.random.default_rng(3)
    H, Hk, d, T = 4, 2, 4, 7
    q = rng.standard_normal((H, 3, d))
    k = rng.standard_normal((Hk, T, d))
    v = rng.standard_normal((Hk, T, d))
    q_pos = np.array([4, 5, 6])                 # 3 new tokens after 4 cached
    assert np.allclose(attention(q, k, v, q_pos), _brute_attention(q, k, v, q_pos), rtol=1e-12, atol=1e-13)
    q_pos = np.arange(T)
    q = rng.standard_normal((H, T, d))
    assert np.allclose(attention(q, k, v, q_pos), _brute_attention(q, k, v, q_pos), rtol=1e-12, atol=1e-13)


def test_attention_invariants():
    rng = np.random.default_rng(4)
    H, Hk, S, d = 8, 2, 11, 16
    q, k, v = (rng.standard_normal((h, S, d)) for h in (H, Hk, Hk))
    o, p = attention(q, k, v, np.arange(S), return_probs=True)
    assert np.allclose(p.sum(-1), 1.0, rtol=0, atol=1e-14)          # rows sum to 1
    assert np.all(np.triu(p, 1) == 0.0)                              # nothing above the diagonal
    for h in range(H):                                              # token 0 sees only itself
        assert np.array_equal(o[0, h * d:(h + 1) * d], v[h // (H // Hk), 0])
    # q = 0: uniform weights over the visible prefix
    o0 = attention(np.zeros_like(q), k, v, np.arange(S))
    for i in range(S):
        assert np.allclose(o0[i, :d], v[0, :i + 1].mean(0), rtol=1e-13)
    # GQA equals MHA with each kv head repeated for consecutive query heads
    rep = H // Hk
    om = attention(q, np.repeat(k, rep, 0), np.repeat(v, rep, 0), np.arange(S))
    assert np.allclose(o, om, rtol=0, atol=1e-14)
    # causality: later keys/values do not change earlier rows
    k2, v2 = k.copy(), v.copy()
    k2[:, 6:] += 5.0
    v2[:, 6:] -= 3.0
    assert np.array_equal(attention(q, k2, v2, np.arange(S))[:6], o[:6])
    # two keys: softmax weight of key 1 is sigmoid((s1 - s0)/sqrt(d))
    qq = np.zeros((1, 2, 4)); qq[0, 1] = [1, 0, 0, 0]
    kk = np.zeros((1, 2, 4)); kk[0, 0] = [0.5, 0, 0, 0]; kk[0, 1] = [2.5, 0, 0, 0]
    vv = np.zeros((1, 2, 4)); vv[0, 1, 0] = 1.0
    w1 = 1.0 / (1.0 + math.exp(-(2.5 - 0.5) / 2.0))
    assert attention(qq, kk, vv, np.arange(2))[1, 0] == pytest.approx(w1, rel=1e-15)


def test_softmax_rows_closed_form():
    s = np.array([[0.0, math.log(3.0), -np.inf]])
    assert np.allclose(softmax_rows(s), [[0.25, 0.75, 0.0]], rtol=1e-15)


# ------------------------------------------------------------------------ FFN
def test_silu_values():
    """F.silu ([W] 前馈神经网络层) = z * sigmoid(z)."""
    z = np.array([0.0, 1.0, -1.0, 50.0, -800.0])
    ref = [0.0, 0.7310585786300049, -0.2689414213699951, 50.0, 0.0]
    assert np.allclose(silu(z), ref, rtol=1e-15, atol=1e-300)


def test_feed_forward_brute_force():
    rng = np.random.default_rng(5)
    D, F, S = 3, 5, 2                            # non-square: a transposed operand fails
    x, w1, w3, w2 = (rng.standard_normal(s) for s in ((S, D), (F, D), (F, D), (D, F)))
    ref = np.zeros((S, D))
    for s in range(S):
        g = []
        for f in range(F):
            a = sum(x[s, t] * w1[f, t] for t in range(D))
            b = sum(x[s, t] * w3[f, t] for t in range(D))
            g.append(a / (1.0 + math.exp(-a)) * b)
        for o in range(D):
            ref[s, o] = sum(g[f] * w2[o, f] for f in range(F))
    assert np.allclose(feed_forward(x, w1, w3, w2), ref, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------------- block
def _tiny_params(n_layers=1):
    return Params(dim=8, n_layers=n_layers, n_heads=2, n_kv_heads=1, vocab_size=11, ffn_hidden=6,
                  norm_eps=1e-5, rope_theta=10000.0)


def _rand_weights(p, rng, std=0.3):
    w = {'tok_embeddings.weight': rng.standard_normal((p.vocab_size, p.dim)),
         'norm.weight': rng.uniform(0.5, 1.5, p.dim),
         'output.weight': rng.standard_normal((p.vocab_size, p.dim)) * std}
    d = p.head_dim
    for i in range(p.n_layers):
        pre = f'layers.{i}.'
        w[pre + 'attention_norm.weight'] = rng.uniform(0.5, 1.5, p.dim)
        w[pre + 'ffn_norm.weight'] = rng.uniform(0.5, 1.5, p.dim)
        w[pre + 'attention.wq.weight'] = rng.standard_normal((p.n_heads * d, p.dim)) * std
        w[pre + 'attention.wk.weight'] = rng.standard_normal((p.n_kv_heads * d, p.dim)) * std
        w[pre + 'attention.wv.weight'] = rng.standard_normal((p.n_kv_heads * d, p.dim)) * std
        w[pre + 'attention.wo.weight'] = rng.standard_normal((p.dim, p.n_heads * d)) * std
        w[pre + 'feed_forward.w1.weight'] = rng.standard_normal((p.ffn_hidden, p.dim)) * std
        w[pre + 'feed_forward.w3.weight'] = rng.standard_normal((p.ffn_hidden, p.dim)) * std
        w[pre + 'feed_forward.w2.weight'] = rng.standard_normal((p.dim, p.ffn_hidden)) * std
    return w


def _brute_block(p, w, x, pos0):
    """Whole decoder block with scalar loops, following [W] step by step."""
    S, D = x.shape
    d, H, Hk = p.head_dim, p.n_heads, p.n_kv_heads
    pre = 'layers.0.'

    def norm(row, g):
        r = 1.0 / math.sqrt(sum(t * t for t in row) / len(row) + p.norm_eps)
        return [row[t] * r * g[t] for t in range(len(row))]

    def matvec(W, row):
        return [sum(W[o, t] * row[t] for t in range(len(row))) for o in range(W.shape[0])]

    def rot(vec, m):
        out = list(vec)
        for i in range(d // 2):
            ang = m * p.rope_theta ** (-(2.0 * i) / d)
            a, b = vec[2 * i], vec[2 * i + 1]
            out[2 * i] = a * math.cos(ang) - b * math.sin(ang)
            out[2 * i + 1] = a * math.sin(ang) + b * math.cos(ang)
        return out

    xn = [norm(list(x[s]), w[pre + 'attention_norm.weight']) for s in range(S)]
    qs = [matvec(w[pre + 'attention.wq.weight'], r) for r in xn]
    ks = [matvec(w[pre + 'attention.wk.weight'], r) for r in xn]
    vs = [matvec(w[pre + 'attention.wv.weight'], r) for r in xn]
    q = np.array([[rot(qs[s][h * d:(h + 1) * d], pos0 + s) for s in range(S)] for h in range(H)])
    k = np.array([[rot(ks[s][g * d:(g + 1) * d], pos0 + s) for s in range(S)] for g in range(Hk)])
    v = np.array([[vs[s][g * d:(g + 1) * d] for s in range(S)] for g in range(Hk)])
    o = _brute_attention(q, k, v, np.arange(S))
    out = np.zeros_like(x)
    for s in range(S):
        h = [x[s, t] + a for t, a in enumerate(matvec(w[pre + 'attention.wo.weight'], list(o[s])))]
        hn = norm(h, w[pre + 'ffn_norm.weight'])
        a = matvec(w[pre + 'feed_forward.w1.weight'], hn)
        b = matvec(w[pre + 'feed_forward.w3.weight'], hn)
        g = [a[f] / (1.0 + math.exp(-a[f])) * b[f] for f in range(len(a))]
        out[s] = [h[t] + y for t, y in enumerate(matvec(w[pre + 'feed_forward.w2.weight'], g))]
    return out


def test_block_brute_force():
    """Decoder block = [W] 构建Transformer层 .. 前馈神经网络层 with scalar loops."""
    p = _tiny_params()
    rng = np.random.default_rng(6)
    w = _rand_weights(p, rng)
    x = rng.standard_normal((5, p.dim))
    ref = _brute_block(p, w, x, 0)
    assert np.allclose(Oracle(p, w).layer(0, x, None, 0), ref, rtol=1e-12, atol=1e-12)


def test_block_residual_structure():
    """[W] 相加与归一化: zero wo and w2 make the block the identity; zero w2 alone
    leaves x + attention."""
    p = _tiny_params()
    rng = np.random.default_rng(7)
    w = _rand_weights(p, rng)
    x = rng.standard_normal((4, p.dim))
    w0 = dict(w)
    w0['layers.0.attention.wo.weight'] = np.zeros_like(w['layers.0.attention.wo.weight'])
    w0['layers.0.feed_forward.w2.weight'] = np.zeros_like(w['layers.0.feed_forward.w2.weight'])
    assert np.array_equal(Oracle(p, w0).layer(0, x, None, 0), x)
    w1 = dict(w)
    w1['layers.0.feed_forward.w2.weight'] = np.zeros_like(w['layers.0.feed_forward.w2.weight'])
    y = Oracle(p, w1).layer(0, x, None, 0)
    assert not np.allclose(y, x)
    # rows of a subset equal the full computation
    full = Oracle(p, w).layer(0, x, None, 0)
    assert np.allclose(Oracle(p, w).layer(0, x, None, 0, rows=np.array([1, 3])), full[[1, 3]], rtol=1e-14)


# --------------------------------------------------------- KV-cache decode
def test_decode_equals_recompute():
    """[D] KV-Cache chapter: decoding token t with the cache gives the same logits
    as a full forward pass over t+1 tokens (tiny model, 8 steps)."""
    p = Params(dim=32, n_layers=2, n_heads=4, n_kv_heads=2, vocab_size=50, ffn_hidden=48,
               norm_eps=1e-5, rope_theta=500000.0)
    rng = np.random.default_rng(8)
    w = _rand_weights(p, rng)
    orc = Oracle(p, w)
    toks = list(rng.integers(0, p.vocab_size, 17))
    lg, caches = orc.prefill(np.array([toks]))
    assert rel_l2(lg[0], orc.forward(np.array(toks))) < 1e-14
    for _ in range(8):
        nxt = int(argmax(lg)[0])
        toks.append(nxt)
        lg = orc.decode_step(np.array([nxt]), caches)
        full = orc.forward(np.array(toks))
        assert rel_l2(lg[0], full) < 1e-12
    assert caches[0].length == 25


def test_float32_noise_floor():
    """The float32 oracle stays far inside the 1e-3 fp32 tolerance of float64."""
    p = Params(dim=64, n_layers=2, n_heads=4, n_kv_heads=2, vocab_size=97, ffn_hidden=160)
    rng = np.random.default_rng(9)
    w = _rand_weights(p, rng, std=0.1)
    toks = rng.integers(0, p.vocab_size, (2, 13))
    a, _ = Oracle(p, w, np.float64).prefill(toks)
    b, _ = Oracle(p, w, np.float32).prefill(toks)
    assert rel_l2(b, a) < 1e-5


def test_argmax_ties_lowest_index():
    """[W] 预测下一个输出 uses torch.argmax; the first maximal index wins."""
    lg = np.array([[1.0, 3.0, 3.0, 2.0], [5.0, 5.0, 5.0, 5.0]])
    assert list(argmax(lg)) == [1, 0]


def test_embed_and_logits_brute_force():
    """[W] 分词器与编码 (row gather) and 预测下一个输出 (one final rms_norm, then
    the last row times output^T)."""
    p = _tiny_params()
    rng = np.random.default_rng(10)
    w = _rand_weights(p, rng)
    orc = Oracle(p, w)
    toks = np.array([3, 0, 10, 3])
    assert np.array_equal(orc.embed(toks), w['tok_embeddings.weight'][[3, 0, 10, 3]])
    x = rng.standard_normal(p.dim)
    r = 1.0 / math.sqrt(sum(t * t for t in x) / p.dim + p.norm_eps)
    xf = [x[t] * r * w['norm.weight'][t] for t in range(p.dim)]
    ref = [sum(xf[t] * w['output.weight'][o, t] for t in range(p.dim)) for o in range(p.vocab_size)]
    assert np.allclose(orc.logits(x), ref, rtol=1e-13, atol=1e-14)
