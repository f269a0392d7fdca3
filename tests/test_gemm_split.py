"""Model check of the stream-K work split shared by the wide and skinny
tcgen05 GEMMs (gemm_tc.cu), run on the CPU.

The (tile, k-block) units of the split region, taken tile-major, are cut into
G equal contiguous ranges, one per CTA; a range falls into pieces, one per
tile it touches. The kernels' fixup terminates and sums in a fixed order
because of properties of that split, checked here for many shapes and grid
sizes: every unit is covered once; a split tile has exactly one owner piece
(holding k-block 0), which is the last piece of its CTA's range; every other
piece of the tile is the first piece of its CTA's range and comes from the
CTAs (owner, c_hi] given by the owner formula; so a CTA writes at most one
share slot and owners wait only for pieces that wait for nothing. The
arithmetic mirrors the device functions sk_first / sk_owner and the wide
kernel's work iterator; the two are kept in step by hand."""
import random

import pytest


def sk_first(c, U, G):
    return U * c // G


def sk_owner(u, U, G):
    return ((u + 1) * G - 1) // U


def pieces(c, G, kb, T, T_dp, G_sk):
    """The wide kernel's work sequence for CTA c: whole tiles c, c+G, ...
    below T_dp, then its stream-K range over tiles [T_dp, T)."""
    out = []
    dp_n = (T_dp - c + G - 1) // G if T_dp > c else 0
    out += [(c + i * G, 0, kb) for i in range(dp_n)]
    U = (T - T_dp) * kb
    if c < G_sk:
        u, u1 = sk_first(c, U, G_sk), sk_first(c + 1, U, G_sk)
        while u < u1:
            tile, klo = T_dp + u // kb, u % kb
            n = min(u1 - u, kb - klo)
            out.append((tile, klo, n))
            u += n
    return out


def check_split(T, kb, G, T_dp, G_sk):
    U = (T - T_dp) * kb
    cover = {}
    owner_of, shares_of = {}, {}
    for c in range(max(G, G_sk)):
        ps = pieces(c, G, kb, T, T_dp, G_sk)
        n_share = 0
        for idx, (tile, klo, n) in enumerate(ps):
            assert n > 0
            for k in range(klo, klo + n):
                assert (tile, k) not in cover, 'unit covered twice'
                cover[(tile, k)] = c
            if klo == 0 and n == kb:
                continue
            assert tile >= T_dp, 'a data-parallel tile was split'
            first_sk = idx == sum(1 for p in ps if p[0] < T_dp)
            if klo == 0:
                assert idx == len(ps) - 1, 'owner piece is not the last of its range'
                owner_of[tile] = c
            else:
                assert first_sk, 'share piece is not the first of its range'
                shares_of.setdefault(tile, []).append(c)
                n_share += 1
        assert n_share <= 1, 'a CTA would need two share slots'
    assert len(cover) == T * kb, 'units missing'
    for tile, c in owner_of.items():
        t0 = (tile - T_dp) * kb
        c_own, c_hi = sk_owner(t0, U, G_sk), sk_owner(t0 + kb - 1, U, G_sk)
        assert c_own == c
        # the skinny kernel counts contributors with a non-empty range
        need = sum(1 for cc in range(c_own + 1, c_hi + 1) if sk_first(cc + 1, U, G_sk) > sk_first(cc, U, G_sk))
        assert sorted(shares_of.get(tile, [])) == [cc for cc in range(c_own + 1, c_hi + 1)
                                                   if sk_first(cc + 1, U, G_sk) > sk_first(cc, U, G_sk)]
        assert need == len(shares_of.get(tile, []))
    assert set(shares_of) <= set(owner_of), 'shares of a tile with no owner'


@pytest.mark.parametrize('N,K', [(6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336), (128256, 4096),
                                 (1000, 4096), (520, 4104), (384, 256), (128, 64)])
@pytest.mark.parametrize('G', [148, 132, 7])
def test_skinny_split(N, K, G):
    """Skinny GEMM: every 128-row weight tile is in the stream-K region."""
    T, kb = (N + 127) // 128, (K + 63) // 64
    check_split(T, kb, G, 0, G)


def test_wide_split_random_shapes():
    """Wide GEMM: data-parallel tiles below T_dp, stream-K over G_sk CTAs."""
    rng = random.Random(5)
    for _ in range(300):
        T, kb, G = rng.randint(1, 400), rng.randint(1, 240), rng.choice([148, 132, 64, 7])
        sk = rng.randint(0, T)
        U = sk * kb
        G_sk = min(G, max(1, U // 8)) if sk else 0
        check_split(T, kb, G, T - sk, G_sk)
