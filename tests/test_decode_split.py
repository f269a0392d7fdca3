"""Model check of the decode-attention work split (attention.cu), run on the CPU.

The (sequence, kv head, 32-key tile) triples, T in all, are split into W
ranges, one per decoding warp. On long launches the last quarter of every
range is cut into two sub-chunks that warps claim from a counter once their
own part is done. The kernel's partial slots, its merge and its chunk queue
rely on properties of that geometry, checked here for many sizes: chunk
starts increase and tile the sequence exactly; with claimed sub-chunks every
chunk holds tiles and the chunk of tile x is found by the closed form the
merge uses; the slot (b*Hk + g) + chunk of every piece is unique and below
the scratch bound; the merge's piece list for a (b, g) is exactly the chunks
that hold its tiles; the claim order covers every sub-chunk once; and a
loader running at most two tiles ahead of its consumer never has more than
three chunks queued. The arithmetic mirrors the device functions dm_split,
dm_chunk_start and dm_chunk_of and is kept in step with them by hand."""
import random

import pytest

W_B200 = 148 * 4
DM_SUB = 3
DM_TAIL_MIN = 128
CUT = [0, 75, 90, 100]


def dm_split(T, W, BHk):
    return T >= DM_TAIL_MIN * W and BHk * 24 >= W


def dm_chunks(T, W, tail):
    return W * DM_SUB if tail else W


def dm_chunk_start(T, W, tail, k):
    if not tail:
        return T * k // W
    r, sub = divmod(k, DM_SUB)
    a = T * r // W
    if sub == 0:
        return a
    return a + (T * (r + 1) // W - a) * CUT[sub] // 100


def dm_chunk_of(T, W, tail, x):
    r = ((x + 1) * W - 1) // T
    if not tail:
        return r
    a = T * r // W
    ln = T * (r + 1) // W - a
    sub = 0
    while sub < DM_SUB - 1 and a + ln * CUT[sub + 1] // 100 <= x:
        sub += 1
    return r * DM_SUB + sub


def tiles_of(lens):
    return [(n + 31) // 32 if n > 0 else 0 for n in lens]


def check_geometry(lens, Hk, W):
    nt = tiles_of(lens)
    T = Hk * sum(nt)
    tail = dm_split(T, W, len(lens) * Hk)
    K = dm_chunks(T, W, tail)
    starts = [dm_chunk_start(T, W, tail, k) for k in range(K + 1)]
    assert starts[0] == 0 and starts[-1] == T
    assert all(a <= b for a, b in zip(starts, starts[1:]))
    if tail:
        assert all(a < b for a, b in zip(starts, starts[1:])), 'an empty chunk with claimed sub-chunks'
    # chunk_of agrees with the starts on every tile (sampled for long sequences)
    xs = range(T) if T <= 20000 else random.Random(T).sample(range(T), 20000)
    for x in xs:
        k = dm_chunk_of(T, W, tail, x)
        assert starts[k] <= x < starts[k + 1], (x, k)
    # pieces: chunks cut at (b, g) boundaries; slots unique, within B*Hk + chunks
    slots = set()
    t0 = 0
    for b, n in enumerate(nt):
        for g in range(Hk):
            if n == 0:
                continue
            lo, hi = t0, t0 + n              # tiles of (b, g)
            held = [k for k in range(K) if starts[k] < starts[k + 1] and starts[k] < hi and starts[k + 1] > lo]
            # the merge's list: every chunk between chunk(lo) and chunk(hi - 1) when
            # every range holds tiles, else the warp of each tile
            if T >= W:
                listed = list(range(dm_chunk_of(T, W, tail, lo), dm_chunk_of(T, W, tail, hi - 1) + 1))
            else:
                listed = [((lo + i + 1) * W - 1) // T for i in range(n)]
            assert listed == held, (b, g)
            for k in held:
                s = b * Hk + g + k
                assert s not in slots
                assert s < len(lens) * Hk + K
                slots.add(s)
            t0 = hi
    assert t0 == T
    return T, tail


@pytest.mark.parametrize('B,Hk,cmax', [(1, 8, 1024), (1, 8, 131072), (8, 8, 16384), (8, 8, 65536), (32, 8, 4224),
                                       (32, 8, 16384), (64, 8, 1024), (160, 2, 8192), (3, 2, 300), (13, 6, 700)])
def test_geometry_uniform_and_ragged(B, Hk, cmax):
    rng = random.Random(B * 1000 + cmax)
    check_geometry([cmax] * B, Hk, W_B200)
    check_geometry([rng.randint(1, cmax) for _ in range(B)], Hk, W_B200)
    check_geometry([0 if b % 3 == 1 else cmax - b for b in range(B)], Hk, W_B200)   # empty sequences


def test_claimed_sub_chunks_are_used_exactly_on_long_launches():
    assert check_geometry([16384] * 32, 8, W_B200)[1]         # 221 tiles per warp
    assert check_geometry([65536] * 8, 8, W_B200)[1]
    assert not check_geometry([4224] * 32, 8, W_B200)[1]      # the batch-32 decode step
    assert not check_geometry([131072], 8, W_B200)[1]         # one sequence: too many pieces per (b, g)


@pytest.mark.parametrize('W', [4, 12, 592])
def test_geometry_other_grids(W):
    rng = random.Random(W)
    for _ in range(30):
        B = rng.randint(1, 40)
        Hk = rng.choice([1, 2, 8])
        check_geometry([rng.randint(0, 40000) for _ in range(B)], Hk, W)


def simulate_claims(T, W, rng):
    """Warps stream their own part, then claim sub-chunk c % W, 1 + c // W for
    c = 0, 1, ... in whatever order they run out of work (random speeds). Every
    claimed sub-chunk is streamed exactly once, and the chunk queue of a warp
    (chunks its loader moved on to that its consumer has not reached, with the
    loader at most two tiles ahead) never holds more than three."""
    tail = True
    counter = 0
    n_claims = (DM_SUB - 1) * W
    done = {}
    speed = [rng.uniform(0.8, 1.25) for _ in range(W)]
    chunks_of = {w: [w * DM_SUB] for w in range(W)}
    active = set(range(W))
    # event loop: the warp whose current work ends first claims next
    finish = {w: (dm_chunk_start(T, W, tail, w * DM_SUB + 1) - dm_chunk_start(T, W, tail, w * DM_SUB)) / speed[w]
              for w in range(W)}
    while active:
        w = min(active, key=lambda v: finish[v])
        c = counter
        counter += 1
        if c >= n_claims:
            active.discard(w)
            continue
        k = (c % W) * DM_SUB + 1 + c // W
        assert k not in done
        done[k] = w
        chunks_of[w].append(k)
        ln = dm_chunk_start(T, W, tail, k + 1) - dm_chunk_start(T, W, tail, k)
        assert ln >= 1
        finish[w] += ln / speed[w]
    assert sorted(done) == sorted(r * DM_SUB + s for r in range(W) for s in range(1, DM_SUB))
    # chunk queue depth: replay each warp's tile stream with the loader two tiles ahead
    for w, ks in chunks_of.items():
        tiles = [(k, i) for k in ks for i in range(dm_chunk_start(T, W, tail, k + 1) - dm_chunk_start(T, W, tail, k))]
        for pos in range(len(tiles)):
            ahead = tiles[pos:pos + 3]                    # consumed tile and the two issued after it
            loader_next = tiles[pos + 3][0] if pos + 3 < len(tiles) else None
            queued = {k for k, _ in ahead[1:] if k != ahead[0][0]}
            if loader_next is not None and loader_next != ahead[-1][0]:
                queued.add(loader_next)                   # the loader has already moved to its next chunk
            assert len(queued) <= 3


@pytest.mark.parametrize('T,W', [(128 * 592, 592), (221 * 592 + 17, 592), (130 * 12, 12)])
def test_claims_cover_the_tail_once(T, W):
    simulate_claims(T, W, random.Random(T))
