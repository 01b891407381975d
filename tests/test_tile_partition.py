"""The work split of the tensor-core decode kernels, restated on the CPU.

The 16-token tiles of all (sequence, kv head) rows form one sequence of W
tiles (prefix P over sequences: P[b+1] - P[b] = Hkv * ceil(len_b / 16)).
Owner w (a warp, or a CTA of four warps) takes tiles [w W / N, (w + 1) W / N)
with N = min(owners, W) and writes one partial per row piece to slot
wpu * (w + b Hkv + kv head) + (warp within the owner).  The merge finds a
row's slots from the owners f .. l whose ranges meet the row's tiles.  These
checks run the same index arithmetic over random length mixes: every tile is
covered exactly once, no slot is written twice, every slot stays inside the
workspace, and the merge reads exactly the slots that were written."""
import random

import pytest


def _prefix(lens, Hkv, max_T):
    P = [0]
    for L in lens:
        L = min(max(L, 0), max_T)
        P.append(P[-1] + (L + 15) // 16 * Hkv)
    return P


def _sequence_of(P, x):
    b, hi = 0, len(P) - 1
    while hi - b > 1:
        mid = (b + hi) >> 1
        if P[mid] <= x:
            b = mid
        else:
            hi = mid
    return b


def _split(lens, Hkv, max_T, owners, wpu):
    B = len(lens)
    P = _prefix(lens, Hkv, max_T)
    W = P[B]
    N = min(owners, W)
    written, covered = {}, set()
    for w in range(N):
        x, x1 = w * W // N, (w + 1) * W // N
        assert x < x1                       # every owner gets at least one tile
        b = _sequence_of(P, x)
        while x < x1:
            while P[b + 1] <= x:
                b += 1
            tb = (P[b + 1] - P[b]) // Hkv
            rel = x - P[b]
            kvh, tt = rel // tb, rel % tb
            te = min(tb, tt + (x1 - x))
            assert te > tt
            for sub in range(wpu):          # each warp of the owner writes its slot
                slot = wpu * (w + b * Hkv + kvh) + sub
                assert slot not in written
                assert slot < wpu * (owners + B * Hkv)   # inside the workspace
                written[slot] = (b, kvh)
            for k in range(tt, te):
                assert (b, kvh, k) not in covered
                covered.add((b, kvh, k))
            x += te - tt
    return P, W, N, written, covered


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("wpu", [1, 4])
def test_every_tile_once_and_merge_reads_written_slots(seed, wpu):
    rng = random.Random(seed * 7 + wpu)
    for _ in range(300):
        B = rng.randint(1, 12)
        Hkv = rng.choice([1, 2, 4, 8])
        max_T = rng.choice([16, 20, 64, 100, 512, 4096])
        lens = [rng.choice([0, 1, 15, 16, 17, rng.randint(0, max_T), max_T, max_T + 5, -3]) for _ in range(B)]
        owners = rng.choice([1, 4, 7, 12, 40, 148 * 3, 148 * 12])
        P, W, N, written, covered = _split(lens, Hkv, max_T, owners, wpu)
        for b in range(B):
            tb = (P[b + 1] - P[b]) // Hkv
            for kvh in range(Hkv):
                assert all((b, kvh, k) in covered for k in range(tb))
                if tb == 0:
                    continue
                S = P[b] + kvh * tb
                E = S + tb
                f = ((S + 1) * N + W - 1) // W - 1
                last = (E * N + W - 1) // W - 1
                merge = sorted(wpu * (o + b * Hkv + kvh) + sub for o in range(f, last + 1) for sub in range(wpu))
                mine = sorted(s for s, v in written.items() if v == (b, kvh))
                assert merge == mine, (b, kvh)


def test_full_size_llama_shape():
    """The bench shape: 16 sequences x 8 kv heads x 32768 tokens over 148 x 3 x 4 warps."""
    P, W, N, written, covered = _split([32768] * 16, 8, 32768, 148 * 3 * 4, 1)
    assert W == 16 * 8 * 2048 and len(covered) == W
    assert len(written) <= N + 16 * 8
