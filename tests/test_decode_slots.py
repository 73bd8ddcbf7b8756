"""Host-side model of the balanced decode's work split and partial-slot numbering (no GPU).

The stream kernel orders the T live 8-key sub-tiles of all (batch, kv head) pairs by
(b, g, list position) and gives warp w the slice [w c, (w + 1) c), c = ceil(T / P);
the warp's partial for pair (b, g) goes to slot w + J(b, g), where J counts the
non-empty pairs before (b, g). The combine kernel, knowing only the per-batch counts,
reads slots w0 + J .. w1 + J with w0 = s // c, w1 = (s + n - 1) // c (s, n: the pair's
first item and count). This model restates those formulas and checks, on random count
mixes (empty entries, tiny and long contexts, more warps than items), that every item
is processed once, no two (warp, pair) partials share a slot, slots stay below
P + B * Hkv (the workspace bound), and the combine reads exactly the pair's slots.
"""

import random

import pytest


def _simulate(counts, Hkv, P):
    B = len(counts)
    T = Hkv * sum(counts)
    if T == 0:
        return
    c = (T + P - 1) // P
    seq, nz = [], 0                        # item -> (b, g, J)
    for b in range(B):
        for g in range(Hkv):
            seq += [(b, g, Hkv * nz + g)] * counts[b]
        nz += counts[b] > 0
    written, covered = {}, 0
    for w in range(P):
        lo = w * c
        for x in range(lo, min(lo + c, T)):
            b, g, J = seq[x]
            slot = w + J
            assert slot < P + B * Hkv
            assert written.setdefault(slot, (w, b, g)) == (w, b, g)   # one owner per slot
            covered += 1
    assert covered == T
    nz = 0
    for b in range(B):                     # the combine's view
        n = counts[b]
        if n:
            before = sum(counts[:b])
            for g in range(Hkv):
                s = Hkv * before + g * n
                w0, w1 = s // c, (s + n - 1) // c
                mine = sorted(sl for sl, (_, bb, gg) in written.items() if (bb, gg) == (b, g))
                assert mine == [w + Hkv * nz + g for w in range(w0, w1 + 1)]
            nz += 1


@pytest.mark.parametrize("seed", range(6))
def test_slots_are_unique_bounded_and_found_by_the_combine(seed):
    rng = random.Random(seed)
    for _ in range(300):
        B = rng.randint(1, 40)
        Hkv = rng.choice([1, 2, 4, 8])
        counts = [rng.choice([0, rng.randint(1, 4), rng.randint(1, 520)]) for _ in range(B)]
        P = rng.choice([1, 3, 37, 592, 1776])
        _simulate(counts, Hkv, P)


def test_bench_shape():
    # B = 8, 8 kv heads, contexts up to 4096 keys (512 sub-tiles), one wave of 1776 warps
    rng = random.Random(1004)
    _simulate([rng.randint(16, 512) for _ in range(8)], 8, 1776)
