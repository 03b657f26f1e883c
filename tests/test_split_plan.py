"""The split-KV work plan, modelled on the host: every page of every sequence
belongs to exactly one worker piece, piece slots c + b are unique and below
G + B - 1, and the combine's worker range for sequence b is exactly the set of
workers holding its pages.  (The kernels compute the same integer formulas:
worker c takes pages [c*T/G, (c+1)*T/G); page g belongs to worker
((g+1)*G - 1) // T.)"""
import numpy as np
import pytest


def npages(L):
    return (L + 63) // 64 if L > 0 else 0


def plan(lens, G):
    T = sum(npages(L) for L in lens)
    pieces = []
    prefix = np.concatenate([[0], np.cumsum([npages(L) for L in lens])])
    for c in range(G):
        s, e = c * T // G, (c + 1) * T // G
        for b, L in enumerate(lens):
            n = npages(L)
            lo, hi = max(s, prefix[b]), min(e, prefix[b] + n)
            if n and lo < hi:
                pieces.append((c, b, lo - prefix[b], hi - prefix[b]))
    return T, prefix, pieces


def worker_of_page(g, T, G):
    return ((g + 1) * G - 1) // T


@pytest.mark.parametrize("seed", range(20))
def test_plan_invariants(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 40))
    lens = [int(x) for x in rng.integers(0, 3000, B)]
    if seed % 3 == 0:
        lens[int(rng.integers(0, B))] = 0
    G = int(rng.choice([1, 2, 3, 7, 74, 148, 500]))
    T, prefix, pieces = plan(lens, G)
    covered = {}
    for c, b, p0, p1 in pieces:
        for p in range(p0, p1):
            assert (b, p) not in covered
            covered[(b, p)] = c
    assert len(covered) == T
    slots = [c + b for c, b, _, _ in pieces]
    assert len(set(slots)) == len(slots)
    assert all(0 <= s < G + B - 1 for s in slots)
    for b, L in enumerate(lens):
        n = npages(L)
        if n == 0:
            continue
        c0 = worker_of_page(prefix[b], T, G)
        c1 = worker_of_page(prefix[b] + n - 1, T, G)
        # the combine visits workers c0..c1 and skips those with an empty page range
        visited = [c for c in range(c0, c1 + 1) if c * T // G < (c + 1) * T // G]
        assert sorted({c for c, bb, _, _ in pieces if bb == b}) == visited
    for g in range(T):
        c = worker_of_page(g, T, G)
        assert c * T // G <= g < (c + 1) * T // G
