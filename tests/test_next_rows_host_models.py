"""Host models of the index logic of the two cache-write kernels (the same integer steps as the device code):

* jf_commit_kv moves the accepted rows in passes of `ch` copies, each pass reading all of its sources before
  writing any destination; for every strictly increasing path and every pass size this equals the oracle;
* jf_tree_kv_append finds a node's sequence by a binary search for the last sequence whose first node is at or
  before it; with empty sequences in the batch this must still give the sequence that holds the node."""
import numpy as np
import pytest

from oracle.commit_kv import commit_kv


def commit_in_passes(dense, P, path, L, ch):
    """The kernel's pass structure on one sequence's dense slot array."""
    out = dense.copy()
    for i0 in range(1, L + 1, ch):
        n = min(ch, L + 1 - i0)
        staged = [out[P + path[i0 + c]].copy() for c in range(n)]  # phase 1: every source of the pass
        for c in range(n):                                          # phase 2: every destination
            out[P + i0 + c] = staged[c]
    return out


@pytest.mark.parametrize("ch", [1, 2, 3, 4, 8, 64])
def test_commit_passes_equal_the_oracle(ch):
    rng = np.random.default_rng(ch)
    for _ in range(300):
        N = int(rng.integers(2, 40))
        P = int(rng.integers(0, 20))
        L = int(rng.integers(0, N))
        path = [0] + sorted(rng.choice(np.arange(1, N), size=L, replace=False).tolist())
        dense = rng.standard_normal((P + N, 2))
        got = commit_in_passes(dense, P, path, L, ch)
        npages = (P + N + 15) // 16
        cache = np.zeros((npages, 16, 1, 2))
        for s_ in range(P + N):
            cache[s_ // 16, s_ % 16, 0] = dense[s_]
        kk, _, _ = commit_kv(cache, cache, np.arange(npages)[None], [P], [0, N], [path], [L])
        want = np.array([kk[s_ // 16, s_ % 16, 0] for s_ in range(P + L + 1)])
        assert np.array_equal(got[:P + L + 1], want)


def find_sequence(offsets, t):
    """The kernel's search: the last b in [0, B) with offsets[b] <= t, then a containment check."""
    B = len(offsets) - 1
    lo, hi = 0, B - 1
    while lo < hi:
        mid = (lo + hi + 1) >> 1
        if offsets[mid] <= t:
            lo = mid
        else:
            hi = mid - 1
    return lo if offsets[lo] <= t < offsets[lo + 1] else -1


def test_sequence_search_with_empty_sequences():
    rng = np.random.default_rng(0)
    for _ in range(500):
        B = int(rng.integers(1, 12))
        nodes = rng.integers(0, 4, B)
        nodes[int(rng.integers(B))] += 1
        offsets = np.concatenate([[0], np.cumsum(nodes)])
        for t in range(int(offsets[-1])):
            b = find_sequence(offsets, t)
            assert b >= 0 and offsets[b] <= t < offsets[b + 1]
