"""Pins of the KV-commit oracle (oracle/commit_kv.py) against a hand-worked example, a dense formulation and the
meaning of the result (the committed cache reads as the accepted text)."""
import numpy as np
import pytest

from oracle.accept import accept
from oracle.commit_kv import commit_kv
from tree_verify_attention_jf_b200 import synth


def test_hand_worked_example():
    # one sequence, 1 kv head, 2 dims; logical page 0 -> physical page 1, logical page 1 -> physical page 0.
    # prefix 14, tree of 5 nodes at slots 14..18; accepted path [0, 2, 4] (L = 2).
    k = np.zeros((2, 16, 1, 2), np.float32)
    for pg in range(2):
        for off in range(16):
            k[pg, off, 0] = [100 * pg + off + 1, -(100 * pg + off + 1)]
    v = 2 * k
    k0, v0 = k.copy(), v.copy()
    bt = np.array([[1, 0]])
    kk, vv, newp = commit_kv(k, v, bt, [14], [0, 5], [[0, 2, 4]], [2])
    # slot 15 (page 1, offset 15) <- slot 16 (page 0, offset 0), whose K is [1, -1]
    # slot 16 (page 0, offset 0)  <- slot 18 (page 0, offset 2), whose K is [3, -3]
    assert kk[1, 15, 0].tolist() == [1.0, -1.0] and vv[1, 15, 0].tolist() == [2.0, -2.0]
    assert kk[0, 0, 0].tolist() == [3.0, -3.0] and vv[0, 0, 0].tolist() == [6.0, -6.0]
    changed = np.argwhere(np.any(kk != k, axis=(2, 3)))
    assert sorted(map(tuple, changed.tolist())) == [(0, 0), (1, 15)]
    assert newp.tolist() == [17]
    assert np.array_equal(k, k0) and np.array_equal(v, v0)  # inputs untouched


def rooted_tree(rng, n, max_depth):
    """parent[0] = -1; parent[i] uniform over the earlier nodes shallower than max_depth."""
    par = -np.ones(n, np.int64)
    depth = np.zeros(n, np.int64)
    for i in range(1, n):
        allowed = [j for j in range(i) if depth[j] < max_depth]
        par[i] = allowed[int(rng.integers(len(allowed)))]
        depth[i] = depth[par[i]] + 1
    return par


def random_case(seed, B=3, H=2, D=4, max_depth=6):
    rng = np.random.default_rng(seed)
    prefix = rng.integers(0, 40, B)
    nodes = rng.integers(0, 30, B)
    offsets = np.concatenate([[0], np.cumsum(nodes)])
    pages_per = [(int(p) + int(n) + 15) // 16 for p, n in zip(prefix, nodes)]
    npages = sum(pages_per) + 3
    perm = rng.permutation(npages)
    bt = np.zeros((B, max(pages_per) + 1), np.int64)
    c = 0
    for b in range(B):
        bt[b, :pages_per[b]] = perm[c:c + pages_per[b]]
        c += pages_per[b]
    k = rng.standard_normal((npages, 16, H, D)).astype(np.float32)
    v = rng.standard_normal((npages, 16, H, D)).astype(np.float32)
    path = -np.ones((B, max_depth + 1), np.int64)
    L = np.zeros(B, np.int64)
    toks = []
    for b in range(B):
        n = int(nodes[b])
        par = rooted_tree(rng, n, max_depth)
        toks.append(rng.integers(0, 1000, n))
        if n == 0:
            continue
        end = int(rng.integers(0, n))
        pth = [end]
        while pth[-1] != 0:
            pth.append(int(par[pth[-1]]))
        pth.reverse()
        pth = pth[:max_depth + 1]
        L[b] = len(pth) - 1
        path[b, :len(pth)] = pth
    return k, v, bt, prefix, offsets, path, L, toks


@pytest.mark.parametrize("seed", range(12))
def test_matches_dense_formulation(seed):
    k, v, bt, prefix, offsets, path, L, _ = random_case(seed)
    kk, vv, newp = commit_kv(k, v, bt, prefix, offsets, path, L)
    exp_k, exp_v = k.copy(), v.copy()
    for b in range(len(prefix)):
        P, N = int(prefix[b]), int(offsets[b + 1] - offsets[b])
        n = P + N
        pg = bt[b][np.arange(n) // 16]
        off = np.arange(n) % 16
        dk, dv = k[pg, off].copy(), v[pg, off].copy()  # the sequence's slots, dense
        if N > 0:
            idx = P + path[b, 1:L[b] + 1]
            dk[P + 1:P + 1 + L[b]] = dk[idx]  # numpy reads the right side first
            dv[P + 1:P + 1 + L[b]] = dv[idx]
            m = P + 1 + L[b]
            exp_k[pg[:m], off[:m]] = dk[:m]
            exp_v[pg[:m], off[:m]] = dv[:m]
        assert newp[b] == (P + L[b] + 1 if N > 0 else P)
    assert np.array_equal(kk, exp_k) and np.array_equal(vv, exp_v)


@pytest.mark.parametrize("seed", range(6))
def test_committed_cache_reads_as_the_accepted_text(seed):
    # token ids ride along as cache values: the committed prefix must read prefix tokens, root, accepted tokens
    k, v, bt, prefix, offsets, path, L, toks = random_case(seed + 100, H=1, D=1)
    rng = np.random.default_rng(seed)
    seqs = []
    for b in range(len(prefix)):
        P, N = int(prefix[b]), int(offsets[b + 1] - offsets[b])
        text = np.concatenate([rng.integers(0, 1000, P), toks[b]]).astype(np.float32)
        for s in range(P + N):
            k[bt[b][s // 16], s % 16, 0, 0] = text[s]
        seqs.append(text)
    kk, _, newp = commit_kv(k, v, bt, prefix, offsets, path, L)
    for b in range(len(prefix)):
        P, N = int(prefix[b]), int(offsets[b + 1] - offsets[b])
        got = [kk[bt[b][s // 16], s % 16, 0, 0] for s in range(int(newp[b]))]
        want = list(seqs[b][:P]) + ([toks[b][j] for j in path[b, :L[b] + 1]] if N > 0 else [])
        assert got == want


def test_with_the_accept_oracle_walk():
    # the path comes from the accept oracle on a planted walk; the committed prefix holds the planted tokens
    rng = np.random.default_rng(3)
    N, V = 20, 50
    par = rooted_tree(rng, N, 6)
    tok = rng.integers(0, V, N)
    tgt, paths = synth.target_logits_with_path(4, par[None], tok[None], V)
    acc_len, path, _ = accept(tok[None], par[None], tgt, 6)
    k = np.zeros((4, 16, 1, 1), np.float32)
    bt = np.array([[2, 0, 3, 1]])
    P = 9
    for j in range(N):
        s = P + j
        k[bt[0][s // 16], s % 16, 0, 0] = tok[j]
    kk, _, newp = commit_kv(k, k.copy(), bt, [P], [0, N], path, acc_len)
    got = [kk[bt[0][s // 16], s % 16, 0, 0] for s in range(P, int(newp[0]))]
    assert got == [tok[j] for j in paths[0][:acc_len[0] + 1]]


def test_nothing_accepted_and_empty_tree_leave_the_cache():
    k, v, bt, prefix, offsets, path, L, _ = random_case(7)
    L0 = np.zeros_like(L)
    kk, vv, newp = commit_kv(k, v, bt, prefix, offsets, path, L0)
    assert np.array_equal(kk, k) and np.array_equal(vv, v)
    nodes = np.diff(offsets)
    assert newp.tolist() == [int(p) + (1 if n > 0 else 0) for p, n in zip(prefix, nodes)]


def test_sources_that_are_later_destinations():
    # path [0, 2, 3]: slot P+2 is copy 1's source and copy 2's destination
    k = np.arange(2 * 16 * 1 * 1, dtype=np.float32).reshape(2, 16, 1, 1)
    bt = np.array([[0, 1]])
    kk, _, _ = commit_kv(k, k.copy(), bt, [5], [0, 6], [[0, 2, 3]], [2])
    assert kk[0, 6, 0, 0] == 7 and kk[0, 7, 0, 0] == 8
