"""Pins for oracle.tree_attention against things other than itself:
torch SDPA (float64, CPU) on contiguous sequences that the test scatters into pages, closed forms
(star at P=0, zero queries), and invariances (page permutation, relabelling, unrelated branch)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle.tree_attention import tree_attention, ancestor_sets
from tree_verify_attention_jf_b200 import synth

PAGE = 16


def paged_from_sequences(rng, kseq, vseq, hkv, d, shuffle=True, spare=3):
    """Scatter contiguous per-sequence K/V [L_b, Hkv, D] into a shared page pool: logical slot t of
    sequence b goes to page bt[b][t // 16], row t % 16.  Written independently of the oracle's gather."""
    npages = [(k.shape[0] + PAGE - 1) // PAGE for k in kseq]
    total = sum(npages) + spare
    ids = rng.permutation(total) if shuffle else np.arange(total)
    kc = rng.standard_normal((total, PAGE, hkv, d)) * 50.0  # garbage in unused rows/pages
    vc = rng.standard_normal((total, PAGE, hkv, d)) * 50.0
    bt = np.full((len(kseq), max(npages)), -1, dtype=np.int32)
    pos = 0
    for b, (k, v) in enumerate(zip(kseq, vseq)):
        for lp in range(npages[b]):
            phys = int(ids[pos]); pos += 1
            bt[b, lp] = phys
            lo, hi = lp * PAGE, min((lp + 1) * PAGE, k.shape[0])
            kc[phys, :hi - lo] = k[lo:hi]
            vc[phys, :hi - lo] = v[lo:hi]
    return kc, vc, bt


def sdpa_one(qv, K, V, scale):
    """One query row [Hq, D] against keys [L, Hkv, D] with torch SDPA (float64), GQA by repeat."""
    hq, hkv = qv.shape[0], K.shape[1]
    g = hq // hkv
    qt = torch.from_numpy(qv).double()[:, None, :]                     # [Hq, 1, D]
    kt = torch.from_numpy(K).double().permute(1, 0, 2).repeat_interleave(g, 0)  # [Hq, L, D]
    vt = torch.from_numpy(V).double().permute(1, 0, 2).repeat_interleave(g, 0)
    return F.scaled_dot_product_attention(qt, kt, vt, scale=scale)[:, 0, :].numpy()


def make_case(seed, prefix_lens, parents, hq=4, hkv=2, d=16):
    rng = np.random.default_rng(seed)
    kseq, vseq = [], []
    for P, par in zip(prefix_lens, parents):
        L = P + len(par)
        kseq.append(rng.standard_normal((L, hkv, d)))
        vseq.append(rng.standard_normal((L, hkv, d)))
    kc, vc, bt = paged_from_sequences(rng, kseq, vseq, hkv, d)
    T = sum(len(p) for p in parents)
    q = rng.standard_normal((T, hq, d))
    offs = np.concatenate([[0], np.cumsum([len(p) for p in parents])]).astype(np.int32)
    parent = np.concatenate(parents).astype(np.int32)
    return dict(q=q, k_cache=kc, v_cache=vc, block_table=bt, prefix_lens=np.array(prefix_lens, np.int32),
                tree_offsets=offs, parent=parent, sm_scale=0.3), kseq, vseq


def run(case, **kw):
    return tree_attention(case["q"], case["k_cache"], case["v_cache"], case["block_table"],
                          case["prefix_lens"], case["tree_offsets"], case["parent"], case["sm_scale"], **kw)


def root_path(par, v):
    path = []
    while v >= 0:
        path.append(v)
        v = int(par[v])
    return path[::-1]


def test_chain_equals_causal_attention():
    P, N = 37, 12
    case, kseq, vseq = make_case(1, [P], [synth.chain_tree(N)])
    out, _ = run(case)
    for n in range(N):
        ref = sdpa_one(case["q"][n], kseq[0][:P + n + 1], vseq[0][:P + n + 1], 0.3)
        np.testing.assert_allclose(out[n], ref, rtol=1e-12, atol=1e-12)


def test_star_at_empty_prefix_is_own_value():
    N = 9
    case, kseq, vseq = make_case(2, [0], [synth.star_tree(N)])
    out, lse = run(case)
    for n in range(N):
        for h in range(4):
            np.testing.assert_array_equal(out[n, h], vseq[0][n, h // 2])
            assert lse[n, h] == pytest.approx(0.3 * float(case["q"][n, h] @ kseq[0][n, h // 2]), abs=1e-12)


def test_star_equals_prefix_plus_self():
    P, N = 21, 7
    case, kseq, vseq = make_case(3, [P], [synth.star_tree(N)])
    out, _ = run(case)
    for n in range(N):
        idx = list(range(P)) + [P + n]
        ref = sdpa_one(case["q"][n], kseq[0][idx], vseq[0][idx], 0.3)
        np.testing.assert_allclose(out[n], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [4, 5, 6])
def test_path_extraction_branch_factorisation(seed):
    """out[v] == causal attention over prefix ++ path(v) at its last position, for every node, in a
    forest of random trees across a batch with ragged prefixes (including P = 0 and page-straddling)."""
    rng = np.random.default_rng(seed)
    prefix_lens = [0, 15, 33]
    parents = [synth.uniform_parent_tree(rng, n, 6) for n in (11, 20, 5)]
    case, kseq, vseq = make_case(seed, prefix_lens, parents)
    out, lse = run(case)
    for b, (P, par) in enumerate(zip(prefix_lens, parents)):
        o = int(case["tree_offsets"][b])
        for v in range(len(par)):
            idx = list(range(P)) + [P + u for u in root_path(par, v)]
            ref = sdpa_one(case["q"][o + v], kseq[b][idx], vseq[b][idx], 0.3)
            np.testing.assert_allclose(out[o + v], ref, rtol=1e-11, atol=1e-12)


def test_zero_queries_closed_form():
    """q = 0: every visible score is 0, so lse = ln(#visible) and out = mean of the visible values."""
    rng = np.random.default_rng(7)
    P = 19
    par = synth.uniform_parent_tree(rng, 14, 5)
    case, kseq, vseq = make_case(7, [P], [par])
    case["q"][:] = 0.0
    out, lse = run(case)
    for v in range(len(par)):
        path = root_path(par, v)
        np.testing.assert_allclose(lse[v], np.log(P + len(path)), rtol=0, atol=1e-13)
        idx = list(range(P)) + [P + u for u in path]
        mean = vseq[0][idx].mean(axis=0)  # [Hkv, D]
        np.testing.assert_allclose(out[v], np.repeat(mean, 2, axis=0), rtol=1e-12, atol=1e-13)


def test_page_permutation_invariance():
    rng = np.random.default_rng(8)
    par = synth.uniform_parent_tree(rng, 10, 4)
    case, _, _ = make_case(8, [40], [par])
    out1, lse1 = run(case)
    perm = rng.permutation(case["k_cache"].shape[0])
    inv = np.argsort(perm)
    case2 = dict(case)
    case2["k_cache"] = case["k_cache"][perm]
    case2["v_cache"] = case["v_cache"][perm]
    bt = case["block_table"].copy()
    bt[bt >= 0] = inv[bt[bt >= 0]]
    case2["block_table"] = bt
    out2, lse2 = run(case2)
    np.testing.assert_array_equal(out1, out2)
    np.testing.assert_array_equal(lse1, lse2)


def test_relabel_and_unrelated_branch():
    rng = np.random.default_rng(9)
    P = 24
    par = np.array([-1, 0, 0, 1, 1, 2, -1, 6], dtype=np.int32)
    case, kseq, vseq = make_case(9, [P], [par])
    out, _ = run(case)
    # Topological relabelling: swap the subtrees' order; K/V slots and queries move with the nodes.
    order = [0, 2, 1, 5, 3, 4, 6, 7]           # new index i holds old node order[i]
    newpos = {old: new for new, old in enumerate(order)}
    par2 = np.array([-1 if par[o] < 0 else newpos[int(par[o])] for o in order], dtype=np.int32)
    k2 = [np.concatenate([kseq[0][:P], kseq[0][P:][order]])]
    v2 = [np.concatenate([vseq[0][:P], vseq[0][P:][order]])]
    kc, vc, bt = paged_from_sequences(np.random.default_rng(1), k2, v2, 2, 16)
    case2 = dict(case, q=case["q"][order], k_cache=kc, v_cache=vc, block_table=bt, parent=par2)
    out2, _ = run(case2)
    np.testing.assert_allclose(out2, out[order], rtol=1e-12, atol=1e-13)
    # An extra branch appended at the end leaves every existing node unchanged.
    par3 = np.concatenate([par, [3, 8]]).astype(np.int32)
    extra = np.random.default_rng(2).standard_normal((2, 2, 16))
    k3 = [np.concatenate([kseq[0], extra])]
    v3 = [np.concatenate([vseq[0], -extra])]
    kc3, vc3, bt3 = paged_from_sequences(np.random.default_rng(3), k3, v3, 2, 16)
    q3 = np.concatenate([case["q"], np.random.default_rng(4).standard_normal((2, 4, 16))])
    case3 = dict(case, q=q3, k_cache=kc3, v_cache=vc3, block_table=bt3, parent=par3,
                 tree_offsets=np.array([0, 10], np.int32))
    out3, _ = run(case3)
    np.testing.assert_allclose(out3[:8], out, rtol=1e-12, atol=1e-13)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(10)
    par = synth.uniform_parent_tree(rng, 12, 5)
    case, _, _ = make_case(10, [30], [par])
    out, lse = run(case)
    rows = [(3, 1), (11, 0), (0, 3)]
    out_s, lse_s = run(case, rows=rows)
    for t, h in rows:
        np.testing.assert_allclose(out_s[t, h], out[t, h], rtol=1e-13, atol=1e-15)
        assert lse_s[t, h] == pytest.approx(lse[t, h], abs=1e-13)
    assert np.isnan(out_s[5, 2]).all()


def test_invalid_parent_rejected():
    with pytest.raises(ValueError):
        ancestor_sets(np.array([-1, 1], dtype=np.int32))
    with pytest.raises(ValueError):
        ancestor_sets(np.array([-2], dtype=np.int32))


def test_planted_values_show_ancestors():
    """Planted-V probe at a long prefix: with V = 8 e_j on tree slot j and zero queries, coordinate j
    of node n's output is 8 / (P + depth(n)) exactly when j is on n's path, and the prefix part alone
    otherwise."""
    inp = synth.attention_inputs(11, 4, 1, [64], [synth.uniform_parent_tree(np.random.default_rng(11), 16, 8)],
                                 head_dim=32)
    inp = synth.plant_tree_values(inp, magnitude=8.0, base_scale=0.0)
    inp.q[:] = 0.0
    out, _ = tree_attention(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.prefix_lens,
                            inp.tree_offsets, inp.parent, inp.sm_scale)
    par = inp.parent
    for v in range(16):
        path = set(root_path(par, v))
        for j in range(16):
            want = 8.0 / (64 + len(path)) if j in path else 0.0
            np.testing.assert_allclose(out[v, :, j], want, atol=1e-14)
