"""GPU parity of jf_build_tree and jf_accept (through the C ABI) against the oracle: bit-exact tree
structure, tokens, depths, accepted lengths, paths and bonus tokens; scores within 1e-5."""
import numpy as np
import pytest
import torch

from oracle.accept import accept as oracle_accept
from oracle.build_tree import build_tree as oracle_build
from tree_verify_attention_jf_b200 import api, synth, workloads

pytestmark = pytest.mark.gpu

SCORE_ABS = 1e-5


def gpu_build(x, roots, topk, budget, max_depth):
    xt = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    rt = torch.from_numpy(np.ascontiguousarray(roots, dtype=np.int32)).cuda()
    res = api.build_tree(xt, rt, topk, budget, max_depth)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in res.items()}


def check_build(x, roots, topk, budget, max_depth, margin_guard=True):
    ref, margin = oracle_build(x, roots, topk, budget, max_depth, return_margin=True)
    if margin_guard:
        # the decision gaps are far above float64 rounding, so the pop order is unique
        assert margin.min() > 1e-9, margin
    got = gpu_build(x, roots, topk, budget, max_depth)
    np.testing.assert_array_equal(got["parent"], ref["parent"])
    np.testing.assert_array_equal(got["token"], ref["token"])
    np.testing.assert_array_equal(got["depth"], ref["depth"])
    np.testing.assert_allclose(got["score"], ref["score"], rtol=0, atol=SCORE_ABS)
    return got, ref


def test_build_full_workload():
    x, roots = workloads.build_inputs()
    check_build(x, roots, 4, 256, 16)


@pytest.mark.parametrize("V,topk,budget,max_depth,depths", [
    (1000, 4, 64, 8, 8), (37, 3, 40, 5, 6), (8193, 8, 300, 12, 16), (20000, 1, 17, 16, 16),
    (50, 2, 1, 3, 3), (5000, 5, 6, 4, 4), (3000, 4, 1024, 40, 40),
])
def test_build_shapes(V, topk, budget, max_depth, depths):
    x, roots = synth.draft_logits(V + topk, 3, depths, V, plant=min(8, V))
    check_build(x, roots, topk, budget, max_depth)


def test_build_ties_follow_the_tie_break():
    # every row flat: all candidates of a depth tie, so (depth, parent, rank) order decides
    x = np.zeros((2, 4, 64), dtype=np.float32)
    x[1, 2] = 1.5
    check_build(x, np.array([3, 4]), 3, 40, 4, margin_guard=False)


def test_build_ties_across_chunks():
    # three logit values over a five-chunk vocabulary: thousands of equal maxima per row, in every lane and
    # chunk, so the per-warp top-k filter and the (logit desc, id asc) tie-break decide the children; every
    # depth-1 node ties, so (parent position, rank) orders depth 2.  Depths stay far apart in key.
    rng = np.random.default_rng(5)
    x = rng.integers(0, 3, size=(2, 4, 20000)).astype(np.float32)
    got, ref = check_build(x, np.array([1, 2]), 4, 21, 3, margin_guard=False)
    assert (got["depth"] == 2).sum() == 2 * 16


@pytest.mark.parametrize("hot", [40, 300, 700])
def test_build_many_tied_maxima_per_chunk(hot):
    # `hot` entries of every 4096-entry chunk share the row's largest logit, so that tens to hundreds of
    # elements per chunk pass the per-warp filter (700 is more than a chunk's candidate list holds); the
    # lowest ids among them must win
    rng = np.random.default_rng(11 + hot)
    V = 20000
    x = rng.normal(0.0, 2.0, size=(2, 4, V)).astype(np.float32)
    for c0 in range(0, V, 4096):
        n = min(4096, V - c0)
        for b in range(2):
            for d in range(4):
                idx = c0 + rng.choice(n, size=min(hot, n), replace=False)
                x[b, d, idx] = 12.0 + d
    check_build(x, np.array([1, 2]), 4, 60, 4, margin_guard=False)


def gpu_accept(tok, par, tgt, max_depth):
    res = api.accept(torch.from_numpy(np.ascontiguousarray(tok, dtype=np.int32)).cuda(),
                     torch.from_numpy(np.ascontiguousarray(par, dtype=np.int32)).cuda(),
                     torch.from_numpy(np.ascontiguousarray(tgt)).cuda(), max_depth)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in res.items()}


def test_accept_full_workload():
    x, roots = workloads.build_inputs()
    tree = oracle_build(x, roots, 4, 256, 16)
    tgt, paths = synth.target_logits_with_path(55, tree["parent"], tree["token"], synth.VOCAB)
    acc, path, bonus = oracle_accept(tree["token"], tree["parent"], tgt, 16)
    got = gpu_accept(tree["token"], tree["parent"], tgt, 16)
    np.testing.assert_array_equal(got["accepted_len"], acc)
    np.testing.assert_array_equal(got["path"], path)
    np.testing.assert_array_equal(got["bonus"], bonus)
    assert [len(p) - 1 for p in paths] == acc.tolist()


@pytest.mark.parametrize("seed", range(6))
def test_accept_random_small(seed):
    rng = np.random.default_rng(seed)
    B, N, V = 3, int(rng.integers(1, 300)), int(rng.integers(2, 40))
    par = np.stack([synth.bushy_tree(rng, N, 4, 12) for _ in range(B)])
    tok = rng.integers(0, V, size=(B, N)).astype(np.int32)
    tgt = rng.integers(0, 3, size=(B, N, V)).astype(np.float32)  # many ties: lowest id wins
    for md in (0, 3, 12):
        acc, path, bonus = oracle_accept(tok, par, tgt, md)
        got = gpu_accept(tok, par, tgt, md)
        np.testing.assert_array_equal(got["accepted_len"], acc)
        np.testing.assert_array_equal(got["path"], path)
        np.testing.assert_array_equal(got["bonus"], bonus)


def test_accept_flags_bad_parent():
    par = np.array([[-1, 0, 5, 1]], dtype=np.int32)
    tok = np.zeros((1, 4), dtype=np.int32)
    tgt = np.zeros((1, 4, 8), dtype=np.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = dict(accepted_len=torch.full((1,), -7, dtype=torch.int32, device="cuda"),
               path=torch.full((1, 4), -7, dtype=torch.int32, device="cuda"),
               bonus=torch.full((1,), -7, dtype=torch.int32, device="cuda"))
    api.accept(torch.from_numpy(tok).cuda(), torch.from_numpy(par).cuda(), torch.from_numpy(tgt).cuda(), 3, out=out,
               dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
    assert int(out["accepted_len"].item()) == -7


def test_pipeline_build_attend_accept():
    """The whole hot path on the device: build the tree, attend over it, walk the accepted path."""
    V = 4096
    x, roots = synth.draft_logits(77, 2, 16, V)
    tree = check_build(x, roots, 4, 64, 16)[0]
    # attention over the built trees (node 0 hangs off the prefix; local parents as built)
    pars = [tree["parent"][b] for b in range(2)]
    inp = synth.attention_inputs(78, 32, 8, [700, 1500], pars, interleave=True)
    from tests.gpu_util import compare, run_attention
    from oracle.tree_attention import tree_attention_inputs
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)
    tgt, paths = synth.target_logits_with_path(79, tree["parent"], tree["token"], V)
    got = gpu_accept(tree["token"], tree["parent"], tgt, 16)
    assert got["accepted_len"].tolist() == [len(p) - 1 for p in paths]


def test_build_and_accept_replay_in_a_cuda_graph():
    """jf_build_tree (two launches) and jf_accept (a cluster launch) are capturable; a replay on fresh draft
    logits written into the captured buffer gives the oracle's tree and accepted path."""
    V, B = 8192, 3
    x1, roots = synth.draft_logits(91, B, 16, V)
    x2, _ = synth.draft_logits(92, B, 16, V)
    xt = torch.from_numpy(np.ascontiguousarray(x1)).cuda()
    rt = torch.from_numpy(np.ascontiguousarray(roots, dtype=np.int32)).cuda()
    ws = api.build_tree_workspace(B, 16, V, 4, "cuda")
    tree = api.build_tree(xt, rt, 4, 128, 16, workspace=ws)
    torch.cuda.synchronize()
    ref2 = oracle_build(x2, roots, 4, 128, 16)
    tgt_np, paths = synth.target_logits_with_path(93, ref2["parent"], ref2["token"], V)
    tgt = torch.from_numpy(tgt_np).cuda()
    acc = dict(accepted_len=torch.empty(B, dtype=torch.int32, device="cuda"),
               path=torch.empty(B, 17, dtype=torch.int32, device="cuda"),
               bonus=torch.empty(B, dtype=torch.int32, device="cuda"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        api.build_tree(xt, rt, 4, 128, 16, workspace=ws, out=tree)
        api.accept(tree["token"], tree["parent"], tgt, 16, out=acc)
    xt.copy_(torch.from_numpy(np.ascontiguousarray(x2)))
    g.replay()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(tree["parent"].cpu().numpy(), ref2["parent"])
    np.testing.assert_array_equal(tree["token"].cpu().numpy(), ref2["token"])
    ref_len, ref_path, ref_bonus = oracle_accept(ref2["token"], ref2["parent"], tgt_np, 16)
    np.testing.assert_array_equal(acc["accepted_len"].cpu().numpy(), ref_len)
    np.testing.assert_array_equal(acc["path"].cpu().numpy(), ref_path)
    np.testing.assert_array_equal(acc["bonus"].cpu().numpy(), ref_bonus)
    assert acc["accepted_len"].cpu().tolist() == [len(p) - 1 for p in paths]
