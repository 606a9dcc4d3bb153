"""GPU parity of jf_tree_attention (through the C ABI) against the float64 oracle."""
import numpy as np
import pytest
import torch

from oracle.tree_attention import tree_attention_inputs
from tests.gpu_util import compare, run_attention, to_dev
from tree_verify_attention_jf_b200 import api, synth, workloads

pytestmark = pytest.mark.gpu


def test_tiny_workload():
    inp = workloads.attention_workload("tiny")
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)


@pytest.mark.parametrize("group", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("P", [0, 1, 15, 16, 17, 31, 130])
def test_mask_probes_planted_values(group, P):
    """Small prefixes so tree slots carry real weight; V = 8 e_j on tree slot j makes every ancestor's
    contribution visible in its own coordinate.  Ragged node counts across the batch."""
    rng = np.random.default_rng(100 + P * 17 + group)
    nodes = [1, 16, 64, 256] if group <= 4 else [1, 16, 64, 200]
    pars = [synth.uniform_parent_tree(rng, n, 12) for n in nodes]
    hkv = 2
    inp = synth.attention_inputs(200 + P + group, hkv * group, hkv, [P + i for i in range(len(nodes))], pars,
                                 interleave=True)
    inp = synth.plant_tree_values(inp, magnitude=2.0, base_scale=0.5, seed=P)
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)


@pytest.mark.parametrize("P", [0, 17, 130, 4000])
@pytest.mark.parametrize("group", [4, 8])
def test_mask_exact_with_uniform_weights(group, P):
    """Zero queries make every visible key weigh exactly 1/|visible|; with V = 2 e_j on tree slot j and
    zero prefix values, coordinate j of a node's output is 2/(P + depth) when j is on its path and 0
    otherwise.  A relative bound of 2^-8 then exposes any mask error at any prefix length (the
    absolute tolerance alone cannot at long prefixes)."""
    rng = np.random.default_rng(300 + P + group)
    pars = [synth.uniform_parent_tree(rng, n, 14) for n in (256, 33, 100)]
    inp = synth.attention_inputs(400 + P + group, 2 * group, 2, [P, P + 3, P + 16], pars, interleave=True)
    inp = synth.plant_tree_values(inp, magnitude=2.0, base_scale=0.0, seed=1)
    inp.q[:] = 0.0
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    np.testing.assert_allclose(out, ref, rtol=2 ** -8, atol=1e-7)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-4)


def test_chain_and_deep_tree():
    par = synth.chain_tree(256)
    inp = synth.attention_inputs(7, 8, 2, [33], [par])
    inp = synth.plant_tree_values(inp, magnitude=2.0, base_scale=0.5, seed=3)
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)


def test_star_at_empty_prefix_is_exact():
    inp = synth.attention_inputs(8, 4, 1, [0, 0], [synth.star_tree(50), synth.star_tree(7)])
    out, _ = run_attention(inp)
    for b in range(2):
        o = int(inp.tree_offsets[b])
        for n in range(int(inp.tree_offsets[b + 1]) - o):
            slot = n
            page = int(inp.block_table[b, slot // 16])
            v = inp.v_cache[page, slot % 16, 0]
            np.testing.assert_array_equal(out[o + n], np.broadcast_to(v, (4, 128)))


def test_page_permutation_is_bit_identical():
    inp = workloads.attention_workload("tiny")
    out1, lse1 = run_attention(inp)
    rng = np.random.default_rng(5)
    perm = rng.permutation(inp.k_cache.shape[0])
    inv = np.argsort(perm)
    bt = inp.block_table.copy()
    bt[bt >= 0] = inv[bt[bt >= 0]]
    import dataclasses
    inp2 = dataclasses.replace(inp, k_cache=inp.k_cache[perm], v_cache=inp.v_cache[perm], block_table=bt)
    out2, lse2 = run_attention(inp2)
    np.testing.assert_array_equal(out1, out2)
    np.testing.assert_array_equal(lse1, lse2)


def test_nan_in_unused_cache_slots_does_not_leak():
    inp = synth.attention_inputs(9, 4, 1, [20], [synth.uniform_parent_tree(np.random.default_rng(9), 10, 5)])
    # slots 30..31 of the last used page are past the sequence: poison them
    k = inp.k_cache.copy()
    v = inp.v_cache.copy()
    page = int(inp.block_table[0, 1])
    k[page, 14:] = np.nan
    v[page, 14:] = np.nan
    import dataclasses
    inp2 = dataclasses.replace(inp, k_cache=k, v_cache=v)
    out, lse = run_attention(inp2)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)


@pytest.mark.parametrize("name", ["qwen3_8b", "serving"])
def test_full_size_workloads(name):
    inp = workloads.attention_workload(name)
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)


def test_qwen3_30b_whole_workload():
    """Every row of the Qwen3-30B-A3B workload (4 sequences x 256 nodes x 32 q heads over 32768-token prefixes):
    every (sequence, kv head) unit is cut between several CTAs, so this covers the split partials and their
    merge at full length."""
    inp = workloads.attention_workload("qwen3_30b_a3b")
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)


def test_qwen3_30b_exact_mask_probe():
    """The exact uniform-weight probe at the Qwen3-30B-A3B shape (g = 8, P = 32768, 256-node bushy trees):
    zero queries weigh every visible key 1/|visible| exactly, prefix V is zero and tree slot j carries 2 e_j, so
    coordinate j of a node's output is nonzero exactly when j is on its root path.  At this prefix length a mask
    error moves an output by far less than the absolute tolerance; the relative bound 2^-8 still exposes it."""
    inp = workloads.attention_workload("qwen3_30b_a3b")
    inp = synth.plant_tree_values(inp, magnitude=2.0, base_scale=0.0, seed=4)
    inp.q[:] = 0.0
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    assert (ref != 0).sum() > 0
    np.testing.assert_allclose(out, ref, rtol=2 ** -8, atol=1e-9)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-4)


def test_max_batch_ragged_with_empty_sequences():
    """The largest batch the call takes (1024 sequences) with ragged trees of 0..8 nodes, about a quarter of the
    sequences empty, over prefixes of 0..300 tokens in one interleaved page pool, g = 4: every row against the
    oracle."""
    rng = np.random.default_rng(31)
    B = 1024
    ns = rng.integers(0, 9, size=B)
    ns[rng.random(B) < 0.25] = 0
    prefix = rng.integers(0, 301, size=B)
    parents = [synth.uniform_parent_tree(rng, int(n), 4) for n in ns]
    inp = synth.attention_inputs(32, 8, 2, [int(p) for p in prefix], parents, interleave=True)
    assert (ns == 0).sum() > 200 and inp.q.shape[0] == ns.sum()
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)


def test_one_unit_cut_over_every_cta():
    """One sequence, one kv head with g = 4 and 16 nodes (a single unit of 64 rows) over a 131072-token prefix: the
    unit's 1025 kv tiles are split over every CTA, and the combine merges one segment from each of them."""
    rng = np.random.default_rng(33)
    inp = synth.attention_inputs(34, 4, 1, [131072], [synth.bushy_tree(rng, 16)])
    out, lse = run_attention(inp)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out, ref, lse, lse_ref)


def test_workspace_reuse_and_determinism():
    """One workspace, never initialised, serves calls with different splits in turn (the Qwen3-8B workload cuts
    each unit over about five CTAs, the serving workload over two): what one call leaves there never leaks into
    the next, and a repeated call gives the same bits (the merge order is fixed)."""
    inp = workloads.attention_workload("qwen3_8b")
    srv = workloads.attention_workload("serving")
    ws = api.AttentionWorkspace(torch.device("cuda"))
    ws.buf.fill_(0x5A)  # the workspace needs no initialisation
    d, ds = to_dev(inp), to_dev(srv)
    a, la = run_attention(inp, ws=ws, dev=d)
    s1, ls1 = run_attention(srv, ws=ws, dev=ds)
    b, lb = run_attention(inp, ws=ws, dev=d)
    s2, ls2 = run_attention(srv, ws=ws, dev=ds)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(ls1, ls2)
    ref, lse_ref = tree_attention_inputs(inp)
    compare(b, ref, lb, lse_ref)


def test_cuda_graph_replay_matches_eager():
    """The call is capturable in a CUDA graph (the attention launch and the combine launch that follows it
    with a programmatic dependency); replays give the eager result bit for bit."""
    inp = workloads.attention_workload("qwen3_8b")
    ws = api.AttentionWorkspace(torch.device("cuda"))
    d = to_dev(inp)
    eager, eager_lse = run_attention(inp, ws=ws, dev=d)
    T, Hq = inp.q.shape[:2]
    out = torch.full_like(d["q"], float("nan"))
    lse = torch.full((T, Hq), float("nan"), dtype=torch.float32, device="cuda")

    def call():
        api.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["prefix_lens"],
                           d["tree_offsets"], d["parent"], inp.sm_scale, out=out, lse=lse, workspace=ws)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        call()
    for _ in range(3):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.float().cpu().numpy(), eager)
        np.testing.assert_array_equal(lse.cpu().numpy(), eager_lse)


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def test_device_checks_flag_bad_sequences_only():
    rng = np.random.default_rng(11)
    pars = [synth.uniform_parent_tree(rng, n, 6) for n in (12, 20, 9)]
    inp = synth.attention_inputs(12, 8, 2, [40, 300, 17], pars, interleave=True)
    ref, lse_ref = tree_attention_inputs(inp)
    # 1. a parent index out of range in sequence 1
    bad = inp.parent.copy()
    bad[12 + 5] = 7  # parent[5] = 7 >= 5
    import dataclasses
    st = _status()
    out, lse = run_attention(dataclasses.replace(inp, parent=bad), status=st)
    assert int(st.item()) == 4
    assert np.isnan(out[12:32]).all()  # untouched
    for sl in (slice(0, 12), slice(32, 41)):
        compare(out[sl], ref[sl], lse[sl], lse_ref[sl])
    # 2. a page id out of range in sequence 2
    bt = inp.block_table.copy()
    bt[2, 0] = 10 ** 6
    st = _status()
    out, _ = run_attention(dataclasses.replace(inp, block_table=bt), status=st)
    assert int(st.item()) == 4
    assert np.isnan(out[32:41]).all()
    compare(out[0:32], ref[0:32])
    # 3. malformed tree_offsets: nothing is computed
    offs = inp.tree_offsets.copy()
    offs[1] = 50
    st = _status()
    out, _ = run_attention(dataclasses.replace(inp, tree_offsets=offs), status=st)
    assert int(st.item()) == 4
    assert np.isnan(out).all()


def test_capacity_overflow_flagged():
    inp = synth.attention_inputs(13, 4, 1, [40], [synth.chain_tree(10)])
    import dataclasses
    st = _status()
    # claim a longer prefix than the block table can hold: 3 pages x 16 = 48 < 60 + 10
    out, _ = run_attention(dataclasses.replace(inp, prefix_lens=np.array([60], np.int32)), status=st)
    assert int(st.item()) == 4
    assert np.isnan(out).all()
