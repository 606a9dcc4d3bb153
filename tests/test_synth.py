"""The seeded generators: deterministic, bf16-exact, page pools are permutations, tree shapes hold."""
import numpy as np

from tree_verify_attention_jf_b200 import synth, workloads


def test_deterministic_and_bf16_exact():
    a = workloads.attention_workload("tiny")
    b = workloads.attention_workload("tiny")
    np.testing.assert_array_equal(a.q, b.q)
    np.testing.assert_array_equal(a.block_table, b.block_table)
    np.testing.assert_array_equal(synth.bf16_round(a.k_cache), a.k_cache)
    assert a.q.shape == (16, 4, 128) and a.k_cache.shape[1:] == (16, 1, 128)


def test_page_pool_is_permutation():
    bt, total = synth.page_pool(np.random.default_rng(0), [5, 3, 7], interleave=True)
    used = bt[bt >= 0]
    assert sorted(used.tolist()) == list(range(total))
    bt2, total2 = synth.page_pool(np.random.default_rng(0), [5, 3], interleave=False)
    assert sorted(bt2[0].tolist()) == list(range(5)) and sorted(bt2[1, :3].tolist()) == [5, 6, 7]


def test_tree_shapes():
    rng = np.random.default_rng(3)
    par = synth.bushy_tree(rng, 256, 4, 16)
    assert par[0] == -1 and all(0 <= par[i] < i for i in range(1, 256))
    assert np.bincount(par[1:], minlength=256).max() <= 4
    lvl = np.zeros(256, int)
    for i in range(1, 256):
        lvl[i] = lvl[par[i]] + 1
    assert lvl.max() <= 16
    par = synth.uniform_parent_tree(rng, 64, 12)
    dep = np.zeros(64, int)
    for i in range(64):
        dep[i] = 1 if par[i] < 0 else dep[par[i]] + 1
    assert dep.max() <= 12 and all(par[i] < i for i in range(64))


def test_serving_workload_shape():
    w = workloads.attention_workload("serving")
    assert w.batch == 16 and w.total_nodes == 16 * 64
    assert ((w.prefix_lens >= 1024) & (w.prefix_lens <= 8192)).all()


def test_draft_plant_is_top():
    x, roots = synth.draft_logits(1, 2, 3, 500)
    for b in range(2):
        for k in range(3):
            top8 = np.sort(x[b, k])[-8:]
            assert top8[-1] - np.sort(x[b, k])[-9] > 0.5
