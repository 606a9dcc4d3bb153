"""Pins of the tree-KV append oracle (oracle/kv_append.py): rotary identities, a hand-worked example, a
complex-number formulation, and where the nodes land in the paged cache."""
import numpy as np
import pytest

from oracle.kv_append import node_positions, rope, tree_kv_append


def test_position_zero_is_identity():
    x = np.random.default_rng(0).standard_normal((5, 128))
    assert np.array_equal(rope(x, np.zeros(5), 1e6), x)


def test_hand_worked_d4():
    # d = 4: pairs (0, 2) and (1, 3); angles pos * [1, theta^-1/2].  x = e0 at pos = pi/2 goes to e2 (the first
    # pair turns by pi/2); x = e1 at pos = pi/2 with theta = 10^4 turns by 0.01 * pi/2.
    got = rope([1.0, 0.0, 0.0, 0.0], np.pi / 2, 1e4)
    assert np.allclose(got, [0.0, 0.0, 1.0, 0.0], atol=1e-15)
    got = rope([0.0, 1.0, 0.0, 0.0], np.pi / 2, 1e4)
    a = 0.01 * np.pi / 2
    assert np.allclose(got, [0.0, np.cos(a), 0.0, np.sin(a)], atol=1e-15)


def test_pair_norms_are_kept():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 128))
    y = rope(x, rng.integers(0, 100000, 7), 1e6)
    n = lambda z: z[:, :64] ** 2 + z[:, 64:] ** 2
    assert np.allclose(n(y), n(x), rtol=1e-12)


def test_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for m, n, s in [(5, 3, 100), (1000, 17, 40000), (0, 0, 7)]:
        a = rope(q, m, 1e6) @ rope(k, n, 1e6)
        b = rope(q, m + s, 1e6) @ rope(k, n + s, 1e6)
        assert abs(a - b) < 1e-9 * max(1.0, abs(a))


@pytest.mark.parametrize("theta", [1e4, 1e6])
def test_matches_complex_formulation(theta):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((9, 3, 128))
    pos = rng.integers(0, 50000, 9)
    z = x[..., :64] + 1j * x[..., 64:]
    freq = theta ** (-np.arange(64) / 64.0)            # theta^(-2i/d) with d = 128
    w = z * np.exp(1j * pos[:, None, None] * freq)
    want = np.concatenate([w.real, w.imag], axis=-1)
    assert np.allclose(rope(x, pos[:, None], theta), want, atol=1e-9)


def test_nodes_land_in_their_slots_with_their_positions():
    rng = np.random.default_rng(4)
    B, H, Hq, d = 2, 2, 4, 128
    prefix = np.array([5, 20])
    nodes = np.array([4, 13])
    offsets = np.concatenate([[0], np.cumsum(nodes)])
    depth = np.concatenate([[0, 1, 1, 2], [0, 1, 2, 3, 1, 2, 2, 3, 4, 1, 2, 3, 5]])
    bt = np.array([[3, 1, 0], [2, 4, 5]])
    kc = rng.standard_normal((6, 16, H, d))
    vc = rng.standard_normal((6, 16, H, d))
    kn = rng.standard_normal((offsets[-1], H, d))
    vn = rng.standard_normal((offsets[-1], H, d))
    q = rng.standard_normal((offsets[-1], Hq, d))
    k2, v2, q2 = tree_kv_append(kn, vn, q, kc, vc, bt, prefix, offsets, depth, 1e6)
    assert node_positions(prefix, offsets, depth).tolist() == (prefix[0] + depth[:4]).tolist() + \
        (prefix[1] + depth[4:]).tolist()
    touched = set()
    for b in range(B):
        for j in range(nodes[b]):
            t, s = offsets[b] + j, prefix[b] + j
            pg, off = bt[b][s // 16], s % 16
            touched.add((pg, off))
            pos = prefix[b] + depth[t]
            z = (kn[t, :, :64] + 1j * kn[t, :, 64:]) * np.exp(1j * pos * 1e6 ** (-np.arange(64) / 64.0))
            assert np.allclose(k2[pg, off], np.concatenate([z.real, z.imag], axis=-1), atol=1e-9)
            assert np.array_equal(v2[pg, off], vn[t])
            zq = (q[t, :, :64] + 1j * q[t, :, 64:]) * np.exp(1j * pos * 1e6 ** (-np.arange(64) / 64.0))
            assert np.allclose(q2[t], np.concatenate([zq.real, zq.imag], axis=-1), atol=1e-9)
    for pg in range(6):
        for off in range(16):
            if (pg, off) not in touched:
                assert np.array_equal(k2[pg, off], kc[pg, off]) and np.array_equal(v2[pg, off], vc[pg, off])
