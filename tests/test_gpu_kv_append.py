"""GPU parity of jf_tree_kv_append (through the C ABI) against the float64 oracle rounded once to bf16: rotated K
and q, V byte for byte, untouched slots unchanged, positions up to 10^5, device checks, CUDA-graph replay."""
import numpy as np
import pytest
import torch

from oracle.kv_append import tree_kv_append as oracle_append
from tests.test_oracle_commit import rooted_tree
from tree_verify_attention_jf_b200 import api

pytestmark = pytest.mark.gpu


def bf16_rne(x):
    """float64 -> nearest bf16 value (ties to even), as float64."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def bf16_bits_to_f64(a):
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_bf16(rng, shape):
    x = rng.standard_normal(shape).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)  # truncation to bf16 bits; any bf16 values will do


def make_case(seed, B, Hkv, Hq, max_prefix=200, max_nodes=40, big_prefix=None):
    rng = np.random.default_rng(seed)
    prefix = rng.integers(0, max_prefix, B) if big_prefix is None else np.full(B, big_prefix)
    nodes = rng.integers(1, max_nodes, B)
    offsets = np.concatenate([[0], np.cumsum(nodes)]).astype(np.int32)
    depth = np.concatenate([_depths(rooted_tree(rng, int(n), 16)) for n in nodes]).astype(np.int32)
    pages_per = [(int(p) + int(n) + 15) // 16 for p, n in zip(prefix, nodes)]
    npages = sum(pages_per) + 2
    perm = rng.permutation(npages)
    bt = np.zeros((B, max(pages_per) + 1), np.int32)
    c = 0
    for b in range(B):
        bt[b, :pages_per[b]] = perm[c:c + pages_per[b]]
        c += pages_per[b]
    T = int(offsets[-1])
    return dict(kc=rand_bf16(rng, (npages, 16, Hkv, 128)), vc=rand_bf16(rng, (npages, 16, Hkv, 128)),
                kn=rand_bf16(rng, (T, Hkv, 128)), vn=rand_bf16(rng, (T, Hkv, 128)), q=rand_bf16(rng, (T, Hq, 128)),
                bt=bt, prefix=prefix.astype(np.int32), offsets=offsets, depth=depth)


def _depths(par):
    d = np.zeros(len(par), np.int64)
    for i in range(1, len(par)):
        d[i] = d[par[i]] + 1
    return d


def dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run(c, theta, with_q=True, status=None):
    d = {k: dev(v) for k, v in c.items()}
    api.tree_kv_append(d["kn"], d["vn"], d["kc"], d["vc"], d["bt"], d["prefix"], d["offsets"], d["depth"], theta,
                       q=d["q"] if with_q else None, dev_status=status)
    torch.cuda.synchronize()
    return bits(d["kc"]), bits(d["vc"]), bits(d["q"])


def check(c, theta, got):
    kk, vv, qq = got
    f = bf16_bits_to_f64
    rk, rv, rq = oracle_append(f(c["kn"]), f(c["vn"]), f(c["q"]), f(c["kc"]), f(c["vc"]), c["bt"], c["prefix"],
                               c["offsets"], c["depth"], theta)
    assert np.array_equal(vv, (rv.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))
    for got_bits, ref in ((kk, rk), (qq, rq)):
        want = bf16_rne(ref)
        g = f(got_bits)
        diff = g != want
        # one rounding from float64 each side: only a tie decided differently by the last bits of cos/sin could
        # differ, by one bf16 step
        assert diff.mean() < 1e-4, diff.mean()
        ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(want), 1e-30))[1] - 8)
        assert np.all(np.abs(g - want)[diff] <= ulp[diff])


@pytest.mark.parametrize("seed,B,Hkv,Hq,theta", [
    (0, 3, 8, 32, 1e6), (1, 8, 4, 32, 1e4), (2, 1, 1, 8, 5e5), (3, 16, 8, 16, 1e6),
])
def test_append_matches_oracle(seed, B, Hkv, Hq, theta):
    c = make_case(seed, B, Hkv, Hq)
    check(c, theta, run(c, theta))


def test_append_at_large_positions():
    c = make_case(5, 2, 1, 4, big_prefix=100000)
    check(c, 1e6, run(c, 1e6))


def test_append_without_q_leaves_q():
    c = make_case(6, 2, 2, 4)
    kk, vv, qq = run(c, 1e6, with_q=False)
    assert np.array_equal(qq, c["q"])


def test_append_device_checks_skip_the_node():
    c = make_case(7, 3, 2, 4)
    c["depth"][2] = -1
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kk, vv, qq = run(c, 1e6, status=st)
    assert int(st.item()) == 4  # JF_ERR_DEVICE_CHECK
    # the rest is committed as the oracle says; node 2 left its slot and its q row as they were
    b0 = 0 if c["offsets"][1] > 2 else 1
    s = int(c["prefix"][b0]) + 2 - int(c["offsets"][b0])
    pg, off = int(c["bt"][b0][s // 16]), s % 16
    assert np.array_equal(kk[pg, off], c["kc"][pg, off]) and np.array_equal(qq[2], c["q"][2])


def test_append_replays_in_a_cuda_graph():
    c = make_case(8, 4, 8, 32)
    d = {k: dev(v) for k, v in c.items()}
    k0, v0, q0 = d["kc"].clone(), d["vc"].clone(), d["q"].clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            api.tree_kv_append(d["kn"], d["vn"], d["kc"], d["vc"], d["bt"], d["prefix"], d["offsets"], d["depth"],
                               1e6, q=d["q"])
    d["kc"].copy_(k0)
    d["vc"].copy_(v0)
    d["q"].copy_(q0)
    g.replay()
    torch.cuda.synchronize()
    check(c, 1e6, (bits(d["kc"]), bits(d["vc"]), bits(d["q"])))
