"""GPU parity of jf_commit_kv (through the C ABI) against the oracle: the committed caches byte for byte, the new
prefix lengths exactly, device checks, aliasing of new_prefix_lens with prefix_lens, and CUDA-graph replay."""
import numpy as np
import pytest
import torch

from oracle.commit_kv import commit_kv as oracle_commit
from tests.test_oracle_commit import rooted_tree
from tree_verify_attention_jf_b200 import api

pytestmark = pytest.mark.gpu


def make_case(seed, B, H, max_depth, max_prefix=70, max_nodes=60, chain=False):
    rng = np.random.default_rng(seed)
    prefix = rng.integers(0, max_prefix, B)
    nodes = rng.integers(0, max_nodes, B)
    nodes[0] = max(int(nodes[0]), 2)
    offsets = np.concatenate([[0], np.cumsum(nodes)])
    pages_per = [(int(p) + int(n) + 15) // 16 for p, n in zip(prefix, nodes)]
    npages = sum(pages_per) + 5
    perm = rng.permutation(npages)
    bt = np.zeros((B, max(pages_per) + 2), np.int32)
    c = 0
    for b in range(B):
        bt[b, :pages_per[b]] = perm[c:c + pages_per[b]]
        c += pages_per[b]
    # arbitrary bf16 bit patterns (NaN and inf patterns included): the copy must be byte-exact
    k = rng.integers(-32768, 32768, (npages, 16, H, 128)).astype(np.int16)
    v = rng.integers(-32768, 32768, (npages, 16, H, 128)).astype(np.int16)
    path = -np.ones((B, max_depth + 1), np.int32)
    L = np.zeros(B, np.int32)
    for b in range(B):
        n = int(nodes[b])
        if n == 0:
            continue
        par = np.arange(-1, n - 1) if chain else rooted_tree(rng, n, max(max_depth, 1))
        end = int(rng.integers(0, n))
        pth = [end]
        while pth[-1] != 0:
            pth.append(int(par[pth[-1]]))
        pth.reverse()
        pth = pth[:max_depth + 1]
        L[b] = len(pth) - 1
        path[b, :len(pth)] = pth
    return dict(k=k, v=v, bt=bt, prefix=prefix.astype(np.int32), offsets=offsets.astype(np.int32), path=path, L=L)


def to_dev(c):
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    kv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.bfloat16)
    return dict(k=kv(c["k"]), v=kv(c["v"]), bt=i32(c["bt"]), prefix=i32(c["prefix"]), offsets=i32(c["offsets"]),
                path=i32(c["path"]), L=i32(c["L"]))


def run(c, alias=False, status=None):
    d = to_dev(c)
    newp = d["prefix"] if alias else None
    out = api.commit_kv(d["k"], d["v"], d["bt"], d["prefix"], d["offsets"], d["path"], d["L"], new_prefix_lens=newp,
                        dev_status=status)
    torch.cuda.synchronize()
    return d["k"].view(torch.int16).cpu().numpy(), d["v"].view(torch.int16).cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("seed,B,H,max_depth,chain", [
    (0, 3, 8, 6, False), (1, 16, 4, 16, False), (2, 1, 1, 32, True), (3, 5, 64, 8, False), (4, 7, 8, 40, True),
    (5, 2, 2, 0, False), (6, 9, 16, 12, False),
])
def test_commit_matches_oracle(seed, B, H, max_depth, chain):
    c = make_case(seed, B, H, max_depth, chain=chain)
    kk, vv, newp = run(c)
    rk, rv, rp = oracle_commit(c["k"], c["v"], c["bt"], c["prefix"], c["offsets"], c["path"], c["L"])
    assert np.array_equal(newp, rp)
    assert np.array_equal(kk, rk) and np.array_equal(vv, rv)


def test_commit_new_prefix_may_alias_prefix():
    c = make_case(11, 8, 8, 10)
    kk, vv, newp = run(c, alias=True)
    rk, rv, rp = oracle_commit(c["k"], c["v"], c["bt"], c["prefix"], c["offsets"], c["path"], c["L"])
    assert np.array_equal(newp, rp) and np.array_equal(kk, rk) and np.array_equal(vv, rv)


def test_commit_device_checks_leave_the_sequence():
    c = make_case(12, 4, 8, 10)
    good = c["path"].copy()
    c["path"][1, 1:3] = [3, 3]   # not strictly increasing (sequence 1)
    c["L"][1] = max(int(c["L"][1]), 2)
    c["L"][2] = 11               # past max_depth (sequence 2)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kk, vv, newp = run(c, status=st)
    assert int(st.item()) == 4  # JF_ERR_DEVICE_CHECK
    keep = [0, 3]
    L_ok = c["L"].copy()
    L_ok[1] = 0
    L_ok[2] = 0
    rk, rv, rp = oracle_commit(c["k"], c["v"], c["bt"], c["prefix"], c["offsets"], np.where(
        np.arange(4)[:, None] == 1, good, c["path"]), L_ok)
    assert np.array_equal(kk, rk) and np.array_equal(vv, rv)
    for b in keep:
        assert newp[b] == rp[b]
    assert newp[1] == c["prefix"][1] and newp[2] == c["prefix"][2]


def test_commit_replays_in_a_cuda_graph():
    c = make_case(13, 6, 8, 12)
    d = to_dev(c)
    k0, v0 = d["k"].clone(), d["v"].clone()
    newp = torch.empty_like(d["prefix"])
    api.commit_kv(d["k"], d["v"], d["bt"], d["prefix"], d["offsets"], d["path"], d["L"], new_prefix_lens=newp)
    torch.cuda.synchronize()
    eager_k, eager_v = d["k"].clone(), d["v"].clone()
    d["k"].copy_(k0)
    d["v"].copy_(v0)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            api.commit_kv(d["k"], d["v"], d["bt"], d["prefix"], d["offsets"], d["path"], d["L"], new_prefix_lens=newp)
    d["k"].copy_(k0)
    d["v"].copy_(v0)
    newp.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(d["k"].view(torch.int16), eager_k.view(torch.int16))
    assert torch.equal(d["v"].view(torch.int16), eager_v.view(torch.int16))
    rp = oracle_commit(c["k"], c["v"], c["bt"], c["prefix"], c["offsets"], c["path"], c["L"])[2]
    assert np.array_equal(newp.cpu().numpy(), rp)
