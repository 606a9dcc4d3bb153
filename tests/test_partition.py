"""Host-side model of the attention kernel's stream-K partition (the same integer formulas as the
device plan): every (unit, kv tile) pair is covered exactly once, a unit's sharing CTAs are exactly
those that hold one of its kv tiles, partial slots never collide, every CTA's range is non-empty, and
a CTA that starts segments in mid-range gets correspondingly fewer kv tiles.

A unit is one (sequence, kv head, pair of 128-row M tiles).  It costs SEG_COST + kt positions: SEG_COST
leading positions (the price of starting a segment in mid-kernel) and then its kt positions, position t
reading kv tile (t - rot) mod kt, rot being where the owner of the unit's last position starts."""

import collections

import numpy as np
import pytest

BN, BM = 128, 128
SEG_COST = 3
Q_TILES = 2  # M tiles per unit


def pairs(N, group):
    return ((N * group + BM - 1) // BM + Q_TILES - 1) // Q_TILES


def plan(prefix, nodes, hkv, group):
    work = []
    for P, N in zip(prefix, nodes):
        if N == 0:
            work.append(0)
            continue
        kt = (P + N + BN - 1) // BN
        work.append(hkv * pairs(N, group) * (kt + SEG_COST))
    cum = np.concatenate([[0], np.cumsum(work)]).astype(np.int64)
    return cum


def segments(prefix, nodes, hkv, group, grid):
    cum = plan(prefix, nodes, hkv, group)
    W = int(cum[-1])
    G = min(grid, W)
    cta_of = lambda x: ((x + 1) * G - 1) // W
    out = []
    for c in range(G):
        x, xend = c * W // G, (c + 1) * W // G
        assert xend > x
        b = 0
        while x < xend:
            while cum[b + 1] <= x:
                b += 1
            P, N = prefix[b], nodes[b]
            kt = (P + N + BN - 1) // BN
            mtn = pairs(N, group)
            span = kt + SEG_COST
            unit = (x - cum[b]) // span
            u0, u1 = cum[b] + unit * span, cum[b] + unit * span + span
            e = min(xend, u1)
            t0, t1 = x - u0 - SEG_COST, e - u0 - SEG_COST
            x = e
            if t1 <= 0:
                continue
            c0, c1 = cta_of(u0 + SEG_COST), cta_of(u1 - 1)
            slot = 2 * c + 1 if c == c0 else 2 * c
            rot = max(c1 * W // G - u0 - SEG_COST, 0)
            out.append(dict(cta=c, b=b, kvh=unit // mtn, mt=unit % mtn, kb=max(t0, 0), ke=t1, c0=c0, c1=c1,
                            slot=slot, range=(c * W // G, (c + 1) * W // G), kt=kt, rot=rot,
                            start=u0 + SEG_COST - c * W // G))  # local time of position 0
    return out, W, G


@pytest.mark.parametrize("prefix,nodes,hkv,group,grid", [
    ([256], [16], 1, 4, 148),
    ([4096], [256], 8, 4, 148),
    ([32768] * 4, [256] * 4, 4, 8, 148),
    (list(np.random.default_rng(0).integers(1024, 8193, 16)), [64] * 16, 8, 4, 148),
    ([0, 5, 300, 17], [3, 0, 256, 1], 2, 2, 7),
    ([10] * 50, [1] * 50, 1, 1, 148),
    ([131072], [16], 1, 4, 148),  # one unit cut over every CTA
])
def test_cover_exactly_once(prefix, nodes, hkv, group, grid):
    segs, W, G = segments(prefix, nodes, hkv, group, grid)
    seen = {}
    for s in segs:
        assert 0 <= s["rot"] < s["kt"]
        for t in range(s["kb"], s["ke"]):
            key = (s["b"], s["kvh"], s["mt"], (t - s["rot"]) % s["kt"])
            assert key not in seen
            seen[key] = s["cta"]
    tiles = sum(hkv * pairs(N, group) * ((P + N + BN - 1) // BN) for P, N in zip(prefix, nodes) if N > 0)
    assert len(seen) == tiles
    assert W == tiles + SEG_COST * sum(hkv * pairs(N, group) for N in nodes if N > 0)
    # the pieces of a unit agree on its rotation, and the owner of the last position reads tile 0 first
    for s in segs:
        if s["cta"] == s["c1"] and s["c0"] != s["c1"]:
            assert (s["kb"] - s["rot"]) % s["kt"] == 0
    per_cta = {}
    for s in segs:
        per_cta.setdefault(s["cta"], []).append(s)
    for c, ss in per_cta.items():
        lo, hi = ss[0]["range"]
        real = sum(x["ke"] - x["kb"] for x in ss)
        assert real + SEG_COST * (len(ss) - 1) <= hi - lo
    units = {}
    for s in segs:
        units.setdefault((s["b"], s["kvh"], s["mt"]), []).append(s)
    slots = set()
    for u, ss in units.items():
        ctas = sorted(x["cta"] for x in ss)
        assert ctas == list(range(ss[0]["c0"], ss[0]["c1"] + 1))
        if len(ss) > 1:
            for x in ss:
                assert x["slot"] not in slots
                slots.add(x["slot"])
                assert x["slot"] < 2 * G


def test_pairs_of_one_kv_head_read_in_step():
    """Qwen3-30B-A3B shape (4 sequences, 32768-token prefix, 256-node trees, 4 kv heads, 8 q heads per kv
    head: 8 units per (sequence, kv head)): at every CTA-local time the units of one (sequence, kv head)
    read tile x or tile x + (kt - W / G) (rounding: +-1), x the local time, with a few reads two such
    steps ahead (a CTA whose range lies inside one unit)."""
    segs, W, G = segments([32768] * 4, [256] * 4, 4, 8, 148)
    kt = segs[0]["kt"]
    lag = kt - W // G
    phases = collections.defaultdict(collections.Counter)
    for s in segs:
        for t in range(s["kb"], s["ke"]):
            tau = s["start"] + t  # CTA-local time of this position
            phases[(s["b"], s["kvh"])][((t - s["rot"]) % kt - tau) % kt] += 1
    assert len(phases) == 16
    for grp, c in phases.items():
        assert sum(c.values()) == 8 * kt
        main = sum(v for k, v in c.items() if k in (0, lag - 1, lag, lag + 1))
        assert main >= 0.95 * 8 * kt, (grp, sorted(c.items()))
        assert set(c) <= {0, lag - 1, lag, lag + 1, 2 * lag - 2, 2 * lag - 1, 2 * lag, 2 * lag + 1}, sorted(c.items())
