"""The five seeded workloads (shapes only; data from :mod:`synth`).

* ``tiny``          batch 1, 4 q heads / 1 kv head, prefix 256, 16-node uniform-parent tree (depth <= 8)
* ``qwen3_8b``      batch 1, 32 q / 8 kv heads, prefix 4096, 256-node tree (branching <= 4, <= 16 levels)
* ``serving``       batch 16, 32 q / 8 kv heads, prefixes ~ U{1024..8192}, 64-node trees (depth <= 12),
                    one shared page pool with all sequences' pages interleaved
* ``qwen3_30b_a3b`` batch 4, 32 q / 4 kv heads, prefix 32768, 256-node trees (branching <= 4, <= 16 levels)
* ``build_accept``  batch 8, draft logits fp32 [8, 16, 151936], top-4, budget 256, target logits
                    fp32 [8, 256, 151936] agreeing with the built tree on a path of length ~ U{1..16}

Shapes come from the JetFlow/JetSpec pages (Qwen3-8B dense, Qwen3-30B-A3B MoE, budgets 16..256,
"4. Experimental results"; tree construction up to a budget of 256, "2. Method").  Seeds 1..5.
"""
from __future__ import annotations

import numpy as np

from . import synth

SEEDS = {"tiny": 1, "qwen3_8b": 2, "serving": 3, "qwen3_30b_a3b": 4, "build_accept": 5}

ATTENTION_WORKLOADS = ("tiny", "qwen3_8b", "serving", "qwen3_30b_a3b")


def attention_workload(name: str, seed_offset: int = 0) -> synth.AttentionInputs:
    seed = SEEDS[name] + seed_offset
    rng = np.random.default_rng(seed * 7919)
    if name == "tiny":
        par = synth.uniform_parent_tree(rng, 16, max_depth=8)
        return synth.attention_inputs(seed, 4, 1, [256], [par])
    if name == "qwen3_8b":
        par = synth.bushy_tree(rng, 256, 4, 16)
        return synth.attention_inputs(seed, 32, 8, [4096], [par])
    if name == "serving":
        prefixes = [int(x) for x in rng.integers(1024, 8193, size=16)]
        pars = [synth.uniform_parent_tree(rng, 64, max_depth=12) for _ in range(16)]
        return synth.attention_inputs(seed, 32, 8, prefixes, pars, interleave=True)
    if name == "qwen3_30b_a3b":
        pars = [synth.bushy_tree(rng, 256, 4, 16) for _ in range(4)]
        return synth.attention_inputs(seed, 32, 4, [32768] * 4, pars)
    raise KeyError(name)


BUILD = dict(batch=8, depths=16, vocab=synth.VOCAB, topk=4, budget=256, max_depth=16)


def build_inputs(seed_offset: int = 0, batch: int = BUILD["batch"], vocab: int = BUILD["vocab"],
                 depths: int = BUILD["depths"]):
    """Draft logits [batch, depths, vocab] and root tokens for the build+accept workload."""
    return synth.draft_logits(SEEDS["build_accept"] + seed_offset, batch, depths, vocab)
