"""GPU parity of jf_tree_attention_fp8 (8-bit E4M3 KV cache, through the C ABI) against the float64 oracle
oracle.tree_attention_fp8 (the bf16 path's definition on the decoded, scaled cache)."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle.fp8_kv import tree_attention_fp8
from tests.gpu_util import compare
from tree_verify_attention_jf_b200 import api, synth, workloads

pytestmark = pytest.mark.gpu

K_SCALE, V_SCALE = 1.0 / 128, 1.0 / 64  # N(0, 0.5) cache values -> codes within +-448


def run_fp8(inp, k_codes, v_codes, k_scale=K_SCALE, v_scale=V_SCALE, with_lse=True, status=None):
    dev = "cuda"
    bf = lambda a: synth.to_bf16_tensor(a).to(dev)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(dev)
    q = bf(inp.q)
    T, Hq = inp.q.shape[:2]
    out = torch.full_like(q, float("nan"))
    lse = torch.full((max(T, 1), Hq), float("nan"), dtype=torch.float32, device=dev) if with_lse else None
    api.tree_attention_fp8(q, u8(k_codes), u8(v_codes), k_scale, v_scale, i32(inp.block_table), i32(inp.prefix_lens),
                           i32(inp.tree_offsets), i32(inp.parent), inp.sm_scale, out=out, lse=lse, dev_status=status)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), (lse.cpu().numpy() if with_lse else None)


def reference(inp, k_codes, v_codes, k_scale=K_SCALE, v_scale=V_SCALE, rows=None):
    return tree_attention_fp8(inp.q, k_codes, v_codes, k_scale, v_scale, inp.block_table, inp.prefix_lens,
                              inp.tree_offsets, inp.parent, inp.sm_scale, inp.num_kv_heads, rows)


def codes_of(inp):
    return synth.e4m3_cache(inp.k_cache, K_SCALE), synth.e4m3_cache(inp.v_cache, V_SCALE)


def test_tiny_workload():
    inp = workloads.attention_workload("tiny")
    kc, vc = codes_of(inp)
    out, lse = run_fp8(inp, kc, vc)
    ref, lse_ref = reference(inp, kc, vc)
    compare(out, ref, lse, lse_ref)


@pytest.mark.parametrize("group", [1, 4, 8, 16])
@pytest.mark.parametrize("P", [0, 17, 130])
def test_mask_probes_planted_values(group, P):
    rng = np.random.default_rng(900 + P * 3 + group)
    nodes = [1, 16, 64, 200]
    pars = [synth.uniform_parent_tree(rng, n, 12) for n in nodes]
    hkv = 2
    inp = synth.attention_inputs(910 + P + group, hkv * group, hkv, [P + i for i in range(len(nodes))], pars,
                                 interleave=True)
    inp = synth.plant_tree_values(inp, magnitude=2.0, base_scale=0.5, seed=P)
    kc, vc = codes_of(inp)
    out, lse = run_fp8(inp, kc, vc)
    ref, lse_ref = reference(inp, kc, vc)
    compare(out, ref, lse, lse_ref)


@pytest.mark.parametrize("P", [0, 130, 4000])
def test_mask_exact_with_uniform_weights(P):
    """Zero queries weigh every visible key equally; V codes plant 2 e_j on tree slot j (exact in E4M3), zero prefix
    values: the output is exact up to the bf16 rounding of the result, at any prefix length."""
    rng = np.random.default_rng(950 + P)
    pars = [synth.uniform_parent_tree(rng, n, 14) for n in (256, 33, 100)]
    inp = synth.attention_inputs(960 + P, 8, 2, [P, P + 3, P + 16], pars, interleave=True)
    inp = synth.plant_tree_values(inp, magnitude=2.0, base_scale=0.0, seed=1)
    inp.q[:] = 0.0
    kc, vc = codes_of(inp)
    out, lse = run_fp8(inp, kc, vc)
    ref, lse_ref = reference(inp, kc, vc)
    np.testing.assert_allclose(out, ref, rtol=2 ** -8, atol=1e-7)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-4)


def test_serving_shaped_batch():
    """Serving shape (32 q / 8 kv heads, 64-node trees, interleaved page pool), 6 sequences with prefixes drawn from
    U[1024, 8192]; every row against the oracle."""
    rng = np.random.default_rng(33)
    prefixes = [int(x) for x in rng.integers(1024, 8193, size=6)]
    pars = [synth.uniform_parent_tree(rng, 64, max_depth=12) for _ in range(6)]
    inp = synth.attention_inputs(34, 32, 8, prefixes, pars, interleave=True)
    kc, vc = codes_of(inp)
    out, lse = run_fp8(inp, kc, vc)
    ref, lse_ref = reference(inp, kc, vc)
    compare(out, ref, lse, lse_ref)


def test_qwen3_8b_shape_and_scales():
    """The Qwen3-8B shape (256-node tree, 4096 prefix); a different pair of scales gives the oracle's result too."""
    inp = workloads.attention_workload("qwen3_8b")
    ks, vs = 1.0 / 150, 1.0 / 96
    kc, vc = synth.e4m3_cache(inp.k_cache, ks), synth.e4m3_cache(inp.v_cache, vs)
    out, lse = run_fp8(inp, kc, vc, ks, vs)
    ref, lse_ref = reference(inp, kc, vc, ks, vs)
    compare(out, ref, lse, lse_ref)


def test_qwen3_30b_whole_workload():
    """Every row of the Qwen3-30B-A3B workload over 8-bit caches (4 sequences x 256 nodes x 32 q heads, 32768-token
    prefixes, g = 8): every unit is cut between several CTAs, so the conversion, the split partials and their
    merge all run at full length."""
    inp = workloads.attention_workload("qwen3_30b_a3b")
    kc, vc = codes_of(inp)
    out, lse = run_fp8(inp, kc, vc)
    ref, lse_ref = reference(inp, kc, vc)
    compare(out, ref, lse, lse_ref)


def test_max_batch_ragged_with_empty_sequences():
    """1024 sequences with ragged trees of 0..8 nodes (about a quarter empty) over prefixes of 0..300 tokens, g = 4:
    every CTA runs many one- to three-tile segments, so landed tiles are still being converted when the next
    segment's Q tiles go out."""
    rng = np.random.default_rng(41)
    B = 1024
    ns = rng.integers(0, 9, size=B)
    ns[rng.random(B) < 0.25] = 0
    prefix = rng.integers(0, 301, size=B)
    parents = [synth.uniform_parent_tree(rng, int(n), 4) for n in ns]
    inp = synth.attention_inputs(42, 8, 2, [int(p) for p in prefix], parents, interleave=True)
    kc, vc = codes_of(inp)
    out, lse = run_fp8(inp, kc, vc)
    ref, lse_ref = reference(inp, kc, vc)
    compare(out, ref, lse, lse_ref)


def test_one_unit_cut_over_every_cta():
    """One unit (16 nodes, g = 4) over a 131072-token prefix: its 1025 kv tiles are split over every CTA, and
    each CTA's segment converts a handful of tiles and writes a partial."""
    rng = np.random.default_rng(43)
    inp = synth.attention_inputs(44, 4, 1, [131072], [synth.bushy_tree(rng, 16)])
    kc, vc = codes_of(inp)
    out, lse = run_fp8(inp, kc, vc)
    ref, lse_ref = reference(inp, kc, vc)
    compare(out, ref, lse, lse_ref)


def test_nan_codes_in_unused_slots_do_not_leak():
    inp = synth.attention_inputs(971, 4, 1, [20], [synth.uniform_parent_tree(np.random.default_rng(9), 10, 5)])
    kc, vc = codes_of(inp)
    page = int(inp.block_table[0, 1])
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[page, 14:] = 0x7F  # E4M3 NaN in the slots past the sequence (30, 31)
    vc2[page, 14:] = 0xFF
    out, lse = run_fp8(inp, kc2, vc2)
    ref, lse_ref = reference(inp, kc, vc)
    compare(out, ref, lse, lse_ref)


def test_page_permutation_is_bit_identical():
    inp = workloads.attention_workload("tiny")
    kc, vc = codes_of(inp)
    out1, lse1 = run_fp8(inp, kc, vc)
    perm = np.random.default_rng(5).permutation(kc.shape[0])
    inv = np.argsort(perm)
    bt = inp.block_table.copy()
    bt[bt >= 0] = inv[bt[bt >= 0]]
    out2, lse2 = run_fp8(dataclasses.replace(inp, block_table=bt), kc[perm], vc[perm])
    np.testing.assert_array_equal(out1, out2)
    np.testing.assert_array_equal(lse1, lse2)
