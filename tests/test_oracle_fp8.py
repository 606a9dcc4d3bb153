"""Pins of the 8-bit KV oracle (oracle/fp8_kv.py): the E4M3 format's named codes, agreement with torch's
float8_e4m3fn conversion (an independent implementation) on all codes and on random values, ties to even,
saturation, and closed forms of the cache scales in attention."""
import numpy as np
import torch

from oracle.fp8_kv import e4m3_decode, e4m3_encode, quantize_cache, tree_attention_fp8
from oracle.tree_attention import tree_attention
from tree_verify_attention_jf_b200 import synth


def test_named_codes():
    d = e4m3_decode(np.array([0x38, 0x7E, 0x08, 0x07, 0x01, 0x00, 0x80, 0xB8, 0xFE, 0x7F, 0xFF], np.uint8))
    assert d[:9].tolist() == [1.0, 448.0, 2.0 ** -6, 7 * 2.0 ** -9, 2.0 ** -9, 0.0, -0.0, -1.0, -448.0]
    assert np.isnan(d[9]) and np.isnan(d[10])
    assert np.signbit(d[6])


def test_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def test_encoding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1.0, 30.0, 150.0)])
    x = x[np.abs(x) <= 448.0].astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3_encode(x), want)


def test_round_trip_and_ties_to_even():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    assert np.array_equal(e4m3_encode(e4m3_decode(codes)), codes)
    # exact midpoints: 1 + 1/16 lies between 1.0 (mantissa 0) and 1.125 (mantissa 1) -> 1.0;
    # 1 + 3/16 lies between 1.125 and 1.25 (mantissa 2) -> 1.25
    assert e4m3_decode(e4m3_encode([1.0625, 1.1875])).tolist() == [1.0, 1.25]


def test_saturation():
    assert e4m3_encode([500.0, 1e9, -1e9, 448.0]).tolist() == [0x7E, 0x7E, 0xFE, 0x7E]


def small_case(seed):
    rng = np.random.default_rng(seed)
    parent = synth.uniform_parent_tree(rng, 12, 5)
    return synth.attention_inputs(seed, 4, 2, [40], [parent], interleave=False)


def test_v_scale_multiplies_the_output():
    inp = small_case(1)
    kc, vc = quantize_cache(inp.k_cache, 0.01), quantize_cache(inp.v_cache, 0.01)
    a, _ = tree_attention_fp8(inp.q, kc, vc, 0.01, 0.01, inp.block_table, inp.prefix_lens, inp.tree_offsets,
                              inp.parent, inp.sm_scale)
    b, _ = tree_attention_fp8(inp.q, kc, vc, 0.01, 0.03, inp.block_table, inp.prefix_lens, inp.tree_offsets,
                              inp.parent, inp.sm_scale)
    assert np.allclose(b, 3 * a, rtol=1e-12, atol=1e-14)


def test_k_scale_acts_on_the_softmax_scale():
    inp = small_case(2)
    kc, vc = quantize_cache(inp.k_cache, 0.01), quantize_cache(inp.v_cache, 0.01)
    a, la = tree_attention_fp8(inp.q, kc, vc, 0.02, 0.01, inp.block_table, inp.prefix_lens, inp.tree_offsets,
                               inp.parent, inp.sm_scale)
    b, lb = tree_attention_fp8(inp.q, kc, vc, 0.01, 0.01, inp.block_table, inp.prefix_lens, inp.tree_offsets,
                               inp.parent, 2 * inp.sm_scale)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14) and np.allclose(la, lb, rtol=1e-12)


def test_quantized_attention_stays_near_the_bf16_one():
    # E4M3 keeps 3 mantissa bits (relative step 2^-3): with a scale that maps the cache's largest value to 448,
    # the output moves by a few percent of its scale at most
    inp = small_case(3)
    ks = np.abs(inp.k_cache).max() / 448.0
    vs = np.abs(inp.v_cache).max() / 448.0
    a, _ = tree_attention_fp8(inp.q, quantize_cache(inp.k_cache, ks), quantize_cache(inp.v_cache, vs), ks, vs,
                              inp.block_table, inp.prefix_lens, inp.tree_offsets, inp.parent, inp.sm_scale)
    b, _ = tree_attention(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.prefix_lens, inp.tree_offsets,
                          inp.parent, inp.sm_scale)
    assert np.abs(a - b).max() < 0.1 * np.abs(b).max()
