"""Failure detection on the GPU without a fault: the debug build (libjf_debug.so: 50 ms wait limit) can make the
attention kernel's first wait run out (jf_debug_hold) before any copy or MMA is issued.  The call must return,
report JF_ERR_TIMEOUT in dev_status, write no output, and leave the context usable: the next call (hold released)
gives the oracle's result."""
import numpy as np
import pytest
import torch

from oracle.tree_attention import tree_attention_inputs
from tests.gpu_util import compare, to_dev
from tree_verify_attention_jf_b200 import _lib, synth, workloads

pytestmark = pytest.mark.gpu


def call(L, inp, d, out, lse, ws, status):
    T, Hq = inp.q.shape[:2]
    num_pages, page, Hkv, D = inp.k_cache.shape
    ptr = lambda t: None if t is None else t.data_ptr()
    return L.jf_tree_attention(ptr(d["q"]), ptr(d["k_cache"]), ptr(d["v_cache"]), ptr(d["block_table"]),
                               inp.block_table.shape[1], ptr(d["prefix_lens"]), ptr(d["tree_offsets"]),
                               ptr(d["parent"]), inp.batch, T, Hq, Hkv, D, page, num_pages, inp.sm_scale, ptr(out),
                               ptr(lse), ptr(ws), ws.numel(), ptr(status), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name", ["tiny", "qwen3_8b"])
def test_wait_that_runs_out_reports_timeout_and_the_context_survives(name):
    L = _lib.debug_lib()
    inp = workloads.attention_workload(name)
    d = to_dev(inp)
    T, Hq = inp.q.shape[:2]
    ws = torch.empty(L.jf_tree_attention_workspace_size(0, 0, 0, 0), dtype=torch.uint8, device="cuda")
    out = torch.full_like(d["q"], float("nan"))
    lse = torch.full((T, Hq), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.jf_debug_hold(1) == _lib.JF_OK
    try:
        assert call(L, inp, d, out, lse, ws, status) == _lib.JF_OK  # launched; the failure is reported on the device
        torch.cuda.synchronize()  # returns: no hang, no fault
    finally:
        assert L.jf_debug_hold(0) == _lib.JF_OK
    assert int(status.item()) == _lib.JF_ERR_TIMEOUT
    assert torch.isnan(out.float()).all()  # nothing was written
    # the context is usable and the same call now gives the oracle's result
    status.zero_()
    assert call(L, inp, d, out, lse, ws, status) == _lib.JF_OK
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, lse_ref = tree_attention_inputs(inp)
    compare(out.float().cpu().numpy(), ref, lse.cpu().numpy(), lse_ref)


def test_wait_that_runs_out_on_the_8bit_cache_path():
    """The same hold on jf_tree_attention_fp8 (the 8-bit cache instantiation of the kernel): JF_ERR_TIMEOUT,
    nothing written, and the released call gives the oracle's result on the decoded cache."""
    from oracle.fp8_kv import tree_attention_fp8
    L = _lib.debug_lib()
    inp = workloads.attention_workload("tiny")
    k_scale, v_scale = 1.0 / 128, 1.0 / 64
    kc, vc = synth.e4m3_cache(inp.k_cache, k_scale), synth.e4m3_cache(inp.v_cache, v_scale)
    d = to_dev(inp)
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()
    kd, vd = u8(kc), u8(vc)
    T, Hq = inp.q.shape[:2]
    num_pages, page, Hkv, D = inp.k_cache.shape
    ws = torch.empty(L.jf_tree_attention_workspace_size(0, 0, 0, 0), dtype=torch.uint8, device="cuda")
    out = torch.full_like(d["q"], float("nan"))
    lse = torch.full((T, Hq), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call8():
        return L.jf_tree_attention_fp8(d["q"].data_ptr(), kd.data_ptr(), vd.data_ptr(), k_scale, v_scale,
                                       d["block_table"].data_ptr(), inp.block_table.shape[1],
                                       d["prefix_lens"].data_ptr(), d["tree_offsets"].data_ptr(),
                                       d["parent"].data_ptr(), inp.batch, T, Hq, Hkv, D, page, num_pages,
                                       inp.sm_scale, out.data_ptr(), lse.data_ptr(), ws.data_ptr(), ws.numel(),
                                       status.data_ptr(), torch.cuda.current_stream().cuda_stream)

    assert L.jf_debug_hold(1) == _lib.JF_OK
    try:
        assert call8() == _lib.JF_OK
        torch.cuda.synchronize()
    finally:
        assert L.jf_debug_hold(0) == _lib.JF_OK
    assert int(status.item()) == _lib.JF_ERR_TIMEOUT
    assert torch.isnan(out.float()).all()
    status.zero_()
    assert call8() == _lib.JF_OK
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, lse_ref = tree_attention_fp8(inp.q, kc, vc, k_scale, v_scale, inp.block_table, inp.prefix_lens,
                                      inp.tree_offsets, inp.parent, inp.sm_scale, inp.num_kv_heads, None)
    compare(out.float().cpu().numpy(), ref, lse.cpu().numpy(), lse_ref)
