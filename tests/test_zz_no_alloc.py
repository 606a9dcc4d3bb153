"""jf_build_tree_noalloc: the tree-build call for hosts that cannot allocate device memory when they call
this library (a serving engine that gives all spare memory to its KV-cache pool at start-up, a plugin
framework whose per-call hook must not allocate).  It keeps its scratch in a fixed 1 MiB device array
inside libjf.so instead of a caller-provided workspace.

This file is collected last on purpose: if it fails, a run that stops at the first failure has already
run every other test.  It passes both on its own in a fresh process and after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

from tree_verify_attention_jf_b200 import _lib, api, synth, workloads

SCORE_ABS = 1e-5  # the score tolerance of the other build tests


def noalloc_fn():
    fn = _lib.lib().jf_build_tree_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, i, i, i, i, i, i, vp, vp, vp, vp, vp, vp]
    fn.restype = i
    return fn


def call_noalloc(x, roots, topk, budget, max_depth):
    B, depths, V = x.shape
    dev = x.device
    out = {k: torch.full((B, budget), -7, dtype=torch.int32, device=dev) for k in ("parent", "token", "depth")}
    out["score"] = torch.full((B, budget), float("nan"), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    code = noalloc_fn()(x.data_ptr(), roots.data_ptr(), B, depths, V, topk, budget, max_depth, out["parent"].data_ptr(),
                        out["token"].data_ptr(), out["score"].data_ptr(), out["depth"].data_ptr(), status.data_ptr(),
                        torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return code, int(status.item()), {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.gpu
def test_matches_workspace_variant_on_two_calls_in_a_row():
    cases = [workloads.build_inputs(), synth.draft_logits(91, 3, 12, 50000)]
    for (x_np, roots_np), (topk, budget, max_depth) in zip(cases, [(4, 256, 16), (3, 100, 12)]):
        x = torch.from_numpy(x_np).cuda()
        roots = torch.from_numpy(roots_np).cuda()
        ref = {k: v.cpu().numpy() for k, v in api.build_tree(x, roots, topk, budget, max_depth).items()}
        code, status, got = call_noalloc(x, roots, topk, budget, max_depth)
        assert code == _lib.JF_OK and status == 0
        for k in ("parent", "token", "depth"):
            np.testing.assert_array_equal(got[k], ref[k])
        np.testing.assert_allclose(got["score"], ref["score"], rtol=0, atol=SCORE_ABS)


def test_rejects_calls_beyond_the_scratch_limit():
    # 64 sequences x 16 depths x 38 chunks x 80 bytes > 1 MiB: refused before anything is launched.  Every
    # pointer is null, so that if the size check ever stopped refusing this call, the null-pointer check
    # would still turn it into JF_ERR_INVALID_ARG (and this test would fail) without launching a kernel.
    code = noalloc_fn()(None, None, 64, 16, 151936, 4, 256, 16, None, None, None, None, None, None)
    assert code == _lib.JF_ERR_UNSUPPORTED
