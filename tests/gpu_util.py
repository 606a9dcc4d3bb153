"""Helpers shared by the GPU tests: move seeded inputs to the device, run the C-ABI path, compare."""
import numpy as np
import torch

from tree_verify_attention_jf_b200 import api, synth

# Attention tolerance: bf16 output vs float64 oracle (max-abs 2e-2, mean-abs 2e-3), plus an LSE bound.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 2e-3
# Error relative to the output's RMS.  The kernel rounds twice in bf16 (unit roundoff u = 2^-9): every softmax
# weight before the PV product and the output itself; each contributes at most u relative, so the RMS of the
# error stays below about 2u.  The bound is 4u = 2^-7.  Unlike the absolute bounds it does not loosen when the
# output is small (long prefixes average V towards zero).
REL_RMS = 2 ** -7


def to_dev(inp: synth.AttentionInputs, device="cuda"):
    bf = lambda a: synth.to_bf16_tensor(a).to(device)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    return dict(q=bf(inp.q), k_cache=bf(inp.k_cache), v_cache=bf(inp.v_cache), block_table=i32(inp.block_table),
                prefix_lens=i32(inp.prefix_lens), tree_offsets=i32(inp.tree_offsets), parent=i32(inp.parent))


def run_attention(inp: synth.AttentionInputs, ws=None, status=None, dev=None, with_lse=True):
    d = dev if dev is not None else to_dev(inp)
    T, Hq = inp.q.shape[:2]
    lse = torch.full((max(T, 1), Hq), float("nan"), dtype=torch.float32, device="cuda") if with_lse else None
    out = torch.full_like(d["q"], float("nan"))
    api.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["prefix_lens"], d["tree_offsets"],
                       d["parent"], inp.sm_scale, out=out, lse=lse, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), (lse.cpu().numpy() if with_lse else None)


def compare(out, ref, lse=None, lse_ref=None, rows=None):
    if rows is not None:
        t = np.array([r[0] for r in rows])
        h = np.array([r[1] for r in rows])
        out, ref = out[t, h], ref[t, h]
        if lse is not None:
            lse, lse_ref = lse[t, h], lse_ref[t, h]
    assert np.isfinite(out).all()
    err = np.abs(out - ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) + 1e-12
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()), rel_rms=float(np.sqrt(np.mean(err ** 2)) / rms))
    assert stats["max_abs"] <= MAX_ABS, stats
    assert stats["mean_abs"] <= MEAN_ABS, stats
    assert stats["rel_rms"] <= REL_RMS, stats
    if lse is not None:
        lerr = float(np.abs(lse - lse_ref).max())
        stats["lse_max_abs"] = lerr
        assert lerr <= LSE_ABS, stats
    return stats
