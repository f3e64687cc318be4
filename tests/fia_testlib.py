"""Test glue: move a workloads.Problem onto the GPU, run it through the C ABI
(paged_attention_02_b200.FiaOp) and compare against the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances for fp16/bf16 outputs and fp32 lse against the fp64 oracle.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 5e-3


def run_gpu(p, device="cuda", **overrides):
    """Run problem ``p`` through libfia; returns (op, out_cpu_f64, lse_cpu_f64)."""
    import paged_attention_02_b200 as fia
    d = lambda t: None if t is None else t.to(device).contiguous()
    kw = dict(mask_type=p.mask_type, slopes=d(p.slopes), pse=d(p.pse), sink=d(p.sink),
              k_scale=d(p.k_scale), k_offset=d(p.k_offset), v_scale=d(p.v_scale),
              v_offset=d(p.v_offset), want_lse=p.want_lse,
              kv_layout=int(getattr(p, "kv_layout", 0)),
              k_antiquant_mode=int(getattr(p, "k_antiquant_mode", 0)),
              v_antiquant_mode=int(getattr(p, "v_antiquant_mode", 0)),
              band=getattr(p, "band", None))
    kw.update(overrides)
    op = fia.FiaOp(d(p.query), d(p.key_cache), d(p.value_cache), d(p.block_tables),
                   [int(x) for x in p.seq_len], [int(x) for x in p.kv_seq_len], p.head_num,
                   p.kv_head_num, p.qk_scale, **kw)
    out, lse = op.run()
    torch.cuda.synchronize()
    ew = op.error_word()
    assert ew == 0, "kernel error word set: %#x, trail %s" % (ew, op.error_trail())
    o = out.float().double().cpu().numpy()
    l = lse.double().cpu().numpy() if lse is not None else None
    return op, o, l


def compare(out, lse, ref_out, ref_lse, what=""):
    """Element-wise parity: max/mean |err| on out, |err| on lse (inf == inf)."""
    assert out.shape == ref_out.shape, (out.shape, ref_out.shape)
    assert np.all(np.isfinite(out)), "%s: non-finite output" % what
    err = np.abs(out - ref_out)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= MAX_ABS and mean <= MEAN_ABS, "%s: max %.3g mean %.3g" % (what, mx, mean)
    if lse is not None:
        inf_ref = np.isinf(ref_lse)
        assert np.array_equal(np.isinf(lse), inf_ref), "%s: lse inf pattern differs" % what
        if (~inf_ref).any():
            le = float(np.abs(lse[~inf_ref] - ref_lse[~inf_ref]).max())
            assert le <= LSE_ABS, "%s: lse err %.3g" % (what, le)
    return mx, mean


def sample_rows(p, n, seed):
    """Seeded sample of (token, head) rows, always including the first and
    last token of every sequence."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cu = p.cu_seq()
    rows = set()
    for b in range(p.batch):
        if p.seq_len[b] == 0:
            continue
        for t in (int(cu[b]), int(cu[b + 1]) - 1):
            rows.add((t, int(rng.integers(p.head_num))))
    while len(rows) < n:
        rows.add((int(rng.integers(p.n_tokens)), int(rng.integers(p.head_num))))
    return sorted(rows)
