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


def lse_err(lse, ref_lse):
    """max |err| of the finite lse entries (0 when there are none)."""
    fin = ~np.isinf(ref_lse)
    return float(np.abs(lse[fin] - ref_lse[fin]).max()) if fin.any() else 0.0


def compare_full(p, out, lse):
    """Every element of problem p's output against the oracle; prints and
    returns (max|err|, mean|err|, lse |err|)."""
    import oracle
    ref_out, ref_lse = oracle.attention(p)
    mx, mean = compare(out, lse, ref_out, ref_lse, p.name)
    le = lse_err(lse, ref_lse) if lse is not None else 0.0
    print("%-28s %9d rows  max|err| %.3e  mean|err| %.3e  lse|err| %.3e"
          % (p.name, out.shape[0] * out.shape[1], mx, mean, le))
    return mx, mean, le


def head_slice(p, kvh, h0, n):
    """Sub-problem of p with the n query heads kvh * g + h0 .. + n - 1 (all
    reading KV head kvh) and that KV head alone: same tokens, block table and
    cache rows, so its result must equal those heads' rows of p's result.
    Only inputs are sliced; nothing is computed."""
    import dataclasses
    g = p.head_num // p.kv_head_num
    assert 0 <= h0 and h0 + n <= g
    hs = slice(kvh * g + h0, kvh * g + h0 + n)
    kv_ax = 1 if p.kv_layout == 1 else 2
    cut = lambda t: t.narrow(kv_ax, kvh, 1).contiguous()
    per_ch = lambda t, mode: (None if t is None else
                              (t[kvh:kvh + 1].contiguous() if mode == 0 else t))
    return dataclasses.replace(
        p, name=p.name + "_kvh%d_h%d" % (kvh, h0), query=p.query[:, hs].contiguous(),
        key_cache=cut(p.key_cache), value_cache=cut(p.value_cache), head_num=n, kv_head_num=1,
        slopes=None if p.slopes is None else p.slopes[hs].contiguous(),
        pse=None if p.pse is None else p.pse[:, hs].contiguous(),
        sink=None if p.sink is None else p.sink[hs].contiguous(),
        k_scale=per_ch(p.k_scale, p.k_antiquant_mode), k_offset=per_ch(p.k_offset, p.k_antiquant_mode),
        v_scale=per_ch(p.v_scale, p.v_antiquant_mode), v_offset=per_ch(p.v_offset, p.v_antiquant_mode))


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
