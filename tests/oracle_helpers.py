"""Helpers shared by the oracle pins: golden-fixture loading and an
independent dense reference built on torch's scaled_dot_product_attention."""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

from workloads import Problem

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

_CONST = {"ln2": math.log(2.0), "ln3": math.log(3.0), "log2": math.log(2.0),
          "log3": math.log(3.0), "log5": math.log(5.0), "log7": math.log(7.0),
          "log1.75": math.log(1.75), "inf": math.inf}
_TD = {"f16": torch.float16, "bf16": torch.bfloat16, "i8": torch.int8}


def _num(x):
    return _CONST[x] if isinstance(x, str) else float(x)


def _fill(x, shape, nan):
    """Nested lists with ``None`` placeholders -> float array of ``shape``."""
    if x is None:
        return np.full(shape, nan, dtype=np.float64)
    if not shape:
        return np.float64(_num(x))
    return np.stack([_fill(e, shape[1:], nan) for e in x])


def load_golden(name: str):
    with open(os.path.join(GOLDEN_DIR, name)) as f:
        g = json.load(f)
    dt = _TD[g["dtype"]]
    kvdt = _TD[g.get("kv_dtype", g["dtype"])]
    H, KVH, D, bs = g["head_num"], g["kv_head_num"], g["head_size"], g["block_size"]
    nblk = len(g["key"])
    nan = 0.0 if kvdt == torch.int8 else float("nan")
    k = _fill(g["key"], (nblk, bs, KVH, D), nan)
    v = _fill(g["value"], (nblk, bs, KVH, D), nan)
    q = _fill(g["query"], (int(sum(g["seq_len"])), H, D), 0.0)
    f32 = lambda key, shape: (torch.tensor(_fill(g[key], shape, 0.0), dtype=torch.float32)
                              if key in g else None)
    p = Problem(
        name=name, query=torch.tensor(q, dtype=torch.float32).to(dt),
        key_cache=torch.tensor(k, dtype=torch.float32).to(kvdt),
        value_cache=torch.tensor(v, dtype=torch.float32).to(kvdt),
        block_tables=torch.tensor(g["block_tables"], dtype=torch.int32),
        seq_len=np.array(g["seq_len"], dtype=np.int32),
        kv_seq_len=np.array(g["kv_seq_len"], dtype=np.int32),
        head_num=H, kv_head_num=KVH, qk_scale=_num(g["qk_scale"]), mask_type=g["mask_type"],
        slopes=f32("slopes", (H,)), sink=f32("sink", (H,)),
        k_scale=f32("k_scale", (KVH, D)), k_offset=f32("k_offset", (KVH, D)),
        v_scale=f32("v_scale", (KVH, D)), v_offset=f32("v_offset", (KVH, D)),
    )
    exp_out = _fill(g["expect_out"], (p.n_tokens, H, D), 0.0)
    exp_lse = _fill(g["expect_lse"], (p.n_tokens, H), 0.0)
    return p, exp_out, exp_lse


def dense_sdpa(p: Problem) -> np.ndarray:
    """Independent reference: gather each sequence's K/V into a dense tensor
    with torch indexing, dequantise int8 with torch ops, and run torch's
    scaled_dot_product_attention in float64.  A learnable sink becomes one
    extra key with zero key/value rows whose additive mask entry is the sink
    logit.  Returns out [nTokens, H, D] float64."""
    H, KVH, D, bs = p.head_num, p.kv_head_num, p.head_size, p.block_size
    g = H // KVH
    cu = p.cu_seq()
    out = np.zeros((p.n_tokens, H, D), dtype=np.float64)
    kc = p.key_cache.to(torch.float64)
    vc = p.value_cache.to(torch.float64)
    if getattr(p, "kv_layout", 0) == 1:          # BnNBsD -> BnBsH view
        kc, vc = kc.transpose(1, 2), vc.transpose(1, 2)
    km, vm = int(getattr(p, "k_antiquant_mode", 0)), int(getattr(p, "v_antiquant_mode", 0))
    if p.kv_is_int8:
        # per-channel pairs are applied to the whole pool here; per-token
        # pairs ([B, S]) after each sequence's gather below
        if not km:
            ko = torch.zeros(KVH, D, dtype=torch.float64) if p.k_offset is None else p.k_offset.double()
            kc = (kc + ko) * p.k_scale.double()
        if not vm:
            vo = torch.zeros(KVH, D, dtype=torch.float64) if p.v_offset is None else p.v_offset.double()
            vc = (vc + vo) * p.v_scale.double()
    for b in range(p.batch):
        ql, kl = int(p.seq_len[b]), int(p.kv_seq_len[b])
        if ql == 0:
            continue
        t = torch.arange(kl)
        blk = p.block_tables[b].long()[t // bs]
        kd = kc[blk, t % bs]                              # [kl, KVH, D]
        vd = vc[blk, t % bs]
        if p.kv_is_int8 and km:
            off = p.k_offset[b, :kl].double() if p.k_offset is not None else torch.zeros(kl, dtype=torch.float64)
            kd = (kd + off[:, None, None]) * p.k_scale[b, :kl].double()[:, None, None]
        if p.kv_is_int8 and vm:
            off = p.v_offset[b, :kl].double() if p.v_offset is not None else torch.zeros(kl, dtype=torch.float64)
            vd = (vd + off[:, None, None]) * p.v_scale[b, :kl].double()[:, None, None]
        q = p.query[cu[b]:cu[b + 1]].to(torch.float64)    # [ql, H, D]
        kd = kd.repeat_interleave(g, dim=1)               # GQA: head h -> kv head h // g
        vd = vd.repeat_interleave(g, dim=1)
        bias = torch.zeros(H, ql, kl, dtype=torch.float64)
        if p.mask_type in (3, 9):
            allowed = torch.ones(ql, kl, dtype=torch.bool).tril(diagonal=kl - ql)
            bias = bias.masked_fill(~allowed, float("-inf"))
        if getattr(p, "band", None) is not None:
            pre, nxt = p.band
            rel = torch.arange(kl)[None, :] - (torch.arange(ql)[:, None] + (kl - ql))   # t - qpos
            inside = (rel >= -pre) & (rel <= nxt)
            bias = bias.masked_fill(~inside, float("-inf"))
        if p.mask_type == 3:
            rel = (torch.arange(kl)[None, :] - (torch.arange(ql)[:, None] + (kl - ql))).double()
            bias = bias + p.slopes.double()[:, None, None] * rel[None]
        if p.pse is not None:
            bias = bias + p.pse[b, :, :ql, :kl].double()
        if p.sink is not None:
            kd = torch.cat([kd, torch.zeros(1, H, D, dtype=torch.float64)], 0)
            vd = torch.cat([vd, torch.zeros(1, H, D, dtype=torch.float64)], 0)
            bias = torch.cat([bias, p.sink.double()[:, None, None].expand(H, ql, 1)], 2)
        if kd.shape[0] == 0:
            continue
        o = F.scaled_dot_product_attention(q.transpose(0, 1), kd.transpose(0, 1),
                                           vd.transpose(0, 1), attn_mask=bias,
                                           scale=p.qk_scale)
        out[cu[b]:cu[b + 1]] = o.transpose(0, 1).numpy()
    return out
