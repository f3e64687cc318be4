"""The bench's algorithmic work counts (the numerators of its roofline
figures) against brute force on small problems."""
import numpy as np
import pytest

import bench
import workloads as W


def _brute_pairs(p):
    tot = 0
    for b in range(p.batch):
        ql, kl = int(p.seq_len[b]), int(p.kv_seq_len[b])
        for i in range(ql):
            qpos = kl - ql + i
            for t in range(kl):
                if p.band is not None:
                    ok = qpos - p.band[0] <= t <= qpos + p.band[1]
                elif p.mask_type in (W.MASK_CAUSAL, W.MASK_ALIBI):
                    ok = t <= qpos
                else:
                    ok = True
                tot += ok
    return tot * p.head_num


@pytest.mark.parametrize("kw", [
    dict(mask_type=W.MASK_NONE),
    dict(mask_type=W.MASK_CAUSAL),
    dict(mask_type=W.MASK_ALIBI, alibi_slopes=True),
    dict(band=(4, 1)),
    dict(band=(-2, 5)),
    dict(band=(0, 0)),
    dict(band=(100, 100)),
])
def test_unmasked_pairs_brute_force(kw):
    p = W.make_problem(seed=1, seq_len=[7, 3, 1], kv_seq_len=[20, 3, 9], head_num=2,
                       kv_head_num=1, head_size=64, block_size=16, **kw)
    assert bench.unmasked_pairs(p) == _brute_pairs(p)
    assert bench.flops(p) == 4.0 * 64 * _brute_pairs(p)


@pytest.mark.parametrize("kmode,vmode", [("channel", "channel"), ("token", "token"),
                                         ("channel", "token"), ("token", "channel")])
def test_kv_bytes_counts_per_token_params_once(kmode, vmode):
    p = W.make_problem(seed=2, seq_len=[1, 1], kv_seq_len=[30, 50], head_num=4, kv_head_num=2,
                       head_size=128, block_size=16, kv_dtype="i8", k_antiquant=kmode,
                       v_antiquant=vmode)
    cache = 80 * 2 * 128 * 1 * 2                    # tokens x KVH x D x int8 x (K, V)
    per_token = 80 * 4 * 2 * ((kmode == "token") + (vmode == "token"))   # scale + offset
    assert bench.kv_bytes(p) == cache + per_token
