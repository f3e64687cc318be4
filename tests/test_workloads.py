"""The named benchmark workloads follow their configurations: shapes,
lengths, dtypes, scales, masks and value ranges (the input recipe)."""
import math

import numpy as np
import torch

import workloads as W


def _common(p, B, H, KVH, D, bs, dtype):
    assert p.batch == B and p.head_num == H and p.kv_head_num == KVH
    assert p.head_size == D and p.block_size == bs
    assert p.query.dtype == dtype
    assert p.query.shape == (int(np.sum(p.seq_len)), H, D)
    # block tables: the entries a sequence reads are distinct blocks of the pool
    used = []
    for b in range(B):
        need = -(-int(p.kv_seq_len[b]) // bs)
        used += [int(x) for x in p.block_tables[b, :need]]
    assert len(set(used)) == len(used)
    assert all(0 <= x < p.key_cache.shape[0] for x in used)


def test_tiny_decode():
    p = W.tiny_decode()
    _common(p, 2, 4, 4, 64, 16, torch.float16)
    assert list(p.seq_len) == [1, 1] and list(p.kv_seq_len) == [37, 64]
    assert p.key_cache.shape[0] == 8 and p.key_cache.dtype == torch.float16
    assert p.qk_scale == 1 / 8 and p.mask_type == W.MASK_NONE and p.want_lse


def test_prefill_prefix():
    p = W.prefill_prefix()
    _common(p, 4, 32, 8, 128, 128, torch.bfloat16)
    assert list(p.seq_len) == [128, 256, 512, 1024]
    assert list(p.kv_seq_len - p.seq_len) == [0, 512, 1024, 3072]
    assert math.isclose(p.qk_scale, 1 / math.sqrt(128), rel_tol=1e-7)
    assert p.mask_type == W.MASK_CAUSAL
    q = p.query.float()
    assert abs(float(q.mean())) < 0.01 and abs(float(q.std()) - 1) < 0.01     # ~N(0, 1)


def test_decode_large_batch():
    p = W.decode_large_batch()
    _common(p, 64, 32, 8, 128, 128, torch.bfloat16)
    assert all(int(x) == 1 for x in p.seq_len)
    assert all(1024 <= int(x) <= 8192 for x in p.kv_seq_len)
    assert len(set(int(x) for x in p.kv_seq_len)) > 32                          # spread, not constant
    assert p.mask_type == W.MASK_NONE and p.want_lse


def test_alibi_prefill_both_forms():
    a = W.alibi_prefill(False)
    _common(a, 2, 32, 32, 128, 128, torch.float16)
    assert list(a.seq_len) == [2048, 2048] and list(a.kv_seq_len) == [2048, 2048]
    assert a.mask_type == W.MASK_ALIBI
    h = np.arange(32)
    np.testing.assert_allclose(a.slopes.numpy(), 2.0 ** (-8.0 * (h + 1) / 32), rtol=1e-6)
    b = W.alibi_prefill(True)
    assert b.mask_type == W.MASK_CAUSAL and b.slopes is None
    assert b.pse.shape == (2, 32, 2048, 2048) and b.pse.dtype == torch.float16
    # the pse holds fp16(slope_h * (t - qpos)) on the visible (causal) entries
    for hh, i, t in [(0, 100, 3), (31, 2047, 0), (7, 1000, 1000), (15, 5, 2)]:
        want = np.float16(a.slopes[hh].item() * (t - i))
        assert b.pse[0, hh, i, t].item() == float(want)


def test_int8_long_decode():
    p = W.int8_long_decode()
    _common(p, 16, 64, 8, 128, 128, torch.bfloat16)
    assert all(int(x) == 32768 for x in p.kv_seq_len)
    assert p.key_cache.dtype == torch.int8 and p.value_cache.dtype == torch.int8
    k = p.key_cache[:64].to(torch.int16)
    assert int(k.min()) >= -127 and int(k.max()) <= 127
    for s in (p.k_scale, p.v_scale):
        assert s.shape == (8, 128) and float(s.min()) >= 0.005 and float(s.max()) <= 0.02
    for o in (p.k_offset, p.v_offset):
        assert o.shape == (8, 128) and abs(float(o.std()) - 0.1) < 0.02
    assert p.sink is not None and p.sink.shape == (64,)
