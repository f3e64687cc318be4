"""Pins for the CPU oracle: each test ties it to something other than itself.

Citations are to the pages' sections:
  * aclnnFusedInferAttentionScoreV4 / V3, "Formula";
  * V3 "lse" restriction bullet (subtract the max, exponentiate, sum, add
    the log of the sum back);
  * V4/V3 paged-attention bullet (blocks listed in blockTables form one
    logically contiguous K/V sequence);
  * ATB PrefixEncoder parameter table (qkScale, maskType, slopes, heads);
  * V4 empty-tensor rule (no key/value: out all 0, lse all inf).
"""
import dataclasses
import math
import zlib
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle_helpers import GOLDEN_DIR, dense_sdpa, load_golden


# ---------------------------------------------------------------------------
# Hand-worked closed forms (tests/golden/*.json).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", sorted(f for f in os.listdir(GOLDEN_DIR) if f.endswith(".json")))
def test_golden_rows(name):
    p, exp_out, exp_lse = load_golden(name)
    out, lse = oracle.attention(p)
    np.testing.assert_allclose(out, exp_out, rtol=0, atol=1e-6)
    fin = np.isfinite(exp_lse)
    np.testing.assert_allclose(lse[fin], exp_lse[fin], rtol=0, atol=1e-6)
    assert np.all(np.isinf(lse[~fin]) & (lse[~fin] > 0))


# ---------------------------------------------------------------------------
# Library routine: torch scaled_dot_product_attention (float64) on the
# densely gathered sequences.
# ---------------------------------------------------------------------------
SDPA_CASES = [
    dict(seq_len=[1, 1, 1], kv_seq_len=[5, 17, 33], head_num=4, kv_head_num=4, head_size=16,
         block_size=4, dtype="f16", mask_type=W.MASK_NONE),
    dict(seq_len=[3, 7], kv_seq_len=[9, 7], head_num=8, kv_head_num=2, head_size=8,
         block_size=4, dtype="bf16", mask_type=W.MASK_CAUSAL),
    dict(seq_len=[5, 4], kv_seq_len=[11, 4], head_num=4, kv_head_num=1, head_size=8,
         block_size=2, dtype="f16", mask_type=W.MASK_ALIBI, alibi_slopes=True),
    dict(seq_len=[4, 2], kv_seq_len=[6, 5], head_num=2, kv_head_num=2, head_size=8,
         block_size=4, dtype="f16", mask_type=W.MASK_CAUSAL, pse=True),
    dict(seq_len=[1, 1], kv_seq_len=[13, 3], head_num=4, kv_head_num=2, head_size=8,
         block_size=4, dtype="bf16", sink=True),
    dict(seq_len=[1, 2], kv_seq_len=[9, 6], head_num=8, kv_head_num=2, head_size=16,
         block_size=4, dtype="bf16", kv_dtype="i8", sink=True, mask_type=W.MASK_CAUSAL),
    dict(seq_len=[1], kv_seq_len=[7], head_num=2, kv_head_num=1, head_size=8,
         block_size=4, dtype="f16", kv_dtype="i8", int8_offsets=False),
]


@pytest.mark.parametrize("case", range(len(SDPA_CASES)))
def test_matches_torch_sdpa(case):
    p = W.make_problem(seed=100 + case, spare_blocks=2, **SDPA_CASES[case])
    out, _ = oracle.attention(p)
    ref = dense_sdpa(p)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("kw", [
    dict(mask_type=W.MASK_CAUSAL),
    dict(band=(3, 1), sink=True),
    dict(kv_dtype="i8", k_antiquant="token", v_antiquant="channel", sink=True),
    dict(mask_type=W.MASK_CAUSAL, pse=True),
    dict(kv_layout=1, mask_type=W.MASK_ALIBI, alibi_slopes=True),
])
def test_row_subset_matches_full(kw):
    """The sampled-rows mode (used by the full-size GPU tests) gives exactly
    the rows of the full computation, for every feature it is sampled with."""
    p = W.make_problem(seed=7, seq_len=[3, 5], kv_seq_len=[10, 5], head_num=4, kv_head_num=2,
                       head_size=8, block_size=4, **kw)
    out, lse = oracle.attention(p)
    rows = [(0, 1), (7, 3), (4, 0)]
    so, sl = oracle.attention(p, rows=rows)
    for r, (t, h) in enumerate(rows):
        assert np.array_equal(so[r], out[t, h]) and sl[r] == lse[t, h]


# ---------------------------------------------------------------------------
# Invariants.
# ---------------------------------------------------------------------------
def test_rows_sum_to_one_and_lse_is_logsumexp():
    """Weights sum to 1 (no sink) and lse = log(sum_t exp(s_t)) computed
    directly with math.fsum (no max subtraction)."""
    p = W.make_problem(seed=8, seq_len=[2, 3], kv_seq_len=[9, 3], head_num=2, kv_head_num=1,
                       head_size=8, block_size=4, dtype="f16", mask_type=W.MASK_CAUSAL)
    cu = p.cu_seq()
    for b in range(p.batch):
        for i in range(int(p.seq_len[b])):
            for h in range(p.head_num):
                probs, _, lse = oracle.row_probs(p, b, i, h)
                assert math.isclose(math.fsum(probs), 1.0, abs_tol=1e-12)
                # scores from the dense gather, in float64
                kl = int(p.kv_seq_len[b])
                qpos = kl - int(p.seq_len[b]) + i
                t = np.arange(kl)
                blk = p.block_tables[b].numpy()[t // p.block_size]
                k = p.key_cache.double().numpy()[blk, t % p.block_size, h // 2]
                q = p.query.double().numpy()[cu[b] + i, h]
                s = [p.qk_scale * float(np.dot(q, k[j])) for j in range(qpos + 1)]
                assert math.isclose(lse, math.log(math.fsum(math.exp(x) for x in s)),
                                    rel_tol=0, abs_tol=1e-12)
                assert np.all(probs[qpos + 1:] == 0.0)


def test_rows_with_sink_sum_to_one_minus_sink_weight():
    p = W.make_problem(seed=9, seq_len=[1, 1], kv_seq_len=[6, 11], head_num=4, kv_head_num=2,
                       head_size=8, block_size=4, dtype="bf16", sink=True)
    for b in range(2):
        for h in range(4):
            probs, _, lse = oracle.row_probs(p, b, 0, h)
            sink_w = math.exp(float(p.sink[h]) - lse)
            assert math.isclose(math.fsum(probs) + sink_w, 1.0, abs_tol=1e-12)


def test_block_permutation_invariance_exact():
    p = W.make_problem(seed=10, seq_len=[3, 1, 4], kv_seq_len=[19, 8, 30], head_num=4,
                       kv_head_num=2, head_size=8, block_size=4, mask_type=W.MASK_CAUSAL,
                       spare_blocks=3)
    out, lse = oracle.attention(p)
    for s in range(3):
        out2, lse2 = oracle.attention(W.permute_blocks(p, 50 + s))
        assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_unread_cache_slots_and_table_padding_are_ignored():
    """NaN in the slots past kvSeqLen and garbage table padding change nothing."""
    base = dict(seq_len=[1, 2], kv_seq_len=[6, 9], head_num=2, kv_head_num=2, head_size=8,
                block_size=4, mask_type=W.MASK_CAUSAL, max_blocks=5)
    p = W.make_problem(seed=11, **base)
    q = W.make_problem(seed=11, tail_fill=float("nan"), pad_value=123456, **base)
    a, la = oracle.attention(p)
    b, lb = oracle.attention(q)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_single_key_returns_value_row_exactly():
    p = W.make_problem(seed=12, seq_len=[1, 1], kv_seq_len=[1, 1], head_num=4, kv_head_num=2,
                       head_size=8, block_size=4, dtype="bf16", sink=False)
    out, _ = oracle.attention(p)
    for b in range(2):
        blk = int(p.block_tables[b, 0])
        for h in range(4):
            assert np.array_equal(out[b, h], p.value_cache[blk, 0, h // 2].double().numpy())


def test_dominant_key_selects_its_value_row():
    """Make one key's score exceed all others by > 110; the output is that
    key's value row (up to e^-110)."""
    p = W.make_problem(seed=13, seq_len=[1], kv_seq_len=[23], head_num=1, kv_head_num=1,
                       head_size=8, block_size=4, dtype="f16", qk_scale=1.0)
    q = p.query[0, 0].double()
    for target in range(23):
        kc = p.key_cache.clone()
        blk = int(p.block_tables[0, target // 4])
        kc[blk, target % 4, 0] = (q * 200.0 / float(q.norm() ** 2)).to(torch.float16)
        pp = dataclasses.replace(p, key_cache=kc)
        out, _ = oracle.attention(pp)
        v = p.value_cache[blk, target % 4, 0].double().numpy()
        np.testing.assert_allclose(out[0, 0], v, rtol=0, atol=1e-30)


def test_gqa_equals_mha_with_repeated_kv_heads():
    p = W.make_problem(seed=14, seq_len=[2, 3], kv_seq_len=[7, 12], head_num=6, kv_head_num=2,
                       head_size=8, block_size=4, mask_type=W.MASK_CAUSAL)
    out, lse = oracle.attention(p)
    mha = dataclasses.replace(p, kv_head_num=6,
                              key_cache=p.key_cache.repeat_interleave(3, dim=2).contiguous(),
                              value_cache=p.value_cache.repeat_interleave(3, dim=2).contiguous())
    out2, lse2 = oracle.attention(mha)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_zero_scale_gives_mean_of_values():
    p = W.make_problem(seed=15, seq_len=[1, 1], kv_seq_len=[5, 12], head_num=2, kv_head_num=2,
                       head_size=8, block_size=4, qk_scale=0.0)
    out, lse = oracle.attention(p)
    for b in range(2):
        kl = int(p.kv_seq_len[b])
        t = np.arange(kl)
        blk = p.block_tables[b].numpy()[t // 4]
        for h in range(2):
            v = p.value_cache.double().numpy()[blk, t % 4, h]
            np.testing.assert_allclose(out[b, h], v.mean(0), rtol=0, atol=1e-14)
            assert math.isclose(lse[b, h], math.log(kl), abs_tol=1e-14)


def test_alibi_with_zero_slopes_equals_causal():
    base = dict(seq_len=[3, 2], kv_seq_len=[8, 2], head_num=2, kv_head_num=1, head_size=8,
                block_size=4)
    p = W.make_problem(seed=16, mask_type=W.MASK_ALIBI, alibi_slopes=True, **base)
    p = dataclasses.replace(p, slopes=torch.zeros(2))
    c = W.make_problem(seed=16, mask_type=W.MASK_CAUSAL, **base)
    a, la = oracle.attention(p)
    b, lb = oracle.attention(c)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_pse_equal_to_alibi_bias_matches_alibi_path():
    """The full pse tensor holding the ALiBi bias (with the causal mask)
    reproduces the slope form up to the pse tensor's fp16 rounding."""
    base = dict(seq_len=[4, 3], kv_seq_len=[9, 3], head_num=2, kv_head_num=2, head_size=8,
                block_size=4, dtype="f16")
    a = W.make_problem(seed=17, mask_type=W.MASK_ALIBI, alibi_slopes=True, **base)
    b = W.make_problem(seed=17, mask_type=W.MASK_CAUSAL, pse=True, **base)
    oa, _ = oracle.attention(a)
    ob, _ = oracle.attention(b)
    np.testing.assert_allclose(oa, ob, rtol=0, atol=5e-3)


def test_sink_limits():
    base = dict(seq_len=[1, 1], kv_seq_len=[5, 9], head_num=2, kv_head_num=2, head_size=8,
                block_size=4)
    p = W.make_problem(seed=18, **base)
    s = W.make_problem(seed=18, sink=True, **base)
    out, lse = oracle.attention(p)
    lo = dataclasses.replace(s, sink=torch.full((2,), -1e30))
    o2, l2 = oracle.attention(lo)
    np.testing.assert_allclose(o2, out, rtol=0, atol=1e-15)
    np.testing.assert_allclose(l2, lse, rtol=0, atol=1e-15)
    hi = dataclasses.replace(s, sink=torch.full((2,), 1e4))
    o3, l3 = oracle.attention(hi)
    np.testing.assert_allclose(o3, 0.0, atol=1e-300)
    np.testing.assert_allclose(l3, 1e4, rtol=1e-12)


def test_int8_unit_scale_zero_offset_equals_float_cache():
    """scale 1 / offset 0 int8 cache equals the fp16 cache holding the same
    integers (exactly representable)."""
    p = W.make_problem(seed=19, seq_len=[1, 1], kv_seq_len=[7, 13], head_num=4, kv_head_num=2,
                       head_size=8, block_size=4, dtype="f16", kv_dtype="i8",
                       int8_offsets=False, qk_scale=0.01)
    one = torch.ones(2, 8)
    pi = dataclasses.replace(p, k_scale=one, v_scale=one, k_offset=torch.zeros(2, 8),
                             v_offset=None)
    pf = dataclasses.replace(p, key_cache=p.key_cache.to(torch.float16),
                             value_cache=p.value_cache.to(torch.float16), k_scale=None,
                             v_scale=None, k_offset=None, v_offset=None)
    a, la = oracle.attention(pi)
    b, lb = oracle.attention(pf)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_empty_kv_rows():
    p = W.make_problem(seed=20, seq_len=[1, 1], kv_seq_len=[0, 4], head_num=2, kv_head_num=2,
                       head_size=8, block_size=4)
    out, lse = oracle.attention(p)
    assert np.all(out[0] == 0.0) and np.all(np.isposinf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


def test_planted_mistake_is_caught():
    """A wrong GQA mapping (h % KVH instead of h // g) planted on the CPU
    side of the comparison must fail the SDPA pin: the pin has teeth."""
    p = W.make_problem(seed=21, seq_len=[1], kv_seq_len=[9], head_num=4, kv_head_num=2,
                       head_size=8, block_size=4)
    ref = dense_sdpa(p)
    # planted: interleave heads the other way
    perm = [0, 2, 1, 3]
    wrong = dataclasses.replace(p, query=p.query[:, perm].contiguous())
    out, _ = oracle.attention(wrong)
    assert not np.allclose(out[:, perm], ref, atol=1e-6)


@pytest.mark.parametrize("kind", ["decode_gqa_sink", "prefill_causal", "int8_offsets", "alibi_mtp"])
def test_oracle_bnnbsd_layout_matches_bnbsh(kind):
    """The same cache stored BnNBsD ([numBlocks, KVH, bs, D], V3 paged attention
    constraints) gives exactly the BnBsH result: the layout only moves rows.
    KVH > 1 and bs > 1 with distinct values, so a swapped (head, row) index in
    either resolve changes the answer."""
    cfg = dict(
        decode_gqa_sink=dict(seq_len=[1, 1, 1], kv_seq_len=[37, 80, 5], head_num=8,
                             kv_head_num=2, head_size=64, block_size=16, sink=True),
        prefill_causal=dict(seq_len=[20, 7], kv_seq_len=[45, 7], head_num=4, kv_head_num=2,
                            head_size=64, block_size=16, mask_type=W.MASK_CAUSAL),
        int8_offsets=dict(seq_len=[1, 2], kv_seq_len=[70, 33], head_num=8, kv_head_num=4,
                          head_size=128, block_size=16, kv_dtype="i8", sink=True),
        alibi_mtp=dict(seq_len=[3, 2], kv_seq_len=[40, 64], head_num=6, kv_head_num=3,
                       head_size=64, block_size=32, mask_type=W.MASK_ALIBI, alibi_slopes=True),
    )[kind]
    p = W.make_problem(seed=zlib.crc32(kind.encode()), **cfg)
    q = W.to_bnnbsd(p)
    assert q.kv_layout == 1 and q.block_size == p.block_size
    assert tuple(q.key_cache.shape) == (p.key_cache.shape[0], p.kv_head_num, p.block_size,
                                        p.head_size)
    o1, l1 = oracle.attention(p)
    o2, l2 = oracle.attention(q)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # and it is not the same numbers by accident: reading the BnNBsD pool as
    # if it were BnBsH (same shape only when KVH == bs) is impossible here, so
    # check instead that permuting heads inside the pool changes the result
    swapped = dataclasses.replace(q, key_cache=q.key_cache.flip(1).contiguous())
    o3, _ = oracle.attention(swapped)
    assert not np.allclose(o1, o3)


def _int8_problem(k_antiquant="token", v_antiquant="token", **kw):
    cfg = dict(seq_len=[1, 2, 1], kv_seq_len=[70, 33, 5], head_num=8, kv_head_num=2,
               head_size=128, block_size=16, kv_dtype="i8", sink=True)
    cfg.update(kw)
    return W.make_problem(seed=zlib.crc32((k_antiquant + v_antiquant).encode()) % 1000,
                          k_antiquant=k_antiquant, v_antiquant=v_antiquant, **cfg)


@pytest.mark.parametrize("km,vm", [(1, 1), (1, 0), (0, 1)])
def test_oracle_per_token_reduces_to_per_channel_for_constant_scales(km, vm):
    """V3 fake-quantization modes: per-token (scale/offset per (b, t), [B, S])
    and per-channel ([KVH, D]) are the same dequantisation when every scale
    (offset) is one constant: the results agree bitwise, in any mix of K/V
    modes."""
    p = _int8_problem()
    S = p.k_scale.shape[1]
    def with_modes(pp, mk, mv):
        ks = (p.batch, S) if mk else (p.kv_head_num, p.head_size)
        vs = (p.batch, S) if mv else (p.kv_head_num, p.head_size)
        return dataclasses.replace(pp, k_scale=torch.full(ks, 0.0125), k_offset=torch.full(ks, 0.25),
                                   v_scale=torch.full(vs, 0.015625), v_offset=torch.full(vs, -0.5),
                                   k_antiquant_mode=mk, v_antiquant_mode=mv)
    o0, l0 = oracle.attention(with_modes(p, 0, 0))
    o1, l1 = oracle.attention(with_modes(p, km, vm))
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_oracle_per_token_uses_each_tokens_own_scale():
    """Per-token scales are indexed by (sequence, cached position): against
    torch SDPA on the pool dequantised token by token; doubling every V scale
    doubles the output exactly and leaves lse alone; scales of positions past
    kvSeqLen are never read."""
    p = _int8_problem(sink=False)
    out, lse = oracle.attention(p)
    ref_out = dense_sdpa(p)
    assert np.abs(out - ref_out).max() < 1e-9
    p2 = dataclasses.replace(p, v_scale=p.v_scale * 2, v_offset=p.v_offset)
    out2, lse2 = oracle.attention(p2)
    assert np.array_equal(out2, 2 * out) and np.array_equal(lse2, lse)
    ks = p.k_scale.clone()
    for b in range(p.batch):
        ks[b, int(p.kv_seq_len[b]):] = float("nan")      # never read
    out3, lse3 = oracle.attention(dataclasses.replace(p, k_scale=ks))
    assert np.array_equal(out3, out) and np.array_equal(lse3, lse)
    ks2 = p.k_scale.clone()
    ks2[1, 3] *= 3.0                                      # a read position of sequence 1
    out4, _ = oracle.attention(dataclasses.replace(p, k_scale=ks2))
    rows_seq1 = slice(int(p.seq_len[0]), int(p.seq_len[0] + p.seq_len[1]))
    assert not np.allclose(out4[rows_seq1], out[rows_seq1])
    assert np.array_equal(out4[:int(p.seq_len[0])], out[:int(p.seq_len[0])])


def _band_problem(band, mask=W.MASK_NONE, **kw):
    cfg = dict(seq_len=[40, 1, 7, 3], kv_seq_len=[100, 90, 7, 60], head_num=4, kv_head_num=2,
               head_size=64, block_size=16)
    cfg.update(kw)
    return W.make_problem(seed=23, mask_type=mask, band=band, **cfg)


def test_oracle_band_special_cases():
    """Band mask (V3 sparseMode 4, preTokens / nextTokens): with preTokens
    past every key and nextTokens = 0 it is the causal mask; with both past
    every key it is no mask (bitwise)."""
    big = 10 ** 6
    causal = oracle.attention(_band_problem(None, mask=W.MASK_CAUSAL))
    band_causal = oracle.attention(_band_problem((big, 0)))
    assert all(np.array_equal(x, y) for x, y in zip(causal, band_causal))
    full = oracle.attention(_band_problem(None))
    band_full = oracle.attention(_band_problem((big, big)))
    assert all(np.array_equal(x, y) for x, y in zip(full, band_full))


def test_oracle_band_single_key():
    """preTokens = nextTokens = 0 leaves each row exactly one key, its own
    position qpos: out is that key's value row (softmax of one score is 1) and
    lse is the scaled score itself."""
    p = _band_problem((0, 0), want_lse=True)
    out, lse = oracle.attention(p)
    g = p.head_num // p.kv_head_num
    bs = p.block_size
    cu = p.cu_seq()
    q = p.query.double()
    for b in range(p.batch):
        kl, ql = int(p.kv_seq_len[b]), int(p.seq_len[b])
        for i in range(ql):
            qpos = kl - ql + i
            blk = int(p.block_tables[b, qpos // bs])
            for h in range(p.head_num):
                kvh = h // g
                k = p.key_cache[blk, qpos % bs, kvh].double()
                v = p.value_cache[blk, qpos % bs, kvh].double().numpy()
                r = cu[b] + i
                assert np.array_equal(out[r, h], v)
                score = p.qk_scale * float(q[r, h] @ k)
                assert abs(lse[r, h] - score) <= 1e-12 * max(1.0, abs(score))


@pytest.mark.parametrize("band", [(20, 3), (0, 0), (5, -2), (-3, 40)])
def test_oracle_band_against_sdpa(band):
    """Against torch SDPA with the band written out as an additive mask
    (t - qpos in [-preTokens, nextTokens]); rows whose band holds no key give
    out 0 and lse +inf (the empty-row rule)."""
    p = _band_problem(band, sink=True)
    out, lse = oracle.attention(p)
    ref = dense_sdpa(p)
    empty = np.isinf(lse)
    cu = p.cu_seq()
    # which rows must be empty: band interval clipped to [0, kvSeqLen) is void
    for b in range(p.batch):
        kl, ql = int(p.kv_seq_len[b]), int(p.seq_len[b])
        for i in range(ql):
            qpos = kl - ql + i
            lo, hi = max(0, qpos - band[0]), min(kl - 1, qpos + band[1])
            assert bool(empty[cu[b] + i].all()) == (hi < lo)
    assert np.all(out[empty] == 0)
    assert np.abs(out[~empty] - ref[~empty]).max() < 1e-9
