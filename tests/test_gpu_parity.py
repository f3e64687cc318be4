"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Tolerances: max |err| <= 2e-2 and mean |err| <= 2e-3 on
the fp16/bf16 output, |err| <= 5e-3 on the fp32 lse; gather/index work is
checked bit-exactly (single key, dominant key, block permutation)."""
import dataclasses
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from fia_testlib import compare, compare_full, head_slice, run_gpu

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------
# Small cases, full comparison.  Sizes span several tiles and a ragged tail.
# ---------------------------------------------------------------------------
DECODE_CASES = {
    "mha_d64_bs16_f16": dict(seq_len=[1, 1, 1], kv_seq_len=[37, 64, 1], head_num=4, kv_head_num=4,
                             head_size=64, block_size=16, dtype="f16", qk_scale=0.125),
    "gqa4_bs16_ragged_bf16": dict(seq_len=[1] * 5, kv_seq_len=[1, 15, 129, 700, 1000],
                                  head_num=16, kv_head_num=4, head_size=128, block_size=16),
    "gqa8_bs128_bf16": dict(seq_len=[1] * 3, kv_seq_len=[300, 1025, 2049], head_num=32,
                            kv_head_num=4, head_size=128, block_size=128),
    "gqa16_bs64_f16_sink": dict(seq_len=[1, 1], kv_seq_len=[513, 77], head_num=16, kv_head_num=1,
                                head_size=128, block_size=64, dtype="f16", sink=True),
    "mtp_causal_q3_g4": dict(seq_len=[3, 4, 1], kv_seq_len=[45, 260, 9], head_num=8,
                             kv_head_num=2, head_size=128, block_size=32, mask_type=W.MASK_CAUSAL),
    "mtp_alibi_q2_g4": dict(seq_len=[2, 2], kv_seq_len=[100, 333], head_num=8, kv_head_num=2,
                            head_size=128, block_size=16, mask_type=W.MASK_ALIBI,
                            alibi_slopes=True, dtype="f16"),
    "decode_pse": dict(seq_len=[1, 2], kv_seq_len=[90, 200], head_num=4, kv_head_num=2,
                       head_size=64, block_size=16, mask_type=W.MASK_CAUSAL, pse=True, dtype="f16"),
    "nan_tail_slots": dict(seq_len=[1, 1], kv_seq_len=[70, 131], head_num=8, kv_head_num=2,
                           head_size=128, block_size=64, tail_fill=float("nan"), pad_value=-1),
    "int8_sink_offsets": dict(seq_len=[1, 1, 1], kv_seq_len=[200, 1500, 65], head_num=16,
                              kv_head_num=2, head_size=128, block_size=128, kv_dtype="i8",
                              sink=True),
    "int8_symmetric_f16": dict(seq_len=[1, 1], kv_seq_len=[333, 64], head_num=8, kv_head_num=8,
                               head_size=128, block_size=32, dtype="f16", kv_dtype="i8",
                               int8_offsets=False),
    "int8_mtp_causal": dict(seq_len=[2, 3], kv_seq_len=[50, 700], head_num=8, kv_head_num=2,
                            head_size=128, block_size=64, kv_dtype="i8",
                            mask_type=W.MASK_CAUSAL),
    # block sizes that are not powers of two, and the largest accepted (256):
    # TMA boxes of gcd(blockSize, 64) rows
    "bs48_gqa4_bf16": dict(seq_len=[1, 1, 1], kv_seq_len=[100, 481, 48], head_num=16,
                           kv_head_num=4, head_size=128, block_size=48),
    "bs80_mtp_causal_f16": dict(seq_len=[2, 1], kv_seq_len=[333, 80], head_num=8, kv_head_num=2,
                                head_size=128, block_size=80, dtype="f16",
                                mask_type=W.MASK_CAUSAL),
    "bs256_gqa8_sink": dict(seq_len=[1, 1], kv_seq_len=[700, 2000], head_num=32, kv_head_num=4,
                            head_size=128, block_size=256, sink=True),
    "bs80_d64": dict(seq_len=[1, 1], kv_seq_len=[161, 79], head_num=4, kv_head_num=2,
                     head_size=64, block_size=80),
    "int8_bs48": dict(seq_len=[1, 1], kv_seq_len=[500, 47], head_num=16, kv_head_num=2,
                      head_size=128, block_size=48, kv_dtype="i8", sink=True),
    "int8_bs256_per_token": dict(seq_len=[1, 1], kv_seq_len=[1000, 300], head_num=16,
                                 kv_head_num=2, head_size=128, block_size=256, kv_dtype="i8",
                                 k_antiquant="token", v_antiquant="token"),
}

PREFILL_CASES = {
    "causal_gqa_prefix_bs16": dict(seq_len=[37, 130], kv_seq_len=[100, 300], head_num=8,
                                   kv_head_num=2, head_size=128, block_size=16,
                                   mask_type=W.MASK_CAUSAL),
    "causal_bs128_f16": dict(seq_len=[256, 129], kv_seq_len=[256, 400], head_num=4, kv_head_num=4,
                             head_size=128, block_size=128, dtype="f16", mask_type=W.MASK_CAUSAL),
    "nomask_d64_bs32": dict(seq_len=[70, 200], kv_seq_len=[70, 333], head_num=4, kv_head_num=2,
                            head_size=64, block_size=32),
    "alibi_causal": dict(seq_len=[200, 64], kv_seq_len=[200, 300], head_num=4, kv_head_num=4,
                         head_size=128, block_size=64, mask_type=W.MASK_ALIBI, alibi_slopes=True,
                         dtype="f16"),
    "pse_causal": dict(seq_len=[150, 40], kv_seq_len=[150, 260], head_num=4, kv_head_num=4,
                       head_size=128, block_size=64, mask_type=W.MASK_CAUSAL, pse=True,
                       dtype="f16"),
    "sink_gqa": dict(seq_len=[140, 30], kv_seq_len=[300, 30], head_num=8, kv_head_num=2,
                     head_size=128, block_size=32, mask_type=W.MASK_CAUSAL, sink=True),
    "nan_tail_slots_prefill": dict(seq_len=[100, 50], kv_seq_len=[150, 50], head_num=4,
                                   kv_head_num=1, head_size=128, block_size=64,
                                   mask_type=W.MASK_CAUSAL, tail_fill=float("nan")),
    "wide_group_decode_shape": dict(seq_len=[1, 1], kv_seq_len=[300, 129], head_num=32,
                                    kv_head_num=1, head_size=128, block_size=16),
    # tile pairing: odd group size -> one pair + one single tile per KV head
    "odd_group_g3": dict(seq_len=[150, 20], kv_seq_len=[400, 20], head_num=6, kv_head_num=2,
                         head_size=128, block_size=32, mask_type=W.MASK_CAUSAL),
    # g = 1: consecutive token tiles pair up with unequal key-tile counts
    "mha_three_tiles_prefix": dict(seq_len=[300], kv_seq_len=[700], head_num=2, kv_head_num=2,
                                   head_size=128, block_size=64, mask_type=W.MASK_CAUSAL,
                                   dtype="f16"),
    # pse rows 16-byte aligned: fetched by TMA into per-warp slots
    "pse_tma_rows_aligned": dict(seq_len=[200, 70], kv_seq_len=[264, 70], head_num=4,
                                 kv_head_num=2, head_size=128, block_size=16,
                                 mask_type=W.MASK_CAUSAL, pse=True),
    "pse_no_mask_d64": dict(seq_len=[130], kv_seq_len=[256], head_num=2, kv_head_num=2,
                            head_size=64, block_size=32, pse=True, dtype="f16"),
    "d64_pairs_causal_sink": dict(seq_len=[256, 100], kv_seq_len=[300, 400], head_num=8,
                                  kv_head_num=2, head_size=64, block_size=64,
                                  mask_type=W.MASK_CAUSAL, sink=True),
    # block sizes that are not powers of two, and 256: TMA boxes of
    # gcd(blockSize, 128) rows, block runs that straddle key tiles
    "bs48_causal_prefix": dict(seq_len=[140, 60], kv_seq_len=[400, 60], head_num=8,
                               kv_head_num=2, head_size=128, block_size=48,
                               mask_type=W.MASK_CAUSAL),
    "bs80_nomask_d64_f16": dict(seq_len=[130, 50], kv_seq_len=[250, 81], head_num=4,
                                kv_head_num=2, head_size=64, block_size=80, dtype="f16"),
    "bs256_causal_prefix_sink": dict(seq_len=[200, 129], kv_seq_len=[900, 129], head_num=8,
                                     kv_head_num=2, head_size=128, block_size=256,
                                     mask_type=W.MASK_CAUSAL, sink=True),
    "bs256_alibi_f16": dict(seq_len=[300], kv_seq_len=[300], head_num=4, kv_head_num=4,
                            head_size=128, block_size=256, dtype="f16",
                            mask_type=W.MASK_ALIBI, alibi_slopes=True),
    "bs48_pse_causal": dict(seq_len=[150], kv_seq_len=[200], head_num=4, kv_head_num=2,
                            head_size=128, block_size=48, mask_type=W.MASK_CAUSAL, pse=True),
    # ALiBi with the in-tile bias as an extra QK^T K-step: GQA pairs whose two
    # tiles carry different heads' slopes, a long prefix (biases in the
    # hundreds), D = 64; a negative qkScale takes the softmax-side bias instead
    "alibi_gqa_long_prefix_bf16": dict(seq_len=[200, 64], kv_seq_len=[2300, 64], head_num=8,
                                       kv_head_num=2, head_size=128, block_size=64,
                                       mask_type=W.MASK_ALIBI, alibi_slopes=True),
    "alibi_d64_gqa_f16": dict(seq_len=[130, 260], kv_seq_len=[400, 260], head_num=8,
                              kv_head_num=4, head_size=64, block_size=32, dtype="f16",
                              mask_type=W.MASK_ALIBI, alibi_slopes=True),
    "alibi_negative_scale_f16": dict(seq_len=[150], kv_seq_len=[300], head_num=4, kv_head_num=4,
                                     head_size=128, block_size=64, dtype="f16", qk_scale=-0.05,
                                     mask_type=W.MASK_ALIBI, alibi_slopes=True),
}


# int8 cache with more than 16 query rows per KV head: prefix prefill over an
# int8 cache and multi-token decode with seqLen * g > 16 take the tensor-core
# kernel, which dequantises each K / V tile into the query dtype in shared
# memory (V3 fake-quantization: per-channel and per-token scale / offset).
INT8_PREFILL_CASES = {
    "i8_prefix_causal_gqa_bs16_sink": dict(seq_len=[37, 130], kv_seq_len=[100, 300], head_num=8,
                                           kv_head_num=2, head_size=128, block_size=16,
                                           mask_type=W.MASK_CAUSAL, kv_dtype="i8", sink=True),
    "i8_prefix_per_token_bs64": dict(seq_len=[200, 64], kv_seq_len=[500, 64], head_num=8,
                                     kv_head_num=2, head_size=128, block_size=64,
                                     mask_type=W.MASK_CAUSAL, kv_dtype="i8",
                                     k_antiquant="token", v_antiquant="token"),
    "i8_channel_k_token_v_alibi_f16": dict(seq_len=[150, 40], kv_seq_len=[150, 260], head_num=4,
                                           kv_head_num=4, head_size=128, block_size=128,
                                           dtype="f16", mask_type=W.MASK_ALIBI,
                                           alibi_slopes=True, kv_dtype="i8",
                                           k_antiquant="channel", v_antiquant="token"),
    "i8_token_k_channel_v_symmetric": dict(seq_len=[130], kv_seq_len=[700], head_num=2,
                                           kv_head_num=1, head_size=128, block_size=32,
                                           kv_dtype="i8", k_antiquant="token",
                                           v_antiquant="channel", int8_offsets=False),
    "i8_pse_causal_f16": dict(seq_len=[150, 40], kv_seq_len=[150, 260], head_num=4,
                              kv_head_num=2, head_size=128, block_size=64,
                              mask_type=W.MASK_CAUSAL, pse=True, dtype="f16", kv_dtype="i8"),
    "i8_pse_tma_rows_bs16": dict(seq_len=[200, 70], kv_seq_len=[264, 70], head_num=4,
                                 kv_head_num=2, head_size=128, block_size=16,
                                 mask_type=W.MASK_CAUSAL, pse=True, kv_dtype="i8"),
    "i8_band_prefill": dict(seq_len=[300, 130], kv_seq_len=[700, 130], head_num=8,
                            kv_head_num=2, head_size=128, block_size=64, band=(200, 0),
                            kv_dtype="i8", sink=True),
    "i8_mtp_g8_q3_causal_sink": dict(seq_len=[3, 3, 2], kv_seq_len=[700, 1500, 40], head_num=64,
                                     kv_head_num=8, head_size=128, block_size=128,
                                     mask_type=W.MASK_CAUSAL, kv_dtype="i8", sink=True),
    "i8_g32_per_token_bs48": dict(seq_len=[1, 1], kv_seq_len=[513, 90], head_num=64,
                                  kv_head_num=2, head_size=128, block_size=48, kv_dtype="i8",
                                  k_antiquant="token", v_antiquant="token"),
    "i8_bs80_odd_group_f16": dict(seq_len=[150, 20], kv_seq_len=[400, 20], head_num=6,
                                  kv_head_num=2, head_size=128, block_size=80, dtype="f16",
                                  mask_type=W.MASK_CAUSAL, kv_dtype="i8"),
    "i8_bs256_mha_three_tiles": dict(seq_len=[300], kv_seq_len=[700], head_num=2, kv_head_num=2,
                                     head_size=128, block_size=256, mask_type=W.MASK_CAUSAL,
                                     kv_dtype="i8"),
}


@pytest.mark.parametrize("name", sorted(INT8_PREFILL_CASES))
def test_int8_prefill_small(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, spare_blocks=2,
                       **INT8_PREFILL_CASES[name])
    op, out, lse = run_gpu(p, path=2)
    assert op.plan_info()["path"] == 2
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, name)
    assert op.error_word() == 0


# Decode-shaped calls with more than 16 rows per KV head (MTP with g * seqLen
# > 16, wide GQA groups): the decode kernels in 16-row chunks per unit.
DECODE_CHUNK_CASES = {
    "chunk_mtp_g8_q3_causal_sink": dict(seq_len=[3, 3, 2], kv_seq_len=[700, 1500, 40], head_num=64,
                                        kv_head_num=8, head_size=128, block_size=128,
                                        mask_type=W.MASK_CAUSAL, sink=True),
    "chunk_g32_decode_f16": dict(seq_len=[1, 1, 1], kv_seq_len=[300, 1000, 77], head_num=32,
                                 kv_head_num=1, head_size=128, block_size=64, dtype="f16"),
    "chunk_i8_mtp_g8_q3": dict(seq_len=[3, 2], kv_seq_len=[900, 300], head_num=16, kv_head_num=2,
                               head_size=128, block_size=64, kv_dtype="i8",
                               mask_type=W.MASK_CAUSAL, sink=True),
    "chunk_i8_per_token_g16_q2": dict(seq_len=[2, 1], kv_seq_len=[400, 160], head_num=32,
                                      kv_head_num=2, head_size=128, block_size=32, kv_dtype="i8",
                                      k_antiquant="token", v_antiquant="channel",
                                      mask_type=W.MASK_CAUSAL),
    "chunk_alibi_g32_q2_f16": dict(seq_len=[1, 2], kv_seq_len=[513, 90], head_num=64,
                                   kv_head_num=2, head_size=128, block_size=128, dtype="f16",
                                   mask_type=W.MASK_ALIBI, alibi_slopes=True, sink=True),
    "chunk_pse_q5_g4_d64": dict(seq_len=[5, 3], kv_seq_len=[90, 200], head_num=8, kv_head_num=2,
                                head_size=64, block_size=16, mask_type=W.MASK_CAUSAL, pse=True,
                                dtype="f16"),
    "chunk_band_q6_g8_d64": dict(seq_len=[6, 2], kv_seq_len=[500, 64], head_num=16,
                                 kv_head_num=2, head_size=64, block_size=16, band=(77, 1)),
    "chunk_128_rows_bs48": dict(seq_len=[16, 1], kv_seq_len=[700, 33], head_num=16, kv_head_num=2,
                                head_size=128, block_size=48, mask_type=W.MASK_CAUSAL),
}


@pytest.mark.parametrize("name", sorted(DECODE_CHUNK_CASES))
def test_decode_row_chunks(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, spare_blocks=2,
                       **DECODE_CHUNK_CASES[name])
    op, out, lse = run_gpu(p)
    assert op.plan_info()["path"] == 1
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, name)


# Every (sequence, KV head) in a single split: the decode units finish their
# rows (sink, int8 V dequantisation, lse) and the combine kernel is skipped.
SINGLE_SPLIT_CASES = {
    "one_split_bf16_sink": dict(seq_len=[1, 1, 1], kv_seq_len=[37, 100, 1], head_num=8,
                                kv_head_num=2, head_size=128, block_size=16, sink=True),
    "one_split_i8_channel_sink_f16": dict(seq_len=[1, 2], kv_seq_len=[120, 64], head_num=16,
                                          kv_head_num=2, head_size=128, block_size=32,
                                          dtype="f16", kv_dtype="i8", sink=True,
                                          mask_type=W.MASK_CAUSAL),
    "one_split_i8_per_token": dict(seq_len=[1, 1], kv_seq_len=[90, 128], head_num=8,
                                   kv_head_num=1, head_size=128, block_size=64, kv_dtype="i8",
                                   k_antiquant="token", v_antiquant="token"),
    "one_split_d64_chunks": dict(seq_len=[3, 1], kv_seq_len=[70, 20], head_num=16, kv_head_num=2,
                                 head_size=64, block_size=16, mask_type=W.MASK_CAUSAL),
}


@pytest.mark.parametrize("name", sorted(SINGLE_SPLIT_CASES))
def test_single_split_decode_skips_combine(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, spare_blocks=2,
                       **SINGLE_SPLIT_CASES[name])
    op, out, lse = run_gpu(p)
    info = op.plan_info()
    assert info["path"] == 1 and info["kernels_per_run"] == 1
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, name)


@pytest.mark.parametrize("name", sorted(DECODE_CASES))
def test_decode_small(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, spare_blocks=2, **DECODE_CASES[name])
    op, out, lse = run_gpu(p)
    assert op.plan_info()["path"] == 1
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, name)


@pytest.mark.parametrize("name", sorted(PREFILL_CASES))
def test_prefill_small(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, spare_blocks=2, **PREFILL_CASES[name])
    op, out, lse = run_gpu(p, path=2)
    assert op.plan_info()["path"] == 2
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, name)


def test_tiny_decode_config():
    p = W.tiny_decode()
    _, out, lse = run_gpu(p)
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, "tiny_decode")


# ---------------------------------------------------------------------------
# Bit-exact gather checks through the real kernels.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kind", ["decode", "prefill"])
def test_single_key_returns_value_row_bitwise(kind):
    if kind == "decode":
        p = W.make_problem(seed=31, seq_len=[1, 1], kv_seq_len=[1, 1], head_num=8, kv_head_num=2,
                           head_size=128, block_size=16)
    else:
        p = W.make_problem(seed=31, seq_len=[1, 1], kv_seq_len=[1, 1], head_num=32,
                           kv_head_num=1, head_size=128, block_size=16)
    _, out, _ = run_gpu(p, path=2 if kind == "prefill" else 0)
    for b in range(2):
        blk = int(p.block_tables[b, 0])
        for h in range(p.head_num):
            v = p.value_cache[blk, 0, h // (p.head_num // p.kv_head_num)].double().numpy()
            assert np.array_equal(out[b, h], v)


@pytest.mark.parametrize("kind", ["decode", "prefill"])
def test_dominant_key_bit_exact_gather(kind):
    """For every logical position t, make key t dominate (score margin > 110)
    and check the output equals V[t] bit for bit: the block-table resolve
    reached the right physical row."""
    kv = 48
    if kind == "decode":
        p = W.make_problem(seed=32, seq_len=[1], kv_seq_len=[kv], head_num=4, kv_head_num=1,
                           head_size=128, block_size=16, dtype="f16", qk_scale=1.0)
    else:
        p = W.make_problem(seed=32, seq_len=[1], kv_seq_len=[kv], head_num=32, kv_head_num=1,
                           head_size=128, block_size=16, dtype="f16", qk_scale=1.0)
    q = p.query[0, 0].double()
    qs = p.query.clone()
    qs[0, :] = p.query[0, 0]              # every head asks the same question
    for target in range(0, kv, 5):
        kc = p.key_cache.clone()
        blk = int(p.block_tables[0, target // 16])
        kc[blk, target % 16, 0] = (q * 200.0 / float(q.norm() ** 2)).to(torch.float16)
        pp = dataclasses.replace(p, key_cache=kc, query=qs)
        _, out, _ = run_gpu(pp, path=2 if kind == "prefill" else 0)
        v = p.value_cache[blk, target % 16, 0].double().numpy()
        for h in range(p.head_num):
            assert np.array_equal(out[0, h], v), (target, h)


@pytest.mark.parametrize("kind", ["decode", "prefill", "prefill_int8"])
def test_block_permutation_bitwise_invariant(kind):
    if kind == "decode":
        base = dict(seq_len=[1, 1, 1], kv_seq_len=[100, 513, 64], head_num=8, kv_head_num=2,
                    head_size=128, block_size=16)
    else:
        base = dict(seq_len=[70, 128], kv_seq_len=[170, 128], head_num=4, kv_head_num=2,
                    head_size=128, block_size=16, mask_type=W.MASK_CAUSAL)
        if kind == "prefill_int8":
            base.update(kv_dtype="i8", k_antiquant="token")
    p = W.make_problem(seed=33, spare_blocks=5, **base)
    _, out, lse = run_gpu(p)
    _, out2, lse2 = run_gpu(W.permute_blocks(p, 7))
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


@pytest.mark.parametrize("kind", ["decode", "prefill"])
def test_run_to_run_determinism(kind):
    if kind == "decode":
        p = W.make_problem(seed=34, seq_len=[1] * 4, kv_seq_len=[3000, 20, 900, 4097],
                           head_num=16, kv_head_num=2, head_size=128, block_size=64, sink=True)
    else:
        p = W.make_problem(seed=34, seq_len=[300, 20], kv_seq_len=[500, 20], head_num=8,
                           kv_head_num=2, head_size=128, block_size=64, mask_type=W.MASK_CAUSAL)
    op, out, lse = run_gpu(p)
    for _ in range(3):
        o2, l2 = op.run()
        torch.cuda.synchronize()
        assert np.array_equal(o2.float().double().cpu().numpy(), out)
        assert np.array_equal(l2.double().cpu().numpy(), lse)


def test_empty_kv_rows_and_empty_query():
    p = W.make_problem(seed=35, seq_len=[1, 1], kv_seq_len=[0, 40], head_num=4, kv_head_num=2,
                       head_size=128, block_size=16)
    _, out, lse = run_gpu(p)
    assert np.all(out[0] == 0) and np.all(np.isposinf(lse[0]))
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, "empty_kv")
    e = W.make_problem(seed=35, seq_len=[0, 0], kv_seq_len=[0, 0], head_num=4, kv_head_num=2,
                       head_size=128, block_size=16)
    op, out, _ = run_gpu(e)
    assert op.plan_info()["path"] == 0 and out.size == 0


# ---------------------------------------------------------------------------
# The five named workloads (and the f-row workloads) at full size, in the
# launch configuration the benchmark times: every output element and every
# lse against the oracle.
# ---------------------------------------------------------------------------
def _full_size(p):
    op, out, lse = run_gpu(p)
    compare_full(p, out, lse)
    return op, out, lse


def test_config_prefill_prefix_full():
    op, _, _ = _full_size(W.prefill_prefix())
    assert op.plan_info()["path"] == 2


def test_config_decode_large_batch_full():
    op, _, _ = _full_size(W.decode_large_batch())
    assert op.plan_info()["path"] == 1


def test_config_tiny_decode_full():
    op, _, _ = _full_size(W.tiny_decode())
    assert op.plan_info()["path"] == 1


def test_config_alibi_prefill_and_pse_agree():
    a = W.alibi_prefill(False)
    _, oa, la = _full_size(a)
    b = W.alibi_prefill(True)
    _, ob, lb = _full_size(b)
    # same bias in two forms: slope generated in registers vs fp16 pse tensor
    assert float(np.abs(oa - ob).max()) <= 2e-2


def test_config_int8_long_decode_full():
    op, _, _ = _full_size(W.int8_long_decode())
    assert op.plan_info()["path"] == 1


def test_config_bnnbsd_full():
    """The two BnNBsD bench workloads at full size."""
    op, _, _ = _full_size(W.decode_large_batch_bnnbsd())
    assert op.plan_info()["path"] == 1
    op, _, _ = _full_size(W.prefill_prefix_bnnbsd())
    assert op.plan_info()["path"] == 2


def test_config_mtp_decode_full():
    op, _, _ = _full_size(W.mtp_decode())
    assert op.plan_info()["path"] == 1


def test_config_int8_per_token_decode_full():
    _full_size(W.int8_per_token_decode())


def test_int8_prefix_prefill_full():
    op, _, _ = _full_size(W.int8_prefix_prefill())
    assert op.plan_info()["path"] == 2


def test_int8_mtp_decode_full():
    op, _, _ = _full_size(W.int8_mtp_decode())
    assert op.plan_info()["path"] == 1          # 3 tokens x g=8 = 24 rows: two 16-row chunks


def test_config_sliding_window_prefill_full():
    p = W.sliding_window_prefill()
    op, _, lse = _full_size(p)
    assert op.plan_info()["path"] == 2
    assert np.all(np.isfinite(lse))          # every row sees at least itself


# ---------------------------------------------------------------------------
# Consistency pins (one operator for Q_S = 1 and Q_S > 1 -- V3 / V4 Formula;
# deterministic by default -- V3 / V4 determinism statement).
# ---------------------------------------------------------------------------
# Each problem takes the prefill (tcgen05) kernel: seqLen * g > 16 rows per KV
# head.  Its heads, cut into groups small enough for the decode (split-KV)
# kernels, must give the same rows.
KERNEL_AGREE_CASES = {
    "decode_shape_g32_bf16": dict(seq_len=[1, 1, 1], kv_seq_len=[300, 1000, 77], head_num=32,
                                  kv_head_num=1, head_size=128, block_size=64),
    "mtp_causal_g8_q3": dict(seq_len=[2, 3], kv_seq_len=[200, 650], head_num=16, kv_head_num=2,
                             head_size=128, block_size=32, mask_type=W.MASK_CAUSAL),
    "alibi_sink_g32_f16": dict(seq_len=[1, 2], kv_seq_len=[513, 90], head_num=64, kv_head_num=2,
                               head_size=128, block_size=128, dtype="f16",
                               mask_type=W.MASK_ALIBI, alibi_slopes=True, sink=True),
    "band_d64_g16_q2": dict(seq_len=[2, 1], kv_seq_len=[400, 160], head_num=32, kv_head_num=2,
                            head_size=64, block_size=16, band=(100, 0)),
    # int8 cache: the int8 decode kernel against the dequantising prefill kernel
    "i8_decode_shape_g32_sink": dict(seq_len=[1, 1, 1], kv_seq_len=[300, 1000, 77], head_num=32,
                                     kv_head_num=1, head_size=128, block_size=64, kv_dtype="i8",
                                     sink=True),
    "i8_per_token_g16_q2": dict(seq_len=[2, 1], kv_seq_len=[400, 160], head_num=32,
                                kv_head_num=2, head_size=128, block_size=32, kv_dtype="i8",
                                k_antiquant="token", v_antiquant="token",
                                mask_type=W.MASK_CAUSAL),
}


@pytest.mark.parametrize("name", sorted(KERNEL_AGREE_CASES))
def test_decode_and_prefill_kernels_agree(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, **KERNEL_AGREE_CASES[name])
    op, out, lse = run_gpu(p, path=2)
    assert op.plan_info()["path"] == 2
    compare_full(p, out, lse)
    # the whole problem on the decode kernels, in 16-row chunks
    dop, dout, dlse = run_gpu(p, path=1)
    assert dop.plan_info()["path"] == 1
    compare_full(p, dout, dlse)
    assert float(np.abs(dout - out).max()) <= 2e-2
    g = p.head_num // p.kv_head_num
    qmax = int(max(p.seq_len))
    # heads per decode-sized group: the largest divisor of g with n * qmax <= 16
    n = max(d for d in range(1, g + 1) if g % d == 0 and d * qmax <= 16)
    for kvh in range(p.kv_head_num):
        for h0 in range(0, g, n):
            q = head_slice(p, kvh, h0, n)
            qop, qout, qlse = run_gpu(q)
            assert qop.plan_info()["path"] == 1
            hs = slice(kvh * g + h0, kvh * g + h0 + n)
            compare(qout, qlse, out[:, hs], lse[:, hs], q.name + " vs prefill kernel")


@pytest.mark.parametrize("kv_dtype", ["bf16", "i8"])
def test_split_count_does_not_change_result(kv_dtype):
    """One sequence planned alone (many short splits) and inside a large batch
    (few long splits): the same rows up to rounding, and both match the
    oracle."""
    big = W.make_problem(name="split_batch_" + kv_dtype, seed=61,
                         seq_len=[1] * 24, kv_seq_len=[8000] + [6000] * 23, head_num=32,
                         kv_head_num=8, head_size=128, block_size=128, kv_dtype=kv_dtype,
                         sink=True)
    alone = dataclasses.replace(big, name="split_alone_" + kv_dtype, query=big.query[:1].clone(),
                                block_tables=big.block_tables[:1].clone(),
                                seq_len=big.seq_len[:1].copy(), kv_seq_len=big.kv_seq_len[:1].copy())
    op_b, out_b, lse_b = run_gpu(big)
    op_a, out_a, lse_a = run_gpu(alone)
    sa, sb = op_a.plan_info()["split_tokens"], op_b.plan_info()["split_tokens"]
    assert sa < sb and 8000 // sa > 2 * (8000 // sb), (sa, sb)
    compare_full(alone, out_a, lse_a)
    compare(out_a, lse_a, out_b[:1], lse_b[:1], "split %d vs %d" % (sa, sb))


DETERMINISM_CASES = {
    "int8_decode_sink": dict(seq_len=[1] * 3, kv_seq_len=[3000, 70, 1500], head_num=16,
                             kv_head_num=2, head_size=128, block_size=128, kv_dtype="i8",
                             sink=True),
    "int8_per_token_mtp": dict(seq_len=[2, 1], kv_seq_len=[900, 2500], head_num=16,
                               kv_head_num=2, head_size=128, block_size=64, kv_dtype="i8",
                               k_antiquant="token", v_antiquant="token",
                               mask_type=W.MASK_CAUSAL),
    "band_prefill": dict(seq_len=[300, 130], kv_seq_len=[700, 130], head_num=8, kv_head_num=2,
                         head_size=128, block_size=64, band=(200, 0)),
    "int8_prefill_mixed_modes": dict(seq_len=[300, 130], kv_seq_len=[700, 130], head_num=8,
                                     kv_head_num=2, head_size=128, block_size=64, kv_dtype="i8",
                                     k_antiquant="token", v_antiquant="channel",
                                     mask_type=W.MASK_CAUSAL, sink=True),
    "band_decode": dict(seq_len=[1, 1], kv_seq_len=[4000, 1300], head_num=16, kv_head_num=4,
                        head_size=128, block_size=128, band=(255, 0)),
    "alibi_prefill_f16": dict(seq_len=[200, 64], kv_seq_len=[200, 300], head_num=4,
                              kv_head_num=4, head_size=128, block_size=64,
                              mask_type=W.MASK_ALIBI, alibi_slopes=True, dtype="f16"),
}


@pytest.mark.parametrize("name", sorted(DETERMINISM_CASES))
def test_run_to_run_determinism_more_kernels(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, **DETERMINISM_CASES[name])
    op, out, lse = run_gpu(p)
    for _ in range(3):
        o2, l2 = op.run()
        torch.cuda.synchronize()
        assert np.array_equal(o2.float().double().cpu().numpy(), out)
        assert np.array_equal(l2.double().cpu().numpy(), lse)
    assert op.error_word() == 0


# BnNBsD cache layout [numBlocks, kvHeadNum, blockSize, headSize] (V3 paged
# attention constraints: BnBsH or BnNBsD, the latter recommended): the kernels
# read each (block, KV head) run as one TMA box.  Checked against the oracle on
# the same cache, and bitwise against the BnBsH run of the same problem (the
# layout only changes where rows come from).
BNNBSD_CASES = {
    "decode_gqa4_bs16_ragged": dict(seq_len=[1] * 4, kv_seq_len=[1, 15, 700, 1000], head_num=16,
                                    kv_head_num=4, head_size=128, block_size=16),
    "decode_bs128_sink_f16": dict(seq_len=[1, 1], kv_seq_len=[513, 2049], head_num=16,
                                  kv_head_num=2, head_size=128, block_size=128, dtype="f16",
                                  sink=True),
    "decode_int8_offsets_sink": dict(seq_len=[1, 1, 2], kv_seq_len=[300, 1025, 64], head_num=16,
                                     kv_head_num=2, head_size=128, block_size=64, kv_dtype="i8",
                                     sink=True),
    "decode_mtp_causal_d64": dict(seq_len=[3, 1], kv_seq_len=[45, 260], head_num=8, kv_head_num=2,
                                  head_size=64, block_size=32, mask_type=W.MASK_CAUSAL),
    "prefill_causal_gqa_bs64": dict(seq_len=[130, 300], kv_seq_len=[130, 700], head_num=8,
                                    kv_head_num=2, head_size=128, block_size=64,
                                    mask_type=W.MASK_CAUSAL),
    "prefill_alibi_mha_bs32_f16": dict(seq_len=[200], kv_seq_len=[333], head_num=4, kv_head_num=4,
                                       head_size=128, block_size=32, dtype="f16",
                                       mask_type=W.MASK_ALIBI, alibi_slopes=True),
    "prefill_pse_causal_bs128": dict(seq_len=[140], kv_seq_len=[400], head_num=4, kv_head_num=2,
                                     head_size=128, block_size=128, mask_type=W.MASK_CAUSAL,
                                     pse=True),
    "prefill_nomask_d64_bs16": dict(seq_len=[129, 40], kv_seq_len=[129, 90], head_num=4,
                                    kv_head_num=1, head_size=64, block_size=16),
    "decode_bs48_gqa": dict(seq_len=[1, 1], kv_seq_len=[500, 47], head_num=16, kv_head_num=2,
                            head_size=128, block_size=48),
    "prefill_bs256_causal": dict(seq_len=[200, 60], kv_seq_len=[600, 60], head_num=8,
                                 kv_head_num=2, head_size=128, block_size=256,
                                 mask_type=W.MASK_CAUSAL),
    "decode_int8_bs80": dict(seq_len=[1, 2], kv_seq_len=[321, 700], head_num=16, kv_head_num=2,
                             head_size=128, block_size=80, kv_dtype="i8"),
}


@pytest.mark.parametrize("name", sorted(BNNBSD_CASES))
def test_bnnbsd_layout(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, spare_blocks=3,
                       **BNNBSD_CASES[name])
    q = W.to_bnnbsd(p)
    _, out_q, lse_q = run_gpu(q)
    ref_out, ref_lse = oracle.attention(q)
    compare(out_q, lse_q, ref_out, ref_lse, name)
    _, out_p, lse_p = run_gpu(p)
    assert np.array_equal(out_q, out_p) and np.array_equal(lse_q, lse_p)


# Per-token int8 dequantisation (V3 fake-quantization: scale/offset per
# (sequence, cached token), [B, S] f32; K and V modes may differ, e.g.
# per-channel keys with per-token values).
PER_TOKEN_CASES = {
    "tok_kv_bf16_sink": dict(seq_len=[1, 1, 1], kv_seq_len=[300, 1025, 7], head_num=16,
                             kv_head_num=2, head_size=128, block_size=64, kv_dtype="i8",
                             sink=True, k_antiquant="token", v_antiquant="token"),
    "k_channel_v_token_f16": dict(seq_len=[1, 1], kv_seq_len=[513, 64], head_num=8, kv_head_num=1,
                                  head_size=128, block_size=16, dtype="f16", kv_dtype="i8",
                                  k_antiquant="channel", v_antiquant="token"),
    "k_token_v_channel_sym": dict(seq_len=[1, 1], kv_seq_len=[200, 4100], head_num=16,
                                  kv_head_num=4, head_size=128, block_size=128, kv_dtype="i8",
                                  int8_offsets=False, k_antiquant="token", v_antiquant="channel"),
    "tok_mtp_causal_nt2": dict(seq_len=[2, 1, 2], kv_seq_len=[90, 33, 700], head_num=16,
                               kv_head_num=2, head_size=128, block_size=32, kv_dtype="i8",
                               mask_type=W.MASK_CAUSAL, k_antiquant="token", v_antiquant="token"),
    "tok_bnnbsd": dict(seq_len=[1, 1], kv_seq_len=[777, 129], head_num=16, kv_head_num=2,
                       head_size=128, block_size=64, kv_dtype="i8", sink=True,
                       k_antiquant="token", v_antiquant="token", kv_layout=1),
}


@pytest.mark.parametrize("name", sorted(PER_TOKEN_CASES))
def test_int8_per_token_antiquant(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, spare_blocks=2,
                       **PER_TOKEN_CASES[name])
    _, out, lse = run_gpu(p)
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, name)


# Band mask (V3 sparseMode 4 with preTokens / nextTokens; sliding window is
# nextTokens = 0): prefill skips the key tiles outside the band, decode reads
# only the band's keys; rows whose band holds no key give out 0, lse +inf.
BAND_CASES = {
    "prefill_gqa_window200": dict(seq_len=[300, 130], kv_seq_len=[700, 130], head_num=8,
                                  kv_head_num=2, head_size=128, block_size=64, band=(200, 0)),
    "prefill_mha_band_f16": dict(seq_len=[400], kv_seq_len=[512], head_num=4, kv_head_num=4,
                                 head_size=128, block_size=32, dtype="f16", band=(150, 20)),
    "prefill_empty_rows_sink": dict(seq_len=[200, 50], kv_seq_len=[260, 50], head_num=4,
                                    kv_head_num=2, head_size=64, block_size=16, sink=True,
                                    band=(-3, 10)),
    "prefill_pse_window": dict(seq_len=[140], kv_seq_len=[400], head_num=4, kv_head_num=2,
                               head_size=128, block_size=128, pse=True, band=(100, 0)),
    "decode_window256": dict(seq_len=[1] * 3, kv_seq_len=[4000, 100, 1300], head_num=16,
                             kv_head_num=4, head_size=128, block_size=128, band=(255, 0)),
    "decode_mtp_band_d64": dict(seq_len=[3, 2], kv_seq_len=[500, 64], head_num=8, kv_head_num=2,
                                head_size=64, block_size=16, band=(77, 1)),
    "decode_int8_window": dict(seq_len=[1, 2], kv_seq_len=[3000, 777], head_num=16,
                               kv_head_num=2, head_size=128, block_size=64, kv_dtype="i8",
                               sink=True, band=(500, 0)),
    "decode_band_excludes_all": dict(seq_len=[1, 1], kv_seq_len=[300, 40], head_num=8,
                                     kv_head_num=2, head_size=128, block_size=16, band=(-50, 60)),
}


@pytest.mark.parametrize("band", [(255, 0), (0, 0), (-70, 200), (10 ** 6, 10 ** 6), (5, -3)])
def test_band_decode_plan_covers_only_the_band(band):
    """Phase 1 under a band mask splits only the keys the band can reach: per
    sequence [kvSeqLen - seqLen - pre, kvSeqLen + next) clipped to the
    sequence, its start rounded down to a 64-key tile (empty when the band
    misses every key, which still gets one unit for the empty-row output)."""
    import paged_attention_02_b200 as fia
    kv = [4000, 100, 1300, 64, 1]
    p = W.make_problem(seed=77, seq_len=[1, 2, 1, 3, 1], kv_seq_len=kv, head_num=16,
                       kv_head_num=4, head_size=128, block_size=64, band=band)
    d = lambda t: None if t is None else t.cuda().contiguous()
    op = fia.FiaOp(d(p.query), d(p.key_cache), d(p.value_cache), d(p.block_tables),
                   [int(x) for x in p.seq_len], kv, p.head_num, p.kv_head_num, p.qk_scale,
                   band=band)
    info = op.plan_info()
    assert info["path"] == 1
    split = info["split_tokens"]
    assert split > 0 and split % 64 == 0
    units = 0
    for ql, kl in zip(p.seq_len, kv):
        lo = max(0, kl - int(ql) - band[0])
        hi = min(kl, kl + band[1])
        if hi <= lo:
            lo = hi = 0
        lo = lo // 64 * 64
        units += max(1, -(-(hi - lo) // split)) * p.kv_head_num
    assert info["work_items"] == units


@pytest.mark.parametrize("name", sorted(BAND_CASES))
def test_band_mask(name):
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, spare_blocks=2,
                       **BAND_CASES[name])
    _, out, lse = run_gpu(p)
    ref_out, ref_lse = oracle.attention(p)
    compare(out, lse, ref_out, ref_lse, name)


# ---------------------------------------------------------------------------
# CUDA graphs: fia_run (plan upload + kernels) captured once, replayed.
# ---------------------------------------------------------------------------
GRAPH_CASES = {
    "decode": dict(seq_len=[1] * 3, kv_seq_len=[700, 33, 2000], head_num=16, kv_head_num=4,
                   head_size=128, block_size=64),
    "decode_int8_sink": dict(seq_len=[1, 1], kv_seq_len=[1500, 90], head_num=16, kv_head_num=2,
                             head_size=128, block_size=128, kv_dtype="i8", sink=True),
    "prefill_causal": dict(seq_len=[200, 64], kv_seq_len=[300, 64], head_num=8, kv_head_num=2,
                           head_size=128, block_size=64, mask_type=W.MASK_CAUSAL),
}


@pytest.mark.parametrize("name", sorted(GRAPH_CASES))
def test_cuda_graph_capture_and_replay(name):
    """A captured fia_run replays to the eager result bitwise and reads its
    inputs at replay time (new query values in place give the eager result on
    the new values)."""
    import paged_attention_02_b200 as fia
    p = W.make_problem(name=name, seed=zlib.crc32(name.encode()) % 10000, **GRAPH_CASES[name])
    d = lambda t: None if t is None else t.cuda().contiguous()
    q = d(p.query)
    op = fia.FiaOp(q, d(p.key_cache), d(p.value_cache), d(p.block_tables),
                   [int(x) for x in p.seq_len], [int(x) for x in p.kv_seq_len], p.head_num,
                   p.kv_head_num, p.qk_scale, mask_type=p.mask_type, sink=d(p.sink),
                   k_scale=d(p.k_scale), k_offset=d(p.k_offset), v_scale=d(p.v_scale),
                   v_offset=d(p.v_offset), want_lse=True)
    out, lse = op.run()
    torch.cuda.synchronize()
    ref_o, ref_l = out.clone(), lse.clone()
    out.zero_()
    lse.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        op.run()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    q.copy_((q.float() * 0.5 + 0.25).to(q.dtype))
    g.replay()
    torch.cuda.synchronize()
    got_o, got_l = out.clone(), lse.clone()
    assert not torch.equal(got_o, ref_o)
    op.run()
    torch.cuda.synchronize()
    assert torch.equal(out, got_o) and torch.equal(lse, got_l)
    assert op.error_word() == 0
    del g


@pytest.mark.parametrize("kind", ["decode", "prefill"])
def test_flat_query_and_cache_forms_are_bitwise_equal(kind):
    """The 2-D query form [nTokens, H * D] and the 3-D cache form
    [numBlocks, blockSize, kvHeadNum * D] (same memory) give the same result
    as the 4-D forms, bit for bit."""
    import paged_attention_02_b200 as fia
    cfg = dict(decode=dict(seq_len=[1, 2], kv_seq_len=[300, 77], mask_type=W.MASK_CAUSAL),
               prefill=dict(seq_len=[150, 40], kv_seq_len=[400, 40],
                            mask_type=W.MASK_CAUSAL))[kind]
    p = W.make_problem(seed=91, head_num=8, kv_head_num=2, head_size=128, block_size=32, **cfg)
    _, ref, ref_lse = run_gpu(p)
    q = p.query.cuda().contiguous()
    k = p.key_cache.cuda().contiguous()
    v = p.value_cache.cuda().contiguous()
    n, h, d = q.shape
    nb, bs, kvh, _ = k.shape
    op = fia.FiaOp(q.view(n, h * d), k.view(nb, bs, kvh * d), v.view(nb, bs, kvh * d),
                   p.block_tables.cuda().contiguous(), [int(x) for x in p.seq_len],
                   [int(x) for x in p.kv_seq_len], p.head_num, p.kv_head_num, p.qk_scale,
                   mask_type=p.mask_type)
    out, lse = op.run()
    torch.cuda.synchronize()
    assert op.error_word() == 0
    assert np.array_equal(out.view(n, h, d).float().double().cpu().numpy(), ref)
    assert np.array_equal(lse.double().cpu().numpy(), ref_lse)
