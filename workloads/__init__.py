"""Seeded synthetic inputs for paged fused inference attention.

This module only *draws* inputs: random values, block-table permutations and
sequence lengths.  It holds none of the attention arithmetic, so both the
CUDA path and the CPU oracle can be fed from it without sharing any of the
method's code.

Layouts follow the ATB PrefixEncoder parameter table (ascendtb_01_0320,
"AtbSelfAttentionPrefixEncoderGetWorkspaceSize Members"):

* query       ``[nTokens, headNum, headSize]``; the tokens of all sequences
  are concatenated in batch order.
* key / value ``[numBlocks, blockSize, kvHeadNum, headSize]`` (the BnBsH
  paged cache of aclnnFusedInferAttentionScoreV3, paged-attention bullets).
* blockTables ``[batch, maxBlockNum]`` int32; entry ``[b][j]`` is the
  physical block holding logical block ``j`` of sequence ``b``.
* seqLen / kvSeqLen: host int32 arrays ``[batch]``.

Random draws use ``numpy.random.Generator(PCG64(seed))``; floating values are
drawn in fp32 and rounded to fp16/bf16 by torch (round-to-nearest-even).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

MASK_NONE = 0
MASK_ALIBI = 3
MASK_CAUSAL = 9

_TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "i8": torch.int8}


@dataclasses.dataclass
class Problem:
    """One call's worth of host-side (CPU) inputs."""

    name: str
    query: torch.Tensor                 # [nTokens, H, D]  f16 | bf16
    key_cache: torch.Tensor             # [numBlocks, bs, KVH, D] (kv_layout 1: [numBlocks, KVH, bs, D])
    value_cache: torch.Tensor           # same shape / dtype as key_cache
    block_tables: torch.Tensor          # [B, maxBlockNum] int32
    seq_len: np.ndarray                 # [B] int32 (host)
    kv_seq_len: np.ndarray              # [B] int32 (host)
    head_num: int
    kv_head_num: int
    qk_scale: float
    mask_type: int = MASK_NONE
    slopes: Optional[torch.Tensor] = None     # [H] f32
    pse: Optional[torch.Tensor] = None        # [B, H, maxQ, maxKV] f16 | bf16
    sink: Optional[torch.Tensor] = None       # [H] f32
    k_scale: Optional[torch.Tensor] = None    # [KVH, D] f32
    k_offset: Optional[torch.Tensor] = None   # [KVH, D] f32
    v_scale: Optional[torch.Tensor] = None    # [KVH, D] f32
    v_offset: Optional[torch.Tensor] = None   # [KVH, D] f32
    want_lse: bool = True
    kv_layout: int = 0                        # 0 BnBsH, 1 BnNBsD
    k_antiquant_mode: int = 0                 # int8: 0 per-channel [KVH, D], 1 per-token [B, S]
    v_antiquant_mode: int = 0
    band: Optional[Tuple[int, int]] = None    # (preTokens, nextTokens): band mask

    @property
    def batch(self) -> int:
        return int(self.seq_len.shape[0])

    @property
    def head_size(self) -> int:
        return int(self.query.shape[2])

    @property
    def block_size(self) -> int:
        return int(self.key_cache.shape[2 if self.kv_layout == 1 else 1])

    @property
    def n_tokens(self) -> int:
        return int(self.query.shape[0])

    @property
    def out_dtype(self) -> torch.dtype:
        return self.query.dtype

    @property
    def kv_is_int8(self) -> bool:
        return self.key_cache.dtype == torch.int8

    def cu_seq(self) -> np.ndarray:
        """Token offset of each sequence inside ``query`` (length B+1)."""
        return np.concatenate([[0], np.cumsum(self.seq_len.astype(np.int64))])


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(_TORCH_DTYPES[dtype])


def make_problem(
    *,
    name: str = "custom",
    seed: int,
    seq_len: Sequence[int],
    kv_seq_len: Sequence[int],
    head_num: int,
    kv_head_num: int,
    head_size: int,
    block_size: int,
    dtype: str = "bf16",
    kv_dtype: Optional[str] = None,
    qk_scale: Optional[float] = None,
    mask_type: int = MASK_NONE,
    alibi_slopes: bool = False,
    pse: bool = False,
    sink: bool = False,
    spare_blocks: int = 0,
    pad_value: int = -1,
    tail_fill: Optional[float] = None,
    int8_offsets: bool = True,
    want_lse: bool = True,
    max_blocks: Optional[int] = None,
    kv_layout: int = 0,
    k_antiquant: str = "channel",
    v_antiquant: str = "channel",
    band: Optional[Tuple[int, int]] = None,
) -> Problem:
    """Draw a seeded problem.

    * K/V pool: ``numBlocks = sum_b ceil(kvSeqLen_b / blockSize) + spare_blocks``
      blocks, filled N(0,1) (or uniform int8 in [-127, 127]).  A seeded
      ``rng.permutation(numBlocks)`` is dealt out to the sequences in batch
      order; unused block-table entries hold ``pad_value``.
    * ``tail_fill``: value written into the cache slots past kvSeqLen in each
      sequence's last block (e.g. NaN) to prove they are never read.
    * ALiBi slopes are ``2**(-8(h+1)/H)`` (caller-supplied, as the
      PrefixEncoder ``slopes`` parameter is).
    * int8 scales ``U(0.005, 0.02)`` and offsets ``N(0, 0.1)``, per
      ``k_antiquant`` / ``v_antiquant``: ``"channel"`` ``[KVH, D]`` or
      ``"token"`` ``[B, S]`` with ``S = max kvSeqLen + 3`` (a row stride
      longer than any sequence).
    * ``kv_layout=1``: the same cache stored BnNBsD ``[numBlocks, KVH, bs, D]``
      (drawn as above, then transposed).
    * ``pse``: the ALiBi bias written out as a full ``[B, H, maxQ, maxKV]``
      tensor of the query dtype, ``pse[b,h,i,t] = slope_h * (t - qpos_i)``
      with ``qpos_i = kvSeqLen_b - seqLen_b + i``.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    seq_len = np.asarray(seq_len, dtype=np.int32)
    kv_seq_len = np.asarray(kv_seq_len, dtype=np.int32)
    B = int(seq_len.shape[0])
    H, KVH, D, bs = head_num, kv_head_num, head_size, block_size
    kv_dtype = kv_dtype or dtype
    if qk_scale is None:
        qk_scale = 1.0 / math.sqrt(D)
    n_tokens = int(seq_len.sum())
    blocks_per_seq = [(int(k) + bs - 1) // bs for k in kv_seq_len]
    num_blocks = max(1, sum(blocks_per_seq) + spare_blocks)
    mb = max(1, max(blocks_per_seq) if blocks_per_seq else 1)
    if max_blocks is not None:
        mb = max(mb, max_blocks)

    query = _round(rng.standard_normal((n_tokens, H, D), dtype=np.float32), dtype)
    if kv_dtype == "i8":
        kc = torch.from_numpy(rng.integers(-127, 128, (num_blocks, bs, KVH, D)).astype(np.int8))
        vc = torch.from_numpy(rng.integers(-127, 128, (num_blocks, bs, KVH, D)).astype(np.int8))
    else:
        kc = _round(rng.standard_normal((num_blocks, bs, KVH, D), dtype=np.float32), kv_dtype)
        vc = _round(rng.standard_normal((num_blocks, bs, KVH, D), dtype=np.float32), kv_dtype)

    perm = rng.permutation(num_blocks).astype(np.int32)
    bt = np.full((B, mb), pad_value, dtype=np.int32)
    pos = 0
    for b in range(B):
        n = blocks_per_seq[b]
        bt[b, :n] = perm[pos:pos + n]
        pos += n

    if tail_fill is not None and kv_dtype != "i8":
        for b in range(B):
            kl = int(kv_seq_len[b])
            if kl % bs:
                blk = int(bt[b, kl // bs])
                kc[blk, kl % bs:] = tail_fill
                vc[blk, kl % bs:] = tail_fill

    slopes_t = None
    if alibi_slopes or pse:
        slopes_np = np.array([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=np.float32)
        slopes_t = torch.from_numpy(slopes_np)

    pse_t = None
    if pse:
        maxq = int(seq_len.max()) if B else 0
        maxkv = int(kv_seq_len.max()) if B else 0
        pse_t = torch.zeros((B, H, maxq, maxkv), dtype=_TORCH_DTYPES[dtype])
        t = torch.arange(maxkv, dtype=torch.float32)
        for b in range(B):
            q0 = int(kv_seq_len[b]) - int(seq_len[b])
            i = torch.arange(maxq, dtype=torch.float32) + q0
            rel = (t[None, :] - i[:, None])                       # [maxQ, maxKV]
            pse_t[b] = (slopes_t[:, None, None] * rel[None]).to(pse_t.dtype)

    sink_t = None
    if sink:
        sink_t = torch.from_numpy(rng.standard_normal(H, dtype=np.float32))

    ks = ko = vs = vo = None
    modes = {"channel": 0, "token": 1}
    km, vm = modes[k_antiquant], modes[v_antiquant]
    if kv_dtype == "i8":
        S = int(kv_seq_len.max()) + 3 if B else 3
        kshape = (B, S) if km else (KVH, D)
        vshape = (B, S) if vm else (KVH, D)
        ks = torch.from_numpy(rng.uniform(0.005, 0.02, kshape).astype(np.float32))
        vs = torch.from_numpy(rng.uniform(0.005, 0.02, vshape).astype(np.float32))
        if int8_offsets:
            ko = torch.from_numpy((0.1 * rng.standard_normal(kshape)).astype(np.float32))
            vo = torch.from_numpy((0.1 * rng.standard_normal(vshape)).astype(np.float32))

    p = Problem(
        name=name, query=query, key_cache=kc, value_cache=vc,
        block_tables=torch.from_numpy(bt), seq_len=seq_len, kv_seq_len=kv_seq_len,
        head_num=H, kv_head_num=KVH, qk_scale=float(qk_scale), mask_type=mask_type,
        slopes=slopes_t if mask_type == MASK_ALIBI else None, pse=pse_t, sink=sink_t,
        k_scale=ks, k_offset=ko, v_scale=vs, v_offset=vo, want_lse=want_lse,
        k_antiquant_mode=km if kv_dtype == "i8" else 0,
        v_antiquant_mode=vm if kv_dtype == "i8" else 0,
        band=tuple(band) if band is not None else None,
    )
    return to_bnnbsd(p) if kv_layout == 1 else p


def to_bnnbsd(p: Problem) -> Problem:
    """The same problem with its K/V pool stored BnNBsD ``[numBlocks, KVH, bs, D]``
    (a pure transpose of the BnBsH pool; the block table is unchanged)."""
    if p.kv_layout == 1:
        return p
    return dataclasses.replace(p, key_cache=p.key_cache.transpose(1, 2).contiguous(),
                               value_cache=p.value_cache.transpose(1, 2).contiguous(),
                               kv_layout=1)


# ---------------------------------------------------------------------------
# The five named workloads.
# ---------------------------------------------------------------------------

def tiny_decode() -> Problem:
    """Tiny paged decode: B=2, H=KVH=4, D=64, bs=16, kvSeqLen=[37,64], fp16,
    qkScale=1/8, 8 blocks dealt from a seeded permutation, no mask."""
    return make_problem(name="tiny_decode", seed=1, seq_len=[1, 1], kv_seq_len=[37, 64],
                        head_num=4, kv_head_num=4, head_size=64, block_size=16,
                        dtype="f16", qk_scale=1.0 / 8.0, mask_type=MASK_NONE,
                        spare_blocks=1)


def prefill_prefix() -> Problem:
    """Prefix-encoder prefill, causal: B=4, new=[128,256,512,1024] on cached
    prefixes [0,512,1024,3072], H=32, KVH=8, D=128, bs=128, bf16."""
    new = [128, 256, 512, 1024]
    prefix = [0, 512, 1024, 3072]
    return make_problem(name="prefill_prefix_causal_gqa", seed=2, seq_len=new,
                        kv_seq_len=[a + b for a, b in zip(new, prefix)],
                        head_num=32, kv_head_num=8, head_size=128, block_size=128,
                        dtype="bf16", mask_type=MASK_CAUSAL)


def decode_large_batch() -> Problem:
    """Decode, B=64, kvSeqLen ~ U[1024, 8192], H=32, KVH=8, D=128, bs=128,
    bf16, shuffled block tables over one shared pool."""
    rng = np.random.Generator(np.random.PCG64(3))
    kv = rng.integers(1024, 8193, 64).astype(np.int32)
    return make_problem(name="decode_large_batch", seed=3, seq_len=[1] * 64, kv_seq_len=kv,
                        head_num=32, kv_head_num=8, head_size=128, block_size=128,
                        dtype="bf16", mask_type=MASK_NONE)


def alibi_prefill(full_pse: bool = False) -> Problem:
    """ALiBi prefill: B=2, seqLen=kvSeqLen=2048, H=KVH=32, D=128, bs=128, fp16,
    slopes 2^(-8(h+1)/32), causal.  ``full_pse`` passes the same bias as a
    [B, N, 2048, 2048] fp16 pse tensor with the internally generated causal
    mask instead of the slope form."""
    return make_problem(name="alibi_prefill_pse" if full_pse else "alibi_prefill",
                        seed=4, seq_len=[2048, 2048], kv_seq_len=[2048, 2048],
                        head_num=32, kv_head_num=32, head_size=128, block_size=128,
                        dtype="f16", mask_type=MASK_CAUSAL if full_pse else MASK_ALIBI,
                        alibi_slopes=not full_pse, pse=full_pse)


def int8_long_decode() -> Problem:
    """Long-context INT8-KV decode: B=16, kvSeqLen=32768, H=64, KVH=8, D=128,
    bs=128, bf16 query, int8 K/V with per-channel fp32 scale ~U(0.005,0.02)
    and offset ~N(0,0.1), per-head learnable sink ~N(0,1)."""
    return make_problem(name="int8_long_decode_sink", seed=5, seq_len=[1] * 16,
                        kv_seq_len=[32768] * 16, head_num=64, kv_head_num=8, head_size=128,
                        block_size=128, dtype="bf16", kv_dtype="i8", mask_type=MASK_NONE,
                        sink=True)


def decode_large_batch_bnnbsd() -> Problem:
    """decode_large_batch with its pool stored BnNBsD [numBlocks, KVH, bs, D]."""
    return dataclasses.replace(to_bnnbsd(decode_large_batch()), name="decode_large_batch_bnnbsd")


def prefill_prefix_bnnbsd() -> Problem:
    """prefill_prefix with its pool stored BnNBsD [numBlocks, KVH, bs, D]."""
    return dataclasses.replace(to_bnnbsd(prefill_prefix()), name="prefill_prefix_bnnbsd")


def mtp_decode() -> Problem:
    """Multi-token (speculative) decode: 4 new tokens per sequence, causal
    among themselves, on the decode_large_batch sequences (B=64, kvSeqLen ~
    U[1024, 8192] including the 4 new tokens, H=32, KVH=8 so 16 rows per KV
    head, D=128, bs=128, bf16)."""
    rng = np.random.Generator(np.random.PCG64(3))
    kv = rng.integers(1024, 8193, 64).astype(np.int32)
    return make_problem(name="mtp_decode_causal", seed=6, seq_len=[4] * 64, kv_seq_len=kv,
                        head_num=32, kv_head_num=8, head_size=128, block_size=128,
                        dtype="bf16", mask_type=MASK_CAUSAL)


def int8_per_token_decode() -> Problem:
    """int8_long_decode with per-token dequantisation: K and V scale / offset
    of shape [B, S] fp32 (one pair per cached token, shared by the KV heads)."""
    return make_problem(name="int8_long_decode_per_token", seed=7, seq_len=[1] * 16,
                        kv_seq_len=[32768] * 16, head_num=64, kv_head_num=8, head_size=128,
                        block_size=128, dtype="bf16", kv_dtype="i8", mask_type=MASK_NONE,
                        sink=True, k_antiquant="token", v_antiquant="token")


def sliding_window_prefill() -> Problem:
    """Sliding-window prefill (band mask, preTokens=1023, nextTokens=0: each
    token sees itself and the 1023 before it): B=2, seqLen=kvSeqLen=4096,
    H=32, KVH=8, D=128, bs=128, bf16."""
    return make_problem(name="sliding_window_prefill", seed=8, seq_len=[4096, 4096],
                        kv_seq_len=[4096, 4096], head_num=32, kv_head_num=8, head_size=128,
                        block_size=128, dtype="bf16", mask_type=MASK_NONE, band=(1023, 0))


def causal_mha_prefill() -> Problem:
    """alibi_prefill's shapes with the plain causal mask and no bias (B=2,
    seqLen=kvSeqLen=2048, H=KVH=32, D=128, bs=128, fp16): the cost of the
    ALiBi bias is measured against it."""
    return make_problem(name="causal_mha_prefill", seed=4, seq_len=[2048, 2048],
                        kv_seq_len=[2048, 2048], head_num=32, kv_head_num=32, head_size=128,
                        block_size=128, dtype="f16", mask_type=MASK_CAUSAL)


def int8_prefix_prefill() -> Problem:
    """prefill_prefix (B=4, new=[128,256,512,1024] on prefixes
    [0,512,1024,3072], H=32, KVH=8, D=128, bs=128, causal, bf16 query) over an
    int8 cache with per-channel fp32 scale ~U(0.005,0.02) and offset
    ~N(0,0.1), per-head learnable sink ~N(0,1)."""
    new = [128, 256, 512, 1024]
    prefix = [0, 512, 1024, 3072]
    return make_problem(name="int8_prefix_prefill", seed=9, seq_len=new,
                        kv_seq_len=[a + b for a, b in zip(new, prefix)],
                        head_num=32, kv_head_num=8, head_size=128, block_size=128,
                        dtype="bf16", kv_dtype="i8", mask_type=MASK_CAUSAL, sink=True)


def int8_mtp_decode() -> Problem:
    """Multi-token decode over the long int8 cache: 3 new tokens per sequence
    (causal among themselves) on int8_long_decode's shapes (B=16,
    kvSeqLen=32768, H=64, KVH=8, so 24 rows per KV head, D=128, bs=128, bf16
    query, per-channel scale / offset, sink)."""
    return make_problem(name="int8_mtp_decode", seed=10, seq_len=[3] * 16,
                        kv_seq_len=[32768] * 16, head_num=64, kv_head_num=8, head_size=128,
                        block_size=128, dtype="bf16", kv_dtype="i8", mask_type=MASK_CAUSAL,
                        sink=True)


NAMED = {
    "tiny_decode": tiny_decode,
    "prefill_prefix": prefill_prefix,
    "decode_large_batch": decode_large_batch,
    "alibi_prefill": lambda: alibi_prefill(False),
    "alibi_prefill_pse": lambda: alibi_prefill(True),
    "int8_long_decode": int8_long_decode,
    "decode_large_batch_bnnbsd": decode_large_batch_bnnbsd,
    "prefill_prefix_bnnbsd": prefill_prefix_bnnbsd,
    "mtp_decode": mtp_decode,
    "int8_per_token_decode": int8_per_token_decode,
    "sliding_window_prefill": sliding_window_prefill,
    "causal_mha_prefill": causal_mha_prefill,
    "int8_prefix_prefill": int8_prefix_prefill,
    "int8_mtp_decode": int8_mtp_decode,
}


def permute_blocks(p: Problem, seed: int) -> Problem:
    """Same logical problem with the physical blocks of the pool shuffled and
    the block table rewritten to match (paging is logical contiguity)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    nb = p.key_cache.shape[0]
    perm = torch.from_numpy(rng.permutation(nb).astype(np.int64))     # new -> old
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(nb)
    bt = p.block_tables.clone()
    valid = bt >= 0
    bt[valid] = inv[bt[valid].long()].to(torch.int32)
    return dataclasses.replace(p, key_cache=p.key_cache[perm].contiguous(),
                               value_cache=p.value_cache[perm].contiguous(), block_tables=bt)


def unused_entries(p: Problem) -> List[tuple]:
    """Block-table positions that are never read (past ceil(kvSeqLen/bs))."""
    bs = p.block_size
    out = []
    for b in range(p.batch):
        need = (int(p.kv_seq_len[b]) + bs - 1) // bs
        out += [(b, j) for j in range(need, p.block_tables.shape[1])]
    return out
