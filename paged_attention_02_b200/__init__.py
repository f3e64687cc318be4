"""B200-native paged fused inference attention.

    out = Softmax(qkScale * Q K^T + bias) V

over a paged K/V cache, for prefill / prefix-encoder and decode, on sm_100a
kernels behind the C ABI of ``include/fia.h`` (libfia.so).  This module is the
thin Python face of that ABI: it turns torch CUDA tensors into ``fia_tensor``
descriptors, allocates the workspace phase 1 asks for, and calls the two
phases.  All arithmetic runs in the CUDA kernels; nothing here computes
attention, and a missing libfia.so raises at import.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import (FIA_KV_BNBSH, FIA_KV_BNNBSD, FIA_MASK_ALIBI, FIA_MASK_CAUSAL, FIA_MASK_NONE,
                   FIA_PATH_AUTO, FIA_PATH_DECODE, FIA_PATH_TENSOR, FiaError, fia_ext,
                   fia_plan_info, fia_tensor)

__all__ = ["FiaOp", "fused_infer_attention", "FIA_MASK_NONE", "FIA_MASK_ALIBI",
           "FIA_MASK_CAUSAL", "FIA_KV_BNBSH", "FIA_KV_BNNBSD", "FIA_PATH_AUTO",
           "FIA_PATH_DECODE", "FIA_PATH_TENSOR", "FiaError", "tensor_desc",
           "validate_block_tables"]

_DT = {torch.float16: _lib.FIA_F16, torch.bfloat16: _lib.FIA_BF16, torch.float32: _lib.FIA_F32,
       torch.int8: _lib.FIA_I8, torch.int32: _lib.FIA_I32}


def tensor_desc(t: Optional[torch.Tensor]) -> Optional[fia_tensor]:
    """fia_tensor describing a contiguous torch tensor (None -> None)."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("fia tensors must be contiguous")
    if t.dim() > 4:
        raise ValueError("fia tensors have at most 4 dims")
    d = fia_tensor()
    d.data = ctypes.c_void_p(t.data_ptr()) if t.numel() > 0 else ctypes.c_void_p(t.data_ptr() or None)
    d.dtype = _DT[t.dtype]
    d.ndim = t.dim()
    for i, n in enumerate(t.shape):
        d.dims[i] = int(n)
    return d


def _ptr(d: Optional[fia_tensor]):
    return ctypes.pointer(d) if d is not None else None


def validate_block_tables(block_tables, kv_seq_len: Sequence[int], block_size: int,
                          num_blocks: int) -> None:
    """Debug check of a block table, on the host (the kernels, like the
    operator they implement, do not validate block ids).  Every entry a
    sequence reads -- entries j < ceil(kvSeqLen / blockSize) of its row --
    must name a block in [0, numBlocks); entries past that are never read and
    may hold anything.  Copies the table to the host; raises ValueError naming
    the first bad entry."""
    bt = block_tables.detach().to("cpu")
    if bt.dim() != 2 or bt.shape[0] < len(kv_seq_len):
        raise ValueError("block table must be [batch, maxBlockNum]")
    for b, kl in enumerate(kv_seq_len):
        need = (int(kl) + block_size - 1) // block_size
        if need > bt.shape[1]:
            raise ValueError("sequence %d needs %d blocks, the table row has %d"
                             % (b, need, bt.shape[1]))
        row = bt[b, :need]
        bad = ((row < 0) | (row >= num_blocks)).nonzero()
        if bad.numel():
            j = int(bad[0, 0])
            raise ValueError("block_tables[%d][%d] = %d is outside [0, %d)"
                             % (b, j, int(row[j]), num_blocks))


class FiaOp:
    """One planned call (phase 1 done); ``run()`` enqueues phase 2.

    Arguments follow ``fia_get_workspace_size``: query ``[nTokens, H, D]``,
    ``band=(preTokens, nextTokens)``: band mask (sliding window with
    nextTokens = 0) instead of mask_type, which must then be FIA_MASK_NONE.
    int8 caches take k_scale/k_offset/v_scale/v_offset per (KV head, channel)
    ``[kvHeadNum, D]``, or per (sequence, token) ``[batch, S]`` with
    ``k_antiquant_mode`` / ``v_antiquant_mode`` = 1.
    key/value caches ``[numBlocks, blockSize, kvHeadNum, D]`` (``kv_layout=
    FIA_KV_BNNBSD``: ``[numBlocks, kvHeadNum, blockSize, D]``), block table
    ``[batch, maxBlockNum]`` int32 (all on the same CUDA device), host
    sequence lengths.  ``out`` / ``lse`` are allocated when not given
    (``want_lse=False`` skips lse).  Tensors are referenced, not copied: keep
    them unchanged while runs are in flight.  ``check_block_tables=True``
    runs ``validate_block_tables`` on the table first (a host copy: debugging only).
    ``path``: 0 automatic, ``FIA_PATH_DECODE`` (1) or ``FIA_PATH_TENSOR`` (2)
    forces the split-KV decode kernels or the tensor-core kernel.
    """

    def __init__(self, query, key, value, block_tables, seq_len: Sequence[int],
                 kv_seq_len: Sequence[int], head_num: int, kv_head_num: int, qk_scale: float,
                 mask_type: int = FIA_MASK_NONE, slopes=None, pse=None, sink=None, k_scale=None,
                 k_offset=None, v_scale=None, v_offset=None, out=None, lse=None,
                 want_lse: bool = True, kv_layout: int = FIA_KV_BNBSH,
                 k_antiquant_mode: int = 0, v_antiquant_mode: int = 0,
                 band: Optional[Tuple[int, int]] = None, check_block_tables: bool = False,
                 path: int = 0):
        dev = query.device
        if check_block_tables:
            bnnbsd = int(kv_layout) == FIA_KV_BNNBSD
            validate_block_tables(block_tables, kv_seq_len,
                                  int(key.shape[2] if bnnbsd else key.shape[1]), int(key.shape[0]))
        self.out = out if out is not None else torch.empty_like(query)
        if lse is None and want_lse:
            lse = torch.empty((query.shape[0], head_num), dtype=torch.float32, device=dev)
        self.lse = lse
        self._keep = [query, key, value, block_tables, slopes, pse, sink, k_scale, k_offset,
                      v_scale, v_offset, self.out, self.lse]
        self._d = {n: tensor_desc(t) for n, t in
                   dict(q=query, k=key, v=value, bt=block_tables, slopes=slopes, pse=pse,
                        sink=sink, ks=k_scale, ko=k_offset, vs=v_scale, vo=v_offset,
                        out=self.out, lse=self.lse).items()}
        self._ext = fia_ext(_ptr(self._d["pse"]), _ptr(self._d["sink"]), _ptr(self._d["ks"]),
                            _ptr(self._d["ko"]), _ptr(self._d["vs"]), _ptr(self._d["vo"]),
                            _ptr(self._d["lse"]), int(kv_layout), int(k_antiquant_mode),
                            int(v_antiquant_mode), _lib.FIA_SPARSE_BAND if band else 0,
                            int(band[0]) if band else 0, int(band[1]) if band else 0, int(path))
        b = len(seq_len)
        self._sl = (ctypes.c_int32 * max(b, 1))(*[int(x) for x in seq_len])
        self._kl = (ctypes.c_int32 * max(b, 1))(*[int(x) for x in kv_seq_len])
        self._op = ctypes.c_void_p()
        ws = ctypes.c_uint64(0)
        with torch.cuda.device(dev):
            st = _lib.fia_get_workspace_size(
                _ptr(self._d["q"]), _ptr(self._d["k"]), _ptr(self._d["v"]), _ptr(self._d["bt"]),
                self._sl, self._kl, b, _ptr(self._d["slopes"]), int(mask_type), int(head_num),
                int(kv_head_num), float(qk_scale), ctypes.pointer(self._ext), _ptr(self._d["out"]),
                ctypes.byref(ws), ctypes.byref(self._op))
        if st != _lib.FIA_OK:
            raise FiaError(st, "fia_get_workspace_size")
        self.workspace_size = int(ws.value)
        # 256-byte aligned device workspace (torch's allocator aligns to 512 B)
        self.workspace = torch.empty(max(self.workspace_size, 1), dtype=torch.uint8, device=dev)
        self._timing = None

    def run(self, stream: Optional[torch.cuda.Stream] = None):
        s = stream if stream is not None else torch.cuda.current_stream(self.out.device)
        st = _lib.fia_run(ctypes.c_void_p(self.workspace.data_ptr()), self.workspace_size,
                          self._op, ctypes.c_void_p(s.cuda_stream))
        if st != _lib.FIA_OK:
            raise FiaError(st, "fia_run")
        return self.out, self.lse

    def plan_info(self) -> dict:
        info = fia_plan_info()
        st = _lib.fia_op_get_plan_info(self._op, ctypes.byref(info))
        if st != _lib.FIA_OK:
            raise FiaError(st, "fia_op_get_plan_info")
        return {f: getattr(info, f) for f, _ in fia_plan_info._fields_}

    def error_word(self) -> int:
        """Value of the kernels' error word after the last run (syncs the device)."""
        off = self.plan_info()["error_word_offset"]
        if self.workspace_size == 0:
            return 0
        return int(self.workspace[off:off + 4].view(torch.int32).item())

    def error_trail(self) -> list:
        """Records the kernels left when a bounded wait ran out (syncs the device):
        dicts with the wait site, block, thread, three site values and the
        barrier's raw state."""
        if self.workspace_size == 0:
            return []
        off = self.plan_info()["error_word_offset"]
        words = self.workspace[off:off + (4 + 8 * 31) * 4].view(torch.int32).cpu().tolist()
        n = min(words[1] & 0xffffffff, 31)
        out = []
        for k in range(n):
            r = [w & 0xffffffff for w in words[4 + 8 * k: 12 + 8 * k]]
            out.append(dict(where=r[0], block=r[1], thread=r[2], x0=r[3], x1=r[4], x2=r[5],
                            bar=(r[7] << 32) | r[6]))
        return out

    def set_wait_limit(self, wait_limit_ns: int = 0, stall: bool = False):
        """Bound every internal wait of this op's kernels by ``wait_limit_ns``
        (0: the 2 s default).  ``stall=True`` is a test hook that makes the
        kernels time out on purpose (see fia_op_set_wait_limit in fia.h)."""
        st = _lib.fia_op_set_wait_limit(self._op, int(wait_limit_ns), 1 if stall else 0)
        if st != _lib.FIA_OK:
            raise FiaError(st, "fia_op_set_wait_limit")

    def set_timing_events(self, start: Optional[torch.cuda.Event], stop: Optional[torch.cuda.Event]):
        """Have run() record ``start``/``stop`` around its kernels only."""
        if start is None:
            st = _lib.fia_op_set_timing_events(self._op, None, None)
        else:
            s = torch.cuda.current_stream(self.out.device)
            start.record(s)    # make sure the events exist before taking their handles
            stop.record(s)
            st = _lib.fia_op_set_timing_events(self._op, ctypes.c_void_p(start.cuda_event),
                                               ctypes.c_void_p(stop.cuda_event))
        if st != _lib.FIA_OK:
            raise FiaError(st, "fia_op_set_timing_events")
        self._timing = (start, stop)

    def close(self):
        if getattr(self, "_op", None) is not None and self._op.value:
            _lib.fia_op_destroy(self._op)
            self._op = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fused_infer_attention(query, key, value, block_tables, seq_len, kv_seq_len, head_num,
                          kv_head_num, qk_scale, mask_type=FIA_MASK_NONE, slopes=None, pse=None,
                          sink=None, k_scale=None, k_offset=None, v_scale=None, v_offset=None,
                          want_lse=True, kv_layout=FIA_KV_BNBSH, k_antiquant_mode=0,
                          v_antiquant_mode=0, band=None, check_block_tables=False):
    """One-shot call: plan, run on the current stream, return (out, lse)."""
    op = FiaOp(query, key, value, block_tables, seq_len, kv_seq_len, head_num, kv_head_num,
               qk_scale, mask_type, slopes, pse, sink, k_scale, k_offset, v_scale, v_offset,
               want_lse=want_lse, kv_layout=kv_layout, k_antiquant_mode=k_antiquant_mode,
               v_antiquant_mode=v_antiquant_mode, band=band,
               check_block_tables=check_block_tables)
    out, lse = op.run()
    op._keep.append(op.workspace)
    return out, lse
