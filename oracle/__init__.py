"""CPU oracle for paged fused inference attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never touches the CUDA library and
the CUDA library never touches it.

The arithmetic lives in ``fia_oracle.c`` (plain C, double precision, naive
block-table resolve, full softmax rows), written from the
aclnnFusedInferAttentionScoreV4/V3 "Formula" sections, the V3 ``lse``
restriction bullet and the ATB PrefixEncoder parameter table.  This module
only compiles it with gcc and marshals numpy/torch buffers into it.

Pins (tests/test_oracle_pins.py) tie it to things other than itself:
torch's scaled_dot_product_attention on contiguous inputs, hand-worked golden
rows (tests/golden/), rows summing to one, block-permutation invariance,
single-key and dominant-key outputs, GQA == MHA with repeated KV heads,
qkScale = 0 closed form, lse == log-sum-exp by math.fsum, the int8 dequant
special cases and the sink limits.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fia_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libfia_oracle.so")
_lock = threading.Lock()
_lib = None

_DT = {torch.float16: 0, torch.bfloat16: 1, torch.int8: 2}

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_D = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile fia_oracle.c into a shared library next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            common = [_P, _I, _P, _P, _I, _I64, _I, _P, _I, _P, _P, _I, _I, _I, _I, _D, _I, _P,
                      _P, _I, _I, _I, _P, _P, _P, _P, _P]
            lib.fia_oracle_attention.argtypes = common + [_P, _I64, _I, _P, _P, _I, _I, _I, _I64, _I64,
                                                          _I, _I64, _I64]
            lib.fia_oracle_attention.restype = _I
            lib.fia_oracle_row_probs.argtypes = common + [_I, _I, _I, _P, _P, _P, _I, _I, _I, _I64, _I64,
                                                          _I, _I64, _I64]
            lib.fia_oracle_row_probs.restype = _I
            lib.fia_oracle_max_threads.restype = _I
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().fia_oracle_max_threads())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous()
    return ctypes.c_void_p(t.data_ptr())


def _layout(p) -> int:
    """KV cache layout of problem p: 0 BnBsH (default), 1 BnNBsD."""
    return int(getattr(p, "kv_layout", 0))


def _quant_modes(p):
    """(k_mode, v_mode, k_row_stride, v_row_stride): per-channel (0) or
    per-token (1) int8 dequantisation; per-token tensors are [B, S]."""
    km, vm = int(getattr(p, "k_antiquant_mode", 0)), int(getattr(p, "v_antiquant_mode", 0))
    ks = p.k_scale.shape[-1] if (km == 1 and p.k_scale is not None) else 0
    vs = p.v_scale.shape[-1] if (vm == 1 and p.v_scale is not None) else 0
    return [km, vm, int(ks), int(vs)]


def _band(p):
    """(band, preTokens, nextTokens) of problem p (band mask, V3 sparseMode 4)."""
    if getattr(p, "band", None) is None:
        return [0, 0, 0]
    pre, nxt = p.band
    return [1, int(pre), int(nxt)]


def _common(p, keep):
    """Positional argument prefix shared by both entry points."""
    q = p.query.contiguous()
    kc = p.key_cache.contiguous()
    vc = p.value_cache.contiguous()
    bt = p.block_tables.to(torch.int32).contiguous()
    sl = torch.from_numpy(np.ascontiguousarray(p.seq_len, dtype=np.int32))
    kl = torch.from_numpy(np.ascontiguousarray(p.kv_seq_len, dtype=np.int32))
    f32 = lambda t: None if t is None else t.to(torch.float32).contiguous()
    slopes, sink = f32(p.slopes), f32(p.sink)
    ks, ko, vs, vo = f32(p.k_scale), f32(p.k_offset), f32(p.v_scale), f32(p.v_offset)
    pse = None if p.pse is None else p.pse.contiguous()
    keep += [q, kc, vc, bt, sl, kl, slopes, sink, ks, ko, vs, vo, pse]
    pse_dt = _DT[pse.dtype] if pse is not None else 0
    pse_q = pse.shape[2] if pse is not None else 0
    pse_kv = pse.shape[3] if pse is not None else 0
    # block size: [numBlocks, blockSize, KVH, D] (BnBsH) or [numBlocks, KVH, blockSize, D]
    bs = kc.shape[2] if _layout(p) == 1 else kc.shape[1]
    return [_ptr(q), _DT[q.dtype], _ptr(kc), _ptr(vc), _DT[kc.dtype], kc.shape[0], bs,
            _ptr(bt), bt.shape[1], _ptr(sl), _ptr(kl), sl.shape[0],
            p.head_num, p.kv_head_num, q.shape[2], float(p.qk_scale), int(p.mask_type),
            _ptr(slopes), _ptr(pse), pse_dt, pse_q, pse_kv, _ptr(sink),
            _ptr(ks), _ptr(ko), _ptr(vs), _ptr(vo)]


def attention(p, rows: Optional[Sequence[Tuple[int, int]]] = None,
              threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Reference output (float64, unrounded) and lse (float64) for problem ``p``.

    ``rows=None``: out ``[nTokens, H, D]``, lse ``[nTokens, H]``.
    ``rows=[(token, head), ...]``: out ``[len(rows), D]``, lse ``[len(rows)]``.
    """
    lib = _load()
    keep = []
    args = _common(p, keep)
    D = p.query.shape[2]
    if rows is None:
        out = np.zeros((p.query.shape[0], p.head_num, D), dtype=np.float64)
        lse = np.zeros((p.query.shape[0], p.head_num), dtype=np.float64)
        rows_arr, n_rows = None, 0
    else:
        rows_np = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
        n_rows = rows_np.shape[0]
        out = np.zeros((n_rows, D), dtype=np.float64)
        lse = np.zeros((n_rows,), dtype=np.float64)
        rows_arr = rows_np
    rc = lib.fia_oracle_attention(*args,
                                  rows_arr.ctypes.data_as(_P) if rows_arr is not None else None,
                                  n_rows, int(threads),
                                  out.ctypes.data_as(_P), lse.ctypes.data_as(_P), _layout(p),
                                  *_quant_modes(p), *_band(p))
    if rc != 0:
        raise ValueError("oracle rejected the problem (code %d)" % rc)
    return out, lse


def row_probs(p, b: int, i: int, h: int) -> Tuple[np.ndarray, np.ndarray, float]:
    """Softmax weights over logical positions t < kvSeqLen[b] for one row,
    plus that row's output and lse."""
    lib = _load()
    keep = []
    args = _common(p, keep)
    kvlen = int(p.kv_seq_len[b])
    probs = np.zeros((max(kvlen, 1),), dtype=np.float64)
    out = np.zeros((p.query.shape[2],), dtype=np.float64)
    lse = np.zeros((1,), dtype=np.float64)
    rc = lib.fia_oracle_row_probs(*args, b, i, h, probs.ctypes.data_as(_P),
                                  out.ctypes.data_as(_P), lse.ctypes.data_as(_P), _layout(p),
                                  *_quant_modes(p), *_band(p))
    if rc != 0:
        raise ValueError("oracle rejected the row (code %d)" % rc)
    return probs[:kvlen], out, float(lse[0])
