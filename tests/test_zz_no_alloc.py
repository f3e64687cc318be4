"""fia_decode_run_static: decode with the library's own fixed scratch array.

This entry point is for callers that cannot allocate device memory when they
run attention (an engine whose device memory all belongs to its own pool, or a
serving loop where cudaMalloc is forbidden): it takes no workspace and
allocates nothing.  These tests call it through the C ABI and check that it
reproduces fia_run (the workspace entry point) on the same op -- the same plan
and the same kernels, so bit for bit -- on calls in a row, with an op of
another shape and cache dtype run through the shared array in between (each
call must fully replace what the previous one left there), and that the
kernels' error word, which on this path lives in the array, reads zero.  This
file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from fia_testlib import run_gpu

pytestmark = pytest.mark.gpu


def _stream_ptr():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _static_run(op):
    from paged_attention_02_b200 import _lib
    op.out.fill_(float("nan"))
    op.lse.fill_(float("nan"))
    st = _lib.fia_decode_run_static(op._op, _stream_ptr())
    assert st == _lib.FIA_OK, _lib.fia_status_string(st)
    torch.cuda.synchronize()
    word = ctypes.c_uint32(123)
    assert _lib.fia_decode_static_error_word(op._op, ctypes.byref(word)) == _lib.FIA_OK
    assert word.value == 0, hex(word.value)
    return op.out.float().double().cpu().numpy(), op.lse.double().cpu().numpy()


def test_static_scratch_decode_matches_workspace_run():
    from paged_attention_02_b200 import _lib
    # two decode ops of different shapes and cache dtypes: the larger bf16 op
    # first, then the smaller int8 op (fewer splits, different plan layout)
    a = W.make_problem(name="static_decode_bf16", seed=77, seq_len=[1, 1, 2, 1],
                       kv_seq_len=[900, 33, 2500, 4100], head_num=16, kv_head_num=2,
                       head_size=128, block_size=64, sink=True, mask_type=W.MASK_CAUSAL)
    b = W.make_problem(name="static_decode_i8", seed=79, seq_len=[1, 3],
                       kv_seq_len=[300, 1200], head_num=8, kv_head_num=2, head_size=128,
                       block_size=128, kv_dtype="i8", mask_type=W.MASK_CAUSAL)
    ops = []
    for p in (a, b):
        op, ref_out, ref_lse = run_gpu(p)                # existing entry point: fia_run
        assert op.plan_info()["path"] == 1
        assert op.workspace_size <= _lib.FIA_STATIC_WORKSPACE_BYTES
        ops.append((op, ref_out, ref_lse))
    assert ops[0][0].plan_info()["work_items"] != ops[1][0].plan_info()["work_items"]
    for call in range(2):
        for op, ref_out, ref_lse in ops:
            out, lse = _static_run(op)
            assert np.array_equal(out, ref_out), "call %d: output differs from fia_run" % call
            assert np.array_equal(lse, ref_lse), "call %d: lse differs from fia_run" % call


def test_static_scratch_rejects_prefill_and_oversized_ops():
    from paged_attention_02_b200 import _lib
    # prefill-path op: not a decode op
    p = W.make_problem(seed=78, seq_len=[130], kv_seq_len=[200], head_num=4, kv_head_num=4,
                       head_size=128, block_size=64, mask_type=W.MASK_CAUSAL)
    op, _, _ = run_gpu(p)
    assert op.plan_info()["path"] == 2
    assert _lib.fia_decode_run_static(op._op, _stream_ptr()) == _lib.FIA_ERR_UNSUPPORTED
    word = ctypes.c_uint32(0)
    assert _lib.fia_decode_static_error_word(op._op, ctypes.byref(word)) == _lib.FIA_ERR_UNSUPPORTED
    # a decode op whose scratch would exceed the fixed array: 600 sequences x
    # 4096 keys x 8 KV heads; the table may name the same blocks repeatedly
    # (ids are not validated), so the cache itself stays small.  Nothing is
    # launched: the size check comes first.
    import paged_attention_02_b200 as fia
    B, KVH, D, bs = 600, 8, 128, 128
    dev = torch.device("cuda")
    q = torch.zeros(B, 64, D, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(32, bs, KVH, D, dtype=torch.bfloat16, device=dev)
    bt = (torch.arange(B * 32, dtype=torch.int32, device=dev) % 32).reshape(B, 32)
    big = fia.FiaOp(q, kc, kc.clone(), bt, [1] * B, [4096] * B, 64, KVH, 0.1)
    assert big.plan_info()["path"] == 1
    assert big.workspace_size > _lib.FIA_STATIC_WORKSPACE_BYTES
    assert _lib.fia_decode_run_static(big._op, _stream_ptr()) == _lib.FIA_ERR_WORKSPACE
    assert _lib.fia_decode_run_static(None, _stream_ptr()) == _lib.FIA_ERR_NULLPTR
    assert _lib.fia_decode_static_error_word(None, ctypes.byref(word)) == _lib.FIA_ERR_NULLPTR
