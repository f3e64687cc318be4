"""Failure detection on the GPU, without a GPU fault.

Every wait of the kernels on an on-chip barrier is bounded; a wait that runs
out sets the error word (wait site << 8 | 1), leaves trail records, lets every
role of the CTA leave, waits for the CTA's copies and MMAs still in flight,
releases TMEM and returns.  The test hook of fia_op_set_wait_limit makes one
role wait on a barrier that nothing signals, with a 1 ms limit, so the exit
runs for real; the host then reads the error report, and the same op, with the
default limit restored, must give the oracle's result (the context is intact).
(V3 long-sequence restriction: an over-long run ends in a device time-out
error; here the time-out is the kernels' own and reports through a status.)
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from fia_testlib import compare, run_gpu

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000          # 1 ms
SITE_DECODE_STALL = 3         # decode kernels: the hook's wait
SITE_PREFILL_STALL = 35       # prefill softmax warps: the hook's wait
# Prefill wait sites: producer 10-12, issuer 20-27, softmax warps 30-35, int8
# converters 40-44.  With the softmax warps stalled, the issuer's wait for
# their P (or a wait further up the pipeline) can run out first; each is a
# time-out of a wait that nothing completed.
PREFILL_SITES = (set(range(10, 13)) | set(range(20, 28)) | set(range(30, 36)) |
                 set(range(40, 45)))

CASES = {
    "decode_bf16": (dict(seq_len=[1, 1, 1], kv_seq_len=[900, 70, 3000], head_num=16,
                         kv_head_num=2, head_size=128, block_size=64, sink=True),
                    1, SITE_DECODE_STALL),
    "decode_int8_per_token": (dict(seq_len=[1, 2], kv_seq_len=[1500, 333], head_num=16,
                                   kv_head_num=2, head_size=128, block_size=64, kv_dtype="i8",
                                   k_antiquant="token", v_antiquant="token",
                                   mask_type=W.MASK_CAUSAL),
                              1, SITE_DECODE_STALL),
    "prefill_causal_gqa": (dict(seq_len=[300, 130], kv_seq_len=[700, 130], head_num=8,
                                kv_head_num=2, head_size=128, block_size=64,
                                mask_type=W.MASK_CAUSAL),
                           2, SITE_PREFILL_STALL),
    "prefill_int8_per_token": (dict(seq_len=[300, 130], kv_seq_len=[700, 130], head_num=8,
                                    kv_head_num=2, head_size=128, block_size=64, kv_dtype="i8",
                                    k_antiquant="token", v_antiquant="channel",
                                    mask_type=W.MASK_CAUSAL),
                               2, SITE_PREFILL_STALL),
    "prefill_pse_mha_f16": (dict(seq_len=[200], kv_seq_len=[264], head_num=4, kv_head_num=4,
                                 head_size=128, block_size=32, dtype="f16",
                                 mask_type=W.MASK_CAUSAL, pse=True),
                            2, SITE_PREFILL_STALL),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_bounded_wait_times_out_and_reports(name):
    kw, path, site = CASES[name]
    p = W.make_problem(name=name, seed=500 + len(name), **kw)
    op, out_ok, lse_ok = run_gpu(p)
    assert op.plan_info()["path"] == path
    op.set_wait_limit(LIMIT_NS, stall=True)
    op.run()
    torch.cuda.synchronize()          # the run returns: no hang, no fault
    ew = op.error_word()
    sites = {site} if path == 1 else PREFILL_SITES
    assert ew & 0xff == 1 and (ew >> 8) in sites, hex(ew)
    trail = op.error_trail()
    assert trail and all(r["where"] in sites for r in trail), trail
    assert all(r["block"] < op.plan_info()["grid"] for r in trail)
    # default limit again: the same op, the same device, the oracle's result
    op.set_wait_limit(0, stall=False)
    out, lse = op.run()
    torch.cuda.synchronize()
    assert op.error_word() == 0
    o = out.float().double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.array_equal(o, out_ok) and np.array_equal(l, lse_ok)
    ref_o, ref_l = oracle.attention(p)
    compare(o, l, ref_o, ref_l, name)


def test_static_scratch_path_reports_time_out():
    """fia_decode_run_static: the error word lives in the library's array and
    is read with fia_decode_static_error_word."""
    from paged_attention_02_b200 import _lib
    p = W.make_problem(name="static_stall", seed=503, seq_len=[1, 1], kv_seq_len=[2000, 90],
                       head_num=16, kv_head_num=2, head_size=128, block_size=128)
    op, out_ok, _ = run_gpu(p)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    word = ctypes.c_uint32(0)
    op.set_wait_limit(LIMIT_NS, stall=True)
    assert _lib.fia_decode_run_static(op._op, stream) == _lib.FIA_OK
    torch.cuda.synchronize()
    assert _lib.fia_decode_static_error_word(op._op, ctypes.byref(word)) == _lib.FIA_OK
    assert word.value == (SITE_DECODE_STALL << 8) | 1, hex(word.value)
    op.set_wait_limit(0, stall=False)
    assert _lib.fia_decode_run_static(op._op, stream) == _lib.FIA_OK
    torch.cuda.synchronize()
    assert _lib.fia_decode_static_error_word(op._op, ctypes.byref(word)) == _lib.FIA_OK
    assert word.value == 0
    assert np.array_equal(op.out.float().double().cpu().numpy(), out_ok)


def test_wait_limit_argument_rules():
    from paged_attention_02_b200 import _lib
    p = W.make_problem(seed=504, seq_len=[1], kv_seq_len=[64], head_num=4, kv_head_num=4,
                       head_size=128, block_size=16)
    op, _, _ = run_gpu(p)
    assert _lib.fia_op_set_wait_limit(None, 0, 0) == _lib.FIA_ERR_NULLPTR
    assert _lib.fia_op_set_wait_limit(op._op, 0, 2) == _lib.FIA_ERR_PARAM
    assert _lib.fia_op_set_wait_limit(op._op, 5_000_000_000, 0) == _lib.FIA_OK
