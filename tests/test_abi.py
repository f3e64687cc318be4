"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/fia.h declares, and phase 1 rejects bad inputs with
the documented status codes before touching any device (aclnn
GetWorkspaceSize "implements input parameter verification")."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            names += re.findall(r"FIA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_library_builds_and_exports_every_declared_symbol():
    import __graft_entry__
    build = __graft_entry__.load_builder()
    build.build()
    lib = ctypes.CDLL(build.LIB_PATH)
    names = _declared_functions()
    assert len(names) >= 6
    for n in names:
        assert hasattr(lib, n), "missing export %s" % n


def test_status_strings():
    import paged_attention_02_b200 as fia
    from paged_attention_02_b200 import _lib
    for s in range(8):
        assert fia._lib.fia_status_string(s)
    assert _lib.fia_status_string(99) == "unknown status"


def _call(**kw):
    """Phase 1 on CPU tensors (only shapes and dtypes are read)."""
    from paged_attention_02_b200 import _lib, tensor_desc
    from paged_attention_02_b200._lib import fia_ext
    B, H, KVH, D, bs = 2, 4, 2, 128, 16
    t = dict(q=torch.zeros(3, H, D, dtype=torch.bfloat16),
             k=torch.zeros(8, bs, KVH, D, dtype=torch.bfloat16),
             v=torch.zeros(8, bs, KVH, D, dtype=torch.bfloat16),
             bt=torch.zeros(B, 4, dtype=torch.int32),
             out=torch.zeros(3, H, D, dtype=torch.bfloat16),
             slopes=None, pse=None, sink=None, lse=None, ks=None, vs=None)
    args = dict(seq=[1, 2], kv=[20, 33], batch=B, mask=9, H=H, KVH=KVH, scale=0.1)
    for k, v in kw.items():
        if k in t:
            t[k] = v
        else:
            args[k] = v
    d = {k: tensor_desc(v) for k, v in t.items()}
    P = lambda x: ctypes.pointer(x) if x is not None else None
    ext = fia_ext(P(d["pse"]), P(d["sink"]), P(d["ks"]), None, P(d["vs"]), None, P(d["lse"]),
                  int(args.get("layout", 0)), int(args.get("kmode", 0)), int(args.get("vmode", 0)),
                  int(args.get("sparse", 0)), int(args.get("pre", 0)), int(args.get("next", 0)),
                  int(args.get("path", 0)))
    if args["seq"] is None:                       # NULL host length arrays
        sl = kl = None
    else:
        n = max(len(args["seq"]), 1)
        sl = (ctypes.c_int32 * n)(*args["seq"])
        kl = (ctypes.c_int32 * n)(*args["kv"])
    ws = ctypes.c_uint64(123)
    op = ctypes.c_void_p()
    st = _lib.fia_get_workspace_size(P(d["q"]), P(d["k"]), P(d["v"]), P(d["bt"]), sl, kl,
                                     args["batch"], P(d["slopes"]), args["mask"], args["H"],
                                     args["KVH"], args["scale"], ctypes.pointer(ext), P(d["out"]),
                                     ctypes.byref(ws), ctypes.byref(op))
    if op.value:
        _lib.fia_op_destroy(op)
    return st


def test_phase1_rejects_bad_inputs():
    from paged_attention_02_b200 import _lib as L
    assert _call(H=6, KVH=4) == L.FIA_ERR_PARAM                                   # H % KVH
    assert _call(mask=5) == L.FIA_ERR_PARAM                                       # mask code
    assert _call(seq=[2, 2]) == L.FIA_ERR_SHAPE                                   # sum != nTokens
    assert _call(seq=[1, 2], kv=[20, 1]) == L.FIA_ERR_PARAM                       # seqLen > kvSeqLen
    assert _call(kv=[20, 80]) == L.FIA_ERR_SHAPE                                  # table too short
    assert _call(k=torch.zeros(8, 16, 2, 128, dtype=torch.float16),
                 v=torch.zeros(8, 16, 2, 128, dtype=torch.float16)) == L.FIA_ERR_DTYPE
    assert _call(out=torch.zeros(3, 4, 128, dtype=torch.float16)) == L.FIA_ERR_DTYPE
    assert _call(bt=torch.zeros(2, 4, dtype=torch.float32)) == L.FIA_ERR_DTYPE
    assert _call(v=torch.zeros(9, 16, 2, 128, dtype=torch.bfloat16)) == L.FIA_ERR_SHAPE
    assert _call(mask=3) == L.FIA_ERR_NULLPTR                                     # ALiBi w/o slopes
    assert _call(mask=9, slopes=torch.zeros(4)) == L.FIA_ERR_PARAM                # slopes w/o ALiBi
    assert _call(sink=torch.zeros(3)) == L.FIA_ERR_SHAPE
    assert _call(lse=torch.zeros(3, 4, dtype=torch.float16)) == L.FIA_ERR_DTYPE
    assert _call(pse=torch.zeros(2, 4, 2, 16, dtype=torch.bfloat16)) == L.FIA_ERR_SHAPE
    assert _call(scale=float("nan")) == L.FIA_ERR_PARAM
    assert _call(batch=-1) == L.FIA_ERR_PARAM


def test_phase1_rejects_more_bad_inputs():
    """The remaining phase-1 rejection rules (each case breaks exactly one)."""
    from paged_attention_02_b200 import _lib as L
    bf = lambda *sh: torch.zeros(*sh, dtype=torch.bfloat16)
    ok = (L.FIA_ERR_CUDA, L.FIA_OK)               # valid: no GPU here, phase 1 stops at encoding
    # null pointers
    assert L.fia_get_workspace_size(None, None, None, None, None, None, 0, None, 0, 0, 0, 0.0,
                                    None, None, None, None) == L.FIA_ERR_NULLPTR
    assert _call(q=None) == L.FIA_ERR_NULLPTR
    assert _call(bt=None) == L.FIA_ERR_NULLPTR
    assert _call(out=None) == L.FIA_ERR_NULLPTR
    assert _call(seq=None) == L.FIA_ERR_NULLPTR                                   # batch 2, no lengths
    # head counts
    assert _call(H=0) == L.FIA_ERR_PARAM
    assert _call(KVH=0) == L.FIA_ERR_PARAM
    assert _call(H=2048, KVH=2, q=bf(3, 2048, 128), out=bf(3, 2048, 128)) == L.FIA_ERR_PARAM
    # query / output shapes; the 2-D query form [nTokens, H * D] is accepted
    assert _call(q=bf(3, 4, 128, 1), out=bf(3, 4, 128, 1)) == L.FIA_ERR_SHAPE
    assert _call(q=bf(3, 5, 128), out=bf(3, 5, 128)) == L.FIA_ERR_SHAPE
    assert _call(q=bf(3, 512), out=bf(3, 512)) in ok
    assert _call(q=bf(3, 510), out=bf(3, 510)) == L.FIA_ERR_SHAPE
    assert _call(out=bf(3, 4, 64)) == L.FIA_ERR_SHAPE
    # cache shapes: the 3-D BnBsH form [numBlocks, blockSize, kvHeadNum * D] is accepted
    assert _call(k=bf(8, 16, 256), v=bf(8, 16, 256)) in ok
    assert _call(k=bf(8, 16, 250), v=bf(8, 16, 250)) == L.FIA_ERR_SHAPE
    assert _call(k=bf(8, 4096), v=bf(8, 4096)) == L.FIA_ERR_SHAPE                  # 2-D cache
    assert _call(v=bf(8, 16, 256)) == L.FIA_ERR_SHAPE                             # k 4-D, v 3-D
    # block table
    assert _call(bt=torch.zeros(8, dtype=torch.int32)) == L.FIA_ERR_SHAPE
    assert _call(bt=torch.zeros(3, 4, dtype=torch.int32)) == L.FIA_ERR_SHAPE     # 3 rows, batch 2
    # lengths
    assert _call(seq=[-1, 4]) == L.FIA_ERR_PARAM
    assert _call(kv=[-1, 33]) == L.FIA_ERR_PARAM
    # pse
    assert _call(pse=torch.zeros(2, 4, 2, 40, dtype=torch.float16)) == L.FIA_ERR_DTYPE
    assert _call(pse=bf(2, 4, 2, 40)) in ok
    assert _call(pse=bf(2, 4, 1, 40)) == L.FIA_ERR_SHAPE                          # maxQ is 2
    assert _call(mask=3, slopes=torch.zeros(4), pse=bf(2, 4, 2, 40)) == L.FIA_ERR_PARAM
    # sink / lse / slopes dtypes and shapes
    assert _call(sink=torch.zeros(4, dtype=torch.float16)) == L.FIA_ERR_DTYPE
    assert _call(sink=torch.zeros(4)) in ok
    assert _call(mask=3, slopes=torch.zeros(3)) == L.FIA_ERR_SHAPE
    assert _call(lse=torch.zeros(3, 5)) == L.FIA_ERR_SHAPE
    assert _call(lse=torch.zeros(3, 4)) in ok


def test_phase1_int8_rules():
    from paged_attention_02_b200 import _lib as L
    k8 = torch.zeros(8, 16, 2, 128, dtype=torch.int8)
    assert _call(k=k8, v=k8) == L.FIA_ERR_NULLPTR                                 # scales missing
    ks = torch.ones(2, 128)
    # scales on a bf16 cache are a parameter error
    assert _call(ks=ks, vs=ks) == L.FIA_ERR_PARAM
    # more than 16 rows per KV head (9 new tokens x g=2) takes the tensor-core
    # path, which also reads an int8 cache
    ok = (L.FIA_ERR_CUDA, L.FIA_OK)               # valid: no GPU here, phase 1 stops at encoding
    q = torch.zeros(10, 4, 128, dtype=torch.bfloat16)
    assert _call(k=k8, v=k8, ks=ks, vs=ks, q=q, out=q.clone(), seq=[1, 9]) in ok
    # an int8 cache needs headSize 128 (one 128-byte row per key) on both paths
    k64 = torch.zeros(8, 16, 2, 64, dtype=torch.int8)
    ks64 = torch.ones(2, 64)
    for seq, n in (([1, 2], 3), ([1, 9], 10)):
        q = torch.zeros(n, 4, 64, dtype=torch.bfloat16)
        assert _call(k=k64, v=k64, ks=ks64, vs=ks64, q=q, out=q.clone(), seq=seq) == L.FIA_ERR_UNSUPPORTED


def test_phase1_path_choice():
    from paged_attention_02_b200 import _lib as L
    ok = (L.FIA_ERR_CUDA, L.FIA_OK)               # valid: no GPU here, phase 1 stops at encoding
    assert _call(path=3) == L.FIA_ERR_PARAM
    assert _call(path=-1) == L.FIA_ERR_PARAM
    for path in (0, 1, 2):
        assert _call(path=path) in ok
    # the decode kernels take at most 8 chunks of 16 rows per KV head: 65
    # new tokens x g = 2 is 130 rows
    q = torch.zeros(66, 4, 128, dtype=torch.bfloat16)
    k = torch.zeros(16, 16, 2, 128, dtype=torch.bfloat16)
    bt = torch.zeros(2, 8, dtype=torch.int32)
    assert _call(q=q, out=q.clone(), k=k, v=k.clone(), bt=bt, seq=[1, 65], kv=[20, 100],
                 path=1) == L.FIA_ERR_PARAM
    assert _call(q=q, out=q.clone(), k=k, v=k.clone(), bt=bt, seq=[1, 65], kv=[20, 100],
                 path=2) in ok


def test_phase1_build_limits():
    from paged_attention_02_b200 import _lib as L
    q = torch.zeros(3, 4, 96, dtype=torch.bfloat16)
    k = torch.zeros(8, 16, 2, 96, dtype=torch.bfloat16)
    assert _call(q=q, out=q.clone(), k=k, v=k.clone()) == L.FIA_ERR_UNSUPPORTED   # D=96
    k = torch.zeros(8, 24, 2, 128, dtype=torch.bfloat16)
    assert _call(k=k, v=k.clone(), bt=torch.zeros(2, 8, dtype=torch.int32)) == L.FIA_ERR_UNSUPPORTED


def test_phase1_without_gpu_reports_cuda_error():
    from paged_attention_02_b200 import _lib as L
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _call() == L.FIA_ERR_CUDA


def test_empty_query_is_a_noop_op():
    from paged_attention_02_b200 import _lib as L
    q = torch.zeros(0, 4, 128, dtype=torch.bfloat16)
    assert _call(q=q, out=q.clone(), seq=[0, 0], kv=[0, 0]) == L.FIA_OK


def test_run_rejects_null_op_and_missing_workspace():
    from paged_attention_02_b200 import _lib as L
    assert L.fia_run(None, 0, None, None) == L.FIA_ERR_NULLPTR
    assert L.fia_op_set_timing_events(None, None, None) == L.FIA_ERR_NULLPTR
    assert L.fia_op_get_plan_info(None, None) == L.FIA_ERR_NULLPTR


def test_phase1_kv_layout_rules():
    """BnNBsD cache [numBlocks, kvHeadNum, blockSize, headSize] (V3 paged
    attention constraints: BnBsH or BnNBsD): validated by phase 1."""
    from paged_attention_02_b200 import _lib as L
    bn = lambda: torch.zeros(8, 2, 16, 128, dtype=torch.bfloat16)
    assert _call(layout=2) == L.FIA_ERR_PARAM                                     # unknown layout
    assert _call(layout=1) == L.FIA_ERR_SHAPE                                     # BnBsH dims given
    assert _call(layout=1, k=torch.zeros(8, 16, 256, dtype=torch.bfloat16),
                 v=torch.zeros(8, 16, 256, dtype=torch.bfloat16)) == L.FIA_ERR_SHAPE  # 3-D
    assert _call(layout=1, k=bn(), v=torch.zeros(8, 2, 16, 64, dtype=torch.bfloat16)) == \
        L.FIA_ERR_SHAPE                                                            # k != v
    # valid BnNBsD inputs pass validation; without a GPU, phase 1 stops at the
    # tensor-map encoding
    assert _call(layout=1, k=bn(), v=bn()) in (L.FIA_ERR_CUDA, L.FIA_OK)
    # the table must cover kvSeqLen with the BnNBsD block size (dims[2] = 16)
    assert _call(layout=1, k=bn(), v=bn(), kv=[20, 80]) == L.FIA_ERR_SHAPE


def test_phase1_per_token_antiquant_rules():
    """Per-token int8 dequantisation (V3 fake-quantization: scale/offset
    (B, S) or (1, B, S), f32; K and V modes may differ)."""
    from paged_attention_02_b200 import _lib as L
    k8 = torch.zeros(8, 16, 2, 128, dtype=torch.int8)
    ch = torch.ones(2, 128)                       # per-channel [KVH, D]
    tok = torch.ones(2, 40)                       # per-token [B=2, S=40 >= max kvSeqLen 33]
    ok = (L.FIA_ERR_CUDA, L.FIA_OK)               # valid: no GPU here, phase 1 stops at encoding
    assert _call(k=k8, v=k8, ks=tok, vs=tok, kmode=1, vmode=1) in ok
    assert _call(k=k8, v=k8, ks=ch, vs=tok, kmode=0, vmode=1) in ok
    assert _call(k=k8, v=k8, ks=tok, vs=ch, kmode=1, vmode=0) in ok
    assert _call(k=k8, v=k8, ks=tok[None], vs=tok[None], kmode=1, vmode=1) in ok      # (1, B, S)
    assert _call(k=k8, v=k8, ks=tok, vs=tok, kmode=2) == L.FIA_ERR_PARAM              # unknown mode
    assert _call(k=k8, v=k8, ks=tok, vs=tok, kmode=0, vmode=1) == L.FIA_ERR_SHAPE     # K expects [KVH, D]
    assert _call(k=k8, v=k8, ks=torch.ones(3, 40), vs=tok, kmode=1, vmode=1) == L.FIA_ERR_SHAPE  # B
    assert _call(k=k8, v=k8, ks=torch.ones(2, 30), vs=tok, kmode=1, vmode=1) == L.FIA_ERR_SHAPE  # S < 33
    assert _call(k=k8, v=k8, ks=torch.ones(2, 40, dtype=torch.float16), vs=tok, kmode=1,
                 vmode=1) == L.FIA_ERR_DTYPE
    # a mode on a bf16 cache is a parameter error
    assert _call(kmode=1) == L.FIA_ERR_PARAM


def test_phase1_band_rules():
    """Band mask (V3 sparseMode 4): replaces maskType (which must be
    FIA_MASK_NONE) and needs preTokens + nextTokens >= 0."""
    from paged_attention_02_b200 import _lib as L
    ok = (L.FIA_ERR_CUDA, L.FIA_OK)
    assert _call(mask=0, sparse=4, pre=100, next=0) in ok
    assert _call(mask=0, sparse=4, pre=-5, next=5) in ok
    assert _call(mask=0, sparse=4, pre=2 ** 62, next=2 ** 62) in ok        # huge limits clamp
    assert _call(mask=9, sparse=4, pre=100, next=0) == L.FIA_ERR_PARAM      # with causal
    assert _call(mask=0, sparse=4, pre=3, next=-4) == L.FIA_ERR_PARAM       # empty band
    assert _call(mask=0, sparse=3, pre=3, next=0) == L.FIA_ERR_PARAM        # other sparse modes
