// fia_host.cu -- the C ABI of include/fia.h: validation, launch planning,
// TMA descriptor encoding and the two-phase call.
//
// Phase 1 (fia_get_workspace_size) mirrors the first-phase call of the aclnn
// FusedInferAttentionScore API and the ATB PrefixEncoder
// GetWorkspaceSize call: it verifies the inputs and sizes the workspace.
// seqLen / kvSeqLen are host arrays (the PrefixEncoder parameter table puts
// them on the host), so the whole work decomposition is planned here:
//   * decode path (up to 16 rows -- new token x head of the group -- per KV
//     head, or up to 128 with fewer than 64 new tokens; fia_ext.path may
//     force either path): split-KV units of whole 64-key tiles and 16-row
//     chunks (8 over an int8 cache past 16 rows), sized so the grid fills the
//     SMs several times, ordered longest first; one combine item per
//     (sequence, kv head, chunk), and no combine launch when every item has
//     a single split;
//   * prefill path: (sequence, 128-token tile, head) items, costed by the
//     number of 128-key tiles they read, assigned longest-processing-time
//     first to one persistent CTA per SM.
// Phase 2 (fia_run) uploads the plan (pinned host memory, one async copy)
// into the caller's workspace and launches the kernels on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <functional>
#include <mutex>
#include <numeric>
#include <queue>
#include <vector>

#include "../../include/fia.h"
#include "fia_device.cuh"
#include "fia_plan.h"

namespace {
// NVTX range over one API call (a no-op unless a profiler is attached), so a
// timeline shows planning and each run's launches by name.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace

using namespace fia;

struct fia_op {
    int32_t path = 0;          // 0 no-op, 1 decode, 2 prefill
    int32_t device = -1;       // the device current at phase 1 (runs must use it)
    int32_t q_dtype = 0;       // 0 f16, 1 bf16
    bool kv_int8 = false;
    CUtensorMap tq{}, tk{}, tv{}, tp{};
    CommonArgs common{};
    const float *k_scale = nullptr, *k_offset = nullptr, *v_scale = nullptr, *v_offset = nullptr;
    // plan, uploaded to the front of the workspace by every fia_run
    uint8_t *plan_host = nullptr;      // pinned
    size_t plan_bytes = 0;
    size_t off_seq = 0, off_units = 0, off_citems = 0, off_err = 0, off_cta = 0, off_items = 0;
    size_t off_part_ml = 0, off_part_o = 0;
    uint64_t ws_size = 0;
    int32_t grid = 0, grid2 = 0;
    int32_t direct = 0;             // decode: no combine (every item has one split)
    int32_t max_rows = 0;           // decode: max seqLen * g
    int32_t k_mode = 0, v_mode = 0;     // int8 dequant modes (fia_antiquant_mode)
    int64_t k_tok_stride = 0, v_tok_stride = 0;
    int64_t work_items = 0;
    int32_t split_tokens = 0;
    cudaEvent_t ev_start = nullptr, ev_stop = nullptr;
    // prefill plans small enough to travel as a kernel parameter
    PlanBytes<kInlinePlanBytes> *inline_plan = nullptr;
};

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int64_t numel(const fia_tensor *t) {
    int64_t n = 1;
    for (int i = 0; i < t->ndim; ++i) n *= t->dims[i];
    return n;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// FIA_OK when the current device is the one the op was planned on (its TMA
// descriptors and pointers belong to that device), FIA_ERR_PARAM when another
// device is current, FIA_ERR_CUDA when the query fails.
fia_status check_device(const fia_op *op) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    return cur == op->device ? FIA_OK : FIA_ERR_PARAM;
}

int gcd_int(int a, int b) { return b == 0 ? a : gcd_int(b, a % b); }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 3-D tiled map over a row-major [rows, mid, inner] tensor, 128-byte swizzle;
// the box is box_inner x box_mid x box_rows.
bool encode_3d(CUtensorMap *m, CUtensorMapDataType dt, int esize, void *base, uint64_t inner,
               uint64_t mid, uint64_t rows, uint32_t box_inner, uint32_t box_rows,
               uint32_t box_mid = 1) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, mid, rows};
    cuuint64_t strides[2] = {inner * esize, inner * mid * esize};
    cuuint32_t box[3] = {box_inner, box_mid, box_rows};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, dt, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

fia_status check_f32_vec(const fia_tensor *t, int64_t a, int64_t b /*0 = 1-D*/) {
    if (!t || !t->data) return FIA_ERR_NULLPTR;
    if (t->dtype != FIA_F32) return FIA_ERR_DTYPE;
    if (b == 0) {
        if (numel(t) != a || t->ndim < 1) return FIA_ERR_SHAPE;
    } else {
        if (numel(t) != a * b) return FIA_ERR_SHAPE;
        if (t->ndim >= 2 && t->dims[t->ndim - 1] != b) return FIA_ERR_SHAPE;
    }
    return FIA_OK;
}

}  // namespace

extern "C" {

const char *fia_status_string(fia_status s) {
    switch (s) {
    case FIA_OK: return "ok";
    case FIA_ERR_NULLPTR: return "a required pointer is NULL";
    case FIA_ERR_PARAM: return "a scalar parameter is out of range";
    case FIA_ERR_DTYPE: return "unsupported or mismatched dtype";
    case FIA_ERR_SHAPE: return "inconsistent tensor shapes";
    case FIA_ERR_UNSUPPORTED: return "configuration not supported by this library";
    case FIA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FIA_ERR_CUDA: return "a CUDA call failed";
    }
    return "unknown status";
}

fia_status fia_get_workspace_size(const fia_tensor *query, const fia_tensor *key,
                                  const fia_tensor *value, const fia_tensor *blockTables,
                                  const int32_t *seqLen, const int32_t *kvSeqLen, int32_t batch,
                                  const fia_tensor *slopes, int32_t maskType, int32_t headNum,
                                  int32_t kvHeadNum, float qkScale, const fia_ext *ext,
                                  fia_tensor *attnOut, uint64_t *workspaceSize, fia_op **op) {
    NvtxRange range("fia_get_workspace_size");
    if (!workspaceSize || !op) return FIA_ERR_NULLPTR;
    *workspaceSize = 0;
    *op = nullptr;
    if (!query || !key || !value || !blockTables || !attnOut) return FIA_ERR_NULLPTR;
    if (batch < 0) return FIA_ERR_PARAM;
    if (batch > 0 && (!seqLen || !kvSeqLen)) return FIA_ERR_NULLPTR;
    if (headNum <= 0 || kvHeadNum <= 0 || headNum > 1024) return FIA_ERR_PARAM;
    if (headNum % kvHeadNum != 0) return FIA_ERR_PARAM;
    if (!std::isfinite(qkScale)) return FIA_ERR_PARAM;
    if (maskType != FIA_MASK_NONE && maskType != FIA_MASK_ALIBI && maskType != FIA_MASK_CAUSAL)
        return FIA_ERR_PARAM;
    // band mask (sparseMode 4): replaces maskType; the band must not be empty
    const int32_t sparse = ext ? ext->sparseMode : (int32_t)FIA_SPARSE_NONE;
    if (sparse != FIA_SPARSE_NONE && sparse != FIA_SPARSE_BAND) return FIA_ERR_PARAM;
    const bool band = (sparse == FIA_SPARSE_BAND);
    // limits past +-2^40 cut nothing (lengths < 2^31); clamping first keeps
    // the sum below from overflowing
    const int64_t kLim = int64_t(1) << 40;
    int64_t pre_tok = band ? std::max(-kLim, std::min(ext->preTokens, kLim)) : 0;
    int64_t next_tok = band ? std::max(-kLim, std::min(ext->nextTokens, kLim)) : 0;
    if (band && (maskType != FIA_MASK_NONE || pre_tok + next_tok < 0)) return FIA_ERR_PARAM;


    // ---- dtypes ----
    if (query->dtype != FIA_F16 && query->dtype != FIA_BF16) return FIA_ERR_DTYPE;
    if (attnOut->dtype != query->dtype) return FIA_ERR_DTYPE;
    if (key->dtype != value->dtype) return FIA_ERR_DTYPE;
    const bool kv_int8 = key->dtype == FIA_I8;
    if (!kv_int8 && key->dtype != query->dtype) return FIA_ERR_DTYPE;
    if (blockTables->dtype != FIA_I32) return FIA_ERR_DTYPE;

    // ---- shapes ----
    if (query->ndim != 2 && query->ndim != 3) return FIA_ERR_SHAPE;
    const int64_t n_tokens = query->dims[0];
    int64_t D = 0;
    if (query->ndim == 3) {
        if (query->dims[1] != headNum) return FIA_ERR_SHAPE;
        D = query->dims[2];
    } else {
        if (query->dims[1] % headNum != 0) return FIA_ERR_SHAPE;
        D = query->dims[1] / headNum;
    }
    if (n_tokens < 0 || D <= 0) return FIA_ERR_SHAPE;
    if (numel(attnOut) != n_tokens * headNum * D || attnOut->dims[0] != n_tokens)
        return FIA_ERR_SHAPE;
    int64_t nb = 0, bs = 0;
    const int32_t kv_layout = ext ? ext->kvLayout : (int32_t)FIA_KV_BNBSH;
    if (kv_layout == FIA_KV_BNNBSD) {
        if (key->ndim != 4 || key->dims[1] != kvHeadNum || key->dims[3] != D) return FIA_ERR_SHAPE;
        nb = key->dims[0];
        bs = key->dims[2];
    } else if (kv_layout == FIA_KV_BNBSH) {
        if (key->ndim == 4) {
            if (key->dims[2] != kvHeadNum || key->dims[3] != D) return FIA_ERR_SHAPE;
        } else if (key->ndim == 3) {
            if (key->dims[2] != (int64_t)kvHeadNum * D) return FIA_ERR_SHAPE;
        } else {
            return FIA_ERR_SHAPE;
        }
        nb = key->dims[0];
        bs = key->dims[1];
    } else {
        return FIA_ERR_PARAM;
    }
    if (value->ndim != key->ndim) return FIA_ERR_SHAPE;
    for (int i = 0; i < key->ndim; ++i)
        if (value->dims[i] != key->dims[i]) return FIA_ERR_SHAPE;
    if (blockTables->ndim != 2 || blockTables->dims[0] != batch) return FIA_ERR_SHAPE;
    const int64_t max_blocks = blockTables->dims[1];

    // ---- host lengths ----
    int64_t sum_q = 0, max_q = 0, max_kv = 0, need_blocks = 0;
    for (int b = 0; b < batch; ++b) {
        if (seqLen[b] < 0 || kvSeqLen[b] < 0) return FIA_ERR_PARAM;
        if (kvSeqLen[b] > 0 && seqLen[b] > kvSeqLen[b]) return FIA_ERR_PARAM;
        sum_q += seqLen[b];
        max_q = std::max<int64_t>(max_q, seqLen[b]);
        max_kv = std::max<int64_t>(max_kv, kvSeqLen[b]);
        if (bs > 0) need_blocks = std::max<int64_t>(need_blocks, (kvSeqLen[b] + bs - 1) / bs);
    }
    if (sum_q != n_tokens) return FIA_ERR_SHAPE;
    if (need_blocks > max_blocks) return FIA_ERR_SHAPE;

    // ---- optional tensors ----
    const fia_tensor *pse = ext ? ext->pse : nullptr;
    const fia_tensor *sink = ext ? ext->sink : nullptr;
    const fia_tensor *lse = ext ? ext->lse : nullptr;
    if (maskType == FIA_MASK_ALIBI) {
        fia_status s = check_f32_vec(slopes, headNum, 0);
        if (s != FIA_OK) return s;
    } else if (slopes) {
        return FIA_ERR_PARAM;   // the PrefixEncoder table: slopes only with the ALiBi mask
    }
    if (pse) {
        if (!pse->data) return FIA_ERR_NULLPTR;
        if (pse->dtype != query->dtype) return FIA_ERR_DTYPE;
        if (pse->ndim != 4 || pse->dims[0] != batch || pse->dims[1] != headNum ||
            pse->dims[2] < max_q || pse->dims[3] < max_kv)
            return FIA_ERR_SHAPE;
        if (maskType == FIA_MASK_ALIBI) return FIA_ERR_PARAM;
    }
    if (sink) {
        fia_status s = check_f32_vec(sink, headNum, 0);
        if (s != FIA_OK) return s;
    }
    if (lse) {
        if (!lse->data && n_tokens > 0) return FIA_ERR_NULLPTR;
        if (lse->dtype != FIA_F32) return FIA_ERR_DTYPE;
        if (numel(lse) != n_tokens * headNum || (lse->ndim > 0 && lse->dims[0] != n_tokens))
            return FIA_ERR_SHAPE;
    }
    const fia_tensor *ks = ext ? ext->kScale : nullptr, *ko = ext ? ext->kOffset : nullptr;
    const fia_tensor *vs = ext ? ext->vScale : nullptr, *vo = ext ? ext->vOffset : nullptr;
    const int32_t k_mode = ext ? ext->kAntiquantMode : (int32_t)FIA_ANTIQUANT_PER_CHANNEL;
    const int32_t v_mode = ext ? ext->vAntiquantMode : (int32_t)FIA_ANTIQUANT_PER_CHANNEL;
    if ((k_mode != FIA_ANTIQUANT_PER_CHANNEL && k_mode != FIA_ANTIQUANT_PER_TOKEN) ||
        (v_mode != FIA_ANTIQUANT_PER_CHANNEL && v_mode != FIA_ANTIQUANT_PER_TOKEN))
        return FIA_ERR_PARAM;
    int64_t k_tok_stride = 0, v_tok_stride = 0;
    if (kv_int8) {
        // per-channel: [kvHeadNum, headSize]; per-token: [batch, S] or
        // [1, batch, S] with S >= max kvSeqLen.  Returns the row stride S.
        auto check_quant = [&](const fia_tensor *t, int32_t mode, int64_t *stride) -> fia_status {
            if (mode == FIA_ANTIQUANT_PER_CHANNEL) return check_f32_vec(t, kvHeadNum, D);
            if (!t || !t->data) return FIA_ERR_NULLPTR;
            if (t->dtype != FIA_F32) return FIA_ERR_DTYPE;
            int64_t bd, sd;
            if (t->ndim == 2) {
                bd = t->dims[0];
                sd = t->dims[1];
            } else if (t->ndim == 3 && t->dims[0] == 1) {
                bd = t->dims[1];
                sd = t->dims[2];
            } else {
                return FIA_ERR_SHAPE;
            }
            if (bd != batch || sd < std::max<int64_t>(max_kv, 1)) return FIA_ERR_SHAPE;
            if (*stride != 0 && *stride != sd) return FIA_ERR_SHAPE;   // scale vs offset
            *stride = sd;
            return FIA_OK;
        };
        fia_status st;
        if ((st = check_quant(ks, k_mode, &k_tok_stride)) != FIA_OK) return st;
        if (ko && (st = check_quant(ko, k_mode, &k_tok_stride)) != FIA_OK) return st;
        if ((st = check_quant(vs, v_mode, &v_tok_stride)) != FIA_OK) return st;
        if (vo && (st = check_quant(vo, v_mode, &v_tok_stride)) != FIA_OK) return st;
    } else if (ks || vs || ko || vo || k_mode != 0 || v_mode != 0) {
        return FIA_ERR_PARAM;
    }

    // ---- build limits ----
    const int g = headNum / kvHeadNum;
    if (D != 64 && D != 128) return FIA_ERR_UNSUPPORTED;
    if (bs < 16 || bs > 256 || bs % 16 != 0) return FIA_ERR_UNSUPPORTED;
    if (nb * bs >= (int64_t(1) << 31) || n_tokens >= (int64_t(1) << 31)) return FIA_ERR_UNSUPPORTED;
    if (band && max_kv >= (int64_t(1) << 30)) return FIA_ERR_UNSUPPORTED;
    // Kernel choice.  The tensor-core kernel's 128-row tiles hold one query
    // head's new tokens, so they are well filled only for long new-token
    // runs; decode-shaped calls (up to 16 rows per KV head, or fewer than 64
    // new tokens and at most 8 chunks of 16 rows) take the decode kernels,
    // one unit per 16-row chunk, the chunks of one key range side by side so
    // that the later reads of each K/V tile come from L2.
    const int32_t path_hint = ext ? ext->path : (int32_t)FIA_PATH_AUTO;
    if (path_hint != FIA_PATH_AUTO && path_hint != FIA_PATH_DECODE && path_hint != FIA_PATH_TENSOR)
        return FIA_ERR_PARAM;
    const int64_t rows_per_kvh = max_q * g;
    const bool fits_decode = rows_per_kvh <= (int64_t)kDecodeRows * kDecodeMaxChunks;
    if (path_hint == FIA_PATH_DECODE && !fits_decode) return FIA_ERR_PARAM;
    const bool decode = path_hint == FIA_PATH_DECODE ||
                        (path_hint == FIA_PATH_AUTO &&
                         (rows_per_kvh <= kDecodeRows || (fits_decode && max_q < 64)));
    // int8 rows are one 128-byte TMA box row per key on both paths
    if (kv_int8 && D != 128) return FIA_ERR_UNSUPPORTED;

    fia_op *o = new fia_op();
    o->q_dtype = query->dtype == FIA_BF16 ? 1 : 0;
    o->kv_int8 = kv_int8;
    if (n_tokens == 0) {
        *op = o;
        return FIA_OK;
    }
    // pointers: TMA and vector stores need 16-byte alignment
    if (!query->data || !attnOut->data || !key->data || !value->data) {
        delete o;
        return FIA_ERR_NULLPTR;
    }
    if (max_kv > 0 && !blockTables->data) {
        delete o;
        return FIA_ERR_NULLPTR;
    }
    if (!aligned16(query->data) || !aligned16(attnOut->data) || !aligned16(key->data) ||
        !aligned16(value->data)) {
        delete o;
        return FIA_ERR_PARAM;
    }

    // ---- device facts ----
    int dev = 0, nsm = 0, cc_major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        delete o;
        return FIA_ERR_CUDA;
    }
    if (cc_major != 10) {
        delete o;
        return FIA_ERR_UNSUPPORTED;
    }

    CommonArgs &c = o->common;
    c.q = query->data;
    c.out = attnOut->data;
    c.lse = lse ? reinterpret_cast<float *>(lse->data) : nullptr;
    c.bt = reinterpret_cast<const int32_t *>(blockTables->data);
    c.slopes = maskType == FIA_MASK_ALIBI ? reinterpret_cast<const float *>(slopes->data) : nullptr;
    c.pse = pse ? pse->data : nullptr;
    c.pse_q = pse ? pse->dims[2] : 0;
    c.pse_kv = pse ? pse->dims[3] : 0;
    c.pse_vec = pse ? ((c.pse_kv % 8) == 0 && aligned16(pse->data)) : 0;
    c.sink = sink ? reinterpret_cast<const float *>(sink->data) : nullptr;
    c.bt_stride = (int32_t)max_blocks;
    c.H = headNum;
    c.KVH = kvHeadNum;
    c.g = g;
    c.D = (int32_t)D;
    c.bs = (int32_t)bs;
    c.kv_layout = kv_layout;
    c.band = band ? 1 : 0;
    // beyond +-(max kvSeqLen + 1) a band limit cuts nothing; clamped there the
    // kernels' int32 position arithmetic cannot overflow (kvSeqLen < 2^30)
    c.pre = (int32_t)std::max<int64_t>(-(max_kv + 1), std::min<int64_t>(pre_tok, max_kv + 1));
    c.next = (int32_t)std::max<int64_t>(-(max_kv + 1), std::min<int64_t>(next_tok, max_kv + 1));
    c.mask_type = maskType;
    c.scale_log2 = qkScale * 1.4426950408889634f;
    c.wait_ns = kWaitLimitNs;
    c.stall = 0;
    o->device = dev;
    if (kv_int8) {
        o->k_mode = k_mode;
        o->v_mode = v_mode;
        o->k_tok_stride = k_tok_stride;
        o->v_tok_stride = v_tok_stride;
        o->k_scale = reinterpret_cast<const float *>(ks->data);
        o->k_offset = ko ? reinterpret_cast<const float *>(ko->data) : nullptr;
        o->v_scale = reinterpret_cast<const float *>(vs->data);
        o->v_offset = vo ? reinterpret_cast<const float *>(vo->data) : nullptr;
    }

    // ---- TMA descriptors ----
    const CUtensorMapDataType tdt =
        query->dtype == FIA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const int kv_es = kv_int8 ? 1 : 2;
    const CUtensorMapDataType kdt = kv_int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : tdt;
    const uint32_t box_inner = kv_int8 ? 128u : 64u;
    const int box_rows = decode ? gcd_int((int)bs, kDecodeTile) : gcd_int((int)bs, kPrefillBN);
    c.box_rows = box_rows;
    // K/V maps: {D, KVH, blocks*bs} (BnBsH, box of one head x rows) or
    // {D, bs, blocks*KVH} (BnNBsD, box of rows x one head); both land in
    // shared memory as `rows` consecutive 128-byte rows
    bool enc_ok;
    if (kv_layout == FIA_KV_BNNBSD)
        enc_ok = encode_3d(&o->tk, kdt, kv_es, key->data, D, bs, nb * kvHeadNum, box_inner, 1,
                           box_rows) &&
                 encode_3d(&o->tv, kdt, kv_es, value->data, D, bs, nb * kvHeadNum, box_inner, 1,
                           box_rows);
    else
        enc_ok = encode_3d(&o->tk, kdt, kv_es, key->data, D, kvHeadNum, nb * bs, box_inner, box_rows) &&
                 encode_3d(&o->tv, kdt, kv_es, value->data, D, kvHeadNum, nb * bs, box_inner, box_rows);
    if (!decode)
        enc_ok = enc_ok && encode_3d(&o->tq, tdt, 2, query->data, D, headNum, n_tokens, 64, kPrefillBM);
    if (!decode && pse && (pse->dims[3] % 8) == 0 && aligned16(pse->data)) {
        // pse viewed as {maxKV, maxQ, B*H}; one softmax warp fetches two
        // {64 keys, 16 rows} boxes per key tile (128-byte swizzle)
        auto fn = encode_fn();
        cuuint64_t dims[3] = {(cuuint64_t)pse->dims[3], (cuuint64_t)pse->dims[2],
                              (cuuint64_t)(pse->dims[0] * pse->dims[1])};
        cuuint64_t strides[2] = {(cuuint64_t)pse->dims[3] * 2,
                                 (cuuint64_t)(pse->dims[2] * pse->dims[3] * 2)};
        cuuint32_t box[3] = {64, 16, 1};
        cuuint32_t es[3] = {1, 1, 1};
        enc_ok = enc_ok && fn &&
                 fn(&o->tp, tdt, 3, pse->data, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        c.pse_tma = 1;
    }
    if (!enc_ok) {
        delete o;
        return FIA_ERR_CUDA;
    }

    // ---- plan ----
    std::vector<SeqInfo> seq(batch);
    {
        int32_t cu = 0;
        for (int b = 0; b < batch; ++b) {
            seq[b] = {cu, seqLen[b], kvSeqLen[b], 0};
            cu += seqLen[b];
        }
    }
    size_t off = 0;
    o->off_seq = off;
    off = align_up(off + sizeof(SeqInfo) * std::max(batch, 1), 256);
    o->off_err = off;
    off = align_up(off + kErrRegionBytes, 256);
    std::vector<uint8_t> host;
    if (decode) {
        o->path = 1;
        // Rows per unit: 16, or, for an int8 cache past 16 rows per KV head,
        // 8, so that every unit runs the int8 kernel's single-column-tile
        // instance (no spills, four CTAs per SM); the extra reads of each
        // K/V tile by the other chunks of its key range come from L2.
        const int chunk_rows = (kv_int8 && max_q * g > kDecodeRows) ? kDecodeRows / 2 : kDecodeRows;
        c.chunk_rows = chunk_rows;
        o->max_rows = (int32_t)std::min<int64_t>(max_q * g, chunk_rows);   // per unit
        const bool causal = (maskType != FIA_MASK_NONE);
        (void)causal;
        // keys a sequence's rows can see: all of [0, kvSeqLen), or under a band
        // [minQpos - pre, maxQpos + next] with the start rounded down to a
        // 64-key tile (TMA boxes stay block-aligned)
        auto key_range = [&](int b, int64_t *lo, int64_t *hi) {
            const int64_t kl = kvSeqLen[b], ql = seqLen[b];
            *lo = 0;
            *hi = kl;
            if (band) {
                *lo = std::max<int64_t>(0, kl - ql - pre_tok);
                *hi = std::min<int64_t>(kl, kl + next_tok);
                if (*hi <= *lo) *hi = *lo = 0;
                *lo = (*lo / kDecodeTile) * kDecodeTile;
            }
        };
        // 16-row chunks of sequence b's seqLen * g rows
        auto chunks = [&](int b) { return (int)((int64_t(seqLen[b]) * g + chunk_rows - 1) / chunk_rows); };
        int64_t total = 0;
        for (int b = 0; b < batch; ++b) {
            int64_t lo, hi;
            key_range(b, &lo, &hi);
            total += (hi - lo) * kvHeadNum * chunks(b);
        }
        const int64_t target_units = (int64_t)nsm * 2 * 4;
        int64_t split = (total + target_units - 1) / std::max<int64_t>(target_units, 1);
        split = std::max<int64_t>(2 * kDecodeTile, align_up(std::max<int64_t>(split, 1), kDecodeTile));
        o->split_tokens = (int32_t)split;
        std::vector<DecodeUnit> units;
        std::vector<CombineItem> citems;
        int32_t slot = 0;
        for (int b = 0; b < batch; ++b) {
            if (seqLen[b] == 0) continue;
            int64_t lo, hi;
            key_range(b, &lo, &hi);
            const int ns = (int)std::max<int64_t>(1, (hi - lo + split - 1) / split);
            const int nch = chunks(b);
            for (int kvh = 0; kvh < kvHeadNum; ++kvh) {
                // chunk c owns slots slot + c * ns .. + ns - 1 (one per split)
                for (int ch = 0; ch < nch; ++ch) {
                    CombineItem ci{};
                    ci.slot0 = slot + ch * ns;
                    ci.nsplit = ns;
                    ci.b = b;
                    ci.kvh = kvh;
                    ci.r0 = ch * chunk_rows;
                    citems.push_back(ci);
                }
                for (int s = 0; s < ns; ++s) {
                    for (int ch = 0; ch < nch; ++ch) {
                        DecodeUnit u{};
                        u.b = b;
                        u.kvh = kvh;
                        u.t_begin = (int32_t)std::min<int64_t>(hi, lo + s * split);
                        u.t_end = (int32_t)std::min<int64_t>(hi, lo + (s + 1) * split);
                        u.slot = slot + ch * ns + s;
                        u.r0 = ch * chunk_rows;
                        units.push_back(u);
                    }
                }
                slot += nch * ns;
            }
        }
        std::stable_sort(units.begin(), units.end(), [](const DecodeUnit &x, const DecodeUnit &y) {
            return (x.t_end - x.t_begin) > (y.t_end - y.t_begin);
        });
        o->off_units = off;
        off = align_up(off + sizeof(DecodeUnit) * std::max<size_t>(units.size(), 1), 256);
        o->off_citems = off;
        off = align_up(off + sizeof(CombineItem) * std::max<size_t>(citems.size(), 1), 256);
        o->plan_bytes = off;
        o->off_part_ml = off;
        off = align_up(off + sizeof(float2) * kDecodeRows * std::max(slot, 1), 256);
        o->off_part_o = off;
        off = align_up(off + sizeof(float) * kDecodeRows * D * std::max(slot, 1), 256);
        o->ws_size = off;
        o->grid = (int32_t)units.size();
        // every (sequence, KV head, chunk) in one split: the decode units
        // finish their rows themselves and the combine launch is skipped
        bool one_split = true;
        for (const CombineItem &ci : citems) one_split = one_split && ci.nsplit == 1;
        o->direct = one_split ? 1 : 0;
        o->grid2 = one_split ? 0 : (int32_t)citems.size();
        o->work_items = (int64_t)units.size();
        host.assign(o->plan_bytes, 0);
        std::memcpy(host.data() + o->off_seq, seq.data(), sizeof(SeqInfo) * batch);
        std::memcpy(host.data() + o->off_units, units.data(), sizeof(DecodeUnit) * units.size());
        std::memcpy(host.data() + o->off_citems, citems.data(), sizeof(CombineItem) * citems.size());
    } else {
        o->path = 2;
        const bool causal = (maskType != FIA_MASK_NONE);
        // Pairs of 128-token tiles that read the same KV head: two heads of a
        // GQA group (same tile), else two consecutive tiles of one head.  Tile
        // 0 of a pair needs no more key tiles than tile 1.  Under a band mask
        // a tile's key tiles start past 0 too, so g = 1 tiles stay unpaired
        // (both tiles of a pair then always share one key-tile range).
        // (The kernel derives the same ranges from the same rule.)
        auto ntiles = [&](int b, int q0) {
            const int64_t ql = seqLen[b], kl = kvSeqLen[b];
            const int64_t rows = std::min<int64_t>(kPrefillBM, ql - q0);
            const int64_t qmin = kl - ql + q0, qmax = qmin + rows - 1;
            int64_t lo = 0, hi = causal ? std::min(kl, qmax + 1) : kl;
            if (band) {
                lo = std::max<int64_t>(0, qmin - pre_tok);
                hi = std::min<int64_t>(kl, qmax + next_tok + 1);
            }
            if (hi <= lo) return 0;
            return (int)((hi + kPrefillBN - 1) / kPrefillBN - lo / kPrefillBN);
        };
        struct Cand {
            PrefillItem it;
            double cost;
        };
        std::vector<Cand> items;
        auto add = [&](int b, int kvh, int q0a, int ha, int q0b, int hb) {
            PrefillItem it{};
            it.b = b;
            it.kvh = kvh;
            it.q0[0] = q0a; it.h[0] = ha;
            it.q0[1] = q0b; it.h[1] = hb;
            const int nb = ntiles(b, q0b);
            items.push_back({it, nb + 0.75});
        };
        for (int b = 0; b < batch; ++b) {
            const int ql = seqLen[b];
            const int nqt = (ql + kPrefillBM - 1) / kPrefillBM;
            if (g >= 2) {
                for (int qt = 0; qt < nqt; ++qt) {
                    const int q0 = qt * kPrefillBM;
                    for (int kvh = 0; kvh < kvHeadNum; ++kvh) {
                        int h = kvh * g;
                        for (; h + 1 < (kvh + 1) * g; h += 2) add(b, kvh, q0, h, q0, h + 1);
                        if (h < (kvh + 1) * g) add(b, kvh, 0, -1, q0, h);
                    }
                }
            } else {
                for (int h = 0; h < headNum; ++h) {
                    int qt = 0;
                    if (!band)
                        for (; qt + 1 < nqt; qt += 2)
                            add(b, h, qt * kPrefillBM, h, (qt + 1) * kPrefillBM, h);
                    for (; qt < nqt; ++qt) add(b, h, 0, -1, qt * kPrefillBM, h);
                }
            }
        }
        std::stable_sort(items.begin(), items.end(),
                         [](const Cand &x, const Cand &y) { return x.cost > y.cost; });
        const int grid = (int)std::min<int64_t>(nsm, (int64_t)items.size());
        std::vector<std::vector<PrefillItem>> per(grid);
        using Load = std::pair<double, int>;
        std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
        for (int i = 0; i < grid; ++i) heap.push({0.0, i});
        for (const Cand &cd : items) {
            Load l = heap.top();
            heap.pop();
            per[l.second].push_back(cd.it);
            heap.push({l.first + cd.cost, l.second});
        }
        // A CTA's total, hence the makespan, does not depend on the order of its
        // items.  Ordered by (sequence, KV head), every CTA sweeps the KV heads
        // at about the same pace, so the K/V tiles in use at any moment are
        // those of a few heads and stay in L2 between their items (longest
        // first, the items of all heads run at once and K/V is re-read).
        for (auto &v : per)
            std::stable_sort(v.begin(), v.end(), [](const PrefillItem &x, const PrefillItem &y) {
                return x.b != y.b ? x.b < y.b : x.kvh < y.kvh;
            });
        std::vector<int32_t> cta_off(grid + 1, 0);
        std::vector<PrefillItem> flat;
        flat.reserve(items.size());
        for (int i = 0; i < grid; ++i) {
            cta_off[i] = (int32_t)flat.size();
            flat.insert(flat.end(), per[i].begin(), per[i].end());
        }
        cta_off[grid] = (int32_t)flat.size();
        o->off_cta = off;
        off = align_up(off + sizeof(int32_t) * (grid + 1), 256);
        o->off_items = off;
        off = align_up(off + sizeof(PrefillItem) * std::max<size_t>(flat.size(), 1), 256);
        o->plan_bytes = off;
        o->ws_size = off;
        o->grid = grid;
        o->work_items = (int64_t)flat.size();
        host.assign(o->plan_bytes, 0);
        std::memcpy(host.data() + o->off_seq, seq.data(), sizeof(SeqInfo) * batch);
        std::memcpy(host.data() + o->off_cta, cta_off.data(), sizeof(int32_t) * (grid + 1));
        std::memcpy(host.data() + o->off_items, flat.data(), sizeof(PrefillItem) * flat.size());
        if (o->plan_bytes <= (size_t)kInlinePlanBytes) {
            // the plan rides in the launch parameters; the workspace keeps only
            // the error words (cleared by the kernel itself)
            o->inline_plan = new PlanBytes<kInlinePlanBytes>();
            std::memset(o->inline_plan->b, 0, sizeof(o->inline_plan->b));
            std::memcpy(o->inline_plan->b, host.data(), o->plan_bytes);
            o->off_err = 0;
            o->ws_size = align_up(kErrRegionBytes, 256);
            *workspaceSize = o->ws_size;
            *op = o;
            return FIA_OK;
        }
    }
    if (cudaMallocHost(reinterpret_cast<void **>(&o->plan_host), o->plan_bytes) != cudaSuccess) {
        cudaGetLastError();
        delete o;
        return FIA_ERR_CUDA;
    }
    std::memcpy(o->plan_host, host.data(), o->plan_bytes);
    *workspaceSize = o->ws_size;
    *op = o;
    return FIA_OK;
}

fia_status fia_run(void *workspace, uint64_t workspaceSize, fia_op *op, void *stream_ptr) {
    if (!op) return FIA_ERR_NULLPTR;
    if (op->path == 0) return FIA_OK;
    NvtxRange range(op->path == 1 ? "fia_run decode" : "fia_run prefill");
    if (!workspace || workspaceSize < op->ws_size ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return FIA_ERR_WORKSPACE;
    const fia_status dst = check_device(op);
    if (dst != FIA_OK) return dst;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_ptr);
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    if (!op->inline_plan &&
        cudaMemcpyAsync(ws, op->plan_host, op->plan_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    CommonArgs c = op->common;
    c.seq = reinterpret_cast<const SeqInfo *>(ws + op->off_seq);
    c.err = reinterpret_cast<uint32_t *>(ws + op->off_err);
    if (op->ev_start && cudaEventRecord(op->ev_start, s) != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    cudaError_t e = cudaSuccess;
    if (op->path == 1) {
        DecodeArgs d{};
        d.c = c;
        d.units = reinterpret_cast<const DecodeUnit *>(ws + op->off_units);
        d.part_o = reinterpret_cast<float *>(ws + op->off_part_o);
        d.part_ml = reinterpret_cast<float2 *>(ws + op->off_part_ml);
        d.k_scale = op->k_scale;
        d.k_offset = op->k_offset;
        d.v_scale = op->v_scale;
        d.v_offset = op->v_offset;
        d.k_tok_stride = op->k_tok_stride;
        d.v_tok_stride = op->v_tok_stride;
        d.k_mode = op->k_mode;
        d.v_mode = op->v_mode;
        d.n_units = op->grid;
        d.max_rows = op->max_rows;
        d.direct = op->direct;
        if (op->grid > 0) e = launch_decode(d, op->tk, op->tv, op->q_dtype, op->kv_int8, op->grid, s);
        if (e == cudaSuccess && op->grid2 > 0) {
            CombineArgs cb{};
            cb.c = c;
            cb.items = reinterpret_cast<const CombineItem *>(ws + op->off_citems);
            cb.part_o = d.part_o;
            cb.part_ml = d.part_ml;
            cb.v_scale = op->v_scale;
            cb.v_offset = op->v_offset;
            cb.v_mode = op->v_mode;
            cb.n_items = op->grid2;
            e = launch_combine(cb, op->q_dtype, op->kv_int8, op->grid2, s);
        }
    } else {
        PrefillArgs p{};
        p.c = c;
        p.plan = op->inline_plan ? nullptr : ws;
        p.off_seq = (int32_t)op->off_seq;
        p.off_cta = (int32_t)op->off_cta;
        p.off_items = (int32_t)op->off_items;
        p.k_scale = op->k_scale;
        p.k_offset = op->k_offset;
        p.v_scale = op->v_scale;
        p.v_offset = op->v_offset;
        p.k_tok_stride = op->k_tok_stride;
        p.v_tok_stride = op->v_tok_stride;
        p.k_mode = op->k_mode;
        p.v_mode = op->v_mode;
        if (op->grid > 0)
            e = launch_prefill(p, op->tq, op->tk, op->tv, op->tp, op->q_dtype, op->kv_int8,
                               op->grid, op->inline_plan ? op->inline_plan->b : nullptr, s);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    if (op->ev_stop && cudaEventRecord(op->ev_stop, s) != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    return FIA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode with library-owned scratch (fia_decode_run_static).  The scratch is a
// file-scope device array; host code only ever sees its address through
// cudaGetSymbolAddress, looked up once per device and cached.
// ---------------------------------------------------------------------------
namespace {
constexpr int kMaxStaticDevices = 64;
static __device__ __align__(256) uint8_t g_fia_static_ws[FIA_STATIC_WORKSPACE_BYTES];
std::mutex g_static_mu;
void *g_static_addr[kMaxStaticDevices] = {};
}  // namespace

extern "C" {

fia_status fia_decode_run_static(fia_op *op, void *stream_ptr) {
    if (!op) return FIA_ERR_NULLPTR;
    if (op->path == 0) return FIA_OK;
    if (op->path != 1) return FIA_ERR_UNSUPPORTED;
    if (op->ws_size > FIA_STATIC_WORKSPACE_BYTES) return FIA_ERR_WORKSPACE;
    NvtxRange range("fia_decode_run_static");
    const fia_status dst = check_device(op);
    if (dst != FIA_OK) return dst;
    const int dev = op->device;
    if (dev < 0 || dev >= kMaxStaticDevices) return FIA_ERR_UNSUPPORTED;
    uint8_t *ws = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_static_mu);
        if (!g_static_addr[dev]) {
            void *addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_fia_static_ws) != cudaSuccess || !addr) {
                cudaGetLastError();
                return FIA_ERR_CUDA;
            }
            g_static_addr[dev] = addr;
        }
        ws = reinterpret_cast<uint8_t *>(g_static_addr[dev]);
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_ptr);
    // The plan (which also clears the error word) is rewritten on every call;
    // every partial the combine reads is written by the decode kernel first.
    if (cudaMemcpyAsync(ws, op->plan_host, op->plan_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    CommonArgs c = op->common;
    c.seq = reinterpret_cast<const SeqInfo *>(ws + op->off_seq);
    c.err = reinterpret_cast<uint32_t *>(ws + op->off_err);
    DecodeArgs d{};
    d.c = c;
    d.units = reinterpret_cast<const DecodeUnit *>(ws + op->off_units);
    d.part_o = reinterpret_cast<float *>(ws + op->off_part_o);
    d.part_ml = reinterpret_cast<float2 *>(ws + op->off_part_ml);
    d.k_scale = op->k_scale;
    d.k_offset = op->k_offset;
    d.v_scale = op->v_scale;
    d.v_offset = op->v_offset;
    d.k_tok_stride = op->k_tok_stride;
    d.v_tok_stride = op->v_tok_stride;
    d.k_mode = op->k_mode;
    d.v_mode = op->v_mode;
    d.n_units = op->grid;
    d.max_rows = op->max_rows;
    d.direct = op->direct;
    if (op->ev_start && cudaEventRecord(op->ev_start, s) != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    cudaError_t e = cudaSuccess;
    if (op->grid > 0) e = launch_decode(d, op->tk, op->tv, op->q_dtype, op->kv_int8, op->grid, s);
    if (e == cudaSuccess && op->grid2 > 0) {
        CombineArgs cb{};
        cb.c = c;
        cb.items = reinterpret_cast<const CombineItem *>(ws + op->off_citems);
        cb.part_o = d.part_o;
        cb.part_ml = d.part_ml;
        cb.v_scale = op->v_scale;
        cb.v_offset = op->v_offset;
        cb.v_mode = op->v_mode;
        cb.n_items = op->grid2;
        e = launch_combine(cb, op->q_dtype, op->kv_int8, op->grid2, s);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    if (op->ev_stop && cudaEventRecord(op->ev_stop, s) != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    return FIA_OK;
}

fia_status fia_decode_static_error_word(const fia_op *op, uint32_t *word) {
    if (!op || !word) return FIA_ERR_NULLPTR;
    *word = 0;
    if (op->path == 0) return FIA_OK;
    if (op->path != 1) return FIA_ERR_UNSUPPORTED;
    const fia_status dst = check_device(op);
    if (dst != FIA_OK) return dst;
    if (cudaMemcpyFromSymbol(word, g_fia_static_ws, sizeof(uint32_t), op->off_err,
                             cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return FIA_ERR_CUDA;
    }
    return FIA_OK;
}

void fia_op_destroy(fia_op *op) {
    if (!op) return;
    if (op->plan_host) cudaFreeHost(op->plan_host);
    delete op->inline_plan;
    delete op;
}

fia_status fia_op_set_timing_events(fia_op *op, void *start, void *stop) {
    if (!op) return FIA_ERR_NULLPTR;
    if ((start == nullptr) != (stop == nullptr)) return FIA_ERR_PARAM;
    op->ev_start = reinterpret_cast<cudaEvent_t>(start);
    op->ev_stop = reinterpret_cast<cudaEvent_t>(stop);
    return FIA_OK;
}

fia_status fia_op_set_wait_limit(fia_op *op, uint64_t wait_limit_ns, int32_t stall) {
    if (!op) return FIA_ERR_NULLPTR;
    if (stall != 0 && stall != 1) return FIA_ERR_PARAM;
    op->common.wait_ns = wait_limit_ns ? wait_limit_ns : kWaitLimitNs;
    op->common.stall = stall;
    return FIA_OK;
}

fia_status fia_op_get_plan_info(const fia_op *op, fia_plan_info *info) {
    if (!op || !info) return FIA_ERR_NULLPTR;
    info->path = op->path;
    info->kernels_per_run = op->path == 1 ? ((op->grid > 0) + (op->grid2 > 0)) : (op->path == 2 && op->grid > 0);
    info->work_items = op->work_items;
    info->grid = op->grid;
    info->split_tokens = op->split_tokens;
    info->error_word_offset = (int64_t)op->off_err;
    return FIA_OK;
}

}  // extern "C"
