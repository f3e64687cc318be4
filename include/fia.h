/*
 * fia.h -- C ABI of the B200 paged fused-inference-attention library (libfia.so).
 *
 * Operation (aclnnFusedInferAttentionScoreV4 "Formula"; V3 "Formula"):
 *
 *     attnOut = Softmax(qkScale * Q K^T + bias) V
 *
 * over a paged K/V cache (V4/V3 paged-attention bullets: the blocks that
 * blockTables lists for a sequence form one logically contiguous K/V run),
 * with GQA head grouping, an internally generated causal mask, an ALiBi bias
 * from per-head slopes, an optional full pse-shift bias, an optional lse
 * output, an optional per-head learnable sink and an optional int8 K/V cache
 * with per-channel dequantisation.  One call covers both the prefill /
 * prefix-encoder case (several new tokens per sequence attending to the cached
 * prefix and to themselves) and single-token decode.
 *
 * Call pattern (the two-phase convention of the aclnn API and of the ATB
 * PrefixEncoder interface, "Definition"):
 *
 *     fia_get_workspace_size(...)  -> validates everything, plans the launch,
 *                                     reports the workspace size, returns an op
 *     fia_run(workspace, size, op, stream)
 *                                  -> enqueues the kernels on the stream
 *     fia_op_destroy(op)
 *
 * Conventions that hold for every entry point:
 *  - Every tensor is dense, row-major and contiguous.  `data` is a DEVICE
 *    pointer unless a parameter says "host".  The caller owns every buffer;
 *    the op keeps pointers, not copies, so the tensors and the workspace must
 *    stay alive and unchanged until the stream has finished fia_run.
 *  - Phase 1 launches nothing and reads or writes no device memory.  It does
 *    query the current device's attributes and encodes TMA descriptors, so it
 *    needs a CUDA device (it returns FIA_ERR_CUDA without one).
 *  - fia_run is asynchronous on `stream`, allocates nothing and does not
 *    synchronise.  It may be called any number of times on the same op.
 *  - Block ids in blockTables are not validated on the device; the V3 page's
 *    paged-attention constraints leave that check to the caller as well.
 *    Entries past ceil(kvSeqLen[b] / blockSize) are never read.
 *  - An op belongs to the device that was current when phase 1 ran (its
 *    pointers and TMA descriptors refer to that device's memory).  Every call
 *    that launches work checks that the same device is current and returns
 *    FIA_ERR_PARAM otherwise.
 *  - Errors are returned as fia_status; nothing is printed and nothing aborts.
 */
#ifndef FIA_H
#define FIA_H

#include <stdint.h>

#if defined(__GNUC__)
#define FIA_API __attribute__((visibility("default")))
#else
#define FIA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FIA_OK = 0,
    FIA_ERR_NULLPTR = 1,     /* a required pointer is NULL                        */
    FIA_ERR_PARAM = 2,       /* a scalar parameter is out of range                */
    FIA_ERR_DTYPE = 3,       /* a tensor has a dtype the operation does not take  */
    FIA_ERR_SHAPE = 4,       /* tensor ranks / extents are inconsistent           */
    FIA_ERR_UNSUPPORTED = 5, /* valid per the pages but not built (e.g. D=96)     */
    FIA_ERR_WORKSPACE = 6,   /* workspace NULL, misaligned or smaller than needed */
    FIA_ERR_CUDA = 7         /* a CUDA runtime / driver call failed               */
} fia_status;

typedef enum { FIA_F16 = 0, FIA_BF16 = 1, FIA_F32 = 2, FIA_I8 = 3, FIA_I32 = 4 } fia_dtype;

/* A dense row-major tensor: dims[0] is the slowest axis.  ndim <= 4. */
typedef struct {
    void *data;
    fia_dtype dtype;
    int32_t ndim;
    int64_t dims[4];
} fia_tensor;

/* maskType codes of the ATB PrefixEncoder table ("maskType" row). */
typedef enum {
    FIA_MASK_NONE = 0,   /* no mask: every key t < kvSeqLen[b] is visible              */
    FIA_MASK_ALIBI = 3,  /* MASK_TYPE_ALIBI_COMPRESS: causal mask plus the ALiBi bias
                            slope_h * (t - qpos), generated in registers from `slopes` */
    FIA_MASK_CAUSAL = 9  /* MASK_TYPE_CAUSAL_MASK: internally generated causal mask     */
} fia_mask_type;

/* Optional extensions; the struct pointer and every field may be NULL. */
/* Paged KV cache layout (aclnnFusedInferAttentionScoreV3, paged attention
   constraints: the cache may be BnBsH or BnNBsD, BnNBsD being the one the page
   recommends for performance).  key and value use the same layout.
     FIA_KV_BNBSH   [numBlocks, blockSize, kvHeadNum, headSize] (4-D) or
                    [numBlocks, blockSize, kvHeadNum * headSize] (3-D)
     FIA_KV_BNNBSD  [numBlocks, kvHeadNum, blockSize, headSize] (4-D only): the
                    rows of one (block, KV head) are contiguous. */
typedef enum { FIA_KV_BNBSH = 0, FIA_KV_BNNBSD = 1 } fia_kv_layout;

/* int8 KV dequantisation modes (V3 fake-quantization: per-channel mode, and
   per-token mode with scale/offset of shape (B, S) or (1, B, S), f32). */
typedef enum { FIA_ANTIQUANT_PER_CHANNEL = 0, FIA_ANTIQUANT_PER_TOKEN = 1 } fia_antiquant_mode;

/* sparse modes (V3 sparseMode): 0 = mask from maskType, 4 = band */
typedef enum { FIA_SPARSE_NONE = 0, FIA_SPARSE_BAND = 4 } fia_sparse_mode;

/* kernel choice (fia_ext.path).  FIA_PATH_AUTO picks the split-KV decode
   kernels when the rows per KV head (max seqLen * headNum / kvHeadNum) are at
   most 16, or at most 128 with max seqLen < 64 (in 16-row chunks), and the
   tensor-core prefill kernel otherwise.  FIA_PATH_DECODE / FIA_PATH_TENSOR
   force one (the result agrees to rounding; FIA_PATH_DECODE with more than
   128 rows per KV head is FIA_ERR_PARAM). */
typedef enum { FIA_PATH_AUTO = 0, FIA_PATH_DECODE = 1, FIA_PATH_TENSOR = 2 } fia_path;

typedef struct {
    /* pse-shift bias [batch, headNum, maxQ, maxKV], the query's dtype, added to
       the scaled scores: s += pse[b][h][i][t] for new token i and key position t
       (V4 "alibi fullmask" restrictions: shape [B, N, maxQ, maxKV]).  Needs
       maxQ >= max seqLen and maxKV >= max kvSeqLen.  Not combinable with
       FIA_MASK_ALIBI. */
    const fia_tensor *pse;
    /* learnable sink [headNum] f32 (V4 learnableSinkOptional): a raw logit,
       not scaled by qkScale, that joins the softmax denominator with no value
       row.  lse includes it. */
    const fia_tensor *sink;
    /* int8 K/V dequantisation (V3 fake-quantization bullets).  The cache value
       x stands for scale * (x + offset).  kScale and vScale are required when
       key/value are FIA_I8; a NULL offset means 0 (symmetric).  Per key / value
       mode (kAntiquantMode / vAntiquantMode below):
         FIA_ANTIQUANT_PER_CHANNEL  [kvHeadNum, headSize] f32: one pair per
                                    (KV head, channel);
         FIA_ANTIQUANT_PER_TOKEN    [batch, S] or [1, batch, S] f32 with
                                    S >= max kvSeqLen: one pair per (sequence,
                                    cached token position), shared by every
                                    KV head and channel of that token.
       Scale and offset of one operand use the same mode; K and V may differ
       (e.g. per-channel keys with per-token values). */
    const fia_tensor *kScale;
    const fia_tensor *kOffset;
    const fia_tensor *vScale;
    const fia_tensor *vOffset;
    /* lse output [nTokens, headNum] f32 (V3 "lse" bullet): m + log(sum exp(s - m)).
       Rows with no visible key get +inf. */
    fia_tensor *lse;
    /* KV cache layout, a fia_kv_layout value (0, the default, is BnBsH).  A
       zero-initialised fia_ext keeps the default. */
    int32_t kvLayout;
    /* int8 dequantisation modes of K and V, fia_antiquant_mode values (0, the
       default, is per-channel). */
    int32_t kAntiquantMode;
    int32_t vAntiquantMode;
    /* Band mask (V3 sparseMode 4 with preTokens / nextTokens): with
       sparseMode = FIA_SPARSE_BAND, new token i (absolute position qpos =
       kvSeqLen - seqLen + i) sees the cached keys t with
       qpos - preTokens <= t <= qpos + nextTokens (and t < kvSeqLen);
       maskType must then be FIA_MASK_NONE, and preTokens + nextTokens >= 0.
       A row whose band holds no key gets out 0 and lse +inf.  The default
       (0) leaves masking to maskType.  Sliding-window attention is the band
       with nextTokens = 0. */
    int32_t sparseMode;
    int64_t preTokens;
    int64_t nextTokens;
    /* kernel choice, a fia_path value (0, the default, is automatic). */
    int32_t path;
} fia_ext;

typedef struct fia_op fia_op;

/*
 * Phase 1 (ATB AtbSelfAttentionPrefixEncoderGetWorkspaceSize; the aclnn
 * ...GetWorkspaceSize call, the phase in which the V4/V3 pages check the inputs).
 *
 *  query        [nTokens, headNum, headSize] or [nTokens, headNum*headSize], f16|bf16.
 *               The new tokens of all sequences, concatenated in batch order.
 *  key, value   [numBlocks, blockSize, kvHeadNum, headSize] or
 *               [numBlocks, blockSize, kvHeadNum*headSize]; the query's dtype, or
 *               FIA_I8 with ext->kScale/vScale.  Same shape.
 *  blockTables  [batch, maxBlockNum] int32, device.  maxBlockNum must cover
 *               ceil(kvSeqLen[b] / blockSize) for every b.
 *  seqLen       host int32[batch]: new tokens per sequence; sum == nTokens.
 *  kvSeqLen     host int32[batch]: cached tokens per sequence INCLUDING the new
 *               ones (the new tokens' K/V are already in the cache); new token
 *               i of sequence b sits at position qpos = kvSeqLen[b]-seqLen[b]+i.
 *               seqLen[b] <= kvSeqLen[b] unless kvSeqLen[b] == 0 (rows with no
 *               keys: out 0, lse +inf).
 *  batch        number of sequences, >= 0.
 *  slopes       [headNum] f32 device, required for FIA_MASK_ALIBI, else NULL.
 *  maskType     FIA_MASK_NONE | FIA_MASK_ALIBI | FIA_MASK_CAUSAL.
 *  headNum      > 0;  kvHeadNum > 0 and headNum % kvHeadNum == 0; query head h
 *               reads KV head h / (headNum / kvHeadNum).
 *  qkScale      multiplies Q K^T before the bias is added (PrefixEncoder
 *               parameter table, qkScale row: the scale applies to the product).
 *  ext          optional extensions (see fia_ext), may be NULL.
 *  attnOut      [nTokens, headNum, headSize] (or 2-D), the query's dtype.
 *  workspaceSize  out: bytes of device workspace fia_run needs (0 if none).
 *  op           out: the planned operation; free with fia_op_destroy.
 *
 * Supported build limits: headSize in {64, 128} (128 with an int8 cache);
 * blockSize a multiple of 16, 16 <= blockSize <= 256; headNum <= 1024.
 * Everything else the pages allow returns FIA_ERR_UNSUPPORTED.  With an int8
 * cache on the tensor-core path (fia_path, below) the products run in f16:
 * q * kScale (per-channel keys), the cache values plus their offsets, and
 * per-token dequantised values must lie within f16 range (|v| < 65504).
 * nTokens == 0 returns FIA_OK with workspaceSize 0 and an op whose run is a no-op.
 */
FIA_API fia_status fia_get_workspace_size(const fia_tensor *query, const fia_tensor *key,
                                  const fia_tensor *value, const fia_tensor *blockTables,
                                  const int32_t *seqLen, const int32_t *kvSeqLen, int32_t batch,
                                  const fia_tensor *slopes, int32_t maskType, int32_t headNum,
                                  int32_t kvHeadNum, float qkScale, const fia_ext *ext,
                                  fia_tensor *attnOut, uint64_t *workspaceSize, fia_op **op);

/*
 * Phase 2 (ATB AtbSelfAttentionPrefixEncoder; aclnn second-phase call).
 *  workspace      device buffer of at least workspaceSize bytes, 256-byte aligned
 *                 (may be NULL only when workspaceSize was 0).  Its contents
 *                 are scratch: fia_run overwrites them.
 *  stream         a cudaStream_t (0 = legacy default stream), passed as void*.
 * Returns FIA_ERR_WORKSPACE for a NULL/misaligned/too-small workspace,
 * FIA_ERR_PARAM when the current device is not the op's, and FIA_ERR_CUDA when
 * a copy or launch fails (the op stays usable).
 */
FIA_API fia_status fia_run(void *workspace, uint64_t workspaceSize, fia_op *op, void *stream);

/* Frees the op (host memory only).  NULL is a no-op. */
FIA_API void fia_op_destroy(fia_op *op);

/* Static, human-readable text for a status code. */
FIA_API const char *fia_status_string(fia_status s);

/*
 * Measurement hook: when both events are non-NULL, fia_run records `start`
 * immediately before its main attention kernel and `stop` immediately after
 * its last kernel, on the run's stream, so that cudaEventElapsedTime gives the
 * device time of the kernels alone (the plan upload is excluded).  Pass NULLs
 * to switch it off.  Events are cudaEvent_t handles passed as void*, owned by
 * the caller.
 */
FIA_API fia_status fia_op_set_timing_events(fia_op *op, void *start, void *stop);

/*
 * Introspection of the plan phase 1 chose (for tests and reports).
 *   path            0 = no-op, 1 = decode (split-KV + combine), 2 = prefill (tcgen05)
 *   kernels_per_run number of kernel launches one fia_run makes
 *   work_items      decode: split units; prefill: (q-tile, head) items
 *   grid            CTAs of the main kernel
 *   (NULL op or info -> FIA_ERR_NULLPTR)
 */
typedef struct {
    int32_t path;
    int32_t kernels_per_run;
    int64_t work_items;
    int32_t grid;
    int32_t split_tokens;     /* decode: keys per split unit (0 otherwise)            */
    int64_t error_word_offset;/* byte offset in the workspace of a uint32 that a kernel
                                 sets non-zero when a bounded internal wait runs out;
                                 fia_run clears it                                     */
} fia_plan_info;

FIA_API fia_status fia_op_get_plan_info(const fia_op *op, fia_plan_info *info);

/*
 * Failure detection (V3 long-sequence restriction: an over-long run ends in a
 * device time-out error; here every internal wait of the kernels is bounded
 * instead).  Each wait on an on-chip barrier gives up after a time limit
 * (default 2 s); the kernel then sets the error word (error_word_offset above;
 * bits 8.. name the wait site, bit 0 = time-out), records up to 31 trail
 * entries after it, lets every role of the CTA leave, waits for its copies and
 * MMAs still in flight, releases its resources and returns.  The run's output
 * is then undefined, and the device stays usable.
 *   wait_limit_ns  new limit for this op's runs (0 restores the default).
 *   stall          test hook, 0 or 1: with 1, one role of every CTA first waits
 *                  on a barrier that nothing signals, so that the time-out path
 *                  runs and its report can be checked.  Never set it in service.
 * FIA_ERR_NULLPTR for a NULL op, FIA_ERR_PARAM for another stall value.
 */
FIA_API fia_status fia_op_set_wait_limit(fia_op *op, uint64_t wait_limit_ns, int32_t stall);

/*
 * Decode without a caller workspace (no counterpart in the pages: the aclnn and
 * ATB interfaces always take a caller-allocated workspace).
 *
 * For callers that cannot allocate device memory when they run attention --
 * an engine whose device memory is all handed out by its own pool at start-up,
 * or a runtime that forbids cudaMalloc/cudaFree on its serving path -- this runs
 * a decode-path op (split-KV decode + combine; fia_op_get_plan_info path == 1)
 * with its scratch in a fixed array inside libfia.so instead of the `workspace`
 * argument of fia_run.  Inputs and outputs are still the caller's tensors given
 * to fia_get_workspace_size.  Nothing here allocates: no cudaMalloc, no
 * cudaFree, no allocating library call.
 *
 *  - The array is FIA_STATIC_WORKSPACE_BYTES (32 MiB) per device.  Every GPU
 *    that loads the library holds it until the process exits.
 *  - An op whose workspaceSize exceeds it gets FIA_ERR_WORKSPACE; a prefill op
 *    gets FIA_ERR_UNSUPPORTED; a no-op op returns FIA_OK.  Nothing is launched
 *    in those cases.
 *  - Call it with the op's device current (FIA_ERR_PARAM otherwise).  The first
 *    call on a device looks up the array's device address
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *    A failed lookup returns FIA_ERR_CUDA.
 *  - All calls on a device share the one array, which keeps the last call's
 *    contents.  Calls that overlap on the GPU (two streams, or two host threads
 *    without ordering) race on it: serialise them.
 *  - Asynchronous on `stream` (a cudaStream_t passed as void*), like fia_run.
 *    Timing events set with fia_op_set_timing_events are recorded around its
 *    kernels as for fia_run.
 *  - The kernels' error word (see fia_op_set_wait_limit) lives in the array:
 *    read it with fia_decode_static_error_word.
 */
#define FIA_STATIC_WORKSPACE_BYTES (32u * 1024u * 1024u)
FIA_API fia_status fia_decode_run_static(fia_op *op, void *stream);

/*
 * The error word of the last fia_decode_run_static call of this op's shape on
 * the op's device (0 = every internal wait completed).  Copies 4 bytes out of
 * the library's array with cudaMemcpyFromSymbol, which waits for the device
 * to finish its queued work.  *word is 0 for a no-op op.  FIA_ERR_UNSUPPORTED
 * for a prefill op, FIA_ERR_PARAM when another device is current,
 * FIA_ERR_CUDA when the copy fails.
 */
FIA_API fia_status fia_decode_static_error_word(const fia_op *op, uint32_t *word);

#ifdef __cplusplus
}
#endif

#endif /* FIA_H */
