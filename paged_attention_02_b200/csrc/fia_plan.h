// fia_plan.h -- launch parameters shared by the host planner and the kernels.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace fia {

// Per-sequence facts, uploaded to the workspace by fia_run.
struct SeqInfo {
    int32_t cu_q;    // first token of the sequence inside query / attnOut
    int32_t qlen;    // seqLen[b]
    int32_t kvlen;   // kvSeqLen[b]
    int32_t pad;
};

// Decode work unit: one (sequence, kv head, row chunk, key range) split.
// Rows are the seqLen * g (new token, head-in-group) pairs of the group,
// row n = token * g + head-in-group; a unit takes rows r0 .. r0 + 15.
struct DecodeUnit {
    int32_t b, kvh, t_begin, t_end;
    int32_t slot;    // partial-result slot (logical split order within its chunk)
    int32_t r0;      // first row of the chunk
    int32_t pad[2];
};

// Decode combine item: the splits of one (sequence, kv head, row chunk).
struct CombineItem {
    int32_t slot0, nsplit, b, kvh;
    int32_t r0;      // first row of the chunk
    int32_t pad[3];
};

// Prefill work item: a pair of 128-new-token tiles of one sequence that read
// the same KV head, processed together by one CTA (they share every K/V tile).
// Tile 0 needs no more key tiles than tile 1; h[0] < 0 when tile 0 is absent.
struct PrefillItem {
    int32_t b, kvh;
    int32_t q0[2];   // first new token of each tile within the sequence
    int32_t h[2];    // query head of each tile
    int32_t pad[2];
};

constexpr int kDecodeRows = 16;      // rows (new token x head-in-group) per decode unit
constexpr int kDecodeMaxChunks = 8;  // row chunks per (sequence, KV head) on the decode path
constexpr int kDecodeTile = 64;      // keys per decode pipeline stage
constexpr int kPrefillBM = 128;      // new tokens per prefill item
constexpr int kPrefillBN = 128;      // keys per prefill tile

struct CommonArgs {
    const void *q;          // [nTokens, H, D]
    void *out;              // [nTokens, H, D]
    float *lse;             // [nTokens, H] or null
    const int32_t *bt;      // [B, bt_stride]
    const SeqInfo *seq;     // workspace
    const float *slopes;    // [H] (mask 3) or null
    const void *pse;        // [B, H, pse_q, pse_kv] or null
    const float *sink;      // [H] or null
    uint32_t *err;          // workspace error word
    int64_t pse_q, pse_kv;
    int32_t bt_stride;
    int32_t H, KVH, g, D, bs, box_rows;
    int32_t mask_type;
    int32_t pse_vec;        // pse rows 16-byte aligned (vector loads allowed)
    int32_t pse_tma;        // prefill: pse boxes fetched by TMA (tensor map tp)
    int32_t kv_layout;      // 0: [blocks, bs, KVH, D]; 1: [blocks, KVH, bs, D]
    int32_t band;           // band mask: keys qpos - pre .. qpos + next
    int32_t pre, next;      // band limits (clamped to +-2^30)
    int32_t chunk_rows;     // decode: rows per unit chunk (16, or 8 for int8 past 16 rows)
    float scale_log2;       // qkScale * log2(e)
    // Failure detection: every bounded wait gives up after wait_ns.  With
    // stall set (a test hook), one role first waits on a barrier that nothing
    // signals, so the time-out exit runs and reports through the error word.
    uint64_t wait_ns;
    int32_t stall;
};

// TMA coordinates (y, z) of cache row `off` of block `blk`, KV head kvh, in
// the K/V tensor maps: {D, KVH, blocks*bs} for layout 0, {D, bs, blocks*KVH}
// for layout 1 (the box is one head x rows, or rows x one head).
__device__ __forceinline__ void kv_box_yz(const CommonArgs &c, int kvh, int blk, int off, int &y,
                                          int &z) {
    if (c.kv_layout) {
        y = off;
        z = blk * c.KVH + kvh;
    } else {
        y = kvh;
        z = blk * c.bs + off;
    }
}

struct DecodeArgs {
    CommonArgs c;
    const DecodeUnit *units;
    float *part_o;          // [slots][16][D]
    float2 *part_ml;        // [slots][16] (m in log2 units, l)
    const float *k_scale, *k_offset;   // int8 only
    const float *v_scale, *v_offset;   // int8 only (used here in per-token mode)
    int64_t k_tok_stride, v_tok_stride;   // per-token mode: row stride S of [B, S]
    int32_t k_mode, v_mode;  // int8 dequant: 0 per (KV head, channel), 1 per (b, token)
    int32_t n_units;
    int32_t max_rows;       // max over sequences of seqLen * g (<= kDecodeRows)
    int32_t direct;         // every item has one split: units write the output (no combine)
};

struct CombineArgs {
    CommonArgs c;
    const CombineItem *items;
    const float *part_o;
    const float2 *part_ml;
    const float *v_scale, *v_offset;   // int8 only
    int32_t v_mode;         // int8: 1 = per-token V, already applied in the partials
    int32_t n_items;
};

struct PrefillArgs {
    CommonArgs c;
    // Plan location: either the workspace (device pointer `plan`) or the
    // kernel's inline plan parameter; offsets are bytes from the plan start.
    const uint8_t *plan;
    int32_t off_seq, off_cta, off_items;
    // int8 cache: K and V tiles are dequantised, (x + offset) * scale, into
    // the query dtype in shared memory before the MMAs read them
    const float *k_scale, *k_offset;   // per channel [KVH, D] or per token [B, S]
    const float *v_scale, *v_offset;
    int64_t k_tok_stride, v_tok_stride;   // per-token mode: row stride S of [B, S]
    int32_t k_mode, v_mode;  // 0 per (KV head, channel), 1 per (b, token)
};

// A plan of at most this many bytes travels as a kernel parameter (no
// host-to-device copy per run).
constexpr int kInlinePlanBytes = 24576;
template <int N> struct PlanBytes {
    uint8_t b[N];
};

// Kernel launchers (defined in the .cu files).
cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap &tk, const CUtensorMap &tv,
                          int q_dtype, bool kv_int8, int grid, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs &a, int q_dtype, bool kv_int8, int grid,
                           cudaStream_t s);
// inline_plan: nullptr (plan in the workspace) or kInlinePlanBytes of host data.
// tp: pse tensor map (used when a.c.pse_tma).
cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &tq, const CUtensorMap &tk,
                           const CUtensorMap &tv, const CUtensorMap &tp, int q_dtype, bool kv_int8,
                           int grid, const uint8_t *inline_plan, cudaStream_t s);

}  // namespace fia
