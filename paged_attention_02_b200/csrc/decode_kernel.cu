// decode_kernel.cu -- split-KV paged decode attention for sm_100a.
//
// Decode (Q_S = 1, aclnnFusedInferAttentionScoreV3 "When Q_S is 1" section;
// also the few-token MTP case) is bound by HBM: every cached K/V row of the
// sequence is read once per KV head and reused by all g = headNum/kvHeadNum
// query heads of its group.  The work is split along the key axis (V3 advises
// splitting S for long sequences), each split writes an unnormalised partial
// (O, m, l), and a second kernel merges the splits with the lse rule of the
// V3 "lse" bullet (max, rescaled exponent sums, log of the sum added back).
//
// Kernel 1 (one CTA per split unit (b, kvh, 16-row chunk, [t0, t1))).  K/V rows of the unit
// stream through a ring of shared-memory tiles (64 keys each) filled by TMA:
// one 3-D box per (block run, 128-byte column group), the physical row coming
// from the block table, so every cached byte is fetched once, 128-byte
// swizzled.  4 warps split each tile 16 keys apiece and run m16n8k16
// tensor-core MMAs; warps merge their (m, l, O) in shared memory and the CTA
// writes one partial per unit.
//   * fia_decode_kernel (fp16/bf16 cache): the g*qlen query rows of the
//     group form the 16-row A operand; S = Q K^T (keys as N), online softmax
//     in fp32 on the accumulator fragments, O += P V with P from registers.
//   * fia_decode_i8_kernel (int8 cache): keys are the 16-row A operand and
//     the query rows the N = 8 columns (S^T = K Q'^T, O^T = V^T P^T), so no
//     MMA row is padding.  Bytes are widened to f16 in registers by placing
//     each byte (+128) under the f16 exponent pattern for 1024, i.e. the
//     exact value 1152 + x; the 1152 bias is removed afterwards (for K from
//     the per-row constant, for V through a per-row sum of P from one extra
//     MMA against ones).  The per-channel K scale is folded into q (with a
//     power-of-two range fix), the K offset becomes one additive constant per
//     row, and the V scale/offset are applied once in the combine.  A fifth
//     warp only requests tiles: a compute warp issuing the refills carried
//     about a thousand cycles of barrier and TMA issue per tile (clock
//     stamps) and, being the last to finish each tile, set every warp's pace.
// Kernel 2, fia_combine_kernel: one CTA per (b, kvh, row); merges the unit
//   partials in fixed logical order (deterministic), adds the learnable sink
//   to the denominator, applies int8 V dequantisation, writes out and lse.
//   When every (b, kvh, chunk) has a single split the units apply the same
//   rules themselves (finish_unit) and this kernel is not launched.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "fia_device.cuh"
#include "fia_plan.h"

namespace fia {

// The last step of a decode unit, once its 4 warps' (m, l, O) sit in shared
// memory (ow [4][16][D], mlw [4][16]): merge them per row, then either write
// the unit's partial for the combine kernel or, when every (sequence, KV
// head, chunk) has a single split (a.direct), finish the rows here with the
// combine's rules (sink in the denominator, int8 per-channel V, lse) and
// save the combine launch.
template <typename T, int D, bool INT8>
__device__ __forceinline__ void finish_unit(const DecodeArgs &a, const DecodeUnit &u,
                                            const SeqInfo &si, int R, const float *ow,
                                            const float2 *mlw) {
    const int g = a.c.g;
    float *po = a.part_o + (int64_t)u.slot * kDecodeRows * D;
    float2 *pml = a.part_ml + (int64_t)u.slot * kDecodeRows;
    for (int idx = threadIdx.x; idx < R * D; idx += blockDim.x) {
        const int row = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, mlw[w * kDecodeRows + row].x);
        float acc = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float2 ml = mlw[w * kDecodeRows + row];
                const float f = ex2(ml.x - M);
                acc = fmaf(ow[(w * kDecodeRows + row) * D + d], f, acc);
                L = fmaf(ml.y, f, L);
            }
        }
        if (!a.direct) {
            po[row * D + d] = acc;
            if (d == 0) pml[row] = make_float2(M, L);
            continue;
        }
        const int n = u.r0 + row;                  // row of the group
        const int head = u.kvh * g + n % g;
        const int64_t o_idx = (int64_t)(si.cu_q + n / g) * a.c.H + head;
        float val = 0.f, lse = INFINITY;
        if (M != -INFINITY) {
            const float sink2 = a.c.sink ? a.c.sink[head] * kLog2e : -INFINITY;
            const float M2 = fmaxf(M, sink2);
            const float f = ex2(M - M2);
            L *= f;
            acc *= f;
            const float Lt = L + (a.c.sink ? ex2(sink2 - M2) : 0.f);
            if constexpr (INT8) {
                if (!a.v_mode) {      // per-channel V (per-token V is in acc already)
                    const float vs = a.v_scale[u.kvh * D + d];
                    const float vo = a.v_offset ? a.v_offset[u.kvh * D + d] : 0.f;
                    acc = vs * fmaf(vo, L, acc);
                }
            }
            val = acc / Lt;
            lse = (M2 + log2f(Lt)) * kLn2;
        }
        T *out = reinterpret_cast<T *>(a.c.out);
        if constexpr (MmaType<T>::bf16) out[o_idx * D + d] = __float2bfloat16_rn(val);
        else out[o_idx * D + d] = __float2half_rn(val);
        if (d == 0 && a.c.lse) a.c.lse[o_idx] = lse;
    }
}

template <int D>
struct DecodeCfg {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kHalves = kRowBytes / 128;               // 128-byte column groups
    static constexpr int kTileBytes = kDecodeTile * kRowBytes;    // one of K or V
    static constexpr int kStages = (2 * kTileBytes >= 32768) ? 3 : 4;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kMergeBytes = 4 * kDecodeRows * D * 4 + 4 * kDecodeRows * 8;
    static constexpr int kDataBytes =
        (kStages * kStageBytes > kMergeBytes) ? kStages * kStageBytes : kMergeBytes;
    // full[S], empty[S], one barrier nothing signals (test hook), abort flag
    static constexpr int kBarBytes = ((2 * kStages + 1) * 8 + 4 + 15) & ~15;
    static constexpr int kSmem = 1024 /*align slack*/ + kDataBytes + kBarBytes;
    static_assert(kRowBytes % 128 == 0, "row must be a whole number of 128-byte groups");
};

struct DecodeI8Cfg;

template <typename T, int D>
__global__ void __launch_bounds__(128, 2)
fia_decode_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv) {
    using Cfg = DecodeCfg<D>;
    constexpr int STAGES = Cfg::kStages;
    constexpr int KT = D / 16;           // k-steps of the QK^T MMA
    constexpr bool MMA_BF16 = MmaType<T>::bf16;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kDataBytes);
    uint64_t *empty = full + STAGES;
    uint64_t *never = empty + STAGES;       // test hook: nothing arrives on it
    volatile int *abort_flag = reinterpret_cast<volatile int *>(never + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int r = lane >> 2;       // fragment row group
    const int c = lane & 3;        // fragment column pair

    const DecodeUnit u = a.units[blockIdx.x];
    const SeqInfo si = a.c.seq[u.b];
    const int g = a.c.g;
    const int R = min(a.c.chunk_rows, si.qlen * g - u.r0);   // rows of this unit's chunk
    const int n_tiles = (u.t_end - u.t_begin + kDecodeTile - 1) / kDecodeTile;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        mbar_init(never, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
    }
    __syncthreads();

    const int32_t *bt_row = a.c.bt + (int64_t)u.b * a.c.bt_stride;
    auto issue = [&](int j) {
        const int s = j % STAGES;
        const int t0 = u.t_begin + j * kDecodeTile;
        const int t1 = min(t0 + kDecodeTile, u.t_end);
        const int br = a.c.box_rows;
        const int nbox = (t1 - t0 + br - 1) / br;
        uint8_t *kst = smem + s * Cfg::kStageBytes;
        uint8_t *vst = kst + Cfg::kTileBytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(nbox * br * 128 * Cfg::kHalves * 2));
        for (int bi = 0; bi < nbox; ++bi) {
            const int t = t0 + bi * br;
            int y, z;
            kv_box_yz(a.c, u.kvh, bt_row[t / a.c.bs], t % a.c.bs, y, z);
            for (int hv = 0; hv < Cfg::kHalves; ++hv) {
                const int off = hv * kDecodeTile * 128 + bi * br * 128;
                const int col = hv * 64;
                tma_load_3d(kst + off, &tk, &full[s], col, y, z);
                tma_load_3d(vst + off, &tv, &full[s], col, y, z);
            }
        }
    };
    int n_issued = 0;      // tiles requested (thread 0)
    if (tid == 0) {
        for (int j = 0; j < STAGES && j < n_tiles; ++j) issue(j);
        n_issued = min(STAGES, n_tiles);
    }
    // Test hook: every warp first waits on a barrier nothing signals; the
    // bounded wait gives up, and the CTA takes the error exit below with its
    // first tiles' copies still in flight.
    int n_run = n_tiles;
    if (a.c.stall) {
        const bool got = mbar_wait(never, 0, abort_flag, a.c.err, 3, a.c.wait_ns);
        if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0) fail_trail(a.c.err, 3, (uint32_t)u.b, (uint32_t)u.kvh, 0u, never);
            n_run = 0;
        }
    }

    // ---- per-row constants and the Q operand (rows ra = r, rb = r + 8) ----
    const int ra = r, rb = r + 8;
    int head_a = 0, head_b = 0, qi_a = 0, qi_b = 0;
    const bool va = ra < R, vb = rb < R;
    if (va) { qi_a = (u.r0 + ra) / g; head_a = u.kvh * g + (u.r0 + ra) % g; }
    if (vb) { qi_b = (u.r0 + rb) / g; head_b = u.kvh * g + (u.r0 + rb) % g; }
    const int qpos_a = si.kvlen - si.qlen + qi_a;
    const int qpos_b = si.kvlen - si.qlen + qi_b;
    const T *qp = reinterpret_cast<const T *>(a.c.q);
    const T *qa_ptr = qp + ((int64_t)(si.cu_q + qi_a) * a.c.H + head_a) * D;
    const T *qb_ptr = qp + ((int64_t)(si.cu_q + qi_b) * a.c.H + head_b) * D;

    uint32_t qf[KT][4];
    const float sc_a = a.c.scale_log2, sc_b = a.c.scale_log2;   // multiplies the raw accumulator
    const float add_a = 0.f, add_b = 0.f;                       // per-row additive term (log2 units)
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
        const int d0 = kk * 16 + 2 * c;
        qf[kk][0] = va ? *reinterpret_cast<const uint32_t *>(qa_ptr + d0) : 0u;
        qf[kk][1] = vb ? *reinterpret_cast<const uint32_t *>(qb_ptr + d0) : 0u;
        qf[kk][2] = va ? *reinterpret_cast<const uint32_t *>(qa_ptr + d0 + 8) : 0u;
        qf[kk][3] = vb ? *reinterpret_cast<const uint32_t *>(qb_ptr + d0 + 8) : 0u;
    }
    const bool causal = (a.c.mask_type == 9 || a.c.mask_type == 3);
    const bool alibi = a.c.mask_type == 3;
    const float slope_a = (alibi && va) ? a.c.slopes[head_a] * kLog2e : 0.f;
    const float slope_b = (alibi && vb) ? a.c.slopes[head_b] * kLog2e : 0.f;
    const T *pse_a = nullptr, *pse_b = nullptr;
    if (a.c.pse) {
        const T *pb = reinterpret_cast<const T *>(a.c.pse);
        if (va) pse_a = pb + (((int64_t)u.b * a.c.H + head_a) * a.c.pse_q + qi_a) * a.c.pse_kv;
        if (vb) pse_b = pb + (((int64_t)u.b * a.c.H + head_b) * a.c.pse_q + qi_b) * a.c.pse_kv;
    }

    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    float o[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

    bool ok = true;
    for (int j = 0; j < n_run; ++j) {
        const int s = j % STAGES;
        // every lane waits; the warp leaves together if any lane gave up
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (j / STAGES) & 1, abort_flag, a.c.err, 1,
                                               a.c.wait_ns))) {
            ok = false;
            break;
        }
        __syncwarp();      // ldmatrix / mma.sync below are warp-collective (.aligned)
        const uint32_t kst = smem_u32(smem + s * Cfg::kStageBytes);
        const uint32_t vst = kst + Cfg::kTileBytes;
        const int tw = u.t_begin + j * kDecodeTile + warp * 16;   // first key of this warp

        // ---- S = Q K^T over this warp's 16 keys ----
        float sacc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
        {
            const int mi = lane >> 3;
            const int tok = warp * 16 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) {
                const int chunk = 2 * kk + (mi & 1);
                const uint32_t addr = kst + (chunk >> 3) * (kDecodeTile * 128) + swz128(tok, chunk & 7);
                uint32_t b00, b01, b10, b11;
                ldsm_x4(addr, b00, b01, b10, b11);
                mma_16816<MMA_BF16>(sacc[0], qf[kk], b00, b01);
                mma_16816<MMA_BF16>(sacc[1], qf[kk], b10, b11);
            }
        }

        // ---- scores, masks, online softmax ----
        float sv[2][4];
        float mx_a = -INFINITY, mx_b = -INFINITY;
        // Interior tile without bias: every key of the 16 is visible to every
        // row (rows past R only carry zeros and are never written out).
        const bool simple = !alibi && !a.c.pse && (tw + 16 <= u.t_end) &&
                            (!causal || tw + 15 <= si.kvlen - si.qlen) &&
                            (!a.c.band || (tw >= si.kvlen - 1 - a.c.pre &&
                                           tw + 15 <= si.kvlen - si.qlen + a.c.next));
        if (simple) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    sv[nt][e] = fmaf(sacc[nt][e], sc_a, add_a);
                    sv[nt][2 + e] = fmaf(sacc[nt][2 + e], sc_b, add_b);
                }
            mx_a = fmax3(fmax3(sv[0][0], sv[0][1], sv[1][0]), sv[1][1], -INFINITY);
            mx_b = fmax3(fmax3(sv[0][2], sv[0][3], sv[1][2]), sv[1][3], -INFINITY);
        } else {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = tw + nt * 8 + 2 * c + e;
                    const bool in = t < u.t_end;
                    float x = fmaf(sacc[nt][e], sc_a, add_a);
                    float y = fmaf(sacc[nt][2 + e], sc_b, add_b);
                    if (alibi) {
                        x = fmaf(slope_a, (float)(t - qpos_a), x);
                        y = fmaf(slope_b, (float)(t - qpos_b), y);
                    }
                    if (pse_a && in) x = fmaf(to_f32<T>(pse_a[t]), kLog2e, x);
                    if (pse_b && in) y = fmaf(to_f32<T>(pse_b[t]), kLog2e, y);
                    const bool ka = in && va && !(causal && t > qpos_a) &&
                                    !(a.c.band && (t < qpos_a - a.c.pre || t > qpos_a + a.c.next));
                    const bool kb = in && vb && !(causal && t > qpos_b) &&
                                    !(a.c.band && (t < qpos_b - a.c.pre || t > qpos_b + a.c.next));
                    sv[nt][e] = ka ? x : -INFINITY;
                    sv[nt][2 + e] = kb ? y : -INFINITY;
                    mx_a = fmaxf(mx_a, sv[nt][e]);
                    mx_b = fmaxf(mx_b, sv[nt][2 + e]);
                }
            }
            __syncwarp();
        }
#pragma unroll
        for (int x = 1; x <= 2; x <<= 1) {
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, x));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, x));
        }
        // Running max raised only when it grows by more than 2^8 (P stays
        // <= 2^8, fine for f16/bf16); O, l and m stay mutually consistent.
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const bool up_a = mn_a > m_a + 8.0f, up_b = mn_b > m_b + 8.0f;
        float al_a = 1.0f, al_b = 1.0f;
        if (up_a) { al_a = ex2(m_a - mn_a); m_a = mn_a; }
        if (up_b) { al_b = ex2(m_b - mn_b); m_b = mn_b; }
        const float mu_a = (m_a == -INFINITY) ? 0.f : m_a;
        const float mu_b = (m_b == -INFINITY) ? 0.f : m_b;
        float ps_a = 0.f, ps_b = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                sv[nt][e] = ex2(sv[nt][e] - mu_a);
                sv[nt][2 + e] = ex2(sv[nt][2 + e] - mu_b);
                ps_a += sv[nt][e];
                ps_b += sv[nt][2 + e];
            }
        }
        l_a = fmaf(l_a, al_a, ps_a);
        l_b = fmaf(l_b, al_b, ps_b);
        if (__any_sync(0xffffffffu, up_a || up_b)) {
#pragma unroll
            for (int jj = 0; jj < D / 8; ++jj) {
                o[jj][0] *= al_a; o[jj][1] *= al_a;
                o[jj][2] *= al_b; o[jj][3] *= al_b;
            }
        }
        uint32_t pa[4];
        pa[0] = pack2<T>(sv[0][0], sv[0][1]);
        pa[1] = pack2<T>(sv[0][2], sv[0][3]);
        pa[2] = pack2<T>(sv[1][0], sv[1][1]);
        pa[3] = pack2<T>(sv[1][2], sv[1][3]);

        // ---- O += P V ----  (V rows past the unit's end are zeroed: P is 0
        // there but the slots may hold NaN garbage)
        const bool tail = (tw + 16 > u.t_end);
        {
            uint32_t mk0 = 0xffffffffu, mk1 = 0xffffffffu;
            if (tail) {
                const int t0 = tw + 2 * c;
                mk0 = (t0 < u.t_end ? 0x0000ffffu : 0u) | (t0 + 1 < u.t_end ? 0xffff0000u : 0u);
                mk1 = (t0 + 8 < u.t_end ? 0x0000ffffu : 0u) | (t0 + 9 < u.t_end ? 0xffff0000u : 0u);
            }
            const int mi = lane >> 3;
            const int tok = warp * 16 + (mi & 1) * 8 + (lane & 7);
            auto pv_tile = [&](auto masked) {
#pragma unroll
                for (int jj = 0; jj < D / 16; ++jj) {
                    const int chunk = 2 * jj + (mi >> 1);
                    const uint32_t addr = vst + (chunk >> 3) * (kDecodeTile * 128) + swz128(tok, chunk & 7);
                    uint32_t v0, v1, v2, v3;
                    ldsm_x4_t(addr, v0, v1, v2, v3);
                    if (decltype(masked)::value) { v0 &= mk0; v1 &= mk1; v2 &= mk0; v3 &= mk1; }
                    mma_16816<MMA_BF16>(o[2 * jj], pa, v0, v1);
                    mma_16816<MMA_BF16>(o[2 * jj + 1], pa, v2, v3);
                }
            };
            if (tail) pv_tile(std::true_type{});
            else pv_tile(std::false_type{});
        }

        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        bool stop = false;
        if (tid == 0 && j + STAGES < n_tiles) {
            if (mbar_wait(&empty[s], (j / STAGES) & 1, abort_flag, a.c.err, 2, a.c.wait_ns)) {
                issue(j + STAGES);
                ++n_issued;
            } else {
                stop = true;
            }
        }
        __syncwarp();
        // a failed wait ends the key loop for the whole warp at once (lane 0
        // alone leaving would strand its siblings at a warp barrier)
        if (__any_sync(0xffffffffu, stop)) { ok = false; break; }
    }
    (void)ok;

    // ---- merge the 4 warps' (m, l, O) and write this unit's partial ----
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, x);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, x);
    }
    __syncthreads();   // every warp is done with the stage buffers
    // Error exit (the flag is final here: no wait follows): the copies of the
    // last STAGES requested tiles may still be in flight; wait for them before
    // the buffers are reused below and before the CTA ends.  Earlier tiles'
    // copies completed before their stage was requested again.
    if (*abort_flag) {
        if (tid == 0)
            for (int j = max(0, n_issued - STAGES); j < n_issued; ++j)
                mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1);
        __syncthreads();
    }
    float *ow = reinterpret_cast<float *>(smem);                          // [4][16][D]
    float2 *mlw = reinterpret_cast<float2 *>(smem + 4 * kDecodeRows * D * 4);  // [4][16]
    float *oww = ow + warp * kDecodeRows * D;
#pragma unroll
    for (int jj = 0; jj < D / 8; ++jj) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int d = jj * 8 + 2 * c + e;
            oww[ra * D + d] = o[jj][e];
            oww[rb * D + d] = o[jj][2 + e];
        }
    }
    if (c == 0) {
        mlw[warp * kDecodeRows + ra] = make_float2(m_a, l_a);
        mlw[warp * kDecodeRows + rb] = make_float2(m_b, l_b);
    }
    __syncthreads();
    finish_unit<T, D, false>(a, u, si, R, ow, mlw);
}

// ---------------------------------------------------------------------------
// int8 KV decode with the keys as the MMA row dimension.
//
// S^T = K Q'^T and O^T = V^T P^T: the 16 keys of a warp are the 16-row A
// operand (widened from int8 in registers) and the query rows of the group
// (g heads x qlen tokens) are the N = 8 column tiles (NT of them).  No MMA row
// is padding, each (key, row) exponential is computed once, and the O^T
// accumulator is 32 floats per thread per column tile, so four CTAs fit an SM.
//   * K (A of S^T): key rows r and r + 8 of the warp; k-step kk = 4G + i
//     covers dims 64G + 16c + 4i + {0..3} for thread column c, so one 16-byte
//     shared load per key row brings four k-steps.  Q'^T (B) uses the same
//     dims for query row 8nt + r.
//   * P^T (B of O^T): the S^T accumulator packed to f16 and transposed in
//     registers with movmatrix (keys x rows -> rows x keys).
//   * V^T (A of O^T): M tile mt, row rho holds output dim
//     64 (rho >> 3) + 8 (rho & 7) + mt, so a thread's dims of one key row are
//     two runs of 8 contiguous bytes (two 8-byte shared loads).
// int8 decode: warps 0-3 compute, warp 4 (from thread kI8Producer) requests
// the tiles.  Four CTAs per SM for the per-channel single-column-tile kernel
// (96 registers), three for the others (their extra state spills at 96).
constexpr int kI8Producer = 128;
struct DecodeI8Cfg {
    static constexpr int D = 128;
    static constexpr int kTileBytes = kDecodeTile * D;          // one of K or V
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kStages = 3;
    static constexpr int kMergeBytes = 4 * kDecodeRows * D * 4 + 4 * kDecodeRows * 8;
    static constexpr int kDataBytes =
        (kStages * kStageBytes > kMergeBytes) ? kStages * kStageBytes : kMergeBytes;
    // full[S], empty[S], one barrier nothing signals (test hook), abort flag
    static constexpr int kBarBytes = ((2 * kStages + 1) * 8 + 4 + 15) & ~15;
    // per-token dequantisation parameters, per warp: [2 buffers][4 arrays:
    // K scale, K offset, V scale, V offset][16 keys] fp32, after the barriers
    static constexpr int kOffTok = kDataBytes + kBarBytes;
    static constexpr int kTokBytes = 4 * 2 * 4 * 16 * 4;
    static constexpr int kSmem = 1024 /*align slack*/ + kOffTok + kTokBytes;
};

template <typename T, int NT, bool KTOK, bool VTOK>
__global__ void __launch_bounds__(160, (NT == 1 && !KTOK && !VTOK) ? 4 : 3)
fia_decode_i8_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv) {
    using Cfg = DecodeI8Cfg;
    constexpr int D = Cfg::D;
    constexpr int STAGES = Cfg::kStages;
    constexpr int KT = D / 16;                 // k-steps of S^T
    constexpr int MT = D / 16;                 // M tiles of O^T
    constexpr uint32_t F = 0x64646464u;        // f16 exponent bytes of 1024
    static_assert(KT % 4 == 0, "keys are read 64 dims (4 k-steps) at a time");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kDataBytes);
    uint64_t *empty = full + STAGES;
    uint64_t *never = empty + STAGES;       // test hook: nothing arrives on it
    volatile int *abort_flag = reinterpret_cast<volatile int *>(never + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int r = lane >> 2;       // fragment row group
    const int c = lane & 3;        // fragment column pair

    const DecodeUnit u = a.units[blockIdx.x];
    const SeqInfo si = a.c.seq[u.b];
    const int g = a.c.g;
    const int R = min(a.c.chunk_rows, si.qlen * g - u.r0);   // rows of this unit's chunk
    const int n_tiles = (u.t_end - u.t_begin + kDecodeTile - 1) / kDecodeTile;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        mbar_init(never, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
    }
    __syncthreads();

    const int32_t *bt_row = a.c.bt + (int64_t)u.b * a.c.bt_stride;
    auto issue = [&](int j) {
        const int s = j % STAGES;
        const int t0 = u.t_begin + j * kDecodeTile;
        const int t1 = min(t0 + kDecodeTile, u.t_end);
        const int br = a.c.box_rows;
        const int nbox = (t1 - t0 + br - 1) / br;
        uint8_t *kst = smem + s * Cfg::kStageBytes;
        uint8_t *vst = kst + Cfg::kTileBytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(nbox * br * 128 * 2));
        for (int bi = 0; bi < nbox; ++bi) {
            const int t = t0 + bi * br;
            int y, z;
            kv_box_yz(a.c, u.kvh, bt_row[t / a.c.bs], t % a.c.bs, y, z);
            tma_load_3d(kst + bi * br * 128, &tk, &full[s], 0, y, z);
            tma_load_3d(vst + bi * br * 128, &tv, &full[s], 0, y, z);
        }
    };
    int n_issued = 0;      // tiles requested (producer thread)
    if (tid == kI8Producer) {
        for (int j = 0; j < STAGES && j < n_tiles; ++j) issue(j);
        n_issued = min(STAGES, n_tiles);
    }
    // Test hook: every warp first waits on a barrier nothing signals; the
    // bounded wait gives up, and the CTA takes the error exit below with its
    // first tiles' copies still in flight.
    int n_run = n_tiles;
    if (a.c.stall) {
        const bool got = mbar_wait(never, 0, abort_flag, a.c.err, 3, a.c.wait_ns);
        if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0) fail_trail(a.c.err, 3, (uint32_t)u.b, (uint32_t)u.kvh, 0u, never);
            n_run = 0;
        }
    }
    if (warp == 4) {
        // producer: refill each stage as soon as the four compute warps are
        // done with it.  A compute warp issuing the refills after its own
        // share of a tile carried about a thousand cycles of barrier and TMA
        // issue per tile (clock stamps), and its pace set every warp's data.
        if (lane == 0 && n_run > 0) {
            for (int j = 0; j + STAGES < n_tiles; ++j) {
                if (!mbar_wait(&empty[j % STAGES], (j / STAGES) & 1, abort_flag, a.c.err, 2,
                               a.c.wait_ns))
                    break;
                issue(j + STAGES);
                ++n_issued;
            }
        }
        __syncwarp();
        n_run = 0;
    }

    // ---- Q'^T fragments: this thread holds query row nb = 8nt + r ----
    // Per-channel K: q'_d = q_d * kScale_d, scaled per row by a power of two
    // so that max |q'| lands below 2^11 (inside f16 range); sc undoes it on
    // the accumulator.  add = qkScale * sum_d q_d sK_d oK_d (key offset) minus
    // 1152 * sum_d q'_d (the bias of the widened key bytes), in log2 units.
    // Per-token K (scale sK_t, offset oK_t per cached token): q' = q, and a
    // score is qkScale * sK_t * (sum_d q_d k_td + oK_t * sum_d q_d): sc and add
    // stay in raw units and qs = sum_d q_d; sK_t and oK_t join per key.
    constexpr bool ktok = KTOK, vtok = VTOK;     // per-token K / V (else per-channel)
    uint32_t qb[NT][KT][2];
    float sc_b[NT], add_b[NT], qs_b[NT];
    {
        const T *qp = reinterpret_cast<const T *>(a.c.q);
        const float *ks = ktok ? nullptr : a.k_scale + u.kvh * D;
        const float *ko = (!ktok && a.k_offset) ? a.k_offset + u.kvh * D : nullptr;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int nb = 8 * nt + r;
            const bool vr = nb < R;
            const int qi = vr ? (u.r0 + nb) / g : 0;
            const int head = vr ? u.kvh * g + (u.r0 + nb) % g : 0;
            const T *qrow = qp + ((int64_t)(si.cu_q + qi) * a.c.H + head) * D;
            float qv[KT][4];
            float mx = 0.f, cs = 0.f;
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int d = (kk >> 2) * 64 + 16 * c + 4 * (kk & 3) + e;
                    const float o = ktok ? 1.f : (ko ? ko[d] : 0.f);
                    qv[kk][e] = vr ? to_f32<T>(qrow[d]) * (ktok ? 1.f : ks[d]) : 0.f;
                    mx = fmaxf(mx, fabsf(qv[kk][e]));
                    cs = fmaf(qv[kk][e], o, cs);
                }
            }
#pragma unroll
            for (int x = 1; x <= 2; x <<= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
                cs += __shfl_xor_sync(0xffffffffu, cs, x);
            }
            int ex = 0;
            if (mx > 0.f) { frexpf(mx, &ex); ex = 11 - ex; }
            float sq = 0.f;
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) {
                qb[nt][kk][0] = pack2<__half>(ldexpf(qv[kk][0], ex), ldexpf(qv[kk][1], ex));
                qb[nt][kk][1] = pack2<__half>(ldexpf(qv[kk][2], ex), ldexpf(qv[kk][3], ex));
                const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&qb[nt][kk][0]));
                const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&qb[nt][kk][1]));
                sq += (f0.x + f0.y) + (f1.x + f1.y);
            }
#pragma unroll
            for (int x = 1; x <= 2; x <<= 1) sq += __shfl_xor_sync(0xffffffffu, sq, x);
            if (ktok) {
                sc_b[nt] = ldexpf(1.0f, -ex);
                add_b[nt] = -1152.0f * sq * sc_b[nt];
                qs_b[nt] = cs;
            } else {
                sc_b[nt] = ldexpf(a.c.scale_log2, -ex);
                add_b[nt] = cs * a.c.scale_log2 - 1152.0f * sq * sc_b[nt];
                qs_b[nt] = 0.f;
            }
        }
    }

    // ---- accumulator columns: this thread holds query rows 8nt + 2c + e ----
    const bool causal = (a.c.mask_type == 9 || a.c.mask_type == 3);
    const bool alibi = a.c.mask_type == 3;
    float sc[NT][2], add[NT][2], qs[NT][2], slope[NT][2];
    int qpos[NT][2];
    bool vrow[NT][2];
    const T *pse_row[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = 8 * nt + 2 * c + e;
            // the B-layout thread holding row n is lane 4 (2c + e) of the column tile
            sc[nt][e] = __shfl_sync(0xffffffffu, sc_b[nt], 4 * (2 * c + e));
            add[nt][e] = __shfl_sync(0xffffffffu, add_b[nt], 4 * (2 * c + e));
            qs[nt][e] = ktok ? __shfl_sync(0xffffffffu, qs_b[nt], 4 * (2 * c + e)) : 0.f;
            vrow[nt][e] = n < R;
            const int qi = vrow[nt][e] ? (u.r0 + n) / g : 0;
            const int head = vrow[nt][e] ? u.kvh * g + (u.r0 + n) % g : 0;
            qpos[nt][e] = si.kvlen - si.qlen + qi;
            slope[nt][e] = (alibi && vrow[nt][e]) ? a.c.slopes[head] * kLog2e : 0.f;
            pse_row[nt][e] = nullptr;
            if (a.c.pse && vrow[nt][e])
                pse_row[nt][e] = reinterpret_cast<const T *>(a.c.pse) +
                                 (((int64_t)u.b * a.c.H + head) * a.c.pse_q + qi) * a.c.pse_kv;
        }
    }

    float m[NT][2], l[NT][2];
    float o[NT][MT][4];
    float osum[NT][4];
    float voff[NT][2];      // per-token V: sum_t p_t sV_t oV_t per row
    // per-token scale / offset rows of this sequence
    const float *ksr = ktok ? a.k_scale + (int64_t)u.b * a.k_tok_stride : nullptr;
    const float *kor = (ktok && a.k_offset) ? a.k_offset + (int64_t)u.b * a.k_tok_stride : nullptr;
    const float *vsr = vtok ? a.v_scale + (int64_t)u.b * a.v_tok_stride : nullptr;
    const float *vor = (vtok && a.v_offset) ? a.v_offset + (int64_t)u.b * a.v_tok_stride : nullptr;
    // This warp's 16 keys of key tile jt: their per-token parameters are
    // copied into shared-memory buffer jt & 1 one tile ahead (lane L copies
    // array L >> 4 and array 2 + (L >> 4) for key L & 15), so their latency
    // hides behind the previous tile.  Keys past the unit's end and absent
    // offsets read as 0 (the key loop then needs no bounds tests: a zero V
    // scale keeps 0 * garbage out of P).  One commit group per call.
    float *tokbuf = reinterpret_cast<float *>(smem + Cfg::kOffTok) + warp * 128;
    auto tok_fetch = [&](int jt) {
        const int t = u.t_begin + jt * kDecodeTile + warp * 16 + (lane & 15);
        const float *s0 = (lane < 16) ? ksr : kor;
        const float *s1 = (lane < 16) ? vsr : vor;
        float *dst = tokbuf + (jt & 1) * 64;
        if (s0 && t < u.t_end) cp_async4(smem_u32(dst + lane), s0 + t);
        else dst[lane] = 0.f;
        if (s1 && t < u.t_end) cp_async4(smem_u32(dst + 32 + lane), s1 + t);
        else dst[32 + lane] = 0.f;
        cp_async_commit();
    };
    if constexpr (KTOK || VTOK) { if (warp < 4) tok_fetch(0); }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        voff[nt][0] = voff[nt][1] = 0.f;
        m[nt][0] = m[nt][1] = -INFINITY;
        l[nt][0] = l[nt][1] = 0.f;
        osum[nt][0] = osum[nt][1] = osum[nt][2] = osum[nt][3] = 0.f;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    }
    const uint32_t ones = 0x3C003C00u;          // f16x2 (1, 1)
    const uint32_t ones4[4] = {ones, ones, ones, ones};

    bool ok = true;
    for (int j = 0; j < n_run; ++j) {
        const int s = j % STAGES;
        // every lane waits; the warp leaves together if any lane gave up
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (j / STAGES) & 1, abort_flag, a.c.err, 1,
                                               a.c.wait_ns))) {
            ok = false;
            break;
        }
        const float *tok = tokbuf + (j & 1) * 64;
        if constexpr (KTOK || VTOK) {
            // buffer (j + 1) & 1 was last read in tile j - 1, before a __syncwarp
            if (j + 1 < n_tiles) tok_fetch(j + 1);
            else cp_async_commit();
            cp_async_wait<1>();            // this tile's group has landed
        }
        __syncwarp();      // movmatrix / mma.sync below are warp-collective (.aligned);
                           // also makes every lane's parameter copies visible
        const uint32_t kst = smem_u32(smem + s * Cfg::kStageBytes);
        const uint32_t vst = kst + Cfg::kTileBytes;
        const int tw = u.t_begin + j * kDecodeTile + warp * 16;   // first key of this warp

        // ---- S^T = K Q'^T over this warp's 16 keys ----
        float sacc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
        {
            const int ka = warp * 16 + r, kb = ka + 8;
#pragma unroll
            for (int G = 0; G < KT / 4; ++G) {
                uint32_t wa[4], wb[4];
                lds128(kst + swz128(ka, 4 * G + c), wa);
                lds128(kst + swz128(kb, 4 * G + c), wb);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    // bytes biased to 128 + k under the f16 exponent pattern:
                    // f16 values 1152 + k, exact (the bias is in add)
                    const uint32_t xa = wa[i] ^ 0x80808080u, xb = wb[i] ^ 0x80808080u;
                    const uint32_t A[4] = {prmt(xa, F, 0x4140u), prmt(xb, F, 0x4140u),
                                           prmt(xa, F, 0x4342u), prmt(xb, F, 0x4342u)};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816<false>(sacc[nt], A, qb[nt][4 * G + i][0], qb[nt][4 * G + i][1]);
                }
            }
        }

        // ---- scores, masks, online softmax (columns = query rows) ----
        // accumulator element q of column tile nt: key tw + r + 8 (q >> 1),
        // row 8nt + 2c + (q & 1)
        const bool simple = !alibi && !a.c.pse && (tw + 16 <= u.t_end) &&
                            (!causal || tw + 15 <= si.kvlen - si.qlen) &&
                            (!a.c.band || (tw >= si.kvlen - 1 - a.c.pre &&
                                           tw + 15 <= si.kvlen - si.qlen + a.c.next));
        float sv[NT][4];
        float mx[NT][2];
        // per-token K of this thread's keys tw + r and tw + r + 8 (keys past
        // the unit's end are masked below and never read)
        float kf[2] = {1.f, 1.f}, kof[2] = {0.f, 0.f};
        if constexpr (KTOK) {
#pragma unroll
            for (int hk = 0; hk < 2; ++hk) {
                kf[hk] = tok[r + 8 * hk] * a.c.scale_log2;
                kof[hk] = tok[16 + r + 8 * hk];
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = q & 1;
                float x = ktok ? fmaf(sacc[nt][q], sc[nt][e], fmaf(kof[q >> 1], qs[nt][e], add[nt][e])) *
                                     kf[q >> 1]
                               : fmaf(sacc[nt][q], sc[nt][e], add[nt][e]);
                if (!simple) {
                    const int t = tw + r + 8 * (q >> 1);
                    const bool in = t < u.t_end;
                    if (alibi) x = fmaf(slope[nt][e], (float)(t - qpos[nt][e]), x);
                    if (pse_row[nt][e] && in) x = fmaf(to_f32<T>(pse_row[nt][e][t]), kLog2e, x);
                    const bool keep = in && vrow[nt][e] && !(causal && t > qpos[nt][e]) &&
                                      !(a.c.band && (t < qpos[nt][e] - a.c.pre ||
                                                     t > qpos[nt][e] + a.c.next));
                    x = keep ? x : -INFINITY;
                }
                sv[nt][q] = x;
            }
            mx[nt][0] = fmaxf(sv[nt][0], sv[nt][2]);
            mx[nt][1] = fmaxf(sv[nt][1], sv[nt][3]);
        }
        if (!simple) __syncwarp();     // reconverge after the per-key pse loads
#pragma unroll
        for (int x = 4; x <= 16; x <<= 1)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mx[nt][0] = fmaxf(mx[nt][0], __shfl_xor_sync(0xffffffffu, mx[nt][0], x));
                mx[nt][1] = fmaxf(mx[nt][1], __shfl_xor_sync(0xffffffffu, mx[nt][1], x));
            }
        // Running max raised only when it grows by more than 2^8 (P stays
        // <= 2^8, fine for f16); O, l and m stay mutually consistent.
        bool up_any = false;
        float al[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float mn = fmaxf(m[nt][e], mx[nt][e]);
                al[nt][e] = 1.0f;
                if (mn > m[nt][e] + 8.0f) {
                    al[nt][e] = ex2(m[nt][e] - mn);
                    m[nt][e] = mn;
                    up_any = true;
                }
            }
        }
        // per-token V of this thread's keys: P is scaled by sV_t before it
        // meets the value bytes, and sum_t p_t sV_t oV_t is kept per row
        float vf[2] = {1.f, 1.f}, vof[2] = {0.f, 0.f};
        if constexpr (VTOK) {
#pragma unroll
            for (int hk = 0; hk < 2; ++hk) {
                vf[hk] = tok[32 + r + 8 * hk];
                vof[hk] = tok[48 + r + 8 * hk];
            }
        }
        __syncwarp();      // movmatrix and mma.sync below are .aligned
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float mu0 = (m[nt][0] == -INFINITY) ? 0.f : m[nt][0];
            const float mu1 = (m[nt][1] == -INFINITY) ? 0.f : m[nt][1];
            float p0 = ex2(sv[nt][0] - mu0), p1 = ex2(sv[nt][1] - mu1);
            float p2 = ex2(sv[nt][2] - mu0), p3 = ex2(sv[nt][3] - mu1);
            l[nt][0] = fmaf(l[nt][0], al[nt][0], p0 + p2);
            l[nt][1] = fmaf(l[nt][1], al[nt][1], p1 + p3);
            if constexpr (VTOK) {
                p0 *= vf[0]; p1 *= vf[0]; p2 *= vf[1]; p3 *= vf[1];
                voff[nt][0] = fmaf(voff[nt][0], al[nt][0], fmaf(p0, vof[0], p2 * vof[1]));
                voff[nt][1] = fmaf(voff[nt][1], al[nt][1], fmaf(p1, vof[0], p3 * vof[1]));
            }
            // P^T fragments: (keys x rows) f16 tiles transposed to (rows x keys)
            pb[nt][0] = movmatrix_trans(pack2<__half>(p0, p1));     // keys 2c, 2c+1
            pb[nt][1] = movmatrix_trans(pack2<__half>(p2, p3));     // keys 2c+8, 2c+9
        }
        if (__any_sync(0xffffffffu, up_any)) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    o[nt][mt][0] *= al[nt][0]; o[nt][mt][1] *= al[nt][1];
                    o[nt][mt][2] *= al[nt][0]; o[nt][mt][3] *= al[nt][1];
                }
                osum[nt][0] *= al[nt][0]; osum[nt][1] *= al[nt][1];
                osum[nt][2] *= al[nt][0]; osum[nt][3] *= al[nt][1];
            }
        }

        // ---- O^T += V^T P^T ----  (V rows past the unit's end are zeroed: P
        // is 0 there but the slots may hold NaN garbage)
        {
            const int k0 = warp * 16 + 2 * c;
            const int tg = tw + 2 * c;
            const bool tail = (tw + 16 > u.t_end);
            // dims 8r .. 8r+7 (rows rho = r) and 64 + 8r .. (rows rho = r + 8)
            const uint32_t lo_off = ((uint32_t)(r >> 1) << 4), hi_off = ((uint32_t)(4 + (r >> 1)) << 4);
            const uint32_t in8 = 8u * (uint32_t)(r & 1);
            uint2 vl[4], vh[4];     // key rows k0, k0+1, k0+8, k0+9
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                const int kr = k0 + (kq & 1) + 8 * (kq >> 1);
                const uint32_t rowb = vst + (uint32_t)kr * 128u;
                const uint32_t sw = (uint32_t)(kr & 7) << 4;
                vl[kq] = lds64(rowb + (lo_off ^ sw) + in8);
                vh[kq] = lds64(rowb + (hi_off ^ sw) + in8);
                if (tail && tg + (kq & 1) + 8 * (kq >> 1) >= u.t_end) {
                    vl[kq] = make_uint2(0u, 0u);
                    vh[kq] = make_uint2(0u, 0u);
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {           // M tiles 4h .. 4h+3
                const uint32_t a0 = h ? vl[0].y : vl[0].x, a1 = h ? vl[1].y : vl[1].x;
                const uint32_t b0 = h ? vh[0].y : vh[0].x, b1 = h ? vh[1].y : vh[1].x;
                const uint32_t c0 = h ? vl[2].y : vl[2].x, c1 = h ? vl[3].y : vl[3].x;
                const uint32_t d0 = h ? vh[2].y : vh[2].x, d1 = h ? vh[3].y : vh[3].x;
                // key pairs interleaved byte by byte, then biased (+128)
                const uint32_t xa01 = prmt(a0, a1, 0x5140u) ^ 0x80808080u;   // rho r, keys 2c/2c+1
                const uint32_t xa23 = prmt(a0, a1, 0x7362u) ^ 0x80808080u;
                const uint32_t xb01 = prmt(b0, b1, 0x5140u) ^ 0x80808080u;   // rho r+8
                const uint32_t xb23 = prmt(b0, b1, 0x7362u) ^ 0x80808080u;
                const uint32_t xc01 = prmt(c0, c1, 0x5140u) ^ 0x80808080u;   // rho r, keys 2c+8/+9
                const uint32_t xc23 = prmt(c0, c1, 0x7362u) ^ 0x80808080u;
                const uint32_t xd01 = prmt(d0, d1, 0x5140u) ^ 0x80808080u;   // rho r+8
                const uint32_t xd23 = prmt(d0, d1, 0x7362u) ^ 0x80808080u;
#pragma unroll
                for (int q = 0; q < 4; ++q) {       // M tile mt = 4h + q: byte q of each word
                    const uint32_t sel = (q & 1) ? 0x4342u : 0x4140u;
                    const uint32_t A[4] = {prmt((q < 2) ? xa01 : xa23, F, sel),
                                           prmt((q < 2) ? xb01 : xb23, F, sel),
                                           prmt((q < 2) ? xc01 : xc23, F, sel),
                                           prmt((q < 2) ? xd01 : xd23, F, sel)};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816<false>(o[nt][4 * h + q], A, pb[nt][0], pb[nt][1]);
                }
            }
            // sum_k p~ per row with the same rounding and accumulation as O
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_16816<false>(osum[nt], ones4, pb[nt][0], pb[nt][1]);
        }

        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    (void)ok;
    if constexpr (KTOK || VTOK) cp_async_wait<0>();   // no copy outlives the loop

    // ---- merge the 4 warps' (m, l, O) and write this unit's partial ----
#pragma unroll
    for (int x = 4; x <= 16; x <<= 1)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            l[nt][0] += __shfl_xor_sync(0xffffffffu, l[nt][0], x);
            l[nt][1] += __shfl_xor_sync(0xffffffffu, l[nt][1], x);
            if constexpr (VTOK) {
                voff[nt][0] += __shfl_xor_sync(0xffffffffu, voff[nt][0], x);
                voff[nt][1] += __shfl_xor_sync(0xffffffffu, voff[nt][1], x);
            }
        }
    __syncthreads();   // every warp is done with the stage buffers
    // Error exit (the flag is final here: no wait follows): the copies of the
    // last STAGES requested tiles may still be in flight; wait for them before
    // the buffers are reused below and before the CTA ends.  Earlier tiles'
    // copies completed before their stage was requested again.
    if (*abort_flag) {
        if (tid == kI8Producer)
            for (int j = max(0, n_issued - STAGES); j < n_issued; ++j)
                mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1);
        __syncthreads();
    }
    float *ow = reinterpret_cast<float *>(smem);                               // [4][16][D]
    float2 *mlw = reinterpret_cast<float2 *>(smem + 4 * kDecodeRows * D * 4);  // [4][16]
    float *oww = ow + warp * kDecodeRows * D;
    if (warp < 4) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int n = 8 * nt + 2 * c + e;
#pragma unroll
                // per-token V: + sum_t p_t sV_t oV_t (exactly 0 otherwise)
                for (int mt = 0; mt < MT; ++mt) {
                    oww[n * D + 8 * r + mt] = fmaf(-1152.0f, osum[nt][e], o[nt][mt][e]) + voff[nt][e];
                    oww[n * D + 64 + 8 * r + mt] =
                        fmaf(-1152.0f, osum[nt][e], o[nt][mt][2 + e]) + voff[nt][e];
                }
                if (r == 0) mlw[warp * kDecodeRows + n] = make_float2(m[nt][e], l[nt][e]);
            }
        }
    }
    __syncthreads();
    finish_unit<T, D, true>(a, u, si, R, ow, mlw);
}

// ---------------------------------------------------------------------------
template <typename T, int D, bool INT8>
__global__ void __launch_bounds__(D)
fia_combine_kernel(const __grid_constant__ CombineArgs a) {
    // one CTA per (sequence, kv head, row of a chunk); one thread per channel d
    const CombineItem it = a.items[blockIdx.x];
    const SeqInfo si = a.c.seq[it.b];
    const int g = a.c.g;
    const int row = blockIdx.y;                 // row within the chunk (partial slot row)
    const int n = it.r0 + row;                  // row of the group
    if (row >= a.c.chunk_rows || n >= si.qlen * g) return;
    const int d = threadIdx.x;
    const int head = it.kvh * g + n % g;
    const int token = si.cu_q + n / g;
    T *out = reinterpret_cast<T *>(a.c.out);
    float M = -INFINITY;
    for (int s = 0; s < it.nsplit; ++s)
        M = fmaxf(M, a.part_ml[(int64_t)(it.slot0 + s) * kDecodeRows + row].x);
    float val = 0.f, lse = INFINITY;
    if (M != -INFINITY) {
        const float sink2 = a.c.sink ? a.c.sink[head] * kLog2e : -INFINITY;
        const float M2 = fmaxf(M, sink2);
        float L = 0.f, acc = 0.f;
        for (int s = 0; s < it.nsplit; ++s) {
            const int64_t slot = it.slot0 + s;
            const float2 ml = a.part_ml[slot * kDecodeRows + row];
            if (ml.x == -INFINITY) continue;
            const float f = ex2(ml.x - M2);
            L = fmaf(ml.y, f, L);
            acc = fmaf(a.part_o[(slot * kDecodeRows + row) * D + d], f, acc);
        }
        const float Lt = L + (a.c.sink ? ex2(sink2 - M2) : 0.f);
        if constexpr (INT8) {
            // per-channel V: out_d = sV_d (sum_t p_t v_td + oV_d sum_t p_t) / L;
            // per-token V was applied token by token in the partials
            if (!a.v_mode) {
                const float vs = a.v_scale[it.kvh * D + d];
                const float vo = a.v_offset ? a.v_offset[it.kvh * D + d] : 0.f;
                acc = vs * fmaf(vo, L, acc);
            }
        }
        val = acc / Lt;
        lse = (M2 + log2f(Lt)) * kLn2;
    }
    if constexpr (MmaType<T>::bf16) {
        out[((int64_t)token * a.c.H + head) * D + d] = __float2bfloat16_rn(val);
    } else {
        out[((int64_t)token * a.c.H + head) * D + d] = __float2half_rn(val);
    }
    if (d == 0 && a.c.lse) a.c.lse[(int64_t)token * a.c.H + head] = lse;
}

// ---------------------------------------------------------------------------
template <typename T, int D>
static cudaError_t launch_decode_t(const DecodeArgs &a, const CUtensorMap &tk,
                                   const CUtensorMap &tv, int grid, cudaStream_t s) {
    auto kern = fia_decode_kernel<T, D>;
    const int smem = DecodeCfg<D>::kSmem;
    cudaError_t e = ensure_smem_attr<fia_decode_kernel<T, D>>(smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 128, smem, s>>>(a, tk, tv);
    return cudaGetLastError();
}

template <typename T, int NT, bool KTOK, bool VTOK>
static cudaError_t launch_decode_i8_m(const DecodeArgs &a, const CUtensorMap &tk,
                                      const CUtensorMap &tv, int grid, cudaStream_t s) {
    auto kern = fia_decode_i8_kernel<T, NT, KTOK, VTOK>;
    const int smem = DecodeI8Cfg::kSmem;
    cudaError_t e = ensure_smem_attr<fia_decode_i8_kernel<T, NT, KTOK, VTOK>>(smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kI8Producer + 32, smem, s>>>(a, tk, tv);
    return cudaGetLastError();
}

// dequantisation modes as compile-time flags: the per-channel kernel carries
// no per-token code
template <typename T, int NT>
static cudaError_t launch_decode_i8_t(const DecodeArgs &a, const CUtensorMap &tk,
                                      const CUtensorMap &tv, int grid, cudaStream_t s) {
    if (a.k_mode) return a.v_mode ? launch_decode_i8_m<T, NT, true, true>(a, tk, tv, grid, s)
                                  : launch_decode_i8_m<T, NT, true, false>(a, tk, tv, grid, s);
    return a.v_mode ? launch_decode_i8_m<T, NT, false, true>(a, tk, tv, grid, s)
                    : launch_decode_i8_m<T, NT, false, false>(a, tk, tv, grid, s);
}

cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap &tk, const CUtensorMap &tv,
                          int q_dtype, bool kv_int8, int grid, cudaStream_t s) {
    const bool bf = (q_dtype == 1);
    if (a.c.D == 128) {
        if (kv_int8) {
            // query rows per KV head: one or two N = 8 column tiles
            if (a.max_rows <= 8)
                return bf ? launch_decode_i8_t<__nv_bfloat16, 1>(a, tk, tv, grid, s)
                          : launch_decode_i8_t<__half, 1>(a, tk, tv, grid, s);
            return bf ? launch_decode_i8_t<__nv_bfloat16, 2>(a, tk, tv, grid, s)
                      : launch_decode_i8_t<__half, 2>(a, tk, tv, grid, s);
        }
        return bf ? launch_decode_t<__nv_bfloat16, 128>(a, tk, tv, grid, s)
                  : launch_decode_t<__half, 128>(a, tk, tv, grid, s);
    }
    if (a.c.D == 64 && !kv_int8)
        return bf ? launch_decode_t<__nv_bfloat16, 64>(a, tk, tv, grid, s)
                  : launch_decode_t<__half, 64>(a, tk, tv, grid, s);
    return cudaErrorInvalidValue;
}

template <typename T, int D, bool INT8>
static cudaError_t launch_combine_t(const CombineArgs &a, int grid, cudaStream_t s) {
    fia_combine_kernel<T, D, INT8><<<dim3(grid, kDecodeRows), D, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs &a, int q_dtype, bool kv_int8, int grid,
                           cudaStream_t s) {
    const bool bf = (q_dtype == 1);
    if (a.c.D == 128) {
        if (kv_int8) return bf ? launch_combine_t<__nv_bfloat16, 128, true>(a, grid, s)
                               : launch_combine_t<__half, 128, true>(a, grid, s);
        return bf ? launch_combine_t<__nv_bfloat16, 128, false>(a, grid, s)
                  : launch_combine_t<__half, 128, false>(a, grid, s);
    }
    if (a.c.D == 64 && !kv_int8)
        return bf ? launch_combine_t<__nv_bfloat16, 64, false>(a, grid, s)
                  : launch_combine_t<__half, 64, false>(a, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace fia
