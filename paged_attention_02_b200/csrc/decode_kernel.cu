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
// Kernel 1, fia_decode_kernel: one CTA per split unit (b, kvh, [t0, t1)).
//   * K/V rows of the unit stream through a STAGES-deep ring of shared-memory
//     tiles (64 keys each) filled by TMA: one 3-D box per (block run, 128-byte
//     column group), the physical row coming from the block table, so every
//     cached byte is fetched once, 128-byte swizzled for conflict-free reads.
//   * 4 warps split each tile 16 keys apiece.  The g*qlen query rows of the
//     group form the 16-row A operand of m16n8k16 tensor-core MMAs:
//     S = Q K^T (keys as N), online softmax in fp32 on the accumulator
//     fragments, then O += P V with P fed straight from registers.
//   * int8 caches are widened to f16 in registers by placing each byte (+128)
//     under the f16 exponent pattern for 1024, i.e. the exact value 1152 + x;
//     the 1152 bias is removed afterwards (for K from the per-row constant,
//     for V through a per-row sum of P from one extra MMA against ones).  The
//     per-channel K scale is folded into q (with a power-of-two range fix), the
//     K offset becomes one additive constant per row, and the V scale/offset
//     are applied once in the combine.
//   * Warps merge their (m, l, O) in shared memory and the CTA writes one
//     partial per unit.
// Kernel 2, fia_combine_kernel: one CTA per (b, kvh, row); merges the unit
//   partials in fixed logical order (deterministic), adds the learnable sink
//   to the denominator, applies int8 V dequantisation, writes out and lse.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "fia_device.cuh"
#include "fia_plan.h"

namespace fia {

template <int D, bool INT8>
struct DecodeCfg {
    static constexpr int kRowBytes = D * (INT8 ? 1 : 2);
    static constexpr int kHalves = kRowBytes / 128;               // 128-byte column groups
    static constexpr int kTileBytes = kDecodeTile * kRowBytes;    // one of K or V
    static constexpr int kStages = (2 * kTileBytes >= 32768) ? 3 : 4;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kMergeBytes = 4 * kDecodeRows * D * 4 + 4 * kDecodeRows * 8;
    static constexpr int kDataBytes =
        (kStages * kStageBytes > kMergeBytes) ? kStages * kStageBytes : kMergeBytes;
    static constexpr int kSmem = 1024 /*align slack*/ + kDataBytes + 2 * kStages * 8 + 16;
    static_assert(kRowBytes % 128 == 0, "row must be a whole number of 128-byte groups");
};

int decode_smem_bytes(int D, bool kv_int8) {
    if (D == 64) return kv_int8 ? -1 : DecodeCfg<64, false>::kSmem;
    if (D == 128) return kv_int8 ? DecodeCfg<128, true>::kSmem : DecodeCfg<128, false>::kSmem;
    return -1;
}

template <typename T, int D, bool INT8>
__global__ void __launch_bounds__(128, INT8 ? 3 : 2)
fia_decode_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv) {
    using Cfg = DecodeCfg<D, INT8>;
    constexpr int STAGES = Cfg::kStages;
    constexpr int KT = D / 16;           // k-steps of the QK^T MMA
    constexpr bool MMA_BF16 = INT8 ? false : MmaType<T>::bf16;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kDataBytes);
    uint64_t *empty = full + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + STAGES);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int r = lane >> 2;       // fragment row group
    const int c = lane & 3;        // fragment column pair

    const DecodeUnit u = a.units[blockIdx.x];
    const SeqInfo si = a.c.seq[u.b];
    const int g = a.c.g;
    const int R = si.qlen * g;
    const int n_tiles = (u.t_end - u.t_begin + kDecodeTile - 1) / kDecodeTile;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
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
            const int blk = bt_row[t / a.c.bs];
            const int prow = blk * a.c.bs + (t % a.c.bs);
            for (int hv = 0; hv < Cfg::kHalves; ++hv) {
                const int off = hv * kDecodeTile * 128 + bi * br * 128;
                const int col = INT8 ? hv * 128 : hv * 64;
                tma_load_3d(kst + off, &tk, &full[s], col, u.kvh, prow);
                tma_load_3d(vst + off, &tv, &full[s], col, u.kvh, prow);
            }
        }
    };
    if (tid == 0) {
        for (int j = 0; j < STAGES && j < n_tiles; ++j) issue(j);
    }

    // ---- per-row constants and the Q operand (rows ra = r, rb = r + 8) ----
    const int ra = r, rb = r + 8;
    int head_a = 0, head_b = 0, qi_a = 0, qi_b = 0;
    const bool va = ra < R, vb = rb < R;
    if (va) { qi_a = ra / g; head_a = u.kvh * g + ra % g; }
    if (vb) { qi_b = rb / g; head_b = u.kvh * g + rb % g; }
    const int qpos_a = si.kvlen - si.qlen + qi_a;
    const int qpos_b = si.kvlen - si.qlen + qi_b;
    const T *qp = reinterpret_cast<const T *>(a.c.q);
    const T *qa_ptr = qp + ((int64_t)(si.cu_q + qi_a) * a.c.H + head_a) * D;
    const T *qb_ptr = qp + ((int64_t)(si.cu_q + qi_b) * a.c.H + head_b) * D;

    uint32_t qf[KT][4];
    float sc_a = a.c.scale_log2, sc_b = a.c.scale_log2;   // multiplies the raw accumulator
    float add_a = 0.f, add_b = 0.f;                       // per-row additive term (log2 units)
    if constexpr (!INT8) {
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
            const int d0 = kk * 16 + 2 * c;
            qf[kk][0] = va ? *reinterpret_cast<const uint32_t *>(qa_ptr + d0) : 0u;
            qf[kk][1] = vb ? *reinterpret_cast<const uint32_t *>(qb_ptr + d0) : 0u;
            qf[kk][2] = va ? *reinterpret_cast<const uint32_t *>(qa_ptr + d0 + 8) : 0u;
            qf[kk][3] = vb ? *reinterpret_cast<const uint32_t *>(qb_ptr + d0 + 8) : 0u;
        }
    } else {
        // q'_d = q_d * kScale_d (fp32).  This thread holds dims 16kk+4c+{0..3};
        // the same order is used for the int8 key words below.
        const float *ks = a.k_scale + u.kvh * D;
        const float *ko = a.k_offset ? a.k_offset + u.kvh * D : nullptr;
        float qa[KT][4], qb[KT][4];
        float mx_a = 0.f, mx_b = 0.f, cs_a = 0.f, cs_b = 0.f;
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = kk * 16 + 4 * c + e;
                const float s = ks[d];
                const float o = ko ? ko[d] : 0.f;
                qa[kk][e] = va ? to_f32<T>(qa_ptr[d]) * s : 0.f;
                qb[kk][e] = vb ? to_f32<T>(qb_ptr[d]) * s : 0.f;
                mx_a = fmaxf(mx_a, fabsf(qa[kk][e]));
                mx_b = fmaxf(mx_b, fabsf(qb[kk][e]));
                cs_a = fmaf(qa[kk][e], o, cs_a);
                cs_b = fmaf(qb[kk][e], o, cs_b);
            }
        }
#pragma unroll
        for (int x = 1; x <= 2; x <<= 1) {
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, x));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, x));
            cs_a += __shfl_xor_sync(0xffffffffu, cs_a, x);
            cs_b += __shfl_xor_sync(0xffffffffu, cs_b, x);
        }
        // Scale each row by a power of two so that max|q'| lands below 2^11
        // (well inside f16 range), then undo it on the fp32 accumulator.
        int ea = 0, eb = 0;
        if (mx_a > 0.f) { frexpf(mx_a, &ea); ea = 11 - ea; }
        if (mx_b > 0.f) { frexpf(mx_b, &eb); eb = 11 - eb; }
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
            qf[kk][0] = pack2<__half>(ldexpf(qa[kk][0], ea), ldexpf(qa[kk][1], ea));
            qf[kk][1] = pack2<__half>(ldexpf(qb[kk][0], eb), ldexpf(qb[kk][1], eb));
            qf[kk][2] = pack2<__half>(ldexpf(qa[kk][2], ea), ldexpf(qa[kk][3], ea));
            qf[kk][3] = pack2<__half>(ldexpf(qb[kk][2], eb), ldexpf(qb[kk][3], eb));
        }
        sc_a = ldexpf(a.c.scale_log2, -ea);
        sc_b = ldexpf(a.c.scale_log2, -eb);
        // The MMA sees each key byte as the f16 value 1152 + k (see the QK loop),
        // so the raw score carries 1152 * sum_d q'_d, with q' exactly as the MMA
        // saw it (f16): remove it here, together with the key offset term.
        float sq_a = 0.f, sq_b = 0.f;
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
            const float2 fa0 = __half22float2(*reinterpret_cast<const __half2 *>(&qf[kk][0]));
            const float2 fa1 = __half22float2(*reinterpret_cast<const __half2 *>(&qf[kk][2]));
            const float2 fb0 = __half22float2(*reinterpret_cast<const __half2 *>(&qf[kk][1]));
            const float2 fb1 = __half22float2(*reinterpret_cast<const __half2 *>(&qf[kk][3]));
            sq_a += (fa0.x + fa0.y) + (fa1.x + fa1.y);
            sq_b += (fb0.x + fb0.y) + (fb1.x + fb1.y);
        }
#pragma unroll
        for (int x = 1; x <= 2; x <<= 1) {
            sq_a += __shfl_xor_sync(0xffffffffu, sq_a, x);
            sq_b += __shfl_xor_sync(0xffffffffu, sq_b, x);
        }
        add_a = cs_a * a.c.scale_log2 - 1152.0f * sq_a * sc_a;
        add_b = cs_b * a.c.scale_log2 - 1152.0f * sq_b * sc_b;
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
    // int8: sum of the (f16-rounded) P each row fed to the MMA, to remove the
    // 1152 bias of the value operand (see the PV loop)
    float osum[4] = {0.f, 0.f, 0.f, 0.f};
    float o[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
        const int s = j % STAGES;
        if (!mbar_wait(&full[s], (j / STAGES) & 1, abort_flag, a.c.err, 1)) { ok = false; break; }
        __syncwarp();      // ldmatrix / mma.sync below are warp-collective (.aligned)
        const uint32_t kst = smem_u32(smem + s * Cfg::kStageBytes);
        const uint32_t vst = kst + Cfg::kTileBytes;
        const int tw = u.t_begin + j * kDecodeTile + warp * 16;   // first key of this warp

        // ---- S = Q K^T over this warp's 16 keys ----
        float sacc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
        if constexpr (!INT8) {
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
        } else {
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int tok = warp * 16 + nt * 8 + r;
                    // bytes biased to 128 + k under the f16 exponent pattern:
                    // f16 values 1152 + k, exact; the 1152 * sum(q') term is
                    // removed from the row constant above
                    const uint32_t w = lds32(kst + swz128(tok, kk) + 4 * c) ^ 0x80808080u;
                    mma_16816<false>(sacc[nt], qf[kk], prmt(w, 0x64646464u, 0x4140u),
                                     prmt(w, 0x64646464u, 0x4342u));
                }
            }
        }

        // ---- scores, masks, online softmax ----
        float sv[2][4];
        float mx_a = -INFINITY, mx_b = -INFINITY;
        // Interior tile without bias: every key of the 16 is visible to every
        // row (rows past R only carry zeros and are never written out).
        const bool simple = !alibi && !a.c.pse && (tw + 16 <= u.t_end) &&
                            (!causal || tw + 15 <= si.kvlen - si.qlen);
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
                    const bool ka = in && va && !(causal && t > qpos_a);
                    const bool kb = in && vb && !(causal && t > qpos_b);
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
            if constexpr (INT8) {
                osum[0] *= al_a; osum[1] *= al_a;
                osum[2] *= al_b; osum[3] *= al_b;
            }
        }
        using PT = typename std::conditional<INT8, __half, T>::type;
        uint32_t pa[4];
        pa[0] = pack2<PT>(sv[0][0], sv[0][1]);
        pa[1] = pack2<PT>(sv[0][2], sv[0][3]);
        pa[2] = pack2<PT>(sv[1][0], sv[1][1]);
        pa[3] = pack2<PT>(sv[1][2], sv[1][3]);

        // ---- O += P V ----  (V rows past the unit's end are zeroed: P is 0
        // there but the slots may hold NaN garbage)
        const bool tail = (tw + 16 > u.t_end);
        if constexpr (!INT8) {
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
        } else {
            const int tk0 = warp * 16 + 2 * c;
            const int tg = tw + 2 * c;
            const uint32_t z0 = (tail && tg >= u.t_end) ? 0u : 0xffffffffu;
            const uint32_t z1 = (tail && tg + 1 >= u.t_end) ? 0u : 0xffffffffu;
            const uint32_t z2 = (tail && tg + 8 >= u.t_end) ? 0u : 0xffffffffu;
            const uint32_t z3 = (tail && tg + 9 >= u.t_end) ? 0u : 0xffffffffu;
#pragma unroll
            for (int i = 0; i < D / 32; ++i) {
                const int chunk = 2 * i + (r >> 2);
                const int wo = 4 * (r & 3);
                uint32_t w0 = lds32(vst + swz128(tk0, chunk) + wo);
                uint32_t w1 = lds32(vst + swz128(tk0 + 1, chunk) + wo);
                uint32_t w2 = lds32(vst + swz128(tk0 + 8, chunk) + wo);
                uint32_t w3 = lds32(vst + swz128(tk0 + 9, chunk) + wo);
                if (tail) { w0 &= z0; w1 &= z1; w2 &= z2; w3 &= z3; }
                const uint32_t x01 = prmt(w0, w1, 0x5140u) ^ 0x80808080u;
                const uint32_t x23 = prmt(w0, w1, 0x7362u) ^ 0x80808080u;
                const uint32_t y01 = prmt(w2, w3, 0x5140u) ^ 0x80808080u;
                const uint32_t y23 = prmt(w2, w3, 0x7362u) ^ 0x80808080u;
                // values as f16 (1152 + v), exact; the bias is removed at the end
                const uint32_t F = 0x64646464u;
                mma_16816<false>(o[4 * i + 0], pa, prmt(x01, F, 0x4140u), prmt(y01, F, 0x4140u));
                mma_16816<false>(o[4 * i + 1], pa, prmt(x01, F, 0x4342u), prmt(y01, F, 0x4342u));
                mma_16816<false>(o[4 * i + 2], pa, prmt(x23, F, 0x4140u), prmt(y23, F, 0x4140u));
                mma_16816<false>(o[4 * i + 3], pa, prmt(x23, F, 0x4342u), prmt(y23, F, 0x4342u));
            }
            // sum_t p~_t per row with the same rounding and accumulation as O
            const uint32_t ones = 0x3C003C00u;   // f16x2 (1, 1)
            mma_16816<false>(osum, pa, ones, ones);
        }

        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (tid == 0 && j + STAGES < n_tiles) {
            if (!mbar_wait(&empty[s], (j / STAGES) & 1, abort_flag, a.c.err, 2)) { ok = false; break; }
            issue(j + STAGES);
        }
        __syncwarp();
    }
    (void)ok;

    // ---- merge the 4 warps' (m, l, O) and write this unit's partial ----
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, x);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, x);
    }
    __syncthreads();   // every warp is done with the stage buffers
    float *ow = reinterpret_cast<float *>(smem);                          // [4][16][D]
    float2 *mlw = reinterpret_cast<float2 *>(smem + 4 * kDecodeRows * D * 4);  // [4][16]
    float *oww = ow + warp * kDecodeRows * D;
#pragma unroll
    for (int jj = 0; jj < D / 8; ++jj) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            int d;
            if constexpr (!INT8) {
                d = jj * 8 + 2 * c + e;
            } else {
                // n-tile jj = 4i + q covers dims 32i + 4n + q for column n
                d = (jj >> 2) * 32 + 4 * (2 * c + e) + (jj & 3);
            }
            if constexpr (INT8) {
                oww[ra * D + d] = fmaf(-1152.0f, osum[0], o[jj][e]);
                oww[rb * D + d] = fmaf(-1152.0f, osum[2], o[jj][2 + e]);
            } else {
                oww[ra * D + d] = o[jj][e];
                oww[rb * D + d] = o[jj][2 + e];
            }
        }
    }
    if (c == 0) {
        mlw[warp * kDecodeRows + ra] = make_float2(m_a, l_a);
        mlw[warp * kDecodeRows + rb] = make_float2(m_b, l_b);
    }
    __syncthreads();
    float *po = a.part_o + (int64_t)u.slot * kDecodeRows * D;
    float2 *pml = a.part_ml + (int64_t)u.slot * kDecodeRows;
    for (int idx = tid; idx < R * D; idx += blockDim.x) {
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
        po[row * D + d] = acc;
        if (d == 0) pml[row] = make_float2(M, L);
    }
}

// ---------------------------------------------------------------------------
template <typename T, int D, bool INT8>
__global__ void __launch_bounds__(D)
fia_combine_kernel(const __grid_constant__ CombineArgs a) {
    // one CTA per (sequence, kv head, row); one thread per channel d
    const CombineItem it = a.items[blockIdx.x];
    const SeqInfo si = a.c.seq[it.b];
    const int g = a.c.g;
    const int row = blockIdx.y;
    if (row >= si.qlen * g) return;
    const int d = threadIdx.x;
    const int head = it.kvh * g + row % g;
    const int token = si.cu_q + row / g;
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
            const float vs = a.v_scale[it.kvh * D + d];
            const float vo = a.v_offset ? a.v_offset[it.kvh * D + d] : 0.f;
            acc = vs * fmaf(vo, L, acc);
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
template <typename T, int D, bool INT8>
static cudaError_t launch_decode_t(const DecodeArgs &a, const CUtensorMap &tk,
                                   const CUtensorMap &tv, int grid, cudaStream_t s) {
    auto kern = fia_decode_kernel<T, D, INT8>;
    const int smem = DecodeCfg<D, INT8>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 128, smem, s>>>(a, tk, tv);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap &tk, const CUtensorMap &tv,
                          int q_dtype, bool kv_int8, int grid, cudaStream_t s) {
    const bool bf = (q_dtype == 1);
    if (a.c.D == 128) {
        if (kv_int8) return bf ? launch_decode_t<__nv_bfloat16, 128, true>(a, tk, tv, grid, s)
                               : launch_decode_t<__half, 128, true>(a, tk, tv, grid, s);
        return bf ? launch_decode_t<__nv_bfloat16, 128, false>(a, tk, tv, grid, s)
                  : launch_decode_t<__half, 128, false>(a, tk, tv, grid, s);
    }
    if (a.c.D == 64 && !kv_int8)
        return bf ? launch_decode_t<__nv_bfloat16, 64, false>(a, tk, tv, grid, s)
                  : launch_decode_t<__half, 64, false>(a, tk, tv, grid, s);
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
