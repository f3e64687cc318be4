// prefill_kernel.cu -- paged prefill / prefix-encoder attention on sm_100a
// tensor cores (tcgen05 UMMA, TMEM accumulators, TMA-staged paged K/V).
//
// Computes, for 128 new tokens of one sequence and one query head at a time,
//     O = Softmax(qkScale * Q K^T + bias) V
// (aclnnFusedInferAttentionScoreV4 / V3 "Formula"; ATB PrefixEncoder: new
// tokens attend to the cached prefix and to themselves, maskType 9 causal
// generated internally, maskType 3 ALiBi from per-head slopes; V4 alibi
// fullmask = pse tensor; V4 learnable sink; V3 lse bullet).
//
// One persistent CTA per SM walks a host-planned, longest-first list of
// (sequence, 128-token tile, head) items.  Warp roles:
//   warp 0   TMA producer: Q tile once per item, then K and V tiles of 128
//            keys, each tile gathered block by block through the block table
//            into a 2-stage ring (128-byte swizzled, K-major rows).
//   warp 1   UMMA issuer (one elected lane): S_j = Q K_j^T into one of two
//            TMEM S buffers, then O += P_{j-1} V_{j-1} into the TMEM O buffer,
//            so the next QK^T overlaps the softmax of the previous tile.
//            It also zeroes the V rows past kvSeqLen in a ragged last tile.
//   warps 2-5 softmax + epilogue, one query row per thread (TMEM lane):
//            tcgen05.ld the S row, scale / mask / bias in registers, online
//            softmax in fp32 (log2 domain, rescale of O in TMEM only when the
//            running max grows by more than 2^8), P rounded to the input dtype
//            into shared memory for the PV MMA; at the end O / l, the sink
//            term and lse.
// Every mbarrier wait is bounded in time (see fia_device.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "fia_device.cuh"
#include "fia_plan.h"

namespace fia {

template <int D>
struct PrefillCfg {
    static constexpr int kHalves = D / 64;                 // 128-byte column groups
    static constexpr int kTileBytes = 128 * D * 2;         // Q, K or V tile (128 rows)
    static constexpr int kGroupBytes = 128 * 128;          // one 128-row x 128-byte group
    static constexpr int kKStages = 3;
    static constexpr int kVStages = 3;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTileBytes;                   // K[s]
    static constexpr int kOffV = kOffK + kKStages * kTileBytes;        // V[s]
    static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
    // q_full, q_empty, k_full[3], k_empty[3], v_full[3], v_empty[3],
    // s_full[2], s_empty[2], p_full, pv_done, o_full
    static constexpr int kNumBar = 2 + 4 * 3 + 4 + 3;
    static constexpr int kUsed = kOffBar + kNumBar * 8 + 16;
    // Keep one CTA per SM (each CTA holds all 512 TMEM columns).
    static constexpr int kSmem = 1024 + (kUsed > 118 * 1024 ? kUsed : 118 * 1024);
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
};

int prefill_smem_bytes(int D) {
    if (D == 64) return PrefillCfg<64>::kSmem;
    if (D == 128) return PrefillCfg<128>::kSmem;
    return -1;
}

struct ItemGeom {
    int b, q0, h, kvh, cu_q, qlen, kvlen, rows, kv_end, n;
};

__device__ __forceinline__ ItemGeom item_geom(const PrefillArgs &a, int idx) {
    const PrefillItem it = a.items[idx];
    const SeqInfo si = a.c.seq[it.b];
    ItemGeom g;
    g.b = it.b; g.q0 = it.q0; g.h = it.h; g.kvh = it.h / a.c.g;
    g.cu_q = si.cu_q; g.qlen = si.qlen; g.kvlen = si.kvlen;
    g.rows = min(kPrefillBM, si.qlen - it.q0);
    const bool causal = (a.c.mask_type == 9 || a.c.mask_type == 3);
    g.kv_end = causal ? min(si.kvlen, si.kvlen - si.qlen + it.q0 + g.rows) : si.kvlen;
    if (g.kv_end < 0) g.kv_end = 0;
    g.n = (g.kv_end + kPrefillBN - 1) / kPrefillBN;
    return g;
}

// Bounded wait; on failure lane 0 leaves a trail record (item, tile, parity).
#define FIA_WAIT(bar, parity, where)                                                      \
    do {                                                                                  \
        const uint32_t _par = (parity);                                                   \
        if (!mbar_wait((bar), _par, abort_flag, a.c.err, (where))) {                      \
            if (lane == 0) fail_trail(a.c.err, (where), (uint32_t)idx, (uint32_t)dbg_j,   \
                                      _par, (bar));                                       \
            goto done;                                                                    \
        }                                                                                 \
    } while (0)

enum { kModePlain = 0, kModeAlibi = 1, kModePse = 2 };

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(192, 1)
fia_prefill_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tq,
                   const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
    using Cfg = PrefillCfg<D>;
    constexpr int KS = Cfg::kKStages, VS = Cfg::kVStages;
    constexpr bool BF = MmaType<T>::bf16;
    constexpr uint32_t IDESC_QK = umma_idesc_f16(BF, false, false, 128, kPrefillBN);
    constexpr uint32_t IDESC_PV = umma_idesc_f16(BF, false, true, 128, D);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *q_full = bars + 0;
    uint64_t *q_empty = bars + 1;
    uint64_t *k_full = bars + 2;            // [KS]
    uint64_t *k_empty = k_full + KS;        // [KS]
    uint64_t *v_full = k_empty + KS;        // [VS]
    uint64_t *v_empty = v_full + VS;        // [VS]
    uint64_t *s_full = v_empty + VS;        // [2]
    uint64_t *s_empty = s_full + 2;         // [2]  (released by the PV that read P from it)
    uint64_t *p_full = s_empty + 2;
    uint64_t *pv_done = p_full + 1;
    uint64_t *o_full = pv_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + Cfg::kNumBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < KS; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
        for (int s = 0; s < VS; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&s_full[s], 1); mbar_init(&s_empty[s], 1); }
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        mbar_init(o_full, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int dbg_j = -1;     // tile index recorded in failure trails

    const int it_begin = a.cta_off[blockIdx.x];
    const int it_end = a.cta_off[blockIdx.x + 1];
    const uint32_t sm_q = smem_u32(smem + Cfg::kOffQ);
    const uint32_t sm_k0 = smem_u32(smem + Cfg::kOffK);
    const uint32_t sm_v0 = smem_u32(smem + Cfg::kOffV);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t q_it = 0, kv_it = 0;
            const int br = a.c.box_rows;
            for (int idx = it_begin; idx < it_end; ++idx) {
                const ItemGeom gm = item_geom(a, idx);
                if (gm.n == 0) continue;
                FIA_WAIT(q_empty, (q_it & 1) ^ 1, 10);
                mbar_arrive_expect_tx(q_full, Cfg::kTileBytes);
                for (int hv = 0; hv < Cfg::kHalves; ++hv)
                    tma_load_3d(smem + Cfg::kOffQ + hv * Cfg::kGroupBytes, &tq, q_full, hv * 64,
                                gm.h, gm.cu_q + gm.q0);
                ++q_it;
                const int32_t *bt_row = a.c.bt + (int64_t)gm.b * a.c.bt_stride;
                for (int j = 0; j < gm.n; ++j, ++kv_it) {
                    dbg_j = j;
                    const int t0 = j * kPrefillBN;
                    const int t1 = min(t0 + kPrefillBN, gm.kvlen);
                    const int nbox = (t1 - t0 + br - 1) / br;
                    const uint32_t bytes = (uint32_t)(nbox * br * 128 * Cfg::kHalves);
                    const int ks = kv_it % KS, vs = kv_it % VS;
                    FIA_WAIT(&k_empty[ks], ((kv_it / KS) & 1) ^ 1, 11);
                    uint8_t *kd = smem + Cfg::kOffK + ks * Cfg::kTileBytes;
                    mbar_arrive_expect_tx(&k_full[ks], bytes);
                    for (int bi = 0; bi < nbox; ++bi) {
                        const int t = t0 + bi * br;
                        const int prow = bt_row[t / a.c.bs] * a.c.bs + (t % a.c.bs);
                        for (int hv = 0; hv < Cfg::kHalves; ++hv)
                            tma_load_3d(kd + hv * Cfg::kGroupBytes + bi * br * 128, &tk, &k_full[ks],
                                        hv * 64, gm.kvh, prow);
                    }
                    FIA_WAIT(&v_empty[vs], ((kv_it / VS) & 1) ^ 1, 12);
                    uint8_t *vd = smem + Cfg::kOffV + vs * Cfg::kTileBytes;
                    mbar_arrive_expect_tx(&v_full[vs], bytes);
                    for (int bi = 0; bi < nbox; ++bi) {
                        const int t = t0 + bi * br;
                        const int prow = bt_row[t / a.c.bs] * a.c.bs + (t % a.c.bs);
                        for (int hv = 0; hv < Cfg::kHalves; ++hv)
                            tma_load_3d(vd + hv * Cfg::kGroupBytes + bi * br * 128, &tv, &v_full[vs],
                                        hv * 64, gm.kvh, prow);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        uint32_t q_it = 0, kv_it = 0, s_it = 0, p_it = 0;
        for (int idx = it_begin; idx < it_end; ++idx) {
            const ItemGeom gm = item_geom(a, idx);
            if (gm.n == 0) continue;
            FIA_WAIT(q_full, q_it & 1, 20);
            ++q_it;
            const uint32_t kv_base = kv_it;
            const uint32_t s_base = s_it;
            for (int j = 0; j <= gm.n; ++j) {
                dbg_j = j;
                if (j < gm.n) {
                    // S_j = Q K_j^T  into TMEM buffer j % 2
                    const uint32_t kvi = kv_base + j;
                    const int ks = kvi % KS;
                    FIA_WAIT(&k_full[ks], (kvi / KS) & 1, 21);
                    const int sb = s_it & 1;
                    FIA_WAIT(&s_empty[sb], ((s_it >> 1) & 1) ^ 1, 22);
                    __syncwarp();
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t kbase = sm_k0 + ks * Cfg::kTileBytes;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * Cfg::kGroupBytes + (kk & 3) * 32;
                            umma_ss(tmem + (sb ? Cfg::kColS1 : Cfg::kColS0),
                                    umma_desc_sw128(sm_q + off, 16, 1024),
                                    umma_desc_sw128(kbase + off, 16, 1024), IDESC_QK, kk > 0);
                        }
                        umma_commit(&s_full[sb]);
                        umma_commit(&k_empty[ks]);
                        if (j == gm.n - 1) umma_commit(q_empty);
                    }
                    __syncwarp();
                    ++s_it;
                }
                if (j >= 1) {
                    // O += P_{j-1} V_{j-1}; P is in TMEM (aliasing S buffer (j-1) % 2)
                    const int jj = j - 1;
                    const uint32_t kvi = kv_base + jj;
                    const int vs = kvi % VS;
                    const int sb = (s_base + jj) & 1;
                    FIA_WAIT(p_full, p_it & 1, 23);
                    FIA_WAIT(&v_full[vs], (kvi / VS) & 1, 24);
                    __syncwarp();
                    const uint32_t vbase = sm_v0 + vs * Cfg::kTileBytes;
                    const int valid = gm.kvlen - jj * kPrefillBN;
                    if (valid < kPrefillBN) {
                        // rows past kvSeqLen: P is 0 there, but the slots may
                        // hold anything (NaN * 0 = NaN in the MMA) -> zero them.
                        uint8_t *vd = smem + Cfg::kOffV + vs * Cfg::kTileBytes;
                        const int nbytes = (kPrefillBN - valid) * 128;
                        for (int hv = 0; hv < Cfg::kHalves; ++hv) {
                            uint4 *p = reinterpret_cast<uint4 *>(vd + hv * Cfg::kGroupBytes + valid * 128);
                            for (int x = lane; x < nbytes / 16; x += 32) p[x] = make_uint4(0, 0, 0, 0);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t pcol = tmem + (sb ? Cfg::kColS1 : Cfg::kColS0);
#pragma unroll
                        for (int kk = 0; kk < kPrefillBN / 16; ++kk) {
                            umma_ts(tmem + Cfg::kColO, pcol + kk * 8,
                                    umma_desc_sw128(vbase + kk * 2048, Cfg::kGroupBytes, 1024),
                                    IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(pv_done);
                        umma_commit(&v_empty[vs]);
                        umma_commit(&s_empty[sb]);
                        if (jj == gm.n - 1) umma_commit(o_full);
                    }
                    __syncwarp();
                    ++p_it;
                }
            }
            kv_it = kv_base + gm.n;
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const bool causal = (a.c.mask_type == 9 || a.c.mask_type == 3);
        const float sl2 = a.c.scale_log2;
        // plain mode with a positive scale: mask raw scores and fold the scale
        // into the exponent (one FFMA per element)
        const bool fold = (MODE == kModePlain) && (sl2 > 0.f);
        uint32_t s_it = 0, p_it = 0, o_it = 0;
        T *outp = reinterpret_cast<T *>(a.c.out);
        for (int idx = it_begin; idx < it_end; ++idx) {
            const ItemGeom gm = item_geom(a, idx);
            const int i = gm.q0 + row;
            const bool valid = i < gm.qlen;
            const int qpos = gm.kvlen - gm.qlen + i;
            const int64_t orow = ((int64_t)(gm.cu_q + i) * a.c.H + gm.h);
            if (gm.n == 0) {
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(outp + orow * D);
                    for (int x = 0; x < D * 2 / 16; ++x) dst[x] = make_uint4(0, 0, 0, 0);
                    if (a.c.lse) a.c.lse[orow] = INFINITY;
                }
                __syncwarp();
                continue;
            }
            float slope2 = 0.f;
            if constexpr (MODE == kModeAlibi) slope2 = a.c.slopes[gm.h] * kLog2e;
            const T *pse_row = nullptr;
            if constexpr (MODE == kModePse) {
                // rows past seqLen read row 0 of the sequence (their output is dropped)
                pse_row = reinterpret_cast<const T *>(a.c.pse) +
                          (((int64_t)gm.b * a.c.H + gm.h) * a.c.pse_q + (valid ? i : 0)) * a.c.pse_kv;
            }
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < gm.n; ++j) {
                dbg_j = j;
                const int sb = s_it & 1;
                const uint32_t scol = t_lane + (sb ? Cfg::kColS1 : Cfg::kColS0);
                const int tb = j * kPrefillBN;
                FIA_WAIT(&s_full[sb], (s_it >> 1) & 1, 30);
                __syncwarp();          // tcgen05.ld/st below are warp-collective (.aligned)
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) tmem_ld32(scol + cc * 32, sr[cc]);
                tmem_ld_wait();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) reg_fence32(sr[cc]);
                ++s_it;

                // ---- scores (log2 units unless folded), bias, masks ----
                const bool edge = (tb + kPrefillBN > gm.kvlen) || (causal && tb + kPrefillBN - 1 > qpos);
                if constexpr (MODE == kModeAlibi) {
                    const float base = slope2 * (float)(tb - qpos);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                        for (int x = 0; x < 32; ++x) {
                            const float bias = fmaf(slope2, (float)(cc * 32 + x), base);
                            sr[cc][x] = __float_as_uint(fmaf(__uint_as_float(sr[cc][x]), sl2, bias));
                        }
                } else if constexpr (MODE == kModePse) {
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
                        for (int x8 = 0; x8 < 4; ++x8) {
                            const int t = tb + cc * 32 + x8 * 8;
                            T pv[8];
                            if (a.c.pse_vec && t + 8 <= gm.kvlen) {
                                *reinterpret_cast<uint4 *>(pv) =
                                    __ldg(reinterpret_cast<const uint4 *>(pse_row + t));
                            } else {
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    pv[e] = (t + e < gm.kvlen) ? pse_row[t + e] : pv[0];
                            }
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const float bias = to_f32<T>(pv[e]) * kLog2e;
                                sr[cc][x8 * 8 + e] = __float_as_uint(
                                    fmaf(__uint_as_float(sr[cc][x8 * 8 + e]), sl2, bias));
                            }
                        }
                    }
                    __syncwarp();      // reconverge after the per-row pse loads
                } else if (!fold) {
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            sr[cc][x] = __float_as_uint(__uint_as_float(sr[cc][x]) * sl2);
                }
                if (edge) {
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                        for (int x = 0; x < 32; ++x) {
                            const int t = tb + cc * 32 + x;
                            const bool keep = (t < gm.kvlen) && !(causal && t > qpos);
                            if (!keep) sr[cc][x] = __float_as_uint(-INFINITY);
                        }
                }
                // tree max (8 independent chains)
                float mx8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mx8[k] = __uint_as_float(sr[0][k]);
#pragma unroll
                for (int e = 8; e < 128; ++e)
                    mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(sr[e >> 5][e & 31]));
                float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                if (fold) mx = (mx == -INFINITY) ? -INFINITY : mx * sl2;

                // running max: exact on the first tile, afterwards raised only
                // when it grows by more than 2^8 (O and l stay consistent with m)
                const float m_new = fmaxf(m, mx);
                bool need = false;
                float alpha = 1.0f;
                if (j == 0) {
                    m = m_new;
                } else if (m_new > m + 8.0f) {
                    need = true;
                    alpha = ex2(m - m_new);
                    m = m_new;
                    l *= alpha;
                }
                const float mu = (m == -INFINITY) ? 0.f : m;

                // P = 2^(s - m) in the input dtype, stored over S's first 64 columns
                float ls8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) ls8[k] = 0.f;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t pk[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        float p0, p1;
                        if (fold) {
                            p0 = ex2(fmaf(__uint_as_float(sr[cc][2 * x]), sl2, -mu));
                            p1 = ex2(fmaf(__uint_as_float(sr[cc][2 * x + 1]), sl2, -mu));
                        } else {
                            p0 = ex2(__uint_as_float(sr[cc][2 * x]) - mu);
                            p1 = ex2(__uint_as_float(sr[cc][2 * x + 1]) - mu);
                        }
                        ls8[(2 * x) & 7] += p0;
                        ls8[(2 * x + 1) & 7] += p1;
                        pk[x] = pack2<T>(p0, p1);
                    }
                    tmem_st16(scol + cc * 16, pk);
                }
                l += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));

                // The previous PV must be complete before this warp signals P_j:
                // (1) O may be rescaled below; (2) it keeps every softmax warp
                // within one tile of the others, so the 4 arrivals that complete
                // a p_full phase always belong to the same tile, and pv_done can
                // never run two phases ahead of this parity wait.
                if (j > 0) {
                    FIA_WAIT(pv_done, (p_it - 1) & 1, 31);
                    __syncwarp();
                    tc_fence_after();
                }
                // rescale O (rare)
                if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t orr[32];
                        tmem_ld32(t_lane + Cfg::kColO + cc * 32, orr);
                        tmem_ld_wait();
                        reg_fence32(orr);
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            orr[x] = __float_as_uint(__uint_as_float(orr[x]) * alpha);
                        tmem_st32(t_lane + Cfg::kColO + cc * 32, orr);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full);
                ++p_it;
            }

            // ---- epilogue: O / l (+ sink), lse ----
            dbg_j = gm.n;
            FIA_WAIT(o_full, o_it & 1, 32);
            ++o_it;
            __syncwarp();
            tc_fence_after();
            const float mu = (m == -INFINITY) ? 0.f : m;
            float M = mu, lt = l;
            if (a.c.sink) {
                const float s2 = a.c.sink[gm.h] * kLog2e;
                M = fmaxf(mu, s2);
                lt = l * ex2(mu - M) + ex2(s2 - M);
            }
            const float oscale = ex2(mu - M) / lt;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t orr[32];
                tmem_ld32(t_lane + Cfg::kColO + cc * 32, orr);
                tmem_ld_wait();
                reg_fence32(orr);
                if (valid) {
                    uint32_t pk[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x)
                        pk[x] = pack2<T>(__uint_as_float(orr[2 * x]) * oscale,
                                         __uint_as_float(orr[2 * x + 1]) * oscale);
                    uint4 *dst = reinterpret_cast<uint4 *>(outp + orow * D + cc * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
                __syncwarp();
            }
            if (valid && a.c.lse) a.c.lse[orow] = (M + log2f(lt)) * kLn2;
            tc_fence_before();
            __syncwarp();
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

template <typename T, int D, int MODE>
static cudaError_t launch_prefill_t(const PrefillArgs &a, const CUtensorMap &tq,
                                    const CUtensorMap &tk, const CUtensorMap &tv, int grid,
                                    cudaStream_t s) {
    auto kern = fia_prefill_kernel<T, D, MODE>;
    const int smem = PrefillCfg<D>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 192, smem, s>>>(a, tq, tk, tv);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_prefill_mode(const PrefillArgs &a, const CUtensorMap &tq,
                                       const CUtensorMap &tk, const CUtensorMap &tv, int grid,
                                       cudaStream_t s) {
    if (a.c.pse) return launch_prefill_t<T, D, kModePse>(a, tq, tk, tv, grid, s);
    if (a.c.mask_type == 3) return launch_prefill_t<T, D, kModeAlibi>(a, tq, tk, tv, grid, s);
    return launch_prefill_t<T, D, kModePlain>(a, tq, tk, tv, grid, s);
}

cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &tq, const CUtensorMap &tk,
                           const CUtensorMap &tv, int q_dtype, int grid, cudaStream_t s) {
    const bool bf = (q_dtype == 1);
    if (a.c.D == 128)
        return bf ? launch_prefill_mode<__nv_bfloat16, 128>(a, tq, tk, tv, grid, s)
                  : launch_prefill_mode<__half, 128>(a, tq, tk, tv, grid, s);
    if (a.c.D == 64)
        return bf ? launch_prefill_mode<__nv_bfloat16, 64>(a, tq, tk, tv, grid, s)
                  : launch_prefill_mode<__half, 64>(a, tq, tk, tv, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace fia
