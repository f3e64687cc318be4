// prefill_kernel.cu -- paged prefill / prefix-encoder attention on sm_100a
// tensor cores (tcgen05 UMMA, TMEM accumulators, TMA-staged paged K/V).
//
// Computes, for tiles of 128 new tokens of one sequence and one query head,
//     O = Softmax(qkScale * Q K^T + bias) V
// (aclnnFusedInferAttentionScoreV4 / V3 "Formula"; ATB PrefixEncoder: new
// tokens attend to the cached prefix and to themselves, maskType 9 causal
// generated internally, maskType 3 ALiBi from per-head slopes; V4 alibi
// fullmask = pse tensor; V4 learnable sink; V3 lse bullet).
//
// One persistent CTA per SM walks a host-planned (longest-first) list of tile
// PAIRS: two 128-token tiles that read the same KV head (two heads of one GQA
// group, or two consecutive tiles of one head), so every K/V tile fetched
// serves 2 x 128 query rows.  Warp roles (18 warps):
//   warp 0     TMA producer: both Q tiles once per pair, then K and V tiles
//              of 128 keys, each gathered block by block through the block
//              table (2-stage K and V rings, 128-byte swizzle).
//   warp 1     UMMA issuer (one lane): S_X = Q_X K_j^T into TMEM, and
//              O_X += P_X V_j with P_X read from TMEM (TS form).  One thread's
//              tcgen05.mma ops run in issue order, so QK_X(j+1) may be issued
//              right after PV_X(j) over the same TMEM columns.  It zeroes the V
//              rows past kvSeqLen in a ragged last tile.
//   warps 2-9  softmax + epilogue of tile 0, warps 10-17 of tile 1: each warp
//              owns 16 query rows (TMEM lanes) of its lane quadrant; lanes t
//              and t + 16 hold the two 64-key halves of one row (16x32bx2
//              TMEM access), so row maxima and sums are combined with one
//              shuffle.  S -> registers, scale / mask / bias, online softmax
//              in fp32 (log2 domain; O rescaled in TMEM only when the running
//              max grows by more than 2^8), P in the input dtype written back
//              over S; at the end O / l, sink, lse (each lane writes half of
//              its row).
//   warps 18-19 (int8 cache only) converters: the producer lands raw int8 K
//              and V tiles in rings of their own; the products then run in
//              f16.  Per item the converters rewrite the Q tiles as f16(q *
//              kScale) (per-channel keys) or f16(q); per tile each thread
//              turns 16 values of 8 rows into f16 -- per channel x + offset,
//              widened exactly (the V scale joins in the epilogue), per token
//              (x + offset) * scale (V3 fake-quantization bullets) -- written
//              straight into the swizzled K / V stage the MMAs read.
// TMEM (512 columns): S_0 | S_1 | O_0 | O_1.  While one softmax group works on
// its S, the tensor core runs the other tile's PV and QK^T.
// Modes (template MODE): plain (causal or none), plain GQA (the same for
// g >= 2 over a 16-bit cache), ALiBi with the bias in the softmax (int8 cache
// or qkScale <= 0), ALiBi through the MMA (16-bit cache, qkScale > 0: the
// in-tile part of the bias is one more K-step of each QK^T block, the rest a
// per-row constant; key tiles run last to first), pse.  In the plain GQA,
// band and ALiBi-through-MMA instances an item's epilogue runs inside the
// next item's first key tile, and the issuer sends that item's first QK of
// tile 0 right after this item's last PV of tile 0.
// Each CTA's items are ordered by (sequence, KV head) on the host, so the
// CTAs sweep the KV heads together and K/V stays in L2 between items.
// Every mbarrier wait is bounded in time (see fia_device.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "fia_device.cuh"
#include "fia_plan.h"
#include "prefill_common.cuh"

namespace fia {

// 128 rows x 128 bytes of zeros (static storage starts zeroed): copied by the
// bulk-copy engine over the V rows past kvSeqLen of a ragged last key tile.
static __device__ __align__(128) uint8_t g_zero_rows[kPrefillBN * 128];

template <int D, int MODE = kModePlain, bool I8 = false>
struct PrefillCfg {
    static constexpr int kHalves = D / 64;                 // 128-byte column groups
    static constexpr int kTileBytes = 128 * D * 2;         // Q, K or V tile (128 rows)
    static constexpr int kGroupBytes = 128 * 128;          // one 128-row x 128-byte group
    static constexpr int kRawBytes = 128 * D;              // an int8 K or V tile
    // pse mode gives one K and one V stage to the per-warp pse slots; an int8
    // cache gives one V stage to its raw int8 rings (K and V, kRawStages each)
    static constexpr int kKStages = (MODE == kModePse) ? 1 : 2;
    static constexpr int kVStages = (MODE == kModePse || I8) ? 1 : 2;
    static constexpr int kRawStages = !I8 ? 0 : (MODE == kModePse) ? 1 : 2;
    static constexpr int kOffQ = 0;                                    // Q[2]
    static constexpr int kOffK = kOffQ + 2 * kTileBytes;               // K[s]
    static constexpr int kOffV = kOffK + kKStages * kTileBytes;        // V[s]
    // pse mode: two 16-row x 64-key pse boxes (2 x 2 KB, 128-byte swizzle)
    // per softmax warp, fetched by that warp one key tile ahead
    static constexpr int kOffPse = kOffV + kVStages * kTileBytes;
    static constexpr int kPseBytes = (MODE == kModePse) ? 16 * 4096 : 0;
    static constexpr int kOffRaw = kOffPse + kPseBytes;      // raw K[RS], raw V[RS]
    // kModeAlibiMma: the bias operands of the extra QK^T K-step, unswizzled
    // K-major 8-row x 16-byte core matrices: per tile of the pair the Q side
    // (one core matrix shared by all 16 row groups, then a zero one for K
    // columns 8..15), then the K side (16 groups of 8 key rows, each group's
    // core matrix followed by its zero one)
    static constexpr int kOffExt = kOffRaw + 2 * kRawStages * kRawBytes;
    static constexpr int kExtBytes = (MODE == kModeAlibiMma) ? 2 * 256 + 2 * 2048 : 0;
    static constexpr int kOffBar = kOffExt + kExtBytes;
    static_assert(kOffRaw % 1024 == 0, "swizzled TMA destinations are 1024-byte aligned");
    // q_full, q_empty, k_full/k_empty[KS], v_full/v_empty[VS],
    // s_full[2], p_full[2], o_full[2], pse_full[16], vz_full,
    // mma_drain (error exit), never (test hook: nothing arrives on it),
    // rk_full/rk_empty[RS], rv_full/rv_empty[RS] (int8 rings), q_conv (int8:
    // the converted Q tiles are ready)
    static constexpr int kNumBar = 2 + 2 * kKStages + 2 * kVStages + 6 + 16 + 1 + 2 + 4 * kRawStages + 1;
    static constexpr int kUsed = kOffBar + kNumBar * 8 + 16;
    // Keep one CTA per SM (each CTA holds all 512 TMEM columns).
    static constexpr int kSmem = 1024 + (kUsed > 118 * 1024 ? kUsed : 118 * 1024);
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t col_s(int x) { return (uint32_t)x * 128u; }
    static constexpr uint32_t col_o(int x) { return 256u + (uint32_t)x * D; }
    // producer, UMMA, 2 x 8 softmax warps (+ 2 int8 converters: five warps on
    // each SM sub-partition either way, so the register budget is unchanged)
    static constexpr int kThreads = I8 ? 640 : 576;
    static_assert(!I8 || D == 128, "int8 tiles are one 128-byte row per key");
};

// Bounded wait of a single-lane role (TMA producer, MMA issuer); on failure
// the lane leaves a trail record (item, tile, parity) and goes to the exit.
#define FIA_WAIT(bar, parity, where)                                                      \
    do {                                                                                  \
        const uint32_t _par = (parity);                                                   \
        if (!mbar_wait((bar), _par, abort_flag, a.c.err, (where), a.c.wait_ns)) {         \
            fail_trail(a.c.err, (where), (uint32_t)idx, (uint32_t)dbg_j, _par, (bar));    \
            goto done;                                                                    \
        }                                                                                 \
    } while (0)

// Bounded wait of a whole softmax warp: every lane polls, and the warp leaves
// together when any lane gave up, so no lane reaches the warp-collective
// (.sync.aligned) tcgen05 loads and stores or the shuffles that follow without
// its siblings; pending TMEM stores are waited for before leaving.
#define FIA_WAIT_W(bar, parity, where)                                                    \
    do {                                                                                  \
        const uint32_t _par = (parity);                                                   \
        const bool _ok = mbar_wait((bar), _par, abort_flag, a.c.err, (where), a.c.wait_ns); \
        if (!__all_sync(0xffffffffu, _ok)) {                                              \
            if (lane == 0) fail_trail(a.c.err, (where), (uint32_t)idx, (uint32_t)dbg_j,   \
                                      _par, (bar));                                       \
            tmem_st_wait();                                                               \
            goto done;                                                                    \
        }                                                                                 \
    } while (0)

// Dequantise one int8 tile (128 keys x 128 dims in 128-byte swizzled rows at
// `raw`) into T at `dst`: two 64-column groups of 128-byte swizzled rows, the
// layout TMA gives a 16-bit cache, so the MMAs read it unchanged.  The thread
// (rl, c) converts dims 16c .. 16c + 15 of rows 8 it + rl; rows at or past
// `valid` (past kvSeqLen, or never loaded) become zeros.  sc / of: TOK, the
// tile's per-token rows (sc[r], of[r]); otherwise this thread's 16 channels
// (sc[i], of[i]).  of may be null.
//
// value = (x + offset) * scale: the sign-flipped byte x + 128 placed at
// mantissa bits 8..15 of 1.0 is the float v = 1 + (x + 128) / 2^15 (exact), and
// value = v * (2^15 scale) + (offset - 2^15 - 128) * scale: one FMA per value,
// rounded once, plus the rounding of the constant (about 0.004 scale, far
// below the final rounding to T).
template <typename T, bool TOK, bool FULL>
__device__ __forceinline__ void dequant_tile(const uint8_t *__restrict__ raw,
                                             uint8_t *__restrict__ dst, int rl, int c, int valid,
                                             const float *sc, const float *of) {
    float S[16], C[16];
    if constexpr (!TOK) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float s = __ldg(sc + i);
            const float o = of ? __ldg(of + i) : 0.f;
            S[i] = s * 32768.f;
            C[i] = (o - 32896.f) * s;
        }
    }
    const uint32_t kOne = 0x3F800000u;
    const int src_chunk = (c ^ rl) << 4;
    const int lo_chunk = (((2 * c) & 7) ^ rl) << 4;
    const int hi_chunk = (((2 * c + 1) & 7) ^ rl) << 4;
    uint8_t *grp = dst + (c >> 2) * (128 * 128);
#pragma unroll
    for (int it = 0; it < 16; ++it) {
        const int r = it * 8 + rl;
        const uint4 w4 = *reinterpret_cast<const uint4 *>(raw + r * 128 + src_chunk);
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
        float ts = 0.f, tc = 0.f;
        if constexpr (TOK) {
            // rows past the tile's keys read the last valid row's parameters
            const int rr = FULL ? r : min(r, valid - 1);
            const float s = __ldg(sc + rr);
            const float o = of ? __ldg(of + rr) : 0.f;
            ts = s * 32768.f;
            tc = (o - 32896.f) * s;
        }
        uint32_t o8[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t x = w[i] ^ 0x80808080u;
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                v[e] = __uint_as_float(prmt(x, kOne, 0x7604u | ((uint32_t)e << 4)));
            uint64_t y01, y23;
            if constexpr (TOK) {
                const uint64_t S2 = f2pack(ts, ts), C2 = f2pack(tc, tc);
                y01 = ffma2(f2pack(v[0], v[1]), S2, C2);
                y23 = ffma2(f2pack(v[2], v[3]), S2, C2);
            } else {
                y01 = ffma2(f2pack(v[0], v[1]), f2pack(S[4 * i], S[4 * i + 1]),
                            f2pack(C[4 * i], C[4 * i + 1]));
                y23 = ffma2(f2pack(v[2], v[3]), f2pack(S[4 * i + 2], S[4 * i + 3]),
                            f2pack(C[4 * i + 2], C[4 * i + 3]));
            }
            float a0, a1, a2, a3;
            f2unpack(y01, a0, a1);
            f2unpack(y23, a2, a3);
            o8[2 * i] = pack2<T>(a0, a1);
            o8[2 * i + 1] = pack2<T>(a2, a3);
        }
        if (!FULL && r >= valid) {
#pragma unroll
            for (int k = 0; k < 8; ++k) o8[k] = 0u;
        }
        uint8_t *row = grp + r * 128;
        *reinterpret_cast<uint4 *>(row + lo_chunk) = make_uint4(o8[0], o8[1], o8[2], o8[3]);
        *reinterpret_cast<uint4 *>(row + hi_chunk) = make_uint4(o8[4], o8[5], o8[6], o8[7]);
    }
}

// int8 cache, per-channel mode: one tile's bytes widened exactly to f16,
// x + 128 placed under the f16 exponent pattern of 1024 (the value 1152 + x)
// minus 1152, with OFS plus the channel's offset (one f16 rounding); the
// scale is applied elsewhere (folded into Q for K, in the epilogue for V).
// Same layout and thread mapping as
// dequant_tile; rows at or past `valid` become zeros.  of: this thread's 16
// channels' offsets (OFS).
template <bool FULL, bool OFS>
__device__ __forceinline__ void widen_tile(const uint8_t *__restrict__ raw,
                                           uint8_t *__restrict__ dst, int rl, int c, int valid,
                                           const float *of) {
    __half2 o2[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        o2[k] = (OFS && of) ? __floats2half2_rn(__ldg(of + 2 * k), __ldg(of + 2 * k + 1))
                            : __floats2half2_rn(0.f, 0.f);
    const __half2 k1152 = __floats2half2_rn(1152.f, 1152.f);
    const uint32_t kF = 0x64646464u;
    const int src_chunk = (c ^ rl) << 4;
    const int lo_chunk = (((2 * c) & 7) ^ rl) << 4;
    const int hi_chunk = (((2 * c + 1) & 7) ^ rl) << 4;
    uint8_t *grp = dst + (c >> 2) * (128 * 128);
#pragma unroll
    for (int it = 0; it < 16; ++it) {
        const int r = it * 8 + rl;
        const uint4 w4 = *reinterpret_cast<const uint4 *>(raw + r * 128 + src_chunk);
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
        uint32_t o8[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t x = w[i] ^ 0x80808080u;
            const uint32_t h01 = prmt(x, kF, 0x4140u), h23 = prmt(x, kF, 0x4342u);
            __half2 y01 = __hsub2(*reinterpret_cast<const __half2 *>(&h01), k1152);
            __half2 y23 = __hsub2(*reinterpret_cast<const __half2 *>(&h23), k1152);
            if constexpr (OFS) {
                y01 = __hadd2(y01, o2[2 * i]);
                y23 = __hadd2(y23, o2[2 * i + 1]);
            }
            o8[2 * i] = *reinterpret_cast<uint32_t *>(&y01);
            o8[2 * i + 1] = *reinterpret_cast<uint32_t *>(&y23);
        }
        if (!FULL && r >= valid) {
#pragma unroll
            for (int k = 0; k < 8; ++k) o8[k] = 0u;
        }
        uint8_t *row = grp + r * 128;
        *reinterpret_cast<uint4 *>(row + lo_chunk) = make_uint4(o8[0], o8[1], o8[2], o8[3]);
        *reinterpret_cast<uint4 *>(row + hi_chunk) = make_uint4(o8[4], o8[5], o8[6], o8[7]);
    }
}

// int8 cache: a Q tile (128 rows x 128 dims of T in two 64-column groups of
// 128-byte swizzled rows) rewritten in place as f16(q * scale_d), so the
// products run in f16 against the widened keys.  Thread u of 64 takes chunk
// position p = u & 15 (group p >> 3, chunk p & 7) of rows (u >> 4) + 4 i; the
// eight threads of a quarter warp cover one row's eight chunks.  sc: the
// per-channel K scale of the KV head, or null (per-token keys: scale 1).
template <typename T>
__device__ __forceinline__ void q_to_f16(uint8_t *__restrict__ q, int u, const float *sc) {
    const int p = u & 15, hv = p >> 3, cl = p & 7;
    float s8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) s8[e] = sc ? __ldg(sc + hv * 64 + cl * 8 + e) : 1.f;
    uint8_t *grp = q + hv * (128 * 128);
#pragma unroll 4
    for (int r = u >> 4; r < 128; r += 4) {
        uint4 *ptr = reinterpret_cast<uint4 *>(grp + r * 128 + ((cl ^ (r & 7)) << 4));
        const uint4 w4 = *ptr;
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
        uint32_t o4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float f0, f1;
            if constexpr (MmaType<T>::bf16) {
                f0 = __uint_as_float(w[i] << 16);
                f1 = __uint_as_float(w[i] & 0xffff0000u);
            } else {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
                f0 = f.x;
                f1 = f.y;
            }
            o4[i] = pack2<__half>(f0 * s8[2 * i], f1 * s8[2 * i + 1]);
        }
        *ptr = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
}

// Bounded wait of a converter warp (no TMEM state to settle): the warp leaves
// together when any lane gave up.
#define FIA_WAIT_C(bar, parity, where)                                                    \
    do {                                                                                  \
        const uint32_t _par = (parity);                                                   \
        const bool _ok = mbar_wait((bar), _par, abort_flag, a.c.err, (where), a.c.wait_ns); \
        if (!__all_sync(0xffffffffu, _ok)) {                                              \
            if (lane == 0) fail_trail(a.c.err, (where), (uint32_t)idx, (uint32_t)dbg_j,   \
                                      _par, (bar));                                       \
            goto done;                                                                    \
        }                                                                                 \
    } while (0)

template <typename T, int D, int MODE, int PB, bool BAND, bool I8>
__global__ void __launch_bounds__(PrefillCfg<D, MODE, I8>::kThreads, 1)
fia_prefill_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tq,
                   const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                   const __grid_constant__ CUtensorMap tp, const __grid_constant__ PlanBytes<PB> pl) {
    using Cfg = PrefillCfg<D, MODE, I8>;
    constexpr int KS = Cfg::kKStages, VS = Cfg::kVStages, RS = Cfg::kRawStages;
    // int8 cache: the products run in f16 (Q, the widened K / V and P)
    using MT = std::conditional_t<I8, __half, T>;
    constexpr bool BF = MmaType<MT>::bf16;
    // ALiBi through the MMA: S gains slope / qkScale * (t - t0) for key t of a
    // tile starting at key t0, the rest of the bias is one constant per row
    constexpr bool XB = (MODE == kModeAlibiMma);
    static_assert(!XB || !I8, "the bias K-step is for 16-bit caches");
    // Instances whose pairs end both tiles on the same key tile (GQA pairs,
    // band: GQA pairs or single tiles; ALiBi through the MMA: key tiles last
    // to first) run an item's epilogue inside the next item's first key tile
    // and send that item's first QK_0 early.  Elsewhere (first-to-last MHA
    // pairs, whose tile 0 ends a key tile early and hides its epilogue there;
    // pse and int8, short of registers) the epilogue follows the item at once.
    constexpr bool DEFER = (BAND || XB || MODE == kModePlainGqa) && !I8 && MODE != kModePse;
    constexpr uint32_t IDESC_QK = umma_idesc_f16(BF, false, false, 128, kPrefillBN);
    constexpr uint32_t IDESC_PV = umma_idesc_f16(BF, false, true, 128, D);

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned start, kept an offset of the shared array so that
    // plain loads and stores through it stay shared-memory accesses
    const uint32_t sm_raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((sm_raw + 1023u) & ~1023u) - sm_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *q_full = bars + 0;
    uint64_t *q_empty = bars + 1;
    uint64_t *k_full = bars + 2;            // [KS]
    uint64_t *k_empty = k_full + KS;        // [KS]
    uint64_t *v_full = k_empty + KS;        // [VS]
    uint64_t *v_empty = v_full + VS;        // [VS]
    uint64_t *s_full = v_empty + VS;        // [2]  QK_X done
    uint64_t *p_full = s_full + 2;          // [2]  P_X written (4 warps)
    uint64_t *o_full = p_full + 2;          // [2]  last PV_X of the pair done
    uint64_t *pse_full = o_full + 2;        // [16] per softmax warp (pse mode)
    uint64_t *vz_full = pse_full + 16;      // zero rows copied over a ragged V tile
    uint64_t *mma_drain = vz_full + 1;      // error exit: every MMA issued so far is done
    uint64_t *never = mma_drain + 1;        // test hook: nothing arrives on it
    uint64_t *rk_full = never + 1;          // [RS] int8 rings (I8 only)
    uint64_t *rk_empty = rk_full + RS;
    uint64_t *rv_full = rk_empty + RS;
    uint64_t *rv_empty = rv_full + RS;
    uint64_t *q_conv = rv_empty + RS;       // int8: Q in f16 (2 converter warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + Cfg::kNumBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (PB >= kInlinePlanBytes && blockIdx.x == 0 && tid == 0 && a.c.err) {
        // nothing clears the error words per run on this path; a wait can
        // only give up seconds after this store
        a.c.err[0] = 0u;
        a.c.err[1] = 0u;
    }
    if (tid == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        // int8: the two converter warps fill the K / V stages
        for (int s = 0; s < KS; ++s) { mbar_init(&k_full[s], I8 ? 2 : 1); mbar_init(&k_empty[s], 1); }
        for (int s = 0; s < VS; ++s) { mbar_init(&v_full[s], I8 ? 2 : 1); mbar_init(&v_empty[s], 1); }
        for (int s = 0; s < RS; ++s) {
            mbar_init(&rk_full[s], 1);
            mbar_init(&rk_empty[s], 2);
            mbar_init(&rv_full[s], 1);
            mbar_init(&rv_empty[s], 2);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s_full[x], 1);
            mbar_init(&p_full[x], 8);
            mbar_init(&o_full[x], 1);
        }
        for (int x = 0; x < 16; ++x) mbar_init(&pse_full[x], 1);
        mbar_init(vz_full, 1);
        mbar_init(mma_drain, 1);
        mbar_init(never, 1);
        mbar_init(q_conv, 2);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
        if (MODE == kModePse && a.c.pse_tma) tma_prefetch_desc(&tp);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    if constexpr (XB) {
        // bias operands (16-byte rows): [0, 8) / [16, 24) Q side of tiles 0 / 1
        // (written per item by the producer), [8, 16) / [24, 32) zeros; then
        // per group of 8 keys 8 rows x = (x, x, x, 0 ...) -- the column offset
        // inside the key tile, exact in 16 bits, meeting the three parts of the
        // slope -- and 8 zero rows
        uint4 *ext = reinterpret_cast<uint4 *>(smem + Cfg::kOffExt);
        for (int r16 = tid; r16 < 288; r16 += Cfg::kThreads) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            const int L = r16 - 32;
            if (L >= 0 && (L & 15) < 8) {
                const float xv = (float)((L >> 4) * 8 + (L & 15));
                v.x = pack2<MT>(xv, xv);
                v.y = pack2<MT>(xv, 0.f);
            }
            ext[r16] = v;
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int dbg_j = -1;     // tile index recorded in failure trails
    int idx = -1;
    // Copies each role has requested and (for the error exit) seen complete:
    // producer Q / K / V tiles, issuer zero-row copies, softmax pse boxes.
    uint32_t req_q = 0, req_k = 0, req_v = 0, req_vz = 0, seen_vz = 0, req_ps = 0, seen_ps = 0;

    // the plan: inline kernel parameter, or the workspace copy
    const uint8_t *plan = (PB >= kInlinePlanBytes) ? pl.b : a.plan;
    const SeqInfo *seqs = reinterpret_cast<const SeqInfo *>(plan + a.off_seq);
    const int32_t *cta_off = reinterpret_cast<const int32_t *>(plan + a.off_cta);
    const PrefillItem *items = reinterpret_cast<const PrefillItem *>(plan + a.off_items);
    const int it_begin = cta_off[blockIdx.x];
    const int it_end = cta_off[blockIdx.x + 1];
    const uint32_t sm_q = smem_u32(smem + Cfg::kOffQ);
    const uint32_t sm_k0 = smem_u32(smem + Cfg::kOffK);
    const uint32_t sm_v0 = smem_u32(smem + Cfg::kOffV);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int br = a.c.box_rows;
            for (idx = it_begin; idx < it_end; ++idx) {
                const PairGeom gm = pair_geom<BAND>(a, items, seqs, idx);
                if (gm.nB == 0) continue;
                FIA_WAIT(q_empty, (req_q & 1) ^ 1, 10);
                if constexpr (XB) {
                    // Q side of the bias step: slope / qkScale (log2 units over
                    // the scale folded into the exponent) as the sum of three
                    // 16-bit parts, in each of the 8 rows of the shared core matrix
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        if (!gm.t[x].valid) continue;
                        const float sv = a.c.slopes[gm.t[x].h] * kLog2e / a.c.scale_log2;
                        const float s0 = round_to<MT>(sv);
                        const float s1 = round_to<MT>(sv - s0);
                        const float s2 = sv - s0 - s1;
                        const uint32_t w0 = pack2<MT>(s0, s1), w1 = pack2<MT>(s2, 0.f);
                        const uint32_t qx = smem_u32(smem + Cfg::kOffExt + x * 256);
#pragma unroll
                        for (int r8 = 0; r8 < 8; ++r8) sts128(qx + r8 * 16, w0, w1, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                }
                mbar_arrive_expect_tx(q_full, (gm.t[0].valid ? 2 : 1) * Cfg::kTileBytes);
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (!gm.t[x].valid) continue;
                    for (int hv = 0; hv < Cfg::kHalves; ++hv)
                        tma_load_3d(smem + Cfg::kOffQ + x * Cfg::kTileBytes + hv * Cfg::kGroupBytes,
                                    &tq, q_full, hv * 64, gm.t[x].h, gm.cu_q + gm.t[x].q0);
                }
                ++req_q;
                const int32_t *bt_row = a.c.bt + (int64_t)gm.b * a.c.bt_stride;
                for (int j = 0; j < gm.nB; ++j) {
                    dbg_j = j;
                    // key tiles last to first in the ALiBi-through-MMA mode
                    const int t0 = (XB ? gm.j0 + gm.nB - 1 - j : gm.j0 + j) * kPrefillBN;
                    const int t1 = min(t0 + kPrefillBN, gm.kvlen);
                    const int nbox = (t1 - t0 + br - 1) / br;
                    const uint32_t bytes = (uint32_t)(nbox * br * 128 * Cfg::kHalves);
                    if constexpr (I8) {
                        // raw int8 rows (one 128-byte box row per key) into the rings
                        const uint32_t rbytes = (uint32_t)(nbox * br * 128);
                        const int rks = req_k % RS;
                        FIA_WAIT(&rk_empty[rks], ((req_k / RS) & 1) ^ 1, 11);
                        uint8_t *kd = smem + Cfg::kOffRaw + rks * Cfg::kRawBytes;
                        mbar_arrive_expect_tx(&rk_full[rks], rbytes);
                        for (int bi = 0; bi < nbox; ++bi) {
                            const int t = t0 + bi * br;
                            int y, z;
                            kv_box_yz(a.c, gm.kvh, bt_row[t / a.c.bs], t % a.c.bs, y, z);
                            tma_load_3d(kd + bi * br * 128, &tk, &rk_full[rks], 0, y, z);
                        }
                        ++req_k;
                        const int rvs = req_v % RS;
                        FIA_WAIT(&rv_empty[rvs], ((req_v / RS) & 1) ^ 1, 12);
                        uint8_t *vd = smem + Cfg::kOffRaw + (RS + rvs) * Cfg::kRawBytes;
                        mbar_arrive_expect_tx(&rv_full[rvs], rbytes);
                        for (int bi = 0; bi < nbox; ++bi) {
                            const int t = t0 + bi * br;
                            int y, z;
                            kv_box_yz(a.c, gm.kvh, bt_row[t / a.c.bs], t % a.c.bs, y, z);
                            tma_load_3d(vd + bi * br * 128, &tv, &rv_full[rvs], 0, y, z);
                        }
                        ++req_v;
                        continue;
                    }
                    const int ks = req_k % KS, vs = req_v % VS;
                    FIA_WAIT(&k_empty[ks], ((req_k / KS) & 1) ^ 1, 11);
                    uint8_t *kd = smem + Cfg::kOffK + ks * Cfg::kTileBytes;
                    mbar_arrive_expect_tx(&k_full[ks], bytes);
                    for (int bi = 0; bi < nbox; ++bi) {
                        const int t = t0 + bi * br;
                        int y, z;
                        kv_box_yz(a.c, gm.kvh, bt_row[t / a.c.bs], t % a.c.bs, y, z);
                        for (int hv = 0; hv < Cfg::kHalves; ++hv)
                            tma_load_3d(kd + hv * Cfg::kGroupBytes + bi * br * 128, &tk, &k_full[ks],
                                        hv * 64, y, z);
                    }
                    ++req_k;
                    FIA_WAIT(&v_empty[vs], ((req_v / VS) & 1) ^ 1, 12);
                    uint8_t *vd = smem + Cfg::kOffV + vs * Cfg::kTileBytes;
                    mbar_arrive_expect_tx(&v_full[vs], bytes);
                    for (int bi = 0; bi < nbox; ++bi) {
                        const int t = t0 + bi * br;
                        int y, z;
                        kv_box_yz(a.c, gm.kvh, bt_row[t / a.c.bs], t % a.c.bs, y, z);
                        for (int hv = 0; hv < Cfg::kHalves; ++hv)
                            tma_load_3d(vd + hv * Cfg::kGroupBytes + bi * br * 128, &tv, &v_full[vs],
                                        hv * 64, y, z);
                    }
                    ++req_v;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        // One lane runs this role; the other 31 go straight to the teardown.
        // The issuing warp shares its SM sub-partition with four busy softmax
        // warps and is starved of issue slots, so every instruction here is
        // expensive: no warp-level syncs, each block of MMAs issued from one
        // asm statement with descriptors prepared before the wait that
        // precedes it.
        if (lane != 0) goto done;
        uint32_t q_it = 0, kv_it = 0, p_it[2] = {0, 0};
        bool qk0_early = false;     // the next item's first QK_0 went out already
        constexpr int NKQ = D / 16;                     // K-steps of QK^T
        constexpr uint32_t kHi = umma_desc_hi_sw128(1024);
        constexpr uint32_t kTileStep = Cfg::kTileBytes >> 4;
        const uint32_t q_lo = umma_desc_lo(sm_q, 16);
        const uint32_t k_lo = umma_desc_lo(sm_k0, 16);
        const uint32_t v_lo = umma_desc_lo(sm_v0, Cfg::kGroupBytes);
        // first-step Q descriptors of the two tiles (the fused blocks derive the rest)
        const uint64_t q0d = ((uint64_t)kHi << 32) | q_lo;
        const uint64_t q1d = ((uint64_t)kHi << 32) | (q_lo + kTileStep);
        // K-major 128-row operand (a Q or K tile): 16 columns per K-step
        auto kmajor = [&](uint32_t lo, uint64_t (&d)[NKQ]) {
#pragma unroll
            for (int kk = 0; kk < NKQ; ++kk)
                d[kk] = ((uint64_t)kHi << 32) |
                        (lo + (((kk >> 2) * Cfg::kGroupBytes + (kk & 3) * 32) >> 4));
        };
        // MN-major V tile: 16 keys (2048 bytes) per K-step
        auto vmajor = [&](uint32_t lo, uint64_t (&d)[8]) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) d[kk] = ((uint64_t)kHi << 32) | (lo + kk * (2048 >> 4));
        };
        // TMEM addresses of P (the PV A operand) of tile x
        auto ptmem = [&](int x, uint32_t (&d)[8]) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) d[kk] = tmem + Cfg::col_s(x) + kk * 8;
        };
        // bias step operands: tile x's Q side (every 8-row group reads the
        // same core matrix: stride 0), the key-column side (8-key groups 256
        // bytes apart); each K-step's second core matrix 128 bytes on
        const uint32_t sm_ext = smem_u32(smem + Cfg::kOffExt);
        auto qxd = [&](int x) {
            return ((uint64_t)umma_desc_hi_none(0) << 32) | umma_desc_lo(sm_ext + x * 256, 128);
        };
        auto kxd = [&]() {
            return ((uint64_t)umma_desc_hi_none(256) << 32) | umma_desc_lo(sm_ext + 512, 128);
        };
        auto qk = [&](int x, const uint64_t (&qd)[NKQ], const uint64_t (&kd)[NKQ]) {
            if constexpr (NKQ == 8) umma_ss_x8(tmem + Cfg::col_s(x), qd, kd, IDESC_QK, 0u);
            else umma_ss_x4(tmem + Cfg::col_s(x), qd, kd, IDESC_QK, 0u);
            if constexpr (XB) umma_ss(tmem + Cfg::col_s(x), qxd(x), kxd(), IDESC_QK, 1u);
        };
        // At the last key tile of an item whose two tiles end together, the
        // next item's first QK_0 goes out right after PV_0 instead of after
        // tile 1's last P, so tile 0's softmax warps can start the next item
        // (its epilogue follows that item's first tile).  Its inputs cannot
        // wait on anything issued later: the next Q was requested once this
        // item's last QK finished, and the next K tile takes the stage of
        // K(nB - 2), freed before that.  (int8: the converted Q has its own
        // barrier; not done there.)  Returns false if a wait gave up.
        auto qk0_next = [&](const PairGeom &g0, uint64_t (&qd)[NKQ], uint64_t (&kd)[NKQ]) -> bool {
            if constexpr (!DEFER) return true;
            if (idx + 1 >= it_end) return true;
            const PairGeom gn = pair_geom<BAND>(a, items, seqs, idx + 1);
            if (gn.nB == 0 || gn.nA == 0) return true;
            if (XB && gn.nA != gn.nB) return true;      // its tile 0 starts later
            const uint32_t k0 = kv_it + g0.nB;
            const int ks0 = k0 % KS;
            kmajor(k_lo + ks0 * kTileStep, kd);
            if (!mbar_wait(q_full, q_it & 1, abort_flag, a.c.err, 20, a.c.wait_ns)) return false;
            if (!mbar_wait(&k_full[ks0], (k0 / KS) & 1, abort_flag, a.c.err, 21, a.c.wait_ns))
                return false;
            tc_fence_after();
            kmajor(q_lo, qd);
            qk(0, qd, kd);
            umma_commit(&s_full[0]);
            qk0_early = true;
            return true;
        };
        static_assert(kPrefillBN / 16 == 8, "PV issue assumes 8 key steps per tile");
        static_assert(NKQ == 4 || NKQ == 8, "QK issue assumes D = 64 or 128");
        for (idx = it_begin; idx < it_end; ++idx) {
            const PairGeom gm = pair_geom<BAND>(a, items, seqs, idx);
            if (gm.nB == 0) continue;
            dbg_j = -1;
            // descriptors are rebuilt before each wait rather than kept live:
            // registers are scarce (96 per thread) and the softmax roles need them
            uint64_t qd[NKQ], kd[NKQ], vd[8];
            uint32_t pa[8];
            FIA_WAIT(I8 ? q_conv : q_full, q_it & 1, 20);
            ++q_it;
            const uint32_t kv_base = kv_it;
            // Tile 0 takes part in iterations [a0, a0 + nA).  Key tiles run
            // first to last (a0 = 0), or in the ALiBi-through-MMA mode last to
            // first, where tile 0's fewer key tiles are the last iterations:
            // the diagonal tile, whose bias is the largest, then fixes the
            // running maximum and the lazy O rescale is rarely needed.
            const int a0 = XB ? gm.nB - gm.nA : 0;
            auto t0_on = [&](int jj) { return jj >= a0 && jj < a0 + gm.nA; };
            {
                // QK for key tile 0 (both tiles)
                const int ks = kv_base % KS;
                kmajor(k_lo + ks * kTileStep, kd);
                FIA_WAIT(&k_full[ks], (kv_base / KS) & 1, 21);
                tc_fence_after();
                if (gm.nA > 0 && a0 == 0 && !qk0_early) {
                    kmajor(q_lo, qd);
                    qk(0, qd, kd);
                    umma_commit(&s_full[0]);
                }
                qk0_early = false;
                kmajor(q_lo + kTileStep, qd);
                qk(1, qd, kd);
                umma_commit(&s_full[1]);
                umma_commit(&k_empty[ks]);
                if (gm.nB == 1) umma_commit(q_empty);
            }
            for (int j = 0; j < gm.nB; ++j) {
                dbg_j = j;
                const uint32_t kvi = kv_base + j;
                const int vs = kvi % VS;
                const bool more = (j + 1 < gm.nB);
                const uint32_t kn = kv_base + j + 1;
                const int ksn = kn % KS;
                vmajor(v_lo + vs * kTileStep, vd);
                kmajor(k_lo + ksn * kTileStep, kd);
                FIA_WAIT(&v_full[vs], (kvi / VS) & 1, 24);
                const int valid = gm.kvlen - (XB ? gm.j0 + gm.nB - 1 - j : gm.j0 + j) * kPrefillBN;
                if (!I8 && valid < kPrefillBN) {     // (int8: the converters write the zeros)
                    // rows past kvSeqLen: P is 0 there, but the slots may hold
                    // anything (NaN * 0 = NaN in the MMA): the bulk-copy engine
                    // writes zeros over them after the V tile has landed.
                    uint8_t *vdst = smem + Cfg::kOffV + vs * Cfg::kTileBytes;
                    const uint32_t nbytes = (uint32_t)(kPrefillBN - valid) * 128u;
                    mbar_arrive_expect_tx(vz_full, nbytes * Cfg::kHalves);
                    for (int hv = 0; hv < Cfg::kHalves; ++hv)
                        bulk_load(vdst + hv * Cfg::kGroupBytes + valid * 128, g_zero_rows, nbytes,
                                  vz_full);
                    ++req_vz;
                    FIA_WAIT(vz_full, seen_vz & 1, 27);
                    ++seen_vz;
                }
                if constexpr (KS >= 2) {
                    // Every wait comes before a block, so each tile's PV(j) and
                    // QK(j+1) go out back to back.  K(j+1) was requested a whole
                    // key tile earlier: waiting for it up front almost never waits.
                    // QK_X(j+1) is issued after PV_X(j), so its S-ready commit also
                    // tells the softmax warps that PV_X(j) is done with O.
                    if (more) FIA_WAIT(&k_full[ksn], (kn / KS) & 1, 22);
                    if (t0_on(j)) {
                        FIA_WAIT(&p_full[0], p_it[0] & 1, 23);
                        ++p_it[0];
                        tc_fence_after();
                        const uint32_t acc0 = j > a0 ? 1u : 0u;
                        if constexpr (NKQ == 8) {
                            if (t0_on(j + 1)) {
                                if constexpr (XB)
                                    umma_pv_qk_x(tmem + Cfg::col_o(0), tmem + Cfg::col_s(0), vd[0],
                                                 IDESC_PV, acc0, tmem + Cfg::col_s(0),
                                                 q0d, kd[0], IDESC_QK, qxd(0), kxd(), &s_full[0]);
                                else
                                    umma_pv_qk(tmem + Cfg::col_o(0), tmem + Cfg::col_s(0), vd[0],
                                               IDESC_PV, acc0, tmem + Cfg::col_s(0), q0d,
                                               kd[0], IDESC_QK, &s_full[0]);
                            } else {
                                ptmem(0, pa);
                                umma_ts_x8(tmem + Cfg::col_o(0), pa, vd, IDESC_PV, acc0);
                                umma_commit(&o_full[0]);
                                if (!more && !qk0_next(gm, qd, kd)) {
                                    fail_trail(a.c.err, 20, (uint32_t)idx, (uint32_t)dbg_j, q_it & 1, q_full);
                                    goto done;
                                }
                            }
                        } else {
                            ptmem(0, pa);
                            kmajor(q_lo, qd);
                            umma_ts_x8(tmem + Cfg::col_o(0), pa, vd, IDESC_PV, acc0);
                            if (t0_on(j + 1)) {
                                qk(0, qd, kd);
                                umma_commit(&s_full[0]);
                            } else {
                                umma_commit(&o_full[0]);
                                if (!more && !qk0_next(gm, qd, kd)) {
                                    fail_trail(a.c.err, 20, (uint32_t)idx, (uint32_t)dbg_j, q_it & 1, q_full);
                                    goto done;
                                }
                            }
                        }
                    } else if (t0_on(j + 1)) {
                        // tile 0's first key tile is the next one (reverse order)
                        tc_fence_after();
                        kmajor(q_lo, qd);
                        qk(0, qd, kd);
                        umma_commit(&s_full[0]);
                    }
                    FIA_WAIT(&p_full[1], p_it[1] & 1, 25);
                    ++p_it[1];
                    tc_fence_after();
                    if (NKQ == 8 && more) {
                        if constexpr (XB)
                            umma_pv_qk_x(tmem + Cfg::col_o(1), tmem + Cfg::col_s(1), vd[0], IDESC_PV,
                                         j > 0 ? 1u : 0u, tmem + Cfg::col_s(1), q1d, kd[0], IDESC_QK,
                                         qxd(1), kxd(), &s_full[1]);
                        else
                            umma_pv_qk(tmem + Cfg::col_o(1), tmem + Cfg::col_s(1), vd[0], IDESC_PV,
                                       j > 0 ? 1u : 0u, tmem + Cfg::col_s(1), q1d, kd[0], IDESC_QK,
                                       &s_full[1]);
                    } else {
                        ptmem(1, pa);
                        kmajor(q_lo + kTileStep, qd);
                        umma_ts_x8(tmem + Cfg::col_o(1), pa, vd, IDESC_PV, j > 0 ? 1u : 0u);
                        if (more) {
                            qk(1, qd, kd);
                            umma_commit(&s_full[1]);
                        }
                    }
                    umma_commit(&v_empty[vs]);
                    if (more) {
                        umma_commit(&k_empty[ksn]);
                        if (j + 1 == gm.nB - 1) umma_commit(q_empty);
                    } else {
                        umma_commit(&o_full[1]);
                    }
                } else {
                    // One K stage: K(j+1) is loaded only after QK(j) of both
                    // tiles, so it is waited for between the PV and QK blocks.
                    if (j < gm.nA) {
                        ptmem(0, pa);
                        kmajor(q_lo, qd);
                        FIA_WAIT(&p_full[0], p_it[0] & 1, 23);
                        ++p_it[0];
                        tc_fence_after();
                        umma_ts_x8(tmem + Cfg::col_o(0), pa, vd, IDESC_PV, j > 0 ? 1u : 0u);
                        if (j == gm.nA - 1) umma_commit(&o_full[0]);
                        if (j + 1 < gm.nA) {
                            FIA_WAIT(&k_full[ksn], (kn / KS) & 1, 22);
                            tc_fence_after();
                            qk(0, qd, kd);
                            umma_commit(&s_full[0]);
                        }
                    }
                    ptmem(1, pa);
                    kmajor(q_lo + kTileStep, qd);
                    FIA_WAIT(&p_full[1], p_it[1] & 1, 25);
                    ++p_it[1];
                    tc_fence_after();
                    umma_ts_x8(tmem + Cfg::col_o(1), pa, vd, IDESC_PV, j > 0 ? 1u : 0u);
                    umma_commit(&v_empty[vs]);
                    if (j == gm.nB - 1) umma_commit(&o_full[1]);
                    if (more) {
                        FIA_WAIT(&k_full[ksn], (kn / KS) & 1, 26);
                        tc_fence_after();
                        qk(1, qd, kd);
                        umma_commit(&s_full[1]);
                        umma_commit(&k_empty[ksn]);
                        if (j + 1 == gm.nB - 1) umma_commit(q_empty);
                    }
                }
            }
            kv_it = kv_base + gm.nB;
        }
    } else if (!I8 || warp < 18) {
        // ------------------------------------------------------------ softmax + epilogue
        // 8 warps per tile: warp (quadrant q, sub-block u) owns query rows
        // 32q + 16u .. +15 (TMEM lanes); lane t holds row 32q + 16u + (t & 15)
        // and key columns 64h .. 64h + 63 of S with h = t >> 4.
        const int sw = warp - 2;
        const int X = sw >> 3;                     // which tile of the pair
        const int sub = (sw >> 2) & 1;             // which 16 rows of the quadrant
        const int quad = warp & 3;
        const int half = lane >> 4;                // which 64 key columns (per lane)
        const int row = quad * 32 + sub * 16 + (lane & 15);
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32 + sub * 16) << 16);
        const uint32_t scol = t_lane + Cfg::col_s(X);                  // S (+64 for h = 1)
        constexpr int DH = D / 2;                                      // O columns per lane
        const uint32_t ocol = t_lane + Cfg::col_o(X);                  // O (+DH for h = 1)
        const bool causal = (a.c.mask_type == 9 || a.c.mask_type == 3);
        const float sl2 = a.c.scale_log2;
        // plain mode with a positive scale: mask raw scores and fold the scale
        // into the exponent (one FFMA per element)
        const bool fold = (MODE == kModePlain || MODE == kModePlainGqa || XB) && (sl2 > 0.f);
        uint32_t s_it = 0, p_it = 0, o_it = 0;
        T *outp = reinterpret_cast<T *>(a.c.out);
        const bool pse_tma = (MODE == kModePse) && a.c.pse_tma;
        uint8_t *pslot = smem + Cfg::kOffPse + sw * 4096;
        uint64_t *pbar = &pse_full[sw];
        // lane 0 fetches this warp's two pse boxes (16 rows x 64 keys each) of
        // the item's key tile jt (counted from its first key tile j0)
        auto pse_fetch = [&](const PairGeom &g2, const SubGeom &s2, int jt) {
            if (lane == 0) {
                ++req_ps;
                mbar_arrive_expect_tx(pbar, 4096);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    tma_load_3d(pslot + hh * 2048, &tp, pbar, (g2.j0 + jt) * kPrefillBN + 64 * hh,
                                s2.q0 + 32 * quad + 16 * sub, g2.b * a.c.H + s2.h);
            }
        };

        // Epilogue of a finished item -- O / l (+ sink), lse; each lane writes
        // D/2 columns -- from the state the item left (ep_h < 0: none pending).
        // DEFER: it runs after the next item's first P is in TMEM and before
        // that P is signalled: the PV that overwrites O waits for the signal,
        // and the softmax of the new item's first tile overlaps the wait for
        // the old item's last PV instead of following the epilogue.  Returns
        // false if the wait for that PV gave up (the caller takes the error exit).
        float ep_m = 0.f, ep_l = 0.f;
        int ep_row = -1, ep_h = -1, ep_kvh = 0;
        auto epilogue = [&]() -> bool {
            const bool got = mbar_wait(&o_full[X], o_it & 1, abort_flag, a.c.err, 32, a.c.wait_ns);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) fail_trail(a.c.err, 32, (uint32_t)idx, (uint32_t)dbg_j, o_it & 1, &o_full[X]);
                tmem_st_wait();
                return false;
            }
            ++o_it;
            __syncwarp();
            tc_fence_after();
            const float mu = (ep_m == -INFINITY) ? 0.f : ep_m;
            float M = mu, lt = ep_l;
            if (a.c.sink) {
                const float s2 = a.c.sink[ep_h] * kLog2e;
                M = fmaxf(mu, s2);
                lt = ep_l * ex2(mu - M) + ex2(s2 - M);
            }
            // a row with no visible key (possible under a band mask): out 0,
            // lse +inf, with or without a sink
            const bool no_key = BAND && (ep_m == -INFINITY);
            const float oscale = no_key ? 0.f : ex2(mu - M) / lt;
            const int64_t orow = (int64_t)ep_row * a.c.H + ep_h;
#pragma unroll
            for (int cc = 0; cc < DH / 32; ++cc) {
                uint32_t orr[32];
                tmem_ld16x2_32<DH>(ocol + cc * 32, orr);
                tmem_ld_wait();
                reg_fence32(orr);
                if (ep_row >= 0) {
                    uint32_t pk[16];
                    if (I8 && a.v_mode == 0) {
                        // per-channel V: the widened values carry the offset; the
                        // scale multiplies each output channel here
                        const float *vsc = a.v_scale + ep_kvh * D + DH * half + cc * 32;
#pragma unroll
                        for (int x = 0; x < 16; ++x)
                            pk[x] = pack2<T>(__uint_as_float(orr[2 * x]) * (oscale * __ldg(vsc + 2 * x)),
                                             __uint_as_float(orr[2 * x + 1]) *
                                                 (oscale * __ldg(vsc + 2 * x + 1)));
                    } else {
#pragma unroll
                        for (int x = 0; x < 16; ++x)
                            pk[x] = pack2<T>(__uint_as_float(orr[2 * x]) * oscale,
                                             __uint_as_float(orr[2 * x + 1]) * oscale);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(outp + orow * D + DH * half + cc * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
                __syncwarp();
            }
            if (ep_row >= 0 && a.c.lse && half == 0)
                a.c.lse[orow] = no_key ? INFINITY : (M + log2f(lt)) * kLn2;
            tc_fence_before();
            __syncwarp();
            ep_h = -1;
            return true;
        };

        // test hook: wait on a barrier nothing signals, so the bounded wait
        // gives up and the whole CTA takes the error exit
        if (a.c.stall) FIA_WAIT_W(never, 0, 35);
        for (idx = it_begin; idx < it_end; ++idx) {
            const PairGeom gm = pair_geom<BAND>(a, items, seqs, idx);
            const SubGeom sg = gm.t[X];
            if (!sg.valid) continue;
            const int i = sg.q0 + row;
            const bool valid = i < gm.qlen;
            const int qpos = gm.kvlen - gm.qlen + i;
            // under a band mask the keys this row may see are [klo, khi)
            int klo = 0, khi = gm.kvlen;
            if constexpr (BAND) {
                klo = max(0, qpos - a.c.pre);
                khi = min(khi, qpos + a.c.next + 1);
            }
            const int64_t orow = ((int64_t)(gm.cu_q + i) * a.c.H + sg.h);
            if (sg.n == 0) {
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(outp + orow * D + DH * half);
                    for (int x = 0; x < DH * 2 / 16; ++x) dst[x] = make_uint4(0, 0, 0, 0);
                    if (a.c.lse && half == 0) a.c.lse[orow] = INFINITY;
                }
                __syncwarp();
                continue;
            }
            float slope2 = 0.f;
            if constexpr (MODE == kModeAlibi || XB) slope2 = a.c.slopes[sg.h] * kLog2e;
            const T *pse_row = nullptr;
            if constexpr (MODE == kModePse) {
                // rows past seqLen read row 0 of the sequence (their output is dropped)
                pse_row = reinterpret_cast<const T *>(a.c.pse) +
                          (((int64_t)gm.b * a.c.H + sg.h) * a.c.pse_q + (valid ? i : 0)) * a.c.pse_kv;
            }
            float m = -INFINITY, l = 0.f;
            if (pse_tma) pse_fetch(gm, sg, 0);
            for (int j = 0; j < sg.n; ++j) {
                dbg_j = j;
                // this tile's key tile (last to first in the ALiBi-through-MMA mode)
                const int kt = XB ? gm.j0 + sg.n - 1 - j : gm.j0 + j;
                const int tb = kt * kPrefillBN + 64 * half;            // first key of this lane
                FIA_WAIT_W(&s_full[X], s_it & 1, 30);
                ++s_it;
                __syncwarp();          // tcgen05.ld/st below are warp-collective (.aligned)
                tc_fence_after();
                uint32_t sr[2][32];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) tmem_ld16x2_32<64>(scol + cc * 32, sr[cc]);
                tmem_ld_wait();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) reg_fence32(sr[cc]);

                // ---- scores (log2 units unless folded), bias, masks ----
                const bool edge = BAND ? (tb < klo) || (tb + 64 > khi)
                                       : (tb + 64 > gm.kvlen) || (causal && tb + 63 > qpos);
                if constexpr (MODE == kModeAlibi) {
                    // bias slope * (t - qpos) in log2 units, two keys at a time:
                    // every 8 keys the bias pair is one rounding of slope times
                    // the exact key offsets (integers below 2^24), and in between
                    // it steps by 2 slope (at most three roundings of drift,
                    // < 4e-4 in log2 units for |bias| < 2^12)
                    const float t0 = (float)(tb - qpos);
                    const uint64_t sp2 = f2pack(slope2, slope2), sl2x2 = f2pack(sl2, sl2);
                    const uint64_t eight2 = f2pack(8.f, 8.f);
                    const float st = 2.f * slope2;
                    const uint64_t step2 = f2pack(st, st);
                    uint64_t off2 = f2pack(t0, t0 + 1.f);
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                        for (int x4 = 0; x4 < 4; ++x4) {
                            uint64_t b2 = fmul2(sp2, off2);
                            off2 = fadd2(off2, eight2);
#pragma unroll
                            for (int x1 = 0; x1 < 4; ++x1) {
                                const int x = 4 * x4 + x1;
                                const uint64_t s2 = f2pack(__uint_as_float(sr[cc][2 * x]),
                                                           __uint_as_float(sr[cc][2 * x + 1]));
                                const uint64_t y2 = ffma2(s2, sl2x2, b2);
                                float y0, y1;
                                f2unpack(y2, y0, y1);
                                sr[cc][2 * x] = __float_as_uint(y0);
                                sr[cc][2 * x + 1] = __float_as_uint(y1);
                                if (x1 < 3) b2 = fadd2(b2, step2);
                            }
                        }
                } else if (MODE == kModePse && pse_tma) {
                    // this lane's row of pse box `half` for tile j (128-byte swizzle)
                    FIA_WAIT_W(pbar, seen_ps & 1, 34);
                    ++seen_ps;
                    const int r16 = lane & 15;
                    const uint32_t prow = smem_u32(pslot) + half * 2048 + r16 * 128;
#pragma unroll
                    for (int c16 = 0; c16 < 8; ++c16) {
                        uint32_t w4[4];
                        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3])
                                     : "r"(prow + ((c16 ^ (r16 & 7)) << 4)));
                        const T *pv = reinterpret_cast<const T *>(w4);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int col = c16 * 8 + e;
                            const float bias = to_f32<T>(pv[e]) * kLog2e;
                            sr[col >> 5][col & 31] = __float_as_uint(
                                fmaf(__uint_as_float(sr[col >> 5][col & 31]), sl2, bias));
                        }
                    }
                    // the slot is free: fetch the next tile's boxes (generic-proxy
                    // reads ordered before the async-proxy write)
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (j + 1 < sg.n) pse_fetch(gm, sg, j + 1);
                } else if constexpr (MODE == kModePse) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
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
                                    pv[e] = (t + e < gm.kvlen) ? pse_row[t + e] : pse_row[0];
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
                    for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            sr[cc][x] = __float_as_uint(__uint_as_float(sr[cc][x]) * sl2);
                }
                if (edge) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                        for (int x = 0; x < 32; ++x) {
                            const int t = tb + cc * 32 + x;
                            const bool keep = BAND ? (t >= klo) && (t < khi)
                                                   : (t < gm.kvlen) && !(causal && t > qpos);
                            if (!keep) sr[cc][x] = __float_as_uint(-INFINITY);
                        }
                }
                // tree max over this lane's 64 columns, then with lane t ^ 16
#define FIA_EL(e) __uint_as_float(sr[(e) >> 5][(e) & 31])
                float mx4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) mx4[k] = fmaxf(FIA_EL(k), FIA_EL(k + 4));
#pragma unroll
                for (int e = 8; e < 64; e += 8)
#pragma unroll
                    for (int k = 0; k < 4; ++k) mx4[k] = fmax3(mx4[k], FIA_EL(e + k), FIA_EL(e + 4 + k));
#undef FIA_EL
                float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                if (fold) mx = (mx == -INFINITY) ? -INFINITY : mx * sl2;
                // bias step mode: S holds slope * (t - t0) of the tile's first key
                // t0; slope * (t0 - qpos) is the same for the whole row of the tile
                float cb = 0.f;
                if constexpr (XB) {
                    cb = slope2 * (float)(kt * kPrefillBN - qpos);
                    mx += cb;
                }

                // running max: exact on the first tile, afterwards raised only
                // when it grows by more than 2^8 (O and l stay consistent with m)
                const float m_new = fmaxf(m, mx);
                bool need = false;
                float alpha = 1.0f;
                if (j == 0 || m == -INFINITY) {
                    // (no key seen yet: O and l are exact zeros, nothing to rescale)
                    m = m_new;
                } else if (m_new > m + 8.0f) {
                    need = true;
                    alpha = ex2(m - m_new);
                    m = m_new;
                    l *= alpha;
                }
                const float mu = (m == -INFINITY) ? 0.f : m;

                // P = 2^(s - m) in the input dtype over this lane's half row
                const uint64_t negmu2 = f2pack(cb - mu, cb - mu);
                const uint64_t sl2x2 = f2pack(sl2, sl2);
                uint64_t acc2[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) acc2[k] = f2pack(0.f, 0.f);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint32_t pk[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const uint64_t s2 = f2pack(__uint_as_float(sr[cc][2 * x]),
                                                   __uint_as_float(sr[cc][2 * x + 1]));
                        const uint64_t xx = fold ? ffma2(s2, sl2x2, negmu2) : fadd2(s2, negmu2);
                        float a0, a1;
                        f2unpack(xx, a0, a1);
                        const uint64_t pp = f2pack(ex2(a0), ex2(a1));
                        acc2[x & 3] = fadd2(acc2[x & 3], pp);
                        float p0, p1;
                        f2unpack(pp, p0, p1);
                        pk[x] = pack2<MT>(p0, p1);
                    }
                    // packed P columns 32h + 16cc .. +15 (keys 64h + 32cc ..)
                    tmem_st16x2_16<32>(scol + cc * 16, pk);
                }
                {
                    const uint64_t s01 = fadd2(fadd2(acc2[0], acc2[1]), fadd2(acc2[2], acc2[3]));
                    float l0, l1;
                    f2unpack(s01, l0, l1);
                    l += l0 + l1;
                }

                // Rescale this lane's half of its O row (rare).  The previous PV
                // of this tile must be done with O first.  (The softmax warps
                // cannot drift apart: S for the next key tile is only produced
                // after all eight warps have signalled this P.)
                // (S of tile j was written by QK(j), which the issuer put after
                // PV(j - 1): that PV is done with O.)
                if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int cc = 0; cc < DH / 32; ++cc) {
                        uint32_t orr[32];
                        tmem_ld16x2_32<DH>(ocol + cc * 32, orr);
                        tmem_ld_wait();
                        reg_fence32(orr);
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            orr[x] = __float_as_uint(__uint_as_float(orr[x]) * alpha);
                        tmem_st16x2_32<DH>(ocol + cc * 32, orr);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (DEFER && j == 0 && ep_h >= 0 && !epilogue()) goto done;
                if (lane == 0) mbar_arrive(&p_full[X]);
                ++p_it;
            }

            // DEFER: the item's epilogue runs inside the next item's first key
            // tile (or after the last item); its state waits here
            dbg_j = sg.n;
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            ep_m = m;
            ep_l = l;
            ep_row = valid ? gm.cu_q + i : -1;
            ep_h = sg.h;
            ep_kvh = gm.kvh;
            // (pairs that do not end both tiles together -- never in the
            // deferring instances' plans -- take the epilogue at once)
            if (!DEFER || (!BAND && !XB && gm.nA != gm.nB)) {
                if (!epilogue()) goto done;
            }
        }
        if (DEFER && ep_h >= 0 && !epilogue()) goto done;
    } else if constexpr (I8) {
        // ------------------------------------------------------------ int8 converters
        // Eight consecutive threads take eight consecutive rows of one 16-byte
        // chunk, so the swizzled loads and stores of a quarter warp hit
        // distinct banks.  K runs one tile ahead of V -- K(0), K(1), V(0),
        // K(2), V(1), ... -- since the issuer wants V(j) and K(j + 1) together
        // and the K stage frees a whole tile earlier than the single V stage.
        const int u = tid - 18 * 32;
        const int rl = u & 7;
        const int c = u >> 3;
        uint32_t rk_it = 0, rv_it = 0, k_it = 0, v_it = 0, q_it = 0;
        for (idx = it_begin; idx < it_end; ++idx) {
            const PairGeom gm = pair_geom<BAND>(a, items, seqs, idx);
            if (gm.nB > 0) {
                // the pair's Q tiles, in place, to f16 (times the per-channel
                // K scale); each warp converts half of the rows
                dbg_j = -1;
                FIA_WAIT_C(q_full, q_it & 1, 44);
                ++q_it;
                const float *ksc = a.k_mode == 0 ? a.k_scale + gm.kvh * D : nullptr;
#pragma unroll 1
                for (int x = 0; x < 2; ++x)
                    if (gm.t[x].valid) q_to_f16<T>(smem + Cfg::kOffQ + x * Cfg::kTileBytes, u, ksc);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(q_conv);
            }
            for (int s = 0; s <= gm.nB; ++s) {
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    const bool is_v = (h == 1);
                    const int j = is_v ? s - 1 : s;
                    if (j < 0 || j >= gm.nB) continue;
                    dbg_j = j;
                    const int t0 = (gm.j0 + j) * kPrefillBN;
                    const int valid = min(kPrefillBN, gm.kvlen - t0);
                    const uint32_t rit = is_v ? rv_it : rk_it;
                    const uint32_t sit = is_v ? v_it : k_it;
                    const int nst = is_v ? VS : KS;
                    uint64_t *rfull = (is_v ? rv_full : rk_full) + rit % RS;
                    uint64_t *rempty = (is_v ? rv_empty : rk_empty) + rit % RS;
                    uint64_t *dfull = (is_v ? v_full : k_full) + sit % nst;
                    uint64_t *dempty = (is_v ? v_empty : k_empty) + sit % nst;
                    FIA_WAIT_C(dempty, ((sit / nst) & 1) ^ 1, is_v ? 43 : 41);
                    FIA_WAIT_C(rfull, (rit / RS) & 1, is_v ? 42 : 40);
                    const uint8_t *raw =
                        smem + Cfg::kOffRaw + ((is_v ? RS : 0) + rit % RS) * Cfg::kRawBytes;
                    uint8_t *dst = smem + (is_v ? Cfg::kOffV : Cfg::kOffK) + (sit % nst) * Cfg::kTileBytes;
                    const bool tok = is_v ? a.v_mode != 0 : a.k_mode != 0;
                    const float *sc = is_v ? a.v_scale : a.k_scale;
                    const float *of = is_v ? a.v_offset : a.k_offset;
                    if (tok) {
                        // per token: (x + offset) * scale in f16
                        const int64_t row0 = (int64_t)gm.b * (is_v ? a.v_tok_stride : a.k_tok_stride) + t0;
                        if (valid == kPrefillBN)
                            dequant_tile<MT, true, true>(raw, dst, rl, c, valid, sc + row0,
                                                         of ? of + row0 : nullptr);
                        else
                            dequant_tile<MT, true, false>(raw, dst, rl, c, valid, sc + row0,
                                                          of ? of + row0 : nullptr);
                    } else {
                        // per channel: x + offset exactly widened; the scale is
                        // folded into Q (keys) or applied in the epilogue (values)
                        const int ch0 = gm.kvh * D + 16 * c;
                        // (one instance per tile shape: a null offset adds zeros)
                        const float *ofc = of ? of + ch0 : nullptr;
                        if (valid == kPrefillBN) widen_tile<true, true>(raw, dst, rl, c, valid, ofc);
                        else widen_tile<false, true>(raw, dst, rl, c, valid, ofc);
                    }
                    // the MMAs (async proxy) read what was stored here, and TMA
                    // refills the raw stage that was read here
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(dfull);
                        mbar_arrive(rempty);
                    }
                    if (is_v) { ++rv_it; ++v_it; } else { ++rk_it; ++k_it; }
                }
            }
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    // Error exit: every role has left its loop, so the flag is final here.
    // Wait for what may still be in flight -- the producer's latest copy into
    // each ring stage (earlier ones completed before their stage was requested
    // again), the issuer's MMAs and zero-row copy, a softmax warp's prefetched
    // pse boxes -- before shared memory and TMEM are released.
    if (*abort_flag) {
        if (warp == 0 && lane == 0) {
            if (req_q > 0) mbar_wait_drain(q_full, (req_q - 1) & 1);
            if constexpr (I8) {
                for (uint32_t i = (req_k > RS ? req_k - RS : 0u); i < req_k; ++i)
                    mbar_wait_drain(&rk_full[i % RS], (i / RS) & 1);
                for (uint32_t i = (req_v > RS ? req_v - RS : 0u); i < req_v; ++i)
                    mbar_wait_drain(&rv_full[i % RS], (i / RS) & 1);
            } else {
                for (uint32_t i = (req_k > KS ? req_k - KS : 0u); i < req_k; ++i)
                    mbar_wait_drain(&k_full[i % KS], (i / KS) & 1);
                for (uint32_t i = (req_v > VS ? req_v - VS : 0u); i < req_v; ++i)
                    mbar_wait_drain(&v_full[i % VS], (i / VS) & 1);
            }
        } else if (warp == 1 && lane == 0) {
            umma_commit(mma_drain);
            mbar_wait_drain(mma_drain, 0);
            if (req_vz > seen_vz) mbar_wait_drain(vz_full, seen_vz & 1);
        } else if (warp >= 2 && lane == 0 && req_ps > seen_ps) {
            mbar_wait_drain(&pse_full[warp - 2], seen_ps & 1);
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 1) {
        __syncwarp();          // lanes 1-31 left the issuer role early; dealloc is .aligned
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

template <typename T, int D, int MODE, bool BAND, bool I8>
static cudaError_t launch_prefill_t(const PrefillArgs &a, const CUtensorMap &tq,
                                    const CUtensorMap &tk, const CUtensorMap &tv,
                                    const CUtensorMap &tp, int grid,
                                    const uint8_t *inline_plan, cudaStream_t s) {
    using Cfg = PrefillCfg<D, MODE, I8>;
    const int smem = Cfg::kSmem;
    if (inline_plan) {
        auto kern = fia_prefill_kernel<T, D, MODE, kInlinePlanBytes, BAND, I8>;
        cudaError_t e =
            ensure_smem_attr<fia_prefill_kernel<T, D, MODE, kInlinePlanBytes, BAND, I8>>(smem);
        if (e != cudaSuccess) return e;
        // inline_plan points at a full PlanBytes<kInlinePlanBytes> kept by the op
        kern<<<grid, Cfg::kThreads, smem, s>>>(
            a, tq, tk, tv, tp, *reinterpret_cast<const PlanBytes<kInlinePlanBytes> *>(inline_plan));
    } else {
        auto kern = fia_prefill_kernel<T, D, MODE, 16, BAND, I8>;
        cudaError_t e = ensure_smem_attr<fia_prefill_kernel<T, D, MODE, 16, BAND, I8>>(smem);
        if (e != cudaSuccess) return e;
        PlanBytes<16> pl{};
        kern<<<grid, Cfg::kThreads, smem, s>>>(a, tq, tk, tv, tp, pl);
    }
    return cudaGetLastError();
}

template <typename T, int D, bool I8>
static cudaError_t launch_prefill_mode(const PrefillArgs &a, const CUtensorMap &tq,
                                       const CUtensorMap &tk, const CUtensorMap &tv,
                                       const CUtensorMap &tp, int grid, const uint8_t *ip,
                                       cudaStream_t s) {
    // a band mask excludes maskType (no causal, no ALiBi): its own instances
    // keep the band's range checks out of the other kernels
    if (a.c.band) {
        if (a.c.mask_type != 0) return cudaErrorInvalidValue;
        if (a.c.pse) return launch_prefill_t<T, D, kModePse, true, I8>(a, tq, tk, tv, tp, grid, ip, s);
        return launch_prefill_t<T, D, kModePlain, true, I8>(a, tq, tk, tv, tp, grid, ip, s);
    }
    if (a.c.pse) return launch_prefill_t<T, D, kModePse, false, I8>(a, tq, tk, tv, tp, grid, ip, s);
    if (a.c.mask_type == 3) {
        if constexpr (!I8) {
            if (a.c.scale_log2 > 0.f)
                return launch_prefill_t<T, D, kModeAlibiMma, false, I8>(a, tq, tk, tv, tp, grid, ip, s);
        }
        return launch_prefill_t<T, D, kModeAlibi, false, I8>(a, tq, tk, tv, tp, grid, ip, s);
    }
    if constexpr (!I8) {
        if (a.c.g >= 2) return launch_prefill_t<T, D, kModePlainGqa, false, I8>(a, tq, tk, tv, tp, grid, ip, s);
    }
    return launch_prefill_t<T, D, kModePlain, false, I8>(a, tq, tk, tv, tp, grid, ip, s);
}

cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &tq, const CUtensorMap &tk,
                           const CUtensorMap &tv, const CUtensorMap &tp, int q_dtype, bool kv_int8,
                           int grid, const uint8_t *inline_plan, cudaStream_t s) {
    const bool bf = (q_dtype == 1);
    if (kv_int8) {
        if (a.c.D != 128) return cudaErrorInvalidValue;
        return bf ? launch_prefill_mode<__nv_bfloat16, 128, true>(a, tq, tk, tv, tp, grid, inline_plan, s)
                  : launch_prefill_mode<__half, 128, true>(a, tq, tk, tv, tp, grid, inline_plan, s);
    }
    if (a.c.D == 128)
        return bf ? launch_prefill_mode<__nv_bfloat16, 128, false>(a, tq, tk, tv, tp, grid, inline_plan, s)
                  : launch_prefill_mode<__half, 128, false>(a, tq, tk, tv, tp, grid, inline_plan, s);
    if (a.c.D == 64)
        return bf ? launch_prefill_mode<__nv_bfloat16, 64, false>(a, tq, tk, tv, tp, grid, inline_plan, s)
                  : launch_prefill_mode<__half, 64, false>(a, tq, tk, tv, tp, grid, inline_plan, s);
    return cudaErrorInvalidValue;
}

}  // namespace fia
