// chunk_state.cuh -- the sequential state pass of the chunked delta rule on the
// sm_100a tensor cores, fed by the per-chunk -W, u and P of chunk_wy.cu.
//
// Same mathematics as the chunkwise form of "Linear attention and Gated
// DeltaNet" (ch. 28, "The chunked form: recurrence as matrix multiplication";
// D2L 12.5, "Training it: the WY trick"): with W = T diag(beta e^G) K,
// u = T diag(beta) V and P = scale tril(Q K^T * D) of each chunk computed, and
// Qh = scale e^G Q,
//
//   U   = u - W S                                (values actually written)
//   O   = Qh S + P U
//   S  <- e^(G_last) S + (K * e^(G_last - G))^T U
//
// Every product runs as tcgen05.mma with M = 128 in transposed form (d_v is
// the MMA's M).  A tcgen05.mma costs the tensor pipe about the same time for
// any N up to 128, so the two products of the state share one MMA of N = 128:
//
//   [O^T | U^T] = S^T [Qh ; -W]^T   A = S^T (TMEM, bf16)  B = [Qh rows | -W rows] (smem)
//   U^T        += u^T               (epilogue)
//   S^T        += U~^T K            A = U~^T (TMEM, bf16) B = K tile (smem)
//   O^T        += U^T P^T           A = U^T (TMEM, bf16)  B = P (smem)
//
// with U~ = U * e^(G_last - G) (the decay of K folded into U's rows).  The CTA
// owns one (b, h); its state stays in TMEM (fp32 accumulator, pre-scaled by
// the next chunk's decay, plus a bf16 copy that feeds the next products), and
// [O | U] alternates between two TMEM buffers (one when the SM also hosts a WY
// group) so that the output of one chunk drains while the next one runs.  The U and state epilogues run in two
// halves with a barrier each, so that the tensor pipe starts on the first half
// of a contraction while the second is converted.  Warp roles: 0 TMA + gates,
// 2 TMEM allocation, 3 MMA issue, 4-7 Qh (in place over the q tile) and the
// output rows, 8-15 U and the state (two warps per TMEM lane quarter).  Stages
// of k, q, -W, u^T and P tiles arrive by TMA (128-byte swizzle) three chunks
// ahead.
//
// A partial last chunk has beta = 0, g = 0 past its end (rows past the
// tensor's end are zero-filled by TMA; rows of the next head are masked),
// which equals zero padding.  Every wait is bounded: on a timeout the kernel
// records it in the status word, lets its own copies land and exits.
#pragma once

#include "chunk_tc_common.cuh"

namespace dn {
namespace state {

using namespace sm100;
using namespace tc;

constexpr int kSideWarp0 = 4;     // Qh / output warps 4..7
constexpr int kSideThreads = 128;
constexpr int kChainWarp0 = 8;    // state warps 8 ..
// Warps of the state pass: 8 warps of producer, MMA issue and Qh / output rows, then the
// U and state epilogue warps, kNQ per TMEM lane quarter (each takes 1 / kNQ of a pass's
// columns).  With the per-key gate the pass shares its CTA shape with the KDA WY groups
// (16 warps), else it has 24.
// Alone on its SM (and without the per-key gate) a state pass has warps of its own that
// write the output rows (four; eight with the gated norm), so that the side warps only
// transform stages and run ahead.
template <int GATE, bool HOSTED = false, int PRO = 0>
struct Roles {
    static constexpr int kChainWarps = GATE == kGatePerKey ? 8 : 16;
    static constexpr bool kSplitOut = !HOSTED && GATE != kGatePerKey;
    static constexpr int kOutWarp0 = kChainWarp0 + kChainWarps;     // output warps (kSplitOut)
    static constexpr int kOutWarps = kSplitOut ? (PRO == 2 ? 8 : 4) : 0;
    static constexpr int kOutThreads = kSplitOut ? kOutWarps * 32 : kSideThreads;   // who writes the rows
    static constexpr int kNT = (kChainWarp0 + kChainWarps + kOutWarps) * 32;
    static constexpr int kChainThreads = kChainWarps * 32;
    static constexpr int kNQ = kChainWarps / 4;
};
static_assert(kSideThreads == (kChainWarp0 - kSideWarp0) * 32, "named-barrier thread count of the side warps");
constexpr int kHostedNT = Roles<kGateScalar, true>::kNT;   // 24 warps: with a hosted WY group, 32
// named barriers: 1 Qh / output warps, 5 output warps (split), kCtaBar all the pass's threads
constexpr uint32_t kCtaBar = 3;

// TMEM columns (32-bit, 128 lanes)
constexpr uint32_t TM_SACC = 0;     // S^T fp32 [dv lanes][dk cols], pre-scaled by the coming chunk's decay
constexpr uint32_t TM_OU = 128;     // kOuBufs x [O^T | U^T] fp32, [dv][C | C], by chunk
constexpr uint32_t TM_COLS = 512;   // allocated (a hosted WY group uses the columns past Layout::kCols)

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t SZ_STAGE = 73728;    // one chunk's tiles:
constexpr uint32_t ST_K = 0;            //   K [d-block][64 rows][128 B]                        16 KiB
constexpr uint32_t ST_B = 16384;        //   [d-block][q -> Qh rows 0-63 | -W rows 64-127][128 B] 32 KiB
constexpr uint32_t ST_UT = 49152;       //   u^T [128 rows (dv)][128 B (C)]                      16 KiB
constexpr uint32_t ST_P = 65536;        //   P [64 rows (i)][128 B (j)]                           8 KiB

// Two layouts: alone on its SM (three stages, two [O|U] buffers, all 512 TMEM
// columns), or hosting a WY group (two stages, one [O|U] buffer, 384 columns;
// the group gets the other 128 and the shared memory past STATE_BYTES).  ZB
// (the gated norm on the output rows, alone on its SM): two stages, and in the
// room of the third z of two chunks and one chunk's output rows in fp32.
template <bool HOSTED, bool ZB = false>
struct Layout {
    static_assert(!(HOSTED && ZB), "the gated norm runs on a state pass alone on its SM");
    static constexpr int kStages = HOSTED || ZB ? 2 : 3;
    static constexpr int kOuBufs = HOSTED ? 1 : 2;
    static constexpr uint32_t TM_ST = TM_OU + 128 * kOuBufs;   // S^T bf16 pairs [dv][dk/2]
    static constexpr uint32_t TM_UT = TM_ST + 64;               // U^T bf16 pairs [dv][C/2]
    static constexpr uint32_t kCols = TM_UT + 32;
    static constexpr uint32_t SZ_Z = kC * kD * 2;               // z of one chunk [64 rows][d_v] bf16
    static constexpr uint32_t OFF_Z = kStages * SZ_STAGE;       // ZB: two of them
    static constexpr uint32_t OFF_OB = OFF_Z + 2 * SZ_Z;        // ZB: output rows [64][d_v] fp32
    static constexpr uint32_t OFF_GATE = ZB ? OFF_OB + kC * kD * 4 : OFF_Z;   // 4 gate slots
    static constexpr uint32_t OFF_BAR = OFF_GATE + 4 * GATE_FLOATS * 4;   // mbarriers, TMEM slot, flag
    static constexpr uint32_t STATE_BYTES = OFF_BAR + 256;
};
constexpr uint32_t STAGE_TX = SZ_STAGE;

// barrier indices; where a waiter could otherwise see a barrier two phases on,
// there is one per chunk parity
enum {
    B_FULL0 = 0, B_FREE0 = 3,                            // TMA stages (3 each)
    B_GATE0 = 6,                                         // gate slots (4)
    B_WS = 10, B_KU, B_PU0, B_PU1,                       // MMA completions
    B_READY0, B_READY1, B_READY2, B_OFREE0, B_OFREE1,    // Qh / output warps -> MMA (Qh per stage)
    B_UTA, B_UTB, B_STA, B_STB,                          // state warps -> MMA (first / second half)
    B_SC,                                                // state warps -> MMA: fp32 state rescaled
    B_COUNT
};
static_assert(8 * B_COUNT + 16 <= 256, "barrier area");

struct Args {
    const CUtensorMap* tm_k;        // k; per-key gate: the workspace's K~
    const CUtensorMap* tm_q;        // q; per-key gate: the workspace's Qh
    const CUtensorMap* tm_w;
    const CUtensorMap* tm_u;
    const CUtensorMap* tm_p;
    const unsigned int* flags;      // ready flags of the workspace tiles; null: all written already
    const float* beta;
    const float* g;
    const float* S0;
    __nv_bfloat16* o;
    float* S_T;
    int T;
    float scale;
    unsigned int* status;
    int test_flags;
    const float* gam;               // per-key gate: the workspace's e^Gamma_last per tile and channel
    float* snaps;                   // null, or [heads][n_snap][d_k][d_v]: the state after every
    int snap_every, n_snap;         //   snap_every chunks (full chunks only)
    // the layer's prologue inside the kernels (scalar gate): beta and g hold the raw inputs
    // b and a, q and k are normalised per row (per-head A_log, dt_bias; H heads per batch row)
    int prologue;
    const float* A_log;
    const float* dt_bias;
    int H;
    int rep = 1;
    // a packed batch of N sequences (null: B rows of T tokens): the chunk tables of
    // varlen_table_kernel; `head` is then s H + h for sequence s and head h
    const int* vl = nullptr;
    int vl_N = 0;
    // with the prologue: the layer's gated RMSNorm on the output rows (0 none, 1 SiLU(z),
    // 2 sigmoid(z)); o then receives y = w * o / sqrt(mean(o^2) + eps) * act(z) token-major
    // [B][T][H][d_v], the layout of z
    int norm = 0;
    const __nv_bfloat16* z = nullptr;
    const float* norm_w = nullptr;
    float eps = 0.f;
    // with the prologue: the workspace's 1 / ||q_i|| rows, written by the WY tiles
    const float* rq = nullptr;
    // the workspace (128-byte aligned) and its tile count: each tile's lines are dropped
    // from L2 once its loads have landed (null: kept)
    uint8_t* scratch = nullptr;
    long long scratch_tiles = 0;
};

// Drop tile t's workspace lines from L2 (one warp): -W, u^T, P, the 1 / ||q_i|| row
// with the prologue, and K~, Qh and e^Gamma_last with the per-key gate.  The tile's
// loads have landed in shared memory and nothing reads it again in this call, so the
// lines need never be written back to memory.
template <int GATE, int PRO>
__device__ __forceinline__ void drop_tile(const Args& ar, int64_t t, int lane) {
    const int64_t nt = ar.scratch_tiles;
    uint8_t* const base = ar.scratch;
    uint8_t* const w = base + t * (int64_t)kWsWBytes;
    uint8_t* const u = base + nt * (int64_t)kWsWBytes + t * (int64_t)kWsUBytes;
    uint8_t* const p = base + nt * (int64_t)(kWsWBytes + kWsUBytes) + t * (int64_t)kWsPBytes;
    for (int l = lane; l < (int)(kWsWBytes / 128); l += 32) {
        discard_l2(w + 128 * l);
        discard_l2(u + 128 * l);
    }
    for (int l = lane; l < (int)(kWsPBytes / 128); l += 32) discard_l2(p + 128 * l);
    constexpr int64_t kBeforeRq = (int64_t)(kWsWBytes + kWsUBytes + kWsPBytes);
    if (PRO && lane < (int)(kWsRqBytes / 128)) discard_l2(base + nt * kBeforeRq + t * (int64_t)kWsRqBytes + 128 * lane);
    if constexpr (GATE == kGatePerKey) {
        uint8_t* const kt = base + nt * (int64_t)kWsTileBytes + t * (int64_t)kWsKtBytes;
        uint8_t* const qh = base + nt * (int64_t)(kWsTileBytes + kWsKtBytes) + t * (int64_t)kWsQhBytes;
        uint8_t* const gm = base + nt * (int64_t)(kWsTileBytes + kWsKtBytes + kWsQhBytes) + t * (int64_t)kWsGamBytes;
        for (int l = lane; l < (int)(kWsKtBytes / 128); l += 32) {
            discard_l2(kt + 128 * l);
            discard_l2(qh + 128 * l);
        }
        if (lane < (int)(kWsGamBytes / 128)) discard_l2(gm + 128 * lane);
    }
}

// Gate slot with the per-key gate: e^Gamma_last of each key channel.
constexpr int G_KGAM = 0;

// TMEM loads and stores of N consecutive 32-bit columns of the thread's lane.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&r)[N]) {
    static_assert(N == 8 || N == 16 || N == 32, "column count");
    if constexpr (N == 8) tmem_ld8(taddr, r);
    else if constexpr (N == 16) tmem_ld16(taddr, r);
    else tmem_ld32(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&u)[N]) {
    static_assert(N == 4 || N == 8 || N == 16, "column count");
    if constexpr (N == 4) tmem_st4(taddr, u);
    else if constexpr (N == 8) tmem_st8(taddr, u);
    else tmem_st16(taddr, u);
}
template <int N>
__device__ __forceinline__ void tmem_st_f32(uint32_t taddr, const float (&v)[N]) {
    static_assert(N == 16 || N == 32, "column count");
    if constexpr (N == 16) tmem_st16(taddr, reinterpret_cast<const uint32_t(&)[16]>(v));
    else tmem_st32(taddr, v);
}

// z of chunk c (64 token-major rows of d_v, H d_v elements apart) into the shared
// buffer zb by the NTHR output threads, 16 bytes a copy; rows past the chunk's
// end are zero-filled and not read.
template <int NTHR>
__device__ __forceinline__ void z_load(const Args& ar, uint32_t zb, int64_t bh, int c, int Cc, int oid) {
    const int64_t b = bh / ar.H, h = bh % ar.H;
    const __nv_bfloat16* z0 = ar.z + ((b * ar.T + (int64_t)c * kC) * ar.H + h) * kD;
#pragma unroll
    for (int u = 0; u < 1024 / NTHR; ++u) {
        const int x = oid + NTHR * u;              // 0..1023: (row, 16-byte chunk)
        const int i = x >> 4, ch = x & 15;
        const bool in = i < Cc;
        cp_async16(zb + (uint32_t)(i * kD * 2 + ch * 16), z0 + (in ? (int64_t)i * ar.H * kD + ch * 8 : 0),
                   in ? 16u : 0u);
    }
    cp_async_commit();
}

// Output rows of chunk cp with the layer's gated RMSNorm, in two steps by the
// 256 output threads (8 warps).  First each thread copies 32 positions of its
// value channel j (= TMEM lane) of the chunk's o (fp32, TMEM) into the
// row-major buffer ob (warps 0-3 positions 0-31, warps 4-7 positions 32-63);
// then, after a barrier, thread t takes channels 8 (t mod 16) .. + 7 of rows
// t / 16 + 16 u: the 16 threads of a row sum its squares by shuffles, and each
// forms y_ij = w_j o_ij / sqrt(mean_j o_ij^2 + eps) act(z_ij) for its eight
// channels (16-byte loads of o and z, a 16-byte store of y, token-major like
// z).  (The prologue's 1 / ||q_i|| is already in o: Qh and P carry it.)
__device__ __forceinline__ void norm_stage(uint32_t oc, float* __restrict__ ob, int j, int hh) {
    float v[32];
    tmem_ld32(oc + hh * 32, v);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) ob[(hh * 32 + e) * kD + j] = v[e];
}
__device__ __forceinline__ void norm_rows(const Args& ar, const float* __restrict__ ob,
                                          const __nv_bfloat16* __restrict__ zb, int64_t bh, int cp, int Cc,
                                          int oid) {
    const int64_t b = bh / ar.H, h = bh % ar.H;
    const int64_t row0 = (b * ar.T + (int64_t)cp * kC) * ar.H + h;   // token-major row of position 0
    const int c8 = (oid & 15) * 8;                                   // first channel of the thread
    const bool silu = ar.norm == 1;
    float w[8];
    *reinterpret_cast<float4*>(w) = *reinterpret_cast<const float4*>(ar.norm_w + c8);
    *reinterpret_cast<float4*>(w + 4) = *reinterpret_cast<const float4*>(ar.norm_w + c8 + 4);
#pragma unroll 2
    for (int u = 0; u < 4; ++u) {
        const int i = (oid >> 4) + 16 * u;
        float x[8];
        *reinterpret_cast<float4*>(x) = *reinterpret_cast<const float4*>(ob + i * kD + c8);
        *reinterpret_cast<float4*>(x + 4) = *reinterpret_cast<const float4*>(ob + i * kD + c8 + 4);
        const uint4 zv = *reinterpret_cast<const uint4*>(zb + i * kD + c8);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += x[e] * x[e];
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        ss += __shfl_xor_sync(0xffffffffu, ss, 4);
        ss += __shfl_xor_sync(0xffffffffu, ss, 8);
        const float f = rsqrtf(ss * (1.f / (float)kD) + ar.eps);
        const __nv_bfloat162* z2 = reinterpret_cast<const __nv_bfloat162*>(&zv);
        uint32_t y[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 zz = __bfloat1622float2(z2[e]);
            const float s0 = __fdividef(1.f, 1.f + __expf(-zz.x)), s1 = __fdividef(1.f, 1.f + __expf(-zz.y));
            const float g0 = silu ? zz.x * s0 : s0, g1 = silu ? zz.y * s1 : s1;
            y[e] = pack_bf16x2(x[2 * e] * f * w[2 * e] * g0, x[2 * e + 1] * f * w[2 * e + 1] * g1);
        }
        if (i < Cc)
            *reinterpret_cast<uint4*>(ar.o + (row0 + (int64_t)i * ar.H) * kD + c8) = make_uint4(y[0], y[1], y[2], y[3]);
    }
}

// The state pass of head `head`, run by threads 0 .. kNT - 1 of a CTA whose
// shared memory starts (1024-aligned) at sm.  HOSTED: the caller allocated the
// TMEM (base tmem_given) and shares the SM with a WY group.
// PRO: the layer's prologue (raw gates, unit q and k) is compiled in (scalar gate),
// 1 alone, 2 with the gated RMSNorm on the output rows.
template <int GATE, bool HOSTED, int PRO = 0>
__device__ __forceinline__ void state_pass(uint8_t* sm, const Args& ar, int64_t head, uint32_t tmem_given) {
    using L = Layout<HOSTED, PRO == 2>;
    constexpr int kStages = L::kStages;
    constexpr uint32_t OFF_GATE = L::OFF_GATE, OFF_BAR = L::OFF_BAR;
    constexpr uint32_t TM_ST = L::TM_ST, TM_UT = L::TM_UT;
    using R = Roles<GATE, HOSTED, PRO>;
    constexpr int kNT = R::kNT, kChainThreads = R::kChainThreads, kNQ = R::kNQ;
    constexpr bool kSplitOut = R::kSplitOut;
    const CUtensorMap& tm_k = *ar.tm_k;
    const CUtensorMap& tm_q = *ar.tm_q;
    const CUtensorMap& tm_w = *ar.tm_w;
    const CUtensorMap& tm_u = *ar.tm_u;
    const CUtensorMap& tm_p = *ar.tm_p;
    const unsigned int* __restrict__ flags = ar.flags;
    const float* __restrict__ beta = ar.beta;
    const float* __restrict__ g = ar.g;
    const float* S0 = ar.S0;
    __nv_bfloat16* __restrict__ o = ar.o;
    float* S_T = ar.S_T;
    const int T = ar.T;
    const float scale = ar.scale;
    unsigned int* status = ar.status;
    const int test_flags = ar.test_flags;
    const uint32_t sb = smem_u32(sm);
    float* gates = reinterpret_cast<float*>(sm + OFF_GATE);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_BAR + 8 * B_COUNT + 8);
    Ctl ctl{sb + OFF_BAR, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = head;
    // the chain: its first row of q / k / v / o, its tokens, its tiles (tile0 + c tstep)
    // and its key rows
    int64_t row_base = bh * T, krow_base = key_head(bh, ar.H, ar.rep) * T, tile0;
    int len = T, tstep = 1;
    if (ar.vl) {
        const VarlenTables vt{ar.vl, ar.vl_N};
        const int s = (int)(head / ar.H), h = (int)(head % ar.H);
        const int beg = vt.cu()[s];
        len = vt.cu()[s + 1] - beg;
        row_base = krow_base = (int64_t)h * T + beg;
        tile0 = (int64_t)vt.coff()[s] * ar.H + h;
        tstep = ar.H;
    }
    const int n = (len + kC - 1) / kC;
    if (!ar.vl) tile0 = bh * n;
    if (n == 0) {
        // an empty sequence of a packed batch: its final state is its initial one
        if (S_T)
            for (int x = tid; x < kD * kD; x += kNT) S_T[bh * kD * kD + x] = S0 ? S0[bh * kD * kD + x] : 0.f;
        return;
    }

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(ctl.bar(i), i >= B_UTA ? kChainThreads
                                  : i == B_OFREE0 || i == B_OFREE1 ? R::kOutThreads
                                  : i >= B_READY0 ? kSideThreads : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (!HOSTED && warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    named_bar_sync(kCtaBar, kNT);
    tc_fence_after();
    const uint32_t tmem = HOSTED ? tmem_given : *tmem_slot;

    if (warp == 0) {
        // ================= producer: gates + TMA ================================
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_w);
            prefetch_tmap(&tm_u);
            prefetch_tmap(&tm_p);
        }
        int issued = 0;
        constexpr bool KDA = GATE == kGatePerKey;
        // beta / g of the next chunk, loaded one chunk ahead
        float nb0 = 0.f, nb1 = 0.f, ng0 = 0.f, ng1 = 0.f;
        const float eA = PRO ? expf(ar.A_log[bh % ar.H]) : 0.f;
        const float dtb = PRO ? ar.dt_bias[bh % ar.H] : 0.f;
        auto fetch = [&](int cc) {
            const int64_t t0 = row_base + (int64_t)cc * kC;
            const int Cn = min(kC, len - cc * kC);
            nb0 = lane < Cn ? beta[t0 + lane] : 0.f;
            nb1 = lane + 32 < Cn ? beta[t0 + lane + 32] : 0.f;
            if (GATE == kGateScalar) {
                ng0 = lane < Cn ? g[t0 + lane] : 0.f;
                ng1 = lane + 32 < Cn ? g[t0 + lane + 32] : 0.f;
            }
        };
        if (!KDA) fetch(0);
        for (int cc = 0; cc < n; ++cc) {
            const int s = cc % kStages;
            if (!KDA) {
                float b0 = nb0, b1 = nb1, a0 = ng0, a1 = ng1;
                if (cc + 1 < n) fetch(cc + 1);
                if (PRO) {
                    // beta and g from the raw inputs, as the WY side computes them (here, one
                    // chunk after the loads were issued, so their latency stays hidden)
                    const int Cn = min(kC, len - cc * kC);
                    if (lane < Cn) gdn_raw_gates_fast(b0, a0, eA, dtb, (float)ar.prologue);
                    if (lane + 32 < Cn) gdn_raw_gates_fast(b1, a1, eA, dtb, (float)ar.prologue);
                }
                chunk_gates(gates + (cc & 3) * GATE_FLOATS, b0, b1, a0, a1, lane);
                __syncwarp();
                if (lane == 0) mbar_arrive(ctl.bar(B_GATE0 + (cc & 3)));
            }
            // the stage is free once the products of chunk cc - 3 are done
            if (cc >= kStages) {
                bool ok = lane == 0 ? ctl.wait(B_FREE0 + s, (uint32_t)((cc - kStages) / kStages) & 1u) : true;
                if (!__shfl_sync(0xffffffffu, (int)ok, 0)) break;
            }
            if (!(test_flags & 1) && flags) {
                // this chunk's workspace tiles are written (by another CTA, possibly right now)
                bool ok = lane == 0 ? wait_flag(flags + tile0 + (int64_t)cc * tstep, abort_flag) : true;
                if (!__shfl_sync(0xffffffffu, (int)ok, 0)) break;
            }
            if (KDA) {
                // the chunk's decays per key channel, from the workspace, into slot cc % 4:
                // its previous reader (chunk cc - 4) is done once chunk cc - 3's products are
                const float4 gv = test_flags & 1 ? make_float4(1.f, 1.f, 1.f, 1.f)
                                                 : reinterpret_cast<const float4*>(ar.gam + (tile0 + (int64_t)cc * tstep) * kD)[lane];
                reinterpret_cast<float4*>(gates + (cc & 3) * GATE_FLOATS + G_KGAM)[lane] = gv;
                __syncwarp();
                if (lane == 0) mbar_arrive(ctl.bar(B_GATE0 + (cc & 3)));
            }
            if (lane == 0 && !(test_flags & 1)) {
                fence_async_global();
                const int64_t tile = tile0 + (int64_t)cc * tstep;
                // q and k rows of the chunk; with the per-key gate, Qh and K~ rows of the tile
                const int y = KDA ? (int)(tile * kC) : (int)(krow_base + (int64_t)cc * kC);
                const uint32_t st = sb + s * SZ_STAGE;
                const uint32_t fb = ctl.bar(B_FULL0 + s);
                mbar_arrive_expect_tx(fb, PRO ? STAGE_TX + kC * 4 : STAGE_TX);
                tma_load_2d(st + ST_K + 0, &tm_k, 0, y, fb);
                tma_load_2d(st + ST_K + 8192, &tm_k, 64, y, fb);
                tma_load_2d(st + ST_B + 0, &tm_q, 0, y, fb);
                tma_load_2d(st + ST_B + 16384, &tm_q, 64, y, fb);
                tma_load_2d(st + ST_B + 8192, &tm_w, 0, (int)(tile * kC), fb);
                tma_load_2d(st + ST_B + 24576, &tm_w, 64, (int)(tile * kC), fb);
                tma_load_2d(st + ST_UT, &tm_u, 0, (int)(tile * kD), fb);
                tma_load_2d(st + ST_P, &tm_p, 0, (int)(tile * kC), fb);
                // with the prologue: the WY tile's 1 / ||q_i|| row (published with the tile)
                // into the chunk's gate slot, for Qh; its previous reader, chunk cc - 4's
                // side warps, finished before chunk cc - 3's products, which freed this stage
                if (PRO) bulk_load(smem_u32(gates + (cc & 3) * GATE_FLOATS + G_RQ), ar.rq + tile * kC, kC * 4, fb);
            }
            if (!(test_flags & 1)) issued = cc + 1;
            // chunk cc - 3's workspace tile (its loads landed before the stage was freed) is
            // dropped from L2, after this chunk's loads are under way
            if (cc >= kStages && ar.scratch && !(test_flags & 1))
                drop_tile<GATE, PRO>(ar, tile0 + (int64_t)(cc - kStages) * tstep, lane);
        }
        if (*abort_flag && lane == 0) {
            // let every load this CTA issued land before its shared memory is released
            for (int cc = max(0, issued - kStages); cc < issued; ++cc)
                mbar_wait_bounded(ctl.bar(B_FULL0 + cc % kStages), (uint32_t)(cc / kStages) & 1u, kWaitNs);
        }
    } else if (warp == 3) {
        // ================= MMA issue (one thread) ====================================
        if (lane == 0) {
            const uint32_t I_SW = idesc_bf16(128, 128, 0, 0);       // [O|U] = S^T [Qh;-W]^T
            const uint32_t I_KU = idesc_bf16(128, 128, 0, 1);       // B MN-major
            const uint32_t I_PU = idesc_bf16(128, 64, 0, 0);
            bool ok = true;
            for (int c = 0; ok && c < n; ++c) {
                const uint32_t par = (uint32_t)c & 1u;
                const int s = c % kStages;
                const uint32_t st = sb + s * SZ_STAGE;
                const uint32_t ou = tmem + TM_OU + (c % L::kOuBufs) * 128;
                // [O|U]^T = S^T [Qh;-W]^T: once the tiles are in and this buffer's output of
                // chunk c - 2 is out, the first half of d_k as soon as the state's first half
                // is written, then the second
                ok = ctl.wait(B_FULL0 + s, (uint32_t)(c / kStages) & 1u) &&
                     ctl.wait(B_READY0 + s, (uint32_t)(c / kStages) & 1u) &&
                     (c < L::kOuBufs || ctl.wait(B_OFREE0 + ((c - L::kOuBufs) & 1),
                                                 (uint32_t)((c - L::kOuBufs) >> 1) & 1u)) &&
                     ctl.wait(B_STA, par);
                if (!ok) break;
                tc_fence_after();
                // the stage's operand descriptors once; a step along K is a constant added to
                // the start-address field (address / 16; the stage is 1024-byte aligned and the
                // offsets stay inside the field)
                const uint64_t dB = sw128_desc(st + ST_B, 16, 1024);     // [Qh | -W] rows, K-major
                const uint64_t dK = sw128_desc(st + ST_K, 8192, 1024);   // K, MN-major
                const uint64_t dP = sw128_desc(st + ST_P, 16, 1024);     // P, K-major
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(ou, tmem + TM_ST + kk * 8, dB + (uint64_t)(2 * kk), I_SW, kk > 0);
                ok = ctl.wait(B_STB, par);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 4; kk < 8; ++kk)
                    mma_bf16_ts(ou, tmem + TM_ST + kk * 8, dB + (uint64_t)(16384 / 16 + 2 * (kk & 3)), I_SW, 1);
                mma_commit(ctl.bar(B_WS));
                // S^T += U^T K~ (the decayed keys), positions 0-31 then 32-63, once the fp32
                // state has been rescaled for this chunk; then O^T += U^T P^T, off the chain
                ok = ctl.wait(B_UTA, par) && ctl.wait(B_SC, par);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    mma_bf16_ts(tmem + TM_SACC, tmem + TM_UT + kk * 8, dK + (uint64_t)(128 * kk), I_KU, 1);
                ok = ctl.wait(B_UTB, par);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 2; kk < 4; ++kk)
                    mma_bf16_ts(tmem + TM_SACC, tmem + TM_UT + kk * 8, dK + (uint64_t)(128 * kk), I_KU, 1);
                mma_commit(ctl.bar(B_KU));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(ou, tmem + TM_UT + kk * 8, dP + (uint64_t)(2 * kk), I_PU, 1);
                mma_commit(ctl.bar(B_PU0 + (c & 1)));
                mma_commit(ctl.bar(B_FREE0 + s));        // the stage's last reader is done
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp >= kSideWarp0 && warp < kChainWarp0) {
        // ================= Qh of each chunk, output rows of the previous one (128 threads)
        const int sid = tid - kSideWarp0 * 32;     // 0..127
        const int q = warp & 3;                    // TMEM lane quarter
        const int j = (q << 5) + lane;             // value channel = TMEM lane
        for (int c = 0; c <= n; ++c) {
            if (c < n) {
                // ---- Qh = scale e^G Q in place over the q tile (rows 0-63 of each d-block);
                //      with the prologue, Q's rows also normalised
                const int s = c % kStages;
                const int Cc = min(kC, len - c * kC);
                float* gs = gates + (c & 3) * GATE_FLOATS;
                const uint32_t st = sb + s * SZ_STAGE;
                bool ok = ctl.wait(B_GATE0 + (c & 3), (uint32_t)(c >> 2) & 1u) &&
                          ctl.wait(B_FULL0 + s, (uint32_t)(c / kStages) & 1u);
                if (!ok) *abort_flag = 1;
                if (named_bar_any(1, kSideThreads, !ok)) break;
                // (with the per-key gate the workspace holds Qh already)
                // (loads four at a time: the ld / st helpers keep their order, so one load per
                // iteration would wait out each load's latency in turn)
#pragma unroll
                for (int u0 = 0; u0 < (GATE == kGatePerKey ? 0 : 8); u0 += 4) {
                    uint4 w[4];
                    uint32_t a[4];
#pragma unroll
                    for (int uu = 0; uu < 4; ++uu) {
                        const int x = sid + (u0 + uu) * kSideThreads;   // (d-block, row, 16-byte chunk)
                        const int blk = x >> 9, i = (x >> 3) & 63, ch = x & 7;
                        a[uu] = st + ST_B + blk * 16384 + sw128_off(i, ch);
                        w[uu] = ld_shared_v4(a[uu]);
                    }
#pragma unroll
                    for (int uu = 0; uu < 4; ++uu) {
                        const int i = ((sid + (u0 + uu) * kSideThreads) >> 3) & 63;
                        // (with the prologue Qh also takes 1 / ||q_i||, which landed with the stage).
                        // The row's factor is rounded to bf16 and applied by packed bf16 multiplies:
                        // the side warps share the SM's issue slots with the chain's epilogues, and
                        // their instruction count, not this one rounding, showed in the chain
                        const float f = i < Cc ? (PRO ? scale * gs[G_EG + i] * gs[G_RQ + i] : scale * gs[G_EG + i]) : 0.f;
                        const uint32_t f2 = pack_bf16x2(f, f);
                        st_shared_v4(a[uu], mul_bf16x2(w[uu].x, f2), mul_bf16x2(w[uu].y, f2), mul_bf16x2(w[uu].z, f2),
                                     mul_bf16x2(w[uu].w, f2));
                    }
                }
                // ---- K~ = K (.) e^(G_last - G) in place over the k tile: each position's decay to
                //      the chunk's end folded into its key, so that the KU product reads U itself
                //      (no gate: the factor is 1; per-key gate: the workspace holds K~)
#pragma unroll
                for (int u0 = 0; u0 < (GATE == kGateScalar ? 8 : 0); u0 += 4) {
                    uint4 w[4];
                    uint32_t a[4];
#pragma unroll
                    for (int uu = 0; uu < 4; ++uu) {
                        const int x = sid + (u0 + uu) * kSideThreads;   // (d-block, row, 16-byte chunk)
                        const int blk = x >> 9, i = (x >> 3) & 63, ch = x & 7;
                        a[uu] = st + ST_K + blk * 8192 + sw128_off(i, ch);
                        w[uu] = ld_shared_v4(a[uu]);
                    }
#pragma unroll
                    for (int uu = 0; uu < 4; ++uu) {
                        const float f = gs[G_ET + (((sid + (u0 + uu) * kSideThreads) >> 3) & 63)];
                        const uint32_t f2 = pack_bf16x2(f, f);
                        st_shared_v4(a[uu], mul_bf16x2(w[uu].x, f2), mul_bf16x2(w[uu].y, f2), mul_bf16x2(w[uu].z, f2),
                                     mul_bf16x2(w[uu].w, f2));
                    }
                }
                fence_async_smem();
                mbar_arrive(ctl.bar(B_READY0 + s));
            }
            if (!kSplitOut && c >= 1) {
                // ---- output rows of chunk c - 1 --------------------------------------------
                const int cp = c - 1;
                const int Cc = min(kC, len - cp * kC);
                bool ok = ctl.wait(B_PU0 + (cp & 1), (uint32_t)(cp >> 1) & 1u);
                if (!ok) *abort_flag = 1;
                if (named_bar_any(1, kSideThreads, !ok)) break;
                tc_fence_after();
                __nv_bfloat16* ob = o + (row_base + (int64_t)cp * kC) * kD + j;
                const uint32_t oc = tmem + ((uint32_t)(q << 5) << 16) + TM_OU + (cp % L::kOuBufs) * 128;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tmem_ld32(oc + hh * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int i = hh * 32 + e;
                        if (i < Cc) ob[(int64_t)i * kD] = __float2bfloat16_rn(v[e]);
                    }
                }
                tc_fence_before();
                mbar_arrive(ctl.bar(B_OFREE0 + (cp & 1)));
            }
        }
    } else if (kSplitOut && warp >= R::kOutWarp0) {
        // ================= output rows of each chunk (128 threads) =======================
        const int q = warp & 3;                    // TMEM lane quarter
        const int j = (q << 5) + lane;             // value channel = TMEM lane
        constexpr int kOT = R::kOutThreads;
        const int oid = tid - R::kOutWarp0 * 32;   // 0 .. kOT - 1
        // with the gated norm, z of each chunk is copied in one chunk ahead
        const uint32_t zbuf = sb + L::OFF_Z;
        if (PRO == 2) z_load<kOT>(ar, zbuf, bh, 0, min(kC, len), oid);
        for (int cp = 0; cp < n; ++cp) {
            const int Cc = min(kC, len - cp * kC);
            bool ok = ctl.wait(B_PU0 + (cp & 1), (uint32_t)(cp >> 1) & 1u);
            if (!ok) *abort_flag = 1;
            if (PRO == 2) cp_async_wait_all();
            if (named_bar_any(5, kOT, !ok)) break;
            // every thread is past chunk cp - 1, whose z buffer now takes chunk cp + 1
            if (PRO == 2 && cp + 1 < n)
                z_load<kOT>(ar, zbuf + ((cp + 1) & 1) * L::SZ_Z, bh, cp + 1, min(kC, len - (cp + 1) * kC), oid);
            tc_fence_after();
            const uint32_t oc = tmem + ((uint32_t)(q << 5) << 16) + TM_OU + (cp % L::kOuBufs) * 128;
            if constexpr (PRO == 2) {
                float* ob = reinterpret_cast<float*>(sm + L::OFF_OB);
                norm_stage(oc, ob, j, oid >> 7);
                tc_fence_before();
                mbar_arrive(ctl.bar(B_OFREE0 + (cp & 1)));        // the TMEM buffer is read
                named_bar_sync(5, kOT);
                norm_rows(ar, ob, reinterpret_cast<const __nv_bfloat16*>(sm + L::OFF_Z + (cp & 1) * L::SZ_Z), bh, cp,
                          Cc, oid);
            } else {
                __nv_bfloat16* ob = o + (row_base + (int64_t)cp * kC) * kD + j;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tmem_ld32(oc + hh * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int i = hh * 32 + e;
                        if (i < Cc) ob[(int64_t)i * kD] = __float2bfloat16_rn(v[e]);
                    }
                }
                tc_fence_before();
                mbar_arrive(ctl.bar(B_OFREE0 + (cp & 1)));
            }
        }
        // no copy of this thread is still in flight when the shared memory is released
        if (PRO == 2) cp_async_wait_all();
    } else if (warp >= kChainWarp0) {
        // ================= U and the state (kChainThreads threads) =================
        // kNQ warps per TMEM lane quarter; each pass splits its columns among them
        constexpr int SCOLS = 64 / kNQ;              // d_k columns of a state pass, per thread
        constexpr int UPOS = 32 / kNQ;               // positions of a U pass, per thread
        const int q = warp & 3;
        const int hc = (warp - kChainWarp0) >> 2;    // which part of each pass
        const int j = (q << 5) + lane;               // value channel = TMEM lane
        const uint32_t lane_off = (uint32_t)(q << 5) << 16;
        bool ok = ctl.wait(B_GATE0, 0);
        if (ok) {
            // S0 -> TMEM: its bf16 copy (which the first products read; signalled at once),
            // then the fp32 accumulator pre-scaled by chunk 0's decay
            const float gamma0 = GATE == kGatePerKey ? 0.f : gates[G_GAMMA];
#pragma unroll 1
            for (int p = 0; p < 2; ++p) {
                const int c0 = 64 * p + SCOLS * hc;      // d_k columns c0 .. c0 + SCOLS - 1
                float v[SCOLS];
#pragma unroll
                for (int e = 0; e < SCOLS; ++e) v[e] = S0 ? S0[(bh * kD + c0 + e) * kD + j] : 0.f;
                uint32_t pk[SCOLS / 2];
#pragma unroll
                for (int e = 0; e < SCOLS / 2; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                tmem_st_cols(tmem + lane_off + TM_ST + c0 / 2, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(ctl.bar(p == 0 ? B_STA : B_STB));
#pragma unroll
                for (int e = 0; e < SCOLS; ++e) v[e] *= GATE == kGatePerKey ? gates[G_KGAM + c0 + e] : gamma0;
                tmem_st_f32(tmem + lane_off + TM_SACC + c0, v);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_SC));
        }
        for (int c = 0; ok && c < n; ++c) {
            const uint32_t par = (uint32_t)c & 1u;
            const uint32_t st = sb + (c % kStages) * SZ_STAGE;
            // ---- U = u - W S -> bf16 pairs in TMEM, in two passes over positions 0-31 and
            //      32-63 (the KU product reads U itself: the decays are in K~) -------------
            ok = ctl.wait(B_WS, par) && ctl.wait(B_FULL0 + c % kStages, (uint32_t)(c / kStages) & 1u);
            if (!ok) break;
            tc_fence_after();
            {
                // both halves' columns requested at once: the second half waits no second latency
                float v[2][UPOS];
                const uint32_t ub = tmem + lane_off + TM_OU + (c % L::kOuBufs) * 128 + 64 + UPOS * hc;
                tmem_ld_cols(ub, v[0]);
                tmem_ld_cols(ub + 32, v[1]);
                tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const int i0 = 32 * p + UPOS * hc;   // positions i0 .. i0 + UPOS - 1
#pragma unroll
                    for (int ch = 0; ch < UPOS / 8; ++ch) {
                        const uint4 w = ld_shared_v4(st + ST_UT + sw128_off(j, (i0 >> 3) + ch));
                        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(h2[e]);
                            v[p][8 * ch + 2 * e] += f.x;
                            v[p][8 * ch + 2 * e + 1] += f.y;
                        }
                    }
                    uint32_t pk[UPOS / 2];
#pragma unroll
                    for (int e = 0; e < UPOS / 2; ++e) pk[e] = pack_bf16x2(v[p][2 * e], v[p][2 * e + 1]);
                    tmem_st_cols(tmem + lane_off + TM_UT + (i0 >> 1), pk);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(ctl.bar(p == 0 ? B_UTA : B_UTB));
                }
            }
            // ---- state: S_{c+1} = gamma_c S_c + dS (already summed in TMEM), in two passes
            //      over d_k 0-63 and 64-127: the bf16 copy first (the next chunk's first
            //      products wait for it), then the fp32 accumulator pre-scaled by the next
            //      chunk's decay (the next KU product waits for that) ---------------------
            ok = ctl.wait(B_KU, par) && (c + 1 >= n || ctl.wait(B_GATE0 + ((c + 1) & 3), (uint32_t)((c + 1) >> 2) & 1u));
            if (!ok) break;
            tc_fence_after();
            const bool last = c + 1 == n;
            const float* gsn = gates + ((c + 1) & 3) * GATE_FLOATS;
            // snapshot s = (c + 1) / snap_every - 1 of the state after this chunk
            const bool snap = ar.snaps && (c + 1) % ar.snap_every == 0 && (c + 1) / ar.snap_every <= ar.n_snap;
            float* snap_out = snap ? ar.snaps + ((bh * ar.n_snap + (c + 1) / ar.snap_every - 1) * kD) * kD + j
                                   : nullptr;
            const float gnext = last || GATE == kGatePerKey ? 1.f : gsn[G_GAMMA];
            {
                // both halves' columns requested at once; the bf16 copies first (each half
                // signalled as soon as it is stored), the fp32 rescale after both
                float v[2][SCOLS];
                const uint32_t sa = tmem + lane_off + TM_SACC + SCOLS * hc;
                tmem_ld_cols(sa, v[0]);
                tmem_ld_cols(sa + 64, v[1]);
                tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const int c0 = 64 * p + SCOLS * hc;  // d_k columns c0 .. c0 + SCOLS - 1
                    if (snap) {
#pragma unroll
                        for (int e = 0; e < SCOLS; ++e) snap_out[(c0 + e) * kD] = v[p][e];
                    }
                    if (last) {
                        if (S_T) {
#pragma unroll
                            for (int e = 0; e < SCOLS; ++e) S_T[(bh * kD + c0 + e) * kD + j] = v[p][e];
                        }
                    } else {
                        uint32_t pk[SCOLS / 2];
#pragma unroll
                        for (int e = 0; e < SCOLS / 2; ++e) pk[e] = pack_bf16x2(v[p][2 * e], v[p][2 * e + 1]);
                        tmem_st_cols(tmem + lane_off + TM_ST + c0 / 2, pk);
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    mbar_arrive(ctl.bar(p == 0 ? B_STA : B_STB));
                }
                if (!last) {
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const int c0 = 64 * p + SCOLS * hc;
#pragma unroll
                        for (int e = 0; e < SCOLS; ++e)
                            v[p][e] *= GATE == kGatePerKey ? gsn[G_KGAM + c0 + e] : gnext;
                        tmem_st_f32(sa + 64 * p, v[p]);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_SC));
        }
        if (!ok) *abort_flag = 1;
    }

    named_bar_sync(kCtaBar, kNT);
    if (*abort_flag && tid == 0) atomicOr(status, 1u);
    // the last chunks' tiles (every product is done)
    if (warp == 0 && ar.scratch && !(test_flags & 1) && !*abort_flag)
        for (int cd = max(0, n - kStages); cd < n; ++cd) drop_tile<GATE, PRO>(ar, tile0 + (int64_t)cd * tstep, lane);
    if (!HOSTED && warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace state
}  // namespace dn
