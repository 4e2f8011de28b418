// chunk_wy_kda.cuh -- the state-independent part of one chunk for the per-key
// gate (KDA: "A walk through of the DeltaNet family of linear attention
// variants", its KDA update: each key channel forgets at its own rate), on
// tensor cores, as a device function run by a group of 8 warps: a whole CTA in
// chunk_wy_kda.cu (two per SM), or one of two groups of a CTA in the
// single-launch prefill of chunk_tc.cu.
//
// Chunk algebra ("Linear attention and Gated DeltaNet", ch. 28, "The chunked
// form", with the decay promoted to one value per key channel).  With Gamma_i
// the inclusive prefix sum of g over the chunk, per channel:
//
//   A_ij = beta_i sum_d k_id k_jd e^(Gamma_id - Gamma_jd)          (j < i)
//   P_ij = scale  sum_d q_id k_jd e^(Gamma_id - Gamma_jd)          (j <= i)
//   T = (I + A)^-1,  W = T diag(beta) (K (.) e^Gamma),  u = T diag(beta) V
//
// and the state pass needs Qh = scale Q (.) e^Gamma, K~ = K (.) e^(Gamma_last -
// Gamma) and gam = e^Gamma_last.
//
// The decays cannot leave the sum over d as row and column factors of one
// product: Gamma falls by about 3 per position and channel, and e^-Gamma_j
// overflows long before the end of a chunk.  So the gram is split by the
// 16-row block I of i, and block I uses its own reference position
// m_I = 16 I + 8:
//
//   e^(Gamma_i - Gamma_j) = e^(Gamma_i - Gamma_mI) e^(Gamma_mI - Gamma_j)
//
// For j < 16 I both factors are at most e^(decay over 8 positions); inside
// the block likewise.  Block I is one tcgen05 product of [K^;Q^] (rows scaled
// by e^(Gamma_i - Gamma_m(i))) with the first 16 (I + 1) rows of K scaled by
// e^(Gamma_mI - Gamma_j): four products of N = 16, 32, 48, 64 into TMEM, of
// which row i reads its own block's.  The exponent is capped at 80 (e^80 is
// far inside bf16 and fp32): the results are exact up to rounding while no
// channel decays by more than e^-80 over 8 consecutive positions.
//
// Steps, one 64-channel d-block at a time for the gram:
//   TMA       K and Q, stacked per d-block as [K rows | Q rows]
//   CUDA core g -> Gamma (log2 units) by a prefix sum over positions
//   CUDA core scaled operands: [K^;Q^] in place, the four B tiles, K (.) e^Gamma
//             for W; Qh, K~ and gam straight to the workspace
//   tcgen05   D_I += [K^;Q^] B_I^T  (I = 0..3)
// then, as for the scalar gate (chunk_wy.cuh):
//   CUDA core A and P from the D_I; T = (I + A)^-1; T diag(beta) as bf16
//   TMA       V over the dead K/Q tiles
//   tcgen05   W^T = (K (.) e^Gamma)^T (T diag(beta))^T, u^T = V^T (T diag(beta))^T
//   epilogue  -W and u^T by TMA stores, as for the scalar gate
//
// The ready flag of a tile is raised as for the scalar gate: by kStoreTid,
// during the group's next tile (while warps 0-5 form the M blocks), or by the
// caller after the group's last tile.  Every wait is bounded; on a timeout the
// group sets its abort flag and stops.
#pragma once

#include "chunk_wy.cuh"

namespace dn {
namespace kda {

using namespace sm100;
using namespace tc;
using wy::fidx;
using wy::kNT;

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [K0 | Q0 | K1 | Q1] -> [K^0 | Q^0 | K^1 | Q^1]; then V = [V0 | V1];
                                        // last, the -W and u^T output tiles
constexpr uint32_t OFF_KW = 32768;      // K (.) e^Gamma = [Kw0 | Kw1] (the A operand of W^T)
constexpr uint32_t OFF_G = 49152;       // Gamma log2(e) of the current d-block, fp32 [64][68];
                                        // after the gram A (fp32 64 x 68), then T diag(beta) (bf16)
constexpr uint32_t OFF_T = OFF_G + 64 * 68 * 4;   // T (fp32 64 x 68), after the gram
constexpr uint32_t OFF_B = 67584;       // the current d-block's B tiles: K rows 0 .. 16 (I + 1) - 1
                                        // scaled by e^(Gamma_mI - Gamma_j), I = 0..3
constexpr uint32_t OFF_GATE = OFF_B + 20480;      // beta [64]
constexpr uint32_t OFF_TAB = OFF_GATE + 256;      // per d-block factor tables [18][64] fp32 (below); the
                                                  // prefix-sum segment totals [4][64] before them
constexpr uint32_t OFF_BAR = OFF_TAB + 18 * 64 * 4;
constexpr uint32_t GROUP_BYTES = 93184;     // one group's shared memory, a multiple of 1024
// (the last 16 bytes of a group stay free: a CTA keeps its TMEM address there)
static_assert(OFF_BAR + 64 <= GROUP_BYTES - 16, "group layout");
static_assert(OFF_T + 64 * 68 * 4 <= OFF_GATE, "T stays inside the dead B tiles");
static_assert(OFF_G + 64 * 68 * 4 <= OFF_B && OFF_B % 1024 == 0, "layout");
static_assert(2 * (GROUP_BYTES + 1024) <= 232448, "two groups per SM");

// B tile I: 16 (I + 1) rows of 128 bytes (64 channels), 128-byte swizzle
__host__ __device__ constexpr uint32_t b_off(int I) { return 1024u * (uint32_t)(I * (I + 1)); }
// TMEM: D_I at column d_col(I), 16 (I + 1) wide; W^T and u^T at 0 and 64 after the gram
__host__ __device__ constexpr uint32_t d_col(int I) { return 8u * (uint32_t)(I * (I + 1)); }
constexpr uint32_t TM_W = 0, TM_U = 64;
constexpr uint32_t TM_COLS = 256;
static_assert(b_off(3) + 8192 == 20480 && d_col(3) + 64 <= TM_COLS, "B tiles and D columns");

constexpr float kCap2 = 80.f * 1.4426950408889634f;   // exponent cap, log2 units

// Factor tables of one d-block, by 16-row block b (m_b = 16 b + 8) and channel:
//   TAB_EM + b      e^Gamma_mb
//   TAB_FC + b      e^(Gamma_last - Gamma_mb)
//   TAB_R + p(I,b)  e^(Gamma_mI - Gamma_mb), I >= b, p(I, b) = I (I + 1) / 2 + b
// so that every factor of row i (block b) is e1 = e^(Gamma_i - Gamma_mb) or
// r1 = e^(Gamma_mb - Gamma_i) times one table entry: two exponentials per element.
constexpr int TAB_EM = 0, TAB_FC = 4, TAB_R = 8, TAB_ROWS = 18;
__host__ __device__ constexpr int tab_pair(int I, int b) { return I * (I + 1) / 2 + b; }

constexpr int kStoreTid = wy::kStoreTid;   // issues the output stores and raises the ready flags
// B_FULL completes twice per tile (K and Q; V); B_MMA three times (the gram's
// two d-blocks; W and u), so its waiters count its completions.
enum { B_FULL = 0, B_MMA = 1 };

__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}

// x (.) f as 8 bf16 (one 16-byte chunk)
__device__ __forceinline__ uint4 scaled8(const float (&x)[8], const float (&f)[8]) {
    return make_uint4(pack_bf16x2(x[0] * f[0], x[1] * f[1]), pack_bf16x2(x[2] * f[2], x[3] * f[3]),
                      pack_bf16x2(x[4] * f[4], x[5] * f[5]), pack_bf16x2(x[6] * f[6], x[7] * f[7]));
}

__device__ __forceinline__ void st_shared_u4(uint32_t a, const uint4& v) { st_shared_v4(a, v.x, v.y, v.z, v.w); }

// One group of kNT threads and its resources.
struct Group {
    uint8_t* sm;             // 1024-aligned shared memory of GROUP_BYTES
    uint32_t sb;
    uint32_t tmem;           // first of the group's TM_COLS TMEM columns
    uint32_t bar;            // named barrier of the group's kNT threads
    int tid, warp, lane;     // within the group
    Ctl ctl;
    uint32_t mma_waits;      // completions of B_MMA this thread has waited for
};

__device__ __forceinline__ Group make_group(uint8_t* sm, uint32_t tmem, uint32_t bar, int tid) {
    Group x;
    x.sm = sm;
    x.sb = smem_u32(sm);
    x.tmem = tmem;
    x.bar = bar;
    x.tid = tid;
    x.warp = tid >> 5;
    x.lane = tid & 31;
    x.ctl = Ctl{x.sb + OFF_BAR, reinterpret_cast<volatile int*>(sm + OFF_BAR + 20)};
    x.mma_waits = 0;
    return x;
}

// Barriers and the abort flag of a group (one thread, before the group's first tile).
__device__ __forceinline__ void init_group(const Group& x) {
    mbar_init(x.ctl.bar(B_FULL), 1);
    mbar_init(x.ctl.bar(B_MMA), 1);
    *x.ctl.abort = 0;
}

struct Args {
    const CUtensorMap* tm_q;
    const CUtensorMap* tm_k;
    const CUtensorMap* tm_v;
    const CUtensorMap* tm_w;
    const CUtensorMap* tm_u;
    __nv_bfloat16* p_out;
    __nv_bfloat16* kt_out;
    __nv_bfloat16* qh_out;
    float* gam_out;
    unsigned int* flags;
    const float* beta;
    const float* g;
    int T, n;
    float scale;
    int test_flags;
    unsigned int* counter;   // tile counter of the single launch (null: the caller picks every tile)
    int BH, G;               // with a counter: heads and WY groups (a ticket x is tile G + x)
};

// Thread kStoreTid, during a tile: the inputs of the tile that `ticket` names
// (if any) into L2: K, Q and V by tensor prefetches, beta and the 32 KiB of g
// of a full chunk by bulk prefetches.
__device__ __forceinline__ void prefetch_next(const Args& ar, unsigned int ticket) {
    if (!ar.counter) return;
    const int64_t tn = (int64_t)ar.G + ticket;
    if (tn >= (int64_t)ar.BH * ar.n) return;
    const int cn = (int)(tn / ar.BH);
    const int64_t y = (tn - (int64_t)cn * ar.BH) * ar.T + (int64_t)cn * kC;
    tma_prefetch_2d(ar.tm_k, 0, (int)y);
    tma_prefetch_2d(ar.tm_k, 64, (int)y);
    tma_prefetch_2d(ar.tm_q, 0, (int)y);
    tma_prefetch_2d(ar.tm_q, 64, (int)y);
    tma_prefetch_2d(ar.tm_v, 0, (int)y);
    tma_prefetch_2d(ar.tm_v, 64, (int)y);
    if (ar.T - cn * kC >= kC) {
        bulk_prefetch_l2(ar.beta + y, kC * 4);
        bulk_prefetch_l2(ar.g + y * kD, kC * kD * 4);
    }
}

// The ticket taken during the group's last tile (after kda_tile returned true).
__device__ __forceinline__ unsigned int next_ticket(const Group& x) {
    return *reinterpret_cast<volatile const unsigned int*>(x.sm + OFF_BAR + 24);
}

// Thread kStoreTid: raise the previous tile's ready flag once its stores
// (issued by this thread) are complete; as wy::publish_pending.
__device__ __forceinline__ void publish_pending(const Args& ar, int64_t& pending) {
    if (pending < 0) return;
    bulk_wait_all();
    fence_async_global();
    st_release_gpu(ar.flags + pending, 1u);
    pending = -1;
}

// Next completion of B_MMA (every thread of the group waits for each one).
__device__ __forceinline__ bool wait_mma(Group& x) {
    const bool ok = x.ctl.wait(B_MMA, x.mma_waits & 1u);
    ++x.mma_waits;
    return ok;
}

// Chunk c of head bh.  `pending` (thread kStoreTid's copy counts) is the
// group's tile whose flag is still to be raised, or -1; on return it is this
// tile.  With a tile counter, thread 0 also takes the group's next ticket
// (next_ticket()).  Returns false (the group's abort flag set) if a wait gave up.
__device__ __forceinline__ bool kda_tile(Group& x, const Args& ar, int c, int64_t bh, int64_t& pending) {
    uint8_t* sm = x.sm;
    const uint32_t sb = x.sb;
    float* bs = reinterpret_cast<float*>(sm + OFF_GATE);              // beta of the chunk
    float* segt = reinterpret_cast<float*>(sm + OFF_TAB);             // prefix-sum segment totals
    float* tab = reinterpret_cast<float*>(sm + OFF_TAB);              // factor tables
    float* Gm = reinterpret_cast<float*>(sm + OFF_G);                 // Gamma log2(e), [64][68]
    float* Am = reinterpret_cast<float*>(sm + OFF_G);
    float* Tm = reinterpret_cast<float*>(sm + OFF_T);
    const Ctl& ctl = x.ctl;
    const uint32_t tmem = x.tmem;
    const int tid = x.tid, warp = x.warp, lane = x.lane;
    const uint32_t kBar = x.bar;
    const int T = ar.T, n = ar.n;
    const float scale = ar.scale;
    const float* __restrict__ beta = ar.beta;
    const float* __restrict__ g = ar.g;
    __nv_bfloat16* __restrict__ p_out = ar.p_out;
    __nv_bfloat16* __restrict__ kt_out = ar.kt_out;
    __nv_bfloat16* __restrict__ qh_out = ar.qh_out;
    float* __restrict__ gam_out = ar.gam_out;
    const CUtensorMap& tm_q = *ar.tm_q;
    const CUtensorMap& tm_k = *ar.tm_k;
    const CUtensorMap& tm_v = *ar.tm_v;
    const CUtensorMap& tm_w = *ar.tm_w;
    const CUtensorMap& tm_u = *ar.tm_u;
    const int64_t tile = bh * n + c;
    const int Cc = min(kC, T - c * kC);
    const int64_t t0 = bh * T + (int64_t)c * kC;
    const bool load = !(ar.test_flags & 1);
    int loads = 0;                                   // load phases issued (thread 0)
    bool ok = true;
    // the group's next ticket, taken now (by the thread that prefetches for it and hands
    // it on) and used after the tile: its latency is hidden
    const unsigned int ticket = tid == kStoreTid && ar.counter ? atomicAdd(ar.counter, 1u) : 0u;

    if (tid == 0 && load) {
        const uint32_t fb = ctl.bar(B_FULL);
        mbar_arrive_expect_tx(fb, 4 * 8192);
        tma_load_2d(sb + OFF_KQ + 0, &tm_k, 0, (int)t0, fb);
        tma_load_2d(sb + OFF_KQ + 16384, &tm_k, 64, (int)t0, fb);
        tma_load_2d(sb + OFF_KQ + 8192, &tm_q, 0, (int)t0, fb);
        tma_load_2d(sb + OFF_KQ + 24576, &tm_q, 64, (int)t0, fb);
        loads = 1;
    }
    if (warp == 0) {
        bs[lane] = lane < Cc ? beta[t0 + lane] : 0.f;
        bs[lane + 32] = lane + 32 < Cc ? beta[t0 + lane + 32] : 0.f;
    }

    // g of thread (segment of 16 positions, channel), one d-block ahead: the second
    // d-block's loads are under way while the first is processed
    const int gch = tid & 63, gseg = tid >> 6;
    float gv[16];
    auto load_g = [&](int bb) {
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int i = 16 * gseg + r;
            gv[r] = i < Cc ? g[(t0 + i) * kD + 64 * bb + gch] : 0.f;   // zero past the end: identity steps
        }
    };
    load_g(0);
    for (int b = 0; b < 2; ++b) {
        // ---- Gamma of channels 64 b .. 64 b + 63 --------------------------------------
        {
            const int ch = gch, seg = gseg;
            float acc[16];
            float run = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                run += gv[r];
                acc[r] = run;
            }
            if (b == 0) load_g(1);
            segt[seg * 64 + ch] = run;
            named_bar_sync(kBar, kNT);
            float off = 0.f;
            for (int s2 = 0; s2 < seg; ++s2) off += segt[s2 * 64 + ch];
            const float L2E = 1.4426950408889634f;
#pragma unroll
            for (int r = 0; r < 16; ++r) Gm[fidx(16 * seg + r, ch)] = (acc[r] + off) * L2E;
        }
        // the K/Q tiles have landed (first d-block); the previous d-block's products
        // have read the B tiles (second)
        ok = b == 0 ? ctl.wait(B_FULL, 0) : wait_mma(x);
        if (named_bar_any(kBar, kNT, !ok)) goto done;
        tc_fence_after();
        // ---- factor tables (over the segment totals, read by now) ----------------------
        for (int idx = tid; idx < TAB_ROWS * 64; idx += kNT) {
            const int tr = idx >> 6, ch = idx & 63;
            float v;
            if (tr < TAB_FC) {
                v = ex2_approx(Gm[fidx(16 * tr + 8, ch)]);
            } else if (tr < TAB_R) {
                v = ex2_approx(Gm[fidx(63, ch)] - Gm[fidx(16 * (tr - TAB_FC) + 8, ch)]);
            } else {
                const int p = tr - TAB_R;                       // (I, b) in the order of tab_pair
                const int I = (int)((0x3333222110ull >> (4 * p)) & 15), bb = (int)((0x3210210100ull >> (4 * p)) & 15);
                v = ex2_approx(Gm[fidx(16 * I + 8, ch)] - Gm[fidx(16 * bb + 8, ch)]);
            }
            tab[idx] = v;
        }
        named_bar_sync(kBar, kNT);

        // ---- scaled operands: (row i, 8-channel chunk gq) per item, two per thread ------
#pragma unroll 1
        for (int u = 0; u < 2; ++u) {
            const int x = tid + u * kNT;
            const int i = x >> 3, gq = x & 7, blk = i >> 4;
            float gi[8], gm[8], kv[8], qv[8], e1[8], r1[8], f[8], t8[8];
            load8(Gm + fidx(i, 8 * gq), gi);
            load8(Gm + fidx(16 * blk + 8, 8 * gq), gm);
            const uint32_t ka = sb + OFF_KQ + b * 16384 + sw128_off(i, gq);
            unpack8(ld_shared_v4(ka), kv);
            unpack8(ld_shared_v4(ka + 8192), qv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                e1[e] = ex2_approx(fminf(gi[e] - gm[e], kCap2));
                r1[e] = ex2_approx(fminf(gm[e] - gi[e], kCap2));
            }
            const float* trow = tab + 8 * gq;
            const int64_t grow = (tile * kC + i) * kD + 64 * b + 8 * gq;   // workspace element
            // K (.) e^Gamma for W, and Qh = scale Q (.) e^Gamma
            load8(trow + (TAB_EM + blk) * 64, t8);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = e1[e] * t8[e];
            st_shared_u4(sb + OFF_KW + b * 8192 + sw128_off(i, gq), scaled8(kv, f));
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] *= scale;
            const uint4 qh = scaled8(qv, f);
            st_global_v4(qh_out + grow, qh.x, qh.y, qh.z, qh.w);
            // K~ = K (.) e^(Gamma_last - Gamma)
            load8(trow + (TAB_FC + blk) * 64, t8);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = r1[e] * t8[e];
            const uint4 kt = scaled8(kv, f);
            st_global_v4(kt_out + grow, kt.x, kt.y, kt.z, kt.w);
            if (i == 63) {
                float4* gp = reinterpret_cast<float4*>(gam_out + tile * kD + 64 * b + 8 * gq);
                gp[0] = make_float4(ex2_approx(gi[0]), ex2_approx(gi[1]), ex2_approx(gi[2]), ex2_approx(gi[3]));
                gp[1] = make_float4(ex2_approx(gi[4]), ex2_approx(gi[5]), ex2_approx(gi[6]), ex2_approx(gi[7]));
            }
            // B tiles of the blocks I >= blk: K (.) e^(Gamma_mI - Gamma)
#pragma unroll 1
            for (int I = blk; I < 4; ++I) {
                load8(trow + (TAB_R + tab_pair(I, blk)) * 64, t8);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = r1[e] * t8[e];
                st_shared_u4(sb + OFF_B + b_off(I) + sw128_off(i, gq), scaled8(kv, f));
            }
            // [K^;Q^] in place: rows scaled by e^(Gamma_i - Gamma_m(i))
            st_shared_u4(ka, scaled8(kv, e1));
            st_shared_u4(ka + 8192, scaled8(qv, e1));
        }
        fence_async_smem();
        tc_fence_before();
        named_bar_sync(kBar, kNT);
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int I = 0; I < 4; ++I) {
                const uint32_t idesc = idesc_bf16(128, 16 * (I + 1), 0, 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + d_col(I), sw128_desc(sb + OFF_KQ + b * 16384 + kk * 32, 16, 1024),
                             sw128_desc(sb + OFF_B + b_off(I) + kk * 32, 16, 1024), idesc, (b | kk) > 0);
            }
            mma_commit(ctl.bar(B_MMA));
        }
    }
    ok = wait_mma(x);
    if (named_bar_any(kBar, kNT, !ok)) goto done;
    tc_fence_after();
    if (tid == 0 && load) {
        // V over the K/Q tiles, which the gram has read
        const uint32_t fb = ctl.bar(B_FULL);
        mbar_arrive_expect_tx(fb, 2 * 8192);
        tma_load_2d(sb + OFF_KQ + 0, &tm_v, 0, (int)t0, fb);
        tma_load_2d(sb + OFF_KQ + 8192, &tm_v, 64, (int)t0, fb);
        loads = 2;
    }

    // ---- A (lanes 0-63) and P (lanes 64-127) from the D_I: row i reads D of its own
    //      block; warps 0-3 take columns 0-31, warps 4-7 columns 32-63 ------------------
    {
        const int q = warp & 3, h = warp >> 2;
        const int i = ((q & 1) << 5) + lane;          // row within A or P
        const int blo = (q & 1) * 2;                  // blocks of the warp's lanes: blo, blo + 1
        const uint32_t lane_base = tmem + ((uint32_t)(q << 5) << 16);
        const int j0 = 32 * h;
        if (q < 2) {
            if (!(q == 0 && h == 1)) {                // rows 0-31 x columns 32-63: above the diagonal
                float vlo[32], vhi[32];
                tmem_ld32(lane_base + d_col(blo) + j0, vlo);
                tmem_ld32(lane_base + d_col(blo + 1) + j0, vhi);
                tmem_wait_ld();
                const float bi = bs[i];
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    float a[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = j0 + 4 * q4 + e;
                        const float v = lane < 16 ? vlo[4 * q4 + e] : vhi[4 * q4 + e];
                        a[e] = j < i ? bi * v : 0.f;
                    }
                    *reinterpret_cast<float4*>(Am + fidx(i, j0 + 4 * q4)) = make_float4(a[0], a[1], a[2], a[3]);
                }
                if (warp == 0 || warp == 5) {
                    // the diagonal blocks of the rows just written: 0 and 1 (warp 0), 2 and 3 (warp 5)
                    __syncwarp();
                    wy::wy_diag2(Am, Tm, warp == 0 ? 0 : 2, lane);
                }
            }
        } else {
            __nv_bfloat16* prow = p_out + (tile * kC + i) * kC + j0;
            if (q == 2 && h == 1) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) st_global_v4(prow + 8 * q4, 0u, 0u, 0u, 0u);
            } else {
                float vlo[32], vhi[32];
                tmem_ld32(lane_base + d_col(blo) + j0, vlo);
                tmem_ld32(lane_base + d_col(blo + 1) + j0, vhi);
                tmem_wait_ld();
                const float si = i < Cc ? scale : 0.f;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float pv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = j0 + 8 * q4 + e;
                        const float v = lane < 16 ? vlo[8 * q4 + e] : vhi[8 * q4 + e];
                        pv[e] = j <= i ? si * v : 0.f;
                    }
                    st_global_v4(prow + 8 * q4, pack_bf16x2(pv[0], pv[1]), pack_bf16x2(pv[2], pv[3]),
                                 pack_bf16x2(pv[4], pv[5]), pack_bf16x2(pv[6], pv[7]));
                }
            }
        }
    }
    tc_fence_before();
    named_bar_sync(kBar, kNT);

    // ---- T = (I + A)^-1; warp 6 raises the previous tile's ready flag meanwhile --------
    wy::wy_solve(Am, Tm, warp, lane, kBar, [&] {
        if (tid == kStoreTid) {
            publish_pending(ar, pending);
            prefetch_next(ar, ticket);
        }
    });

    // ---- T diag(beta) as a bf16 operand tile over A (zero above the block diagonal) ---
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int x = tid + u * kNT;
        const int i = x >> 3, ch = x & 7;
        uint32_t b4[4] = {0u, 0u, 0u, 0u};
        if ((ch >> 1) <= (i >> 4)) {
            const float4 t0v = *reinterpret_cast<const float4*>(Tm + fidx(i, 8 * ch));
            const float4 t1v = *reinterpret_cast<const float4*>(Tm + fidx(i, 8 * ch + 4));
            const float4 c0 = *reinterpret_cast<const float4*>(bs + 8 * ch);
            const float4 c1 = *reinterpret_cast<const float4*>(bs + 8 * ch + 4);
            b4[0] = pack_bf16x2(t0v.x * c0.x, t0v.y * c0.y); b4[1] = pack_bf16x2(t0v.z * c0.z, t0v.w * c0.w);
            b4[2] = pack_bf16x2(t1v.x * c1.x, t1v.y * c1.y); b4[3] = pack_bf16x2(t1v.z * c1.z, t1v.w * c1.w);
        }
        st_shared_v4(sb + OFF_G + sw128_off(i, ch), b4[0], b4[1], b4[2], b4[3]);
    }
    fence_async_smem();
    tc_fence_before();
    named_bar_sync(kBar, kNT);

    // ---- W^T = Kw^T Tb^T, u^T = V^T Tb^T ----------------------------------------------
    if (tid == 0) {
        ok = ctl.wait(B_FULL, 1);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, 64, 1, 0);    // A MN-major, B K-major
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + TM_W, sw128_desc(sb + OFF_KW + kk * 2048, 8192, 1024),
                         sw128_desc(sb + OFF_G + kk * 32, 16, 1024), idesc, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + TM_U, sw128_desc(sb + OFF_KQ + kk * 2048, 8192, 1024),
                         sw128_desc(sb + OFF_G + kk * 32, 16, 1024), idesc, kk > 0);
            mma_commit(ctl.bar(B_MMA));
        }
    }
    {
        const bool ok2 = wait_mma(x);               // (every thread counts the completion)
        ok = ok && ok2;
    }
    if (named_bar_any(kBar, kNT, !ok)) goto done;
    tc_fence_after();

    // ---- -W row-major [64][128] and u^T [128][64] over V ----------------------------------
    {
        // warp w: TMEM lane quarter w % 4 (-W: d_k channels; u^T: d_v rows), positions
        // 32 (w / 4) .. 32 (w / 4) + 31 of both
        const int q = warp & 3, hh = warp >> 2;
        const int r = (q << 5) + lane;
        const uint32_t lanes = tmem + ((uint32_t)(q << 5) << 16);
        float v[32];
        // -W row-major [64 positions][128 d_k] as two [64][128 B] column blocks: lane r is column r
        tmem_ld32(lanes + TM_W + hh * 32, v);
        tmem_wait_ld();
        const uint32_t base = sb + OFF_KQ + (uint32_t)(r >> 6) * 8192 + (uint32_t)(r & 7) * 2;
        const int ch = (r & 63) >> 3;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int i = hh * 32 + e;
            st_shared_b16(base + (uint32_t)(i * 128 + ((ch ^ (i & 7)) << 4)), __float2bfloat16_rn(-v[e]));
        }
        // u^T [128 d_v][64 positions]: lane r is row r
        tmem_ld32(lanes + TM_U + hh * 32, v);
        tmem_wait_ld();
        const uint32_t dst = sb + OFF_KQ + 16384;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
            st_shared_v4(dst + sw128_off(r, hh * 4 + q4), pack_bf16x2(v[8 * q4 + 0], v[8 * q4 + 1]),
                         pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]), pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]),
                         pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
    }
    fence_async_smem();
    tc_fence_before();
    named_bar_sync(kBar, kNT);
    if (tid == kStoreTid) {
        tma_store_2d(&tm_w, 0, (int)(tile * kC), sb + OFF_KQ);
        tma_store_2d(&tm_w, 64, (int)(tile * kC), sb + OFF_KQ + 8192);
        tma_store_2d(&tm_u, 0, (int)(tile * kD), sb + OFF_KQ + 16384);
        bulk_commit_group();
        // the staging tiles are read: the space is free for the next tile's loads
        bulk_wait_read_all();
        pending = tile;
    }
    if (tid == kStoreTid) *reinterpret_cast<volatile unsigned int*>(x.sm + OFF_BAR + 24) = ticket;
    tc_fence_before();
    named_bar_sync(kBar, kNT);
    return true;

done:
    tc_fence_before();
    named_bar_sync(kBar, kNT);
    if (tid == 0) {
        // let the loads land before the shared memory is reused or released
        if (loads > 0) mbar_wait_bounded(ctl.bar(B_FULL), (uint32_t)(loads - 1), kWaitNs);
    }
    if (tid == kStoreTid) {
        publish_pending(ar, pending);
        bulk_wait_all();
    }
    *ctl.abort = 1;
    return false;
}


}  // namespace kda
}  // namespace dn
