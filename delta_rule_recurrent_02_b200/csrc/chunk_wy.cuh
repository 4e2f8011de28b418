// chunk_wy.cuh -- the state-independent part of one chunk of the chunked delta
// rule (the "WY transform" of "Linear attention and Gated DeltaNet", ch. 28,
// "The chunked form", and D2L 12.5, "Training it: the WY trick"), as a device
// function run by a group of 8 warps: a whole CTA in chunk_wy.cu, or one of
// four groups of a CTA in the single-launch prefill of chunk_tc.cu.
//
// Inside a chunk of C = 64 tokens, with G_i the inclusive cumulative
// log-decay and D_ij = e^(G_i - G_j),
//
//   A = strict_tril(beta_i k_i.k_j D_ij),   T = (I + A)^-1   (unit lower)
//   W = T diag(beta e^G) K,                 u = T diag(beta) V
//   P = scale tril(q_i.k_j D_ij)            (the intra-chunk attention)
//
// written to the workspace as bf16 tiles: -W [64 rows][128] (row-major,
// negated so that S^T (-W)^T = -(W S)^T), u^T [128][64] and P [64][64], then
// the tile's ready flag (release).  Steps of one tile:
//
//   TMA       K and Q tiles, stacked per 64-column block as [K rows | Q rows]
//   tcgen05   [K;Q] K^T -> TMEM (bf16 -> fp32): K K^T for A, Q K^T for P
//   TMA       V, into the dead K/Q space beside T (it lands during the solve)
//   CUDA core masks and decay -> A (fp32, shared memory); P (bf16) straight to
//             the workspace
//   CUDA core T = (I + A)^-1 at the start of that space: the 16 x 16 diagonal blocks
//             D_k = (I + A_kk)^-1 by forward substitution, M_kl = D_k A_kl,
//             then T_kl = -sum_{m=l}^{k-1} M_km T_ml in three rounds (fp32);
//             then T diag(beta e^G) and T diag(beta) as bf16 operand tiles
//   TMA       K again (from L2) over T
//   tcgen05   W^T = K^T (T diag(beta e^G))^T, u^T = V^T (T diag(beta))^T -> TMEM
//   epilogue  TMEM -> bf16 tiles in shared memory -> TMA stores to the workspace
//
// The ready flag of a tile is raised once its stores are complete, and by a
// thread with time to spare: the output stores are issued by kStoreTid (warp 6),
// which raises the flag during the group's next tile, while warps 0-5 form the
// M blocks and warp 6 has nothing else to do (after the group's last tile, the
// caller raises it with publish_pending()).  The gpu-scope release costs about
// 1.5k cycles under load; there it is off the group's critical path.  Tiles of
// the first two chunks are the exception: every state pass starts by waiting
// for them, so their flags go up as soon as their stores are complete.
//
// A partial last chunk has beta = 0 and g = 0 past its end: those rows of A
// and P, and those columns of W^T and u^T, are zero (equal to zero padding).
// Rows past the end of the tensor are zero-filled by TMA; rows of the next
// head are multiplied by those zeros.  Every wait is bounded; on a timeout the
// group stops.
#pragma once

#include "chunk_tc_common.cuh"

namespace dn {
namespace wy {

using namespace sm100;
using namespace tc;

constexpr int kNT = 256;        // 8 warps per group
constexpr int kStoreTid = 192;  // issues the output stores and raises the ready flags

// TMEM columns (32-bit, 128 lanes)
constexpr uint32_t TM_G = 0;    // gram [K;Q] K^T: lanes 0-63 K K^T, 64-127 Q K^T
constexpr uint32_t TM_W = 0;    // W^T fp32 [dk][C], after the gram has been read
constexpr uint32_t TM_U = 64;   // u^T fp32 [dv][C]
constexpr uint32_t TM_COLS = 128;

// shared memory (bytes from a 1024-aligned base), in the order of use:
//   [0, 32K)      the gram's [K0 | Q0 | K1 | Q1] (d-block b's 64 x 64 bf16 K and Q tiles)
//   [0, 17K)      T (fp32, padded rows), while V = [V0 | V1] lands in [17K, 33K)
//   [0, 16K)      K = [K0 | K1] again, beside V, for W and u
//   [0, 32K)      the -W and u^T output tiles
//   [33K, 50K)    A, then M = D^-1 A; then the bf16 Tw, Tb operand tiles
constexpr uint32_t OFF_KV = 0;
constexpr uint32_t OFF_T = 0;           // fp32 64 x 68: T = (I + A)^-1
constexpr uint32_t OFF_V = 17408;       // V tiles, loaded once the gram has read K and Q
constexpr uint32_t OFF_A = 33792;       // fp32 64 x 68: A, then M = D^-1 A; then the bf16 tiles
constexpr uint32_t OFF_TW = OFF_A;      //   T diag(beta e^G), K-major B [N=i][K=j]: [64 rows][128 B]
constexpr uint32_t OFF_TB = OFF_A + 8192;   // T diag(beta), same layout
constexpr uint32_t OFF_GATE = OFF_A + 17408;   // one gate slot
constexpr uint32_t OFF_BAR = OFF_GATE + GATE_FLOATS * 4;
constexpr uint32_t GROUP_BYTES = 54272;  // one group's shared memory, a multiple of 1024
// (the last 16 bytes of a group stay free: a CTA keeps its TMEM address there)
static_assert(OFF_BAR + 64 <= GROUP_BYTES - 16, "group layout");
static_assert(OFF_T + 64 * 68 * 4 <= OFF_V && OFF_V + 16384 <= OFF_A, "T, V and A overlap");
static_assert(OFF_V % 1024 == 0 && OFF_A % 1024 == 0 && OFF_TB % 1024 == 0, "128-byte swizzle atoms");
enum { B_FULL = 0, B_MMA = 1 };

// fp32 64 x 64 matrix, rows padded to 68 floats: 16-byte aligned rows, and
// rows r and r + 1 start 4 banks apart (conflict-free row, column and 16 x 16
// block accesses)
constexpr int kFS = 68;
__device__ __forceinline__ int fidx(int i, int j) { return i * kFS + j; }

// acc[e] += sum_m X[xr + ii][xc + m] * Y[yr + m][yc + j0 + e] over a 16 x 16
// block pair; lane -> (ii = lane / 2, j0 = 8 (lane % 2)).
__device__ __forceinline__ void blk16(const float* X, int xr, int xc, const float* Y, int yr, int yc,
                                      float (&acc)[8], int lane) {
    const int ii = lane >> 1, j0 = (lane & 1) * 8;
    float xrow[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(X + fidx(xr + ii, xc + 4 * q));
        xrow[4 * q + 0] = v.x; xrow[4 * q + 1] = v.y; xrow[4 * q + 2] = v.z; xrow[4 * q + 3] = v.w;
    }
    // packed fp32 FMAs (two IEEE-rounded FMAs per instruction: the same results as eight
    // scalar ones, in half the issue slots the SM's four groups share)
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const float4 a = *reinterpret_cast<const float4*>(Y + fidx(yr + m, yc + j0));
        const float4 b = *reinterpret_cast<const float4*>(Y + fidx(yr + m, yc + j0 + 4));
        ffma2(acc[0], acc[1], xrow[m], a.x, a.y);
        ffma2(acc[2], acc[3], xrow[m], a.z, a.w);
        ffma2(acc[4], acc[5], xrow[m], b.x, b.y);
        ffma2(acc[6], acc[7], xrow[m], b.z, b.w);
    }
}

__device__ __forceinline__ void blk16_store(float* Z, int zr, int zc, const float (&acc)[8], int lane) {
    const int ii = lane >> 1, j0 = (lane & 1) * 8;
    *reinterpret_cast<float4*>(Z + fidx(zr + ii, zc + j0)) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(Z + fidx(zr + ii, zc + j0 + 4)) = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// T_zr,zc = -acc (fp32).
__device__ __forceinline__ void blk16_store_neg(float* Tm, int zr, int zc, const float (&acc)[8], int lane) {
    const int ii = lane >> 1, j0 = (lane & 1) * 8;
    *reinterpret_cast<float4*>(Tm + fidx(zr + ii, zc + j0)) = make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
    *reinterpret_cast<float4*>(Tm + fidx(zr + ii, zc + j0 + 4)) = make_float4(-acc[4], -acc[5], -acc[6], -acc[7]);
}

__device__ __forceinline__ void zero8(float (&a)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = 0.f;
}


// One group of kNT threads and its resources.  Each mbarrier completes two
// phases per tile (parities 0 then 1), so a group can run tile after tile.
struct Group {
    uint8_t* sm;             // 1024-aligned shared memory of GROUP_BYTES
    uint32_t sb;             // its shared-space address
    uint32_t tmem;           // first of the group's TM_COLS TMEM columns
    uint32_t bar;            // named barrier of the group's kNT threads
    int tid, warp, lane;     // within the group
    Ctl ctl;
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
    return x;
}

// The ticket taken during the group's last tile (after wy_tile returned true).
__device__ __forceinline__ unsigned int next_ticket(const Group& x) {
    return *reinterpret_cast<volatile const unsigned int*>(x.sm + OFF_BAR + 24);
}

// Barriers and the abort flag of a group (one thread, before the group's first tile).
__device__ __forceinline__ void init_group(const Group& x) {
    mbar_init(x.ctl.bar(B_FULL), 1);
    mbar_init(x.ctl.bar(B_MMA), 1);
    *x.ctl.abort = 0;
    *reinterpret_cast<volatile unsigned int*>(x.sm + OFF_BAR + 28) = 0u;   // no tile's K, Q preloaded
}


struct Args {
    const CUtensorMap* tm_q;
    const CUtensorMap* tm_k;
    const CUtensorMap* tm_v;
    const CUtensorMap* tm_w;
    const CUtensorMap* tm_u;
    __nv_bfloat16* p_out;
    unsigned int* flags;
    const float* beta;
    const float* g;
    int T, n;
    float scale;
    int test_flags;
    unsigned int* counter;   // tile counter of the single launch (null: the caller picks every tile)
    int BH, G;               // with a counter: heads and WY groups (a ticket x is tile G + x)
    // the layer's prologue inside the kernels: beta and g hold the raw inputs b and a,
    // q and k are normalised per row (the per-head A_log, dt_bias; H heads per batch row)
    int prologue;
    const float* A_log;
    const float* dt_bias;
    int H;
    int rep = 1;
    // a packed batch of sequences (null: B independent rows of T tokens): the chunk
    // tables of varlen_tables(), with N sequences; c is then the batch's global chunk
    // index and bh the head
    const int* vl = nullptr;
    int vl_N = 0;
    float* rq = nullptr;     // with the prologue: the workspace's 1 / ||q_i|| rows
};

// Thread kStoreTid, at the end of a tile whose stores have read their staging space:
// the K and Q tiles of the tile that `ticket` names (the group's next) into that
// space, on B_FULL's next phase, so that they land during this tile's tail.  Returns
// whether it did (not for the last tile, a packed batch or without a tile counter).
__device__ __forceinline__ bool preload_next(const Args& ar, const Ctl& ctl, uint32_t sb, unsigned int ticket) {
    if (!ar.counter || ar.vl || (ar.test_flags & 1)) return false;
    const int64_t tn = (int64_t)ar.G + ticket;
    if (tn >= (int64_t)ar.BH * ar.n) return false;
    const int cn = (int)(tn / ar.BH);
    const int64_t bhn = tn - (int64_t)cn * ar.BH;
    const int yk = (int)(key_head(bhn, ar.H, ar.rep) * ar.T + (int64_t)cn * kC);
    const uint32_t fb = ctl.bar(B_FULL);
    mbar_arrive_expect_tx(fb, 4 * 8192);
    tma_load_2d(sb + OFF_KV + 0, ar.tm_k, 0, yk, fb);
    tma_load_2d(sb + OFF_KV + 16384, ar.tm_k, 64, yk, fb);
    tma_load_2d(sb + OFF_KV + 8192, ar.tm_q, 0, yk, fb);
    tma_load_2d(sb + OFF_KV + 24576, ar.tm_q, 64, yk, fb);
    return true;
}

// Thread kStoreTid, during a tile: the inputs of the tile that `ticket` names
// (if any) into L2, so that its loads at the group's next tile hit L2: K, Q
// and V by tensor prefetches, beta and g of a full chunk by bulk prefetches.
__device__ __forceinline__ void prefetch_next(const Args& ar, unsigned int ticket, bool gated) {
    if (!ar.counter) return;
    const int64_t tn = (int64_t)ar.G + ticket;
    if (tn >= (int64_t)ar.BH * ar.n) return;
    const int cn = (int)(tn / ar.BH);
    const int64_t bhn = tn - (int64_t)cn * ar.BH;
    const int64_t y = bhn * ar.T + (int64_t)cn * kC;
    const int64_t yk = key_head(bhn, ar.H, ar.rep) * ar.T + (int64_t)cn * kC;
    tma_prefetch_2d(ar.tm_k, 0, (int)yk);
    tma_prefetch_2d(ar.tm_k, 64, (int)yk);
    tma_prefetch_2d(ar.tm_q, 0, (int)yk);
    tma_prefetch_2d(ar.tm_q, 64, (int)yk);
    tma_prefetch_2d(ar.tm_v, 0, (int)y);
    tma_prefetch_2d(ar.tm_v, 64, (int)y);
    if (ar.T - cn * kC >= kC) {
        bulk_prefetch_l2(ar.beta + y, kC * 4);
        if (gated) bulk_prefetch_l2(ar.g + y, kC * 4);
    }
}

// The 16 x 16 diagonal inverses D_k = (I + A_kk)^-1 of blocks kb and kb + 1
// into T, by forward substitution: one warp, lane -> (block kb + lane / 16,
// column lane % 16).  A's rows of those blocks must be visible to the warp.
__device__ __forceinline__ void wy_diag2(const float* Am, float* Tm, int kb, int lane) {
    {
        const int k0 = (kb + (lane >> 4)) * 16, jj = lane & 15;
        float x[16];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
            float p0 = (ii == jj) ? 1.f : 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
            for (int m = 0; m + 3 < ii; m += 4) {
                const float4 av = *reinterpret_cast<const float4*>(Am + fidx(k0 + ii, k0 + m));
                p0 -= av.x * x[m]; p1 -= av.y * x[m + 1]; p2 -= av.z * x[m + 2]; p3 -= av.w * x[m + 3];
            }
#pragma unroll
            for (int m = ii & ~3; m < ii; ++m) p0 -= Am[fidx(k0 + ii, k0 + m)] * x[m];
            x[ii] = (p0 + p1) + (p2 + p3);
        }
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) Tm[fidx(k0 + ii, k0 + jj)] = x[ii];
    }
}

// T = (I + A)^-1 for the unit-lower 64 x 64 system of one chunk, in fp32 on
// CUDA cores, by a group of 8 warps (named barrier `bar`, kNT threads), once
// the diagonal inverses D_k are in Tm (wy_diag2) and the group has passed a
// barrier.  Am holds A (strictly lower; the blocks above its diagonal blocks
// are never read) and is overwritten by M; Tm receives T on and below the
// block diagonal: M_kl = D_k A_kl, then T_kl = -sum_{m=l}^{k-1} M_km T_ml in
// three rounds (block forward substitution).  idle() is run by warps 6 and 7
// while the others form M.  Ends with a group barrier.
template <class Idle>
__device__ __forceinline__ void wy_solve(float* Am, float* Tm, int warp, int lane, uint32_t bar, Idle idle) {
    // ---- M_kl = D_k A_kl (k > l), in place of A_kl -------------------------------------
    if (warp < 6) {
        // (k, l) = (1,0) (2,0) (3,0) (2,1) (3,1) (3,2) for warps 0..5
        const int k = (0x332321 >> (4 * warp)) & 15, l = (0x211000 >> (4 * warp)) & 15;
        float acc[8];
        zero8(acc);
        blk16(Tm, 16 * k, 16 * k, Am, 16 * k, 16 * l, acc, lane);
        __syncwarp();
        blk16_store(Am, 16 * k, 16 * l, acc, lane);
    } else {
        idle();                                       // warps 6 and 7 have nothing else to do
    }
    named_bar_sync(bar, kNT);
    // ---- T_kl = -sum_{m=l}^{k-1} M_km T_ml, three rounds; one block product per warp
    //      and round, (k, m, l) from the tables below (4 bits each) ----------------------
    {
        // round 1, warps 0-5: T_10, T_21, T_32 complete; T_20, T_31, T_30 start (m = l)
        // round 2, warps 3-5: T_20, T_31 complete (m = l + 1); T_30 continues (m = 1)
        // round 3, warp 5:    T_30 completes (m = 2)
        float acc[8];
        zero8(acc);
        if (warp < 6) {
            const int k = (0x332321 >> (4 * warp)) & 15, l = (0x010210 >> (4 * warp)) & 15;
            blk16(Am, 16 * k, 16 * l, Tm, 16 * l, 16 * l, acc, lane);
            if (warp < 3) blk16_store_neg(Tm, 16 * k, 16 * l, acc, lane);
        }
        named_bar_sync(bar, kNT);
        if (warp >= 3 && warp < 6) {
            const int k = (0x332 >> (4 * (warp - 3))) & 15, m = (0x121 >> (4 * (warp - 3))) & 15;
            const int l = (0x010 >> (4 * (warp - 3))) & 15;
            blk16(Am, 16 * k, 16 * m, Tm, 16 * m, 16 * l, acc, lane);
            if (warp < 5) blk16_store_neg(Tm, 16 * k, 16 * l, acc, lane);
        }
        named_bar_sync(bar, kNT);
        if (warp == 5) {
            blk16(Am, 48, 32, Tm, 32, 0, acc, lane);
            blk16_store_neg(Tm, 48, 0, acc, lane);
        }
    }
    named_bar_sync(bar, kNT);
}

// Thread kStoreTid of a group: raise the ready flag of the group's previous
// tile, if one is pending, once its stores (issued by this thread) are
// complete.  The proxy fence orders those async-proxy writes before the
// release; the other threads' writes of the tile (P) precede it through the
// group barriers.  A reader that acquires the flag and fences its async proxy
// reads the tiles.
__device__ __forceinline__ void publish_pending(const Args& ar, int64_t& pending) {
    if (pending < 0) return;
    bulk_wait_all();
    fence_async_global();
    st_release_gpu(ar.flags + pending, 1u);
    pending = -1;
}

// Chunk c of head bh (of a packed batch: global chunk c of head bh, see
// Args::vl).  `pending` (thread kStoreTid's copy counts) is the
// group's tile whose flag is still to be raised, or -1; on return it is this
// tile.  With a tile counter, thread kStoreTid also takes the group's next
// ticket, prefetches that tile's inputs into L2, and hands the ticket on
// (next_ticket() once this returns).  Returns false (the group's
// abort flag set) if a wait gave up.
// PRO: the layer's prologue (raw gates, unit q and k) is compiled in.
template <int GATE, bool PRO = false>
__device__ __forceinline__ bool wy_tile(const Group& x, const Args& ar, int c, int64_t bh, int64_t& pending) {
    const uint32_t sb = x.sb;
    float* gs = reinterpret_cast<float*>(x.sm + OFF_GATE);
    float* Am = reinterpret_cast<float*>(x.sm + OFF_A);
    float* Tm = reinterpret_cast<float*>(x.sm + OFF_T);
    const Ctl& ctl = x.ctl;
    volatile int* abort_flag = ctl.abort;
    const uint32_t tmem = x.tmem;
    const int tid = x.tid, warp = x.warp, lane = x.lane;
    const int T = ar.T, n = ar.n;
    const float scale = ar.scale;
    const float* __restrict__ beta = ar.beta;
    const float* __restrict__ g = ar.g;
    __nv_bfloat16* __restrict__ p_out = ar.p_out;
    const CUtensorMap& tm_q = *ar.tm_q;
    const CUtensorMap& tm_k = *ar.tm_k;
    const CUtensorMap& tm_v = *ar.tm_v;
    const CUtensorMap& tm_w = *ar.tm_w;
    const CUtensorMap& tm_u = *ar.tm_u;
    int64_t tile, t0, t0k;
    int Cc;
    if (ar.vl) {
        // chunk cs of sequence s: rows cu[s] + 64 cs .. of head bh in the packed [H][T][d] arrays
        const VarlenTables vt{ar.vl, ar.vl_N};
        const int s = vt.seq_of()[c];
        const int cs = c - vt.coff()[s];
        const int beg = vt.cu()[s], len = vt.cu()[s + 1] - beg;
        tile = (int64_t)c * ar.H + bh;
        Cc = min(kC, len - cs * kC);
        t0 = bh * T + beg + (int64_t)cs * kC;
        t0k = t0;
    } else {
        tile = bh * n + c;
        Cc = min(kC, T - c * kC);
        t0 = bh * T + (int64_t)c * kC;
        t0k = key_head(bh, ar.H, ar.rep) * T + (int64_t)c * kC;   // q and k rows
    }
    const bool load = !(ar.test_flags & 1);
    int loads = 0;                                   // load groups issued (thread 0)
    // the next ticket, taken now (by the thread that prefetches for it and hands it on)
    // and used after the tile: its latency is hidden
    const unsigned int ticket = tid == kStoreTid && ar.counter ? atomicAdd(ar.counter, 1u) : 0u;

    if (tid == 0 && load) {
        // (unless the group's previous tile issued them at its end)
        if (*reinterpret_cast<volatile const unsigned int*>(x.sm + OFF_BAR + 28) == 0u) {
            const uint32_t fb = ctl.bar(B_FULL);
            const int y = (int)t0k;
            mbar_arrive_expect_tx(fb, 4 * 8192);
            tma_load_2d(sb + OFF_KV + 0, &tm_k, 0, y, fb);
            tma_load_2d(sb + OFF_KV + 16384, &tm_k, 64, y, fb);
            tma_load_2d(sb + OFF_KV + 8192, &tm_q, 0, y, fb);
            tma_load_2d(sb + OFF_KV + 24576, &tm_q, 64, y, fb);
        }
        loads = 1;
    }
    if (warp == 2) {
        float b0 = lane < Cc ? beta[t0 + lane] : 0.f;
        float b1 = lane + 32 < Cc ? beta[t0 + lane + 32] : 0.f;
        float a0 = 0.f, a1 = 0.f;
        if (GATE == kGateScalar) {
            a0 = lane < Cc ? g[t0 + lane] : 0.f;
            a1 = lane + 32 < Cc ? g[t0 + lane + 32] : 0.f;
        }
        if (PRO) {
            // beta and g from the raw inputs (positions past the end stay identity steps)
            const int h = (int)(bh % ar.H);
            const float eA = expf(ar.A_log[h]), dtb = ar.dt_bias[h];
            const float bm = (float)ar.prologue;
            if (lane < Cc) gdn_raw_gates_fast(b0, a0, eA, dtb, bm);
            if (lane + 32 < Cc) gdn_raw_gates_fast(b1, a1, eA, dtb, bm);
        }
        chunk_gates(gs, b0, b1, a0, a1, lane);
    }
    bool ok = true;
    if (tid == 0) {
        // [K;Q] K^T once the tiles have landed; with the prologue [K;Q][K;Q]^T (the same
        // cost for N = 128 as for 64), whose diagonal holds ||k_i||^2 and ||q_i||^2
        ok = ctl.wait(B_FULL, 0);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, PRO ? 128 : 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a = sb + OFF_KV + (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(tmem + TM_G, sw128_desc(a, 16, 1024), sw128_desc(a, 16, 1024), idesc, kk > 0);
            }
            mma_commit(ctl.bar(B_MMA));
        }
    }
    named_bar_sync(x.bar, kNT);                       // gates visible
    ok = ok && ctl.wait(B_MMA, 0);
    if (named_bar_any(x.bar, kNT, !ok)) goto done;
    tc_fence_after();
    if (tid == 0 && load) {
        // V into the second half of the K/Q space, which the gram has read; the
        // phase also counts the K tiles issued after the solve
        const uint32_t fb = ctl.bar(B_FULL);
        mbar_arrive_expect_tx(fb, 4 * 8192);
        tma_load_2d(sb + OFF_V + 0, &tm_v, 0, (int)t0, fb);
        tma_load_2d(sb + OFF_V + 8192, &tm_v, 64, (int)t0, fb);
        loads = 2;
    }

    // ---- A = strict_tril(beta_i (K K^T)_ij D_ij) from TMEM lanes 0-63 (warps 0, 1, 4, 5)
    //      and P = scale tril((Q K^T)_ij D_ij) from lanes 64-127 (warps 2, 3, 6, 7), 32
    //      columns per thread --------------------------------------------------------------
    {
        const int q = warp & 3;
        const int i = ((q & 1) << 5) + lane;
        const int j0 = (warp >> 2) << 5;
        const float g2i = gs[G_G2 + i];
        float rq_i = 0.f;
        if constexpr (PRO) {
            // 1 / max(||x_i||, 1e-12) from the gram's diagonal, before A and P: the key
            // norms by warps 0 and 5 (whose A columns hold the diagonal) into the gate
            // slot, with T diag(beta e^G) taking r_kj by scaling beta e^G; the query norms
            // by the P warps 2, 3 and 7 for their own rows (warps 2 and 3 also write them
            // to the workspace, published with the tile, for the state pass's Qh)
            const bool kdiag = q < 2 && j0 == (q << 5);
            const bool qdiag = q >= 2 && !(q == 2 && j0 == 32);
            if (kdiag || qdiag) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(q << 5) << 16) + TM_G + (kdiag ? j0 : 64 + ((q - 2) << 5)), v);
                tmem_wait_ld();
                float dsq = v[0];
#pragma unroll
                for (int e = 1; e < 32; ++e) dsq = lane == e ? v[e] : dsq;
                const float rn = fminf(rsqrtf(dsq), 1e12f);
                if (kdiag) {
                    gs[G_RK + i] = rn;
                    gs[G_BEG + i] *= rn;
                } else {
                    rq_i = rn;
                    if (j0 == 0 && ar.rq) ar.rq[tile * kC + i] = rn;
                }
            }
            named_bar_sync(x.bar, kNT);
        }
        if (q == 0 && j0 == 32) {
            // A rows 0-31 x columns 32-63 lie above the diagonal: never read
        } else if (q < 2) {
            float v[32];
            tmem_ld32(tmem + ((uint32_t)(q << 5) << 16) + TM_G + j0, v);
            tmem_wait_ld();
            const float bi = PRO ? gs[G_BETA + i] * gs[G_RK + i] : gs[G_BETA + i];   // zero past the chunk's end
            const float* g2c = gs + G_G2;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                const float4 gj = *reinterpret_cast<const float4*>(g2c + j0 + 4 * q4);
                const float gjv[4] = {gj.x, gj.y, gj.z, gj.w};
                // with the prologue, column j also takes r_kj
                const float4 rk = PRO ? *reinterpret_cast<const float4*>(gs + G_RK + j0 + 4 * q4)
                                      : make_float4(1.f, 1.f, 1.f, 1.f);
                const float rkv[4] = {rk.x, rk.y, rk.z, rk.w};
                float a[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j0 + 4 * q4 + e;
                    a[e] = j < i ? bi * v[4 * q4 + e] * (PRO ? decay2(g2i, gjv[e]) * rkv[e] : decay2(g2i, gjv[e]))
                                 : 0.f;
                }
                *reinterpret_cast<float4*>(Am + fidx(i, j0 + 4 * q4)) = make_float4(a[0], a[1], a[2], a[3]);
            }
            if (warp == 0 || warp == 5) {
                // the diagonal blocks of the rows just written: 0 and 1 (warp 0), 2 and 3 (warp 5)
                __syncwarp();
                wy_diag2(Am, Tm, warp == 0 ? 0 : 2, lane);
            }
        } else {
            // P row i, columns j0 .. j0 + 31 -> workspace (row-major [64][64])
            __nv_bfloat16* prow = p_out + (tile * kC + i) * kC + j0;
            if (q == 2 && j0 == 32) {
                // warp 6: the previous tile's ready flag, then zeros: rows 0-31 x
                // columns 32-63 lie above the diagonal
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) st_global_v4(prow + 8 * q4, 0u, 0u, 0u, 0u);
            } else {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(q << 5) << 16) + TM_G + j0, v);
                tmem_wait_ld();
                // (with the prologue, row i also takes 1 / ||q_i||, so that the state pass's
                // output rows come out normalised)
                const float si = i < Cc ? (PRO ? scale * rq_i : scale) : 0.f;
                const float* g2c = gs + G_G2;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 ga = *reinterpret_cast<const float4*>(g2c + j0 + 8 * q4);
                    const float4 gb = *reinterpret_cast<const float4*>(g2c + j0 + 8 * q4 + 4);
                    const float gjv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                    float pv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = j0 + 8 * q4 + e;
                        pv[e] = j <= i ? si * v[8 * q4 + e] * decay2(g2i, gjv[e]) : 0.f;
                    }
                    st_global_v4(prow + 8 * q4, pack_bf16x2(pv[0], pv[1]), pack_bf16x2(pv[2], pv[3]),
                                 pack_bf16x2(pv[4], pv[5]), pack_bf16x2(pv[6], pv[7]));
                }
            }
        }
    }
    tc_fence_before();
    named_bar_sync(x.bar, kNT);

    // ---- T = (I + A)^-1; warp 6 raises the previous tile's ready flag meanwhile --------
    wy_solve(Am, Tm, warp, lane, x.bar, [&] {
        if (tid == kStoreTid) {
            publish_pending(ar, pending);
            prefetch_next(ar, ticket, GATE == kGateScalar);
        }
    });
    // ---- T diag(beta e^G) and T diag(beta) as bf16 operand tiles, over A (zero above
    //      the block diagonal, where T was never written) ----------------------------------
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int x = tid + u * kNT;                   // 0..511: (row, 8-column chunk)
        const int i = x >> 3, ch = x & 7;
        uint32_t w4[4] = {0u, 0u, 0u, 0u}, b4[4] = {0u, 0u, 0u, 0u};
        if ((ch >> 1) <= (i >> 4)) {
            float4 t0v = *reinterpret_cast<const float4*>(Tm + fidx(i, 8 * ch));
            float4 t1v = *reinterpret_cast<const float4*>(Tm + fidx(i, 8 * ch + 4));
            if (PRO) {
                const float ri = gs[G_RK + i];
                t0v.x *= ri; t0v.y *= ri; t0v.z *= ri; t0v.w *= ri;
                t1v.x *= ri; t1v.y *= ri; t1v.z *= ri; t1v.w *= ri;
            }
            // (with the prologue beta e^G / ||k||: W = T diag(beta e^G) K / ||k|| by rows of K)
            const float4 e0 = *reinterpret_cast<const float4*>(gs + G_BEG + 8 * ch);
            const float4 e1 = *reinterpret_cast<const float4*>(gs + G_BEG + 8 * ch + 4);
            const float4 c0 = *reinterpret_cast<const float4*>(gs + G_BETA + 8 * ch);
            const float4 c1 = *reinterpret_cast<const float4*>(gs + G_BETA + 8 * ch + 4);
            w4[0] = pack_bf16x2(t0v.x * e0.x, t0v.y * e0.y); w4[1] = pack_bf16x2(t0v.z * e0.z, t0v.w * e0.w);
            w4[2] = pack_bf16x2(t1v.x * e1.x, t1v.y * e1.y); w4[3] = pack_bf16x2(t1v.z * e1.z, t1v.w * e1.w);
            b4[0] = pack_bf16x2(t0v.x * c0.x, t0v.y * c0.y); b4[1] = pack_bf16x2(t0v.z * c0.z, t0v.w * c0.w);
            b4[2] = pack_bf16x2(t1v.x * c1.x, t1v.y * c1.y); b4[3] = pack_bf16x2(t1v.z * c1.z, t1v.w * c1.w);
        }
        st_shared_v4(sb + OFF_TW + sw128_off(i, ch), w4[0], w4[1], w4[2], w4[3]);
        st_shared_v4(sb + OFF_TB + sw128_off(i, ch), b4[0], b4[1], b4[2], b4[3]);
    }
    fence_async_smem();
    named_bar_sync(x.bar, kNT);

    // ---- K (L2-resident by now) over T, then W^T = K^T Tw^T, u^T = V^T Tb^T -------------
    if (tid == 0) {
        if (load) {
            const uint32_t fb = ctl.bar(B_FULL);     // the phase V opened
            tma_load_2d(sb + OFF_KV + 0, &tm_k, 0, (int)t0k, fb);
            tma_load_2d(sb + OFF_KV + 8192, &tm_k, 64, (int)t0k, fb);
        }
        ok = ctl.wait(B_FULL, 1);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, 64, 1, 0);    // A MN-major, B K-major
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + TM_W, sw128_desc(sb + OFF_KV + kk * 2048, 8192, 1024),
                         sw128_desc(sb + OFF_TW + kk * 32, 16, 1024), idesc, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + TM_U, sw128_desc(sb + OFF_V + kk * 2048, 8192, 1024),
                         sw128_desc(sb + OFF_TB + kk * 32, 16, 1024), idesc, kk > 0);
            mma_commit(ctl.bar(B_MMA));
        }
    }
    ok = ok && ctl.wait(B_MMA, 1);
    if (named_bar_any(x.bar, kNT, !ok)) goto done;
    tc_fence_after();
    // ---- TMEM -> bf16 -W and u^T tiles over K and V (read by now), then TMA stores -------
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
        const uint32_t base = sb + OFF_KV + (uint32_t)(r >> 6) * 8192 + (uint32_t)(r & 7) * 2;
        const int ch = (r & 63) >> 3;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int i = hh * 32 + e;
            st_shared_b16(base + (uint32_t)(i * 128 + ((ch ^ (i & 7)) << 4)), __float2bfloat16_rn(-v[e]));
        }
        // u^T [128 d_v][64 positions]: lane r is row r
        tmem_ld32(lanes + TM_U + hh * 32, v);
        tmem_wait_ld();
        const uint32_t dst = sb + OFF_KV + 16384;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
            st_shared_v4(dst + sw128_off(r, hh * 4 + q4), pack_bf16x2(v[8 * q4 + 0], v[8 * q4 + 1]),
                         pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]), pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]),
                         pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
    }
    fence_async_smem();
    named_bar_sync(x.bar, kNT);
    if (tid == kStoreTid) {
        tma_store_2d(&tm_w, 0, (int)(tile * kC), sb + OFF_KV);
        tma_store_2d(&tm_w, 64, (int)(tile * kC), sb + OFF_KV + 8192);
        tma_store_2d(&tm_u, 0, (int)(tile * kD), sb + OFF_KV + 16384);
        bulk_commit_group();
        // the staging tiles are read: the space takes the next tile's K and Q at once;
        // the flag waits until the stores are complete
        bulk_wait_read_all();
        *reinterpret_cast<volatile unsigned int*>(x.sm + OFF_BAR + 28) = preload_next(ar, ctl, sb, ticket) ? 1u : 0u;
        pending = tile;
        // the first two chunk columns gate the start of every state pass: their flags go up
        // as soon as the stores are complete, not during the group's next tile
        if (c < 2) publish_pending(ar, pending);
    }
    if (tid == kStoreTid) *reinterpret_cast<volatile unsigned int*>(x.sm + OFF_BAR + 24) = ticket;
    tc_fence_before();
    named_bar_sync(x.bar, kNT);
    return true;

done:
    tc_fence_before();
    named_bar_sync(x.bar, kNT);
    if (tid == 0) {
        // let the loads land before the shared memory is reused or released
        if (loads > 0) mbar_wait_bounded(ctl.bar(B_FULL), (uint32_t)(loads - 1), kWaitNs);
    }
    if (tid == kStoreTid) {
        publish_pending(ar, pending);
        bulk_wait_all();
    }
    *abort_flag = 1;
    return false;
}

}  // namespace wy
}  // namespace dn
