// chunk_tc.cu -- chunked delta-rule prefill on the sm_100a tensor cores.
//
// Same mathematics as the chunkwise form of "Linear attention and Gated
// DeltaNet" (ch. 28, "The chunked form: recurrence as matrix multiplication";
// D2L 12.5, "Training it: the WY trick"): inside a chunk of C = 64 tokens,
// with G_i the inclusive cumulative log-decay and D_ij = e^(G_i - G_j),
//
//   A   = strict_tril(beta_i k_i.k_j D_ij),     T = (I + A)^-1      (UT transform)
//   W   = T diag(beta e^G) K,                   u = T diag(beta) V
//   U   = u - W S                                (values actually written)
//   O   = Qh S + P U,   Qh = scale e^G * Q,     P = scale tril(Q K^T * D)
//   S  <- e^(G_last) S + (K * e^(G_last - G))^T U
//
// Every product runs as tcgen05.mma with M = 128 by computing the transposed
// products (the d_v or d_k dimension is the MMA's M, the chunk is its N):
//
//   gram   [K;Q] K^T       A = K,Q tiles (smem)    B = K tile            -> TMEM G
//   W^T  = K^T Tw^T        A = K tile (MN-major)   B = T diag(beta e^G)  -> TMEM W
//   u^T  = V^T Tb^T        A = V tile (MN-major)   B = T diag(beta)      -> TMEM U
//   U^T += -S^T W^T        A = S^T (TMEM, bf16)    B = W^T (smem)        -> TMEM U
//   O^T  = S^T Qh^T        A = S^T (TMEM, bf16)    B = Qh (smem)         -> TMEM O
//   S^T += U^T K~          A = U^T (TMEM, bf16)    B = K~ (smem)         -> TMEM S
//   O^T += U^T P^T         A = U^T (TMEM, bf16)    B = P (smem)          -> TMEM O
//
// The CTA owns one (b, h) and runs two pipelines that overlap:
//   * the chunk-parallel "prework" of chunk c+1 (gram -> masks -> 64 x 64
//     unit-lower inverse on the CUDA cores -> W, u, Qh, K~, P), and
//   * the sequential state chain of chunk c (U, S, O), whose state stays in
//     TMEM (fp32 accumulator, pre-scaled by the next chunk's decay) with a
//     bf16 copy in TMEM that feeds the next products directly.
// Warp roles: 0 TMA + gate precompute, 1 prework MMA issue, 2 TMEM allocation,
// 3 state-chain MMA issue, 4-11 prework, 12-15 state chain and output.  Stages of q, k, v tiles arrive
// by TMA (128-byte swizzle) two chunks ahead.
//
// A partial last chunk treats rows >= Cc as beta = 0, g = 0 (rows past the
// tensor's end are zero-filled by TMA; rows of the next head are masked),
// which equals zero padding.  Every wait is bounded: on a timeout the kernel
// records it in the status word, lets its own copies land and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "dn_common.cuh"
#include "dn_kernels.h"
#include "sm100.cuh"

namespace dn {

using namespace sm100;

namespace {

constexpr int kC = 64;          // chunk
constexpr int kD = 128;         // d_k = d_v
constexpr int kNT = 512;        // 16 warps
constexpr int kPreWarp0 = 4;    // prework warps 4..11
constexpr int kPreThreads = 256;
constexpr int kChainWarp0 = 12; // chain warps 12..15
constexpr int kChainThreads = 128;

// TMEM columns (32-bit, 128 lanes)
constexpr uint32_t TM_SACC = 0;     // S^T fp32 [dv lanes][dk cols], pre-scaled by the coming chunk's decay
constexpr uint32_t TM_ST = 128;     // S^T bf16 pairs [dv][dk/2]
constexpr uint32_t TM_UT = 192;     // U^T bf16 pairs [dv][C/2]
constexpr uint32_t TM_U = 224;      // U^T fp32 accumulator [dv][C]
constexpr uint32_t TM_O = 288;      // O^T fp32 accumulator [dv][C]
constexpr uint32_t TM_G = 352;      // gram: lanes 0-63 K K^T, 64-127 Q K^T
constexpr uint32_t TM_W = 416;      // W^T fp32 [dk][C]
constexpr uint32_t TM_UK = 480;     // (U * e^(G_last - G))^T bf16 pairs [dv][C/2]
constexpr uint32_t TM_COLS = 512;

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // 2 stages x 32 KiB: [d-block][K rows 0-63 | Q rows 64-127][128 B]
constexpr uint32_t SZ_KQ = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x 16 KiB: [d-block][64 rows][128 B]
constexpr uint32_t SZ_V = 16384;
constexpr uint32_t OFF_QH = 98304;      // Qh (even chunks), K-major B [N=i][K=c]: [c-block][64 rows][128 B]
constexpr uint32_t OFF_QH1 = 147456;    // Qh (odd chunks)
constexpr uint32_t OFF_WT = 114688;     // W^T, MN-major B [K=c rows][N=i]: [128 rows][128 B]
constexpr uint32_t OFF_TW = 131072;     // T diag(beta e^G), K-major B [N=i][K=j]: [64 rows][128 B]
constexpr uint32_t OFF_TB = 139264;     // T diag(beta), same layout
constexpr uint32_t OFF_PM = 163840;     // 2 x P, K-major B [N=i][K=j]: [64 rows][128 B]
constexpr uint32_t OFF_A = 180224;      // fp32 64 x 68: A, then M = D^-1 A
constexpr uint32_t OFF_T = 197632;      // fp32 64 x 68: T = (I + A)^-1
constexpr uint32_t OFF_GATE = 215040;   // 4 gate slots
constexpr uint32_t GATE_FLOATS = 384;
constexpr uint32_t OFF_BAR = OFF_GATE + 4 * GATE_FLOATS * 4;   // mbarriers, TMEM slot, flag
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;
constexpr uint32_t STAGE_TX = 6 * 8192;
constexpr uint64_t kWaitNs = 1000000000ull;

// gate slot layout (floats)
constexpr int G_BETA = 0, G_G2 = 64, G_EG = 128, G_ET = 192, G_BEG = 256, G_GAMMA = 320;

// barrier indices
enum {
    B_FULL0 = 0, B_FULL1, B_FREE0, B_FREE1,              // TMA stages
    B_GATE0, B_GATE1, B_GATE2, B_GATE3,                  // gate slots
    B_GRAM, B_WU, B_WS, B_WSQS, B_KUPU,                  // MMA completions
    B_TW, B_READY, B_KP0, B_KP1, B_GFREE,                // prework -> MMA
    B_UT, B_UFREE, B_ST, B_OFREE,                        // chain -> MMA
    B_COUNT
};

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
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const float4 a = *reinterpret_cast<const float4*>(Y + fidx(yr + m, yc + j0));
        const float4 b = *reinterpret_cast<const float4*>(Y + fidx(yr + m, yc + j0 + 4));
        acc[0] += xrow[m] * a.x; acc[1] += xrow[m] * a.y; acc[2] += xrow[m] * a.z; acc[3] += xrow[m] * a.w;
        acc[4] += xrow[m] * b.x; acc[5] += xrow[m] * b.y; acc[6] += xrow[m] * b.z; acc[7] += xrow[m] * b.w;
    }
}

__device__ __forceinline__ void blk16_store(float* Z, int zr, int zc, const float (&acc)[8], float sign, int lane) {
    const int ii = lane >> 1, j0 = (lane & 1) * 8;
    *reinterpret_cast<float4*>(Z + fidx(zr + ii, zc + j0)) =
        make_float4(sign * acc[0], sign * acc[1], sign * acc[2], sign * acc[3]);
    *reinterpret_cast<float4*>(Z + fidx(zr + ii, zc + j0 + 4)) =
        make_float4(sign * acc[4], sign * acc[5], sign * acc[6], sign * acc[7]);
}

// Store -acc as T block rows (fp32) and as the bf16 B tiles T diag(beta e^G)
// and T diag(beta): lane (ii, j0) owns 8 consecutive columns = one 16-byte chunk.
__device__ __forceinline__ void blk16_store_t(float* Tm, uint32_t tw, uint32_t tb, const float* gs, int zr, int zc,
                                              const float (&acc)[8], int lane, int g_beta, int g_beg) {
    const int ii = lane >> 1, j0 = (lane & 1) * 8;
    float t[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = -acc[e];
    *reinterpret_cast<float4*>(Tm + fidx(zr + ii, zc + j0)) = make_float4(t[0], t[1], t[2], t[3]);
    *reinterpret_cast<float4*>(Tm + fidx(zr + ii, zc + j0 + 4)) = make_float4(t[4], t[5], t[6], t[7]);
    const float4 b0 = *reinterpret_cast<const float4*>(gs + g_beta + zc + j0);
    const float4 b1 = *reinterpret_cast<const float4*>(gs + g_beta + zc + j0 + 4);
    const float4 w0 = *reinterpret_cast<const float4*>(gs + g_beg + zc + j0);
    const float4 w1 = *reinterpret_cast<const float4*>(gs + g_beg + zc + j0 + 4);
    const int row = zr + ii, ch = (zc + j0) >> 3;
    st_shared_v4(tw + sw128_off(row, ch), pack_bf16x2(t[0] * w0.x, t[1] * w0.y), pack_bf16x2(t[2] * w0.z, t[3] * w0.w),
                 pack_bf16x2(t[4] * w1.x, t[5] * w1.y), pack_bf16x2(t[6] * w1.z, t[7] * w1.w));
    st_shared_v4(tb + sw128_off(row, ch), pack_bf16x2(t[0] * b0.x, t[1] * b0.y), pack_bf16x2(t[2] * b0.z, t[3] * b0.w),
                 pack_bf16x2(t[4] * b1.x, t[5] * b1.y), pack_bf16x2(t[6] * b1.z, t[7] * b1.w));
}

__device__ __forceinline__ void zero8(float (&a)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = 0.f;
}

// e^(G_i - G_j) = 2^(G2_i - G2_j) with G2 = G log2(e), for j <= i (the
// exponent is <= 0 for g <= 0; very old positions underflow to 0).
__device__ __forceinline__ float decay2(float g2i, float g2j) { return exp2f(g2i - g2j); }

// Scale 8 bf16 values (one 16-byte chunk) by f and store them at dst.
__device__ __forceinline__ void scale_chunk(uint32_t src, uint32_t dst, float f) {
    const uint4 w = ld_shared_v4(src);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
    const float2 e0 = __bfloat1622float2(h[0]), e1 = __bfloat1622float2(h[1]);
    const float2 e2 = __bfloat1622float2(h[2]), e3 = __bfloat1622float2(h[3]);
    st_shared_v4(dst, pack_bf16x2(f * e0.x, f * e0.y), pack_bf16x2(f * e1.x, f * e1.y),
                 pack_bf16x2(f * e2.x, f * e2.y), pack_bf16x2(f * e3.x, f * e3.y));
}

struct Ctl {
    uint32_t bar0;                 // address of barrier 0
    volatile int* abort;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
    // bounded wait; gives up early once another role has aborted
    __device__ bool wait(int i, uint32_t parity) const {
        const uint32_t b = bar(i);
        if (mbar_try_wait(b, parity)) return true;
        const uint64_t t0 = globaltimer_ns();
        while (true) {
            if (mbar_try_wait_sleep(b, parity, 20000u)) return true;
            if (*abort) return false;
            if (globaltimer_ns() - t0 > kWaitNs) {
                *abort = 1;
                return false;
            }
        }
    }
};

}  // namespace

template <int GATE>
__global__ void __launch_bounds__(kNT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ beta,
                const float* __restrict__ g, const float* S0, __nv_bfloat16* __restrict__ o,
                float* S_T, int T, float scale, unsigned int* status, int test_flags) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the __shared__ array itself so that
    // every access below compiles to a shared-memory (not generic) instruction
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    float* gates = reinterpret_cast<float*>(sm + OFF_GATE);
    float* Am = reinterpret_cast<float*>(sm + OFF_A);
    float* Tm = reinterpret_cast<float*>(sm + OFF_T);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_BAR + 8 * B_COUNT + 8);
    Ctl ctl{sb + OFF_BAR, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.x;
    const int n = (T + kC - 1) / kC;

    if (tid == 0) {
        const uint32_t counts[B_COUNT] = {1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1,
                                          kPreThreads, kPreThreads, kPreThreads, kPreThreads, kPreThreads,
                                          kChainThreads, kChainThreads, kChainThreads, kChainThreads};
        for (int i = 0; i < B_COUNT; ++i) mbar_init(ctl.bar(i), counts[i]);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================= producer: gates + TMA ================================
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        int issued = 0;
        // beta / g of the next chunk, loaded one chunk ahead
        float nb0 = 0.f, nb1 = 0.f, ng0 = 0.f, ng1 = 0.f;
        auto fetch = [&](int cc) {
            const int64_t t0 = bh * T + (int64_t)cc * kC;
            const int Cn = min(kC, T - cc * kC);
            nb0 = lane < Cn ? beta[t0 + lane] : 0.f;
            nb1 = lane + 32 < Cn ? beta[t0 + lane + 32] : 0.f;
            if (GATE == kGateScalar) {
                ng0 = lane < Cn ? g[t0 + lane] : 0.f;
                ng1 = lane + 32 < Cn ? g[t0 + lane + 32] : 0.f;
            }
        };
        fetch(0);
        for (int cc = 0; cc < n; ++cc) {
            const int s = cc & 1;
            // gates of chunk cc into slot cc % 4
            float* gs = gates + (cc & 3) * GATE_FLOATS;
            const int64_t t0 = bh * T + (int64_t)cc * kC;
            const float b0 = nb0, b1 = nb1;
            float a0 = ng0, a1 = ng1;
            if (cc + 1 < n) fetch(cc + 1);
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const float y0 = __shfl_up_sync(0xffffffffu, a0, o2);
                const float y1 = __shfl_up_sync(0xffffffffu, a1, o2);
                if (lane >= o2) { a0 += y0; a1 += y1; }
            }
            a1 += __shfl_sync(0xffffffffu, a0, 31);
            const float Glast = __shfl_sync(0xffffffffu, a1, 31);
            const float L2E = 1.4426950408889634f;
            gs[G_BETA + lane] = b0; gs[G_BETA + lane + 32] = b1;
            gs[G_G2 + lane] = a0 * L2E; gs[G_G2 + lane + 32] = a1 * L2E;
            const float e0 = expf(a0), e1 = expf(a1);
            gs[G_EG + lane] = e0; gs[G_EG + lane + 32] = e1;
            gs[G_BEG + lane] = b0 * e0; gs[G_BEG + lane + 32] = b1 * e1;
            gs[G_ET + lane] = expf(Glast - a0); gs[G_ET + lane + 32] = expf(Glast - a1);
            if (lane == 0) gs[G_GAMMA] = expf(Glast);
            __syncwarp();
            if (lane == 0) mbar_arrive(ctl.bar(B_GATE0 + (cc & 3)));
            // the stage is free once the state product of chunk cc - 2 is done
            if (cc >= 2) {
                bool ok = lane == 0 ? ctl.wait(B_FREE0 + s, (uint32_t)((cc - 2) >> 1) & 1u) : true;
                if (!__shfl_sync(0xffffffffu, (int)ok, 0)) break;
            }
            if (lane == 0 && !(test_flags & 1)) {
                const int y = (int)t0;
                const uint32_t kq = sb + OFF_KQ + s * SZ_KQ, vv = sb + OFF_V + s * SZ_V;
                const uint32_t fb = ctl.bar(B_FULL0 + s);
                mbar_arrive_expect_tx(fb, STAGE_TX);
                tma_load_2d(kq + 0, &tm_k, 0, y, fb);
                tma_load_2d(kq + 16384, &tm_k, 64, y, fb);
                tma_load_2d(kq + 8192, &tm_q, 0, y, fb);
                tma_load_2d(kq + 24576, &tm_q, 64, y, fb);
                tma_load_2d(vv + 0, &tm_v, 0, y, fb);
                tma_load_2d(vv + 8192, &tm_v, 64, y, fb);
            }
            if (!(test_flags & 1)) issued = cc + 1;
        }
        if (*abort_flag && lane == 0) {
            // let every load this CTA issued land before its shared memory is released
            for (int cc = max(0, issued - 2); cc < issued; ++cc)
                mbar_wait_bounded(ctl.bar(B_FULL0 + (cc & 1)), (uint32_t)(cc >> 1) & 1u, kWaitNs);
        }
    } else if (warp == 1 || warp == 3) {
        // ================= MMA issue: warp 1 lane 0 the prework products (gram, W, u),
        // warp 3 lane 0 the state-chain products; each commits its own MMAs =====
        if (lane == 0) {
            const uint32_t I_GRAM = idesc_bf16(128, 64, 0, 0);
            const uint32_t I_MNK = idesc_bf16(128, 64, 1, 0);       // A MN-major, B K-major
            const uint32_t I_WS = idesc_bf16(128, 64, 0, 1, 1);     // -A, B MN-major
            const uint32_t I_KK = idesc_bf16(128, 64, 0, 0);
            const uint32_t I_KU = idesc_bf16(128, 128, 0, 1);
            bool ok = true;
            if (warp == 1) {
                for (int c = 0; ok && c < n; ++c) {
                    const uint32_t par = (uint32_t)c & 1u;
                    // [K;Q] K^T once the stage has landed and the previous gram was read
                    ok = ctl.wait(B_FULL0 + (c & 1), (uint32_t)(c >> 1) & 1u) && (c == 0 || ctl.wait(B_GFREE, par ^ 1u));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t kq = sb + OFF_KQ + (c & 1) * SZ_KQ, vv = sb + OFF_V + (c & 1) * SZ_V;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t a = kq + (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_bf16(tmem + TM_G, sw128_desc(a, 16, 1024), sw128_desc(a, 16, 1024), I_GRAM, kk > 0);
                    }
                    mma_commit(ctl.bar(B_GRAM));
                    // W^T = K^T Tw^T and u^T = V^T Tb^T once T is ready and U was read
                    ok = ctl.wait(B_TW, par) && (c == 0 || ctl.wait(B_UFREE, par ^ 1u));
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + TM_W, sw128_desc(kq + kk * 2048, 16384, 1024),
                                 sw128_desc(sb + OFF_TW + kk * 32, 16, 1024), I_MNK, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + TM_U, sw128_desc(vv + kk * 2048, 8192, 1024),
                                 sw128_desc(sb + OFF_TB + kk * 32, 16, 1024), I_MNK, kk > 0);
                    mma_commit(ctl.bar(B_WU));
                }
            } else {
                for (int c = 0; ok && c < n; ++c) {
                    const uint32_t par = (uint32_t)c & 1u;
                    // U^T += -S^T W^T (the chain's critical product), then O^T = S^T Qh^T
                    // once the previous output has been read
                    ok = ctl.wait(B_READY, par) && ctl.wait(B_ST, par);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tmem + TM_U, tmem + TM_ST + kk * 8,
                                    sw128_desc(sb + OFF_WT + kk * 2048, 8192, 1024), I_WS, 1);
                    mma_commit(ctl.bar(B_WS));
                    ok = c == 0 || ctl.wait(B_OFREE, par ^ 1u);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tmem + TM_O, tmem + TM_ST + kk * 8,
                                    sw128_desc((c & 1 ? sb + OFF_QH1 : sb + OFF_QH) + (kk >> 2) * 8192 + (kk & 3) * 32,
                                               16, 1024), I_KK, kk > 0);
                    mma_commit(ctl.bar(B_WSQS));
                    // S^T += U^T K~ ; O^T += U^T P^T
                    ok = ctl.wait(B_UT, par) && ctl.wait(B_KP0 + (c & 1), (uint32_t)(c >> 1) & 1u);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t kq = sb + OFF_KQ + (c & 1) * SZ_KQ, pm = sb + OFF_PM + (c & 1) * 8192;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tmem + TM_SACC, tmem + TM_UK + kk * 8, sw128_desc(kq + kk * 2048, 16384, 1024),
                                    I_KU, 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tmem + TM_O, tmem + TM_UT + kk * 8, sw128_desc(pm + kk * 32, 16, 1024), I_KK, 1);
                    mma_commit(ctl.bar(B_KUPU));
                    mma_commit(ctl.bar(B_FREE0 + (c & 1)));   // the stage's last reader is done
                }
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp >= kPreWarp0 && warp < kChainWarp0) {
        // ================= prework (256 threads) ================================
        const int pt = tid - kPreWarp0 * 32;       // 0..255
        const int pw = warp - kPreWarp0;           // 0..7
        const int q = warp & 3;                    // TMEM lane quarter
        const int h = pw >> 2;                     // column half
        const int r = (q << 5) + lane;             // TMEM lane (row)
        const uint32_t lane_off = (uint32_t)(q << 5) << 16;
        // the blocks of T above the block diagonal are zero for every chunk
#pragma unroll
        for (int u = 0; u < 4; ++u) st_shared_v4(sb + OFF_TW + (uint32_t)(pt + u * kPreThreads) * 16, 0u, 0u, 0u, 0u);
        for (int c = 0; c < n; ++c) {
            const int s = c & 1;
            const uint32_t par = (uint32_t)c & 1u;
            const int Cc = min(kC, T - c * kC);
            const float* gs = gates + (c & 3) * GATE_FLOATS;
            const uint32_t kq = sb + OFF_KQ + s * SZ_KQ;
            bool ok = ctl.wait(B_GATE0 + (c & 3), (uint32_t)(c >> 2) & 1u) && ctl.wait(B_GRAM, par) &&
                      ctl.wait(B_FULL0 + s, (uint32_t)(c >> 1) & 1u);
            if (!ok) *abort_flag = 1;
            if (named_bar_any(1, kPreThreads, !ok)) break;
            tc_fence_after();
            // ---- gram rows: A = strict_tril(beta_i (K K^T)_ij D_ij) (fp32, for the solve)
            //      and P = scale tril((Q K^T)_ij D_ij) (bf16 B tile), rows i < Cc --------
            {
                float v[32];
                tmem_ld32(tmem + lane_off + TM_G + h * 32, v);
                tmem_wait_ld();
                const float* g2p = gs + G_G2 + h * 32;
                if (r < 64) {
                    const int i = r;
                    const float bi = i < Cc ? gs[G_BETA + i] : 0.f;
                    const float g2i = gs[G_G2 + i];
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 gj = *reinterpret_cast<const float4*>(g2p + 4 * q4);
                        const float gjv[4] = {gj.x, gj.y, gj.z, gj.w};
                        float a[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = h * 32 + q4 * 4 + e;
                            a[e] = j < i ? bi * v[q4 * 4 + e] * decay2(g2i, gjv[e]) : 0.f;
                        }
                        *reinterpret_cast<float4*>(Am + fidx(i, h * 32 + q4 * 4)) = make_float4(a[0], a[1], a[2], a[3]);
                    }
                } else {
                    const int i = r - 64;
                    const float si = i < Cc ? scale : 0.f;
                    const float g2i = gs[G_G2 + i];
                    const uint32_t pm = sb + OFF_PM + (c & 1) * 8192;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 ga = *reinterpret_cast<const float4*>(g2p + 8 * q4);
                        const float4 gb = *reinterpret_cast<const float4*>(g2p + 8 * q4 + 4);
                        const float gjv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                        float p[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = h * 32 + q4 * 8 + e;
                            p[e] = j <= i ? si * v[q4 * 8 + e] * decay2(g2i, gjv[e]) : 0.f;
                        }
                        st_shared_v4(pm + sw128_off(i, h * 4 + q4), pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]),
                                     pack_bf16x2(p[4], p[5]), pack_bf16x2(p[6], p[7]));
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_KP0 + (c & 1)));
            mbar_arrive(ctl.bar(B_GFREE));
            named_bar_sync(1, kPreThreads);
            // ---- 16 x 16 diagonal inverses D_k = (I + A_kk)^-1 into T -------------
            if (pw < 4 && lane < 16) {
                const int k0 = pw * 16, jj = lane;
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
            named_bar_sync(1, kPreThreads);
            // ---- M_kl = D_k A_kl (k > l), in place of A_kl ----------------------------
            if (pw < 6) {
                const int kb[6] = {1, 2, 3, 2, 3, 3}, lb[6] = {0, 0, 0, 1, 1, 2};
                const int k = kb[pw], l = lb[pw];
                float acc[8];
                zero8(acc);
                blk16(Tm, 16 * k, 16 * k, Am, 16 * k, 16 * l, acc, lane);
                __syncwarp();
                blk16_store(Am, 16 * k, 16 * l, acc, 1.f, lane);
            } else {
                // warps 6, 7: diagonal blocks D_k of T -> bf16 Tw / Tb chunks
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int x = (pw - 6) * 32 + lane + u * 64;     // 0..127
                    const int blk = x >> 5, i = 16 * blk + ((x >> 1) & 15), j0 = 16 * blk + 8 * (x & 1);
                    const float4 t0 = *reinterpret_cast<const float4*>(Tm + fidx(i, j0));
                    const float4 t1 = *reinterpret_cast<const float4*>(Tm + fidx(i, j0 + 4));
                    const float4 b0 = *reinterpret_cast<const float4*>(gs + G_BETA + j0);
                    const float4 b1 = *reinterpret_cast<const float4*>(gs + G_BETA + j0 + 4);
                    const float4 w0 = *reinterpret_cast<const float4*>(gs + G_BEG + j0);
                    const float4 w1 = *reinterpret_cast<const float4*>(gs + G_BEG + j0 + 4);
                    st_shared_v4(sb + OFF_TW + sw128_off(i, j0 >> 3), pack_bf16x2(t0.x * w0.x, t0.y * w0.y),
                                 pack_bf16x2(t0.z * w0.z, t0.w * w0.w), pack_bf16x2(t1.x * w1.x, t1.y * w1.y),
                                 pack_bf16x2(t1.z * w1.z, t1.w * w1.w));
                    st_shared_v4(sb + OFF_TB + sw128_off(i, j0 >> 3), pack_bf16x2(t0.x * b0.x, t0.y * b0.y),
                                 pack_bf16x2(t0.z * b0.z, t0.w * b0.w), pack_bf16x2(t1.x * b1.x, t1.y * b1.y),
                                 pack_bf16x2(t1.z * b1.z, t1.w * b1.w));
                }
            }
            named_bar_sync(1, kPreThreads);
            // ---- T_kl = -sum_{m=l}^{k-1} M_km T_ml, three rounds ----------------------
            {
                float acc[8];
                zero8(acc);
                const uint32_t tw = sb + OFF_TW, tb = sb + OFF_TB;
                if (pw == 0) { blk16(Am, 16, 0, Tm, 0, 0, acc, lane); blk16_store_t(Tm, tw, tb, gs, 16, 0, acc, lane, G_BETA, G_BEG); }
                if (pw == 1) { blk16(Am, 32, 16, Tm, 16, 16, acc, lane); blk16_store_t(Tm, tw, tb, gs, 32, 16, acc, lane, G_BETA, G_BEG); }
                if (pw == 2) { blk16(Am, 48, 32, Tm, 32, 32, acc, lane); blk16_store_t(Tm, tw, tb, gs, 48, 32, acc, lane, G_BETA, G_BEG); }
                if (pw == 3) blk16(Am, 32, 0, Tm, 0, 0, acc, lane);
                if (pw == 4) blk16(Am, 48, 16, Tm, 16, 16, acc, lane);
                if (pw == 5) blk16(Am, 48, 0, Tm, 0, 0, acc, lane);
                named_bar_sync(1, kPreThreads);
                if (pw == 3) { blk16(Am, 32, 16, Tm, 16, 0, acc, lane); blk16_store_t(Tm, tw, tb, gs, 32, 0, acc, lane, G_BETA, G_BEG); }
                if (pw == 4) { blk16(Am, 48, 32, Tm, 32, 16, acc, lane); blk16_store_t(Tm, tw, tb, gs, 48, 16, acc, lane, G_BETA, G_BEG); }
                if (pw == 5) blk16(Am, 48, 16, Tm, 16, 0, acc, lane);
                named_bar_sync(1, kPreThreads);
                if (pw == 5) { blk16(Am, 48, 32, Tm, 32, 0, acc, lane); blk16_store_t(Tm, tw, tb, gs, 48, 0, acc, lane, G_BETA, G_BEG); }
            }
            fence_async_smem();
            mbar_arrive(ctl.bar(B_TW));
            // ---- Qh into this chunk's buffer (the previous user, two chunks back, is done) ----
            {
                const uint32_t qh = (c & 1) ? sb + OFF_QH1 : sb + OFF_QH;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int x = pt + u * kPreThreads;        // 0..1023
                    const int blk = x >> 9, i = (x >> 3) & 63, ch = x & 7;
                    const float f = i < Cc ? scale * gs[G_EG + i] : 0.f;
                    scale_chunk(kq + blk * 16384 + 8192 + sw128_off(i, ch), qh + blk * 8192 + sw128_off(i, ch), f);
                }
            }
            // ---- W^T (TMEM) -> smem once W is computed and the previous chunk's product read it
            ok = ctl.wait(B_WU, par) && (c == 0 || ctl.wait(B_WS, par ^ 1u));
            if (!ok) *abort_flag = 1;
            if (named_bar_any(1, kPreThreads, !ok)) break;
            tc_fence_after();
            {
                float v[32];
                tmem_ld32(tmem + lane_off + TM_W + h * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    st_shared_v4(sb + OFF_WT + sw128_off(r, h * 4 + q4),
                                 pack_bf16x2(v[8 * q4 + 0], v[8 * q4 + 1]), pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                                 pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]), pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_READY));
        }
    } else if (warp >= kChainWarp0) {
        // ================= state chain and output (128 threads) =================
        const int j = ((warp & 3) << 5) + lane;      // value channel = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
        bool ok = ctl.wait(B_GATE0, 0);
        if (!ok) *abort_flag = 1;
        ok = !named_bar_any(2, kChainThreads, !ok);
        if (ok) {
            // S0 -> TMEM: fp32 pre-scaled by chunk 0's decay, and its bf16 copy
            const float gamma0 = gates[G_GAMMA];
#pragma unroll 1
            for (int pc = 0; pc < 4; ++pc) {
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = S0 ? S0[(bh * kD + pc * 32 + e) * kD + j] : 0.f;
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                tmem_st16(tmem + lane_off + TM_ST + pc * 16, pk);
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= gamma0;
                tmem_st32(tmem + lane_off + TM_SACC + pc * 32, v);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_ST));
        }
        for (int c = 0; ok && c < n; ++c) {
            const uint32_t par = (uint32_t)c & 1u;
            const int Cc = min(kC, T - c * kC);
            // ---- U^T -> bf16 pairs in TMEM ------------------------------------------
            ok = ctl.wait(B_WS, par);
            if (!ok) *abort_flag = 1;
            if (named_bar_any(2, kChainThreads, !ok)) { ok = false; break; }
            tc_fence_after();
            const float* gsc = gates + (c & 3) * GATE_FLOATS;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float v[32];
                tmem_ld32(tmem + lane_off + TM_U + hh * 32, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                tmem_st16(tmem + lane_off + TM_UT + hh * 16, pk);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 et = *reinterpret_cast<const float4*>(gsc + G_ET + hh * 32 + 4 * q4);
                    pk[2 * q4] = pack_bf16x2(v[4 * q4 + 0] * et.x, v[4 * q4 + 1] * et.y);
                    pk[2 * q4 + 1] = pack_bf16x2(v[4 * q4 + 2] * et.z, v[4 * q4 + 3] * et.w);
                }
                tmem_st16(tmem + lane_off + TM_UK + hh * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_UT));
            mbar_arrive(ctl.bar(B_UFREE));
            // ---- state: S_{c+1} = gamma_c S_c + dS (already summed in TMEM) ---------------
            ok = ctl.wait(B_KUPU, par) && (c + 1 >= n || ctl.wait(B_GATE0 + ((c + 1) & 3), (uint32_t)((c + 1) >> 2) & 1u));
            if (!ok) *abort_flag = 1;
            if (named_bar_any(2, kChainThreads, !ok)) { ok = false; break; }
            tc_fence_after();
            const bool last = c + 1 == n;
            const float gnext = last ? 1.f : gates[((c + 1) & 3) * GATE_FLOATS + G_GAMMA];
#pragma unroll 1
            for (int pc = 0; pc < 4; ++pc) {
                float v[32];
                tmem_ld32(tmem + lane_off + TM_SACC + pc * 32, v);
                tmem_wait_ld();
                if (last) {
                    if (S_T) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) S_T[(bh * kD + pc * 32 + e) * kD + j] = v[e];
                    }
                } else {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                    tmem_st16(tmem + lane_off + TM_ST + pc * 16, pk);
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] *= gnext;
                    tmem_st32(tmem + lane_off + TM_SACC + pc * 32, v);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_ST));
            // ---- output rows of this chunk -----------------------------------------------
            __nv_bfloat16* ob = o + (bh * T + (int64_t)c * kC) * kD + j;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float v[32];
                tmem_ld32(tmem + lane_off + TM_O + hh * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = hh * 32 + e;
                    if (i < Cc) ob[(int64_t)i * kD] = __float2bfloat16_rn(v[e]);
                }
            }
            tc_fence_before();
            mbar_arrive(ctl.bar(B_OFREE));
        }
        if (!ok) *abort_flag = 1;
    }

    __syncthreads();
    if (*abort_flag && tid == 0) atomicOr(status, 1u);
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ---- host side ---------------------------------------------------------------

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [rows, 128] bf16 row-major, 64 x 64 boxes, 128-byte swizzle, zero fill past the end.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int GATE>
cudaError_t launch_tc_gate(const ChunkArgs& a, cudaStream_t st) {
    CUtensorMap tq, tk, tv;
    const uint64_t rows = (uint64_t)(a.B * a.H * a.T);
    if (!make_tmap(&tq, a.q, rows) || !make_tmap(&tk, a.k, rows) || !make_tmap(&tv, a.v, rows))
        return cudaErrorInvalidValue;
    auto kern = chunk_tc_kernel<GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.B * a.H), kNT, SMEM_BYTES, st>>>(tq, tk, tv, a.beta, a.g, a.S0,
                                                          static_cast<__nv_bfloat16*>(a.o), a.S_T, (int)a.T,
                                                          a.scale, a.status, a.test_flags);
    return cudaGetLastError();
}

}  // namespace

bool tc_supports(const ChunkArgs& a) {
    return a.bf16 && a.chunk == kC && a.dk == kD && a.dv == kD && a.gate != kGatePerKey &&
           a.B * a.H * a.T < (int64_t(1) << 31);
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t st) {
    if (a.B * a.H == 0) return cudaSuccess;
    return a.gate == kGateScalar ? launch_tc_gate<kGateScalar>(a, st) : launch_tc_gate<kGateNone>(a, st);
}

}  // namespace dn
