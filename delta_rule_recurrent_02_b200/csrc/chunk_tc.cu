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
//   O   = scale (e^G * Q) S + P U,              P = scale tril(Q K^T * D)
//   S  <- e^(G_last) S + (K * e^(G_last - G))^T U
//
// Every product is issued as tcgen05.mma (bf16 operands in shared memory,
// fp32 accumulators in TMEM) with M = 128 by computing the transposed
// products: the d_v (or d_k) dimension is the MMA's M, the chunk is its N.
//
//   gram   [K;Q] K^T          M=128 (64 key rows, 64 query rows) N=64  K=d_k
//   W^T  = K^T (T diag(beta e^G))^T                      M=d_k  N=64   K=64
//   u^T  = V^T (T diag(beta))^T                          M=d_v  N=64   K=64
//   U^T  = u^T - S^T W^T                                 M=d_v  N=64   K=d_k
//   O1^T = S^T Q^T                                       M=d_v  N=64   K=d_k
//   dS^T = U^T (K * e^(G_last - G))                      M=d_v  N=d_k  K=64
//   O2^T = U^T P^T                                       M=d_v  N=64   K=64
//
// The fp32 state lives in registers (thread = one value column j, one half of
// the key channels) and a bf16 copy S^T in shared memory feeds the MMAs; the
// 64 x 64 unit-lower system is inverted in fp32 on the CUDA cores (blocked:
// 16 x 16 diagonal inverses by forward substitution, then the off-diagonal
// blocks by block products).  q, k and v tiles arrive by TMA (128-byte
// swizzle) into a double-buffered stage, prefetched two chunks ahead.
//
// One CTA owns one (b, h) for the whole sequence.  A partial last chunk is
// handled by treating rows >= Cc as beta = 0, g = 0 (rows past the tensor's
// end are zero-filled by TMA; rows of the next head are masked out), which
// equals zero padding.  Every wait on an mbarrier is bounded; on a timeout
// the kernel records it in the status word, drains its own copies and exits.
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
constexpr int kNT = 256;        // 8 warps: two warpgroups
// TMEM columns (fp32, 128 lanes)
constexpr uint32_t TM_G = 0, TM_W = 64, TM_U = 128, TM_O1 = 192, TM_O2 = 256, TM_S = 320;
constexpr uint32_t TM_COLS = 512;
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // 2 stages x 32 KiB: [d-block][K rows 0-63 | Q rows 64-127][128 B]
constexpr uint32_t SZ_KQ = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x 16 KiB: [d-block][64 rows][128 B]
constexpr uint32_t SZ_V = 16384;
constexpr uint32_t OFF_ST = 98304;      // S^T bf16, K-major A: [c-block][128 rows j][128 B]   32 KiB
constexpr uint32_t OFF_UT = 131072;     // U^T bf16, K-major A: [128 rows][128 B]; fp32 A during the solve
constexpr uint32_t OFF_WT = 147456;     // W^T bf16, MN-major B: [128 rows c][128 B]; fp32 T during the solve
constexpr uint32_t OFF_KT = 163840;     // K * e^(G_last - G), MN-major B: [c-block][64 rows][128 B]
constexpr uint32_t OFF_TW = 180224;     // T diag(beta e^G), K-major B [64 rows i][128 B]
constexpr uint32_t OFF_TB = 188416;     // T diag(beta)
constexpr uint32_t OFF_PM = 196608;     // P, K-major B [64 rows i][128 B]
constexpr uint32_t OFF_MISC = 204800;   // gates, barriers, TMEM slot, flags
constexpr uint32_t SMEM_BYTES = OFF_MISC + 2048 + 1024;
constexpr uint32_t STAGE_TX = 6 * 8192; // six 64 x 64 bf16 boxes per stage
constexpr uint64_t kWaitNs = 1000000000ull;

__device__ __forceinline__ int aidx(int i, int j) { return i * 64 + (j ^ (i & 31)); }

}  // namespace

template <int GATE>
__global__ void __launch_bounds__(kNT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ beta,
                const float* __restrict__ g, const float* S0, __nv_bfloat16* __restrict__ o,
                float* S_T, int T, float scale, unsigned int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    float* bs = reinterpret_cast<float*>(sm + OFF_MISC);   // beta (0 past the chunk's end)
    float* Gs = bs + 64;                                      // inclusive cumulative log-decay
    float* eGs = Gs + 64;                                     // e^G_i
    float* eTs = eGs + 64;                                    // e^(G_last - G_i)
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_MISC + 1024);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC + 1024 + 64);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 1024 + 72);
    float* Am = reinterpret_cast<float*>(sm + OFF_UT);
    float* Tm = reinterpret_cast<float*>(sm + OFF_WT);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2;                              // warpgroup: which half of the columns
    const int row = ((warp & 3) << 5) + lane;              // TMEM lane of this thread
    const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
    const int64_t bh = blockIdx.x;
    const int nchunks = (T + kC - 1) / kC;
    const uint32_t bar_full[2] = {smem_u32(&bars[0]), smem_u32(&bars[1])};
    const uint32_t bar_mma = smem_u32(&bars[2]);

    if (tid == 0) {
        mbar_init(bar_full[0], 1);
        mbar_init(bar_full[1], 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), TM_COLS);
        tmem_relinquish();
    }

    // State: this thread holds S[c][j] for j = row, c = 64 wg + n.
    float Sreg[64];
    {
        const float* src = S0 ? S0 + (bh * kD + wg * 64) * kD + row : nullptr;
#pragma unroll
        for (int n = 0; n < 64; ++n) Sreg[n] = src ? src[(int64_t)n * kD] : 0.f;
        const uint32_t st = sb + OFF_ST + wg * 16384;
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8)
            st_shared_v4(st + sw128_off(row, q8),
                         pack_bf16x2(Sreg[8 * q8 + 0], Sreg[8 * q8 + 1]), pack_bf16x2(Sreg[8 * q8 + 2], Sreg[8 * q8 + 3]),
                         pack_bf16x2(Sreg[8 * q8 + 4], Sreg[8 * q8 + 5]), pack_bf16x2(Sreg[8 * q8 + 6], Sreg[8 * q8 + 7]));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto issue = [&](int cc) {
        const int s = cc & 1;
        const int y = (int)(bh * T + (int64_t)cc * kC);
        const uint32_t kq = sb + OFF_KQ + s * SZ_KQ, vv = sb + OFF_V + s * SZ_V;
        mbar_arrive_expect_tx(bar_full[s], STAGE_TX);
        tma_load_2d(kq + 0, &tm_k, 0, y, bar_full[s]);
        tma_load_2d(kq + 16384, &tm_k, 64, y, bar_full[s]);
        tma_load_2d(kq + 8192, &tm_q, 0, y, bar_full[s]);
        tma_load_2d(kq + 24576, &tm_q, 64, y, bar_full[s]);
        tma_load_2d(vv + 0, &tm_v, 0, y, bar_full[s]);
        tma_load_2d(vv + 8192, &tm_v, 64, y, bar_full[s]);
    };
    int issued = 0;      // chunks whose loads were issued (leader only)
    if (tid == 0) {
        issue(0);
        issued = 1;
        if (nchunks > 1) { issue(1); issued = 2; }
    }

    // gate values of the next chunk, prefetched by warp 0
    float nb0 = 0.f, nb1 = 0.f, ng0 = 0.f, ng1 = 0.f;
    auto fetch_gates = [&](int cc) {
        const int64_t t0 = bh * T + (int64_t)cc * kC;
        const int Cn = min(kC, T - cc * kC);
        nb0 = lane < Cn ? beta[t0 + lane] : 0.f;
        nb1 = lane + 32 < Cn ? beta[t0 + lane + 32] : 0.f;
        if (GATE == kGateScalar) {
            ng0 = lane < Cn ? g[t0 + lane] : 0.f;
            ng1 = lane + 32 < Cn ? g[t0 + lane + 32] : 0.f;
        }
    };
    if (warp == 0) fetch_gates(0);

    uint32_t mma_phase = 0;
    bool good = true;
    auto wait_mma = [&]() {
        good &= mbar_wait_bounded(bar_mma, mma_phase, kWaitNs);
        mma_phase ^= 1u;
        tc_fence_after();
    };
    // barrier that also spreads a timeout to every thread; returns true to stop
    auto sync_check = [&]() -> bool {
        if (!good) *abort_flag = 1;
        __syncthreads();
        return *abort_flag != 0;
    };

    int c = 0;
    for (; c < nchunks; ++c) {
        const int s = c & 1;
        const int c0 = c * kC;
        const int Cc = min(kC, T - c0);
        const uint32_t KQ = sb + OFF_KQ + s * SZ_KQ;
        const uint32_t VS = sb + OFF_V + s * SZ_V;

        // ---- gates of this chunk (warp 0) ----------------------------------
        if (warp == 0) {
            float b0 = nb0, b1 = nb1, a0 = ng0, a1 = ng1;
            if (c + 1 < nchunks) fetch_gates(c + 1);
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const float y0 = __shfl_up_sync(0xffffffffu, a0, o2);
                const float y1 = __shfl_up_sync(0xffffffffu, a1, o2);
                if (lane >= o2) { a0 += y0; a1 += y1; }
            }
            a1 += __shfl_sync(0xffffffffu, a0, 31);
            const float Glast = __shfl_sync(0xffffffffu, a1, 31);
            bs[lane] = b0; bs[lane + 32] = b1;
            Gs[lane] = a0; Gs[lane + 32] = a1;
            eGs[lane] = expf(a0); eGs[lane + 32] = expf(a1);
            eTs[lane] = expf(Glast - a0); eTs[lane + 32] = expf(Glast - a1);
        }
        // ---- gram: [K;Q] K^T -------------------------------------------------
        // every thread observes the stage's TMA completion (it reads the K tile below)
        good &= mbar_wait_bounded(bar_full[s], (uint32_t)(c >> 1) & 1u, kWaitNs);
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a = KQ + (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(tmem + TM_G, sw128_desc(a, 16, 1024), sw128_desc(a, 16, 1024),
                         idesc_bf16(128, 64, 0, 0), kk > 0);
            }
            mma_commit(bar_mma);
        }
        if (sync_check()) break;
        wait_mma();
        {
            float r[32];
            tmem_ld32(tmem + lane_off + TM_G + wg * 32, r);
            tmem_wait_ld();
            const int jb = wg * 32;
            if (row < 64) {                     // K K^T rows -> A (fp32)
                const int i = row;
                const float bi = bs[i], Gi = Gs[i];
#pragma unroll
                for (int n = 0; n < 32; ++n) {
                    const int j = jb + n;
                    float a = 0.f;
                    if (j < i && i < Cc) a = bi * r[n] * expf(Gi - Gs[j]);
                    Am[aidx(i, j)] = a;
                }
            } else {                            // Q K^T rows -> P (bf16)
                const int i = row - 64;
                const float Gi = Gs[i];
                float p[32];
#pragma unroll
                for (int n = 0; n < 32; ++n) {
                    const int j = jb + n;
                    p[n] = (j <= i && i < Cc) ? scale * r[n] * expf(Gi - Gs[j]) : 0.f;
                }
                const uint32_t pm = sb + OFF_PM;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    st_shared_v4(pm + sw128_off(i, wg * 4 + q4),
                                 pack_bf16x2(p[8 * q4 + 0], p[8 * q4 + 1]), pack_bf16x2(p[8 * q4 + 2], p[8 * q4 + 3]),
                                 pack_bf16x2(p[8 * q4 + 4], p[8 * q4 + 5]), pack_bf16x2(p[8 * q4 + 6], p[8 * q4 + 7]));
            }
        }
        // K * e^(G_last - G) into the MN-major B tile (same swizzled layout as the TMA tile)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int x = tid + u * kNT;            // 0..1023
            const int blk = x >> 9, t = (x >> 3) & 63, ch = x & 7;
            const uint4 w = ld_shared_v4(KQ + blk * 16384 + sw128_off(t, ch));
            const float f = t < Cc ? eTs[t] : 0.f;
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
            float2 e0 = __bfloat1622float2(h[0]), e1 = __bfloat1622float2(h[1]);
            float2 e2 = __bfloat1622float2(h[2]), e3 = __bfloat1622float2(h[3]);
            st_shared_v4(sb + OFF_KT + blk * 8192 + sw128_off(t, ch),
                         pack_bf16x2(f * e0.x, f * e0.y), pack_bf16x2(f * e1.x, f * e1.y),
                         pack_bf16x2(f * e2.x, f * e2.y), pack_bf16x2(f * e3.x, f * e3.y));
        }
        // zero T
#pragma unroll
        for (int u = 0; u < 16; ++u) Tm[tid + u * kNT] = 0.f;
        tc_fence_before();
        if (sync_check()) break;

        // ---- T = (I + A)^-1, blocked ----------------------------------------
        if (warp < 4 && lane < 16) {            // 16 x 16 diagonal inverses
            const int k0 = warp * 16, jj = lane;
            float x[16];
#pragma unroll
            for (int ii = 0; ii < 16; ++ii) {
                float acc = (ii == jj) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < ii; ++m) acc -= Am[aidx(k0 + ii, k0 + m)] * x[m];
                x[ii] = acc;
            }
#pragma unroll
            for (int ii = 0; ii < 16; ++ii) Tm[(k0 + ii) * 64 + k0 + jj] = x[ii];
        }
        __syncthreads();
        {
            const int ii = tid >> 4, jj = tid & 15;
            // T_kl = -D_k sum_{m=l}^{k-1} A_km T_ml, by block diagonals d = k - l
#pragma unroll
            for (int d = 1; d <= 3; ++d) {
                float X[3];
#pragma unroll
                for (int b = 0; b < 4 - d; ++b) {
                    const int l = b, k = b + d;
                    float acc = 0.f;
                    for (int mb = l; mb < k; ++mb)
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            acc += Am[aidx(16 * k + ii, 16 * mb + m)] * Tm[(16 * mb + m) * 64 + 16 * l + jj];
                    X[b] = acc;
                }
                __syncthreads();
#pragma unroll
                for (int b = 0; b < 4 - d; ++b) Tm[(16 * (b + d) + ii) * 64 + 16 * b + jj] = X[b];
                __syncthreads();
#pragma unroll
                for (int b = 0; b < 4 - d; ++b) {
                    const int l = b, k = b + d;
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        acc += Tm[(16 * k + ii) * 64 + 16 * k + m] * Tm[(16 * k + m) * 64 + 16 * l + jj];
                    X[b] = -acc;
                }
                __syncthreads();
#pragma unroll
                for (int b = 0; b < 4 - d; ++b) Tm[(16 * (b + d) + ii) * 64 + 16 * b + jj] = X[b];
                __syncthreads();
            }
        }
        // T diag(beta e^G) and T diag(beta) as bf16 K-major B tiles
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int x = tid + u * kNT;            // 0..511
            const int i = x >> 3, ch = x & 7;
            float tw[8], tb[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int j = ch * 8 + e;
                const float t = Tm[i * 64 + j];
                tb[e] = t * bs[j];
                tw[e] = tb[e] * eGs[j];
            }
            st_shared_v4(sb + OFF_TW + sw128_off(i, ch), pack_bf16x2(tw[0], tw[1]), pack_bf16x2(tw[2], tw[3]),
                         pack_bf16x2(tw[4], tw[5]), pack_bf16x2(tw[6], tw[7]));
            st_shared_v4(sb + OFF_TB + sw128_off(i, ch), pack_bf16x2(tb[0], tb[1]), pack_bf16x2(tb[2], tb[3]),
                         pack_bf16x2(tb[4], tb[5]), pack_bf16x2(tb[6], tb[7]));
        }
        fence_async_smem();
        if (sync_check()) break;

        // ---- W^T = K^T Tw^T, u^T = V^T Tb^T ------------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + TM_W, sw128_desc(KQ + kk * 2048, 16384, 1024),
                         sw128_desc(sb + OFF_TW + kk * 32, 16, 1024), idesc_bf16(128, 64, 1, 0), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + TM_U, sw128_desc(VS + kk * 2048, 8192, 1024),
                         sw128_desc(sb + OFF_TB + kk * 32, 16, 1024), idesc_bf16(128, 64, 1, 0), kk > 0);
            mma_commit(bar_mma);
        }
        wait_mma();
        {
            float r[32];
            tmem_ld32(tmem + lane_off + TM_W + wg * 32, r);
            tmem_wait_ld();
            const uint32_t wt = sb + OFF_WT;       // row = key channel c = row, columns i
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                st_shared_v4(wt + sw128_off(row, wg * 4 + q4),
                             pack_bf16x2(r[8 * q4 + 0], r[8 * q4 + 1]), pack_bf16x2(r[8 * q4 + 2], r[8 * q4 + 3]),
                             pack_bf16x2(r[8 * q4 + 4], r[8 * q4 + 5]), pack_bf16x2(r[8 * q4 + 6], r[8 * q4 + 7]));
        }
        fence_async_smem();
        tc_fence_before();
        if (sync_check()) break;

        // ---- U^T = u^T - S^T W^T, O1^T = S^T Q^T -------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + TM_U, sw128_desc(sb + OFF_ST + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         sw128_desc(sb + OFF_WT + kk * 2048, 8192, 1024), idesc_bf16(128, 64, 0, 1, 1), 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + TM_O1, sw128_desc(sb + OFF_ST + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         sw128_desc(KQ + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, 0, 0), kk > 0);
            mma_commit(bar_mma);
        }
        wait_mma();
        {
            float r[32];
            tmem_ld32(tmem + lane_off + TM_U + wg * 32, r);
            tmem_wait_ld();
            const uint32_t ut = sb + OFF_UT;       // row = value channel j, columns = token i
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                st_shared_v4(ut + sw128_off(row, wg * 4 + q4),
                             pack_bf16x2(r[8 * q4 + 0], r[8 * q4 + 1]), pack_bf16x2(r[8 * q4 + 2], r[8 * q4 + 3]),
                             pack_bf16x2(r[8 * q4 + 4], r[8 * q4 + 5]), pack_bf16x2(r[8 * q4 + 6], r[8 * q4 + 7]));
        }
        fence_async_smem();
        tc_fence_before();
        if (sync_check()) break;

        // ---- dS^T = U^T K~, O2^T = U^T P^T -------------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + TM_S, sw128_desc(sb + OFF_UT + kk * 32, 16, 1024),
                         sw128_desc(sb + OFF_KT + kk * 2048, 8192, 1024), idesc_bf16(128, 128, 0, 1), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + TM_O2, sw128_desc(sb + OFF_UT + kk * 32, 16, 1024),
                         sw128_desc(sb + OFF_PM + kk * 32, 16, 1024), idesc_bf16(128, 64, 0, 0), kk > 0);
            mma_commit(bar_mma);
        }
        wait_mma();
        if (tid == 0 && good && c + 2 < nchunks) {   // stage s is free again
            issue(c + 2);
            issued = c + 3;
        }
        {
            // state update S <- e^(G_last) S + dS and its bf16 copy S^T
            const float gamma = eGs[63];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float r[32];
                tmem_ld32(tmem + lane_off + TM_S + wg * 64 + h * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < 32; ++n) Sreg[h * 32 + n] = gamma * Sreg[h * 32 + n] + r[n];
            }
            const uint32_t st = sb + OFF_ST + wg * 16384;
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8)
                st_shared_v4(st + sw128_off(row, q8),
                             pack_bf16x2(Sreg[8 * q8 + 0], Sreg[8 * q8 + 1]), pack_bf16x2(Sreg[8 * q8 + 2], Sreg[8 * q8 + 3]),
                             pack_bf16x2(Sreg[8 * q8 + 4], Sreg[8 * q8 + 5]), pack_bf16x2(Sreg[8 * q8 + 6], Sreg[8 * q8 + 7]));
            // output o[i][j] = scale e^G_i O1 + O2 for this thread's j = row, i = 32 wg + n
            float r1[32], r2[32];
            tmem_ld32(tmem + lane_off + TM_O1 + wg * 32, r1);
            tmem_ld32(tmem + lane_off + TM_O2 + wg * 32, r2);
            tmem_wait_ld();
            __nv_bfloat16* ob = o + (bh * T + c0) * kD + row;
#pragma unroll
            for (int n = 0; n < 32; ++n) {
                const int i = wg * 32 + n;
                if (i < Cc) ob[(int64_t)i * kD] = __float2bfloat16_rn(scale * eGs[i] * r1[n] + r2[n]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (sync_check()) break;
    }

    const bool aborted = *abort_flag != 0;
    if (aborted) {
        if (tid == 0) {
            // let every load this CTA issued land before the CTA's shared memory is released
            for (int cc = c; cc < issued; ++cc)
                mbar_wait_bounded(bar_full[cc & 1], (uint32_t)(cc >> 1) & 1u, kWaitNs);
            atomicOr(status, 1u);
        }
    } else if (S_T) {
        float* dst = S_T + (bh * kD + wg * 64) * kD + row;
#pragma unroll
        for (int n = 0; n < 64; ++n) dst[(int64_t)n * kD] = Sreg[n];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
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
                                                          a.scale, a.status);
    return cudaGetLastError();
}

}  // namespace

bool tc_supports(const ChunkArgs& a) {
    return a.bf16 && a.chunk == kC && a.dk == kD && a.dv == kD && a.gate != kGatePerKey && a.T >= 1 &&
           a.B * a.H * a.T < (int64_t(1) << 31);
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t st) {
    if (a.B * a.H == 0) return cudaSuccess;
    return a.gate == kGateScalar ? launch_tc_gate<kGateScalar>(a, st) : launch_tc_gate<kGateNone>(a, st);
}

}  // namespace dn
