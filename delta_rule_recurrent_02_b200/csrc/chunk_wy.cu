// chunk_wy.cu -- the UT/WY transform of every chunk, in parallel over
// (b, h, chunk), on the sm_100a tensor cores and CUDA cores.
//
// Same mathematics as "Linear attention and Gated DeltaNet" (ch. 28, "The
// chunked form") and D2L 12.5 ("Training it: the WY trick"): inside a chunk
// of C = 64 tokens, with G_i the inclusive cumulative log-decay and
// D_ij = e^(G_i - G_j),
//
//   A = strict_tril(beta_i k_i.k_j D_ij),   T = (I + A)^-1   (unit lower)
//   W = T diag(beta e^G) K,                 u = T diag(beta) V
//
// Nothing here depends on the state, so every chunk is an independent CTA (two
// fit on an SM).  W^T and u^T leave as bf16 [128][64] tiles of the workspace,
// which the state-pass kernel (chunk_tc.cu) streams back with TMA.  One CTA:
//
//   TMA       K (loaded twice, stacked, so that the gram has M = 128) and V
//   tcgen05   [K;K] K^T -> TMEM (bf16 -> fp32)
//   CUDA core masks and decay -> A (fp32, shared memory)
//   CUDA core T = (I + A)^-1: the 16 x 16 diagonal blocks D_k = (I + A_kk)^-1
//             by forward substitution, M_kl = D_k A_kl, then
//             T_kl = -sum_{m=l}^{k-1} M_km T_ml in three rounds (fp32);
//             T diag(beta e^G) and T diag(beta) as bf16 operand tiles
//   tcgen05   W^T = K^T (T diag(beta e^G))^T, u^T = V^T (T diag(beta))^T -> TMEM
//   epilogue  TMEM -> bf16 -> workspace
//
// A partial last chunk has beta = 0 and g = 0 past its end: those rows of A,
// and those columns of W^T and u^T, are zero (equal to zero padding).  Rows
// past the end of the tensor are zero-filled by TMA; rows of the next head
// are multiplied by those zeros.  Every wait is bounded; on a timeout the CTA
// records it in the status word and exits.
#include "chunk_tc_common.cuh"
#include "dn_kernels.h"

namespace dn {

using namespace sm100;
using namespace tc;

namespace {

constexpr int kNT = 256;        // 8 warps

// TMEM columns (32-bit, 128 lanes)
constexpr uint32_t TM_G = 0;    // gram [K;K] K^T (lanes 64-127 repeat lanes 0-63)
constexpr uint32_t TM_W = 0;    // W^T fp32 [dk][C], after the gram has been read
constexpr uint32_t TM_U = 64;   // u^T fp32 [dv][C]
constexpr uint32_t TM_COLS = 128;

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_K = 0;           // [d-block][K rows | K rows again][128 B] = 32 KiB
constexpr uint32_t OFF_TW = 8192;       // T diag(beta e^G) in d-block 0's copy, once the gram is done
constexpr uint32_t OFF_TB = 24576;      // T diag(beta) in d-block 1's copy
constexpr uint32_t OFF_V = 32768;       // [d-block][64 rows][128 B] = 16 KiB
constexpr uint32_t OFF_A = 49152;       // fp32 64 x 68: A, then M = D^-1 A
constexpr uint32_t OFF_T = 66560;       // fp32 64 x 68: T = (I + A)^-1
constexpr uint32_t OFF_GATE = 83968;    // one gate slot
constexpr uint32_t OFF_BAR = OFF_GATE + GATE_FLOATS * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
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
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const float4 a = *reinterpret_cast<const float4*>(Y + fidx(yr + m, yc + j0));
        const float4 b = *reinterpret_cast<const float4*>(Y + fidx(yr + m, yc + j0 + 4));
        acc[0] += xrow[m] * a.x; acc[1] += xrow[m] * a.y; acc[2] += xrow[m] * a.z; acc[3] += xrow[m] * a.w;
        acc[4] += xrow[m] * b.x; acc[5] += xrow[m] * b.y; acc[6] += xrow[m] * b.z; acc[7] += xrow[m] * b.w;
    }
}

__device__ __forceinline__ void blk16_store(float* Z, int zr, int zc, const float (&acc)[8], int lane) {
    const int ii = lane >> 1, j0 = (lane & 1) * 8;
    *reinterpret_cast<float4*>(Z + fidx(zr + ii, zc + j0)) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(Z + fidx(zr + ii, zc + j0 + 4)) = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// Eight consecutive entries t[0..7] of T at (row, col0..col0+7) -> one
// 16-byte chunk of each bf16 operand tile, T diag(beta e^G) and T diag(beta).
__device__ __forceinline__ void store_t_tiles(uint32_t tw, uint32_t tb, const float* gs, int row, int col0,
                                              const float (&t)[8]) {
    const float4 b0 = *reinterpret_cast<const float4*>(gs + G_BETA + col0);
    const float4 b1 = *reinterpret_cast<const float4*>(gs + G_BETA + col0 + 4);
    const float4 w0 = *reinterpret_cast<const float4*>(gs + G_BEG + col0);
    const float4 w1 = *reinterpret_cast<const float4*>(gs + G_BEG + col0 + 4);
    const uint32_t off = sw128_off(row, col0 >> 3);
    st_shared_v4(tw + off, pack_bf16x2(t[0] * w0.x, t[1] * w0.y), pack_bf16x2(t[2] * w0.z, t[3] * w0.w),
                 pack_bf16x2(t[4] * w1.x, t[5] * w1.y), pack_bf16x2(t[6] * w1.z, t[7] * w1.w));
    st_shared_v4(tb + off, pack_bf16x2(t[0] * b0.x, t[1] * b0.y), pack_bf16x2(t[2] * b0.z, t[3] * b0.w),
                 pack_bf16x2(t[4] * b1.x, t[5] * b1.y), pack_bf16x2(t[6] * b1.z, t[7] * b1.w));
}

// T_zr,zc = -acc: into T (fp32) and into the two bf16 operand tiles.
__device__ __forceinline__ void blk16_store_t(float* Tm, uint32_t tw, uint32_t tb, const float* gs, int zr, int zc,
                                              const float (&acc)[8], int lane) {
    const int ii = lane >> 1, j0 = (lane & 1) * 8;
    float t[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = -acc[e];
    *reinterpret_cast<float4*>(Tm + fidx(zr + ii, zc + j0)) = make_float4(t[0], t[1], t[2], t[3]);
    *reinterpret_cast<float4*>(Tm + fidx(zr + ii, zc + j0 + 4)) = make_float4(t[4], t[5], t[6], t[7]);
    store_t_tiles(tw, tb, gs, zr + ii, zc + j0, t);
}

__device__ __forceinline__ void zero8(float (&a)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = 0.f;
}

}  // namespace

template <int GATE>
__global__ void __launch_bounds__(kNT, 2)
chunk_wy_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const float* __restrict__ beta, const float* __restrict__ g, __nv_bfloat16* __restrict__ w_out,
                __nv_bfloat16* __restrict__ u_out, int T, int n, unsigned int* status, int test_flags) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the __shared__ array itself so that
    // every access below compiles to a shared-memory (not generic) instruction
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    float* gs = reinterpret_cast<float*>(sm + OFF_GATE);
    float* Am = reinterpret_cast<float*>(sm + OFF_A);
    float* Tm = reinterpret_cast<float*>(sm + OFF_T);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 16);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_BAR + 20);
    Ctl ctl{sb + OFF_BAR, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t tile = blockIdx.x;                 // (b h) n + c
    const int64_t bh = tile / n;
    const int c = (int)(tile - bh * n);
    const int Cc = min(kC, T - c * kC);
    const int64_t t0 = bh * T + (int64_t)c * kC;
    const bool load = !(test_flags & 1);

    if (tid == 0) {
        mbar_init(ctl.bar(B_FULL), 1);
        mbar_init(ctl.bar(B_MMA), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (tid == 0 && load) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        const uint32_t fb = ctl.bar(B_FULL);
        const int y = (int)t0;
        mbar_arrive_expect_tx(fb, 6 * 8192);
        tma_load_2d(sb + OFF_K + 0, &tm_k, 0, y, fb);
        tma_load_2d(sb + OFF_K + 16384, &tm_k, 64, y, fb);
        tma_load_2d(sb + OFF_K + 8192, &tm_k, 0, y, fb);
        tma_load_2d(sb + OFF_K + 24576, &tm_k, 64, y, fb);
        tma_load_2d(sb + OFF_V + 0, &tm_v, 0, y, fb);
        tma_load_2d(sb + OFF_V + 8192, &tm_v, 64, y, fb);
    }
    if (warp == 2) {
        const float b0 = lane < Cc ? beta[t0 + lane] : 0.f;
        const float b1 = lane + 32 < Cc ? beta[t0 + lane + 32] : 0.f;
        float a0 = 0.f, a1 = 0.f;
        if (GATE == kGateScalar) {
            a0 = lane < Cc ? g[t0 + lane] : 0.f;
            a1 = lane + 32 < Cc ? g[t0 + lane + 32] : 0.f;
        }
        chunk_gates(gs, b0, b1, a0, a1, lane);
    }
    bool ok = true;
    if (tid == 0) {
        // [K;K] K^T once K has landed
        ok = ctl.wait(B_FULL, 0);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a = sb + OFF_K + (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(tmem + TM_G, sw128_desc(a, 16, 1024), sw128_desc(a, 16, 1024), idesc, kk > 0);
            }
            mma_commit(ctl.bar(B_MMA));
        }
    }
    __syncthreads();                                  // gates visible
    ok = ok && ctl.wait(B_MMA, 0);
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();

    // ---- A = strict_tril(beta_i (K K^T)_ij D_ij): lane r holds row r mod 64; the two
    //      copies of a row split its columns, the two warps of a lane quarter again ----
    {
        const int q = warp & 3;
        const int r = (q << 5) + lane;
        const int i = r & 63;
        const int j0 = ((r >> 6) << 5) + ((warp >> 2) << 4);
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(q << 5) << 16) + TM_G + j0, v);
        tmem_wait_ld();
        const float bi = gs[G_BETA + i];              // zero past the chunk's end
        const float g2i = gs[G_G2 + i];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const float4 gj = *reinterpret_cast<const float4*>(gs + G_G2 + j0 + 4 * q4);
            const float gjv[4] = {gj.x, gj.y, gj.z, gj.w};
            float a[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = j0 + 4 * q4 + e;
                a[e] = j < i ? bi * v[4 * q4 + e] * decay2(g2i, gjv[e]) : 0.f;
            }
            *reinterpret_cast<float4*>(Am + fidx(i, j0 + 4 * q4)) = make_float4(a[0], a[1], a[2], a[3]);
        }
        // the K copy is free now: zero the operand tiles (their blocks above the
        // block diagonal stay zero)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint32_t off = (uint32_t)(tid + u * kNT) * 16;    // 512 chunks of 16 B per tile
            st_shared_v4(sb + OFF_TW + off, 0u, 0u, 0u, 0u);
            st_shared_v4(sb + OFF_TB + off, 0u, 0u, 0u, 0u);
        }
    }
    tc_fence_before();
    __syncthreads();

    // ---- 16 x 16 diagonal inverses D_k = (I + A_kk)^-1 into T ------------------------
    if (warp < 4 && lane < 16) {
        const int k0 = warp * 16, jj = lane;
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
    __syncthreads();
    // ---- M_kl = D_k A_kl (k > l), in place of A_kl; warps 6, 7: D_k -> operand tiles ----
    if (warp < 6) {
        // (k, l) = (1,0) (2,0) (3,0) (2,1) (3,1) (3,2) for warps 0..5
        const int k = (0x332321 >> (4 * warp)) & 15, l = (0x211000 >> (4 * warp)) & 15;
        float acc[8];
        zero8(acc);
        blk16(Tm, 16 * k, 16 * k, Am, 16 * k, 16 * l, acc, lane);
        __syncwarp();
        blk16_store(Am, 16 * k, 16 * l, acc, lane);
    } else {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int x = (warp - 6) * 32 + lane + u * 64;     // 0..127
            const int blk = x >> 5, i = 16 * blk + ((x >> 1) & 15), j0 = 16 * blk + 8 * (x & 1);
            const float4 t0v = *reinterpret_cast<const float4*>(Tm + fidx(i, j0));
            const float4 t1v = *reinterpret_cast<const float4*>(Tm + fidx(i, j0 + 4));
            const float t[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
            store_t_tiles(sb + OFF_TW, sb + OFF_TB, gs, i, j0, t);
        }
    }
    __syncthreads();
    // ---- T_kl = -sum_{m=l}^{k-1} M_km T_ml, three rounds ------------------------------
    {
        float acc[8];
        zero8(acc);
        const uint32_t tw = sb + OFF_TW, tb = sb + OFF_TB;
        if (warp == 0) { blk16(Am, 16, 0, Tm, 0, 0, acc, lane); blk16_store_t(Tm, tw, tb, gs, 16, 0, acc, lane); }
        if (warp == 1) { blk16(Am, 32, 16, Tm, 16, 16, acc, lane); blk16_store_t(Tm, tw, tb, gs, 32, 16, acc, lane); }
        if (warp == 2) { blk16(Am, 48, 32, Tm, 32, 32, acc, lane); blk16_store_t(Tm, tw, tb, gs, 48, 32, acc, lane); }
        if (warp == 3) blk16(Am, 32, 0, Tm, 0, 0, acc, lane);
        if (warp == 4) blk16(Am, 48, 16, Tm, 16, 16, acc, lane);
        if (warp == 5) blk16(Am, 48, 0, Tm, 0, 0, acc, lane);
        __syncthreads();
        if (warp == 3) { blk16(Am, 32, 16, Tm, 16, 0, acc, lane); blk16_store_t(Tm, tw, tb, gs, 32, 0, acc, lane); }
        if (warp == 4) { blk16(Am, 48, 32, Tm, 32, 16, acc, lane); blk16_store_t(Tm, tw, tb, gs, 48, 16, acc, lane); }
        if (warp == 5) blk16(Am, 48, 16, Tm, 16, 0, acc, lane);
        __syncthreads();
        if (warp == 5) { blk16(Am, 48, 32, Tm, 32, 0, acc, lane); blk16_store_t(Tm, tw, tb, gs, 48, 0, acc, lane); }
    }
    fence_async_smem();
    __syncthreads();

    // ---- W^T = K^T Tw^T, u^T = V^T Tb^T ------------------------------------------------
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, 1, 0);    // A MN-major, B K-major
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + TM_W, sw128_desc(sb + OFF_K + kk * 2048, 16384, 1024),
                     sw128_desc(sb + OFF_TW + kk * 32, 16, 1024), idesc, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + TM_U, sw128_desc(sb + OFF_V + kk * 2048, 8192, 1024),
                     sw128_desc(sb + OFF_TB + kk * 32, 16, 1024), idesc, kk > 0);
        mma_commit(ctl.bar(B_MMA));
    }
    ok = ctl.wait(B_MMA, 1);
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    // ---- TMEM -> bf16 rows of the workspace: warps 0-3 W^T, 4-7 u^T ------------------
    {
        const int q = warp & 3;
        const int r = (q << 5) + lane;
        const bool is_u = warp >= 4;
        __nv_bfloat16* out = (is_u ? u_out : w_out) + (tile * kD + r) * kC;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float v[32];
            tmem_ld32(tmem + ((uint32_t)(q << 5) << 16) + (is_u ? TM_U : TM_W) + hh * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                st_global_v4(out + hh * 32 + q4 * 8, pack_bf16x2(v[8 * q4 + 0], v[8 * q4 + 1]),
                             pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]), pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]),
                             pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
        }
    }

done:
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // let the loads land before the shared memory is released
        if (load) mbar_wait_bounded(ctl.bar(B_FULL), 0, kWaitNs);
        atomicOr(status, 1u);
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ---- host side ---------------------------------------------------------------

namespace {

template <int GATE>
cudaError_t launch_wy_gate(const ChunkArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                           __nv_bfloat16* w_ws, __nv_bfloat16* u_ws, int n, cudaStream_t st) {
    auto kern = chunk_wy_kernel<GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.B * a.H * n), kNT, SMEM_BYTES, st>>>(tk, tv, a.beta, a.g, w_ws, u_ws, (int)a.T, n,
                                                              a.status, a.test_flags);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_wy(const ChunkArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                            __nv_bfloat16* w_ws, __nv_bfloat16* u_ws, cudaStream_t st) {
    const int n = (int)((a.T + kC - 1) / kC);
    return a.gate == kGateScalar ? launch_wy_gate<kGateScalar>(a, tk, tv, w_ws, u_ws, n, st)
                                 : launch_wy_gate<kGateNone>(a, tk, tv, w_ws, u_ws, n, st);
}

}  // namespace dn
