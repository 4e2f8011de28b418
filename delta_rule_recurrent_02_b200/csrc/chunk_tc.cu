// chunk_tc.cu -- the sequential state pass of the chunked delta rule on the
// sm_100a tensor cores, fed by the per-chunk W and u of chunk_wy.cu.
//
// Same mathematics as the chunkwise form of "Linear attention and Gated
// DeltaNet" (ch. 28, "The chunked form: recurrence as matrix multiplication";
// D2L 12.5, "Training it: the WY trick"): with W = T diag(beta e^G) K and
// u = T diag(beta) V of each chunk already computed,
//
//   U   = u - W S                                (values actually written)
//   O   = Qh S + P U,   Qh = scale e^G * Q,     P = scale tril(Q K^T * D)
//   S  <- e^(G_last) S + (K * e^(G_last - G))^T U
//
// Every product runs as tcgen05.mma with M = 128 by computing the transposed
// products (d_v is the MMA's M, the chunk its N):
//
//   gram   [K;Q] K^T       A = K,Q tiles (smem)    B = K tile            -> TMEM G (Q rows used)
//   U^T  = -S^T W^T        A = S^T (TMEM, bf16)    B = W^T (smem)        -> TMEM U  (+ u^T in the epilogue)
//   O^T  = S^T Qh^T        A = S^T (TMEM, bf16)    B = Qh (smem)         -> TMEM O
//   S^T += U~^T K          A = U~^T (TMEM, bf16)   B = K tile (smem)     -> TMEM S
//   O^T += U^T P^T         A = U^T (TMEM, bf16)    B = P (smem)          -> TMEM O
//
// with U~ = U * e^(G_last - G) (the decay of K folded into U's rows).  The CTA
// owns one (b, h); its state stays in TMEM (fp32 accumulator, pre-scaled by
// the next chunk's decay, plus a bf16 copy that feeds the next products).
// Warp roles: 0 TMA + gates, 1 gram MMA issue, 2 TMEM allocation, 3 state
// MMA issue, 4-7 P and Qh of the coming chunk, 8-15 state and output (two
// warps per TMEM lane quarter, each half of the columns).  Stages of q, k,
// W^T and u^T tiles arrive by TMA (128-byte swizzle) two chunks ahead.
//
// A partial last chunk treats rows >= Cc as beta = 0, g = 0 (rows past the
// tensor's end are zero-filled by TMA; rows of the next head are masked),
// which equals zero padding.  Every wait is bounded: on a timeout the kernel
// records it in the status word, lets its own copies land and exits.
#include "chunk_tc_common.cuh"
#include "dn_kernels.h"

namespace dn {

using namespace sm100;
using namespace tc;

namespace {

constexpr int kNT = 512;          // 16 warps
constexpr int kSideWarp0 = 4;     // P / Qh warps 4..7
constexpr int kSideThreads = 128;
constexpr int kChainWarp0 = 8;    // state warps 8..15
constexpr int kChainThreads = 256;
static_assert(kSideThreads == (kChainWarp0 - kSideWarp0) * 32 && kChainThreads == kNT - kChainWarp0 * 32,
              "named-barrier thread counts must match the warps of each role");

// TMEM columns (32-bit, 128 lanes)
constexpr uint32_t TM_SACC = 0;     // S^T fp32 [dv lanes][dk cols], pre-scaled by the coming chunk's decay
constexpr uint32_t TM_ST = 128;     // S^T bf16 pairs [dv][dk/2]
constexpr uint32_t TM_UT = 192;     // U^T bf16 pairs [dv][C/2]
constexpr uint32_t TM_U = 224;      // -(W S)^T fp32 accumulator [dv][C]
constexpr uint32_t TM_O = 288;      // O^T fp32 accumulator [dv][C]
constexpr uint32_t TM_G = 352;      // gram: lanes 0-63 K K^T (unused), 64-127 Q K^T
constexpr uint32_t TM_UK = 416;     // U~^T bf16 pairs [dv][C/2]
constexpr uint32_t TM_COLS = 512;

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t SZ_STAGE = 65536;    // one chunk's tiles:
constexpr uint32_t ST_KQ = 0;           //   [d-block][K rows 0-63 | Q rows 64-127][128 B]  32 KiB
constexpr uint32_t ST_WT = 32768;       //   W^T [128 rows (dk)][128 B (C)]                  16 KiB
constexpr uint32_t ST_UT = 49152;       //   u^T [128 rows (dv)][128 B (C)]                  16 KiB
constexpr uint32_t OFF_QH = 131072;     // 2 x Qh, K-major B [N=i][K=c]: [c-block][64 rows][128 B]
constexpr uint32_t OFF_PM = 163840;     // 2 x P, K-major B [N=i][K=j]: [64 rows][128 B]
constexpr uint32_t OFF_GATE = 180224;   // 4 gate slots
constexpr uint32_t OFF_BAR = OFF_GATE + 4 * GATE_FLOATS * 4;   // mbarriers, TMEM slot, flag
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;
constexpr uint32_t STAGE_TX = 65536;

// barrier indices
enum {
    B_FULL0 = 0, B_FULL1, B_FREE0, B_FREE1,              // TMA stages
    B_GATE0, B_GATE1, B_GATE2, B_GATE3,                  // gate slots
    B_GRAM, B_WS, B_WSQS, B_KUPU,                        // MMA completions
    B_READY, B_KP0, B_KP1, B_GFREE,                      // P / Qh warps -> MMA
    B_UT, B_ST, B_OFREE,                                 // state warps -> MMA
    B_COUNT
};

// Scale 8 bf16 values (one 16-byte chunk) by f and store them at dst.
__device__ __forceinline__ void scale_chunk(uint32_t src, uint32_t dst, float f) {
    const uint4 w = ld_shared_v4(src);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
    const float2 e0 = __bfloat1622float2(h[0]), e1 = __bfloat1622float2(h[1]);
    const float2 e2 = __bfloat1622float2(h[2]), e3 = __bfloat1622float2(h[3]);
    st_shared_v4(dst, pack_bf16x2(f * e0.x, f * e0.y), pack_bf16x2(f * e1.x, f * e1.y),
                 pack_bf16x2(f * e2.x, f * e2.y), pack_bf16x2(f * e3.x, f * e3.y));
}

}  // namespace

template <int GATE>
__global__ void __launch_bounds__(kNT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_u,
                const float* __restrict__ beta, const float* __restrict__ g, const float* S0,
                __nv_bfloat16* __restrict__ o, float* S_T, int T, float scale, unsigned int* status,
                int test_flags) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the __shared__ array itself so that
    // every access below compiles to a shared-memory (not generic) instruction
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    float* gates = reinterpret_cast<float*>(sm + OFF_GATE);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_BAR + 8 * B_COUNT + 8);
    Ctl ctl{sb + OFF_BAR, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.x;
    const int n = (T + kC - 1) / kC;

    if (tid == 0) {
        const uint32_t counts[B_COUNT] = {1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1,
                                          kSideThreads, kSideThreads, kSideThreads, kSideThreads,
                                          kChainThreads, kChainThreads, kChainThreads};
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
            prefetch_tmap(&tm_w);
            prefetch_tmap(&tm_u);
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
            const float b0 = nb0, b1 = nb1, a0 = ng0, a1 = ng1;
            if (cc + 1 < n) fetch(cc + 1);
            chunk_gates(gates + (cc & 3) * GATE_FLOATS, b0, b1, a0, a1, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(ctl.bar(B_GATE0 + (cc & 3)));
            // the stage is free once the state product of chunk cc - 2 is done
            if (cc >= 2) {
                bool ok = lane == 0 ? ctl.wait(B_FREE0 + s, (uint32_t)((cc - 2) >> 1) & 1u) : true;
                if (!__shfl_sync(0xffffffffu, (int)ok, 0)) break;
            }
            if (lane == 0 && !(test_flags & 1)) {
                const int y = (int)(bh * T + (int64_t)cc * kC);
                const int yw = (int)((bh * n + cc) * kD);
                const uint32_t st = sb + s * SZ_STAGE;
                const uint32_t fb = ctl.bar(B_FULL0 + s);
                mbar_arrive_expect_tx(fb, STAGE_TX);
                tma_load_2d(st + ST_KQ + 0, &tm_k, 0, y, fb);
                tma_load_2d(st + ST_KQ + 16384, &tm_k, 64, y, fb);
                tma_load_2d(st + ST_KQ + 8192, &tm_q, 0, y, fb);
                tma_load_2d(st + ST_KQ + 24576, &tm_q, 64, y, fb);
                tma_load_2d(st + ST_WT, &tm_w, 0, yw, fb);
                tma_load_2d(st + ST_UT, &tm_u, 0, yw, fb);
            }
            if (!(test_flags & 1)) issued = cc + 1;
        }
        if (*abort_flag && lane == 0) {
            // let every load this CTA issued land before its shared memory is released
            for (int cc = max(0, issued - 2); cc < issued; ++cc)
                mbar_wait_bounded(ctl.bar(B_FULL0 + (cc & 1)), (uint32_t)(cc >> 1) & 1u, kWaitNs);
        }
    } else if (warp == 1 || warp == 3) {
        // ================= MMA issue: warp 1 lane 0 the gram, warp 3 lane 0 the
        // state products; each commits its own MMAs ====================================
        if (lane == 0) {
            const uint32_t I_GRAM = idesc_bf16(128, 64, 0, 0);
            const uint32_t I_WS = idesc_bf16(128, 64, 0, 1, 1);     // -A, B MN-major
            const uint32_t I_KK = idesc_bf16(128, 64, 0, 0);
            const uint32_t I_KU = idesc_bf16(128, 128, 0, 1);
            bool ok = true;
            if (warp == 1) {
                for (int c = 0; ok && c < n; ++c) {
                    // [K;Q] K^T once the stage has landed and the previous gram was read
                    ok = ctl.wait(B_FULL0 + (c & 1), (uint32_t)(c >> 1) & 1u) &&
                         (c == 0 || ctl.wait(B_GFREE, ((uint32_t)c & 1u) ^ 1u));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t kq = sb + (c & 1) * SZ_STAGE + ST_KQ;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t a = kq + (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_bf16(tmem + TM_G, sw128_desc(a, 16, 1024), sw128_desc(a, 16, 1024), I_GRAM, kk > 0);
                    }
                    mma_commit(ctl.bar(B_GRAM));
                }
            } else {
                for (int c = 0; ok && c < n; ++c) {
                    const uint32_t par = (uint32_t)c & 1u;
                    const uint32_t st = sb + (c & 1) * SZ_STAGE;
                    // U^T = -S^T W^T (the chain's critical product) once the tiles and the state are there
                    ok = ctl.wait(B_FULL0 + (c & 1), (uint32_t)(c >> 1) & 1u) && ctl.wait(B_ST, par);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tmem + TM_U, tmem + TM_ST + kk * 8,
                                    sw128_desc(st + ST_WT + kk * 2048, 8192, 1024), I_WS, kk > 0);
                    mma_commit(ctl.bar(B_WS));
                    // O^T = S^T Qh^T once Qh is written and the previous output was read
                    ok = ctl.wait(B_READY, par) && (c == 0 || ctl.wait(B_OFREE, par ^ 1u));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t qh = sb + OFF_QH + (c & 1) * 16384;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tmem + TM_O, tmem + TM_ST + kk * 8,
                                    sw128_desc(qh + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), I_KK, kk > 0);
                    mma_commit(ctl.bar(B_WSQS));
                    // S^T += U~^T K ; O^T += U^T P^T
                    ok = ctl.wait(B_UT, par) && ctl.wait(B_KP0 + (c & 1), (uint32_t)(c >> 1) & 1u);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t pm = sb + OFF_PM + (c & 1) * 8192;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tmem + TM_SACC, tmem + TM_UK + kk * 8,
                                    sw128_desc(st + ST_KQ + kk * 2048, 16384, 1024), I_KU, 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tmem + TM_O, tmem + TM_UT + kk * 8, sw128_desc(pm + kk * 32, 16, 1024), I_KK, 1);
                    mma_commit(ctl.bar(B_KUPU));
                    mma_commit(ctl.bar(B_FREE0 + (c & 1)));   // the stage's last reader is done
                }
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp >= kSideWarp0 && warp < kChainWarp0) {
        // ================= P and Qh of each chunk (128 threads) ====================
        const int sid = tid - kSideWarp0 * 32;     // 0..127
        const int q = warp & 3;                    // TMEM lane quarter
        for (int c = 0; c < n; ++c) {
            const uint32_t par = (uint32_t)c & 1u;
            const int Cc = min(kC, T - c * kC);
            const float* gs = gates + (c & 3) * GATE_FLOATS;
            const uint32_t kq = sb + (c & 1) * SZ_STAGE + ST_KQ;
            bool ok = ctl.wait(B_GATE0 + (c & 3), (uint32_t)(c >> 2) & 1u) && ctl.wait(B_GRAM, par) &&
                      ctl.wait(B_FULL0 + (c & 1), (uint32_t)(c >> 1) & 1u);
            if (!ok) *abort_flag = 1;
            if (named_bar_any(1, kSideThreads, !ok)) break;
            tc_fence_after();
            // ---- P = scale tril((Q K^T)_ij D_ij), rows i < Cc, from TMEM lanes 64-127 ----
            if (q >= 2) {
                const int i = ((q - 2) << 5) + lane;
                const float si = i < Cc ? scale : 0.f;
                const float g2i = gs[G_G2 + i];
                const uint32_t pm = sb + OFF_PM + (c & 1) * 8192;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tmem_ld32(tmem + ((uint32_t)(q << 5) << 16) + TM_G + hh * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 ga = *reinterpret_cast<const float4*>(gs + G_G2 + hh * 32 + 8 * q4);
                        const float4 gb = *reinterpret_cast<const float4*>(gs + G_G2 + hh * 32 + 8 * q4 + 4);
                        const float gjv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                        float p[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int jj = hh * 32 + q4 * 8 + e;
                            p[e] = jj <= i ? si * v[q4 * 8 + e] * decay2(g2i, gjv[e]) : 0.f;
                        }
                        st_shared_v4(pm + sw128_off(i, hh * 4 + q4), pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]),
                                     pack_bf16x2(p[4], p[5]), pack_bf16x2(p[6], p[7]));
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_KP0 + (c & 1)));
            mbar_arrive(ctl.bar(B_GFREE));
            // ---- Qh into this chunk's buffer (its previous reader, two chunks back, is done) ----
            {
                const uint32_t qh = sb + OFF_QH + (c & 1) * 16384;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int x = sid + u * kSideThreads;     // 0..1023
                    const int blk = x >> 9, i = (x >> 3) & 63, ch = x & 7;
                    const float f = i < Cc ? scale * gs[G_EG + i] : 0.f;
                    scale_chunk(kq + blk * 16384 + 8192 + sw128_off(i, ch), qh + blk * 8192 + sw128_off(i, ch), f);
                }
            }
            fence_async_smem();
            mbar_arrive(ctl.bar(B_READY));
        }
    } else if (warp >= kChainWarp0) {
        // ================= state chain and output (256 threads) =================
        const int q = warp & 3;
        const int hc = (warp - kChainWarp0) >> 2;    // column half
        const int j = (q << 5) + lane;               // value channel = TMEM lane
        const uint32_t lane_off = (uint32_t)(q << 5) << 16;
        bool ok = ctl.wait(B_GATE0, 0);
        if (!ok) *abort_flag = 1;
        ok = !named_bar_any(2, kChainThreads, !ok);
        if (ok) {
            // S0 -> TMEM: fp32 pre-scaled by chunk 0's decay, and its bf16 copy
            const float gamma0 = gates[G_GAMMA];
#pragma unroll 1
            for (int pc = 2 * hc; pc < 2 * hc + 2; ++pc) {
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
            const uint32_t st = sb + (c & 1) * SZ_STAGE;
            // ---- U = u - W S -> bf16 pairs in TMEM, plain and decayed (U~) --------------
            ok = ctl.wait(B_WS, par) && ctl.wait(B_FULL0 + (c & 1), (uint32_t)(c >> 1) & 1u);
            if (!ok) *abort_flag = 1;
            if (named_bar_any(2, kChainThreads, !ok)) { ok = false; break; }
            tc_fence_after();
            const float* gsc = gates + (c & 3) * GATE_FLOATS;
            {
                float v[32];
                tmem_ld32(tmem + lane_off + TM_U + hc * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const uint4 w = ld_shared_v4(st + ST_UT + sw128_off(j, hc * 4 + ch));
                    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h2[e]);
                        v[8 * ch + 2 * e] += f.x;
                        v[8 * ch + 2 * e + 1] += f.y;
                    }
                }
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                tmem_st16(tmem + lane_off + TM_UT + hc * 16, pk);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 et = *reinterpret_cast<const float4*>(gsc + G_ET + hc * 32 + 4 * q4);
                    pk[2 * q4] = pack_bf16x2(v[4 * q4 + 0] * et.x, v[4 * q4 + 1] * et.y);
                    pk[2 * q4 + 1] = pack_bf16x2(v[4 * q4 + 2] * et.z, v[4 * q4 + 3] * et.w);
                }
                tmem_st16(tmem + lane_off + TM_UK + hc * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ctl.bar(B_UT));
            // ---- state: S_{c+1} = gamma_c S_c + dS (already summed in TMEM) ---------------
            ok = ctl.wait(B_KUPU, par) && (c + 1 >= n || ctl.wait(B_GATE0 + ((c + 1) & 3), (uint32_t)((c + 1) >> 2) & 1u));
            if (!ok) *abort_flag = 1;
            if (named_bar_any(2, kChainThreads, !ok)) { ok = false; break; }
            tc_fence_after();
            const bool last = c + 1 == n;
            const float gnext = last ? 1.f : gates[((c + 1) & 3) * GATE_FLOATS + G_GAMMA];
#pragma unroll 1
            for (int pc = 2 * hc; pc < 2 * hc + 2; ++pc) {
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
            {
                __nv_bfloat16* ob = o + (bh * T + (int64_t)c * kC) * kD + j;
                float v[32];
                tmem_ld32(tmem + lane_off + TM_O + hc * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = hc * 32 + e;
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

template <int GATE>
cudaError_t launch_tc_gate(const ChunkArgs& a, cudaStream_t st) {
    const uint64_t rows = (uint64_t)(a.B * a.H * a.T);
    const int64_t n = (a.T + kC - 1) / kC;
    const uint64_t ws_rows = (uint64_t)(a.B * a.H * n * kD);
    __nv_bfloat16* w_ws = static_cast<__nv_bfloat16*>(a.ws);
    __nv_bfloat16* u_ws = w_ws + ws_rows * kC;
    CUtensorMap tq, tk, tv, tw, tu;
    if (!make_tmap(&tq, a.q, kD, rows, 64) || !make_tmap(&tk, a.k, kD, rows, 64) ||
        !make_tmap(&tv, a.v, kD, rows, 64) || !make_tmap(&tw, w_ws, kC, ws_rows, 128) ||
        !make_tmap(&tu, u_ws, kC, ws_rows, 128))
        return cudaErrorInvalidValue;
    cudaError_t e = launch_chunk_wy(a, tk, tv, w_ws, u_ws, st);
    if (e != cudaSuccess) return e;
    auto kern = chunk_tc_kernel<GATE>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.B * a.H), kNT, SMEM_BYTES, st>>>(tq, tk, tw, tu, a.beta, a.g, a.S0,
                                                          static_cast<__nv_bfloat16*>(a.o), a.S_T, (int)a.T,
                                                          a.scale, a.status, a.test_flags);
    return cudaGetLastError();
}

}  // namespace

bool tc_supports(const ChunkArgs& a) {
    const int64_t n = (a.T + kC - 1) / kC;
    return a.bf16 && a.chunk == kC && a.dk == kD && a.dv == kD && a.gate != kGatePerKey &&
           a.B * a.H * a.T < (int64_t(1) << 31) && a.B * a.H * n * kD < (int64_t(1) << 31);
}

size_t tc_workspace_bytes(const ChunkArgs& a) {
    const int64_t n = (a.T + kC - 1) / kC;
    return (size_t)(a.B * a.H * n) * 2 * kWsTileBytes;
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t st) {
    if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
    return a.gate == kGateScalar ? launch_tc_gate<kGateScalar>(a, st) : launch_tc_gate<kGateNone>(a, st);
}

}  // namespace dn
