// chunk_general.cu -- the generalised delta rule of RWKV-7 ("DeltaNet: Memory
// That Edits", D2L 12.5, "The generalized delta rule") in chunks, on the CUDA
// cores in fp32:
//
//   S_t = (diag(w_t) - (a_t * kappa_t) kappa_t^T) S_{t-1} + k_t v_t^T,
//   o_t = S_t^T (scale q_t),
//
// with a per-channel decay w_t = e^(wlog_t), a removal key kappa_t, a
// per-channel removal rate a_t and a write key k_t that need not equal kappa_t.
// The page states only the recurrence.  Its chunkwise form, derived from it and
// checked against it in fp64 (the oracle's chunked restatement): inside a chunk
// of Cc tokens, with l_s = a_s * kappa_s, G_t = sum_{s<=t} wlog_s per channel
// (inclusive, chunk-local), Gp_s = G_{s-1} (G_0 = 0) and U_s = kappa_s^T S_{s-1}
// the content the step removes,
//
//   M_sj = sum_c kappa_sc e^(Gp_sc - G_jc) l_jc          (j < s)
//   N_sj = sum_c kappa_sc e^(Gp_sc - G_jc) k_jc          (j < s)
//   (I + M) U = (kappa * e^Gp) S_0 + N V                   (forward substitution)
//   o_t  = scale [ (q_t * e^G_t)^T S_0 + sum_{s<=t} (Pk_ts v_s - Pl_ts U_s) ],
//          Pk_ts = sum_c q_tc e^(G_tc - G_sc) k_sc,  Pl_ts = same with l_s
//   S   <- e^(G_C) * S_0 + sum_s (e^(G_C - G_s) * k_s) v_s^T - (e^(G_C - G_s) * l_s) U_s
//
// Every exponent is a sum of log-decays over a span of the chunk, so it is <= 0
// when wlog <= 0: nothing overflows.  The pairwise decays stay inside the sums
// over channels (exact per pair, as the per-key gate needs).
//
// One CTA owns one (b, h) and a 32-wide slice of the value dimension (columns
// of S evolve independently); the state slice stays in shared memory for the
// whole sequence.  Chunks of 1..32 tokens (the five key-side tiles of a chunk
// are kept in shared memory).  A partial last chunk just has fewer rows.
//
// Once the pairwise sums are formed, the key-side tiles are replaced in place by
// their decayed forms (q e^G, kappa e^Gp, k e^(G_C - G), l e^(G_C - G)), so that
// the right-hand side, the output rows and the state update are plain sums of
// products; those read 4 rows a warp as float4 broadcasts (rows padded to a
// multiple of 4 floats), one value column per lane.  The system is solved by
// 16-row blocks: the diagonal inverses at once, then block after block.
#include "dn_common.cuh"
#include "dn_kernels.h"

namespace dn {

namespace {

constexpr int kNT = 256;     // threads per CTA
constexpr int kDVT = 32;     // value columns per CTA
constexpr int kCmax = 32;    // largest chunk
constexpr int kVS = kDVT + 1;
constexpr int kCS = kCmax + 4;   // rows of M, N, Pk, Pl: 16-byte aligned

template <int DK>
struct GenSmem {
    static constexpr int KS = DK + 4;
    static constexpr int kQ = 0;                           // q        [Cmax][KS]
    static constexpr int kR = kQ + kCmax * KS;             // kappa    [Cmax][KS]
    static constexpr int kL = kR + kCmax * KS;             // a*kappa  [Cmax][KS]
    static constexpr int kW = kL + kCmax * KS;             // k        [Cmax][KS]
    static constexpr int kG = kW + kCmax * KS;             // G        [Cmax][KS]
    static constexpr int kV = kG + kCmax * KS;             // V        [Cmax][VS]
    static constexpr int kU = kV + kCmax * kVS;            // RHS -> U [Cmax][VS]
    static constexpr int kM = kU + kCmax * kVS;            // M        [Cmax][CS]
    static constexpr int kN = kM + kCmax * kCS;            // N        [Cmax][CS]
    static constexpr int kPk = kN + kCmax * kCS;           // Pk       [Cmax][CS]
    static constexpr int kPl = kPk + kCmax * kCS;          // Pl       [Cmax][CS]
    static constexpr int kS = kPl + kCmax * kCS;           // S slice  [DK][VS]
    static constexpr int kD = kS + DK * kVS;               // (I + M_bb)^-1 [2 blocks][16][17]
    static constexpr int kTotal = kD + 2 * 16 * 17;
    static constexpr size_t bytes = sizeof(float) * kTotal;
};

template <int DK, typename Tin>
__global__ void __launch_bounds__(kNT)
chunk_general_kernel(const Tin* __restrict__ q, const float* __restrict__ wlog, const Tin* __restrict__ kappa,
                     const float* __restrict__ a, const Tin* __restrict__ kw, const Tin* __restrict__ v,
                     const float* S0, Tin* __restrict__ o, float* S_T, int T, int DV, int chunk, float scale) {
    using L = GenSmem<DK>;
    constexpr int KS = L::KS;
    extern __shared__ float sm[];
    float* Qs = sm + L::kQ;
    float* Rs = sm + L::kR;
    float* Ls = sm + L::kL;
    float* Ws = sm + L::kW;
    float* Gm = sm + L::kG;
    float* Vs = sm + L::kV;
    float* Us = sm + L::kU;
    float* Mm = sm + L::kM;
    float* Nm = sm + L::kN;
    float* Pk = sm + L::kPk;
    float* Pl = sm + L::kPl;
    float* Ss = sm + L::kS;
    float* Dm = sm + L::kD;

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int ntiles = DV / kDVT;
    const int64_t bh = blockIdx.x / ntiles;
    const int col0 = (blockIdx.x % ntiles) * kDVT;
    const int64_t tok0 = bh * (int64_t)T;

    for (int x = tid; x < DK * kDVT; x += kNT) {
        const int i = x / kDVT, j = x % kDVT;
        Ss[i * kVS + j] = S0 ? S0[(bh * DK + i) * DV + col0 + j] : 0.f;
    }

    for (int c0 = 0; c0 < T; c0 += chunk) {
        const int Cc = min(chunk, T - c0);
        __syncthreads();   // the previous chunk is consumed
        // ---- the chunk's tiles -----------------------------------------------------
        for (int x = tid; x < Cc * DK; x += kNT) {
            const int i = x / DK, c = x % DK;
            const int64_t off = (tok0 + c0 + i) * DK + c;
            const float r = ld_elem(kappa + off);
            Qs[i * KS + c] = ld_elem(q + off);
            Rs[i * KS + c] = r;
            Ls[i * KS + c] = a[off] * r;
            Ws[i * KS + c] = ld_elem(kw + off);
            Gm[i * KS + c] = wlog[off];
        }
        for (int x = tid; x < kCmax * kDVT; x += kNT) {
            const int i = x / kDVT, j = x % kDVT;
            Vs[i * kVS + j] = i < Cc ? ld_elem(v + (tok0 + c0 + i) * DV + col0 + j) : 0.f;
        }
        __syncthreads();
        // ---- G: inclusive prefix sum of the log-decays over the chunk, per channel -----
        for (int c = tid; c < DK; c += kNT) {
            float acc = 0.f;
            for (int i = 0; i < Cc; ++i) {
                acc += Gm[i * KS + c];
                Gm[i * KS + c] = acc;
            }
        }
        __syncthreads();
        // ---- pairwise sums over channels: M, N (j < i), Pk, Pl (j <= i), read as float4 along
        //      the channels (row j per lane: distinct bank groups; row i broadcast) -----------
        for (int p = tid; p < kCmax * kCmax; p += kNT) {
            const int i = p / kCmax, j = p % kCmax;
            float m = 0.f, nn = 0.f, pk = 0.f, pl = 0.f;
            if (j <= i && i < Cc) {
                const float* gi = Gm + i * KS;
                const float* gj = Gm + j * KS;
                const float* qi = Qs + i * KS;
                const float* lj = Ls + j * KS;
                const float* wj = Ws + j * KS;
                if (j < i) {
                    const float* gp = Gm + (i - 1) * KS;   // Gp_i = G_{i-1}
                    const float* ri = Rs + i * KS;
#pragma unroll 2
                    for (int c = 0; c < DK; c += 4) {
                        const float4 gi4 = *reinterpret_cast<const float4*>(gi + c);
                        const float4 gj4 = *reinterpret_cast<const float4*>(gj + c);
                        const float4 gp4 = *reinterpret_cast<const float4*>(gp + c);
                        const float4 qi4 = *reinterpret_cast<const float4*>(qi + c);
                        const float4 ri4 = *reinterpret_cast<const float4*>(ri + c);
                        const float4 lj4 = *reinterpret_cast<const float4*>(lj + c);
                        const float4 wj4 = *reinterpret_cast<const float4*>(wj + c);
                        const float g_i[4] = {gi4.x, gi4.y, gi4.z, gi4.w}, g_j[4] = {gj4.x, gj4.y, gj4.z, gj4.w};
                        const float g_p[4] = {gp4.x, gp4.y, gp4.z, gp4.w}, q_i[4] = {qi4.x, qi4.y, qi4.z, qi4.w};
                        const float r_i[4] = {ri4.x, ri4.y, ri4.z, ri4.w}, l_j[4] = {lj4.x, lj4.y, lj4.z, lj4.w};
                        const float w_j[4] = {wj4.x, wj4.y, wj4.z, wj4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float e2 = __expf(g_i[e] - g_j[e]) * q_i[e];
                            const float e1 = __expf(g_p[e] - g_j[e]) * r_i[e];
                            pk = fmaf(e2, w_j[e], pk);
                            pl = fmaf(e2, l_j[e], pl);
                            m = fmaf(e1, l_j[e], m);
                            nn = fmaf(e1, w_j[e], nn);
                        }
                    }
                } else {
                    // the diagonal: e^(G_i - G_i) = 1
#pragma unroll 2
                    for (int c = 0; c < DK; c += 4) {
                        const float4 qi4 = *reinterpret_cast<const float4*>(qi + c);
                        const float4 lj4 = *reinterpret_cast<const float4*>(lj + c);
                        const float4 wj4 = *reinterpret_cast<const float4*>(wj + c);
                        pk = fmaf(qi4.x, wj4.x, fmaf(qi4.y, wj4.y, fmaf(qi4.z, wj4.z, fmaf(qi4.w, wj4.w, pk))));
                        pl = fmaf(qi4.x, lj4.x, fmaf(qi4.y, lj4.y, fmaf(qi4.z, lj4.z, fmaf(qi4.w, lj4.w, pl))));
                    }
                }
            }
            Mm[i * kCS + j] = m;
            Nm[i * kCS + j] = nn;
            Pk[i * kCS + j] = scale * pk;
            Pl[i * kCS + j] = scale * pl;
        }
        __syncthreads();
        // ---- the decayed tiles, in place (the raw ones are read for the last time above):
        //      q e^G (output), kappa e^Gp (right-hand side), k and l times e^(G_C - G) (state)
        for (int x = tid; x < Cc * DK; x += kNT) {
            const int i = x / DK, c = x % DK;
            const float gi = Gm[i * KS + c], gc = Gm[(Cc - 1) * KS + c];
            const float gp = i > 0 ? Gm[(i - 1) * KS + c] : 0.f;
            const float ed = __expf(gc - gi);
            Qs[i * KS + c] *= __expf(gi);
            Rs[i * KS + c] *= __expf(gp);
            Ws[i * KS + c] *= ed;
            Ls[i * KS + c] *= ed;
        }
        __syncthreads();
        // e^(G_C) per channel, for the state's decay (row 0 of G is free now)
        for (int c = tid; c < DK; c += kNT) Gm[c] = __expf(Gm[(Cc - 1) * KS + c]);
        // ---- right-hand side: (kappa e^Gp) S_0 + N V; warp w: rows 4w .. 4w + 3, lane: column
        {
            const int j = lane, i0 = warp * 4;
            if (i0 < Cc) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
                for (int c = 0; c < DK; c += 4) {
                    const float s0 = Ss[c * kVS + j], s1 = Ss[(c + 1) * kVS + j];
                    const float s2 = Ss[(c + 2) * kVS + j], s3 = Ss[(c + 3) * kVS + j];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float4 rv = *reinterpret_cast<const float4*>(Rs + (i0 + r) * KS + c);
                        acc[r] = fmaf(rv.x, s0, fmaf(rv.y, s1, fmaf(rv.z, s2, fmaf(rv.w, s3, acc[r]))));
                    }
                }
                // N V over positions < i0 + 4 (N is zero on and above the diagonal and past Cc)
                for (int m = 0; m < i0 + 4; m += 4) {
                    const float v0 = Vs[m * kVS + j], v1 = Vs[(m + 1) * kVS + j];
                    const float v2 = Vs[(m + 2) * kVS + j], v3 = Vs[(m + 3) * kVS + j];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float4 nv = *reinterpret_cast<const float4*>(Nm + (i0 + r) * kCS + m);
                        acc[r] = fmaf(nv.x, v0, fmaf(nv.y, v1, fmaf(nv.z, v2, fmaf(nv.w, v3, acc[r]))));
                    }
                }
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    if (i0 + r < Cc) Us[(i0 + r) * kVS + j] = acc[r];
            }
        }
        __syncthreads();
        // ---- (I + M) U = rhs by 16-row blocks: both diagonal inverses at once (one warp a
        //      block, lane = column), then U_b = D_b (rhs_b - M_b,<b U_<b) -----------------
        {
            const int nb = (Cc + 15) >> 4;
            if (warp < nb && lane < 16) {
                const int k0 = warp * 16, jj = lane;
                float xr[16];
#pragma unroll
                for (int ii = 0; ii < 16; ++ii) {
                    float p0 = ii == jj ? 1.f : 0.f, p1 = 0.f;
                    if (k0 + ii < Cc) {
#pragma unroll
                        for (int m = 0; m < ii; m += 2) {
                            p0 -= Mm[(k0 + ii) * kCS + k0 + m] * xr[m];
                            if (m + 1 < ii) p1 -= Mm[(k0 + ii) * kCS + k0 + m + 1] * xr[m + 1];
                        }
                    }
                    xr[ii] = p0 + p1;
                }
#pragma unroll
                for (int ii = 0; ii < 16; ++ii) Dm[(warp * 16 + ii) * 17 + jj] = xr[ii];
            }
            __syncthreads();
            for (int bb = 0; bb < nb; ++bb) {
                const int r0 = 16 * bb;
                if (bb > 0) {
                    for (int x = tid; x < 16 * kDVT; x += kNT) {
                        const int i = r0 + x / kDVT, j = x % kDVT;
                        if (i < Cc) {
                            float a4[4] = {0.f, 0.f, 0.f, 0.f};
                            for (int m = 0; m < r0; m += 4) {
#pragma unroll
                                for (int u = 0; u < 4; ++u)
                                    a4[u] = fmaf(Mm[i * kCS + m + u], Us[(m + u) * kVS + j], a4[u]);
                            }
                            Us[i * kVS + j] -= (a4[0] + a4[1]) + (a4[2] + a4[3]);
                        }
                    }
                    __syncthreads();
                }
                float val[16 * kDVT / kNT];
#pragma unroll
                for (int u = 0; u < 16 * kDVT / kNT; ++u) {
                    const int x = tid + u * kNT;
                    const int ii = x / kDVT, j = x % kDVT;
                    const float* drow = Dm + (bb * 16 + ii) * 17;
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int t = 0; t < 16; t += 2) {
                        if (t <= ii && r0 + t < Cc) a0 = fmaf(drow[t], Us[(r0 + t) * kVS + j], a0);
                        if (t + 1 <= ii && r0 + t + 1 < Cc) a1 = fmaf(drow[t + 1], Us[(r0 + t + 1) * kVS + j], a1);
                    }
                    val[u] = a0 + a1;
                }
                __syncthreads();
#pragma unroll
                for (int u = 0; u < 16 * kDVT / kNT; ++u) {
                    const int x = tid + u * kNT;
                    const int ii = x / kDVT, j = x % kDVT;
                    if (r0 + ii < Cc) Us[(r0 + ii) * kVS + j] = val[u];
                }
                __syncthreads();
            }
            // rows of U past a short chunk are zero for the products below
            for (int x = Cc * kDVT + tid; x < kCmax * kDVT; x += kNT) Us[(x / kDVT) * kVS + x % kDVT] = 0.f;
            __syncthreads();
        }
        // ---- output: scale (q e^G) S_0 + Pk V - Pl U (Pk, Pl carry the scale); warp w: rows
        //      4w .. 4w + 3, lane: column --------------------------------------------------
        {
            const int j = lane, i0 = warp * 4;
            if (i0 < Cc) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f}, pv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
                for (int c = 0; c < DK; c += 4) {
                    const float s0 = Ss[c * kVS + j], s1 = Ss[(c + 1) * kVS + j];
                    const float s2 = Ss[(c + 2) * kVS + j], s3 = Ss[(c + 3) * kVS + j];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float4 qv = *reinterpret_cast<const float4*>(Qs + (i0 + r) * KS + c);
                        acc[r] = fmaf(qv.x, s0, fmaf(qv.y, s1, fmaf(qv.z, s2, fmaf(qv.w, s3, acc[r]))));
                    }
                }
                for (int m = 0; m < i0 + 4; m += 4) {
                    const float v0 = Vs[m * kVS + j], v1 = Vs[(m + 1) * kVS + j];
                    const float v2 = Vs[(m + 2) * kVS + j], v3 = Vs[(m + 3) * kVS + j];
                    const float u0 = Us[m * kVS + j], u1 = Us[(m + 1) * kVS + j];
                    const float u2 = Us[(m + 2) * kVS + j], u3 = Us[(m + 3) * kVS + j];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float4 kv = *reinterpret_cast<const float4*>(Pk + (i0 + r) * kCS + m);
                        const float4 lv = *reinterpret_cast<const float4*>(Pl + (i0 + r) * kCS + m);
                        pv[r] = fmaf(kv.x, v0, fmaf(kv.y, v1, fmaf(kv.z, v2, fmaf(kv.w, v3, pv[r]))));
                        pv[r] = fmaf(-lv.x, u0, fmaf(-lv.y, u1, fmaf(-lv.z, u2, fmaf(-lv.w, u3, pv[r]))));
                    }
                }
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    if (i0 + r < Cc) st_elem(o + (tok0 + c0 + i0 + r) * DV + col0 + j, scale * acc[r] + pv[r]);
            }
        }
        __syncthreads();
        // ---- state: e^(G_C) * S_0 + sum_s (k e^(G_C - G))_s v_s^T - (l e^(G_C - G))_s U_s;
        //      warp w: key channels 16w .. 16w + 15 (+ 128), lane: column ----------------
        {
            const int j = lane;
            for (int cb = warp * 16; cb < DK; cb += 16 * (kNT / 32)) {
                float acc[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = 0.f;
                for (int s2 = 0; s2 < Cc; ++s2) {
                    const float vv = Vs[s2 * kVS + j], uu = Us[s2 * kVS + j];
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const float4 kw4 = *reinterpret_cast<const float4*>(Ws + s2 * KS + cb + 4 * e4);
                        const float4 l4 = *reinterpret_cast<const float4*>(Ls + s2 * KS + cb + 4 * e4);
                        acc[4 * e4 + 0] = fmaf(kw4.x, vv, fmaf(-l4.x, uu, acc[4 * e4 + 0]));
                        acc[4 * e4 + 1] = fmaf(kw4.y, vv, fmaf(-l4.y, uu, acc[4 * e4 + 1]));
                        acc[4 * e4 + 2] = fmaf(kw4.z, vv, fmaf(-l4.z, uu, acc[4 * e4 + 2]));
                        acc[4 * e4 + 3] = fmaf(kw4.w, vv, fmaf(-l4.w, uu, acc[4 * e4 + 3]));
                    }
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int c = cb + e;
                    Ss[c * kVS + j] = Gm[c] * Ss[c * kVS + j] + acc[e];
                }
            }
        }
    }
    __syncthreads();
    if (S_T) {
        for (int x = tid; x < DK * kDVT; x += kNT) {
            const int i = x / kDVT, j = x % kDVT;
            S_T[(bh * DK + i) * DV + col0 + j] = Ss[i * kVS + j];
        }
    }
}

template <int DK, typename Tin>
cudaError_t launch_general_t(const GeneralArgs& a, cudaStream_t st) {
    using L = GenSmem<DK>;
    auto kern = chunk_general_kernel<DK, Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return e;
    const int64_t blocks = a.B * a.H * (a.dv / kDVT);
    kern<<<(unsigned)blocks, kNT, L::bytes, st>>>(
        static_cast<const Tin*>(a.q), a.wlog, static_cast<const Tin*>(a.kappa), a.a, static_cast<const Tin*>(a.k),
        static_cast<const Tin*>(a.v), a.S0, static_cast<Tin*>(a.o), a.S_T, (int)a.T, a.dv, a.chunk, a.scale);
    return counted(cudaGetLastError());
}

}  // namespace

int general_max_chunk() { return kCmax; }

cudaError_t launch_chunk_general(const GeneralArgs& a, cudaStream_t st) {
    if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
    if (a.dk == 64) return a.bf16 ? launch_general_t<64, __nv_bfloat16>(a, st) : launch_general_t<64, float>(a, st);
    return a.bf16 ? launch_general_t<128, __nv_bfloat16>(a, st) : launch_general_t<128, float>(a, st);
}

}  // namespace dn
