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
#include "dn_common.cuh"
#include "dn_kernels.h"

namespace dn {

namespace {

constexpr int kNT = 256;     // threads per CTA
constexpr int kDVT = 32;     // value columns per CTA
constexpr int kCmax = 32;    // largest chunk
constexpr int kVS = kDVT + 1;
constexpr int kCS = kCmax + 1;

template <int DK>
struct GenSmem {
    static constexpr int KS = DK + 1;
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
    static constexpr int kTotal = kS + DK * kVS;
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
        for (int x = tid; x < Cc * kDVT; x += kNT) {
            const int i = x / kDVT, j = x % kDVT;
            Vs[i * kVS + j] = ld_elem(v + (tok0 + c0 + i) * DV + col0 + j);
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
        // ---- pairwise sums over channels: M, N (j < i), Pk, Pl (j <= i) ---------------
        for (int p = tid; p < Cc * Cc; p += kNT) {
            const int i = p / Cc, j = p % Cc;
            float m = 0.f, nn = 0.f, pk = 0.f, pl = 0.f;
            if (j <= i) {
                const float* gi = Gm + i * KS;
                const float* gj = Gm + j * KS;
                const float* gp = i > 0 ? Gm + (i - 1) * KS : nullptr;   // Gp_i = G_{i-1}
                const float* ri = Rs + i * KS;
                const float* qi = Qs + i * KS;
                const float* lj = Ls + j * KS;
                const float* wj = Ws + j * KS;
#pragma unroll 4
                for (int c = 0; c < DK; ++c) {
                    const float e2 = expf(gi[c] - gj[c]);
                    pk += qi[c] * e2 * wj[c];
                    pl += qi[c] * e2 * lj[c];
                    if (j < i) {
                        const float e1 = expf(gp[c] - gj[c]);
                        m += ri[c] * e1 * lj[c];
                        nn += ri[c] * e1 * wj[c];
                    }
                }
            }
            Mm[i * kCS + j] = m;
            Nm[i * kCS + j] = nn;
            Pk[i * kCS + j] = scale * pk;
            Pl[i * kCS + j] = scale * pl;
        }
        __syncthreads();
        // ---- right-hand side: (kappa * e^Gp) S_0 + N V ---------------------------------
        {
            const int j = lane;
            for (int i = warp; i < Cc; i += kNT / 32) {
                const float* ri = Rs + i * KS;
                float acc = 0.f;
                if (i > 0) {
                    const float* gp = Gm + (i - 1) * KS;
#pragma unroll 8
                    for (int c = 0; c < DK; ++c) acc += ri[c] * expf(gp[c]) * Ss[c * kVS + j];
                } else {
#pragma unroll 8
                    for (int c = 0; c < DK; ++c) acc += ri[c] * Ss[c * kVS + j];
                }
                for (int m = 0; m < i; ++m) acc += Nm[i * kCS + m] * Vs[m * kVS + j];
                Us[i * kVS + j] = acc;
            }
        }
        __syncthreads();
        // ---- forward substitution (I + M) U = rhs, 4 columns per warp ----------------
        {
            const int j = warp * 4 + (lane >> 3);
            const int part = lane & 7;
            for (int i = 1; i < Cc; ++i) {
                float acc = 0.f;
                for (int m = part; m < i; m += 8) acc += Mm[i * kCS + m] * Us[m * kVS + j];
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                if (part == 0) Us[i * kVS + j] -= acc;
                __syncwarp();
            }
        }
        __syncthreads();
        // ---- output: scale (q * e^G) S_0 + Pk V - Pl U --------------------------------
        {
            const int j = lane;
            for (int i = warp; i < Cc; i += kNT / 32) {
                const float* qi = Qs + i * KS;
                const float* gi = Gm + i * KS;
                float acc = 0.f;
#pragma unroll 8
                for (int c = 0; c < DK; ++c) acc += qi[c] * expf(gi[c]) * Ss[c * kVS + j];
                acc *= scale;
                for (int m = 0; m <= i; ++m) acc += Pk[i * kCS + m] * Vs[m * kVS + j] - Pl[i * kCS + m] * Us[m * kVS + j];
                st_elem(o + (tok0 + c0 + i) * DV + col0 + j, acc);
            }
        }
        __syncthreads();
        // ---- state: e^(G_C) * S_0 + sum_s (e^(G_C - G_s) * k_s) v_s^T - (e^(G_C - G_s) * l_s) U_s
        {
            const int j = lane;
            const float* gl = Gm + (Cc - 1) * KS;
            for (int c = warp; c < DK; c += kNT / 32) {
                float acc = 0.f;
                for (int s = 0; s < Cc; ++s) {
                    const float e = expf(gl[c] - Gm[s * KS + c]);
                    acc += e * (Ws[s * KS + c] * Vs[s * kVS + j] - Ls[s * KS + c] * Us[s * kVS + j]);
                }
                Ss[c * kVS + j] = expf(gl[c]) * Ss[c * kVS + j] + acc;
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
