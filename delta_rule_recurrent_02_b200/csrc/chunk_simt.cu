// chunk_simt.cu -- chunked delta-rule prefill on the CUDA cores, fp32 math.
//
// The chunkwise form of "Linear attention and Gated DeltaNet" (ch. 28, "The
// chunked form: recurrence as matrix multiplication"), with the per-key
// decay of KDA folded in.  Inside a chunk of Cc <= 64 tokens, with
// Gamma_i = sum_{m<=i} g_m (per key channel; one value for a scalar gate,
// zero without a gate):
//
//   A_ij  = beta_i sum_c k_ic k_jc e^(Gamma_ic - Gamma_jc)        j <  i
//   P_ij  =        sum_c q_ic k_jc e^(Gamma_ic - Gamma_jc)        j <= i
//   (I + A) U = diag(beta) (V - (K * e^Gamma) S)                    (UT transform)
//   O     = (Q * e^Gamma) S + P U
//   S    <- Diag(e^Gamma_last) S + (K * e^(Gamma_last - Gamma))^T U
//
// which is the page's system with its right-hand side factored as
// beta * (V - e^G (K S_0)).  A partial last chunk just uses Cc < chunk rows,
// which equals zero padding with g = 0 and beta = 0.
//
// This is the fp32 path (fp32 or bf16 storage, fp32 arithmetic, any chunk
// size 1..64).  One CTA owns one (b, h) and a 32-wide slice of the value
// dimension: columns of S evolve independently given K, beta and g, so the
// slices need no communication.  The state slice stays in shared memory for
// the whole sequence; the only HBM traffic is the token tiles, o, and S0/S_T.
#include "dn_common.cuh"
#include "dn_kernels.h"

namespace dn {

namespace {

constexpr int kNT = 256;     // threads per CTA
constexpr int kDVT = 32;     // value columns per CTA
constexpr int kCmax = 64;    // largest chunk
constexpr int kVS = kDVT + 1;
constexpr int kCS = kCmax + 4;   // A, P rows: 16-byte aligned (read as float4 along a row)

// Row strides are multiples of 4 floats, and so every region's offset: rows of K, Q
// and P are read as float4, broadcast to a warp, along the contraction.
template <int DK, int GATE>
struct SimtSmem {
    static constexpr int KS = DK + 4;
    static constexpr int kK = 0;                              // K      [Cmax][KS]
    static constexpr int kQ = kK + kCmax * KS;                // Q      [Cmax][KS]
    static constexpr int kG = kQ + kCmax * KS;                // Gamma  [Cmax][KS] or [Cmax]
    static constexpr int kGn = (GATE == kGatePerKey) ? kCmax * KS : kCmax;
    static constexpr int kKx = kG + kGn;                      // scaled K (per-key only)
    static constexpr int kKxn = (GATE == kGatePerKey) ? kCmax * KS : 0;
    static constexpr int kV = kKx + kKxn;                     // V -> R -> U [Cmax][VS]
    static constexpr int kA = kV + kCmax * kVS;               // A      [Cmax][CS]
    static constexpr int kP = kA + kCmax * kCS;               // P      [Cmax][CS]
    static constexpr int kS = kP + kCmax * kCS;               // S      [DK][VS]
    static constexpr int kB = kS + DK * kVS;                  // beta   [Cmax]
    static constexpr int kE = kB + kCmax;                     // e^G_i  [Cmax]
    static constexpr int kT = kE + kCmax;                     // e^(G_last - G_i) [Cmax]
    static constexpr int kD = kT + kCmax;                     // (I + A_bb)^-1 [4 blocks][16][17]
    static constexpr int kTotal = kD + 4 * 16 * 17;
    static constexpr size_t bytes = sizeof(float) * kTotal;
};

}  // namespace

template <int DK, int GATE, typename Tin, bool PRO = false>
__global__ void __launch_bounds__(kNT)
chunk_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                  const Tin* __restrict__ v, const float* __restrict__ beta,
                  const float* __restrict__ g, const float* S0,
                  Tin* __restrict__ o, float* S_T, int T, int DV, int chunk,
                  float scale, float* snaps, int snap_every, int n_snap,
                  const float* A_log = nullptr, const float* dt_bias = nullptr, int H = 1, float bmul = 1.f) {
    using L = SimtSmem<DK, GATE>;
    constexpr int KS = L::KS;
    extern __shared__ float sm[];
    float* Ks = sm + L::kK;
    float* Qs = sm + L::kQ;
    float* Gm = sm + L::kG;
    float* Kx = sm + L::kKx;
    float* Vs = sm + L::kV;
    float* Am = sm + L::kA;
    float* Pm = sm + L::kP;
    float* Ss = sm + L::kS;
    float* bs = sm + L::kB;
    float* eG = sm + L::kE;
    float* eT = sm + L::kT;
    float* Dm = sm + L::kD;

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int ntiles = DV / kDVT;
    const int64_t bh = blockIdx.x / ntiles;
    const int col0 = (blockIdx.x % ntiles) * kDVT;
    const int64_t tok0 = bh * (int64_t)T;

    // state slice S[:, col0 : col0 + 32]
    for (int x = tid; x < DK * kDVT; x += kNT) {
        const int i = x / kDVT, j = x % kDVT;
        Ss[i * kVS + j] = S0 ? S0[(bh * DK + i) * DV + col0 + j] : 0.f;
    }

    // Token tiles of the next chunk are prefetched into registers while the
    // current chunk is computed, so HBM latency is off the critical path.
    constexpr int NVK = kCmax * DK / 4 / kNT;      // float4-groups of K (or Q, or g) per thread
    constexpr int NVV = kCmax * kDVT / 4 / kNT;    // float4-groups of the V slice per thread
    float4 pk[NVK], pq[NVK], pg[GATE == kGatePerKey ? NVK : 1], pv[NVV];
    float pb = 0.f, ps = 0.f;
    auto prefetch = [&](int c0) {
        const int Cc = min(chunk, T - c0);
        const int64_t t0 = tok0 + c0;
#pragma unroll
        for (int u = 0; u < NVK; ++u) {
            const int x = tid + u * kNT;             // group index: row x / (DK/4), col 4 * (x % (DK/4))
            if (x < Cc * DK / 4) {
                const int64_t off = (t0 + x / (DK / 4)) * DK + 4 * (x % (DK / 4));
                pk[u] = ld4(k + off);
                pq[u] = ld4(q + off);
                if (GATE == kGatePerKey) pg[u] = *reinterpret_cast<const float4*>(g + off);
            }
        }
#pragma unroll
        for (int u = 0; u < NVV; ++u) {
            const int x = tid + u * kNT;
            if (x < Cc * kDVT / 4)
                pv[u] = ld4(v + (t0 + x / (kDVT / 4)) * DV + col0 + 4 * (x % (kDVT / 4)));
        }
        if (tid < Cc) {
            pb = beta[t0 + tid];
            if (GATE == kGateScalar) ps = g[t0 + tid];
        }
    };
    if (T > 0) prefetch(0);

    for (int c0 = 0; c0 < T; c0 += chunk) {
        const int Cc = min(chunk, T - c0);
        __syncthreads();   // previous chunk fully consumed
        // ---- the chunk's tiles: registers -> shared memory -----------------
#pragma unroll
        for (int u = 0; u < NVK; ++u) {
            const int x = tid + u * kNT;
            if (x < Cc * DK / 4) {
                const int i = x / (DK / 4), c = 4 * (x % (DK / 4));
                float* kd = Ks + i * KS + c;
                float* qd = Qs + i * KS + c;
                kd[0] = pk[u].x; kd[1] = pk[u].y; kd[2] = pk[u].z; kd[3] = pk[u].w;
                qd[0] = scale * pq[u].x; qd[1] = scale * pq[u].y; qd[2] = scale * pq[u].z; qd[3] = scale * pq[u].w;
                if (GATE == kGatePerKey) {
                    float* gd = Gm + i * KS + c;
                    gd[0] = pg[u].x; gd[1] = pg[u].y; gd[2] = pg[u].z; gd[3] = pg[u].w;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < NVV; ++u) {
            const int x = tid + u * kNT;
            if (x < Cc * kDVT / 4) {
                float* vd = Vs + (x / (kDVT / 4)) * kVS + 4 * (x % (kDVT / 4));
                vd[0] = pv[u].x; vd[1] = pv[u].y; vd[2] = pv[u].z; vd[3] = pv[u].w;
            }
        }
        // rows of V past a short chunk's end are zero: the blocked products read whole rows
        for (int x = Cc * kDVT + tid; x < kCmax * kDVT; x += kNT) Vs[(x / kDVT) * kVS + x % kDVT] = 0.f;
        if (tid < Cc) {
            float bb = pb, aa = ps;
            if (PRO) gdn_raw_gates(bb, aa, expf(A_log[bh % H]), dt_bias[bh % H], bmul);
            bs[tid] = bb;
            if (GATE == kGateScalar) Gm[tid] = aa;
        }
        __syncthreads();
        if (PRO) {
            // unit k and q rows, x / max(||x||, 1e-12), one warp per row (Qs holds scale q)
            for (int i = warp; i < Cc; i += kNT / 32) {
                float sk = 0.f, sq = 0.f;
                for (int c = lane; c < DK; c += 32) {
                    const float kv = Ks[i * KS + c], qv = Qs[i * KS + c];
                    sk += kv * kv;
                    sq += qv * qv;
                }
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, o2);
                    sq += __shfl_xor_sync(0xffffffffu, sq, o2);
                }
                const float rk = 1.f / fmaxf(sqrtf(sk), 1e-12f);
                const float as = fabsf(scale);
                const float rq = as > 0.f ? 1.f / fmaxf(sqrtf(sq) / as, 1e-12f) : 0.f;
                for (int c = lane; c < DK; c += 32) {
                    Ks[i * KS + c] *= rk;
                    Qs[i * KS + c] *= rq;
                }
            }
            __syncthreads();
        }
        if (c0 + chunk < T) prefetch(c0 + chunk);
        // ---- cumulative log-decay (inclusive) ---------------------------
        if (GATE == kGateScalar) {
            if (warp == 0) {
                float a0 = lane < Cc ? Gm[lane] : 0.f;
                float a1 = lane + 32 < Cc ? Gm[lane + 32] : 0.f;
#pragma unroll
                for (int o2 = 1; o2 < 32; o2 <<= 1) {
                    const float y0 = __shfl_up_sync(0xffffffffu, a0, o2);
                    const float y1 = __shfl_up_sync(0xffffffffu, a1, o2);
                    if (lane >= o2) { a0 += y0; a1 += y1; }
                }
                a1 += __shfl_sync(0xffffffffu, a0, 31);
                if (lane < Cc) Gm[lane] = a0;
                if (lane + 32 < Cc) Gm[lane + 32] = a1;
                __syncwarp();
                const float Glast = Gm[Cc - 1];
                for (int i = lane; i < Cc; i += 32) {
                    eG[i] = expf(Gm[i]);
                    eT[i] = expf(Glast - Gm[i]);
                }
            }
        } else if (GATE == kGatePerKey) {
            for (int c = tid; c < DK; c += kNT) {
                float acc = 0.f;
                for (int i = 0; i < Cc; ++i) {
                    acc += Gm[i * KS + c];
                    Gm[i * KS + c] = acc;
                }
            }
        } else {
            for (int i = tid; i < Cc; i += kNT) { eG[i] = 1.f; eT[i] = 1.f; }
        }
        __syncthreads();
        // ---- pairwise decayed products: A (strict lower) and P (lower) ---
        if (GATE != kGatePerKey) {
            // warp w: rows 8w .. 8w + 7 (K and Q rows read as broadcast float4 along c);
            // lane: columns lane and lane + 32.  Whole 64 x 64 tiles are written (zero
            // outside the chunk), so the later products need no bounds
            const int i0 = warp * 8;
            float ka[8][2], qa[8][2];
#pragma unroll
            for (int r = 0; r < 8; ++r) ka[r][0] = ka[r][1] = qa[r][0] = qa[r][1] = 0.f;
#pragma unroll 2
            for (int c = 0; c < DK; c += 4) {
                const float4 kj0 = *reinterpret_cast<const float4*>(Ks + lane * KS + c);
                const float4 kj1 = *reinterpret_cast<const float4*>(Ks + (lane + 32) * KS + c);
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float4 ki = *reinterpret_cast<const float4*>(Ks + (i0 + r) * KS + c);
                    const float4 qi = *reinterpret_cast<const float4*>(Qs + (i0 + r) * KS + c);
                    ka[r][0] = fmaf(ki.x, kj0.x, fmaf(ki.y, kj0.y, fmaf(ki.z, kj0.z, fmaf(ki.w, kj0.w, ka[r][0]))));
                    ka[r][1] = fmaf(ki.x, kj1.x, fmaf(ki.y, kj1.y, fmaf(ki.z, kj1.z, fmaf(ki.w, kj1.w, ka[r][1]))));
                    qa[r][0] = fmaf(qi.x, kj0.x, fmaf(qi.y, kj0.y, fmaf(qi.z, kj0.z, fmaf(qi.w, kj0.w, qa[r][0]))));
                    qa[r][1] = fmaf(qi.x, kj1.x, fmaf(qi.y, kj1.y, fmaf(qi.z, kj1.z, fmaf(qi.w, kj1.w, qa[r][1]))));
                }
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i = i0 + r;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = lane + 32 * h;
                    const bool in = i < Cc && j <= i;
                    const float d = (GATE == kGateScalar && in) ? expf(Gm[i] - Gm[j]) : 1.f;
                    Am[i * kCS + j] = (in && j < i) ? bs[i] * ka[r][h] * d : 0.f;
                    Pm[i * kCS + j] = in ? qa[r][h] * d : 0.f;
                }
            }
        } else {
            for (int p = tid; p < kCmax * kCmax; p += kNT) {
                const int i = p / kCmax, j = p % kCmax;
                float kd = 0.f, qd = 0.f;
                if (j <= i && i < Cc) {
                    // float4 along the channels: row j per lane lands in distinct bank groups
                    const float* ki = Ks + i * KS;
                    const float* qi = Qs + i * KS;
                    const float* kj = Ks + j * KS;
                    const float* gi = Gm + i * KS;
                    const float* gj = Gm + j * KS;
#pragma unroll 2
                    for (int c = 0; c < DK; c += 4) {
                        const float4 ki4 = *reinterpret_cast<const float4*>(ki + c);
                        const float4 qi4 = *reinterpret_cast<const float4*>(qi + c);
                        const float4 kj4 = *reinterpret_cast<const float4*>(kj + c);
                        const float4 gi4 = *reinterpret_cast<const float4*>(gi + c);
                        const float4 gj4 = *reinterpret_cast<const float4*>(gj + c);
                        const float w0 = kj4.x * __expf(gi4.x - gj4.x), w1 = kj4.y * __expf(gi4.y - gj4.y);
                        const float w2 = kj4.z * __expf(gi4.z - gj4.z), w3 = kj4.w * __expf(gi4.w - gj4.w);
                        kd = fmaf(ki4.x, w0, fmaf(ki4.y, w1, fmaf(ki4.z, w2, fmaf(ki4.w, w3, kd))));
                        qd = fmaf(qi4.x, w0, fmaf(qi4.y, w1, fmaf(qi4.z, w2, fmaf(qi4.w, w3, qd))));
                    }
                }
                Am[i * kCS + j] = (j < i && i < Cc) ? bs[i] * kd : 0.f;
                Pm[i * kCS + j] = (j <= i && i < Cc) ? qd : 0.f;
            }
        }
        if (GATE == kGatePerKey) {
            __syncthreads();   // P used the raw q; now Q <- Q * e^Gamma, Kx <- K * e^Gamma
            for (int x = tid; x < Cc * DK; x += kNT) {
                const int i = x / DK, c = x % DK;
                const float e = expf(Gm[i * KS + c]);
                Qs[i * KS + c] *= e;
                Kx[i * KS + c] = Ks[i * KS + c] * e;
            }
        }
        __syncthreads();
        // ---- right-hand side: beta * (V - (K * e^Gamma) S) ---------------
        //      warp w: rows 8w .. 8w + 7 (K rows as broadcast float4 along c); lane: column
        {
            const int j = lane, i0 = warp * 8;
            if (i0 < Cc) {
                const float* kb = (GATE == kGatePerKey) ? Kx : Ks;
                float acc[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) acc[r] = 0.f;
#pragma unroll 2
                for (int c = 0; c < DK; c += 4) {
                    const float s0 = Ss[c * kVS + j], s1 = Ss[(c + 1) * kVS + j];
                    const float s2 = Ss[(c + 2) * kVS + j], s3 = Ss[(c + 3) * kVS + j];
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const float4 kv = *reinterpret_cast<const float4*>(kb + (i0 + r) * KS + c);
                        acc[r] = fmaf(kv.x, s0, fmaf(kv.y, s1, fmaf(kv.z, s2, fmaf(kv.w, s3, acc[r]))));
                    }
                }
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int i = i0 + r;
                    if (i < Cc) {
                        const float a = (GATE != kGatePerKey) ? acc[r] * eG[i] : acc[r];
                        Vs[i * kVS + j] = bs[i] * (Vs[i * kVS + j] - a);
                    }
                }
            }
        }
        __syncthreads();
        // ---- (I + A) U = rhs by 16-row blocks: the diagonal inverses D_b = (I + A_bb)^-1 of
        //      every block at once (forward substitution, one warp per block, lane = column),
        //      then U_b = D_b (rhs_b - sum_{m < 16 b} A_bm U_m) block after block.  Rows and
        //      columns past Cc are identity / zero (never read by the later steps) ----------
        {
            const int nb = (Cc + 15) >> 4;
            if (warp < nb && lane < 16) {
                const int k0 = warp * 16, jj = lane;
                float x[16];
#pragma unroll
                for (int ii = 0; ii < 16; ++ii) {
                    float p0 = ii == jj ? 1.f : 0.f, p1 = 0.f;
                    if (k0 + ii < Cc) {
#pragma unroll
                        for (int m = 0; m < ii; m += 2) {
                            p0 -= Am[(k0 + ii) * kCS + k0 + m] * x[m];
                            if (m + 1 < ii) p1 -= Am[(k0 + ii) * kCS + k0 + m + 1] * x[m + 1];
                        }
                    }
                    x[ii] = p0 + p1;
                }
#pragma unroll
                for (int ii = 0; ii < 16; ++ii) Dm[(warp * 16 + ii) * 17 + jj] = x[ii];
            }
            __syncthreads();
            for (int b = 0; b < nb; ++b) {
                const int r0 = 16 * b;
                // rhs_b -= A_b,<b U_<b : 16 x kDVT outputs, two per thread
                if (b > 0) {
                    for (int x = tid; x < 16 * kDVT; x += kNT) {
                        const int i = r0 + x / kDVT, j = x % kDVT;
                        if (i < Cc) {
                            float a4[4] = {0.f, 0.f, 0.f, 0.f};
                            for (int m = 0; m < r0; m += 4) {
#pragma unroll
                                for (int u = 0; u < 4; ++u)
                                    a4[u] = fmaf(Am[i * kCS + m + u], Vs[(m + u) * kVS + j], a4[u]);
                            }
                            Vs[i * kVS + j] -= (a4[0] + a4[1]) + (a4[2] + a4[3]);
                        }
                    }
                    __syncthreads();
                }
                // U_b = D_b rhs_b (all reads before any write)
                float val[16 * kDVT / kNT];
#pragma unroll
                for (int u = 0; u < 16 * kDVT / kNT; ++u) {
                    const int x = tid + u * kNT;
                    const int ii = x / kDVT, j = x % kDVT;
                    const float* drow = Dm + (b * 16 + ii) * 17;
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int t = 0; t < 16; t += 2) {
                        if (t <= ii) a0 = fmaf(drow[t], Vs[(r0 + t) * kVS + j], a0);
                        if (t + 1 <= ii) a1 = fmaf(drow[t + 1], Vs[(r0 + t + 1) * kVS + j], a1);
                    }
                    val[u] = a0 + a1;
                }
                __syncthreads();
#pragma unroll
                for (int u = 0; u < 16 * kDVT / kNT; ++u) {
                    const int x = tid + u * kNT;
                    const int ii = x / kDVT, j = x % kDVT;
                    if (r0 + ii < Cc) Vs[(r0 + ii) * kVS + j] = val[u];
                }
                __syncthreads();
            }
        }
        // ---- output: O = (Q * e^Gamma) S + P U ---------------------------
        //      warp w: rows 8w .. 8w + 7 (Q and P rows as broadcast float4); lane: column
        {
            const int j = lane, i0 = warp * 8;
            if (i0 < Cc) {
                float acc[8], pu[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) acc[r] = pu[r] = 0.f;
#pragma unroll 2
                for (int c = 0; c < DK; c += 4) {
                    const float s0 = Ss[c * kVS + j], s1 = Ss[(c + 1) * kVS + j];
                    const float s2 = Ss[(c + 2) * kVS + j], s3 = Ss[(c + 3) * kVS + j];
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const float4 qv = *reinterpret_cast<const float4*>(Qs + (i0 + r) * KS + c);
                        acc[r] = fmaf(qv.x, s0, fmaf(qv.y, s1, fmaf(qv.z, s2, fmaf(qv.w, s3, acc[r]))));
                    }
                }
                // P U over positions 0 .. i0 + 7 (P is zero above the diagonal and past Cc,
                // and so are the rows of U past Cc)
                for (int m = 0; m < i0 + 8; m += 4) {
                    const float u0 = Vs[m * kVS + j], u1 = Vs[(m + 1) * kVS + j];
                    const float u2 = Vs[(m + 2) * kVS + j], u3 = Vs[(m + 3) * kVS + j];
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const float4 pv = *reinterpret_cast<const float4*>(Pm + (i0 + r) * kCS + m);
                        pu[r] = fmaf(pv.x, u0, fmaf(pv.y, u1, fmaf(pv.z, u2, fmaf(pv.w, u3, pu[r]))));
                    }
                }
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int i = i0 + r;
                    if (i < Cc) {
                        const float a = (GATE != kGatePerKey) ? acc[r] * eG[i] : acc[r];
                        st_elem(o + (tok0 + c0 + i) * DV + col0 + j, a + pu[r]);
                    }
                }
            }
        }
        if (GATE == kGatePerKey) {
            __syncthreads();   // Kx <- K * e^(Gamma_last - Gamma)
            for (int x = tid; x < Cc * DK; x += kNT) {
                const int i = x / DK, c = x % DK;
                Kx[i * KS + c] = Ks[i * KS + c] * expf(Gm[(Cc - 1) * KS + c] - Gm[i * KS + c]);
            }
        }
        __syncthreads();
        // ---- state: S <- Diag(e^Gamma_last) S + (K * e^(Gamma_last - Gamma))^T U
        //      warp w: key channels 8w .. 8w + 7 (+ 64) (K rows as broadcast float4); lane: column
        {
            const int j = lane;
            for (int cb = warp * 8; cb < DK; cb += 8 * (kNT / 32)) {
                float acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
                const float* kb = (GATE == kGatePerKey) ? Kx : Ks;
                for (int i = 0; i < Cc; ++i) {
                    const float u = (GATE == kGatePerKey) ? Vs[i * kVS + j] : Vs[i * kVS + j] * eT[i];
                    const float4 k0 = *reinterpret_cast<const float4*>(kb + i * KS + cb);
                    const float4 k1 = *reinterpret_cast<const float4*>(kb + i * KS + cb + 4);
                    acc[0] = fmaf(k0.x, u, acc[0]); acc[1] = fmaf(k0.y, u, acc[1]);
                    acc[2] = fmaf(k0.z, u, acc[2]); acc[3] = fmaf(k0.w, u, acc[3]);
                    acc[4] = fmaf(k1.x, u, acc[4]); acc[5] = fmaf(k1.y, u, acc[5]);
                    acc[6] = fmaf(k1.z, u, acc[6]); acc[7] = fmaf(k1.w, u, acc[7]);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int c = cb + e;
                    const float dec = (GATE == kGatePerKey) ? expf(Gm[(Cc - 1) * KS + c])
                                      : (GATE == kGateScalar) ? expf(Gm[Cc - 1]) : 1.f;
                    Ss[c * kVS + j] = dec * Ss[c * kVS + j] + acc[e];
                }
            }
        }
        // ---- snapshot: the state after chunks 1 .. (s + 1) snap_every (full chunks only)
        if (snaps) {
            const int ci = c0 / chunk + 1;               // chunks done
            if (ci % snap_every == 0 && ci / snap_every <= n_snap) {
                __syncthreads();
                const int64_t sn = bh * n_snap + ci / snap_every - 1;
                for (int x = tid; x < DK * kDVT; x += kNT) {
                    const int i = x / kDVT, j = x % kDVT;
                    snaps[(sn * DK + i) * DV + col0 + j] = Ss[i * kVS + j];
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

template <int DK, int GATE, typename Tin, bool PRO = false>
static cudaError_t launch_simt_t(const ChunkArgs& a, cudaStream_t st) {
    using L = SimtSmem<DK, GATE>;
    auto kern = chunk_simt_kernel<DK, GATE, Tin, PRO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return e;
    const int64_t grid = a.B * a.H * (a.dv / kDVT);
    kern<<<(unsigned)grid, kNT, L::bytes, st>>>(
        static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
        a.beta, a.g, a.S0, static_cast<Tin*>(a.o), a.S_T, (int)a.T, a.dv, a.chunk, a.scale, a.snaps, a.snap_every,
        a.n_snap, a.A_log, a.dt_bias, (int)a.H, (float)a.prologue);
    return counted(cudaGetLastError());
}

template <int DK, typename Tin>
static cudaError_t launch_simt_gate(const ChunkArgs& a, cudaStream_t st) {
    switch (a.gate) {
        case kGateNone: return launch_simt_t<DK, kGateNone, Tin>(a, st);
        case kGateScalar:
            return a.prologue ? launch_simt_t<DK, kGateScalar, Tin, true>(a, st)
                              : launch_simt_t<DK, kGateScalar, Tin>(a, st);
        default: return launch_simt_t<DK, kGatePerKey, Tin>(a, st);
    }
}

cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t st) {
    if (a.B * a.H == 0) return cudaSuccess;
    if (a.dk == 128)
        return a.bf16 ? launch_simt_gate<128, __nv_bfloat16>(a, st) : launch_simt_gate<128, float>(a, st);
    return a.bf16 ? launch_simt_gate<64, __nv_bfloat16>(a, st) : launch_simt_gate<64, float>(a, st);
}

}  // namespace dn
