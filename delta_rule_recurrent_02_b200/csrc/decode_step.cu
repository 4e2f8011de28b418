// decode_step.cu -- one recurrent step of the delta rule per (sequence, head).
//
// "Linear attention and Gated DeltaNet" (ch. 28), "The recurrent form": for
// each head, decay the d_k x d_v fp32 state, predict p = S~^T k, write
// S = S~ + k (beta (v - p))^T and read o = S^T (scale q); for KDA the decay
// scales row i (key channel i) by exp(g_i) ("A walk through of the DeltaNet
// family", the KDA recurrence).  The page calls the step memory-bound on the
// state; the kernel therefore streams each state exactly once in and once
// out of HBM and does everything else on chip.
//
// One CTA owns one head.  Thread (rs, cg) holds rows rs, rs + RS, ... and the
// four columns 4cg .. 4cg+3 of S in registers (a warp covers one full 512-byte
// row per 128-bit access, so every load and store is coalesced).  The two
// reductions over rows (p = S~^T k and S~^T q') go through shared memory;
// the output uses o = S~^T q' + (q'.k) delta, which needs S~ only, so the
// state is read once and written once.
#include "dn_common.cuh"
#include "dn_kernels.h"

namespace dn {

// PRO: the Gated DeltaNet layer's prologue ("The full layer", steps 4 and 5):
// q and k normalised per head, beta = bmul sigmoid(b) (bmul 1, or 2 for the
// gate in (0, 2)), g = -exp(A_log) softplus(a + dt_bias), from the raw b and a
// in `beta` and `g` (scalar gate).
// NORM: the layer's gated RMSNorm ("The full layer", step 7) on the step's
// output row: o <- weight * o / sqrt(mean(o^2) + eps) * act(z), act = SiLU
// (NORM 1) or the logistic sigmoid (NORM 2); z [B, H, d_v], weight [d_v].
template <int DK, int DV, typename Tin, int GATE, bool PRO = false, int NORM = 0>
__global__ void __launch_bounds__(2 * DV)
decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                   const Tin* __restrict__ v, const float* __restrict__ beta,
                   const float* __restrict__ g, float* __restrict__ S,
                   Tin* __restrict__ o, float scale, const float* __restrict__ A_log = nullptr,
                   const float* __restrict__ dt_bias = nullptr, int H = 1, int rep = 1, float bmul = 1.f,
                   const Tin* __restrict__ z = nullptr, const float* __restrict__ nw = nullptr,
                   float eps = 0.f) {
    constexpr int NT = 2 * DV;     // threads
    constexpr int TPR = DV / 4;    // threads per state row
    constexpr int RS = NT / TPR;   // row sets (8)
    constexpr int RPT = DK / RS;   // rows per thread
    const int64_t head = blockIdx.x;
    const int64_t khead = rep == 1 ? head : (head / H) * (H / rep) + (head % H) / rep;   // q and k row
    const int tid = threadIdx.x;
    const int cg = tid % TPR;
    const int rs = tid / TPR;

    __shared__ float ks[DK], qs[DK], as[DK];
    __shared__ float4 red_p[RS][TPR], red_q[RS][TPR];
    __shared__ float qk_s;
    __shared__ float rn_s[2];

    float* Sh = S + head * (DK * DV);
    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m)
        s[m] = ld_stream_f4(Sh + (rs + RS * m) * DV + cg * 4);

    for (int i = tid; i < DK; i += NT) {
        ks[i] = ld_elem(k + khead * DK + i);
        qs[i] = (PRO ? 1.f : scale) * ld_elem(q + khead * DK + i);
        if (GATE == kGatePerKey) as[i] = expf(g[head * DK + i]);
    }
    const float4 vv = ld4(v + head * DV + cg * 4);
    float b = beta[head];
    float a = (GATE == kGateScalar) ? g[head] : 0.f;
    if (PRO) gdn_raw_gates(b, a, expf(A_log[head % H]), dt_bias[head % H], bmul);
    if (GATE == kGateScalar) a = expf(a);
    else a = 1.0f;
    __syncthreads();
    // q . k; with the prologue also ||k||^2 and ||q||^2 of the raw rows: k and q enter
    // every product linearly, so their factors rk = 1 / max(||k||, 1e-12) and
    // rq = scale / max(||q||, 1e-12) are applied to the reduced sums below instead of
    // to the rows (no pass over the rows, no barrier of its own)
    if (tid < 32) {
        float x = 0.f, sk = 0.f, sq = 0.f;
        for (int i = tid; i < DK; i += 32) {
            x += qs[i] * ks[i];
            if (PRO) {
                sk += ks[i] * ks[i];
                sq += qs[i] * qs[i];
            }
        }
        x = warp_sum(x);
        if (PRO) {
            sk = warp_sum(sk);
            sq = warp_sum(sq);
        }
        if (tid == 0) {
            qk_s = x;
            if (PRO) {
                rn_s[0] = fminf(rsqrtf(sk), 1e12f);
                rn_s[1] = scale * fminf(rsqrtf(sq), 1e12f);
            }
        }
    }

    float4 p4 = make_float4(0.f, 0.f, 0.f, 0.f), q4 = p4;
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int r = rs + RS * m;
        const float d = (GATE == kGatePerKey) ? as[r] : a;
        if (GATE != kGateNone) {
            s[m].x *= d; s[m].y *= d; s[m].z *= d; s[m].w *= d;
        }
        const float kr = ks[r], qr = qs[r];
        p4.x += kr * s[m].x; p4.y += kr * s[m].y; p4.z += kr * s[m].z; p4.w += kr * s[m].w;
        q4.x += qr * s[m].x; q4.y += qr * s[m].y; q4.z += qr * s[m].z; q4.w += qr * s[m].w;
    }
    red_p[rs][cg] = p4;
    red_q[rs][cg] = q4;
    __syncthreads();

    float4 pred = make_float4(0.f, 0.f, 0.f, 0.f), qsum = pred;
#pragma unroll
    for (int r = 0; r < RS; ++r) {
        const float4 x = red_p[r][cg], y = red_q[r][cg];
        pred.x += x.x; pred.y += x.y; pred.z += x.z; pred.w += x.w;
        qsum.x += y.x; qsum.y += y.y; qsum.z += y.z; qsum.w += y.w;
    }
    // with the prologue: the unit k's and the scaled unit q's sums (rk, rq are visible
    // after the barrier above)
    const float rk = PRO ? rn_s[0] : 1.f, rq = PRO ? rn_s[1] : 1.f;
    if (PRO) {
        pred.x *= rk; pred.y *= rk; pred.z *= rk; pred.w *= rk;
        qsum.x *= rq; qsum.y *= rq; qsum.z *= rq; qsum.w *= rq;
    }
    float4 dl;
    dl.x = b * (vv.x - pred.x); dl.y = b * (vv.y - pred.y);
    dl.z = b * (vv.z - pred.z); dl.w = b * (vv.w - pred.w);
    // the state takes (rk k_raw) dl^T: rk rides on dl
    const float4 dk = PRO ? make_float4(rk * dl.x, rk * dl.y, rk * dl.z, rk * dl.w) : dl;

#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int r = rs + RS * m;
        const float kr = ks[r];
        float4 x = s[m];
        x.x += kr * dk.x; x.y += kr * dk.y; x.z += kr * dk.z; x.w += kr * dk.w;
        st_stream_f4(Sh + r * DV + cg * 4, x);
    }
    if (rs == 0) {
        const float qk = PRO ? rq * rk * qk_s : qk_s;
        float4 ov;
        ov.x = qsum.x + qk * dl.x; ov.y = qsum.y + qk * dl.y;
        ov.z = qsum.z + qk * dl.z; ov.w = qsum.w + qk * dl.w;
        if (NORM) {
            // the row's mean square over the TPR threads of row set 0 (a warp, or half of one)
            float ss = ov.x * ov.x + ov.y * ov.y + ov.z * ov.z + ov.w * ov.w;
            constexpr unsigned kMask = TPR >= 32 ? 0xffffffffu : ((1u << TPR) - 1u);
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(kMask, ss, off);
            const float r = 1.f / sqrtf(ss / (float)DV + eps);
            const float4 zz = ld4(z + head * DV + cg * 4);
            const float4 ww = *reinterpret_cast<const float4*>(nw + cg * 4);
            auto act = [](float x) { return NORM == 1 ? x / (1.f + __expf(-x)) : 1.f / (1.f + __expf(-x)); };
            ov.x = ov.x * r * ww.x * act(zz.x); ov.y = ov.y * r * ww.y * act(zz.y);
            ov.z = ov.z * r * ww.z * act(zz.z); ov.w = ov.w * r * ww.w * act(zz.w);
        }
        st4(o + head * DV + cg * 4, ov);
    }
}

template <int DK, int DV, typename Tin>
static cudaError_t launch_decode_gate(const DecodeArgs& a, cudaStream_t st) {
    const unsigned grid = (unsigned)(a.B * a.H);
    const Tin* q = static_cast<const Tin*>(a.q);
    const Tin* k = static_cast<const Tin*>(a.k);
    const Tin* v = static_cast<const Tin*>(a.v);
    Tin* o = static_cast<Tin*>(a.o);
    if (a.prologue) {
        const Tin* z = static_cast<const Tin*>(a.z);
        if (a.norm == 1)
            decode_step_kernel<DK, DV, Tin, kGateScalar, true, 1><<<grid, 2 * DV, 0, st>>>(
                q, k, v, a.beta, a.g, a.S, o, a.scale, a.A_log, a.dt_bias, (int)a.H, a.rep, (float)a.prologue, z,
                a.norm_weight, a.eps);
        else if (a.norm == 2)
            decode_step_kernel<DK, DV, Tin, kGateScalar, true, 2><<<grid, 2 * DV, 0, st>>>(
                q, k, v, a.beta, a.g, a.S, o, a.scale, a.A_log, a.dt_bias, (int)a.H, a.rep, (float)a.prologue, z,
                a.norm_weight, a.eps);
        else
            decode_step_kernel<DK, DV, Tin, kGateScalar, true><<<grid, 2 * DV, 0, st>>>(
                q, k, v, a.beta, a.g, a.S, o, a.scale, a.A_log, a.dt_bias, (int)a.H, a.rep, (float)a.prologue);
        return counted(cudaGetLastError());
    }
    switch (a.gate) {
        case kGateNone:
            decode_step_kernel<DK, DV, Tin, kGateNone><<<grid, 2 * DV, 0, st>>>(q, k, v, a.beta, a.g, a.S, o, a.scale,
                                                                          nullptr, nullptr, (int)a.H, a.rep);
            break;
        case kGateScalar:
            decode_step_kernel<DK, DV, Tin, kGateScalar><<<grid, 2 * DV, 0, st>>>(q, k, v, a.beta, a.g, a.S, o, a.scale,
                                                                          nullptr, nullptr, (int)a.H, a.rep);
            break;
        default:
            decode_step_kernel<DK, DV, Tin, kGatePerKey><<<grid, 2 * DV, 0, st>>>(q, k, v, a.beta, a.g, a.S, o, a.scale,
                                                                          nullptr, nullptr, (int)a.H, a.rep);
            break;
    }
    return counted(cudaGetLastError());
}

template <int DK, int DV>
static cudaError_t launch_decode_dims(const DecodeArgs& a, cudaStream_t st) {
    return a.bf16 ? launch_decode_gate<DK, DV, __nv_bfloat16>(a, st)
                  : launch_decode_gate<DK, DV, float>(a, st);
}

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t st) {
    if (a.B * a.H == 0) return cudaSuccess;
    if (a.dk == 128 && a.dv == 128) return launch_decode_dims<128, 128>(a, st);
    if (a.dk == 128 && a.dv == 64) return launch_decode_dims<128, 64>(a, st);
    if (a.dk == 64 && a.dv == 128) return launch_decode_dims<64, 128>(a, st);
    return launch_decode_dims<64, 64>(a, st);
}

}  // namespace dn
