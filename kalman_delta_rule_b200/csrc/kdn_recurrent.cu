// Fused recurrent Diagonal-KDN kernel (KDA article, "fused recurrent kernel" regime:
// one token at a time with vector operations; explainer "对角近似" for the diagonal
// uncertainty).  One CTA owns one (sequence, head, d_v tile): the memory tile lives
// in registers as float4 rows, the d_k-length uncertainty in the first d_k threads.
//
// Per token:
//   P^- = alpha^2 P + sigma;  g = P^- k / (r + sum P^- k^2)       (threads = key channels)
//   a_j = sum_i alpha_i k_i S_ij;  b_j = sum_i alpha_i q_i S_ij   (column sums over rows)
//   u_j = v_j - a_j;  o_j = b_j + (q.g) u_j;  S_ij <- alpha_i S_ij + g_i u_j
//   P = P^- / (1 + mu P^- k^2 / r)
// o_t = S_t^T q_t expands to (D S)^T q + (q.g) u, so S is read once and written once.
//
// Isotropic KDN (explainer "各向同性近似"; aifromscratch "Approximation 2"): one
// uncertainty p per head, held by every thread; per token the channel sums of alpha^2,
// sigma, k^2 and q k give p^- = mean(alpha^2) p + mean(sigma), g = p^- k / (r + p^- |k|^2)
// and p = p^- / (1 + mu p^- |k|^2 / (d_k r)).
//
// Decode is the same kernel on one token per sequence with the state in HBM updated
// in place (one tile per head so the uncertainty read and write stay in one CTA).
#include "kdn_common.cuh"
#include "kdn_launch.h"

namespace kdn {

template <int DK, int DVT>
struct RecShape {
    static constexpr int nw_raw = DK * DVT / 1024;
    static constexpr int nw_lo = DK / 32 > 1 ? DK / 32 : 1;
    static constexpr int NW = nw_raw < nw_lo ? nw_lo : (nw_raw > 16 ? 16 : nw_raw);
    static constexpr int NT = NW * 32;
    static constexpr int TPR = DVT / 4;       // threads per memory row (4 columns each)
    static constexpr int RPP = NT / TPR;      // rows per pass
    static constexpr int NPASS = DK / RPP;    // rows held per thread
    static_assert(NT % TPR == 0, "row split");
    static_assert(DK % RPP == 0 && NPASS >= 1, "row passes");
    static_assert(NT >= DK, "one thread per key channel");
};

template <int DK, int DVT, typename Tin, bool ISO>
__global__ void __launch_bounds__(RecShape<DK, DVT>::NT)
recurrent_kernel(TokenArgs a, int write_p_all_tiles)
{
    using Sh = RecShape<DK, DVT>;
    constexpr int NW = Sh::NW, TPR = Sh::TPR, RPP = Sh::RPP, NPASS = Sh::NPASS;

    const Tin *__restrict__ q = static_cast<const Tin *>(a.q);
    const Tin *__restrict__ k = static_cast<const Tin *>(a.k);
    const Tin *__restrict__ v = static_cast<const Tin *>(a.v);
    const Tin *__restrict__ alpha = static_cast<const Tin *>(a.alpha);
    const Tin *__restrict__ sigma = static_cast<const Tin *>(a.sigma);
    const Tin *__restrict__ r = static_cast<const Tin *>(a.r);
    Tin *__restrict__ o = static_cast<Tin *>(a.o);

    const int ntiles = a.dv / DVT;
    const int tile = blockIdx.x % ntiles;
    const int sh = blockIdx.x / ntiles;   // sequence * H + head
    const int s = sh / a.H, h = sh % a.H;
    int t0, t1;
    seq_range(a, s, t0, t1);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = tid % TPR, rs = tid / TPR;
    const int col0 = tile * DVT + c * 4;

    __shared__ float ak_s[2][DK], aq_s[2][DK], al_s[2][DK];
    __shared__ float g_s[DK];
    __shared__ float redA[RPP][DVT], redB[RPP][DVT];
    __shared__ float u_s[DVT];
    __shared__ float wsum[ISO ? 4 : 2][NW];

    // memory tile -> registers
    float4 S[NPASS];
    const size_t sbase = (size_t)sh * DK * a.dv;
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
        const int row = p * RPP + rs;
        S[p] = a.S0 ? __ldcs(reinterpret_cast<const float4 *>(a.S0 + sbase + (size_t)row * a.dv + col0))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float P = 1.f;   // diagonal: channel tid's uncertainty; isotropic: the head's (every thread)
    if (ISO) {
        if (a.P0) P = a.P0[sh];
    } else if (tid < DK && a.P0) {
        P = a.P0[(size_t)sh * DK + tid];
    }

    const float mu = a.mu;
    for (int t = t0; t < t1; ++t) {
        const int buf = t & 1;
        const size_t th = (size_t)t * a.H + h;
        // ---- per key channel: predict and the two gain reductions
        float pm = 0.f, kk = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f, x4 = 0.f;
        if (tid < DK) {
            const size_t e = th * DK + tid;
            const float al = ldf(alpha + e), sg = ldf(sigma + e), qq = ldf(q + e);
            kk = ldf(k + e);
            if (ISO) {
                x1 = kk * kk;
                x2 = qq * kk;
                x3 = al * al;
                x4 = sg;
            } else {
                pm = fmaf(al * al, P, sg);
                const float pk = pm * kk;
                x1 = pk * kk;
                x2 = qq * pk;
            }
            ak_s[buf][tid] = al * kk;
            aq_s[buf][tid] = al * qq;
            al_s[buf][tid] = al;
        }
        float vj = 0.f;
        if (tid < DVT) vj = ldf(v + th * a.dv + tile * DVT + tid);
        const float rr = ldf(r + th);
        x1 = warp_sum(x1);
        x2 = warp_sum(x2);
        if (ISO) {
            x3 = warp_sum(x3);
            x4 = warp_sum(x4);
        }
        if (lane == 0) {
            wsum[0][warp] = x1;
            wsum[1][warp] = x2;
            if constexpr (ISO) { wsum[2][warp] = x3; wsum[3][warp] = x4; }
        }
        __syncthreads();
        float sx1 = 0.f, sx2 = 0.f, sx3 = 0.f, sx4 = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            sx1 += wsum[0][w];
            sx2 += wsum[1][w];
            if constexpr (ISO) { sx3 += wsum[2][w]; sx4 += wsum[3][w]; }
        }
        float den, qg;
        if (ISO) {
            constexpr float inv_dk = 1.f / DK;
            pm = fmaf(sx3 * inv_dk, P, sx4 * inv_dk);
            den = fmaf(pm, sx1, rr);
            qg = pm * sx2 / den;
            if (tid < DK) g_s[tid] = pm * kk / den;
            P = pm / fmaf(mu * sx1 * inv_dk / rr, pm, 1.f);
        } else {
            den = rr + sx1;
            qg = sx2 / den;
            if (tid < DK) {
                g_s[tid] = pm * kk / den;
                P = pm / fmaf(mu * kk * kk / rr, pm, 1.f);
            }
        }
        // ---- column partial sums of (alpha*k)^T S and (alpha*q)^T S over this thread's rows
        float4 A = make_float4(0.f, 0.f, 0.f, 0.f), B = A;
#pragma unroll
        for (int p = 0; p < NPASS; ++p) {
            const int i = p * RPP + rs;
            const float w1 = ak_s[buf][i], w2 = aq_s[buf][i];
            A.x = fmaf(w1, S[p].x, A.x); A.y = fmaf(w1, S[p].y, A.y);
            A.z = fmaf(w1, S[p].z, A.z); A.w = fmaf(w1, S[p].w, A.w);
            B.x = fmaf(w2, S[p].x, B.x); B.y = fmaf(w2, S[p].y, B.y);
            B.z = fmaf(w2, S[p].z, B.z); B.w = fmaf(w2, S[p].w, B.w);
        }
        *reinterpret_cast<float4 *>(&redA[rs][c * 4]) = A;
        *reinterpret_cast<float4 *>(&redB[rs][c * 4]) = B;
        __syncthreads();
        if (tid < DVT) {
            float sa = 0.f, sb = 0.f;
#pragma unroll
            for (int j = 0; j < RPP; ++j) { sa += redA[j][tid]; sb += redB[j][tid]; }
            const float u = vj - sa;
            u_s[tid] = u;
            stf(o + th * a.dv + tile * DVT + tid, fmaf(qg, u, sb));
        }
        __syncthreads();
        // ---- write: S <- diag(alpha) S + g u^T
        const float4 u4 = *reinterpret_cast<const float4 *>(&u_s[c * 4]);
#pragma unroll
        for (int p = 0; p < NPASS; ++p) {
            const int i = p * RPP + rs;
            const float al = al_s[buf][i], gi = g_s[i];
            S[p].x = fmaf(al, S[p].x, gi * u4.x);
            S[p].y = fmaf(al, S[p].y, gi * u4.y);
            S[p].z = fmaf(al, S[p].z, gi * u4.z);
            S[p].w = fmaf(al, S[p].w, gi * u4.w);
        }
    }

    if (a.S_out) {
#pragma unroll
        for (int p = 0; p < NPASS; ++p) {
            const int row = p * RPP + rs;
            __stcs(reinterpret_cast<float4 *>(a.S_out + sbase + (size_t)row * a.dv + col0), S[p]);
        }
    }
    if (a.P_out && (tile == 0 || write_p_all_tiles)) {
        if (ISO) {
            if (tid == 0) a.P_out[sh] = P;
        } else if (tid < DK) {
            a.P_out[(size_t)sh * DK + tid] = P;
        }
    }
}

template <int DK, int DVT, typename Tin>
static cudaError_t launch_rec(const TokenArgs &a, cudaStream_t st) {
    const unsigned grid = (unsigned)((size_t)a.nseq * a.H * (a.dv / DVT));
    if (a.iso) recurrent_kernel<DK, DVT, Tin, true><<<grid, RecShape<DK, DVT>::NT, 0, st>>>(a, 0);
    else recurrent_kernel<DK, DVT, Tin, false><<<grid, RecShape<DK, DVT>::NT, 0, st>>>(a, 0);
    return cudaGetLastError();
}

template <int DK, typename Tin>
static cudaError_t dispatch_dvt(const TokenArgs &a, int dvt, cudaStream_t st) {
    switch (dvt) {
        case 32: return launch_rec<DK, 32, Tin>(a, st);
        case 64: return launch_rec<DK, 64, Tin>(a, st);
        case 128: return launch_rec<DK, 128, Tin>(a, st);
        case 256: return launch_rec<DK, 256, Tin>(a, st);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
static cudaError_t dispatch_dk(const TokenArgs &a, int dvt, cudaStream_t st) {
    switch (a.dk) {
        case 32: return dispatch_dvt<32, Tin>(a, dvt, st);
        case 64: return dispatch_dvt<64, Tin>(a, dvt, st);
        case 128: return dispatch_dvt<128, Tin>(a, dvt, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_recurrent(const TokenArgs &a, bool bf16_in, int dvt, cudaStream_t st) {
    if (a.nseq == 0 || a.H == 0) return cudaSuccess;
    return bf16_in ? dispatch_dk<bf16>(a, dvt, st) : dispatch_dk<float>(a, dvt, st);
}

}  // namespace kdn
