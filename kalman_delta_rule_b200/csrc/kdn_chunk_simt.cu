// Chunkwise Diagonal-KDN forward on CUDA cores, fp32 arithmetic (KDA article,
// "chunkwise" regime: provisional errors corrected by a causal triangular solve).
//
// One CTA owns one (sequence, head, d_v tile) and walks the sequence chunk by chunk
// (chunk C <= 64, restarting at sequence starts; the last chunk may be partial).
// Inside a chunk with local tokens t = 0..L-1 and b_t = sum_{j<=t} log alpha_j
// (per channel, inclusive), the recurrence unrolls exactly to
//     u_t + sum_{s<t} A_ts u_s = v_t - S0^T (e^{b_t} k_t),    A_ts = k_t . (e^{b_t - b_s} g_s)
//     o_t = S0^T (e^{b_t} q_t) + sum_{s<=t} Aq_ts u_s,         Aq_ts = q_t . (e^{b_t - b_s} g_s)
//     S_L = e^{b_{L-1}} S0 + sum_s (e^{b_{L-1} - b_s} g_s) u_s^T
// so U = (I + A)^-1 W with W = V - K~ S0 (forward substitution).  The pairwise decay
// factors are formed per term, which keeps the path exact for any alpha in [0, 1]
// (log alpha is floored at -80, i.e. alpha < 2e-35 acts as 0).
//
// The uncertainty recursion and the gain of the chunk's tokens are computed first
// (one thread per key channel), with the chunk's per-token gain denominators reduced
// across channels.  This kernel is the fp32-exact path; the bf16 throughput path is
// the tensor-core kernel.
//
// Isotropic KDN (explainer "各向同性近似"): the head's single uncertainty runs first,
// from per-token channel sums (thread = token), p^- = mean(alpha^2) p + mean(sigma),
// p = p^- / (1 + mu p^- |k|^2 / (d_k r)); the gain numerators are then p^-_t k_t.
#include "kdn_common.cuh"
#include "kdn_launch.h"

namespace kdn {

namespace {
constexpr int CMAX = 64;
constexpr int LDC = CMAX + 1;   // padded row length of the channel-major [dk][C] arrays
constexpr int NT = 256;

template <int DK, int DVT>
struct SimtSmem {
    static constexpr int kK = 0;                    // [DK][LDC] k, then k~ = e^{b} k
    static constexpr int kQ = kK + DK * LDC;        // [DK][LDC] q, then q~
    static constexpr int kG = kQ + DK * LDC;        // [DK][LDC] gain, then e^{b_last - b_s} g
    static constexpr int kB = kG + DK * LDC;        // [DK][LDC] cumulative log decay
    static constexpr int kS = kB + DK * LDC;        // [DK][DVT] memory tile
    static constexpr int kA = kS + DK * DVT;        // [C][LDC] A (strictly lower)
    static constexpr int kAq = kA + CMAX * LDC;     // [C][LDC] Aq (lower incl. diagonal)
    static constexpr int kU = kAq + CMAX * LDC;     // [C][DVT] W, solved in place into U
    static constexpr int kR = kU + CMAX * DVT;      // [C] r
    static constexpr int kID = kR + CMAX;           // [C] 1 / gain denominator
    static constexpr int kGC = kID + CMAX;          // [DK] e^{b_last}
    static constexpr int total = kGC + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};
}  // namespace

template <int DK, int DVT, typename Tin>
__global__ void __launch_bounds__(NT, 1) chunk_simt_kernel(TokenArgs a, int C)
{
    using L_ = SimtSmem<DK, DVT>;
    extern __shared__ float sm[];
    float *Ks = sm + L_::kK, *Qs = sm + L_::kQ, *Gs = sm + L_::kG, *Bs = sm + L_::kB;
    float *Ss = sm + L_::kS, *As = sm + L_::kA, *Aqs = sm + L_::kAq, *Us = sm + L_::kU;
    float *Rs = sm + L_::kR, *IDs = sm + L_::kID, *GCs = sm + L_::kGC;

    const Tin *__restrict__ q = static_cast<const Tin *>(a.q);
    const Tin *__restrict__ k = static_cast<const Tin *>(a.k);
    const Tin *__restrict__ v = static_cast<const Tin *>(a.v);
    const Tin *__restrict__ alpha = static_cast<const Tin *>(a.alpha);
    const Tin *__restrict__ sigma = static_cast<const Tin *>(a.sigma);
    const Tin *__restrict__ r = static_cast<const Tin *>(a.r);
    Tin *__restrict__ o = static_cast<Tin *>(a.o);

    const int ntiles = a.dv / DVT;
    const int tile = blockIdx.x % ntiles;
    const int sh = blockIdx.x / ntiles;
    const int s_ = sh / a.H, h = sh % a.H;
    int t0, t1;
    seq_range(a, s_, t0, t1);
    const int tid = threadIdx.x;
    const int H = a.H, dv = a.dv;
    const float mu = a.mu;

    // memory tile and uncertainty
    const size_t sbase = (size_t)sh * DK * dv + (size_t)tile * DVT;
    for (int e = tid; e < DK * DVT; e += NT) {
        const int i = e / DVT, j = e % DVT;
        Ss[e] = a.S0 ? a.S0[sbase + (size_t)i * dv + j] : 0.f;
    }
    float P = 1.f;   // diagonal: channel tid; isotropic: the head's (thread 0 carries it)
    if (a.iso) {
        if (a.P0) P = a.P0[sh];
    } else if (tid < DK && a.P0) {
        P = a.P0[(size_t)sh * DK + tid];
    }
    __syncthreads();

    for (int c0 = t0; c0 < t1; c0 += C) {
        const int L = min(C, t1 - c0);
        if (tid < L) Rs[tid] = ldf(r + (size_t)(c0 + tid) * H + h);
        __syncthreads();
        if (a.iso) {
            // channel sums of alpha^2, sigma, k^2 per token (A's rows are free until A is formed)
            if (tid < L) {
                float sa = 0.f, ss = 0.f, sk = 0.f;
                for (int i = 0; i < DK; ++i) {
                    const size_t e = ((size_t)(c0 + tid) * H + h) * DK + i;
                    const float al = ldf(alpha + e), kk = ldf(k + e);
                    sa = fmaf(al, al, sa);
                    ss += ldf(sigma + e);
                    sk = fmaf(kk, kk, sk);
                }
                As[tid * LDC + 0] = sa;
                As[tid * LDC + 1] = ss;
                As[tid * LDC + 2] = sk;
            }
            __syncthreads();
            if (tid == 0) {
                constexpr float inv_dk = 1.f / DK;
                for (int t = 0; t < L; ++t) {
                    const float pm = fmaf(As[t * LDC] * inv_dk, P, As[t * LDC + 1] * inv_dk);
                    As[t * LDC + 3] = pm;
                    P = pm / fmaf(mu * As[t * LDC + 2] * inv_dk / Rs[t], pm, 1.f);
                }
            }
            __syncthreads();
        }
        // ---- uncertainty recursion, gain numerators, cumulative log decay (thread = key channel)
        if (tid < DK) {
            float b = 0.f;
            for (int t = 0; t < L; ++t) {
                const size_t e = ((size_t)(c0 + t) * H + h) * DK + tid;
                const float al = ldf(alpha + e), sg = ldf(sigma + e), kk = ldf(k + e);
                b += fmaxf(logf(al), -80.f);
                const float pm = a.iso ? As[t * LDC + 3] : fmaf(al * al, P, sg);
                Ks[tid * LDC + t] = kk;
                Qs[tid * LDC + t] = ldf(q + e);
                Gs[tid * LDC + t] = pm * kk;
                Bs[tid * LDC + t] = b;
                if (!a.iso) P = pm / fmaf(mu * kk * kk / Rs[t], pm, 1.f);
            }
        }
        __syncthreads();
        // ---- gain denominators r_t + sum_i P^-_i k_i^2
        if (tid < L) {
            float acc = 0.f;
            for (int i = 0; i < DK; ++i) acc = fmaf(Gs[i * LDC + tid], Ks[i * LDC + tid], acc);
            IDs[tid] = 1.f / (Rs[tid] + acc);
        }
        __syncthreads();
        for (int e = tid; e < DK * L; e += NT) {
            const int i = e / L, t = e % L;
            Gs[i * LDC + t] *= IDs[t];
        }
        __syncthreads();
        // ---- A (s < t) and Aq (s <= t) with pairwise decay factors
        {
            const int t = tid % CMAX, sg = tid / CMAX;   // 4 groups of s
            float accA[CMAX / 4], accQ[CMAX / 4];
#pragma unroll
            for (int j = 0; j < CMAX / 4; ++j) { accA[j] = 0.f; accQ[j] = 0.f; }
            if (t < L) {
                for (int i = 0; i < DK; ++i) {
                    const float kt = Ks[i * LDC + t], qt = Qs[i * LDC + t], bt = Bs[i * LDC + t];
#pragma unroll
                    for (int j = 0; j < CMAX / 4; ++j) {
                        const int s = sg + 4 * j;
                        if (s <= t) {
                            const float w = Gs[i * LDC + s] * expf(bt - Bs[i * LDC + s]);
                            accA[j] = fmaf(kt, w, accA[j]);
                            accQ[j] = fmaf(qt, w, accQ[j]);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < CMAX / 4; ++j) {
                    const int s = sg + 4 * j;
                    if (s <= t) {
                        As[t * LDC + s] = (s < t) ? accA[j] : 0.f;
                        Aqs[t * LDC + s] = accQ[j];
                    }
                }
            }
        }
        __syncthreads();
        // ---- decayed operands: k~ = e^{b_t} k, q~ = e^{b_t} q, g' = e^{b_last - b_s} g
        for (int e = tid; e < DK * L; e += NT) {
            const int i = e / L, t = e % L;
            const float bt = Bs[i * LDC + t], bl = Bs[i * LDC + L - 1];
            const float gt = expf(bt);
            Ks[i * LDC + t] *= gt;
            Qs[i * LDC + t] *= gt;
            Gs[i * LDC + t] *= expf(bl - bt);
            if (t == L - 1) GCs[i] = gt;
        }
        __syncthreads();
        // ---- W = V - K~ S0 (into U) and O1 = Q~ S0 (registers)
        constexpr int RPT = NT / DVT;                 // token rows per pass
        float o1[CMAX / RPT];
        {
            const int j = tid % DVT, t_ = tid / DVT;
#pragma unroll
            for (int m = 0; m < CMAX / RPT; ++m) {
                const int t = t_ + m * RPT;
                o1[m] = 0.f;
                if (t < L) {
                    float w = 0.f, oq = 0.f;
                    for (int i = 0; i < DK; ++i) {
                        const float sv = Ss[i * DVT + j];
                        w = fmaf(Ks[i * LDC + t], sv, w);
                        oq = fmaf(Qs[i * LDC + t], sv, oq);
                    }
                    const float vv = ldf(v + ((size_t)(c0 + t) * H + h) * dv + tile * DVT + j);
                    Us[t * DVT + j] = vv - w;
                    o1[m] = oq;
                }
            }
        }
        __syncthreads();
        // ---- forward substitution (I + A) U = W, NPC lanes per column
        {
            constexpr int NPC = NT / DVT;
            const int col = tid / NPC, part = tid % NPC;
            for (int t = 1; t < L; ++t) {
                float acc = 0.f;
                for (int s = part; s < t; s += NPC) acc = fmaf(As[t * LDC + s], Us[s * DVT + col], acc);
#pragma unroll
                for (int off = NPC / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (part == 0) Us[t * DVT + col] -= acc;
                __syncwarp();
            }
        }
        __syncthreads();
        // ---- O = Q~ S0 + Aq U
        {
            const int j = tid % DVT, t_ = tid / DVT;
#pragma unroll
            for (int m = 0; m < CMAX / RPT; ++m) {
                const int t = t_ + m * RPT;
                if (t < L) {
                    float acc = o1[m];
                    for (int s = 0; s <= t; ++s) acc = fmaf(Aqs[t * LDC + s], Us[s * DVT + j], acc);
                    stf(o + ((size_t)(c0 + t) * H + h) * dv + tile * DVT + j, acc);
                }
            }
        }
        // ---- S <- e^{b_last} S0 + G'^T U
        for (int e = tid; e < DK * DVT; e += NT) {
            const int i = e / DVT, j = e % DVT;
            float acc = GCs[i] * Ss[e];
            for (int s = 0; s < L; ++s) acc = fmaf(Gs[i * LDC + s], Us[s * DVT + j], acc);
            Ss[e] = acc;
        }
        __syncthreads();
    }

    if (a.S_out)
        for (int e = tid; e < DK * DVT; e += NT) {
            const int i = e / DVT, j = e % DVT;
            a.S_out[sbase + (size_t)i * dv + j] = Ss[e];
        }
    if (a.P_out && tile == 0) {
        if (a.iso) {
            if (tid == 0) a.P_out[sh] = P;
        } else if (tid < DK) {
            a.P_out[(size_t)sh * DK + tid] = P;
        }
    }
}

template <int DK, int DVT, typename Tin>
static cudaError_t launch_simt(const TokenArgs &a, int C, cudaStream_t st) {
    constexpr size_t smem = SimtSmem<DK, DVT>::bytes;
    auto kern = chunk_simt_kernel<DK, DVT, Tin>;
    KernelSetup ks;
    cudaError_t e = kernel_setup(reinterpret_cast<const void *>(kern), smem, NT, false, &ks);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.nseq * a.H * (a.dv / DVT));
    kern<<<grid, NT, smem, st>>>(a, C);
    return cudaGetLastError();
}

template <typename Tin>
static cudaError_t dispatch_simt(const TokenArgs &a, int C, cudaStream_t st) {
    const int dvt = a.dv >= 64 ? 64 : 32;
    switch (a.dk * 1000 + dvt) {
        case 32032: return launch_simt<32, 32, Tin>(a, C, st);
        case 32064: return launch_simt<32, 64, Tin>(a, C, st);
        case 64032: return launch_simt<64, 32, Tin>(a, C, st);
        case 64064: return launch_simt<64, 64, Tin>(a, C, st);
        case 128032: return launch_simt<128, 32, Tin>(a, C, st);
        case 128064: return launch_simt<128, 64, Tin>(a, C, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_chunk_simt(const TokenArgs &a, bool bf16_in, int C, cudaStream_t st) {
    if (a.nseq == 0 || a.H == 0) return cudaSuccess;
    if (C < 1 || C > CMAX) return cudaErrorInvalidValue;
    return bf16_in ? dispatch_simt<bf16>(a, C, st) : dispatch_simt<float>(a, C, st);
}

}  // namespace kdn
