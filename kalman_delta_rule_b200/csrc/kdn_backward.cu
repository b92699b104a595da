// Backward pass of the Diagonal KDN (the chunkwise regime is the training regime: KDA article,
// "chunkwise" section; the recurrence is the explainer's diagonal approximation, "对角近似").
//
// Gradients of  L = <o, d_o> + <S_T, dS_T> + <P_T, dP_T>  with respect to q, k, v, alpha, sigma,
// r, S0 and P0, by reverse-mode differentiation of the token recurrence
//     P^- = alpha^2 P + sigma,  den = r + sum_i P^-_i k_i^2,  g = P^- k / den,
//     W = diag(alpha) S,  u = v - W^T k,  S' = W + g u^T,  o = S'^T q,
//     P' = P^- / (1 + c P^-),  c = mu k^2 / r.
// Reverse step of one token (^ marks an adjoint; S^ arrives from the later tokens):
//     S^ += q d_o^T;  dq = S' d_o;  g^ = S^ u;  u^ = S^T g;  dv = u^;
//     W^ = S^ - k u^T;  k^ += -W u^;  alpha^ += rowsum(W^ o S);  S^ <- diag(alpha) W^;
//     den^ = -(g^ . g) / den;  P^-^ = g^ k / den + den^ k^2 + P'^ z^2   (z = 1 / (1 + c P^-));
//     c^ = -P'^ P'^2;  k^ += g^ P^- / den + 2 den^ P^- k + c^ 2 mu k / r;
//     r^ = den^ - sum_i c^_i mu k_i^2 / r^2;  sigma^ = P^-^;  alpha^ += 2 alpha P P^-^;  P^ = alpha^2 P^-^.
//
// Four launches:
//   tape  the uncertainty forward; writes P before each token, den and g per token: the
//         chunk-parallel gain scan (bf16, d_k = 128, diagonal), else one CTA per (sequence, head),
//         thread = key channel;
//   state (one CTA per (sequence, head, 16-column block of d_v), thread = key channel = row of S):
//         the memory forward with S checkpoints every 16 tokens and u of every token taped, then
//         the reverse sweep chunk by chunk: the chunk's inputs are staged in shared memory, the
//         chunk is re-stepped from its checkpoint (with the taped u, so without the cross-row
//         reduction) into shared-memory sub-checkpoints every 4 tokens, and the
//         state before each token is re-stepped from the nearest sub-checkpoint (never
//         reconstructed by dividing by alpha, which loses it when alpha is small).  Writes dv and
//         adds its column block's share of dq, g^, the S-part of k^ and the S-part of alpha^ into
//         them with fire-and-forget atomic adds (dq into the output, the others into three token
//         vectors cleared before the tape);
//   local (one warp per (token, head), every token in parallel): writes den^ and the parts of P^-^
//         and k^ that do not depend on the later tokens' P^;
//   prev  the one serial part of the uncertainty adjoint, P^ <- alpha^2 (P^-^local + P^ z^2), and
//         the outputs that need P^: dk, dalpha, dsigma, dr and dP0 -- for the diagonal variant a
//         chunk-parallel reverse affine scan, else one CTA per (sequence, head).
// Token rows are staged into shared memory with 16-byte asynchronous copies, a group of tokens at
// a time, so each group costs one memory round trip.  Everything is fp32 on the CUDA cores;
// inputs may be bf16 (widened exactly).
#include "kdn_common.cuh"
#include "kdn_launch.h"

namespace kdn {

namespace {
constexpr int DB = 16;    // d_v columns per state CTA
constexpr int CK = 16;    // tokens between the DRAM checkpoints of S (four CTAs per SM fit)
constexpr int NS = 4;     // tokens between the shared-memory sub-checkpoints
constexpr int GT = 32;    // tokens per group in the uncertainty kernels

struct BwdWs {
    float *Pprev, *g, *den, *dden, *utape, *ckpt, *part;
    long long ntok;
    int nblk;
};

__device__ __forceinline__ uint32_t smem_addr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
}
// n rows of row_bytes (a multiple of 16) from src + row * stride_bytes into dst, rows packed;
// every thread of the block takes a share of the 16-byte pieces
__device__ __forceinline__ void stage_rows(void *dst, const void *src, size_t stride_bytes, int n, int row_bytes) {
    const int per = row_bytes >> 4, nt = blockDim.x;
    for (int x = threadIdx.x; x < n * per; x += nt) {
        const int rr = x / per, c = x - rr * per;
        cp_async16(static_cast<char *>(dst) + (size_t)rr * row_bytes + c * 16,
                   static_cast<const char *>(src) + (size_t)rr * stride_bytes + c * 16);
    }
}
__device__ __forceinline__ float lds(const float *p) { return *p; }
// 16 consecutive staged values (16-byte aligned) as 8 column pairs, in 128-bit shared loads
__device__ __forceinline__ void lds16x2(const float *p, f32x2 (&x)[8]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const ulonglong2 v = reinterpret_cast<const ulonglong2 *>(p)[q];
        x[2 * q] = v.x;
        x[2 * q + 1] = v.y;
    }
}
__device__ __forceinline__ void lds16x2(const bf16 *p, f32x2 (&x)[8]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint4 v = reinterpret_cast<const uint4 *>(p)[q];
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int m = 0; m < 4; ++m)
            x[4 * q + m] = pk2(__uint_as_float(w[m] << 16), __uint_as_float(w[m] & 0xffff0000u));
    }
}
__device__ __forceinline__ float lds(const bf16 *p) {
    return __uint_as_float(((unsigned)*reinterpret_cast<const unsigned short *>(p)) << 16);
}

// Sums 16 per-lane values over the 32 lanes of a warp (each step exchanges half of the
// remaining values).  Lanes 2m and 2m+1 end with the total of value `which`.
__device__ __forceinline__ float reduce16(float (&v)[16], int lane, int &which) {
    const unsigned FULL = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 16;
        const float send = up ? v[i] : v[i + 8], keep = up ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 8;
        const float send = up ? v[i] : v[i + 4], keep = up ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 4;
        const float send = up ? v[i] : v[i + 2], keep = up ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, 4);
    }
    {
        const bool up = lane & 2;
        const float send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(FULL, send, 2);
    }
    v[0] += __shfl_xor_sync(FULL, v[0], 1);
    which = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
    return v[0];
}

}  // namespace

// ================================================================= tape
// dynamic shared memory: P^- and P^- k^2 [GT][dk]; den, r, 1/r [GT]; alpha, sigma, k rows of a
// group [GT][dk] (input type)
template <typename T>
__global__ void __launch_bounds__(128) bwd_tape_kernel(const BwdArgs b, const BwdWs w)
{
    extern __shared__ float smf[];
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    float *pm_s = smf, *x_s = pm_s + GT * dk, *den_s = x_s + GT * dk, *r_s = den_s + GT, *ir_s = r_s + GT;
    T *al_s = reinterpret_cast<T *>(ir_s + 2 * GT), *sg_s = al_s + GT * dk, *k_s = sg_s + GT * dk;
    const T *alpha = static_cast<const T *>(a.alpha), *sigma = static_cast<const T *>(a.sigma);
    const T *k = static_cast<const T *>(a.k), *r = static_cast<const T *>(a.r);
    const int chain = blockIdx.x, s = chain / H, h = chain % H;
    const int i = threadIdx.x, warp = i >> 5, lane = i & 31, nw = dk >> 5;
    const size_t rstride = (size_t)H * dk * sizeof(T);
    const int rbytes = dk * (int)sizeof(T);
    int t0, t1;
    seq_range(a, s, t0, t1);
    float P = a.P0 ? a.P0[(size_t)chain * dk + i] : 1.f;
    for (int tb = t0; tb < t1; tb += GT) {
        const int n = min(GT, t1 - tb);
        const size_t row0 = ((size_t)tb * H + h) * dk;
        stage_rows(al_s, alpha + row0, rstride, n, rbytes);
        stage_rows(sg_s, sigma + row0, rstride, n, rbytes);
        stage_rows(k_s, k + row0, rstride, n, rbytes);
        if (i < n) {
            const float rr = ldf(r + (size_t)(tb + i) * H + h);
            r_s[i] = rr;
            ir_s[i] = 1.f / rr;
        }
        cp_async_wait_all();
        __syncthreads();
        for (int tt = 0; tt < n; ++tt) {
            const float al = lds(al_s + tt * dk + i), kk = lds(k_s + tt * dk + i);
            w.Pprev[((size_t)(tb + tt) * H + h) * dk + i] = P;
            const float pm = fmaf(al * al, P, lds(sg_s + tt * dk + i));
            pm_s[tt * dk + i] = pm;
            x_s[tt * dk + i] = pm * kk * kk;
            P = pm / fmaf(a.mu * kk * kk * ir_s[tt], pm, 1.f);
        }
        __syncthreads();
        for (int tt = warp; tt < n; tt += nw) {
            float x = 0.f;
            for (int c = lane; c < dk; c += 32) x += x_s[tt * dk + c];
            x = warp_sum(x);
            if (lane == 0) {
                den_s[tt] = r_s[tt] + x;
                w.den[(size_t)(tb + tt) * H + h] = den_s[tt];
            }
        }
        __syncthreads();
        for (int tt = 0; tt < n; ++tt) {
            const size_t e = ((size_t)(tb + tt) * H + h) * dk + i;
            w.g[e] = pm_s[tt * dk + i] * lds(k_s + tt * dk + i) / den_s[tt];
        }
        __syncthreads();
    }
}

// ================================================================= state
// dynamic shared memory, per chunk of CK tokens: g rows [CK][dk] fp32; sub-checkpoints
// [CK/NS][DB/4][dk] float4; u per token [CK][DB]; reduction partials [4][DB]; u^ [DB]; then alpha, k, q
// rows [CK][dk] and the column block of v (forward) or d_o (reverse) [CK][DB] in the input type
template <typename T>
__global__ void __launch_bounds__(128, 4) bwd_state_kernel(const BwdArgs b, const BwdWs w)
{
    extern __shared__ float smf[];
    const TokenArgs &a = b.a;
    const int dk = a.dk, dv = a.dv, H = a.H;
    float *g_s = smf;
    float *sub = g_s + CK * dk;               // [CK/NS][DB/4][dk] float4 (thread i's 16 columns, conflict-free)
    float *us = sub + (CK / NS) * DB * dk;    // [CK][DB]
    float *red = us + CK * DB;                // [4][DB]
    float *uh = red + 4 * DB;                 // [DB]
    T *al_s = reinterpret_cast<T *>(uh + DB), *k_s = al_s + CK * dk, *q_s = k_s + CK * dk;
    T *v_s = q_s + CK * dk, *do_s = v_s;      // v in the forward, d_o in the reverse

    const T *q = static_cast<const T *>(a.q), *k = static_cast<const T *>(a.k), *v = static_cast<const T *>(a.v);
    const T *alpha = static_cast<const T *>(a.alpha), *d_o = static_cast<const T *>(b.d_o);
    const int chain = blockIdx.x / w.nblk, blk = blockIdx.x % w.nblk, col0 = blk * DB;
    const int s = chain / H, h = chain % H;
    const int i = threadIdx.x, warp = i >> 5, lane = i & 31, nw = dk >> 5;
    int t0, t1;
    seq_range(a, s, t0, t1);
    const long long slot0 = t0 / CK + s;      // checkpoint slots of this sequence: slot0 + chunk
    const size_t tokstride = (size_t)w.ntok * H * dk;
    auto ckpt_at = [&](int m) { return w.ckpt + (((size_t)(slot0 + m) * H + h) * w.nblk + blk) * DB * dk; };

    // the chunk's per-token inputs into shared memory (forward: v; reverse: q, d_o and the taped u)
    auto stage = [&](int c0, int L, bool rev) {
        __syncthreads();   // the previous chunk is done with the staged inputs
        const size_t row0 = ((size_t)c0 * H + h) * dk, vrow0 = ((size_t)c0 * H + h) * dv + col0;
        const size_t rstride = (size_t)H * dk * sizeof(T), vstride = (size_t)H * dv * sizeof(T);
        stage_rows(al_s, alpha + row0, rstride, L, dk * (int)sizeof(T));
        stage_rows(k_s, k + row0, rstride, L, dk * (int)sizeof(T));
        stage_rows(g_s, w.g + row0, (size_t)H * dk * 4, L, dk * 4);
        if (rev) {
            stage_rows(q_s, q + row0, rstride, L, dk * (int)sizeof(T));
            stage_rows(do_s, d_o + vrow0, vstride, L, DB * (int)sizeof(T));
            stage_rows(us, w.utape + vrow0, (size_t)H * dv * 4, L, DB * 4);
        } else {
            stage_rows(v_s, v + vrow0, vstride, L, DB * (int)sizeof(T));
        }
        cp_async_wait_all();
        __syncthreads();
    };
    // 16 consecutive shared floats (16-byte aligned) as 8 column pairs
    auto lds8x2 = [&](const float *p, f32x2 (&x)[8]) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const ulonglong2 v = reinterpret_cast<const ulonglong2 *>(p)[q];
            x[2 * q] = v.x;
            x[2 * q + 1] = v.y;
        }
    };
    // u_j = v_j - sum_i alpha_i k_i S_ij for staged token tt of the chunk at c0 -> the u tape and
    // dst[DB] (shared), then into u
    auto forward_u = [&](int c0, int tt, const f32x2 (&S)[8], float *dst, f32x2 (&u)[8]) {
        const float ak = lds(al_s + tt * dk + i) * lds(k_s + tt * dk + i);
        const f32x2 ak2 = pk2(ak, ak);
        float p[16];
#pragma unroll
        for (int jp = 0; jp < 8; ++jp) {
            const f32x2 x = mul2(ak2, S[jp]);
            p[2 * jp] = x2(x);
            p[2 * jp + 1] = y2(x);
        }
        int which;
        const float tot = reduce16(p, lane, which);
        if ((lane & 1) == 0) red[warp * DB + which] = tot;
        __syncthreads();
        if (i < DB) {
            float x = 0.f;
            for (int ww = 0; ww < nw; ++ww) x += red[ww * DB + i];
            dst[i] = lds(v_s + tt * DB + i) - x;
            w.utape[((size_t)(c0 + tt) * H + h) * dv + col0 + i] = dst[i];
        }
        __syncthreads();
        lds8x2(dst, u);
    };
    auto step = [&](int tt, f32x2 (&S)[8], const f32x2 (&u)[8]) {
        const float al = lds(al_s + tt * dk + i), gg = g_s[tt * dk + i];
        const f32x2 al2 = pk2(al, al), gg2 = pk2(gg, gg);
#pragma unroll
        for (int jp = 0; jp < 8; ++jp) S[jp] = fma2(gg2, u[jp], mul2(al2, S[jp]));
    };

    f32x2 S[8], Sh[8], u[8];
#pragma unroll
    for (int jp = 0; jp < 8; ++jp) {
        const size_t e = ((size_t)chain * dk + i) * dv + col0 + 2 * jp;
        S[jp] = a.S0 ? pk2(a.S0[e], a.S0[e + 1]) : pk2(0.f, 0.f);
    }

    // ---- forward: checkpoints every CK tokens
    const int nchk = (t1 - t0 + CK - 1) / CK;
    for (int m = 0; m < nchk; ++m) {
        const int c0 = t0 + m * CK, L = min(CK, t1 - c0);
        float *ck = ckpt_at(m);
#pragma unroll
        for (int jp = 0; jp < 8; ++jp) {
            ck[(2 * jp) * dk + i] = x2(S[jp]);
            ck[(2 * jp + 1) * dk + i] = y2(S[jp]);
        }
        stage(c0, L, false);
        for (int tt = 0; tt < L; ++tt) {
            forward_u(c0, tt, S, uh, u);
            step(tt, S, u);
        }
    }

    // ---- reverse, chunk by chunk
#pragma unroll
    for (int jp = 0; jp < 8; ++jp) {
        const size_t e = ((size_t)chain * dk + i) * dv + col0 + 2 * jp;
        Sh[jp] = b.dS_T ? pk2(b.dS_T[e], b.dS_T[e + 1]) : pk2(0.f, 0.f);
    }
    for (int m = nchk - 1; m >= 0; --m) {
        const int c0 = t0 + m * CK, L = min(CK, t1 - c0);
        const float *ck = ckpt_at(m);
#pragma unroll
        for (int jp = 0; jp < 8; ++jp) S[jp] = pk2(ck[(2 * jp) * dk + i], ck[(2 * jp + 1) * dk + i]);
        stage(c0, L, true);
        for (int tt = 0; tt < L; ++tt) {
            if (tt % NS == 0) {
                ulonglong2 *sb = reinterpret_cast<ulonglong2 *>(sub) + (size_t)(tt / NS) * 4 * dk + i;
#pragma unroll
                for (int q = 0; q < 4; ++q) sb[q * dk] = make_ulonglong2(S[2 * q], S[2 * q + 1]);
            }
            lds8x2(us + tt * DB, u);
            step(tt, S, u);
        }
        for (int js = (L - 1) / NS; js >= 0; --js) {
            for (int tt = min(L, js * NS + NS) - 1; tt >= js * NS; --tt) {
                const int t = c0 + tt;
                // state before token t, re-stepped from the sub-checkpoint
                f32x2 Sp[8], uu[8];
                {
                    const ulonglong2 *sb = reinterpret_cast<const ulonglong2 *>(sub) + (size_t)js * 4 * dk + i;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const ulonglong2 v = sb[q * dk];
                        Sp[2 * q] = v.x;
                        Sp[2 * q + 1] = v.y;
                    }
                }
                for (int oo = js * NS; oo < tt; ++oo) {
                    lds8x2(us + oo * DB, uu);
                    step(oo, Sp, uu);
                }
                const float al = lds(al_s + tt * dk + i), kk = lds(k_s + tt * dk + i), gg = g_s[tt * dk + i];
                const float qq = lds(q_s + tt * dk + i);
                const f32x2 al2 = pk2(al, al), gg2 = pk2(gg, gg), qq2 = pk2(qq, qq), nk2 = pk2(-kk, -kk);
                f32x2 dq2 = pk2(0.f, 0.f), gp2 = dq2;
                float p[16];
                f32x2 dov[8];
                lds8x2(us + tt * DB, uu);
                lds16x2(do_s + tt * DB, dov);
#pragma unroll
                for (int jp = 0; jp < 8; ++jp) {
                    const f32x2 do2 = dov[jp];
                    const f32x2 St = fma2(gg2, uu[jp], mul2(al2, Sp[jp]));
                    Sh[jp] = fma2(qq2, do2, Sh[jp]);
                    dq2 = fma2(St, do2, dq2);
                    gp2 = fma2(Sh[jp], uu[jp], gp2);
                    const f32x2 x = mul2(Sh[jp], gg2);
                    p[2 * jp] = x2(x);
                    p[2 * jp + 1] = y2(x);
                }
                int which;
                const float tot = reduce16(p, lane, which);
                if ((lane & 1) == 0) red[warp * DB + which] = tot;
                __syncthreads();
                if (i < DB) {
                    float x = 0.f;
                    for (int ww = 0; ww < nw; ++ww) x += red[ww * DB + i];
                    uh[i] = x;
                    b.dv[((size_t)t * H + h) * dv + col0 + i] = x;
                }
                __syncthreads();
                f32x2 kp2 = pk2(0.f, 0.f), ap2 = kp2;
                lds8x2(uh, uu);
#pragma unroll
                for (int jp = 0; jp < 8; ++jp) {
                    const f32x2 Wh = fma2(nk2, uu[jp], Sh[jp]);
                    kp2 = fma2(mul2(al2, Sp[jp]), uu[jp], kp2);
                    ap2 = fma2(Wh, Sp[jp], ap2);
                    Sh[jp] = mul2(al2, Wh);
                }
                const size_t e = ((size_t)t * H + h) * dk + i;
                atomicAdd(b.dq + e, x2(dq2) + y2(dq2));
                atomicAdd(w.part + e, x2(gp2) + y2(gp2));
                atomicAdd(w.part + tokstride + e, -(x2(kp2) + y2(kp2)));
                atomicAdd(w.part + 2 * tokstride + e, x2(ap2) + y2(ap2));
            }
        }
    }
    if (b.dS0) {
#pragma unroll
        for (int jp = 0; jp < 8; ++jp) {
            const size_t e = ((size_t)chain * dk + i) * dv + col0 + 2 * jp;
            b.dS0[e] = x2(Sh[jp]);
            b.dS0[e + 1] = y2(Sh[jp]);
        }
    }
}

// ================================================================= local
// One warp per (token, head), lanes over the key channels.  Writes den^ = -(g^ . g) / den and
// overwrites the sums of g^ and k^_S with
//   A  = g^ k / den + den^ k^2                      (P^-^ without the later tokens' part)
//   Kl = k^_S + g^ P^- / den + 2 den^ P^- k         (k^ without the uncertainty-update part)
template <typename T>
__global__ void __launch_bounds__(256) bwd_local_kernel(const BwdArgs b, const BwdWs w)
{
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    const long long th = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (th >= w.ntok * H) return;
    const T *alpha = static_cast<const T *>(a.alpha), *sigma = static_cast<const T *>(a.sigma);
    const T *k = static_cast<const T *>(a.k);
    const size_t tokstride = (size_t)w.ntok * H * dk;
    const float dn = w.den[th];
    float gh[4], kS[4], xg = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = lane + 32 * m;
        gh[m] = kS[m] = 0.f;
        if (c < dk) {
            const size_t e = (size_t)th * dk + c;
            gh[m] = w.part[e];
            kS[m] = w.part[tokstride + e];
            xg = fmaf(gh[m], w.g[e], xg);
        }
    }
    const float dd = -warp_sum(xg) / dn;
    if (lane == 0) w.dden[th] = dd;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = lane + 32 * m;
        if (c < dk) {
            const size_t e = (size_t)th * dk + c;
            const float al = ldf(alpha + e), kk = ldf(k + e);
            const float pm = fmaf(al * al, w.Pprev[e], ldf(sigma + e));
            w.part[e] = gh[m] * kk / dn + dd * kk * kk;
            w.part[tokstride + e] = kS[m] + gh[m] * pm / dn + 2.f * dd * pm * kk;
        }
    }
}

// ================================================================= prev
// dynamic shared memory, per group of GT tokens: A, Kl, alpha^_S, P before the token [GT][dk]
// fp32; r-terms [GT][dk]; 1/r, den^ [GT]; alpha, sigma, k rows [GT][dk] in the input type
template <typename T>
__global__ void __launch_bounds__(128) bwd_prev_kernel(const BwdArgs b, const BwdWs w)
{
    extern __shared__ float smf[];
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    float *A_s = smf, *K_s = A_s + GT * dk, *aS_s = K_s + GT * dk, *pp_s = aS_s + GT * dk, *x_s = pp_s + GT * dk;
    float *r_s = x_s + GT * dk, *dd_s = r_s + GT;
    T *al_s = reinterpret_cast<T *>(dd_s + GT), *sg_s = al_s + GT * dk, *k_s = sg_s + GT * dk;
    const T *alpha = static_cast<const T *>(a.alpha), *sigma = static_cast<const T *>(a.sigma);
    const T *k = static_cast<const T *>(a.k), *r = static_cast<const T *>(a.r);
    const int chain = blockIdx.x, s = chain / H, h = chain % H;
    const int i = threadIdx.x, warp = i >> 5, lane = i & 31, nw = dk >> 5;
    const float mu = a.mu;
    const size_t tokstride = (size_t)w.ntok * H * dk;
    const size_t rstride = (size_t)H * dk * sizeof(T), fstride = (size_t)H * dk * 4;
    int t0, t1;
    seq_range(a, s, t0, t1);
    float Ph = b.dP_T ? b.dP_T[(size_t)chain * dk + i] : 0.f;
    for (int te = t1; te > t0; te -= GT) {
        const int tb = max(t0, te - GT), n = te - tb;
        const size_t row0 = ((size_t)tb * H + h) * dk;
        stage_rows(A_s, w.part + row0, fstride, n, dk * 4);
        stage_rows(K_s, w.part + tokstride + row0, fstride, n, dk * 4);
        stage_rows(aS_s, w.part + 2 * tokstride + row0, fstride, n, dk * 4);
        stage_rows(pp_s, w.Pprev + row0, fstride, n, dk * 4);
        stage_rows(al_s, alpha + row0, rstride, n, dk * (int)sizeof(T));
        stage_rows(sg_s, sigma + row0, rstride, n, dk * (int)sizeof(T));
        stage_rows(k_s, k + row0, rstride, n, dk * (int)sizeof(T));
        if (i < n) {
            r_s[i] = 1.f / ldf(r + (size_t)(tb + i) * H + h);   // 1/r
            dd_s[i] = w.dden[(size_t)(tb + i) * H + h];
        }
        cp_async_wait_all();
        __syncthreads();
        for (int tt = n - 1; tt >= 0; --tt) {
            const size_t e = ((size_t)(tb + tt) * H + h) * dk + i;
            const int o = tt * dk + i;
            const float al = lds(al_s + o), kk = lds(k_s + o), ir = r_s[tt], Pp = pp_s[o];
            const float pm = fmaf(al * al, Pp, lds(sg_s + o));
            const float mk = mu * kk * ir;                 // mu k / r
            const float z = 1.f / fmaf(mk * kk, pm, 1.f);
            const float Pt = pm * z;
            const float pmh = A_s[o] + Ph * z * z;
            const float ch = -Ph * Pt * Pt;
            b.dk[e] = K_s[o] + ch * 2.f * mk;
            x_s[o] = -ch * mk * kk * ir;
            b.dsigma[e] = pmh;
            b.dalpha[e] = aS_s[o] + 2.f * al * Pp * pmh;
            Ph = al * al * pmh;
        }
        __syncthreads();
        for (int tt = warp; tt < n; tt += nw) {
            float x = 0.f;
            for (int c = lane; c < dk; c += 32) x += x_s[tt * dk + c];
            x = warp_sum(x);
            if (lane == 0) b.dr[(size_t)(tb + tt) * H + h] = dd_s[tt] + x;
        }
        __syncthreads();
    }
    if (b.dP0) b.dP0[(size_t)chain * dk + i] = Ph;
}

// ================================================================= prev, chunk-parallel
// The serial part of the uncertainty adjoint, P^ <- alpha^2 (P^-^local + P^ z^2), is affine in P^
// per key channel (P^_before = a P^_after + b, a = alpha^2 z^2, b = alpha^2 P^-^local), so it is
// scanned like the forward uncertainty, over chunks of PC tokens counted from the sequence end:
// a unit (chunk, chain) composes its chunk's maps (thread = key channel), publishes the
// aggregate as tagged 64-bit words, walks over the later chunks' words to the last published
// chunk-start value (decoupled look-back, bounded waits), publishes its own, and walks its
// tokens again with the incoming P^ to write dk, dsigma, dalpha and dr.  Tickets go out
// chunk-major in that order, so every unit a look-back waits for was taken earlier by a running
// CTA.  A sequence without tokens gets one empty unit, which passes dP_T through to dP0.
namespace {
constexpr int PC = 64;
constexpr int PSEG = 4;   // segments of PC / PSEG tokens per chunk
enum : unsigned { TAG_AGG = 1, TAG_INCL = 2 };
struct PrevWs {
    unsigned *counter;
    unsigned long long *words;   // per unit [3][dk]: aggregate (a, b), chunk-start P^
    long long nchunks_max;
};
__device__ __forceinline__ unsigned long long tagged(float x, unsigned tag) {
    return ((unsigned long long)tag << 32) | __float_as_uint(x);
}
__device__ __forceinline__ unsigned tag_of(unsigned long long v) { return (unsigned)(v >> 32); }
__device__ __forceinline__ float value_of(unsigned long long v) { return __uint_as_float((unsigned)v); }
__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
struct PrevUnit { long long u; int j, chain, h, lo, hi, nch; };
}  // namespace

// dynamic shared memory: dr terms [PC][dk]; 1/r, den^ [PC]; segment maps and incoming P^
// [PSEG][dk] float2; the claimed unit.  Thread = key channel x segment of PC / PSEG tokens
// (segment 0 holds the latest tokens).
template <typename T>
__global__ void __launch_bounds__(512) bwd_prev_scan_kernel(const BwdArgs b, const BwdWs w, const PrevWs pw)
{
    extern __shared__ float smf[];
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    float *x_s = smf, *ir_s = x_s + PC * dk, *dd_s = ir_s + PC;
    float2 *seg_s = reinterpret_cast<float2 *>(dd_s + PC);       // [PSEG][dk]: (a, b), then (P^_in, -)
    PrevUnit *claimed = reinterpret_cast<PrevUnit *>(seg_s + PSEG * dk);
    const T *alpha = static_cast<const T *>(a.alpha), *sigma = static_cast<const T *>(a.sigma);
    const T *k = static_cast<const T *>(a.k), *r = static_cast<const T *>(a.r);
    const int tid = threadIdx.x, nt = blockDim.x, warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
    const int i = tid % dk, sg = tid / dk;
    const float mu = a.mu;
    const size_t tokstride = (size_t)w.ntok * H * dk;
    const int nchains = a.nseq * H;
    const long long units = pw.nchunks_max * nchains;
    for (;;) {
        if (tid == 0) {
            PrevUnit n;
            for (;;) {
                n.u = (long long)atomicAdd(pw.counter, 1u);
                if (n.u >= units) break;
                n.j = (int)(n.u / nchains);
                n.chain = (int)(n.u - (long long)n.j * nchains);
                const int s = n.chain / H;
                n.h = n.chain - s * H;
                int t0, t1;
                seq_range(a, s, t0, t1);
                n.nch = (t1 - t0 + PC - 1) / PC;
                // a sequence longer than max_seqlen has chunks past the work list
                if (n.j == 0 && n.nch > pw.nchunks_max) raise_error(a.err, ERR_ARG);
                if (n.j < n.nch || n.j == 0) {
                    n.hi = t1 - n.j * PC;
                    n.lo = max(t0, n.hi - PC);
                    break;
                }
            }
            *claimed = n;
        }
        __syncthreads();
        const PrevUnit cu = *claimed;
        if (cu.u >= units) break;
        const int L = cu.hi - cu.lo;
        for (int tt = tid; tt < L; tt += nt) {
            const size_t th = (size_t)(cu.lo + tt) * H + cu.h;
            ir_s[tt] = 1.f / ldf(r + th);
            dd_s[tt] = w.dden[th];
        }
        __syncthreads();
        // this thread's tokens (chunk offsets), walked from the latest
        const int seg_hi = L - sg * (PC / PSEG), seg_lo = max(0, seg_hi - PC / PSEG);

        // pass 1: the segment's composite map, P^ at its start = ra P^ at its end + rb
        float ra = 1.f, rb = 0.f;
#pragma unroll 4
        for (int tt = seg_hi - 1; tt >= seg_lo; --tt) {
            const size_t e = ((size_t)(cu.lo + tt) * H + cu.h) * dk + i;
            const float al = ldf(alpha + e), kk = ldf(k + e);
            const float pm = fmaf(al * al, ldf(w.Pprev + e), ldf(sigma + e));
            const float mk = mu * kk * ir_s[tt];
            const float z = 1.f / fmaf(mk * kk, pm, 1.f);
            const float aa = al * al, at = aa * z * z;
            rb = fmaf(at, rb, aa * ldf(w.part + e));
            ra *= at;
        }
        seg_s[sg * dk + i] = make_float2(ra, rb);
        __syncthreads();

        // segment-0 threads (one per key channel): the chunk's map, its publication, the
        // incoming P^ at the chunk end (dP_T for the last chunk, else the later chunks' words),
        // and the incoming P^ of every segment.  The last chunk publishes no aggregate, so every
        // walk ends at a start value.
        if (sg == 0) {
            float ca = 1.f, cb = 0.f;
#pragma unroll
            for (int q = 0; q < PSEG; ++q) {
                const float2 m = seg_s[q * dk + i];
                cb = fmaf(m.x, cb, m.y);
                ca *= m.x;
            }
            unsigned long long *wd = pw.words + (size_t)cu.u * 3 * dk + i;
            if (cu.j > 0 && cu.j + 1 < cu.nch) {
                st_relaxed(wd, tagged(ca, TAG_AGG));
                st_relaxed(wd + dk, tagged(cb, TAG_AGG));
            }
            float ph_end = 0.f;
            if (cu.j == 0) {
                ph_end = b.dP_T ? b.dP_T[(size_t)cu.chain * dk + i] : 0.f;
            } else {
                // walk to the nearest later chunk whose start value is published, then back through
                // the aggregates of the chunks in between, each applied as its owner applies it:
                // the result does not depend on which words were published when (bit-reproducible)
                auto words_of = [&](int jj) { return pw.words + ((size_t)jj * nchains + cu.chain) * 3 * dk + i; };
                bool timed_out = false;
                int jj = cu.j - 1;
                float x = 0.f;
                for (;; --jj) {
                    const unsigned long long *dj = words_of(jj);
                    unsigned long long w0 = 0ull, w1 = 0ull, w2 = ld_relaxed(dj + 2 * dk);
                    const long long ts = clock64();
                    while (tag_of(w2) != TAG_INCL) {
                        w0 = ld_relaxed(dj);
                        w1 = ld_relaxed(dj + dk);
                        if (jj > 0 && tag_of(w0) == TAG_AGG && tag_of(w1) == TAG_AGG) break;
                        // give up after ~1 s, or at once when another wait already gave up
                        if (clock64() - ts > 2000000000ll || (a.err && (*(volatile unsigned *)a.err & ERR_TIMEOUT))) {
                            timed_out = true;
                            break;
                        }
                        __nanosleep(32);
                        w2 = ld_relaxed(dj + 2 * dk);
                    }
                    if (timed_out) {
                        raise_error(a.err, ERR_TIMEOUT);
                        break;
                    }
                    if (tag_of(w2) == TAG_INCL || jj == 0) {
                        x = value_of(w2);
                        break;
                    }
                }
                if (!timed_out) {
                    for (int k2 = jj + 1; k2 < cu.j; ++k2) {   // aggregates seen published by the walk
                        const unsigned long long *dq = words_of(k2);
                        x = fmaf(value_of(ld_relaxed(dq)), x, value_of(ld_relaxed(dq + dk)));
                    }
                }
                ph_end = timed_out ? 0.f : x;
            }
            st_relaxed(wd + 2 * dk, tagged(fmaf(ca, ph_end, cb), TAG_INCL));
            float in = ph_end;
#pragma unroll
            for (int q = 0; q < PSEG; ++q) {
                const float2 m = seg_s[q * dk + i];
                seg_s[q * dk + i] = make_float2(in, 0.f);
                in = fmaf(m.x, in, m.y);
            }
        }
        __syncthreads();

        // pass 2: the token adjoints with the incoming P^ (the serial kernel's arithmetic)
        float ph = seg_s[sg * dk + i].x;
#pragma unroll 4
        for (int tt = seg_hi - 1; tt >= seg_lo; --tt) {
            const size_t e = ((size_t)(cu.lo + tt) * H + cu.h) * dk + i;
            const float al = ldf(alpha + e), kk = ldf(k + e), ir = ir_s[tt], Pp = ldf(w.Pprev + e);
            const float pm = fmaf(al * al, Pp, ldf(sigma + e));
            const float mk = mu * kk * ir;
            const float z = 1.f / fmaf(mk * kk, pm, 1.f);
            const float Pt = pm * z;
            const float pmh = ldf(w.part + e) + ph * z * z;
            const float ch = -ph * Pt * Pt;
            b.dk[e] = ldf(w.part + tokstride + e) + ch * 2.f * mk;
            x_s[tt * dk + i] = -ch * mk * kk * ir;
            b.dsigma[e] = pmh;
            b.dalpha[e] = ldf(w.part + 2 * tokstride + e) + 2.f * al * Pp * pmh;
            ph = al * al * pmh;
        }
        if (sg == PSEG - 1 && cu.j >= cu.nch - 1 && b.dP0) b.dP0[(size_t)cu.chain * dk + i] = ph;
        __syncthreads();
        for (int tt = warp; tt < L; tt += nw) {
            float x = 0.f;
            for (int c = lane; c < dk; c += 32) x += x_s[tt * dk + c];
            x = warp_sum(x);
            if (lane == 0) b.dr[(size_t)(cu.lo + tt) * H + cu.h] = dd_s[tt] + x;
        }
        __syncthreads();   // the staged values and the claimed unit are free for the next unit
    }
}

// ================================================================= isotropic variant
// One uncertainty p per head (explainer "各向同性近似"): p^- = a p + s with a = mean(alpha^2),
// s = mean(sigma); g = p^- k / den, den = r + p^- K2, K2 = |k|^2; p' = p^- z, z = 1/(1 + c p^-),
// c = mu K2 / (d_k r).  Adjoint of one token (p^ arrives from the later tokens):
//     p^-^ = (g^.k - (g^.g) K2) / den + p^ z^2;   c^ = -p^ p'^2;   p^ <- a p^-^
//     k^ = k^_S + g^ p^- / den - 2 (g^.g) p^- k / den + c^ 2 mu k / (d_k r)
//     r^ = -(g^.g) / den - c^ mu K2 / (d_k r^2);  sigma^ = p^-^ / d_k;  alpha^ = alpha^_S + 2 alpha p p^-^ / d_k
// The memory state pass is the diagonal one (it only needs g and alpha).  Per-token scalars
// live in the first 8 floats of the (token, head) row of the P tape:
//     [0] p before the token, [1] a, [2] mean sigma (forward), then p^-^ (adjoint), [3] K2,
//     [4] the local part of p^-^, [5] the local part of r^, [6] p^-, [7] c^ (adjoint).
namespace {
constexpr int SC_P = 0, SC_A = 1, SC_K2 = 3, SC_AL = 4, SC_RL = 5, SC_PM = 6;
}

// The isotropic uncertainty forward in three launches, with the expressions of a serial walk:
// the channel sums of every (token, head) (one warp each: mean alpha^2, mean sigma and |k|^2 into
// the token's scalar row); the scalar recursion of each head (one warp per (sequence, head): the
// lanes load 32 tokens' sums at a time and lane 0 carries p through them), which writes p before
// the token, p^- and den; then g = p^- k / den for every channel (one warp per (token, head)).
namespace {
constexpr int SC_S = 2;   // mean sigma of the token, until SC_PMH takes the slot in the adjoint
}

template <typename T>
__global__ void __launch_bounds__(256) bwd_tape_iso_sums_kernel(const BwdArgs b, const BwdWs w)
{
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    const long long th = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (th >= w.ntok * H) return;
    const T *alpha = static_cast<const T *>(a.alpha), *sigma = static_cast<const T *>(a.sigma);
    const T *k = static_cast<const T *>(a.k);
    const float inv_dk = 1.f / dk;
    float xa = 0.f, xs = 0.f, xk = 0.f;
    for (int c = lane; c < dk; c += 32) {
        const size_t e = (size_t)th * dk + c;
        const float al = ldf(alpha + e), kk = ldf(k + e);
        xa = fmaf(al, al, xa);
        xs += ldf(sigma + e);
        xk = fmaf(kk, kk, xk);
    }
    xa = warp_sum(xa); xs = warp_sum(xs); xk = warp_sum(xk);
    if (lane == 0) {
        float *sc = w.Pprev + (size_t)th * dk;
        sc[SC_A] = xa * inv_dk;
        sc[SC_S] = xs * inv_dk;
        sc[SC_K2] = xk;
    }
}

template <typename T>
__global__ void __launch_bounds__(32) bwd_tape_iso_chain_kernel(const BwdArgs b, const BwdWs w)
{
    __shared__ float aa_s[32], s_s[32], k2_s[32], r_s[32], p_s[32];
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    const T *r = static_cast<const T *>(a.r);
    const int chain = blockIdx.x, s = chain / H, h = chain % H;
    const int lane = threadIdx.x;
    const float inv_dk = 1.f / dk;
    int t0, t1;
    seq_range(a, s, t0, t1);
    float p = a.P0 ? a.P0[chain] : 1.f;   // lane 0's running uncertainty
    for (int tb = t0; tb < t1; tb += 32) {
        const int n = min(32, t1 - tb);
        if (lane < n) {
            const size_t th = (size_t)(tb + lane) * H + h;
            const float *sc = w.Pprev + th * dk;
            aa_s[lane] = sc[SC_A];
            s_s[lane] = sc[SC_S];
            k2_s[lane] = sc[SC_K2];
            r_s[lane] = ldf(r + th);
        }
        __syncwarp();
        if (lane == 0) {
            for (int tt = 0; tt < n; ++tt) {
                p_s[tt] = p;
                const float pm = fmaf(aa_s[tt], p, s_s[tt]);
                p = pm / fmaf(a.mu * k2_s[tt] * inv_dk / r_s[tt], pm, 1.f);
            }
        }
        __syncwarp();
        if (lane < n) {
            const size_t th = (size_t)(tb + lane) * H + h;
            float *sc = w.Pprev + th * dk;
            const float pm = fmaf(aa_s[lane], p_s[lane], s_s[lane]);
            sc[SC_P] = p_s[lane];
            sc[SC_PM] = pm;
            w.den[th] = fmaf(pm, k2_s[lane], r_s[lane]);
        }
        __syncwarp();
    }
}

template <typename T>
__global__ void __launch_bounds__(256) bwd_tape_iso_gain_kernel(const BwdArgs b, const BwdWs w)
{
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    const long long th = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (th >= w.ntok * H) return;
    const T *k = static_cast<const T *>(a.k);
    const float pm = w.Pprev[(size_t)th * dk + SC_PM], den = w.den[th];
    for (int c = lane; c < dk; c += 32) {
        const size_t e = (size_t)th * dk + c;
        w.g[e] = pm * ldf(k + e) / den;
    }
}

// one warp per (token, head): the local parts of k^ (over the k^_S sum), p^-^ and r^ (tape scalars)
template <typename T>
__global__ void __launch_bounds__(256) bwd_local_iso_kernel(const BwdArgs b, const BwdWs w)
{
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    const long long th = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (th >= w.ntok * H) return;
    const T *k = static_cast<const T *>(a.k);
    const size_t tokstride = (size_t)w.ntok * H * dk;
    float *sc = w.Pprev + (size_t)th * dk;
    const float dn = w.den[th], pm = sc[SC_PM], K2 = sc[SC_K2];
    float gh[4], kS[4], kk[4], gk = 0.f, gg = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = lane + 32 * m;
        gh[m] = kS[m] = kk[m] = 0.f;
        if (c < dk) {
            const size_t e = (size_t)th * dk + c;
            gh[m] = w.part[e];
            kS[m] = w.part[tokstride + e];
            kk[m] = ldf(k + e);
            gk = fmaf(gh[m], kk[m], gk);
            gg = fmaf(gh[m], w.g[e], gg);
        }
    }
    gk = warp_sum(gk);
    gg = warp_sum(gg);
    if (lane == 0) {
        sc[SC_AL] = (gk - gg * K2) / dn;
        sc[SC_RL] = -gg / dn;
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = lane + 32 * m;
        if (c < dk) {
            w.part[tokstride + (size_t)th * dk + c] = kS[m] + gh[m] * pm / dn - 2.f * gg * pm * kk[m] / dn;
        }
    }
}

// The isotropic uncertainty adjoint in two launches.  Its serial part is a scalar per head, so
// one warp per (sequence, head) walks it: the lanes form the per-token terms of 32 tokens at a
// time (z, the head's a, the local part of p^-^), lane 0 carries p^ through them (two dependent
// operations per token), and the lanes then write p^-^ and c^ of their tokens (slots SC_PMH,
// SC_CH of the token's scalar row) and dr.  A second launch, one warp per (token, head), forms
// dk, dsigma and dalpha of every channel.  The expressions are the one-CTA-per-head kernel's.
namespace {
constexpr int SC_PMH = 2, SC_CH = 7;
}

template <typename T>
__global__ void __launch_bounds__(32) bwd_prev_iso_chain_kernel(const BwdArgs b, const BwdWs w)
{
    __shared__ float z_s[32], aa_s[32], al_s[32], ph_s[32];
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    const T *r = static_cast<const T *>(a.r);
    const int chain = blockIdx.x, s = chain / H, h = chain % H;
    const int lane = threadIdx.x;
    const float mu = a.mu, inv_dk = 1.f / dk;
    int t0, t1;
    seq_range(a, s, t0, t1);
    float ph = b.dP_T ? b.dP_T[chain] : 0.f;   // lane 0's running p^
    for (int te = t1; te > t0; te -= 32) {
        const int tb = max(t0, te - 32), n = te - tb;
        float pt = 0.f, mk = 0.f, K2 = 0.f, ir = 0.f;
        float *sc = nullptr;
        if (lane < n) {
            const size_t th = (size_t)(tb + lane) * H + h;
            sc = w.Pprev + th * dk;
            const float aa = sc[SC_A], pm = sc[SC_PM];
            K2 = sc[SC_K2];
            ir = 1.f / ldf(r + th);
            mk = mu * inv_dk * ir;
            const float z = 1.f / fmaf(mk * K2, pm, 1.f);
            pt = pm * z;
            z_s[lane] = z;
            aa_s[lane] = aa;
            al_s[lane] = sc[SC_AL];
        }
        __syncwarp();
        if (lane == 0) {
            for (int tt = n - 1; tt >= 0; --tt) {
                ph_s[tt] = ph;
                const float z = z_s[tt];
                const float pmh = al_s[tt] + ph * z * z;
                ph = aa_s[tt] * pmh;
            }
        }
        __syncwarp();
        if (lane < n) {
            const float p_in = ph_s[lane], z = z_s[lane];
            const float pmh = al_s[lane] + p_in * z * z;
            const float ch = -p_in * pt * pt;
            sc[SC_PMH] = pmh;
            sc[SC_CH] = ch;
            b.dr[(size_t)(tb + lane) * H + h] = sc[SC_RL] - ch * mk * K2 * ir;
        }
        __syncwarp();
    }
    if (b.dP0 && lane == 0) b.dP0[chain] = ph;
}

template <typename T>
__global__ void __launch_bounds__(256) bwd_prev_iso_out_kernel(const BwdArgs b, const BwdWs w)
{
    const TokenArgs &a = b.a;
    const int dk = a.dk, H = a.H;
    const long long th = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (th >= w.ntok * H) return;
    const T *alpha = static_cast<const T *>(a.alpha), *k = static_cast<const T *>(a.k);
    const T *r = static_cast<const T *>(a.r);
    const size_t tokstride = (size_t)w.ntok * H * dk;
    const float *sc = w.Pprev + (size_t)th * dk;
    const float mu = a.mu, inv_dk = 1.f / dk;
    const float pp = sc[SC_P], pmh = sc[SC_PMH], ch = sc[SC_CH];
    const float ir = 1.f / ldf(r + th);
    const float mk = mu * inv_dk * ir;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = lane + 32 * m;
        if (c < dk) {
            const size_t e = (size_t)th * dk + c;
            const float al = ldf(alpha + e), kk = ldf(k + e);
            b.dk[e] = w.part[tokstride + e] + ch * 2.f * mk * kk;
            b.dsigma[e] = pmh * inv_dk;
            b.dalpha[e] = w.part[2 * tokstride + e] + 2.f * al * pp * pmh * inv_dk;
        }
    }
}

// ================================================================= host
namespace {
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
long long ckpt_slots(long long ntok, int nseq) { return ntok / CK + nseq + 1; }
}  // namespace

size_t backward_workspace_bytes(long long ntok, int nseq, int H, int dk, int dv) {
    const size_t th = (size_t)ntok * H;
    size_t n = 0;
    n += align256(th * dk * 4);                                     // P before each token
    n += align256(th * dk * 4);                                     // g
    n += align256(th * 4);                                          // den
    n += align256(th * 4);                                          // den^
    n += align256(th * dv * 4);                                     // u of every token
    n += align256((size_t)ckpt_slots(ntok, nseq) * H * dk * dv * 4);   // S checkpoints
    n += align256((size_t)3 * th * dk * 4);                         // sums of g^, k^_S, alpha^_S
    return n;
}

template <typename T>
static cudaError_t launch_local(const BwdArgs &b, const BwdWs &w, cudaStream_t st) {
    const long long rows = w.ntok * b.a.H;
    if (rows == 0) return cudaSuccess;
    if (b.a.iso)
        bwd_local_iso_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(b, w);
    else
        bwd_local_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(b, w);
    return cudaGetLastError();
}

// the kernel's dynamic shared-memory limit, set once per device and context
static cudaError_t set_smem(const void *kern, size_t smem) {
    KernelSetup ks;
    return kernel_setup(kern, smem, 128, true, &ks);
}

// The uncertainty forward as the chunk-parallel gain scan (bf16, d_k = 128, diagonal): P before
// each token, g and den, with its look-back words in the checkpoint region (written by the
// state pass only later).
static cudaError_t launch_tape_scan(const BwdArgs &b, const BwdWs &w, int nchunks_max, cudaStream_t st) {
    const TokenArgs &a = b.a;
    ScanArgs sa{};
    sa.k = a.k; sa.alpha = a.alpha; sa.sigma = a.sigma; sa.r = a.r; sa.P0 = a.P0;
    sa.g = w.g; sa.P_prev = w.Pprev; sa.den = w.den;
    sa.cu = a.cu; sa.T = a.T; sa.nseq = a.nseq; sa.H = a.H; sa.dk = a.dk; sa.mu = a.mu;
    sa.nchunks_max = nchunks_max; sa.nchains = a.nseq * a.H; sa.err = a.err;
    return launch_gain_scan_tma(sa, w.ntok, w.ckpt, st);
}

// bytes of the chunk-parallel adjoint's ticket counter and look-back words
static size_t prev_scan_bytes(long long nchains, long long nchunks_max, int dk) {
    return 256 + (size_t)nchains * (size_t)(nchunks_max > 0 ? nchunks_max : 1) * 3 * dk * 8;
}

// The serial uncertainty adjoint as the chunk-parallel scan, its words in the checkpoint
// region (the state pass is done with it)
template <typename T>
static cudaError_t launch_prev_scan(const BwdArgs &b, const BwdWs &w, long long nchunks_max, cudaStream_t st) {
    const int dk = b.a.dk;
    const long long nchains = (long long)b.a.nseq * b.a.H;
    PrevWs pw;
    pw.counter = reinterpret_cast<unsigned *>(w.ckpt);
    pw.words = reinterpret_cast<unsigned long long *>(reinterpret_cast<uint8_t *>(w.ckpt) + 256);
    pw.nchunks_max = nchunks_max > 0 ? nchunks_max : 1;
    cudaError_t e = cudaMemsetAsync(w.ckpt, 0, prev_scan_bytes(nchains, nchunks_max, dk), st);
    if (e != cudaSuccess) return e;
    const size_t smem = ((size_t)PC * dk + 2 * PC) * sizeof(float) + (size_t)PSEG * dk * sizeof(float2) + sizeof(PrevUnit);
    const int nt = dk * PSEG;
    KernelSetup ks;
    e = kernel_setup(reinterpret_cast<const void *>(bwd_prev_scan_kernel<T>), smem, nt, true, &ks);
    if (e != cudaSuccess) return e;
    // persistent CTAs; units go out by ticket to resident CTAs only
    long long grid = (long long)ks.sms * (ks.blocks_per_sm > 0 ? ks.blocks_per_sm : 1);
    const long long units = pw.nchunks_max * nchains;
    if (grid > units) grid = units;
    bwd_prev_scan_kernel<T><<<(unsigned)grid, nt, smem, st>>>(b, w, pw);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_bwd_typed(const BwdArgs &b, const BwdWs &w, bool tape_scan, bool prev_scan,
                                    int nchunks_max, cudaStream_t st) {
    const int chains = b.a.nseq * b.a.H, dk = b.a.dk;
    // the state pass adds its column blocks' shares into dq and the three sums
    const size_t thd = (size_t)w.ntok * b.a.H * dk * 4;
    cudaError_t e = cudaMemsetAsync(b.dq, 0, thd, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(w.part, 0, 3 * thd, st);
    if (e != cudaSuccess) return e;
    if (tape_scan) {
        e = launch_tape_scan(b, w, nchunks_max, st);
        if (e != cudaSuccess) return e;
    } else if (b.a.iso) {
        const long long rows = w.ntok * b.a.H;
        if (rows > 0) {
            bwd_tape_iso_sums_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(b, w);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            bwd_tape_iso_chain_kernel<T><<<chains, 32, 0, st>>>(b, w);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            bwd_tape_iso_gain_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(b, w);
        }
    } else {
        const size_t tsm = ((size_t)2 * GT * dk + 4 * GT) * sizeof(float) + (size_t)3 * GT * dk * sizeof(T);
        e = set_smem(reinterpret_cast<const void *>(bwd_tape_kernel<T>), tsm);
        if (e != cudaSuccess) return e;
        bwd_tape_kernel<T><<<chains, dk, tsm, st>>>(b, w);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t ssm = ((size_t)CK * dk + (CK / NS) * DB * dk + CK * DB + 4 * DB + DB) * sizeof(float) +
                       ((size_t)3 * CK * dk + CK * DB) * sizeof(T);
    e = set_smem(reinterpret_cast<const void *>(bwd_state_kernel<T>), ssm);
    if (e != cudaSuccess) return e;
    bwd_state_kernel<T><<<(unsigned)chains * w.nblk, dk, ssm, st>>>(b, w);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_local<T>(b, w, st);
    if (e != cudaSuccess) return e;
    if (b.a.iso) {
        bwd_prev_iso_chain_kernel<T><<<chains, 32, 0, st>>>(b, w);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        const long long rows = w.ntok * b.a.H;
        if (rows > 0) bwd_prev_iso_out_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(b, w);
        return cudaGetLastError();
    }
    if (prev_scan) return launch_prev_scan<T>(b, w, nchunks_max, st);
    const size_t psm = ((size_t)5 * GT * dk + 2 * GT) * sizeof(float) + (size_t)3 * GT * dk * sizeof(T);
    e = set_smem(reinterpret_cast<const void *>(bwd_prev_kernel<T>), psm);
    if (e != cudaSuccess) return e;
    bwd_prev_kernel<T><<<chains, dk, psm, st>>>(b, w);
    return cudaGetLastError();
}

cudaError_t launch_backward(const BwdArgs &b, bool bf16_in, long long ntok, long long nchunks_max, void *workspace,
                            cudaStream_t st) {
    const TokenArgs &a = b.a;
    const size_t th = (size_t)ntok * a.H;
    uint8_t *p = static_cast<uint8_t *>(workspace);
    BwdWs w;
    w.ntok = ntok;
    w.nblk = a.dv / DB;
    w.Pprev = reinterpret_cast<float *>(p); p += align256(th * a.dk * 4);
    w.g = reinterpret_cast<float *>(p); p += align256(th * a.dk * 4);
    w.den = reinterpret_cast<float *>(p); p += align256(th * 4);
    w.dden = reinterpret_cast<float *>(p); p += align256(th * 4);
    w.utape = reinterpret_cast<float *>(p); p += align256(th * a.dv * 4);
    const size_t ckpt_bytes = (size_t)ckpt_slots(ntok, a.nseq) * a.H * a.dk * a.dv * 4;
    w.ckpt = reinterpret_cast<float *>(p); p += align256(ckpt_bytes);
    w.part = reinterpret_cast<float *>(p);
    // the scan's look-back words must fit the checkpoint region (they may not for packed
    // sequences of very different lengths, whose work list is nseq x H x the longest's chunks)
    const bool tape_scan = !a.iso && ntok > 0 && gain_scan_tma_supported(a.dk, bf16_in) &&
                           scan_tma_workspace_bytes((long long)a.nseq * a.H, nchunks_max) <= ckpt_bytes;
    const bool prev_scan = !a.iso && prev_scan_bytes((long long)a.nseq * a.H, nchunks_max, a.dk) <= ckpt_bytes;
    const int ncm = (int)(nchunks_max < (1ll << 30) ? nchunks_max : (1ll << 30));
    return bf16_in ? launch_bwd_typed<bf16>(b, w, tape_scan, prev_scan, ncm, st)
                   : launch_bwd_typed<float>(b, w, tape_scan, prev_scan, ncm, st);
}

}  // namespace kdn
