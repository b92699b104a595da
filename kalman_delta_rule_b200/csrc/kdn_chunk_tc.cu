// Chunkwise Diagonal-KDN forward on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), bf16 inputs, fp32 state.  (KDA article, "chunkwise" regime:
// provisional errors corrected by a causal triangular solve, with interaction matrices
// carrying the cumulative decay; explainer "对角近似" for the diagonal uncertainty.)
//
// One CTA owns one (sequence, head, d_v tile of DVT columns); d_k = 128, chunk C = 64.
// Per chunk (local tokens t, s in [0, L)), with Gam_t = prod_{j<=t} alpha_j per channel
// (decay referenced to the chunk start) and den_t = r_t + sum_i P^-_{t,i} k_{t,i}^2:
//   prep (independent of the memory S):
//     uncertainty recursion in eight 8-token segments joined by the Moebius composites
//     of the segments' 2x2 maps (CUDA cores, thread = key-channel pair x segment)
//     K~ = k Gam,  Q~ = q Gam,  G^ = P^- k / Gam   (the gain is G^ Gam / den)
//     MMA1   [A; Aq] = [K~; Q~] G^^T, columns scaled by 1/den  -> A (s < t), Aq (s <= t)
//     T = (I + A)^{-1} = (I - N + N^2 - N^3) D with D the 16x16 diagonal-block inverses
//     (CUDA cores) and N = D L (L: A below the block diagonal), on the tensor cores (M = 64)
//     MMA_X  X = Aq T                                (M = 64)
//     MMA2   [w; X K~] = [T; X] K~ ,  Q' = Q~ - X K~
//   serial (carries S in TMEM, fp32):
//     MMA4   [U; O] = [-w; Q'] S + [T; X] V          (K = 128 + 64)
//     MMA5   S += G^^T (U / den) ;  then S <- Gam_{L-1} S (rows)
// which is the serial recurrence unrolled exactly: U = (I + A)^{-1}(V - K S0),
// O = Q S0 + Aq U, S_next = Gam_{L-1} S0 + sum_s (Gam_{L-1}/Gam_s) g_s u_s^T.
// The factored decay needs Gam_{L-1} >= 1e-30 per channel; a chunk outside that range
// sets KDN_ERR_RANGE in the device error word (the fp32 CUDA-core path has no limit).
//
// Isotropic KDN (explainer "各向同性近似"; aifromscratch "Approximation 2"): the prep
// replaces the per-channel recursion by per-token channel sums (alpha^2, sigma, k^2),
// and one warp runs the head's scalar uncertainty as a warp-wide scan of the tokens'
// 2x2 maps; P^- of every channel is then the head's p^-, and the rest is unchanged.
#include <mutex>

#include "kdn_common.cuh"
#include "kdn_launch.h"
#include "kdn_tc.cuh"

namespace kdn {

namespace {
constexpr int C = 64, DK = 128, NT = 512, LDA = 68;   // LDA: padded fp32 row stride of A

template <int DVT>
struct TcSmem {
    static constexpr uint32_t Q = 0;                        // q tile (TMA); then bf16 D and L of the inverse
    static constexpr uint32_t K = Q + 16384;                // k tile (TMA); then A fp32 [64][LDA] at K + 1024
    static constexpr uint32_t AL = K + 16384;               // alpha tile (TMA); then Aq bf16 64 x 64 at AL + 8192
    static constexpr uint32_t SG = AL + 16384;              // sigma tile (TMA); then bf16 N and N^2
    static constexpr uint32_t V = SG + 16384;               // v tile (TMA), DVT*128 B
    static constexpr uint32_t KQ = V + DVT * 128;           // [K~; Q~] bf16, K-major, 2 atoms of 128 rows
    static constexpr uint32_t G = KQ + 32768;               // G^ bf16, 64 token rows x 128 ch
    static constexpr uint32_t Y = G + 16384;                // [T; X] bf16 128 x 64; prep: segment composites
    static constexpr uint32_t A4 = Y + 16384;               // [-w; Q'] bf16 128 x 128; prep: P^- fp32 [64][128]
    static constexpr uint32_t S = A4 + 32768;               // S bf16, 128 channel rows x DVT (MN-major)
    static constexpr uint32_t U = S + DVT * 256;            // U / den bf16 64 x DVT; prep: Gam every 4 tokens
    static constexpr uint32_t MISC = U + DVT * 128;
    static constexpr uint32_t MISC_BYTES = 2048;
    static constexpr uint32_t total = MISC + MISC_BYTES;
    static constexpr uint32_t TMA_BYTES = 4 * 16384 + DVT * 128;
    static constexpr uint32_t AF = K + 1024, AQ = AL + 8192;
    // bf16 64x64 operands of the tensor-core triangular inverse (rows of 128 B)
    static constexpr uint32_t DB = Q, LB = Q + 8192, NB = SG, N2B = SG + 8192, RB = K + 1024;
    static_assert(AF + 64 * LDA * 4 <= AQ, "A fp32 tile overlaps Aq");
    static_assert(DVT * 128 >= 16 * 128 * 4, "U must hold the decay table");
};

struct TcParams {
    TokenArgs a;
    CUtensorMap tq, tk, tv, tal, tsg;
};

// T = (I + A)^{-1} for a strictly lower 64x64 fp32 A (row stride LDA), blocked by 16:
// the four 16x16 diagonal blocks by forward substitution, then block levels
// T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj with 1x4 output strips whose dot products are
// split over `ks` adjacent lanes.  T's strictly-upper blocks are used as scratch.
// pack 8 floats (scaled) into one 16-byte bf16 chunk
__device__ __forceinline__ uint4 pack8(const float *v, float sc = 1.f) {
    uint4 w;
    w.x = tc::pack_bf16x2(v[0] * sc, v[1] * sc);
    w.y = tc::pack_bf16x2(v[2] * sc, v[3] * sc);
    w.z = tc::pack_bf16x2(v[4] * sc, v[5] * sc);
    w.w = tc::pack_bf16x2(v[6] * sc, v[7] * sc);
    return w;
}
}  // namespace

template <int DVT, bool ISO>
__global__ void __launch_bounds__(NT, 1) chunk_tc_kernel(const __grid_constant__ TcParams prm)
{
    using L_ = TcSmem<DVT>;
    using namespace tc;
    constexpr int NC = DVT / 4;   // d_v columns per warp in the epilogues (four warps share a lane quadrant)
    extern __shared__ uint8_t smraw[];
    const uint32_t raw_u32 = smem_u32(smraw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;     // 1024-B aligned base (swizzle atoms)
    uint8_t *sm = smraw + (sb - raw_u32);

    float *misc = reinterpret_cast<float *>(sm + L_::MISC);
    float *r_s = misc;              // [64] r_t
    float *mur = misc + 64;         // [64] mu / r_t
    float *invden = misc + 128;     // [64] 1 / den_t (0 past the chunk end)
    float *gamc = misc + 192;       // [128] chunk decay Gam_{L-1}
    float *pst = misc + 320;        // [128] uncertainty at the chunk start (isotropic: pst[0])
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(misc + 448);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_mma + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const TokenArgs &a = prm.a;
    const bf16 *__restrict__ rin = static_cast<const bf16 *>(a.r);
    bf16 *__restrict__ out = static_cast<bf16 *>(a.o);
    const int ntiles = a.dv / DVT;
    const int tile = blockIdx.x % ntiles;
    const int sh = blockIdx.x / ntiles;
    const int sq_ = sh / a.H, h = sh % a.H;
    int t0, t1;
    seq_range(a, sq_, t0, t1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, cg = warp >> 2;     // TMEM lane quadrant, column group
    const int H = a.H, dv = a.dv;
    const float mu = a.mu;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        *abort_flag = 0;
        tma_prefetch_desc(&prm.tq); tma_prefetch_desc(&prm.tk); tma_prefetch_desc(&prm.tv);
        tma_prefetch_desc(&prm.tal); tma_prefetch_desc(&prm.tsg);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t T_PREP = tmem, T_D4 = tmem + 128, T_S = tmem + 256;
    const uint32_t lane_off = ((uint32_t)quad * 32u) << 16;
    const int row = quad * 32 + lane;   // TMEM lane this thread reads in M=128 epilogues
    const int cb0 = cg * NC;            // first d_v column of this thread's epilogue slice

    // ---- initial memory tile -> TMEM (lane = key channel) and its bf16 operand copy
    const size_t sbase = (size_t)sh * DK * dv + (size_t)tile * DVT;
    {
        float v[NC];
#pragma unroll
        for (int j = 0; j < NC; j += 4) {
            float4 x = a.S0 ? *reinterpret_cast<const float4 *>(a.S0 + sbase + (size_t)row * dv + cb0 + j)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            v[j] = x.x; v[j + 1] = x.y; v[j + 2] = x.z; v[j + 3] = x.w;
        }
        tmem_st<NC>(T_S + lane_off + cb0, v);
        const uint32_t atom = (uint32_t)(cb0 >> 6) * 16384u;
#pragma unroll
        for (int chn = 0; chn < NC / 8; ++chn)
            *reinterpret_cast<uint4 *>(sm + L_::S + atom + swz(row, (((cb0 & 63) >> 3) + chn) * 16)) = pack8(v + chn * 8);
    }
    if (ISO) {
        if (tid == 0) pst[0] = a.P0 ? a.P0[sh] : 1.f;
    } else if (tid < DK) {
        pst[tid] = a.P0 ? a.P0[(size_t)sh * DK + tid] : 1.f;
    }

    const int nchunks = (t1 - t0 + C - 1) / C;
    uint32_t tma_phase = 0, mma_phase = 0;
    if (tid == 0 && nchunks > 0) {
        mbar_expect_tx(bar_tma, L_::TMA_BYTES);
        for (int b = 0; b < 2; ++b) {
            tma_load_3d(sm + L_::Q + b * 8192, &prm.tq, b * 64, h, t0, bar_tma);
            tma_load_3d(sm + L_::K + b * 8192, &prm.tk, b * 64, h, t0, bar_tma);
            tma_load_3d(sm + L_::AL + b * 8192, &prm.tal, b * 64, h, t0, bar_tma);
            tma_load_3d(sm + L_::SG + b * 8192, &prm.tsg, b * 64, h, t0, bar_tma);
        }
        for (int b = 0; b < DVT / 64; ++b) tma_load_3d(sm + L_::V + b * 8192, &prm.tv, tile * DVT + b * 64, h, t0, bar_tma);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    constexpr uint32_t ID_M128_N64_KK = idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_M64_N64_KM = idesc_bf16(64, 64, false, true);
    constexpr uint32_t ID_M128_N128_KM = idesc_bf16(128, 128, false, true);
    constexpr uint32_t ID_M128_NV_KM = idesc_bf16(128, DVT, false, true);
    constexpr uint32_t ID_M128_NV_MM = idesc_bf16(128, DVT, true, true);

    auto wait_mma = [&]() {
        if (!mbar_wait(bar_mma, mma_phase)) atomicExch(abort_flag, 1);
        mma_phase ^= 1u;
        tc_fence_after();
    };

    for (int c = 0; c < nchunks; ++c) {
        const int c0 = t0 + c * C;
        const int L = min(C, t1 - c0);
        const int nxt = c0 + C;
        const bool more = c + 1 < nchunks;
        if (tid < C) {
            const float rr = (tid < L) ? ldf(rin + (size_t)(c0 + tid) * H + h) : 1.f;
            r_s[tid] = rr;
            mur[tid] = mu / rr;
        }
        if (!mbar_wait(bar_tma, tma_phase)) atomicExch(abort_flag, 1);
        tma_phase ^= 1u;
        __syncthreads();
        if (*abort_flag) break;

        if constexpr (ISO) {
            // ---- isotropic: per-token channel sums, the decay table, then the head's
            //      uncertainty by a warp scan of the tokens' maps [[a, s], [c a, c s + 1]]
            //      with a = mean alpha^2, s = mean sigma, c = mu |k|^2 / (d_k r)
            float *tsum = reinterpret_cast<float *>(sm + L_::Y);                  // [64][4]
            float *segp = tsum + 256;                                             // [8][128]
            float *pms = reinterpret_cast<float *>(sm + L_::A4);                  // [64] p^-
            float *gst = reinterpret_cast<float *>(sm + L_::U);                   // [16][128]
            {
                const uint32_t atom8 = (uint32_t)(lane >> 4) * 8192u, bir = (uint32_t)(lane & 15) * 8u;
                float xa[4], xs[4], xk[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t off = atom8 + swz(warp * 4 + j, bir);
                    const uint2 aw = *reinterpret_cast<const uint2 *>(sm + L_::AL + off);
                    const uint2 sw = *reinterpret_cast<const uint2 *>(sm + L_::SG + off);
                    const uint2 kw = *reinterpret_cast<const uint2 *>(sm + L_::K + off);
                    const float a0 = bf16_lo(aw.x), a1 = bf16_hi(aw.x), a2 = bf16_lo(aw.y), a3 = bf16_hi(aw.y);
                    const float k0 = bf16_lo(kw.x), k1 = bf16_hi(kw.x), k2 = bf16_lo(kw.y), k3 = bf16_hi(kw.y);
                    xa[j] = fmaf(a0, a0, fmaf(a1, a1, fmaf(a2, a2, a3 * a3)));
                    xs[j] = (bf16_lo(sw.x) + bf16_hi(sw.x)) + (bf16_lo(sw.y) + bf16_hi(sw.y));
                    xk[j] = fmaf(k0, k0, fmaf(k1, k1, fmaf(k2, k2, k3 * k3)));
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        xa[j] += __shfl_xor_sync(0xffffffffu, xa[j], off);
                        xs[j] += __shfl_xor_sync(0xffffffffu, xs[j], off);
                        xk[j] += __shfl_xor_sync(0xffffffffu, xk[j], off);
                    }
                if (lane < 4) {
                    const float va = lane == 0 ? xa[0] : (lane == 1 ? xa[1] : (lane == 2 ? xa[2] : xa[3]));
                    const float vs = lane == 0 ? xs[0] : (lane == 1 ? xs[1] : (lane == 2 ? xs[2] : xs[3]));
                    const float vk = lane == 0 ? xk[0] : (lane == 1 ? xk[1] : (lane == 2 ? xk[2] : xk[3]));
                    *reinterpret_cast<float4 *>(tsum + (warp * 4 + lane) * 4) = make_float4(va, vs, vk, 0.f);
                }
            }
            const int cp = tid & 63, sgi = tid >> 6, ch = cp * 2;
            const uint32_t coff = (uint32_t)(ch >> 6) * 8192u, cb = (uint32_t)(ch & 63) * 2u;
            const int tb = sgi * 8, te = min(L, tb + 8);
            uint32_t aw8[8];
            float ga = 1.f, gb = 1.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                aw8[j] = *reinterpret_cast<const uint32_t *>(sm + L_::AL + coff + swz(tb + j, cb));
                if (tb + j < te) { ga *= bf16_lo(aw8[j]); gb *= bf16_hi(aw8[j]); }
            }
            *reinterpret_cast<float2 *>(segp + sgi * 128 + ch) = make_float2(ga, gb);
            __syncthreads();
            float gama = 1.f, gamb = 1.f;
            for (int q2 = 0; q2 < sgi; ++q2) {
                const float2 x = *reinterpret_cast<const float2 *>(segp + q2 * 128 + ch);
                gama *= x.x;
                gamb *= x.y;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int t = tb + j;
                if ((t & 3) == 0) *reinterpret_cast<float2 *>(gst + (t >> 2) * 128 + ch) = make_float2(gama, gamb);
                if (t < te) { gama *= bf16_lo(aw8[j]); gamb *= bf16_hi(aw8[j]); }
            }
            if (te == L && tb < L) {
                gamc[ch] = gama;
                gamc[ch + 1] = gamb;
                if (!(gama >= 1e-30f) || !(gamb >= 1e-30f)) raise_error(a.err, ERR_RANGE);
            }
            if (warp == 0) {
                constexpr float inv_dk = 1.f / DK;
                const float p0 = pst[0];
                float ta[2], ts[2], tc[2];
                float m00 = 1.f, m01 = 0.f, m10 = 0.f, m11 = 1.f;   // this lane's two tokens composed
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int t = 2 * lane + u;
                    ta[u] = 1.f; ts[u] = 0.f; tc[u] = 0.f;
                    if (t < L) {
                        const float4 x = *reinterpret_cast<const float4 *>(tsum + t * 4);
                        ta[u] = x.x * inv_dk;
                        ts[u] = x.y * inv_dk;
                        tc[u] = mur[t] * x.z * inv_dk;
                    }
                    // [[a, s], [c a, c s + 1]] applied after the composite so far
                    const float y00 = ta[u] * m00 + ts[u] * m10, y01 = ta[u] * m01 + ts[u] * m11;
                    m10 = fmaf(tc[u], y00, m10);
                    m11 = fmaf(tc[u], y01, m11);
                    m00 = y00;
                    m01 = y01;
                }
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {   // inclusive scan: lane's maps after the earlier lanes'
                    const float n00 = __shfl_up_sync(0xffffffffu, m00, off), n01 = __shfl_up_sync(0xffffffffu, m01, off);
                    const float n10 = __shfl_up_sync(0xffffffffu, m10, off), n11 = __shfl_up_sync(0xffffffffu, m11, off);
                    if (lane >= off) {
                        const float y00 = fmaf(m00, n00, m01 * n10), y01 = fmaf(m00, n01, m01 * n11);
                        const float y10 = fmaf(m10, n00, m11 * n10), y11 = fmaf(m10, n01, m11 * n11);
                        const float sc = 1.f / y11;
                        m00 = y00 * sc; m01 = y01 * sc; m10 = y10 * sc; m11 = 1.f;
                    }
                }
                float e00 = __shfl_up_sync(0xffffffffu, m00, 1), e01 = __shfl_up_sync(0xffffffffu, m01, 1);
                float e10 = __shfl_up_sync(0xffffffffu, m10, 1), e11 = __shfl_up_sync(0xffffffffu, m11, 1);
                if (lane == 0) { e00 = 1.f; e01 = 0.f; e10 = 0.f; e11 = 1.f; }
                float p = fmaf(e00, p0, e01) / fmaf(e10, p0, e11);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int t = 2 * lane + u;
                    if (t < L) {
                        const float pm = fmaf(ta[u], p, ts[u]);
                        pms[t] = pm;
                        p = __fdividef(pm, fmaf(tc[u], pm, 1.f));
                    }
                }
                __syncwarp();
                if (lane == (L - 1) >> 1) pst[0] = p;
            }
        } else {
        // ---- uncertainty recursion (thread = channel pair cp x 8-token segment sgi).  Each
        //      segment first composes the 2x2 maps of its tokens (predict [[a, s],[0,1]] then
        //      update [[1,0],[c,1]]); a segment then starts from the composites before it.
        //      Output: P^- per (token, channel) and the decay Gam before every 4th token.
        {
            float *pmv = reinterpret_cast<float *>(sm + L_::A4);                  // [64][128] P^-
            float *comp = reinterpret_cast<float *>(sm + L_::Y);                  // [7][128][4]
            float *gst = reinterpret_cast<float *>(sm + L_::U);                   // [16][128]
            const int cp = tid & 63, sgi = tid >> 6, ch = cp * 2;
            const uint32_t coff = (uint32_t)(ch >> 6) * 8192u, cb = (uint32_t)(ch & 63) * 2u;
            const float p0a = pst[ch], p0b = pst[ch + 1];
            const int tb = sgi * 8, te = min(L, tb + 8);
            // this thread's 8 tokens of alpha, sigma, k (2 channels each) and mu / r, loaded up front
            uint32_t aw8[8], sw8[8], kw8[8];
            float mr8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t off = coff + swz(tb + j, cb);
                aw8[j] = *reinterpret_cast<const uint32_t *>(sm + L_::AL + off);
                sw8[j] = *reinterpret_cast<const uint32_t *>(sm + L_::SG + off);
                kw8[j] = *reinterpret_cast<const uint32_t *>(sm + L_::K + off);
                mr8[j] = mur[tb + j];
            }
            if (sgi < 7 && te > tb) {
                float a00 = 1.f, a01 = 0.f, a10 = 0.f, a11 = 1.f, ga = 1.f;
                float b00 = 1.f, b01 = 0.f, b10 = 0.f, b11 = 1.f, gb = 1.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (tb + j < te) {
                        {
                            const float al = bf16_lo(aw8[j]), sg = bf16_lo(sw8[j]), kk = bf16_lo(kw8[j]);
                            const float aa = al * al, cc = mr8[j] * kk * kk;
                            const float y00 = fmaf(aa, a00, sg * a10), y01 = fmaf(aa, a01, sg * a11);
                            a10 = fmaf(cc, y00, a10); a11 = fmaf(cc, y01, a11); a00 = y00; a01 = y01; ga *= al;
                        }
                        {
                            const float al = bf16_hi(aw8[j]), sg = bf16_hi(sw8[j]), kk = bf16_hi(kw8[j]);
                            const float aa = al * al, cc = mr8[j] * kk * kk;
                            const float y00 = fmaf(aa, b00, sg * b10), y01 = fmaf(aa, b01, sg * b11);
                            b10 = fmaf(cc, y00, b10); b11 = fmaf(cc, y01, b11); b00 = y00; b01 = y01; gb *= al;
                        }
                    }
                }
                const float sa = 1.f / a11, sb2 = 1.f / b11;
                *reinterpret_cast<float4 *>(comp + (sgi * 128 + ch) * 4) = make_float4(a00 * sa, a01 * sa, a10 * sa, ga);
                *reinterpret_cast<float4 *>(comp + (sgi * 128 + ch + 1) * 4) = make_float4(b00 * sb2, b01 * sb2, b10 * sb2, gb);
            }
            __syncthreads();
            float Pa = p0a, Pb = p0b, gama = 1.f, gamb = 1.f;
            for (int q2 = 0; q2 < sgi; ++q2) {
                const float4 ca = *reinterpret_cast<const float4 *>(comp + (q2 * 128 + ch) * 4);
                const float4 cb4 = *reinterpret_cast<const float4 *>(comp + (q2 * 128 + ch + 1) * 4);
                Pa = fmaf(ca.x, Pa, ca.y) / fmaf(ca.z, Pa, 1.f);
                Pb = fmaf(cb4.x, Pb, cb4.y) / fmaf(cb4.z, Pb, 1.f);
                gama *= ca.w;
                gamb *= cb4.w;
            }
            float pma8[8], pmb8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int t = tb + j;
                if ((t & 3) == 0) *reinterpret_cast<float2 *>(gst + (t >> 2) * 128 + ch) = make_float2(gama, gamb);
                pma8[j] = 0.f;
                pmb8[j] = 0.f;
                if (t < te) {
                    const float ala = bf16_lo(aw8[j]), alb = bf16_hi(aw8[j]), ka = bf16_lo(kw8[j]), kb = bf16_hi(kw8[j]);
                    const float pma = fmaf(ala * ala, Pa, bf16_lo(sw8[j])), pmb = fmaf(alb * alb, Pb, bf16_hi(sw8[j]));
                    pma8[j] = pma;
                    pmb8[j] = pmb;
                    Pa = __fdividef(pma, fmaf(mr8[j] * ka * ka, pma, 1.f));
                    Pb = __fdividef(pmb, fmaf(mr8[j] * kb * kb, pmb, 1.f));
                    gama *= ala;
                    gamb *= alb;
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (tb + j < te) *reinterpret_cast<float2 *>(pmv + (tb + j) * 128 + ch) = make_float2(pma8[j], pmb8[j]);
            if (te == L && tb < L) {     // this thread processed the chunk's last token
                pst[ch] = Pa;
                pst[ch + 1] = Pb;
                gamc[ch] = gama;
                gamc[ch + 1] = gamb;
                if (!(gama >= 1e-30f) || !(gamb >= 1e-30f)) raise_error(a.err, ERR_RANGE);
            }
        }
        }
        __syncthreads();
        // ---- elementwise pass (warp = 4 tokens, lane = 4 channels; 8-byte accesses):
        //      K~ = k Gam, Q~ = q Gam, G^ = P^- k / Gam, and den_t = r_t + sum_i P^-_i k_i^2
        {
            const float *pmv = reinterpret_cast<const float *>(sm + L_::A4);
            const float *gst = reinterpret_cast<const float *>(sm + L_::U);
            const int cq = lane, g = warp, c4 = cq * 4;
            const uint32_t atom8 = (uint32_t)(cq >> 4) * 8192u, atom16 = (uint32_t)(cq >> 4) * 16384u;
            const uint32_t bir = (uint32_t)(cq & 15) * 8u;
            float4 gam = *reinterpret_cast<const float4 *>(gst + g * 128 + c4);
            uint2 aw[4], kw[4], qw[4];
            float4 pm[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {   // loads for the warp's four tokens first
                const int t = g * 4 + j;
                const uint32_t off = swz(t, bir);
                aw[j] = *reinterpret_cast<const uint2 *>(sm + L_::AL + atom8 + off);
                kw[j] = *reinterpret_cast<const uint2 *>(sm + L_::K + atom8 + off);
                qw[j] = *reinterpret_cast<const uint2 *>(sm + L_::Q + atom8 + off);
                if constexpr (ISO) {
                    const float x = pmv[t];
                    pm[j] = make_float4(x, x, x, x);
                } else {
                    pm[j] = *reinterpret_cast<const float4 *>(pmv + t * 128 + c4);
                }
            }
            float xs[4];
            uint2 kq[4], qq[4], gg[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = g * 4 + j;
                kq[j] = make_uint2(0u, 0u); qq[j] = kq[j]; gg[j] = kq[j]; xs[j] = 0.f;
                if (t < L) {
                    gam.x *= bf16_lo(aw[j].x); gam.y *= bf16_hi(aw[j].x); gam.z *= bf16_lo(aw[j].y); gam.w *= bf16_hi(aw[j].y);
                    const float k0 = bf16_lo(kw[j].x), k1 = bf16_hi(kw[j].x), k2 = bf16_lo(kw[j].y), k3 = bf16_hi(kw[j].y);
                    const float p0 = pm[j].x * k0, p1 = pm[j].y * k1, p2 = pm[j].z * k2, p3 = pm[j].w * k3;
                    xs[j] = fmaf(p0, k0, fmaf(p1, k1, fmaf(p2, k2, p3 * k3)));
                    kq[j].x = pack_bf16x2(k0 * gam.x, k1 * gam.y);
                    kq[j].y = pack_bf16x2(k2 * gam.z, k3 * gam.w);
                    qq[j].x = pack_bf16x2(bf16_lo(qw[j].x) * gam.x, bf16_hi(qw[j].x) * gam.y);
                    qq[j].y = pack_bf16x2(bf16_lo(qw[j].y) * gam.z, bf16_hi(qw[j].y) * gam.w);
                    gg[j].x = pack_bf16x2(__fdividef(p0, gam.x), __fdividef(p1, gam.y));
                    gg[j].y = pack_bf16x2(__fdividef(p2, gam.z), __fdividef(p3, gam.w));
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = g * 4 + j;
                const uint32_t off = swz(t, bir);
                *reinterpret_cast<uint2 *>(sm + L_::KQ + atom16 + off) = kq[j];
                *reinterpret_cast<uint2 *>(sm + L_::KQ + atom16 + swz(64 + t, bir)) = qq[j];
                *reinterpret_cast<uint2 *>(sm + L_::G + atom8 + off) = gg[j];
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int j = 0; j < 4; ++j) xs[j] += __shfl_xor_sync(0xffffffffu, xs[j], off);
            if (lane < 4) {
                const int t = g * 4 + lane;
                const float xv = lane == 0 ? xs[0] : (lane == 1 ? xs[1] : (lane == 2 ? xs[2] : xs[3]));
                invden[t] = (t < L) ? __fdividef(1.f, r_s[t] + xv) : 0.f;
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA1: [A; Aq] = [K~; Q~] G^^T   (M=128, N=64, K=128)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ka = (uint32_t)(ks >> 2), ko = (uint32_t)(ks & 3) * 32u;
                mma_bf16(T_PREP, sdesc(sb + L_::KQ + ka * 16384u + ko, 16, 1024), sdesc(sb + L_::G + ka * 8192u + ko, 16, 1024),
                         ID_M128_N64_KK, ks > 0);
            }
            mma_commit(bar_mma);
        }
        wait_mma();
        // rows 0..63 -> A (fp32, strictly lower) ; rows 64..127 -> Aq (bf16, lower incl. diagonal); columns / den
        float *Af = reinterpret_cast<float *>(sm + L_::AF);
        {
            const int s0 = cg * 16;
            float v[16];
            tmem_ld16(T_PREP + lane_off + s0, v);
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                const float4 d4 = *reinterpret_cast<const float4 *>(invden + s0 + j);
                v[j] *= d4.x; v[j + 1] *= d4.y; v[j + 2] *= d4.z; v[j + 3] *= d4.w;
            }
            if (row < 64) {
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4 *>(Af + row * LDA + s0 + j) =
                        make_float4(s0 + j < row ? v[j] : 0.f, s0 + j + 1 < row ? v[j + 1] : 0.f,
                                    s0 + j + 2 < row ? v[j + 2] : 0.f, s0 + j + 3 < row ? v[j + 3] : 0.f);
            } else {
                const int t = row - 64;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (s0 + j > t) v[j] = 0.f;
#pragma unroll
                for (int chn = 0; chn < 2; ++chn)
                    *reinterpret_cast<uint4 *>(sm + L_::AQ + swz(t, (cg * 2 + chn) * 16)) = pack8(v + chn * 8);
            }
        }
        tc_fence_before();
        __syncthreads();
        // ---- T = (I + A)^{-1} on the tensor cores.  With D the four 16x16 diagonal-block inverses
        //      (CUDA cores) and L the blocks of A below the block diagonal, N = D L is nilpotent
        //      (N^4 = 0) and T = (I + D L)^{-1} D = (I - N + N^2 - N^3) D.
        {
            float *Db4 = reinterpret_cast<float *>(sm + L_::Y);   // [4][16][16] fp32 diagonal blocks of D
            if (tid < 64) {
                const int o = (tid >> 4) * 16, j = tid & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
                for (int r = 1; r < 16; ++r) {
                    const float *arow = Af + (o + r) * LDA + o;
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < r; ++c) acc[c & 3] = fmaf(arow[c], x[c], acc[c & 3]);
                    if (r > j) x[r] = -((acc[0] + acc[1]) + (acc[2] + acc[3]));
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) Db4[(o + r) * 16 + j] = x[r];
            }
            __syncthreads();
            {   // bf16 D (block diagonal) and L (below the block diagonal): one 16-byte chunk per thread each
                const int r = tid >> 3, cc = tid & 7, b = r >> 4, cb = cc >> 1;
                float dv8[8], lv8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int c = cc * 8 + e;
                    dv8[e] = (cb == b) ? Db4[r * 16 + (c & 15)] : 0.f;
                    lv8[e] = (cb < b) ? Af[r * LDA + c] : 0.f;
                }
                *reinterpret_cast<uint4 *>(sm + L_::DB + swz(r, cc * 16)) = pack8(dv8);
                *reinterpret_cast<uint4 *>(sm + L_::LB + swz(r, cc * 16)) = pack8(lv8);
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            // M=64 x N=64 x K=64 product: A operand K-major (rows of 128 B), B operand MN-major
            auto mma64 = [&](uint32_t dcol, uint32_t aoff, uint32_t boff) {
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(dcol, sdesc(sb + aoff + ks * 32u, 16, 1024), sdesc(sb + boff + ks * 2048u, 8192, 1024),
                                 ID_M64_N64_KM, ks > 0);
                    mma_commit(bar_mma);
                }
                wait_mma();
            };
            // M=64 accumulator rows: row m sits in lane (m%16) + 32*(m/16); this warp reads
            // columns cg*16 .. cg*16+15 of rows quad*16 + lane (lanes < 16)
            const int m64 = quad * 16 + lane;
            auto store64 = [&](uint32_t dst, float (&v)[16]) {
                if (lane < 16) {
#pragma unroll
                    for (int chn = 0; chn < 2; ++chn)
                        *reinterpret_cast<uint4 *>(sm + dst + swz(m64, (cg * 2 + chn) * 16)) = pack8(v + chn * 8);
                }
            };
            auto sync_tc = [&]() {
                fence_async_smem();
                tc_fence_before();
                __syncthreads();
            };
            mma64(T_PREP, L_::DB, L_::LB);                        // N = D L
            { float v[16]; tmem_ld16(T_PREP + lane_off + cg * 16, v); store64(L_::NB, v); }
            sync_tc();
            mma64(T_PREP + 64, L_::NB, L_::NB);                   // N^2
            { float v[16]; tmem_ld16(T_PREP + 64 + lane_off + cg * 16, v); store64(L_::N2B, v); }
            sync_tc();
            mma64(T_D4, L_::N2B, L_::NB);                         // N^3 (the state-update columns are free here)
            {   // R = I - N + N^2 - N^3
                float n1[16], n2[16], n3[16];
                tmem_ld16(T_PREP + lane_off + cg * 16, n1);
                tmem_ld16(T_PREP + 64 + lane_off + cg * 16, n2);
                tmem_ld16(T_D4 + lane_off + cg * 16, n3);
#pragma unroll
                for (int j = 0; j < 16; ++j) n1[j] = (cg * 16 + j == m64 ? 1.f : 0.f) - n1[j] + n2[j] - n3[j];
                store64(L_::RB, n1);
            }
            sync_tc();
            mma64(T_PREP, L_::RB, L_::DB);                        // T = R D
            {   // T -> bf16, rows 0..63 of Y (zero above the diagonal)
                float v[16];
                tmem_ld16(T_PREP + lane_off + cg * 16, v);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (cg * 16 + j > m64) v[j] = 0.f;
                store64(L_::Y, v);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA_X: X = Aq T   (M=64, N=64, K=64; T read as MN-major B from Y rows 0..63)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_PREP + 64, sdesc(sb + L_::AQ + ks * 32u, 16, 1024), sdesc(sb + L_::Y + ks * 2048u, 8192, 1024),
                         ID_M64_N64_KM, ks > 0);
            mma_commit(bar_mma);
            if (more) {   // q, k and sigma tiles of the next chunk (the inverse's operands are consumed)
                mbar_expect_tx(bar_tma, L_::TMA_BYTES);
                for (int b = 0; b < 2; ++b) {
                    tma_load_3d(sm + L_::Q + b * 8192, &prm.tq, b * 64, h, nxt, bar_tma);
                    tma_load_3d(sm + L_::K + b * 8192, &prm.tk, b * 64, h, nxt, bar_tma);
                    tma_load_3d(sm + L_::SG + b * 8192, &prm.tsg, b * 64, h, nxt, bar_tma);
                }
            }
        }
        wait_mma();
        if (tid == 0 && more)   // alpha tile of the next chunk (Aq consumed)
            for (int b = 0; b < 2; ++b) tma_load_3d(sm + L_::AL + b * 8192, &prm.tal, b * 64, h, nxt, bar_tma);
        // X -> bf16, rows 64..127 of Y.  M=64 accumulator: row m sits in lane (m%16) + 32*(m/16).
        {
            float v[16];
            tmem_ld16(T_PREP + 64 + lane_off + cg * 16, v);
            if (lane < 16) {
                const int t = quad * 16 + lane;
#pragma unroll
                for (int chn = 0; chn < 2; ++chn)
                    *reinterpret_cast<uint4 *>(sm + L_::Y + swz(64 + t, (cg * 2 + chn) * 16)) = pack8(v + chn * 8);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA2: [w; X K~] = [T; X] K~   (M=128, N=128 channels, K=64 tokens; K~ as MN-major B)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_PREP, sdesc(sb + L_::Y + ks * 32u, 16, 1024), sdesc(sb + L_::KQ + ks * 2048u, 16384, 1024),
                         ID_M128_N128_KM, ks > 0);
            mma_commit(bar_mma);
        }
        wait_mma();
        // rows 0..63 -> -w ; rows 64..127 -> Q' = Q~ - X K~   (bf16 into A4)
        {
            float v[32];
            tmem_ld32(T_PREP + lane_off + cg * 32, v);
            const uint32_t atom = (uint32_t)(cg >> 1) * 16384u;
#pragma unroll
            for (int chn = 0; chn < 4; ++chn) {
                const uint32_t boff = swz(row, ((cg & 1) * 4 + chn) * 16);
                if (row < 64) {
                    *reinterpret_cast<uint4 *>(sm + L_::A4 + atom + boff) = pack8(v + chn * 8, -1.f);
                } else {
                    const uint4 q4 = *reinterpret_cast<const uint4 *>(sm + L_::KQ + atom + boff);
                    const uint32_t *qp = reinterpret_cast<const uint32_t *>(&q4);
                    float w8[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        w8[2 * e] = bf16_lo(qp[e]) - v[chn * 8 + 2 * e];
                        w8[2 * e + 1] = bf16_hi(qp[e]) - v[chn * 8 + 2 * e + 1];
                    }
                    *reinterpret_cast<uint4 *>(sm + L_::A4 + atom + boff) = pack8(w8);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA4: [U; O] = [-w; Q'] S + [T; X] V   (M=128, N=DVT, K=128+64)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ka = (uint32_t)(ks >> 2), ko = (uint32_t)(ks & 3) * 32u;
                mma_bf16(T_D4, sdesc(sb + L_::A4 + ka * 16384u + ko, 16, 1024), sdesc(sb + L_::S + ks * 2048u, 16384, 1024),
                         ID_M128_NV_KM, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_D4, sdesc(sb + L_::Y + ks * 32u, 16, 1024), sdesc(sb + L_::V + ks * 2048u, 8192, 1024),
                         ID_M128_NV_KM, 1);
            mma_commit(bar_mma);
        }
        wait_mma();
        if (tid == 0 && more)
            for (int b = 0; b < DVT / 64; ++b)
                tma_load_3d(sm + L_::V + b * 8192, &prm.tv, tile * DVT + b * 64, h, nxt, bar_tma);
        // rows 0..63 -> U / den (bf16, zero past the chunk end); rows 64..127 -> o (global)
        {
            float v[NC];
            tmem_ld<NC>(T_D4 + lane_off + cb0, v);
            if (row < 64) {
                const float sc = invden[row];
                const uint32_t blk = (uint32_t)(cb0 >> 6) * 8192u;
#pragma unroll
                for (int chn = 0; chn < NC / 8; ++chn)
                    *reinterpret_cast<uint4 *>(sm + L_::U + blk + swz(row, (((cb0 & 63) >> 3) + chn) * 16)) =
                        pack8(v + chn * 8, sc);
            } else if (row - 64 < L) {
                bf16 *dst = out + ((size_t)(c0 + row - 64) * H + h) * dv + tile * DVT + cb0;
#pragma unroll
                for (int chn = 0; chn < NC / 8; ++chn) *reinterpret_cast<uint4 *>(dst + chn * 8) = pack8(v + chn * 8);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA5: S += G^^T (U / den)   (M=128 channels, N=DVT, K=64 tokens; both operands MN-major)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_S, sdesc(sb + L_::G + ks * 2048u, 8192, 1024), sdesc(sb + L_::U + ks * 2048u, 8192, 1024),
                         ID_M128_NV_MM, 1);
            mma_commit(bar_mma);
        }
        wait_mma();
        // ---- decay the rows by the chunk's Gam_{L-1}; refresh the bf16 operand copy
        {
            const float gC = gamc[row];
            float v[NC];
            tmem_ld<NC>(T_S + lane_off + cb0, v);
#pragma unroll
            for (int j = 0; j < NC; ++j) v[j] *= gC;
            tmem_st<NC>(T_S + lane_off + cb0, v);
            const uint32_t atom = (uint32_t)(cb0 >> 6) * 16384u;
#pragma unroll
            for (int chn = 0; chn < NC / 8; ++chn)
                *reinterpret_cast<uint4 *>(sm + L_::S + atom + swz(row, (((cb0 & 63) >> 3) + chn) * 16)) = pack8(v + chn * 8);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (*abort_flag) break;
    }

    // ---- final state
    if (!*abort_flag) {
        if (a.S_out) {
            float v[NC];
            tmem_ld<NC>(T_S + lane_off + cb0, v);
#pragma unroll
            for (int j = 0; j < NC; j += 4)
                *reinterpret_cast<float4 *>(a.S_out + sbase + (size_t)row * dv + cb0 + j) =
                    make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
        if (a.P_out && tile == 0) {
            if (ISO) {
                if (tid == 0) a.P_out[sh] = pst[0];
            } else if (tid < DK) {
                a.P_out[(size_t)sh * DK + tid] = pst[tid];
            }
        }
    } else {
        raise_error(a.err, ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [ntok, H, d] bf16 viewed as a 3-D tensor {d, H, ntok}; box = 64 channels x 1 head x 64 tokens, 128B swizzle
bool make_token_map(CUtensorMap *m, const void *base, int d, int H, long long ntok) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)ntok};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DVT, bool ISO>
static cudaError_t launch_tc(const TcParams &prm, cudaStream_t st) {
    constexpr size_t smem = TcSmem<DVT>::total + 1024;
    auto kern = chunk_tc_kernel<DVT, ISO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)prm.a.nseq * prm.a.H * (prm.a.dv / DVT));
    kern<<<grid, NT, smem, st>>>(prm);
    return cudaGetLastError();
}

bool chunk_tc_supported(int dk, int dv, bool bf16_in, int chunk, long long ntok) {
    return bf16_in && chunk == C && dk == DK && (dv == 64 || dv == 128 || dv == 256) && ntok > 0 && encode_fn() != nullptr;
}

cudaError_t launch_chunk_tc(const TokenArgs &a, long long ntok, int dvt, cudaStream_t st) {
    if (a.nseq == 0 || a.H == 0) return cudaSuccess;
    TcParams prm;
    prm.a = a;
    if (!make_token_map(&prm.tq, a.q, DK, a.H, ntok) || !make_token_map(&prm.tk, a.k, DK, a.H, ntok) ||
        !make_token_map(&prm.tv, a.v, a.dv, a.H, ntok) || !make_token_map(&prm.tal, a.alpha, DK, a.H, ntok) ||
        !make_token_map(&prm.tsg, a.sigma, DK, a.H, ntok))
        return cudaErrorInvalidValue;
    if (dvt == 128) return a.iso ? launch_tc<128, true>(prm, st) : launch_tc<128, false>(prm, st);
    if (dvt == 64) return a.iso ? launch_tc<64, true>(prm, st) : launch_tc<64, false>(prm, st);
    return cudaErrorInvalidValue;
}

}  // namespace kdn
