// Chunkwise Diagonal-KDN forward on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), bf16 inputs, fp32 state.  (KDA article, "chunkwise" regime:
// provisional errors corrected by a causal triangular solve, with interaction matrices
// carrying the cumulative decay; explainer "对角近似" for the diagonal uncertainty.)
//
// One CTA owns one (sequence, head, d_v tile of DVT columns); d_k = 128, chunk C = 64.
// Per chunk (local tokens t, s in [0, L)), with Gam_t = prod_{j<=t} alpha_j per channel
// and the chunk's geometric-middle reference rho = Gam_{L-1}^{-1/2}:
//   prep (independent of the memory S):
//     uncertainty recursion and gain g_t (CUDA cores, thread = key channel)
//     K~ = k Gam rho,  Q~ = q Gam rho,  G~ = g / (Gam rho),  G' = G~ Gam_{L-1}^{1/2}
//     MMA1   [A; Aq] = [K~; Q~] G~^T                 -> A (s < t), Aq (s <= t)
//     T = (I + A)^{-1}                               (CUDA cores, blocked 16x16)
//     MMA_X  X = Aq T                                (M = 64)
//     MMA2   [w; X K~] = [T; X] K~ ,  Q' = Q~ - X K~
//   serial (carries S in TMEM, fp32):
//     S0' = Gam_{L-1}^{1/2} S (bf16 operand),  TMEM S <- Gam_{L-1} S
//     MMA4   [U; O] = [-w; Q'] S0' + [T; X] V        (K = 128 + 64)
//     MMA5   S += G'^T U
// which is the serial recurrence unrolled exactly: U = (I + A)^{-1}(V - K S0),
// O = Q S0 + Aq U, S_next = Gam_{L-1} S0 + sum_s (Gam_{L-1}/Gam_s) g_s u_s^T.
// The factored decay needs Gam_{L-1} >= 1e-30 per channel; a chunk outside that range
// sets KDN_ERR_RANGE in the device error word (the fp32 CUDA-core path has no limit).
#include <mutex>

#include "kdn_common.cuh"
#include "kdn_launch.h"
#include "kdn_tc.cuh"

namespace kdn {

namespace {
constexpr int C = 64, DK = 128, NT = 256;

template <int DVT>
struct TcSmem {
    static constexpr uint32_t Q = 0;                        // q tile (TMA) 16 KB; later T fp32 [64][64]
    static constexpr uint32_t K = Q + 16384;                // k tile (TMA) 16 KB; later A fp32 [64][64]
    static constexpr uint32_t V = K + 16384;                // v tile (TMA) DVT*128 B
    static constexpr uint32_t KQ = V + DVT * 128;           // [K~; Q~] bf16, K-major, 2 atoms of 128 rows
    static constexpr uint32_t G = KQ + 32768;               // G~ bf16, 64 token rows x 128 ch
    static constexpr uint32_t GP = G + 16384;               // alpha tile (TMA), turned into G' in place
    static constexpr uint32_t AQ = GP + 16384;              // Aq bf16, 64 x 64
    static constexpr uint32_t Y = AQ + 8192;                // [T; X] bf16, 128 x 64
    static constexpr uint32_t A4 = Y + 16384;               // [-w; Q'] bf16 128 x 128; pass A: g numerators fp32
    static constexpr uint32_t S = A4 + 32768;               // S0' bf16, 128 channel rows x DVT (MN-major)
    static constexpr uint32_t U = S + DVT * 256;            // U bf16, 64 token rows x DVT (MN-major)
    static constexpr uint32_t SIG = (DVT >= 128) ? U : U + DVT * 128;   // sigma tile (TMA) 16 KB
    static constexpr uint32_t MISC = SIG + 16384;
    static constexpr uint32_t MISC_BYTES = 2048;
    static constexpr uint32_t total = MISC + MISC_BYTES;
    static constexpr uint32_t TMA_BYTES = 4 * 16384 + DVT * 128;
};

struct TcParams {
    TokenArgs a;
    CUtensorMap tq, tk, tv, tal, tsg;
};

__device__ __forceinline__ float bf16_at(const uint8_t *base, uint32_t off) {
    return __uint_as_float(((uint32_t) * reinterpret_cast<const unsigned short *>(base + off)) << 16);
}
__device__ __forceinline__ void st_bf16(uint8_t *base, uint32_t off, float v) {
    *reinterpret_cast<__nv_bfloat16 *>(base + off) = __float2bfloat16_rn(v);
}

// T = (I + A)^{-1} for a strictly lower 64x64 fp32 A (row-major), blocked by 16.
// T's strictly-upper blocks are used as scratch; readers mask them out.
__device__ void tri_inverse64(const float *A, float *T, int tid) {
    if (tid < 64) {
        const int o = (tid >> 4) * 16, j = tid & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
            if (r > j) {
                float acc = 0.f;
#pragma unroll
                for (int s = 0; s < r; ++s)
                    if (s >= j) acc = fmaf(A[(o + r) * 64 + o + s], x[s], acc);
                x[r] = -acc;
            }
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) T[(o + r) * 64 + o + j] = x[r];
    }
    __syncthreads();
    for (int lvl = 1; lvl < 4; ++lvl) {
        const int nblk = 4 - lvl;
        for (int e = tid; e < nblk * 256; e += NT) {
            const int bj = e >> 8, bi = bj + lvl, rr = (e >> 4) & 15, cc = e & 15;
            float acc = 0.f;
            for (int kb = bj; kb < bi; ++kb)
#pragma unroll
                for (int s = 0; s < 16; ++s)
                    acc = fmaf(A[(bi * 16 + rr) * 64 + kb * 16 + s], T[(kb * 16 + s) * 64 + bj * 16 + cc], acc);
            T[(bj * 16 + rr) * 64 + bi * 16 + cc] = acc;   // M_ij parked in the upper block (bj, bi)
        }
        __syncthreads();
        for (int e = tid; e < nblk * 256; e += NT) {
            const int bj = e >> 8, bi = bj + lvl, rr = (e >> 4) & 15, cc = e & 15;
            float acc = 0.f;
            for (int u = 0; u <= rr; ++u)
                acc = fmaf(T[(bi * 16 + rr) * 64 + bi * 16 + u], T[(bj * 16 + u) * 64 + bi * 16 + cc], acc);
            T[(bi * 16 + rr) * 64 + bj * 16 + cc] = -acc;
        }
        __syncthreads();
    }
}
}  // namespace

template <int DVT>
__global__ void __launch_bounds__(NT, 1) chunk_tc_kernel(const __grid_constant__ TcParams prm)
{
    using L_ = TcSmem<DVT>;
    using namespace tc;
    extern __shared__ uint8_t smraw[];
    const uint32_t raw_u32 = smem_u32(smraw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;     // 1024-B aligned base (swizzle atoms)
    uint8_t *sm = smraw + (sb - raw_u32);

    float *misc = reinterpret_cast<float *>(sm + L_::MISC);
    float *r_s = misc;              // [64]
    float *invden = misc + 64;      // [64]
    float *gamc = misc + 128;       // [128] chunk decay Gam_{L-1}
    float *gam31 = misc + 256;      // [128] Gam_31 (start of the second half of the chunk)
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(misc + 384);
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
    const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;

    // ---- initial memory tile -> TMEM (lane = key channel), uncertainty -> registers
    const size_t sbase = (size_t)sh * DK * dv + (size_t)tile * DVT;
    if (warp < 4) {
        const int i = tid;
#pragma unroll 1
        for (int cb = 0; cb < DVT; cb += 32) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                float4 x = a.S0 ? *reinterpret_cast<const float4 *>(a.S0 + sbase + (size_t)i * dv + cb + j)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
                v[j] = x.x; v[j + 1] = x.y; v[j + 2] = x.z; v[j + 3] = x.w;
            }
            tmem_st32(T_S + lane_off + cb, v);
        }
    }
    float P = 1.f;
    if (tid < DK && a.P0) P = a.P0[(size_t)sh * DK + tid];

    const int nchunks = (t1 - t0 + C - 1) / C;
    uint32_t tma_phase = 0, mma_phase = 0;
    if (tid == 0 && nchunks > 0) {
        mbar_expect_tx(bar_tma, L_::TMA_BYTES);
        for (int b = 0; b < 2; ++b) {
            tma_load_3d(sm + L_::Q + b * 8192, &prm.tq, b * 64, h, t0, bar_tma);
            tma_load_3d(sm + L_::K + b * 8192, &prm.tk, b * 64, h, t0, bar_tma);
            tma_load_3d(sm + L_::GP + b * 8192, &prm.tal, b * 64, h, t0, bar_tma);
            tma_load_3d(sm + L_::SIG + b * 8192, &prm.tsg, b * 64, h, t0, bar_tma);
        }
        for (int b = 0; b < DVT / 64; ++b) tma_load_3d(sm + L_::V + b * 8192, &prm.tv, tile * DVT + b * 64, h, t0, bar_tma);
    }
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
        if (tid < C) r_s[tid] = (tid < L) ? ldf(rin + (size_t)(c0 + tid) * H + h) : 1.f;
        if (!mbar_wait(bar_tma, tma_phase)) atomicExch(abort_flag, 1);
        tma_phase ^= 1u;
        __syncthreads();
        if (*abort_flag) break;

        // ---- pass A: uncertainty recursion and gain numerators (thread = key channel)
        {
            float *gnum = reinterpret_cast<float *>(sm + L_::A4);
            if (tid < DK) {
                const int i = tid;
                const uint32_t coff = (uint32_t)(i >> 6) * 8192u, cb = (uint32_t)(i & 63) * 2u;
                float gam = 1.f;
                for (int t = 0; t < L; ++t) {
                    const uint32_t off = coff + swz(t, cb);
                    const float al = bf16_at(sm + L_::GP, off), sg = bf16_at(sm + L_::SIG, off);
                    const float kk = bf16_at(sm + L_::K, off);
                    const float mr = mu / r_s[t];
                    const float pm = fmaf(al * al, P, sg);
                    const float gn = pm * kk;
                    gnum[t * 128 + i] = gn;
                    P = __fdividef(pm, fmaf(mr * kk, gn, 1.f));
                    gam *= al;
                    if (t == 31) gam31[i] = gam;
                }
                gamc[i] = gam;
            }
            __syncthreads();
            // gain denominators r_t + sum_i P^-_i k_i^2 (4 threads per token)
            {
                const int t = tid >> 2, part = tid & 3;
                float acc = 0.f;
                if (t < L) {
#pragma unroll 8
                    for (int j = 0; j < 32; ++j) {
                        const int ch = part * 32 + j;
                        acc = fmaf(gnum[t * 128 + ch], bf16_at(sm + L_::K, (uint32_t)(ch >> 6) * 8192u + swz(t, (ch & 63) * 2)), acc);
                    }
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (part == 0) invden[t] = (t < L) ? 1.f / (r_s[t] + acc) : 0.f;
            }
            __syncthreads();
            // ---- pass B: decayed operands (thread = channel x half of the chunk)
            {
                const int i = tid & 127, half = tid >> 7;
                const float gC = gamc[i];
                if (half == 0 && L > 0 && !(gC >= 1e-30f)) raise_error(a.err, ERR_RANGE);
                const float rho = rsqrtf(gC), sqg = sqrtf(gC);
                const uint32_t coff = (uint32_t)(i >> 6) * 8192u, cb = (uint32_t)(i & 63) * 2u;
                const uint32_t kqoff = (uint32_t)(i >> 6) * 16384u;
                float gam = half ? gam31[i] : 1.f;
                for (int t = half * 32; t < half * 32 + 32; ++t) {
                    const uint32_t off = coff + swz(t, cb);
                    float kt = 0.f, qt = 0.f, gt = 0.f, gp = 0.f;
                    if (t < L) {
                        const float al = bf16_at(sm + L_::GP, off);
                        gam *= al;
                        const float gr = gam * rho;
                        const float g = gnum[t * 128 + i] * invden[t];
                        kt = bf16_at(sm + L_::K, off) * gr;
                        qt = bf16_at(sm + L_::Q, off) * gr;
                        gt = __fdividef(g, gr);
                        gp = gt * sqg;
                    }
                    st_bf16(sm + L_::KQ, kqoff + swz(t, cb), kt);
                    st_bf16(sm + L_::KQ, kqoff + swz(64 + t, cb), qt);
                    st_bf16(sm + L_::G, off, gt);
                    st_bf16(sm + L_::GP, off, gp);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA1: [A; Aq] = [K~; Q~] G~^T   (M=128, N=64, K=128)
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
        // rows 0..63 -> A (fp32, strictly lower); rows 64..127 -> Aq (bf16, lower incl. diagonal)
        float *Af = reinterpret_cast<float *>(sm + L_::K);
        float *Tf = reinterpret_cast<float *>(sm + L_::Q);
        if (warp < 4) {
            const int row = warp * 32 + lane;
#pragma unroll 1
            for (int hb = 0; hb < 2; ++hb) {
                float v[32];
                tmem_ld32(T_PREP + lane_off + hb * 32, v);
                if (row < 64) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) Af[row * 64 + hb * 32 + j] = (hb * 32 + j < row) ? v[j] : 0.f;
                } else {
                    const int t = row - 64;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint4 w4;
                        uint32_t *wp = reinterpret_cast<uint32_t *>(&w4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int s0 = hb * 32 + ch * 8 + 2 * e;
                            wp[e] = pack_bf16x2(s0 <= t ? v[ch * 8 + 2 * e] : 0.f, s0 + 1 <= t ? v[ch * 8 + 2 * e + 1] : 0.f);
                        }
                        *reinterpret_cast<uint4 *>(sm + L_::AQ + swz(t, (hb * 4 + ch) * 16)) = w4;
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tri_inverse64(Af, Tf, tid);
        // T -> bf16, rows 0..63 of Y (row t, column s; zero above the diagonal)
        {
            const int t = tid >> 2, q4 = tid & 3;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int chn = q4 * 2 + m;
                uint4 w4;
                uint32_t *wp = reinterpret_cast<uint32_t *>(&w4);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s0 = chn * 8 + 2 * e;
                    wp[e] = pack_bf16x2(s0 <= t ? Tf[t * 64 + s0] : 0.f, s0 + 1 <= t ? Tf[t * 64 + s0 + 1] : 0.f);
                }
                *reinterpret_cast<uint4 *>(sm + L_::Y + swz(t, chn * 16)) = w4;
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
            if (c + 1 < nchunks) {   // q and k tiles of the next chunk (their space is free now)
                const int n0 = c0 + C;
                mbar_expect_tx(bar_tma, L_::TMA_BYTES);
                for (int b = 0; b < 2; ++b) {
                    tma_load_3d(sm + L_::Q + b * 8192, &prm.tq, b * 64, h, n0, bar_tma);
                    tma_load_3d(sm + L_::K + b * 8192, &prm.tk, b * 64, h, n0, bar_tma);
                }
            }
        }
        wait_mma();
        // X -> bf16, rows 64..127 of Y.  M=64 accumulator: row m sits in lane (m%16) + 32*(m/16).
        if (warp < 4) {
            float v[32], v2[32];
            tmem_ld32(T_PREP + 64 + lane_off, v);
            tmem_ld32(T_PREP + 64 + lane_off + 32, v2);
            if (lane < 16) {
                const int t = warp * 16 + lane;
#pragma unroll
                for (int chn = 0; chn < 8; ++chn) {
                    uint4 w4;
                    uint32_t *wp = reinterpret_cast<uint32_t *>(&w4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s0 = chn * 8 + 2 * e;
                        const float x0 = s0 < 32 ? v[s0] : v2[s0 - 32];
                        const float x1 = s0 + 1 < 32 ? v[s0 + 1] : v2[s0 + 1 - 32];
                        wp[e] = pack_bf16x2(x0, x1);
                    }
                    *reinterpret_cast<uint4 *>(sm + L_::Y + swz(64 + t, chn * 16)) = w4;
                }
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
        if (warp < 4) {
            const int row = warp * 32 + lane;
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                float v[32];
                tmem_ld32(T_PREP + lane_off + cb * 32, v);
                const uint32_t atom = (uint32_t)(cb >> 1) * 16384u;
#pragma unroll
                for (int chn = 0; chn < 4; ++chn) {
                    const uint32_t boff = swz(row, ((cb & 1) * 4 + chn) * 16);
                    uint4 w4;
                    uint32_t *wp = reinterpret_cast<uint32_t *>(&w4);
                    if (row < 64) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) wp[e] = pack_bf16x2(-v[chn * 8 + 2 * e], -v[chn * 8 + 2 * e + 1]);
                    } else {
                        const uint4 q4 = *reinterpret_cast<const uint4 *>(sm + L_::KQ + atom + boff);
                        const uint32_t *qp = reinterpret_cast<const uint32_t *>(&q4);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            wp[e] = pack_bf16x2(bf16_lo(qp[e]) - v[chn * 8 + 2 * e], bf16_hi(qp[e]) - v[chn * 8 + 2 * e + 1]);
                    }
                    *reinterpret_cast<uint4 *>(sm + L_::A4 + atom + boff) = w4;
                }
            }
            // ---- memory tile: S0' = Gam^{1/2} S (bf16 operand), TMEM S <- Gam S
            const int i = row;
            const float gC = gamc[i], sqg = sqrtf(gC);
#pragma unroll 1
            for (int cb = 0; cb < DVT / 32; ++cb) {
                float v[32];
                tmem_ld32(T_S + lane_off + cb * 32, v);
                const uint32_t atom = (uint32_t)(cb >> 1) * 16384u;
#pragma unroll
                for (int chn = 0; chn < 4; ++chn) {
                    uint4 w4;
                    uint32_t *wp = reinterpret_cast<uint32_t *>(&w4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) wp[e] = pack_bf16x2(sqg * v[chn * 8 + 2 * e], sqg * v[chn * 8 + 2 * e + 1]);
                    *reinterpret_cast<uint4 *>(sm + L_::S + atom + swz(i, ((cb & 1) * 4 + chn) * 16)) = w4;
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= gC;
                tmem_st32(T_S + lane_off + cb * 32, v);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA4: [U; O] = [-w; Q'] S0' + [T; X] V   (M=128, N=DVT, K=128+64)
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
        if (tid == 0 && c + 1 < nchunks)
            for (int b = 0; b < DVT / 64; ++b)
                tma_load_3d(sm + L_::V + b * 8192, &prm.tv, tile * DVT + b * 64, h, c0 + C, bar_tma);
        // rows 0..63 -> U (bf16, zero past the chunk end); rows 64..127 -> o (global)
        if (warp < 4) {
            const int row = warp * 32 + lane;
#pragma unroll 1
            for (int cb = 0; cb < DVT / 32; ++cb) {
                float v[32];
                tmem_ld32(T_D4 + lane_off + cb * 32, v);
                if (row < 64) {
                    const bool live = row < L;
                    const uint32_t blk = (uint32_t)(cb >> 1) * 8192u;
#pragma unroll
                    for (int chn = 0; chn < 4; ++chn) {
                        uint4 w4;
                        uint32_t *wp = reinterpret_cast<uint32_t *>(&w4);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            wp[e] = live ? pack_bf16x2(v[chn * 8 + 2 * e], v[chn * 8 + 2 * e + 1]) : 0u;
                        *reinterpret_cast<uint4 *>(sm + L_::U + blk + swz(row, ((cb & 1) * 4 + chn) * 16)) = w4;
                    }
                } else if (row - 64 < L) {
                    bf16 *dst = out + ((size_t)(c0 + row - 64) * H + h) * dv + tile * DVT + cb * 32;
#pragma unroll
                    for (int chn = 0; chn < 4; ++chn) {
                        uint4 w4;
                        uint32_t *wp = reinterpret_cast<uint32_t *>(&w4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) wp[e] = pack_bf16x2(v[chn * 8 + 2 * e], v[chn * 8 + 2 * e + 1]);
                        *reinterpret_cast<uint4 *>(dst + chn * 8) = w4;
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA5: S += G'^T U   (M=128 channels, N=DVT, K=64 tokens; both operands MN-major)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_S, sdesc(sb + L_::GP + ks * 2048u, 8192, 1024), sdesc(sb + L_::U + ks * 2048u, 8192, 1024),
                         ID_M128_NV_MM, 1);
            mma_commit(bar_mma);
        }
        wait_mma();
        if (tid == 0 && c + 1 < nchunks)
            for (int b = 0; b < 2; ++b) {
                tma_load_3d(sm + L_::GP + b * 8192, &prm.tal, b * 64, h, c0 + C, bar_tma);
                tma_load_3d(sm + L_::SIG + b * 8192, &prm.tsg, b * 64, h, c0 + C, bar_tma);
            }
        __syncthreads();
        if (*abort_flag) break;
    }

    // ---- final state
    if (!*abort_flag) {
        if (warp < 4 && a.S_out) {
            const int i = tid;
#pragma unroll 1
            for (int cb = 0; cb < DVT; cb += 32) {
                float v[32];
                tmem_ld32(T_S + lane_off + cb, v);
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(a.S_out + sbase + (size_t)i * dv + cb + j) =
                        make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
        }
        if (a.P_out && tid < DK && tile == 0) a.P_out[(size_t)sh * DK + tid] = P;
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
static bool make_map(CUtensorMap *m, const void *base, int d, int H, long long ntok) {
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

template <int DVT>
static cudaError_t launch_tc(const TcParams &prm, cudaStream_t st) {
    constexpr size_t smem = TcSmem<DVT>::total + 1024;
    auto kern = chunk_tc_kernel<DVT>;
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
    if (!make_map(&prm.tq, a.q, DK, a.H, ntok) || !make_map(&prm.tk, a.k, DK, a.H, ntok) ||
        !make_map(&prm.tv, a.v, a.dv, a.H, ntok) || !make_map(&prm.tal, a.alpha, DK, a.H, ntok) ||
        !make_map(&prm.tsg, a.sigma, DK, a.H, ntok))
        return cudaErrorInvalidValue;
    if (dvt == 128) return launch_tc<128>(prm, st);
    if (dvt == 64) return launch_tc<64>(prm, st);
    return cudaErrorInvalidValue;
}

}  // namespace kdn
