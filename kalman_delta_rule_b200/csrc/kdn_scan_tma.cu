// The uncertainty / gain scan for bf16 inputs with d_k = 128: the same single pass with a
// decoupled look-back as the generic scan (explainer, closing paragraph of "各向同性近似": the
// uncertainty recursion is a Moebius map whose 2x2 matrices compose), with
//  - the chunk's alpha, sigma and k tiles fetched by TMA into one stage per CTA, four CTAs per
//    SM, so the loads of one CTA overlap the arithmetic of the others;
//  - look-back words that carry their own tag (64-bit (value, tag) per key channel), so a
//    reader never needs a fence or a flag, and every channel walks back on its own;
//  - thread = key-channel pair x 16-token segment in the composite and re-expansion passes.
// Outputs: g_t = P^-_t k_t / den_t (fp32), k_t^T g_t, and the uncertainty after each sequence;
// for the backward also P before each token and den_t.
#include "kdn_common.cuh"
#include "kdn_launch.h"
#include "kdn_tc.cuh"

namespace kdn {

namespace {
constexpr int C = 64, DK = 128, NT = 256;
enum : unsigned { TAG_AGG = 1, TAG_INCL = 2 };

struct ScanTmaSmem {
    static constexpr uint32_t STAGE = 3 * 16384;          // alpha, sigma, k tiles of one chunk
    // segment composites fp32 (normalised maps [[m00, m01], [m10, 1]]): (m00, m01) [4][128] and
    // m10 [4][128]; the last segment's m10 slots then hold the uncertainty at the chunk start
    // (the re-expansion never reads that segment's composite)
    static constexpr uint32_t COMP01 = STAGE;
    static constexpr uint32_t COMP10 = COMP01 + 4 * 128 * 8;
    static constexpr uint32_t MISC = COMP10 + 4 * 128 * 4;  // mu / r [64], sum P^- k^2 [64]
    static constexpr uint32_t CTL = MISC + 512;             // 2 mbarriers, the claimed unit
    static constexpr uint32_t total = CTL + 64;             // four CTAs per SM: <= 56 KB with the alignment pad
};

struct ScanTmaArgs {
    ScanArgs a;
    CUtensorMap tal, tsg, tk;
    unsigned long long *words;   // per unit [4][128]: aggregate (m00, m01, m10), end-of-chunk P
};

__device__ __forceinline__ f32x2 bf2(uint32_t w) { return pk2(tc::bf16_lo(w), tc::bf16_hi(w)); }
__device__ __forceinline__ float mob(float m00, float m01, float m10, float m11, float x) {
    return fmaf(m00, x, m01) / fmaf(m10, x, m11);
}
__device__ __forceinline__ unsigned long long tagged(float x, unsigned tag) {
    return ((unsigned long long)tag << 32) | __float_as_uint(x);
}
__device__ __forceinline__ unsigned tag_of(unsigned long long w) { return (unsigned)(w >> 32); }
__device__ __forceinline__ float value_of(unsigned long long w) { return __uint_as_float((unsigned)w); }
__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Sums 16 per-lane values over the 32 lanes of a warp with 16 shuffles (each step exchanges
// half of the remaining values).  Lanes 2m and 2m+1 end with the total of value `which`.
__device__ __forceinline__ float warp_reduce16(float (&v)[16], int lane, int &which) {
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

__global__ void __launch_bounds__(NT, 4) gain_scan_tma_kernel(const __grid_constant__ ScanTmaArgs sa)
{
    using L_ = ScanTmaSmem;
    using namespace tc;
    extern __shared__ uint8_t smraw[];
    const uint32_t raw_u32 = smem_u32(smraw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
    uint8_t *sm = smraw + (sb - raw_u32);
    float *comp01 = reinterpret_cast<float *>(sm + L_::COMP01);
    float *comp10 = reinterpret_cast<float *>(sm + L_::COMP10);
    float *pst = comp10 + 3 * 128;
    float *mur = reinterpret_cast<float *>(sm + L_::MISC);
    float *dsum = mur + 64;
    uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + L_::CTL);   // [2]

    const ScanArgs &a = sa.a;
    const bf16 *__restrict__ rin = static_cast<const bf16 *>(a.r);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const long long units = (long long)a.nchunks_max * a.nchains;
    const int cp = (warp & 1) * 32 + lane, sgi = warp >> 1, ch = cp * 2, tb = sgi * 16;
    const uint32_t catom = (uint32_t)(ch >> 6) * 8192u, bch = (uint32_t)(ch & 63) * 2u;

    if (tid == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_full + 1, 1);
        mbar_fence_init();
        tma_prefetch_desc(&sa.tal);
        tma_prefetch_desc(&sa.tsg);
        tma_prefetch_desc(&sa.tk);
    }
    __syncthreads();

    struct Unit { long long u; int c, chain, h, c0, L, nch; };
    static_assert(sizeof(Unit) <= 48, "claimed unit slot");
    static_assert(L_::total + 1024 <= 57344, "four CTAs per SM");
    Unit *claimed = reinterpret_cast<Unit *>(sm + L_::CTL + 16);
    // next unit with tokens: thread 0 takes tickets (skipping chunks past a sequence's end) and
    // decodes the unit once for the block
    auto claim = [&]() -> Unit {
        if (tid == 0) {
            Unit n;
            for (;;) {
                n.u = (long long)atomicAdd(a.counter, 1u);
                if (n.u >= units) break;
                const unsigned uu = (unsigned)n.u, nc = (unsigned)a.nchains;
                n.c = (int)(uu / nc);
                n.chain = (int)(uu - (unsigned)n.c * nc);
                const int s = n.chain / H;
                n.h = n.chain - s * H;
                int t0, t1;
                if (a.cu) { t0 = __ldg(a.cu + s); t1 = __ldg(a.cu + s + 1); }
                else { t0 = s * a.T; t1 = t0 + a.T; }
                n.nch = (t1 - t0 + C - 1) / C;
                if (n.c == 0 && n.nch > a.nchunks_max) raise_error(a.err, ERR_ARG);
                if (n.c < n.nch) {
                    n.c0 = t0 + n.c * C;
                    n.L = min(C, t1 - n.c0);
                    break;
                }
            }
            *claimed = n;
        }
        __syncthreads();
        return *claimed;
    };
    // the unit's tiles into stage st (thread 0), its r into r_next (threads < 64)
    float r_next = 1.f;
    auto fetch = [&](const Unit &n, int st) {
        if (tid == 0) {
            mbar_expect_tx(bar_full + st, L_::STAGE);
            uint8_t *dst = sm + st * L_::STAGE;
            for (int b = 0; b < 2; ++b) {
                tma_load_3d(dst + b * 8192, &sa.tal, b * 64, n.h, n.c0, bar_full + st);
                tma_load_3d(dst + 16384 + b * 8192, &sa.tsg, b * 64, n.h, n.c0, bar_full + st);
                tma_load_3d(dst + 32768 + b * 8192, &sa.tk, b * 64, n.h, n.c0, bar_full + st);
            }
        }
        r_next = (tid < n.L) ? ldf(rin + (size_t)(n.c0 + tid) * H + n.h) : 1.f;
    };

    // One stage: a unit's tiles are fetched when the unit is claimed; four CTAs per SM keep the
    // loads of one CTA under the arithmetic of the others.
    for (int it = 0;; ++it) {
        const Unit cur = claim();
        if (cur.u >= units) break;
        fetch(cur, 0);
        const long long u = cur.u;
        const int c = cur.c, chain = cur.chain, h = cur.h, c0 = cur.c0, L = cur.L, nch = cur.nch;
        const float r_cur = r_next;   // threads < 64: r of token tid
        if (tid < C) {
            mur[tid] = a.mu / r_next;
            dsum[tid] = 0.f;
        }
        const bool abort = !mbar_wait(bar_full, (uint32_t)(it & 1));   // the stage's it-th use: parity it & 1
        if (__syncthreads_or(abort)) {
            // the copy that timed out is the only one in flight: one more bounded wait for it
            // before the CTA exits and its shared memory goes away
            if (tid == 0) mbar_wait(bar_full, (uint32_t)(it & 1));
            raise_error(a.err, ERR_TIMEOUT);
            break;
        }
        uint8_t *tile = sm;

        // ---- segment composites of the uncertainty maps (predict [[a, s],[0,1]], update [[1,0],[c,1]]);
        //      channels ch and ch + 1 in the two lanes of packed f32x2 arithmetic
        {
            f32x2 m00 = pk2(1.f, 1.f), m01 = pk2(0.f, 0.f), m10 = m01, m11 = m00;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (tb + j < L) {
                    const uint32_t off = catom + swz(tb + j, bch);
                    const f32x2 al = bf2(*reinterpret_cast<const uint32_t *>(tile + off));
                    const f32x2 sg = bf2(*reinterpret_cast<const uint32_t *>(tile + 16384 + off));
                    const f32x2 kk = bf2(*reinterpret_cast<const uint32_t *>(tile + 32768 + off));
                    const float mr = mur[tb + j];
                    const f32x2 aa = mul2(al, al), cc = mul2(mul2(pk2(mr, mr), kk), kk);
                    const f32x2 y00 = fma2(aa, m00, mul2(sg, m10)), y01 = fma2(aa, m01, mul2(sg, m11));
                    m10 = fma2(cc, y00, m10);
                    m11 = fma2(cc, y01, m11);
                    m00 = y00;
                    m01 = y01;
                }
            }
            const float sa_ = 1.f / x2(m11), sb_ = 1.f / y2(m11);
            *reinterpret_cast<float4 *>(comp01 + (sgi * 128 + ch) * 2) =
                make_float4(x2(m00) * sa_, x2(m01) * sa_, y2(m00) * sb_, y2(m01) * sb_);
            *reinterpret_cast<float2 *>(comp10 + sgi * 128 + ch) = make_float2(x2(m10) * sa_, y2(m10) * sb_);
        }
        __syncthreads();

        // ---- warps 0-3 (thread = key channel): aggregate, its publication, decoupled look-back
        if (warp < 4) {
            const int cc = tid;
            unsigned long long *wd = sa.words + (size_t)u * 4 * DK + cc;
            float g00 = 1.f, g01 = 0.f, g10 = 0.f, g11 = 1.f;
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                const float2 c01 = *reinterpret_cast<const float2 *>(comp01 + (q2 * 128 + cc) * 2);
                const float4 cm = make_float4(c01.x, c01.y, comp10[q2 * 128 + cc], 0.f);
                const float n00 = fmaf(cm.x, g00, cm.y * g10), n01 = fmaf(cm.x, g01, cm.y * g11);
                const float n10 = fmaf(cm.z, g00, g10), n11 = fmaf(cm.z, g01, g11);
                const float sc = 1.f / n11;
                g00 = n00 * sc; g01 = n01 * sc; g10 = n10 * sc; g11 = 1.f;
            }
            if (c > 0) {
                st_relaxed(wd + 0 * DK, tagged(g00, TAG_AGG));
                st_relaxed(wd + 1 * DK, tagged(g01, TAG_AGG));
                st_relaxed(wd + 2 * DK, tagged(g10, TAG_AGG));
            }
            float p0;
            if (c == 0) {
                p0 = a.P0 ? a.P0[(size_t)chain * DK + cc] : 1.f;
            } else {
                // walk back to the nearest published end-of-chunk uncertainty, then forward through the
                // aggregates of the chunks in between, each applied as its owner applies it: the start
                // value does not depend on which words were published when (bit-reproducible)
                auto words_of = [&](int j) { return sa.words + ((size_t)j * a.nchains + chain) * 4 * DK + cc; };
                bool timed_out = false;
                int j = c - 1;
                float x = 1.f;
                for (;; --j) {
                    const unsigned long long *dj = words_of(j);
                    unsigned long long w0 = 0ull, w1 = 0ull, w2 = 0ull, w3 = ld_relaxed(dj + 3 * DK);
                    const long long ts = clock64();
                    while (tag_of(w3) != TAG_INCL) {
                        w0 = ld_relaxed(dj);
                        w1 = ld_relaxed(dj + DK);
                        w2 = ld_relaxed(dj + 2 * DK);
                        if (tag_of(w0) == TAG_AGG && tag_of(w1) == TAG_AGG && tag_of(w2) == TAG_AGG) break;
                        // give up after ~1 s, or at once when another wait already gave up
                        if (clock64() - ts > 2000000000ll || (a.err && (*(volatile unsigned *)a.err & ERR_TIMEOUT))) {
                            timed_out = true;
                            break;
                        }
                        __nanosleep(32);
                        w3 = ld_relaxed(dj + 3 * DK);
                    }
                    if (timed_out) {
                        raise_error(a.err, ERR_TIMEOUT);
                        break;
                    }
                    if (tag_of(w3) == TAG_INCL) {
                        x = value_of(w3);
                        break;
                    }
                }
                if (!timed_out) {
                    for (int jj = j + 1; jj < c; ++jj) {   // aggregates seen published by the walk
                        const unsigned long long *dq = words_of(jj);
                        x = mob(value_of(ld_relaxed(dq)), value_of(ld_relaxed(dq + DK)), value_of(ld_relaxed(dq + 2 * DK)), 1.f, x);
                    }
                }
                p0 = timed_out ? 1.f : x;
            }
            pst[cc] = p0;
            const float pe = mob(g00, g01, g10, 1.f, p0);
            st_relaxed(wd + 3 * DK, tagged(pe, TAG_INCL));
            if (c == nch - 1 && a.P_out) a.P_out[(size_t)chain * DK + cc] = pe;
        }
        __syncthreads();

        // ---- re-expansion: P^- k per token and channel (written fp32 over the token's alpha and
        //      sigma words, which only this thread reads), the gain denominators, g and k^T g
        {
            float Pa = pst[ch], Pb = pst[ch + 1];
            for (int q2 = 0; q2 < sgi; ++q2) {
                const float4 c01 = *reinterpret_cast<const float4 *>(comp01 + (q2 * 128 + ch) * 2);
                const float2 c10 = *reinterpret_cast<const float2 *>(comp10 + q2 * 128 + ch);
                const float4 ca = make_float4(c01.x, c01.y, c10.x, 0.f), cb = make_float4(c01.z, c01.w, c10.y, 0.f);
                Pa = mob(ca.x, ca.y, ca.z, 1.f, Pa);
                Pb = mob(cb.x, cb.y, cb.z, 1.f, Pb);
            }
            float xs[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                xs[j] = 0.f;
                if (tb + j < L) {
                    const uint32_t off = catom + swz(tb + j, bch);
                    const f32x2 al = bf2(*reinterpret_cast<const uint32_t *>(tile + off));
                    const f32x2 sg = bf2(*reinterpret_cast<const uint32_t *>(tile + 16384 + off));
                    const f32x2 kk = bf2(*reinterpret_cast<const uint32_t *>(tile + 32768 + off));
                    const float mr = mur[tb + j];
                    if (a.P_prev)
                        *reinterpret_cast<float2 *>(a.P_prev + ((size_t)(c0 + tb + j) * H + h) * DK + ch) =
                            make_float2(Pa, Pb);
                    const f32x2 pm = fma2(mul2(al, al), pk2(Pa, Pb), sg);
                    const f32x2 pk = mul2(pm, kk);
                    const f32x2 dn = fma2(mul2(pk2(mr, mr), kk), pk, pk2(1.f, 1.f));
                    Pa = __fdividef(x2(pm), x2(dn));
                    Pb = __fdividef(y2(pm), y2(dn));
                    *reinterpret_cast<float *>(tile + off) = x2(pk);
                    *reinterpret_cast<float *>(tile + 16384 + off) = y2(pk);
                    xs[j] = fmaf(x2(pk), x2(kk), y2(pk) * y2(kk));
                }
            }
            int which;
            const float tot = warp_reduce16(xs, lane, which);
            if ((lane & 1) == 0 && tb + which < L) atomicAdd(dsum + tb + which, tot);
        }
        __syncthreads();
        if (tid < C && tid < L) {
            const float x = dsum[tid];
            const float dn = r_cur + x, inv = 1.f / dn;
            dsum[tid] = inv;
            if (a.den) a.den[(size_t)(c0 + tid) * H + h] = dn;
            if (a.beta) a.beta[(size_t)(c0 + tid) * H + h] = x * inv;
        }
        __syncthreads();
        if (a.g) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (tb + j < L) {
                    const float inv = dsum[tb + j];
                    const uint32_t off = catom + swz(tb + j, bch);
                    *reinterpret_cast<float2 *>(a.g + ((size_t)(c0 + tb + j) * H + h) * DK + ch) =
                        make_float2(*reinterpret_cast<const float *>(tile + off) * inv,
                                    *reinterpret_cast<const float *>(tile + 16384 + off) * inv);
                }
            }
        }
        __syncthreads();   // the stage, composites and sums are free for the next unit
    }
}

size_t scan_tma_workspace_bytes(long long nchains, long long nchunks_max) {
    return 256 + (size_t)(nchains * nchunks_max) * 4 * DK * 8;
}

bool gain_scan_tma_supported(int dk, bool bf16_in) { return bf16_in && dk == DK; }

cudaError_t launch_gain_scan_tma(const ScanArgs &a, long long ntok, void *workspace, cudaStream_t st) {
    if (a.nchains == 0 || a.nchunks_max == 0) return cudaSuccess;
    const long long units = (long long)a.nchains * a.nchunks_max;
    ScanTmaArgs sa;
    sa.a = a;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    sa.a.counter = reinterpret_cast<unsigned *>(ws);
    sa.words = reinterpret_cast<unsigned long long *>(ws + 256);
    if (!make_token_map(&sa.tal, a.alpha, DK, a.H, ntok) || !make_token_map(&sa.tsg, a.sigma, DK, a.H, ntok) ||
        !make_token_map(&sa.tk, a.k, DK, a.H, ntok))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(ws, 0, scan_tma_workspace_bytes(a.nchains, a.nchunks_max), st);
    if (e != cudaSuccess) return e;
    constexpr size_t smem = ScanTmaSmem::total + 1024;
    KernelSetup ks;
    e = kernel_setup(reinterpret_cast<const void *>(gain_scan_tma_kernel), smem, NT, true, &ks);
    if (e != cudaSuccess) return e;
    // four CTAs per SM; units go out by ticket to resident CTAs only, so extra CTAs are harmless
    long long grid = (long long)ks.sms * 4;
    if (grid > units) grid = units;
    gain_scan_tma_kernel<<<(unsigned)grid, NT, smem, st>>>(sa);
    return cudaGetLastError();
}

}  // namespace kdn
