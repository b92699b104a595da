// The uncertainty / gain scan of the Diagonal KDN on its own (explainer, closing
// paragraph of "各向同性近似": the uncertainty recursion is a Moebius map whose 2x2
// matrices compose, so it parallelises as an associative scan).
//
// Per key channel, one token maps the uncertainty P as
//     predict  x -> a x + s        = [[a, s], [0, 1]],   a = alpha^2, s = sigma
//     update   x -> x / (1 + c x)  = [[1, 0], [c, 1]],   c = mu k^2 / r
// acting projectively (x -> (m00 x + m01) / (m10 x + m11)).  The kernel runs one pass
// over 64-token chunks with a decoupled look-back:
//   1. a chunk composes its tokens' matrices (four segments in parallel, then joined)
//      and publishes the aggregate;
//   2. it walks back over its predecessors, composing their aggregates until it meets a
//      published end-of-chunk uncertainty (or the sequence start), which fixes its own
//      starting uncertainty; it then publishes its end-of-chunk uncertainty;
//   3. it re-expands its tokens: P^- per token and channel, the gain denominator
//      den_t = r_t + sum_i P^-_i k_i^2, the gain g_t = P^- k / den_t and k^T g.
// Work is handed out by a ticket counter in chunk-major order, so every predecessor of
// a chunk was taken by a CTA that is already running; waits are bounded.
#include <mutex>

#include "kdn_common.cuh"
#include "kdn_launch.h"

namespace kdn {

namespace {
constexpr int SC = 64, SNT = 256;
enum : int { FLAG_NONE = 0, FLAG_AGG = 1, FLAG_INCL = 2 };

template <int DK, typename Tin>
struct ScanSmem {
    static constexpr int NCP = DK / 2, NSEG = SNT / NCP, SEG = SC / NSEG;
    static constexpr size_t tile = (size_t)SC * DK * sizeof(Tin);
    static constexpr size_t AL = 0, SG = AL + tile, KK = SG + tile;
    static constexpr size_t PMK = KK + tile;                                  // fp32 [SC][DK]  P^- k
    static constexpr size_t COMP = PMK + (size_t)SC * DK * 4;                 // fp32 [NSEG][DK][4]
    static constexpr size_t RS = COMP + (size_t)NSEG * DK * 16;               // fp32 [SC] mu / r, [SC] r
    static constexpr size_t PST = RS + 2 * SC * 4;                            // fp32 [DK] chunk-start P
    static constexpr size_t total = PST + DK * 4 + 64;
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float mob(float m00, float m01, float m10, float m11, float x) {
    return fmaf(m00, x, m01) / fmaf(m10, x, m11);
}
}  // namespace

template <int DK, typename Tin>
__global__ void __launch_bounds__(SNT) gain_scan_kernel(ScanArgs a)
{
    using L_ = ScanSmem<DK, Tin>;
    constexpr int NCP = L_::NCP, NSEG = L_::NSEG, SEG = L_::SEG;
    extern __shared__ __align__(16) uint8_t sm[];
    Tin *al_s = reinterpret_cast<Tin *>(sm + L_::AL);
    Tin *sg_s = reinterpret_cast<Tin *>(sm + L_::SG);
    Tin *k_s = reinterpret_cast<Tin *>(sm + L_::KK);
    float *pmk = reinterpret_cast<float *>(sm + L_::PMK);
    float *comp = reinterpret_cast<float *>(sm + L_::COMP);
    float *mur = reinterpret_cast<float *>(sm + L_::RS);
    float *r_s = mur + SC;
    float *pst = reinterpret_cast<float *>(sm + L_::PST);
    int *ctl = reinterpret_cast<int *>(sm + L_::PST + DK * 4);   // [0] ticket, [1] flag, [2] abort

    const Tin *__restrict__ kin = static_cast<const Tin *>(a.k);
    const Tin *__restrict__ ain = static_cast<const Tin *>(a.alpha);
    const Tin *__restrict__ sin_ = static_cast<const Tin *>(a.sigma);
    const Tin *__restrict__ rin = static_cast<const Tin *>(a.r);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H;
    const long long units = (long long)a.nchunks_max * a.nchains;

    for (;;) {
        if (tid == 0) ctl[0] = (int)atomicAdd(a.counter, 1u);
        __syncthreads();
        const long long u = ctl[0];
        __syncthreads();
        if (u >= units) break;
        const int c = (int)(u / a.nchains), chain = (int)(u % a.nchains);
        const int s = chain / H, h = chain % H;
        int t0, t1;
        if (a.cu) { t0 = __ldg(a.cu + s); t1 = __ldg(a.cu + s + 1); } else { t0 = s * a.T; t1 = t0 + a.T; }
        const int nch = (t1 - t0 + SC - 1) / SC;
        if (c == 0 && tid == 0 && nch > a.nchunks_max) raise_error(a.err, ERR_ARG);
        if (c >= nch) continue;
        const int c0 = t0 + c * SC, L = min(SC, t1 - c0);

        // ---- stage the chunk's alpha, sigma, k (rows t < L) and mu / r
        {
            constexpr int VEC = 16 / sizeof(Tin), NV = DK / VEC;
            for (int e = tid; e < L * NV; e += SNT) {
                const int t = e / NV, v = e % NV;
                const size_t g = ((size_t)(c0 + t) * H + h) * DK + v * VEC;
                reinterpret_cast<uint4 *>(al_s + t * DK)[v] = __ldg(reinterpret_cast<const uint4 *>(ain + g));
                reinterpret_cast<uint4 *>(sg_s + t * DK)[v] = __ldg(reinterpret_cast<const uint4 *>(sin_ + g));
                reinterpret_cast<uint4 *>(k_s + t * DK)[v] = __ldg(reinterpret_cast<const uint4 *>(kin + g));
            }
            if (tid < SC) {
                const float rr = tid < L ? ldf(rin + (size_t)(c0 + tid) * H + h) : 1.f;
                r_s[tid] = rr;
                mur[tid] = a.mu / rr;
            }
        }
        __syncthreads();

        // ---- segment composites: thread = (channel pair, segment)
        const int cp = tid % NCP, sgi = tid / NCP, ch = cp * 2;
        const int tb = sgi * SEG, te = min(L, tb + SEG);
        {
            float m[2][4] = {{1.f, 0.f, 0.f, 1.f}, {1.f, 0.f, 0.f, 1.f}};
            for (int t = tb; t < te; ++t) {
                const float mr = mur[t];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float al = to_f(al_s[t * DK + ch + q]), sg = to_f(sg_s[t * DK + ch + q]);
                    const float kk = to_f(k_s[t * DK + ch + q]);
                    const float aa = al * al, cc = mr * kk * kk;
                    const float y00 = fmaf(aa, m[q][0], sg * m[q][2]), y01 = fmaf(aa, m[q][1], sg * m[q][3]);
                    m[q][2] = fmaf(cc, y00, m[q][2]);
                    m[q][3] = fmaf(cc, y01, m[q][3]);
                    m[q][0] = y00;
                    m[q][1] = y01;
                }
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float sc = 1.f / m[q][3];
                float *cpm = comp + ((size_t)sgi * DK + ch + q) * 4;
                cpm[0] = m[q][0] * sc; cpm[1] = m[q][1] * sc; cpm[2] = m[q][2] * sc; cpm[3] = 1.f;
            }
        }
        __syncthreads();

        // ---- chunk aggregate (thread = channel) and its publication
        float g00 = 1.f, g01 = 0.f, g10 = 0.f, g11 = 1.f;
        float *desc = a.desc + (size_t)u * 4 * DK;
        if (tid < DK) {
            for (int q = 0; q < NSEG; ++q) {
                const float *cm = comp + ((size_t)q * DK + tid) * 4;
                const float n00 = fmaf(cm[0], g00, cm[1] * g10), n01 = fmaf(cm[0], g01, cm[1] * g11);
                const float n10 = fmaf(cm[2], g00, cm[3] * g10), n11 = fmaf(cm[2], g01, cm[3] * g11);
                const float sc = 1.f / n11;
                g00 = n00 * sc; g01 = n01 * sc; g10 = n10 * sc; g11 = 1.f;
            }
            if (c > 0) {
                __stcg(desc + 0 * DK + tid, g00);
                __stcg(desc + 1 * DK + tid, g01);
                __stcg(desc + 2 * DK + tid, g10);
            }
        }
        if (c > 0) {
            __threadfence();
            __syncthreads();
            if (tid == 0) atomicExch(a.flags + u, FLAG_AGG);
        }

        // ---- look-back for the chunk's starting uncertainty
        if (c == 0) {
            if (tid < DK) pst[tid] = a.P0 ? a.P0[(size_t)chain * DK + tid] : 1.f;
        } else {
            // walk back to the nearest chunk whose end-of-chunk uncertainty is published, then
            // forward through the aggregates of the chunks in between, each applied as its owner
            // applies it: the start value does not depend on which flags were set when
            int j = c - 1, f = FLAG_NONE;
            for (;;) {
                const long long uj = (long long)j * a.nchains + chain;
                if (tid == 0) {
                    volatile int *fp = a.flags + uj;
                    int fl = *fp;
                    const long long tstart = clock64();
                    while (fl == FLAG_NONE) {
                        // give up after ~1 s, or at once when another wait already gave up
                        if (clock64() - tstart > 2000000000ll || (a.err && (*(volatile unsigned *)a.err & ERR_TIMEOUT))) break;
                        __nanosleep(64);
                        fl = *fp;
                    }
                    if (fl == FLAG_NONE) { raise_error(a.err, ERR_TIMEOUT); fl = -1; }
                    ctl[1] = fl;
                }
                __syncthreads();
                f = ctl[1];
                __syncthreads();   // ctl[1] is read by every thread before it is replaced
                if (f == FLAG_INCL || f < 0) break;
                --j;
            }
            __threadfence();
            if (tid < DK) {
                float x = 1.f;
                if (f >= 0) {
                    x = __ldcg(a.desc + ((size_t)((long long)j * a.nchains + chain) * 4 + 3) * DK + tid);
                    for (int jj = j + 1; jj < c; ++jj) {   // aggregates whose flags the walk saw
                        const float *dq = a.desc + (size_t)((long long)jj * a.nchains + chain) * 4 * DK;
                        x = mob(__ldcg(dq + tid), __ldcg(dq + DK + tid), __ldcg(dq + 2 * DK + tid), 1.f, x);
                    }
                }
                pst[tid] = x;
            }
        }
        __syncthreads();
        // ---- publish the end-of-chunk uncertainty
        if (tid < DK) {
            const float pe = mob(g00, g01, g10, g11, pst[tid]);
            __stcg(desc + 3 * DK + tid, pe);
            if (c == nch - 1 && a.P_out) a.P_out[(size_t)chain * DK + tid] = pe;
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) atomicExch(a.flags + u, FLAG_INCL);

        // ---- re-expansion: P^- k per token and channel (thread = channel pair x segment)
        {
            float P[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float x = pst[ch + q];
                for (int q2 = 0; q2 < sgi; ++q2) {
                    const float *cm = comp + ((size_t)q2 * DK + ch + q) * 4;
                    x = mob(cm[0], cm[1], cm[2], cm[3], x);
                }
                P[q] = x;
            }
            for (int t = tb; t < te; ++t) {
                const float mr = mur[t];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float al = to_f(al_s[t * DK + ch + q]), sg = to_f(sg_s[t * DK + ch + q]);
                    const float kk = to_f(k_s[t * DK + ch + q]);
                    const float pm = fmaf(al * al, P[q], sg);
                    const float pk = pm * kk;
                    pmk[t * DK + ch + q] = pk;
                    P[q] = pm / fmaf(mr * kk, pk, 1.f);
                }
            }
        }
        __syncthreads();
        // ---- gain denominators, gain and k^T g (warp per token row)
        for (int t = warp; t < L; t += SNT / 32) {
            constexpr int PER = DK / 32;
            float x = 0.f, pv[PER];
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                const int chh = lane * PER + e;
                pv[e] = pmk[t * DK + chh];
                x = fmaf(pv[e], to_f(k_s[t * DK + chh]), x);
            }
            x = warp_sum(x);
            const float inv = 1.f / (r_s[t] + x);
            const size_t th = (size_t)(c0 + t) * H + h;
            if (a.g) {
                float *gd = a.g + th * DK + lane * PER;
#pragma unroll
                for (int e = 0; e < PER; ++e) gd[e] = pv[e] * inv;
            }
            if (a.beta && lane == 0) a.beta[th] = x * inv;
        }
        __syncthreads();
    }
}

template <int DK, typename Tin>
static cudaError_t launch_scan_t(const ScanArgs &a, cudaStream_t st) {
    constexpr size_t smem = ScanSmem<DK, Tin>::total;
    auto kern = gain_scan_kernel<DK, Tin>;
    KernelSetup ks;
    cudaError_t e = kernel_setup(reinterpret_cast<const void *>(kern), smem, SNT, false, &ks);
    if (e != cudaSuccess) return e;
    const long long units = (long long)a.nchunks_max * a.nchains;
    long long grid = (long long)ks.sms * (ks.blocks_per_sm > 0 ? ks.blocks_per_sm : 1);
    if (grid > units) grid = units;
    if (grid < 1) grid = 1;
    kern<<<(unsigned)grid, SNT, smem, st>>>(a);
    return cudaGetLastError();
}

size_t scan_workspace_bytes(long long nchains, long long nchunks_max, int dk) {
    const long long units = nchains * nchunks_max;
    const size_t flags = ((size_t)units * 4 + 255) / 256 * 256;
    const size_t generic = 256 + flags + (size_t)units * 4 * dk * 4;
    const size_t tma = dk == 128 ? scan_tma_workspace_bytes(nchains, nchunks_max) : 0;
    return generic > tma ? generic : tma;
}

cudaError_t launch_gain_scan(ScanArgs a, bool bf16_in, long long ntok, void *workspace, cudaStream_t st) {
    if (a.nchains == 0 || a.nchunks_max == 0) return cudaSuccess;
    if (gain_scan_tma_supported(a.dk, bf16_in)) return launch_gain_scan_tma(a, ntok, workspace, st);
    const long long units = (long long)a.nchains * a.nchunks_max;
    const size_t flags = ((size_t)units * 4 + 255) / 256 * 256;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    a.counter = reinterpret_cast<unsigned *>(ws);
    a.flags = reinterpret_cast<int *>(ws + 256);
    a.desc = reinterpret_cast<float *>(ws + 256 + flags);
    cudaError_t e = cudaMemsetAsync(ws, 0, 256 + flags, st);   // ticket counter and chunk flags
    if (e != cudaSuccess) return e;
    switch (a.dk * 2 + (bf16_in ? 1 : 0)) {
        case 64: return launch_scan_t<32, float>(a, st);
        case 65: return launch_scan_t<32, bf16>(a, st);
        case 128: return launch_scan_t<64, float>(a, st);
        case 129: return launch_scan_t<64, bf16>(a, st);
        case 256: return launch_scan_t<128, float>(a, st);
        case 257: return launch_scan_t<128, bf16>(a, st);
    }
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- allocation-free variant
// Scratch of kdn_gain_scan_noalloc: a fixed device array (one copy on every GPU that loads
// the library, held until the process exits) used instead of a caller-provided workspace.
constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;
static __device__ __align__(256) unsigned char g_scan_scratch[kNoAllocScratchBytes];

// Device address of the current GPU's scratch array.  In host code the array's name only
// stands for the symbol, so the address is looked up once per device and context (with that
// device current) and cached.
static cudaError_t scratch_address(void **out) {
    return symbol_address(reinterpret_cast<const void *>(&g_scan_scratch), out);
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t launch_gain_scan_noalloc(const ScanArgs &a, bool bf16_in, long long ntok, cudaStream_t st) {
    void *ws = nullptr;
    cudaError_t e = scratch_address(&ws);
    if (e != cudaSuccess) return e;
    return launch_gain_scan(a, bf16_in, ntok, ws, st);   // clears the ticket counter and flags it uses
}

}  // namespace kdn
