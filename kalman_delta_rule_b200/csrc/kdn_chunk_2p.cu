// Chunkwise Diagonal-KDN forward in two launches on the tcgen05 tensor cores (KDA article,
// "chunkwise" regime; explainer "对角近似" for the diagonal uncertainty and, closing
// paragraph of "各向同性近似", the Moebius form of its recursion).
//
// Everything of a chunk that does not involve the memory S is independent across chunks
// once the uncertainty at the chunk start is known, and that uncertainty comes from an
// associative (Moebius) scan.  So the work splits into
//
//   prep  (one unit = one 64-token chunk of one (sequence, head); every unit in parallel):
//         compose the chunk's 2x2 uncertainty maps, take the starting uncertainty from the
//         chunk's predecessors by decoupled look-back, re-expand P^- per token, form the
//         decayed operands and 1/den, then [A; Aq] (the intra-chunk interaction matrices with
//         their pairwise decay), T = (I + A)^{-1}, X = Aq T, [w; X K~] = [T; X] K~, and write
//         one record per unit: [-w; Q'] (Q' = Q~ - X K~), [T; X], G', 1/den, Gam_L;
//   state (one CTA per (sequence, head, d_v tile); chunks in order):
//         [U; O] = [-w; Q'] S + [T; X] V,   S <- Gam_L S + G'^T (U / den).
// Here Gam_t is the decay from the chunk start through token t (per channel), Gam_L the whole
// chunk's, K~ = k Gam_t, Q~ = q Gam_t and G' = P^- k Gam_L / Gam_t: every operand of the state
// kernel is at most its undecayed value, whatever the decay.  A and Aq are formed on the tensor
// cores from operands referenced to the chunk end when every channel's Gam_L >= 2^-100, else on
// the CUDA cores from log-space pairwise decay factors, so any alpha in [0, 1] is in range.
//
// Records are stored exactly in the state kernel's shared-memory operand layout (128-byte
// swizzled atoms), so the state kernel fetches each with one bulk copy, double-buffered,
// and its per-chunk critical path is two MMAs and two TMEM epilogues.
//
// Isotropic KDN (one uncertainty per head): the prep first sums alpha^2, sigma and k^2 over the
// channels of every token; each channel then carries the head's map (channel means) through the
// same composite / look-back / re-expansion machinery, and the records are the same.
//
// The prep kernel runs two 256-thread CTAs per SM; work is handed out by a ticket counter
// in chunk-major order, so every predecessor of a unit belongs to a CTA that is already
// running, and every wait is bounded (a wait that gives up records KDN_ERR_TIMEOUT).
#include <mutex>

#include "kdn_common.cuh"
#include "kdn_launch.h"
#include "kdn_tc.cuh"

namespace kdn {

namespace {
constexpr int C = 64, DK = 128, PNT = 256, SNT = 256;
constexpr int ADS = 36;   // padded fp32 row stride of the diagonal blocks (conflict-free row-wise float4 access)
constexpr int XLD = 65;   // padded row stride (words) of the out-of-range path's [channel][token] staging
// A chunk whose decay Gam_L (product of its alphas) is at least this on every channel takes the
// factored tensor-core form (operands up to 1 / Gam_L); below it, the pairwise CUDA-core form.
constexpr float kMinChunkDecay = 0x1p-100f;

// one unit's record; each part in the state kernel's operand layout
struct Rec {
    static constexpr uint32_t A4 = 0;          // [-w; Q'] bf16: 2 channel atoms x 128 rows x 128 B
    static constexpr uint32_t Y = 32768;       // [T; X] bf16: 128 rows x 64 tokens
    static constexpr uint32_t G = 49152;       // G' bf16: 2 channel atoms x 64 token rows
    static constexpr uint32_t MISC = 65536;    // 1/den [64] fp32, then Gam_L [128] fp32
    static constexpr uint32_t BYTES = MISC + 768;
};

struct PrepSmem {
    static constexpr uint32_t KQ = 0;                  // [K; Q] decayed bf16, 2 channel atoms x 128 rows
    static constexpr uint32_t G = 32768;               // G' bf16 (record part)
    static constexpr uint32_t W = 49152;               // work region, reused phase by phase:
    static constexpr uint32_t COMP = W;                //   segment composites fp32 [4][128][4]
    static constexpr uint32_t AQ = W;                  //   Aq bf16 64 x 64
    static constexpr uint32_t DB = W + 8192;           //   D bf16 64 x 64 (the two 32x32 diagonal-block inverses)
    static constexpr uint32_t LB = W + 16384;          //   L: A's lower-left 32x32 block
    static constexpr uint32_t NB = W + 24576;          //   I - N, N = D L
    static constexpr uint32_t ADG = W + 32768;         //   fp32 [2][32][ADS]: A's diagonal blocks, then D's
    static constexpr uint32_t A4 = W;                  //   [-w; Q'] (record part), once the inverse is done
    static constexpr uint32_t Y = W + 43008;           //   [T; X] (record part)
    static constexpr uint32_t MISC = W + 59392;        // 1/den [64], Gam_L [128] (record tail)
    static constexpr uint32_t RS = MISC + 768;         // r [64]
    static constexpr uint32_t MUR = RS + 256;          // mu / r [64]
    static constexpr uint32_t PST = MUR + 256;         // uncertainty at the chunk start [128]
    static constexpr uint32_t DSUM = PST + 512;        // sum_i P^- k^2 per token [64]
    static constexpr uint32_t TSUM = DSUM + 256;       // isotropic: per-token sums of alpha^2, sigma, k^2 [64][4]
    static constexpr uint32_t HCOMP = TSUM + 1024;     // isotropic: the head map's segment composites [4][4]
    static constexpr uint32_t CTL = HCOMP + 64;        // mbarrier, ticket, TMEM slot, flags
    static constexpr uint32_t total = CTL + 64;
    // out-of-range units (pairwise decay on the CUDA cores), staged one half of the channels at a time
    static constexpr uint32_t XKQ = 0;                 // (k, q) bf16 pairs [64][XLD], over K~/Q~
    static constexpr uint32_t XPK = XKQ + 64 * XLD * 4;  // P^- k fp32 [64][XLD]
    static constexpr uint32_t XLG = W + 8192;          // log2 decay from the chunk start fp32 [64][XLD]
    static constexpr uint32_t LSUM = W + 26624;        // per-segment log2 decay sums [4][128]
    static constexpr uint32_t XAA = W + 8192;          // A (rows 0..63) and Aq fp32 [128][XLD], once staged
    static_assert(COMP + 4 * 128 * 16 <= DB, "composites overlap D");
    static_assert(ADG + 64 * ADS * 4 <= Y && Y + 16384 <= MISC && A4 + 32768 <= Y, "work region");
    static_assert(XPK + 64 * XLD * 4 <= W && XLG + 64 * XLD * 4 <= LSUM && LSUM + 2048 <= Y, "staging");
    static_assert(XAA + 128 * XLD * 4 <= Y, "A staging");
};

template <int DVT>
struct StateSmem {
    // operand tiles are 64-column swizzle atoms; a 32-column tile uses half of one
    static constexpr uint32_t W64 = DVT < 64 ? 64 : DVT;
    static constexpr uint32_t STAGE = 67584;               // a record, rounded up to 1 KB
    static constexpr uint32_t V_BYTES = W64 * 128;         // v tile (64 tokens x W64 columns)
    static constexpr uint32_t V0 = 2 * STAGE;              // two v tiles
    static constexpr uint32_t S = V0 + 2 * V_BYTES;        // S bf16, 128 channel rows x DVT (MN-major)
    static constexpr uint32_t U = S + W64 * 256;           // U / den bf16, 64 token rows x DVT
    static constexpr uint32_t CTL = U + W64 * 128;         // 3 mbarriers, TMEM slot
    static constexpr uint32_t total = CTL + 64;
};

// Units of packed (varlen) problems are numbered densely, chunk-major over the chunks that exist,
// with the sequences of each chunk level in order of length (longest first):
//     unit (c, s, h) = U[c] + pos[s] * H + h      (for c < the sequence's chunk count)
// U[c] = H x #{(c', s) : c' < c, chunks(s) > c'}; pos = rank of s by chunk count, order = pos^-1.
// Dense batches use unit = c * nchains + chain.
struct UnitTable {
    long long *U;      // [cmax + 1]; U[cmax] = number of units
    int *order, *pos;  // [nseq]
    int *hist, *fill;  // [cmax + 1] scratch of the table kernel
    int cmax;          // ceil(T / 64): bounds every sequence's chunk count
};

struct PrepArgs {
    TokenArgs a;
    long long nchunks_max;
    int nchains;
    unsigned *counter;
    unsigned long long *desc;   // per unit [4][128] tagged words: aggregate map (m00, m01, m10), end-of-chunk P
    uint8_t *rec;     // per unit Rec::BYTES
    const long long *U;         // varlen unit table (NULL: dense numbering)
    const int *order, *pos;
    int cmax;
};

struct StateArgs {
    TokenArgs a;
    CUtensorMap tv;
    const uint8_t *rec;
    long long nchunks_max;
    int nchains;
    const long long *U;         // varlen unit table (NULL: dense numbering)
    const int *order;
};

__device__ __forceinline__ float mob(float m00, float m01, float m10, float m11, float x) {
    return fmaf(m00, x, m01) / fmaf(m10, x, m11);
}

__device__ __forceinline__ uint4 pack8(const float *v, float sc = 1.f) {
    uint4 w;
    w.x = tc::pack_bf16x2(v[0] * sc, v[1] * sc);
    w.y = tc::pack_bf16x2(v[2] * sc, v[3] * sc);
    w.z = tc::pack_bf16x2(v[4] * sc, v[5] * sc);
    w.w = tc::pack_bf16x2(v[6] * sc, v[7] * sc);
    return w;
}

__device__ __forceinline__ uint32_t ldg_u32(const bf16 *p) { return __ldg(reinterpret_cast<const unsigned *>(p)); }

// a bf16 pair (low half = channel ch) widened to f32x2
__device__ __forceinline__ f32x2 bf2(uint32_t w) { return pk2(tc::bf16_lo(w), tc::bf16_hi(w)); }

// Failure paths: after a bounded wait gave up, one more bounded wait for the tcgen05 operations
// (a fresh commit covers every earlier one) or the copy a CTA issued, before its tensor and shared
// memory are released.  Out of line, so the kernels' register allocation does not carry them.
__device__ __noinline__ void drain_mma(uint64_t *bar, uint32_t phase) {
    tc::mma_commit(bar);
    tc::mbar_wait(bar, phase);
}
__device__ __noinline__ void drain_copy(uint64_t *bar, uint32_t parity) { tc::mbar_wait(bar, parity); }

// Look-back descriptors are 64-bit words (value, tag): each word carries its own status, so a
// reader that sees a tag also sees that word's value, with no fence between writer and flag.
enum : unsigned { TAG_NONE = 0, TAG_AGG = 1, TAG_INCL = 2 };
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

// one token of the uncertainty walk on a key-channel pair's bf16 words (alpha, sigma, k):
// returns P^- of the pair and advances P (isotropic: the head's map from the token sums)
template <bool ISO>
__device__ __forceinline__ f32x2 uncertainty_step(const float *mur, const float *tsum, int t, uint32_t aa,
                                                  uint32_t ss, uint32_t kk2, float &Pa, float &Pb) {
    if constexpr (!ISO) {   // both channels of the pair at once (f32x2)
        const f32x2 al = bf2(aa), kk = bf2(kk2);
        const f32x2 pm = fma2(mul2(al, al), pk2(Pa, Pb), bf2(ss));
        const float mr = mur[t];
        const f32x2 dn = fma2(mul2(mul2(pk2(mr, mr), kk), kk), pm, pk2(1.f, 1.f));
        Pa = __fdividef(x2(pm), x2(dn));
        Pb = __fdividef(y2(pm), y2(dn));
        return pm;
    } else {   // the head's map, the same on every channel
        const float4 iso = *reinterpret_cast<const float4 *>(tsum + t * 4);
        const float pma = fmaf(iso.x, Pa, iso.y), pmb = fmaf(iso.x, Pb, iso.y);
        Pa = __fdividef(pma, fmaf(iso.z, pma, 1.f));
        Pb = __fdividef(pmb, fmaf(iso.z, pmb, 1.f));
        return pk2(pma, pmb);
    }
}

// What the out-of-range form of a prep unit needs from the kernel (thread = key-channel pair
// ch, ch + 1 x 16-token segment sgi starting at token tb of the chunk).
struct PairwiseCtx {
    uint8_t *sm;
    const bf16 *q, *k, *alpha, *sigma;
    const float *mur, *tsum;
    float *lsum, *dsum;
    int tid, warp, ch, tb, sgi, L, c0, h, H;
    uint32_t atom16, atom8, bch;
    float Ps_a, Ps_b;   // uncertainty of the pair at the segment start
};

// A unit whose chunk decay leaves the factored range (some channel's Gam_L < 2^-100: an alpha = 0
// reset, or strong decay): A and Aq are formed on the CUDA cores with every pairwise decay factor
// 2^(lg_t - lg_s) <= 1 from log-space sums lg_t = sum log2 max(alpha, 2^-126) (a zero decay acts as
// 2^-126, so a factor across it is below 2^-126 instead of 0), written fp32 to XAA (rows 0..63 A,
// 64..127 Aq, before the 1/den column scale); then the operands referenced to the chunk start, K~ =
// k Gam_t, Q~ = q Gam_t and G' = P^- k 2^(lg_L - lg_t), and the gain denominators' sums.  Kept out
// of line (rare path): the unit's tokens are re-read from global memory, and its registers do not
// weigh on the factored path's.
template <bool ISO>
__device__ __noinline__ void pairwise_unit(const PairwiseCtx &x) {
    using L_ = PrepSmem;
    using namespace tc;
    const int tid = x.tid, ch = x.ch, tb = x.tb, sgi = x.sgi, L = x.L, c0 = x.c0, h = x.h, H = x.H;
    auto lg2 = [](float al) { return __log2f(fmaxf(al, 0x1p-126f)); };
    auto tok = [&](const bf16 *base, int t) { return ldg_u32(base + ((size_t)(c0 + t) * H + h) * DK + ch); };
    {   // per-segment sums of log2 alpha
        float la = 0.f, lb = 0.f;
        for (int j = 0; j < 16; ++j)
            if (tb + j < L) {
                const uint32_t aa = tok(x.alpha, tb + j);
                la += lg2(bf16_lo(aa));
                lb += lg2(bf16_hi(aa));
            }
        x.lsum[sgi * 128 + ch] = la;
        x.lsum[sgi * 128 + ch + 1] = lb;
    }
    __syncthreads();
    float lga = 0.f, lgb = 0.f, lLa = 0.f, lLb = 0.f;   // at the segment start; over the chunk
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2) {
        const float xa = x.lsum[q2 * 128 + ch], xb = x.lsum[q2 * 128 + ch + 1];
        if (q2 < sgi) { lga += xa; lgb += xb; }
        lLa += xa;
        lLb += xb;
    }
    // A_ts = sum_i k_ti pk_si 2^(lg_ti - lg_si) (s < t), Aq_ts likewise with q (s <= t), one half of
    // the channels at a time staged as [channel][token]: (k, q) bf16 pairs, P^- k and lg in fp32.
    // Thread = token row tr x column set {sgc + 4 j}.
    uint32_t *kqr = reinterpret_cast<uint32_t *>(x.sm + L_::XKQ);
    float *pks = reinterpret_cast<float *>(x.sm + L_::XPK);
    float *lgs = reinterpret_cast<float *>(x.sm + L_::XLG);
    const int tr = tid & 63, sgc = tid >> 6;
    float accA[16], accQ[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) { accA[j] = 0.f; accQ[j] = 0.f; }
    for (int half = 0; half < 2; ++half) {
        if ((x.warp & 1) == half) {   // the owners of this half's channels stage their tokens
            float Pa = x.Ps_a, Pb = x.Ps_b, lta = lga, ltb = lgb;
            const int c2 = ch - 64 * half;
            for (int j = 0; j < 16; ++j) {
                const int t = tb + j;
                uint32_t kqa = 0u, kqb = 0u;
                float pka = 0.f, pkb = 0.f;
                if (t < L) {
                    const uint32_t aa = tok(x.alpha, t), kk2 = tok(x.k, t), qq2 = tok(x.q, t);
                    const f32x2 pm = uncertainty_step<ISO>(x.mur, x.tsum, t, aa, tok(x.sigma, t), kk2, Pa, Pb);
                    lta += lg2(bf16_lo(aa));
                    ltb += lg2(bf16_hi(aa));
                    pka = x2(pm) * bf16_lo(kk2);
                    pkb = y2(pm) * bf16_hi(kk2);
                    kqa = (kk2 & 0xffffu) | (qq2 << 16);
                    kqb = (kk2 >> 16) | (qq2 & 0xffff0000u);
                }
                kqr[c2 * XLD + t] = kqa;
                kqr[(c2 + 1) * XLD + t] = kqb;
                pks[c2 * XLD + t] = pka;
                pks[(c2 + 1) * XLD + t] = pkb;
                lgs[c2 * XLD + t] = lta;
                lgs[(c2 + 1) * XLD + t] = ltb;
            }
        }
        __syncthreads();
        if (tid < C) {   // this half's share of the gain denominators sum_i P^-_i k_i^2
            float acc = 0.f;
            for (int c2 = 0; c2 < 64; ++c2) acc = fmaf(pks[c2 * XLD + tid], bf16_lo(kqr[c2 * XLD + tid]), acc);
            x.dsum[tid] += acc;
        }
        for (int c2 = 0; c2 < 64; ++c2) {
            const uint32_t kq = kqr[c2 * XLD + tr];
            const float kt = bf16_lo(kq), qt = bf16_hi(kq), lt = lgs[c2 * XLD + tr];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int s_ = sgc + 4 * j;
                if (s_ <= tr) {
                    const float w = pks[c2 * XLD + s_] * exp2f(lt - lgs[c2 * XLD + s_]);
                    accA[j] = fmaf(kt, w, accA[j]);
                    accQ[j] = fmaf(qt, w, accQ[j]);
                }
            }
        }
        __syncthreads();
    }
    float *aaf = reinterpret_cast<float *>(x.sm + L_::XAA);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        aaf[tr * XLD + sgc + 4 * j] = accA[j];
        aaf[(64 + tr) * XLD + sgc + 4 * j] = accQ[j];
    }
    // the operands of the rest of the unit, referenced to the chunk start
    float Pa = x.Ps_a, Pb = x.Ps_b, lta = lga, ltb = lgb;
    for (int j = 0; j < 16; ++j) {
        const int t = tb + j;
        uint32_t kq = 0u, qq = 0u, gg = 0u;
        if (t < L) {
            const uint32_t aa = tok(x.alpha, t), kk2 = tok(x.k, t);
            const f32x2 pm = uncertainty_step<ISO>(x.mur, x.tsum, t, aa, tok(x.sigma, t), kk2, Pa, Pb);
            const f32x2 kk = bf2(kk2), qk = bf2(tok(x.q, t));
            lta += lg2(bf16_lo(aa));
            ltb += lg2(bf16_hi(aa));
            const float ga = exp2f(lta), gb = exp2f(ltb);
            kq = pack_bf16x2(x2(kk) * ga, y2(kk) * gb);
            qq = pack_bf16x2(x2(qk) * ga, y2(qk) * gb);
            gg = pack_bf16x2(x2(pm) * x2(kk) * exp2f(lLa - lta), y2(pm) * y2(kk) * exp2f(lLb - ltb));
        }
        *reinterpret_cast<uint32_t *>(x.sm + L_::KQ + x.atom16 + swz(t, x.bch)) = kq;
        *reinterpret_cast<uint32_t *>(x.sm + L_::KQ + x.atom16 + swz(64 + t, x.bch)) = qq;
        *reinterpret_cast<uint32_t *>(x.sm + L_::G + x.atom8 + swz(t, x.bch)) = gg;
    }
}

// ================================================================= prep
template <bool ISO, bool PACKED>
__global__ void __launch_bounds__(PNT, 2) chunk_prep_kernel(const __grid_constant__ PrepArgs pa)
{
    using L_ = PrepSmem;
    using namespace tc;
    extern __shared__ uint8_t smraw[];
    const uint32_t raw_u32 = smem_u32(smraw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
    uint8_t *sm = smraw + (sb - raw_u32);

    float *invden = reinterpret_cast<float *>(sm + L_::MISC);
    float *gamc = invden + 64;
    float *r_s = reinterpret_cast<float *>(sm + L_::RS);
    float *mur = reinterpret_cast<float *>(sm + L_::MUR);
    float *pst = reinterpret_cast<float *>(sm + L_::PST);
    float *dsum = reinterpret_cast<float *>(sm + L_::DSUM);
    float *tsum = reinterpret_cast<float *>(sm + L_::TSUM);
    float *lsum = reinterpret_cast<float *>(sm + L_::LSUM);
    float *hcomp = reinterpret_cast<float *>(sm + L_::HCOMP);
    float *comp = reinterpret_cast<float *>(sm + L_::COMP);
    float *adg = reinterpret_cast<float *>(sm + L_::ADG);
    uint64_t *bar_mma = reinterpret_cast<uint64_t *>(sm + L_::CTL);
    long long *ticket = reinterpret_cast<long long *>(sm + L_::CTL + 8);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L_::CTL + 16);
    int *ctl = reinterpret_cast<int *>(sm + L_::CTL + 20);   // [0] look-back flag, [1] abort, [2] out-of-range unit

    const TokenArgs &a = pa.a;
    const bf16 *__restrict__ qin = static_cast<const bf16 *>(a.q);
    const bf16 *__restrict__ kin = static_cast<const bf16 *>(a.k);
    const bf16 *__restrict__ ain = static_cast<const bf16 *>(a.alpha);
    const bf16 *__restrict__ sin_ = static_cast<const bf16 *>(a.sigma);
    const bf16 *__restrict__ rin = static_cast<const bf16 *>(a.r);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, cg = warp >> 2;     // TMEM lane quadrant, column half
    const int H = a.H;
    constexpr bool packed = PACKED;   // packed (varlen) unit numbering through the unit table
    const long long units = packed ? pa.U[pa.cmax] : pa.nchunks_max * pa.nchains;
    int level = 0;   // packed: this CTA's chunk level (its tickets only grow)

    // the state kernel (launched next, as a programmatic dependent) may start its prologue
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid == 0) {
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        ctl[1] = 0;
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t T_A = *tmem_slot;
    const uint32_t lane_off = ((uint32_t)quad * 32u) << 16;
    const int row = quad * 32 + lane;     // TMEM lane of this thread in M=128 epilogues
    const int m64 = quad * 16 + lane;     // row of an M=64 accumulator (lanes < 16)
    uint32_t mma_phase = 0;

    constexpr uint32_t ID_M128_N64_KK = idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_M64_N64_KM = idesc_bf16(64, 64, false, true);
    constexpr uint32_t ID_M128_N128_KM = idesc_bf16(128, 128, false, true);

    auto wait_mma = [&]() {
        if (!mbar_wait(bar_mma, mma_phase)) atomicExch(&ctl[1], 1);
        mma_phase ^= 1u;
        tc_fence_after();
    };
    auto sync_tc = [&]() {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
    };
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
    // 64 x 64 bf16 tile from an M=64 accumulator: row m sits in lane (m % 16) + 32 (m / 16)
    auto store64 = [&](uint32_t dst, int row0, const float (&v)[32]) {
        if (lane < 16) {
#pragma unroll
            for (int chn = 0; chn < 4; ++chn)
                *reinterpret_cast<uint4 *>(sm + dst + swz(row0 + m64, (cg * 4 + chn) * 16)) = pack8(v + chn * 8);
        }
    };

    // unit u -> its chunk c, chain, rank among the packed sequences, and the chain's token range
    auto decode = [&](long long u, int &lvl, int &c, int &chain, int &rank, int &t0, int &t1) {
        rank = 0;
        if constexpr (PACKED) {
            while (lvl < pa.cmax && pa.U[lvl + 1] <= u) ++lvl;
            c = lvl;
            const int idx = (int)(u - pa.U[c]);
            rank = idx / H;
            chain = pa.order[rank] * H + idx % H;
        } else {
            c = (int)(u / pa.nchains);
            chain = (int)(u % pa.nchains);
        }
        seq_range(a, chain / H, t0, t1);
    };
    for (;;) {
        if (tid == 0) {
            *ticket = (long long)atomicAdd(pa.counter, 1u);
            ctl[2] = 0;   // the unit's decay-range class (set below when it leaves the factored range)
        }
        __syncthreads();
        const long long u = *ticket;
        if (u >= units || ctl[1]) break;
        int c, chain, rank, t0, t1;
        decode(u, level, c, chain, rank, t0, t1);
        const int h = chain % H;
        const int nch = (t1 - t0 + C - 1) / C;
        if (!packed && c == 0 && tid == 0 && nch > pa.nchunks_max) raise_error(a.err, ERR_ARG);
        if (c >= nch) {
            __syncthreads();   // every thread has read the ticket before it is replaced
            continue;
        }
        const int c0 = t0 + c * C, L = min(C, t1 - c0);

        if (tid < C) {
            const float rr = tid < L ? ldf(rin + (size_t)(c0 + tid) * H + h) : 1.f;
            r_s[tid] = rr;
            mur[tid] = a.mu / rr;
            dsum[tid] = 0.f;
            if (ISO) *reinterpret_cast<float4 *>(tsum + tid * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // thread = key-channel pair cp x 16-token segment sgi; alpha, sigma, k of its tokens
        const int cp = (warp & 1) * 32 + lane, sgi = warp >> 1, ch = cp * 2, tb = sgi * 16;
        float hexcl[4];   // isotropic, warp 0: the head map composed over the tokens before 2 lane
        uint32_t aw[16], sw[16], kw[16], qw[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            aw[j] = 0u; sw[j] = 0u; kw[j] = 0u;
            if (tb + j < L) {
                const size_t e = ((size_t)(c0 + tb + j) * H + h) * DK + ch;
                aw[j] = ldg_u32(ain + e);
                sw[j] = ldg_u32(sin_ + e);
                kw[j] = ldg_u32(kin + e);
            }
        }
        if (tid == 0) bulk_wait_read0();   // the previous record's bulk stores have read shared memory
        __syncthreads();

        // isotropic (explainer "各向同性近似"): every channel carries the head's uncertainty, with
        // the maps of the channel means a = mean alpha^2, s = mean sigma, c = mu |k|^2 / (d_k r)
        if constexpr (ISO) {
            float xa[16], xg[16], xk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float a0 = bf16_lo(aw[j]), a1 = bf16_hi(aw[j]), k0 = bf16_lo(kw[j]), k1 = bf16_hi(kw[j]);
                xa[j] = fmaf(a0, a0, a1 * a1);
                xg[j] = bf16_lo(sw[j]) + bf16_hi(sw[j]);
                xk[j] = fmaf(k0, k0, k1 * k1);
            }
            int which;
            const float sa_ = warp_reduce16(xa, lane, which);
            const float sg_ = warp_reduce16(xg, lane, which);
            const float sk_ = warp_reduce16(xk, lane, which);
            if ((lane & 1) == 0 && tb + which < L) {
                atomicAdd(tsum + (tb + which) * 4 + 0, sa_);
                atomicAdd(tsum + (tb + which) * 4 + 1, sg_);
                atomicAdd(tsum + (tb + which) * 4 + 2, sk_);
            }
            __syncthreads();
            if (tid < C) {   // the token's map parameters, in place
                constexpr float inv_dk = 1.f / DK;
                const float4 x = *reinterpret_cast<const float4 *>(tsum + tid * 4);
                *reinterpret_cast<float4 *>(tsum + tid * 4) =
                    make_float4(x.x * inv_dk, x.y * inv_dk, mur[tid] * x.z * inv_dk, x.z);
            }
            __syncthreads();
        }
        // ---- segment composites of the uncertainty maps (predict [[a, s],[0,1]], update [[1,0],[c,1]])
        if constexpr (!ISO) {   // both channels of the pair at once (f32x2)
            f32x2 m00 = pk2(1.f, 1.f), m01 = pk2(0.f, 0.f), m10 = m01, m11 = m00, gm = m00;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (tb + j < L) {
                    const float mr = mur[tb + j];
                    const f32x2 al = bf2(aw[j]), kk = bf2(kw[j]), sg = bf2(sw[j]);
                    const f32x2 aa = mul2(al, al), cc = mul2(mul2(pk2(mr, mr), kk), kk);
                    const f32x2 y00 = fma2(aa, m00, mul2(sg, m10)), y01 = fma2(aa, m01, mul2(sg, m11));
                    m10 = fma2(cc, y00, m10); m11 = fma2(cc, y01, m11); m00 = y00; m01 = y01; gm = mul2(gm, al);
                }
            }
            const float sa = 1.f / x2(m11), sbb = 1.f / y2(m11);
            *reinterpret_cast<float4 *>(comp + (sgi * 128 + ch) * 4) = make_float4(x2(m00) * sa, x2(m01) * sa, x2(m10) * sa, x2(gm));
            *reinterpret_cast<float4 *>(comp + (sgi * 128 + ch + 1) * 4) = make_float4(y2(m00) * sbb, y2(m01) * sbb, y2(m10) * sbb, y2(gm));
        } else {
            // isotropic: the per-channel decay products, and (one thread per segment) the head map's
            // composite -- the same map on every channel, so it is composed once
            float ga = 1.f, gb = 1.f;
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (tb + j < L) { ga *= bf16_lo(aw[j]); gb *= bf16_hi(aw[j]); }
            comp[(sgi * 128 + ch) * 4 + 3] = ga;
            comp[(sgi * 128 + ch + 1) * 4 + 3] = gb;
            if (warp == 0) {   // the head map's prefix composites over the chunk: lane l = tokens 2l, 2l + 1
                // map of token t: x -> (a x + s) / (c (a x + s) + 1), the matrix [[a, s], [c a, c s + 1]]
                auto tmap = [&](int t, float (&m)[4]) {
                    if (t < L) {
                        const float4 iso = *reinterpret_cast<const float4 *>(tsum + t * 4);
                        m[0] = iso.x; m[1] = iso.y; m[2] = iso.z * iso.x; m[3] = fmaf(iso.z, iso.y, 1.f);
                    } else {
                        m[0] = 1.f; m[1] = 0.f; m[2] = 0.f; m[3] = 1.f;
                    }
                };
                // x <- y after x (2x2 product y x), normalised so that (1,1) = 1
                auto after = [](float (&x)[4], const float (&y)[4]) {
                    const float n00 = fmaf(y[0], x[0], y[1] * x[2]), n01 = fmaf(y[0], x[1], y[1] * x[3]);
                    const float n10 = fmaf(y[2], x[0], y[3] * x[2]), n11 = fmaf(y[2], x[1], y[3] * x[3]);
                    const float sc = 1.f / n11;
                    x[0] = n00 * sc; x[1] = n01 * sc; x[2] = n10 * sc; x[3] = 1.f;
                };
                float m[4], m1[4];
                tmap(2 * lane, m);
                tmap(2 * lane + 1, m1);
                after(m, m1);   // the lane's two tokens
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {   // inclusive scan over the lanes
                    float o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[e] = __shfl_up_sync(0xffffffffu, m[e], off);
                    if (lane >= off) {
                        float y[4] = {m[0], m[1], m[2], m[3]};
                        m[0] = o[0]; m[1] = o[1]; m[2] = o[2]; m[3] = o[3];
                        after(m, y);   // this lane's part after the earlier lanes'
                    }
                }
                // the lane's exclusive prefix (tokens before 2l), kept for the per-token pass below
#pragma unroll
                for (int e = 0; e < 4; ++e) hexcl[e] = __shfl_up_sync(0xffffffffu, m[e], 1);
                if (lane == 0) { hexcl[0] = 1.f; hexcl[1] = 0.f; hexcl[2] = 0.f; hexcl[3] = 1.f; }
                if (lane == 31) *reinterpret_cast<float4 *>(hcomp) = make_float4(m[0], m[1], m[2], m[3]);
            }
        }
        // q of the thread's tokens (consumed after the look-back)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            qw[j] = 0u;
            if (tb + j < L) qw[j] = ldg_u32(qin + ((size_t)(c0 + tb + j) * H + h) * DK + ch);
        }
        __syncthreads();

        // ---- warps 0-3 (thread = key channel): chunk aggregate, its publication and the
        //      decoupled look-back, every channel on its own.
        const uint32_t atom16 = (uint32_t)(ch >> 6) * 16384u, atom8 = (uint32_t)(ch >> 6) * 8192u;
        const uint32_t bch = (uint32_t)(ch & 63) * 2u;
        auto gamma_start = [&](float &ga, float &gb) {
            ga = 1.f;
            gb = 1.f;
            for (int q2 = 0; q2 < sgi; ++q2) {
                ga *= comp[(q2 * 128 + ch) * 4 + 3];
                gb *= comp[(q2 * 128 + ch + 1) * 4 + 3];
            }
        };
        if (warp < 4) {
            const int cc = tid;   // key channel
            {   // the chunk's decay Gam_L per channel, from the segments' decay products
                const float gl = comp[cc * 4 + 3] * comp[(128 + cc) * 4 + 3] * comp[(256 + cc) * 4 + 3] *
                                 comp[(384 + cc) * 4 + 3];
                gamc[cc] = gl;
                if (!(gl >= kMinChunkDecay)) ctl[2] = 1;
            }
        }
        if (warp < 4 && (!ISO || tid == 0)) {   // isotropic: one uncertainty per head, one walk
            const int cc = tid;   // key channel
            unsigned long long *desc = pa.desc + (size_t)u * 4 * DK + cc;
            float g00 = 1.f, g01 = 0.f, g10 = 0.f, g11 = 1.f;
            if constexpr (ISO) {   // the whole chunk's head map, from the scan
                g00 = hcomp[0]; g01 = hcomp[1]; g10 = hcomp[2];
            } else {
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const float4 cm = *reinterpret_cast<const float4 *>(comp + (q2 * 128 + cc) * 4);
                    const float n00 = fmaf(cm.x, g00, cm.y * g10), n01 = fmaf(cm.x, g01, cm.y * g11);
                    const float n10 = fmaf(cm.z, g00, g10), n11 = fmaf(cm.z, g01, g11);
                    const float sc = 1.f / n11;
                    g00 = n00 * sc; g01 = n01 * sc; g10 = n10 * sc; g11 = 1.f;
                }
            }
            if (c > 0) {   // publish the aggregate
                st_relaxed(desc + 0 * DK, tagged(g00, TAG_AGG));
                st_relaxed(desc + 1 * DK, tagged(g01, TAG_AGG));
                st_relaxed(desc + 2 * DK, tagged(g10, TAG_AGG));
            }
            float p0;
            if (c == 0) {
                p0 = a.P0 ? a.P0[ISO ? (size_t)chain : (size_t)chain * DK + cc] : 1.f;
            } else {   // walk back to the nearest published end-of-chunk uncertainty, then forward
                       // through the aggregates of the chunks in between, each applied as its owner
                       // applies it: the start value does not depend on which words were published
                       // when (bit-reproducible)
                auto words_of = [&](int j) {
                    const long long uj = packed ? pa.U[j] + (long long)rank * H + h : (long long)j * pa.nchains + chain;
                    return pa.desc + (size_t)uj * 4 * DK + cc;
                };
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
            st_relaxed(desc + 3 * DK, tagged(pe, TAG_INCL));
            if (c == nch - 1 && a.P_out) {
                if (!ISO) a.P_out[(size_t)chain * DK + cc] = pe;
                else if (cc == 0) a.P_out[chain] = pe;
            }
        }
        __syncthreads();

        // ---- re-expansion fused with the chunk operands: P^- per token (from the chunk-start
        //      uncertainty through the earlier segments' composites), the gain denominators'
        //      partial sums, and the decayed operands.
        //      In range (every channel's chunk decay Gam_L >= kMinChunkDecay) the operands are
        //      referenced to the chunk END: K' = k Gam_t / Gam_L and Q' = q Gam_t / Gam_L (between
        //      k and k / Gam_L), G' = P^- k Gam_L / Gam_t (at most P^- k), so MMA1's A = K' G'^T
        //      carries the pairwise decay Gam_t / Gam_s of every pair exactly, and MMA2 takes
        //      Gam_L back as a column scale.
        //      Out of range (an alpha = 0 reset, or strong decay) A and Aq are formed on the CUDA
        //      cores with every pairwise factor 2^(lg_t - lg_s) <= 1 taken from log-space decay
        //      sums, and the operands are referenced to the chunk START: K~ = k Gam_t, Q~ = q Gam_t,
        //      G' = P^- k 2^(lg_L - lg_t); every factor is at most 1, so nothing overflows.
        const bool out_of_range = ctl[2] != 0;   // CTA-uniform
        float Ps_a, Ps_b;   // uncertainty at the segment start
        if constexpr (ISO) {
            // warp 0: the head's P^- of every token from the chunk-start uncertainty and the exclusive
            // prefix maps, the gain denominators r + p^- |k|^2, and the uncertainty after each token
            float *ppost = lsum;   // [64]
            if (warp == 0) {
                float P = mob(hexcl[0], hexcl[1], hexcl[2], hexcl[3], pst[0]);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = 2 * lane + e;
                    if (t < L) {
                        const float4 iso = *reinterpret_cast<const float4 *>(tsum + t * 4);
                        const float pm = fmaf(iso.x, P, iso.y);
                        P = __fdividef(pm, fmaf(iso.z, pm, 1.f));
                        dsum[t] = pm;
                        invden[t] = __fdividef(1.f, fmaf(pm, iso.w, r_s[t]));
                    } else {
                        invden[t] = 0.f;
                    }
                    ppost[t] = P;
                }
            }
            __syncthreads();
            Ps_a = sgi == 0 ? pst[0] : ppost[tb - 1];
            Ps_b = Ps_a;
        } else {
            Ps_a = pst[ch];
            Ps_b = pst[ch + 1];
            for (int q2 = 0; q2 < sgi; ++q2) {
                const float4 ca = *reinterpret_cast<const float4 *>(comp + (q2 * 128 + ch) * 4);
                const float4 cb = *reinterpret_cast<const float4 *>(comp + (q2 * 128 + ch + 1) * 4);
                Ps_a = mob(ca.x, ca.y, ca.z, 1.f, Ps_a);
                Ps_b = mob(cb.x, cb.y, cb.z, 1.f, Ps_b);
            }
        }
        auto store_operands = [&](int t, uint32_t kq, uint32_t qq, uint32_t gg) {
            *reinterpret_cast<uint32_t *>(sm + L_::KQ + atom16 + swz(t, bch)) = kq;
            *reinterpret_cast<uint32_t *>(sm + L_::KQ + atom16 + swz(64 + t, bch)) = qq;
            *reinterpret_cast<uint32_t *>(sm + L_::G + atom8 + swz(t, bch)) = gg;
        };
        if (ISO && !out_of_range) {   // P^- of the head per token (dsum) and 1/den are ready
            float gama, gamb;
            gamma_start(gama, gamb);
            f32x2 up = pk2(__fdividef(gama, gamc[ch]), __fdividef(gamb, gamc[ch + 1]));
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int t = tb + j;
                uint32_t kq = 0u, qq = 0u, gg = 0u;
                if (t < L) {
                    const float pm = dsum[t];
                    const f32x2 kk = bf2(kw[j]);
                    up = mul2(up, bf2(aw[j]));
                    const f32x2 kg = mul2(kk, up), qg = mul2(bf2(qw[j]), up);
                    kq = pack_bf16x2(x2(kg), y2(kg));
                    qq = pack_bf16x2(x2(qg), y2(qg));
                    gg = pack_bf16x2(__fdividef(pm * x2(kk), x2(up)), __fdividef(pm * y2(kk), y2(up)));
                }
                store_operands(t, kq, qq, gg);
            }
        } else if (!out_of_range) {
            float Pa = Ps_a, Pb = Ps_b, gama, gamb;
            gamma_start(gama, gamb);
            // up = Gam_t / Gam_L, in [1, 2^100]: K' = k up, Q' = q up, G' = P^- k / up
            f32x2 up = pk2(gama / gamc[ch], gamb / gamc[ch + 1]);
            float xs[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int t = tb + j;
                uint32_t kq = 0u, qq = 0u, gg = 0u;
                xs[j] = 0.f;
                if (t < L) {
                    const f32x2 pm = uncertainty_step<ISO>(mur, tsum, t, aw[j], sw[j], kw[j], Pa, Pb);
                    const f32x2 kk = bf2(kw[j]);
                    up = mul2(up, bf2(aw[j]));
                    const f32x2 pk = mul2(pm, kk), kg = mul2(kk, up), qg = mul2(bf2(qw[j]), up);
                    kq = pack_bf16x2(x2(kg), y2(kg));
                    qq = pack_bf16x2(x2(qg), y2(qg));
                    gg = pack_bf16x2(__fdividef(x2(pk), x2(up)), __fdividef(y2(pk), y2(up)));
                    xs[j] = fmaf(x2(pk), x2(kk), y2(pk) * y2(kk));
                }
                store_operands(t, kq, qq, gg);
            }
            int which;
            const float tot = warp_reduce16(xs, lane, which);
            if ((lane & 1) == 0 && tb + which < L) atomicAdd(dsum + tb + which, tot);
        } else {
            PairwiseCtx x;
            x.sm = sm; x.q = qin; x.k = kin; x.alpha = ain; x.sigma = sin_;
            x.mur = mur; x.tsum = tsum; x.lsum = lsum; x.dsum = dsum;
            x.tid = tid; x.warp = warp; x.ch = ch; x.tb = tb; x.sgi = sgi; x.L = L; x.c0 = c0; x.h = h; x.H = H;
            x.atom16 = atom16; x.atom8 = atom8; x.bch = bch; x.Ps_a = Ps_a; x.Ps_b = Ps_b;
            pairwise_unit<ISO>(x);
        }
        __syncthreads();
        if (tid < C && !(ISO && !out_of_range)) invden[tid] = tid < L ? __fdividef(1.f, r_s[tid] + dsum[tid]) : 0.f;
        sync_tc();

        // ---- MMA1 (in range): [A; Aq] = [K'; Q'] G'^T   (M=128, N=64 tokens, K=128 channels)
        if (!out_of_range) {
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t ka = (uint32_t)(ks >> 2), ko = (uint32_t)(ks & 3) * 32u;
                    mma_bf16(T_A, sdesc(sb + L_::KQ + ka * 16384u + ko, 16, 1024),
                             sdesc(sb + L_::G + ka * 8192u + ko, 16, 1024), ID_M128_N64_KK, ks > 0);
                }
                mma_commit(bar_mma);
            }
            wait_mma();
        }
        // rows 0..63: A (strictly lower) -> its lower-left 32x32 block L (bf16) and its two
        // diagonal blocks (fp32); rows 64..127: Aq (lower incl. diagonal, bf16); columns / den
        {
            const int s0 = cg * 32;
            float v[32];
            if (!out_of_range) {
                tmem_ld32(T_A + lane_off + s0, v);
            } else {
                const float *src = reinterpret_cast<const float *>(sm + L_::XAA) + row * XLD + s0;
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = src[j];
                __syncthreads();   // every row is read before the epilogue reuses the region
            }
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 d4 = *reinterpret_cast<const float4 *>(invden + s0 + j);
                v[j] *= d4.x; v[j + 1] *= d4.y; v[j + 2] *= d4.z; v[j + 3] *= d4.w;
            }
            if (row < 64) {
                const int t = row, b = t >> 5, tr = t & 31;
                const bool lower_left = (b == 1 && cg == 0);
#pragma unroll
                for (int chn = 0; chn < 4; ++chn) {
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(sm + L_::LB + swz(t, (cg * 4 + chn) * 16)) = lower_left ? pack8(v + chn * 8) : z;
                }
                if (b == cg) {
                    float *dst = adg + (b * 32 + tr) * ADS;
#pragma unroll
                    for (int jj = 0; jj < 32; jj += 4)
                        *reinterpret_cast<float4 *>(dst + jj) =
                            make_float4(jj < tr ? v[jj] : 0.f, jj + 1 < tr ? v[jj + 1] : 0.f, jj + 2 < tr ? v[jj + 2] : 0.f,
                                        jj + 3 < tr ? v[jj + 3] : 0.f);
                }
            } else {
                const int t = row - 64;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (s0 + j > t) v[j] = 0.f;
#pragma unroll
                for (int chn = 0; chn < 4; ++chn)
                    *reinterpret_cast<uint4 *>(sm + L_::AQ + swz(t, (cg * 4 + chn) * 16)) = pack8(v + chn * 8);
            }
        }
        __syncthreads();
        // ---- T = (I + A)^{-1}: D = the two 32x32 diagonal-block inverses, each from the inverses
        //      D1, D2 of its two 16x16 diagonal blocks (forward substitution, thread = one column of
        //      one 16-block) and its lower-left block -D2 A21 D1 (two 16x16 products on every thread);
        //      then N = D L (N^2 = 0), T = (I - N) D
        {
            if (tid < 64) {
                float x[16];
                const int b16 = tid >> 4, j = tid & 15, o = (b16 & 1) * 16;
                float *blk = adg + ((b16 >> 1) * 32 + o) * ADS + o;   // the 16-block's first entry
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
                for (int r = 1; r < 16; ++r) {   // A's row r is zero from column r on
                    const float4 *arow = reinterpret_cast<const float4 *>(blk + r * ADS);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int q4 = 0; q4 < (r + 3) / 4; ++q4) {
                        const float4 a4 = arow[q4];
                        acc[0] = fmaf(a4.x, x[4 * q4], acc[0]);
                        acc[1] = fmaf(a4.y, x[4 * q4 + 1], acc[1]);
                        acc[2] = fmaf(a4.z, x[4 * q4 + 2], acc[2]);
                        acc[3] = fmaf(a4.w, x[4 * q4 + 3], acc[3]);
                    }
                    if (r > j) x[r] = -((acc[0] + acc[1]) + (acc[2] + acc[3]));
                }
                __syncwarp();   // the 16-block's rows are read (its columns belong to this warp's half)
#pragma unroll
                for (int r = 0; r < 16; ++r) blk[r * ADS + j] = x[r];
            }
            __syncthreads();
            // Y = A21 D1 (fp32 [2][16][16] in the N tile, written later), then the lower-left block
            // -D2 Y over A21; thread = two entries (32-block, row, column)
            float *yt = reinterpret_cast<float *>(sm + L_::NB);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int idx = tid * 2 + e, b = idx >> 8, r = (idx >> 4) & 15, cc = idx & 15;
                const float *a21 = adg + (b * 32 + 16 + r) * ADS, *d1 = adg + (b * 32) * ADS + cc;
                float acc = 0.f;
                for (int m = cc; m < 16; ++m) acc = fmaf(a21[m], d1[m * ADS], acc);   // D1 is lower triangular
                yt[idx] = acc;
            }
            __syncthreads();
            float z[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int idx = tid * 2 + e, b = idx >> 8, r = (idx >> 4) & 15, cc = idx & 15;
                const float *d2 = adg + (b * 32 + 16 + r) * ADS + 16;
                float acc = 0.f;
                for (int m = 0; m <= r; ++m) acc = fmaf(d2[m], yt[(b * 16 + m) * 16 + cc], acc);   // D2 too
                z[e] = -acc;
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {   // over A21: every read of it was before the last barrier
                const int idx = tid * 2 + e, b = idx >> 8, r = (idx >> 4) & 15, cc = idx & 15;
                adg[(b * 32 + 16 + r) * ADS + cc] = z[e];
            }
            __syncthreads();
            // bf16 D: 64 rows x 8 chunks of 16 B, two chunks per thread
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = tid >> 2, cc = (tid & 3) * 2 + half, rb = r >> 5, cb = cc >> 2;
                float d8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) d8[e] = (cb == rb) ? adg[(rb * 32 + (r & 31)) * ADS + (cc & 3) * 8 + e] : 0.f;
                *reinterpret_cast<uint4 *>(sm + L_::DB + swz(r, cc * 16)) = pack8(d8);
            }
        }
        sync_tc();
        mma64(T_A, L_::DB, L_::LB);                           // N = D L
        {   // I - N (bf16; N^2 = 0, so (I + D L)^{-1} = I - N)
            float v[32];
            tmem_ld32(T_A + lane_off + cg * 32, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = (cg * 32 + j == m64 ? 1.f : 0.f) - v[j];
            store64(L_::NB, 0, v);
        }
        sync_tc();
        mma64(T_A + 64, L_::NB, L_::DB);                      // T = (I - N) D
        {   // T -> rows 0..63 of Y
            float v[32];
            tmem_ld32(T_A + 64 + lane_off + cg * 32, v);
            store64(L_::Y, 0, v);
        }
        sync_tc();
        mma64(T_A + 128, L_::AQ, L_::Y);                      // X = Aq T (T as MN-major B)
        {   // X -> rows 64..127 of Y, 16 columns at a time
            for (int hh = 0; hh < 2; ++hh) {
                float v[16];
                tmem_ld16(T_A + 128 + lane_off + cg * 32 + hh * 16, v);
                if (lane < 16) {
#pragma unroll
                    for (int chn = 0; chn < 2; ++chn)
                        *reinterpret_cast<uint4 *>(sm + L_::Y + swz(64 + m64, (cg * 4 + hh * 2 + chn) * 16)) = pack8(v + chn * 8);
                }
            }
        }
        sync_tc();

        // ---- MMA2: [w; X K~] = [T; X] K~   (M=128, N=128 channels, K=64 tokens; K~ MN-major)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_A + 128, sdesc(sb + L_::Y + ks * 32u, 16, 1024), sdesc(sb + L_::KQ + ks * 2048u, 16384, 1024),
                         ID_M128_N128_KM, ks > 0);
            mma_commit(bar_mma);
        }
        wait_mma();
        // rows 0..63 -> -w ; rows 64..127 -> Q' = Q~ - X K~   (bf16, record layout), 16 columns at a
        // time; operands referenced to the chunk end take the chunk decay Gam_L back per column
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
            float v[16], gl[16];
            tmem_ld16(T_A + 128 + lane_off + cg * 64 + hh * 16, v);
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                const float4 g4 = out_of_range ? make_float4(1.f, 1.f, 1.f, 1.f)
                                               : *reinterpret_cast<const float4 *>(gamc + cg * 64 + hh * 16 + e);
                gl[e] = g4.x; gl[e + 1] = g4.y; gl[e + 2] = g4.z; gl[e + 3] = g4.w;
            }
            const uint32_t atom = (uint32_t)cg * 16384u;
#pragma unroll
            for (int chn = 0; chn < 2; ++chn) {
                const uint32_t boff = atom + swz(row, (hh * 2 + chn) * 16);
                float w8[8];
                if (row < 64) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) w8[e] = -v[chn * 8 + e] * gl[chn * 8 + e];
                } else {
                    const uint4 q4 = *reinterpret_cast<const uint4 *>(sm + L_::KQ + boff);
                    const uint32_t *qp = reinterpret_cast<const uint32_t *>(&q4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        w8[2 * e] = (bf16_lo(qp[e]) - v[chn * 8 + 2 * e]) * gl[chn * 8 + 2 * e];
                        w8[2 * e + 1] = (bf16_hi(qp[e]) - v[chn * 8 + 2 * e + 1]) * gl[chn * 8 + 2 * e + 1];
                    }
                }
                *reinterpret_cast<uint4 *>(sm + L_::A4 + boff) = pack8(w8);
            }
        }
        sync_tc();
        // ---- the unit's record (bulk stores; drained before the next unit reuses the buffers)
        if (tid == 0) {
            uint8_t *dst = pa.rec + (size_t)u * Rec::BYTES;
            bulk_store(dst + Rec::A4, sm + L_::A4, 32768);
            bulk_store(dst + Rec::Y, sm + L_::Y, 16384);
            bulk_store(dst + Rec::G, sm + L_::G, 16384);
            bulk_store(dst + Rec::MISC, sm + L_::MISC, 768);
            bulk_commit();
        }
    }
    if (ctl[1]) {
        raise_error(a.err, ERR_TIMEOUT);
        // an MMA wait gave up: one more bounded wait for everything this CTA issued before its
        // tensor memory is released
        if (tid == 0) drain_mma(bar_mma, mma_phase);
    }
    if (tid == 0) bulk_wait0();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(T_A, 256);
}

// ================================================================= state
template <int DVT>
__global__ void __launch_bounds__(SNT, 1) chunk_state_kernel(const __grid_constant__ StateArgs sa)
{
    using L_ = StateSmem<DVT>;
    using namespace tc;
    constexpr int NC = DVT / 2;           // d_v columns per thread in the epilogues
    constexpr int CW = NC < 32 ? NC : 32;  // columns per TMEM load
    extern __shared__ uint8_t smraw[];
    const uint32_t raw_u32 = smem_u32(smraw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
    uint8_t *sm = smraw + (sb - raw_u32);
    uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + L_::CTL);   // [2]
    uint64_t *bar_mma = bar_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_mma + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const TokenArgs &a = sa.a;
    bf16 *__restrict__ out = static_cast<bf16 *>(a.o);
    const int ntiles = a.dv / DVT;
    const int tile = blockIdx.x % ntiles;
    const bool packed = sa.U != nullptr;
    // packed problems: chains in order of length, longest first (the long chains start first)
    const int rank = packed ? (int)(blockIdx.x / ntiles) / a.H : 0;
    const int chain = packed ? sa.order[rank] * a.H + (int)(blockIdx.x / ntiles) % a.H : (int)(blockIdx.x / ntiles);
    const int s = chain / a.H, h = chain % a.H;
    int t0, t1;
    seq_range(a, s, t0, t1);
    int nch = (t1 - t0 + C - 1) / C;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, cg = warp >> 2;
    const int H = a.H, dv = a.dv;
    if (!packed && nch > sa.nchunks_max) {   // records exist for nchunks_max chunks only
        if (tid == 0) raise_error(a.err, ERR_ARG);
        nch = (int)sa.nchunks_max;
    }

    if (tid == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_full + 1, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        *abort_flag = 0;
        tma_prefetch_desc(&sa.tv);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t T_S = tmem, T_D4 = tmem + 256;
    const uint32_t lane_off = ((uint32_t)quad * 32u) << 16;
    const int row = quad * 32 + lane;
    const int cb0 = cg * NC;

    // the v tile: whole 64-column boxes; a 32-column tile is one half of its box
    const int vx0 = (tile * DVT) & ~63;
    const uint32_t voff = (uint32_t)((tile * DVT) & 63) * 2u;
    int last0 = -1, last1 = -1;         // thread 0: the chunk last fetched into stage 0 / 1
    auto issue = [&](int c, int st) {   // record and v tile of chunk c into stage st
        if (st == 0) last0 = c; else last1 = c;
        const long long uc = packed ? sa.U[c] + (long long)rank * H + h : (long long)c * sa.nchains + chain;
        const uint8_t *src = sa.rec + (size_t)uc * Rec::BYTES;
        mbar_expect_tx(bar_full + st, Rec::BYTES + L_::V_BYTES);
        bulk_load(sm + st * L_::STAGE, src, Rec::BYTES, bar_full + st);
        for (int b = 0; b < (int)(L_::W64 / 64); ++b)
            tma_load_3d(sm + L_::V0 + st * L_::V_BYTES + b * 8192, &sa.tv, vx0 + b * 64, h, t0 + c * C, bar_full + st);
    };

    // initial memory tile -> TMEM (lane = key channel) and its bf16 operand copy
    const size_t sbase = (size_t)chain * DK * dv + (size_t)tile * DVT;
#pragma unroll
    for (int p = 0; p < NC / CW; ++p) {
        float v[CW];
        const int col = cb0 + p * CW;
#pragma unroll
        for (int j = 0; j < CW; j += 4) {
            float4 x = a.S0 ? *reinterpret_cast<const float4 *>(a.S0 + sbase + (size_t)row * dv + col + j)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            v[j] = x.x; v[j + 1] = x.y; v[j + 2] = x.z; v[j + 3] = x.w;
        }
        tmem_st<CW>(T_S + lane_off + col, v);
        const uint32_t atom = (uint32_t)(col >> 6) * 16384u;
#pragma unroll
        for (int chn = 0; chn < CW / 8; ++chn)
            *reinterpret_cast<uint4 *>(sm + L_::S + atom + swz(row, (((col & 63) >> 3) + chn) * 16)) = pack8(v + chn * 8);
    }
    // launched as a programmatic dependent of the prep kernel: everything above overlaps the
    // prep's tail; the records are read only once the whole prep grid has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0 && nch > 0) issue(0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    constexpr uint32_t ID_M128_NV_KM = idesc_bf16(128, DVT, false, true);
    constexpr uint32_t ID_M128_NV_MM = idesc_bf16(128, DVT, true, true);
    uint32_t mma_phase = 0;
    auto wait_mma = [&]() {
        if (!mbar_wait(bar_mma, mma_phase)) atomicExch(abort_flag, 1);
        mma_phase ^= 1u;
        tc_fence_after();
    };

    for (int c = 0; c < nch; ++c) {
        const int st = c & 1;
        const int c0 = t0 + c * C, L = min(C, t1 - c0);
        const uint32_t stg = (uint32_t)st * L_::STAGE;
        const float *invden = reinterpret_cast<const float *>(sm + stg + Rec::MISC);
        const float *gamc = invden + 64;
        if (!mbar_wait(bar_full + st, (uint32_t)((c >> 1) & 1))) atomicExch(abort_flag, 1);
        __syncthreads();
        if (*abort_flag) break;
        if (tid == 0 && c + 1 < nch) issue(c + 1, st ^ 1);

        // ---- MMA4: [U; O] = [-w; Q'] S + [T; X] V   (M=128, N=DVT, K=128+64)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ka = (uint32_t)(ks >> 2), ko = (uint32_t)(ks & 3) * 32u;
                mma_bf16(T_D4, sdesc(sb + stg + Rec::A4 + ka * 16384u + ko, 16, 1024),
                         sdesc(sb + L_::S + ks * 2048u, 16384, 1024), ID_M128_NV_KM, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_D4, sdesc(sb + stg + Rec::Y + ks * 32u, 16, 1024),
                         sdesc(sb + L_::V0 + st * L_::V_BYTES + ks * 2048u + voff, 8192, 1024), ID_M128_NV_KM, 1);
            mma_commit(bar_mma);
        }
        // ---- the memory's rows decayed by the chunk's Gam_L while MMA4 (which reads the bf16
        //      copy) runs: S <- Gam_L S, before MMA5 adds G'^T (U / den), G' = P^- k Gam_L / Gam_s
        {
            const float gC = gamc[row];
#pragma unroll
            for (int p = 0; p < NC / CW; ++p) {
                float v[CW];
                const int col = cb0 + p * CW;
                tmem_ld<CW>(T_S + lane_off + col, v);
#pragma unroll
                for (int j = 0; j < CW; ++j) v[j] *= gC;
                tmem_st<CW>(T_S + lane_off + col, v);
            }
        }
        wait_mma();
        // rows 0..63 -> U / den (bf16); rows 64..127 -> o (global, tokens of the chunk)
#pragma unroll
        for (int p = 0; p < NC / CW; ++p) {
            float v[CW];
            const int col = cb0 + p * CW;
            tmem_ld<CW>(T_D4 + lane_off + col, v);
            if (row < 64) {
                const float sc = invden[row];
                const uint32_t blk = (uint32_t)(col >> 6) * 8192u;
#pragma unroll
                for (int chn = 0; chn < CW / 8; ++chn)
                    *reinterpret_cast<uint4 *>(sm + L_::U + blk + swz(row, (((col & 63) >> 3) + chn) * 16)) =
                        pack8(v + chn * 8, sc);
            } else if (row - 64 < L) {
                bf16 *dst = out + ((size_t)(c0 + row - 64) * H + h) * dv + tile * DVT + col;
#pragma unroll
                for (int chn = 0; chn < CW / 8; ++chn) *reinterpret_cast<uint4 *>(dst + chn * 8) = pack8(v + chn * 8);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- MMA5: S += G'^T (U / den)   (M=128 channels, N=DVT, K=64 tokens; both MN-major)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_S, sdesc(sb + stg + Rec::G + ks * 2048u, 8192, 1024), sdesc(sb + L_::U + ks * 2048u, 8192, 1024),
                         ID_M128_NV_MM, 1);
            mma_commit(bar_mma);
        }
        wait_mma();
        // ---- refresh the bf16 operand copy of the memory
        {
#pragma unroll
            for (int p = 0; p < NC / CW; ++p) {
                float v[CW];
                const int col = cb0 + p * CW;
                tmem_ld<CW>(T_S + lane_off + col, v);
                const uint32_t atom = (uint32_t)(col >> 6) * 16384u;
#pragma unroll
                for (int chn = 0; chn < CW / 8; ++chn)
                    *reinterpret_cast<uint4 *>(sm + L_::S + atom + swz(row, (((col & 63) >> 3) + chn) * 16)) =
                        pack8(v + chn * 8);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (!*abort_flag) {
        if (a.S_out) {
#pragma unroll
            for (int p = 0; p < NC / CW; ++p) {
                float v[CW];
                const int col = cb0 + p * CW;
                tmem_ld<CW>(T_S + lane_off + col, v);
#pragma unroll
                for (int j = 0; j < CW; j += 4)
                    *reinterpret_cast<float4 *>(a.S_out + sbase + (size_t)row * dv + col + j) =
                        make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
        }
        // a sequence without tokens had no prep unit: its uncertainty passes through here
        if (nch == 0 && a.P_out && tile == 0) {
            if (!a.iso && tid < DK) a.P_out[(size_t)chain * DK + tid] = a.P0 ? a.P0[(size_t)chain * DK + tid] : 1.f;
            else if (a.iso && tid == 0) a.P_out[chain] = a.P0 ? a.P0[chain] : 1.f;
        }
    } else {
        raise_error(a.err, ERR_TIMEOUT);
        // a wait gave up: one more bounded wait for the MMAs and copies this CTA issued before
        // its tensor and shared memory are released
        if (tid == 0) {
            drain_mma(bar_mma, mma_phase);
            if (last0 >= 0) drain_copy(bar_full, (uint32_t)((last0 >> 1) & 1));
            if (last1 >= 0) drain_copy(bar_full + 1, (uint32_t)((last1 >> 1) & 1));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ================================================================= unit table (packed problems)
// One CTA: chunk counts of the sequences, their histogram, U by two block-wide prefix sums,
// and the ranks of the sequences by chunk count (equal counts in any order).
__global__ void __launch_bounds__(1024) unit_table_kernel(const int32_t *__restrict__ cu, int nseq, int H, UnitTable t)
{
    constexpr int NTH = 1024;
    __shared__ long long part[NTH];
    const int tid = threadIdx.x;
    const int n = t.cmax + 1;
    for (int i = tid; i < n; i += NTH) { t.hist[i] = 0; t.fill[i] = 0; }
    __syncthreads();
    for (int q = tid; q < nseq; q += NTH) {
        const int nc = min((__ldg(cu + q + 1) - __ldg(cu + q) + C - 1) / C, t.cmax);
        atomicAdd(t.hist + nc, 1);
    }
    __syncthreads();
    const int per = (n + NTH - 1) / NTH, b = min(n, tid * per), e = min(n, b + per);
    // exclusive prefix over the threads' partial sums (Hillis-Steele in shared memory)
    auto block_exclusive = [&](long long own) -> long long {
        part[tid] = own;
        __syncthreads();
        for (int off = 1; off < NTH; off <<= 1) {
            const long long x = tid >= off ? part[tid - off] : 0;
            __syncthreads();
            part[tid] += x;
            __syncthreads();
        }
        const long long incl = part[tid];
        __syncthreads();
        return incl - own;
    };
    // sequences with more than c chunks: nseq - (inclusive prefix of the histogram at c)
    long long acc = 0;
    for (int i = b; i < e; ++i) acc += t.hist[i];
    acc = block_exclusive(acc);
    for (int i = b; i < e; ++i) { acc += t.hist[i]; t.U[i] = acc; }
    __syncthreads();
    for (int i = b; i < e; ++i) t.hist[i] = nseq - (int)t.U[i];
    __syncthreads();
    // U[c] = H x (units of the chunk levels below c)
    acc = 0;
    for (int i = b; i < e; ++i) acc += t.hist[i];
    acc = block_exclusive(acc);
    for (int i = b; i < e; ++i) { t.U[i] = (long long)H * acc; acc += t.hist[i]; }
    __syncthreads();
    // rank = sequences with more chunks + place among the equal ones
    for (int q = tid; q < nseq; q += NTH) {
        const int nc = min((__ldg(cu + q + 1) - __ldg(cu + q) + C - 1) / C, t.cmax);
        const int r = t.hist[nc] + atomicAdd(t.fill + nc, 1);
        t.pos[q] = r;
        t.order[r] = q;
    }
}

// ================================================================= host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// the driver's tensor-map encoder, resolved once through the runtime (no link against libcuda)
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

bool chunk_tc_supported(int dk, int dv, bool bf16_in, int chunk, long long ntok) {
    return bf16_in && chunk == C && dk == DK && (dv == 64 || dv == 128 || dv == 256) && ntok > 0 && encode_fn() != nullptr;
}

namespace {
size_t round256(size_t x) { return (x + 255) / 256 * 256; }
size_t table_bytes(long long cmax, long long nseq) {
    return round256((size_t)(cmax + 1) * 8) + 2 * round256((size_t)nseq * 4) + 2 * round256((size_t)(cmax + 1) * 4);
}
}  // namespace

// units: upper bound of the number of units; cmax > 0 for packed problems (their unit table)
size_t two_phase_workspace_bytes(long long units, long long cmax, long long nseq) {
    const size_t table = cmax > 0 ? table_bytes(cmax, nseq) : 0;
    return 256 + table + (size_t)units * 4 * DK * 8 + (size_t)units * Rec::BYTES;
}

template <int DVT>
static cudaError_t launch_state(const StateArgs &sa, unsigned grid, cudaStream_t st) {
    constexpr size_t smem = StateSmem<DVT>::total + 1024;
    auto kern = chunk_state_kernel<DVT>;
    KernelSetup ks;
    cudaError_t e = kernel_setup(reinterpret_cast<const void *>(kern), smem, SNT, false, &ks);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the CTAs may start while the prep kernel finishes
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(SNT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, sa);
}

cudaError_t launch_chunk_two_phase(const TokenArgs &a, long long ntok, long long nchunks_max, void *workspace,
                                   cudaStream_t st) {
    const long long nchains = (long long)a.nseq * a.H;
    if (nchains == 0) return cudaSuccess;
    const bool packed = a.cu != nullptr;
    // packed: sum_s ceil(len_s / 64) <= T / 64 + nseq units per head
    const long long cmax = packed ? (ntok + C - 1) / C : 0;
    const long long units = packed ? (ntok / C + a.nseq) * a.H : nchains * nchunks_max;
    const size_t desc_bytes = (size_t)units * 4 * DK * 8;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *tab = ws + 256;
    const size_t tbytes = packed ? table_bytes(cmax, a.nseq) : 0;

    PrepArgs pa;
    pa.a = a;
    pa.nchunks_max = nchunks_max;
    pa.nchains = (int)nchains;
    pa.counter = reinterpret_cast<unsigned *>(ws);
    pa.desc = reinterpret_cast<unsigned long long *>(ws + 256 + tbytes);
    pa.rec = ws + 256 + tbytes + desc_bytes;
    pa.U = nullptr;
    pa.order = nullptr;
    pa.pos = nullptr;
    pa.cmax = (int)cmax;
    UnitTable t{};
    if (packed) {
        t.U = reinterpret_cast<long long *>(tab);
        t.order = reinterpret_cast<int *>(tab + round256((size_t)(cmax + 1) * 8));
        t.pos = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(t.order) + round256((size_t)a.nseq * 4));
        t.hist = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(t.pos) + round256((size_t)a.nseq * 4));
        t.fill = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(t.hist) + round256((size_t)(cmax + 1) * 4));
        t.cmax = (int)cmax;
        pa.U = t.U;
        pa.order = t.order;
        pa.pos = t.pos;
    }

    StateArgs sa;
    sa.a = a;
    sa.rec = pa.rec;
    sa.nchunks_max = nchunks_max;
    sa.nchains = (int)nchains;
    sa.U = pa.U;
    sa.order = pa.order;
    if (!make_token_map(&sa.tv, a.v, a.dv, a.H, ntok)) return cudaErrorInvalidValue;

    cudaError_t e = cudaSuccess;
    if (units > 0) {
        e = cudaMemsetAsync(ws, 0, 256, st);   // ticket counter
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(pa.desc, 0, desc_bytes, st);   // look-back words (untagged)
        if (e != cudaSuccess) return e;
        if (packed) {
            unit_table_kernel<<<1, 1024, 0, st>>>(a.cu, a.nseq, a.H, t);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        constexpr size_t psmem = PrepSmem::total + 1024;
        auto prep = a.iso ? (packed ? chunk_prep_kernel<true, true> : chunk_prep_kernel<true, false>)
                          : (packed ? chunk_prep_kernel<false, true> : chunk_prep_kernel<false, false>);
        // all of the unified L1 / shared array as shared memory, so that two CTAs fit on an SM
        KernelSetup ks;
        e = kernel_setup(reinterpret_cast<const void *>(prep), psmem, PNT, true, &ks);
        if (e != cudaSuccess) return e;
        // two CTAs fit on an SM (registers and shared memory); the occupancy query can report
        // fewer.  Extra CTAs are harmless: units go out by ticket to resident CTAs only.
        long long grid = (long long)ks.sms * (ks.blocks_per_sm > 2 ? ks.blocks_per_sm : 2);
        if (grid > units) grid = units;
        prep<<<(unsigned)grid, PNT, psmem, st>>>(pa);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // the narrowest d_v tile whose CTAs still fit on the SMs at one per SM (more chains in flight,
    // shorter MMAs and epilogues); with more chains than that, the widest
    int sms = 148;
    {
        KernelSetup ks;
        e = kernel_setup(reinterpret_cast<const void *>(chunk_state_kernel<128>), StateSmem<128>::total + 1024, SNT,
                         false, &ks);
        if (e != cudaSuccess) return e;
        sms = ks.sms;
    }
    int dvt = a.dv < 128 ? a.dv : 128;
    for (int w = 32; w <= dvt; w *= 2)
        if (nchains * (a.dv / w) <= sms) { dvt = w; break; }
    const unsigned sgrid = (unsigned)(nchains * (a.dv / dvt));
    if (dvt == 32) return launch_state<32>(sa, sgrid, st);
    return dvt == 64 ? launch_state<64>(sa, sgrid, st) : launch_state<128>(sa, sgrid, st);
}

}  // namespace kdn
