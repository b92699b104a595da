// Shared device helpers of the B200 KDN library: typed loads/stores, reductions,
// the device error word and the launch-argument structs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kdn.h"

namespace kdn {

// bits of the device error word (reported by kdn_last_device_error)
enum : unsigned { ERR_TIMEOUT = 1u, ERR_RANGE = 2u, ERR_ARG = 4u };

__device__ __forceinline__ void raise_error(unsigned *err, unsigned bit) {
    if (err) atomicOr(err, bit);
}

typedef __nv_bfloat16 bf16;

// ------------------------------------------------------------ scalar / vector I/O
__device__ __forceinline__ float ldf(const float *p) { return __ldg(p); }
__device__ __forceinline__ float ldf(const bf16 *p) {
    unsigned short u = __ldg(reinterpret_cast<const unsigned short *>(p));
    return __uint_as_float(((unsigned)u) << 16);
}

__device__ __forceinline__ float4 ldf4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float4 ldf4(const bf16 *p) {
    uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

__device__ __forceinline__ void stf4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void stf4(bf16 *p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<unsigned *>(&a);
    u.y = *reinterpret_cast<unsigned *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}
__device__ __forceinline__ void stf(float *p, float v) { *p = v; }
__device__ __forceinline__ void stf(bf16 *p, float v) { *p = __float2bfloat16_rn(v); }

// Two fp32 lanes in one 64-bit register pair, for sm_100's packed f32x2 arithmetic (x = the low
// lane, y = the high one); mul2 / fma2 round each lane as the scalar instruction would.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pk2(float x, float y) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
    return r;
}
__device__ __forceinline__ float x2(f32x2 r) { return __uint_as_float((unsigned)r); }
__device__ __forceinline__ float y2(f32x2 r) { return __uint_as_float((unsigned)(r >> 32)); }
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ------------------------------------------------------------ argument packs
struct TokenArgs {
    const void *q, *k, *v, *alpha, *sigma, *r;  // [ntok, H, d] / [ntok, H]
    void *o;                                     // [ntok, H, dv]
    const float *S0, *P0;                        // [N, H, dk, dv], [N, H, dk] ([N, H] isotropic) (NULL -> 0 / 1)
    float *S_out, *P_out;                        // may be NULL
    const int32_t *cu;                           // device [N+1] or NULL (dense: seq s = [s*T, (s+1)*T))
    int T;                                       // dense sequence length (ignored with cu)
    int nseq, H, dk, dv;
    float mu;
    int iso;                                     // 1: isotropic KDN (one uncertainty per head)
    unsigned *err;
};

struct ScanArgs {
    const void *k, *alpha, *sigma, *r;          // [ntok, H, dk] / [ntok, H]
    const float *P0;                            // [N, H, dk] or NULL (ones)
    float *g, *beta, *P_out;                    // [ntok, H, dk], [ntok, H], [N, H, dk]; each may be NULL
    float *P_prev, *den;                        // [ntok, H, dk], [ntok, H]: P before each token and the gain
                                                // denominator (the backward's tape); NULL = not written
    const int32_t *cu;                          // device [N+1] or NULL
    int T, nseq, H, dk;
    float mu;
    int nchunks_max, nchains;                   // chunk-major work list: nchunks_max x (nseq * H)
    unsigned *counter;                          // workspace: ticket counter
    int *flags;                                 // workspace: per (chunk, chain) publication flag
    float *desc;                                // workspace: per (chunk, chain) [4][dk] aggregate + end value
    unsigned *err;
};

__device__ __forceinline__ void seq_range(const TokenArgs &a, int s, int &t0, int &t1) {
    if (a.cu) {
        t0 = __ldg(a.cu + s);
        t1 = __ldg(a.cu + s + 1);
    } else {
        t0 = s * a.T;
        t1 = t0 + a.T;
    }
}

}  // namespace kdn
