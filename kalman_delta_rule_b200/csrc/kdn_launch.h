// Host-side launchers of the KDN kernels (internal to libkdn.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "kdn_common.cuh"

namespace kdn {

// Launch set-up of a kernel on the current device and context, done once and cached: the
// dynamic shared-memory limit set to `smem` (and the whole unified L1/shared array as shared
// memory when `max_carveout`), the SM count and the occupancy at `threads` per CTA.
struct KernelSetup {
    int sms;            // multiprocessors of the device
    int blocks_per_sm;  // resident CTAs per SM at this shared memory and block size
};
cudaError_t kernel_setup(const void *kern, size_t smem, int threads, bool max_carveout, KernelSetup *out);
// Device address of a __device__ symbol on the current device and context, looked up once
// (with that device current) and cached; looked up again after the context changes.
cudaError_t symbol_address(const void *symbol, void **out);

// token-serial fused recurrence; dvt = d_v tile per CTA (32/64/128/256, divides d_v)
cudaError_t launch_recurrent(const TokenArgs &a, bool bf16_in, int dvt, cudaStream_t st);

// chunkwise forward on CUDA cores in fp32 (chunk C <= 64); any dtype
cudaError_t launch_chunk_simt(const TokenArgs &a, bool bf16_in, int C, cudaStream_t st);

// chunkwise forward on tcgen05 tensor cores (bf16 inputs, d_k = 128, chunk 64) in two launches:
// a chunk-parallel prep kernel (uncertainty by decoupled look-back, intra-chunk matrices,
// triangular inverse) writing per-chunk operand records to the workspace, then the
// chunk-serial state kernel
bool chunk_tc_supported(int dk, int dv, bool bf16_in, int chunk, long long ntok);
// units: upper bound of the (chunk, sequence x head) units; cmax > 0 for packed problems
size_t two_phase_workspace_bytes(long long units, long long cmax, long long nseq);
cudaError_t launch_chunk_two_phase(const TokenArgs &a, long long ntok, long long nchunks_max, void *workspace,
                                   cudaStream_t st);
// [ntok, H, d] bf16 as a TMA tensor map with 64 x 1 x 64 boxes and 128-byte swizzle
bool make_token_map(CUtensorMap *m, const void *base, int d, int H, long long ntok);

// backward of the diagonal KDN (three launches: uncertainty tape, memory state pass,
// uncertainty adjoint); all gradients fp32
struct BwdArgs {
    TokenArgs a;                                 // forward inputs (o, S_out, P_out unused)
    const void *d_o;                             // [ntok, H, dv], input dtype
    const float *dS_T, *dP_T;                    // [N, H, dk, dv], [N, H, dk]; NULL = 0
    float *dq, *dk, *dv, *dalpha, *dsigma, *dr;  // token layouts
    float *dS0, *dP0;                            // may be NULL
};
size_t backward_workspace_bytes(long long ntok, int nseq, int H, int dk, int dv);
cudaError_t launch_backward(const BwdArgs &b, bool bf16_in, long long ntok, long long nchunks_max, void *workspace,
                            cudaStream_t st);

// failure-detection self-test: bounded waits that run out and record ERR_TIMEOUT
cudaError_t launch_bounded_wait_selftest(long long limit_cycles, unsigned *err, cudaStream_t st);

// single-pass Moebius scan of the uncertainty with decoupled look-back (workspace-backed)
size_t scan_workspace_bytes(long long nchains, long long nchunks_max, int dk);
cudaError_t launch_gain_scan(ScanArgs a, bool bf16_in, long long ntok, void *workspace, cudaStream_t st);
// the same scan on the library's fixed scratch array (no allocation, no caller workspace)
size_t noalloc_scratch_bytes();
cudaError_t launch_gain_scan_noalloc(const ScanArgs &a, bool bf16_in, long long ntok, cudaStream_t st);
// bf16, d_k = 128: TMA-staged scan with tagged look-back words (its own workspace layout)
bool gain_scan_tma_supported(int dk, bool bf16_in);
size_t scan_tma_workspace_bytes(long long nchains, long long nchunks_max);
cudaError_t launch_gain_scan_tma(const ScanArgs &a, long long ntok, void *workspace, cudaStream_t st);

}  // namespace kdn
