// C ABI of libkdn.so: argument validation, workspace sizing, dispatch to the kernels,
// and the device error word.  Declarations and the contract are in include/kdn.h.
#include <math.h>

#include "kdn_common.cuh"
#include "kdn_launch.h"

namespace {

__device__ unsigned g_kdn_err;  // bits kdn::ERR_*; one copy per device

// the current device's error word (address looked up once per device and context)
unsigned *err_word() {
    void *p = nullptr;
    if (kdn::symbol_address(reinterpret_cast<const void *>(&g_kdn_err), &p) != cudaSuccess) return nullptr;
    return static_cast<unsigned *>(p);
}

bool dk_ok(int d) { return d == 32 || d == 64 || d == 128; }
bool dv_ok(int d) { return d == 32 || d == 64 || d == 128 || d == 256; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

struct Resolved {
    long long ntok;
    int nseq;
    bool bf16;
    long long nchunks_max;   // gain scan work list (chunks of 64 per sequence, upper bound)
};

kdn_status_t check_problem(const kdn_problem_t *p, Resolved *out) {
    if (!p) return KDN_ERR_INVALID_ARG;
    if (p->B < 0 || p->T < 0 || p->H <= 0) return KDN_ERR_INVALID_ARG;
    if (!(p->mu > 0.f) || !isfinite(p->mu)) return KDN_ERR_INVALID_ARG;
    if (p->in_dtype != KDN_DTYPE_F32 && p->in_dtype != KDN_DTYPE_BF16) return KDN_ERR_INVALID_ARG;
    if (p->variant != KDN_VARIANT_DIAGONAL && p->variant != KDN_VARIANT_ISOTROPIC) return KDN_ERR_INVALID_ARG;
    if (!dk_ok(p->d_k) || !dv_ok(p->d_v)) return KDN_ERR_UNSUPPORTED;
    if (p->chunk != 0 && p->chunk != 16 && p->chunk != 32 && p->chunk != 64) return KDN_ERR_UNSUPPORTED;
    if (p->cu_seqlens) {
        if (p->B != 1 || p->num_seqs < 0) return KDN_ERR_INVALID_ARG;
        out->nseq = p->num_seqs;
    } else {
        out->nseq = p->B;
    }
    out->ntok = (long long)p->B * p->T;
    out->bf16 = p->in_dtype == KDN_DTYPE_BF16;
    if (p->max_seqlen < 0) return KDN_ERR_INVALID_ARG;
    const long long ml = (p->max_seqlen > 0 && p->max_seqlen < p->T) ? p->max_seqlen : p->T;
    out->nchunks_max = (ml + 63) / 64;
    if (out->ntok > (1ll << 31) / 2) return KDN_ERR_UNSUPPORTED;
    return KDN_OK;
}

kdn_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? KDN_OK : KDN_ERR_CUDA; }

// the tensor-core chunk kernels serve this problem (bf16, d_k = 128, chunk 64, work list
// within 2^31 units)
bool two_phase_path(const kdn_problem_t *p, const Resolved &rv) {
    const long long units = p->cu_seqlens ? (rv.ntok / 64 + rv.nseq) * p->H : (long long)rv.nseq * p->H * rv.nchunks_max;
    return kdn::chunk_tc_supported(p->d_k, p->d_v, rv.bf16, p->chunk, rv.ntok) && units < (1ll << 31);
}
size_t two_phase_bytes(const kdn_problem_t *p, const Resolved &rv) {
    if (p->cu_seqlens) {   // packed: sum_s ceil(len_s / 64) <= T / 64 + num_seqs units per head
        const long long units = (rv.ntok / 64 + rv.nseq) * p->H;
        return kdn::two_phase_workspace_bytes(units, (rv.ntok + 63) / 64, rv.nseq);
    }
    return kdn::two_phase_workspace_bytes((long long)rv.nseq * p->H * rv.nchunks_max, 0, 0);
}

}  // namespace

extern "C" {

const char *kdn_status_string(kdn_status_t s) {
    switch (s) {
        case KDN_OK: return "ok";
        case KDN_ERR_INVALID_ARG: return "invalid argument";
        case KDN_ERR_UNSUPPORTED: return "unsupported size, dtype or chunk";
        case KDN_ERR_CUDA: return "CUDA runtime or launch error";
        case KDN_ERR_TIMEOUT: return "a bounded device wait gave up";
        case KDN_ERR_RANGE: return "value outside the supported range (reserved; no kernel reports it)";
        case KDN_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char *kdn_version(void) { return "kdn-b200 0.1 sm_100a"; }

kdn_status_t kdn_workspace_size(const kdn_problem_t *p, size_t *bytes) {
    Resolved rv;
    kdn_status_t st = check_problem(p, &rv);
    if (st != KDN_OK) return st;
    if (!bytes) return KDN_ERR_INVALID_ARG;
    size_t n = kdn::scan_workspace_bytes((long long)rv.nseq * p->H, rv.nchunks_max, p->d_k);
    if (two_phase_path(p, rv)) {
        const size_t m = two_phase_bytes(p, rv);
        if (m > n) n = m;
    }
    *bytes = n;
    return KDN_OK;
}

kdn_status_t kdn_forward_chunkwise(const kdn_problem_t *p, const void *q, const void *k, const void *v,
                                   const void *alpha, const void *sigma, const void *r, const float *S0,
                                   const float *P0, void *o, float *S_out, float *P_out, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    Resolved rv;
    kdn_status_t st = check_problem(p, &rv);
    if (st != KDN_OK) return st;
    if (rv.nseq == 0 || (rv.ntok == 0 && !S_out && !P_out)) return KDN_OK;
    if (rv.ntok > 0 && (!q || !k || !v || !alpha || !sigma || !r || !o)) return KDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, sigma, r, o, S0, P0, S_out, P_out};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDN_ERR_INVALID_ARG;
    if ((S_out && S_out == S0) || (P_out && P_out == P0)) return KDN_ERR_INVALID_ARG;
    if (!p->cu_seqlens && rv.nseq > 0 && p->T == 0 && !S_out && !P_out) return KDN_OK;

    kdn::TokenArgs a{};
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.sigma = sigma; a.r = r; a.o = o;
    a.S0 = S0; a.P0 = P0; a.S_out = S_out; a.P_out = P_out;
    a.cu = p->cu_seqlens; a.T = p->T; a.nseq = rv.nseq; a.H = p->H; a.dk = p->d_k; a.dv = p->d_v;
    a.mu = p->mu; a.iso = p->variant == KDN_VARIANT_ISOTROPIC; a.err = err_word();
    cudaStream_t cs = static_cast<cudaStream_t>(stream);

    if (p->chunk == 0) {
        const int dvt = p->d_v < 64 ? p->d_v : 64;
        return cuda_status(kdn::launch_recurrent(a, rv.bf16, dvt, cs));
    }
    if (two_phase_path(p, rv) && workspace && aligned256(workspace) && workspace_bytes >= two_phase_bytes(p, rv))
        return cuda_status(kdn::launch_chunk_two_phase(a, rv.ntok, rv.nchunks_max, workspace, cs));
    return cuda_status(kdn::launch_chunk_simt(a, rv.bf16, p->chunk, cs));
}

static kdn_status_t decode_impl(int N, int n_tokens, int H, int d_k, int d_v, kdn_dtype_t in_dtype, float mu,
                                const void *q, const void *k, const void *v, const void *alpha, const void *sigma,
                                const void *r, float *S, float *P, void *o, void *stream, bool iso) {
    if (N < 0 || n_tokens < 0 || H <= 0 || !(mu > 0.f) || !isfinite(mu)) return KDN_ERR_INVALID_ARG;
    if (in_dtype != KDN_DTYPE_F32 && in_dtype != KDN_DTYPE_BF16) return KDN_ERR_INVALID_ARG;
    if (!dk_ok(d_k) || !dv_ok(d_v)) return KDN_ERR_UNSUPPORTED;
    if (N == 0 || n_tokens == 0) return KDN_OK;
    if ((long long)N * n_tokens > (1ll << 30)) return KDN_ERR_UNSUPPORTED;
    const void *ptrs[] = {q, k, v, alpha, sigma, r, S, P, o};
    for (const void *ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return KDN_ERR_INVALID_ARG;
    kdn::TokenArgs a{};
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.sigma = sigma; a.r = r; a.o = o;
    a.S0 = S; a.P0 = P; a.S_out = S; a.P_out = P;
    a.cu = nullptr; a.T = n_tokens; a.nseq = N; a.H = H; a.dk = d_k; a.dv = d_v; a.mu = mu; a.err = err_word();
    a.iso = iso;
    // one tile per head: the in-place state and uncertainty are read and written by one CTA
    return cuda_status(kdn::launch_recurrent(a, in_dtype == KDN_DTYPE_BF16, d_v, static_cast<cudaStream_t>(stream)));
}

kdn_status_t kdn_decode_tokens(int N, int n_tokens, int H, int d_k, int d_v, kdn_dtype_t in_dtype, float mu,
                               const void *q, const void *k, const void *v, const void *alpha, const void *sigma,
                               const void *r, float *S, float *P, void *o, void *stream) {
    return decode_impl(N, n_tokens, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o, stream, false);
}

kdn_status_t kdn_decode_tokens_iso(int N, int n_tokens, int H, int d_k, int d_v, kdn_dtype_t in_dtype, float mu,
                                   const void *q, const void *k, const void *v, const void *alpha, const void *sigma,
                                   const void *r, float *S, float *P, void *o, void *stream) {
    return decode_impl(N, n_tokens, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o, stream, true);
}

kdn_status_t kdn_decode_step(int N, int H, int d_k, int d_v, kdn_dtype_t in_dtype, float mu, const void *q,
                             const void *k, const void *v, const void *alpha, const void *sigma, const void *r,
                             float *S, float *P, void *o, void *stream) {
    return kdn_decode_tokens(N, 1, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o, stream);
}

static kdn_status_t scan_args(const kdn_problem_t *p, const void *k, const void *alpha, const void *sigma,
                              const void *r, const float *P0, float *g, float *beta_eff, float *P_out,
                              kdn::ScanArgs *a, Resolved *rv, bool *empty) {
    kdn_status_t st = check_problem(p, rv);
    if (st != KDN_OK) return st;
    if (p->variant != KDN_VARIANT_DIAGONAL) return KDN_ERR_UNSUPPORTED;
    *empty = rv->nseq == 0 || rv->ntok == 0;
    if (*empty) return KDN_OK;
    if (!k || !alpha || !sigma || !r) return KDN_ERR_INVALID_ARG;
    const void *ptrs[] = {k, alpha, sigma, r, P0, g, beta_eff, P_out};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDN_ERR_INVALID_ARG;
    *a = kdn::ScanArgs{};
    a->k = k; a->alpha = alpha; a->sigma = sigma; a->r = r; a->P0 = P0;
    a->g = g; a->beta = beta_eff; a->P_out = P_out;
    a->cu = p->cu_seqlens; a->T = p->T; a->nseq = rv->nseq; a->H = p->H; a->dk = p->d_k; a->mu = p->mu;
    a->nchunks_max = (int)rv->nchunks_max; a->nchains = rv->nseq * p->H;
    return KDN_OK;
}

kdn_status_t kdn_gain_scan(const kdn_problem_t *p, const void *k, const void *alpha, const void *sigma,
                           const void *r, const float *P0, float *g, float *beta_eff, float *P_out,
                           void *workspace, size_t workspace_bytes, void *stream) {
    Resolved rv;
    kdn::ScanArgs a;
    bool empty = false;
    kdn_status_t st = scan_args(p, k, alpha, sigma, r, P0, g, beta_eff, P_out, &a, &rv, &empty);
    if (st != KDN_OK || empty) return st;
    const size_t need = kdn::scan_workspace_bytes((long long)rv.nseq * p->H, rv.nchunks_max, p->d_k);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return KDN_ERR_WORKSPACE;
    a.err = err_word();
    return cuda_status(kdn::launch_gain_scan(a, rv.bf16, rv.ntok, workspace, static_cast<cudaStream_t>(stream)));
}

kdn_status_t kdn_gain_scan_noalloc(const kdn_problem_t *p, const void *k, const void *alpha, const void *sigma,
                                   const void *r, const float *P0, float *g, float *beta_eff, float *P_out,
                                   void *stream) {
    Resolved rv;
    kdn::ScanArgs a;
    bool empty = false;
    kdn_status_t st = scan_args(p, k, alpha, sigma, r, P0, g, beta_eff, P_out, &a, &rv, &empty);
    if (st != KDN_OK || empty) return st;
    if (kdn::scan_workspace_bytes((long long)rv.nseq * p->H, rv.nchunks_max, p->d_k) > kdn::noalloc_scratch_bytes())
        return KDN_ERR_UNSUPPORTED;
    a.err = err_word();
    return cuda_status(kdn::launch_gain_scan_noalloc(a, rv.bf16, rv.ntok, static_cast<cudaStream_t>(stream)));
}

kdn_status_t kdn_backward_workspace_size(const kdn_problem_t *p, size_t *bytes) {
    Resolved rv;
    kdn_status_t st = check_problem(p, &rv);
    if (st != KDN_OK) return st;
    if (!bytes) return KDN_ERR_INVALID_ARG;
    *bytes = kdn::backward_workspace_bytes(rv.ntok, rv.nseq, p->H, p->d_k, p->d_v);
    return KDN_OK;
}

kdn_status_t kdn_backward(const kdn_problem_t *p, const void *q, const void *k, const void *v, const void *alpha,
                          const void *sigma, const void *r, const float *S0, const float *P0, const void *d_o,
                          const float *dS_T, const float *dP_T, float *dq, float *dk, float *dv, float *dalpha,
                          float *dsigma, float *dr, float *dS0, float *dP0, void *workspace, size_t workspace_bytes,
                          void *stream) {
    Resolved rv;
    kdn_status_t st = check_problem(p, &rv);
    if (st != KDN_OK) return st;
    if (rv.nseq == 0) return KDN_OK;
    if (rv.ntok > 0 && (!q || !k || !v || !alpha || !sigma || !r || !d_o || !dq || !dk || !dv || !dalpha ||
                        !dsigma || !dr))
        return KDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, sigma, r, S0, P0, d_o, dS_T, dP_T, dq, dk, dv, dalpha, dsigma, dr, dS0, dP0};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDN_ERR_INVALID_ARG;
    const size_t need = kdn::backward_workspace_bytes(rv.ntok, rv.nseq, p->H, p->d_k, p->d_v);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return KDN_ERR_WORKSPACE;

    kdn::BwdArgs b{};
    kdn::TokenArgs &a = b.a;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.sigma = sigma; a.r = r;
    a.S0 = S0; a.P0 = P0;
    a.cu = p->cu_seqlens; a.T = p->T; a.nseq = rv.nseq; a.H = p->H; a.dk = p->d_k; a.dv = p->d_v;
    a.mu = p->mu; a.iso = p->variant == KDN_VARIANT_ISOTROPIC; a.err = err_word();
    b.d_o = d_o; b.dS_T = dS_T; b.dP_T = dP_T;
    b.dq = dq; b.dk = dk; b.dv = dv; b.dalpha = dalpha; b.dsigma = dsigma; b.dr = dr; b.dS0 = dS0; b.dP0 = dP0;
    return cuda_status(kdn::launch_backward(b, rv.bf16, rv.ntok, rv.nchunks_max, workspace,
                                            static_cast<cudaStream_t>(stream)));
}

kdn_status_t kdn_selftest_bounded_wait(long long limit_cycles, void *stream) {
    if (limit_cycles < 1000 || limit_cycles > 4000000000ll) return KDN_ERR_INVALID_ARG;
    unsigned *err = err_word();
    if (!err) return KDN_ERR_CUDA;
    return cuda_status(kdn::launch_bounded_wait_selftest(limit_cycles, err, static_cast<cudaStream_t>(stream)));
}

int kdn_execution_path(const kdn_problem_t *p) {
    Resolved rv;
    if (check_problem(p, &rv) != KDN_OK) return -1;
    if (p->chunk == 0) return 0;
    return two_phase_path(p, rv) ? 3 : 1;
}

kdn_status_t kdn_last_device_error(void *stream) {
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(cs) != cudaSuccess) return KDN_ERR_CUDA;
    unsigned *ew = err_word();
    if (!ew) return KDN_ERR_CUDA;
    unsigned bits = 0;
    if (cudaMemcpyAsync(&bits, ew, sizeof(bits), cudaMemcpyDeviceToHost, cs) != cudaSuccess) return KDN_ERR_CUDA;
    if (cudaMemsetAsync(ew, 0, sizeof(unsigned), cs) != cudaSuccess) return KDN_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return KDN_ERR_CUDA;
    if (bits & kdn::ERR_TIMEOUT) return KDN_ERR_TIMEOUT;
    if (bits & kdn::ERR_RANGE) return KDN_ERR_RANGE;
    if (bits & kdn::ERR_ARG) return KDN_ERR_INVALID_ARG;
    return KDN_OK;
}

}  // extern "C"
