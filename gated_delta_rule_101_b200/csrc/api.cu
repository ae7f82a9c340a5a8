// libkda C ABI: argument validation and kernel dispatch.
//
// Every check here runs on the host before any launch, so a rejected call
// leaves all outputs untouched. The library allocates nothing: the caller
// provides every buffer (see include/kda.h).
#include "kda_internal.cuh"

namespace {

constexpr int KDA_VERSION = 100;  // 0.1.0

bool valid_dtype(int dtype) { return dtype == KDA_BF16 || dtype == KDA_F32; }
bool valid_gate(int gate) { return gate >= KDA_GATE_CHANNEL && gate <= KDA_GATE_CHANNEL_LOGIT_BF16; }

// The gate tensor is required unless there is no gate; the tensor-core path reads
// per-channel gates through TMA (16-byte base) and head gates as fp32 scalars.
int check_gate_ptr(const void *log_alpha, int gate, bool tma) {
    if (gate == KDA_GATE_NONE) return KDA_OK;
    if (!log_alpha) return KDA_ERR_INVALID_ARG;
    const bool fp32 = gate == KDA_GATE_CHANNEL || gate == KDA_GATE_CHANNEL_LOGIT;
    const uintptr_t align = gate == KDA_GATE_HEAD ? 4u : (tma ? 16u : (fp32 ? 4u : 2u));
    return ((uintptr_t)log_alpha & (align - 1)) == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
}

// The tensor-core kernels take bf16 inputs in chunks of 64; everything else (fp32
// inputs, and chunks of 32 in either dtype) runs on the CUDA-core kernel.
bool tensor_core_path(int C, int dtype) { return dtype == KDA_BF16 && C == KDA_CHUNK; }

// Validates the shape arguments shared by the size query and the call.
int check_prefill_shape(int B, int64_t T, int H, int C, int n_seqs, int dtype) {
    if (C != KDA_CHUNK && C != KDA_CHUNK_SMALL) return KDA_ERR_UNSUPPORTED;
    if (!valid_dtype(dtype)) return KDA_ERR_UNSUPPORTED;
    if (B <= 0 || T < 0 || H <= 0 || n_seqs < 0) return KDA_ERR_INVALID_ARG;
    if (n_seqs > 0 && B != 1) return KDA_ERR_INVALID_ARG;
    if (n_seqs == 0 && T == 0) return KDA_ERR_INVALID_ARG;
    // grid limits: y = H (<= 65535); x = sequences
    if (H > 65535) return KDA_ERR_INVALID_ARG;
    if (T > (int64_t)INT32_MAX) return KDA_ERR_INVALID_ARG;  // offsets are int32
    return KDA_OK;
}

// Checks a kda_io and turns it into the kernels' options. `out_ok`: the call supports an
// output gate; `esize`: bytes per element of the output gate (it has q's dtype).
int make_io(const kda_io *io, bool out_ok, int esize, kda::IoOpts *opts) {
    *opts = kda::IoOpts{};
    if (!io) return KDA_OK;
    if (!(io->qk_l2norm_eps >= 0.f) || !(io->out_norm_eps >= 0.f)) return KDA_ERR_INVALID_ARG;  // also NaN
    if (io->qk_l2norm_eps > 1e30f || io->out_norm_eps > 1e30f) return KDA_ERR_INVALID_ARG;
    opts->flags = (io->qk_l2norm ? kda::IO_QK_L2NORM : 0) | (io->beta_logits ? kda::IO_BETA_LOGITS : 0);
    opts->l2_eps = io->qk_l2norm_eps;
    if (io->out_gate) {
        if (!out_ok) return KDA_ERR_UNSUPPORTED;
        // the prefill epilogue reads eight gate values (16 bytes) per lane, the weights as float4
        const uintptr_t align = esize == 2 ? 16u : (uintptr_t)esize;
        if (((uintptr_t)io->out_gate & (align - 1)) != 0) return KDA_ERR_INVALID_ARG;
        if (io->out_norm_weight && ((uintptr_t)io->out_norm_weight & 15u) != 0) return KDA_ERR_INVALID_ARG;
        opts->out_gate = io->out_gate;  // (fp32 gates are read as float4 by the prefill epilogue)
        opts->out_w = io->out_norm_weight;
        opts->out_eps = io->out_norm_eps;
    }
    return KDA_OK;
}

}  // namespace

extern "C" {

const char *kda_strerror(int status) {
    switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: unsupported chunk size, dtype or gate layout";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: kernel launch failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: bounded device wait expired";
    case KDA_ERR_SCRATCH_LIMIT:
        return "KDA_ERR_SCRATCH_LIMIT: problem needs more than the fixed scratch of "
               "kda_chunk_fwd_noalloc";
    default: return "unknown kda status";
    }
}

int kda_version(void) { return KDA_VERSION; }

int kda_chunk_fwd_workspace_size(int B, int64_t T, int H, int C, int n_seqs, int dtype,
                                 size_t *bytes) {
    if (!bytes) return KDA_ERR_INVALID_ARG;
    const int st = check_prefill_shape(B, T, H, C, n_seqs, dtype);
    if (st != KDA_OK) return st;
    *bytes = tensor_core_path(C, dtype) ? kda::prefill_tc_workspace(B, T, H, n_seqs) : 0;
    return KDA_OK;
}

int kda_chunk_fwd_launches(int B, int64_t T, int H, int C, int n_seqs, int dtype, int *n_kernels) {
    return kda_chunk_fwd_io_launches(B, T, H, C, n_seqs, dtype, nullptr, n_kernels);
}

int kda_chunk_fwd_io_launches(int B, int64_t T, int H, int C, int n_seqs, int dtype, const kda_io *io,
                              int *n_kernels) {
    if (!n_kernels) return KDA_ERR_INVALID_ARG;
    const int st = check_prefill_shape(B, T, H, C, n_seqs, dtype);
    if (st != KDA_OK) return st;
    const bool out_epi = io && io->out_gate;
    const int64_t n_tok = n_seqs > 0 ? T : (int64_t)B * T;
    *n_kernels = (tensor_core_path(C, dtype) ? kda::prefill_tc_launches(B, T, H, n_seqs, io && io->qk_l2norm) : 1) +
                 (out_epi && n_tok > 0 ? 1 : 0);
    return KDA_OK;
}

int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *S0, void *o, float *S_T, int B, int64_t T,
                  int H, int C, const int32_t *cu_seqlens, int n_seqs,
                  const int32_t *cu_seqlens_host, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream) {
    return kda_chunk_fwd_gated(q, k, v, log_alpha, KDA_GATE_CHANNEL, beta, S0, o, S_T, B, T, H, C,
                               cu_seqlens, n_seqs, cu_seqlens_host, dtype, workspace,
                               workspace_bytes, stream);
}

int kda_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *log_alpha,
                        int gate, const float *beta, const float *S0, void *o, float *S_T, int B,
                        int64_t T, int H, int C, const int32_t *cu_seqlens, int n_seqs,
                        const int32_t *cu_seqlens_host, int dtype, void *workspace,
                        size_t workspace_bytes, void *stream) {
    return kda_chunk_fwd_io(q, k, v, log_alpha, gate, beta, S0, o, S_T, B, T, H, C, cu_seqlens, n_seqs,
                            cu_seqlens_host, dtype, workspace, workspace_bytes, nullptr, stream);
}

int kda_chunk_fwd_io(const void *q, const void *k, const void *v, const void *log_alpha, int gate,
                     const float *beta, const float *S0, void *o, float *S_T, int B, int64_t T, int H,
                     int C, const int32_t *cu_seqlens, int n_seqs, const int32_t *cu_seqlens_host,
                     int dtype, void *workspace, size_t workspace_bytes, const kda_io *io,
                     void *stream) {
    int st = check_prefill_shape(B, T, H, C, n_seqs, dtype);
    if (st != KDA_OK) return st;
    if (!valid_gate(gate)) return KDA_ERR_UNSUPPORTED;
    kda::IoOpts opts;
    const bool tc = tensor_core_path(C, dtype);
    st = make_io(io, true, dtype == KDA_BF16 ? 2 : 4, &opts);
    if (st != KDA_OK) return st;
    if (opts.out_gate && ((uintptr_t)opts.out_gate & 15u) != 0) return KDA_ERR_INVALID_ARG;  // vector rows
    if (opts.out_gate && ((uintptr_t)o & 15u) != 0) return KDA_ERR_INVALID_ARG;
    const bool packed = n_seqs > 0;
    if (packed != (cu_seqlens != nullptr)) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !beta || !o)) return KDA_ERR_INVALID_ARG;
    if (T > 0 && check_gate_ptr(log_alpha, gate, tc) != KDA_OK)
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens_host) {
        if (!packed || cu_seqlens_host[0] != 0 || cu_seqlens_host[n_seqs] != T)
            return KDA_ERR_INVALID_ARG;
        for (int s = 0; s < n_seqs; ++s)
            if (cu_seqlens_host[s + 1] < cu_seqlens_host[s]) return KDA_ERR_INVALID_ARG;
    }
    size_t need = 0;
    st = kda_chunk_fwd_workspace_size(B, T, H, C, n_seqs, dtype, &need);
    if (st != KDA_OK) return st;
    if (need > 0 && (!workspace || workspace_bytes < need)) return KDA_ERR_WORKSPACE;
    if (need > 0 && ((uintptr_t)workspace & 15u) != 0) return KDA_ERR_WORKSPACE;

    const int nseq = packed ? n_seqs : B;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t err;
    if (tc) {
        // TMA requires 16-byte aligned tensor bases
        if (T > 0 && ((((uintptr_t)q | (uintptr_t)k | (uintptr_t)v) & 15u) != 0))
            return KDA_ERR_INVALID_ARG;
        if ((S0 && ((uintptr_t)S0 & 15u)) || (S_T && ((uintptr_t)S_T & 15u)) || ((uintptr_t)o & 15u))
            return KDA_ERR_INVALID_ARG;
        err = kda::launch_prefill_tc(q, k, v, log_alpha, gate, beta, S0, o, S_T, B, T, H,
                                     cu_seqlens, n_seqs, workspace, opts, s);
    } else {
        err = kda::launch_prefill_simt(q, k, v, log_alpha, gate, beta, S0, o, S_T, nseq, T, H,
                                       cu_seqlens, dtype, C, opts, s);
    }
    if (err == cudaSuccess && opts.out_gate)
        err = kda::launch_out_epilogue(o, opts, (packed ? T : (int64_t)B * T) * H, dtype, s);
    if (err == cudaErrorInvalidValue) return KDA_ERR_INVALID_ARG;
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_chunk_bwd_workspace_size(int B, int64_t T, int H, int n_seqs, size_t *bytes) {
    if (!bytes) return KDA_ERR_INVALID_ARG;
    const int st = check_prefill_shape(B, T, H, KDA_CHUNK, n_seqs, KDA_F32);
    if (st != KDA_OK) return st;
    const bool packed = n_seqs > 0;
    const int64_t n_tok = packed ? T : (int64_t)B * T;
    *bytes = kda::bwd_workspace(n_tok, H, kda::bwd_chunk_slots(B, T, n_seqs));
    return KDA_OK;
}

int kda_chunk_bwd(const void *q, const void *k, const void *v, const void *log_alpha, int gate,
                  const float *beta, const float *S0, const void *dout, const float *dS_T, float *dq,
                  float *dk, float *dv, float *dgate, float *dbeta, float *dS0, int B, int64_t T, int H,
                  const int32_t *cu_seqlens, int n_seqs, const int32_t *cu_seqlens_host, int dtype,
                  const kda_io *io, void *workspace, size_t workspace_bytes, void *stream) {
    int st = check_prefill_shape(B, T, H, KDA_CHUNK, n_seqs, dtype);
    if (st != KDA_OK) return st;
    if (!valid_gate(gate)) return KDA_ERR_UNSUPPORTED;
    kda::IoOpts opts;
    st = make_io(io, false, dtype == KDA_BF16 ? 2 : 4, &opts);  // no output epilogue
    if (st != KDA_OK) return st;
    const bool packed = n_seqs > 0;
    if (packed != (cu_seqlens != nullptr)) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !beta || !dout || !dq || !dk || !dv || !dbeta))
        return KDA_ERR_INVALID_ARG;
    if (T > 0 && gate != KDA_GATE_NONE && !dgate) return KDA_ERR_INVALID_ARG;
    if (T > 0 && check_gate_ptr(log_alpha, gate, false) != KDA_OK) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens_host) {
        if (!packed || cu_seqlens_host[0] != 0 || cu_seqlens_host[n_seqs] != T) return KDA_ERR_INVALID_ARG;
        for (int s2 = 0; s2 < n_seqs; ++s2)
            if (cu_seqlens_host[s2 + 1] < cu_seqlens_host[s2]) return KDA_ERR_INVALID_ARG;
    }
    size_t need = 0;
    st = kda_chunk_bwd_workspace_size(B, T, H, n_seqs, &need);
    if (st != KDA_OK) return st;
    if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 15u) != 0) return KDA_ERR_WORKSPACE;
    kda::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0; a.dout = dout;
    a.dS_T = dS_T; a.dq = dq; a.dk = dk; a.dv = dv; a.dgate = dgate; a.dbeta = dbeta; a.dS0 = dS0;
    a.B = B; a.T = T; a.H = H; a.cu = cu_seqlens; a.n_seqs = n_seqs;
    a.n_tok = packed ? T : (int64_t)B * T;
    a.chunk_slots = kda::bwd_chunk_slots(B, T, n_seqs);
    a.workspace = workspace;
    a.io = opts;
    const cudaError_t err = kda::launch_bwd(a, gate, dtype, (cudaStream_t)stream);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_get_device_status(int *status) {
    if (!status) return KDA_ERR_INVALID_ARG;
    return kda::read_device_status(status) == 0 ? KDA_OK : KDA_ERR_CUDA;
}

int kda_set_wait_limit_ns(uint64_t ns) {
    return kda::set_wait_limit_ns((unsigned long long)ns) == 0 ? KDA_OK : KDA_ERR_CUDA;
}

int kda_selftest_wait_timeout(const int32_t *flag, int32_t *result, void *stream) {
    if (!flag || !result) return KDA_ERR_INVALID_ARG;
    if (((uintptr_t)flag & 3u) != 0 || ((uintptr_t)result & 3u) != 0) return KDA_ERR_INVALID_ARG;
    return kda::launch_wait_selftest(flag, result, (cudaStream_t)stream) == cudaSuccess ? KDA_OK
                                                                                        : KDA_ERR_CUDA;
}

int kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, float *S, void *o, int N, int H, int dtype,
                    void *stream) {
    return kda_decode_step_gated(q, k, v, log_alpha, KDA_GATE_CHANNEL, beta, S, o, N, H, dtype,
                                 stream);
}

int kda_decode_step_gated(const void *q, const void *k, const void *v, const void *log_alpha,
                          int gate, const float *beta, float *S, void *o, int N, int H,
                          int dtype, void *stream) {
    return kda_decode_step_io(q, k, v, log_alpha, gate, beta, S, o, N, H, dtype, nullptr, stream);
}

int kda_decode_step_io(const void *q, const void *k, const void *v, const void *log_alpha, int gate,
                       const float *beta, float *S, void *o, int N, int H, int dtype, const kda_io *io,
                       void *stream) {
    if (!valid_dtype(dtype) || !valid_gate(gate)) return KDA_ERR_UNSUPPORTED;
    kda::IoOpts opts;
    const int io_st = make_io(io, true, dtype == KDA_BF16 ? 2 : 4, &opts);
    if (io_st != KDA_OK) return io_st;
    if (N <= 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if ((int64_t)N * H > (int64_t)INT32_MAX) return KDA_ERR_INVALID_ARG;
    if (!q || !k || !v || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    if (check_gate_ptr(log_alpha, gate, false) != KDA_OK) return KDA_ERR_INVALID_ARG;
    if (((uintptr_t)S & 15u) != 0) return KDA_ERR_INVALID_ARG;  // 128-bit state accesses
    const cudaError_t err = kda::launch_decode(q, k, v, log_alpha, gate, beta, S, o, N, H, dtype, opts,
                                               (cudaStream_t)stream);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
