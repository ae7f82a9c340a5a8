// Internal declarations shared by the libkda translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "kda.h"

namespace kda {

constexpr int D = KDA_HEAD_DIM;  // dk = dv
constexpr int CH = KDA_CHUNK;    // chunk length

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Log forget rate of key channel c for token-head row `row` (= token * H + head), in
// each kda_gate layout: per channel (fp32 or bf16, rows of 128), one per row (a
// head-wide scalar gate), or none (rate 1, log 0).
// log sigmoid(z) = min(z, 0) - log(1 + exp(-|z|)), so that nothing overflows; for small
// x = exp(-|z|) the logarithm is its Taylor series x - x^2 / 2 (relative error below
// x^2 / 3 < 4e-7), which keeps full relative precision where 1 + x would round to 1.
__device__ __forceinline__ float log_sigmoid(float z) {
    const float x = __expf(-fabsf(z));
    const float l = x < 1e-3f ? x * (1.f - 0.5f * x) : __logf(1.f + x);
    return fminf(z, 0.f) - l;
}
// Fast division (__fdividef: within 2 ulp; 0 once 1 + e^-z overflows) instead of the
// correctly rounded one, whose multi-instruction sequence dominated the output epilogue.
__device__ __forceinline__ float sigmoid(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

// Fused input and output transformations of the layer around the operator
// (blog.gzher.com "Kimi K3论文：Kimi Linear", section 3: q, k = L2Norm(...),
// beta = Sigmoid(W_beta x), and a head-wise RMSNorm with a sigmoid output gate before
// the output projection). Flags of IoOpts::flags:
constexpr int IO_QK_L2NORM = 1;    // q and k rows are L2-normalised in the kernel
constexpr int IO_BETA_LOGITS = 2;  // beta holds logits: the kernel uses sigmoid(beta)
struct IoOpts {
    int flags = 0;
    float l2_eps = 0.f;             // added to the sum of squares of a q / k row
    const void *out_gate = nullptr;  // [tokens][H][128] dtype, or null: no output gate and norm
    const float *out_w = nullptr;    // [128] RMSNorm weight, or null for ones
    float out_eps = 0.f;             // added to the mean square of an output row
};

// Per-channel gate layouts (one value per key channel, fp32 or bf16): log rates or logits.
template <int GATE>
constexpr bool per_channel_gate() {
    return GATE == KDA_GATE_CHANNEL || GATE == KDA_GATE_CHANNEL_BF16 || GATE == KDA_GATE_CHANNEL_LOGIT ||
           GATE == KDA_GATE_CHANNEL_LOGIT_BF16;
}
template <int GATE>
constexpr bool bf16_gate() {
    return GATE == KDA_GATE_CHANNEL_BF16 || GATE == KDA_GATE_CHANNEL_LOGIT_BF16;
}
template <int GATE>
constexpr bool logit_gate() {
    return GATE == KDA_GATE_CHANNEL_LOGIT || GATE == KDA_GATE_CHANNEL_LOGIT_BF16;
}

template <int GATE>
__device__ __forceinline__ float gate_log(const void *la, int64_t row, int c) {
    if constexpr (GATE == KDA_GATE_CHANNEL) {
        return static_cast<const float *>(la)[row * D + c];
    } else if constexpr (GATE == KDA_GATE_CHANNEL_BF16) {
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(la)[row * D + c]);
    } else if constexpr (GATE == KDA_GATE_HEAD) {
        return static_cast<const float *>(la)[row];
    } else if constexpr (GATE == KDA_GATE_CHANNEL_LOGIT) {
        return log_sigmoid(static_cast<const float *>(la)[row * D + c]);
    } else if constexpr (GATE == KDA_GATE_CHANNEL_LOGIT_BF16) {
        return log_sigmoid(__bfloat162float(static_cast<const __nv_bfloat16 *>(la)[row * D + c]));
    } else {
        return 0.f;
    }
}

// Calls f(std::integral_constant<int, GATE>) for a runtime gate layout (validated by
// the caller).
template <class F>
auto with_gate(int gate, F &&f) {
    switch (gate) {
    case KDA_GATE_CHANNEL_BF16: return f(std::integral_constant<int, KDA_GATE_CHANNEL_BF16>{});
    case KDA_GATE_HEAD: return f(std::integral_constant<int, KDA_GATE_HEAD>{});
    case KDA_GATE_NONE: return f(std::integral_constant<int, KDA_GATE_NONE>{});
    case KDA_GATE_CHANNEL_LOGIT: return f(std::integral_constant<int, KDA_GATE_CHANNEL_LOGIT>{});
    case KDA_GATE_CHANNEL_LOGIT_BF16: return f(std::integral_constant<int, KDA_GATE_CHANNEL_LOGIT_BF16>{});
    default: return f(std::integral_constant<int, KDA_GATE_CHANNEL>{});
    }
}

// Where a sequence's tokens live: [start, start + len) in token rows.
struct SeqSpan {
    int64_t start;
    int64_t len;
};

// Rows of this chunk that belong to the sequence (the chunk starts at row c0 of it).
__device__ __forceinline__ int chunk_rows(int64_t seq_len, int64_t c0) {
    const int64_t left = seq_len - c0;
    return left < CH ? (int)left : CH;
}

__device__ __forceinline__ SeqSpan seq_span(const int32_t *cu, int64_t T, int s) {
    if (cu) return {(int64_t)cu[s], (int64_t)cu[s + 1] - (int64_t)cu[s]};
    return {(int64_t)s * T, T};
}

// ---- launchers (host side); each returns cudaGetLastError() of its launch ----
cudaError_t launch_decode(const void *q, const void *k, const void *v, const void *log_alpha,
                          int gate, const float *beta, float *S, void *o, int N, int H,
                          int dtype, const IoOpts &io, cudaStream_t stream);

cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v,
                                const void *log_alpha, int gate, const float *beta, const float *S0,
                                void *o, float *S_T, int n_seqs, int64_t T, int H,
                                const int32_t *cu_seqlens, int dtype, int C, const IoOpts &io,
                                cudaStream_t stream);

// Tensor-core prefill (bf16 q/k/v): workspace bytes and launcher.
size_t prefill_tc_workspace(int B, int64_t T, int H, int n_seqs);
// l2norm: q and k are normalised in the kernel (no fused grid). The output epilogue is
// not counted (launch_out_epilogue, one more launch).
int prefill_tc_launches(int B, int64_t T, int H, int n_seqs, bool l2norm = false);
// Runs every fused step of `io` except the output epilogue.
cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const void *log_alpha,
                              int gate, const float *beta, const float *S0, void *o, float *S_T, int B,
                              int64_t T, int H, const int32_t *cu_seqlens, int n_seqs,
                              void *workspace, const IoOpts &io, cudaStream_t stream);

// Output epilogue (RMSNorm over each row's 128 channels, weights, sigmoid gate), in place
// on the `rows` rows of o (dtype KDA_BF16 or KDA_F32). Nothing is launched without
// io.out_gate or rows.
cudaError_t launch_out_epilogue(void *o, const IoOpts &io, int64_t rows, int dtype, cudaStream_t stream);

// Backward pass (kda_chunk_bwd): arguments of one call.
struct BwdArgs {
    const void *q, *k, *v, *log_alpha;
    const float *beta, *S0;
    const void *dout;
    const float *dS_T;
    float *dq, *dk, *dv, *dgate, *dbeta, *dS0;
    int B;
    int64_t T;
    int H;
    const int32_t *cu;
    int n_seqs;
    int64_t n_tok;        // tokens in all (B * T, or T packed)
    int64_t chunk_slots;  // replayed chunks in all (bwd_chunk_slots)
    void *workspace;
    IoOpts io;
};
size_t bwd_workspace(int64_t n_tok, int H, int64_t chunk_slots);
int64_t bwd_chunk_slots(int B, int64_t T, int n_seqs);
cudaError_t launch_bwd(const BwdArgs &a, int gate, int dtype, cudaStream_t stream);

// Reads and clears the device status: *status is a mask of KDA_STATUS_TIMEOUT (a bounded
// wait gave up) and KDA_STATUS_BAD_INPUT (a KDA_DEBUG build refused device offsets).
int read_device_status(int *status);
// Reads and clears the fp32 path's count of refused device offsets (KDA_DEBUG builds).
int read_simt_bad_input(int *count);
// Sets the bounded waits' time limit (0: the default of one second).
int set_wait_limit_ns(unsigned long long ns);
// Runs the bounded-wait self-test kernel (see kda_selftest_wait_timeout).
cudaError_t launch_wait_selftest(const int32_t *flag, int32_t *result, cudaStream_t stream);

}  // namespace kda
