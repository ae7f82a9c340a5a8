// KDA chunk-parallel prefill on CUDA cores, all arithmetic in fp32.
//
// This is the path for fp32 inputs, where tensor-core operand rounding would
// exceed the fp32 error budget, and for chunks of C = 32 tokens in either input
// dtype (the chunk size is a template parameter, C = 32 or 64; mokono.cn section 4.1
// names 32 to 128 as the useful range). It follows the chunked form of KDA
// (mokono.cn "Kimi Linear：高效注意力机制在长序列处理中的创新应用" section 2.1,
// S_r = P_r S_0 + H_r; blog.gzher.com "Kimi K3论文：Kimi Linear" section 4:
// WY representation, UT transform, state passed from chunk to chunk). For a
// chunk of L <= C tokens with start state S (dk x dv), per key channel c:
//
//   g_r        = sum_{j<=r} log_alpha_j           (reset at every chunk)
//   A_kk[r,i]  = beta_r sum_c k_rc k_ic exp(g_rc - g_ic)   for i < r
//   A_qk[r,i]  =        sum_c q_rc k_ic exp(g_rc - g_ic)   for i <= r
//   (I + A_kk) W = Diag(beta) (exp(g) * K),  (I + A_kk) U = Diag(beta) V
//   V_new = U - W S
//   O     = (exp(g) * Q) S + A_qk V_new
//   S    <- Diag(exp(g_L)) S + (exp(g_L - g) * K)^T V_new
//
// The exp(g_r - g_i) factor is split as exp(g_r) * exp(-g_i) when the chunk's
// total log-decay is at most 80 in every channel (both factors then stay far
// from fp32 overflow); otherwise the pairwise exponentials are taken
// directly. g is accumulated as an unevaluated sum hi + lo (Knuth's two-sum),
// so differences g_r - g_i keep full fp32 precision even when a near-zero
// gate (log_alpha of -1e4, say) makes |g| huge. The triangular systems are solved by forward substitution, one
// thread per right-hand-side column.
//
// Grid: (sequence, head, dv slice of 32 columns). Each CTA walks its
// sequence's chunks in order, keeping its 128 x 32 state slice in shared
// memory; the dk-side work (gates, Grams, W) is repeated by the four slices.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int NT = 256;           // threads per CTA
constexpr int DVS = 32;           // value columns per CTA
constexpr int LD = D + 4;         // row stride of the [64][128] buffers (floats)
constexpr float SAFE_SPAN = 80.f; // max chunk log-decay for the factorised form

// CK: chunk length (32 or 64). About 201 KB for 64, 100 KB for 32; 128 would need
// about 400 KB and does not fit an SM.
template <int CK>
struct SimtSmem {
    static constexpr int LDA = CK + 1;  // row stride of the [CK][CK] buffers
    float q[CK * LD];    // q, then exp(g) * q
    float k[CK * LD];    // k, then exp(g) * k, then W (solved in place)
    float g[CK * LD];    // log_alpha, then g (high part), then exp(g_L - g) * k
    float glo[CK * LD];  // low part of g
    float akk[CK * LDA]; // beta-scaled strict-lower Gram
    float aqk[CK * LDA]; // inclusive-lower Gram
    float vu[CK * DVS];  // v slice, then U (solved in place)
    float vn[CK * DVS];  // V_new
    float s[D * DVS];    // state slice S[c][j]
    float gl[D];         // g_L per channel (high part)
    float gllo[D];       // g_L per channel (low part)
    float einv[D];       // exp(-g_L) per channel
    float beta[CK];
};

// Calls of a KDA_DEBUG build whose device offsets failed the checks (always 0 in the
// ordinary build); read and cleared with the rest of the device status.
__device__ int g_simt_bad_input = 0;

template <typename TIn>
__device__ __forceinline__ void load_row8(const TIn *src, float *dst) {
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e] = to_f32(src[e]);
}

template <typename TIn, int GATE, int CK>
__global__ void __launch_bounds__(NT, 1)
prefill_simt_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                    const TIn *__restrict__ v, const void *__restrict__ log_alpha,
                    const float *__restrict__ beta, const float *__restrict__ S0,
                    TIn *__restrict__ o, float *__restrict__ S_T, int64_t T, int H,
                    const int32_t *__restrict__ cu_seqlens, int io_flags, float l2_eps) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    using Smem = SimtSmem<CK>;
    constexpr int LDA = Smem::LDA;
    constexpr int NB = CK / 16;  // Gram blocks of 16 rows (columns) per thread
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

    const int seq = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * DVS;
    const int tid = threadIdx.x;
#ifdef KDA_DEBUG
    // Device offsets of packed sequences are checked by every CTA before any is used
    // (cu[0] = 0, non-decreasing, cu[n_seqs] = T, with n_seqs = gridDim.x); on failure
    // the CTA returns without touching the caller's tensors and the first CTA counts
    // the call in the debug status.
    if (cu_seqlens) {
        const int n_seqs = (int)gridDim.x;
        bool bad = tid == 0 && (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[n_seqs] != T);
        for (int s2 = tid; s2 < n_seqs; s2 += NT) bad |= cu_seqlens[s2 + 1] < cu_seqlens[s2];
        if (__syncthreads_or(bad)) {
            if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
                atomicAdd(&g_simt_bad_input, 1);
            return;
        }
    }
#endif
    const SeqSpan span = seq_span(cu_seqlens, T, seq);
    const int64_t state_off = ((int64_t)seq * H + h) * (int64_t)(D * D);

    for (int e = tid; e < D * DVS; e += NT) {
        const int c = e / DVS, j = e % DVS;
        sm.s[e] = S0 ? S0[state_off + (int64_t)c * D + j0 + j] : 0.f;
    }

    for (int64_t c0 = 0; c0 < span.len; c0 += CK) {
        const int L = span.len - c0 < CK ? (int)(span.len - c0) : CK;
        const int64_t tok0 = span.start + c0;
        __syncthreads();  // previous chunk finished with every buffer

        // ---- load the chunk; rows >= L become k = q = 0, log_alpha = 0, beta = 0
        for (int e = tid; e < CK * (D / 8); e += NT) {
            const int r = e / (D / 8), c8 = (e % (D / 8)) * 8;
            float *dq = sm.q + r * LD + c8, *dk = sm.k + r * LD + c8, *dg = sm.g + r * LD + c8;
            if (r < L) {
                const int64_t off = ((tok0 + r) * H + h) * (int64_t)D + c8;
                load_row8(q + off, dq);
                load_row8(k + off, dk);
#pragma unroll
                for (int x = 0; x < 8; ++x) dg[x] = gate_log<GATE>(log_alpha, (tok0 + r) * H + h, c8 + x);
            } else {
#pragma unroll
                for (int x = 0; x < 8; ++x) dq[x] = dk[x] = dg[x] = 0.f;
            }
        }
        for (int e = tid; e < CK * DVS; e += NT) {
            const int r = e / DVS, j = e % DVS;
            sm.vu[e] = r < L ? to_f32(v[((tok0 + r) * H + h) * (int64_t)D + j0 + j]) : 0.f;
        }
        if (tid < CK) {
            float b = tid < L ? beta[(tok0 + tid) * H + h] : 0.f;
            if ((io_flags & IO_BETA_LOGITS) && tid < L) b = sigmoid(b);
            sm.beta[tid] = b;
        }
        __syncthreads();
        if (io_flags & IO_QK_L2NORM) {  // q and k rows to unit length (rows >= L stay zero)
            const int warp = tid >> 5, lane = tid & 31;
            for (int r = warp; r < CK; r += NT / 32) {
                float sq = 0.f, sk = 0.f;
                for (int c = lane; c < D; c += 32) {
                    sq += sm.q[r * LD + c] * sm.q[r * LD + c];
                    sk += sm.k[r * LD + c] * sm.k[r * LD + c];
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                }
                const float nq = sq + l2_eps > 0.f ? rsqrtf(sq + l2_eps) : 0.f;
                const float nk = sk + l2_eps > 0.f ? rsqrtf(sk + l2_eps) : 0.f;
                for (int c = lane; c < D; c += 32) {
                    sm.q[r * LD + c] *= nq;
                    sm.k[r * LD + c] *= nk;
                }
            }
            __syncthreads();
        }

        // ---- g = chunk-local inclusive cumulative sum of log_alpha, per channel
        bool unsafe = false;
        if (tid < D) {
            float hi = 0.f, lo = 0.f;
            for (int r = 0; r < CK; ++r) {
                const float x = sm.g[r * LD + tid];
                const float s = hi + x, bb = s - hi;  // two-sum: s + err == hi + x exactly
                lo += (hi - (s - bb)) + (x - bb);
                hi = s;
                sm.g[r * LD + tid] = hi;
                sm.glo[r * LD + tid] = lo;
            }
            sm.gl[tid] = hi;
            sm.gllo[tid] = lo;
            sm.einv[tid] = expf(-(hi + lo));
            unsafe = -(hi + lo) > SAFE_SPAN;
        }
        unsafe = __syncthreads_or(unsafe);

        // ---- Grams. Thread (u, t) owns rows r = u + 16b and columns i = t + 16a.
        const int tu = tid / 16, tt = tid % 16;
        float accq[NB][NB], acck[NB][NB];
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int a = 0; a < NB; ++a) accq[b][a] = acck[b][a] = 0.f;
        if (unsafe) {
            // pairwise exponentials from the raw q, k, g, only where i <= r
            for (int c = 0; c < D; ++c) {
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    const int r = tu + 16 * b;
                    const float gr = sm.g[r * LD + c], grl = sm.glo[r * LD + c];
                    const float qv = sm.q[r * LD + c], kv = sm.k[r * LD + c];
#pragma unroll
                    for (int a = 0; a < NB; ++a) {
                        const int i = tt + 16 * a;
                        if (i <= r) {
                            const float d = (gr - sm.g[i * LD + c]) + (grl - sm.glo[i * LD + c]);
                            const float f = sm.k[i * LD + c] * expf(d);
                            accq[b][a] += qv * f;
                            acck[b][a] += kv * f;
                        }
                    }
                }
            }
        }
        __syncthreads();

        // ---- rescale in place: q <- exp(g) q; k <- exp(g) k; g <- exp(g_L - g) k
        for (int e = tid; e < CK * D; e += NT) {
            const int r = e / D, c = e % D;
            const float g = sm.g[r * LD + c], glo = sm.glo[r * LD + c], kv = sm.k[r * LD + c];
            const float eg = expf(g + glo);
            sm.q[r * LD + c] *= eg;
            sm.k[r * LD + c] = kv * eg;
            sm.g[r * LD + c] = kv * expf((sm.gl[c] - g) + (sm.gllo[c] - glo));
        }
        __syncthreads();

        if (!unsafe) {
            // factorised: exp(g_r - g_i) = exp(g_r) * exp(-g_i), and
            // k_i exp(-g_i) = (exp(g_L - g_i) k_i) * exp(-g_L)
            for (int c = 0; c < D; ++c) {
                const float ei = sm.einv[c];
                float qr[NB], kr[NB], ki[NB];
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    const int r = tu + 16 * b;
                    qr[b] = sm.q[r * LD + c];
                    kr[b] = sm.k[r * LD + c];
                }
#pragma unroll
                for (int a = 0; a < NB; ++a) ki[a] = sm.g[(tt + 16 * a) * LD + c] * ei;
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int a = 0; a < NB; ++a) {
                        accq[b][a] += qr[b] * ki[a];
                        acck[b][a] += kr[b] * ki[a];
                    }
            }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int a = 0; a < NB; ++a) {
                const int r = tu + 16 * b, i = tt + 16 * a;
                sm.aqk[r * LDA + i] = i <= r ? accq[b][a] : 0.f;
                sm.akk[r * LDA + i] = i < r ? sm.beta[r] * acck[b][a] : 0.f;
            }
        __syncthreads();

        // ---- forward substitution: (I + A_kk) W = beta * (exp(g) k), (I + A_kk) U = beta * v
        if (tid < D + DVS) {
            float *col = tid < D ? sm.k + tid : sm.vu + (tid - D);
            const int ld = tid < D ? LD : DVS;
            for (int r = 0; r < CK; ++r) {
                float x = sm.beta[r] * col[r * ld];
                for (int i = 0; i < r; ++i) x -= sm.akk[r * LDA + i] * col[i * ld];
                col[r * ld] = x;
            }
        }
        __syncthreads();

        // ---- V_new = U - W S   (thread: column j, rows r = tid/32 + 8m)
        const int j = tid % DVS, rb = tid / DVS;
        {
#pragma unroll
            for (int m = 0; m < CK / 8; ++m) {
                const int r = rb + 8 * m;
                float acc = sm.vu[r * DVS + j];
                for (int c = 0; c < D; ++c) acc -= sm.k[r * LD + c] * sm.s[c * DVS + j];
                sm.vn[r * DVS + j] = acc;
            }
        }
        __syncthreads();

        // ---- O = (exp(g) q) S + A_qk V_new
#pragma unroll
        for (int m = 0; m < CK / 8; ++m) {
            const int r = rb + 8 * m;
            if (r < L) {
                float acc = 0.f;
                for (int c = 0; c < D; ++c) acc += sm.q[r * LD + c] * sm.s[c * DVS + j];
                for (int i = 0; i <= r; ++i) acc += sm.aqk[r * LDA + i] * sm.vn[i * DVS + j];
                o[((tok0 + r) * H + h) * (int64_t)D + j0 + j] = from_f32<TIn>(acc);
            }
        }
        __syncthreads();

        // ---- S <- Diag(exp(g_L)) S + (exp(g_L - g) k)^T V_new
#pragma unroll 4
        for (int m = 0; m < D / 8; ++m) {
            const int c = rb + 8 * m;
            float acc = expf(sm.gl[c] + sm.gllo[c]) * sm.s[c * DVS + j];
            for (int i = 0; i < L; ++i) acc += sm.g[i * LD + c] * sm.vn[i * DVS + j];
            sm.s[c * DVS + j] = acc;
        }
    }
    __syncthreads();
    if (S_T)
        for (int e = tid; e < D * DVS; e += NT) {
            const int c = e / DVS, j = e % DVS;
            S_T[state_off + (int64_t)c * D + j0 + j] = sm.s[e];
        }
}

template <typename TIn, int GATE, int CK>
cudaError_t launch_t(const void *q, const void *k, const void *v, const void *la,
                     const float *beta, const float *S0, void *o, float *S_T, int n_seqs,
                     int64_t T, int H, const int32_t *cu, const IoOpts &io, cudaStream_t stream) {
    const size_t smem = sizeof(SimtSmem<CK>);
    cudaError_t err = cudaFuncSetAttribute(prefill_simt_kernel<TIn, GATE, CK>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid((unsigned)n_seqs, (unsigned)H, D / DVS);
    prefill_simt_kernel<TIn, GATE, CK><<<grid, NT, smem, stream>>>(
        (const TIn *)q, (const TIn *)k, (const TIn *)v, la, beta, S0, (TIn *)o, S_T, T, H, cu, io.flags,
        io.l2_eps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v,
                                const void *log_alpha, int gate, const float *beta,
                                const float *S0, void *o, float *S_T, int n_seqs, int64_t T,
                                int H, const int32_t *cu_seqlens, int dtype, int C, const IoOpts &io,
                                cudaStream_t stream) {
    return with_gate(gate, [&](auto g) {
        constexpr int G = decltype(g)::value;
        auto run = [&](auto ck) {
            constexpr int CK = decltype(ck)::value;
            if (dtype == KDA_BF16)
                return launch_t<__nv_bfloat16, G, CK>(q, k, v, log_alpha, beta, S0, o, S_T, n_seqs, T, H,
                                                      cu_seqlens, io, stream);
            return launch_t<float, G, CK>(q, k, v, log_alpha, beta, S0, o, S_T, n_seqs, T, H,
                                          cu_seqlens, io, stream);
        };
        return C == 32 ? run(std::integral_constant<int, 32>{}) : run(std::integral_constant<int, 64>{});
    });
}

int read_simt_bad_input(int *count) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_simt_bad_input, sizeof(int)) != cudaSuccess) return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_simt_bad_input, &zero, sizeof(int)) != cudaSuccess) return -1;
    *count = v;
    return 0;
}

}  // namespace kda
