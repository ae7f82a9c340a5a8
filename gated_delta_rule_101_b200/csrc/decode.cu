// KDA single-token decode step (recurrent form).
//
// One token of eq. (1), blog.gzher.com "Kimi K3论文：Kimi Linear" section 3,
// for every (sequence, head); section 4 says decode runs this recurrent form
// rather than the chunk kernel. With S' = Diag(alpha) S:
//
//   u = S'^T k,  p = S'^T q,  delta = beta (v - u)
//   S_new = S' + k delta^T,   o = S_new^T q = p + (k . q) delta
//
// so the 64 KiB fp32 state of a head is read once and written once, and the
// step is bound by HBM bandwidth (0.86 FLOP per byte).
//
// Optional fused transformations (IoOpts): q and k L2-normalised, beta given as logits,
// and the output passed through the head-wise RMSNorm and sigmoid output gate.
//
// Layout: one CTA of 256 threads per (sequence, head). Warp w owns state rows
// 16w .. 16w+15; lane l owns columns 4l .. 4l+3, so every warp access to a row
// is one contiguous 512-byte segment (float4 per lane). All 16 row loads are
// issued before any arithmetic to keep 64 KiB per CTA in flight.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;
constexpr int ROWS_PER_WARP = D / DEC_WARPS;  // 16

// Sum over the first four warps (the D = 128 threads that hold one channel each) of a
// value per thread; every one of those threads gets the total. `slot`: 4 floats of
// shared memory. Called by all threads of the CTA (it contains a barrier).
__device__ __forceinline__ float sum_channels(float x, float *slot) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if (tid < D && lane == 0) slot[warp] = x;
    __syncthreads();
    return slot[0] + slot[1] + slot[2] + slot[3];
}

// IO: the call has fused transformations (io); a template parameter, so that the plain
// step carries none of their code.
template <typename TIn, int GATE, bool IO>
__global__ void __launch_bounds__(DEC_THREADS)
decode_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
              const void *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ S, TIn *__restrict__ o, IoOpts io) {
    const int64_t nh = blockIdx.x;  // sequence * H + head
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    __shared__ float s_ka[D], s_qa[D], s_k[D], s_a[D];
    __shared__ float4 s_red[2][DEC_WARPS][D / 4];
    __shared__ float s_delta[D];
    __shared__ float s_qk[4];
    __shared__ float s_sum[3][4];

    float4 *Sp = reinterpret_cast<float4 *>(S + nh * (int64_t)(D * D));
    float4 st[ROWS_PER_WARP];
#pragma unroll
    for (int rr = 0; rr < ROWS_PER_WARP; ++rr)
        st[rr] = __ldcs(Sp + (warp * ROWS_PER_WARP + rr) * (D / 4) + lane);

    float kk = 0.f, qq = 0.f;
    if constexpr (IO) {
        kk = tid < D ? to_f32(k[nh * D + tid]) : 0.f;
        qq = tid < D ? to_f32(q[nh * D + tid]) : 0.f;
        if (io.flags & IO_QK_L2NORM) {  // uniform over the CTA
            const float sk = sum_channels(kk * kk, s_sum[0]);
            const float sq = sum_channels(qq * qq, s_sum[1]);
            kk *= sk + io.l2_eps > 0.f ? rsqrtf(sk + io.l2_eps) : 0.f;
            qq *= sq + io.l2_eps > 0.f ? rsqrtf(sq + io.l2_eps) : 0.f;
        }
    }
    if (tid < D) {
        if constexpr (!IO) {
            kk = to_f32(k[nh * D + tid]);
            qq = to_f32(q[nh * D + tid]);
        }
        const float a = GATE == KDA_GATE_NONE ? 1.f : expf(gate_log<GATE>(log_alpha, nh, tid));
        s_k[tid] = kk;
        s_a[tid] = a;
        s_ka[tid] = kk * a;
        s_qa[tid] = qq * a;
        float qk = qq * kk;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
        if (lane == 0) s_qk[warp] = qk;
    }
    __syncthreads();

    float4 u = make_float4(0.f, 0.f, 0.f, 0.f), p = u;
#pragma unroll
    for (int rr = 0; rr < ROWS_PER_WARP; ++rr) {
        const int i = warp * ROWS_PER_WARP + rr;
        const float ka = s_ka[i], qa = s_qa[i];
        u.x += ka * st[rr].x; u.y += ka * st[rr].y; u.z += ka * st[rr].z; u.w += ka * st[rr].w;
        p.x += qa * st[rr].x; p.y += qa * st[rr].y; p.z += qa * st[rr].z; p.w += qa * st[rr].w;
    }
    s_red[0][warp][lane] = u;
    s_red[1][warp][lane] = p;
    __syncthreads();

    float oj = 0.f;
    if (tid < D) {
        const float *ru = reinterpret_cast<const float *>(&s_red[0][0][0]);
        const float *rp = reinterpret_cast<const float *>(&s_red[1][0][0]);
        float uj = 0.f, pj = 0.f;
#pragma unroll
        for (int w = 0; w < DEC_WARPS; ++w) {
            uj += ru[w * D + tid];
            pj += rp[w * D + tid];
        }
        float b = beta[nh];
        if (IO && (io.flags & IO_BETA_LOGITS)) b = sigmoid(b);
        const float d = b * (to_f32(v[nh * D + tid]) - uj);
        s_delta[tid] = d;
        const float qk = s_qk[0] + s_qk[1] + s_qk[2] + s_qk[3];
        oj = pj + qk * d;
    }
    if (IO && io.out_gate) {  // o <- RMSNorm(o) * w * sigmoid(gate), over the head's 128 channels
        const float ms = sum_channels(oj * oj, s_sum[2]) * (1.f / D);
        if (tid < D) {
            const float w = io.out_w ? io.out_w[tid] : 1.f;
            const float g = to_f32(static_cast<const TIn *>(io.out_gate)[nh * D + tid]);
            oj *= rsqrtf(ms + io.out_eps) * w * sigmoid(g);
        }
    }
    if (tid < D) o[nh * D + tid] = from_f32<TIn>(oj);
    __syncthreads();

    const float4 d4 = reinterpret_cast<const float4 *>(s_delta)[lane];
#pragma unroll
    for (int rr = 0; rr < ROWS_PER_WARP; ++rr) {
        const int i = warp * ROWS_PER_WARP + rr;
        const float a = s_a[i], kk = s_k[i];
        float4 s = st[rr];
        s.x = a * s.x + kk * d4.x;
        s.y = a * s.y + kk * d4.y;
        s.z = a * s.z + kk * d4.z;
        s.w = a * s.w + kk * d4.w;
        __stcs(Sp + i * (D / 4) + lane, s);
    }
}

}  // namespace

cudaError_t launch_decode(const void *q, const void *k, const void *v, const void *log_alpha,
                          int gate, const float *beta, float *S, void *o, int N, int H,
                          int dtype, const IoOpts &io, cudaStream_t stream) {
    const unsigned grid = (unsigned)((int64_t)N * H);
    const bool has_io = io.flags != 0 || io.out_gate != nullptr;
    with_gate(gate, [&](auto g) {
        constexpr int G = decltype(g)::value;
        auto run = [&](auto kernel, auto tin) {
            using TIn = decltype(tin);
            kernel<<<grid, DEC_THREADS, 0, stream>>>((const TIn *)q, (const TIn *)k, (const TIn *)v, log_alpha,
                                                     beta, S, (TIn *)o, io);
        };
        if (dtype == KDA_BF16) {
            if (has_io) run(decode_kernel<__nv_bfloat16, G, true>, __nv_bfloat16{});
            else run(decode_kernel<__nv_bfloat16, G, false>, __nv_bfloat16{});
        } else {
            if (has_io) run(decode_kernel<float, G, true>, float{});
            else run(decode_kernel<float, G, false>, float{});
        }
        return 0;
    });
    return cudaGetLastError();
}

}  // namespace kda
