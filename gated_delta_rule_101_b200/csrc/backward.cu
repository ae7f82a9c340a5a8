// KDA backward pass: gradients of a prefill call, all arithmetic in fp32 on CUDA cores.
//
// The loss is L = sum(o * do) + sum(S_T * dS_T) for the outputs of kda_chunk_fwd. Each
// token's step of eq. (1) (blog.gzher.com "Kimi K3论文：Kimi Linear", section 3),
//
//   S' = Diag(a) S_{t-1},  a = exp(log_alpha_t);   u = S'^T k;   d = beta (v - u);
//   S_t = S' + k d^T;      o_t = S_t^T q,
//
// is differentiated in reverse order with G = dL/dS_t (section 4 of the same page counts
// the training cost of the chunked form; this is the plain recurrent reverse pass that
// any training backward must reproduce):
//
//   G  += q do^T               dq = S_t do
//   dd  = G^T k                dk = G d + S' du,   du = -beta dd,   dv = beta dd
//   dbeta = dd . (v - u)       G' = G + k du^T
//   dlog_alpha = a * rowsum(G' * S_{t-1})           G = Diag(a) G'
//
// and dS0 = G at the start. Value columns never mix in G's recurrence, so the work is
// split into slices of 32 value columns; dq, dk, dlog_alpha and dbeta are sums over all
// columns, so each slice writes its share and a second kernel adds the four shares in a
// fixed order (no atomics: the result is bitwise reproducible).
//
// kda_bwd_slice_kernel, grid (sequence, head, slice), 256 threads. Thread (warp w, lane
// l) holds rows 16w .. 16w+15 of column l of the slice's state and gradient in
// registers. Phase A runs the sequence forward once and keeps the state at every chunk
// start (chunks of BW_CH = 32 tokens) in the workspace. Phase B walks the chunks backwards: it reruns the
// chunk forward from its start state, keeping the state before each token in the
// workspace and u, d in shared memory, then takes the chunk's tokens in reverse.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int BW_NT = 256;
constexpr int BW_J = 32;                    // value columns per slice
constexpr int BW_SLICES = D / BW_J;         // 4
constexpr int BW_ROWS = D / (BW_NT / 32);   // 16 state rows per warp
constexpr int BW_PARTS = 3 * D + 1;         // per token and slice: dq, dk, dlog_alpha shares, dbeta share
constexpr size_t BW_SLICE_STATE = (size_t)D * BW_J;  // floats of one state slice
// Per-token states of the chunk being replayed live in one of BW_SM_SLOTS scratch slots.
// A CTA claims a free slot at its start (atomic compare-and-swap on a per-slot word,
// starting from its SM's index) and frees it at its end. At most two CTAs of this kernel
// are resident per SM (shared memory and __launch_bounds__), so with more slots than
// twice the SMs a free slot always exists; the claim does not depend on CTAs staying on
// one SM.
constexpr int BW_SM_SLOTS = 512;
// Tokens per replayed chunk. 32 keeps a CTA's shared memory (the chunk's q, k, rates, v
// and dout) small enough for two CTAs per SM.
constexpr int BW_CH = 32;
// Tokens of the replayed chunk starting at token c0 of a sequence of seq_len tokens.
__device__ __forceinline__ int bw_chunk_rows(int64_t seq_len, int64_t c0) {
    const int64_t left = seq_len - c0;
    return left < BW_CH ? (int)left : BW_CH;
}

// About 82 KB: two CTAs per SM.
struct BwdSmem {
    float q[BW_CH][D], k[BW_CH][D], a[BW_CH][D];  // the chunk's q, k and per-channel rates a = exp(log_alpha)
    float beta[BW_CH];
    float v[BW_CH][BW_J], dout[BW_CH][BW_J];   // the slice's v and do
    float u[BW_CH][BW_J], dd[BW_CH][BW_J];     // u_t of the forward rerun; d_t (then reused)
    float colsum[2][BW_NT / 32][BW_J];   // per-warp partial column sums, two buffers
    float rows[BW_NT / 32][BW_ROWS][BW_J + 1];  // per-warp row-sum transposition
};

// Sum over the state's 128 rows of x (this thread's 16 rows, column lane), for every
// column: the result is returned to all threads of column lane. One CTA barrier: the
// calls alternate between two buffers (`buf`, flipped here), so a buffer is written
// again only after the barrier of the next call, when every thread has read it.
__device__ __forceinline__ float col_sum(const float (&x)[BW_ROWS], BwdSmem &sm, int &buf) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < BW_ROWS; ++r) s += x[r];
    sm.colsum[buf][warp][lane] = s;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < BW_NT / 32; ++w) t += sm.colsum[buf][w][lane];
    buf ^= 1;
    return t;
}

// Sums over the slice's 32 columns of x (one value per row), for this warp's 16 rows:
// lane r < 16 gets row 16 warp + r. Warp-local.
__device__ __forceinline__ float row_sum(const float (&x)[BW_ROWS], BwdSmem &sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int r = 0; r < BW_ROWS; ++r) sm.rows[warp][r][lane] = x[r];
    __syncwarp();
    float s = 0.f;
    if (lane < BW_ROWS) {
#pragma unroll 8
        for (int j = 0; j < BW_J; ++j) s += sm.rows[warp][lane][j];
    }
    __syncwarp();
    return s;
}

template <typename TIn, int GATE>
__global__ void __launch_bounds__(BW_NT, 2)
kda_bwd_slice_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                     const void *__restrict__ log_alpha, const float *__restrict__ beta,
                     const float *__restrict__ S0, const TIn *__restrict__ dout,
                     const float *__restrict__ dS_T, float *__restrict__ dv, float *__restrict__ dS0,
                     float *__restrict__ parts, float *__restrict__ chunk_states,
                     float *__restrict__ token_states, int *__restrict__ slot_pool,
                     const int32_t *__restrict__ cu, int64_t T, int H,
                     int nck, int io_flags, float l2_eps) {
    extern __shared__ __align__(16) unsigned char bw_smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>(bw_smem_raw);
    const int seq = blockIdx.x, h = blockIdx.y, slice = blockIdx.z, j0 = slice * BW_J;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, r0 = warp * BW_ROWS;
    const SeqSpan span = seq_span(cu, T, seq);
    const int n_chunks = (int)((span.len + BW_CH - 1) / BW_CH);
    const int64_t pair = (int64_t)seq * H + h;
    // the sequence's first chunk slot: seq * nck, or for packed sequences the chunks of
    // the sequences before it (sum of ceil(len / 64))
    int64_t slot0 = (int64_t)seq * nck;
    if (cu) {
        int64_t acc = 0;
        for (int t = tid; t < seq; t += BW_NT) acc += (cu[t + 1] - cu[t] + BW_CH - 1) / BW_CH;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        __shared__ long long chunk_acc[BW_NT / 32];
        if (lane == 0) chunk_acc[warp] = acc;
        __syncthreads();
        slot0 = 0;
#pragma unroll
        for (int w = 0; w < BW_NT / 32; ++w) slot0 += chunk_acc[w];
        __syncthreads();
    }
    __shared__ int slot_s;
    if (tid == 0) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        int got = -1;
        for (int i = 0; i < 2 * BW_SM_SLOTS && got < 0; ++i) {  // bounded: a free slot exists
            const int cand = (int)((smid + (uint32_t)i) % BW_SM_SLOTS);
            if (atomicCAS(slot_pool + cand, 0, 1) == 0) got = cand;
        }
        slot_s = got;
    }
    __syncthreads();
    const int slot = slot_s;
    if (slot < 0) return;  // cannot happen with more slots than SMs
    // this CTA's scratch: a state slice per chunk start, and per token of the current chunk
    const size_t cstride = (size_t)H * BW_SLICES * BW_SLICE_STATE;  // between chunk slots
    float *cbase = chunk_states + ((size_t)slot0 * H + h) * BW_SLICES * BW_SLICE_STATE + slice * BW_SLICE_STATE;
    float *tstates = token_states + (size_t)slot * BW_CH * BW_SLICE_STATE;
    auto st_off = [&](int r) { return (size_t)(r0 + r) * BW_J + lane; };
    int cbuf = 0;  // col_sum's buffer

    // Loads a chunk's q, k, a and beta (rows >= L zero; a = 1 there) and the slice's v, do.
    auto load_chunk = [&](int64_t tok0, int L) {
        for (int e = tid; e < BW_CH * D; e += BW_NT) {
            const int r = e / D, c = e % D;
            const bool live = r < L;
            const int64_t row = (tok0 + r) * H + h;
            sm.q[r][c] = live ? to_f32(q[row * D + c]) : 0.f;
            sm.k[r][c] = live ? to_f32(k[row * D + c]) : 0.f;
            sm.a[r][c] = live ? expf(gate_log<GATE>(log_alpha, row, c)) : 1.f;
        }
        for (int e = tid; e < BW_CH * BW_J; e += BW_NT) {
            const int r = e / BW_J, j = e % BW_J;
            const int64_t row = (tok0 + r) * H + h;
            sm.v[r][j] = r < L ? to_f32(v[row * D + j0 + j]) : 0.f;
            sm.dout[r][j] = r < L ? to_f32(dout[row * D + j0 + j]) : 0.f;
        }
        if (tid < BW_CH) {
            float b = tid < L ? beta[(tok0 + tid) * H + h] : 0.f;
            if ((io_flags & IO_BETA_LOGITS) && tid < L) b = sigmoid(b);
            sm.beta[tid] = b;
        }
        __syncthreads();
        if (io_flags & IO_QK_L2NORM) {  // the rows the forward used
            for (int r = warp; r < BW_CH; r += BW_NT / 32) {
                float sq = 0.f, sk = 0.f;
                for (int c = lane; c < D; c += 32) {
                    sq += sm.q[r][c] * sm.q[r][c];
                    sk += sm.k[r][c] * sm.k[r][c];
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                }
                const float nq = sq + l2_eps > 0.f ? rsqrtf(sq + l2_eps) : 0.f;
                const float nk = sk + l2_eps > 0.f ? rsqrtf(sk + l2_eps) : 0.f;
                for (int c = lane; c < D; c += 32) {
                    sm.q[r][c] *= nq;
                    sm.k[r][c] *= nk;
                }
            }
            __syncthreads();
        }
    };
    // One forward token step on the slice state s (in registers); writes u and d of the
    // token to shared memory row t.
    auto forward_token = [&](float (&s)[BW_ROWS], int t) {
        float ka[BW_ROWS];
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) {
            s[r] *= sm.a[t][r0 + r];
            ka[r] = s[r] * sm.k[t][r0 + r];
        }
        const float u = col_sum(ka, sm, cbuf);
        const float d = sm.beta[t] * (sm.v[t][lane] - u);
        if (warp == 0) {
            sm.u[t][lane] = u;
            sm.dd[t][lane] = d;
        }
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) s[r] += sm.k[t][r0 + r] * d;
    };

    // ---- phase A: the state at every chunk start
    float s[BW_ROWS];
#pragma unroll
    for (int r = 0; r < BW_ROWS; ++r) s[r] = S0 ? S0[pair * D * D + (int64_t)(r0 + r) * D + j0 + lane] : 0.f;
    for (int n = 0; n < n_chunks; ++n) {
        const int64_t tok0 = span.start + (int64_t)n * BW_CH;
        const int L = bw_chunk_rows(span.len, (int64_t)n * BW_CH);
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) cbase[(size_t)n * cstride + st_off(r)] = s[r];
        if (n + 1 == n_chunks) break;  // the last chunk's tokens are replayed in phase B
        load_chunk(tok0, L);
        for (int t = 0; t < L; ++t) forward_token(s, t);
        __syncthreads();
    }

    // ---- phase B: chunks in reverse
    float G[BW_ROWS];
#pragma unroll
    for (int r = 0; r < BW_ROWS; ++r) G[r] = dS_T ? dS_T[pair * D * D + (int64_t)(r0 + r) * D + j0 + lane] : 0.f;
    for (int n = n_chunks - 1; n >= 0; --n) {
        const int64_t tok0 = span.start + (int64_t)n * BW_CH;
        const int L = bw_chunk_rows(span.len, (int64_t)n * BW_CH);
        __syncthreads();
        load_chunk(tok0, L);
        // rerun the chunk forward, keeping the state before each token
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) s[r] = cbase[(size_t)n * cstride + st_off(r)];
        for (int t = 0; t < L; ++t) {
#pragma unroll
            for (int r = 0; r < BW_ROWS; ++r) tstates[(size_t)t * BW_SLICE_STATE + st_off(r)] = s[r];
            forward_token(s, t);
        }
        __syncthreads();
        // s is the state after the chunk's last token; tokens in reverse
        // S_{t-1} of the next token back is loaded while the current token is worked on
        float nxt[BW_ROWS];
        if (L > 0) {
#pragma unroll
            for (int r = 0; r < BW_ROWS; ++r) nxt[r] = tstates[(size_t)(L - 1) * BW_SLICE_STATE + st_off(r)];
        }
        for (int t = L - 1; t >= 0; --t) {
            float prev[BW_ROWS];  // S_{t-1}
#pragma unroll
            for (int r = 0; r < BW_ROWS; ++r) prev[r] = nxt[r];
            if (t > 0) {
#pragma unroll
                for (int r = 0; r < BW_ROWS; ++r) nxt[r] = tstates[(size_t)(t - 1) * BW_SLICE_STATE + st_off(r)];
            }
            const float do_j = sm.dout[t][lane];
            const float d_j = sm.dd[t][lane], u_j = sm.u[t][lane];
            float x[BW_ROWS];
            // G += q do^T;  dq share = S_t do
#pragma unroll
            for (int r = 0; r < BW_ROWS; ++r) {
                G[r] += sm.q[t][r0 + r] * do_j;
                x[r] = s[r] * do_j;
            }
            const float dq_sh = row_sum(x, sm);
            // dd = G^T k
#pragma unroll
            for (int r = 0; r < BW_ROWS; ++r) x[r] = G[r] * sm.k[t][r0 + r];
            const float dd_j = col_sum(x, sm, cbuf);
            const float b = sm.beta[t];
            const float du_j = -b * dd_j;
            float* part = parts + ((size_t)(tok0 + t) * H + h) * (BW_SLICES * BW_PARTS) + (size_t)slice * BW_PARTS;
            if (warp == 0) dv[((tok0 + t) * H + h) * (int64_t)D + j0 + lane] = b * dd_j;
            // dk share = G d + S' du  (S' = Diag(a) S_{t-1})
#pragma unroll
            for (int r = 0; r < BW_ROWS; ++r) x[r] = G[r] * d_j + sm.a[t][r0 + r] * prev[r] * du_j;
            const float dk_sh = row_sum(x, sm);
            // G' = G + k du^T;  dlog_alpha share = a * rowsum(G' * S_{t-1});  G = Diag(a) G'
#pragma unroll
            for (int r = 0; r < BW_ROWS; ++r) {
                G[r] += sm.k[t][r0 + r] * du_j;
                x[r] = G[r] * prev[r];
            }
            const float dl_sh = row_sum(x, sm);
            if (lane < BW_ROWS) {
                const int c = r0 + lane;
                part[c] = dq_sh;
                part[D + c] = dk_sh;
                part[2 * D + c] = sm.a[t][c] * dl_sh;
            }
            // dbeta share = dd . (v - u) over the slice's columns
            {
                float xb = dd_j * (sm.v[t][lane] - u_j);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) xb += __shfl_xor_sync(0xffffffffu, xb, off);
                if (warp == 0 && lane == 0) part[3 * D] = xb;
            }
#pragma unroll
            for (int r = 0; r < BW_ROWS; ++r) {
                G[r] *= sm.a[t][r0 + r];
                s[r] = prev[r];
            }
        }
    }
    if (dS0) {
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) dS0[pair * D * D + (int64_t)(r0 + r) * D + j0 + lane] = G[r];
    }
    __syncthreads();  // every thread is done with the slot
    if (tid == 0) atomicExch(slot_pool + slot, 0);
}

// Adds the four slices' shares of one token-head in a fixed order and writes dq, dk, the
// gate's gradient in its layout, and dbeta. Gate gradients: per-channel log layouts get
// dlog_alpha; a head gate gets its sum over channels; logit layouts (alpha = sigmoid(z))
// get dz = dlog_alpha * (1 - alpha); no gate writes nothing. A q or k normalised in the
// kernel passes its gradient through the normalisation: for x = y / n, n = sqrt(|y|^2 +
// eps), dy = (dx - x (x . dx)) / n.
template <typename TIn, int GATE>
__global__ void __launch_bounds__(D)
kda_bwd_reduce_kernel(const float *__restrict__ parts, const TIn *__restrict__ q, const TIn *__restrict__ k,
                      const void *__restrict__ log_alpha, const float *__restrict__ beta,
                      float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dgate,
                      float *__restrict__ dbeta, int H, int io_flags, float l2_eps) {
    const int64_t row = blockIdx.x;  // token * H + head
    const int c = threadIdx.x, warp = c >> 5, lane = c & 31;
    __shared__ float red[4][4];
    const float *p = parts + (size_t)row * (BW_SLICES * BW_PARTS);
    float gq = 0.f, gk = 0.f, gl = 0.f, gb = 0.f;
#pragma unroll
    for (int sl = 0; sl < BW_SLICES; ++sl) {
        gq += p[sl * BW_PARTS + c];
        gk += p[sl * BW_PARTS + D + c];
        gl += p[sl * BW_PARTS + 2 * D + c];
        if (c == 0) gb += p[sl * BW_PARTS + 3 * D];
    }
    auto block_sum = [&](float x, int slot) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (lane == 0) red[slot][warp] = x;
        __syncthreads();
        return red[slot][0] + red[slot][1] + red[slot][2] + red[slot][3];
    };
    if (io_flags & IO_QK_L2NORM) {
        const float yq = to_f32(q[row * D + c]), yk = to_f32(k[row * D + c]);
        const float sq = block_sum(yq * yq, 0), sk = block_sum(yk * yk, 1);
        const float nq = sq + l2_eps > 0.f ? rsqrtf(sq + l2_eps) : 0.f;
        const float nk = sk + l2_eps > 0.f ? rsqrtf(sk + l2_eps) : 0.f;
        const float xq = yq * nq, xk = yk * nk;
        const float pq = block_sum(xq * gq, 2), pk = block_sum(xk * gk, 3);
        gq = (gq - xq * pq) * nq;
        gk = (gk - xk * pk) * nk;
    }
    dq[row * D + c] = gq;
    dk[row * D + c] = gk;
    if (c == 0) {
        if (io_flags & IO_BETA_LOGITS) {
            const float s = sigmoid(beta[row]);
            gb *= s * (1.f - s);
        }
        dbeta[row] = gb;
    }
    if constexpr (GATE == KDA_GATE_HEAD) {
        __syncthreads();
        const float t = block_sum(gl, 0);
        if (c == 0) dgate[row] = t;
    } else if constexpr (logit_gate<GATE>()) {
        const float a = expf(gate_log<GATE>(log_alpha, row, c));
        dgate[row * D + c] = gl * (1.f - a);
    } else if constexpr (GATE != KDA_GATE_NONE) {
        dgate[row * D + c] = gl;
    }
}

template <typename TIn, int GATE>
cudaError_t launch_bwd_t(const BwdArgs &a, int n_seqs, int nck, cudaStream_t stream) {
    const size_t smem = sizeof(BwdSmem);
    cudaError_t err = cudaFuncSetAttribute(kda_bwd_slice_kernel<TIn, GATE>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int *pool = static_cast<int *>(a.workspace);  // BW_SM_SLOTS words, cleared here
    float *parts = reinterpret_cast<float *>(pool + BW_SM_SLOTS);
    float *cstates = parts + (size_t)a.n_tok * a.H * (BW_SLICES * BW_PARTS);
    float *tstates = cstates + (size_t)a.chunk_slots * a.H * BW_SLICES * BW_SLICE_STATE;
    err = cudaMemsetAsync(pool, 0, BW_SM_SLOTS * sizeof(int), stream);
    if (err != cudaSuccess) return err;
    kda_bwd_slice_kernel<TIn, GATE><<<dim3((unsigned)n_seqs, (unsigned)a.H, BW_SLICES), BW_NT, smem, stream>>>(
        (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, a.log_alpha, a.beta, a.S0,
        (const TIn *)a.dout, a.dS_T, a.dv, a.dS0, parts, cstates, tstates, pool, a.cu, a.T, a.H, nck,
        a.io.flags, a.io.l2_eps);
    err = cudaGetLastError();
    if (err != cudaSuccess || a.n_tok == 0) return err;
    kda_bwd_reduce_kernel<TIn, GATE><<<(unsigned)(a.n_tok * a.H), D, 0, stream>>>(
        parts, (const TIn *)a.q, (const TIn *)a.k, a.log_alpha, a.beta, a.dq, a.dk, a.dgate, a.dbeta, a.H,
        a.io.flags, a.io.l2_eps);
    return cudaGetLastError();
}

}  // namespace

// Replayed chunks of a call: B * ceil(T / BW_CH), or for packed sequences at most
// T / BW_CH + n_seqs (each sequence adds at most one partial chunk).
int64_t bwd_chunk_slots(int B, int64_t T, int n_seqs) {
    return n_seqs > 0 ? T / BW_CH + n_seqs : (int64_t)B * ((T + BW_CH - 1) / BW_CH);
}

// Workspace of kda_chunk_bwd: the replay slots' claim words, the slices' shares per
// token-head, a state slice per chunk slot and head and slice, and the replay slots.
size_t bwd_workspace(int64_t n_tok, int H, int64_t chunk_slots) {
    return (BW_SM_SLOTS + (size_t)n_tok * H * (BW_SLICES * BW_PARTS) +
            (size_t)chunk_slots * H * BW_SLICES * BW_SLICE_STATE + (size_t)BW_SM_SLOTS * BW_CH * BW_SLICE_STATE) *
           sizeof(float);
}

cudaError_t launch_bwd(const BwdArgs &a, int gate, int dtype, cudaStream_t stream) {
    const int n_seqs = a.cu ? a.n_seqs : a.B;
    const int nck = (int)((a.T + BW_CH - 1) / BW_CH);
    return with_gate(gate, [&](auto g) {
        constexpr int G = decltype(g)::value;
        if (dtype == KDA_BF16) return launch_bwd_t<__nv_bfloat16, G>(a, n_seqs, nck, stream);
        return launch_bwd_t<float, G>(a, n_seqs, nck, stream);
    });
}

}  // namespace kda
