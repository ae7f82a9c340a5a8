// KDA chunk-parallel prefill on the 5th-generation tensor cores (bf16 q/k/v).
//
// Algorithm: the chunked form of KDA (mokono.cn "Kimi Linear：高效注意力机制在
// 长序列处理中的创新应用" section 2.1: S_r = P_r S_0 + H_r with WY auxiliaries;
// blog.gzher.com "Kimi K3论文：Kimi Linear" section 4: chunks of C = 64, WY
// representation, UT transform by a strictly lower triangular inverse, state
// passed from chunk to chunk). For one chunk of L <= 64 tokens with start
// state S (dk x dv), per key channel c:
//
//   g_r        = sum_{j<=r} log_alpha_j        (reset at each chunk)
//   A_qk[r,i]  = sum_c q_rc k_ic exp(g_rc - g_ic),           i <= r
//   A_kk[r,i]  = beta_r sum_c k_rc k_ic exp(g_rc - g_ic),    i <  r
//   T          = (I + A_kk)^-1
//   W = T Diag(beta)(exp(g) * K),    U = T Diag(beta) V
//   V_new = U - W S,   O = (exp(g) * Q) S + A_qk V_new
//   S    <- Diag(exp(g_L)) S + (exp(g_L - g) * K)^T V_new
//
// Two kernels share the work:
//
//  * kda_prep_kernel, one CTA per (chunk, head), fully parallel. TMA brings
//    the chunk's q, k, v and log_alpha tiles into shared memory; one tcgen05
//    MMA forms both Grams at once as [Q e^g; K e^g] (K e^-g)^T (M = 128); the
//    64 x 64 unit lower triangular system is inverted in fp32 by blocked
//    forward substitution; two more MMAs give W^T and U^T. The results are
//    written to the workspace as ready-to-use swizzled operand images (a
//    "blob" per chunk and head).
//  * kda_chain_kernel, one CTA per (sequence, head, 64-wide value slice),
//    walks the chunks in order. Per chunk: MMA [Q~; W] S (M = 128: both the
//    output's inter-chunk part and W S), V_new = U - W S in registers, then
//    MMAs [A_qk; 0] V_new (accumulated onto the output rows) and K~^T V_new.
//    The fp32 state slice lives in registers (thread = key row); its bf16
//    copy in shared memory is the B operand of the next chunk's first MMA.
//    Blobs arrive by bulk copy, double-buffered one chunk ahead.
//
// The factorisation exp(g_r - g_i) = exp(g_r) exp(-g_i) used by the Gram MMA
// needs exp(-g) to stay finite; key channels whose log-decay over the chunk
// exceeds 80 are left out of that MMA and added exactly, with pairwise
// exponentials, on CUDA cores.
#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "tc_ptx.cuh"

namespace kda {

// Status word of the tensor-core kernels: 1 after a bounded wait gave up.
// Read and cleared by kda_get_device_status().
__device__ int g_kda_device_status = 0;

namespace {

using namespace ptx;

constexpr int NT = 128;            // threads per CTA in both kernels (4 warps)
constexpr float SAFE_SPAN = 80.f;  // largest chunk log-decay the factorised Gram accepts

// ---- one workspace blob per (chunk, head): operand images for the chain kernel
constexpr uint32_t BLOB_A1 = 0;        // [Q~; W]: 128 x 128 bf16, K-major swizzled   (32 KiB)
constexpr uint32_t BLOB_AQK = 32768;   // A_qk:    64 x 64 bf16                        (8 KiB)
constexpr uint32_t BLOB_KTT = 40960;   // K~^T:    128 x 64 bf16                       (16 KiB)
constexpr uint32_t BLOB_U = 57344;     // U:       64 x 128 bf16 (two 64-column atoms) (16 KiB)
constexpr uint32_t BLOB_GAM = 73728;   // exp(g_L): 128 fp32
constexpr uint32_t BLOB_BYTES = 74240;

// ---- prep kernel shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t P_A1 = 0;          // 32768: Gram A = [Q e^g; K e^g], later [Q~; W]
constexpr uint32_t P_KINV = 32768;    // 16384: Gram B = K e^-g (64 x 128); later solve scratch
constexpr uint32_t P_KTT = 49152;     // 16384: K~^T (128 x 64)
constexpr uint32_t P_XWT = 65536;     // 16384: (beta e^g K)^T (128 x 64)
constexpr uint32_t P_XUT = 81920;     // 16384: (beta V)^T (128 x 64)
constexpr uint32_t P_RAW = 98304;     // 81920: raw TMA tiles, reused after the gates are built
constexpr uint32_t R_Q = 0, R_K = 16384, R_V = 32768, R_G = 49152;  // q, k, v bf16; log_alpha fp32
constexpr uint32_t P_AQK = P_RAW + 0;       // 8192: A_qk image (64 x 64)
constexpr uint32_t P_TB = P_RAW + 8192;     // 8192: T image (64 x 64), B operand of the W/U MMAs
constexpr uint32_t P_UIMG = P_RAW + 16384;  // 16384: U image
constexpr uint32_t P_AKK = P_RAW + 32768;   // 64 x 65 fp32
constexpr uint32_t P_TF = P_RAW + 49408;    // 64 x 65 fp32
constexpr uint32_t P_GAM = 180224;          // 512
constexpr uint32_t P_BETA = 180736;         // 256
constexpr uint32_t P_BADL = 180992;         // 512: list of key channels needing the exact path
constexpr uint32_t P_BAR = 181504;          // 2 mbarriers
constexpr uint32_t P_TMEM = 181520;         // TMEM base address
constexpr uint32_t PREP_SMEM = 181536 + 1024;
constexpr uint32_t PREP_TMEM_COLS = 256;  // Gram 64 + W^T 64 + U^T 64
constexpr int LDA = 65;

// ---- chain kernel shared memory
template <int N>
struct ChainLayout {
    static constexpr uint32_t A1 = 0;                 // 32768
    static constexpr uint32_t A2 = 32768;             // 16384: [A_qk; zeros]
    static constexpr uint32_t KTT = 49152;            // 16384
    static constexpr uint32_t U = 65536;              // N == 128 ? 16384 : 8192
    static constexpr uint32_t U_BYTES = N == 128 ? 16384 : 8192;
    static constexpr uint32_t GAM = U + U_BYTES;      // 512
    static constexpr uint32_t STAGE = ((GAM + 512 + 1023) / 1024) * 1024;
    static constexpr uint32_t SIMG = 2 * STAGE;       // N x 128 bf16
    static constexpr uint32_t VIMG = SIMG + N * 256;  // N x 64 bf16
    static constexpr uint32_t BAR = VIMG + N * 128;   // 3 mbarriers
    static constexpr uint32_t TMEM = BAR + 24;
    static constexpr uint32_t BYTES = TMEM + 8 + 1024;
    static constexpr uint32_t TMEM_COLS = 2 * N < 32 ? 32 : 2 * N;
    static constexpr uint32_t LOAD_BYTES = 32768 + 8192 + 16384 + U_BYTES + 512;
};

__device__ __forceinline__ unsigned char *aligned_smem(unsigned char *raw) {
    return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                             ~uintptr_t(1023));
}

__device__ __forceinline__ void st_bf16(unsigned char *base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(base + off) = __float2bfloat16_rn(x);
}

// Resolves a chunk slot into (sequence, chunk index). Returns false for slots past the end.
__device__ __forceinline__ bool resolve_slot(int slot, const int32_t *chunk_off, int n_seqs,
                                             int nck, int &seq, int &n) {
    if (!chunk_off) {
        seq = slot / nck;
        n = slot % nck;
        return true;
    }
    if (slot >= chunk_off[n_seqs]) return false;
    int lo = 0, hi = n_seqs;  // invariant: chunk_off[lo] <= slot < chunk_off[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (chunk_off[mid] <= slot) lo = mid;
        else hi = mid;
    }
    seq = lo;
    n = slot - chunk_off[lo];
    return true;
}

// =====================================================================================
// chunk offsets of packed sequences: chunk_off[s] = sum_{t<s} ceil(len_t / 64)
// =====================================================================================
__global__ void __launch_bounds__(1024)
chunk_offsets_kernel(const int32_t *__restrict__ cu, int n_seqs, int32_t *__restrict__ out) {
    __shared__ int32_t part[1024];
    const int tid = threadIdx.x;
    const int per = (n_seqs + 1023) / 1024;
    const int s0 = min(tid * per, n_seqs), s1 = min(s0 + per, n_seqs);
    int32_t local = 0;
    for (int s = s0; s < s1; ++s) local += (cu[s + 1] - cu[s] + CH - 1) / CH;
    part[tid] = local;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {  // inclusive Hillis-Steele scan
        const int32_t add = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += add;
        __syncthreads();
    }
    int32_t run = tid > 0 ? part[tid - 1] : 0;
    for (int s = s0; s < s1; ++s) {
        out[s] = run;
        run += (cu[s + 1] - cu[s] + CH - 1) / CH;
    }
    if (tid == 1023) out[n_seqs] = part[1023];
}

// =====================================================================================
// prep: per (chunk, head) gates, Grams, UT inverse, W, U -> workspace blob
// =====================================================================================
__global__ void __launch_bounds__(NT, 1)
kda_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_la,
                const float *__restrict__ beta, unsigned char *__restrict__ ws_blobs,
                const int32_t *__restrict__ chunk_off, const int32_t *__restrict__ cu, int64_t T,
                int H, int n_seqs, int nck) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = aligned_smem(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slot = blockIdx.x, h = blockIdx.y;

    int seq, n;
    if (!resolve_slot(slot, chunk_off, n_seqs, nck, seq, n)) return;
    const SeqSpan span = seq_span(cu, T, seq);
    const int64_t tok0 = span.start + (int64_t)n * CH;
    const int L = chunk_rows(span.len, (int64_t)n * CH);

    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + P_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + P_TMEM);
    float *sgam = reinterpret_cast<float *>(sm + P_GAM);
    float *sbeta = reinterpret_cast<float *>(sm + P_BETA);
    int *badl = reinterpret_cast<int *>(sm + P_BADL);
    bool dead = false;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar_tma, 3 * 16384 + 32768);
        const int x = h * D, y = (int)tok0;
        tma_load_2d(sm + P_RAW + R_Q, &tm_q, x, y, bar_tma);
        tma_load_2d(sm + P_RAW + R_K, &tm_k, x, y, bar_tma);
        tma_load_2d(sm + P_RAW + R_V, &tm_v, x, y, bar_tma);
        tma_load_2d(sm + P_RAW + R_G, &tm_la, x, y, bar_tma);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, PREP_TMEM_COLS);
        tmem_relinquish();
    }
    if (tid < CH) sbeta[tid] = tid < L ? beta[(tok0 + tid) * H + h] : 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sm_base = smem_u32(sm);

    mbar_wait(bar_tma, 0, dead, &g_kda_device_status);

    // ---- gates: thread c owns key channel c (and value column c)
    const int c = tid;
    const __nv_bfloat16 *rq = reinterpret_cast<const __nv_bfloat16 *>(sm + P_RAW + R_Q);
    const __nv_bfloat16 *rk = reinterpret_cast<const __nv_bfloat16 *>(sm + P_RAW + R_K);
    const __nv_bfloat16 *rv = reinterpret_cast<const __nv_bfloat16 *>(sm + P_RAW + R_V);
    float *rg = reinterpret_cast<float *>(sm + P_RAW + R_G);  // log_alpha, overwritten by g
    float gl = 0.f;
    for (int r = 0; r < CH; ++r) {
        gl += r < L ? rg[r * D + c] : 0.f;
        rg[r * D + c] = gl;
    }
    const bool bad = -gl > SAFE_SPAN;
    sgam[c] = expf(gl);

    // ---- operand images (rows >= L are zero)
#pragma unroll 1
    for (int qc = 0; qc < CH / 8; ++qc) {
        uint32_t kt[4], xw[4], xu[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float ktv[2], xwv[2], xuv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int r = qc * 8 + e + u;
                const bool live = r < L;
                const float g = rg[r * D + c];
                const float qv = live ? __bfloat162float(rq[r * D + c]) : 0.f;
                const float kv = live ? __bfloat162float(rk[r * D + c]) : 0.f;
                const float vv = live ? __bfloat162float(rv[r * D + c]) : 0.f;
                const float eg = expf(g);
                const float ke = kv * eg;
                st_bf16(sm, P_A1 + sw128_elem_off(r, c, 128), qv * eg);
                st_bf16(sm, P_A1 + sw128_elem_off(64 + r, c, 128), ke);
                st_bf16(sm, P_KINV + sw128_elem_off(r, c, 64), bad ? 0.f : kv * expf(-g));
                ktv[u] = kv * expf(gl - g);
                xwv[u] = sbeta[r] * ke;
                xuv[u] = sbeta[r] * vv;
            }
            kt[e / 2] = pack_bf16x2(ktv[0], ktv[1]);
            xw[e / 2] = pack_bf16x2(xwv[0], xwv[1]);
            xu[e / 2] = pack_bf16x2(xuv[0], xuv[1]);
        }
        *reinterpret_cast<uint4 *>(sm + P_KTT + sw128_chunk_off(c, qc, 128)) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
        *reinterpret_cast<uint4 *>(sm + P_XWT + sw128_chunk_off(c, qc, 128)) = make_uint4(xw[0], xw[1], xw[2], xw[3]);
        *reinterpret_cast<uint4 *>(sm + P_XUT + sw128_chunk_off(c, qc, 128)) = make_uint4(xu[0], xu[1], xu[2], xu[3]);
    }
    fence_async_smem();
    tc_fence_before();
    const int n_bad = __syncthreads_count(bad);

    // ---- Gram MMA: rows 0..63 = (Q e^g)(K e^-g)^T, rows 64..127 = (K e^g)(K e^-g)^T
    if (tid == 0) {
        tc_fence_after();
        mma_tiles(tmem, sm_base + P_A1, 128, sm_base + P_KINV, 64, D, idesc_bf16(128, 64), false);
        mma_commit(bar_mma);
    }

    // ---- exact contribution of channels left out of the MMA (pairwise exponentials)
    float acc_bad[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) acc_bad[i] = 0.f;
    const int r_own = tid & 63;
    const bool kk_row = tid >= 64;
    if (n_bad > 0) {
        if (tid == 0) {
            int m = 0;
            for (int cc = 0; cc < D; ++cc)
                if (-reinterpret_cast<float *>(sm + P_RAW + R_G)[(CH - 1) * D + cc] > SAFE_SPAN)
                    badl[m++] = cc;
        }
        __syncthreads();
        if (r_own < L) {
            for (int b = 0; b < n_bad; ++b) {
                const int cc = badl[b];
                const float xr = __bfloat162float((kk_row ? rk : rq)[r_own * D + cc]);
                const float gr = rg[r_own * D + cc];
#pragma unroll
                for (int i = 0; i < CH; ++i) {
                    const bool use = i <= r_own;  // (i < L follows from i <= r_own < L)
                    const float f = use ? __bfloat162float(rk[i * D + cc]) *
                                              expf(fminf(gr - rg[i * D + cc], 0.f))
                                        : 0.f;
                    acc_bad[i] += xr * f;
                }
            }
        }
    }

    mbar_wait(bar_mma, 0, dead, &g_kda_device_status);
    tc_fence_after();
    __syncthreads();  // raw tiles are dead from here on: their space is reused below

    {
        float G[CH];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 0, G);
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32, G + 32);
        const int r = r_own;
        if (!kk_row) {
            // A_qk row r (inclusive lower), bf16 image for the chain kernel
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
                uint32_t p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i0 = qq * 8 + 2 * e, i1 = i0 + 1;
                    const float a0 = (i0 <= r && r < L) ? G[i0] + acc_bad[i0] : 0.f;
                    const float a1 = (i1 <= r && r < L) ? G[i1] + acc_bad[i1] : 0.f;
                    p[e] = pack_bf16x2(a0, a1);
                }
                *reinterpret_cast<uint4 *>(sm + P_AQK + sw128_chunk_off(r, qq, 64)) = make_uint4(p[0], p[1], p[2], p[3]);
            }
        } else {
            float *akk = reinterpret_cast<float *>(sm + P_AKK);
            const float b = sbeta[r];
#pragma unroll
            for (int i = 0; i < CH; ++i) akk[r * LDA + i] = (i < r) ? b * (G[i] + acc_bad[i]) : 0.f;
        }
    }
    __syncthreads();

    // ---- T = (I + A_kk)^-1 by blocked forward substitution (16 x 16 blocks), fp32
    {
        const float *akk = reinterpret_cast<const float *>(sm + P_AKK);
        float *tf = reinterpret_cast<float *>(sm + P_TF);
        float *pbuf = reinterpret_cast<float *>(sm + P_KINV);  // 16 x 48 scratch
        if (lane < 16) {  // warp b inverts diagonal block b; lane l -> column l
            const int o = warp * 16, l = lane;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float x = (r == l) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < r; ++m) x -= akk[(o + r) * LDA + o + m] * t[m];
                t[r] = x;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) tf[(o + r) * LDA + o + l] = t[r];
        }
        __syncthreads();
        for (int bi = 1; bi < 4; ++bi) {  // block row bi: T_bj = -T_bb sum_{k=j}^{b-1} A_bk T_kj
            const int nent = bi * 256;
            for (int e = tid; e < nent; e += NT) {
                const int bj = e >> 8, a = (e >> 4) & 15, col = bj * 16 + (e & 15);
                const int row = bi * 16 + a;
                float s = 0.f;
                for (int m = bj * 16; m < bi * 16; ++m) s += akk[row * LDA + m] * tf[m * LDA + col];
                pbuf[a * 48 + col] = s;
            }
            __syncthreads();
            for (int e = tid; e < nent; e += NT) {
                const int bj = e >> 8, a = (e >> 4) & 15, col = bj * 16 + (e & 15);
                float s = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) s += tf[(bi * 16 + a) * LDA + bi * 16 + m] * pbuf[m * 48 + col];
                tf[(bi * 16 + a) * LDA + col] = -s;
            }
            __syncthreads();
        }
        // bf16 image of T (rows r, K = i), zero above the diagonal
        {
            const int r = tid >> 1, half = tid & 1;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i0 = half * 32 + cc * 8 + 2 * e, i1 = i0 + 1;
                    p[e] = pack_bf16x2(i0 <= r ? tf[r * LDA + i0] : 0.f, i1 <= r ? tf[r * LDA + i1] : 0.f);
                }
                *reinterpret_cast<uint4 *>(sm + P_TB + sw128_chunk_off(r, half * 4 + cc, 64)) = make_uint4(p[0], p[1], p[2], p[3]);
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- W^T = (beta e^g K)^T T^T and U^T = (beta V)^T T^T
    if (tid == 0) {
        tc_fence_after();
        mma_tiles(tmem + 64, sm_base + P_XWT, 128, sm_base + P_TB, 64, CH, idesc_bf16(128, 64), false);
        mma_tiles(tmem + 128, sm_base + P_XUT, 128, sm_base + P_TB, 64, CH, idesc_bf16(128, 64), false);
        mma_commit(bar_mma);
    }
    mbar_wait(bar_mma, 1, dead, &g_kda_device_status);
    tc_fence_after();
    {
        float w[CH];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 64, w);
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 96, w + 32);
#pragma unroll
        for (int r = 0; r < CH; ++r) st_bf16(sm, P_A1 + sw128_elem_off(64 + r, c, 128), w[r]);
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 128, w);
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 160, w + 32);
#pragma unroll
        for (int r = 0; r < CH; ++r) st_bf16(sm, P_UIMG + sw128_elem_off(r, c, 64), w[r]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    if (tid == 0) {
        unsigned char *blob = ws_blobs + ((size_t)slot * H + h) * BLOB_BYTES;
        bulk_s2g(blob + BLOB_A1, sm + P_A1, 32768);
        bulk_s2g(blob + BLOB_AQK, sm + P_AQK, 8192);
        bulk_s2g(blob + BLOB_KTT, sm + P_KTT, 16384);
        bulk_s2g(blob + BLOB_U, sm + P_UIMG, 16384);
        bulk_s2g(blob + BLOB_GAM, sm + P_GAM, 512);
        bulk_commit();
        bulk_wait_all();
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, PREP_TMEM_COLS);
}

// =====================================================================================
// chain: per (sequence, head, value slice) state recurrence over the chunks
// =====================================================================================
template <int N>
__global__ void __launch_bounds__(NT, 1)
kda_chain_kernel(const unsigned char *__restrict__ ws_blobs, const int32_t *__restrict__ chunk_off,
                 const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o,
                 float *__restrict__ S_T, const int32_t *__restrict__ cu, int64_t T, int H,
                 int nck) {
    using Lay = ChainLayout<N>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = aligned_smem(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int seq = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * N;
    const SeqSpan span = seq_span(cu, T, seq);
    const int nchunks = (int)((span.len + CH - 1) / CH);
    const int64_t slot0 = chunk_off ? (int64_t)chunk_off[seq] : (int64_t)seq * nck;
    const int64_t state_off = ((int64_t)seq * H + h) * (int64_t)(D * D);

    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + Lay::BAR);  // [2]
    uint64_t *bar_mma = bar_ld + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lay::TMEM);
    bool dead = false;

    auto issue_load = [&](int chunk, int stage) {
        const unsigned char *blob = ws_blobs + ((size_t)(slot0 + chunk) * H + h) * BLOB_BYTES;
        unsigned char *st = sm + stage * Lay::STAGE;
        mbar_arrive_expect_tx(&bar_ld[stage], Lay::LOAD_BYTES);
        bulk_g2s(st + Lay::A1, blob + BLOB_A1, 32768, &bar_ld[stage]);
        bulk_g2s(st + Lay::A2, blob + BLOB_AQK, 8192, &bar_ld[stage]);
        bulk_g2s(st + Lay::KTT, blob + BLOB_KTT, 16384, &bar_ld[stage]);
        bulk_g2s(st + Lay::U, blob + BLOB_U + (N == 128 ? 0 : (uint32_t)(j0 / 64) * 8192),
                 Lay::U_BYTES, &bar_ld[stage]);
        bulk_g2s(st + Lay::GAM, blob + BLOB_GAM, 512, &bar_ld[stage]);
    };

    if (tid == 0) {
        mbar_init(&bar_ld[0], 1);
        mbar_init(&bar_ld[1], 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, Lay::TMEM_COLS);
        tmem_relinquish();
    }
    // zero rows 64..127 of both A2 stage buffers (A2 = [A_qk; 0])
    for (int e = tid; e < 2 * 512; e += NT) {
        const int stage = e >> 9, w16 = e & 511;
        reinterpret_cast<uint4 *>(sm + stage * Lay::STAGE + Lay::A2 + 8192)[w16] = make_uint4(0, 0, 0, 0);
    }
    // state slice: thread c owns key row c, columns j0 .. j0+N-1
    const int c = tid;
    float s_reg[N];
#pragma unroll
    for (int j = 0; j < N; j += 4) {
        float4 v4 = S0 ? *reinterpret_cast<const float4 *>(S0 + state_off + (int64_t)c * D + j0 + j)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        s_reg[j] = v4.x; s_reg[j + 1] = v4.y; s_reg[j + 2] = v4.z; s_reg[j + 3] = v4.w;
    }
#pragma unroll
    for (int j = 0; j < N; ++j) st_bf16(sm, Lay::SIMG + sw128_elem_off(j, c, N), s_reg[j]);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t d1 = tmem, d3 = tmem + N;
    const uint32_t sm_base = smem_u32(sm);
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    if (tid == 0) {
        if (nchunks > 0) issue_load(0, 0);
        if (nchunks > 1) issue_load(1, 1);
    }
    uint32_t mma_phase = 0;

#pragma unroll 1
    for (int n = 0; n < nchunks && !dead; ++n) {
        const int stage = n & 1;
        unsigned char *st = sm + stage * Lay::STAGE;
        const uint32_t st_base = sm_base + stage * Lay::STAGE;
        const int64_t tok0 = span.start + (int64_t)n * CH;
        const int L = chunk_rows(span.len, (int64_t)n * CH);

        mbar_wait(&bar_ld[stage], (uint32_t)(n >> 1) & 1u, dead, &g_kda_device_status);
        // D1 = [Q~; W] S
        if (tid == 0) {
            tc_fence_after();
            mma_tiles(d1, st_base + Lay::A1, 128, sm_base + Lay::SIMG, N, D, idesc_bf16(128, N), false);
            mma_commit(bar_mma);
        }
        mbar_wait(bar_mma, mma_phase, dead, &g_kda_device_status);
        mma_phase ^= 1u;
        tc_fence_after();
        if (warp >= 2) {  // rows 64..127 of D1 hold (W S)[r]; V_new = U - W S
            const int r = tid - 64;
            float ws[N];
#pragma unroll
            for (int j = 0; j < N; j += 32)
                tmem_ld32(d1 + lane_off + j, ws + j);
#pragma unroll
            for (int jc = 0; jc < N / 8; ++jc) {
                const int jg = (N == 128 ? 0 : (j0 & 63)) + jc * 8;  // column inside the U image
                const uint4 u4 = *reinterpret_cast<const uint4 *>(st + Lay::U + sw128_chunk_off(r, jg >> 3, 64));
                const __nv_bfloat16 *ub = reinterpret_cast<const __nv_bfloat16 *>(&u4);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = jc * 8 + e;
                    st_bf16(sm, Lay::VIMG + sw128_elem_off(j, r, N), __bfloat162float(ub[e]) - ws[j]);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // D1 += [A_qk; 0] V_new ; D3 = K~^T V_new
        if (tid == 0) {
            tc_fence_after();
            mma_tiles(d1, st_base + Lay::A2, 128, sm_base + Lay::VIMG, N, CH, idesc_bf16(128, N), true);
            mma_tiles(d3, st_base + Lay::KTT, 128, sm_base + Lay::VIMG, N, CH, idesc_bf16(128, N), false);
            mma_commit(bar_mma);
        }
        mbar_wait(bar_mma, mma_phase, dead, &g_kda_device_status);
        mma_phase ^= 1u;
        tc_fence_after();
        if (warp < 2) {  // rows 0..63 of D1: the chunk's output
            const int r = tid;
            float ov[N];
#pragma unroll
            for (int j = 0; j < N; j += 32)
                tmem_ld32(d1 + lane_off + j, ov + j);
            if (r < L) {
                __nv_bfloat16 *dst = o + ((tok0 + r) * H + h) * (int64_t)D + j0;
#pragma unroll
                for (int j = 0; j < N; j += 8) {
                    uint4 pk = make_uint4(pack_bf16x2(ov[j], ov[j + 1]), pack_bf16x2(ov[j + 2], ov[j + 3]),
                                          pack_bf16x2(ov[j + 4], ov[j + 5]), pack_bf16x2(ov[j + 6], ov[j + 7]));
                    *reinterpret_cast<uint4 *>(dst + j) = pk;
                }
            }
        }
        {  // S <- Diag(exp(g_L)) S + K~^T V_new; thread c = key row c
            float dv[N];
#pragma unroll
            for (int j = 0; j < N; j += 32)
                tmem_ld32(d3 + lane_off + j, dv + j);
            const float gam = reinterpret_cast<const float *>(st + Lay::GAM)[c];
#pragma unroll
            for (int j = 0; j < N; ++j) {
                s_reg[j] = gam * s_reg[j] + dv[j];
                st_bf16(sm, Lay::SIMG + sw128_elem_off(j, c, N), s_reg[j]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && n + 2 < nchunks) issue_load(n + 2, stage);
    }

    if (S_T) {
#pragma unroll
        for (int j = 0; j < N; j += 4)
            *reinterpret_cast<float4 *>(S_T + state_off + (int64_t)c * D + j0 + j) =
                make_float4(s_reg[j], s_reg[j + 1], s_reg[j + 2], s_reg[j + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, Lay::TMEM_COLS);
}

// =====================================================================================
// host side
// =====================================================================================
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [n_tok, H*128] row-major tensor, box of 64 rows x 128 columns starting at (h*128, tok0).
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int esize, int64_t n_tok,
              int H) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)H * D, (cuuint64_t)n_tok};
    cuuint64_t strides[1] = {(cuuint64_t)H * D * esize};
    cuuint32_t box[2] = {D, CH};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int CHAIN_N = 64;

}  // namespace

size_t prefill_tc_workspace(int B, int64_t T, int H, int n_seqs) {
    if (n_seqs > 0) {
        const size_t head = (((size_t)(n_seqs + 1) * 4 + 255) / 256) * 256;
        const size_t slots = (size_t)(T / CH) + (size_t)n_seqs;
        return head + slots * (size_t)H * BLOB_BYTES;
    }
    const size_t nck = (size_t)((T + CH - 1) / CH);
    return (size_t)B * nck * (size_t)H * BLOB_BYTES;
}

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *S0, void *o, float *S_T, int B,
                              int64_t T, int H, const int32_t *cu_seqlens, int n_seqs,
                              void *workspace, cudaStream_t stream) {
    const bool packed = n_seqs > 0;
    const int nseq = packed ? n_seqs : B;
    const int64_t n_tok = packed ? T : (int64_t)B * T;
    const int nck = (int)((T + CH - 1) / CH);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    int32_t *chunk_off = nullptr;
    unsigned char *blobs = ws;
    int64_t slots = (int64_t)B * nck;
    if (packed) {
        chunk_off = reinterpret_cast<int32_t *>(ws);
        blobs = ws + (((size_t)(n_seqs + 1) * 4 + 255) / 256) * 256;
        slots = T / CH + n_seqs;
        chunk_offsets_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, n_seqs, chunk_off);
    }
    cudaError_t err;
    if (n_tok > 0 && slots > 0) {
        CUtensorMap mq, mk, mv, mla;
        if (!make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_tok, H) ||
            !make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_tok, H) ||
            !make_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_tok, H) ||
            !make_map(&mla, log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, n_tok, H))
            return cudaErrorInvalidValue;
        err = cudaFuncSetAttribute(kda_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)PREP_SMEM);
        if (err != cudaSuccess) return err;
        kda_prep_kernel<<<dim3((unsigned)slots, (unsigned)H), NT, PREP_SMEM, stream>>>(
            mq, mk, mv, mla, beta, blobs, chunk_off, cu_seqlens, T, H, n_seqs, nck);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    using Lay = ChainLayout<CHAIN_N>;
    err = cudaFuncSetAttribute(kda_chain_kernel<CHAIN_N>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::BYTES);
    if (err != cudaSuccess) return err;
    kda_chain_kernel<CHAIN_N><<<dim3((unsigned)nseq, (unsigned)H, D / CHAIN_N), NT, Lay::BYTES, stream>>>(
        blobs, chunk_off, S0, (__nv_bfloat16 *)o, S_T, cu_seqlens, T, H, nck);
    return cudaGetLastError();
}

int read_device_status(int *status) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_kda_device_status, sizeof(int)) != cudaSuccess) return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_kda_device_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    *status = v;
    return 0;
}

}  // namespace kda
