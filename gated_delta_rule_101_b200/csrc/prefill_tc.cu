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

#include <type_traits>

#include <utility>

#include "kda_internal.cuh"
#include "tc_ptx.cuh"

namespace kda {

// Status of the tensor-core kernels: the count of bounded waits that gave up (read and
// cleared by kda_get_device_status()) and the waits' time limit.
__device__ ptx::DeviceStatus g_kda_status = {0, 0, ptx::WAIT_LIMIT_NS};

namespace {

using namespace ptx;

constexpr float SAFE_SPAN = 80.f;  // largest chunk log-decay the factorised Gram accepts

// ---- one workspace blob per (chunk, head): operand images for the chain kernel
constexpr uint32_t BLOB_A1 = 0;        // [Q~; W]: 128 x 128 bf16, K-major swizzled   (32 KiB)
constexpr uint32_t BLOB_AQK = 32768;   // A_qk:    64 x 64 bf16                        (8 KiB)
constexpr uint32_t BLOB_KTT = 40960;   // K~:      64 x 128 bf16 (rows = token)        (16 KiB)
constexpr uint32_t BLOB_TB = 57344;    // T Diag(beta): 64 x 64 bf16                  (8 KiB)
constexpr uint32_t BLOB_GAM = 65536;   // exp(g_L): 128 fp32
constexpr uint32_t BLOB_BYTES = 66048;

// ---- prep kernel shared memory (offsets from a 1024-byte aligned base). Every
// operand image is a 128-byte-swizzled tile of 128-byte rows (see tc_ptx.cuh).
// The layout keeps a CTA under 52 KB so that four run on each SM.
//   KINV rows = token i, two 64-channel blocks: (K e^-g)[i][c]; the Gram's K-major B.
//   A1   K-major, rows r' = 0..127, K = key channel c (two 64-channel blocks of 16 KiB).
//        TMA puts q in rows 0..63 and k in rows 64..127; they are scaled in place
//        to Q e^g and K e^g. Rows 64..127 are later replaced by W.
// K~ = exp(g_L - g) K, the chain's MN-major A operand K~^T, goes from registers straight
// to the blob. Once the Gram MMA has completed and the Q~ rows have been stored, KINV and
// the Q rows of A1 take A_kk / T (fp32, rows padded to LDT floats, KINV and the first
// 1 KiB of A1), the solve's scratch (in A1's first Q block) and the A_qk image (A1's
// second Q block), whose space then takes the T Diag(beta) image.
constexpr int PREP_NT = 256;
constexpr uint32_t P_KINV = 0;        // 16384 (dead after the Gram MMA)
constexpr uint32_t P_GTOT = 0;        // 8 x 128 fp32 per-warp log-decay totals (before KINV)
constexpr uint32_t P_A1 = 16384;      // 32768
constexpr uint32_t P_AKK = 0;         // 64 x 68 fp32 (17408): A_kk, then T in place
constexpr uint32_t P_PBUF = 17408;    // 4608: solve scratch (2 x [16][20], then [32][36])
constexpr uint32_t P_AQK = 32768;     // 8192: A_qk image, rows r, columns i
constexpr uint32_t P_TB = 32768;      // 8192: T Diag(beta) image (after A_qk has been stored)
constexpr uint32_t P_BADB = 17408;    // 8 x 3 x 64 fp32 bad-channel batch (Gram readout, before the solve)
constexpr uint32_t P_GAM = 49152;     // 128 fp32: exp(g_L)
constexpr uint32_t P_GL = 49664;      // 128 fp32: g_L
constexpr uint32_t P_BETA = 50176;    // 64 fp32
constexpr uint32_t P_BADL = 50432;    // 128 int
constexpr uint32_t P_BAR = 50944;     // 2 mbarriers
constexpr uint32_t P_TMEM = 50960;
constexpr uint32_t P_NBAD = 50964;    // number of listed bad channels
constexpr uint32_t P_CLAIM = 50968;   // [2] item indices handed to the worker's threads
constexpr uint32_t P_QN = 50976;      // 64 fp32: 1 / |q row| (rows L2-normalised in the kernel)
constexpr uint32_t P_KN = 51232;      // 64 fp32: 1 / |k row|
constexpr uint32_t PREP_SMEM = 51488 + 1024;
constexpr uint32_t PREP_TMEM_COLS = 128;  // Gram 64, then W 128
constexpr uint32_t PREP_TMA_BYTES = 32768;  // q, k
static_assert(P_AKK + 64 * 68 * 4 <= P_PBUF && P_PBUF + 4608 <= P_A1 + 8192,
              "prep layout: A_kk and the solve scratch must fit in KINV and A1's first Q block");
static_assert(P_AQK == P_A1 + 16384 && P_AQK + 8192 <= P_A1 + 16384 + 8192,
              "prep layout: the A_qk / T Diag(beta) image fills A1's second Q block");
static_assert(P_GTOT + 8 * 128 * 4 <= P_KINV + 16384 && P_BADB >= P_AKK + 64 * 68 * 4 &&
              P_BADB + 8 * 3 * 64 * 4 <= P_A1 + 8192 && P_A1 + 32768 <= P_GAM,
              "prep layout: scratch regions (the bad-channel batch shares the solve scratch's space)");
static_assert(4 * (PREP_SMEM + 1024) <= 233472, "four prep CTAs per SM");

// A_kk / T rows are padded to 68 floats: float4 row segments stay aligned, and
// 8 consecutive rows at the same column fall on distinct bank quads.
constexpr int LDT = 68;

// ---- chain kernel shared memory
template <int N>
struct ChainLayout {
    // One stage holds a chunk's blob and its value slice. The M = 128 operands that
    // only have 64 meaningful rows read the 64 rows stored just before or after
    // them as filler: those rows only reach accumulator rows that are dead by then.
    static constexpr uint32_t A1 = 0;                 // 32768 (K-major [Q~; W])
    static constexpr uint32_t A2 = 32768;             // A_qk (8192); rows 64..127 = start of KTT
    static constexpr uint32_t KTT = 40960;            // 16384 (MN-major K~^T: rows i, channels)
    static constexpr uint32_t TB = 57344;             // 8192: T Diag(beta); the U MMA starts 8192 earlier
    static constexpr uint32_t V = 65536;              // value slice: 64 rows x N columns (TMA, 64-column blocks)
    static constexpr uint32_t GAM = V + N * 128;      // 512
    static constexpr uint32_t STAGE = ((GAM + 512 + 1023) / 1024) * 1024;
    static constexpr uint32_t SIMG = 2 * STAGE;       // S bf16, MN-major: rows c (128), N columns
    static constexpr uint32_t VIMG = SIMG + N * 256;  // V_new bf16, MN-major: rows r (64), N columns
    static constexpr uint32_t BAR = VIMG + N * 128;   // 8 mbarriers
    static constexpr uint32_t TMEM = BAR + 64;
    static constexpr uint32_t READY = TMEM + 4;       // chunks whose blobs are known ready
    static constexpr uint32_t BYTES = TMEM + 8 + 1024;
    static constexpr uint32_t TMEM_COLS = 4 * N;      // D1 (two buffers), D3, U
    // A stage is filled in two parts, each released as soon as its readers are done:
    // part 1 (A1, TB, V) feeds the chunk's first MMAs, part 2 (A2, KTT, GAM) the rest.
    static constexpr uint32_t LOAD1_BYTES = 32768 + 8192 + N * 128;
    static constexpr uint32_t LOAD2_BYTES = 8192 + 16384 + 512;
};

// TMEM load of this thread's lane, N/2 consecutive columns.
template <int NH>
__device__ __forceinline__ void tmem_ld_half(uint32_t taddr, float *v) {
    if constexpr (NH == 32) tmem_ld32(taddr, v);
    else tmem_ld64(taddr, v);
}

__device__ __forceinline__ unsigned char *aligned_smem(unsigned char *raw) {
    return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                             ~uintptr_t(1023));
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
// The workspace of packed inputs starts with n_seqs + 2 int32: the n_seqs + 1 chunk
// offsets and a validity word, 1 when the offsets may be used. The ordinary build sets
// it to 1 unconditionally (the device offsets are trusted, or were checked on the host
// from their host copy). A KDA_DEBUG build checks them here (cu[0] = 0, non-decreasing,
// cu[n_seqs] = T); if they fail it counts the call in the device status, writes zero
// chunk offsets and a validity word of 0, and every later kernel of the call returns
// at entry without reading cu_seqlens, so nothing outside the caller's tensors is
// touched and no output is written.
__host__ __device__ constexpr size_t packed_head_bytes(int n_seqs) {
    return (((size_t)(n_seqs + 2) * 4 + 255) / 256) * 256;
}
__device__ __forceinline__ bool packed_offsets_ok(const int32_t *chunk_off, int n_seqs) {
    return chunk_off[n_seqs + 1] != 0;
}

__global__ void __launch_bounds__(1024)
chunk_offsets_kernel(const int32_t *__restrict__ cu, int n_seqs, int64_t T, int32_t *__restrict__ out) {
    __shared__ int32_t part[1024];
    const int tid = threadIdx.x;
    const int per = (n_seqs + 1023) / 1024;
    const int s0 = min(tid * per, n_seqs), s1 = min(s0 + per, n_seqs);
#ifdef KDA_DEBUG
    bool bad = tid == 0 && (cu[0] != 0 || (int64_t)cu[n_seqs] != T);
    for (int s = s0; s < s1; ++s) bad |= cu[s + 1] < cu[s];
    if (__syncthreads_or(bad)) {
        for (int s = tid; s <= n_seqs; s += 1024) out[s] = 0;
        if (tid == 0) {
            out[n_seqs + 1] = 0;
            atomicAdd(&g_kda_status.bad_input, 1);
        }
        return;
    }
#endif
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
    if (tid == 1023) {
        out[n_seqs] = part[1023];
        out[n_seqs + 1] = 1;
    }
}

// =====================================================================================
// prep: per (chunk, head) gates, Grams, UT inverse, W, U -> workspace blob
// =====================================================================================
__device__ __forceinline__ void st_chunk(unsigned char *p, const float (&v)[8]) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                               pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// Shared-memory stride between the prep workers of one CTA.
constexpr uint32_t PREP_PART = ((PREP_SMEM - 1024 + 1023) / 1024) * 1024;

// Arguments of the prep work that are fixed for a launch.
struct PrepArgs {
    const CUtensorMap *tm_q, *tm_k, *tm_la;  // tm_la: per-channel gate layouts only
    const __nv_bfloat16 *q, *k;
    const void *log_alpha;  // in the kernel's kda_gate layout
    const float *beta;
    unsigned char *ws_blobs;
    int64_t T;
    int H;
    int io_flags;   // IO_QK_L2NORM, IO_BETA_LOGITS
    float l2_eps;
    int64_t n_rows;  // token-head rows of the call (tokens x H)
};

// One prep worker: 256 threads with their own shared-memory partition (PREP_SMEM
// bytes, 1024-aligned), PREP_TMEM_COLS TMEM columns, two mbarriers and one named
// barrier. A CTA of kda_prep_kernel is one worker; a CTA of the fused kernel runs three.
template <bool SINGLE>
struct PrepWorker {
    static constexpr bool kSingle = SINGLE;
    // Everything that identifies the worker is recomputed from threadIdx (its threads
    // are PREP_NT consecutive ones, worker g = threadIdx.x / PREP_NT), so that a loop
    // over items keeps few values live across the item's code. SINGLE: the worker is
    // the whole CTA (of PREP_NT threads).
    uint32_t tma_phase;  // parity of the TMA barrier's next completion
    bool dead;
    // Thread 0: ready-flag index of the worker's last blob, not yet published (or -1).
    // It is published once that blob's stores have completed, which the worker checks
    // while it waits for its next item's loads, so that the two waits overlap.
    int pending;
    __device__ __forceinline__ static int g() { return SINGLE ? 0 : (int)(threadIdx.x / PREP_NT); }
    __device__ __forceinline__ static int tid() { return SINGLE ? (int)threadIdx.x : (int)(threadIdx.x % PREP_NT); }
    __device__ __forceinline__ static uint32_t bar_id() { return 1u + (uint32_t)g(); }
    __device__ __forceinline__ static unsigned char *sm() {
        extern __shared__ unsigned char smem_raw[];
        return aligned_smem(smem_raw) + g() * PREP_PART;
    }
    __device__ __forceinline__ void publish_pending(int32_t *ready) {
        if (pending >= 0) {
            bulk_wait_all();
            flag_publish(ready + pending);
            pending = -1;
        }
    }
    __device__ __forceinline__ static void sync() { named_bar_sync(bar_id(), PREP_NT); }
    __device__ __forceinline__ static bool sync_or(bool p) { return named_bar_or(bar_id(), PREP_NT, p); }
    // Worker-wide wait: thread 0 polls, the others sleep at the worker's barrier.
    __device__ __forceinline__ void wait(uint64_t *bar, uint32_t parity) {
        bool ok = true;
        if (tid() == 0) ok = mbar_wait(bar, parity, dead, &g_kda_status);
        dead = sync_or(!ok || dead);
    }
    // Barriers and TMEM; every thread of the worker calls this once, before any item.
    // No barrier here: the first item issues its loads at once, and reads the TMEM
    // address after its first worker barrier. `last_alloc`: no other TMEM allocation
    // follows in this CTA, so the CTA gives up its right to allocate (a CTA that has
    // done so may not allocate again).
    __device__ __forceinline__ void init(bool last_alloc) {
        tma_phase = 0;
        dead = false;
        pending = -1;
        unsigned char *s = sm();
        uint64_t *bars = reinterpret_cast<uint64_t *>(s + P_BAR);
        if (tid() == 0) {
            mbar_init(bars, 1);
            mbar_init(bars + 1, 1);
            fence_mbar_init();
        }
        if (tid() >> 5 == 1) {  // warp 1, so that thread 0 goes on to issue the first loads
            tmem_alloc(reinterpret_cast<uint32_t *>(s + P_TMEM), PREP_TMEM_COLS);
            if (last_alloc) tmem_relinquish();
        }
        tc_fence_before();
    }
    // Frees the worker's TMEM and ends its mbarriers, so that its shared memory and
    // columns can serve another role.
    __device__ __forceinline__ void release(int32_t *ready) {
        tc_fence_before();
        sync();
        tc_fence_after();
        unsigned char *s = sm();
        if (tid() >> 5 == 1) tmem_dealloc(*reinterpret_cast<volatile uint32_t *>(s + P_TMEM), PREP_TMEM_COLS);
        if (tid() == 0) {
            publish_pending(ready);
            uint64_t *bars = reinterpret_cast<uint64_t *>(s + P_BAR);
            mbar_inval(bars);
            mbar_inval(bars + 1);
        }
    }
};

// Prep of one (chunk, head): the chunk's gates, Grams, inverse and W, written to the
// chunk's workspace blob. pf(x, y) is called by thread 0 after it has issued the
// item's loads; it returns false or the coordinates of a later item's tiles, which are
// then warmed in L2. ready != null: publish the blob's ready flag. Thread 0 calls
// hook.before_wait() and hook.after_wait() around its wait for the item's loads (work
// whose latency that wait can hide).
// Log gate of channels c .. c+3 of token-head row `row` (read once: streamed past L1).
template <int GATE>
__device__ __forceinline__ float4 load_gate4(const void *la, int64_t row, int c) {
    if constexpr (GATE == KDA_GATE_CHANNEL) {
        return __ldcs(reinterpret_cast<const float4 *>(static_cast<const float *>(la) + row * D + c));
    } else if constexpr (GATE == KDA_GATE_CHANNEL_BF16) {
        const uint2 raw = __ldcs(reinterpret_cast<const uint2 *>(
            static_cast<const __nv_bfloat16 *>(la) + row * D + c));
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
        return make_float4(lo.x, lo.y, hi.x, hi.y);
    } else if constexpr (logit_gate<GATE>()) {  // z -> log sigmoid(z)
        constexpr int RAW = GATE == KDA_GATE_CHANNEL_LOGIT ? KDA_GATE_CHANNEL : KDA_GATE_CHANNEL_BF16;
        const float4 z = load_gate4<RAW>(la, row, c);
        return make_float4(log_sigmoid(z.x), log_sigmoid(z.y), log_sigmoid(z.z), log_sigmoid(z.w));
    } else if constexpr (GATE == KDA_GATE_HEAD) {
        const float x = __ldcs(static_cast<const float *>(la) + row);
        return make_float4(x, x, x, x);
    } else {
        return make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

struct NoHook {
    __device__ __forceinline__ void before_wait() {}
    __device__ __forceinline__ void after_wait() {}
};
// L2: q and k rows are L2-normalised here (IO_QK_L2NORM); a template parameter, so that
// kernels without it carry none of its code.
template <int GATE, bool L2, class Worker, class Prefetch, class Hook = NoHook>
__device__ __forceinline__ void prep_item(Worker &w, const PrepArgs &a, int slot, int h,
                                          SeqSpan span, int n, Prefetch pf,
                                          int32_t *__restrict__ ready, Hook hook = Hook()) {
    unsigned char *sm = Worker::sm();
    const int tid = Worker::tid(), warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int64_t tok0 = span.start + (int64_t)n * CH;
    const int L = chunk_rows(span.len, (int64_t)n * CH);

    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + P_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    float *sgam = reinterpret_cast<float *>(sm + P_GAM);
    float *sgl = reinterpret_cast<float *>(sm + P_GL);
    float *sbeta = reinterpret_cast<float *>(sm + P_BETA);
    int *badl = reinterpret_cast<int *>(sm + P_BADL);

    if (tid == 0) {
        mbar_arrive_expect_tx(bar_tma, PREP_TMA_BYTES);
        const int x = h * D, y = (int)tok0;
        tma_load_2d(sm + P_A1, a.tm_q, x, y, bar_tma);                  // q, channels 0..63
        tma_load_2d(sm + P_A1 + 16384, a.tm_q, x + 64, y, bar_tma);     // q, channels 64..127
        tma_load_2d(sm + P_A1 + 8192, a.tm_k, x, y, bar_tma);           // k -> rows 64..127
        tma_load_2d(sm + P_A1 + 16384 + 8192, a.tm_k, x + 64, y, bar_tma);
        int pf_x, pf_y;
        if (pf(pf_x, pf_y)) {
            tma_prefetch_l2_2d(a.tm_q, pf_x, pf_y);
            tma_prefetch_l2_2d(a.tm_q, pf_x + 64, pf_y);
            tma_prefetch_l2_2d(a.tm_k, pf_x, pf_y);
            tma_prefetch_l2_2d(a.tm_k, pf_x + 64, pf_y);
            if constexpr (per_channel_gate<GATE>() && !bf16_gate<GATE>()) {  // fp32 boxes of 128 channels
                tma_prefetch_l2_2d(a.tm_la, pf_x, pf_y);
            } else if constexpr (bf16_gate<GATE>()) {  // bf16 boxes of 64
                tma_prefetch_l2_2d(a.tm_la, pf_x, pf_y);
                tma_prefetch_l2_2d(a.tm_la, pf_x + 64, pf_y);
            }
        }
    } else if (GATE == KDA_GATE_HEAD && tid < CH) {
        // A head-wide gate (and beta) of that later item's rows: 4 bytes per token-head,
        // one cache line every 128 / (4 H) rows, so each row's thread asks for its own.
        // Only here does it pay: with per-channel gates the extra work costs more than
        // the two scattered row reads it hides.
        int pf_x, pf_y;
        if (pf(pf_x, pf_y)) {
            const int64_t prow = (int64_t)(pf_y + tid) * H + pf_x / D;
            if (prow < a.n_rows) {
                prefetch_l2(a.beta + prow);
                prefetch_l2(static_cast<const float *>(a.log_alpha) + prow);
            }
        }
    }
    if (tid < CH) {
        float b = tid < L ? a.beta[(tok0 + tid) * H + h] : 0.f;
        if ((a.io_flags & IO_BETA_LOGITS) && tid < L) b = sigmoid(b);
        sbeta[tid] = b;
    }

    // ---- g = chunk-local cumulative sum of log_alpha (rows >= L count as 0), while
    //      the q / k tiles are in flight. Thread (w, f) loads rows 8w .. 8w+7, channels
    //      4f .. 4f+3 straight into registers, sums down its rows, and adds the totals
    //      of the warps before it; g_L is the sum of all eight totals.
    const int f = lane, fblk = f >> 4, fchunk = (f & 15) >> 1, fhalf = (f & 1) * 8;
    float4 g4[8];
    float gls[4], gams[4];
    if constexpr (GATE == KDA_GATE_NONE) {  // no decay: g = 0, exp(g_L) = 1
#pragma unroll
        for (int v = 0; v < 8; ++v) g4[v] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 4; ++e) { gls[e] = 0.f; gams[e] = 1.f; }
        if (warp == 0) {
            *reinterpret_cast<float4 *>(sgl + 4 * f) = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(sgam + 4 * f) = make_float4(1.f, 1.f, 1.f, 1.f);
        }
    } else {
        const int64_t row0 = tok0 * H + h;  // token-head row of the chunk's first token
        if constexpr (logit_gate<GATE>()) {
            // all eight rows' loads first, then log sigmoid: the loads stay in flight together
            constexpr int RAW = GATE == KDA_GATE_CHANNEL_LOGIT ? KDA_GATE_CHANNEL : KDA_GATE_CHANNEL_BF16;
            constexpr float ZERO_LOGIT = 1e30f;  // rows >= L: log sigmoid(+big) = 0
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int r = 8 * warp + v;
                g4[v] = r < L ? load_gate4<RAW>(a.log_alpha, row0 + (int64_t)r * H, 4 * f)
                              : make_float4(ZERO_LOGIT, ZERO_LOGIT, ZERO_LOGIT, ZERO_LOGIT);
            }
#pragma unroll
            for (int v = 0; v < 8; ++v)
                g4[v] = make_float4(log_sigmoid(g4[v].x), log_sigmoid(g4[v].y), log_sigmoid(g4[v].z),
                                    log_sigmoid(g4[v].w));
        } else {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int r = 8 * warp + v;
                g4[v] = r < L ? load_gate4<GATE>(a.log_alpha, row0 + (int64_t)r * H, 4 * f)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int v = 1; v < 8; ++v) {
            g4[v].x += g4[v - 1].x; g4[v].y += g4[v - 1].y;
            g4[v].z += g4[v - 1].z; g4[v].w += g4[v - 1].w;
        }
        float *gtot = reinterpret_cast<float *>(sm + P_GTOT);
        *reinterpret_cast<float4 *>(gtot + warp * D + 4 * f) = g4[7];
        w.sync();
        float4 off = make_float4(0.f, 0.f, 0.f, 0.f), tot = off;
#pragma unroll
        for (int w2 = 0; w2 < 8; ++w2) {
            const float4 t = *reinterpret_cast<const float4 *>(gtot + w2 * D + 4 * f);
            if (w2 < warp) { off.x += t.x; off.y += t.y; off.z += t.z; off.w += t.w; }
            tot.x += t.x; tot.y += t.y; tot.z += t.z; tot.w += t.w;
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            g4[v].x += off.x; g4[v].y += off.y; g4[v].z += off.z; g4[v].w += off.w;
        }
        gls[0] = tot.x; gls[1] = tot.y; gls[2] = tot.z; gls[3] = tot.w;
#pragma unroll
        for (int e = 0; e < 4; ++e) gams[e] = expf(gls[e]);
        if (warp == 0) {
            *reinterpret_cast<float4 *>(sgl + 4 * f) = tot;
            *reinterpret_cast<float4 *>(sgam + 4 * f) = make_float4(gams[0], gams[1], gams[2], gams[3]);
        }
    }
    bool badc[4], any_bad = false;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        badc[e] = -gls[e] > SAFE_SPAN;
        any_bad |= badc[e];
    }
    // (this barrier also ends the reads of the warp totals, whose space becomes KINV)
    const int n_bad = w.sync_or(any_bad) ? 1 : 0;
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + P_TMEM);
    const uint32_t sm_base = smem_u32(sm);
    if (tid == 0) {
        hook.before_wait();
        // The previous item's stores are the only bulk stores in flight; waiting for
        // them here overlaps this item's loads and keeps warp 0 free until now.
        w.publish_pending(ready);
    }
    w.wait(bar_tma, w.tma_phase);
    if (tid == 0) hook.after_wait();
    w.tma_phase ^= 1u;

    // ---- gates and operand images, row by row. BAD selects the exact handling of key
    //      channels whose chunk log-decay exceeds SAFE_SPAN (kept out of the unrolled
    //      common path so that it stays branch-free).
    constexpr bool l2 = L2;
    unsigned char *blob = a.ws_blobs + ((size_t)slot * H + h) * BLOB_BYTES;
    float *sqn = reinterpret_cast<float *>(sm + P_QN);
    float *skn = reinterpret_cast<float *>(sm + P_KN);
    auto gate_rows = [&](auto bad_tag) {
        constexpr bool BAD = decltype(bad_tag)::value;
        unsigned char *blk = sm + P_A1 + fblk * 16384;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int r = 8 * warp + v;
            const bool live = r < L;
            const uint2 qraw = *reinterpret_cast<const uint2 *>(blk + sw128_chunk_off(r, fchunk, 128) + fhalf);
            const uint2 kraw = *reinterpret_cast<const uint2 *>(blk + sw128_chunk_off(64 + r, fchunk, 128) + fhalf);
            const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(&qraw);
            const __nv_bfloat16 *kb = reinterpret_cast<const __nv_bfloat16 *>(&kraw);
            float xq[4], xk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                xq[e] = live ? __bfloat162float(qb[e]) : 0.f;
                xk[e] = live ? __bfloat162float(kb[e]) : 0.f;
            }
            if constexpr (L2) {  // the warp holds the whole row (lane f: channels 4f .. 4f+3)
                float sq = xq[0] * xq[0] + xq[1] * xq[1] + xq[2] * xq[2] + xq[3] * xq[3];
                float sk = xk[0] * xk[0] + xk[1] * xk[1] + xk[2] * xk[2] + xk[3] * xk[3];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                }
                const float nq = sq + a.l2_eps > 0.f ? rsqrtf(sq + a.l2_eps) : 0.f;
                const float nk = sk + a.l2_eps > 0.f ? rsqrtf(sk + a.l2_eps) : 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xq[e] *= nq;
                    xk[e] *= nk;
                }
                if (lane == 0) {
                    sqn[r] = nq;
                    skn[r] = nk;
                }
            }
            const float gs[4] = {g4[v].x, g4[v].y, g4[v].z, g4[v].w};
            // a head-wide gate has one g per row: its two exponentials serve all channels
            const float eg_row = GATE == KDA_GATE_NONE ? 1.f : __expf(gs[0]);
            const float ein_row = GATE == KDA_GATE_NONE ? 1.f : __expf(-gs[0]);
            constexpr bool ROW_GATE = GATE == KDA_GATE_HEAD || GATE == KDA_GATE_NONE;
            float qe[4], ke[4], kin[4], kt[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float x = xq[e];
                const float kk = xk[e];
                const float eg = ROW_GATE ? eg_row : __expf(gs[e]);
                qe[e] = x * eg;
                ke[e] = kk * eg;
                // exp(-g) <= exp(80) for good channels
                const float kin_ = kk * (ROW_GATE ? ein_row : __expf(-gs[e]));
                if constexpr (BAD) {  // g_L from shared memory: keeps gls and badc dead here
                    const float gl_c = sgl[4 * f + e];
                    const bool bad_c = -gl_c > SAFE_SPAN;
                    kin[e] = bad_c ? 0.f : kin_;
                    kt[e] = bad_c ? kk * __expf(gl_c - gs[e]) : kin_ * gams[e];
                } else {
                    kin[e] = kin_;
                    kt[e] = kin_ * gams[e];  // exp(g_L - g) = exp(g_L) exp(-g)
                }
            }
            *reinterpret_cast<uint2 *>(blk + sw128_chunk_off(r, fchunk, 128) + fhalf) =
                make_uint2(pack_bf16x2(qe[0], qe[1]), pack_bf16x2(qe[2], qe[3]));
            *reinterpret_cast<uint2 *>(blk + sw128_chunk_off(64 + r, fchunk, 128) + fhalf) =
                make_uint2(pack_bf16x2(ke[0], ke[1]), pack_bf16x2(ke[2], ke[3]));
            *reinterpret_cast<uint2 *>(blob + BLOB_KTT + fblk * 8192 + sw128_chunk_off(r, fchunk, 64) + fhalf) =
                make_uint2(pack_bf16x2(kt[0], kt[1]), pack_bf16x2(kt[2], kt[3]));
            *reinterpret_cast<uint2 *>(sm + P_KINV + fblk * 8192 + sw128_chunk_off(r, fchunk, 64) + fhalf) =
                make_uint2(pack_bf16x2(kin[0], kin[1]), pack_bf16x2(kin[2], kin[3]));
        }
    };
    if (GATE != KDA_GATE_NONE && n_bad) gate_rows(std::true_type{});
    else gate_rows(std::false_type{});
    fence_async_smem();
    // K~ went to the blob by ordinary stores; a worker of the fused grid publishes the
    // blob to chains that read it with bulk copies, so order them for the async proxy
    if constexpr (!Worker::kSingle) fence_proxy_async_global();
    tc_fence_before();
    w.sync();

    // Each blob image is stored as soon as it is final (bulk copies drain while the CTA
    // keeps computing): exp(g_L) and the Q~ rows of A1 are final now.
    if (tid == 0) {
        bulk_s2g(blob + BLOB_GAM, sm + P_GAM, 512);
        bulk_s2g(blob + BLOB_A1, sm + P_A1, 8192);                   // Q~, channels 0..63
        bulk_s2g(blob + BLOB_A1 + 16384, sm + P_A1 + 16384, 8192);   // Q~, channels 64..127
        bulk_commit();
    }

    // ---- Gram MMA: D[m][i] = sum_c A1[m][c] KINV[i][c]; rows 0..63 Q-rows, 64..127 K-rows
    if (tid == 0) {
        tc_fence_after();
        mma_run<D>(tmem, kmajor(sm_base + P_A1, 128), kmajor(sm_base + P_KINV, 64), idesc_bf16(128, 64), false);
        mma_commit(bar_mma);
        bulk_wait_read();  // the Q~ rows have left shared memory: their space takes A_kk after the MMA
    }
    w.wait(bar_mma, 0);
    tc_fence_after();

    // Readout mapping: warp w reads TMEM lanes 32*(w%4) .. +31 (Gram rows m),
    // columns 32*(w/4) .. +31.
    const int m = 32 * (warp & 3) + lane, cb = 32 * (warp >> 2);
    const int r_own = m & 63;
    const bool kk_row = m >= 64;
    // Output of Gram row r_own, columns i = cb + 8 cq .. +7 (8 values): A_qk (inclusive
    // lower) to its bf16 image, or A_kk (strict lower, times beta_r) to fp32 for the solve.
    auto store_gram8 = [&](int cq, const float *g8) {
        const int r = r_own;
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int i = cb + cq * 8 + e;
            v[e] = kk_row ? (i < r ? sbeta[r] * g8[e] : 0.f) : ((i <= r && r < L) ? g8[e] : 0.f);
        }
        if (!kk_row) {
            st_chunk(sm + P_AQK + sw128_chunk_off(r, (cb >> 3) + cq, 64), v);
        } else {
            float *akk = reinterpret_cast<float *>(sm + P_AKK) + r * LDT + cb + cq * 8;
            *reinterpret_cast<float4 *>(akk) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4 *>(akk + 4) = make_float4(v[4], v[5], v[6], v[7]);
        }
    };
    auto gram_readout = [&](auto bad_tag) {
        constexpr bool BAD = decltype(bad_tag)::value;
        if constexpr (BAD) {
            // Exact pairwise terms of the key channels whose chunk log-decay exceeds
            // SAFE_SPAN (left out of the MMA), added 8 columns at a time so that few
            // registers are live: this path only runs for such chunks.
            int *nbad = reinterpret_cast<int *>(sm + P_NBAD);
            if (tid == 0) {
                int cnt = 0;
                for (int cc = 0; cc < D; ++cc)
                    if (-sgl[cc] > SAFE_SPAN) badl[cnt++] = cc;
                *nbad = cnt;
            }
            w.sync();
            const int nb_total = *nbad;
            float *bb = reinterpret_cast<float *>(sm + P_BADB);  // [8][3][64]: q, k, g per row
            for (int cq = 0; cq < 4; ++cq) {
                float g8[8];
                tmem_ld8(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + cb + 8 * cq, g8);
                for (int b0 = 0; b0 < nb_total; b0 += 8) {
                    for (int e = tid; e < 8 * 64; e += PREP_NT) {  // gather the batch's columns
                        const int bi = e >> 6, r = e & 63;
                        float qx = 0.f, kx = 0.f, gx = 0.f;
                        if (b0 + bi < nb_total) {
                            const int cc = badl[b0 + bi];
                            const int64_t ccol = (int64_t)h * D + cc;
                            float gsum = 0.f;
                            for (int j = 0; j <= r; ++j)
                                gsum += j < L ? gate_log<GATE>(a.log_alpha, (tok0 + j) * H + h, cc) : 0.f;
                            gx = gsum;
                            if (r < L) {
                                qx = __bfloat162float(a.q[(tok0 + r) * H * D + ccol]);
                                kx = __bfloat162float(a.k[(tok0 + r) * H * D + ccol]);
                                if constexpr (L2) {  // the row norms gate_rows found
                                    qx *= sqn[r];
                                    kx *= skn[r];
                                }
                            }
                        }
                        bb[(bi * 3 + 0) * 64 + r] = qx;
                        bb[(bi * 3 + 1) * 64 + r] = kx;
                        bb[(bi * 3 + 2) * 64 + r] = gx;
                    }
                    w.sync();
                    const int nb = min(8, nb_total - b0);
                    for (int bi = 0; bi < nb; ++bi) {
                        const float xr = bb[(bi * 3 + (kk_row ? 1 : 0)) * 64 + r_own];
                        const float grr = bb[(bi * 3 + 2) * 64 + r_own];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int i = cb + 8 * cq + e;
                            const float fi = i <= r_own ? bb[(bi * 3 + 1) * 64 + i] *
                                                              expf(fminf(grr - bb[(bi * 3 + 2) * 64 + i], 0.f))
                                                        : 0.f;
                            g8[e] += xr * fi;
                        }
                    }
                    w.sync();
                }
                store_gram8(cq, g8);
            }
        } else {
            float G[32];
            tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + cb, G);
            const int r = r_own;
            if (!kk_row) {  // A_qk (inclusive lower) -> bf16 image, rows r, columns i
#pragma unroll
                for (int cq = 0; cq < 4; ++cq) {
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = cb + cq * 8 + e;
                        v[e] = (i <= r && r < L) ? G[cq * 8 + e] : 0.f;
                    }
                    st_chunk(sm + P_AQK + sw128_chunk_off(r, (cb >> 3) + cq, 64), v);
                }
            } else {  // A_kk (strict lower, times beta_r) -> fp32 for the solve
                float *akk = reinterpret_cast<float *>(sm + P_AKK);
                const float b = sbeta[r];
#pragma unroll
                for (int e4 = 0; e4 < 32; e4 += 4) {
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = cb + e4 + e;
                        v[e] = i < r ? b * G[e4 + e] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(akk + r * LDT + cb + e4) = make_float4(v[0], v[1], v[2], v[3]);
                }
            }
        }
    };
    if (GATE != KDA_GATE_NONE && n_bad) gram_readout(std::true_type{});
    else gram_readout(std::false_type{});
    fence_async_smem();
    tc_fence_before();
    w.sync();
    if (tid == 0) {  // A_qk is final
        bulk_s2g(blob + BLOB_AQK, sm + P_AQK, 8192);
        bulk_commit();
    }

    // ---- T = (I + A_kk)^-1 in place, by blocks: invert the four 16 x 16 diagonal
    //      blocks, then merge 16 -> 32 -> 64 with [[X, 0], [Y, Z]]^-1 =
    //      [[X^-1, 0], [-Z^-1 Y X^-1, Z^-1]] (each level two small products).
    {
        float *at = reinterpret_cast<float *>(sm + P_AKK);   // A_kk, becoming T (row stride LDT)
        float *pb = reinterpret_cast<float *>(sm + P_PBUF);  // 2 x [16][20] level-1 products
        float *qb = reinterpret_cast<float *>(sm + P_PBUF);  // [32][36] level-2 product
        if (warp < 4) {  // warp b inverts diagonal block b; lane l -> column l
            const int o = warp * 16, l = lane & 15;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float arow[16];
#pragma unroll
                for (int m4 = 0; m4 < 16; m4 += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(at + (o + r) * LDT + o + m4);
                    arow[m4] = a4.x; arow[m4 + 1] = a4.y; arow[m4 + 2] = a4.z; arow[m4 + 3] = a4.w;
                }
                float x0 = (r == l) ? 1.f : 0.f, x1 = 0.f;
#pragma unroll
                for (int mm = 0; mm < r; mm += 2) {
                    x0 -= arow[mm] * t[mm];
                    if (mm + 1 < r) x1 -= arow[mm + 1] * t[mm + 1];
                }
                t[r] = x0 + x1;
            }
            __syncwarp();
            if (lane < 16) {
#pragma unroll
                for (int r = 0; r < 16; ++r) at[(o + r) * LDT + o + l] = t[r];
            }
        }
        w.sync();
        // Merges, as 16 x 8 warp-level tf32 MMA tiles.
        // level 1: blocks (16..31, 0..15) and (48..63, 32..47); warps 0-3 take one 16 x 8
        // tile each (block w/2, columns 8*(w%2) ..).
        if (warp < 4) {  // P = A[o+16.., o..o+15] X^-1
            const int o = 32 * (warp >> 1), n0 = 8 * (warp & 1);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            warp_gemm_16x8<16>(d, at + (o + 16) * LDT + o, LDT, at + o * LDT + o + n0, LDT);
            warp_store_16x8(d, pb + (warp >> 1) * 16 * 20 + n0, 20, 1.f);
        }
        w.sync();
        if (warp < 4) {  // T = -Z^-1 P
            const int o = 32 * (warp >> 1), n0 = 8 * (warp & 1);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            warp_gemm_16x8<16>(d, at + (o + 16) * LDT + o + 16, LDT, pb + (warp >> 1) * 16 * 20 + n0, 20);
            warp_store_16x8(d, at + (o + 16) * LDT + o + n0, LDT, -1.f);
        }
        w.sync();
        // level 2: block (32..63, 0..31); warp w takes the 16 x 8 tile (rows 16*(w/4), cols 8*(w%4)).
        {  // Q = A[32.., 0..31] T[0..31, 0..31]
            const int m0 = 16 * (warp >> 2), n0 = 8 * (warp & 3);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            warp_gemm_16x8<32>(d, at + (32 + m0) * LDT, LDT, at + n0, LDT);
            warp_store_16x8(d, qb + m0 * 36 + n0, 36, 1.f);
        }
        w.sync();
        {  // T[32.., 0..31] = -T[32.., 32..] Q
            const int m0 = 16 * (warp >> 2), n0 = 8 * (warp & 3);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            warp_gemm_16x8<32>(d, at + (32 + m0) * LDT + 32, LDT, qb + n0, 36);
            warp_store_16x8(d, at + (32 + m0) * LDT + n0, LDT, -1.f);
        }
        if (tid == 0) bulk_wait_read();  // A_qk has left shared memory: its space takes T Diag(beta)
        w.sync();
        // image of T Diag(beta): rows r, columns i, zero above the diagonal
        {
            const int r = tid >> 2, qd = tid & 3;
#pragma unroll
            for (int cq = 0; cq < 2; ++cq) {
                const int i0 = qd * 16 + cq * 8;
                const float4 t0 = *reinterpret_cast<const float4 *>(at + r * LDT + i0);
                const float4 t1 = *reinterpret_cast<const float4 *>(at + r * LDT + i0 + 4);
                const float4 b0 = *reinterpret_cast<const float4 *>(sbeta + i0);
                const float4 b1 = *reinterpret_cast<const float4 *>(sbeta + i0 + 4);
                const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = (i0 + e) <= r ? tv[e] * bv[e] : 0.f;
                st_chunk(sm + P_TB + sw128_chunk_off(r, qd * 2 + cq, 64), v);
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    w.sync();

    // ---- W = (T Diag(beta)) (K e^g), M = 64, N = 128. K e^g sits in rows 64..127 of A1,
    //      read here as an MN-major B (K = token i). (U = T Diag(beta) V is formed by the
    //      chain kernel from the blob's T Diag(beta) and its own slice of V.)
    if (tid == 0) {
        bulk_s2g(blob + BLOB_TB, sm + P_TB, 8192);  // T Diag(beta) is final
        bulk_commit();
        tc_fence_after();
        mma_run<CH>(tmem, kmajor(sm_base + P_TB, 64), mnmajor(sm_base + P_A1 + 8192, 16384), idesc_bf16(64, 128, 0, 1), false);
        mma_commit(bar_mma);
    }
    w.wait(bar_mma, 1);
    tc_fence_after();
    {
        // M = 64 accumulator: row r sits in lane 16*(w%4) + (lane < 16) of quarter w%4.
        // Warp half w/4 takes columns 64*(w/4) .. +63, in two loads of 32.
        const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
        const int r = 16 * (warp & 3) + lane;
        unsigned char *wb = sm + P_A1 + (warp >> 2) * 16384;
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
            float a[32];
            tmem_ld32(tmem + lanes + 64u * (uint32_t)(warp >> 2) + 32u * hq, a);
            if (lane < 16) {  // W row r -> A1 row 64 + r, channel block w/4
#pragma unroll
                for (int cq = 0; cq < 4; ++cq) {
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = a[cq * 8 + e];
                    st_chunk(wb + sw128_chunk_off(64 + r, 4 * hq + cq, 128), v);
                }
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    w.sync();

    if (tid == 0) {  // the W rows of A1
        bulk_s2g(blob + BLOB_A1 + 8192, sm + P_A1 + 8192, 8192);
        bulk_s2g(blob + BLOB_A1 + 16384 + 8192, sm + P_A1 + 16384 + 8192, 8192);
        bulk_commit();
        bulk_wait_read();  // shared memory may be reused; the writes complete with the grid
        if (ready) w.pending = slot * H + h;  // a chain in the same grid waits for it

    }
    w.sync();  // the worker's shared memory and TMEM are free for its next item
}


template <int GATE, bool L2>
__global__ void __launch_bounds__(PREP_NT, 4)
kda_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_la, int pf_dist,
                const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                const void *__restrict__ log_alpha, const float *__restrict__ beta,
                unsigned char *__restrict__ ws_blobs, const int32_t *__restrict__ chunk_off,
                const int32_t *__restrict__ cu, int64_t T, int H, int n_seqs, int nck, int io_flags,
                float l2_eps) {
    extern __shared__ unsigned char smem_raw[];
    // The chain kernel after this one may start its CTAs (they wait for this grid to
    // complete before reading a blob): they then take SMs as this grid's last CTAs leave.
    griddep_launch_dependents();
    if (chunk_off && !packed_offsets_ok(chunk_off, n_seqs)) return;
    const int slot = blockIdx.x, h = blockIdx.y;
    int seq, n;
    if (!resolve_slot(slot, chunk_off, n_seqs, nck, seq, n)) return;
    // Warm L2 for the CTA that starts pf_dist launches after this one (about one full
    // residency later): its q, k and log_alpha tiles, so that its own loads find them
    // in L2 instead of waiting on DRAM.
    auto pf = [&](int &x, int &y) {
        const int64_t lin = blockIdx.x + (int64_t)blockIdx.y * gridDim.x + pf_dist;
        int pseq, pn;
        if (pf_dist <= 0 || lin >= (int64_t)gridDim.x * gridDim.y ||
            !resolve_slot((int)(lin % gridDim.x), chunk_off, n_seqs, nck, pseq, pn))
            return false;
        x = (int)(lin / gridDim.x) * D;
        y = (int)(seq_span(cu, T, pseq).start + (int64_t)pn * CH);
        return true;
    };
    const int64_t n_tok = chunk_off ? T : (int64_t)(gridDim.x / nck) * T;  // packed: T tokens in all
    const PrepArgs a{&tm_q, &tm_k, &tm_la, q, k, log_alpha, beta, ws_blobs, T, H, io_flags, l2_eps, n_tok * H};
    PrepWorker<true> w;
    w.init(true);
    prep_item<GATE, L2>(w, a, slot, h, seq_span(cu, T, seq), n, pf, nullptr);
    w.release(nullptr);
}

// =====================================================================================
// chain: per (sequence, head, value slice) state recurrence over the chunks
// =====================================================================================
// 288 threads, warp-specialised. Warps 0-7 are the epilogue warps: warp w reads TMEM
// lane quarter q = w % 4 and handles value columns (N/2)*(w/4) .. +N/2-1 of the slice,
// and thread (q, lane, w/4) keeps state row c = 32q + lane, those columns, in
// registers. Warp 8 issues every MMA and bulk load; a tcgen05.mma issue can stall
// while the tensor pipe is busy, and on its own warp that stall delays no epilogue.
// N = 64 gives two CTAs per (sequence, head), N = 128 one.
constexpr int CHAIN_EPI_WARPS = 8;
constexpr int CHAIN_NT = 32 * (CHAIN_EPI_WARPS + 1);
// Named barriers (id 0 is __syncthreads):
//   BAR_VNEW: the V_new warps (lane quarters 2, 3) arrive once their rows of the V_new
//             image are written; the issuer waits before the MMAs that read it.
//   BAR_END:  every thread, at the end of each chunk: the state image is written and
//             the chunk's TMEM reads are done. It also ORs the threads' `dead` flags,
//             so all warps leave the loop at the same chunk and the barriers' arrivals
//             always pair up, even after a bounded wait has given up.
//   BAR_CHAIN: all 288 threads, around the prologue and the epilogue.
constexpr uint32_t BAR_VNEW = 1, BAR_VNEW_COUNT = 32 * 5;
constexpr uint32_t BAR_END = 2;
constexpr uint32_t BAR_CHAIN = 3;

// Arguments of the chain work that are fixed for a launch.
struct ChainArgs {
    const CUtensorMap *tm_v;
    const unsigned char *ws_blobs;
    const int32_t *chunk_off;
    const float *S0;
    __nv_bfloat16 *o;
    float *S_T;
    const int32_t *cu;
    int64_t T;
    int H;
    int nck;
    const int32_t *ready;  // non-null: wait for each blob's ready flag before reading it
    // Launched as a dependent of the prep kernel (which may still run): everything up
    // to the first blob load only touches the call's inputs, then griddep_wait.
    bool wait_prior = false;
};

// The part of one (sequence, head, slice) recurrence a chain task runs: chunks [c0, c1)
// of the sequence (c1 < 0: to its end), starting from s0 (the (sequence, head) 128 x 128
// state block; null: zeros; s0_identity: the identity) and writing the end state to st
// (a block, or null) and, if write_o, the outputs. u_zero drops U (V_new = -W S): the
// recurrence then applies the chunks' transition matrix Prod (Diag(gamma_L) - K~^T W)
// to s0, which with s0 = I yields that matrix itself.
struct ChainWindow {
    int c0, c1;
    const float *s0;
    bool s0_identity;
    float *st;
    bool write_o;
    bool u_zero;
};
__device__ __forceinline__ ChainWindow full_window(const ChainArgs &a, int seq, int h) {
    const int64_t off = ((int64_t)seq * a.H + h) * (int64_t)(D * D);
    return {0, -1, a.S0 ? a.S0 + off : nullptr, false, a.S_T ? a.S_T + off : nullptr, true, false};
}

// The state recurrence of one (sequence, head, N-column value slice), run by threads
// 0 .. CHAIN_NT-1 of the CTA (tid) on shared memory `sm` (1024-aligned,
// ChainLayout<N>::BYTES - 1024 bytes). ROLE 0: the calling thread's warp decides its
// part. ROLE 1 / 2: compiled for the epilogue warps / the MMA warp only, so that each
// can run under its own register budget. With a.ready set (blobs produced by prep
// workers of the same grid), a watcher warp (ROLE 3, threads CHAIN_NT .. +31) reads
// the blobs' ready flags in chunk order and raises a shared counter, so the threads
// that issue the loads only poll shared memory.
template <int N, int ROLE = 0>
__device__ __forceinline__ void chain_task(unsigned char *sm, const int tid, const ChainArgs &a,
                                           const int seq, const int h, const int j0,
                                           const ChainWindow &win) {
    static_assert(N == 64 || N == 128, "value slices of 64 or 128 columns");
    constexpr int NH = N / 2;  // columns per epilogue thread
    using Lay = ChainLayout<N>;
    const int warp = tid >> 5, lane = tid & 31;
    const bool issuer = ROLE == 0 ? warp == CHAIN_EPI_WARPS : ROLE == 2;
    const bool epi = ROLE == 0 ? warp < CHAIN_EPI_WARPS : ROLE == 1;
    const uint32_t bar_chain_count = a.ready ? CHAIN_NT + 32 : CHAIN_NT;  // + the watcher
    const int q4 = warp & 3, hf = (warp >> 2) & 1;
    const CUtensorMap &tm_v = *a.tm_v;
    const unsigned char *ws_blobs = a.ws_blobs;
    const int32_t *chunk_off = a.chunk_off;
    __nv_bfloat16 *o = a.o;
    const int64_t T = a.T;
    const int H = a.H, nck = a.nck;
    const SeqSpan span = seq_span(a.cu, T, seq);
    const int c0 = win.c0;  // chunk indices below are relative to the window's first chunk
    const int seq_chunks = (int)((span.len + CH - 1) / CH);
    const int c_end = win.c1 < 0 || win.c1 > seq_chunks ? seq_chunks : win.c1;
    const int nchunks = c_end > c0 ? c_end - c0 : 0;
    const int64_t slot0 = (chunk_off ? (int64_t)chunk_off[seq] : (int64_t)seq * nck) + c0;

    uint64_t *bar_ld1 = reinterpret_cast<uint64_t *>(sm + Lay::BAR);  // [2] load part 1, per stage
    uint64_t *bar_ld2 = bar_ld1 + 2;  // [2] load part 2, per stage
    uint64_t *bar_a = bar_ld1 + 4;    // first MMAs done
    uint64_t *bar_b = bar_ld1 + 5;    // state MMA done
    uint64_t *bar_c = bar_ld1 + 6;    // [2] output MMA done, per D1 buffer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lay::TMEM);
    int32_t *ready_upto = reinterpret_cast<int32_t *>(sm + Lay::READY);
    bool dead = false;

    auto blob_of = [&](int chunk) {
        if (a.ready) counter_wait_gt(ready_upto, chunk, dead, &g_kda_status);
        return ws_blobs + ((size_t)(slot0 + chunk) * H + h) * BLOB_BYTES;
    };
    auto issue_load1 = [&](int chunk, int stage) {
        const unsigned char *blob = blob_of(chunk);
        unsigned char *st = sm + stage * Lay::STAGE;
        mbar_arrive_expect_tx(&bar_ld1[stage], Lay::LOAD1_BYTES);
        bulk_g2s(st + Lay::A1, blob + BLOB_A1, 32768, &bar_ld1[stage]);
        bulk_g2s(st + Lay::TB, blob + BLOB_TB, 8192, &bar_ld1[stage]);
#pragma unroll
        for (int b = 0; b < N / 64; ++b)
            tma_load_2d(st + Lay::V + b * 8192, &tm_v, h * D + j0 + 64 * b,
                        (int)(span.start + (int64_t)(c0 + chunk) * CH), &bar_ld1[stage]);
    };
    auto issue_load2 = [&](int chunk, int stage) {
        const unsigned char *blob = blob_of(chunk);
        unsigned char *st = sm + stage * Lay::STAGE;
        mbar_arrive_expect_tx(&bar_ld2[stage], Lay::LOAD2_BYTES);
        bulk_g2s(st + Lay::A2, blob + BLOB_AQK, 8192, &bar_ld2[stage]);
        bulk_g2s(st + Lay::KTT, blob + BLOB_KTT, 16384, &bar_ld2[stage]);
        bulk_g2s(st + Lay::GAM, blob + BLOB_GAM, 512, &bar_ld2[stage]);
    };

    if (tid == 0) {
        for (int b = 0; b < 8; ++b) mbar_init(&bar_ld1[b], 1);
        *ready_upto = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, Lay::TMEM_COLS);
        tmem_relinquish();
    }
    const int c = 32 * q4 + lane;    // state row owned by an epilogue thread
    const int jh = NH * hf;          // first of its NH value columns (inside the slice)
    float s_reg[NH];
    if (epi) {
#pragma unroll
        for (int j = 0; j < NH; j += 4) {
            float4 v4 = win.s0 ? *reinterpret_cast<const float4 *>(win.s0 + (int64_t)c * D + j0 + jh + j)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
            if (win.s0_identity) {
                const int col = j0 + jh + j;
                v4 = make_float4(c == col, c == col + 1, c == col + 2, c == col + 3);
            }
            s_reg[j] = v4.x; s_reg[j + 1] = v4.y; s_reg[j + 2] = v4.z; s_reg[j + 3] = v4.w;
        }
#pragma unroll
        for (int jc = 0; jc < NH / 8; ++jc) {  // row c of the MN-major S image, this thread's chunks
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = s_reg[jc * 8 + e];
            st_chunk(sm + Lay::SIMG + sw128_chunk_off(c, (jh >> 3) + jc, 128), v);
        }
    }
    fence_async_smem();
    tc_fence_before();
    named_bar_sync(BAR_CHAIN, bar_chain_count);
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    if (a.wait_prior) {  // the blobs exist once the prep grid has completed
        griddep_wait();
        fence_proxy_async_global();
    }
    const uint32_t d3 = tmem + 2 * N;  // D1 buffers at columns 0 and N
    const uint32_t du = tmem + 3 * N;  // U = T Diag(beta) V (rows 64..127)
    const uint32_t sm_base = smem_u32(sm);
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;

    if (ROLE == 3) {
        // ------------------------------------------------------------ flag watcher
        if (lane == 0) {
            for (int m = 0; m < nchunks; ++m) {
                if (!flag_wait(a.ready + (size_t)(slot0 + m) * H + h, dead, &g_kda_status)) break;
                st_release_cta(ready_upto, m + 1);
            }
        }
        __syncwarp();
    } else if (issuer) {
        // ------------------------------------------------------------ MMA / load warp
        // DU = [.; T Diag(beta)] V does not depend on the state. With 128 columns, chunk m's
        // is issued at the end of chunk m - 1 (after its V_new has been read from DU), so
        // that the tensor pipe runs it while the epilogue updates the state, and chunk m
        // starts with D1 alone; the next bar_a commit covers it. With 64 columns the
        // product is short and issuing it early measured slower (A/B on one box: 0.2325
        // against 0.2365 ms on B=4, T=4096, H=16; 0.4085 against 0.3932 ms at 128 columns
        // on B=8), so there it follows D1 as before.
        constexpr bool EARLY_DU = N == 128;
        auto issue_du = [&](int m) {
            const int sm_stage = m & 1;
            mbar_wait(&bar_ld1[sm_stage], (uint32_t)(m >> 1) & 1u, dead, &g_kda_status);
            if (!dead) {
                const uint32_t sb = sm_base + sm_stage * Lay::STAGE;
                tc_fence_after();
                mma_run<CH>(du, kmajor(sb + Lay::TB - 8192, 128), mnmajor(sb + Lay::V, 8192),
                            idesc_bf16(128, N, 0, 1), false);
            }
        };
        if (lane == 0) {
            for (int m = 0; m < 2 && m < nchunks; ++m) {
                issue_load1(m, m);
                issue_load2(m, m);
            }
            if (EARLY_DU && nchunks > 0) issue_du(0);
        }
#pragma unroll 1
        for (int n = 0; n < nchunks; ++n) {
            const int stage = n & 1;
            const uint32_t st_base = sm_base + stage * Lay::STAGE;
            const uint32_t d1 = tmem + (uint32_t)((n & 1) * N);
            const uint32_t lph = (uint32_t)(n >> 1) & 1u;
            if (lane == 0) {
                mbar_wait(&bar_ld1[stage], lph, dead, &g_kda_status);
                if (!dead) {  // D1 = [Q~; W] S, then (unless issued early) DU
                    tc_fence_after();
                    mma_run<D>(d1, kmajor(st_base + Lay::A1, 128), mnmajor(sm_base + Lay::SIMG, 16384),
                               idesc_bf16(128, N, 0, 1), false);
                    if constexpr (!EARLY_DU)
                        mma_run<CH>(du, kmajor(st_base + Lay::TB - 8192, 128), mnmajor(st_base + Lay::V, 8192),
                                    idesc_bf16(128, N, 0, 1), false);
                    mma_commit(bar_a);
                }
            }
            __syncwarp();
            named_bar_sync(BAR_VNEW, BAR_VNEW_COUNT);  // V_new image of chunk n written
            if (lane == 0) mbar_wait(&bar_ld2[stage], lph, dead, &g_kda_status);
            if (lane == 0 && !dead) {
                // D3 = K~^T V_new (the state path first), then D1 += [A_qk; 0] V_new
                tc_fence_after();
                mma_run<CH>(d3, mnmajor(st_base + Lay::KTT, 8192), mnmajor(sm_base + Lay::VIMG, 8192),
                            idesc_bf16(128, N, 1, 1), false);
                mma_commit(bar_b);
                mma_run<CH>(d1, kmajor(st_base + Lay::A2, 128), mnmajor(sm_base + Lay::VIMG, 8192),
                            idesc_bf16(128, N, 0, 1), true);
                mma_commit(&bar_c[n & 1]);
                if (EARLY_DU && n + 1 < nchunks) issue_du(n + 1);  // DU(n) has been read: V_new is written
            }
            __syncwarp();
            if (named_bar_or(BAR_END, CHAIN_NT, dead)) {
                dead = true;
                break;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue warps
        // Output of chunk m: rows 0..63 of D1 buffer m % 2, all N columns, read by warps
        // 4 and 5 (lane quarters 0 and 1) once the output MMA of chunk m has completed,
        // while the next chunk's first MMAs run.
        auto store_output = [&](int m) {
            mbar_wait(&bar_c[m & 1], (uint32_t)(m >> 1) & 1u, dead, &g_kda_status);
            tc_fence_after();
            const int r = c;
            const int64_t m0 = (int64_t)(c0 + m) * CH;  // first token of the chunk
            const bool live = r < chunk_rows(span.len, m0);
            __nv_bfloat16 *dst = o + ((span.start + m0 + r) * H + h) * (int64_t)D + j0;
#pragma unroll
            for (int b = 0; b < N / 32; ++b) {
                float ov[32];
                tmem_ld32(tmem + (uint32_t)((m & 1) * N + 32 * b) + lane_off, ov);
                if (live) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 pk = make_uint4(pack_bf16x2(ov[j], ov[j + 1]), pack_bf16x2(ov[j + 2], ov[j + 3]),
                                              pack_bf16x2(ov[j + 4], ov[j + 5]), pack_bf16x2(ov[j + 6], ov[j + 7]));
                        *reinterpret_cast<uint4 *>(dst + 32 * b + j) = pk;
                    }
                }
            }
        };
#pragma unroll 1
        for (int n = 0; n < nchunks; ++n) {
            const int stage = n & 1;
            const uint32_t ph = (uint32_t)n & 1u;
            const unsigned char *st = sm + stage * Lay::STAGE;
            const uint32_t d1 = tmem + (uint32_t)((n & 1) * N);
            const uint32_t lph = (uint32_t)(n >> 1) & 1u;
            if (q4 >= 2) {  // rows 64..127 hold (W S)[r] in D1 and U[r] in DU; V_new = U - W S
                mbar_wait(bar_a, ph, dead, &g_kda_status);
                tc_fence_after();
                const int r = c - 64;
#pragma unroll
                for (int p = 0; p < NH / 32; ++p) {
                    float ws[32], us[32];
                    tmem_ld32(d1 + lane_off + jh + 32 * p, ws);
                    tmem_ld32(du + lane_off + jh + 32 * p, us);
#pragma unroll
                    for (int jc = 0; jc < 4; ++jc) {
                        float v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v[e] = (win.u_zero ? 0.f : us[jc * 8 + e]) - ws[jc * 8 + e];
                        st_chunk(sm + Lay::VIMG + sw128_chunk_off(r, ((jh + 32 * p) >> 3) + jc, 64), v);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                named_bar_arrive(BAR_VNEW, BAR_VNEW_COUNT);
            } else if (hf == 1) {
                if (win.write_o && n > 0) store_output(n - 1);
            } else if (warp == 1) {
                // Part 1 of the stage is free once the first MMAs have completed: refill it
                // with chunk n + 2 while this chunk is still being processed.
                if (lane == 0 && n + 2 < nchunks) {
                    mbar_wait(bar_a, ph, dead, &g_kda_status);
                    if (!dead) issue_load1(n + 2, stage);
                }
                __syncwarp();
            }
            {  // S <- Diag(exp(g_L)) S + K~^T V_new
                mbar_wait(&bar_ld2[stage], lph, dead, &g_kda_status);  // GAM
                mbar_wait(bar_b, ph, dead, &g_kda_status);
                tc_fence_after();
                const float gam = reinterpret_cast<const float *>(st + Lay::GAM)[c];
#pragma unroll
                for (int p = 0; p < NH / 32; ++p) {
                    float dv[32];
                    tmem_ld32(d3 + lane_off + jh + 32 * p, dv);
#pragma unroll
                    for (int jc = 0; jc < 4; ++jc) {
                        float v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            float &s = s_reg[32 * p + jc * 8 + e];
                            s = gam * s + dv[jc * 8 + e];
                            v[e] = s;
                        }
                        st_chunk(sm + Lay::SIMG + sw128_chunk_off(c, ((jh + 32 * p) >> 3) + jc, 128), v);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            if (named_bar_or(BAR_END, CHAIN_NT, dead)) {
                dead = true;
                break;
            }
            // Part 2 is free once the output MMA (the last reader of A2 and KTT) has
            // completed and the state update (the reader of GAM) has passed BAR_END.
            if (tid == 32 && n + 2 < nchunks) {
                mbar_wait(&bar_c[stage], lph, dead, &g_kda_status);
                if (!dead) issue_load2(n + 2, stage);
            }
        }
        if (win.write_o && nchunks > 0 && !dead && q4 < 2 && hf == 1) store_output(nchunks - 1);
        if (win.st) {
#pragma unroll
            for (int j = 0; j < NH; j += 4)
                *reinterpret_cast<float4 *>(win.st + (int64_t)c * D + j0 + jh + j) =
                    make_float4(s_reg[j], s_reg[j + 1], s_reg[j + 2], s_reg[j + 3]);
        }
    }
    tc_fence_before();
    named_bar_sync(BAR_CHAIN, bar_chain_count);
    if (warp == 0) tmem_dealloc(tmem, Lay::TMEM_COLS);
}

template <int N>
__global__ void __launch_bounds__(CHAIN_NT, 1)
kda_chain_kernel(const __grid_constant__ CUtensorMap tm_v,
                 const unsigned char *__restrict__ ws_blobs, const int32_t *__restrict__ chunk_off,
                 const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o,
                 float *__restrict__ S_T, const int32_t *__restrict__ cu, int64_t T, int H,
                 int nck, int wait_prior) {
    extern __shared__ unsigned char smem_raw[];
    if (chunk_off && !packed_offsets_ok(chunk_off, (int)gridDim.x)) return;
    const ChainArgs a{&tm_v, ws_blobs, chunk_off, S0, o, S_T, cu, T, H, nck, nullptr, wait_prior != 0};
    chain_task<N>(aligned_smem(smem_raw), threadIdx.x, a, blockIdx.x, blockIdx.y, blockIdx.z * N,
                  full_window(a, blockIdx.x, blockIdx.y));
}

// =====================================================================================
// segment scan: long sequences with few sequence-heads (batched inputs)
// =====================================================================================
// The chunks of every sequence are cut into n_seg segments of seg_len chunks (the last
// one takes the rest). Within a segment the state obeys S_end = P_k S_start + H_k, with
// P_k the product of the chunks' transitions Diag(gamma_L) - K~^T W and H_k the end
// state reached from zero (mokono.cn "Kimi Linear：高效注意力机制在长序列处理中的创新应用"
// section 2.1: S_r = P_r S_0 + H_r, applied per segment instead of per chunk).
//  * pass 1, all in parallel: segment 0 runs its true chain (outputs; its end state is
//    the start of segment 1); each middle segment k = 1 .. n_seg-2 runs its chain from
//    zero (giving H_k) and, with U dropped, from the identity (giving P_k).
//  * combine: S_start[k+1] = P_k S_start[k] + H_k for k = 1 .. n_seg-2, in fp32.
//  * pass 2, in parallel: segments 1 .. n_seg-1 replay their chains from their true start
//    states (outputs; the last one writes S_T).
// The chain work is about three segments' worth per slice instead of n_seg, spread over
// up to 2 (2 n_seg - 3) CTAs per sequence-head.
struct SegScan {
    float *p, *hh, *start;  // per (sequence-head, segment) 128 x 128 fp32 blocks
    int n_seg, seg_len;
    __host__ __device__ float *blk(float *base, int pair, int k) const {
        return base + ((size_t)pair * n_seg + k) * (size_t)(D * D);
    }
};

template <int N>
__global__ void __launch_bounds__(CHAIN_NT, 1)
kda_seg_pass_kernel(const __grid_constant__ CUtensorMap tm_v,
                    const unsigned char *__restrict__ ws_blobs, const float *__restrict__ S0,
                    __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T, int64_t T, int H,
                    int nck, SegScan sg, int pass) {
    extern __shared__ unsigned char smem_raw[];
    constexpr int SLICES = D / N;
    const int pair = blockIdx.x / SLICES, j0 = (blockIdx.x % SLICES) * N;
    const int seq = pair / H, h = pair % H;
    const int64_t off = (int64_t)pair * (D * D);
    // pass 1 follows the prep kernel as its dependent; pass 2 follows the combine
    const ChainArgs a{&tm_v, ws_blobs, nullptr, S0, o, S_T, nullptr, T, H, nck, nullptr, pass == 1};
    const int L = sg.seg_len;
    ChainWindow win;
    if (pass == 1) {
        const int t = blockIdx.y;  // 0: segment 0; 2k - 1: H_k; 2k: P_k
        const int k = (t + 1) / 2;
        if (t == 0)
            win = {0, L, S0 ? S0 + off : nullptr, false, sg.blk(sg.start, pair, 1), true, false};
        else if (t & 1)
            win = {k * L, (k + 1) * L, nullptr, false, sg.blk(sg.hh, pair, k), false, false};
        else
            win = {k * L, (k + 1) * L, nullptr, true, sg.blk(sg.p, pair, k), false, true};
    } else {
        const int k = blockIdx.y + 1;
        const bool last = k == sg.n_seg - 1;
        win = {k * L, last ? -1 : (k + 1) * L, sg.blk(sg.start, pair, k), false,
               last ? (S_T ? S_T + off : nullptr) : nullptr, true, false};
    }
    chain_task<N>(aligned_smem(smem_raw), threadIdx.x, a, seq, h, j0, win);
}

// S_start[k+1][:, slice] = P_k S_start[k][:, slice] + H_k[:, slice] for k = 1 .. n_seg-2.
// One CTA per (sequence-head, 64-column slice). Thread t owns rows t/4 and t/4 + 64 and
// the 16 columns 4 (t % 4) + 16 m + {0..3}, m = 0..3: per column index the four threads
// of a row read four different banks of the state, and two row values of P_k serve 32
// products. Each step stages P_k in shared memory (rows padded to 129 floats, so that
// the rows a warp reads at one column fall in distinct banks).
constexpr int SEG_COMBINE_NT = 256;
constexpr int SEG_NJ = 16;       // state columns per CTA: (128 / SEG_NJ) CTAs per sequence-head
constexpr int SEG_PLD = D + 1;   // row stride of P_k in shared memory (floats)
constexpr uint32_t SEG_COMBINE_SMEM = (D * SEG_NJ + D * SEG_PLD) * sizeof(float);
static_assert(D * SEG_NJ == 8 * SEG_COMBINE_NT, "one row and 8 columns per thread");
__global__ void __launch_bounds__(SEG_COMBINE_NT)
kda_seg_combine_kernel(SegScan sg) {
    extern __shared__ __align__(16) float seg_smem[];
    float (*s)[SEG_NJ] = reinterpret_cast<float (*)[SEG_NJ]>(seg_smem);  // [128][SEG_NJ] state slice
    float *pm = seg_smem + D * SEG_NJ;                                    // [128][SEG_PLD] P_k
    constexpr int SLICES = D / SEG_NJ;
    const int pair = blockIdx.x / SLICES, j0 = (blockIdx.x % SLICES) * SEG_NJ;
    // thread: state row r, columns jq .. jq + 7 of the slice
    const int tid = threadIdx.x, r = tid >> 1, jq = (tid & 1) * 8;
    const float *s1 = sg.blk(sg.start, pair, 1);
    {
        const float4 *src = reinterpret_cast<const float4 *>(s1 + r * D + j0 + jq);
        *reinterpret_cast<float4 *>(&s[r][jq]) = src[0];
        *reinterpret_cast<float4 *>(&s[r][jq + 4]) = src[1];
    }
    for (int k = 1; k + 1 < sg.n_seg; ++k) {
        const float *pk = sg.blk(sg.p, pair, k);
        {  // all of this thread's loads first, so that they are in flight together
            constexpr int PER = D * 32 / SEG_COMBINE_NT;  // float4 of P_k per thread
            float4 v[PER];
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = tid + i * SEG_COMBINE_NT;
                v[i] = *reinterpret_cast<const float4 *>(pk + (e >> 5) * D + (e & 31) * 4);
            }
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = tid + i * SEG_COMBINE_NT;
                float *dst = pm + (e >> 5) * SEG_PLD + (e & 31) * 4;
                dst[0] = v[i].x; dst[1] = v[i].y; dst[2] = v[i].z; dst[3] = v[i].w;
            }
        }
        float acc[8];
        {
            const float4 *hk = reinterpret_cast<const float4 *>(sg.blk(sg.hh, pair, k) + (size_t)r * D + j0 + jq);
            const float4 h0 = hk[0], h1 = hk[1];
            acc[0] = h0.x; acc[1] = h0.y; acc[2] = h0.z; acc[3] = h0.w;
            acc[4] = h1.x; acc[5] = h1.y; acc[6] = h1.z; acc[7] = h1.w;
        }
        __syncthreads();  // P_k and the state are in shared memory
        const float *prow = pm + r * SEG_PLD;
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
            const float a = prow[c];
            const float4 s0 = *reinterpret_cast<const float4 *>(&s[c][jq]);
            const float4 s4 = *reinterpret_cast<const float4 *>(&s[c][jq + 4]);
            acc[0] += a * s0.x; acc[1] += a * s0.y; acc[2] += a * s0.z; acc[3] += a * s0.w;
            acc[4] += a * s4.x; acc[5] += a * s4.y; acc[6] += a * s4.z; acc[7] += a * s4.w;
        }
        __syncthreads();  // every thread has read the old state and P_k
        const float4 o0 = make_float4(acc[0], acc[1], acc[2], acc[3]);
        const float4 o1 = make_float4(acc[4], acc[5], acc[6], acc[7]);
        *reinterpret_cast<float4 *>(&s[r][jq]) = o0;
        *reinterpret_cast<float4 *>(&s[r][jq + 4]) = o1;
        float4 *out = reinterpret_cast<float4 *>(sg.blk(sg.start, pair, k + 1) + (size_t)r * D + j0 + jq);
        out[0] = o0;
        out[1] = o1;
    }
}

// =====================================================================================
// fused: prep and chain in one cooperative grid (batched inputs)
// =====================================================================================
// One CTA of FUSED_NT threads per SM, all resident at once (cooperative launch). Each
// CTA starts as three prep workers that take (chunk, head) items from a queue in
// chunk order: items of the first n_first chunks are shared by all CTAs, the rest go
// only to CTAs that never run a chain. Once the shared items are all claimed, CTA
// b < n_chain finishes its items and becomes the chain of task b = (seq H + h) D/N +
// slice; a watcher warp of that CTA follows the blobs' ready flags. Prep workers never
// wait on a chain, so every flag a chain waits for is eventually set. n_first is chosen
// so that the CTAs left on prep finish the remaining items about when the chains need
// them.
constexpr int FUSED_NT = 3 * PREP_NT;
template <int N>
constexpr uint32_t fused_smem() {
    return (3 * PREP_PART > ChainLayout<N>::BYTES - 1024 ? 3 * PREP_PART : ChainLayout<N>::BYTES - 1024) + 1024;
}
static_assert(fused_smem<128>() <= 232448, "fused CTA exceeds the shared memory of an SM");
// Registers per thread in the chain role: epilogue warpgroups 0-1 get FUSED_REG_EPI,
// warpgroup 2 (the MMA warp, the watcher and two idle warps) 72, idle warpgroups 3-5
// drop to 24. Their sum must stay within the launch's 80 per thread.
template <int N>
__host__ __device__ constexpr int fused_reg_epi() { return N == 64 ? 144 : 168; }
constexpr int FUSED_REG_MMA = 72, FUSED_REG_IDLE = 24;
static_assert(256 * 168 + 128 * FUSED_REG_MMA + 384 * FUSED_REG_IDLE <= FUSED_NT * 80,
              "register split exceeds the launch's registers");

struct FusedQueue {
    int32_t next_shared;  // items of the first n_first chunks, claimed by every CTA
    int32_t next_rest;    // the other items, claimed by prep-only CTAs
};

template <int N, int GATE>
__global__ void __launch_bounds__(FUSED_NT, 1)
kda_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_v,
                 const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                 const void *__restrict__ log_alpha, const float *__restrict__ beta,
                 unsigned char *__restrict__ ws_blobs, int32_t *__restrict__ ready,
                 FusedQueue *__restrict__ queue, const float *__restrict__ S0,
                 __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T, int64_t T, int H, int B,
                 int nck, int n_first, int n_chain, int io_flags, float l2_eps) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = aligned_smem(smem_raw);
    const int tid = threadIdx.x;
    const int P = B * H;
    const int n_shared = n_first * P, n_total = nck * P;
    const bool chain_cta = (int)blockIdx.x < n_chain;
    {
        const PrepArgs pa{&tm_q, &tm_k, &tm_la, q, k, log_alpha, beta, ws_blobs, T, H, io_flags, l2_eps,
                          (int64_t)B * T * H};
        using Worker = PrepWorker<false>;
        Worker w;
        w.init(false);
        // Thread 0 claims each item one item ahead: the claim's atomics are issued while
        // the current item's loads are in flight. The two slots alternate, so a slot is
        // rewritten only after every thread has passed the item that read it.
        volatile int32_t *claim = reinterpret_cast<volatile int32_t *>(Worker::sm() + P_CLAIM);
        auto claim_next = [&]() {
            int it = atomicAdd(&queue->next_shared, 1);
            if (it >= n_shared) it = chain_cta ? -1 : n_shared + atomicAdd(&queue->next_rest, 1);
            return it < n_total ? it : -1;
        };
        struct ClaimAhead {
            decltype(claim_next) &next;
            volatile int32_t *slot;
            int value;
            __device__ __forceinline__ void before_wait() { value = next(); }
            __device__ __forceinline__ void after_wait() { *slot = value; }
        };
        if (Worker::tid() == 0) claim[0] = claim_next();
        for (int j = 0;; ++j) {
            Worker::sync();
            const int it = claim[j & 1];
            if (it < 0 || w.dead) break;
            const int n = it / P, p = it % P, seq = p / H, h = p % H;
            // warm L2 for the item about one round of all workers later
            auto pf = [&](int &x, int &y) {
                const int pit = it + 3 * (int)gridDim.x;
                if (pit >= n_total) return false;
                const int pp = pit % P;
                x = (pp % H) * D;
                y = (int)((int64_t)(pp / H) * T + (int64_t)(pit / P) * CH);
                return true;
            };
            prep_item<GATE, false>(w, pa, seq * nck + n, h, SeqSpan{(int64_t)seq * T, T}, n, pf, ready,
                      ClaimAhead{claim_next, claim + ((j + 1) & 1), -1});
        }
        w.release(ready);
    }
    __syncthreads();  // every worker is done: shared memory and TMEM pass to the chain
    if (!chain_cta) return;
    const int wg = tid >> 7;
    const ChainArgs ca{&tm_v, ws_blobs, nullptr, S0, o, S_T, nullptr, T, H, nck, ready};
    constexpr int SLICES = D / N;
    const int task = blockIdx.x, pair = task / SLICES, seq = pair / H, h = pair % H;
    const int j0 = (task % SLICES) * N;
    const ChainWindow win = full_window(ca, seq, h);
    if (wg < 2) {
        setmaxnreg_inc<fused_reg_epi<N>()>();
        chain_task<N, 1>(sm, tid, ca, seq, h, j0, win);
    } else if (wg == 2) {
        setmaxnreg_dec<FUSED_REG_MMA>();
        if (tid < CHAIN_NT) chain_task<N, 2>(sm, tid, ca, seq, h, j0, win);
        else if (tid < CHAIN_NT + 32) chain_task<N, 3>(sm, tid, ca, seq, h, j0, win);
    } else {
        setmaxnreg_dec<FUSED_REG_IDLE>();
    }
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

// [n_tok, H*128] row-major tensor; boxes of 64 rows x 64 bf16 or 128 fp32 columns. bf16
// boxes use the 128-byte swizzle, so a box lands in shared memory as one swizzled
// operand block; the fp32 log_alpha box is plain rows.
bool make_map(CUtensorMap *m, const void *ptr, bool bf16, int64_t n_tok, int H) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int esize = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)H * D, (cuuint64_t)n_tok};
    cuuint64_t strides[1] = {(cuuint64_t)H * D * esize};
    cuuint32_t box[2] = {bf16 ? 64u : (cuuint32_t)D, (cuuint32_t)CH};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
              const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              bf16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launches `kernel`; with `after_prep` as a programmatic dependent of the prep kernel just
// launched on the stream, so that its CTAs may start while that kernel's last CTAs run.
template <class... KArgs, class... Args>
cudaError_t launch_maybe_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t stream, bool after_prep, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_prep ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int N>
cudaError_t launch_chain(const CUtensorMap &mv, const unsigned char *blobs, const int32_t *chunk_off,
                         const float *S0, void *o, float *S_T, const int32_t *cu, int64_t T, int H,
                         int nck, int nseq, bool after_prep, cudaStream_t stream) {
    using Lay = ChainLayout<N>;
    cudaError_t err = cudaFuncSetAttribute(kda_chain_kernel<N>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::BYTES);
    if (err != cudaSuccess) return err;
    err = launch_maybe_dependent(kda_chain_kernel<N>, dim3((unsigned)nseq, (unsigned)H, D / N),
                                 dim3(CHAIN_NT), Lay::BYTES, stream, after_prep, mv, blobs, chunk_off,
                                 S0, (__nv_bfloat16 *)o, S_T, cu, T, H, nck, after_prep ? 1 : 0);
    return err != cudaSuccess ? err : cudaGetLastError();
}


// CTAs of the prep kernel resident on the whole GPU at once (its L2 prefetch
// distance); 0 if it cannot be determined.
// Prep CTAs resident at once on the device (the kernel's attributes must be set first).
template <class K>
int prep_residency(K kernel) {
    int dev = 0, n_sm = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, PREP_NT, PREP_SMEM) != cudaSuccess)
        return 0;
    return n_sm * per_sm;
}

}  // namespace

// Workspace of batched inputs: one ready flag per blob and the fused kernel's queue,
// then the blobs.
size_t batched_head_bytes(int B, int nck, int H) {
    return (((size_t)B * nck * H * 4 + sizeof(FusedQueue) + 255) / 256) * 256;
}

// Plan for batched inputs: prep then chains (two kernels), the fused grid, or the
// segment scan. Model (B200 measurements): the standalone prep kernel finishes a
// chunk-head about every PREP_US_TWO per CTA slot, the fused grid's workers about
// every PREP_US_FUSED, three per SM; a 64-column chain takes about CHAIN_US_64 per
// chunk (CHAIN_US_128 for 128 columns). Each alternative is costed and the cheapest
// taken; the fused grid only with a clear margin.
//  * fused grid: n_chain chain CTAs run while the other SMs produce the items of the
//    last chunks; n_first puts the end of that production at about the end of the chains.
//  * segment scan: n_seg segments of seg_len chunks; two passes of about seg_len chunks
//    each after the prep, plus the sequential combine.
struct BatchedPlan {
    int kind;     // 0: prep then chains; 1: fused grid; 2: segment scan
    int n_first;  // fused grid: chunks whose items every CTA shares
    int n_seg, seg_len;
};
// Whether the current device can run the fused grid (cooperative launch, one CTA per
// SM). The kernel's shared-memory attribute is set here, once per device, as the check
// needs it; the answer is cached per device.
template <int GATE>
bool fused_smem_attr() {
    return cudaFuncSetAttribute(kda_fused_kernel<64, GATE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<64>()) == cudaSuccess;
}
bool fused_supported() {
    constexpr int MAX_DEVICES = 128;
    static int ok[MAX_DEVICES];  // 0: not checked, 1: yes, 2: no
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return false;
    if (ok[dev] == 0) {
        int coop = 0, per64 = 0;
        const bool yes =
            cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && coop &&
            fused_smem_attr<KDA_GATE_CHANNEL>() && fused_smem_attr<KDA_GATE_CHANNEL_BF16>() &&
            fused_smem_attr<KDA_GATE_HEAD>() && fused_smem_attr<KDA_GATE_NONE>() &&
            fused_smem_attr<KDA_GATE_CHANNEL_LOGIT>() && fused_smem_attr<KDA_GATE_CHANNEL_LOGIT_BF16>() &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per64, kda_fused_kernel<64, KDA_GATE_CHANNEL>,
                                                          FUSED_NT, fused_smem<64>()) == cudaSuccess &&
            per64 >= 1;
        ok[dev] = yes ? 1 : 2;
    }
    return ok[dev] == 1;
}
// Segments the workspace has room for (it is sized without knowing the device: at most
// 16 segments of at least 8 chunks, and only where 3 segments fit 256 SMs).
int seg_capacity(int B, int H, int nck) {
    const int P = B * H;
    if (2 * P * 3 > 256) return 0;
    const int c = nck / 8;
    return c < 16 ? c : 16;
}
size_t seg_bytes(int B, int H, int nck) {
    const int cap = seg_capacity(B, H, nck);
    return cap >= 3 ? (size_t)3 * B * H * cap * (size_t)(D * D) * sizeof(float) : 0;
}
constexpr double CHAIN_US_64 = 1.45, CHAIN_US_128 = 2.3;  // per chunk, B200
// Whether P sequence-heads run faster as P 128-column chains than as 2 P 64-column ones:
// a 128-column chain takes about CHAIN_US_128 per chunk, a 64-column one CHAIN_US_64,
// one CTA per SM, in waves of n_sm CTAs.
bool wide_chain(int64_t P, int n_sm) {
    const int64_t w64 = (2 * P + n_sm - 1) / n_sm, w128 = (P + n_sm - 1) / n_sm;
    return (double)w128 * CHAIN_US_128 < (double)w64 * CHAIN_US_64;
}
BatchedPlan batched_plan(int B, int H, int nck, int n_sm) {
    constexpr double PREP_US_TWO = 14.4, PREP_US_FUSED = 16.5, COMBINE_US = 2.0, LAUNCH_US = 4.0;
    constexpr int MIN_PREP_CTAS = 8;
    const int P = B * H;
    const double r2 = 3.0 / PREP_US_TWO, rf = 3.0 / PREP_US_FUSED;  // items per us per SM
    const double t_prep = nck * (double)P / (n_sm * r2);
    // prep on every SM, then the chains in waves
    const int n2 = wide_chain(P, n_sm) ? 128 : 64;
    const double waves = (double)((P * (D / n2) + n_sm - 1) / n_sm);
    BatchedPlan best{0, 0, 0, 0};
    double t_best = t_prep + waves * nck * (n2 == 64 ? CHAIN_US_64 : CHAIN_US_128);
    // segment scan
    int n_seg = (n_sm / (2 * P) + 3) / 2;  // pass 1: 2 P (2 n_seg - 3) CTAs in one wave
    const int cap = seg_capacity(B, H, nck);
    n_seg = n_seg < cap ? n_seg : cap;
    if (n_seg >= 3) {
        const int seg_len = (nck + n_seg - 1) / n_seg;
        n_seg = (nck + seg_len - 1) / seg_len;
        const double t = t_prep + 2.0 * seg_len * CHAIN_US_64 + (n_seg - 2) * COMBINE_US + 2 * LAUNCH_US;
        if (n_seg >= 3 && t < t_best) {
            t_best = t;
            best = {2, 0, n_seg, seg_len};
        }
    }
    // fused grid (64-column chains; 128-column chains run about 2.3 us per chunk: no gain)
    const int n_chain = 2 * P;
    if (n_chain + MIN_PREP_CTAS <= n_sm && (int64_t)nck * P < (1ll << 30) && fused_supported()) {
        const int n_prep = n_sm - n_chain;
        int n_first = nck - (int)((double)nck * CHAIN_US_64 * n_prep * rf / P);
        const int lo = nck < 2 ? nck : 2;
        n_first = n_first < lo ? lo : (n_first > nck ? nck : n_first);
        const double t_a = (double)n_first * P / (n_sm * rf);
        const double t_b = (double)(nck - n_first) * P / (n_prep * rf);
        const double t = t_a + (nck * CHAIN_US_64 > t_b ? nck * CHAIN_US_64 : t_b);
        if (t < 0.95 * t_best) {
            t_best = t;
            best = {1, n_first, 0, 0};
        }
    }
    return best;
}

size_t prefill_tc_workspace(int B, int64_t T, int H, int n_seqs) {
    if (n_seqs > 0) {
        const size_t head = packed_head_bytes(n_seqs);
        const size_t slots = (size_t)(T / CH) + (size_t)n_seqs;
        return head + slots * (size_t)H * BLOB_BYTES;
    }
    const int nck = (int)((T + CH - 1) / CH);
    return batched_head_bytes(B, nck, H) + (size_t)B * nck * (size_t)H * BLOB_BYTES +
           seg_bytes(B, H, nck);
}

int sm_count() {
    int dev = 0, n_sm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    return n_sm;
}

// Kernels launch_prefill_tc launches for these arguments (its decisions, restated).
int prefill_tc_launches(int B, int64_t T, int H, int n_seqs, bool l2norm) {
    const bool packed = n_seqs > 0;
    const int64_t n_tok = packed ? T : (int64_t)B * T;
    const int nck = (int)((T + CH - 1) / CH);
    if (!packed && n_tok > 0) {
        const BatchedPlan plan = batched_plan(B, H, nck, sm_count());
        if (plan.kind == 1 && !l2norm) return 1;  // the fused grid
        if (plan.kind == 2) return 4;             // prep, pass 1, combine, pass 2
    }
    const int64_t slots = packed ? T / CH + n_seqs : (int64_t)B * nck;
    return (packed ? 1 : 0) + (n_tok > 0 && slots > 0 ? 1 : 0) + 1;
}

// Tensor map of a per-channel gate (fp32 boxes of 128 channels, bf16 boxes of 64), used
// only for L2 prefetch; the other layouts get a copy of `fallback`, which no kernel reads.
bool make_gate_map(CUtensorMap *m, const void *la, int gate, int64_t n_tok, int H,
                   const CUtensorMap &fallback) {
    if (gate == KDA_GATE_CHANNEL || gate == KDA_GATE_CHANNEL_LOGIT) return make_map(m, la, false, n_tok, H);
    if (gate == KDA_GATE_CHANNEL_BF16 || gate == KDA_GATE_CHANNEL_LOGIT_BF16) return make_map(m, la, true, n_tok, H);
    *m = fallback;
    return true;
}

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const void *log_alpha,
                              int gate, const float *beta, const float *S0, void *o, float *S_T, int B,
                              int64_t T, int H, const int32_t *cu_seqlens, int n_seqs,
                              void *workspace, const IoOpts &io, cudaStream_t stream) {
    const bool packed = n_seqs > 0;
    int io_flags = io.flags;
    float l2_eps = io.l2_eps;
    const int nseq = packed ? n_seqs : B;
    const int64_t n_tok = packed ? T : (int64_t)B * T;
    const int nck = (int)((T + CH - 1) / CH);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    int32_t *chunk_off = nullptr;
    unsigned char *blobs = ws;
    int64_t slots = (int64_t)B * nck;
    const int n_sm = sm_count();
    BatchedPlan plan{0, 0, 0, 0};
    if (packed) {
        chunk_off = reinterpret_cast<int32_t *>(ws);
        blobs = ws + packed_head_bytes(n_seqs);
        slots = T / CH + n_seqs;
        chunk_offsets_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, n_seqs, T, chunk_off);
    } else {
        blobs = ws + batched_head_bytes(B, nck, H);
        // the fused grid's prep workers have no L2 normalisation: with it the call runs
        // the prep and the chains
        plan = n_tok > 0 ? batched_plan(B, H, nck, n_sm) : BatchedPlan{0, 0, 0, 0};
        if ((io_flags & IO_QK_L2NORM) != 0 && plan.kind == 1) plan = BatchedPlan{0, 0, 0, 0};
        if (plan.kind == 1) {
            int32_t *ready = reinterpret_cast<int32_t *>(ws);
            FusedQueue *queue = reinterpret_cast<FusedQueue *>(ready + (size_t)B * nck * H);
            cudaError_t err = cudaMemsetAsync(ws, 0, (size_t)B * nck * H * 4 + sizeof(FusedQueue), stream);
            if (err != cudaSuccess) return err;
            CUtensorMap mq, mk, mla, mv;
            if (!make_map(&mq, q, true, n_tok, H) || !make_map(&mk, k, true, n_tok, H) ||
                !make_gate_map(&mla, log_alpha, gate, n_tok, H, mq) || !make_map(&mv, v, true, n_tok, H))
                return cudaErrorInvalidValue;
            const __nv_bfloat16 *qb = (const __nv_bfloat16 *)q, *kb = (const __nv_bfloat16 *)k;
            __nv_bfloat16 *ob = (__nv_bfloat16 *)o;
            int n_chain = 2 * B * H, n_first = plan.n_first;
            void *args[] = {&mq, &mk, &mla, &mv, &qb, &kb, (void *)&log_alpha, (void *)&beta, &blobs,
                            &ready, &queue, (void *)&S0, &ob, &S_T, &T, &H, &B, (void *)&nck,
                            &n_first, &n_chain, &io_flags, &l2_eps};
            return with_gate(gate, [&](auto g) {
                return cudaLaunchCooperativeKernel((const void *)kda_fused_kernel<64, decltype(g)::value>,
                                                   dim3((unsigned)n_sm), dim3(FUSED_NT), args,
                                                   fused_smem<64>(), stream);
            });
        }
    }
    cudaError_t err;
    const bool prep_launched = n_tok > 0 && slots > 0;
    if (prep_launched) {
        CUtensorMap mq, mk, mla;
        if (!make_map(&mq, q, true, n_tok, H) || !make_map(&mk, k, true, n_tok, H) ||
            !make_gate_map(&mla, log_alpha, gate, n_tok, H, mq))
            return cudaErrorInvalidValue;
        auto launch_prep = [&](auto kernel) {
            cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PREP_SMEM);
            if (e == cudaSuccess)  // four CTAs per SM need the largest shared-memory carveout
                e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
            const int pf_dist = prep_residency(kernel);
            kernel<<<dim3((unsigned)slots, (unsigned)H), PREP_NT, PREP_SMEM, stream>>>(
                mq, mk, mla, pf_dist, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, log_alpha,
                beta, blobs, chunk_off, cu_seqlens, T, H, n_seqs, nck, io_flags, l2_eps);
            return cudaGetLastError();
        };
        err = with_gate(gate, [&](auto g) {
            constexpr int G = decltype(g)::value;
            return (io_flags & IO_QK_L2NORM) ? launch_prep(kda_prep_kernel<G, true>)
                                             : launch_prep(kda_prep_kernel<G, false>);
        });
        if (err != cudaSuccess) return err;
    }
    CUtensorMap mv;
    if (n_tok > 0 && !make_map(&mv, v, true, n_tok, H)) return cudaErrorInvalidValue;
    if (plan.kind == 2) {  // segment scan: pass 1, combine, pass 2
        const int P = B * H, cap = seg_capacity(B, H, nck);
        float *base = reinterpret_cast<float *>(blobs + (size_t)B * nck * H * BLOB_BYTES);
        const size_t per = (size_t)P * cap * (D * D);
        const SegScan sg{base, base + per, base + 2 * per, plan.n_seg, plan.seg_len};
        using Lay = ChainLayout<64>;
        err = cudaFuncSetAttribute(kda_seg_pass_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)Lay::BYTES);
        if (err != cudaSuccess) return err;
        __nv_bfloat16 *ob = (__nv_bfloat16 *)o;
        err = launch_maybe_dependent(kda_seg_pass_kernel<64>, dim3((unsigned)(2 * P), (unsigned)(2 * plan.n_seg - 3)),
                                     dim3(CHAIN_NT), Lay::BYTES, stream, prep_launched, mv, blobs, S0, ob,
                                     S_T, T, H, nck, sg, 1);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(kda_seg_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)SEG_COMBINE_SMEM);
        if (err != cudaSuccess) return err;
        kda_seg_combine_kernel<<<(D / SEG_NJ) * P, SEG_COMBINE_NT, SEG_COMBINE_SMEM, stream>>>(sg);
        kda_seg_pass_kernel<64><<<dim3((unsigned)(2 * P), (unsigned)(plan.n_seg - 1)), CHAIN_NT,
                                  Lay::BYTES, stream>>>(mv, blobs, S0, ob, S_T, T, H, nck, sg, 2);
        return cudaGetLastError();
    }
    // 128-column slices (one CTA per sequence-head) when twice as many 64-column chains
    // would need more waves than that saves (about 75 sequence-heads and up on 148 SMs);
    // otherwise 64-column slices for twice the parallelism.
    if (wide_chain((int64_t)nseq * H, n_sm))
        return launch_chain<128>(mv, blobs, chunk_off, S0, o, S_T, cu_seqlens, T, H, nck, nseq,
                                 prep_launched, stream);
    return launch_chain<64>(mv, blobs, chunk_off, S0, o, S_T, cu_seqlens, T, H, nck, nseq,
                            prep_launched, stream);
}

int read_device_status(int *status) {
    int v[2] = {0, 0};  // timeouts, bad_input
    if (cudaMemcpyFromSymbol(v, g_kda_status, sizeof(v)) != cudaSuccess) return -1;
    const int zero[2] = {0, 0};
    if (cudaMemcpyToSymbol(g_kda_status, zero, sizeof(zero)) != cudaSuccess) return -1;
    int simt_bad = 0;
    if (read_simt_bad_input(&simt_bad) != 0) return -1;
    *status = (v[0] != 0 ? KDA_STATUS_TIMEOUT : 0) | (v[1] + simt_bad != 0 ? KDA_STATUS_BAD_INPUT : 0);
    return 0;
}

int set_wait_limit_ns(unsigned long long ns) {
    const unsigned long long limit = ns ? ns : ptx::WAIT_LIMIT_NS;
    return cudaMemcpyToSymbol(g_kda_status, &limit, sizeof(limit),
                              offsetof(ptx::DeviceStatus, wait_limit_ns)) == cudaSuccess
               ? 0
               : -1;
}

namespace {
// Self-test of the failure path: one warp runs the three kinds of bounded wait the
// kernels use on conditions that never come true (an mbarrier nobody arrives on, a
// global flag nobody sets, a shared counter nobody raises), each with its own `dead`
// flag so that every one of them runs its slow path. No copy or MMA is in flight, so
// the kernel leaves nothing behind when it returns. Bit b of *result is set when wait
// b gave up.
__global__ void __launch_bounds__(32) kda_wait_selftest_kernel(const int32_t *flag, int32_t *result) {
    __shared__ uint64_t bar;
    __shared__ int32_t counter;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        counter = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        int32_t bits = 0;
        bool dead0 = false, dead1 = false, dead2 = false;
        if (!mbar_wait(&bar, 0, dead0, &g_kda_status)) bits |= 1;
        if (!flag_wait(flag, dead1, &g_kda_status)) bits |= 2;
        if (!counter_wait_gt(&counter, 0, dead2, &g_kda_status)) bits |= 4;
        *result = bits;
        mbar_inval(&bar);
    }
}
}  // namespace

cudaError_t launch_wait_selftest(const int32_t *flag, int32_t *result, cudaStream_t stream) {
    kda_wait_selftest_kernel<<<1, 32, 0, stream>>>(flag, result);
    return cudaGetLastError();
}

}  // namespace kda
