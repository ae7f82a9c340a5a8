// kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot
// allocate device memory.
//
// kda_chunk_fwd needs a caller-provided workspace for its bf16 path (the
// per-chunk operand images passed from the prep kernel to the chain kernel).
// Some callers cannot provide one: a plugin running inside a host framework
// that owns every byte of device memory through its own pool and offers its
// plugins no allocation hook, or a latency-critical loop that must not call
// cudaMalloc because cudaMalloc can synchronise the whole device. For them
// this file keeps one fixed scratch buffer in device memory, declared below as
// a static __device__ array, and runs the ordinary kda_chunk_fwd with it.
//
// Properties a caller must know:
//   - The scratch is KDA_NOALLOC_SCRATCH_BYTES (64 MiB) per GPU. It is part of
//     the library's device image: it is reserved on each GPU where that image
//     is loaded (when the CUDA context loads the library's module: at context
//     creation with CUDA_MODULE_LOADING=EAGER, otherwise on the first use of
//     one of its kernels or symbols) and held until the process exits, whether
//     or not this entry point is used.
//   - Problems whose workspace would exceed it are rejected with
//     KDA_ERR_SCRATCH_LIMIT before anything is launched.
//   - All calls on a GPU share the one buffer, and it keeps whatever the last
//     call left in it. Nothing in it needs to start at zero: every call
//     rewrites the parts it reads. Calls that can overlap on the GPU (issued
//     to different streams without ordering between them) race on the buffer
//     and corrupt each other's results; order them on one stream.
//   - The first call on each GPU looks up the buffer's device address
//     (cudaGetSymbolAddress, with that GPU current). Make that first call
//     before any stream capture begins.
//   - The address is kept for the life of the process. A device reset
//     (cudaDeviceReset) unloads the module and invalidates it, so this entry
//     point must not be used after one.
//   - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "kda_internal.cuh"

namespace {

constexpr size_t KDA_NOALLOC_SCRATCH_BYTES = (size_t)64 << 20;

// The scratch itself. In host code this name is only a stand-in for the
// symbol, not a device address: it must never be passed to a kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int KDA_MAX_DEVICES = 128;
void *g_scratch_addr[KDA_MAX_DEVICES];  // device address of the scratch, per GPU
std::mutex g_scratch_mu;

// Device address of the scratch on the current GPU; looked up once per GPU.
int scratch_on_current_device(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= KDA_MAX_DEVICES)
        return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" {

size_t kda_noalloc_scratch_bytes(void) { return KDA_NOALLOC_SCRATCH_BYTES; }

int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *S0, void *o, float *S_T, int B,
                          int64_t T, int H, int C, const int32_t *cu_seqlens, int n_seqs,
                          const int32_t *cu_seqlens_host, int dtype, void *stream) {
    size_t need = 0;
    const int st = kda_chunk_fwd_workspace_size(B, T, H, C, n_seqs, dtype, &need);
    if (st != KDA_OK) return st;
    if (need > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if (need > 0) {
        const int rc = scratch_on_current_device(&scratch);
        if (rc != KDA_OK) return rc;
    }
    return kda_chunk_fwd(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, C, cu_seqlens, n_seqs,
                         cu_seqlens_host, dtype, scratch, need > 0 ? KDA_NOALLOC_SCRATCH_BYTES : 0,
                         stream);
}

}  // extern "C"
