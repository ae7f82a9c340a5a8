// Output epilogue of the KDA layer: head-wise RMSNorm and sigmoid output gate.
//
// blog.gzher.com "Kimi K3论文：Kimi Linear", section 3 (neural parameterisation): the
// operator's output goes through a head-wise RMSNorm and an output gate Sigmoid(W_g x)
// before the output projection. Per (token, head) row of 128 channels:
//
//   o_c <- o_c / sqrt(mean_c' o_c'^2 + eps) * w_c * sigmoid(g_c)
//
// It runs after the prefill kernels of a call, in place on o, whichever plan the call
// took. The step is bound by HBM bandwidth: each row reads o and g and writes o
// (3 x 256 bytes in bf16), with w held in registers.
//
// Layout: one warp per row, lane l on channels 4l .. 4l+3 (one 8-byte bf16 or 16-byte
// fp32 access per lane, a contiguous 256 / 512-byte segment per warp). Each warp takes
// EPI_ROWS rows, all loads issued before any arithmetic; the grid covers every row once.
// It is launched as a programmatic dependent of the call's last kernel: its CTAs may be
// scheduled while that kernel drains, and wait for its completion (griddepcontrol.wait)
// before reading o.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int EPI_NT = 256;
constexpr int EPI_ROWS = 4;  // rows in flight per warp

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    using type = float4;
    __device__ static float4 to_f32(float4 v) { return v; }
    __device__ static float4 from_f32(float4 v) { return v; }
};
template <> struct Vec4<__nv_bfloat16> {
    using type = uint2;  // four bf16
    __device__ static float4 to_f32(uint2 v) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    __device__ static uint2 from_f32(float4 v) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        uint2 r;
        r.x = *reinterpret_cast<const uint32_t *>(&a);
        r.y = *reinterpret_cast<const uint32_t *>(&b);
        return r;
    }
};

template <typename T>
__global__ void __launch_bounds__(EPI_NT)
kda_out_epilogue_kernel(T *__restrict__ o, const T *__restrict__ gate, const float *__restrict__ w,
                        float eps, int64_t rows) {
    using V = Vec4<T>;
    using VT = typename V::type;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * EPI_NT + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * EPI_NT) >> 5;
    const float4 wl = w ? __ldg(reinterpret_cast<const float4 *>(w) + lane) : make_float4(1.f, 1.f, 1.f, 1.f);
    VT *ov = reinterpret_cast<VT *>(o);
    const VT *gv = reinterpret_cast<const VT *>(gate);
    asm volatile("griddepcontrol.wait;" ::: "memory");  // o is final once the previous kernel completed
    for (int64_t r0 = warp0 * EPI_ROWS; r0 < rows; r0 += n_warps * EPI_ROWS) {
        VT ox[EPI_ROWS], gx[EPI_ROWS];
#pragma unroll
        for (int i = 0; i < EPI_ROWS; ++i) {
            if (r0 + i < rows) {
                ox[i] = __ldcs(ov + (r0 + i) * (D / 4) + lane);
                gx[i] = __ldcs(gv + (r0 + i) * (D / 4) + lane);
            }
        }
#pragma unroll
        for (int i = 0; i < EPI_ROWS; ++i) {
            if (r0 + i >= rows) break;  // uniform over the warp
            const float4 x = V::to_f32(ox[i]), g = V::to_f32(gx[i]);
            float ss = x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float inv = rsqrtf(ss * (1.f / D) + eps);
            const float4 y = make_float4(x.x * inv * wl.x * sigmoid(g.x), x.y * inv * wl.y * sigmoid(g.y),
                                         x.z * inv * wl.z * sigmoid(g.z), x.w * inv * wl.w * sigmoid(g.w));
            __stcs(ov + (r0 + i) * (D / 4) + lane, V::from_f32(y));
        }
    }
}

}  // namespace

cudaError_t launch_out_epilogue(void *o, const IoOpts &io, int64_t rows, int dtype, cudaStream_t stream) {
    if (rows <= 0 || !io.out_gate) return cudaSuccess;
    // 8 warps per CTA, EPI_ROWS rows per warp: one pass over the rows (grid-x limit 2^31 - 1)
    const int64_t need = (rows + 8 * EPI_ROWS - 1) / (8 * EPI_ROWS);
    const unsigned grid = (unsigned)(need < 0x7fffffff ? need : 0x7fffffff);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(EPI_NT);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (dtype == KDA_BF16)
        return cudaLaunchKernelEx(&cfg, kda_out_epilogue_kernel<__nv_bfloat16>, static_cast<__nv_bfloat16 *>(o),
                                  static_cast<const __nv_bfloat16 *>(io.out_gate), io.out_w, io.out_eps, rows);
    return cudaLaunchKernelEx(&cfg, kda_out_epilogue_kernel<float>, static_cast<float *>(o),
                              static_cast<const float *>(io.out_gate), io.out_w, io.out_eps, rows);
}

}  // namespace kda
