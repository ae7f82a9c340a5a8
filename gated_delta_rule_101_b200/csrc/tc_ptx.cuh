// Thin inline-PTX wrappers for the sm_100a features the tensor-core path uses:
// mbarriers, TMA (tiled tensor and 1-D bulk copies), and tcgen05 (TMEM
// allocation, MMA issue/commit, TMEM loads). Written from the PTX ISA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace kda {
namespace ptx {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
// Ends an mbarrier's life; required before its memory is used for anything else.
__device__ __forceinline__ void mbar_inval(uint64_t *bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Device status shared by the tensor-core kernels of the library.
//   timeouts:      number of bounded waits that have given up since the host last
//                  read and cleared it (kda_get_device_status).
//   bad_input:     number of calls whose device-side sequence offsets failed the
//                  checks of a KDA_DEBUG build (always 0 in the ordinary build).
//   wait_limit_ns: how long a wait may take before it gives up (one second; tests of
//                  the failure path shorten it through kda_set_wait_limit_ns).
struct DeviceStatus {
    int timeouts;
    int bad_input;
    unsigned long long wait_limit_ns;
};
constexpr unsigned long long WAIT_LIMIT_NS = 1000000000ull;  // the default limit: one second

// Bookkeeping of one wait's slow path. It starts when the wait is first found not
// complete: it notes the time, the limit in force and the timeout count at that moment.
// The wait gives up when its limit has passed, or as soon as the count has moved, that
// is when any CTA has given up on a wait since this one began (so one failure does not
// make every other CTA wait its full limit in turn). A count left over from an earlier
// launch does not count: only changes seen while waiting do, so a timeout that nobody
// has read yet cannot make a later call give up early.
struct WaitClock {
    uint64_t t0, limit;
    int base;
    __device__ __forceinline__ explicit WaitClock(const DeviceStatus *st)
        : t0(global_ns()),
          limit(*reinterpret_cast<const volatile unsigned long long *>(&st->wait_limit_ns)),
          base(*reinterpret_cast<const volatile int *>(&st->timeouts)) {}
    __device__ __forceinline__ bool expired(const DeviceStatus *st) const {
        return *reinterpret_cast<const volatile int *>(&st->timeouts) != base || global_ns() - t0 > limit;
    }
};
__device__ __forceinline__ void record_timeout(DeviceStatus *st, bool &dead) {
    dead = true;
    atomicAdd(&st->timeouts, 1);
}

// Waits for `parity` on `bar`, bounded as WaitClock describes. On giving up it
// counts a timeout in *st and sets `dead`; once `dead` is set every later wait
// returns at once, so the kernel unwinds instead of hanging.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, bool &dead, DeviceStatus *st) {
    if (dead) return false;
    if (mbar_try_wait(bar, parity)) return true;
    const WaitClock clk(st);
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0 && clk.expired(st)) break;
    }
    record_timeout(st, dead);
    return false;
}

// ------------------------------------------------------------------ dependent launch
// A kernel launched with programmatic stream serialization may start while the kernel
// before it on the stream still runs, once every CTA of that one has called
// griddep_launch_dependents (or exited). It must call griddep_wait, which returns when
// the earlier kernel has completed and its writes are visible, before reading them.
// Both are no-ops for kernels launched the ordinary way.
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ cross-CTA flags
// Between CTAs of one cooperative grid (all resident at once): a producer publishes
// data it wrote to global memory with bulk copies by waiting for the copies to
// complete, then flag_publish; a consumer that sees the flag set (flag_wait) may then
// read that data, also with bulk copies. The producer must never wait on its consumer.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void flag_publish(int32_t *flag) {
    fence_proxy_async_global();
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(1) : "memory");
}
__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t *p) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Waits until *flag != 0, with the same limit and failure reporting as mbar_wait.
__device__ __forceinline__ bool flag_wait(const int32_t *flag, bool &dead, DeviceStatus *st) {
    if (dead) return false;
    if (ld_acquire_gpu(flag) != 0) {
        fence_proxy_async_global();
        return true;
    }
    const WaitClock clk(st);
    for (uint32_t i = 1;; ++i) {
        __nanosleep(100);
        if (ld_acquire_gpu(flag) != 0) {
            fence_proxy_async_global();
            return true;
        }
        if ((i & 63u) == 0 && clk.expired(st)) break;
    }
    record_timeout(st, dead);
    return false;
}

// Counter in shared memory raised by one thread and read by others in the CTA.
__device__ __forceinline__ int32_t ld_acquire_cta(const int32_t *p) {
    int32_t v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_cta(int32_t *p, int32_t v) {
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
// Waits until the shared counter *p exceeds v, with the limit and failure reporting of
// mbar_wait; the counter's writer has seen global data the caller will then read with
// bulk copies.
__device__ __forceinline__ bool counter_wait_gt(const int32_t *p, int32_t v, bool &dead, DeviceStatus *st) {
    if (dead) return false;
    if (ld_acquire_cta(p) > v) {
        fence_proxy_async_global();
        return true;
    }
    const WaitClock clk(st);
    for (uint32_t i = 1;; ++i) {
        if (ld_acquire_cta(p) > v) {
            fence_proxy_async_global();
            return true;
        }
        if ((i & 255u) == 0 && clk.expired(st)) break;
    }
    record_timeout(st, dead);
    return false;
}

// CTA-wide wait: thread 0 polls the barrier while every other thread sleeps at
// the CTA barrier (polling threads would take issue slots from co-resident
// CTAs). All threads leave with the same `dead` value.
__device__ __forceinline__ void cta_wait(uint64_t *bar, uint32_t parity, bool &dead, DeviceStatus *status) {
    bool ok = true;
    if (threadIdx.x == 0) ok = mbar_wait(bar, parity, dead, status);
    dead = __syncthreads_or(!ok || dead) != 0;
}

// Named CTA barriers (ids 1..15; id 0 belongs to __syncthreads). `count` is the
// number of threads taking part, a multiple of 32. bar.arrive does not wait; like
// bar.sync it makes the arriving thread's earlier memory accesses visible to the
// threads that wait on the barrier.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(uint32_t id, uint32_t count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// bar.sync that also returns the OR of `pred` over the participating threads.
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------------------ async proxy / TMA
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> shared, completing `bytes` on `bar`. Addresses and
// size must be multiples of 16 bytes.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// 1-D bulk copy shared -> global (bulk-group completion).
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Waits until the shared-memory sources of all committed bulk stores have been read.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// 2-D tiled tensor load into this CTA's shared memory. x is the innermost coordinate.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Brings the cache line of a global address into L2 without waiting for it.
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}
// Brings the box at (x, y) of a tiled tensor into L2 without waiting for it.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

// ------------------------------------------------------------------ register budget
// Moves registers between the warpgroups of a CTA (all four warps of a warpgroup
// execute it). The counts must be multiples of 8 in [24, 256], and the increases of
// all warpgroups together must not exceed what the decreases and the launch leave.
template <int R>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}

// ------------------------------------------------------------------ tcgen05
// TMEM allocation (whole warp). ncols: power of two >= 32.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}
// Arrive once on `bar` when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Loads 32 consecutive 32-bit TMEM columns of this thread's lane
// (lane = 32 * (warp % 4) + lane id) starting at taddr, and waits for them:
// the wait sits in the same asm statement so no use of the registers can be
// scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 8 consecutive columns, with the wait in the same statement.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// 64 consecutive columns in one load, with the wait in the same statement.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float *v) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------------ warp-level MMA
// D (16x8, fp32) += A (16x8) * B (8x8), tf32 inputs. Used only for the 16- and
// 32-wide block products inside the 64 x 64 triangular inverse, which are far
// below tcgen05's 64-row minimum. Fragments (g = lane / 4, t = lane % 4):
//   A: a0 (g, t), a1 (g+8, t), a2 (g, t+4), a3 (g+8, t+4)
//   B: b0 (t, g), b1 (t+4, g)
//   D: d0 (g, 2t), d1 (g, 2t+1), d2 (g+8, 2t), d3 (g+8, 2t+1)
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// One 16 x 8 tile of D = A * B over K (multiple of 8), with A and B read from
// shared memory: A(i, k) = a[i * lda + k], B(k, j) = b[k * ldb + j].
template <int K>
__device__ __forceinline__ void warp_gemm_16x8(float (&d)[4], const float *a, int lda, const float *b,
                                               int ldb) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t af[4] = {to_tf32(a[g * lda + k0 + t]), to_tf32(a[(g + 8) * lda + k0 + t]),
                                to_tf32(a[g * lda + k0 + t + 4]), to_tf32(a[(g + 8) * lda + k0 + t + 4])};
        const uint32_t bf[2] = {to_tf32(b[(k0 + t) * ldb + g]), to_tf32(b[(k0 + t + 4) * ldb + g])};
        mma_tf32_16x8x8(d, af, bf);
    }
}
// Stores a D tile (scaled by s) to c[i * ldc + j].
__device__ __forceinline__ void warp_store_16x8(const float (&d)[4], float *c, int ldc, float s) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    c[g * ldc + 2 * t] = s * d[0];
    c[g * ldc + 2 * t + 1] = s * d[1];
    c[(g + 8) * ldc + 2 * t] = s * d[2];
    c[(g + 8) * ldc + 2 * t + 1] = s * d[3];
}

// ------------------------------------------------------------------ operand layouts
// K-major bf16 operand tiles with the 128-byte swizzle: `rows` rows (a
// multiple of 8), K a multiple of 64. Each group of 64 K-elements is an
// "atom column" of rows x 128 bytes; inside it row r sits at r * 128 and its
// 16-byte chunk q is stored at chunk position q ^ (r % 8). Tiles start on a
// 1024-byte boundary so the swizzle phase matches the hardware's.
__device__ __forceinline__ uint32_t sw128_chunk_off(uint32_t row, uint32_t chunk, uint32_t rows) {
    // chunk: 16-byte chunk index along K (0 .. K/8 - 1)
    const uint32_t kb = chunk >> 3, q = chunk & 7;
    return kb * rows * 128u + row * 128u + ((q ^ (row & 7u)) << 4);
}
__device__ __forceinline__ uint32_t sw128_elem_off(uint32_t row, uint32_t k, uint32_t rows) {
    return sw128_chunk_off(row, k >> 3, rows) + ((k & 7u) << 1);
}

// Shared-memory matrix descriptor for a SWIZZLE_128B operand tile. The tile is
// made of 128-byte rows (64 bf16 elements each, 16-byte chunks XOR-swizzled
// by row % 8), 8-row groups 1024 bytes apart (the stride byte offset).
// K-major operands: rows are M (or N) rows, the 64 elements run along K.
// MN-major operands: rows are K rows, the 64 elements run along M (or N);
// further blocks of 64 M/N elements sit `lbo` bytes apart (leading byte offset).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr, uint32_t lbo = 16) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);   // start address, 16-byte units
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;     // leading byte offset
    d |= (uint64_t)(1024u >> 4) << 32;               // stride byte offset: 8-row group pitch
    d |= (uint64_t)1u << 46;                         // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                         // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: bf16 A and B, fp32 accumulator, M x N; a_mn / b_mn
// select MN-major (1) or K-major (0) operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn = 0, int b_mn = 0) {
    return (1u << 4)    // D format: f32
           | (1u << 7)  // A format: bf16
           | (1u << 10) // B format: bf16
           | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// One MMA operand in shared memory.
//   K-major:  `rows` rows of the tile; 64-element K blocks are rows*128 bytes apart.
//   MN-major: K runs down the rows; `lbo` = bytes between 64-element M/N blocks.
// The descriptor of the kk-th K step (16 elements) is the base descriptor plus
// the step's byte offset in 16-byte units (shared addresses stay below 256 KiB,
// so the 14-bit start-address field never carries).
struct Operand {
    uint64_t base_desc;
    uint32_t rows;  // K-major row count (0 for MN-major)
    __device__ __forceinline__ uint64_t desc(int kk) const {
        const uint32_t off = rows ? ((uint32_t)kk >> 2) * rows * 128u + ((uint32_t)kk & 3u) * 32u
                                  : (uint32_t)kk * 2048u;
        return base_desc + (uint64_t)(off >> 4);
    }
};
__device__ __forceinline__ Operand kmajor(uint32_t base, uint32_t rows) {
    return {sw128_desc(base), rows};
}
__device__ __forceinline__ Operand mnmajor(uint32_t base, uint32_t lbo) {
    return {sw128_desc(base, lbo), 0u};
}

// Issues the K/16 MMAs of D (+)= A * B (A: M x K, B: K x N as described by
// the operands; the instruction descriptor must carry the same majorness).
template <int K>
__device__ __forceinline__ void mma_run(uint32_t d_tmem, Operand a, Operand b, uint32_t idesc,
                                        bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < K / 16; ++kk)
        mma_bf16(d_tmem, a.desc(kk), b.desc(kk), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

}  // namespace ptx
}  // namespace kda
