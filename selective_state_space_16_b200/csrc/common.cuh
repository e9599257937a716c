// common.cuh -- small sm_100a building blocks shared by the scan kernels:
// shared-memory addressing, mbarriers with bounded waits, TMA (cp.async.bulk.tensor)
// loads/stores, proxy fences, bf16 packing and the device status word.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ssm {

// Device status codes written into the workspace status word (same values as ssm_status_t).
constexpr uint32_t kDevTimeout = 4u;

// Layout of the first 256 bytes of every forward workspace.
struct WorkspaceHeader {
    uint32_t epoch;       // flag tag of the previous chunked launch (tags are epoch + 1)
    uint32_t ticket;      // dynamic work-unit counter of the chunked kernel
    uint32_t done;        // CTAs of the current chunked launch that have finished
    uint32_t status;      // device-side error (0 = none); read and cleared by ssm_read_status
    uint32_t where[4];    // first failing wait: kind, unit, chunk, polls
    uint32_t pad[56];
};
static_assert(sizeof(WorkspaceHeader) == 256, "header must stay 256 bytes");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------------
// mbarrier (transaction-counting barrier in shared memory)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

// Bounded wait for phase `parity` of `bar`.  Each try_wait already suspends the
// thread for a hardware-chosen interval; after `limit` unsuccessful tries the
// wait gives up and returns false, so a lost transaction can never hang the GPU.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// As mbar_wait_bounded, sleeping ~128 ns between tries: for a waiter that is far ahead
// (the producer of a ring), so that its polling does not take issue slots from the
// warps it waits for.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        __nanosleep(128);
    }
    return false;
}

// ---------------------------------------------------------------------------------------
// TMA (tensor-map bulk copies) and bulk groups
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// 3-D tiled store shared -> global (elements outside the tensor are dropped).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// 16-byte asynchronous copy global -> shared (cp.async, cached in L2 only); only the
// first src_bytes (0 or 16) are read, the rest of the 16 bytes is zero-filled.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed cp.async groups are still pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Order this thread's generic-proxy shared-memory accesses before later async-proxy
// (TMA) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier `id` over `threads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------------------------------
// Global-memory flags for the inter-CTA carry
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Order this thread's earlier memory accesses before its later ones, GPU scope.
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Programmatic dependent launch: pdl_launch_dependents lets the next kernel of the stream (if
// launched with programmatic serialization) start before this one ends; pdl_wait_primary waits
// until the previous kernel has completed and its writes are visible (a no-op when this kernel
// was launched normally).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ float4 ld_relaxed_gpu_f4(const float4* p) {
    float4 v;
    asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// Record the first device-side failure in the workspace header (later ones are dropped).
__device__ __forceinline__ void report_status(WorkspaceHeader* hdr, uint32_t code, uint32_t kind,
                                              uint32_t unit, uint32_t chunk, uint32_t polls) {
    if (hdr == nullptr) return;
    if (atomicCAS(&hdr->status, 0u, code) == 0u) {
        hdr->where[0] = kind;
        hdr->where[1] = unit;
        hdr->where[2] = chunk;
        hdr->where[3] = polls;
    }
}

// Range checks of the debug build (-DSSM_DEBUG_CHECKS).  dcheck(hdr, ok, site, value)
// returns ok; when ok is false it records kDevBounds in the workspace header with
// where = {site, block, thread, value}, and the caller skips the guarded access, so a bad
// index is reported instead of touching memory.  Release builds compile every check away
// (dcheck is constant true and its arguments are never evaluated for effect).
constexpr uint32_t kDevBounds = 7u;
enum DcheckSite : uint32_t {
    kSiteSeqTile = 1,       // sequential kernel: tile / batch-row slot of a consumer lane in the round
    kSiteSeqTma = 2,        // sequential kernel: TMA destination or coordinate of a stage copy
    kSiteSeqY = 3,          // sequential kernel: y element index
    kSiteSeqState = 4,      // sequential kernel: last_state index
    kSiteChunkKey = 5,      // chunked kernel: look-back key (flags / payload)
    kSiteChunkSmem = 6,     // chunked kernel: shared aggregate / speculative carry index
    kSiteChunkY = 7,        // chunked kernel: y element or last_state index
    kSiteDirect = 8,        // direct kernel: B/C row, y or last_state index
    kSitePack = 9,          // B/C transpose: workspace row index
    kSiteBwdCkpt = 10,      // backward: checkpoint index
    kSiteBwdPart = 11,      // backward: per-CTA dB/dC partial index
    kSiteBwdOut = 12,       // backward: gradient element index
    kSiteBwdSmem = 13,      // backward: shared ring / per-warp buffer offset
};
#ifdef SSM_DEBUG_CHECKS
__device__ __forceinline__ bool dcheck(WorkspaceHeader* hdr, bool ok, uint32_t site, long long value) {
    if (!ok) report_status(hdr, kDevBounds, site, blockIdx.x, threadIdx.x, static_cast<uint32_t>(value));
    return ok;
}
#else
__device__ __forceinline__ constexpr bool dcheck(WorkspaceHeader*, bool, uint32_t, long long) { return true; }
#endif

// ---------------------------------------------------------------------------------------
// Element types
// ---------------------------------------------------------------------------------------
template <typename T>
struct IoTraits;

template <>
struct IoTraits<float> {
    static constexpr int kBytes = 4;
    static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    __device__ __forceinline__ static float to_f32(float v) { return v; }
    __device__ __forceinline__ static float from_f32(float v) { return v; }
};

template <>
struct IoTraits<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    __device__ __forceinline__ static float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ __forceinline__ static __nv_bfloat16 from_f32(float v) { return __float2bfloat16_rn(v); }
};

// A 16-byte group of consecutive elements of one row, unpacked to fp32.
template <typename T>
struct Group16;

template <>
struct Group16<__nv_bfloat16> {
    static constexpr int kN = 8;
    __device__ __forceinline__ static void unpack(const uint4& raw, float (&out)[8]) {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

template <>
struct Group16<float> {
    static constexpr int kN = 4;
    __device__ __forceinline__ static void unpack(const uint4& raw, float (&out)[4]) {
        out[0] = __uint_as_float(raw.x);
        out[1] = __uint_as_float(raw.y);
        out[2] = __uint_as_float(raw.z);
        out[3] = __uint_as_float(raw.w);
    }
};

// Round two fp32 values to bf16 (nearest-even) and pack them, first one in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace ssm
