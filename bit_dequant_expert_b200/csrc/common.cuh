// Shared device helpers of the moe_b200 kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr int kWarp = 32;

// ------------------------------------------------------------------ layout

// Workspace header: sticky error word at byte 0, the small-T router's
// last-block ticket at byte 4 (left at zero by every call), the decode
// kernels' launch counter at byte 8 (monotonic, 64-bit: every decode launch
// adds its grid size, so count / grid size numbers the launches); the rest
// of the first 256 bytes is reserved.  Scratch sections follow, 256-byte
// aligned.
struct WsHeader {
    int32_t error;
    uint32_t route_ticket;
    unsigned long long decode_launches;
    int32_t reserved[60];
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// ------------------------------------------------------------------ errors

// First error wins; later ones are dropped so the report names the root cause.
__device__ __forceinline__ void set_error(int32_t* err, int32_t code) {
    if (err) atomicCAS(err, 0, code);
}

// ------------------------------------------------------------------ bf16

__device__ __forceinline__ float bf16_lo(uint32_t pair) { return __uint_as_float(pair << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t pair) { return __uint_as_float(pair & 0xFFFF0000u); }

// fp32 -> bf16 bits, round to nearest even (hardware conversion).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

// (lo, hi) -> bf16x2 bits, each rounded to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// ------------------------------------------------------------------ loads

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Raises a kernel's dynamic shared-memory limit when a launch needs more than
// was set before on this device (kernel attributes are per device; after the
// first launch of each size the call is skipped, so it stays out of stream
// capture).  `set_bytes` is a per-kernel table of 64 devices.
template <typename Kern>
inline cudaError_t set_smem_once(Kern* k, int bytes, int* set_bytes) {
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return ce;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (__atomic_load_n(&set_bytes[dev], __ATOMIC_ACQUIRE) >= bytes) return cudaSuccess;
    ce = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (ce == cudaSuccess) {
        int cur = __atomic_load_n(&set_bytes[dev], __ATOMIC_ACQUIRE);
        while (cur < bytes && !__atomic_compare_exchange_n(&set_bytes[dev], &cur, bytes, false, __ATOMIC_ACQ_REL,
                                                           __ATOMIC_ACQUIRE)) {
        }
    }
    return ce;
}

// Launch with programmatic dependent launch allowed: the kernel may start
// while the previous grid on the stream finishes, and must execute
// griddepcontrol.wait before touching anything that grid writes or reads.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace moe
