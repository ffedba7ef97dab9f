// Failure-detection self-test: makes one of the two kinds of bounded device
// wait the kernels use expire on purpose, so that a caller can check that an
// expired wait surfaces as MOE_ERR_TIMEOUT in the workspace error word and
// that the CUDA context stays usable afterwards.  Nothing is computed.
//
//   kind 0  a pipeline wait: one thread waits on a shared-memory mbarrier that
//           no thread or copy ever arrives on (the producer/consumer wait of
//           the tensor-core FFN pipeline), through the same bounded wait;
//   kind 1  a grid barrier: the CTAs of the launch count themselves on a
//           64-bit counter in global memory and wait until all are counted
//           (the decode kernels' barrier), with the arrival of one chosen CTA
//           suppressed by a host-set parameter.
//
// Every wait ends after limit_ns of global time at the latest; no CTA depends
// on another for progress beyond that.
#include <cuda_runtime.h>

#include <cstddef>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

// The counter of kind 1: the first 8 reserved bytes of the workspace header
// (byte offset 16), cleared by the host before every launch.
constexpr size_t kCounterOffset = 16;
static_assert(kCounterOffset + 8 <= sizeof(WsHeader), "counter inside the workspace header");
static_assert(kCounterOffset >= offsetof(WsHeader, reserved), "counter in the reserved bytes");

__device__ __forceinline__ unsigned long long counter_load_acquire(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void counter_add_release(unsigned long long* p) {
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(p) : "memory");
}

__global__ void k_wait_selftest(int kind, int skip_cta, uint64_t limit_ns, unsigned long long* counter,
                                int32_t* err) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    if (kind == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        // phase 0 never completes: the wait gives up after limit_ns and records the timeout
        mbar_wait_bounded(&bar, 0, err, limit_ns);
        return;
    }
    if ((int)blockIdx.x != skip_cta) counter_add_release(counter);
    const uint64_t t0 = globaltimer_ns();
    while (counter_load_acquire(counter) < gridDim.x) {
        if (globaltimer_ns() - t0 > limit_ns) {
            set_error(err, MOE_ERR_TIMEOUT);
            break;
        }
        __nanosleep(256);
    }
}

}  // namespace

}  // namespace moe

extern "C" int32_t moe_wait_selftest(int32_t kind, int32_t ctas, int32_t skip_cta, uint64_t limit_ns, void* ws,
                                     void* stream) {
    using namespace moe;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return MOE_ERR_WORKSPACE;
    if (kind != 0 && kind != 1) return MOE_ERR_INVALID_ARG;
    if (limit_ns < 1000ull || limit_ns > 1000000000ull) return MOE_ERR_INVALID_ARG;
    if (kind == 0 && (ctas != 1 || skip_cta != -1)) return MOE_ERR_INVALID_ARG;
    if (kind == 1 && (ctas < 1 || ctas > 148 || skip_cta < -1 || skip_cta >= ctas)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* base = static_cast<uint8_t*>(ws);
    auto* counter = reinterpret_cast<unsigned long long*>(base + kCounterOffset);
    if (cudaMemsetAsync(counter, 0, sizeof(*counter), s) != cudaSuccess) return MOE_ERR_CUDA;
    k_wait_selftest<<<ctas, 32, 0, s>>>(kind, skip_cta, limit_ns, counter, reinterpret_cast<int32_t*>(base));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
