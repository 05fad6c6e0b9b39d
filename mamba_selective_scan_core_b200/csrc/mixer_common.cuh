// Device helpers shared by the prefill and decode kernels of the Mamba mixer
// core: activation loads/stores, the two math flavours (exact and fast),
// small packed-fp32 helpers, and the mbarrier / bulk-tensor-copy wrappers the
// forward stages its tiles with.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------- act dtype
template <typename T> struct Act;
template <> struct Act<float> {
    using storage = float;
    static constexpr int kBytes = 4;
    __device__ __forceinline__ static float load(const float* p) { return *p; }
    __device__ __forceinline__ static float to_f32(float v) { return v; }
    __device__ __forceinline__ static float from_f32(float v) { return v; }
};
template <> struct Act<__nv_bfloat16> {
    using storage = __nv_bfloat16;
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static float to_f32(__nv_bfloat16 v) {
        return __uint_as_float(static_cast<uint32_t>(__bfloat16_as_ushort(v)) << 16);
    }
    __device__ __forceinline__ static float load(const __nv_bfloat16* p) { return to_f32(*p); }
    __device__ __forceinline__ static __nv_bfloat16 from_f32(float v) { return __float2bfloat16_rn(v); }
};

// ---------------------------------------------------------------- fast math
// Single MUFU instructions (inline PTX); used by the bf16 path, whose
// tolerance is set by bf16 rounding of the inputs and outputs.
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_fast(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Math policy.  kExact: CUDA's correctly-rounded-ish libm (expf/log1pf, IEEE
// division) in natural units.  kFast: MUFU ex2/lg2/tanh in log2 units.
//
// Both compute, for the pre-bias step input v = dt + dt_bias:
//   step(v)   : a scaled step size "l" such that Delta = l * step_scale
//   decay(l,a): exp(Delta * a) for a state coefficient a (= A[d, n])
// kExact: l = Delta, step_scale = 1, decay = expf(l * a).
// kFast : l = Delta / ln 2 (log2 of 1 + 2^(v log2 e)), step_scale = ln 2,
//         decay = 2^(l * a)   (= e^(Delta a), since Delta log2(e) = l).
struct MathExact {
    static constexpr float step_scale = 1.0f;
    __device__ __forceinline__ static float silu(float v) { return v / (1.0f + expf(-v)); }
    __device__ __forceinline__ static float step(float dt, float bias) {
        const float v = dt + bias;
        return fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
    }
    __device__ __forceinline__ static float decay(float l, float a) { return expf(l * a); }
};

struct MathFast {
    static constexpr float step_scale = kLn2;
    // SiLU(v) = v sigmoid(v) = h + h tanh(h) with h = v/2, since
    // sigmoid(v) = (1 + tanh(v/2)) / 2: one MUFU op instead of ex2 and rcp
    __device__ __forceinline__ static float silu(float v) {
        const float h = 0.5f * v;
        return fmaf(h, tanh_fast(h), h);
    }
    // bias2 = dt_bias * log2(e), precomputed per channel.
    __device__ __forceinline__ static float step2(float dt, float bias2) {
        const float v2 = fmaf(dt, kLog2e, bias2);
        // log2(1 + 2^v2), exact enough for v2 <= 126; beyond that 2^v2 would
        // overflow and the answer is v2 itself.
        const float l = lg2_fast(1.0f + ex2_fast(fminf(v2, 126.0f)));
        return fmaxf(l, v2);
    }
    __device__ __forceinline__ static float decay(float l, float a) { return ex2_fast(l * a); }
};

// ---------------------------------------------------------------- packed fp32
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// ---------------------------------------------------------------- shared memory
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// lane 0 of the warp does the work of a single-thread role
__device__ __forceinline__ bool elect_one_lane() { return (threadIdx.x & 31) == 0; }

// two floats -> a bf16 pair, round to nearest even, low half first
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

}  // namespace mm

// ---------------------------------------------------------------- TMA + mbarrier
#include <cuda.h>   // CUtensorMap

namespace mm {

// Set when a kernel gave up waiting for its own bulk copies (never expected:
// the wait limits only guard against a hung copy turning into a hung GPU).
__device__ unsigned int g_mm_fault;

// Index checks of the debug build (compiled with MM_CHECK_BOUNDS; the library
// file libmamba_mixer_checked.so): an access of `count` elements from index
// `first` of a buffer of `extent` elements is made only when it lies inside
// the buffer; otherwise it is skipped and recorded -- bit 1 of the device
// fault word and code kStatusBounds in the call's status -- instead of
// faulting.  The release build compiles every check to `true`.
#ifdef MM_CHECK_BOUNDS
constexpr bool kCheckBounds = true;
#else
constexpr bool kCheckBounds = false;
#endif
constexpr unsigned long long kStatusBounds = 3;    // call status code of a skipped access
constexpr unsigned kFaultBounds = 2;               // its bit in the device fault word
__device__ __forceinline__ bool mm_in_bounds(int64_t first, int64_t count, int64_t extent,
                                             unsigned long long* status, unsigned long long epoch) {
    if constexpr (!kCheckBounds) {
        return true;
    } else {
        if (first >= 0 && count >= 0 && first + count <= extent) return true;
        atomicOr(&g_mm_fault, kFaultBounds);
        if (status) atomicExch(status, (epoch << 8) | kStatusBounds);
        return false;
    }
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" :: "r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
// order this thread's earlier generic-proxy accesses of shared memory before
// later async-proxy (bulk copy) writes to it
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" :: "r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// Wait for the phase with the given parity to complete, trying at most
// `limit` times (each try itself waits a bounded, hardware-defined time).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, unsigned limit) {
    for (unsigned i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
// Programmatic dependent launch.  launch_dependents lets the next kernel in
// the stream, when launched as a programmatic dependent, start once every CTA
// of this grid has executed it (or exited).  grid_dependency_wait returns once
// the grid this one depends on has completed and its writes are visible; with
// no such dependency it returns at once.
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// 3-D tiled bulk tensor copy global -> this CTA's shared memory; completion
// is signalled on `bar` as transferred bytes.  No multicast.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n"
        :: "r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
        : "memory");
}

}  // namespace mm
