// Device helpers shared by every kernel of the FLARE++ mixer library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

namespace flarepp {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kNumSMs = 148;

// The device status word of the translation unit that includes this header
// (0 = no failure).  A kernel whose bounded wait runs out stores a nonzero
// code here and returns early.
static __device__ int g_device_status = 0;

__device__ __forceinline__ void record_status(int code) {
    atomicCAS(&g_device_status, 0, code);
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <> __device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

// Two fp32 values rounded to nearest even into a packed pair of the 16-bit
// type T (bf16 or fp16), `lo` in the low half.
template <typename T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// The packed pair of 16-bit values in `w` as two fp32 values (exact).
template <typename T> __device__ __forceinline__ float2 unpack2(uint32_t w);
template <> __device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
template <> __device__ __forceinline__ float2 unpack2<__half>(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the previous kernel of its stream is still
// running; it calls pdl_wait() before its first global-memory access, which
// returns once that kernel has completed and its writes are visible.
// pdl_launch_dependents() lets the next kernel of the stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 2^x on the MUFU unit (PTX ex2.approx, flush-to-zero).
__device__ __forceinline__ float ex2_mufu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Load `D` consecutive elements of type T starting at `src` (16-byte aligned)
// into fp32 registers.
template <typename T, int D>
__device__ __forceinline__ void load_row_f32(const T* __restrict__ src, float (&dst)[D]) {
    if constexpr (sizeof(T) == 4) {
        const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
        for (int i = 0; i < D / 4; ++i) {
            float4 v = s4[i];
            dst[4 * i + 0] = v.x; dst[4 * i + 1] = v.y; dst[4 * i + 2] = v.z; dst[4 * i + 3] = v.w;
        }
    } else {
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            uint4 v = s4[i];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = unpack2<T>(w[j]);
                dst[8 * i + 2 * j + 0] = f.x;
                dst[8 * i + 2 * j + 1] = f.y;
            }
        }
    }
}

// Store `D` fp32 registers as type T (round to nearest even for 16-bit types).
template <typename T, int D>
__device__ __forceinline__ void store_row(T* __restrict__ dst, const float (&src)[D]) {
    if constexpr (sizeof(T) == 4) {
        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int i = 0; i < D / 4; ++i)
            d4[i] = make_float4(src[4 * i], src[4 * i + 1], src[4 * i + 2], src[4 * i + 3]);
    } else {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = pack2<T>(src[8 * i + 2 * j], src[8 * i + 2 * j + 1]);
            d4[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace flarepp
