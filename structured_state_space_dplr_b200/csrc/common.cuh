// common.cuh -- small device helpers shared by the s4dplr kernels.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>
#include <type_traits>

namespace s4 {

// ---------------------------------------------------------------- complex --
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cscale(float2 a, float s) { return make_float2(a.x * s, a.y * s); }
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }
// a * b
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// a * conj(b)
__device__ __forceinline__ float2 cmulc(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
// a * b (DIR < 0) or a * conj(b) (DIR > 0): twiddle tables hold exp(-2 pi i e/D)
template <int DIR>
__device__ __forceinline__ float2 ctw(float2 a, float2 w) {
    if constexpr (DIR < 0) return cmul(a, w); else return cmulc(a, w);
}
// multiply by DIR*i
template <int DIR>
__device__ __forceinline__ float2 mul_i(float2 a) {
    if constexpr (DIR > 0) return make_float2(-a.y, a.x); else return make_float2(a.y, -a.x);
}

// exp(-2 pi i e / d) for 0 <= e < d (exact rational argument to sincospif)
__device__ __forceinline__ float2 unit_root(int e, int d) {
    float s, c;
    sincospif(2.0f * (float)e / (float)d, &s, &c);
    return make_float2(c, -s);
}

// compile-time loops
template <int Begin, int End, typename F>
__device__ __forceinline__ void static_for(F &&f) {
    if constexpr (Begin < End) {
        f(std::integral_constant<int, Begin>{});
        static_for<Begin + 1, End>(f);
    }
}

__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v >> 1); }

}  // namespace s4
