// Shared device helpers for the Gated Delta Rule-2 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <tuple>
#include <vector>

namespace gdr2 {

// Chunk length of the chunkwise form ("Chunkwise training and gate-aware
// backward", ainews.random.gg article: C = 64).
constexpr int kChunk = 64;

// Raises a kernel's dynamic shared-memory limit on the current device the
// first time a launch there needs it, instead of on every launch (the setting
// lasts as long as the device's context). Host only.
inline cudaError_t ensure_dynamic_smem(const void *kernel, int bytes)
{
    static std::mutex mu;
    static std::vector<std::tuple<const void *, int, int>> done;  // kernel, device, bytes
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (const auto &t : done)
        if (std::get<0>(t) == kernel && std::get<1>(t) == dev && std::get<2>(t) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.emplace_back(kernel, dev, bytes);
    return e;
}

// Token range [begin, end) of packed sequence n, with the offsets clamped to
// [0, tokens] and end >= begin, so that malformed offsets cannot move a
// kernel's reads or writes outside the token tensors.
__device__ __forceinline__ void packed_bounds(const int32_t *cu_seqlens, int64_t n, int64_t tokens,
                                              int64_t &begin, int64_t &end)
{
    int64_t s = cu_seqlens[n], e = cu_seqlens[n + 1];
    s = s < 0 ? 0 : (s > tokens ? tokens : s);
    e = e < s ? s : (e > tokens ? tokens : e);
    begin = s;
    end = e;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Loads `N` consecutive elements (N in {1,2,4,8}) as fp32; the address must be
// aligned to N elements.
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T *p, float (&out)[N]);

template <>
__device__ __forceinline__ void load_vec<float, 4>(const float *p, float (&o)[4]) {
    float4 v = *reinterpret_cast<const float4 *>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
template <>
__device__ __forceinline__ void load_vec<float, 2>(const float *p, float (&o)[2]) {
    float2 v = *reinterpret_cast<const float2 *>(p);
    o[0] = v.x; o[1] = v.y;
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 4>(const __nv_bfloat16 *p, float (&o)[4]) {
    uint2 raw = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    o[0] = fa.x; o[1] = fa.y; o[2] = fb.x; o[3] = fb.y;
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 2>(const __nv_bfloat16 *p, float (&o)[2]) {
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(p);
    float2 fa = __bfloat1622float2(a);
    o[0] = fa.x; o[1] = fa.y;
}

}  // namespace gdr2
