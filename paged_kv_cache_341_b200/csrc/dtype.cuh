// Element types of the cache and their 16-byte chunk conversions to and from
// float32 pairs.  16-bit -> float32 is exact; float32 -> 16-bit rounds to
// nearest even.
#ifndef PAGEDATTN_DTYPE_CUH
#define PAGEDATTN_DTYPE_CUH

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace pa {

template <typename T>
struct Chunk;

// float32: 4 values per 16-byte chunk.
template <>
struct Chunk<float> {
  static constexpr int kElems = 4;
  __device__ __forceinline__ static void load(const void* p, float2* out) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = make_float2(v.x, v.y);
    out[1] = make_float2(v.z, v.w);
  }
  __device__ __forceinline__ static void store(void* p, const float2* in) {
    *reinterpret_cast<float4*>(p) = make_float4(in[0].x, in[0].y, in[1].x, in[1].y);
  }
};

// bfloat16: 8 values per chunk; widening is a 16-bit shift of each half word.
template <>
struct Chunk<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ __forceinline__ static float2 widen(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
  __device__ __forceinline__ static void load(const void* p, float2* out) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    out[0] = widen(v.x);
    out[1] = widen(v.y);
    out[2] = widen(v.z);
    out[3] = widen(v.w);
  }
  __device__ __forceinline__ static uint32_t narrow(float2 f) {
    __nv_bfloat162 h = __float22bfloat162_rn(f);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static void store(void* p, const float2* in) {
    *reinterpret_cast<uint4*>(p) = make_uint4(narrow(in[0]), narrow(in[1]), narrow(in[2]), narrow(in[3]));
  }
};

// float16: 8 values per chunk.
template <>
struct Chunk<__half> {
  static constexpr int kElems = 8;
  __device__ __forceinline__ static float2 widen(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
  }
  __device__ __forceinline__ static void load(const void* p, float2* out) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    out[0] = widen(v.x);
    out[1] = widen(v.y);
    out[2] = widen(v.z);
    out[3] = widen(v.w);
  }
  __device__ __forceinline__ static uint32_t narrow(float2 f) {
    __half2 h = __float22half2_rn(f);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static void store(void* p, const float2* in) {
    *reinterpret_cast<uint4*>(p) = make_uint4(narrow(in[0]), narrow(in[1]), narrow(in[2]), narrow(in[3]));
  }
};

}  // namespace pa

#endif
