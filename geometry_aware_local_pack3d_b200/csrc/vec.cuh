// 16-byte vector loads/stores of E = 16 / sizeof(T) elements converted to/from float.
#pragma once

#include "common.cuh"

namespace p3d {

template <typename T> struct Vec;

template <> struct Vec<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void load(const float* p, float (&x)[4]) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  }
  __device__ __forceinline__ static void load_shared(const float* p, float (&x)[4]) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  }
  __device__ __forceinline__ static void store(float* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};

template <> struct Vec<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void unpack(const uint4 t, float (&x)[8]) {
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&x)[8]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), x);
  }
  __device__ __forceinline__ static void load_shared(const __nv_bfloat16* p, float (&x)[8]) {
    unpack(*reinterpret_cast<const uint4*>(p), x);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

}  // namespace p3d
