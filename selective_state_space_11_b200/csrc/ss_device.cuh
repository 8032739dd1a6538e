// ss_device.cuh -- device helpers shared by the selective-scan kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ss {

constexpr int kN = 16;         // state width per channel (d_state)
constexpr int kChunk = 64;     // steps between state checkpoints
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- math -----
// 2^x on the SFU (MUFU.EX2).  Used for every decay exp(Delta*A) =
// 2^(Delta * A*log2e): A is pre-scaled by log2(e) once per channel.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(x) = log(1 + e^x).  For x > 20, e^x > 4.8e8 and log1p(e^x)
// equals x to within 2.1e-9 relative, below fp32 resolution.
__device__ __forceinline__ float softplus_f(float x) {
  return x > 20.f ? x : log1pf(ex2(x * kLog2e));
}

// logistic sigmoid 1 / (1 + e^-x); saturates cleanly at both ends.
__device__ __forceinline__ float sigmoid_f(float x) {
  return __frcp_rn(1.f + ex2(-x * kLog2e));
}

// ------------------------------------------------------------ storage -----
template <typename T> struct Elt;
template <> struct Elt<float> {
  __device__ __forceinline__ static float load(const float* p) { return __ldg(p); }
  __device__ __forceinline__ static float to_f(float v) { return v; }
  __device__ __forceinline__ static float from_f(float v) { return v; }
};
template <> struct Elt<__nv_bfloat16> {
  __device__ __forceinline__ static float load(const __nv_bfloat16* p) {
    return __bfloat162float(__ldg(p));
  }
  __device__ __forceinline__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};
template <> struct Elt<__half> {
  __device__ __forceinline__ static float load(const __half* p) { return __half2float(__ldg(p)); }
  __device__ __forceinline__ static float to_f(__half v) { return __half2float(v); }
  __device__ __forceinline__ static __half from_f(float v) { return __float2half_rn(v); }
};

// Load 8 consecutive elements from a 16-byte aligned address (one or two
// 128-bit loads), converting to fp32.
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void load8(const __half* p, float (&v)[8]) {
  const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
  const __half2* h = reinterpret_cast<const __half2*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// Store 8 consecutive fp32 values (rounded to nearest-even for 16-bit types)
// to a 16-byte aligned address.
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 r;
  uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&t);
  }
  *reinterpret_cast<uint4*>(p) = r;
}
__device__ __forceinline__ void store8(__half* p, const float (&v)[8]) {
  uint4 r;
  uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 t = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&t);
  }
  *reinterpret_cast<uint4*>(p) = r;
}

template <typename T>
__device__ __forceinline__ float ldf(const T* p) { return Elt<T>::load(p); }

template <typename T>
__device__ __forceinline__ void stf(T* p, float v) { *p = Elt<T>::from_f(v); }

// Load up to 8 consecutive elements starting at element index `t` of a row
// of length `len`.  Vector path when the row is 16-byte aligned and all 8 are
// in range; scalar (guarded) otherwise.  Out-of-range elements read as 0.
template <typename T, bool VEC>
__device__ __forceinline__ void load8_row(const T* row, int t, int len, float (&v)[8]) {
  if (VEC && t + 8 <= len) {
    load8(row + t, v);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (t + i < len) ? ldf(row + t + i) : 0.f;
  }
}

template <typename T, bool VEC>
__device__ __forceinline__ void store8_row(T* row, int t, int len, const float (&v)[8]) {
  if (VEC && t + 8 <= len) {
    store8(row + t, v);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (t + i < len) stf(row + t + i, v[i]);
  }
}

}  // namespace ss
