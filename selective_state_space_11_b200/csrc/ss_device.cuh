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
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- math -----
// 2^x on the SFU (MUFU.EX2).  Used for every decay exp(Delta*A) =
// 2^(Delta * A*log2e): A is pre-scaled by log2(e) once per channel.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 1/x on the SFU (MUFU.RCP), maximum error about 1 ulp.
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log(1 + w) for w in [0, 1] from the classical series
//   log(1 + w) = 2 atanh(s) = 2 (s + s^3/3 + s^5/5 + ...),  s = w / (2 + w),
// truncated after s^15/15: with s <= 1/3 the remainder is below 1.5e-9 of the
// result.  Costs one SFU reciprocal and eight FMAs.
__device__ __forceinline__ float log1p_unit(float w) {
  const float s = w * rcp(2.f + w);
  const float u = s * s;
  float q = fmaf(u, 1.f / 15.f, 1.f / 13.f);
  q = fmaf(u, q, 1.f / 11.f);
  q = fmaf(u, q, 1.f / 9.f);
  q = fmaf(u, q, 1.f / 7.f);
  q = fmaf(u, q, 1.f / 5.f);
  q = fmaf(u, q, 1.f / 3.f);
  q = fmaf(u, q, 1.f);
  return (2.f * s) * q;
}

// softplus(x) = log(1 + e^x) = max(x, 0) + log(1 + e^-|x|): no overflow, no
// cancellation, two SFU operations (ex2, rcp).
__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.f) + log1p_unit(ex2(-fabsf(x) * kLog2e));
}

// logistic sigmoid 1 / (1 + e^-x); saturates cleanly at both ends.
__device__ __forceinline__ float sigmoid_f(float x) {
  return rcp(1.f + ex2(-x * kLog2e));
}

// ---------------------------------------------------- packed fp32 pairs -----
// sm_100 executes two fp32 FMAs / multiplies / adds per lane in one
// instruction (fma/mul/add .rn.f32x2): the FP32 pipe does the same work in
// half the issue slots.  A pair lives in a 64-bit register (lo, hi).
typedef unsigned long long f2_t;

__device__ __forceinline__ f2_t pk2(float lo, float hi) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float lo2(f2_t v) { return __uint_as_float((unsigned)(v & 0xffffffffull)); }
__device__ __forceinline__ float hi2(f2_t v) { return __uint_as_float((unsigned)(v >> 32)); }
__device__ __forceinline__ f2_t fma2(f2_t a, f2_t b, f2_t c) {
  f2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2_t mul2(f2_t a, f2_t b) {
  f2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t add2(f2_t a, f2_t b) {
  f2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// (2^lo, 2^hi) of a pair of exponents, two SFU operations.
__device__ __forceinline__ f2_t ex2_2(f2_t e) { return pk2(ex2(lo2(e)), ex2(hi2(e))); }

// -------------------------------------------------------- seq_idx -----
// Packed documents ("seq_idx strict reset", niverel-mamba README): the state
// restarts at every change of the document id.  Bit i of the result is set
// when step t0 + i starts a new document (id differs from step t0 + i - 1),
// for t0 + i < t_end; zero without seq_idx.  Called by all 32 lanes of a
// warp, lane i inspecting step t0 + i, so every warp holds the same mask.
__device__ __forceinline__ unsigned doc_starts32(const int* seq_row, int t0, int t_end) {
  const int t = t0 + (int)(threadIdx.x & 31);
  bool f = false;
  if (seq_row && t > 0 && t < t_end) f = seq_row[t] != seq_row[t - 1];
  return __ballot_sync(0xffffffffu, f);
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialisation may start while the kernel before it in the stream still
// runs; pdl_wait() blocks until that kernel has completed and its memory
// writes are visible (a no-op in a kernel launched without the attribute).
// pdl_trigger() lets the next such kernel start launching.  Code before
// pdl_wait() reads only data no earlier kernel of the chain writes, and
// writes no global memory.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ------------------------------------------------------- async copies -----
// 16-byte global->shared copy that bypasses the register file (cp.async, .cg:
// L2 only).  Bytes past src_bytes are zero-filled, so ragged row tails never
// read past the end of a row.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, int src_bytes) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
// Wait until at most N of this thread's committed copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

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

// PS consecutive elements of a row, held in their storage format so that a
// prefetch does not wait for the data: the loads are issued one tile ahead
// and only unpacked when the tile is consumed.
template <typename T, int PS>
struct RawVec {
  static constexpr int kWords = PS * (int)sizeof(T) / 4;
  static_assert(kWords == 2 || kWords % 4 == 0, "vector width");
  uint32_t w[kWords];

  template <bool VEC>
  __device__ __forceinline__ void load(const T* row, int t, int len) {
    if (VEC && t + PS <= len) {
      const T* src = row + t;
      if (kWords == 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
        w[0] = v.x; w[1] = v.y;
      } else {
#pragma unroll
        for (int i = 0; i < kWords / 4; ++i) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
          w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
      }
    } else if constexpr (sizeof(T) == 4) {
#pragma unroll
      for (int i = 0; i < PS; ++i)
        w[i] = (t + i < len) ? __ldg(reinterpret_cast<const uint32_t*>(row) + t + i) : 0u;
    } else {
      const unsigned short* r16 = reinterpret_cast<const unsigned short*>(row);
#pragma unroll
      for (int i = 0; i < kWords; ++i) {
        const uint32_t a = (t + 2 * i < len) ? __ldg(r16 + t + 2 * i) : 0u;
        const uint32_t b = (t + 2 * i + 1 < len) ? __ldg(r16 + t + 2 * i + 1) : 0u;
        w[i] = a | (b << 16);
      }
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < kWords; ++i) w[i] = 0u;
  }
  __device__ __forceinline__ void unpack(float (&v)[PS]) const {
    const T* e = reinterpret_cast<const T*>(w);
#pragma unroll
    for (int i = 0; i < PS; ++i) v[i] = Elt<T>::to_f(e[i]);
  }
};

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
