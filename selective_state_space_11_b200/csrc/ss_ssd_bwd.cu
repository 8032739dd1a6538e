// ss_ssd_bwd.cu -- Mamba-2 SSD backward for sm_100a: the chunked adjoint.
//
// "Mamba" (stanleyjacob.dev), Part V, "Deep dive: Mamba-2 and state-space
// duality" gives the forward: per (batch b, head h) with scalar A_h and the
// B, C of the head's group,
//   H_t = a_t H_{t-1} + Delta_t x_t B_t^T,  a_t = exp(Delta_t A_h),   H: P x N
//   y_t = (H_t C_t + D_h x_t) SiLU(z_t).
// Its gradient ("Mamba", Part IV Stage 7: the backward of the scan) is taken
// here chunk by chunk.  Inside a chunk of Q = 64 steps let lc_t = A_h sum_{s<=t}
// Delta_s, so that H_t = e^{lc_t} S0 + sum_{s<=t} e^{lc_t - lc_s} Delta_s x_s B_s^T
// with S0 the state entering the chunk, and let Gc = dL/dH at the chunk's last
// step from the later chunks.  With dout_t = dy_t SiLU(z_t):
//   G_t B_t = sum_{s>=t} e^{lc_s - lc_t} (C_s.B_t) dout_s + e^{lc_end - lc_t} Gc B_t
//   dx_t    = Delta_t G_t B_t + D_h dout_t
//   dB_t   += Delta_t [sum_{s>=t} e^{lc_s - lc_t} (dout_s.x_t) C_s + e^{lc_end - lc_t} Gc^T x_t]
//   dC_t   += sum_{s<=t} e^{lc_t - lc_s} Delta_s (dout_t.x_s) B_s + e^{lc_t} S0^T dout_t
//   dz_t    = dy_t (H_t C_t + D_h x_t) sigma(z_t) (1 + z_t (1 - sigma(z_t)))
// and the gradient through the decays goes by dl_t = dL/dlc_t: every factor
// e^{lc_i - lc_j} of the loss adds its term to dl_i and takes it from dl_j;
// the loss terms are the read-outs (intra-chunk and through S0) and
// <Gc, S_end>.  Then dDelta_s = x_s.(G_s B_s) + A_h sum_{t>=s} dl_t and
// dA_h = sum_s Delta_s sum_{t>=s} dl_t.
//
// Between chunks the state and the adjoint obey linear recurrences
//   S_{k+1} = e^{lc_end,k} S_k + U_k,   U_k = sum_u e^{lc_end - lc_u} Delta_u x_u B_u^T
//   dS0_k   = e^{lc_end,k} Gc_k + V_k,  V_k = sum_t e^{lc_t} dout_t C_t^T,  Gc_{k-1} = dS0_k
// so the work splits into three launches: the chunk maps U_k, V_k (one block
// per chunk), a pass over the chunks per state element that turns them into
// S_k and Gc_k in place (and dh0), and the gradient of every chunk (one block
// per chunk).  dB, dC are kept per head and summed over the group's heads, and
// dA, dD, ddt_bias per chunk, in fixed order afterwards: no atomics, results
// are bitwise reproducible.
//
// The contractions inside a chunk run on the tensor cores as warp-level tf32
// MMAs (m16n8k8, fp32 accumulation) whose operands are read from fp32
// shared-memory tiles; each of the 8 warps owns a 16-row slab of a product's
// output.  Rows are 4 banks apart (stride 64 + 4 or N + 4), so the 8 rows x 4
// columns of a fragment load hit distinct banks.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "ss_device.cuh"
#include "ss_ssd_bwd.h"

namespace ss {
namespace {

constexpr int kQ = 64;      // chunk length
constexpr int kP = 64;      // head dimension
constexpr int kT = 256;     // threads per block
constexpr int kS = kQ + 4;  // row stride of the 64-wide tiles

size_t round_up256(size_t x) { return (x + 255) / 256 * 256; }

// An fp32 value as a tf32 MMA operand: the MMA reads the sign, the exponent
// and the top 10 mantissa bits of the register (truncation; relative error
// below 2^-10, well inside the bf16 inputs' own 2^-8).
__device__ __forceinline__ uint32_t tf32(float x) { return __float_as_uint(x); }

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc += A B for the warp's 16 x 8NT output tile at (r0, c0), with A(r, k) =
// fa(r, k), B(k, n) = fb(k, n), k < K.  In an m16n8k8 fragment lane 4g + q holds
// A(g or g+8, q or q+4), B(q or q+4, g) and D(g or g+8, 2q or 2q+1).
// The k-loop is unrolled UNROLL times (default: fully).
template <int NT, int K, int UNROLL = K / 8, typename FA, typename FB>
__device__ __forceinline__ void wmma(float (&acc)[NT][4], int r0, int c0, FA fa, FB fb) {
  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll UNROLL
  for (int k0 = 0; k0 < K; k0 += 8) {
    uint32_t a[4];
    a[0] = tf32(fa(r0 + g, k0 + q));
    a[1] = tf32(fa(r0 + g + 8, k0 + q));
    a[2] = tf32(fa(r0 + g, k0 + q + 4));
    a[3] = tf32(fa(r0 + g + 8, k0 + q + 4));
#pragma unroll
    for (int j = 0; j < NT; ++j)
      mma_tf32(acc[j], a, tf32(fb(k0 + q, c0 + 8 * j + g)), tf32(fb(k0 + q + 4, c0 + 8 * j + g)));
  }
}

template <int NT>
__device__ __forceinline__ void zero(float (&acc)[NT][4]) {
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
}

// f(row, col, v0, v1) for each pair of adjacent outputs (col even) of the warp's tile.
template <int NT, typename F>
__device__ __forceinline__ void each2(const float (&acc)[NT][4], int r0, int c0, F f) {
  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    f(r0 + g, c0 + 8 * j + 2 * q, acc[j][0], acc[j][1]);
    f(r0 + g + 8, c0 + 8 * j + 2 * q, acc[j][2], acc[j][3]);
  }
}

// Delta_t (zero past the sequence end), v_t = dt_t + bias, and the cumulative
// log2 decay lc_t = log2(e) A_h sum_{s<=t} Delta_s of one chunk.  dtg points at
// the chunk's first dt of this (b, h); consecutive steps are nh apart.  Ends
// with a block barrier.
template <typename T>
__device__ __forceinline__ void chunk_delta(const T* dtg, int nh, int nval, float bias, int softplus,
                                            float al2, float* dlt, float* lc, float* vv) {
  const int tid = threadIdx.x;
  if (tid < kQ) {
    float v = 0.f, d = 0.f;
    if (tid < nval) {
      v = Elt<T>::to_f(dtg[(size_t)tid * nh]) + bias;
      d = softplus ? softplus_f(v) : v;
    }
    dlt[tid] = d;
    if (vv) vv[tid] = v;
  }
  __syncthreads();
  if (tid < 32) {
    float a0 = dlt[tid] * al2, a1 = dlt[tid + 32] * al2;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u0 = __shfl_up_sync(0xffffffffu, a0, o), u1 = __shfl_up_sync(0xffffffffu, a1, o);
      if (tid >= o) {
        a0 += u0;
        a1 += u1;
      }
    }
    const float tot = __shfl_sync(0xffffffffu, a0, 31);
    lc[tid] = a0;
    lc[tid + 32] = a1 + tot;
  }
  __syncthreads();
}

// 16-byte loads of 8 storage elements, issued together before any is used
__device__ __forceinline__ uint4 ld16(const void* p) { return __ldg(static_cast<const uint4*>(p)); }

template <typename T> struct Pair;
template <> struct Pair<__nv_bfloat16> {
  __device__ __forceinline__ static float2 f(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
};
template <> struct Pair<__half> {
  __device__ __forceinline__ static float2 f(uint32_t w) {
    __half2 h;
    memcpy(&h, &w, sizeof(h));
    return __half22float2(h);
  }
};

template <typename T>
__device__ __forceinline__ void unpack8(const uint4& r, float (&v)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = Pair<T>::f(w[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// Stage the chunk's x, dout = dy SiLU(z) and (when gdz) the dz factor
// dy sigma(z)(1 + z(1 - sigma(z))) as fp32 [t][p] tiles (row stride kS), and
// its B, C as [t][n] tiles (row stride SN); zero past the sequence end.
// Returns this thread's share of sum x dout.
template <typename T, int N, int SN>
__device__ __forceinline__ float stage_chunk(const T* xg, const T* dyg, const T* zg, const T* bg,
                                             const T* cg, size_t xrow, size_t brow, int nval, float* sx,
                                             float* so, float* sdz, float* sb, float* sc) {
  constexpr int XI = kQ * kP / 8 / kT, BI = kQ * N / 8 / kT;
  const int tid = threadIdx.x;
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
  uint4 xr[XI], yr[XI], zr[XI], br[BI], cr[BI];
#pragma unroll
  for (int i = 0; i < XI; ++i) {
    const int e = (tid + i * kT) * 8, t = e / kP, pp = e % kP;
    const size_t o = (size_t)t * xrow + pp;
    const bool ok = t < nval;
    xr[i] = ok ? ld16(xg + o) : z4;
    yr[i] = ok ? ld16(dyg + o) : z4;
    zr[i] = (ok && zg) ? ld16(zg + o) : z4;
  }
#pragma unroll
  for (int i = 0; i < BI; ++i) {
    const int e = (tid + i * kT) * 8, t = e / N, n = e % N;
    const size_t o = (size_t)t * brow + n;
    const bool ok = t < nval;
    br[i] = ok ? ld16(bg + o) : z4;
    cr[i] = ok ? ld16(cg + o) : z4;
  }
  float dd = 0.f;
#pragma unroll
  for (int i = 0; i < XI; ++i) {
    const int e = (tid + i * kT) * 8, t = e / kP, pp = e % kP;
    float xv[8], dy[8], zv[8], ov[8], fz[8];
    unpack8<T>(xr[i], xv);
    unpack8<T>(yr[i], dy);
    unpack8<T>(zr[i], zv);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      if (zg) {
        const float sg = sigmoid_f(zv[v]);
        ov[v] = dy[v] * zv[v] * sg;
        fz[v] = dy[v] * sg * (1.f + zv[v] * (1.f - sg));
      } else {
        ov[v] = dy[v];
        fz[v] = 0.f;
      }
      dd = fmaf(xv[v], ov[v], dd);
    }
    float* px = sx + t * kS + pp;
    float* po = so + t * kS + pp;
    reinterpret_cast<float4*>(px)[0] = make_float4(xv[0], xv[1], xv[2], xv[3]);
    reinterpret_cast<float4*>(px)[1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
    reinterpret_cast<float4*>(po)[0] = make_float4(ov[0], ov[1], ov[2], ov[3]);
    reinterpret_cast<float4*>(po)[1] = make_float4(ov[4], ov[5], ov[6], ov[7]);
    if (sdz) {
      float* pz = sdz + t * kS + pp;
      reinterpret_cast<float4*>(pz)[0] = make_float4(fz[0], fz[1], fz[2], fz[3]);
      reinterpret_cast<float4*>(pz)[1] = make_float4(fz[4], fz[5], fz[6], fz[7]);
    }
  }
#pragma unroll
  for (int i = 0; i < BI; ++i) {
    const int e = (tid + i * kT) * 8, t = e / N, n = e % N;
    float bv[8], cv[8];
    unpack8<T>(br[i], bv);
    unpack8<T>(cr[i], cv);
    float* pb = sb + t * SN + n;
    float* pc = sc + t * SN + n;
    reinterpret_cast<float4*>(pb)[0] = make_float4(bv[0], bv[1], bv[2], bv[3]);
    reinterpret_cast<float4*>(pb)[1] = make_float4(bv[4], bv[5], bv[6], bv[7]);
    reinterpret_cast<float4*>(pc)[0] = make_float4(cv[0], cv[1], cv[2], cv[3]);
    reinterpret_cast<float4*>(pc)[1] = make_float4(cv[4], cv[5], cv[6], cv[7]);
  }
  return dd;
}

// Copy a (64 x N) fp32 state slab from global memory into a [p][n] tile of row
// stride SN (16-byte loads, all issued first); with acc, also return this
// thread's share of <old tile, new slab>.
template <int N, int SN, bool DOT>
__device__ __forceinline__ float stage_state(float* dst, const float* src) {
  constexpr int SI = kP * N / 4 / kT;
  const int tid = threadIdx.x;
  float4 r[SI];
#pragma unroll
  for (int i = 0; i < SI; ++i) r[i] = __ldg(reinterpret_cast<const float4*>(src) + tid + i * kT);
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < SI; ++i) {
    const int e = (tid + i * kT) * 4;
    float4* d = reinterpret_cast<float4*>(dst + (e / N) * SN + e % N);
    if (DOT) {
      const float4 o = *d;
      dot = fmaf(o.x, r[i].x, fmaf(o.y, r[i].y, fmaf(o.z, r[i].z, fmaf(o.w, r[i].w, dot))));
    }
    *d = r[i];
  }
  return dot;
}

// ------------------------------------------------------------ chunk maps -----
template <int N>
struct MapSm {
  static constexpr int SN = N + 4;
  static constexpr int XW = 0;              // x                              [u][p]
  static constexpr int DW = XW + kQ * kS;   // dout                           [t][p]
  static constexpr int BS = DW + kQ * kS;   // B                              [t][n]
  static constexpr int CS = BS + kQ * SN;   // C                              [t][n]
  static constexpr int DLT = CS + kQ * SN;
  static constexpr int LC = DLT + kQ;
  static constexpr int WU = LC + kQ;        // e^{lc_end - lc_u} Delta_u
  static constexpr int EL = WU + kQ;        // e^{lc_t}
  static constexpr int TOTAL = EL + kQ;
};

template <typename T, int N>
__global__ void __launch_bounds__(kT, 2) ssd_maps_kernel(const SsdBwdParams p) {
  using M = MapSm<N>;
  constexpr int SN = M::SN, NTN = N / 16;
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int k = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int L = p.seqlen, nh = p.nheads, ng = p.ngroups, g = h / (nh / ng);
  const int t0 = k * kQ, nval = min(kQ, L - t0);
  const size_t xrow = (size_t)nh * kP, brow = (size_t)ng * N;
  const size_t xo0 = ((size_t)b * L + t0) * xrow + (size_t)h * kP;
  const T* xg = static_cast<const T*>(p.x) + xo0;
  const T* dyg = static_cast<const T*>(p.dy) + xo0;
  const T* zg = p.z ? static_cast<const T*>(p.z) + xo0 : nullptr;
  const size_t bo0 = ((size_t)b * L + t0) * brow + (size_t)g * N;
  const T* bg = static_cast<const T*>(p.B) + bo0;
  const T* cg = static_cast<const T*>(p.C) + bo0;
  const T* dtg = static_cast<const T*>(p.dt) + ((size_t)b * L + t0) * nh + h;
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;

  chunk_delta<T>(dtg, nh, nval, bias, p.softplus, p.A[h] * kLog2e, sm + M::DLT, sm + M::LC, nullptr);
  const float* dlt = sm + M::DLT;
  const float* lc = sm + M::LC;
  const float lend = lc[kQ - 1];
  if (tid < kQ) {
    sm[M::WU + tid] = ex2(lend - lc[tid]) * dlt[tid];
    sm[M::EL + tid] = ex2(lc[tid]);
  }
  stage_chunk<T, N, SN>(xg, dyg, zg, bg, cg, xrow, brow, nval, sm + M::XW, sm + M::DW, nullptr, sm + M::BS,
                        sm + M::CS);
  __syncthreads();

  // U[p][n] = sum_u WU_u x_u[p] B_u[n], V[p][n] = sum_t EL_t dout_t[p] C_t[n]: warp w owns
  // rows 16 (w % 4) .. + 16 and columns (N / 2)(w / 4) .. + N / 2
  const size_t slab = (((size_t)b * nh + h) * p.nchunk + k) * (size_t)(kP * N);
  const int wr = 16 * (warp & 3), wc = (N / 2) * (warp >> 2);
  float acc[NTN][4];
  zero(acc);
  wmma<NTN, kQ, 2>(acc, wr, wc, [&](int r, int u) { return sm[M::XW + u * kS + r] * sm[M::WU + u]; },
                [&](int u, int n) { return sm[M::BS + u * SN + n]; });
  each2(acc, wr, wc, [&](int r, int c, float v0, float v1) {
    *reinterpret_cast<float2*>(p.su + slab + (size_t)r * N + c) = make_float2(v0, v1);
  });
  zero(acc);
  wmma<NTN, kQ, 2>(acc, wr, wc, [&](int r, int t) { return sm[M::DW + t * kS + r] * sm[M::EL + t]; },
                [&](int t, int n) { return sm[M::CS + t * SN + n]; });
  each2(acc, wr, wc, [&](int r, int c, float v0, float v1) {
    *reinterpret_cast<float2*>(p.gv + slab + (size_t)r * N + c) = make_float2(v0, v1);
  });
  if (tid == 0) p.dec[((size_t)b * nh + h) * p.nchunk + k] = ex2(lend);
}

// --------------------------------------------------- pass over the chunks -----
// One thread per 4 consecutive state elements of a (b, h): forwards, U_k -> S_k
// (the state entering chunk k) in place; backwards, V_k -> Gc_k (the adjoint
// at chunk k's last step) in place; the adjoint left over is dh0.  The
// 16-byte loads of kPassDepth chunks are issued before their stores.
constexpr int kPassDepth = 16;
__device__ __forceinline__ float4 fma4(float d, const float4& s, const float4& u) {
  return make_float4(fmaf(d, s.x, u.x), fmaf(d, s.y, u.y), fmaf(d, s.z, u.z), fmaf(d, s.w, u.w));
}

__global__ void __launch_bounds__(256) ssd_pass_kernel(const SsdBwdParams p, int pn4) {
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (size_t)p.batch * p.nheads * pn4) return;
  const size_t bh = idx / pn4, e = idx % pn4;
  const int K = p.nchunk;
  const float* dec = p.dec + bh * K;
  float4* su = reinterpret_cast<float4*>(p.su) + bh * K * pn4 + e;
  float4* gv = reinterpret_cast<float4*>(p.gv) + bh * K * pn4 + e;
  const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 s = p.h0 ? reinterpret_cast<const float4*>(p.h0)[idx] : zero4;
  for (int k0 = 0; k0 < K; k0 += kPassDepth) {
    float4 u[kPassDepth];
    float d[kPassDepth];
#pragma unroll
    for (int j = 0; j < kPassDepth; ++j)
      if (k0 + j < K) {
        u[j] = su[(size_t)(k0 + j) * pn4];
        d[j] = dec[k0 + j];
      }
#pragma unroll
    for (int j = 0; j < kPassDepth; ++j)
      if (k0 + j < K) {
        su[(size_t)(k0 + j) * pn4] = s;
        s = fma4(d[j], s, u[j]);
      }
  }
  float4 gacc = p.dfinal ? reinterpret_cast<const float4*>(p.dfinal)[idx] : zero4;
  for (int k1 = K - 1; k1 >= 0; k1 -= kPassDepth) {
    float4 v[kPassDepth];
    float d[kPassDepth];
#pragma unroll
    for (int j = 0; j < kPassDepth; ++j)
      if (k1 - j >= 0) {
        v[j] = gv[(size_t)(k1 - j) * pn4];
        d[j] = dec[k1 - j];
      }
#pragma unroll
    for (int j = 0; j < kPassDepth; ++j)
      if (k1 - j >= 0) {
        gv[(size_t)(k1 - j) * pn4] = gacc;
        gacc = fma4(d[j], gacc, v[j]);
      }
  }
  if (p.dh0) reinterpret_cast<float4*>(p.dh0)[idx] = gacc;
}

// ------------------------------------------------------ chunk gradients -----
template <int N>
struct GradSm {
  static constexpr int SN = N + 4;
  static constexpr int X = 0;               // x                              [t][p]
  static constexpr int O = X + kQ * kS;     // dout                           [t][p]
  static constexpr int CBL = O + kQ * kS;   // e^{lc_t - lc_s} C_t.B_s, s<=t  [t][s]
  static constexpr int XDL = CBL + kQ * kS; // e^{lc_t - lc_s} dout_t.x_s, s<=t; then the read-out [t][p]
  static constexpr int SC = XDL + kQ * kS;  // first the dl terms W[t][s], then (S0 C_t)_p
  static constexpr int BG = SC + kQ * kS;   // (Gc B_t)_p                     [t][p]
  static constexpr int DZF = BG + kQ * kS;  // dy sigma(z)(1 + z(1 - sigma(z)))  [t][p]
  static constexpr int BS = DZF + kQ * kS;  // B                              [t][n]
  static constexpr int CS = BS + kQ * SN;   // C                              [t][n]
  static constexpr int ST = CS + kQ * SN;   // S0, then Gc [p][n]; then G_t B_t [t][p] (stride kS)
  static constexpr int DLT = ST + kP * SN;
  static constexpr int LC = DLT + kQ;
  static constexpr int VV = LC + kQ;        // dt + bias
  static constexpr int EL = VV + kQ;        // e^{lc_t}
  static constexpr int ER = EL + kQ;        // e^{lc_end - lc_t} Delta_t
  static constexpr int RW = ER + kQ;        // row sums of W
  static constexpr int CL = RW + kQ;        // column sums of W
  static constexpr int RXGB = CL + kQ;      // x_t . (G_t B_t)
  static constexpr int ROSC = RXGB + kQ;    // dout_t . (S0 C_t)
  static constexpr int RXBG = ROSC + kQ;    // x_t . (Gc B_t)
  static constexpr int RED = RXBG + kQ;     // per-warp partial sums (2 x 8)
  static constexpr int TOTAL = RED + 16;
};

template <typename T, int N>
__global__ void __launch_bounds__(kT, 1) ssd_grad_kernel(const SsdBwdParams p) {
  using M = GradSm<N>;
  constexpr int SN = M::SN, NTN = N / 16;
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, tr = tid >> 4, tc = tid & 15;
  const int k = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int L = p.seqlen, nh = p.nheads, ng = p.ngroups, g = h / (nh / ng);
  const int t0 = k * kQ, nval = min(kQ, L - t0);
  const size_t xrow = (size_t)nh * kP, brow = (size_t)ng * N;
  const size_t xo0 = ((size_t)b * L + t0) * xrow + (size_t)h * kP;
  const T* xg = static_cast<const T*>(p.x) + xo0;
  const T* dyg = static_cast<const T*>(p.dy) + xo0;
  const T* zg = p.z ? static_cast<const T*>(p.z) + xo0 : nullptr;
  const size_t bo0 = ((size_t)b * L + t0) * brow + (size_t)g * N;
  const T* bg = static_cast<const T*>(p.B) + bo0;
  const T* cg = static_cast<const T*>(p.C) + bo0;
  const size_t dto0 = ((size_t)b * L + t0) * nh + h;
  const T* dtg = static_cast<const T*>(p.dt) + dto0;
  const float Ah = p.A[h];
  const float Dh = p.D ? p.D[h] : 0.f;
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
  const size_t slab = (((size_t)b * nh + h) * p.nchunk + k) * (size_t)(kP * N);
  // warp tiles: rows 16 (w % 4) .. + 16; columns 32 (w / 4) .. + 32 of a 64-wide
  // product, (N / 2)(w / 4) .. + N / 2 of an N-wide one
  const int wr = 16 * (warp & 3), w64 = 32 * (warp >> 2), wN = (N / 2) * (warp >> 2);
  const size_t prow = (size_t)nh * N;  // floats between time steps of the per-head dB, dC

  chunk_delta<T>(dtg, nh, nval, bias, p.softplus, Ah * kLog2e, sm + M::DLT, sm + M::LC, sm + M::VV);
  const float* dlt = sm + M::DLT;
  const float* lc = sm + M::LC;
  const float lend = lc[kQ - 1];
  if (tid < kQ) {
    sm[M::EL + tid] = ex2(lc[tid]);
    sm[M::ER + tid] = ex2(lend - lc[tid]) * dlt[tid];
  }

  // ---- stage x, dout, the dz factor, B, C and the state entering the chunk
  float dDp = stage_chunk<T, N, SN>(xg, dyg, zg, bg, cg, xrow, brow, nval, sm + M::X, sm + M::O,
                                          zg ? sm + M::DZF : nullptr, sm + M::BS, sm + M::CS);
  stage_state<N, SN, false>(sm + M::ST, p.su + slab);
  __syncthreads();

  // ---- C_t.B_s and dout_t.x_s, masked and decayed; the dl terms of the intra-chunk read-out
  {
    float cb[4][4], xd[4][4];
    zero(cb);
    zero(xd);
    wmma<4, N>(cb, wr, w64, [&](int r, int n) { return sm[M::CS + r * SN + n]; },
               [&](int n, int c) { return sm[M::BS + c * SN + n]; });
    wmma<4, kP>(xd, wr, w64, [&](int r, int q) { return sm[M::O + r * kS + q]; },
                [&](int q, int c) { return sm[M::X + c * kS + q]; });
    const int gq = lane >> 2, qq = lane & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = wr + gq + 8 * (e >> 1), s = w64 + 8 * j + 2 * qq + (e & 1);
        const float dcy = s <= t ? ex2(lc[t] - lc[s]) : 0.f;
        const float c = dcy * cb[j][e];
        sm[M::CBL + t * kS + s] = c;
        sm[M::XDL + t * kS + s] = dcy * xd[j][e];
        sm[M::SC + t * kS + s] = c * dlt[s] * xd[j][e];
      }
  }
  __syncthreads();
  {
    // row sums (s <= t) and column sums (t >= s) of W: four lanes per row or
    // column, 16 entries each, then a 4-lane reduction
    const int rc = tid >> 2, seg = tid & 3;
    float r = 0.f, c = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int m = 16 * seg + i;
      if (m <= rc) r += sm[M::SC + rc * kS + m];
      if (m >= rc) c += sm[M::SC + m * kS + rc];
    }
    r += __shfl_xor_sync(0xffffffffu, r, 1);
    c += __shfl_xor_sync(0xffffffffu, c, 1);
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    c += __shfl_xor_sync(0xffffffffu, c, 2);
    if (seg == 0) {
      sm[M::RW + rc] = r;
      sm[M::CL + rc] = c;
    }
  }
  __syncthreads();

  // ---- the entering state: (S0 C_t)_p, and this head's
  //      dC_t = e^{lc_t} S0^T dout_t + sum_{s<=t} e^{lc_t - lc_s} Delta_s (dout_t.x_s) B_s
  {
    float sc[4][4];
    zero(sc);
    wmma<4, N>(sc, wr, w64, [&](int r, int n) { return sm[M::CS + r * SN + n]; },
               [&](int n, int c) { return sm[M::ST + c * SN + n]; });
    each2(sc, wr, w64, [&](int r, int c, float v0, float v1) {
      sm[M::SC + r * kS + c] = v0;
      sm[M::SC + r * kS + c + 1] = v1;
    });
    float acc[NTN][4];
    zero(acc);
    wmma<NTN, kP>(acc, wr, wN, [&](int r, int q) { return sm[M::O + r * kS + q] * sm[M::EL + r]; },
                  [&](int q, int n) { return sm[M::ST + q * SN + n]; });
    wmma<NTN, kQ>(acc, wr, wN, [&](int r, int s) { return sm[M::XDL + r * kS + s] * dlt[s]; },
                  [&](int s, int n) { return sm[M::BS + s * SN + n]; });
    float* pdc = p.pdC + (((size_t)b * L + t0) * nh + h) * N;
    each2(acc, wr, wN, [&](int t, int n, float v0, float v1) {
      if (t < nval) *reinterpret_cast<float2*>(pdc + t * prow + n) = make_float2(v0, v1);
    });
  }
  __syncthreads();

  // ---- the adjoint leaving the chunk: <Gc, S0>, (Gc B_t)_p, and this head's
  //      dB_t = e^{lc_end - lc_t} Delta_t Gc^T x_t + Delta_t sum_{s>=t} e^{lc_s - lc_t} (dout_s.x_t) C_s
  float gs = stage_state<N, SN, true>(sm + M::ST, p.gv + slab);
  __syncthreads();
  {
    float bgv[4][4];
    zero(bgv);
    wmma<4, N>(bgv, wr, w64, [&](int r, int n) { return sm[M::BS + r * SN + n]; },
               [&](int n, int c) { return sm[M::ST + c * SN + n]; });
    each2(bgv, wr, w64, [&](int r, int c, float v0, float v1) {
      sm[M::BG + r * kS + c] = v0;
      sm[M::BG + r * kS + c + 1] = v1;
    });
    float acc[NTN][4];
    zero(acc);
    wmma<NTN, kP>(acc, wr, wN, [&](int r, int q) { return sm[M::X + r * kS + q] * sm[M::ER + r]; },
                  [&](int q, int n) { return sm[M::ST + q * SN + n]; });
    wmma<NTN, kQ>(acc, wr, wN, [&](int r, int s) { return sm[M::XDL + s * kS + r] * dlt[r]; },
                  [&](int s, int n) { return sm[M::CS + s * SN + n]; });
    float* pdb = p.pdB + (((size_t)b * L + t0) * nh + h) * N;
    each2(acc, wr, wN, [&](int t, int n, float v0, float v1) {
      if (t < nval) *reinterpret_cast<float2*>(pdb + t * prow + n) = make_float2(v0, v1);
    });
  }
  __syncthreads();

  // ---- the intra-chunk read-out (into the XDL tile) and sum_{s>=t} e^{lc_s - lc_t} (C_s.B_t) dout_s
  //      (into the state tile), both [t][p]
  {
    float yp[4][4], gb[4][4];
    zero(yp);
    zero(gb);
    wmma<4, kQ>(yp, wr, w64, [&](int r, int s) { return sm[M::CBL + r * kS + s] * dlt[s]; },
                [&](int s, int c) { return sm[M::X + s * kS + c]; });
    wmma<4, kQ>(gb, wr, w64, [&](int r, int s) { return sm[M::CBL + s * kS + r]; },
                [&](int s, int c) { return sm[M::O + s * kS + c]; });
    each2(yp, wr, w64, [&](int r, int c, float v0, float v1) {
      sm[M::XDL + r * kS + c] = v0;
      sm[M::XDL + r * kS + c + 1] = v1;
    });
    each2(gb, wr, w64, [&](int r, int c, float v0, float v1) {
      sm[M::ST + r * kS + c] = v0;
      sm[M::ST + r * kS + c + 1] = v1;
    });
  }
  __syncthreads();

  // ---- per (t, p): dx and dz, and the row sums the decay gradient needs
  {
    T* dxg = static_cast<T*>(p.dx) + xo0;
    T* dzg = (p.dz && zg) ? static_cast<T*>(p.dz) + xo0 : nullptr;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = tr + 16 * i;
      const float el = sm[M::EL + t], er = ex2(lend - lc[t]);
      float rx = 0.f, ro = 0.f, rb = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int pp = tc + 16 * j;
        const float xv = sm[M::X + t * kS + pp], ov = sm[M::O + t * kS + pp];
        const float scv = sm[M::SC + t * kS + pp], bgv = sm[M::BG + t * kS + pp];
        const float gbv = fmaf(er, bgv, sm[M::ST + t * kS + pp]);
        rx = fmaf(xv, gbv, rx);
        ro = fmaf(ov, scv, ro);
        rb = fmaf(xv, bgv, rb);
        if (t < nval) {
          const size_t o = (size_t)t * xrow + pp;
          dxg[o] = Elt<T>::from_f(fmaf(dlt[t], gbv, Dh * ov));
          if (dzg) {
            const float yv = fmaf(el, scv, sm[M::XDL + t * kS + pp]) + Dh * xv;
            dzg[o] = Elt<T>::from_f(yv * sm[M::DZF + t * kS + pp]);
          }
        }
      }
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) {
        rx += __shfl_xor_sync(0xffffffffu, rx, o);
        ro += __shfl_xor_sync(0xffffffffu, ro, o);
        rb += __shfl_xor_sync(0xffffffffu, rb, o);
      }
      if (tc == 0) {
        sm[M::RXGB + t] = rx;
        sm[M::ROSC + t] = ro;
        sm[M::RXBG + t] = rb;
      }
    }
  }

  // ---- the decay gradient dl_t, dDelta, and the per-chunk parameter partials
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    gs += __shfl_xor_sync(0xffffffffu, gs, o);
    dDp += __shfl_xor_sync(0xffffffffu, dDp, o);
  }
  if (lane == 0) {
    sm[M::RED + warp] = gs;
    sm[M::RED + 8 + warp] = dDp;
  }
  __syncthreads();
  if (warp == 0) {
    float gsum = 0.f, dsum = 0.f;
    for (int w = 0; w < kT / 32; ++w) {
      gsum += sm[M::RED + w];
      dsum += sm[M::RED + 8 + w];
    }
    float dl[2], t3 = 0.f;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int t = lane + 32 * hh;
      const float x3 = ex2(lend - lc[t]) * dlt[t] * sm[M::RXBG + t];
      dl[hh] = sm[M::RW + t] - sm[M::CL + t] + ex2(lc[t]) * sm[M::ROSC + t] - x3;
      t3 += x3;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) t3 += __shfl_xor_sync(0xffffffffu, t3, o);
    if (lane == 31) dl[1] += ex2(lend) * gsum + t3;  // the chunk end, t = 63
    // q_s = sum_{t>=s} dl_t
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u0 = __shfl_down_sync(0xffffffffu, dl[0], o), u1 = __shfl_down_sync(0xffffffffu, dl[1], o);
      if (lane + o < 32) {
        dl[0] += u0;
        dl[1] += u1;
      }
    }
    dl[0] += __shfl_sync(0xffffffffu, dl[1], 0);
    T* ddtg = static_cast<T*>(p.ddt) + dto0;
    float pa = 0.f, pb = 0.f;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int t = lane + 32 * hh;
      const float dd = fmaf(Ah, dl[hh], sm[M::RXGB + t]);
      const float dv = p.softplus ? dd * sigmoid_f(sm[M::VV + t]) : dd;
      pa = fmaf(dlt[t], dl[hh], pa);
      if (t < nval) {
        ddtg[(size_t)t * nh] = Elt<T>::from_f(dv);
        pb += dv;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      pa += __shfl_xor_sync(0xffffffffu, pa, o);
      pb += __shfl_xor_sync(0xffffffffu, pb, o);
    }
    if (lane == 0) {
      const size_t pi = ((size_t)b * nh + h) * p.nchunk + k;
      p.pA[pi] = pa;
      p.pD[pi] = dsum;
      p.pbias[pi] = pb;
    }
  }
}

// ------------------------------------------------------ fixed-order sums -----
// PT: the type of the partials (fp32 per head on the mma.sync path, fp16 per
// hpc heads on the tcgen05 path); the sum is fp32 in head order either way.
template <typename PT>
__global__ void __launch_bounds__(256) ssd_reduce_bc_kernel(const SsdBwdParams p) {
  const PT* pdB = reinterpret_cast<const PT*>(p.pdB);
  const PT* pdC = reinterpret_cast<const PT*>(p.pdC);
  const int N = p.dstate, ng = p.ngroups, nh = p.nheads / p.hpc, hpg = nh / ng;  // partials
  const size_t total = (size_t)p.batch * p.seqlen * ng * N;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const size_t bt = idx / ((size_t)ng * N);
    const int r = (int)(idx % ((size_t)ng * N)), g = r / N, n = r % N;
    const size_t base = (bt * nh + (size_t)g * hpg) * N + n;
    float sb = 0.f, sc = 0.f;
    for (int hh = 0; hh < hpg; ++hh) {
      sb += Elt<PT>::to_f(pdB[base + (size_t)hh * N]);
      sc += Elt<PT>::to_f(pdC[base + (size_t)hh * N]);
    }
    p.dB[idx] = sb;
    p.dC[idx] = sc;
  }
}

// The same sum over fp16 partials, 8 consecutive n per thread (16-byte loads).
__global__ void __launch_bounds__(256) ssd_reduce_bc8_kernel(const SsdBwdParams p) {
  const int N = p.dstate, ng = p.ngroups, nh = p.nheads / p.hpc, hpg = nh / ng;  // partials
  const size_t total8 = (size_t)p.batch * p.seqlen * ng * N / 8;
  const uint4* pdB = reinterpret_cast<const uint4*>(p.pdB);
  const uint4* pdC = reinterpret_cast<const uint4*>(p.pdC);
  for (size_t i8 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i8 < total8;
       i8 += (size_t)gridDim.x * blockDim.x) {
    const size_t idx = 8 * i8;
    const size_t bt = idx / ((size_t)ng * N);
    const int r = (int)(idx % ((size_t)ng * N)), g = r / N, n = r % N;
    const size_t base8 = ((bt * nh + (size_t)g * hpg) * N + n) / 8;
    float sb[8], sc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sb[j] = sc[j] = 0.f;
    for (int hh = 0; hh < hpg; ++hh) {
      const uint4 vb = pdB[base8 + (size_t)hh * (N / 8)], vc = pdC[base8 + (size_t)hh * (N / 8)];
      const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w}, wc[4] = {vc.x, vc.y, vc.z, vc.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&wb[j]));
        const float2 fc = __half22float2(*reinterpret_cast<const __half2*>(&wc[j]));
        sb[2 * j] += fb.x; sb[2 * j + 1] += fb.y;
        sc[2 * j] += fc.x; sc[2 * j + 1] += fc.y;
      }
    }
    float4* dB = reinterpret_cast<float4*>(p.dB + idx);
    float4* dC = reinterpret_cast<float4*>(p.dC + idx);
    dB[0] = make_float4(sb[0], sb[1], sb[2], sb[3]);
    dB[1] = make_float4(sb[4], sb[5], sb[6], sb[7]);
    dC[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
    dC[1] = make_float4(sc[4], sc[5], sc[6], sc[7]);
  }
}

__global__ void ssd_reduce_param_kernel(const SsdBwdParams p) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= p.nheads) return;
  float a = 0.f, d = 0.f, c = 0.f;
  for (int b = 0; b < p.batch; ++b) {
    const size_t base = ((size_t)b * p.nheads + h) * p.nchunk;
    for (int k = 0; k < p.nchunk; ++k) {
      a += p.pA[base + k];
      d += p.pD[base + k];
      c += p.pbias[base + k];
    }
  }
  p.dA[h] = a;
  if (p.dD) p.dD[h] = d;
  if (p.ddt_bias) p.ddt_bias[h] = c;
}

}  // namespace

int ssd_heads_per_cta(int batch, int nchunk, int nheads, int ngroups, int sms, int cap, bool force) {
  const int hpg = nheads / ngroups;
  for (int d = cap < 8 ? cap : 8; d > 1; --d) {
    if (hpg % d) continue;
    if (force || (long long)nchunk * (nheads / d) * batch >= sms) return d;
  }
  return 1;
}

namespace {

template <typename T, int N>
cudaError_t launch_ssd_bwd_n(const SsdBwdParams& p, DType dt, bool tc_maps, cudaStream_t s) {
  const size_t map_bytes = sizeof(float) * MapSm<N>::TOTAL;
  const size_t grad_bytes = sizeof(float) * GradSm<N>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(ssd_maps_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)map_bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ssd_grad_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)grad_bytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.nchunk, p.nheads, p.batch);
  if (tc_maps) {
    e = launch_ssd_maps_tc(p, dt, s);
    if (e != cudaSuccess) return e;
  } else {
    ssd_maps_kernel<T, N><<<grid, kT, map_bytes, s>>>(p);
  }
  if (tc_maps) {
    e = launch_ssd_pass16(p, s);
    if (e != cudaSuccess) return e;
  } else {
    const int pn4 = kP * N / 4;
    const size_t quads = (size_t)p.batch * p.nheads * pn4;
    ssd_pass_kernel<<<(unsigned)((quads + 255) / 256), 256, 0, s>>>(p, pn4);
  }
  if (tc_maps) {
    e = launch_ssd_grad_tc(p, dt, s);
    if (e != cudaSuccess) return e;
  } else {
    ssd_grad_kernel<T, N><<<grid, kT, grad_bytes, s>>>(p);
  }
  const size_t bc = (size_t)p.batch * p.seqlen * p.ngroups * N;
  const unsigned bc_blocks = (unsigned)std::min<size_t>((bc + 255) / 256, (size_t)148 * 64);
  // dB, dC need only 4-byte alignment: the 16-byte stores of the 8-wide sum
  // are taken when both allow them
  const bool out16 = (reinterpret_cast<uintptr_t>(p.dB) % 16 == 0) && (reinterpret_cast<uintptr_t>(p.dC) % 16 == 0);
  if (tc_maps && out16) {
    const unsigned bc8 = (unsigned)std::min<size_t>((bc / 8 + 255) / 256, (size_t)148 * 64);
    ssd_reduce_bc8_kernel<<<bc8, 256, 0, s>>>(p);
  } else if (tc_maps) {
    ssd_reduce_bc_kernel<__half><<<bc_blocks, 256, 0, s>>>(p);
  } else {
    ssd_reduce_bc_kernel<float><<<bc_blocks, 256, 0, s>>>(p);
  }
  ssd_reduce_param_kernel<<<(p.nheads + 127) / 128, 128, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ssd_bwd_t(const SsdBwdParams& p, DType dt, bool tc_maps, cudaStream_t s) {
  return p.dstate == 64 ? launch_ssd_bwd_n<T, 64>(p, dt, tc_maps, s) : launch_ssd_bwd_n<T, 128>(p, dt, tc_maps, s);
}

}  // namespace

SsdBwdLayout ssd_bwd_layout(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                            int64_t dstate) {
  const size_t nck = (size_t)(seqlen + kQ - 1) / kQ;
  const size_t maps = round_up256((size_t)batch * nheads * nck * headdim * dstate * sizeof(float));
  const size_t per_chunk = round_up256((size_t)batch * nheads * nck * sizeof(float));
  const size_t per_head = round_up256((size_t)batch * seqlen * nheads * dstate * sizeof(float));
  SsdBwdLayout l{};
  l.off_su = 0;
  l.off_gv = maps;
  l.off_dec = 2 * maps;
  l.off_pdB = l.off_dec + per_chunk;
  l.off_pdC = l.off_pdB + per_head;
  l.off_pA = l.off_pdC + per_head;
  l.off_pD = l.off_pA + per_chunk;
  l.off_pbias = l.off_pD + per_chunk;
  l.total = l.off_pbias + per_chunk;
  return l;
}

void ssd_bwd_bind(SsdBwdParams& p, void* workspace) {
  const SsdBwdLayout l = ssd_bwd_layout(p.batch, p.seqlen, p.nheads, p.headdim, p.dstate);
  unsigned char* w = static_cast<unsigned char*>(workspace);
  p.su = reinterpret_cast<float*>(w + l.off_su);
  p.gv = reinterpret_cast<float*>(w + l.off_gv);
  p.dec = reinterpret_cast<float*>(w + l.off_dec);
  p.pdB = reinterpret_cast<float*>(w + l.off_pdB);
  p.pdC = reinterpret_cast<float*>(w + l.off_pdC);
  p.pA = reinterpret_cast<float*>(w + l.off_pA);
  p.pD = reinterpret_cast<float*>(w + l.off_pD);
  p.pbias = reinterpret_cast<float*>(w + l.off_pbias);
}

cudaError_t launch_ssd_bwd(const SsdBwdParams& p, DType dt, bool tc_maps, cudaStream_t s) {
  switch (dt) {
    case DType::BF16: return launch_ssd_bwd_t<__nv_bfloat16>(p, dt, tc_maps, s);
    case DType::F16: return launch_ssd_bwd_t<__half>(p, dt, tc_maps, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ss
