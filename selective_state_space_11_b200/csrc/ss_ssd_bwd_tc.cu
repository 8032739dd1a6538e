// ss_ssd_bwd_tc.cu -- the chunk maps of the Mamba-2 SSD backward on the
// sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Mamba" (stanleyjacob.dev), Part V, "Deep dive: Mamba-2 and state-space
// duality" (the forward) and Part IV Stage 7 (the backward of the scan): the
// state and the adjoint cross a chunk boundary through two linear maps per
// (batch b, head h, chunk k), with lc_t = A_h sum_{s<=t} Delta_s inside the chunk:
//   U_k[p][n] = sum_u e^{lc_end - lc_u} Delta_u x_u[p] B_u[n]    (the state the chunk adds)
//   V_k[p][n] = sum_t e^{lc_t} dout_t[p] C_t[n],  dout = dy SiLU(z)  (the adjoint it adds)
// and the chunk decay e^{lc_end}.  Both maps are (B^T Xw)^T-shaped products:
// with Xw[u][p] = e^{lc_end - lc_u} Delta_u x_u[p] and Dw[t][p] = e^{lc_t} dout_t[p],
//   U^T = B^T Xw,  V^T = C^T Dw      (M = dstate, N = headdim, K = 64 steps).
// One CTA of 4 warps per chunk: thread 0 TMA-loads x, dy, z, B and C as
// 128-byte-swizzled [t][.] tiles, the threads scale x and dout in place (bf16
// or fp16 operands), thread 0 issues the two products (kind::f16, fp32
// accumulation) into TMEM columns [0, 64) and [64, 128), and each thread
// stores its accumulator row (state row n) as column n of the fp32 [p][n]
// slabs that the pass over the chunks reads.  Waits are bounded; a timeout
// sets a bit in the device fault word and the CTA drains and exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstring>
#include <type_traits>

#include "ss_device.cuh"
#include "ss_ssd_bwd.h"
#include "ss_tc.cuh"

namespace ss {

__device__ unsigned int g_tc_fault_bwd = 0;

namespace {

constexpr int kQ = 64, kP = 64, kThreads = 128;
constexpr uint32_t kTmemCols = 128, kR0 = 0, kR1 = 64;
constexpr uint32_t kWaitLimit = 1u << 22;

// Byte offsets in the 1024-aligned block (sized for dstate 128 in both
// variants, which also keeps TMEM to 3 CTAs x 128 columns per SM).
struct MapLay {
  static constexpr int kX = 0;            // x, then Xw        [t][p]
  static constexpr int kDy = 8192;        // dy, then Dw       [t][p]
  static constexpr int kZ = 16384;        // z                 [t][p]
  static constexpr int kB = 24576;        // B  [t][n], 64-wide n blocks 8 KB apart
  static constexpr int kC = kB + 16384;   // C
  static constexpr int kWu = kC + 16384;  // float e^{lc_end - lc_u} Delta_u
  static constexpr int kEl = kWu + 256;   // float e^{lc_t}
  static constexpr int kBars = kEl + 256; // 2 mbarriers: copies, products
  static constexpr int kSlot = kBars + 16;
  static constexpr int kBytes = kSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

template <typename T> struct Pk;
template <> struct Pk<__nv_bfloat16> {
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __device__ __forceinline__ static float2 unpack(uint32_t w) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w));
  }
};
template <> struct Pk<__half> {
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __device__ __forceinline__ static float2 unpack(uint32_t w) {
    return __half22float2(*reinterpret_cast<__half2*>(&w));
  }
};

__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

template <typename T, int N>
__global__ void __launch_bounds__(kThreads, 3)
    ssd_maps_tc_kernel(const SsdBwdParams p, const __grid_constant__ CUtensorMap map_x,
                       const __grid_constant__ CUtensorMap map_dy, const __grid_constant__ CUtensorMap map_z,
                       const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_c) {
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kId = tc::idesc_f16(kBf16, N, 64, true, true);  // B^T Xw, C^T Dw
  constexpr int HP = N == 128 ? 64 : 32;                             // map columns (p) per thread
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc::saddr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* const sm = smem_raw + pad;
  const uint32_t sb = raw + pad;
  float* const swu = reinterpret_cast<float*>(sm + MapLay::kWu);
  float* const sel = reinterpret_cast<float*>(sm + MapLay::kEl);
  uint32_t* const sslot = reinterpret_cast<uint32_t*>(sm + MapLay::kSlot);
  const uint32_t bar_ld = sb + MapLay::kBars, bar_mma = bar_ld + 8;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = 16 * warp + (lane & 15), hx = lane >> 4;
  const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
  const int k = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int L = p.seqlen, nh = p.nheads, ng = p.ngroups, g = h / (nh / ng);
  const int t0 = k * kQ, nval = min(kQ, L - t0);
  const bool gate = p.z != nullptr;

  if (tid == 0) {
    tc::mbar_init(bar_ld, 1);
    tc::mbar_init(bar_mma, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(tc::saddr(sslot), kTmemCols);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *sslot;

  if (tid == 0) {
    tc::expect_tx(bar_ld, (gate ? 3 : 2) * 8192 + 2 * N * 128);
    tc::tma_load_4d(sb + MapLay::kX, &map_x, 0, h, t0, b, bar_ld);
    tc::tma_load_4d(sb + MapLay::kDy, &map_dy, 0, h, t0, b, bar_ld);
    if (gate) tc::tma_load_4d(sb + MapLay::kZ, &map_z, 0, h, t0, b, bar_ld);
#pragma unroll
    for (int nb = 0; nb < N / 64; ++nb) {
      tc::tma_load_4d(sb + MapLay::kB + nb * 8192, &map_b, 64 * nb, g, t0, b, bar_ld);
      tc::tma_load_4d(sb + MapLay::kC + nb * 8192, &map_c, 64 * nb, g, t0, b, bar_ld);
    }
  }
  // Delta and lc (log2 units) of the chunk: warp 3, two steps per lane
  if (warp == 3) {
    const T* dtg = static_cast<const T*>(p.dt) + (static_cast<size_t>(b) * L + t0) * nh + h;
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
    const float A2 = p.A[h] * kLog2e;
    float d2[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      float v = 0.f;
      if (t < nval) {
        const float xv = Elt<T>::to_f(dtg[static_cast<size_t>(t) * nh]) + bias;
        v = p.softplus ? softplus_f(xv) : xv;
      }
      d2[e] = v;
    }
    const float own = (d2[0] + d2[1]) * A2;
    float run = own;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float o = __shfl_up_sync(0xffffffffu, run, off);
      if (lane >= off) run += o;
    }
    const float lc0 = run - own + d2[0] * A2, lc1 = run;
    const float lend = __shfl_sync(0xffffffffu, run, 31);
    swu[2 * lane] = ex2(lend - lc0) * d2[0];
    swu[2 * lane + 1] = ex2(lend - lc1) * d2[1];
    sel[2 * lane] = ex2(lc0);
    sel[2 * lane + 1] = ex2(lc1);
    if (lane == 31) p.dec[(static_cast<size_t>(b) * nh + h) * p.nchunk + k] = ex2(lend);
  }
  bool ok = tc::wait(bar_ld, 0, kWaitLimit);
  if (!ok) atomicOr(&g_tc_fault_bwd, 1u);
  const bool fail1 = __syncthreads_or(!ok);  // weights visible, tiles landed

  if (!fail1) {
    // Xw = x e^{lc_end - lc_r} Delta_r and Dw = dout e^{lc_r}, row r, pieces 4 hx .. +3, in place
    const float wu = swu[r], el = sel[r];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t o = swz(r, 4 * hx + c);
      uint4& xv = *reinterpret_cast<uint4*>(sm + MapLay::kX + o);
      uint4& dv = *reinterpret_cast<uint4*>(sm + MapLay::kDy + o);
      const uint4 zv = gate ? *reinterpret_cast<const uint4*>(sm + MapLay::kZ + o) : make_uint4(0u, 0u, 0u, 0u);
      uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
      const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 x2 = Pk<T>::unpack(xw[i]);
        float2 d2 = Pk<T>::unpack(dw[i]);
        if (gate) {
          const float2 z2 = Pk<T>::unpack(zw[i]);
          d2.x *= z2.x * sigmoid_f(z2.x);
          d2.y *= z2.y * sigmoid_f(z2.y);
        }
        xw[i] = Pk<T>::pack(x2.x * wu, x2.y * wu);
        dw[i] = Pk<T>::pack(d2.x * el, d2.y * el);
      }
      xv = make_uint4(xw[0], xw[1], xw[2], xw[3]);
      dv = make_uint4(dw[0], dw[1], dw[2], dw[3]);
    }
    tc::fence_proxy_async();
  }
  const bool fail2 = __syncthreads_or(fail1);

  if (!fail2 && tid == 0) {
    tc::fence_after();
    const uint64_t db = tc::desc_sw128(sb + MapLay::kB, 8192, 1024);
    const uint64_t dc = tc::desc_sw128(sb + MapLay::kC, 8192, 1024);
    const uint64_t dx = tc::desc_sw128(sb + MapLay::kX, 8192, 1024);
    const uint64_t dd = tc::desc_sw128(sb + MapLay::kDy, 8192, 1024);
#pragma unroll
    for (int kk = 0; kk < kQ / 16; ++kk) tc::mma(tmem + kR0, db + kk * 128, dx + kk * 128, kId, kk > 0);
#pragma unroll
    for (int kk = 0; kk < kQ / 16; ++kk) tc::mma(tmem + kR1, dc + kk * 128, dd + kk * 128, kId, kk > 0);
    tc::commit(bar_mma);
  }
  if (!fail2) {
    ok = tc::wait(bar_mma, 0, kWaitLimit);
    if (!ok) atomicOr(&g_tc_fault_bwd, 2u);
    tc::fence_after();
    if (ok) {
      // accumulator row n = state row n: column n of the [p][n] slabs
      const size_t slab = ((static_cast<size_t>(b) * nh + h) * p.nchunk + k) * static_cast<size_t>(kP * N);
      const int n = N == 128 ? tid : r;
      const int p0 = N == 128 ? 0 : 32 * hx;
      float* su = p.su + slab + n;
      float* gv = p.gv + slab + n;
      if constexpr (N == 128) {
#pragma unroll
        for (int c0 = 0; c0 < HP; c0 += 16) {
          float u[16], v[16];
          tc::ld32x32b_x16(tmem + lane_base + kR0 + c0, u);
          tc::ld32x32b_x16(tmem + lane_base + kR1 + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            su[static_cast<size_t>(p0 + c0 + i) * N] = u[i];
            gv[static_cast<size_t>(p0 + c0 + i) * N] = v[i];
          }
        }
      } else {
        float u[32], v[32];
        tc::ld16x32bx2_x32(tmem + lane_base + kR0, u);
        tc::ld16x32bx2_x32(tmem + lane_base + kR1, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          su[static_cast<size_t>(p0 + i) * N] = u[i];
          gv[static_cast<size_t>(p0 + i) * N] = v[i];
        }
      }
    }
  } else if (tid == 0) {
    // copies may still be in flight after a failed wait: drain them (bounded)
    if (!tc::wait(bar_ld, 0, kWaitLimit)) atomicOr(&g_tc_fault_bwd, 4u);
  }
  if (!fail2 && tid == 0 && !tc::wait(bar_mma, 0, kWaitLimit)) atomicOr(&g_tc_fault_bwd, 4u);
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <typename T, int N>
cudaError_t launch_maps(const SsdBwdParams& p, cudaStream_t s) {
  constexpr bool bf = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap mx, mdy, mz, mb, mc;
  std::memset(&mz, 0, sizeof(mz));
  if (!tc::encode_rows(&mx, bf, p.x, kP, p.nheads, p.seqlen, p.batch) ||
      !tc::encode_rows(&mdy, bf, p.dy, kP, p.nheads, p.seqlen, p.batch) ||
      (p.z && !tc::encode_rows(&mz, bf, p.z, kP, p.nheads, p.seqlen, p.batch)) ||
      !tc::encode_rows(&mb, bf, p.B, N, p.ngroups, p.seqlen, p.batch) ||
      !tc::encode_rows(&mc, bf, p.C, N, p.ngroups, p.seqlen, p.batch))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(ssd_maps_tc_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       MapLay::kAlloc);
  if (e != cudaSuccess) return e;
  ssd_maps_tc_kernel<T, N><<<dim3(p.nchunk, p.nheads, p.batch), kThreads, MapLay::kAlloc, s>>>(p, mx, mdy, mz,
                                                                                               mb, mc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ssd_maps_tc(const SsdBwdParams& p, DType dt, cudaStream_t s) {
  if (p.headdim != kP || (p.dstate != 64 && p.dstate != 128)) return cudaErrorInvalidValue;
  switch (dt) {
    case DType::BF16:
      return p.dstate == 64 ? launch_maps<__nv_bfloat16, 64>(p, s) : launch_maps<__nv_bfloat16, 128>(p, s);
    case DType::F16:
      return p.dstate == 64 ? launch_maps<__half, 64>(p, s) : launch_maps<__half, 128>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t read_tc_fault_bwd(unsigned* bits, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_tc_fault_bwd, sizeof(unsigned));
  if (e != cudaSuccess || !clear) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_tc_fault_bwd, &zero, sizeof(unsigned));
}

}  // namespace ss
