// ss_ssd_bwd_tc.cu -- the chunk maps and the chunk gradients of the Mamba-2
// SSD backward on the sm_100a tensor cores (tcgen05 + TMEM + TMA); the pass
// over the chunks and the fixed-order sums between them are in ss_ssd_bwd.cu.
// The operands of every product here are fp16 (see `Op` below).
//
// The chunk maps:
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
// variants; 2 CTAs x 128 TMEM columns per SM).
struct MapLay {
  static constexpr int kX = 0;            // x, then Xw        [t][p]
  static constexpr int kDy = 8192;        // dy, then Dw       [t][p]
  static constexpr int kZ = 16384;        // z                 [t][p]
  static constexpr int kB = 24576;        // B  [t][n], 64-wide n blocks 8 KB apart
  static constexpr int kC = kB + 16384;   // C
  static constexpr int kSu = kC + 16384;  // fp16 U slab of a head, in operand-tile order (bulk-stored)
  static constexpr int kSv = kSu + 16384; // fp16 V slab
  static constexpr int kWu = kSv + 16384; // float e^{lc_end - lc_u} Delta_u
  static constexpr int kEl = kWu + 256;   // float e^{lc_t}
  static constexpr int kBars = kEl + 256; // 3 mbarriers: copies, products, drain
  static constexpr int kSlot = kBars + 32;
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

// Index (in 16-bit elements) of element (p, n) of a [64 p][N n] operand tile:
// 64-wide n blocks of 64 rows x 128 bytes, 128-byte swizzle.  The state and
// adjoint slabs of the tcgen05 path are stored in this order, so a slab is its
// operand tile as it stands.
__host__ __device__ __forceinline__ uint32_t tile_idx(int p, int n) {
  return static_cast<uint32_t>((n >> 6) * 4096 + p * 64 + ((((n & 63) >> 3) ^ (p & 7)) << 3) + (n & 7));
}

// The tensor-core operands of the backward are fp16 whatever the storage type:
// its 11-bit significand matches tf32's, where bf16's 8 bits are too coarse for
// the derived operands (dout, the decayed masks, the states) of sums that
// cancel.  bf16 inputs that are operands (x, B, C) are converted in place,
// which is exact for values in fp16's range.
using Op = __half;

// Convert `pieces` 16-byte pieces of T at `base` to Op in place, pieces
// tid, tid + nthr, ...
template <typename T>
__device__ __forceinline__ void to_op_inplace(unsigned char* base, int pieces, int tid, int nthr) {
  if constexpr (!std::is_same<T, Op>::value) {
    for (int e = tid; e < pieces; e += nthr) {
      uint4& v = *reinterpret_cast<uint4*>(base + 16 * e);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f2 = Pk<T>::unpack(w[i]);
        w[i] = Pk<Op>::pack(f2.x, f2.y);
      }
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// One CTA of 4 warps per chunk and group of hpc heads (one group of B, C),
// which it takes one after another: B and C are copied and converted to fp16
// once, each head's x, dy, z are copied in, and the head's maps U^T = B^T Xw
// and V^T = C^T Dw go out as fp16 slabs in operand-tile order by two bulk
// stores.
template <typename T, int N>
__global__ void __launch_bounds__(kThreads, 2)
    ssd_maps_tc_kernel(const SsdBwdParams p, const __grid_constant__ CUtensorMap map_x,
                       const __grid_constant__ CUtensorMap map_dy, const __grid_constant__ CUtensorMap map_z,
                       const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_c) {
  constexpr uint32_t kId = tc::idesc_f16(false, N, 64, true, true);  // B^T Xw, C^T Dw (fp16)
  constexpr int HP = N == 128 ? 64 : 32;                             // map columns (p) per thread
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc::saddr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* const sm = smem_raw + pad;
  const uint32_t sb = raw + pad;
  float* const swu = reinterpret_cast<float*>(sm + MapLay::kWu);
  float* const sel = reinterpret_cast<float*>(sm + MapLay::kEl);
  uint32_t* const sslot = reinterpret_cast<uint32_t*>(sm + MapLay::kSlot);
  const uint32_t bar_ld = sb + MapLay::kBars, bar_mma = bar_ld + 8, bar_dr = bar_ld + 16;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = 16 * warp + (lane & 15), hx = lane >> 4;
  const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
  const int k = blockIdx.x, hb = blockIdx.y * p.hpc, b = blockIdx.z;
  const int L = p.seqlen, nh = p.nheads, ng = p.ngroups, g = hb / (nh / ng);
  const int t0 = k * kQ, nval = min(kQ, L - t0);
  const bool gate = p.z != nullptr;

  if (tid == 0) {
    tc::mbar_init(bar_ld, 1);
    tc::mbar_init(bar_mma, 1);
    tc::mbar_init(bar_dr, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(tc::saddr(sslot), kTmemCols);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *sslot;

  uint32_t par = 0;     // phase parity of this head's copy and product barriers
  uint32_t ld_par = 0;  // thread 0: parity of the last armed copy phase
  bool ok = true;
  for (int it = 0; it < p.hpc; ++it, par ^= 1u) {
    const int h = hb + it;
    if (tid == 0) {
      ld_par = par;
      tc::expect_tx(bar_ld, (gate ? 3 : 2) * 8192 + (it == 0 ? 2 * N * 128 : 0));
      tc::tma_load_4d(sb + MapLay::kX, &map_x, 0, h, t0, b, bar_ld);
      tc::tma_load_4d(sb + MapLay::kDy, &map_dy, 0, h, t0, b, bar_ld);
      if (gate) tc::tma_load_4d(sb + MapLay::kZ, &map_z, 0, h, t0, b, bar_ld);
      if (it == 0) {
#pragma unroll
        for (int nb = 0; nb < N / 64; ++nb) {
          tc::tma_load_4d(sb + MapLay::kB + nb * 8192, &map_b, 64 * nb, g, t0, b, bar_ld);
          tc::tma_load_4d(sb + MapLay::kC + nb * 8192, &map_c, 64 * nb, g, t0, b, bar_ld);
        }
      }
      // the previous head's bulk stores must have read the staging buffers
      // before this head's slabs are staged there
      tc::bulk_wait_read_all();
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
    ok = tc::wait(bar_ld, par, kWaitLimit);
    if (!ok) atomicOr(&g_tc_fault_bwd, 1u);
    if (__syncthreads_or(!ok)) break;  // weights visible, tiles landed

    // Xw = x e^{lc_end - lc_r} Delta_r and Dw = dout e^{lc_r}, row r, pieces 4 hx .. +3, in place
    {
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
          xw[i] = Pk<Op>::pack(x2.x * wu, x2.y * wu);
          dw[i] = Pk<Op>::pack(d2.x * el, d2.y * el);
        }
        xv = make_uint4(xw[0], xw[1], xw[2], xw[3]);
        dv = make_uint4(dw[0], dw[1], dw[2], dw[3]);
      }
      if (it == 0) {
        to_op_inplace<T>(sm + MapLay::kB, N * 8, tid, kThreads);
        to_op_inplace<T>(sm + MapLay::kC, N * 8, tid, kThreads);
      }
      tc::fence_proxy_async();
    }
    __syncthreads();

    if (tid == 0) {
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
    ok = tc::wait(bar_mma, par, kWaitLimit);
    if (!ok) atomicOr(&g_tc_fault_bwd, 2u);
    tc::fence_after();
    if (ok) {
      // accumulator row n = state row n: element (p, n) of the fp16 slabs, in
      // operand-tile order (tile_idx), staged for the bulk stores
      const int n = N == 128 ? tid : r;
      const int p0 = N == 128 ? 0 : 32 * hx;
      __half* su = reinterpret_cast<__half*>(sm + MapLay::kSu);
      __half* gv = reinterpret_cast<__half*>(sm + MapLay::kSv);
      if constexpr (N == 128) {
#pragma unroll
        for (int c0 = 0; c0 < HP; c0 += 16) {
          float u[16], v[16];
          tc::ld32x32b_x16(tmem + lane_base + kR0 + c0, u);
          tc::ld32x32b_x16(tmem + lane_base + kR1 + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            su[tile_idx(p0 + c0 + i, n)] = __float2half_rn(u[i]);
            gv[tile_idx(p0 + c0 + i, n)] = __float2half_rn(v[i]);
          }
        }
      } else {
        float u[32], v[32];
        tc::ld16x32bx2_x32(tmem + lane_base + kR0, u);
        tc::ld16x32bx2_x32(tmem + lane_base + kR1, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          su[tile_idx(p0 + i, n)] = __float2half_rn(u[i]);
          gv[tile_idx(p0 + i, n)] = __float2half_rn(v[i]);
        }
      }
      tc::fence_proxy_async();
    }
    // every thread staged its slab columns, read its accumulators and is done
    // with this head's tiles and weights
    tc::fence_before();
    if (__syncthreads_or(!ok)) break;
    tc::fence_after();
    if (tid == 0) {
      const size_t slab = ((static_cast<size_t>(b) * nh + h) * p.nchunk + k) * static_cast<size_t>(kP * N);
      tc::bulk_store(reinterpret_cast<__half*>(p.su) + slab, sb + MapLay::kSu, kP * N * 2);
      tc::bulk_store(reinterpret_cast<__half*>(p.gv) + slab, sb + MapLay::kSv, kP * N * 2);
      tc::bulk_commit();
    }
  }
  // drain (a no-op on the normal path): the last armed copies, every product
  // (one commit tracks all of thread 0's earlier products), the bulk stores
  if (tid == 0) {
    if (!tc::wait(bar_ld, ld_par, kWaitLimit)) atomicOr(&g_tc_fault_bwd, 4u);
    tc::commit(bar_dr);
    if (!tc::wait(bar_dr, 0, kWaitLimit)) atomicOr(&g_tc_fault_bwd, 4u);
    tc::bulk_wait_all();
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------ chunk gradients -----
// One CTA of 8 compute warps and an issuing warp per chunk and group of hpc
// heads, which it takes one after another.  With lc_t = A_h sum_{s<=t} Delta_s (log2
// units below), S0 the state entering the chunk and Gc the adjoint at its last
// step (both from the pass over the chunks), dout_t = dy_t SiLU(z_t):
//   CBL[t][s]  = e^{lc_t - lc_s} C_t.B_s                   (s <= t, else 0)
//   XDL'[t][s] = e^{lc_t - lc_s} (dout_t.x_s) Delta_s      (s <= t, else 0)
//   dC_t = e^{lc_t} S0^T dout_t + sum_s XDL'[t][s] B_s
//   dB_t = e^{lc_end - lc_t} Delta_t Gc^T x_t + sum_s XDL'[s][t] C_s
//   (S0 C_t)_p, (Gc B_t)_p, yp = sum_s CBL[t][s] Delta_s x_s, gb = sum_s CBL[s][t] dout_s
// are ten tcgen05 products (M = 64 steps, fp32 accumulation, all 512 TMEM
// columns): the row scalings e^{lc_t}, e^{lc_end - lc_t} Delta_t and Delta_s
// ride on pre-scaled copies of dout and x, and Delta_s on XDL' itself, which
// then serves dC as stored and dB transposed (an MN-major A operand).  From
// the accumulators each thread forms dx, dz and the row sums of the decay
// gradient for its row segment.  dC and dB accumulate over the CTA's heads
// (the first products of each later head add to them), and after the last
// head each thread stores its segment of the sums as one fp16 partial.
struct GradLay {
  static constexpr int kX = 0;              // x                      [t][p] (TMA)
  static constexpr int kDy = 8192;          // dy                     [t][p] (TMA)
  static constexpr int kZ = 16384;          // z                      [t][p] (TMA)
  static constexpr int kB = 24576;          // B   [t][n], 64-wide n blocks 8 KB apart (TMA)
  static constexpr int kC = kB + 16384;     // C                              (TMA)
  static constexpr int kS0 = kC + 16384;    // S0  [p][n]
  static constexpr int kGc = kS0 + 16384;   // Gc  [p][n]
  static constexpr int kO = kGc + 16384;    // dout                   [t][p]
  static constexpr int kOe = kO + 8192;     // dout e^{lc_t}
  static constexpr int kXr = kOe + 8192;    // x e^{lc_end - lc_t} Delta_t
  static constexpr int kXd = kXr + 8192;    // x Delta_t
  static constexpr int kCbl = kXd + 8192;   // CBL                    [t][s]
  static constexpr int kXdl = kCbl + 8192;  // XDL'                   [t][s]
  static constexpr int kDzf = kXdl + 8192;  // dz factor dy sigma(z)(1 + z(1 - sigma(z)))  [t][p]
  static constexpr int kF = kDzf + 8192;    // fp32 scratch, offsets in floats:
  static constexpr int fDlt = 0, fLc = 64, fVv = 128, fEl = 192;
  static constexpr int fRw = 256;           // [2][64] row sums of W by column half
  static constexpr int fCl = fRw + 128;     // [4][64] column sums of W by row quarter
  static constexpr int fRx = fCl + 256;     // [2][64] x.(G B) by column half
  static constexpr int fRo = fRx + 128;     // [2][64] dout.(S0 C)
  static constexpr int fRb = fRo + 128;     // [2][64] x.(Gc B)
  static constexpr int fRed = fRb + 128;    // [2][8] per-warp <Gc, S0> and sum x dout
  static constexpr int fEnd = fRed + 16;
  static constexpr int kBars = kF + fEnd * 4;  // 4 mbarriers: copies, first and second products, drain
  static constexpr int kSlot = kBars + 32;
  static constexpr int kBytes = kSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

template <typename T>
__device__ __forceinline__ void unpack8f(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = Pk<T>::unpack(w[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
template <typename T>
__device__ __forceinline__ uint4 pack8f(const float* f) {
  return make_uint4(Pk<T>::pack(f[0], f[1]), Pk<T>::pack(f[2], f[3]), Pk<T>::pack(f[4], f[5]),
                    Pk<T>::pack(f[6], f[7]));
}
// K-major descriptor of K16 step kk of a [64 rows][K] tile (64-wide K blocks
// 8 KB apart); MN-major descriptor of K16 step kk of a [K = 64 rows][MN] tile.
__device__ __forceinline__ uint64_t dk(uint32_t tile, int kk) {
  return tc::desc_sw128(tile + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t dmn(uint32_t tile, int kk) {
  return tc::desc_sw128(tile + kk * 2048, 8192, 1024);
}

constexpr int kGradCompute = 256;  // threads of the 8 compute warps
constexpr int kGradThreads = kGradCompute + 32;  // + one warp that issues the copies and products

template <typename T, int N>
__global__ void __launch_bounds__(kGradThreads, 1)
    ssd_grad_tc_kernel(const SsdBwdParams p, const __grid_constant__ CUtensorMap map_x,
                       const __grid_constant__ CUtensorMap map_dy, const __grid_constant__ CUtensorMap map_z,
                       const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_c) {
  using G = GradLay;
  constexpr uint32_t kIdKK = tc::idesc_f16(false, 64, 64, false, false);  // fp16 operands
  constexpr uint32_t kIdKM = tc::idesc_f16(false, 64, 64, false, true);
  constexpr uint32_t kIdMM = tc::idesc_f16(false, 64, 64, true, true);
  constexpr uint32_t kIdNKM = tc::idesc_f16(false, 64, N, false, true);
  constexpr uint32_t kIdNMM = tc::idesc_f16(false, 64, N, true, true);
  constexpr uint32_t cCb = 0, cXd = 64, cSc = 128, cBg = 192, cDc = 256, cDb = 256 + N;  // TMEM columns
  constexpr uint32_t cYp = 0, cGb = 64;  // reuse C B^T's and dout x^T's columns
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc::saddr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* const sm = smem_raw + pad;
  const uint32_t sb = raw + pad;
  float* const f = reinterpret_cast<float*>(sm + G::kF);
  uint32_t* const sslot = reinterpret_cast<uint32_t*>(sm + G::kSlot);
  const uint32_t bar_ld = sb + G::kBars, bar_a = bar_ld + 8, bar_b = bar_ld + 16, bar_dr = bar_ld + 24;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool compute = tid < kGradCompute;               // warp 8 only issues
  constexpr int kIssuer = kGradCompute;
  const int q = warp & 3, cg = warp >> 2;                // lane quarter, column half
  const int r = 16 * q + (lane & 15), hx = lane >> 4;    // row of an M = 64 accumulator
  const int c16 = 32 * cg + 16 * hx;                     // this thread's 16 of 64 columns
  const int c32 = 64 * cg + 32 * hx;                     // its 32 of 128 columns
  const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
  // this CTA: chunk k of heads hb .. hb + hpc - 1 (one group) of batch row b
  const int k = blockIdx.x, hb = blockIdx.y * p.hpc, b = blockIdx.z;
  const int L = p.seqlen, nh = p.nheads, ng = p.ngroups, g = hb / (nh / ng);
  const int t0 = k * kQ, nval = min(kQ, L - t0);
  const bool gate = p.z != nullptr;

  if (tid == 0) {
    tc::mbar_init(bar_ld, 1);
    tc::mbar_init(bar_a, 1);
    tc::mbar_init(bar_b, 1);
    tc::mbar_init(bar_dr, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(tc::saddr(sslot), 512);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *sslot;
  uint32_t par = 0;       // phase parity of this head's barriers
  bool ld_armed = false;  // the issuer has armed bar_ld ...
  uint32_t ld_par = 0;    // ... last in the phase of this parity
  bool ok = true;
  for (int it = 0; it < p.hpc; ++it, par ^= 1u) {
  const int h = hb + it;
  const float Ah = p.A[h];
  const float Dh = p.D ? p.D[h] : 0.f;
  const size_t slab = ((static_cast<size_t>(b) * nh + h) * p.nchunk + k) * static_cast<size_t>(kP * N);
  const size_t dto0 = (static_cast<size_t>(b) * L + t0) * nh + h;
  if (tid == kIssuer) {
    // this head's tiles and fp16 state and adjoint slabs (stored in tile
    // order: one untiled bulk copy each); B and C once, for the first head
    tc::expect_tx(bar_ld, (gate ? 3 : 2) * 8192 + (it == 0 ? 2 * N * 128 : 0) + 2 * kP * N * 2);
    tc::bulk_load(sb + G::kS0, reinterpret_cast<const __half*>(p.su) + slab, kP * N * 2, bar_ld);
    tc::bulk_load(sb + G::kGc, reinterpret_cast<const __half*>(p.gv) + slab, kP * N * 2, bar_ld);
    tc::tma_load_4d(sb + G::kX, &map_x, 0, h, t0, b, bar_ld);
    tc::tma_load_4d(sb + G::kDy, &map_dy, 0, h, t0, b, bar_ld);
    if (gate) tc::tma_load_4d(sb + G::kZ, &map_z, 0, h, t0, b, bar_ld);
    if (it == 0) {
#pragma unroll
      for (int nb = 0; nb < N / 64; ++nb) {
        tc::tma_load_4d(sb + G::kB + nb * 8192, &map_b, 64 * nb, g, t0, b, bar_ld);
        tc::tma_load_4d(sb + G::kC + nb * 8192, &map_c, 64 * nb, g, t0, b, bar_ld);
      }
    }
    ld_armed = true;
    ld_par = par;
  }
  // Delta, v = dt + bias, lc (log2 units) and e^{lc} of the chunk (warp 7)
  if (warp == 7) {
    const T* dtg = static_cast<const T*>(p.dt) + dto0;
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
    const float A2 = Ah * kLog2e;
    float d2[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      float v = 0.f, d = 0.f;
      if (t < nval) {
        v = Elt<T>::to_f(dtg[static_cast<size_t>(t) * nh]) + bias;
        d = p.softplus ? softplus_f(v) : v;
      }
      d2[e] = d;
      f[G::fVv + t] = v;
      f[G::fDlt + t] = d;
    }
    const float own = (d2[0] + d2[1]) * A2;
    float run = own;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float o = __shfl_up_sync(0xffffffffu, run, off);
      if (lane >= off) run += o;
    }
    const float l0 = run - own + d2[0] * A2;
    f[G::fLc + 2 * lane] = l0;
    f[G::fLc + 2 * lane + 1] = run;
    f[G::fEl + 2 * lane] = ex2(l0);
    f[G::fEl + 2 * lane + 1] = ex2(run);
  }
  float gs = 0.f;
  ok = tc::wait(bar_ld, par, kWaitLimit);
  if (!ok) atomicOr(&g_tc_fault_bwd, 1u);
  float dxo = 0.f;  // sum x dout
  do {
    if (__syncthreads_or(!ok)) break;  // Delta arrays, tiles
    // ---- <Gc, S0> from the two tiles (same element order)
    if (compute) {
#pragma unroll
      for (int i = 0; i < kP * N / 8 / 256; ++i) {
        const int e = tid + 256 * i;
        float sv[8], gv[8];
        unpack8f<Op>(*reinterpret_cast<const uint4*>(sm + G::kS0 + 16 * e), sv);
        unpack8f<Op>(*reinterpret_cast<const uint4*>(sm + G::kGc + 16 * e), gv);
#pragma unroll
        for (int j = 0; j < 8; ++j) gs = fmaf(sv[j], gv[j], gs);
      }
    }
    // ---- dout, the dz factor and the scaled copies of dout and x (two
    //      16-byte pieces per thread); x, B and C become fp16 operands in place
    if (compute) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int e = tid + 256 * i, t = e >> 3;
        const uint32_t off = swz(t, e & 7);
        float xv[8], dy[8], o[8], w[8];
        unpack8f<T>(*reinterpret_cast<const uint4*>(sm + G::kX + off), xv);
        unpack8f<T>(*reinterpret_cast<const uint4*>(sm + G::kDy + off), dy);
        if (gate) {
          float zv[8], fz[8];
          unpack8f<T>(*reinterpret_cast<const uint4*>(sm + G::kZ + off), zv);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float sg = sigmoid_f(zv[j]);
            o[j] = dy[j] * zv[j] * sg;
            fz[j] = dy[j] * sg * fmaf(zv[j], 1.f - sg, 1.f);
          }
          *reinterpret_cast<uint4*>(sm + G::kDzf + off) = pack8f<Op>(fz);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) o[j] = dy[j];
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) dxo = fmaf(xv[j], o[j], dxo);
        *reinterpret_cast<uint4*>(sm + G::kO + off) = pack8f<Op>(o);
        const float el = f[G::fEl + t], dl = f[G::fDlt + t];
        const float er = ex2(f[G::fLc + kQ - 1] - f[G::fLc + t]) * dl;
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = o[j] * el;
        *reinterpret_cast<uint4*>(sm + G::kOe + off) = pack8f<Op>(w);
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = xv[j] * er;
        *reinterpret_cast<uint4*>(sm + G::kXr + off) = pack8f<Op>(w);
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = xv[j] * dl;
        *reinterpret_cast<uint4*>(sm + G::kXd + off) = pack8f<Op>(w);
        *reinterpret_cast<uint4*>(sm + G::kX + off) = pack8f<Op>(xv);
      }
      if (it == 0) {
        to_op_inplace<T>(sm + G::kB, N * 8, tid, kGradCompute);
        to_op_inplace<T>(sm + G::kC, N * 8, tid, kGradCompute);
      }
    }
    tc::fence_proxy_async();
    if (__syncthreads_or(false)) break;
    // ---- C B^T, dout x^T (commit), then (S0 C_t), (Gc B_t) and the first terms of dC, dB
    if (tid == kIssuer) {
      tc::fence_after();
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) tc::mma(tmem + cCb, dk(sb + G::kC, kk), dk(sb + G::kB, kk), kIdKK, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) tc::mma(tmem + cXd, dk(sb + G::kO, kk), dk(sb + G::kX, kk), kIdKK, kk > 0);
      tc::commit(bar_a);
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) tc::mma(tmem + cSc, dk(sb + G::kC, kk), dk(sb + G::kS0, kk), kIdKK, kk > 0);
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) tc::mma(tmem + cBg, dk(sb + G::kB, kk), dk(sb + G::kGc, kk), kIdKK, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma(tmem + cDc, dk(sb + G::kOe, kk), dmn(sb + G::kS0, kk), kIdNKM, it > 0 || kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma(tmem + cDb, dk(sb + G::kXr, kk), dmn(sb + G::kGc, kk), kIdNKM, it > 0 || kk > 0);
    }
    // ---- CBL and XDL' rows, and the row / column sums of W = CBL o Delta_s o (dout.x)
    if (compute) {
      ok = tc::wait(bar_a, par, kWaitLimit);
      if (!ok) atomicOr(&g_tc_fault_bwd, 2u);
      tc::fence_after();
      float cb[16], xd[16], w[16];
      tc::ld16x32bx2_x16(tmem + lane_base + cCb + 32 * cg, cb);
      tc::ld16x32bx2_x16(tmem + lane_base + cXd + 32 * cg, xd);
      const float lcr = f[G::fLc + r];
      float cbl[16], xdl[16], rw = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int s = c16 + i;
        const float dcy = s <= r ? ex2(lcr - f[G::fLc + s]) : 0.f;
        const float dls = f[G::fDlt + s];
        cbl[i] = dcy * cb[i];
        xdl[i] = dcy * xd[i] * dls;
        w[i] = cbl[i] * dls * xd[i];
        rw += w[i];
      }
      *reinterpret_cast<uint4*>(sm + G::kCbl + swz(r, c16 / 8)) = pack8f<Op>(cbl);
      *reinterpret_cast<uint4*>(sm + G::kCbl + swz(r, c16 / 8 + 1)) = pack8f<Op>(cbl + 8);
      *reinterpret_cast<uint4*>(sm + G::kXdl + swz(r, c16 / 8)) = pack8f<Op>(xdl);
      *reinterpret_cast<uint4*>(sm + G::kXdl + swz(r, c16 / 8 + 1)) = pack8f<Op>(xdl + 8);
      rw += __shfl_xor_sync(0xffffffffu, rw, 16);
      if (hx == 0) f[G::fRw + 64 * cg + r] = rw;
      // column sums over this half-warp's 16 rows: reduce-scatter, lane j ends
      // with column c16 + j
#pragma unroll
      for (int o = 8, n = 8; o >= 1; o >>= 1, n >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
          const float send = up ? w[i] : w[i + n];
          const float keep = up ? w[i + n] : w[i];
          w[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      f[G::fCl + 64 * q + c16 + (lane & 15)] = w[0];
    }
    tc::fence_proxy_async();
    tc::fence_before();
    if (__syncthreads_or(!ok)) break;
    // ---- the second terms of dC and dB, the intra-chunk read-out and sum_s CBL[s][t] dout_s
    if (tid == kIssuer) {
      tc::fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) tc::mma(tmem + cDc, dk(sb + G::kXdl, kk), dmn(sb + G::kB, kk), kIdNKM, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) tc::mma(tmem + cDb, dmn(sb + G::kXdl, kk), dmn(sb + G::kC, kk), kIdNMM, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) tc::mma(tmem + cYp, dk(sb + G::kCbl, kk), dmn(sb + G::kXd, kk), kIdKM, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) tc::mma(tmem + cGb, dmn(sb + G::kCbl, kk), dmn(sb + G::kO, kk), kIdMM, kk > 0);
      tc::commit(bar_b);
    }
    const bool live = r < nval;
    if (compute) {
    ok = tc::wait(bar_b, par, kWaitLimit);
    if (!ok) atomicOr(&g_tc_fault_bwd, 2u);
    tc::fence_after();
    // ---- after the last head: dC, dB rows summed over this CTA's heads, as
    //      fp16 partials (summed over the group's partials in fp32 by the
    //      fixed-order reduction)
    if (it == p.hpc - 1) {
      const size_t rowo = ((static_cast<size_t>(b) * L + t0 + r) * (nh / p.hpc) + hb / p.hpc) * N;
      __half* pdc = reinterpret_cast<__half*>(p.pdC) + rowo;
      __half* pdb = reinterpret_cast<__half*>(p.pdB) + rowo;
      if constexpr (N == 128) {
        float v[32];
        tc::ld16x32bx2_x32(tmem + lane_base + cDc + 64 * cg, v);
        if (live) {
          uint4* d = reinterpret_cast<uint4*>(pdc + c32);
#pragma unroll
          for (int i = 0; i < 4; ++i) d[i] = pack8f<Op>(v + 8 * i);
        }
        tc::ld16x32bx2_x32(tmem + lane_base + cDb + 64 * cg, v);
        if (live) {
          uint4* d = reinterpret_cast<uint4*>(pdb + c32);
#pragma unroll
          for (int i = 0; i < 4; ++i) d[i] = pack8f<Op>(v + 8 * i);
        }
      } else {
        float v[16];
        tc::ld16x32bx2_x16(tmem + lane_base + cDc + 32 * cg, v);
        if (live) {
          uint4* d = reinterpret_cast<uint4*>(pdc + c16);
#pragma unroll
          for (int i = 0; i < 2; ++i) d[i] = pack8f<Op>(v + 8 * i);
        }
        tc::ld16x32bx2_x16(tmem + lane_base + cDb + 32 * cg, v);
        if (live) {
          uint4* d = reinterpret_cast<uint4*>(pdb + c16);
#pragma unroll
          for (int i = 0; i < 2; ++i) d[i] = pack8f<Op>(v + 8 * i);
        }
      }
    }
    // ---- per (t, p): dx, dz and the row sums of the decay gradient
    {
      float sc[16], bg[16], yp[16], gb[16];
      tc::ld16x32bx2_x16(tmem + lane_base + cSc + 32 * cg, sc);
      tc::ld16x32bx2_x16(tmem + lane_base + cBg + 32 * cg, bg);
      tc::ld16x32bx2_x16(tmem + lane_base + cYp + 32 * cg, yp);
      tc::ld16x32bx2_x16(tmem + lane_base + cGb + 32 * cg, gb);
      const float el = f[G::fEl + r], dlr = f[G::fDlt + r];
      const float er = ex2(f[G::fLc + kQ - 1] - f[G::fLc + r]);
      float rx = 0.f, ro = 0.f, rb = 0.f;
      const size_t xo = (static_cast<size_t>(b) * L + t0 + r) * static_cast<size_t>(nh) * kP + h * kP + c16;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t off = swz(r, c16 / 8 + half);
        float xv[8], ovs[8], fzs[8], dxv[8], dzv[8];
        unpack8f<Op>(*reinterpret_cast<const uint4*>(sm + G::kX + off), xv);  // x, dout, the dz factor: fp16
        unpack8f<Op>(*reinterpret_cast<const uint4*>(sm + G::kO + off), ovs);
        if (gate) unpack8f<Op>(*reinterpret_cast<const uint4*>(sm + G::kDzf + off), fzs);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = 8 * half + j;
          const float ov = ovs[j], fz = gate ? fzs[j] : 0.f;
          const float gbv = fmaf(er, bg[i], gb[i]);
          rx = fmaf(xv[j], gbv, rx);
          ro = fmaf(ov, sc[i], ro);
          rb = fmaf(xv[j], bg[i], rb);
          dxv[j] = fmaf(dlr, gbv, Dh * ov);
          dzv[j] = (fmaf(el, sc[i], yp[i]) + Dh * xv[j]) * fz;
        }
        if (live) {
          *reinterpret_cast<uint4*>(static_cast<T*>(p.dx) + xo + 8 * half) = pack8f<T>(dxv);
          if (p.dz && gate) *reinterpret_cast<uint4*>(static_cast<T*>(p.dz) + xo + 8 * half) = pack8f<T>(dzv);
        }
      }
      rx += __shfl_xor_sync(0xffffffffu, rx, 16);
      ro += __shfl_xor_sync(0xffffffffu, ro, 16);
      rb += __shfl_xor_sync(0xffffffffu, rb, 16);
      if (hx == 0) {
        f[G::fRx + 64 * cg + r] = rx;
        f[G::fRo + 64 * cg + r] = ro;
        f[G::fRb + 64 * cg + r] = rb;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      gs += __shfl_xor_sync(0xffffffffu, gs, o);
      dxo += __shfl_xor_sync(0xffffffffu, dxo, o);
    }
    if (lane == 0) {
      f[G::fRed + warp] = gs;
      f[G::fRed + 8 + warp] = dxo;
    }
    }  // compute warps
    if (__syncthreads_or(!ok)) break;
    // ---- the decay gradient dl_t, dDelta and the per-chunk parameter partials (warp 0)
    if (warp == 0) {
      float gsum = 0.f, dsum = 0.f;
      for (int w8 = 0; w8 < 8; ++w8) {
        gsum += f[G::fRed + w8];
        dsum += f[G::fRed + 8 + w8];
      }
      const float* lc = f + G::fLc;
      const float* dlt = f + G::fDlt;
      const float lend = lc[kQ - 1];
      float dl[2], t3 = 0.f, rxgb[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = lane + 32 * hh;
        const float rwt = f[G::fRw + t] + f[G::fRw + 64 + t];
        const float clt = f[G::fCl + t] + f[G::fCl + 64 + t] + f[G::fCl + 128 + t] + f[G::fCl + 192 + t];
        const float rosc = f[G::fRo + t] + f[G::fRo + 64 + t];
        const float rxbg = f[G::fRb + t] + f[G::fRb + 64 + t];
        rxgb[hh] = f[G::fRx + t] + f[G::fRx + 64 + t];
        const float x3 = ex2(lend - lc[t]) * dlt[t] * rxbg;
        dl[hh] = rwt - clt + f[G::fEl + t] * rosc - x3;
        t3 += x3;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) t3 += __shfl_xor_sync(0xffffffffu, t3, o);
      if (lane == 31) dl[1] += ex2(lend) * gsum + t3;  // the chunk end, t = 63
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {  // suffix sums: q_s = sum_{t >= s} dl_t
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
        const float dd = fmaf(Ah, dl[hh], rxgb[hh]);
        const float dv = p.softplus ? dd * sigmoid_f(f[G::fVv + t]) : dd;
        pa = fmaf(dlt[t], dl[hh], pa);
        if (t < nval) {
          ddtg[static_cast<size_t>(t) * nh] = Elt<T>::from_f(dv);
          pb += dv;
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        pa += __shfl_xor_sync(0xffffffffu, pa, o);
        pb += __shfl_xor_sync(0xffffffffu, pb, o);
      }
      if (lane == 0) {
        const size_t pi = (static_cast<size_t>(b) * nh + h) * p.nchunk + k;
        p.pA[pi] = pa;
        p.pD[pi] = dsum;
        p.pbias[pi] = pb;
      }
    }
  } while (false);
  // the next head's copies, products and Delta arrays overwrite this head's
  // tiles, accumulators and scratch: everyone is done with them here
  tc::fence_proxy_async();
  tc::fence_before();
  if (__syncthreads_or(!ok)) break;
  tc::fence_after();
  }  // heads
  // drain whatever may still be in flight after an early exit (no-op
  // otherwise): the last armed copies, and every product (one commit tracks
  // all the issuer's earlier products)
  if (tid == kIssuer) {
    if (ld_armed && !tc::wait(bar_ld, ld_par, kWaitLimit)) atomicOr(&g_tc_fault_bwd, 4u);
    tc::commit(bar_dr);
    if (!tc::wait(bar_dr, 0, kWaitLimit)) atomicOr(&g_tc_fault_bwd, 4u);
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, 512);
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
  if (p.hpc < 1 || (p.nheads / p.ngroups) % p.hpc != 0) return cudaErrorInvalidValue;
  ssd_maps_tc_kernel<T, N><<<dim3(p.nchunk, p.nheads / p.hpc, p.batch), kThreads, MapLay::kAlloc, s>>>(
      p, mx, mdy, mz, mb, mc);
  return cudaGetLastError();
}

// The pass over the chunks on fp16 slabs: one thread per 16-byte piece (8
// elements) of a (b, h) slab.  Forwards it turns U_k into S_k (the state
// entering chunk k) in place, backwards V_k into Gc_k (the adjoint at chunk
// k's last step); the recurrences run in fp32 registers, only the stored
// slabs are fp16.  h0, dfinal and dh0 are fp32 (b, nh, P, N): the piece's
// 8 elements are 8 consecutive n of one row p there.
constexpr int kPass16Depth = 16;
__global__ void __launch_bounds__(256) ssd_pass16_kernel(const SsdBwdParams p, int pieces) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<size_t>(p.batch) * p.nheads * pieces) return;
  const size_t bh = idx / pieces;
  const int e = static_cast<int>(idx % pieces);
  const int N = p.dstate;
  const int q = e & 511, prow = q >> 3, n0 = 64 * (e >> 9) + 8 * ((q & 7) ^ (prow & 7));
  const size_t ho = (bh * kP + prow) * N + n0;  // fp32 (b, h, p, n) of the piece's first element
  const int K = p.nchunk;
  const float* dec = p.dec + bh * K;
  uint4* su = reinterpret_cast<uint4*>(p.su) + bh * K * pieces + e;
  uint4* gv = reinterpret_cast<uint4*>(p.gv) + bh * K * pieces + e;
  float s[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s[i] = p.h0 ? p.h0[ho + i] : 0.f;
  for (int k0 = 0; k0 < K; k0 += kPass16Depth) {
    uint4 u[kPass16Depth];
    float d[kPass16Depth];
#pragma unroll
    for (int j = 0; j < kPass16Depth; ++j)
      if (k0 + j < K) {
        u[j] = su[static_cast<size_t>(k0 + j) * pieces];
        d[j] = dec[k0 + j];
      }
#pragma unroll
    for (int j = 0; j < kPass16Depth; ++j)
      if (k0 + j < K) {
        su[static_cast<size_t>(k0 + j) * pieces] = pack8f<Op>(s);
        float uv[8];
        unpack8f<Op>(u[j], uv);
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i] = fmaf(d[j], s[i], uv[i]);
      }
  }
  float g[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) g[i] = p.dfinal ? p.dfinal[ho + i] : 0.f;
  for (int k1 = K - 1; k1 >= 0; k1 -= kPass16Depth) {
    uint4 v[kPass16Depth];
    float d[kPass16Depth];
#pragma unroll
    for (int j = 0; j < kPass16Depth; ++j)
      if (k1 - j >= 0) {
        v[j] = gv[static_cast<size_t>(k1 - j) * pieces];
        d[j] = dec[k1 - j];
      }
#pragma unroll
    for (int j = 0; j < kPass16Depth; ++j)
      if (k1 - j >= 0) {
        gv[static_cast<size_t>(k1 - j) * pieces] = pack8f<Op>(g);
        float vv[8];
        unpack8f<Op>(v[j], vv);
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = fmaf(d[j], g[i], vv[i]);
      }
  }
  if (p.dh0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) p.dh0[ho + i] = g[i];
  }
}

template <typename T, int N>
cudaError_t launch_grad(const SsdBwdParams& p, cudaStream_t s) {
  constexpr bool bf = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap mx, mdy, mz, mb, mc;
  std::memset(&mz, 0, sizeof(mz));
  if (!tc::encode_rows(&mx, bf, p.x, kP, p.nheads, p.seqlen, p.batch) ||
      !tc::encode_rows(&mdy, bf, p.dy, kP, p.nheads, p.seqlen, p.batch) ||
      (p.z && !tc::encode_rows(&mz, bf, p.z, kP, p.nheads, p.seqlen, p.batch)) ||
      !tc::encode_rows(&mb, bf, p.B, N, p.ngroups, p.seqlen, p.batch) ||
      !tc::encode_rows(&mc, bf, p.C, N, p.ngroups, p.seqlen, p.batch))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(ssd_grad_tc_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       GradLay::kAlloc);
  if (e != cudaSuccess) return e;
  // hpc heads of one group per CTA
  if (p.hpc < 1 || (p.nheads / p.ngroups) % p.hpc != 0) return cudaErrorInvalidValue;
  ssd_grad_tc_kernel<T, N><<<dim3(p.nchunk, p.nheads / p.hpc, p.batch), kGradThreads, GradLay::kAlloc, s>>>(
      p, mx, mdy, mz, mb, mc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ssd_grad_tc(const SsdBwdParams& p, DType dt, cudaStream_t s) {
  if (p.headdim != kP || (p.dstate != 64 && p.dstate != 128)) return cudaErrorInvalidValue;
  switch (dt) {
    case DType::BF16:
      return p.dstate == 64 ? launch_grad<__nv_bfloat16, 64>(p, s) : launch_grad<__nv_bfloat16, 128>(p, s);
    case DType::F16:
      return p.dstate == 64 ? launch_grad<__half, 64>(p, s) : launch_grad<__half, 128>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

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

cudaError_t launch_ssd_pass16(const SsdBwdParams& p, cudaStream_t s) {
  const int pieces = kP * p.dstate / 8;
  const size_t n = static_cast<size_t>(p.batch) * p.nheads * pieces;
  ssd_pass16_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(p, pieces);
  return cudaGetLastError();
}

cudaError_t read_tc_fault_bwd(unsigned* bits, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_tc_fault_bwd, sizeof(unsigned));
  if (e != cudaSuccess || !clear) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_tc_fault_bwd, &zero, sizeof(unsigned));
}

}  // namespace ss
