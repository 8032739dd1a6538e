// ss_ssd_tc.cu -- Mamba-2 SSD forward on the sm_100a tensor cores: tcgen05
// MMAs with TMEM accumulators, operand tiles brought in by TMA.
//
// "Mamba" (stanleyjacob.dev), Part V, "Deep dive: Mamba-2 and state-space
// duality": with A a scalar per head the selective SSM is, inside a chunk of
// the sequence, a masked quadratic form (dense matrix products) and, between
// chunks, a recurrence on the (headdim x dstate) state.  Per (batch b, head h),
// with the B, C of the head's group and a chunk of Q = 64 steps, cs_t the
// cumulative sum of Delta_k A_h within the chunk (k <= t):
//
//   G  = C B^T                                   (Q x Q, K = dstate)
//   M  = G o [exp(cs_i - cs_j) Delta_j]_{j <= i}  (masked, decayed)
//   Y  = diag(exp cs) C H^T + M X                H: state entering the chunk
//   S  = (w o B)^T X,  w_t = exp(cs_last - cs_t) Delta_t
//   H <- exp(cs_last) H + S^T
//   y  = (Y + D x) SiLU(z)
//
// One CTA of 4 warps per (b, h) walks the chunks in order; 3 CTAs (dstate 128)
// or 4 (dstate 64) share an SM.  Per chunk, thread 0 issues three groups of
// tcgen05.mma (kind::f16, fp32 accumulation in TMEM, 128 columns):
//   a) G -> columns [0, 64), then Yc = C H^T -> [64, 128), each with its own
//      commit (neither needs this chunk's Delta: they start as soon as B and C
//      have landed, and the mask starts as soon as G is done);
//   b) S = B^T Xw -> [0, 64), after the threads have read G;
//   c) Y2 = M X -> [0, 64), after the threads have read S.  The skip term D x
//      rides on M's diagonal (M + D I), so the epilogue needs no x.
// Between them the 128 threads form Delta and cs (warp 3), turn x into Xw and
// G into M, update the fp32 state H (kept in registers: thread n owns state
// row n) and write its bf16 copy, the B operand of the next chunk's C H^T, and
// finally form y = exp(cs_i) Yc + Y2, gate it with SiLU(z) and store it.
// Thread 32 issues the TMA copies, each into a single buffer as soon as the
// products that read the previous contents are done: C after C B^T and C H^T,
// B after B^T Xw, x after M X, z after the epilogue.  dt is read with plain
// loads right after a barrier, one chunk ahead.
//
// Every operand tile is a 128-byte-swizzled stack of 128-byte rows:
//   x, Xw    [t][p]                 (MN-major B of M X; rows of Xw)
//   z        [t][p]                 (read by the epilogue)
//   B, C     [t][n] in 64-wide n blocks (K-major for C B^T and C H^T; MN-major
//                                    A of B^T Xw, blocks 8 KB apart)
//   M        [i][j]                 (K-major A of M X; shares Xw's buffer,
//                                    written after S has read Xw)
//   H copy   [n][p]                 (MN-major B of C H^T)
// Waits on mbarriers are bounded.  On a timeout the kernel sets a bit in a
// device fault word (read with ss_device_fault), leaves the walk, waits
// (bounded) for its copies and products in flight, frees its TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstring>
#include <type_traits>

#include "ss_device.cuh"
#include "ss_internal.h"
#include "ss_ssd_bwd.h"
#include "ss_tc.cuh"

namespace ss {

__device__ unsigned int g_tc_fault = 0;

namespace {

constexpr int kQ = 64;        // chunk length
constexpr int kP = 64;        // head dimension
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kR0 = 0, kR1 = 64;  // TMEM column regions
constexpr uint32_t kWaitLimit = 1u << 22;

// Byte offsets in the (1024-aligned) shared-memory block.
template <int N>
struct TcLayout {
  static constexpr int kX = 0;                 // x [t][p], 8 KB
  static constexpr int kZ = 8192;              // z [t][p], 8 KB
  static constexpr int kB = 2 * 8192;          // B: N / 64 blocks of 8 KB
  static constexpr int kC = kB + N * 128;      // C: likewise
  static constexpr int kW = kC + N * 128;      // Xw, then M
  static constexpr int kH = kW + 8192;         // bf16 state copy, N rows of 128 B
  static constexpr int kCs = kH + N * 128;     // float cs[64] (log2 units)
  static constexpr int kNcs = kCs + 256;       // float -cs_j, padded (see cpos)
  static constexpr int kDl = kNcs + 288;       // float Delta_j, padded
  static constexpr int kBars = kDl + 288;      // 9 mbarriers
  static constexpr int kSlot = kBars + 80;     // TMEM base address
  static constexpr int kBytes = kSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;  // + slack to align the base
};
// mbarrier indices
// kBarNever is never arrived on: the test hook waits on it to make a wait run out.
enum : int { kBarX = 0, kBarZ = 1, kBarB = 2, kBarC = 3, kBarG = 4, kBarYc = 5, kBarS = 6, kBarY = 7, kNumBars = 8,
             kBarNever = 8 };
// Column j of the per-column arrays sits at j + 4 (j >= 32): the two column
// halves a warp reads at once then fall in different banks.
__device__ __forceinline__ int cpos(int j) { return j + ((j >> 5) << 2); }

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

// 8 packed 16-bit values <-> 4 fp32 pairs
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& v, f2_t (&f)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = Pk<T>::unpack(w[i]);
    f[i] = pk2(t.x, t.y);
  }
}
template <typename T>
__device__ __forceinline__ uint32_t pack2(f2_t v) { return Pk<T>::pack(lo2(v), hi2(v)); }
template <typename T>
__device__ __forceinline__ uint4 pack8(const f2_t* f) {
  return make_uint4(pack2<T>(f[0]), pack2<T>(f[1]), pack2<T>(f[2]), pack2<T>(f[3]));
}

// Byte offset of 16-byte piece c of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

template <typename T, int N>
__global__ void __launch_bounds__(kThreads, N == 128 ? 3 : 4)
    ssd_tc_kernel(const SsdParams p, const __grid_constant__ CUtensorMap map_x,
                  const __grid_constant__ CUtensorMap map_z, const __grid_constant__ CUtensorMap map_b,
                  const __grid_constant__ CUtensorMap map_c) {
  using Lay = TcLayout<N>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdG = tc::idesc_f16(kBf16, 64, 64, false, false);   // C B^T
  constexpr uint32_t kIdYc = tc::idesc_f16(kBf16, 64, 64, false, true);   // C H^T
  constexpr uint32_t kIdS = tc::idesc_f16(kBf16, N, 64, true, true);      // B^T Xw
  constexpr uint32_t kIdY2 = tc::idesc_f16(kBf16, 64, 64, false, true);   // M X
  constexpr int HP = N == 128 ? 64 : 32;  // state columns (p) per thread
  constexpr uint32_t kBcBytes = N * 128;
  constexpr int kMma = 0, kTma = 32, kDeltaWarp = 3;  // thread / warp roles

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc::saddr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* const sm = smem_raw + pad;
  const uint32_t sb = raw + pad;  // shared-window address of the block
  float* const scs = reinterpret_cast<float*>(sm + Lay::kCs);
  float* const sncs = reinterpret_cast<float*>(sm + Lay::kNcs);
  float* const sdl = reinterpret_cast<float*>(sm + Lay::kDl);
  uint32_t* const sslot = reinterpret_cast<uint32_t*>(sm + Lay::kSlot);
  auto bar = [&](int i) { return sb + Lay::kBars + 8u * static_cast<uint32_t>(i); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = 16 * warp + (lane & 15);  // row of an M = 64 accumulator this thread reads
  const int hx = lane >> 4;               // which 32 of its 64 columns
  const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
  // state rows: thread n owns H[n][p0 .. p0 + HP)
  const int n_own = N == 128 ? tid : r;
  const int p0 = N == 128 ? 0 : 32 * hx;

  const int b = blockIdx.y, h = blockIdx.x;
  const int L = p.seqlen, nh = p.nheads, ng = p.ngroups;
  const int g = h / (nh / ng);
  const float A2 = p.A[h] * kLog2e;
  const float Dh = p.D ? p.D[h] : 0.f;
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
  const size_t xrow = static_cast<size_t>(nh) * kP;
  const bool gate = p.z != nullptr;
  T* __restrict__ yg = static_cast<T*>(p.y) + static_cast<size_t>(b) * L * xrow + h * kP;
  const T* __restrict__ dtg = static_cast<const T*>(p.dt) + static_cast<size_t>(b) * L * nh + h;
  const int nchunks = (L + kQ - 1) / kQ;

  if (tid == kMma) {
#pragma unroll
    for (int i = 0; i <= kBarNever; ++i) tc::mbar_init(bar(i), 1);
    tc::fence_mbar_init();
  }
  if (tid == kTma) {
    tc::prefetch_map(&map_x);
    if (gate) tc::prefetch_map(&map_z);
    tc::prefetch_map(&map_b);
    tc::prefetch_map(&map_c);
  }
  if (warp == 0) tc::tmem_alloc(tc::saddr(sslot), kTmemCols);

  // the state (fp32 pairs of columns p) and its bf16 operand copy
  f2_t hs[HP / 2];
  {
    const float* h0 = p.h0 ? p.h0 + (static_cast<size_t>(b) * nh + h) * kP * N : nullptr;
#pragma unroll
    for (int i = 0; i < HP / 2; ++i)
      hs[i] = h0 ? pk2(h0[static_cast<size_t>(p0 + 2 * i) * N + n_own], h0[static_cast<size_t>(p0 + 2 * i + 1) * N + n_own])
                 : pk2(0.f, 0.f);
  }
  auto write_state_copy = [&]() {
#pragma unroll
    for (int c = 0; c < HP / 8; ++c)
      *reinterpret_cast<uint4*>(sm + Lay::kH + swz(n_own, p0 / 8 + c)) = pack8<T>(hs + 4 * c);
  };
  write_state_copy();
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();  // barriers initialised, TMEM allocated, state copy written
  tc::fence_after();
  const uint32_t tmem = *sslot;

  // The copy thread arms the load barriers, the MMA thread the product
  // barriers; each remembers the parity of the last phase it armed on each, so
  // that an early exit can drain them.
  uint32_t armed = 0, last_par = 0, next_par = 0;
  auto arm = [&](int i) {
    const uint32_t m = 1u << i;
    armed |= m;
    last_par = (last_par & ~m) | (next_par & m);
    next_par ^= m;
  };
  auto load_xz = [&](int k, const CUtensorMap* map, int off, int i) {
    tc::expect_tx(bar(i), 8192);
    tc::tma_load_4d(sb + off, map, 0, h, k * kQ, b, bar(i));
    arm(i);
  };
  auto load_bc = [&](int k, const CUtensorMap* map, int off, int i) {
    tc::expect_tx(bar(i), kBcBytes);
#pragma unroll
    for (int nb = 0; nb < N / 64; ++nb) tc::tma_load_4d(sb + off + nb * 8192, map, 64 * nb, g, k * kQ, b, bar(i));
    arm(i);
  };
  if (tid == kTma) {
    load_bc(0, &map_b, Lay::kB, kBarB);
    load_bc(0, &map_c, Lay::kC, kBarC);
    load_xz(0, &map_x, Lay::kX, kBarX);
    if (gate) load_xz(0, &map_z, Lay::kZ, kBarZ);
  }
  // raw dt of the first chunk (warp kDeltaWarp, steps 2 lane and 2 lane + 1)
  T dtn[2] = {Elt<T>::from_f(0.f), Elt<T>::from_f(0.f)};
  if (warp == kDeltaWarp) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      if (t < L) dtn[e] = dtg[static_cast<size_t>(t) * nh];
    }
  }

  bool ok = true;
  auto fault = [&](unsigned bit) {
    atomicOr(&g_tc_fault, bit);
    ok = false;
  };
  int k = 0;
  for (; k < nchunks; ++k) {
    const int t0 = k * kQ;
    const int nval = min(kQ, L - t0);
    const uint32_t par = k & 1;
    unsigned char* const xs = sm + Lay::kX;
    unsigned char* const zs = sm + Lay::kZ;

    // ---- a) G = C B^T -> R0, Yc = C H^T -> R1 (need B, C and the state copy only)
    if (tid == kMma) {
      if (!tc::wait(bar(kBarB), par, kWaitLimit) || !tc::wait(bar(kBarC), par, kWaitLimit)) fault(1u);
      // test hook (SS_INJECT_WAIT_TIMEOUT): a wait on a barrier nothing arrives on runs out
      if (p.inject_timeout && k == 0 && !tc::wait(bar(kBarNever), 0, 1u << 12)) fault(1u);
      tc::fence_after();
      const uint64_t dc = tc::desc_sw128(sb + Lay::kC, 16, 1024);
      const uint64_t db = tc::desc_sw128(sb + Lay::kB, 16, 1024);
      const uint64_t dh = tc::desc_sw128(sb + Lay::kH, 8192, 1024);
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) {
        const uint32_t koff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;  // descriptor address units
        tc::mma(tmem + kR0, dc + koff, db + koff, kIdG, kk > 0);
      }
      tc::commit(bar(kBarG));  // the mask starts while C H^T still runs
      arm(kBarG);
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) {
        const uint32_t koff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
        tc::mma(tmem + kR1, dc + koff, dh + kk * (2048 >> 4), kIdYc, kk > 0);
      }
      tc::commit(bar(kBarYc));
      arm(kBarYc);
    }
    // ---- Delta_t and cs_t = log2(e) A_h sum_{k<=t} Delta_k
    if (warp == kDeltaWarp) {
      float d2[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        float v = 0.f;
        if (t < nval) {
          const float xv = Elt<T>::to_f(dtn[e]) + bias;
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
      const float c0 = run - own + d2[0] * A2;
      scs[2 * lane] = c0;
      scs[2 * lane + 1] = run;
      const int q = cpos(2 * lane);
      *reinterpret_cast<float2*>(sncs + q) = make_float2(-c0, -run);
      *reinterpret_cast<float2*>(sdl + q) = make_float2(d2[0], d2[1]);
    }
    if (!tc::wait(bar(kBarX), par, kWaitLimit)) fault(1u);
    if (__syncthreads_or(!ok)) break;  // Delta, cs visible; x of the chunk landed

    // The next chunk's dt: global loads issued right after a barrier, so that
    // the work up to the next barrier (which waits for them) hides their latency.
    if (warp == kDeltaWarp && k + 1 < nchunks) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = t0 + kQ + 2 * lane + e;
        if (t < L) dtn[e] = dtg[static_cast<size_t>(t) * nh];
      }
    }
    // ---- Xw = x w_t, w_t = 2^(cs_last - cs_t) Delta_t (row r, pieces 4 hx .. 4 hx + 3)
    const float cs_last = scs[kQ - 1];
    {
      const float w = ex2(cs_last + sncs[cpos(r)]) * sdl[cpos(r)];
      const f2_t w2 = pk2(w, w);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t o = swz(r, 4 * hx + c);
        f2_t f[4];
        unpack8<T>(*reinterpret_cast<const uint4*>(xs + o), f);
#pragma unroll
        for (int e = 0; e < 4; ++e) f[e] = mul2(f[e], w2);
        *reinterpret_cast<uint4*>(sm + Lay::kW + o) = pack8<T>(f);
      }
    }
    tc::fence_proxy_async();
    // ---- M = G o [2^(cs_i - cs_j) Delta_j]_{j <= i} + D_h I, row r, columns 32 hx .. +31
    uint32_t mp[16];
    if (!tc::wait(bar(kBarG), par, kWaitLimit)) fault(2u);
    tc::fence_after();
    {
      const float csr = scs[r];
      const f2_t csr2 = pk2(csr, csr);
      const float4* ncs4 = reinterpret_cast<const float4*>(sncs + 36 * hx);
      const float4* dl4 = reinterpret_cast<const float4*>(sdl + 36 * hx);
      float gv[16];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        if ((m & 3) == 0) tc::ld16x32bx2_x16_split32(tmem + lane_base + kR0 + 16 * (m >> 2), gv);
        const float4 nc = ncs4[m], dl = dl4[m];
        const f2_t e01 = ex2_2(add2(csr2, pk2(nc.x, nc.y)));
        const f2_t e23 = ex2_2(add2(csr2, pk2(nc.z, nc.w)));
        const int gi = 4 * (m & 3);
        f2_t v01 = mul2(mul2(pk2(gv[gi], gv[gi + 1]), e01), pk2(dl.x, dl.y));
        f2_t v23 = mul2(mul2(pk2(gv[gi + 2], gv[gi + 3]), e23), pk2(dl.z, dl.w));
        const int j = 32 * hx + 4 * m;
        float v[4] = {lo2(v01), hi2(v01), lo2(v23), hi2(v23)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (j + e > r) v[e] = 0.f;
          if (j + e == r) v[e] += Dh;
        }
        mp[2 * m] = Pk<T>::pack(v[0], v[1]);
        mp[2 * m + 1] = Pk<T>::pack(v[2], v[3]);
      }
    }
    tc::fence_before();
    if (__syncthreads_or(!ok)) break;  // G read, Xw written

    // ---- b) S = B^T Xw -> R0; the next chunk's C (once C H^T is done too)
    if (tid == kMma) {
      tc::fence_after();
      const uint64_t dbm = tc::desc_sw128(sb + Lay::kB, 8192, 1024);
      const uint64_t dw = tc::desc_sw128(sb + Lay::kW, 8192, 1024);
#pragma unroll
      for (int kk = 0; kk < kQ / 16; ++kk)
        tc::mma(tmem + kR0, dbm + kk * (2048 >> 4), dw + kk * (2048 >> 4), kIdS, kk > 0);
      tc::commit(bar(kBarS));
      arm(kBarS);
    }
    if (tid == kTma && k + 1 < nchunks) {
      if (!tc::wait(bar(kBarYc), par, kWaitLimit)) fault(2u);
      load_bc(k + 1, &map_c, Lay::kC, kBarC);  // C B^T and C H^T are done
    }
    // the old state copy is overwritten below: C H^T must be done with it
    if (!tc::wait(bar(kBarYc), par, kWaitLimit) || !tc::wait(bar(kBarS), par, kWaitLimit)) fault(2u);
    tc::fence_after();
#pragma unroll
    for (int c = 0; c < 4; ++c)  // M over Xw: S has read Xw
      *reinterpret_cast<uint4*>(sm + Lay::kW + swz(r, 4 * hx + c)) =
          make_uint4(mp[4 * c], mp[4 * c + 1], mp[4 * c + 2], mp[4 * c + 3]);
    {
      const float dec = ex2(cs_last);
      const f2_t dec2 = pk2(dec, dec);
      if constexpr (N == 128) {
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {
          float sv[16];
          tc::ld32x32b_x16(tmem + lane_base + kR0 + c0, sv);
#pragma unroll
          for (int i = 0; i < 8; ++i) hs[c0 / 2 + i] = fma2(dec2, hs[c0 / 2 + i], pk2(sv[2 * i], sv[2 * i + 1]));
        }
      } else {
        float sv[32];
        tc::ld16x32bx2_x32(tmem + lane_base + kR0, sv);
#pragma unroll
        for (int i = 0; i < 16; ++i) hs[i] = fma2(dec2, hs[i], pk2(sv[2 * i], sv[2 * i + 1]));
      }
      write_state_copy();  // C H^T of this chunk is done with the old copy
    }
    tc::fence_proxy_async();
    tc::fence_before();
    if (__syncthreads_or(!ok)) break;  // S read, M and the state copy written

    // ---- c) Y2 = M X -> R0 (the skip term D x rides on M's diagonal); the next chunk's B
    if (tid == kMma) {
      tc::fence_after();
      const uint64_t dmk = tc::desc_sw128(sb + Lay::kW, 16, 1024);
      const uint64_t dx = tc::desc_sw128(sb + Lay::kX, 8192, 1024);
#pragma unroll
      for (int kk = 0; kk < kQ / 16; ++kk) tc::mma(tmem + kR0, dmk + kk * 2, dx + kk * (2048 >> 4), kIdY2, kk > 0);
      tc::commit(bar(kBarY));
      arm(kBarY);
    }
    if (tid == kTma && k + 1 < nchunks) load_bc(k + 1, &map_b, Lay::kB, kBarB);  // C B^T, B^T Xw are done
    if (!tc::wait(bar(kBarY), par, kWaitLimit)) fault(2u);
    tc::fence_after();
    if (tid == kTma && k + 1 < nchunks) load_xz(k + 1, &map_x, Lay::kX, kBarX);  // M X and Xw are done with x
    if (gate && !tc::wait(bar(kBarZ), par, kWaitLimit)) fault(1u);
    // ---- y = (2^cs_i Yc + Y2) SiLU(z)
    {
      float yc[32], y2[32];
      tc::ld16x32bx2_x32(tmem + lane_base + kR1, yc);
      tc::ld16x32bx2_x32(tmem + lane_base + kR0, y2);
      const float er = ex2(scs[r]);
      const f2_t er2 = pk2(er, er), nl2 = pk2(-kLog2e, -kLog2e), one2 = pk2(1.f, 1.f);
      if (r < nval) {
        T* yrow = yg + static_cast<size_t>(t0 + r) * xrow + 32 * hx;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          f2_t zv[4], o[4];
          if (gate) unpack8<T>(*reinterpret_cast<const uint4*>(zs + swz(r, 4 * hx + c)), zv);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 8 * c + 2 * e;
            f2_t v = fma2(er2, pk2(yc[i], yc[i + 1]), pk2(y2[i], y2[i + 1]));
            if (gate) {  // z sigma(z) = z / (1 + 2^(-z log2 e))
              const f2_t d = add2(one2, ex2_2(mul2(zv[e], nl2)));
              v = mul2(v, mul2(zv[e], pk2(rcp(lo2(d)), rcp(hi2(d)))));
            }
            o[e] = v;
          }
          *reinterpret_cast<uint4*>(yrow + 8 * c) = pack8<T>(o);
        }
      }
    }
    tc::fence_before();
    if (__syncthreads_or(!ok)) break;  // TMEM and the z tile are free
    if (tid == kTma && gate && k + 1 < nchunks) load_xz(k + 1, &map_z, Lay::kZ, kBarZ);
  }

  if (k == nchunks && p.final_state) {
    float* fs = p.final_state + (static_cast<size_t>(b) * nh + h) * kP * N;
#pragma unroll
    for (int i = 0; i < HP / 2; ++i) {
      fs[static_cast<size_t>(p0 + 2 * i) * N + n_own] = lo2(hs[i]);
      fs[static_cast<size_t>(p0 + 2 * i + 1) * N + n_own] = hi2(hs[i]);
    }
  }
  // Drain: every armed phase must be complete before the TMEM and the shared
  // memory are given back (a no-op on the normal path, where all were waited).
  if (tid == kMma || tid == kTma) {
#pragma unroll
    for (int i = 0; i < kNumBars; ++i)
      if ((armed >> i) & 1u)
        if (!tc::wait(bar(i), (last_par >> i) & 1u, kWaitLimit)) atomicOr(&g_tc_fault, 4u);
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <typename T, int N>
cudaError_t launch_tc(const SsdParams& p, DType dt, cudaStream_t s) {
  CUtensorMap mx, mz, mb, mc;
  std::memset(&mz, 0, sizeof(mz));
  const bool bf = dt == DType::BF16;
  if (!tc::encode_rows(&mx, bf, p.x, kP, p.nheads, p.seqlen, p.batch) ||
      (p.z && !tc::encode_rows(&mz, bf, p.z, kP, p.nheads, p.seqlen, p.batch)) ||
      !tc::encode_rows(&mb, bf, p.B, N, p.ngroups, p.seqlen, p.batch) ||
      !tc::encode_rows(&mc, bf, p.C, N, p.ngroups, p.seqlen, p.batch))
    return cudaErrorInvalidValue;
  const int smem = TcLayout<N>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(ssd_tc_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  ssd_tc_kernel<T, N><<<dim3(p.nheads, p.batch), kThreads, smem, s>>>(p, mx, mz, mb, mc);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_tc_t(const SsdParams& p, DType dt, cudaStream_t s) {
  if (p.headdim != kP) return cudaErrorInvalidValue;
  if (p.dstate == 64) return launch_tc<T, 64>(p, dt, s);
  if (p.dstate == 128) return launch_tc<T, 128>(p, dt, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_ssd_fwd_tc(const SsdParams& p, DType dt, cudaStream_t s) {
  switch (dt) {
    case DType::BF16: return launch_tc_t<__nv_bfloat16>(p, dt, s);
    case DType::F16: return launch_tc_t<__half>(p, dt, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t read_tc_fault(unsigned* bits, bool clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  unsigned fwd = 0, bwd = 0;
  e = cudaMemcpyFromSymbol(&fwd, g_tc_fault, sizeof(unsigned));
  if (e == cudaSuccess) e = read_tc_fault_bwd(&bwd, clear);
  if (e != cudaSuccess) return e;
  *bits = fwd | bwd;
  if (!clear) return cudaSuccess;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_tc_fault, &zero, sizeof(unsigned));
}

}  // namespace ss
