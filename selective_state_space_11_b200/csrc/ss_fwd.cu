// ss_fwd.cu -- forward selective scan (S6) for sm_100a.
//
// Computes, per (batch b, channel d), with an N = 16 wide diagonal state:
//   Delta_t = softplus(delta_t + bias_d)        ("Mamba", stanleyjacob.dev,
//   h_t     = exp(Delta_t A_d) h_{t-1}            Part IV Stages 3-6 and the
//             + Delta_t B_t u_t                   Part V kernel sketch)
//   y_t     = (C_t . h_t + D_d u_t) SiLU(z_t)
// and writes y, the final state, and the state after every 64th step
// ("Mamba, on a laptop GPU.", "The state lives in registers").
//
// Work decomposition (B200: 148 SMs x 4 SM sub-partitions; the 16 decays per
// token*channel on the SFU are the binding unit):
//   * K = 4 (or 8) lanes per channel, 16/K states per lane in registers, held
//     as fp32 pairs so the FP32 pipe works on two states per instruction
//     (fma/mul .f32x2) and issue slots stay free for the SFU;
//   * per 32-step tile, each thread computes the per-token scalars of 32/K
//     steps of its channel once (softplus, Delta*u, gate, D*u) and publishes
//     (Delta, Delta) and (Delta u, Delta u) pairs in shared memory;
//   * B_t / C_t tiles (shared by every channel of a batch row) are staged once
//     per block, transposed to [t][n] so a lane reads its states with one
//     64/128-bit shared load;
//   * the next tile's u, delta, z, B, C are loaded (in storage format) while
//     the current tile scans, hiding HBM latency;
//   * the K lanes' partial readouts meet in shared memory and the owning
//     thread applies skip and gate and writes y with vector stores.
// Zero-padded steps (Delta = 0) leave the state unchanged (exp(0) = 1), so
// ragged tails run the full tile and only the stores are guarded.
//
// Chunk-parallel path (few channels, long L): L is cut into segments (a
// multiple of 64 steps).  Phase 1 scans each segment from a zero state and
// records its end state e_s and decay product P_s = exp(A * sum Delta); phase 2
// composes the (P_s, e_s) pairs with the associative operator
// (a_l, b_l) then (a_r, b_r) = (a_r a_l, a_r b_l + b_r) ("Mamba", Part V "S6,
// and why selectivity forbids the convolution") in three levels (serial
// folds over per-thread slabs of segments, a shuffle scan over a warp's
// slabs, warps in order through shared memory); phase 3 re-runs every segment
// from its true entering state.  Phases 2 and 3 are launched while the phase
// before them still runs (programmatic dependent launch).
#include "ss_device.cuh"
#include "ss_internal.h"

namespace ss {
namespace {

constexpr int TT = 32;  // steps per tile (two tiles per checkpoint chunk)

// Unrolling of the 4-lane forward (compile-time tuning).
#ifndef SS_FWD_UNROLL
#define SS_FWD_UNROLL 8
#endif
constexpr int kFwdUnroll = SS_FWD_UNROLL;
#ifndef SS_FWD_DECAYS_FIRST
#define SS_FWD_DECAYS_FIRST 1
#endif

enum { kFull = 0, kLocal = 1 };

// Store PS consecutive values of a row (vector store when aligned and in range).
template <typename T, int PS, bool VEC>
__device__ __forceinline__ void store_row(T* row, int t, int len, const float (&v)[PS]) {
  constexpr int kWords = PS * (int)sizeof(T) / 4;
  if (VEC && t + PS <= len) {
    uint32_t w[kWords];
    if constexpr (sizeof(T) == 4) {
#pragma unroll
      for (int i = 0; i < PS; ++i) w[i] = __float_as_uint(v[i]);
    } else {
#pragma unroll
      for (int i = 0; i < kWords; ++i) {
        T pr[2] = {Elt<T>::from_f(v[2 * i]), Elt<T>::from_f(v[2 * i + 1])};
        uint32_t lo = *reinterpret_cast<const unsigned short*>(&pr[0]);
        uint32_t hi = *reinterpret_cast<const unsigned short*>(&pr[1]);
        w[i] = lo | (hi << 16);
      }
    }
    if constexpr (kWords == 2) {
      *reinterpret_cast<uint2*>(row + t) = make_uint2(w[0], w[1]);
    } else {
#pragma unroll
      for (int i = 0; i < kWords / 4; ++i)
        reinterpret_cast<uint4*>(row + t)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < PS; ++i)
      if (t + i < len) row[t + i] = Elt<T>::from_f(v[i]);
  }
}

// MINB: resident blocks per SM the register budget is cut for.  Four give
// the scan its registers; five (96 registers) put a grid of up to 5 x SMs
// blocks in one wave instead of leaving a tail wave of a few blocks.
template <typename T, int K, int CB, bool VEC, int MODE, int MINB, bool SEQ>
__global__ void __launch_bounds__(CB * K, MINB)
fwd_kernel(const FwdParams p) {
  constexpr int NT = CB * K;
  constexpr int SPL = kN / K;   // states per lane
  constexpr int NP = SPL / 2;   // fp32 pairs per lane
  constexpr int PS = TT / K;    // steps per thread in prologue / epilogue
  static_assert(NT == 128 && (K == 4 || K == 8), "B/C staging assumes 128 threads");
  __shared__ __align__(16) f2_t s_dt2[CB][TT + 2];   // (Delta, Delta)
  __shared__ __align__(16) f2_t s_du2[CB][TT + 2];   // (Delta u, Delta u)
  __shared__ __align__(16) float s_B[TT][kN];
  __shared__ __align__(16) float s_C[TT][kN];
  __shared__ __align__(16) float s_yp[CB][K][TT + 4];  // per-lane partial C.h

  const int tid = threadIdx.x;
  const int c = tid / K, j = tid % K;
  const int b = blockIdx.y, seg = blockIdx.z;
  const int d = blockIdx.x * CB + c;
  const bool dvalid = d < p.dim;
  const int dd = dvalid ? d : 0;
  const int L = p.seqlen;
  const int t_begin = seg * p.seg_len;
  const int t_end = min(L, t_begin + p.seg_len);

  const size_t row = ((size_t)b * p.dim + dd) * (size_t)L;
  const T* __restrict__ u_row = static_cast<const T*>(p.u) + row;
  const T* __restrict__ x_row = static_cast<const T*>(p.delta) + row;
  const T* __restrict__ z_row = p.z ? static_cast<const T*>(p.z) + row : nullptr;
  const T* __restrict__ Bb = static_cast<const T*>(p.B) + (size_t)b * kN * L;
  const T* __restrict__ Cb = static_cast<const T*>(p.C) + (size_t)b * kN * L;

  if (MODE == kLocal) pdl_trigger();  // the carry scan may launch and wait for this grid
  f2_t A2[NP], h[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    const float* a = p.A + (size_t)dd * kN + SPL * j + 2 * q;
    A2[q] = pk2(a[0] * kLog2e, a[1] * kLog2e);
  }
  const float Dd = p.D ? p.D[dd] : 0.f;
  const float bias = p.bias ? p.bias[dd] : 0.f;

  const size_t st_idx = ((size_t)b * p.dim + dd) * kN + SPL * j;
  const size_t seg_stride = (size_t)p.batch * p.dim * kN;
#pragma unroll
  for (int q = 0; q < NP; ++q) h[q] = pk2(0.f, 0.f);
  // the state entering the segment: h0, or (chunk-parallel) the carry scan's
  // output, read after pdl_wait() in the first tile
  auto load_hin = [&]() {
    const float* src = nullptr;
    if (MODE == kFull && p.nseg > 1 && seg > 0) src = p.seg_hin + seg * seg_stride + st_idx;
    else if (MODE == kFull && seg == 0 && p.h0) src = p.h0 + st_idx;
    if (src) {
#pragma unroll
      for (int q = 0; q < NP; ++q) h[q] = pk2(src[2 * q], src[2 * q + 1]);
    }
  };
  if (MODE == kFull && p.nseg == 1) load_hin();
  float dsum = 0.f;
  unsigned seg_rst = 0;  // any document start inside this segment
  const int* seq_row = p.seq_idx ? p.seq_idx + (size_t)b * L : nullptr;

  // B / C staging: 128 threads = 2 arrays x 16 rows x 4 groups of 8 steps
  const int g_which = tid >> 6, g_n = (tid >> 2) & 15, g_tg = tid & 3;
  const T* __restrict__ g_src = (g_which ? Cb : Bb) + (size_t)g_n * L;
  const bool g_active = !(MODE == kLocal && g_which == 1);

  RawVec<T, PS> ru, rx, rz;
  RawVec<T, 8> rbc;
  rz.zero();
  rbc.zero();
  auto fetch = [&](int t0) {
    const int t = t0 + PS * j;
    ru.template load<VEC>(u_row, t, t_end);
    rx.template load<VEC>(x_row, t, t_end);
    if (MODE == kFull && z_row) rz.template load<VEC>(z_row, t, t_end);
    if (g_active) rbc.template load<VEC>(g_src, t0 + 8 * g_tg, t_end);
  };
  fetch(t_begin);

  for (int t0 = t_begin; t0 < t_end; t0 += TT) {
    // ---- per-token prologue from the prefetched tile
    float gate[PS], dsk[PS];
    {
      float uv[PS], xv[PS], zv[PS];
      ru.unpack(uv);
      rx.unpack(xv);
      if (MODE == kFull && z_row) rz.unpack(zv);
      const int t = t0 + PS * j;
#pragma unroll
      for (int i = 0; i < PS; ++i) {
        const bool ok = dvalid && (t + i < t_end);
        const float x = xv[i] + bias;
        float dt = p.softplus ? softplus_f(x) : x;
        dt = ok ? dt : 0.f;
        const float du = dt * uv[i];
        s_dt2[c][PS * j + i] = pk2(dt, dt);
        s_du2[c][PS * j + i] = pk2(du, du);
        if (MODE == kFull) {
          gate[i] = z_row ? zv[i] * sigmoid_f(zv[i]) : 1.f;
          dsk[i] = Dd * uv[i];
        }
      }
      if (g_active) {
        float v[8];
        rbc.unpack(v);
        float(*dst)[kN] = g_which ? s_C : s_B;
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[8 * g_tg + i][g_n] = v[i];
      }
    }
    if (t0 + TT < t_end) fetch(t0 + TT);  // next tile's loads fly during this scan
    // steps of this tile that start a new document: their decay is zero
    const unsigned rst = SEQ ? doc_starts32(seq_row, t0, t_end) : 0u;
    if (MODE == kLocal) seg_rst |= rst;
    if (MODE == kFull && p.nseg > 1 && t0 == t_begin) {
      pdl_wait();  // the carry scan has completed
      load_hin();
    }
    __syncthreads();

    // ---- the scan: NP state pairs per lane
#pragma unroll kFwdUnroll
    for (int tt = 0; tt < TT; tt += 4) {
      float acc[4];
#if SS_FWD_DECAYS_FIRST
      // issue the group's 4 x NP decay pairs (SFU) before its recurrence FMAs
      f2_t ag[4][NP], bug[4][NP];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const f2_t dt2 = s_dt2[c][tt + qq];
        const f2_t du2 = s_du2[c][tt + qq];
        f2_t Bp[NP];
        if constexpr (NP == 2) {
          const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(&s_B[tt + qq][SPL * j]);
          Bp[0] = v.x; Bp[1] = v.y;
        } else {
          Bp[0] = *reinterpret_cast<const f2_t*>(&s_B[tt + qq][SPL * j]);
        }
#pragma unroll
        for (int q = 0; q < NP; ++q) {
          ag[qq][q] = ex2_2(mul2(dt2, A2[q]));
          if (rst & (1u << (tt + qq))) ag[qq][q] = pk2(0.f, 0.f);
          bug[qq][q] = mul2(du2, Bp[q]);
        }
        if (MODE == kLocal) dsum += lo2(dt2);
      }
#endif
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
#if SS_FWD_DECAYS_FIRST
#pragma unroll
        for (int q = 0; q < NP; ++q) h[q] = fma2(ag[qq][q], h[q], bug[qq][q]);
#else
        const f2_t dt2 = s_dt2[c][tt + qq];
        const f2_t du2 = s_du2[c][tt + qq];
        f2_t Bp[NP];
        if constexpr (NP == 2) {
          const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(&s_B[tt + qq][SPL * j]);
          Bp[0] = v.x; Bp[1] = v.y;
        } else {
          Bp[0] = *reinterpret_cast<const f2_t*>(&s_B[tt + qq][SPL * j]);
        }
#pragma unroll
        for (int q = 0; q < NP; ++q) {
          f2_t a = ex2_2(mul2(dt2, A2[q]));
          if (rst & (1u << (tt + qq))) a = pk2(0.f, 0.f);
          h[q] = fma2(a, h[q], mul2(du2, Bp[q]));
        }
        if (MODE == kLocal) dsum += lo2(dt2);
#endif
        if (MODE == kFull) {
          f2_t Cp[NP];
          if constexpr (NP == 2) {
            const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(&s_C[tt + qq][SPL * j]);
            Cp[0] = v.x; Cp[1] = v.y;
          } else {
            Cp[0] = *reinterpret_cast<const f2_t*>(&s_C[tt + qq][SPL * j]);
          }
          f2_t r = mul2(Cp[0], h[0]);
#pragma unroll
          for (int q = 1; q < NP; ++q) r = fma2(Cp[q], h[q], r);
          acc[qq] = lo2(r) + hi2(r);
        }
      }
      if (MODE == kFull)
        *reinterpret_cast<float4*>(&s_yp[c][j][tt]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }

    if (MODE == kFull && p.ckpt && dvalid) {
      const int tlast = min(t0 + TT, t_end) - 1;
      if ((tlast % kChunk) == kChunk - 1 || tlast == L - 1) {
        float* dst = p.ckpt + (((size_t)b * p.dim + d) * p.nchunk + tlast / kChunk) * kN + SPL * j;
#pragma unroll
        for (int q = 0; q < NP; ++q)
          *reinterpret_cast<float2*>(dst + 2 * q) = make_float2(lo2(h[q]), hi2(h[q]));
      }
    }
    __syncthreads();

    // ---- epilogue: sum the K lanes' readouts, skip, gate, store y
    if (MODE == kFull) {
      float yv[PS];
#pragma unroll
      for (int i = 0; i < PS; i += 4) {
        const ulonglong2* p0 = reinterpret_cast<const ulonglong2*>(&s_yp[c][0][PS * j + i]);
        f2_t s0 = p0->x, s1 = p0->y;
#pragma unroll
        for (int l = 1; l < K; ++l) {
          const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(&s_yp[c][l][PS * j + i]);
          s0 = add2(s0, v.x);
          s1 = add2(s1, v.y);
        }
        yv[i + 0] = lo2(s0); yv[i + 1] = hi2(s0);
        yv[i + 2] = lo2(s1); yv[i + 3] = hi2(s1);
      }
#pragma unroll
      for (int i = 0; i < PS; ++i) yv[i] = (yv[i] + dsk[i]) * gate[i];
      if (dvalid) store_row<T, PS, VEC>(static_cast<T*>(p.y) + row, t0 + PS * j, t_end, yv);
    }
  }

  if (!dvalid) return;
  if (MODE == kFull) {
    if (t_end == L && p.final_state) {
#pragma unroll
      for (int q = 0; q < NP; ++q)
        *reinterpret_cast<float2*>(p.final_state + st_idx + 2 * q) = make_float2(lo2(h[q]), hi2(h[q]));
    }
  } else {
    const size_t o = seg * seg_stride + st_idx;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      *reinterpret_cast<float2*>(p.seg_end + o + 2 * q) = make_float2(lo2(h[q]), hi2(h[q]));
      // product of the segment's decays: prod_t exp(Delta_t A) = exp(A sum_t Delta_t),
      // zero when a document starts inside the segment
      *reinterpret_cast<float2*>(p.seg_decay + o + 2 * q) =
          seg_rst ? make_float2(0.f, 0.f) : make_float2(ex2(lo2(A2[q]) * dsum), ex2(hi2(A2[q]) * dsum));
    }
  }
}

// Forward scan with two channels per 4-lane group (one warp = 16 channels).
// Shared-memory bandwidth bounds the one-channel scan: each lane reads B_t
// and C_t for its 4 states every step, so every channel pays for its own
// copy.  Here one B_t / C_t load serves two channels, and the per-step
// tokens (Delta, Delta u) are kept once per channel and duplicated into fp32
// pairs in registers.  Tiles are 16 steps; a one-warp block synchronises
// with warp barriers.
#ifndef SS_FWD2_MIN_BLOCKS
#define SS_FWD2_MIN_BLOCKS 12
#endif
template <typename T, bool VEC, int MODE, bool SEQ>
__global__ void __launch_bounds__(32, SS_FWD2_MIN_BLOCKS)
fwd2_kernel(const FwdParams p) {
  constexpr int CB = 16;                 // channels per block
  constexpr int T2 = 16;                 // steps per tile
  constexpr int PS = 8;                  // steps per thread in prologue / epilogue
  constexpr int NP = 2;                  // fp32 pairs per channel per lane (4 states)
  constexpr int TKS = T2 + 1;            // s_tk channel stride (f2_t, padded)
  constexpr int YPS = T2 + 4;            // s_yp lane stride (floats, padded)
  __shared__ __align__(16) f2_t s_tk[CB * TKS];          // (Delta, Delta u) per (channel, step)
  // B_t in columns 0-15 and C_t in 16-31 of one row: the two staging
  // half-warps' transposed stores of a step fill all 32 banks
  __shared__ __align__(16) float s_BC[T2][2 * kN];
  __shared__ __align__(16) float s_yp[CB][4][YPS];       // per-lane partial C.h

  const int tid = threadIdx.x;
  const int pr = tid >> 2, j = tid & 3;   // scan role: channels 2pr, 2pr+1, states 4j..4j+3
  const int ce = tid >> 1, hf = tid & 1;  // prologue / epilogue role: channel ce, steps 8hf..8hf+7
  const int b = blockIdx.y, seg = blockIdx.z;
  const int dbase = blockIdx.x * CB;
  const int L = p.seqlen;
  const int t_begin = seg * p.seg_len;
  const int t_end = min(L, t_begin + p.seg_len);

  // prologue / epilogue role
  const int dE = dbase + ce;
  const bool eval = dE < p.dim;
  const int ddE = eval ? dE : 0;
  const size_t rowE = ((size_t)b * p.dim + ddE) * (size_t)L;
  const T* __restrict__ u_row = static_cast<const T*>(p.u) + rowE;
  const T* __restrict__ x_row = static_cast<const T*>(p.delta) + rowE;
  const T* __restrict__ z_row = p.z ? static_cast<const T*>(p.z) + rowE : nullptr;
  const float DdE = p.D ? p.D[ddE] : 0.f;
  const float biasE = p.bias ? p.bias[ddE] : 0.f;

  // scan role
  const size_t seg_stride = (size_t)p.batch * p.dim * kN;
  f2_t A2[2][NP], h[2][NP];
  float dsum[2] = {0.f, 0.f};
  unsigned seg_rst = 0;  // any document start inside this segment
  const int* seq_row = p.seq_idx ? p.seq_idx + (size_t)b * L : nullptr;
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const int d = dbase + 2 * pr + ch;
    const int dd = d < p.dim ? d : 0;
    const float* a = p.A + (size_t)dd * kN + 4 * j;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      A2[ch][q] = pk2(a[2 * q] * kLog2e, a[2 * q + 1] * kLog2e);
      h[ch][q] = pk2(0.f, 0.f);
    }
    if (MODE == kFull && p.nseg > 1 && seg > 0) {
      const float* src = p.seg_hin + seg * seg_stride + ((size_t)b * p.dim + dd) * kN + 4 * j;
#pragma unroll
      for (int q = 0; q < NP; ++q) h[ch][q] = pk2(src[2 * q], src[2 * q + 1]);
    } else if (MODE == kFull && seg == 0 && p.h0) {
      const float* src = p.h0 + ((size_t)b * p.dim + dd) * kN + 4 * j;
#pragma unroll
      for (int q = 0; q < NP; ++q) h[ch][q] = pk2(src[2 * q], src[2 * q + 1]);
    }
  }

  // B / C staging: thread (array, n) stages a 16-step piece of its row
  const int g_which = tid >> 4, g_n = tid & 15;
  const T* __restrict__ g_src = static_cast<const T*>(g_which ? p.C : p.B) + ((size_t)b * kN + g_n) * L;
  const bool g_active = !(MODE == kLocal && g_which == 1);

  RawVec<T, PS> ru, rx, rz;
  RawVec<T, T2> rbc;
  rz.zero();
  rbc.zero();
  auto fetch = [&](int t0) {
    const int t = t0 + PS * hf;
    ru.template load<VEC>(u_row, t, t_end);
    rx.template load<VEC>(x_row, t, t_end);
    if (MODE == kFull && z_row) rz.template load<VEC>(z_row, t, t_end);
    if (g_active) rbc.template load<VEC>(g_src, t0, t_end);
  };
  fetch(t_begin);

  auto dup_lo = [](f2_t v) { return pk2(lo2(v), lo2(v)); };
  auto dup_hi = [](f2_t v) { return pk2(hi2(v), hi2(v)); };

  for (int t0 = t_begin; t0 < t_end; t0 += T2) {
    // ---- per-token prologue from the prefetched tile
    float gate[PS], dsk[PS];
    {
      float uv[PS], xv[PS], zv[PS];
      ru.unpack(uv);
      rx.unpack(xv);
      if (MODE == kFull && z_row) rz.unpack(zv);
#pragma unroll
      for (int i = 0; i < PS; ++i) {
        const int tt = PS * hf + i;
        const bool ok = eval && (t0 + tt < t_end);
        const float x = xv[i] + biasE;
        float dt = p.softplus ? softplus_f(x) : x;
        dt = ok ? dt : 0.f;
        s_tk[ce * TKS + tt] = pk2(dt, dt * uv[i]);
        if (MODE == kFull) {
          gate[i] = z_row ? zv[i] * sigmoid_f(zv[i]) : 1.f;
          dsk[i] = DdE * uv[i];
        }
      }
      if (g_active) {
        float v[T2];
        rbc.unpack(v);
#pragma unroll
        for (int i = 0; i < T2; ++i) s_BC[i][kN * g_which + g_n] = v[i];
      }
    }
    if (t0 + T2 < t_end) fetch(t0 + T2);  // next tile's loads fly during this scan
    // steps of this tile that start a new document: their decay is zero
    const unsigned rst = SEQ ? doc_starts32(seq_row, t0, min(t_end, t0 + T2)) : 0u;
    if (MODE == kLocal) seg_rst |= rst;
    __syncwarp();

    // ---- the scan: 2 channels x 2 state pairs per lane
#pragma unroll
    for (int tg = 0; tg < T2; tg += 4) {
      float acc[2][4];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const int i = tg + qq;
        f2_t tk[2];
        tk[0] = s_tk[(2 * pr) * TKS + i];  // left to the compiler's schedule
        tk[1] = s_tk[(2 * pr + 1) * TKS + i];
        const ulonglong2 bp = *reinterpret_cast<const ulonglong2*>(&s_BC[i][4 * j]);
        const f2_t Bp[NP] = {bp.x, bp.y};
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const f2_t dt2 = dup_lo(tk[ch]), du2 = dup_hi(tk[ch]);
#pragma unroll
          for (int q = 0; q < NP; ++q) {
            f2_t a = ex2_2(mul2(dt2, A2[ch][q]));
            if (rst & (1u << i)) a = pk2(0.f, 0.f);
            h[ch][q] = fma2(a, h[ch][q], mul2(du2, Bp[q]));
          }
          if (MODE == kLocal) dsum[ch] += lo2(tk[ch]);
        }
        if (MODE == kFull) {
          const ulonglong2 cp = *reinterpret_cast<const ulonglong2*>(&s_BC[i][kN + 4 * j]);
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const f2_t r = fma2(cp.y, h[ch][1], mul2(cp.x, h[ch][0]));
            acc[ch][qq] = lo2(r) + hi2(r);
          }
        }
      }
      if (MODE == kFull) {
#pragma unroll
        for (int ch = 0; ch < 2; ++ch)
          *reinterpret_cast<float4*>(&s_yp[2 * pr + ch][j][tg]) =
              make_float4(acc[ch][0], acc[ch][1], acc[ch][2], acc[ch][3]);
      }
    }

    if (MODE == kFull && p.ckpt) {
      const int tlast = min(t0 + T2, t_end) - 1;
      if ((tlast % kChunk) == kChunk - 1 || tlast == L - 1) {
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int d = dbase + 2 * pr + ch;
          if (d < p.dim) {
            float* dst = p.ckpt + (((size_t)b * p.dim + d) * p.nchunk + tlast / kChunk) * kN + 4 * j;
            *reinterpret_cast<float4*>(dst) =
                make_float4(lo2(h[ch][0]), hi2(h[ch][0]), lo2(h[ch][1]), hi2(h[ch][1]));
          }
        }
      }
    }
    __syncwarp();

    // ---- epilogue: sum the 4 lanes' readouts, skip, gate, store y
    if (MODE == kFull) {
      float yv[PS];
#pragma unroll
      for (int i = 0; i < PS; i += 4) {
        const ulonglong2* p0 = reinterpret_cast<const ulonglong2*>(&s_yp[ce][0][PS * hf + i]);
        f2_t s0 = p0->x, s1 = p0->y;
#pragma unroll
        for (int l = 1; l < 4; ++l) {
          const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(&s_yp[ce][l][PS * hf + i]);
          s0 = add2(s0, v.x);
          s1 = add2(s1, v.y);
        }
        yv[i + 0] = lo2(s0); yv[i + 1] = hi2(s0);
        yv[i + 2] = lo2(s1); yv[i + 3] = hi2(s1);
      }
#pragma unroll
      for (int i = 0; i < PS; ++i) yv[i] = (yv[i] + dsk[i]) * gate[i];
      if (eval) store_row<T, PS, VEC>(static_cast<T*>(p.y) + rowE, t0 + PS * hf, t_end, yv);
    }
  }

#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const int d = dbase + 2 * pr + ch;
    if (d >= p.dim) continue;
    const size_t st_idx = ((size_t)b * p.dim + d) * kN + 4 * j;
    if (MODE == kFull) {
      if (t_end == L && p.final_state)
        *reinterpret_cast<float4*>(p.final_state + st_idx) =
            make_float4(lo2(h[ch][0]), hi2(h[ch][0]), lo2(h[ch][1]), hi2(h[ch][1]));
    } else {
      const size_t o = seg * seg_stride + st_idx;
      *reinterpret_cast<float4*>(p.seg_end + o) =
          make_float4(lo2(h[ch][0]), hi2(h[ch][0]), lo2(h[ch][1]), hi2(h[ch][1]));
      // product of the segment's decays: prod_t exp(Delta_t A) = exp(A sum_t Delta_t),
      // zero when a document starts inside the segment
      *reinterpret_cast<float4*>(p.seg_decay + o) =
          seg_rst ? make_float4(0.f, 0.f, 0.f, 0.f)
                  : make_float4(ex2(lo2(A2[ch][0]) * dsum[ch]), ex2(hi2(A2[ch][0]) * dsum[ch]),
                                ex2(lo2(A2[ch][1]) * dsum[ch]), ex2(hi2(A2[ch][1]) * dsum[ch]));
    }
  }
}

// Phase 2 of the chunk-parallel path: for every (b, d, n) compose the segment
// maps h -> P_s h + e_s in order and write the state entering each segment.
// A warp holds 8 consecutive (b, d, n) entries x 4 segment slabs (lane =
// 8 slab + entry), so a load of one segment's maps reads whole 32-byte
// sectors; a block's warps hold consecutive slabs of the same 8 entries, and
// a block covers all the segments.  Each thread folds its slab (contiguous
// segments) into one (a, e) pair; a 2-step shuffle scan composes the warp's 4
// slabs, the warps' totals are composed in order through shared memory from
// h0, and each thread re-walks its slab from the state entering it.
// CACHE > 0: a thread keeps its (at most CACHE) segment maps in registers, so
// the loads are one round of independent loads and the re-walk reads
// registers; the launcher picks the smallest CACHE that holds a slab.  CACHE
// = 0 re-reads the maps from global memory.
constexpr int kCarryEntries = 8;                  // entries per warp
constexpr int kCarrySlabs = 32 / kCarryEntries;   // slabs per warp
constexpr int kCarryMaxWarps = 32;

template <int CACHE>
__global__ void __launch_bounds__(32 * kCarryMaxWarps)
carry_scan_kernel(const FwdParams p, const int per) {
  constexpr int kCache = CACHE > 0 ? CACHE : 1;
  constexpr int E = kCarryEntries;
  __shared__ float s_a[kCarryMaxWarps][E], s_e[kCarryMaxWarps][E];
  pdl_wait();     // the local pass has completed
  pdl_trigger();  // the full pass may launch: it loads its first tile while this runs
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int ent = lane % E, sl = lane / E;        // entry within the warp, slab within the warp
  const long long ntrip = (long long)p.batch * p.dim * kN;
  const long long tr = (long long)blockIdx.x * E + ent;
  const bool live_tr = tr < ntrip;
  const size_t stride = (size_t)ntrip;
  const size_t col = live_tr ? (size_t)tr : 0;
  const int nmap = p.nseg - 1;  // the last segment's map is never applied
  const int slab = w * kCarrySlabs + sl;
  const int s_lo = min(p.nseg, slab * per), s_hi = min(p.nseg, s_lo + per);
  float cP[kCache], cE[kCache];
  float a = 1.f, e = 0.f;
  if (CACHE > 0) {
#pragma unroll
    for (int k = 0; k < kCache; ++k) {
      const int s = s_lo + k;
      const bool live = live_tr && s < s_hi && s < nmap;
      cP[k] = live ? p.seg_decay[s * stride + col] : 1.f;
      cE[k] = live ? p.seg_end[s * stride + col] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kCache; ++k) {
      e = fmaf(cP[k], e, cE[k]);
      a = cP[k] * a;
    }
  } else if (live_tr) {
    for (int s = s_lo; s < min(s_hi, nmap); ++s) {
      const float P = p.seg_decay[s * stride + col];
      e = fmaf(P, e, p.seg_end[s * stride + col]);
      a = P * a;
    }
  }
  // inclusive scan over the warp's slabs of the same entry (lanes E apart)
#pragma unroll
  for (int off = 1; off < kCarrySlabs; off <<= 1) {
    const float a_up = __shfl_up_sync(0xffffffffu, a, off * E);
    const float e_up = __shfl_up_sync(0xffffffffu, e, off * E);
    if (sl >= off) {
      e = fmaf(a, e_up, e);
      a = a * a_up;
    }
  }
  if (sl == kCarrySlabs - 1) {  // the warp's total map
    s_a[w][ent] = a;
    s_e[w][ent] = e;
  }
  // exclusive prefix within the warp (identity for the first slab)
  float a_ex = __shfl_up_sync(0xffffffffu, a, E);
  float e_ex = __shfl_up_sync(0xffffffffu, e, E);
  if (sl == 0) { a_ex = 1.f; e_ex = 0.f; }
  __syncthreads();
  if (w == 0 && sl == 0) {
    // the state entering each warp's first slab, composed in warp order from h0
    float h = (p.h0 && live_tr) ? p.h0[col] : 0.f;
    for (int k = 0; k < nw; ++k) {
      const float ak = s_a[k][ent], ek = s_e[k][ent];
      s_e[k][ent] = h;
      h = fmaf(ak, h, ek);
    }
  }
  __syncthreads();
  if (!live_tr) return;
  float hin = fmaf(a_ex, s_e[w][ent], e_ex);
  if (CACHE > 0) {
#pragma unroll
    for (int k = 0; k < kCache; ++k) {
      const int s = s_lo + k;
      if (s < s_hi) p.seg_hin[s * stride + col] = hin;
      hin = fmaf(cP[k], hin, cE[k]);
    }
  } else {
    for (int s = s_lo; s < s_hi; ++s) {
      p.seg_hin[s * stride + col] = hin;
      if (s < nmap) hin = fmaf(p.seg_decay[s * stride + col], hin, p.seg_end[s * stride + col]);
    }
  }
}

// Launch with programmatic stream serialisation: the kernel may start before
// the previous kernel in the stream completes, and must pdl_wait() before it
// touches that kernel's results.
template <typename... Args>
cudaError_t launch_pdl(void (*kernel)(Args...), dim3 grid, dim3 block, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_carry_scan(const FwdParams& p, cudaStream_t s) {
  const long long ntrip = (long long)p.batch * p.dim * kN;
  int nw = (p.nseg + kCarrySlabs - 1) / kCarrySlabs;  // warps: one slab per segment if they suffice
  if (nw > kCarryMaxWarps) nw = kCarryMaxWarps;
  const int per = (p.nseg + nw * kCarrySlabs - 1) / (nw * kCarrySlabs);  // segments per slab
  const dim3 blocks((unsigned)((ntrip + kCarryEntries - 1) / kCarryEntries)), threads(32 * nw);
  if (per <= 1) return launch_pdl(carry_scan_kernel<1>, blocks, threads, s, p, per);
  if (per <= 4) return launch_pdl(carry_scan_kernel<4>, blocks, threads, s, p, per);
  if (per <= 16) return launch_pdl(carry_scan_kernel<16>, blocks, threads, s, p, per);
  if (per <= 32) return launch_pdl(carry_scan_kernel<32>, blocks, threads, s, p, per);
  return launch_pdl(carry_scan_kernel<0>, blocks, threads, s, p, per);
}

template <typename T, int K, bool VEC, bool SEQ>
cudaError_t launch_fwd_k(const FwdParams& p, cudaStream_t s) {
  constexpr int CB = 128 / K;
  const dim3 block(128);
  const dim3 g((p.dim + CB - 1) / CB, p.batch, p.nseg);
  const long long blocks = (long long)g.x * g.y * g.z;
  auto full = (K == 4 && blocks > 4LL * p.sms && blocks <= 5LL * p.sms)
                  ? fwd_kernel<T, K, CB, VEC, kFull, 5, SEQ>
                  : fwd_kernel<T, K, CB, VEC, kFull, K == 4 ? 4 : 7, SEQ>;
  if (p.nseg > 1) {
    // local pass -> carry scan -> full pass, each launched while the one
    // before it still runs (programmatic dependent launch)
    const dim3 g1((p.dim + CB - 1) / CB, p.batch, p.nseg - 1);
    fwd_kernel<T, K, CB, VEC, kLocal, K == 4 ? 4 : 7, SEQ><<<g1, block, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = launch_carry_scan(p, s);
    if (e == cudaSuccess) e = launch_pdl(full, g, block, s, p);
    return e;
  }
  full<<<g, block, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T, bool VEC, bool SEQ>
cudaError_t launch_fwd2(const FwdParams& p, cudaStream_t s) {
  constexpr int CB = 16;
  if (p.nseg > 1) {
    // (the pair scan has no pdl_wait(): its full pass follows the carry scan
    // in plain stream order)
    const dim3 g1((p.dim + CB - 1) / CB, p.batch, p.nseg - 1);
    fwd2_kernel<T, VEC, kLocal, SEQ><<<g1, 32, 0, s>>>(p);
    const cudaError_t e = launch_carry_scan(p, s);
    if (e != cudaSuccess) return e;
  }
  const dim3 g((p.dim + CB - 1) / CB, p.batch, p.nseg);
  fwd2_kernel<T, VEC, kFull, SEQ><<<g, 32, 0, s>>>(p);
  return cudaGetLastError();
}

// Two channels per lane group pay off once every SM holds eight or more of
// their one-warp blocks (128 channels per SM); below that the one-channel
// scan keeps more warps in flight.
bool use_fwd2(const FwdParams& p) {
#ifdef SS_FWD_PAIRS
  return SS_FWD_PAIRS && p.lanes == 4;
#else
  return p.lanes == 4 && p.nseg == 1 && (long long)p.batch * p.dim >= 128LL * p.sms;
#endif
}

template <typename T, bool SEQ>
cudaError_t launch_fwd_s(const FwdParams& p, bool vec, cudaStream_t s) {
  if (use_fwd2(p))
    return vec ? launch_fwd2<T, true, SEQ>(p, s) : launch_fwd2<T, false, SEQ>(p, s);
  if (p.lanes == 8)
    return vec ? launch_fwd_k<T, 8, true, SEQ>(p, s) : launch_fwd_k<T, 8, false, SEQ>(p, s);
  return vec ? launch_fwd_k<T, 4, true, SEQ>(p, s) : launch_fwd_k<T, 4, false, SEQ>(p, s);
}

// packed documents get the document-aware kernels; plain rows skip the checks
template <typename T>
cudaError_t launch_fwd_t(const FwdParams& p, bool vec, cudaStream_t s) {
  return p.seq_idx ? launch_fwd_s<T, true>(p, vec, s) : launch_fwd_s<T, false>(p, vec, s);
}

}  // namespace

cudaError_t launch_fwd(const FwdParams& p, DType dt, bool vec, cudaStream_t s) {
  switch (dt) {
    case DType::F32: return launch_fwd_t<float>(p, vec, s);
    case DType::BF16: return launch_fwd_t<__nv_bfloat16>(p, vec, s);
    case DType::F16: return launch_fwd_t<__half>(p, vec, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ss
