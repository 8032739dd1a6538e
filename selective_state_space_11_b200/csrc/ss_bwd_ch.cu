// ss_bwd_ch.cu -- backward selective scan (S6), one thread per channel (sm_100a).
//
// The adjoint of the forward scan for the loss <dy, y> ("Mamba",
// stanleyjacob.dev, Part IV Stage 7: recompute the states instead of storing
// them, then accumulate the gradients of u, Delta, A, B, C, D, z).  With
// g_t = dloss/dh_t and dout_t = dy_t SiLU(z_t):
//   g_t    = Abar_{t+1} g_{t+1} + dout_t C_t
//   dC_t   = sum_d dout_t h_t                 dB_t = sum_d g_t Delta_t u_t
//   du_t   = dout_t D + Delta_t sum_n g_t B_t
//   dDelta = u_t sum_n g_t B_t + sum_n A g_t Abar_t h_{t-1}
//   dA    += Delta_t g_t Abar_t h_{t-1}
//   ddelta = dDelta sigmoid(delta + bias) (softplus on), dbias = sum ddelta
//   dz     = dy (C.h + D u) SiLU'(z),          dD = sum dout u
//
// Work decomposition.  A thread owns one channel and all 16 of its states
// (as eight fp32 pairs, so the FP32 pipe retires two states per instruction),
// 32 channels of one batch row per warp, 128 per block.  Sums over the state
// index (du, dDelta, the recomputed readout for dz) stay in registers; B_t and
// C_t are read from shared memory by every lane of the block; the channel
// sums of dB and dC are a warp reduce-scatter followed by a fixed-order sum of
// the block's four warps.
//
//   1. ch_states_kernel: one block per (128 channels, 64-step chunk, batch
//      row), all chunks in parallel.  From the forward's checkpoint it
//      recomputes the chunk and records the state entering every 4-step
//      sub-chunk (workspace), and forms dC (dout_t h_t summed over channels).
//      For chunks whose carry map is needed (chunk groups after the first) it
//      also composes the chunk's map of the reverse gradient carry
//      c -> P_k c + e_k, P_k = prod_t Abar_t, e_k = sum_s (prod_{r<=s} Abar_r)
//      dout_s C_s, from the decays it forms anyway.
//   2. ch_carry_kernel: composes those maps from the last chunk backwards into
//      the carry entering each chunk group.
//   3. ch_walk_kernel: per block of channels and chunk group, the 8-step
//      tiles latest first ("Mamba, on a laptop GPU.", "The state lives in
//      registers": walk the chunks in reverse, carry the state gradient in
//      registers).  Each 4-step half-tile is recomputed forward from its
//      stored entering state into registers (states and decays), then walked
//      backwards.  The next tile's rows are copied to shared memory with
//      cp.async while the current one is processed.
//   4. ch_reduce_bc_kernel, ch_reduce_param_kernel: dB, dC summed over the
//      channel blocks, dA, dD, dbias over (chunk group, batch row), in a fixed
//      order (no floating-point atomics: results are bitwise reproducible).
//
// State slots.  Lane l keeps state pair (k ^ x) in its register pair k,
// x = (l >> 2) & 7, so the lanes hold the 16 states in different orders.  A
// warp reduce-scatter of 4 steps' per-state values (the channel sums of dB and
// dC) then sends and keeps the same registers in every lane for its first
// three levels (no selects; 64 values, 62 shuffles, every level wide enough to
// overlap its latencies), and ends with lane l holding the warp sum of state
// pair x at step l & 3.  B_t, C_t rows sit in shared memory twice, in natural
// order and with the two pairs of every float4 swapped (the second copy 16
// bytes further on, clear of the first copy's banks), so a lane's slots are
// four 128-bit loads whatever its x.  The workspace keeps per-channel states in
// slot order too, laid out [pair][channel][2]: a warp's 32 channels store or
// load one pair with a single 256-byte access.  Loads and stores of the
// caller's per-state arrays (checkpoints, h0, dfinal, dA, dh0) apply the
// permutation.
#include <cstddef>

#include "ss_device.cuh"
#include "ss_internal.h"

namespace ss {
namespace {

constexpr int CB = kChBlock;     // channels (threads) per block
constexpr int NW = CB / 32;      // warps per block
constexpr int TS = kChSub;       // steps per stored sub-chunk state (4)
constexpr int TL = 8;            // steps per staged tile (two sub-chunks)
constexpr float kLn2f = 0.6931471805599453f;
static_assert(TS == 4, "the reduce-scatter covers 4 steps");

__device__ __forceinline__ f2_t shfl_xor2(f2_t v, int m) {
  return __shfl_xor_sync(0xffffffffu, v, m);
}
__device__ __forceinline__ f2_t sel2(bool c, f2_t a, f2_t b) { return c ? a : b; }

// Warp sums over the 32 lanes (channels) of per-state values of 4 steps held
// in state slots.  Lane l receives the sum of state pair (l >> 2) & 7 at step
// l & 3.  The order of the additions is fixed, so results are reproducible.
__device__ __forceinline__ f2_t warp_sum4(f2_t (&v)[TS][8], int lane) {
#pragma unroll
  for (int s = 0; s < TS; ++s)
#pragma unroll
    for (int k = 0; k < 4; ++k) v[s][k] = add2(v[s][k], shfl_xor2(v[s][k + 4], 16));
#pragma unroll
  for (int s = 0; s < TS; ++s)
#pragma unroll
    for (int k = 0; k < 2; ++k) v[s][k] = add2(v[s][k], shfl_xor2(v[s][k + 2], 8));
#pragma unroll
  for (int s = 0; s < TS; ++s) v[s][0] = add2(v[s][0], shfl_xor2(v[s][1], 4));
  const bool b1 = (lane >> 1) & 1, b0 = lane & 1;
  f2_t k0 = sel2(b1, v[2][0], v[0][0]), k1 = sel2(b1, v[3][0], v[1][0]);
  const f2_t s0 = sel2(b1, v[0][0], v[2][0]), s1 = sel2(b1, v[1][0], v[3][0]);
  k0 = add2(k0, shfl_xor2(s0, 2));
  k1 = add2(k1, shfl_xor2(s1, 2));
  return add2(sel2(b0, k1, k0), shfl_xor2(sel2(b0, k0, k1), 1));
}

// The same over 2 steps: lane l receives the sum of state pair (l >> 2) & 7
// at step (l >> 1) & 1 (lanes l and l ^ 1 agree).
__device__ __forceinline__ f2_t warp_sum2(f2_t (&v)[2][8], int lane) {
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int k = 0; k < 4; ++k) v[s][k] = add2(v[s][k], shfl_xor2(v[s][k + 4], 16));
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int k = 0; k < 2; ++k) v[s][k] = add2(v[s][k], shfl_xor2(v[s][k + 2], 8));
#pragma unroll
  for (int s = 0; s < 2; ++s) v[s][0] = add2(v[s][0], shfl_xor2(v[s][1], 4));
  const bool b1 = (lane >> 1) & 1;
  const f2_t k = add2(sel2(b1, v[1][0], v[0][0]), shfl_xor2(sel2(b1, v[0][0], v[1][0]), 2));
  return add2(k, shfl_xor2(k, 1));
}

// 16 per-state fp32 values at p (natural order) into / out of slot order.
__device__ __forceinline__ void load_slots(const float* p, int x, f2_t (&v)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = *reinterpret_cast<const f2_t*>(p + 2 * (k ^ x));
}
__device__ __forceinline__ void store_slots(float* p, int x, const f2_t (&v)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) *reinterpret_cast<f2_t*>(p + 2 * (k ^ x)) = v[k];
}
// Per-channel state in the workspace's slot layout: pair k of channel d at
// base + (k * dim + d) * 2.
__device__ __forceinline__ void store_pairs(float* base, int dim, int d, const f2_t (&v)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) *reinterpret_cast<f2_t*>(base + ((size_t)k * dim + d) * 2) = v[k];
}
__device__ __forceinline__ void load_pairs(const float* base, int dim, int d, f2_t (&v)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = *reinterpret_cast<const f2_t*>(base + ((size_t)k * dim + d) * 2);
}
// One step's B_t (or C_t) in slot order, from the two shared copies of the row
// (`row` in copy 0; copy 1, `stride` floats later, has its float4 pairs swapped).
__device__ __forceinline__ void lds_slots(const float* row, int stride, int x, f2_t (&v)[8]) {
  const float* r = row + (x & 1) * stride;
#pragma unroll
  for (int G = 0; G < 4; ++G) {
    const ulonglong2 q = *reinterpret_cast<const ulonglong2*>(r + 4 * (G ^ (x >> 1)));
    v[2 * G] = q.x;
    v[2 * G + 1] = q.y;
  }
}
// Value of state n at step t into both copies of a [t][16] table.
__device__ __forceinline__ void sts_both(float* tab, int stride, int t, int n, float v) {
  tab[t * kN + n] = v;
  tab[stride + t * kN + (n ^ 2)] = v;   // the two pairs of each float4 swapped
}
// Sum of the 8 pairs' products a[k] * b[k] (+ c), in two chains of four.
__device__ __forceinline__ float dot8(const f2_t (&a)[8], const f2_t (&b)[8]) {
  f2_t e = mul2(a[0], b[0]), o = mul2(a[1], b[1]);
#pragma unroll
  for (int k = 2; k < 8; k += 2) {
    e = fma2(a[k], b[k], e);
    o = fma2(a[k + 1], b[k + 1], o);
  }
  const f2_t s = add2(e, o);
  return lo2(s) + hi2(s);
}

// Per-token scalars of one step: Delta (masked), sigma(x) for ddelta, the
// gate's dz factor and dout.  `ok` is false past the row's end or for a
// channel beyond d_inner: the step then has Delta = 0 (unit decay, no input)
// and dout = 0, which leaves every state and gradient unchanged.
struct Tok {
  float dt, sx, dzf, dout;
};
__device__ __forceinline__ Tok token(float xv, float zv, float gv, float bias, bool softplus,
                                     bool has_z, bool ok) {
  Tok k;
  const float x = xv + bias;
  float dt = x, sx = 1.f;
  if (softplus) {
    const float w = ex2(-fabsf(x) * kLog2e);
    dt = fmaxf(x, 0.f) + log1p_unit(w);
    const float r = rcp(1.f + w);
    sx = x >= 0.f ? r : w * r;
  }
  float gate = 1.f, dzf = 0.f;
  if (has_z) {
    const float sz = sigmoid_f(zv);
    gate = zv * sz;
    dzf = gv * sz * fmaf(zv, 1.f - sz, 1.f);
  }
  k.dt = ok ? dt : 0.f;
  k.sx = ok ? sx : 0.f;
  k.dzf = dzf;
  k.dout = ok ? gv * gate : 0.f;
  return k;
}

template <typename T>
__device__ __forceinline__ float elt_at(const void* row, int i) {
  return Elt<T>::to_f(reinterpret_cast<const T*>(row)[i]);
}

// Rows of u, delta, z, dy for a block's 128 channels, 32 bytes of each row
// (16 steps of 16-bit data, 8 of fp32): [array][channel][16-byte half].  The
// block copies them together, consecutive threads taking consecutive halves,
// so a warp's copy reads 16 rows of 32 bytes; half q of row r sits in slot
// q ^ ((r >> 2) & 1), which spreads the rows a quarter-warp reads over the banks.
template <typename T>
struct RowStage {
  static constexpr int SL = 32 / (int)sizeof(T);    // steps per stage
  uint4 w[4][CB][2];
};

// Copy the stage starting at step t of channels [d0, d0 + 128) of batch row b
// (cp.async, zero-filled past the row end and past d_inner).  z may be absent.
template <typename T>
__device__ __forceinline__ void stage_rows(RowStage<T>& dst, const BwdParams& p, int b, int d0, int t, int tid) {
  constexpr int ES = (int)sizeof(T);
  const int rbytes = (p.seqlen - t) * ES;          // bytes of the row left from t
#pragma unroll
  for (int arr = 0; arr < 4; ++arr) {
    const void* base = arr == 0 ? p.u : arr == 1 ? p.delta : arr == 2 ? p.z : p.dy;
    if (!base) continue;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int c = tid + m * CB, r = c >> 1, q = c & 1;
      const int d = d0 + r;
      const int nb = d < p.dim ? max(0, min(16, rbytes - 16 * q)) : 0;
      const T* src = static_cast<const T*>(base) + ((size_t)b * p.dim + (d < p.dim ? d : 0)) * p.seqlen + t +
                     q * (16 / ES);
      cp_async16(&dst.w[arr][r][q ^ ((r >> 2) & 1)], nb > 0 ? (const void*)src : base, nb);
    }
  }
}

// The 4 values of array `arr` for steps [s, s + 4) of a stage (s a multiple of 4),
// row `tid`.
template <typename T>
__device__ __forceinline__ void stage_quad(const RowStage<T>& src, int arr, int s, int tid, float (&v)[TS]) {
  constexpr int ES = (int)sizeof(T);
  const int byte = s * ES, q = byte >> 4;
  const unsigned char* ptr =
      reinterpret_cast<const unsigned char*>(&src.w[arr][tid][q ^ ((tid >> 2) & 1)]) + (byte & 15);
  if constexpr (ES == 4) {
    const float4 f = *reinterpret_cast<const float4*>(ptr);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  } else {
    const uint2 r = *reinterpret_cast<const uint2*>(ptr);
    const T* e = reinterpret_cast<const T*>(&r);
#pragma unroll
    for (int i = 0; i < TS; ++i) v[i] = Elt<T>::to_f(e[i]);
  }
}

// =========================================================================
// 1. States pass.
// =========================================================================
#ifndef SS_CH_STATES_MINB
#define SS_CH_STATES_MINB 4
#endif
template <typename T, bool CARRY>
struct StatesSmem {
  RowStage<T> rows[2];           // the chunk's rows, a stage at a time (double-buffered)
  // every member a multiple of 16 bytes, so each starts 16-byte aligned
  float B[2 * kChunk * kN + 16]; // the chunk's B_t in fp32 [t][n], two copies (see lds_slots)
  float C[CARRY ? 2 * kChunk * kN + 16 : 4];
  __align__(16) float red[NW][TL][kN];   // per-warp dC sums of a tile
};

using StatesSmemF = StatesSmem<float, false>;
using StatesSmemFC = StatesSmem<float, true>;
using StatesSmemH = StatesSmem<__nv_bfloat16, false>;
using StatesSmemHC = StatesSmem<__nv_bfloat16, true>;
static_assert(offsetof(StatesSmemF, red) % 16 == 0 && offsetof(StatesSmemH, red) % 16 == 0 &&
              offsetof(StatesSmemFC, C) % 16 == 0 && offsetof(StatesSmemHC, red) % 16 == 0 &&
              offsetof(StatesSmemFC, red) % 16 == 0,
              "16-byte aligned shared members");

template <typename T, bool SEQ, bool CARRY>
__global__ void __launch_bounds__(CB, SS_CH_STATES_MINB) ch_states_kernel(const BwdParams p, int chunk0) {
  constexpr int ES = (int)sizeof(T);
  constexpr int EPP = 16 / ES;                 // elements per 16-byte piece
  constexpr int PPR = kChunk / EPP;            // pieces per 64-step row
  constexpr int NT = kChunk / TL;              // tiles per chunk
  extern __shared__ __align__(16) unsigned char ch_smem[];
  StatesSmem<T, CARRY>& S = *reinterpret_cast<StatesSmem<T, CARRY>*>(ch_smem);
  constexpr int BS = kChunk * kN + 16;         // offset of the second copy of B / C
  constexpr int SL = RowStage<T>::SL;          // steps per row stage
  constexpr int TPS = SL / TL;                 // tiles per row stage

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int x = (lane >> 2) & 7;
  const int d = blockIdx.x * CB + tid;
  const bool dvalid = d < p.dim;
  const int dd = dvalid ? d : p.dim - 1;
  const int kc = chunk0 + blockIdx.y, b = blockIdx.z;
  const int L = p.seqlen;
  const int t0 = kc * kChunk;
  const int ntl = min(NT, (L - t0 + TL - 1) / TL);    // tiles of this chunk inside the row
  const int d0 = blockIdx.x * CB;

  stage_rows<T>(S.rows[0], p, b, d0, t0, tid);   // the first stage's rows in flight
  cp_async_commit();
  // ---- B (and C) of the chunk into fp32 [t][n], both copies
  {
    constexpr int NR = CARRY ? 2 * kN : kN;
    for (int pc = tid; pc < NR * PPR; pc += CB) {
      const int r = pc / PPR, w = pc % PPR;
      const T* brow = static_cast<const T*>(r < kN ? p.B : p.C) + ((size_t)b * kN + (r & (kN - 1))) * L;
      RawVec<T, EPP> rv;
      rv.template load<true>(brow, t0 + w * EPP, L);
      float v[EPP];
      rv.unpack(v);
#pragma unroll
      for (int i = 0; i < EPP; ++i) {
        if (r < kN) sts_both(S.B, BS, w * EPP + i, r, v[i]);
        else sts_both(S.C, BS, w * EPP + i, r - kN, v[i]);
      }
    }
  }

  f2_t A2[8], h[8], pi[8], e[8];
  load_slots(p.A + (size_t)dd * kN, x, A2);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    A2[k] = mul2(A2[k], pk2(kLog2e, kLog2e));
    h[k] = pk2(0.f, 0.f);
    pi[k] = pk2(1.f, 1.f);
    e[k] = pk2(0.f, 0.f);
  }
  if (kc > 0) load_slots(p.ckpt + (((size_t)b * p.dim + dd) * p.nchunk + (kc - 1)) * kN, x, h);
  else if (p.h0) load_slots(p.h0 + ((size_t)b * p.dim + dd) * kN, x, h);
  const float bias = p.bias ? p.bias[dd] : 0.f;
  const bool has_z = p.z != nullptr;
  const int* seq_row = SEQ ? p.seq_idx + (size_t)b * L : nullptr;
  float* part = p.ch_part_dC + ((size_t)b * p.ncb + blockIdx.x) * (size_t)p.lpad * kN;
  __syncthreads();

#pragma unroll 1
  for (int tile = 0; tile < ntl; ++tile) {
    const int tb = t0 + tile * TL;
    const int st = tile / TPS;                   // row stage of this tile
    if (tile % TPS == 0) {
      cp_async_wait_all();
      __syncthreads();                           // the stage's rows (copied by all threads) are visible
      if ((st + 1) * SL < kChunk && t0 + (st + 1) * SL < L) {
        stage_rows<T>(S.rows[(st + 1) & 1], p, b, d0, t0 + (st + 1) * SL, tid);
        cp_async_commit();
      }
    }
    const RowStage<T>& R = S.rows[st & 1];
    const int s0 = (tile % TPS) * TL;            // first step of the tile within the stage
    const unsigned rst = SEQ ? doc_starts32(seq_row, tb, min(L, tb + TL)) : 0u;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float uv[TS], xv[TS], zv[TS], gv[TS];
      stage_quad<T>(R, 0, s0 + TS * hf, tid, uv);
      stage_quad<T>(R, 1, s0 + TS * hf, tid, xv);
      if (has_z) stage_quad<T>(R, 2, s0 + TS * hf, tid, zv);
      else zv[0] = zv[1] = zv[2] = zv[3] = 0.f;
      stage_quad<T>(R, 3, s0 + TS * hf, tid, gv);
      const int ts = tb + TS * hf;             // first step of the sub-chunk
      if (dvalid && ts < L)                    // state entering the sub-chunk
        store_pairs(p.ch_state + ((size_t)b * p.nsub4 + ts / TS) * kN * p.dpad, p.dpad, d, h);
#pragma unroll
      for (int i0 = 0; i0 < TS; i0 += 2) {
        f2_t dc[2][8];
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
          const int i = i0 + ii;
          const int tt = tile * TL + TS * hf + i;  // step within the chunk
          const bool ok = dvalid && ts + i < L;
          const Tok k = token(xv[i], zv[i], gv[i], bias, p.softplus, has_z, ok);
          const float du = k.dt * (ok ? uv[i] : 0.f);
          f2_t Bp[8];
          lds_slots(S.B + tt * kN, BS, x, Bp);
          const f2_t dt2 = pk2(k.dt, k.dt), du2 = pk2(du, du), do2 = pk2(k.dout, k.dout);
          const bool reset = SEQ && ((rst >> (TS * hf + i)) & 1u);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            f2_t a = ex2_2(mul2(dt2, A2[q]));
            if (reset) a = pk2(0.f, 0.f);
            h[q] = fma2(a, h[q], mul2(du2, Bp[q]));
            dc[ii][q] = mul2(do2, h[q]);
            if constexpr (CARRY) pi[q] = mul2(pi[q], a);
          }
          if constexpr (CARRY) {
            f2_t Cp[8];
            lds_slots(S.C + tt * kN, BS, x, Cp);
#pragma unroll
            for (int q = 0; q < 8; ++q) e[q] = fma2(pi[q], mul2(do2, Cp[q]), e[q]);
          }
        }
        const f2_t sm = warp_sum2(dc, lane);
        if (!(lane & 1)) *reinterpret_cast<f2_t*>(&S.red[warp][TS * hf + i0 + ((lane >> 1) & 1)][2 * x]) = sm;
      }
    }
    __syncthreads();
    {  // fixed-order sum of the block's warps: this tile's dC partial
      const int tt = tid / kN, n = tid % kN;   // 8 steps x 16 states = 128 threads
      const int t = tb + tt;
      float v = S.red[0][tt][n];
#pragma unroll
      for (int w = 1; w < NW; ++w) v += S.red[w][tt][n];
      part[(size_t)t * kN + n] = t < L ? v : 0.f;
    }
    __syncthreads();
  }
  // rows of the chunk past the end of the sequence: zero partials
  for (int o = ntl * TL * kN + tid; o < kChunk * kN; o += CB) part[(size_t)t0 * kN + o] = 0.f;
  if (CARRY && dvalid) {
    const size_t o = ((size_t)b * p.nchunk + kc) * kN * p.dpad;
    store_pairs(p.ch_map_e + o, p.dpad, d, e);
    store_pairs(p.ch_map_P + o, p.dpad, d, pi);
  }
}

// =========================================================================
// 2. Carry entering the last step of every chunk group: the gradient reaching
// the final state (or zero), composed through the maps of the later groups'
// chunks, latest first.  One thread per (b, d, 4 states).
// =========================================================================
__global__ void __launch_bounds__(256) ch_carry_kernel(const BwdParams p) {
  // thread (b, pair k, d), d fastest: maps and carries in the slot layout
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)p.batch * 8 * p.dim) return;
  const int d = (int)(i % p.dim);
  const int k = (int)((i / p.dim) % 8), b = (int)(i / ((long long)8 * p.dim));
  const int x = ((d & 31) >> 2) & 7;        // the slot permutation of channel d's lane
  f2_t c = p.dfinal ? *reinterpret_cast<const f2_t*>(p.dfinal + ((size_t)b * p.dim + d) * kN + 2 * (k ^ x))
                    : pk2(0.f, 0.f);
  const int gc = p.group_nsub / (kChunk / TL);  // chunks per group
  for (int g = p.ngroups - 1; g >= 0; --g) {
    *reinterpret_cast<f2_t*>(p.ch_carry + ((((size_t)b * p.ngroups + g) * 8 + k) * p.dpad + d) * 2) = c;
    if (g == 0) break;
    const int k_lo = g * gc, k_hi = min(p.nchunk, k_lo + gc) - 1;
#pragma unroll 4
    for (int kc = k_hi; kc >= k_lo; --kc) {
      const size_t o = ((((size_t)b * p.nchunk + kc) * 8 + k) * p.dpad + d) * 2;
      c = fma2(*reinterpret_cast<const f2_t*>(p.ch_map_P + o), c, *reinterpret_cast<const f2_t*>(p.ch_map_e + o));
    }
  }
}

// =========================================================================
// 3. The reverse walk.
// =========================================================================
// NA: state pairs (of 8) whose decays are kept from the forward recompute of a
// half-tile for its reverse sweep; the others are evaluated again there.
#ifndef SS_CH_WALK_NA
#define SS_CH_WALK_NA 8
#endif
#ifndef SS_CH_WALK_MINB
#define SS_CH_WALK_MINB 2
#endif
template <typename T>
struct WalkSmem {
  static constexpr int RW = TL * (int)sizeof(T) / 16;   // 16-byte words of an 8-step B / C row
  RowStage<T> rows[2];          // u, delta, z, dy rows, a stage at a time (double-buffered)
  uint4 bcr[2][2 * kN][RW];     // B, C rows of a tile
  f2_t hs[2][2][8][CB];         // states entering the tile's two halves, [pair][lane]
  float B[2 * TL * kN + 16];    // the tile's B_t, C_t in fp32 [t][n], two copies each
  float C[2 * TL * kN + 16];
  __align__(16) float red[NW][TL][kN];   // per-warp dB sums
};

using WalkSmemF = WalkSmem<float>;
using WalkSmemH = WalkSmem<__nv_bfloat16>;
static_assert(offsetof(WalkSmemF, hs) % 16 == 0 && offsetof(WalkSmemF, B) % 16 == 0 &&
              offsetof(WalkSmemF, C) % 16 == 0 && offsetof(WalkSmemF, red) % 16 == 0 &&
              offsetof(WalkSmemH, hs) % 16 == 0 && offsetof(WalkSmemH, B) % 16 == 0 &&
              offsetof(WalkSmemH, C) % 16 == 0 && offsetof(WalkSmemH, red) % 16 == 0,
              "16-byte aligned shared members");

template <typename T, bool SEQ, int NA>
__global__ void __launch_bounds__(CB, SS_CH_WALK_MINB) ch_walk_kernel(const BwdParams p) {
  constexpr int ES = (int)sizeof(T);
  constexpr int RW = WalkSmem<T>::RW;
  constexpr int HW = TS * ES;                  // bytes of a 4-step half row (8 or 16)
  constexpr int BS = TL * kN + 16;             // offset of the second copy of B / C
  constexpr int SL = RowStage<T>::SL;          // steps per row stage
  constexpr int TPS = SL / TL;                 // tiles per row stage
  extern __shared__ __align__(16) unsigned char ch_smem[];
  WalkSmem<T>& S = *reinterpret_cast<WalkSmem<T>*>(ch_smem);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int x = (lane >> 2) & 7;
  const int d = blockIdx.x * CB + tid;
  const bool dvalid = d < p.dim;
  const int dd = dvalid ? d : p.dim - 1;
  const int grp = blockIdx.y, b = blockIdx.z;
  const int L = p.seqlen;
  const bool has_z = p.z != nullptr;
  const int ntile = p.nsub;                    // 8-step tiles
  const int tile_lo = grp * p.group_nsub;
  const int tile_hi = min(ntile, tile_lo + p.group_nsub) - 1;
  const size_t row = ((size_t)b * p.dim + dd) * (size_t)L;
  const int* seq_row = SEQ ? p.seq_idx + (size_t)b * L : nullptr;
  float* part = p.ch_part_dB + ((size_t)b * p.ncb + blockIdx.x) * (size_t)p.lpad * kN;

  // Copies for tile `tile`: its B, C rows and entering states into buffer `buf`,
  // and the row stage holding it when the tile is the first of its stage the
  // walk reaches (the stage's last tile, or the group's last tile).
  auto stage = [&](int tile, int buf) {
    const int t = tile * TL;
    if (tile % TPS == TPS - 1 || tile == tile_hi)
      stage_rows<T>(S.rows[(tile / TPS) & 1], p, b, blockIdx.x * CB, (tile / TPS) * SL, tid);
    if (tid < 2 * kN * RW) {
      const int r = tid / RW, w = tid % RW;
      const T* src = static_cast<const T*>(r < kN ? p.B : p.C) + ((size_t)b * kN + (r & (kN - 1))) * L + t;
      const int nb = max(0, min(16, min(TL, L - t) * ES - 16 * w));
      cp_async16(&S.bcr[buf][r][w], nb > 0 ? (const void*)(src + 16 * w / ES) : (const void*)src, nb);
    }
    // entering states of the two halves: per half 8 pairs x 128 channels x 8 bytes,
    // copied as 16-byte pieces (two channels each) by consecutive threads
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int s = 2 * tile + hf;
      const float* src = p.ch_state + ((size_t)b * p.nsub4 + (s < p.nsub4 ? s : 0)) * kN * p.dpad;
#pragma unroll
      for (int m = 0; m < 8 * CB / 2 / CB; ++m) {
        const int c = tid + m * CB;              // piece: pair c / 64, channels 2 (c % 64), +1
        const int k = c / (CB / 2), dl = 2 * (c % (CB / 2));
        const int dg = blockIdx.x * CB + dl;
        // zero-filled past the sequence's sub-chunks and past d_inner
        const int nb = s < p.nsub4 && dg < p.dim ? (dg + 1 < p.dim ? 16 : 8) : 0;
        cp_async16(&S.hs[buf][hf][k][dl], nb ? (const void*)(src + ((size_t)k * p.dpad + dg) * 2) : (const void*)src, nb);
      }
    }
    cp_async_commit();
  };

  f2_t A2[8], carry[8], dA[8];
  load_slots(p.A + (size_t)dd * kN, x, A2);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    A2[k] = mul2(A2[k], pk2(kLog2e, kLog2e));
    carry[k] = dA[k] = pk2(0.f, 0.f);
  }
  // carry = Abar_{t+1} g_{t+1} before the group's last step: composed from the
  // later groups, or (last group) the gradient reaching the final state
  if (p.ngroups > 1) load_pairs(p.ch_carry + ((size_t)b * p.ngroups + grp) * kN * p.dpad, p.dpad, dd, carry);
  else if (p.dfinal) load_slots(p.dfinal + ((size_t)b * p.dim + dd) * kN, x, carry);
  const float Dd = p.D ? p.D[dd] : 0.f;
  const float bias = p.bias ? p.bias[dd] : 0.f;
  float dD_acc = 0.f, dbias_acc = 0.f;

  stage(tile_hi, 0);

#pragma unroll 1
  for (int tile = tile_hi; tile >= tile_lo; --tile) {
    const int buf = (tile_hi - tile) & 1;
    const int t0 = tile * TL;
    cp_async_wait_all();
    __syncthreads();  // this tile's rows are visible; the previous tile is fully consumed
    if (tile < tile_hi) {  // fixed-order sum of the warps' dB of the previous tile
      const int tt = tid / kN, n = tid % kN;
      const int t = t0 + TL + tt;
      float s = S.red[0][tt][n];
#pragma unroll
      for (int w = 1; w < NW; ++w) s += S.red[w][tt][n];
      part[(size_t)t * kN + n] = t < L ? s : 0.f;
    }
    if (tile > tile_lo) stage(tile - 1, buf ^ 1);
    for (int o = tid; o < 2 * kN * TL; o += CB) {  // B, C rows -> fp32 [t][n], both copies
      const int r = o % (2 * kN), i = o / (2 * kN);
      const float v = elt_at<T>(&S.bcr[buf][r][0], i);
      if (r < kN) sts_both(S.B, BS, i, r, v);
      else sts_both(S.C, BS, i, r - kN, v);
    }
    __syncthreads();
    const unsigned rst = SEQ ? doc_starts32(seq_row, t0, min(L, t0 + TL)) : 0u;

#pragma unroll 1
    for (int hf = 1; hf >= 0; --hf) {
      const int tb = t0 + TS * hf;
      // ---- per-token prologue for the half's 4 steps
      float uv[TS], dtv[TS], duv[TS], dov[TS], sxv[TS], dzv[TS];
      {
        float xr[TS], zr[TS], gr[TS];
        const RowStage<T>& R = S.rows[(tile / TPS) & 1];
        const int sq = (tile % TPS) * TL + TS * hf;   // first step of the half within the stage
        stage_quad<T>(R, 0, sq, tid, uv);
        stage_quad<T>(R, 1, sq, tid, xr);
        if (has_z) stage_quad<T>(R, 2, sq, tid, zr);
        else zr[0] = zr[1] = zr[2] = zr[3] = 0.f;
        stage_quad<T>(R, 3, sq, tid, gr);
#pragma unroll
        for (int i = 0; i < TS; ++i) {
          const bool ok = dvalid && tb + i < L;
          const Tok k = token(xr[i], zr[i], gr[i], bias, p.softplus, has_z, ok);
          uv[i] = ok ? uv[i] : 0.f;
          dtv[i] = k.dt;
          duv[i] = k.dt * uv[i];
          dov[i] = k.dout;
          sxv[i] = k.sx;
          dzv[i] = k.dzf;
        }
      }
      // ---- recompute the half's states (and decays) forward from its entering state
      f2_t Hh[TS][8];   // state entering each step
      f2_t Ha[TS][NA > 0 ? NA : 1];
      float ysv[TS];
      {
#pragma unroll
        for (int k = 0; k < 8; ++k) Hh[0][k] = S.hs[buf][hf][k][tid];
#pragma unroll
        for (int i = 0; i < TS; ++i) {
          f2_t Bp[8], Cp[8], hn[8];
          lds_slots(S.B + (TS * hf + i) * kN, BS, x, Bp);
          lds_slots(S.C + (TS * hf + i) * kN, BS, x, Cp);
          const f2_t dt2 = pk2(dtv[i], dtv[i]), du2 = pk2(duv[i], duv[i]);
          const bool reset = SEQ && ((rst >> (TS * hf + i)) & 1u);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            f2_t a = ex2_2(mul2(dt2, A2[q]));
            if (reset) a = pk2(0.f, 0.f);
            if (q < NA) Ha[i][q < NA ? q : 0] = a;
            hn[q] = fma2(a, Hh[i][q], mul2(du2, Bp[q]));
            if (i + 1 < TS) Hh[i + 1 < TS ? i + 1 : 0][q] = hn[q];
          }
          ysv[i] = dot8(Cp, hn);
        }
      }
      // ---- walk the half backwards
      float s1v[TS], s2v[TS];
      f2_t db[TS][8];
#pragma unroll
      for (int i = TS - 1; i >= 0; --i) {
        f2_t Bp[8], Cp[8], g[8], qv[8];
        lds_slots(S.C + (TS * hf + i) * kN, BS, x, Cp);
        lds_slots(S.B + (TS * hf + i) * kN, BS, x, Bp);
        const f2_t dt2 = pk2(dtv[i], dtv[i]), du2 = pk2(duv[i], duv[i]), do2 = pk2(dov[i], dov[i]);
        const bool reset = SEQ && ((rst >> (TS * hf + i)) & 1u);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          g[q] = fma2(do2, Cp[q], carry[q]);
          db[i][q] = mul2(g[q], du2);
          f2_t a;
          if (q < NA) {
            a = Ha[i][q < NA ? q : 0];
          } else {
            a = ex2_2(mul2(dt2, A2[q]));
            if (reset) a = pk2(0.f, 0.f);
          }
          carry[q] = mul2(a, g[q]);
          qv[q] = mul2(carry[q], Hh[i][q]);
          dA[q] = fma2(dt2, qv[q], dA[q]);
        }
        s1v[i] = dot8(g, Bp);
        s2v[i] = dot8(A2, qv) * kLn2f;   // A2 carries log2(e): sum A q = ln2 sum A2 q
      }
      {
        const f2_t sb = warp_sum4(db, lane);
        *reinterpret_cast<f2_t*>(&S.red[warp][TS * hf + (lane & 3)][2 * x]) = sb;
      }
      // ---- the half's du, ddelta, dz
      float duo[TS], ddo[TS], dzo[TS];
#pragma unroll
      for (int i = 0; i < TS; ++i) {
        duo[i] = fmaf(dov[i], Dd, dtv[i] * s1v[i]);
        ddo[i] = fmaf(uv[i], s1v[i], s2v[i]) * sxv[i];
        dzo[i] = fmaf(Dd, uv[i], ysv[i]) * dzv[i];
        dD_acc = fmaf(dov[i], uv[i], dD_acc);
        dbias_acc += ddo[i];
      }
      if (dvalid) {  // the half's 4 steps: one 8-byte (16-bit types) or 16-byte store per array
#pragma unroll
        for (int arr = 0; arr < 3; ++arr) {
          void* dst = arr == 0 ? p.du : arr == 1 ? p.ddelta : p.dz;
          if (!dst) continue;
          T* out = static_cast<T*>(dst) + row + tb;
          uint32_t w[HW / 4];
          T* e = reinterpret_cast<T*>(w);
#pragma unroll
          for (int i = 0; i < TS; ++i) e[i] = Elt<T>::from_f(arr == 0 ? duo[i] : arr == 1 ? ddo[i] : dzo[i]);
          if (tb + TS <= L) {
            if constexpr (ES == 4) *reinterpret_cast<uint4*>(out) = make_uint4(w[0], w[1], w[2], w[3]);
            else *reinterpret_cast<uint2*>(out) = make_uint2(w[0], w[1]);
          } else {  // ragged end of the row
            for (int i = 0; i < L - tb; ++i) out[i] = e[i];
          }
        }
      }
    }
  }
  __syncthreads();
  {  // dB of the group's first tile
    const int tt = tid / kN, n = tid % kN;
    const int t = tile_lo * TL + tt;
    float s = S.red[0][tt][n];
#pragma unroll
    for (int w = 1; w < NW; ++w) s += S.red[w][tt][n];
    part[(size_t)t * kN + n] = t < L ? s : 0.f;
  }
  const size_t part_row = (size_t)grp * p.batch + b;  // partial-sum row (group, batch row)
  if (dvalid) {
    store_slots(p.part_dA + (part_row * p.dim + d) * kN, x, dA);
    p.part_dD[part_row * p.dim + d] = dD_acc;
    p.part_dbias[part_row * p.dim + d] = dbias_acc;
    // after step 0 the carry is Abar_0 g_0 = dloss / dh0
    if (p.dh0 && grp == 0) store_slots(p.dh0 + ((size_t)b * p.dim + d) * kN, x, carry);
  }
}

// =========================================================================
// 4. Fixed-order sums.
// =========================================================================
// dB, dC (batch, 16, L): per block of 64 steps and batch row, add the channel
// blocks' partials in block order, transposed through shared memory so both
// the reads ([t][n]) and the writes ([n][t]) are coalesced.
__global__ void __launch_bounds__(256) ch_reduce_bc_kernel(const BwdParams p) {
  __shared__ float s_t[2][kN][65];
  const int tid = threadIdx.x;
  const int b = blockIdx.y, t0 = blockIdx.x * 64;
  const int L = p.seqlen;
  const int tl = tid >> 2, q4 = tid & 3;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float* src = (q ? p.ch_part_dC : p.ch_part_dB) + ((size_t)b * p.ncb * p.lpad + t0 + tl) * kN + 4 * q4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t0 + tl < L) {
      for (int k = 0; k < p.ncb; ++k) {
        const float4 v = *reinterpret_cast<const float4*>(src + (size_t)k * p.lpad * kN);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
    }
    s_t[q][4 * q4 + 0][tl] = acc.x;
    s_t[q][4 * q4 + 1][tl] = acc.y;
    s_t[q][4 * q4 + 2][tl] = acc.z;
    s_t[q][4 * q4 + 3][tl] = acc.w;
  }
  __syncthreads();
  for (int o = tid; o < 2 * kN * 64; o += 256) {
    const int q = o / (kN * 64), n = (o / 64) % kN, tt = o % 64;
    if (t0 + tt < L) (q ? p.dC : p.dB)[((size_t)b * kN + n) * L + t0 + tt] = s_t[q][n][tt];
  }
}

__global__ void ch_reduce_param_kernel(const BwdParams p) {
  const long long nA = (long long)p.dim * kN, nD = p.dim;
  const int rows = p.ngroups * p.batch;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nA + 2 * nD;
       i += (long long)gridDim.x * blockDim.x) {
    if (i < nA) {
      float s = 0.f;
      for (int r = 0; r < rows; ++r) s += p.part_dA[(size_t)r * nA + i];
      p.dA[i] = s;
    } else {
      const long long r0 = i - nA;
      const int q = r0 >= nD;
      const long long dd = q ? r0 - nD : r0;
      float* out = q ? p.dbias : p.dD;
      if (!out) continue;
      const float* src = q ? p.part_dbias : p.part_dD;
      float s = 0.f;
      for (int r = 0; r < rows; ++r) s += src[(size_t)r * nD + dd];
      out[dd] = s;
    }
  }
}

// Kernels whose shared memory is above the 48 KB static limit get their
// dynamic limit raised once per device.
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes, unsigned long long& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
  if (bit && (__atomic_load_n(&done, __ATOMIC_RELAXED) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  // the largest shared-memory carveout, so shared memory does not cap the blocks per SM
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && bit) __atomic_fetch_or(&done, bit, __ATOMIC_RELAXED);
  return e;
}

template <typename T, bool SEQ>
cudaError_t walk_prepare() {
  static unsigned long long done = 0ull;
  return allow_smem(ch_walk_kernel<T, SEQ, SS_CH_WALK_NA>, sizeof(WalkSmem<T>), done);
}
template <typename T, bool SEQ, bool CARRY>
cudaError_t states_prepare() {
  static unsigned long long done = 0ull;
  return allow_smem(ch_states_kernel<T, SEQ, CARRY>, sizeof(StatesSmem<T, CARRY>), done);
}

template <typename T, bool SEQ>
int walk_blocks_per_sm() {
  if (walk_prepare<T, SEQ>() != cudaSuccess) return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, ch_walk_kernel<T, SEQ, SS_CH_WALK_NA>, CB,
                                                    sizeof(WalkSmem<T>)) != cudaSuccess)
    return 0;
  return n;
}

template <typename T, bool SEQ>
cudaError_t launch_ch_s(const BwdParams& p0, cudaStream_t s) {
  BwdParams p = p0;
  choose_ch_groups(p, walk_blocks_per_sm<T, SEQ>());
  const int plain = p.ngroups > 1 ? p.group_nsub / (kChunk / TL) : p.nchunk;  // chunks of group 0
  cudaError_t e = states_prepare<T, SEQ, false>();
  if (e != cudaSuccess) return e;
  ch_states_kernel<T, SEQ, false><<<dim3(p.ncb, plain, p.batch), CB, sizeof(StatesSmem<T, false>), s>>>(p, 0);
  if (p.ngroups > 1) {
    if ((e = states_prepare<T, SEQ, true>()) != cudaSuccess) return e;
    ch_states_kernel<T, SEQ, true>
        <<<dim3(p.ncb, p.nchunk - plain, p.batch), CB, sizeof(StatesSmem<T, true>), s>>>(p, plain);
    const long long n = (long long)p.batch * 8 * p.dim;
    ch_carry_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
  }
  if ((e = walk_prepare<T, SEQ>()) != cudaSuccess) return e;
  ch_walk_kernel<T, SEQ, SS_CH_WALK_NA><<<dim3(p.ncb, p.ngroups, p.batch), CB, sizeof(WalkSmem<T>), s>>>(p);
  ch_reduce_bc_kernel<<<dim3((p.seqlen + 63) / 64, p.batch), 256, 0, s>>>(p);
  const long long total = (long long)p.dim * kN + 2LL * p.dim;
  long long blocks = (total + 255) / 256;
  if (blocks > (long long)p.sms * 8) blocks = (long long)p.sms * 8;
  ch_reduce_param_kernel<<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ch_t(const BwdParams& p, cudaStream_t s) {
  return p.seq_idx ? launch_ch_s<T, true>(p, s) : launch_ch_s<T, false>(p, s);
}

template <typename T>
void plan_ch_t(BwdParams& p) {
  choose_ch_groups(p, p.seq_idx ? walk_blocks_per_sm<T, true>() : walk_blocks_per_sm<T, false>());
}

}  // namespace

// Chunk groups of the walk: with R walk blocks resident on the GPU, a walk of
// G groups takes about ceil(blocks * G / R) waves of (chunks per group)
// chunk-times.  Groups add carry maps to the states pass (cheap there: it is
// bound by the SFU) and partial rows to the parameter sums; the fewest groups
// within 5% of the best count are taken.
void choose_ch_groups(BwdParams& p, int blocks_per_sm) {
  p.ngroups = 1;
  p.group_nsub = p.nsub;
  const long long base = (long long)p.ncb * p.batch;
  const long long R = (long long)(blocks_per_sm > 0 ? blocks_per_sm : 1) * (p.sms > 0 ? p.sms : 1);
  const int gmax = p.nchunk < kMaxChGroups ? p.nchunk : kMaxChGroups;
  long long best = -1;
  long long cost[kMaxChGroups + 1];
  int gcs[kMaxChGroups + 1];
  for (int g = 1; g <= gmax; ++g) {
    const int gc = (p.nchunk + g - 1) / g;
    gcs[g] = gc;
    cost[g] = (p.nchunk + gc - 1) / gc != g ? -1 : ((base * g + R - 1) / R) * gc;
    if (cost[g] >= 0 && (best < 0 || cost[g] < best)) best = cost[g];
  }
  for (int g = 1; g <= gmax; ++g) {
    if (cost[g] >= 0 && cost[g] * 100 <= best * 105) {
      p.ngroups = g;
      p.group_nsub = gcs[g] * (kChunk / TL);
      return;
    }
  }
}

cudaError_t plan_bwd_ch(BwdParams& p, DType dt) {
  switch (dt) {
    case DType::F32: plan_ch_t<float>(p); break;
    case DType::BF16: plan_ch_t<__nv_bfloat16>(p); break;
    case DType::F16: plan_ch_t<__half>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t launch_bwd_ch(const BwdParams& p, DType dt, cudaStream_t s) {
  switch (dt) {
    case DType::F32: return launch_ch_t<float>(p, s);
    case DType::BF16: return launch_ch_t<__nv_bfloat16>(p, s);
    case DType::F16: return launch_ch_t<__half>(p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ss
