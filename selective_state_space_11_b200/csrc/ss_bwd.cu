// ss_bwd.cu -- backward selective scan (S6) for sm_100a.
//
// Adjoint of the forward scan for the loss <dy, y> ("Mamba", stanleyjacob.dev,
// Part IV Stage 7: recompute the states instead of storing them, accumulate
// gradients for u, Delta, A, B, C, D, z).  With g_t = dloss/dh_t:
//   g_t    = Abar_{t+1} g_{t+1} + dout_t C_t,      dout_t = dy_t SiLU(z_t)
//   dC_t   = sum_d dout_t h_t                       dB_t = sum_d g_t Delta_t u_t
//   du_t   = dout_t D + Delta_t sum_n g_t B_t
//   dDelta = u_t sum_n g_t B_t + sum_n g_t A Abar_t h_{t-1}
//   dA    += g_t Delta_t Abar_t h_{t-1}
//   ddelta = dDelta sigmoid(delta + bias) (softplus on),  dbias = sum ddelta
//   dz     = dy (C.h + D u) SiLU'(z),  dD = sum dout u
//
// Schedule ("Mamba, on a laptop GPU.", "The state lives in registers": walk
// the chunks in reverse, recompute each chunk's states from its checkpoint,
// carry the state gradient across chunk boundaries in registers):
//   1. states_kernel: one block per (64 channels, batch row, 64-step chunk),
//      all chunks in parallel: starting from the forward's 64-step checkpoint
//      it records the state entering every 8-step sub-chunk (workspace).  When
//      the walk runs in chunk groups, it also composes each chunk's map of the
//      reverse gradient carry, c -> P_k c + e_k.
//   1b. group_carry_kernel: composes those maps from the last chunk backwards
//      into the carry entering each group's last step.
//   2. reverse walk (bwd2_kernel: two channels per 4-lane group; bwd_kernel:
//      one): per channel and chunk group, walk the 8-step sub-chunks latest
//      first.  A sub-chunk's states are recomputed from its entering state
//      into registers, then walked backwards with g carried in registers, 4
//      states per lane as fp32 pairs (fma/mul .f32x2).  Inputs for the next
//      sub-chunk are staged while the current one is processed.  Sums over the
//      state index (du, dDelta and the recomputed readout used by dz) meet in
//      shared memory; channel sums of dB, dC are formed per block in a fixed
//      order and written as per-block partials.
//   3. reduce_bc_kernel, reduce_param_kernel: add the per-block partials (dB,
//      dC) and the per-(group, batch row) partials (dA, dD, dbias) in a fixed
//      order -- deterministic, no floating-point atomics (the Metal design on
//      that page reduces with threadgroup memory plus float atomics).
#include <type_traits>

#include "ss_device.cuh"
#include "ss_internal.h"

namespace ss {
namespace {

constexpr int SUB = kSub;    // steps per sub-chunk held in registers (8)
constexpr int KL = 4;        // lanes per channel
constexpr int SPL = 4;       // states per lane
constexpr int NP = 2;        // fp32 pairs per lane

// -------------------------------------------------------------------------
// 1. States entering every 8-step sub-chunk, all 64-step chunks in parallel.
//
// With CARRY the same pass also composes the chunk's map of the reverse
// gradient carry.  Walking a chunk backwards turns the carry c entering its
// last step into P_k c + e_k leaving its first step, with
//   P_k = prod_t Abar_t,   e_k = sum_s (prod_{r <= s} Abar_r) dout_s C_s
// over the chunk's steps (r, s counted from the chunk's first step).  Both are
// accumulated forwards here from the decays the state recompute already
// forms, so the chunk groups of the reverse walk can start from the right
// carry without waiting for the later groups.
// -------------------------------------------------------------------------
#ifndef SS_STATES_CARRY_MINB
#define SS_STATES_CARRY_MINB 5
#endif
#ifndef SS_STATES_MINB
#define SS_STATES_MINB 7
#endif
template <typename T, bool VEC, bool SEQ, bool CARRY>
__global__ void __launch_bounds__(128, CARRY ? SS_STATES_CARRY_MINB : SS_STATES_MINB)
states_kernel(const BwdParams p, int chunk0) {
  // 64 channels: each thread carries the same 4 states of two channels, so one
  // B_t (C_t) load serves both; the tokens (Delta, Delta u) are kept once per
  // channel and duplicated into fp32 pairs in registers.  The chunk is staged
  // in two halves of 32 steps.
  constexpr int CB = 64;
  constexpr int HS = kChunk / 2;
  // channel stride of the token rows: odd, so that 16 consecutive channels'
  // 8-byte entries (32 channels' 4-byte entries) of one step fall in distinct banks
  constexpr int CHP = HS + 1;
  __shared__ __align__(16) f2_t s_tk[CB][CHP];                   // (Delta, Delta u)
  __shared__ __align__(16) float s_do[CARRY ? CB : 1][CHP];      // dout = dy SiLU(z)
  __shared__ __align__(16) float s_B[HS][kN];
  __shared__ __align__(16) float s_C[CARRY ? HS : 1][kN];

  const int tid = threadIdx.x;
  const int pr = tid >> 2, j = tid & 3;  // channels 2pr, 2pr+1; states 4j .. 4j+3
  const int b = blockIdx.y, kc = chunk0 + blockIdx.z;
  const int L = p.seqlen;
  const int t0 = kc * kChunk;

  // per-token role: channel cp, steps [16 part, 16 part + 16) of each half
  const int cp = tid & (CB - 1), part = tid >> 6;
  const int dp = blockIdx.x * CB + cp;
  const bool pvalid = dp < p.dim;
  const size_t prow = ((size_t)b * p.dim + (pvalid ? dp : 0)) * (size_t)L;
  const T* __restrict__ u_row = static_cast<const T*>(p.u) + prow;
  const T* __restrict__ x_row = static_cast<const T*>(p.delta) + prow;
  const T* __restrict__ z_row = CARRY && p.z ? static_cast<const T*>(p.z) + prow : nullptr;
  const T* __restrict__ g_row = CARRY ? static_cast<const T*>(p.dy) + prow : nullptr;
  const float bias = p.bias ? p.bias[pvalid ? dp : 0] : 0.f;
  // B / C tile role: array q (B, or C with CARRY), row n, 8 steps at 8 tg
  const int g_q = tid >> 6, g_n = tid & 15, g_tg = (tid >> 4) & 3;
  const T* __restrict__ bc_row = static_cast<const T*>(g_q ? p.C : p.B) + ((size_t)b * kN + g_n) * L;

  // steps of this chunk that start a new document (their decay is zero);
  // every warp forms the same 64-bit mask
  const int* seq_row = p.seq_idx ? p.seq_idx + (size_t)b * L : nullptr;
  const unsigned long long rst =
      SEQ ? ((unsigned long long)doc_starts32(seq_row, t0, min(L, t0 + 32)) |
             ((unsigned long long)doc_starts32(seq_row, t0 + 32, min(L, t0 + kChunk)) << 32))
          : 0ull;

  f2_t A2[2][NP], h[2][NP], pi[2][NP], e[2][NP];
  float* hs[2];
  bool valid[2];
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const int d = blockIdx.x * CB + 2 * pr + ch;
    valid[ch] = d < p.dim;
    const int dd = valid[ch] ? d : 0;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const float* a = p.A + (size_t)dd * kN + SPL * j + 2 * q;
      A2[ch][q] = pk2(a[0] * kLog2e, a[1] * kLog2e);
      h[ch][q] = pk2(0.f, 0.f);
      pi[ch][q] = pk2(1.f, 1.f);
      e[ch][q] = pk2(0.f, 0.f);
    }
    if (kc > 0 || p.h0) {  // chunk 0 starts from the forward's initial state
      const float4 v = *reinterpret_cast<const float4*>(
          kc > 0 ? p.ckpt + (((size_t)b * p.dim + dd) * p.nchunk + (kc - 1)) * kN + SPL * j
                 : p.h0 + ((size_t)b * p.dim + dd) * kN + SPL * j);
      h[ch][0] = pk2(v.x, v.y);
      h[ch][1] = pk2(v.z, v.w);
    }
    hs[ch] = p.sub_state + ((size_t)b * p.dim + dd) * (size_t)p.nsub * kN + SPL * j;
  }
  const int s0 = kc * (kChunk / SUB);

#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    if (s0 + half * (HS / SUB) >= p.nsub) break;  // past the end of the row
    if (half) __syncthreads();                    // the first half is consumed
    // ---- per-token prologue
#pragma unroll
    for (int pc = 0; pc < 2; ++pc) {
      const int tt = 16 * part + 8 * pc;          // step within the half
      const int t = t0 + HS * half + tt;
      RawVec<T, 8> ru, rx;
      ru.template load<VEC>(u_row, t, L);
      rx.template load<VEC>(x_row, t, L);
      float uv[8], xv[8];
      ru.unpack(uv);
      rx.unpack(xv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool ok = pvalid && (t + i < L);
        const float x = xv[i] + bias;
        float dt = p.softplus ? softplus_f(x) : x;
        dt = ok ? dt : 0.f;
        s_tk[cp][tt + i] = pk2(dt, dt * uv[i]);
      }
    }
    if constexpr (CARRY) {
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        const int tt = 16 * part + 8 * pc;
        const int t = t0 + HS * half + tt;
        RawVec<T, 8> rg;
        rg.template load<VEC>(g_row, t, L);
        float gv[8];
        rg.unpack(gv);
        if (z_row) {
          RawVec<T, 8> rz;
          rz.template load<VEC>(z_row, t, L);
          float zv[8];
          rz.unpack(zv);
#pragma unroll
          for (int i = 0; i < 8; ++i) gv[i] *= zv[i] * sigmoid_f(zv[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) s_do[cp][tt + i] = (pvalid && t + i < L) ? gv[i] : 0.f;
      }
    }
    if (CARRY || g_q == 0) {  // B (and C) tile of the half
      RawVec<T, 8> rb;
      rb.template load<VEC>(bc_row, t0 + HS * half + 8 * g_tg, L);
      float v[8];
      rb.unpack(v);
      float (*dst)[kN] = g_q ? s_C : s_B;
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[8 * g_tg + i][g_n] = v[i];
    }
    __syncthreads();

#pragma unroll
    for (int sb2 = 0; sb2 < HS / SUB; ++sb2) {
      const int sb = (HS / SUB) * half + sb2;
      if (s0 + sb >= p.nsub) break;
      // state entering sub-chunk sb
#pragma unroll
      for (int ch = 0; ch < 2; ++ch)
        if (valid[ch])
          *reinterpret_cast<float4*>(hs[ch] + (size_t)(s0 + sb) * kN) =
              make_float4(lo2(h[ch][0]), hi2(h[ch][0]), lo2(h[ch][1]), hi2(h[ch][1]));
      // without the carry the last sub-chunk's steps are not needed
      if (!CARRY && sb == kChunk / SUB - 1) break;
#pragma unroll
      for (int i = 0; i < SUB; ++i) {
        const int tt = SUB * sb2 + i;             // step within the half
        const int tc = HS * half + tt;            // step within the chunk
        const ulonglong2 bp = *reinterpret_cast<const ulonglong2*>(&s_B[tt][SPL * j]);
        ulonglong2 cpv;
        if constexpr (CARRY) cpv = *reinterpret_cast<const ulonglong2*>(&s_C[tt][SPL * j]);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const f2_t tk = s_tk[2 * pr + ch][tt];
          const f2_t dt2 = pk2(lo2(tk), lo2(tk)), du2 = pk2(hi2(tk), hi2(tk));
          f2_t a0 = ex2_2(mul2(dt2, A2[ch][0])), a1 = ex2_2(mul2(dt2, A2[ch][1]));
          if ((rst >> tc) & 1ull) a0 = a1 = pk2(0.f, 0.f);
          h[ch][0] = fma2(a0, h[ch][0], mul2(du2, bp.x));
          h[ch][1] = fma2(a1, h[ch][1], mul2(du2, bp.y));
          if constexpr (CARRY) {
            const float dov = s_do[2 * pr + ch][tt];
            const f2_t do2 = pk2(dov, dov);
            pi[ch][0] = mul2(pi[ch][0], a0);
            pi[ch][1] = mul2(pi[ch][1], a1);
            e[ch][0] = fma2(pi[ch][0], mul2(do2, cpv.x), e[ch][0]);
            e[ch][1] = fma2(pi[ch][1], mul2(do2, cpv.y), e[ch][1]);
          }
        }
      }
    }
  }
  if constexpr (CARRY) {
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      if (!valid[ch]) continue;
      const int d = blockIdx.x * CB + 2 * pr + ch;
      const size_t o = (((size_t)b * p.dim + d) * p.nchunk + kc) * kN + SPL * j;
      *reinterpret_cast<float4*>(p.chunk_carry + o) =
          make_float4(lo2(e[ch][0]), hi2(e[ch][0]), lo2(e[ch][1]), hi2(e[ch][1]));
      *reinterpret_cast<float4*>(p.chunk_decay + o) =
          make_float4(lo2(pi[ch][0]), hi2(pi[ch][0]), lo2(pi[ch][1]), hi2(pi[ch][1]));
    }
  }
}

// -------------------------------------------------------------------------
// 1b. Carry entering the last step of every chunk group: the gradient that
// reaches the final state (or zero), composed through the chunk maps of the
// later groups, latest first.  One thread per (b, d, 4 states).
// -------------------------------------------------------------------------
__global__ void __launch_bounds__(256) group_carry_kernel(const BwdParams p) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)p.batch * p.dim * (kN / 4)) return;
  const size_t bd = (size_t)(i / (kN / 4));
  const int q4 = (int)(i % (kN / 4));
  float4 c = p.dfinal ? *reinterpret_cast<const float4*>(p.dfinal + bd * kN + 4 * q4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  const int gc = p.group_nsub / (kChunk / SUB);  // chunks per group
  for (int g = p.ngroups - 1; g >= 0; --g) {
    *reinterpret_cast<float4*>(p.group_carry + (bd * p.ngroups + g) * kN + 4 * q4) = c;
    if (g == 0) break;
    const int k_lo = g * gc, k_hi = min(p.nchunk, k_lo + gc) - 1;
#pragma unroll 4
    for (int k = k_hi; k >= k_lo; --k) {
      const size_t o = (bd * p.nchunk + k) * kN + 4 * q4;
      const float4 P = *reinterpret_cast<const float4*>(p.chunk_decay + o);
      const float4 e = *reinterpret_cast<const float4*>(p.chunk_carry + o);
      c = make_float4(fmaf(P.x, c.x, e.x), fmaf(P.y, c.y, e.y), fmaf(P.z, c.z, e.z), fmaf(P.w, c.w, e.w));
    }
  }
}

// -------------------------------------------------------------------------
// 2. The reverse walk over 8-step sub-chunks.
// -------------------------------------------------------------------------
// Two 16-bit storage elements packed in one word -> two floats.
template <typename T>
__device__ __forceinline__ float2 unpack2(unsigned r) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    return make_float2(__uint_as_float(r << 16), __uint_as_float(r & 0xffff0000u));
  } else {
    return __half22float2(*reinterpret_cast<const __half2*>(&r));
  }
}
// Two storage elements (2 * sizeof(T)-byte aligned) -> two floats, one load.
template <typename T>
__device__ __forceinline__ float2 ld_pair(const unsigned char* p) {
  if constexpr (sizeof(T) == 4) {
    return *reinterpret_cast<const float2*>(p);
  } else {
    return unpack2<T>(*reinterpret_cast<const unsigned*>(p));
  }
}
// Four storage elements (4 * sizeof(T)-byte aligned) -> four floats, one load.
template <typename T>
__device__ __forceinline__ float4 ld_quad(const unsigned char* p) {
  if constexpr (sizeof(T) == 4) {
    return *reinterpret_cast<const float4*>(p);
  } else {
    const uint2 r = *reinterpret_cast<const uint2*>(p);
    const float2 a = unpack2<T>(r.x), b = unpack2<T>(r.y);
    return make_float4(a.x, a.y, b.x, b.y);
  }
}

// Shared-memory reads that stay in program order: without this the compiler
// hoists every unrolled step's operands at once and runs out of registers.
// Addresses are a per-thread 32-bit shared base plus a compile-time byte
// offset, which folds into the load's immediate.
__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ f2_t lds_f2(unsigned addr) {
  f2_t v;
  asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ ulonglong2 lds_f4(unsigned addr) {
  ulonglong2 v;
  asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "r"(addr));
  return v;
}

template <typename T, bool VEC, bool SEQ>
__global__ void __launch_bounds__(16 * KL, sizeof(T) == 4 ? 5 : 6)
bwd_kernel(const BwdParams p) {
  constexpr int CB = 16;                     // 16 channels, 64 threads
  constexpr int NT = CB * KL;
  constexpr int ES = (int)sizeof(T);
  constexpr int ROWB = SUB * ES;                   // one 8-step row in storage format
  constexpr int CHB = 4 * ROWB + 8 * ES;           // per-channel stride of the raw tile (padded)
  constexpr int PC = KL * SUB + 8;                 // per-channel stride of s_p (padded)
  constexpr int RED_SLAB = CB * kN + 16;           // padded (step, q) slab of s_red
  static_assert(NT == 64, "mapping assumes 64 threads");
  __shared__ __align__(16) unsigned char s_in[2][CB * CHB];        // u, delta, z, dy rows
  __shared__ __align__(16) unsigned char s_bcr[2][2 * kN * ROWB];  // B, C rows
  __shared__ __align__(16) float4 s_hin[2][NT];                    // entering state per lane
  __shared__ __align__(16) float s_B[SUB][kN];
  __shared__ __align__(16) float s_C[SUB][kN];
  // per step: (Delta, Delta), (Delta u, Delta u), (dout, dout), pad -- one
  // 128-bit load fetches the first two; channel rows padded by 16 bytes
  constexpr int TOKC = 4 * SUB + 2;                                // f2_t per channel row
  __shared__ __align__(16) f2_t s_tok[CB * TOKC];
  __shared__ __align__(16) float s_p[3][CB * PC];                  // per-lane sums over n
  __shared__ __align__(16) float s_red[SUB * 2 * RED_SLAB];        // [step][q][channel][n]

  const int tid = threadIdx.x;
  const int c = tid / KL, j = tid % KL;
  const int b = blockIdx.y, blk = blockIdx.x;
  const int d = blk * CB + c;
  const bool dvalid = d < p.dim;
  const int dd = dvalid ? d : 0;
  const int L = p.seqlen;
  const int Lp = (L + 15) & ~15;
  const bool has_z = p.z != nullptr;
  const int* seq_row = p.seq_idx ? p.seq_idx + (size_t)b * L : nullptr;

  const size_t row = ((size_t)b * p.dim + dd) * (size_t)L;
  // thread (c, j) stages array j of its channel (u, delta, z, dy); threads
  // 0..31 stage one B or C row each; every lane stages its entering state
  const void* arr = j == 0 ? p.u : j == 1 ? p.delta : j == 2 ? p.z : p.dy;
  const T* __restrict__ my_row = arr ? static_cast<const T*>(arr) + row : nullptr;
  const int g_q = tid >> 4, g_n = tid & 15;
  const T* __restrict__ g_row = static_cast<const T*>(g_q ? p.C : p.B) + ((size_t)b * kN + g_n) * L;
  const float* hs = p.sub_state + ((size_t)b * p.dim + dd) * (size_t)p.nsub * kN + SPL * j;

  auto stage = [&](int sc, int buf) {
    const int t = sc * SUB;
    const int nvalid = min(SUB, L - t);
    if (VEC) {
      if (my_row) {
        unsigned char* dst = &s_in[buf][c * CHB + j * ROWB];
#pragma unroll
        for (int k = 0; k < ROWB / 16; ++k) {
          const int bytes = max(0, min(16, nvalid * ES - 16 * k));
          cp_async16(dst + 16 * k, bytes > 0 ? (const void*)(my_row + t + 16 * k / ES) : (const void*)my_row, bytes);
        }
      }
      if (tid < 32) {
        unsigned char* dst = &s_bcr[buf][(g_q * kN + g_n) * ROWB];
#pragma unroll
        for (int k = 0; k < ROWB / 16; ++k) {
          const int bytes = max(0, min(16, nvalid * ES - 16 * k));
          cp_async16(dst + 16 * k, bytes > 0 ? (const void*)(g_row + t + 16 * k / ES) : (const void*)g_row, bytes);
        }
      }
      cp_async16(&s_hin[buf][tid], hs + (size_t)sc * kN, 16);
      cp_async_commit();
    } else {  // rows not 16-byte aligned: plain loads (correct for any L)
      if (my_row) {
        T* dst = reinterpret_cast<T*>(&s_in[buf][c * CHB + j * ROWB]);
#pragma unroll
        for (int i = 0; i < SUB; ++i) dst[i] = i < nvalid ? my_row[t + i] : T(0.f);
      }
      if (tid < 32) {
        T* dst = reinterpret_cast<T*>(&s_bcr[buf][(g_q * kN + g_n) * ROWB]);
#pragma unroll
        for (int i = 0; i < SUB; ++i) dst[i] = i < nvalid ? g_row[t + i] : T(0.f);
      }
      s_hin[buf][tid] = *reinterpret_cast<const float4*>(hs + (size_t)sc * kN);
    }
  };

  f2_t A2[NP], Aq[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    const float* a = p.A + (size_t)dd * kN + SPL * j + 2 * q;
    Aq[q] = pk2(a[0], a[1]);
    A2[q] = pk2(a[0] * kLog2e, a[1] * kLog2e);
  }
  const float Dd = p.D ? p.D[dd] : 0.f;
  const float bias = p.bias ? p.bias[dd] : 0.f;

  // carry = Abar_{t+1} g_{t+1}; before the group's last step it is the
  // carry composed from the later groups, or (one group) the gradient that
  // reaches the final state from outside (zero unless given)
  const int grp = blockIdx.z;
  const int sc_lo = grp * p.group_nsub, sc_hi = min(p.nsub, sc_lo + p.group_nsub) - 1;
  const float* cin = p.ngroups > 1 ? p.group_carry + (((size_t)b * p.dim + dd) * p.ngroups + grp) * kN
                     : p.dfinal     ? p.dfinal + ((size_t)b * p.dim + dd) * kN
                                    : nullptr;
  f2_t carry[NP], dA[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    carry[q] = dA[q] = pk2(0.f, 0.f);
    if (cin) carry[q] = pk2(cin[SPL * j + 2 * q], cin[SPL * j + 2 * q + 1]);
  }
  float dD_acc = 0.f, dbias_acc = 0.f;

  stage(sc_hi, sc_hi & 1);

  for (int sc = sc_hi; sc >= sc_lo; --sc) {
    const int buf = sc & 1;
    const int t0 = sc * SUB;
    // steps of this sub-chunk that start a new document: zero decay, so
    // neither the state nor its gradient crosses the boundary
    const unsigned rst = SEQ ? doc_starts32(seq_row, t0, min(L, t0 + SUB)) : 0u;
    if (VEC) cp_async_wait_all();
    __syncthreads();  // staged tile visible; previous sub-chunk fully consumed
    if (sc > sc_lo) stage(sc - 1, buf ^ 1);

    // ---- B / C to fp32 [step][n]: 64 threads x 4 elements
    {
      const int q = tid >> 5, n = (tid >> 1) & 15, hf = tid & 1;
      const unsigned char* src = &s_bcr[buf][(q * kN + n) * ROWB + 4 * hf * ES];
      const float2 v0 = ld_pair<T>(src), v1 = ld_pair<T>(src + 2 * ES);
      float(*dst)[kN] = q ? s_C : s_B;
      dst[4 * hf + 0][n] = v0.x;
      dst[4 * hf + 1][n] = v0.y;
      dst[4 * hf + 2][n] = v1.x;
      dst[4 * hf + 3][n] = v1.y;
    }
    // ---- per-token prologue: thread (c, j) owns steps 2j, 2j+1
    float e_u[2], e_sx[2], e_dzf[2], e_do[2], e_dt[2];
    {
      const unsigned char* base = &s_in[buf][c * CHB + 2 * j * ES];
      const float2 uu = ld_pair<T>(base);
      const float2 xx = ld_pair<T>(base + ROWB);
      const float2 zz = has_z ? ld_pair<T>(base + 2 * ROWB) : make_float2(0.f, 0.f);
      const float2 gg = ld_pair<T>(base + 3 * ROWB);
      const float uva[2] = {uu.x, uu.y}, xva[2] = {xx.x, xx.y}, zva[2] = {zz.x, zz.y}, gva[2] = {gg.x, gg.y};
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int tt = 2 * j + i;
        const bool ok = dvalid && (t0 + tt < L);
        const float x = xva[i] + bias;
        float dt = x, sx = 1.f;
        if (p.softplus) {
          const float w = ex2(-fabsf(x) * kLog2e);
          dt = fmaxf(x, 0.f) + log1p_unit(w);
          const float r = rcp(1.f + w);
          sx = x >= 0.f ? r : w * r;
        }
        float gate = 1.f, dzf = 0.f;
        if (has_z) {
          const float sz = sigmoid_f(zva[i]);
          gate = zva[i] * sz;
          dzf = gva[i] * sz * fmaf(zva[i], 1.f - sz, 1.f);
        }
        dt = ok ? dt : 0.f;
        const float dout = ok ? gva[i] * gate : 0.f;
        const float du = dt * uva[i];
        *reinterpret_cast<ulonglong2*>(&s_tok[c * TOKC + 4 * tt]) = make_ulonglong2(pk2(dt, dt), pk2(du, du));
        s_tok[c * TOKC + 4 * tt + 2] = pk2(dout, dout);
        e_u[i] = ok ? uva[i] : 0.f;
        e_sx[i] = sx;
        e_dzf[i] = dzf;
        e_do[i] = dout;
        e_dt[i] = dt;
      }
    }
    const float4 hin4 = s_hin[buf][tid];
    __syncthreads();

    // ---- recompute the sub-chunk's states and decays into registers
    const unsigned a_tok = smem_u32(&s_tok[c * TOKC]);             // + 32 i
    const unsigned a_B = smem_u32(&s_B[0][SPL * j]);               // + 64 i
    const unsigned a_C = smem_u32(&s_C[0][SPL * j]);
    const f2_t hin[NP] = {pk2(hin4.x, hin4.y), pk2(hin4.z, hin4.w)};
    f2_t Hh[SUB][NP], Ha[SUB][NP];
    float* sp0 = &s_p[0][c * PC + j * SUB];
    float* sp1 = &s_p[1][c * PC + j * SUB];
    float* sp2 = &s_p[2][c * PC + j * SUB];
    {
      // operands of step i + 1 are loaded before step i is computed
      f2_t hc[NP] = {hin[0], hin[1]};
      ulonglong2 tk = lds_f4(a_tok), bp = lds_f4(a_B), cp = lds_f4(a_C);
#pragma unroll
      for (int i0 = 0; i0 < SUB; i0 += 4) {
        float ys[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = i0 + k;
          ulonglong2 tk_n = tk, bp_n = bp, cp_n = cp;
          if (i + 1 < SUB) {
            tk_n = lds_f4(a_tok + 32 * (i + 1));
            bp_n = lds_f4(a_B + 4 * kN * (i + 1));
            cp_n = lds_f4(a_C + 4 * kN * (i + 1));
          }
          const f2_t dt2 = tk.x, du2 = tk.y;
          const f2_t Bp[NP] = {bp.x, bp.y};
#pragma unroll
          for (int q = 0; q < NP; ++q) {
            f2_t a = ex2_2(mul2(dt2, A2[q]));
            if (rst & (1u << i)) a = pk2(0.f, 0.f);
            hc[q] = fma2(a, hc[q], mul2(du2, Bp[q]));
            Ha[i][q] = a;
            Hh[i][q] = hc[q];
          }
          const f2_t r = fma2(cp.y, hc[1], mul2(cp.x, hc[0]));
          ys[k] = lo2(r) + hi2(r);
          tk = tk_n; bp = bp_n; cp = cp_n;
        }
        *reinterpret_cast<float4*>(sp2 + i0) = make_float4(ys[0], ys[1], ys[2], ys[3]);
      }
    }

    // ---- walk the sub-chunk backwards; operands of step i - 1 are loaded
    // before step i is computed and its dB / dC stored (the stores would
    // otherwise pin the next loads behind them)
    {
      ulonglong2 tk = lds_f4(a_tok + 32 * (SUB - 1)), bp = lds_f4(a_B + 4 * kN * (SUB - 1)),
                 cp = lds_f4(a_C + 4 * kN * (SUB - 1));
      f2_t do2 = lds_f2(a_tok + 32 * (SUB - 1) + 16);
#pragma unroll
      for (int i0 = SUB - 4; i0 >= 0; i0 -= 4) {
        float s1v[4], s2v[4];
#pragma unroll
        for (int k = 3; k >= 0; --k) {
          const int i = i0 + k;
          ulonglong2 tk_n = tk, bp_n = bp, cp_n = cp;
          f2_t do_n = do2;
          if (i > 0) {
            tk_n = lds_f4(a_tok + 32 * (i - 1));
            do_n = lds_f2(a_tok + 32 * (i - 1) + 16);
            bp_n = lds_f4(a_B + 4 * kN * (i - 1));
            cp_n = lds_f4(a_C + 4 * kN * (i - 1));
          }
          const f2_t dt2 = tk.x, du2 = tk.y;
          const f2_t Bp[NP] = {bp.x, bp.y};
          const f2_t Cp[NP] = {cp.x, cp.y};
          f2_t g[NP], qv[NP], dBv[NP], dCv[NP];
#pragma unroll
          for (int q = 0; q < NP; ++q) {
            const f2_t hprev = i > 0 ? Hh[i > 0 ? i - 1 : 0][q] : hin[q];
            g[q] = fma2(do2, Cp[q], carry[q]);
            dCv[q] = mul2(do2, Hh[i][q]);
            dBv[q] = mul2(g[q], du2);
            qv[q] = mul2(g[q], mul2(Ha[i][q], hprev));
            dA[q] = fma2(dt2, qv[q], dA[q]);
            carry[q] = mul2(Ha[i][q], g[q]);
          }
          const f2_t r1 = fma2(g[1], Bp[1], mul2(g[0], Bp[0]));
          const f2_t r2 = fma2(Aq[1], qv[1], mul2(Aq[0], qv[0]));
          s1v[k] = lo2(r1) + hi2(r1);
          s2v[k] = lo2(r2) + hi2(r2);
          *reinterpret_cast<ulonglong2*>(&s_red[(i * 2 + 0) * RED_SLAB + c * kN + SPL * j]) =
              make_ulonglong2(dBv[0], dBv[1]);
          *reinterpret_cast<ulonglong2*>(&s_red[(i * 2 + 1) * RED_SLAB + c * kN + SPL * j]) =
              make_ulonglong2(dCv[0], dCv[1]);
          tk = tk_n; bp = bp_n; cp = cp_n; do2 = do_n;
        }
        *reinterpret_cast<float4*>(sp0 + i0) = make_float4(s1v[0], s1v[1], s1v[2], s1v[3]);
        *reinterpret_cast<float4*>(sp1 + i0) = make_float4(s2v[0], s2v[1], s2v[2], s2v[3]);
      }
    }
    __syncthreads();

    // ---- epilogue: thread (c, j) owns steps 2j, 2j+1
    {
      f2_t S[3];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const float* src = &s_p[q][c * PC + 2 * j];
        S[q] = *reinterpret_cast<const f2_t*>(src);
#pragma unroll
        for (int l = 1; l < KL; ++l) S[q] = add2(S[q], *reinterpret_cast<const f2_t*>(src + l * SUB));
      }
      const float S1[2] = {lo2(S[0]), hi2(S[0])};
      const float S2[2] = {lo2(S[1]), hi2(S[1])};
      const float YS[2] = {lo2(S[2]), hi2(S[2])};
      float duo[2], ddo[2], dzo[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        duo[i] = fmaf(e_do[i], Dd, e_dt[i] * S1[i]);
        const float ddx = fmaf(e_u[i], S1[i], S2[i]) * e_sx[i];
        ddo[i] = ddx;
        dzo[i] = fmaf(Dd, e_u[i], YS[i]) * e_dzf[i];
        dD_acc = fmaf(e_do[i], e_u[i], dD_acc);
        dbias_acc += (dvalid && t0 + 2 * j + i < L) ? ddx : 0.f;
      }
      if (dvalid) {
        const int t = t0 + 2 * j;
        T* du_row = static_cast<T*>(p.du) + row;
        T* dd_row = static_cast<T*>(p.ddelta) + row;
        T* dz_row = has_z ? static_cast<T*>(p.dz) + row : nullptr;
        if (VEC && t + 2 <= L) {
          using V2 = typename std::conditional<sizeof(T) == 4, float2, uint32_t>::type;
          auto pack = [](float a, float bb) -> V2 {
            if constexpr (sizeof(T) == 4) {
              return make_float2(a, bb);
            } else {
              T pr[2] = {Elt<T>::from_f(a), Elt<T>::from_f(bb)};
              return (uint32_t)(*reinterpret_cast<const unsigned short*>(&pr[0])) |
                     ((uint32_t)(*reinterpret_cast<const unsigned short*>(&pr[1])) << 16);
            }
          };
          *reinterpret_cast<V2*>(du_row + t) = pack(duo[0], duo[1]);
          *reinterpret_cast<V2*>(dd_row + t) = pack(ddo[0], ddo[1]);
          if (dz_row) *reinterpret_cast<V2*>(dz_row + t) = pack(dzo[0], dzo[1]);
        } else {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (t + i < L) {
              du_row[t + i] = Elt<T>::from_f(duo[i]);
              dd_row[t + i] = Elt<T>::from_f(ddo[i]);
              if (dz_row) dz_row[t + i] = Elt<T>::from_f(dzo[i]);
            }
          }
        }
      }
    }
    // ---- channel sums of dB, dC for the sub-chunk, fixed order, f32x2 adds
    {
      const int i = tid >> 3, q = (tid >> 2) & 1, ng = tid & 3;
      const float* src = &s_red[(i * 2 + q) * RED_SLAB + 4 * ng];
      ulonglong2 acc = *reinterpret_cast<const ulonglong2*>(src);
#pragma unroll
      for (int cc = 1; cc < CB; ++cc) {
        const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(src + cc * kN);
        acc.x = add2(acc.x, v.x);
        acc.y = add2(acc.y, v.y);
      }
      float* part = (q ? p.part_dC : p.part_dB) +
                    (((size_t)b * p.nblk + blk) * Lp + t0 + i) * kN + 4 * ng;
      if (t0 + i < Lp) *reinterpret_cast<ulonglong2*>(part) = acc;
    }
  }

  const size_t part_row = (size_t)grp * p.batch + b;  // partial-sum row (group, batch row)
  if (dvalid) {
    float* pa = p.part_dA + (part_row * p.dim + d) * kN + SPL * j;
    *reinterpret_cast<float4*>(pa) = make_float4(lo2(dA[0]), hi2(dA[0]), lo2(dA[1]), hi2(dA[1]));
    // after step 0 the carry is Abar_0 g_0 = dloss / dh0
    if (p.dh0 && grp == 0)
      *reinterpret_cast<float4*>(p.dh0 + ((size_t)b * p.dim + d) * kN + SPL * j) =
          make_float4(lo2(carry[0]), hi2(carry[0]), lo2(carry[1]), hi2(carry[1]));
  }
  // the 4 lanes of a channel hold disjoint time steps: combine in a fixed order
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 1);
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 2);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 1);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 2);
  if (dvalid && j == 0) {
    p.part_dD[part_row * p.dim + d] = dD_acc;
    p.part_dbias[part_row * p.dim + d] = dbias_acc;
  }
}

// -------------------------------------------------------------------------
// 2'. Reverse walk, two channels per thread.  Shared-memory bandwidth bounds
// the one-channel walk: every lane re-reads B_t, C_t for its 4 states and
// stages per-channel dB, dC for the channel sums.  Here a thread carries the
// same 4 states of two channels, so one B / C load serves both and dB, dC
// are summed over the pair before staging.  The decays are recomputed in the
// reverse sweep instead of kept (the SFU has room in this pass), leaving the
// 8-step state history of both channels in registers.  Channel and state
// sums are reduced in two 4-step halves to halve their staging buffers.
// -------------------------------------------------------------------------
#ifndef SS_BWD2_WARPS_PER_SM
#define SS_BWD2_WARPS_PER_SM 10   // 16-bit storage; fp32 rows need more registers (8)
#endif
template <typename T, bool VEC, int CB, bool SEQ>
__global__ void __launch_bounds__(2 * CB, (sizeof(T) == 4 ? 8 : SS_BWD2_WARPS_PER_SM) * 16 / CB)
bwd2_kernel(const BwdParams p) {
  static_assert(CB == 16 || CB == 32, "16 or 32 channels per block");
  constexpr int NT = 2 * CB;                       // threads: CB / 2 pairs x 4 lanes
  constexpr int NPR = CB / 2;
  constexpr int ES = (int)sizeof(T);
  constexpr int ROWB = SUB * ES;                   // one 8-step row in storage format
  constexpr int HRB = 4 * ES;                      // half row (4 steps) in storage format
  // Strides below are chosen so that every shared access of a warp is free
  // of bank conflicts: a quarter-warp of 16-byte accesses (or a half-warp of
  // 8-byte ones) touches 32 distinct banks.
  constexpr int CHB = 4 * ROWB + 16;               // raw-tile channel stride (padded)
  constexpr int TKS = SUB + 1;                     // s_tk channel stride (float4, padded)
  // s_s12 holds, per lane j, a slab of CB channels x 4 steps; slab j starts at
  // 4 CB j + {0, 4, 16, 20}[j] floats, so the four slabs sit 0, 4, 16 and 20
  // banks apart with no more padding than that
  constexpr int S12N = 16 * CB + 20;
  constexpr int RSLAB = NPR * kN + 4;              // s_red (step, q) slab (floats)
  __shared__ __align__(16) unsigned char s_in[2][CB * CHB];        // u, delta, z, dy rows
  __shared__ __align__(16) unsigned char s_bcr[2][2 * kN * ROWB];  // B, C rows
  __shared__ __align__(16) float4 s_hin[2][2][NT];                 // entering states
  // B_t (columns 0-15) and C_t (16-31) of each step; a row stride of 36
  // floats puts the two 4-step halves of a transposed store in distinct banks
  constexpr int BCS = 2 * kN + 4;
  __shared__ __align__(16) float s_BC[SUB][BCS];
  // per (channel, step): Delta, Delta u, dout, softplus'(x); one 16-byte row
  // serves both the recompute (first 8 bytes) and the reverse sweep
  __shared__ __align__(16) float4 s_tk[CB * TKS];
  // (dz factor, u) per (channel, step): four 16-byte pieces per channel, piece v
  // of channel c stored at slot v ^ ((c >> 1) & 3) of the channel's four
  __shared__ __align__(16) float4 s_zu[CB * 4];
  __shared__ __align__(16) float s_s12[3][S12N];                   // per-lane g.B, A q, C.h over 4 steps
  __shared__ __align__(16) float s_red[4 * 2 * RSLAB];             // pair-summed dB / dC
  // du, ddelta, dz rows of the last sub-chunk (vector path), as half rows
  // [array][half][channel]: written out as whole 16-byte row pieces at the
  // top of the next iteration
  __shared__ __align__(16) unsigned char s_out[VEC ? 3 * CB * ROWB : 16];

  const int tid = threadIdx.x;
  const int b = blockIdx.y, blk = blockIdx.x;
  const int L = p.seqlen;
  const int Lp = (L + 15) & ~15;
  const bool has_z = p.z != nullptr;
  const int* seq_row = p.seq_idx ? p.seq_idx + (size_t)b * L : nullptr;
  // a one-warp block needs only a warp barrier (which also orders its shared memory)
  auto block_sync = [] {
    if constexpr (NT == 32) __syncwarp();
    else __syncthreads();
  };
  // main-loop role: pair pr (channels 2pr, 2pr+1), states 4j..4j+3
  const int pr = tid >> 2, j = tid & 3;
  // prologue / epilogue role: channel ce, step half k2 (prologue: steps
  // 4k2..4k2+3; epilogue of half h: steps 4h+2k2, 4h+2k2+1).  A quarter-warp
  // holds 8 channels of one k2.
  const int ce = (tid & 7) | ((tid >> 4) << 3), k2 = (tid >> 3) & 1;

  auto dglob = [&](int cl) { return blk * CB + cl; };
  const int dE = dglob(ce);
  const bool eval = dE < p.dim;
  const size_t rowE = ((size_t)b * p.dim + (eval ? dE : 0)) * (size_t)L;

  // store the staged du / ddelta / dz rows of the sub-chunk starting at step t
  auto flush_rows = [&](int t) {
    constexpr int PPR = ROWB / 16;                 // 16-byte pieces per row
    const int nbytes = min(SUB, L - t) * ES;       // a multiple of 16 on the vector path
#pragma unroll
    for (int r = tid; r < 3 * CB * PPR; r += NT) {
      const int cl = r % CB, w = (r / CB) % PPR, a = r / (CB * PPR);
      const int dg = dglob(cl);
      if (dg >= p.dim || 16 * w >= nbytes || (a == 2 && !has_z)) continue;
      void* base = a == 0 ? p.du : a == 1 ? p.ddelta : p.dz;
      unsigned char* dst = static_cast<unsigned char*>(base) + (((size_t)b * p.dim + dg) * L + t) * ES + 16 * w;
      uint4 v;
      if constexpr (PPR == 1) {  // 16-bit rows: the piece is both half rows
        const uint2 lo = *reinterpret_cast<const uint2*>(&s_out[((2 * a + 0) * CB + cl) * HRB]);
        const uint2 hi = *reinterpret_cast<const uint2*>(&s_out[((2 * a + 1) * CB + cl) * HRB]);
        v = make_uint4(lo.x, lo.y, hi.x, hi.y);
      } else {                   // fp32 rows: the piece is half row w
        v = *reinterpret_cast<const uint4*>(&s_out[((2 * a + w) * CB + cl) * HRB]);
      }
      *reinterpret_cast<uint4*>(dst) = v;
    }
  };

  // staging roles: raw rows r = tid, tid + NT (channel r % CB, array r / CB)
  const T* st_row[2];
  int st_c[2], st_a[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int r = tid + NT * k;
    st_c[k] = r % CB;
    st_a[k] = r / CB;
    const int dg = dglob(st_c[k]);
    const void* arr = st_a[k] == 0 ? p.u : st_a[k] == 1 ? p.delta : st_a[k] == 2 ? p.z : p.dy;
    st_row[k] = arr ? static_cast<const T*>(arr) + ((size_t)b * p.dim + (dg < p.dim ? dg : 0)) * L : nullptr;
  }
  const int g_q = tid >> 4, g_n = tid & 15;
  const T* __restrict__ g_row = static_cast<const T*>(g_q ? p.C : p.B) + ((size_t)b * kN + g_n) * L;
  const float* hs[2];
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const int dg = dglob(2 * pr + ch);
    hs[ch] = p.sub_state + ((size_t)b * p.dim + (dg < p.dim ? dg : 0)) * (size_t)p.nsub * kN + SPL * j;
  }

  auto stage = [&](int sc, int buf) {
    const int t = sc * SUB;
    const int nvalid = min(SUB, L - t);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (!st_row[k]) continue;
      unsigned char* dst = &s_in[buf][st_c[k] * CHB + st_a[k] * ROWB];
      if (VEC) {
#pragma unroll
        for (int w = 0; w < ROWB / 16; ++w) {
          const int bytes = max(0, min(16, nvalid * ES - 16 * w));
          cp_async16(dst + 16 * w, bytes > 0 ? (const void*)(st_row[k] + t + 16 * w / ES) : (const void*)st_row[k], bytes);
        }
      } else {
        T* dt_ = reinterpret_cast<T*>(dst);
#pragma unroll
        for (int i = 0; i < SUB; ++i) dt_[i] = i < nvalid ? st_row[k][t + i] : T(0.f);
      }
    }
    if (tid < 32) {
      unsigned char* dst = &s_bcr[buf][(g_q * kN + g_n) * ROWB];
      if (VEC) {
#pragma unroll
        for (int w = 0; w < ROWB / 16; ++w) {
          const int bytes = max(0, min(16, nvalid * ES - 16 * w));
          cp_async16(dst + 16 * w, bytes > 0 ? (const void*)(g_row + t + 16 * w / ES) : (const void*)g_row, bytes);
        }
      } else {
        T* dt_ = reinterpret_cast<T*>(dst);
#pragma unroll
        for (int i = 0; i < SUB; ++i) dt_[i] = i < nvalid ? g_row[t + i] : T(0.f);
      }
    }
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      if (VEC) cp_async16(&s_hin[buf][ch][tid], hs[ch] + (size_t)sc * kN, 16);
      else s_hin[buf][ch][tid] = *reinterpret_cast<const float4*>(hs[ch] + (size_t)sc * kN);
    }
    if (VEC) cp_async_commit();
  };

  // per-channel constants of the main-loop role; the carry entering the
  // group's last step is composed from the later groups, or (one group) the
  // gradient reaching the final state from outside
  const int grp = blockIdx.z;
  const int sc_lo = grp * p.group_nsub, sc_hi = min(p.nsub, sc_lo + p.group_nsub) - 1;
  f2_t A2[2][NP], carry[2][NP], dA[2][NP];
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const int dg = dglob(2 * pr + ch);
    const size_t bd = (size_t)b * p.dim + (dg < p.dim ? dg : 0);
    const float* a = p.A + (size_t)(dg < p.dim ? dg : 0) * kN + SPL * j;
    const float* cin = p.ngroups > 1 ? p.group_carry + (bd * p.ngroups + grp) * kN
                       : p.dfinal     ? p.dfinal + bd * kN
                                      : nullptr;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      A2[ch][q] = pk2(a[2 * q] * kLog2e, a[2 * q + 1] * kLog2e);
      carry[ch][q] = dA[ch][q] = pk2(0.f, 0.f);
      if (cin) carry[ch][q] = pk2(cin[SPL * j + 2 * q], cin[SPL * j + 2 * q + 1]);
    }
  }
  // constants of the epilogue role
  const float DdE = p.D ? p.D[eval ? dE : 0] : 0.f;
  const float biasE = p.bias ? p.bias[eval ? dE : 0] : 0.f;
  float dD_acc = 0.f, dbias_acc = 0.f;

  const unsigned a_tk0 = smem_u32(&s_tk[(2 * pr) * TKS]);          // + 16 i (+ 16 TKS for ch 1)
  auto dup_lo = [](f2_t v) { return pk2(lo2(v), lo2(v)); };
  auto dup_hi = [](f2_t v) { return pk2(hi2(v), hi2(v)); };
  const unsigned a_B = smem_u32(&s_BC[0][SPL * j]);                // + 4 BCS i
  const unsigned a_C = a_B + 4 * kN;

  stage(sc_hi, sc_hi & 1);

  for (int sc = sc_hi; sc >= sc_lo; --sc) {
    const int buf = sc & 1;
    const int t0 = sc * SUB;
    // steps of this sub-chunk that start a new document: zero decay, so
    // neither the state nor its gradient crosses the boundary
    const unsigned rst = SEQ ? doc_starts32(seq_row, t0, min(L, t0 + SUB)) : 0u;
    if (VEC) cp_async_wait_all();
    block_sync();
    if (sc > sc_lo) stage(sc - 1, buf ^ 1);
    if (VEC && sc < sc_hi) flush_rows((sc + 1) * SUB);

    // ---- B / C to fp32 [step][n]: 4 elements per (thread, pass)
#pragma unroll
    for (int e = tid; e < 64; e += NT) {
      const int q = e >> 5, n = (e >> 1) & 15, hf = e & 1;
      const float4 v = ld_quad<T>(&s_bcr[buf][(q * kN + n) * ROWB + 4 * hf * ES]);
      float* dst = &s_BC[4 * hf][kN * q + n];
      dst[0 * BCS] = v.x;
      dst[1 * BCS] = v.y;
      dst[2 * BCS] = v.z;
      dst[3 * BCS] = v.w;
    }
    // ---- per-token prologue: thread (ce, k2) owns steps 4k2 .. 4k2+3
    {
      const int i0 = 4 * k2;
      const unsigned char* base = &s_in[buf][ce * CHB + i0 * ES];
      const float4 uu = ld_quad<T>(base);
      const float4 xx = ld_quad<T>(base + ROWB);
      const float4 zz = has_z ? ld_quad<T>(base + 2 * ROWB) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 gg = ld_quad<T>(base + 3 * ROWB);
      const float uva[4] = {uu.x, uu.y, uu.z, uu.w}, xva[4] = {xx.x, xx.y, xx.z, xx.w},
                  zva[4] = {zz.x, zz.y, zz.z, zz.w}, gva[4] = {gg.x, gg.y, gg.z, gg.w};
      float zu[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tt = i0 + i;
        const bool ok = eval && (t0 + tt < L);
        const float x = xva[i] + biasE;
        float dt = x, sx = 1.f;
        if (p.softplus) {
          const float w = ex2(-fabsf(x) * kLog2e);
          dt = fmaxf(x, 0.f) + log1p_unit(w);
          const float r = rcp(1.f + w);
          sx = x >= 0.f ? r : w * r;
        }
        float gate = 1.f, dzf = 0.f;
        if (has_z) {
          const float sz = sigmoid_f(zva[i]);
          gate = zva[i] * sz;
          dzf = gva[i] * sz * fmaf(zva[i], 1.f - sz, 1.f);
        }
        dt = ok ? dt : 0.f;
        const float dout = ok ? gva[i] * gate : 0.f;
        const float du = dt * uva[i];
        s_tk[ce * TKS + tt] = make_float4(dt, du, dout, sx);
        zu[2 * i] = dzf;
        zu[2 * i + 1] = ok ? uva[i] : 0.f;
      }
      const int zsw = (ce >> 1) & 3;
      s_zu[ce * 4 + ((2 * k2) ^ zsw)] = make_float4(zu[0], zu[1], zu[2], zu[3]);
      s_zu[ce * 4 + ((2 * k2 + 1) ^ zsw)] = make_float4(zu[4], zu[5], zu[6], zu[7]);
    }
    block_sync();

    // ---- recompute both channels' states into registers; readout partials
    f2_t Hh[2][SUB][NP];
    {
      f2_t hc[2][NP];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(&s_hin[buf][ch][tid]);
        hc[ch][0] = v.x;
        hc[ch][1] = v.y;
      }
#pragma unroll
      for (int i = 0; i < SUB; ++i) {
        const f2_t tk[2] = {lds_f2(a_tk0 + 16 * i), lds_f2(a_tk0 + 16 * TKS + 16 * i)};  // (dt, du)
        const ulonglong2 bp = lds_f4(a_B + 4 * BCS * i);
        const f2_t Bp[NP] = {bp.x, bp.y};
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const f2_t dt2 = dup_lo(tk[ch]), du2 = dup_hi(tk[ch]);
#pragma unroll
          for (int q = 0; q < NP; ++q) {
            f2_t a = ex2_2(mul2(dt2, A2[ch][q]));
            if (rst & (1u << i)) a = pk2(0.f, 0.f);
            hc[ch][q] = fma2(a, hc[ch][q], mul2(du2, Bp[q]));
            Hh[ch][i][q] = hc[ch][q];
          }
        }
      }
    }

    // ---- reverse sweep in two 4-step halves, each followed by its sums
#pragma unroll
    for (int h = 1; h >= 0; --h) {
      {
        float s1v[2][4], s2v[2][4], s3v[2][4];
#pragma unroll
        for (int k = 3; k >= 0; --k) {
          const int i = 4 * h + k;
          const ulonglong2 t0v = lds_f4(a_tk0 + 16 * i);                // (dt, du), (do, sx)
          const ulonglong2 t1v = lds_f4(a_tk0 + 16 * TKS + 16 * i);
          const ulonglong2 bp = lds_f4(a_B + 4 * BCS * i);
          const ulonglong2 cp = lds_f4(a_C + 4 * BCS * i);
          const f2_t dt2[2] = {dup_lo(t0v.x), dup_lo(t1v.x)}, du2[2] = {dup_hi(t0v.x), dup_hi(t1v.x)},
                     do2[2] = {dup_lo(t0v.y), dup_lo(t1v.y)};
          const f2_t Bp[NP] = {bp.x, bp.y};
          const f2_t Cp[NP] = {cp.x, cp.y};
          f2_t dBs[NP], dCs[NP];
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            f2_t g[NP], qv[NP], h0v[NP];
            if (i == 0) {
              const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(&s_hin[buf][ch][tid]);
              h0v[0] = v.x;
              h0v[1] = v.y;
            }
#pragma unroll
            for (int q = 0; q < NP; ++q) {
              f2_t a = ex2_2(mul2(dt2[ch], A2[ch][q]));
              if (rst & (1u << i)) a = pk2(0.f, 0.f);
              const f2_t hprev = i > 0 ? Hh[ch][i > 0 ? i - 1 : 0][q] : h0v[q];
              g[q] = fma2(do2[ch], Cp[q], carry[ch][q]);
              const f2_t dCv = mul2(do2[ch], Hh[ch][i][q]);
              const f2_t dBv = mul2(g[q], du2[ch]);
              dCs[q] = ch == 0 ? dCv : add2(dCs[q], dCv);
              dBs[q] = ch == 0 ? dBv : add2(dBs[q], dBv);
              carry[ch][q] = mul2(a, g[q]);
              qv[q] = mul2(carry[ch][q], hprev);
              dA[ch][q] = fma2(dt2[ch], qv[q], dA[ch][q]);
            }
            const f2_t r1 = fma2(g[1], Bp[1], mul2(g[0], Bp[0]));
            // sum_n A qv, taken in the log2e-scaled A (undone in the epilogue)
            const f2_t r2 = fma2(A2[ch][1], qv[1], mul2(A2[ch][0], qv[0]));
            // the recomputed readout C.h_t, needed by dz
            const f2_t r3 = fma2(Cp[1], Hh[ch][i][1], mul2(Cp[0], Hh[ch][i][0]));
            s1v[ch][k] = lo2(r1) + hi2(r1);
            s2v[ch][k] = lo2(r2) + hi2(r2);
            s3v[ch][k] = lo2(r3) + hi2(r3);
          }
          *reinterpret_cast<ulonglong2*>(&s_red[(k * 2 + 0) * RSLAB + pr * kN + SPL * j]) =
              make_ulonglong2(dBs[0], dBs[1]);
          *reinterpret_cast<ulonglong2*>(&s_red[(k * 2 + 1) * RSLAB + pr * kN + SPL * j]) =
              make_ulonglong2(dCs[0], dCs[1]);
        }
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int o = 4 * CB * j + 4 * (j & 1) + 16 * (j >> 1) + 4 * (2 * pr + ch);
          *reinterpret_cast<float4*>(&s_s12[0][o]) = make_float4(s1v[ch][0], s1v[ch][1], s1v[ch][2], s1v[ch][3]);
          *reinterpret_cast<float4*>(&s_s12[1][o]) = make_float4(s2v[ch][0], s2v[ch][1], s2v[ch][2], s2v[ch][3]);
          *reinterpret_cast<float4*>(&s_s12[2][o]) = make_float4(s3v[ch][0], s3v[ch][1], s3v[ch][2], s3v[ch][3]);
        }
      }
      block_sync();

      // ---- epilogue of the half: thread (ce, k2) owns steps 4h + 2k2 + {0, 1}
      {
        f2_t S1 = pk2(0.f, 0.f), S2 = pk2(0.f, 0.f), YS = pk2(0.f, 0.f);
#pragma unroll
        for (int l = 0; l < KL; ++l) {
          const int o = 4 * CB * l + 4 * (l & 1) + 16 * (l >> 1) + 4 * ce + 2 * k2;
          S1 = add2(S1, *reinterpret_cast<const f2_t*>(&s_s12[0][o]));
          S2 = add2(S2, *reinterpret_cast<const f2_t*>(&s_s12[1][o]));
          YS = add2(YS, *reinterpret_cast<const f2_t*>(&s_s12[2][o]));
        }
        const float S1a[2] = {lo2(S1), hi2(S1)}, S2a[2] = {lo2(S2), hi2(S2)}, YSa[2] = {lo2(YS), hi2(YS)};
        const int tt0 = 4 * h + 2 * k2;
        // dz factor and u of the two steps (u zero where the step is not valid)
        const float4 zu = s_zu[ce * 4 + ((2 * h + k2) ^ ((ce >> 1) & 3))];
        const float dzfa[2] = {zu.x, zu.z}, uva[2] = {zu.y, zu.w};
        float duo[2], ddo[2], dzo[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float4 tk = s_tk[ce * TKS + tt0 + i];
          const float dt = tk.x, dout = tk.z;
          const bool ok = eval && t0 + tt0 + i < L;
          const float uv = uva[i];
          duo[i] = fmaf(dout, DdE, dt * S1a[i]);
          const float ddx = fmaf(uv, S1a[i], S2a[i] * kLn2) * tk.w;
          ddo[i] = ddx;
          dzo[i] = fmaf(DdE, uv, YSa[i]) * dzfa[i];
          dD_acc = fmaf(dout, uv, dD_acc);
          dbias_acc += ok ? ddx : 0.f;
        }
        if (VEC) {
          using V2 = typename std::conditional<sizeof(T) == 4, float2, uint32_t>::type;
          auto pack = [](float a, float bb) -> V2 {
            if constexpr (sizeof(T) == 4) {
              return make_float2(a, bb);
            } else {
              T pr2[2] = {Elt<T>::from_f(a), Elt<T>::from_f(bb)};
              return (uint32_t)(*reinterpret_cast<const unsigned short*>(&pr2[0])) |
                     ((uint32_t)(*reinterpret_cast<const unsigned short*>(&pr2[1])) << 16);
            }
          };
          unsigned char* so = &s_out[(h * CB + ce) * HRB + 2 * k2 * ES];
          *reinterpret_cast<V2*>(so) = pack(duo[0], duo[1]);
          *reinterpret_cast<V2*>(so + 2 * CB * HRB) = pack(ddo[0], ddo[1]);
          *reinterpret_cast<V2*>(so + 4 * CB * HRB) = pack(dzo[0], dzo[1]);
        } else if (eval) {
          const int t = t0 + 4 * h + 2 * k2;
          T* du_row = static_cast<T*>(p.du) + rowE;
          T* dd_row = static_cast<T*>(p.ddelta) + rowE;
          T* dz_row = has_z ? static_cast<T*>(p.dz) + rowE : nullptr;
          {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              if (t + i < L) {
                du_row[t + i] = Elt<T>::from_f(duo[i]);
                dd_row[t + i] = Elt<T>::from_f(ddo[i]);
                if (dz_row) dz_row[t + i] = Elt<T>::from_f(dzo[i]);
              }
            }
          }
        }
      }
      // ---- channel sums of the half.  Two warps: warp q sums dB (q = 0) or
      // dC (q = 1), lanes 0-15 over pairs 0-7 and lanes 16-31 over pairs 8-15,
      // then combined.  One warp: half-warp q sums all 8 pairs.
      if constexpr (CB == 16) {
        const int q = tid >> 4, task = tid & 15;
        const int i = task & 3, ng = task >> 2;
        const float* src = &s_red[(i * 2 + q) * RSLAB + 4 * ng];
        ulonglong2 acc = *reinterpret_cast<const ulonglong2*>(src);
#pragma unroll
        for (int k = 1; k < NPR; ++k) {
          const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(src + k * kN);
          acc.x = add2(acc.x, v.x);
          acc.y = add2(acc.y, v.y);
        }
        const int t = t0 + 4 * h + i;
        float* part = (q ? p.part_dC : p.part_dB) + (((size_t)b * p.nblk + blk) * Lp + t) * kN + 4 * ng;
        if (t < Lp) *reinterpret_cast<ulonglong2*>(part) = acc;
      } else {
        const int q = tid >> 5, lane = tid & 31;
        const int hp = lane >> 4, task = lane & 15;
        const int i = task & 3, ng = task >> 2;
        const float* src = &s_red[(i * 2 + q) * RSLAB + (8 * hp) * kN + 4 * ng];
        ulonglong2 acc = *reinterpret_cast<const ulonglong2*>(src);
#pragma unroll
        for (int k = 1; k < 8; ++k) {
          const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(src + k * kN);
          acc.x = add2(acc.x, v.x);
          acc.y = add2(acc.y, v.y);
        }
        // partner holds the other 8 pairs; lanes < 16 add (theirs + partner's)
        const unsigned x0 = __shfl_xor_sync(0xffffffffu, (unsigned)(acc.x & 0xffffffffull), 16);
        const unsigned x1 = __shfl_xor_sync(0xffffffffu, (unsigned)(acc.x >> 32), 16);
        const unsigned y0 = __shfl_xor_sync(0xffffffffu, (unsigned)(acc.y & 0xffffffffull), 16);
        const unsigned y1 = __shfl_xor_sync(0xffffffffu, (unsigned)(acc.y >> 32), 16);
        if (hp == 0) {
          acc.x = add2(acc.x, ((f2_t)x1 << 32) | x0);
          acc.y = add2(acc.y, ((f2_t)y1 << 32) | y0);
          const int t = t0 + 4 * h + i;
          float* part = (q ? p.part_dC : p.part_dB) + (((size_t)b * p.nblk + blk) * Lp + t) * kN + 4 * ng;
          if (t < Lp) *reinterpret_cast<ulonglong2*>(part) = acc;
        }
      }
      if (h == 1) block_sync();  // the second half reuses s_red and s_s12
    }
  }

  if (VEC) {
    block_sync();
    flush_rows(sc_lo * SUB);
  }
  const size_t part_row = (size_t)grp * p.batch + b;  // partial-sum row (group, batch row)
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const int dg = dglob(2 * pr + ch);
    if (dg < p.dim) {
      float* pa = p.part_dA + (part_row * p.dim + dg) * kN + SPL * j;
      *reinterpret_cast<float4*>(pa) =
          make_float4(lo2(dA[ch][0]), hi2(dA[ch][0]), lo2(dA[ch][1]), hi2(dA[ch][1]));
      if (p.dh0 && grp == 0)  // after step 0 the carry is Abar_0 g_0 = dloss / dh0
        *reinterpret_cast<float4*>(p.dh0 + ((size_t)b * p.dim + dg) * kN + SPL * j) =
            make_float4(lo2(carry[ch][0]), hi2(carry[ch][0]), lo2(carry[ch][1]), hi2(carry[ch][1]));
    }
  }
  // the two threads of a channel (lanes 8 apart) hold disjoint steps:
  // combine in a fixed order
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 8);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 8);
  if (eval && k2 == 0) {
    p.part_dD[part_row * p.dim + dE] = dD_acc;
    p.part_dbias[part_row * p.dim + dE] = dbias_acc;
  }
}

// -------------------------------------------------------------------------
// 3. Fixed-order sums.  dB[b,n,t] = sum over blocks of part[b,blk,t,n] (a
// 64-step tile per block, transposed through shared memory so both the
// partial reads and the output writes are coalesced); dA[d,n], dD[d],
// dbias[d] = sum over the (chunk group, batch row) partials, group-major.
// -------------------------------------------------------------------------
__global__ void __launch_bounds__(256) reduce_bc_kernel(const BwdParams p) {
  __shared__ float s_t[2][kN][64 + 1];
  const int L = p.seqlen, Lp = (L + 15) & ~15;
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * 64;
  const int tid = threadIdx.x;
  const int tl = tid >> 2, ng = tid & 3;  // step within tile, group of 4 states
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float* src = (q ? p.part_dC : p.part_dB) + ((size_t)b * p.nblk * Lp + t0 + tl) * kN + 4 * ng;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t0 + tl < Lp) {
      for (int k = 0; k < p.nblk; ++k) {
        const float4 v = *reinterpret_cast<const float4*>(src + (size_t)k * Lp * kN);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
    }
    s_t[q][4 * ng + 0][tl] = acc.x;
    s_t[q][4 * ng + 1][tl] = acc.y;
    s_t[q][4 * ng + 2][tl] = acc.z;
    s_t[q][4 * ng + 3][tl] = acc.w;
  }
  __syncthreads();
  for (int o = tid; o < 2 * kN * 64; o += 256) {
    const int q = o / (kN * 64), n = (o / 64) % kN, tt = o % 64;
    if (t0 + tt < L) (q ? p.dC : p.dB)[((size_t)b * kN + n) * L + t0 + tt] = s_t[q][n][tt];
  }
}

__global__ void reduce_param_kernel(const BwdParams p) {
  const long long nA = (long long)p.dim * kN, nD = p.dim;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nA + 2 * nD;
       i += (long long)gridDim.x * blockDim.x) {
    if (i < nA) {
      float s = 0.f;
      for (int r = 0; r < p.ngroups * p.batch; ++r) s += p.part_dA[(size_t)r * nA + i];
      p.dA[i] = s;
    } else {
      const long long r = i - nA;
      const int q = r >= nD;
      const long long dd = q ? r - nD : r;
      float* out = q ? p.dbias : p.dD;
      if (!out) continue;
      const float* src = q ? p.part_dbias : p.part_dD;
      float s = 0.f;
      for (int r = 0; r < p.ngroups * p.batch; ++r) s += src[(size_t)r * nD + dd];
      out[dd] = s;
    }
  }
}

// Blocks of a kernel that fit on one SM at once (0 on error).
template <typename K>
int resident_blocks(K kernel, int threads) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess) return 0;
  return n;
}

// Chunk groups for the reverse walk.  Each walk block's time is set by the
// chunks of its group; with R blocks resident on the GPU the walk takes about
// ceil(blocks / R) x (chunks per group) block-chunk times.  More groups fill
// the GPU when there are few channel blocks, but every group adds carry maps
// to the states pass and partial rows to the reductions, which that count
// leaves out: the fewest groups within 15% of the best count are taken, and a
// split must save at least 10% over one group.
void choose_groups(BwdParams& p, int blocks_per_sm) {
  p.ngroups = 1;
  p.group_nsub = p.nsub;
  const long long base = (long long)p.nblk * p.batch;
  const long long R = (long long)(blocks_per_sm > 0 ? blocks_per_sm : 1) * (p.sms > 0 ? p.sms : 1);
  const int gmax = p.nchunk < kMaxBwdGroups ? p.nchunk : kMaxBwdGroups;
  long long cost[kMaxBwdGroups + 1];
  int gcs[kMaxBwdGroups + 1];
  const long long one = ((base + R - 1) / R) * p.nchunk;
  long long best = one;
  for (int g = 1; g <= gmax; ++g) {
    const int gc = (p.nchunk + g - 1) / g;          // chunks per group
    gcs[g] = gc;
    cost[g] = (p.nchunk + gc - 1) / gc != g ? -1     // that count leaves a group empty
                                            : ((base * g + R - 1) / R) * gc;
    if (cost[g] >= 0 && cost[g] < best) best = cost[g];
  }
  if (best * 10 > one * 9) return;                  // splitting saves too little
  for (int g = 2; g <= gmax; ++g) {
    if (cost[g] >= 0 && cost[g] * 100 <= best * 115) {
      p.ngroups = g;
      p.group_nsub = gcs[g] * (kChunk / SUB);
      return;
    }
  }
}

// Threads per block of the walk variant, and the chunk groups for p.
template <typename T, bool VEC, bool SEQ>
int plan_walk(BwdParams& p) {
  int threads, per_sm;
  if (p.variant == kBwdPairs32) {
    threads = 64;
    per_sm = resident_blocks(bwd2_kernel<T, VEC, 32, SEQ>, threads);
  } else if (p.variant == kBwdPairs16) {
    threads = 32;
    per_sm = resident_blocks(bwd2_kernel<T, VEC, 16, SEQ>, threads);
  } else {
    threads = 16 * KL;
    per_sm = resident_blocks(bwd_kernel<T, VEC, SEQ>, threads);
  }
  choose_groups(p, per_sm);
  return threads;
}

template <typename T, bool VEC, bool SEQ>
cudaError_t launch_bwd_s(const BwdParams& p0, cudaStream_t s) {
  BwdParams p = p0;
  const int threads = plan_walk<T, VEC, SEQ>(p);
  {
    // the chunks of group 0 need no carry map (nothing is composed through them)
    const int plain = p.ngroups > 1 ? p.group_nsub / (kChunk / SUB) : p.nchunk;
    const dim3 g0((p.dim + 63) / 64, p.batch, plain);
    states_kernel<T, VEC, SEQ, false><<<g0, 128, 0, s>>>(p, 0);
    if (p.ngroups > 1) {
      const dim3 g1((p.dim + 63) / 64, p.batch, p.nchunk - plain);
      states_kernel<T, VEC, SEQ, true><<<g1, 128, 0, s>>>(p, plain);
    }
  }
  if (p.ngroups > 1) {
    const long long n = (long long)p.batch * p.dim * (kN / 4);
    group_carry_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
  }
  {
    const int cb = bwd_block_channels(p.variant);
    const dim3 g((p.dim + cb - 1) / cb, p.batch, p.ngroups);
    if (p.variant == kBwdPairs32) bwd2_kernel<T, VEC, 32, SEQ><<<g, threads, 0, s>>>(p);
    else if (p.variant == kBwdPairs16) bwd2_kernel<T, VEC, 16, SEQ><<<g, threads, 0, s>>>(p);
    else bwd_kernel<T, VEC, SEQ><<<g, threads, 0, s>>>(p);
  }
  {
    const dim3 g((p.seqlen + 63) / 64, p.batch);
    reduce_bc_kernel<<<g, 256, 0, s>>>(p);
    const long long total = (long long)p.dim * kN + 2LL * p.dim;
    long long blocks = (total + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    reduce_param_kernel<<<(unsigned)blocks, 256, 0, s>>>(p);
  }
  return cudaGetLastError();
}

// packed documents get the document-aware kernels; plain rows skip the checks
template <typename T, bool VEC>
cudaError_t launch_bwd_t(const BwdParams& p, cudaStream_t s) {
  return p.seq_idx ? launch_bwd_s<T, VEC, true>(p, s) : launch_bwd_s<T, VEC, false>(p, s);
}

}  // namespace

template <typename T>
void plan_bwd_t(BwdParams& p, bool vec) {
  if (vec) {
    if (p.seq_idx) plan_walk<T, true, true>(p); else plan_walk<T, true, false>(p);
  } else {
    if (p.seq_idx) plan_walk<T, false, true>(p); else plan_walk<T, false, false>(p);
  }
}

cudaError_t plan_bwd(BwdParams& p, DType dt, bool vec) {
  switch (dt) {
    case DType::F32: plan_bwd_t<float>(p, vec); break;
    case DType::BF16: plan_bwd_t<__nv_bfloat16>(p, vec); break;
    case DType::F16: plan_bwd_t<__half>(p, vec); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t launch_bwd(const BwdParams& p, DType dt, bool vec, cudaStream_t s) {
  switch (dt) {
    case DType::F32: return vec ? launch_bwd_t<float, true>(p, s) : launch_bwd_t<float, false>(p, s);
    case DType::BF16:
      return vec ? launch_bwd_t<__nv_bfloat16, true>(p, s) : launch_bwd_t<__nv_bfloat16, false>(p, s);
    case DType::F16: return vec ? launch_bwd_t<__half, true>(p, s) : launch_bwd_t<__half, false>(p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ss
