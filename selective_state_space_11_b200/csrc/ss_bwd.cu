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
// the 64-step chunks in reverse, recompute each chunk from its checkpoint,
// carry the state gradient across chunk boundaries in registers):
//   * 4 lanes per channel, 4 states per lane; 16 channels per block;
//   * per chunk: per-token scalars (Delta, Delta*u, dout) once into shared
//     memory; a forward pass from the checkpoint records the states entering
//     sub-chunks 1..3; then for each 16-step sub-chunk, latest first, the
//     states and decays are recomputed into registers (16 x 4 x 2 values) and
//     walked backwards;
//   * sums over the state index (for du, dDelta and the recomputed readout
//     C.h used by dz) meet in shared memory; sums over channels (dB, dC) are
//     formed per block in a fixed order and written as per-block partials;
//   * a second kernel adds the per-block and per-batch partials in a fixed
//     order -- deterministic, no floating-point atomics (the Metal design on
//     that page reduces with threadgroup memory plus float atomics).
#include "ss_device.cuh"
#include "ss_internal.h"

namespace ss {
namespace {

constexpr int KL = 4, SPL = 4;
constexpr int CH = kChunk;   // 64
constexpr int SUB = 16;      // sub-chunk length held in registers
constexpr int CHP = CH + 4;
constexpr int SUBP = SUB + 4;

__device__ __forceinline__ void load4_row_f(const float* row, int t, int len, bool vec, float (&v)[4]) {
  if (vec && t + 4 <= len) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + t));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = (t + i < len) ? __ldg(row + t + i) : 0.f;
  }
}
template <typename T>
__device__ __forceinline__ void load4_row(const T* row, int t, int len, bool vec, float (&v)[4]) {
  if (vec && t + 4 <= len) {
    const uint2 r = __ldg(reinterpret_cast<const uint2*>(row + t));
    const T* e = reinterpret_cast<const T*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = Elt<T>::to_f(e[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = (t + i < len) ? ldf(row + t + i) : 0.f;
  }
}
template <>
__device__ __forceinline__ void load4_row<float>(const float* row, int t, int len, bool vec, float (&v)[4]) {
  load4_row_f(row, t, len, vec, v);
}
template <typename T>
__device__ __forceinline__ void store4_row(T* row, int t, int len, bool vec, const float (&v)[4]) {
  if (vec && t + 4 <= len) {
    uint2 r;
    T* e = reinterpret_cast<T*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) e[i] = Elt<T>::from_f(v[i]);
    *reinterpret_cast<uint2*>(row + t) = r;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (t + i < len) stf(row + t + i, v[i]);
  }
}
template <>
__device__ __forceinline__ void store4_row<float>(float* row, int t, int len, bool vec, const float (&v)[4]) {
  if (vec && t + 4 <= len) {
    *reinterpret_cast<float4*>(row + t) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (t + i < len) row[t + i] = v[i];
  }
}

template <typename T, int CB, bool VEC>
__global__ void __launch_bounds__(CB * KL, 3)
bwd_kernel(const BwdParams p) {
  constexpr int NT = CB * KL;
  constexpr int NW = NT / 32;
  constexpr int RED_SLAB = CB * kN + 16;  // padded (t, q) slab of the channel-sum buffer
  // dynamic shared memory (about 71 KB at 16 channels per block)
  extern __shared__ __align__(16) float smem[];
  float(*s_dt)[CHP] = reinterpret_cast<float(*)[CHP]>(smem);                 // Delta
  float(*s_du)[CHP] = reinterpret_cast<float(*)[CHP]>(smem + CB * CHP);      // Delta * u
  float(*s_do)[CHP] = reinterpret_cast<float(*)[CHP]>(smem + 2 * CB * CHP);  // dy * SiLU(z)
  float(*s_B)[kN] = reinterpret_cast<float(*)[kN]>(smem + 3 * CB * CHP);
  float(*s_C)[kN] = reinterpret_cast<float(*)[kN]>(smem + 3 * CB * CHP + CH * kN);
  // per-lane partial sums over n: [quantity][channel][lane][step]
  float(*s_p)[CB][KL][SUBP] =
      reinterpret_cast<float(*)[CB][KL][SUBP]>(smem + 3 * CB * CHP + 2 * CH * kN);
  // per-channel dB / dC of the sub-chunk: [step][q][channel][n], slabs padded
  float* s_red = smem + 3 * CB * CHP + 2 * CH * kN + 3 * CB * KL * SUBP;

  const int tid = threadIdx.x;
  const int c = tid / KL, j = tid % KL;
  const int b = blockIdx.y, blk = blockIdx.x;
  const int d = blk * CB + c;
  const bool dvalid = d < p.dim;
  const int dd = dvalid ? d : 0;
  const int L = p.seqlen;
  const int Lp = (L + 15) & ~15;

  const size_t row = ((size_t)b * p.dim + dd) * (size_t)L;
  const T* __restrict__ u_row = static_cast<const T*>(p.u) + row;
  const T* __restrict__ x_row = static_cast<const T*>(p.delta) + row;
  const T* __restrict__ z_row = p.z ? static_cast<const T*>(p.z) + row : nullptr;
  const T* __restrict__ g_row = static_cast<const T*>(p.dy) + row;
  const T* __restrict__ Bb = static_cast<const T*>(p.B) + (size_t)b * kN * L;
  const T* __restrict__ Cb = static_cast<const T*>(p.C) + (size_t)b * kN * L;

  float A2[SPL], Aq[SPL];
#pragma unroll
  for (int k = 0; k < SPL; ++k) {
    Aq[k] = p.A[(size_t)dd * kN + SPL * j + k];
    A2[k] = Aq[k] * kLog2e;
  }
  const float Dd = p.D ? p.D[dd] : 0.f;
  const float bias = p.bias ? p.bias[dd] : 0.f;

  float carry[SPL], dA[SPL];
#pragma unroll
  for (int k = 0; k < SPL; ++k) carry[k] = dA[k] = 0.f;
  float dD_acc = 0.f, dbias_acc = 0.f;

  for (int kc = p.nchunk - 1; kc >= 0; --kc) {
    const int t0 = kc * CH;
    // ---- per-token prologue: thread (c, j) owns steps [16j, 16j+16)
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
      const int tt = 16 * j + 8 * grp;
      const int t = t0 + tt;
      float uv[8], xv[8], zv[8], gv[8];
      load8_row<T, VEC>(u_row, t, L, uv);
      load8_row<T, VEC>(x_row, t, L, xv);
      load8_row<T, VEC>(g_row, t, L, gv);
      if (z_row) load8_row<T, VEC>(z_row, t, L, zv);
      float dt8[8], du8[8], do8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool ok = dvalid && (t + i < L);
        const float x = xv[i] + bias;
        float dt = p.softplus ? softplus_f(x) : x;
        dt = ok ? dt : 0.f;
        const float gate = z_row ? zv[i] * sigmoid_f(zv[i]) : 1.f;
        dt8[i] = dt;
        du8[i] = dt * uv[i];
        do8[i] = ok ? gv[i] * gate : 0.f;
      }
      float4* pd = reinterpret_cast<float4*>(&s_dt[c][tt]);
      float4* pu = reinterpret_cast<float4*>(&s_du[c][tt]);
      float4* po = reinterpret_cast<float4*>(&s_do[c][tt]);
      pd[0] = make_float4(dt8[0], dt8[1], dt8[2], dt8[3]);
      pd[1] = make_float4(dt8[4], dt8[5], dt8[6], dt8[7]);
      pu[0] = make_float4(du8[0], du8[1], du8[2], du8[3]);
      pu[1] = make_float4(du8[4], du8[5], du8[6], du8[7]);
      po[0] = make_float4(do8[0], do8[1], do8[2], do8[3]);
      po[1] = make_float4(do8[4], do8[5], do8[6], do8[7]);
    }
    for (int g = tid; g < 2 * kN * (CH / 8); g += NT) {
      const int which = g / (kN * (CH / 8));
      const int r = g % (kN * (CH / 8));
      const int n = r / (CH / 8), tg = r % (CH / 8);
      float v[8];
      load8_row<T, VEC>((which ? Cb : Bb) + (size_t)n * L, t0 + 8 * tg, L, v);
      float(*dst)[kN] = which ? s_C : s_B;
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[8 * tg + i][n] = v[i];
    }
    __syncthreads();

    // ---- state entering the chunk, and entering sub-chunks 1..3
    float h0[SPL];
    if (kc > 0 && dvalid) {
      const float4 v = *reinterpret_cast<const float4*>(
          p.ckpt + (((size_t)b * p.dim + d) * p.nchunk + (kc - 1)) * kN + SPL * j);
      h0[0] = v.x; h0[1] = v.y; h0[2] = v.z; h0[3] = v.w;
    } else {
#pragma unroll
      for (int k = 0; k < SPL; ++k) h0[k] = 0.f;
    }
    float hb[3][SPL];
    {
      float h[SPL];
#pragma unroll
      for (int k = 0; k < SPL; ++k) h[k] = h0[k];
#pragma unroll
      for (int sb = 0; sb < 3; ++sb) {
#pragma unroll 4
        for (int i = 0; i < SUB; ++i) {
          const int tt = sb * SUB + i;
          const float dt = s_dt[c][tt], du = s_du[c][tt];
          const float4 b4 = *reinterpret_cast<const float4*>(&s_B[tt][SPL * j]);
          const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int k = 0; k < SPL; ++k) h[k] = fmaf(ex2(dt * A2[k]), h[k], du * bv[k]);
        }
#pragma unroll
        for (int k = 0; k < SPL; ++k) hb[sb][k] = h[k];
      }
    }

    for (int sb = 3; sb >= 0; --sb) {
      float hs[SPL];
#pragma unroll
      for (int k = 0; k < SPL; ++k)
        hs[k] = sb == 0 ? h0[k] : (sb == 1 ? hb[0][k] : (sb == 2 ? hb[1][k] : hb[2][k]));
      float Hh[SUB][SPL], Ha[SUB][SPL];
      // recompute the sub-chunk's states and decays
      float hcur[SPL];
#pragma unroll
      for (int k = 0; k < SPL; ++k) hcur[k] = hs[k];
#pragma unroll
      for (int i = 0; i < SUB; i += 4) {
        float ys[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int tt = sb * SUB + i + q;
          const float dt = s_dt[c][tt], du = s_du[c][tt];
          const float4 b4 = *reinterpret_cast<const float4*>(&s_B[tt][SPL * j]);
          const float4 c4 = *reinterpret_cast<const float4*>(&s_C[tt][SPL * j]);
          const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
          const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
          float acc = 0.f;
#pragma unroll
          for (int k = 0; k < SPL; ++k) {
            const float a = ex2(dt * A2[k]);
            hcur[k] = fmaf(a, hcur[k], du * bv[k]);
            Ha[i + q][k] = a;
            Hh[i + q][k] = hcur[k];
            acc = fmaf(cv[k], hcur[k], acc);
          }
          ys[q] = acc;
        }
        *reinterpret_cast<float4*>(&s_p[2][c][j][i]) = make_float4(ys[0], ys[1], ys[2], ys[3]);
      }
      // walk the sub-chunk backwards
#pragma unroll
      for (int i = SUB - 4; i >= 0; i -= 4) {
        float s1v[4], s2v[4];
#pragma unroll
        for (int q = 3; q >= 0; --q) {
          const int ii = i + q;
          const int tt = sb * SUB + ii;
          const float dt = s_dt[c][tt], du = s_du[c][tt], dout = s_do[c][tt];
          const float4 b4 = *reinterpret_cast<const float4*>(&s_B[tt][SPL * j]);
          const float4 c4 = *reinterpret_cast<const float4*>(&s_C[tt][SPL * j]);
          const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
          const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
          float s1 = 0.f, s2 = 0.f, dBv[4], dCv[4];
#pragma unroll
          for (int k = 0; k < SPL; ++k) {
            const float hprev = ii > 0 ? Hh[ii > 0 ? ii - 1 : 0][k] : hs[k];
            const float g = fmaf(dout, cv[k], carry[k]);
            dCv[k] = dout * Hh[ii][k];
            dBv[k] = g * du;
            s1 = fmaf(g, bv[k], s1);
            const float qv = g * Ha[ii][k] * hprev;
            dA[k] = fmaf(dt, qv, dA[k]);
            s2 = fmaf(Aq[k], qv, s2);
            carry[k] = Ha[ii][k] * g;
          }
          s1v[q] = s1;
          s2v[q] = s2;
          *reinterpret_cast<float4*>(&s_red[(ii * 2 + 0) * RED_SLAB + c * kN + SPL * j]) =
              make_float4(dBv[0], dBv[1], dBv[2], dBv[3]);
          *reinterpret_cast<float4*>(&s_red[(ii * 2 + 1) * RED_SLAB + c * kN + SPL * j]) =
              make_float4(dCv[0], dCv[1], dCv[2], dCv[3]);
        }
        *reinterpret_cast<float4*>(&s_p[0][c][j][i]) = make_float4(s1v[0], s1v[1], s1v[2], s1v[3]);
        *reinterpret_cast<float4*>(&s_p[1][c][j][i]) = make_float4(s2v[0], s2v[1], s2v[2], s2v[3]);
      }
      __syncthreads();

      // ---- epilogue for the sub-chunk: thread (c, j) owns steps 4j..4j+3
      {
        const int i0 = 4 * j;
        const int t = t0 + sb * SUB + i0;
        float S[3][4];
#pragma unroll
        for (int q = 0; q < 3; ++q) {
          float4 s = *reinterpret_cast<const float4*>(&s_p[q][c][0][i0]);
#pragma unroll
          for (int l = 1; l < KL; ++l) {
            const float4 v = *reinterpret_cast<const float4*>(&s_p[q][c][l][i0]);
            s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
          }
          S[q][0] = s.x; S[q][1] = s.y; S[q][2] = s.z; S[q][3] = s.w;
        }
        float uv[4], xv[4], zv[4], gv[4];
        load4_row<T>(u_row, t, L, VEC, uv);
        load4_row<T>(x_row, t, L, VEC, xv);
        load4_row<T>(g_row, t, L, VEC, gv);
        if (z_row) load4_row<T>(z_row, t, L, VEC, zv);
        float duo[4], ddo[4], dzo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int tt = sb * SUB + i0 + q;
          const bool ok = dvalid && (t + q < L);
          const float dt = s_dt[c][tt], dout = s_do[c][tt];
          duo[q] = fmaf(dout, Dd, dt * S[0][q]);
          const float dDelta = fmaf(uv[q], S[0][q], S[1][q]);
          const float x = xv[q] + bias;
          const float ddx = p.softplus ? dDelta * sigmoid_f(x) : dDelta;
          ddo[q] = ddx;
          if (z_row) {
            const float out = fmaf(Dd, uv[q], S[2][q]);
            const float sz = sigmoid_f(zv[q]);
            dzo[q] = gv[q] * out * sz * fmaf(zv[q], 1.f - sz, 1.f);
          }
          if (ok) {
            dD_acc = fmaf(dout, uv[q], dD_acc);
            dbias_acc += ddx;
          }
        }
        if (dvalid) {
          store4_row<T>(static_cast<T*>(p.du) + row, t, L, VEC, duo);
          store4_row<T>(static_cast<T*>(p.ddelta) + row, t, L, VEC, ddo);
          if (z_row) store4_row<T>(static_cast<T*>(p.dz) + row, t, L, VEC, dzo);
        }
      }
      // ---- channel sums of dB, dC for the sub-chunk, in a fixed order
      {
        const int warp = tid / 32, lane = tid % 32;
        const int n = lane % kN, q = lane / kN;
        float* part = q ? p.part_dC : p.part_dB;
        for (int ig = warp; ig < SUB / 4; ig += NW) {
          float acc[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float* src = &s_red[((4 * ig + r) * 2 + q) * RED_SLAB + n];
            float sacc = 0.f;
#pragma unroll
            for (int cc = 0; cc < CB; ++cc) sacc += src[cc * kN];
            acc[r] = sacc;
          }
          const int t = t0 + sb * SUB + 4 * ig;
          if (t < Lp) {
            float* dst = part + (((size_t)b * p.nblk + blk) * kN + n) * Lp + t;
            *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
          }
        }
      }
      __syncthreads();
    }
  }

  if (dvalid) {
    float* pa = p.part_dA + ((size_t)b * p.dim + d) * kN + SPL * j;
    *reinterpret_cast<float4*>(pa) = make_float4(dA[0], dA[1], dA[2], dA[3]);
  }
  // the 4 lanes of a channel hold disjoint time ranges: combine in a fixed order
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 1);
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 2);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 1);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 2);
  if (dvalid && j == 0) {
    p.part_dD[(size_t)b * p.dim + d] = dD_acc;
    p.part_dbias[(size_t)b * p.dim + d] = dbias_acc;
  }
}

// Second pass: dB[b,n,t] = sum over blocks, dC likewise; dA[d,n], dD[d],
// dbias[d] = sum over batch rows.  Fixed summation order everywhere.
__global__ void bwd_reduce_kernel(const BwdParams p) {
  const int L = p.seqlen, Lp = (L + 15) & ~15;
  const long long nBC = (long long)p.batch * kN * L;
  const long long nA = (long long)p.dim * kN;
  const long long nD = p.dim;
  const long long total = 2 * nBC + nA + 2 * nD;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    if (i < 2 * nBC) {
      const int q = i >= nBC;
      const long long r = q ? i - nBC : i;
      const int t = (int)(r % L);
      const long long bn = r / L;  // b * 16 + n
      const int n = (int)(bn % kN);
      const int b = (int)(bn / kN);
      const float* src = (q ? p.part_dC : p.part_dB) + ((size_t)b * p.nblk * kN + n) * Lp + t;
      float s = 0.f;
      for (int k = 0; k < p.nblk; ++k) s += src[(size_t)k * kN * Lp];
      (q ? p.dC : p.dB)[r] = s;
    } else if (i < 2 * nBC + nA) {
      const long long r = i - 2 * nBC;
      float s = 0.f;
      for (int b = 0; b < p.batch; ++b) s += p.part_dA[(size_t)b * nA + r];
      p.dA[r] = s;
    } else {
      const long long r = i - 2 * nBC - nA;
      const int q = r >= nD;
      const long long dd = q ? r - nD : r;
      float* out = q ? p.dbias : p.dD;
      if (!out) continue;
      const float* src = q ? p.part_dbias : p.part_dD;
      float s = 0.f;
      for (int b = 0; b < p.batch; ++b) s += src[(size_t)b * nD + dd];
      out[dd] = s;
    }
  }
}

template <int CB>
constexpr size_t bwd_smem_bytes() {
  return sizeof(float) * (3 * CB * CHP + 2 * CH * kN + 3 * CB * KL * SUBP +
                          SUB * 2 * (CB * kN + 16));
}

template <typename T, bool VEC>
cudaError_t launch_bwd_t(const BwdParams& p, cudaStream_t s) {
  constexpr int CB = kBwdChannelsPerBlock;
  constexpr size_t smem = bwd_smem_bytes<CB>();
  // opt in to more than 48 KB of dynamic shared memory, once per device
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !((configured >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(bwd_kernel<T, CB, VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    configured |= 1ull << dev;
  }
  const dim3 g((p.dim + CB - 1) / CB, p.batch);
  bwd_kernel<T, CB, VEC><<<g, CB * KL, smem, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long total = 2LL * p.batch * kN * p.seqlen + (long long)p.dim * kN + 2LL * p.dim;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  bwd_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

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
