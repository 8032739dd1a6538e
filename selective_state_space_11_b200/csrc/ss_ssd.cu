// ss_ssd.cu -- Mamba-2 SSD forward (state-space duality, chunked) for sm_100a.
//
// "Mamba" (stanleyjacob.dev), Part V, "Deep dive: Mamba-2 and state-space
// duality": with A a scalar per head the selective SSM is a masked quadratic
// form inside a chunk of the sequence and a recurrence between chunks, so most
// of the work becomes dense matmuls on the tensor cores.  Per (batch b, head
// h), with the B, C of the head's group and a chunk of Q = 64 steps:
//
//   cs_i = sum_{k<=i} Delta_k A_h                 (within the chunk)
//   Y    = (C B^T o Lmask o Delta_j) X            Lmask[i,j] = exp(cs_i - cs_j), j <= i
//        + diag(exp(cs_i)) C H^T                  H: the P x N state entering the chunk
//   H   <- exp(cs_last) H + X^T diag(exp(cs_last - cs_j) Delta_j) B
//   y    = (Y + D x) SiLU(z)
//
// One block of 4 warps per (b, h) walks the chunks in order.  Warp w owns rows
// 16w .. 16w+15: time steps for C B^T and Y, state rows p for H.  The four
// products are warp-level bf16 (or fp16) tensor-core MMAs (m16n8k16, fp32
// accumulation); the masked C B^T tile goes from accumulator registers
// straight into the A operand of the next product.  The state H stays in fp32
// accumulator registers for the whole sequence; a bf16 copy in shared memory
// is the operand of the C H^T product.  headdim P = 64, d_state N = 64 or 128.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ss_device.cuh"
#include "ss_internal.h"

namespace ss {
namespace {

constexpr int kQ = 64;  // chunk length
constexpr int kP = 64;  // head dimension
constexpr int kThreads = 128;

template <typename T> struct Mma;
template <> struct Mma<__nv_bfloat16> {
  __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};
template <> struct Mma<__half> {
  __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], unsigned addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], unsigned addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ unsigned sm_addr(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

// Shared-memory tiles of one chunk, unpadded.  The 16-byte pieces of each
// row are stored XOR-swizzled by the row index (piece c of row r at c ^ (r & 7)),
// so that the 8 rows an ldmatrix phase reads, and the pieces a staging copy
// writes, fall in distinct bank groups.
template <typename T, int N>
struct SsdSmem {
  T x[kQ][kP];        // x of the chunk           [t][p]
  T xw[kQ][kP];       // x scaled by the state-update weight w_t
  T z[kQ][kP];        // z of the chunk (gate)
  T b[kQ][N];         // B of the chunk           [t][n]
  T c[kQ][N];         // C of the chunk           [t][n]
  T h[kP][N];         // state entering the chunk [p][n] (operand copy)
  float dlt[kQ];      // Delta_t
  float cs[kQ];       // cumulative Delta A within the chunk
};

// Element offset of (row r, column k) in a swizzled tile with W elements per row.
template <int W>
__device__ __forceinline__ int swz(int r, int k) {
  return r * W + ((((k >> 3) ^ r) & 7) | ((k >> 3) & ~7)) * 8 + (k & 7);
}

template <typename T, int N>
__global__ void __launch_bounds__(kThreads, 3) ssd_fwd_kernel(const SsdParams p) {
  using S = SsdSmem<T, N>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  S& sm = *reinterpret_cast<S*>(smem_raw);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y, h = blockIdx.x;
  const int L = p.seqlen, nh = p.nheads, ng = p.ngroups;
  const int g = h / (nh / ng);
  const float Ah = p.A[h];
  const float Dh = p.D ? p.D[h] : 0.f;
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
  const size_t xrow = (size_t)nh * kP;  // elements between time steps of x, z, y
  const size_t brow = (size_t)ng * N;   // elements between time steps of B, C
  const T* __restrict__ xg = static_cast<const T*>(p.x) + (size_t)b * L * xrow + (size_t)h * kP;
  const T* __restrict__ zg = p.z ? static_cast<const T*>(p.z) + (size_t)b * L * xrow + (size_t)h * kP : nullptr;
  T* __restrict__ yg = static_cast<T*>(p.y) + (size_t)b * L * xrow + (size_t)h * kP;
  const T* __restrict__ bg = static_cast<const T*>(p.B) + (size_t)b * L * brow + (size_t)g * N;
  const T* __restrict__ cg = static_cast<const T*>(p.C) + (size_t)b * L * brow + (size_t)g * N;
  const T* __restrict__ dtg = static_cast<const T*>(p.dt) + (size_t)b * L * nh + h;

  // the state: rows p = 16 warp + {lane/4, lane/4 + 8}, columns n = 8 j + 2 (lane%4) + {0,1}
  constexpr int NT = N / 8;  // n8 tiles across the state
  float hacc[NT][4];
  const int r0 = lane >> 2, c0 = 2 * (lane & 3);
  {
    const float* h0 = p.h0 ? p.h0 + ((size_t)b * nh + h) * kP * N : nullptr;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int pr = 16 * warp + r0 + (e >> 1) * 8, nc = 8 * j + c0 + (e & 1);
        hacc[j][e] = h0 ? h0[(size_t)pr * N + nc] : 0.f;
      }
    }
  }

  T* const sx = &sm.x[0][0];
  T* const sxw = &sm.xw[0][0];
  T* const sz = &sm.z[0][0];
  T* const sb = &sm.b[0][0];
  T* const sc = &sm.c[0][0];
  T* const sh = &sm.h[0][0];
  const int nchunks = (L + kQ - 1) / kQ;
  for (int ck = 0; ck < nchunks; ++ck) {
    const int t0 = ck * kQ;
    const int nval = min(kQ, L - t0);
    // ---- stage the chunk: x, z, B, C rows (16-byte async copies, zero past L)
    for (int r = tid; r < kQ * (kP * 2 / 16); r += kThreads) {
      const int t = r / (kP * 2 / 16), q = r % (kP * 2 / 16);
      const bool ok = t < nval;
      const size_t off = (size_t)(t0 + t) * xrow + q * 8;
      cp_async16(sx + swz<kP>(t, q * 8), ok ? (const void*)(xg + off) : (const void*)xg, ok ? 16 : 0);
      if (zg) cp_async16(sz + swz<kP>(t, q * 8), ok ? (const void*)(zg + off) : (const void*)zg, ok ? 16 : 0);
    }
    for (int r = tid; r < kQ * (N * 2 / 16); r += kThreads) {
      const int t = r / (N * 2 / 16), q = r % (N * 2 / 16);
      const bool ok = t < nval;
      const size_t off = (size_t)(t0 + t) * brow + q * 8;
      cp_async16(sb + swz<N>(t, q * 8), ok ? (const void*)(bg + off) : (const void*)bg, ok ? 16 : 0);
      cp_async16(sc + swz<N>(t, q * 8), ok ? (const void*)(cg + off) : (const void*)cg, ok ? 16 : 0);
    }
    cp_async_commit();
    // the operand copy of the state entering this chunk
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int pr = 16 * warp + r0, nc = 8 * j + c0;
      *reinterpret_cast<uint32_t*>(sh + swz<N>(pr, nc)) = Mma<T>::pack(hacc[j][0], hacc[j][1]);
      *reinterpret_cast<uint32_t*>(sh + swz<N>(pr + 8, nc)) = Mma<T>::pack(hacc[j][2], hacc[j][3]);
    }
    // ---- Delta and its cumulative sum within the chunk (warp 0: 2 steps per lane)
    if (warp == 0) {
      float d2[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int t = 2 * lane + k;
        float v = 0.f;
        if (t < nval) {
          const float x = Elt<T>::to_f(dtg[(size_t)(t0 + t) * nh]) + bias;
          v = p.softplus ? softplus_f(x) : x;
        }
        d2[k] = v;
        sm.dlt[t] = v;
      }
      float run = (d2[0] + d2[1]) * Ah;  // inclusive scan of the lane sums
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, run, off);
        if (lane >= off) run += o;
      }
      const float before = run - (d2[0] + d2[1]) * Ah;
      sm.cs[2 * lane] = before + d2[0] * Ah;
      sm.cs[2 * lane + 1] = run;
    }
    cp_async_wait_all();
    __syncthreads();

    const float cs_last = sm.cs[kQ - 1];
    // ---- x scaled by the state-update weight w_t = exp(cs_last - cs_t) Delta_t
    for (int e = tid; e < kQ * kP / 2; e += kThreads) {
      const int t = e / (kP / 2), q = 2 * (e % (kP / 2));
      const float w = __expf(cs_last - sm.cs[t]) * sm.dlt[t];
      const int o = swz<kP>(t, q);
      const float x0 = Elt<T>::to_f(sx[o]), x1 = Elt<T>::to_f(sx[o + 1]);
      *reinterpret_cast<uint32_t*>(sxw + o) = Mma<T>::pack(x0 * w, x1 * w);
    }
    __syncthreads();

    // ---- G = C B^T for rows 16 warp .. +15 (K = N), masked: M[i,j] =
    // G[i,j] exp(cs_i - cs_j) Delta_j for j <= i, else 0
    uint32_t mfrag[kQ / 16][4];  // M as the A operand of M X (k16 chunks of j)
    {
      float gacc[kQ / 8][4];
#pragma unroll
      for (int j = 0; j < kQ / 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) gacc[j][e] = 0.f;
#pragma unroll
      for (int k0 = 0; k0 < N; k0 += 16) {
        uint32_t a[4];
        ldsm_x4(a, sm_addr(sc + swz<N>(16 * warp + (lane & 15), k0 + (lane >> 4) * 8)));
#pragma unroll
        for (int j = 0; j < kQ / 8; j += 2) {  // two n8 tiles (16 steps j) per ldmatrix
          uint32_t bb[4];
          ldsm_x4(bb, sm_addr(sb + swz<N>(8 * j + (lane & 7) + ((lane >> 4) << 3), k0 + ((lane >> 3) & 1) * 8)));
          Mma<T>::run(gacc[j], a, bb[0], bb[1]);
          Mma<T>::run(gacc[j + 1], a, bb[2], bb[3]);
        }
      }
      const int ia = 16 * warp + r0, ib = ia + 8;
      const float csa = sm.cs[ia], csb = sm.cs[ib];
#pragma unroll
      for (int j = 0; j < kQ / 8; ++j) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = (e >> 1) ? ib : ia;
          const int jj = 8 * j + c0 + (e & 1);
          const float csi = (e >> 1) ? csb : csa;
          v[e] = jj <= i ? gacc[j][e] * __expf(csi - sm.cs[jj]) * sm.dlt[jj] : 0.f;
        }
        // accumulator tile pairs (j even, odd) form one k16 A fragment
        const int kk = j >> 1;
        if ((j & 1) == 0) {
          mfrag[kk][0] = Mma<T>::pack(v[0], v[1]);
          mfrag[kk][1] = Mma<T>::pack(v[2], v[3]);
        } else {
          mfrag[kk][2] = Mma<T>::pack(v[0], v[1]);
          mfrag[kk][3] = Mma<T>::pack(v[2], v[3]);
        }
      }
    }

    // ---- Y = diag(exp(cs_i)) C H^T + M X for rows 16 warp .. +15 (columns p)
    float yacc[kP / 8][4];
#pragma unroll
    for (int j = 0; j < kP / 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) yacc[j][e] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < N; k0 += 16) {
      uint32_t a[4];
      ldsm_x4(a, sm_addr(sc + swz<N>(16 * warp + (lane & 15), k0 + (lane >> 4) * 8)));
#pragma unroll
      for (int j = 0; j < kP / 8; j += 2) {  // B operand H^T: stored [p][n] = [N'][K]
        uint32_t bb[4];
        ldsm_x4(bb, sm_addr(sh + swz<N>(8 * j + (lane & 7) + ((lane >> 4) << 3), k0 + ((lane >> 3) & 1) * 8)));
        Mma<T>::run(yacc[j], a, bb[0], bb[1]);
        Mma<T>::run(yacc[j + 1], a, bb[2], bb[3]);
      }
    }
    {
      const float ea = __expf(sm.cs[16 * warp + r0]), eb = __expf(sm.cs[16 * warp + r0 + 8]);
#pragma unroll
      for (int j = 0; j < kP / 8; ++j) {
        yacc[j][0] *= ea; yacc[j][1] *= ea;
        yacc[j][2] *= eb; yacc[j][3] *= eb;
      }
    }
#pragma unroll
    for (int kk = 0; kk < kQ / 16; ++kk) {
#pragma unroll
      for (int j = 0; j < kP / 8; j += 2) {  // B operand X: stored [t][p] = [K][N'] -> .trans
        uint32_t bb[4];
        ldsm_x4_t(bb, sm_addr(sx + swz<kP>(16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3), 8 * j + (lane >> 4) * 8)));
        Mma<T>::run(yacc[j], mfrag[kk], bb[0], bb[1]);
        Mma<T>::run(yacc[j + 1], mfrag[kk], bb[2], bb[3]);
      }
    }
    // ---- y = (Y + D x) SiLU(z), rows t = 16 warp + {r0, r0 + 8}
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int t = 16 * warp + r0 + 8 * half;
      if (t < nval) {
        T* yr = yg + (size_t)(t0 + t) * xrow;
#pragma unroll
        for (int j = 0; j < kP / 8; ++j) {
          const int pc = 8 * j + c0;
          const int o = swz<kP>(t, pc);
          float o0 = yacc[j][2 * half] + Dh * Elt<T>::to_f(sx[o]);
          float o1 = yacc[j][2 * half + 1] + Dh * Elt<T>::to_f(sx[o + 1]);
          if (zg) {
            const float z0 = Elt<T>::to_f(sz[o]), z1 = Elt<T>::to_f(sz[o + 1]);
            o0 *= z0 * sigmoid_f(z0);
            o1 *= z1 * sigmoid_f(z1);
          }
          *reinterpret_cast<uint32_t*>(yr + pc) = Mma<T>::pack(o0, o1);
        }
      }
    }

    // ---- H <- exp(cs_last) H + Xw^T B for state rows p = 16 warp .. +15 (K = t)
    {
      const float el = __expf(cs_last);
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) hacc[j][e] *= el;
#pragma unroll
      for (int kk = 0; kk < kQ / 16; ++kk) {
        uint32_t a[4];  // A = Xw^T: stored [t][p] = [K][M] -> .trans
        ldsm_x4_t(a, sm_addr(sxw + swz<kP>(16 * kk + (lane & 7) + ((lane >> 4) << 3), 16 * warp + ((lane >> 3) & 1) * 8)));
#pragma unroll
        for (int j = 0; j < NT; j += 2) {  // B operand B: stored [t][n] = [K][N'] -> .trans
          uint32_t bb[4];
          ldsm_x4_t(bb, sm_addr(sb + swz<N>(16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3), 8 * j + (lane >> 4) * 8)));
          Mma<T>::run(hacc[j], a, bb[0], bb[1]);
          Mma<T>::run(hacc[j + 1], a, bb[2], bb[3]);
        }
      }
    }
    __syncthreads();  // the next chunk overwrites the tiles
  }

  if (p.final_state) {
    float* fs = p.final_state + ((size_t)b * nh + h) * kP * N;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int pr = 16 * warp + r0, nc = 8 * j + c0;
      *reinterpret_cast<float2*>(fs + (size_t)pr * N + nc) = make_float2(hacc[j][0], hacc[j][1]);
      *reinterpret_cast<float2*>(fs + (size_t)(pr + 8) * N + nc) = make_float2(hacc[j][2], hacc[j][3]);
    }
  }
}

template <typename T, int N>
cudaError_t launch_ssd_n(const SsdParams& p, cudaStream_t s) {
  const size_t smem = sizeof(SsdSmem<T, N>);
  cudaError_t e = cudaFuncSetAttribute(ssd_fwd_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 g(p.nheads, p.batch);
  ssd_fwd_kernel<T, N><<<g, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ssd_t(const SsdParams& p, cudaStream_t s) {
  if (p.dstate == 64) return launch_ssd_n<T, 64>(p, s);
  if (p.dstate == 128) return launch_ssd_n<T, 128>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_ssd_fwd_mma(const SsdParams& p, DType dt, cudaStream_t s) {
  switch (dt) {
    case DType::BF16: return launch_ssd_t<__nv_bfloat16>(p, s);
    case DType::F16: return launch_ssd_t<__half>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ss
