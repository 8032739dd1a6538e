// ss_conv.cu -- causal depthwise conv1d + SiLU for sm_100a.
//
// "Mamba" (stanleyjacob.dev), Part IV Stage 2: before the scan, each of the
// d_inner channels runs its own width-d_conv (4) causal filter, position t
// seeing t-3 .. t, followed by a SiLU.  Part II and Part IV Stage 7: decoding
// keeps the small convolution window and advances it one token at a time.
//
//   pre_t = bias_d + sum_k w[d,k] xin(t - (W-1) + k),   u_t = SiLU(pre_t)
//
// xin(s) is x for s >= 0 and the incoming window (state_in) for s < 0.
//
// The convolution is HBM-bound: 2 + 2 bytes per element in bf16 against 4
// FMAs and 2 SFU operations.  Each thread owns a 32-step piece of one row:
// one 16-byte vector load per 8 steps, the W-1 inputs before the piece as
// scalar loads (they sit in the previous thread's piece and hit L1).
//
// Backward: one block per (batch, channel) row, threads over its 32-step
// pieces.  A thread recomputes pre for its piece plus the W-1 steps after it
// (dx at s needs dpre at s .. s+W-1), forms dx directly, and accumulates dw,
// dbias for its own steps.  The block sums those in a fixed order into a
// per-row partial; a second kernel sums the rows of each channel over the
// batch in order.  No atomics: results are bitwise reproducible.
#include "ss_device.cuh"
#include "ss_internal.h"

namespace ss {
namespace {

constexpr int kPiece = 32;  // steps per thread (forward)
#ifndef SS_CONV_BWD_PIECE
#define SS_CONV_BWD_PIECE 32
#endif
#ifndef SS_CONV_BWD_MINB
#define SS_CONV_BWD_MINB 3
#endif
// steps per thread in the backward: longer pieces recompute a smaller share
// of halo steps; with packed documents the piece and its W-1 halo steps must
// fit the 32-bit document-start mask
template <bool SEQ>
constexpr int bwd_piece() { return SEQ ? 16 : SS_CONV_BWD_PIECE; }

template <typename T>
__device__ __forceinline__ float ldx(const T* p) { return Elt<T>::to_f(*p); }

// window value xin(s) of a row: x for s >= 0, the incoming window for s < 0
template <typename T, int W>
__device__ __forceinline__ float xin(const T* xr, const float* st_row, int s) {
  if (s >= 0) return ldx(xr + s);
  return st_row ? st_row[W - 1 + s] : 0.f;
}

__device__ __forceinline__ float silu_f(float x) { return x * sigmoid_f(x); }

// The W-1 inputs before step t0, oldest first.  A document starting at a step
// r in (t0-(W-1), t0) hides the entries before r (the start at t0 itself is
// applied by the caller's per-step mask).
template <typename T, int W>
__device__ __forceinline__ void init_window(float (&win)[W > 1 ? W - 1 : 1], const T* xr,
                                            const float* st_row, const int* seq_row, int t0) {
#pragma unroll
  for (int j = 0; j < W - 1; ++j) win[j] = xin<T, W>(xr, st_row, t0 - (W - 1) + j);
  if (seq_row) {
#pragma unroll
    for (int j = 1; j < W - 1; ++j) {
      const int r = t0 - (W - 1) + j;
      if (r > 0 && seq_row[r] != seq_row[r - 1]) {
#pragma unroll
        for (int k = 0; k < j; ++k) win[k] = 0.f;
      }
    }
  }
}

// Bit i set when step t0 + i (0 < t0 + i < L, i < 32) starts a new packed
// document (seq_idx changes from the step before): the window restarts
// from zero there, so no input crosses a document boundary.
__device__ __forceinline__ unsigned doc_starts_row(const int* seq_row, int t0, int L) {
  unsigned m = 0;
  if (!seq_row) return 0;
  int prev = t0 > 0 ? seq_row[t0 - 1] : 0;
#pragma unroll 4
  for (int i = 0; i < 32; ++i) {
    const int t = t0 + i;
    if (t >= L) break;
    const int cur = seq_row[t];
    if (t > 0 && cur != prev) m |= 1u << i;
    prev = cur;
  }
  return m;
}

// SEQ: packed documents (seq_idx given); SILU: the SiLU after the conv.  Both
// are compile-time so that plain rows pay for neither.
template <typename T, bool VEC, int W, bool SEQ, bool SILU>
__global__ void __launch_bounds__(256) conv_fwd_kernel(const ConvParams p) {
  const int L = p.seqlen;
  const int npc = (L + kPiece - 1) / kPiece;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long rows = (long long)p.batch * p.dim;
  if (gid >= rows * npc) return;
  const long long row = gid / npc;
  const int pc = (int)(gid - row * npc);
  const int d = (int)(row % p.dim);
  const int t0 = pc * kPiece;
  const T* __restrict__ xr = static_cast<const T*>(p.x) + row * L;
  T* __restrict__ ur = static_cast<T*>(p.u) + row * L;
  const float* st_row = p.state_in ? p.state_in + row * (W - 1) : nullptr;
  const int* seq_row = SEQ ? p.seq_idx + (row / p.dim) * L : nullptr;
  const unsigned rst = SEQ ? doc_starts_row(seq_row, t0, L) : 0u;

  float wk[W];
#pragma unroll
  for (int k = 0; k < W; ++k) wk[k] = p.w[(size_t)d * W + k];
  const float bd = p.bias ? p.bias[d] : 0.f;
  float win[W > 1 ? W - 1 : 1];
  init_window<T, W>(win, xr, st_row, seq_row, t0);

  const int t_end = min(L, t0 + kPiece);
#pragma unroll
  for (int v = 0; v < kPiece / 8; ++v) {
    const int t = t0 + 8 * v;
    if (t >= t_end) break;
    RawVec<T, 8> rx;
    rx.template load<VEC>(xr, t, L);
    float xv[8], uv[8];
    rx.unpack(xv);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (rst & (1u << (8 * v + i))) {
#pragma unroll
        for (int k = 0; k < W - 1; ++k) win[k] = 0.f;
      }
      float pre = fmaf(wk[W - 1], xv[i], bd);
#pragma unroll
      for (int k = 0; k < W - 1; ++k) pre = fmaf(wk[k], win[k], pre);
      uv[i] = SILU ? silu_f(pre) : pre;
      if (t + i < t_end) {  // the window only advances over real steps
#pragma unroll
        for (int k = 0; k + 1 < W - 1; ++k) win[k] = win[k + 1];
        if (W > 1) win[W > 1 ? W - 2 : 0] = xv[i];
      }
    }
    if (VEC && t + 8 <= L) {
      store8(ur + t, uv);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (t + i < L) ur[t + i] = Elt<T>::from_f(uv[i]);
    }
  }
  if (p.state_out && pc == npc - 1) {
#pragma unroll
    for (int j = 0; j < W - 1; ++j) p.state_out[row * (W - 1) + j] = win[j];
  }
}

template <typename T, bool VEC, int W, bool SEQ, bool SILU>
__global__ void __launch_bounds__(256, SS_CONV_BWD_MINB) conv_bwd_kernel(const ConvParams p) {
  constexpr int kBwdPiece = bwd_piece<SEQ>();
  constexpr int H = kBwdPiece + W - 1;  // steps whose dpre a piece needs
  static_assert(!SEQ || H <= 32, "the document-start mask covers 32 steps");
  static_assert(kBwdPiece % 8 == 0, "pieces are whole 8-step vectors");
  const int L = p.seqlen;
  const int npc = (L + kBwdPiece - 1) / kBwdPiece;
  const long long row = blockIdx.x;
  const int d = (int)(row % p.dim);
  const T* __restrict__ xr = static_cast<const T*>(p.x) + row * L;
  const T* __restrict__ gr = static_cast<const T*>(p.du) + row * L;
  T* __restrict__ dxr = static_cast<T*>(p.dx) + row * L;
  const float* st_row = p.state_in ? p.state_in + row * (W - 1) : nullptr;
  const float* dso_row = p.dstate_out ? p.dstate_out + row * (W - 1) : nullptr;

  float wk[W];
#pragma unroll
  for (int k = 0; k < W; ++k) wk[k] = p.w[(size_t)d * W + k];
  const float bd = p.bias ? p.bias[d] : 0.f;
  float dw_acc[W], db_acc = 0.f;
#pragma unroll
  for (int k = 0; k < W; ++k) dw_acc[k] = 0.f;

  const int* seq_row = SEQ ? p.seq_idx + (row / p.dim) * L : nullptr;
  for (int pc = threadIdx.x; pc < npc; pc += blockDim.x) {
    const int t0 = pc * kBwdPiece;
    const unsigned rst = SEQ ? doc_starts_row(seq_row, t0, L) : 0u;  // covers the H steps
    float win[W > 1 ? W - 1 : 1];
    init_window<T, W>(win, xr, st_row, seq_row, t0);
    float dp[H];
#pragma unroll
    for (int v = 0; v < (H + 7) / 8; ++v) {
      const int t = t0 + 8 * v;
      float xv[8], gv[8];
      {
        RawVec<T, 8> rx, rg;
        rx.template load<VEC>(xr, t, L);
        rg.template load<VEC>(gr, t, L);
        rx.unpack(xv);
        rg.unpack(gv);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int h = 8 * v + i;
        if (h >= H) break;
        if (rst & (1u << h)) {
#pragma unroll
          for (int k = 0; k < W - 1; ++k) win[k] = 0.f;
        }
        float pre = fmaf(wk[W - 1], xv[i], bd);
#pragma unroll
        for (int k = 0; k < W - 1; ++k) pre = fmaf(wk[k], win[k], pre);
        float g = t + i < L ? gv[i] : 0.f;
        if (SILU) {
          const float s = sigmoid_f(pre);
          g *= s * fmaf(pre, 1.f - s, 1.f);
        }
        dp[h] = g;
        if (h < kBwdPiece && t + i < L) {  // own steps: parameter gradients
          db_acc += g;
#pragma unroll
          for (int k = 0; k < W - 1; ++k) dw_acc[k] = fmaf(g, win[k], dw_acc[k]);
          dw_acc[W - 1] = fmaf(g, xv[i], dw_acc[W - 1]);
        }
#pragma unroll
        for (int k = 0; k + 1 < W - 1; ++k) win[k] = win[k + 1];
        if (W > 1) win[W > 1 ? W - 2 : 0] = xv[i];
      }
    }
    // dx(s) = sum_k w[k] dpre(s + W-1-k), plus the gradient reaching the
    // outgoing window; pc == 0 also forms the incoming window's gradient
#pragma unroll
    for (int v = 0; v < kBwdPiece / 8; ++v) {
      const int t = t0 + 8 * v;
      if (t >= L) break;
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // x(s) reaches u(s + m) for m < W while no document starts in (s, s + m]
        float g = 0.f;
        bool alive = true;
#pragma unroll
        for (int m = 0; m < W; ++m) {
          const int h = 8 * v + i + m;
          if (m > 0 && (rst & (1u << h))) alive = false;
          if (alive) g = fmaf(wk[W - 1 - m], dp[h], g);
        }
        const int jo = t + i - (L - (W - 1));
        if (dso_row && jo >= 0 && jo < W - 1) g += dso_row[jo];
        o[i] = g;
      }
      if (VEC && t + 8 <= L) {
        store8(dxr + t, o);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (t + i < L) dxr[t + i] = Elt<T>::from_f(o[i]);
      }
    }
    if (pc == 0 && p.dstate_in) {
#pragma unroll
      for (int j = 0; j < W - 1; ++j) {
        const int s = j - (W - 1);  // < 0
        float g = 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k) {
          const int h = s + (W - 1) - k;  // target step, relative to t0 = 0
          // the incoming window belongs to the document at step 0
          const bool alive = (rst & ((2u << (h > 0 ? h : 0)) - 2u)) == 0;
          if (h >= 0 && h < H && alive) g = fmaf(wk[k], dp[h], g);
        }
        const int jo = s - (L - (W - 1));
        if (dso_row && jo >= 0 && jo < W - 1) g += dso_row[jo];
        p.dstate_in[row * (W - 1) + j] = g;
      }
    }
  }

  // fixed-order block sum of (dw, dbias): butterfly within each warp, then
  // warps in order
  __shared__ float s_part[8][W + 1];
  float v[W + 1];
#pragma unroll
  for (int k = 0; k < W; ++k) v[k] = dw_acc[k];
  v[W] = db_acc;
#pragma unroll
  for (int k = 0; k <= W; ++k) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v[k] += __shfl_xor_sync(0xffffffffu, v[k], off);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k <= W; ++k) s_part[warp][k] = v[k];
  }
  __syncthreads();
  if (threadIdx.x <= W) {
    float a = 0.f;
    for (int w8 = 0; w8 < (int)(blockDim.x >> 5); ++w8) a += s_part[w8][threadIdx.x];
    p.part[row * (W + 1) + threadIdx.x] = a;
  }
}

// dw[d,k], dbias[d] = sums over the batch rows of channel d, in batch order
__global__ void conv_reduce_kernel(const ConvParams p) {
  const int W1 = p.width + 1;
  const long long n = (long long)p.dim * W1;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int d = (int)(i / W1), k = (int)(i % W1);
    float a = 0.f;
    for (int b = 0; b < p.batch; ++b) a += p.part[((size_t)b * p.dim + d) * W1 + k];
    if (k < p.width) p.dw[(size_t)d * p.width + k] = a;
    else if (p.dbias) p.dbias[d] = a;
  }
}

template <typename T, int W>
__global__ void __launch_bounds__(256) conv_step_kernel(const ConvParams p) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)p.batch * p.dim) return;
  const int d = (int)(i % p.dim);
  float* st = p.state_out + i * (W - 1);  // in/out
  const float xt = ldx(static_cast<const T*>(p.x) + i);
  float pre = fmaf(p.w[(size_t)d * W + W - 1], xt, p.bias ? p.bias[d] : 0.f);
  float win[W > 1 ? W - 1 : 1];
#pragma unroll
  for (int k = 0; k < W - 1; ++k) {
    win[k] = st[k];
    pre = fmaf(p.w[(size_t)d * W + k], win[k], pre);
  }
  static_cast<T*>(p.u)[i] = Elt<T>::from_f(p.silu ? silu_f(pre) : pre);
#pragma unroll
  for (int k = 0; k + 1 < W - 1; ++k) st[k] = win[k + 1];
  if (W > 1) st[W > 1 ? W - 2 : 0] = xt;
}

template <typename T, bool VEC, int W, bool SEQ, bool SILU>
void launch_conv_fb(const ConvParams& p, int op, cudaStream_t s) {
  const long long rows = (long long)p.batch * p.dim;
  if (op == 0) {
    const long long npc = (p.seqlen + kPiece - 1) / kPiece;
    const long long n = rows * npc;
    conv_fwd_kernel<T, VEC, W, SEQ, SILU><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
  } else {
    constexpr int kBwdPiece = bwd_piece<SEQ>();
    const int npc = (p.seqlen + kBwdPiece - 1) / kBwdPiece;
    int threads = ((npc + 31) / 32) * 32;
    threads = threads < 32 ? 32 : threads > 256 ? 256 : threads;
    conv_bwd_kernel<T, VEC, W, SEQ, SILU><<<(unsigned)rows, threads, 0, s>>>(p);
  }
}

template <typename T, bool VEC, int W>
cudaError_t launch_conv_w(const ConvParams& p, int op, cudaStream_t s) {
  const long long rows = (long long)p.batch * p.dim;
  if (op == 0 || op == 1) {
    if (p.seq_idx) {
      if (p.silu) launch_conv_fb<T, VEC, W, true, true>(p, op, s);
      else launch_conv_fb<T, VEC, W, true, false>(p, op, s);
    } else {
      if (p.silu) launch_conv_fb<T, VEC, W, false, true>(p, op, s);
      else launch_conv_fb<T, VEC, W, false, false>(p, op, s);
    }
  }
  if (op == 1) {
    const long long n = (long long)p.dim * (W + 1);
    long long blocks = (n + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    conv_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(p);
  } else if (op == 2) {
    conv_step_kernel<T, W><<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(p);
  }
  return cudaGetLastError();
}

template <typename T, bool VEC>
cudaError_t launch_conv_v(const ConvParams& p, int op, cudaStream_t s) {
  switch (p.width) {
    case 1: return launch_conv_w<T, VEC, 1>(p, op, s);
    case 2: return launch_conv_w<T, VEC, 2>(p, op, s);
    case 3: return launch_conv_w<T, VEC, 3>(p, op, s);
    case 4: return launch_conv_w<T, VEC, 4>(p, op, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_conv_t(const ConvParams& p, int op, bool vec, cudaStream_t s) {
  return vec ? launch_conv_v<T, true>(p, op, s) : launch_conv_v<T, false>(p, op, s);
}

}  // namespace

cudaError_t launch_conv(const ConvParams& p, int op, DType dt, bool vec, cudaStream_t s) {
  switch (dt) {
    case DType::F32: return launch_conv_t<float>(p, op, vec, s);
    case DType::BF16: return launch_conv_t<__nv_bfloat16>(p, op, vec, s);
    case DType::F16: return launch_conv_t<__half>(p, op, vec, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ss
