// ss_shard.cu -- the two small kernels that sequence sharding adds to the scan.
//
// Sequence sharding splits L into contiguous segments, one per rank.  With the
// state passing of "mamba-metal" README, "Long-context prompts (parallel
// prefill)" -- a segment run from an initial state h0 ends in
//   h_end = P o h0 + E,   P[n] = prod_t exp(Delta_t A_n) = exp(A_n sum_t Delta_t)
// (E: its end state from zero; the map is diagonal in the state because every
// state evolves on its own) -- each rank runs its segment once, the ranks
// exchange (P, E), and each rebuilds the state entering its segment by the
// chain below; the backward chains the adjoints the same way in reverse.
//   segment_decay: P[b][d][n] = 2^(A_n log2(e) sum_t Delta_t) over the segment
//   state_chain:   out[0] = init, out[s+1] = P[s] o out[s] + E[s]        (forward)
//                  out[S-1] = init, out[s-1] = P[s] o out[s] + E[s]      (reverse)
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ss_device.cuh"
#include "ss_internal.h"

namespace ss {
namespace {

constexpr int kDecayThreads = 256;

// One block per (b, d) row: the sum of Delta over the row (strided, then a
// block reduction in fixed order), then P for each state n.
template <typename T>
__global__ void __launch_bounds__(kDecayThreads) segment_decay_kernel(const SegmentDecayParams p) {
  __shared__ float part[kDecayThreads / 32];
  const int row = blockIdx.x;  // b * dim + d
  const int d = row % p.dim;
  const T* dl = static_cast<const T*>(p.delta) + static_cast<size_t>(row) * p.seqlen;
  const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;
  float s = 0.f;
  for (int t = threadIdx.x; t < p.seqlen; t += kDecayThreads) {
    const float v = Elt<T>::to_f(dl[t]) + bias;
    s += p.softplus ? softplus_f(v) : v;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < p.dstate) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kDecayThreads / 32; ++w) tot += part[w];
    const float a = p.A[static_cast<size_t>(d) * p.dstate + threadIdx.x];
    p.P[static_cast<size_t>(row) * p.dstate + threadIdx.x] = ex2(a * kLog2e * tot);
  }
}

__global__ void state_chain_kernel(const StateChainParams p) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<size_t>(p.count)) return;
  const size_t n = static_cast<size_t>(p.count);
  float h = p.init ? p.init[i] : 0.f;
  if (!p.reverse) {
    p.out[i] = h;
    for (int s = 0; s + 1 < p.nseg; ++s) {
      h = fmaf(p.P[s * n + i], h, p.E[s * n + i]);
      p.out[(s + 1) * n + i] = h;
    }
  } else {
    p.out[(p.nseg - 1) * n + i] = h;
    for (int s = p.nseg - 1; s >= 1; --s) {
      h = fmaf(p.P[s * n + i], h, p.E[s * n + i]);
      p.out[(s - 1) * n + i] = h;
    }
  }
}

}  // namespace

cudaError_t launch_segment_decay(const SegmentDecayParams& p, DType dt, cudaStream_t s) {
  const unsigned rows = static_cast<unsigned>(p.batch * p.dim);
  switch (dt) {
    case DType::F32: segment_decay_kernel<float><<<rows, kDecayThreads, 0, s>>>(p); break;
    case DType::BF16: segment_decay_kernel<__nv_bfloat16><<<rows, kDecayThreads, 0, s>>>(p); break;
    case DType::F16: segment_decay_kernel<__half><<<rows, kDecayThreads, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_state_chain(const StateChainParams& p, cudaStream_t s) {
  const unsigned blocks = static_cast<unsigned>((p.count + 255) / 256);
  state_chain_kernel<<<blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ss
