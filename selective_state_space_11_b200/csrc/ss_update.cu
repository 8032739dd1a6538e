// ss_update.cu -- single-step decode state update for sm_100a.
//
// One recurrence step on a cached state, in place ("Mamba", stanleyjacob.dev,
// Part IV Stage 7: one token in, a fixed-size state updated in place, one
// token out; "mamba-metal" README, "O(1) per token via state caching"):
//   h <- exp(Delta A) h + Delta B u,   y = (C.h + D u) SiLU(z),
//   Delta = softplus(delta + bias).
// 4 lanes per channel with 4 states each (one 128-bit state load and store
// per lane); the 4 partial readouts combine with two xor-shuffles in a fixed
// order.  The whole state of a decode batch is a few hundred KB, so the step
// is launch-latency bound: one kernel, no host synchronisation, capturable in
// a CUDA graph.
#include "ss_device.cuh"
#include "ss_internal.h"

namespace ss {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) update_kernel(const UpdateParams p) {
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long ch = gt >> 2;
  const int j = (int)(gt & 3);
  const long long nch = (long long)p.batch * p.dim;
  const bool valid = ch < nch;
  const long long chc = valid ? ch : 0;
  const int b = (int)(chc / p.dim), d = (int)(chc % p.dim);

  const T* u = static_cast<const T*>(p.u);
  const T* dl = static_cast<const T*>(p.delta);
  const T* z = static_cast<const T*>(p.z);
  const T* Bm = static_cast<const T*>(p.B) + (size_t)b * kN + 4 * j;
  const T* Cm = static_cast<const T*>(p.C) + (size_t)b * kN + 4 * j;

  const float uv = ldf(u + chc);
  const float x = ldf(dl + chc) + (p.bias ? p.bias[d] : 0.f);
  const float dt = p.softplus ? softplus_f(x) : x;
  const float du = dt * uv;

  float* st = p.state + chc * kN + 4 * j;
  const float4 h4 = *reinterpret_cast<const float4*>(st);
  float h[4] = {h4.x, h4.y, h4.z, h4.w};
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float a = ex2(dt * p.A[(size_t)d * kN + 4 * j + k] * kLog2e);
    h[k] = fmaf(a, h[k], du * ldf(Bm + k));
    acc = fmaf(ldf(Cm + k), h[k], acc);
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  if (!valid) return;
  *reinterpret_cast<float4*>(st) = make_float4(h[0], h[1], h[2], h[3]);
  if (j == 0) {
    float out = fmaf(p.D ? p.D[d] : 0.f, uv, acc);
    if (z) {
      const float zv = ldf(z + chc);
      out *= zv * sigmoid_f(zv);
    }
    stf(static_cast<T*>(p.y) + chc, out);
  }
}

template <typename T>
cudaError_t launch_t(const UpdateParams& p, cudaStream_t s) {
  const long long threads = (long long)p.batch * p.dim * 4;
  const long long blocks = (threads + 255) / 256;
  update_kernel<T><<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const UpdateParams& p, DType dt, cudaStream_t s) {
  switch (dt) {
    case DType::F32: return launch_t<float>(p, s);
    case DType::BF16: return launch_t<__nv_bfloat16>(p, s);
    case DType::F16: return launch_t<__half>(p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ss
