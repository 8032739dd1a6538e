// ss_ssd_bwd.h -- parameter block, workspace layout and launcher of the Mamba-2
// SSD backward (ss_ssd_bwd.cu).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ss_internal.h"

namespace ss {

struct SsdBwdParams {
  int batch, seqlen, nheads, headdim, ngroups, dstate, softplus;
  int nchunk;                          // ceil(seqlen / 64)
  int hpc;                             // heads per CTA of the tcgen05 chunk gradients, which store one
                                       // dB, dC partial per hpc heads; 1 on the mma.sync path
  const void *x, *dt, *B, *C, *z, *dy; // layouts as in the forward; dy like x
  const float *A, *D, *dt_bias;        // (nh,); D, dt_bias may be null
  const float *h0, *dfinal;            // (b, nh, P, N) or null (zero)
  void *dx, *ddt, *dz;                 // dtype; dz only with z
  float *dA, *dB, *dC, *dD, *ddt_bias; // dB, dC (b, L, ng, N); others (nh,); dD, ddt_bias may be null
  float* dh0;                          // (b, nh, P, N) or null
  // workspace
  float* su;     // (b, nh, nchunk, P, N): the chunk's state map U_k, then the state entering chunk k
  float* gv;     // (b, nh, nchunk, P, N): the chunk's adjoint map V_k, then the adjoint leaving chunk k
  float* dec;    // (b, nh, nchunk): exp(A_h * sum of the chunk's Delta)
  float* pdB;    // (b, L, nh, N): dB of each head, summed over its group afterwards
  float* pdC;
  float *pA, *pD, *pbias;  // (b, nh, nchunk) per-chunk partials of dA, dD, ddt_bias
};

struct SsdBwdLayout {
  size_t off_su, off_gv, off_dec, off_pdB, off_pdC, off_pA, off_pD, off_pbias, total;
};

// Byte offsets of the workspace regions (each 256-byte aligned).
SsdBwdLayout ssd_bwd_layout(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                            int64_t dstate);
void ssd_bwd_bind(SsdBwdParams& p, void* workspace);
// tc: the chunk maps and the chunk gradients on tcgen05 (ss_ssd_bwd_tc.cu)
// instead of the tf32 mma.sync kernels.
cudaError_t launch_ssd_bwd(const SsdBwdParams& p, DType dt, bool tc_maps, cudaStream_t s);
// Heads per CTA for the tcgen05 chunk gradients: the largest divisor of the
// heads per group, up to min(cap, 8), that still gives every SM a CTA (force:
// whatever the grid).
int ssd_heads_per_cta(int batch, int nchunk, int nheads, int ngroups, int sms, int cap, bool force);
cudaError_t launch_ssd_maps_tc(const SsdBwdParams& p, DType dt, cudaStream_t s);
cudaError_t launch_ssd_grad_tc(const SsdBwdParams& p, DType dt, cudaStream_t s);
// The pass over the chunks on the tcgen05 path's fp16 slabs (stored in
// operand-tile order; the workspace keeps its fp32 size).
cudaError_t launch_ssd_pass16(const SsdBwdParams& p, cudaStream_t s);
cudaError_t read_tc_fault_bwd(unsigned* bits, bool clear);

}  // namespace ss
