// ss_internal.h -- kernel parameter blocks and launchers behind the C ABI.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ss {

enum class DType : int { F32 = 0, BF16 = 1, F16 = 2 };

// Forward problem.  Segments split L for the chunk-parallel path; on the
// per-channel path nseg == 1 and seg_len >= L.
struct FwdParams {
  int batch, dim, seqlen;
  int nseg, seg_len;          // seg_len is a multiple of the checkpoint chunk
  int nchunk;                 // ceil(seqlen / 64)
  int lanes;                  // lanes per channel: 4 (4 states each) or 8 (2 each)
  int sms;                    // SM count of the device (sizes the grid's waves)
  const void *u, *delta, *z, *B, *C;
  const float *A, *D, *bias;
  int softplus;
  void* y;
  const float* h0;            // (batch, dim, 16) initial state, or null (zero)
  const int* seq_idx;         // (batch, seqlen) document ids, or null (one document)
  float* final_state;         // (batch, dim, 16) or null
  float* ckpt;                // (batch, dim, nchunk, 16) or null
  // chunk-parallel workspace, each (nseg, batch, dim, 16) fp32
  float* seg_end;             // state at segment end when started from zero
  float* seg_decay;           // product of the segment's decays
  float* seg_hin;             // true state entering each segment
};

// Reverse-walk kernel variants (channels per block, threads per channel).
enum BwdVariant : int {
  kBwdLanes = 0,     // 16 channels, one channel per 4-lane group, 64 threads
  kBwdPairs32 = 1,   // 32 channels, two channels per 4-lane group, 64 threads
  kBwdPairs16 = 2,   // 16 channels, two channels per 4-lane group, 32 threads
  kBwdChannel = 3,   // 128 channels, one channel (all 16 states) per thread (ss_bwd_ch.cu)
};
inline int bwd_block_channels(int variant) { return variant == kBwdPairs32 ? 32 : 16; }

struct BwdParams {
  int batch, dim, seqlen, nchunk, nblk;
  int variant;                // BwdVariant
  int nsub;                   // ceil(seqlen / 8): sub-chunks of the reverse walk
  // The reverse walk runs in parallel over groups of whole 64-step chunks;
  // group g covers sub-chunks [g * group_nsub, min(nsub, (g + 1) * group_nsub)).
  // Set by the launcher (ngroups <= kMaxBwdGroups).
  int ngroups, group_nsub;
  int sms;                    // SM count of the device (sizes the walk's groups)
  const void *u, *delta, *z, *B, *C, *dy;
  const float *A, *D, *bias, *ckpt;
  const float* h0;            // (batch, dim, 16) initial state of the forward, or null
  const int* seq_idx;         // (batch, seqlen) document ids, or null
  const float* dfinal;        // (batch, dim, 16) gradient reaching the final state, or null
  float* dh0;                 // (batch, dim, 16) gradient of the initial state, or null
  int softplus;
  void *du, *ddelta, *dz;
  // workspace
  float* sub_state;           // (batch, dim, nsub, 16): state entering each sub-chunk
  float* part_dB;             // (batch, nblk, Lp, 16) per-block channel sums, Lp = ceil16(L)
  float* part_dC;             // (batch, nblk, Lp, 16)
  float* part_dA;             // (ngroups * batch, dim, 16): per (group, row) sums
  float* part_dD;             // (ngroups * batch, dim)
  float* part_dbias;          // (ngroups * batch, dim)
  // gradient carry across chunks (ngroups > 1): the map carry -> P_k carry + e_k
  // of each chunk, and the carry entering the last step of each group
  float* chunk_carry;         // (batch, dim, nchunk, 16): e_k
  float* chunk_decay;         // (batch, dim, nchunk, 16): P_k
  float* group_carry;         // (batch, dim, ngroups, 16)
  // one-channel-per-thread walk (kBwdChannel), 16-byte aligned rows only
  int nsub4;                  // ceil(seqlen / 4): sub-chunks whose entering state is stored
  int ncb;                    // channel blocks of kChBlock
  int lpad;                   // nchunk * 64: rows of the dB / dC partials
  int dpad;                   // dim rounded up to a multiple of 4: channel stride of the slot layouts
  // Per-channel states below are kept in the walk's slot order, [8 pairs][dpad][2]
  // per (batch, step index): pair k of channel d holds states 2 (k ^ x), +1 with
  // x = ((d % 32) >> 2) & 7.
  float* ch_state;            // (batch, nsub4, 8, dpad, 2): state entering each 4-step sub-chunk
  float* ch_part_dB;          // (batch, ncb, lpad, 16) per-block channel sums
  float* ch_part_dC;          // (batch, ncb, lpad, 16)
  float* ch_map_e;            // (batch, nchunk, 8, dpad, 2): e_k of the chunk's carry map
  float* ch_map_P;            // (batch, nchunk, 8, dpad, 2): P_k
  float* ch_carry;            // (batch, ngroups, 8, dpad, 2): carry entering each group's last step
  // final outputs
  float *dA, *dB, *dC, *dD, *dbias;
};

struct UpdateParams {
  int batch, dim;
  float* state;
  const void *u, *delta, *z, *B, *C;
  const float *A, *D, *bias;
  int softplus;
  void* y;
};

// Tiling constants shared by host and device code.
constexpr int kBwdMinBlockChannels = 16;   // partial-sum buffers are sized for this
constexpr int kSub = 8;       // steps per backward sub-chunk
constexpr int kMaxBwdGroups = 16;          // most chunk groups walked in parallel
constexpr int kChBlock = 128;              // channels per block of the one-channel-per-thread walk
constexpr int kChSub = 4;                  // steps between its stored states
constexpr int kMaxChGroups = 32;           // most chunk groups of that walk

// Causal depthwise conv1d (+ SiLU), its adjoint and its decode step.
struct ConvParams {
  int batch, dim, seqlen, width, silu;
  const void* x;              // (batch, dim, seqlen) [step: (batch, dim)]
  const float *w, *bias;      // (dim, width), (dim,) or null
  const float* state_in;      // (batch, dim, width-1) inputs before t = 0, or null
  const int* seq_idx;         // (batch, seqlen) document ids, or null
  void* u;                    // output (batch, dim, seqlen) [step: (batch, dim)]
  float* state_out;           // (batch, dim, width-1) last inputs, or null [step: in/out window]
  const void* du;             // backward: gradient of u
  const float* dstate_out;    // backward: gradient reaching state_out, or null
  void* dx;                   // backward: gradient of x
  float *dw, *dbias, *dstate_in;
  float* part;                // backward workspace: (batch, dim, width+1) per-row sums
};

// Mamba-2 SSD forward: scalar A per head, grouped B/C, (headdim x dstate) state.
struct SsdParams {
  int batch, seqlen, nheads, headdim, ngroups, dstate, softplus;
  const void *x, *dt, *B, *C, *z;   // (b,L,nh,P), (b,L,nh), (b,L,ng,N) x2, (b,L,nh,P) or null
  const float *A, *D, *dt_bias;     // (nh,) each; D, dt_bias may be null
  const float* h0;                  // (b, nh, P, N) or null
  void* y;                          // (b, L, nh, P)
  float* final_state;               // (b, nh, P, N) or null
  int inject_timeout;               // test hook: the first chunk's copy wait runs out (tcgen05 kernel)
};

// Sequence sharding (ss_shard.cu): the diagonal state transition of a segment
// and the chain of segment states / adjoints.
struct SegmentDecayParams {
  int batch, dim, dstate, seqlen, softplus;
  const void* delta;          // (batch, dim, seqlen)
  const float *A, *delta_bias;
  float* P;                   // (batch, dim, dstate)
};
struct StateChainParams {
  int64_t count;              // elements per segment slab
  int nseg, reverse;
  const float *P, *E, *init;  // (nseg, count) each; init (count,) or null (zero)
  float* out;                 // (nseg, count)
};
cudaError_t launch_segment_decay(const SegmentDecayParams& p, DType dt, cudaStream_t s);
cudaError_t launch_state_chain(const StateChainParams& p, cudaStream_t s);

cudaError_t launch_fwd(const FwdParams& p, DType dt, bool vec, cudaStream_t s);
// SSD forward: tcgen05/TMEM/TMA kernel (ss_ssd_tc.cu) and the warp-level
// mma.sync kernel (ss_ssd.cu).
cudaError_t launch_ssd_fwd_tc(const SsdParams& p, DType dt, cudaStream_t s);
cudaError_t launch_ssd_fwd_mma(const SsdParams& p, DType dt, cudaStream_t s);
// Device fault word of the kernels with bounded waits (synchronizes the device).
cudaError_t read_tc_fault(unsigned* bits, bool clear);
// op: 0 forward, 1 backward (+ fixed-order reduction), 2 decode step
cudaError_t launch_conv(const ConvParams& p, int op, DType dt, bool vec, cudaStream_t s);
cudaError_t launch_bwd(const BwdParams& p, DType dt, bool vec, cudaStream_t s);
// The chunk groups launch_bwd will use (sets p.ngroups, p.group_nsub).
cudaError_t plan_bwd(BwdParams& p, DType dt, bool vec);
// The one-channel-per-thread backward (variant kBwdChannel): its chunk groups,
// given the walk blocks one SM holds, and its launch.
void choose_ch_groups(BwdParams& p, int blocks_per_sm);
cudaError_t plan_bwd_ch(BwdParams& p, DType dt);
cudaError_t launch_bwd_ch(const BwdParams& p, DType dt, cudaStream_t s);
cudaError_t launch_state_update(const UpdateParams& p, DType dt, cudaStream_t s);

}  // namespace ss
