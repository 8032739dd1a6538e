// ss_api.cu -- the C ABI declared in include/ss.h: argument validation, path
// choice, workspace layout, dispatch and error reporting.  No allocation, no
// host synchronisation, no exceptions across the boundary.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "../../include/ss.h"
#include "ss_internal.h"
#include "ss_ssd_bwd.h"

namespace {

thread_local char g_err[512] = "";

ss_status fail(ss_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

constexpr int kN = 16;
constexpr int kChunk = SS_CHECKPOINT_CHUNK;

size_t elt_size(int dtype) { return dtype == SS_F32 ? 4 : 2; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// SM count of the current device, cached per device (cudaDeviceGetAttribute
// is cheap but not free on a decode-sized call).
std::atomic<int> g_sms[64];

int current_sm_count(int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64) {
    int v = g_sms[dev].load(std::memory_order_relaxed);
    if (v > 0) {
      *out = v;
      return 0;
    }
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess || sms <= 0) return -1;
  if (dev >= 0 && dev < 64) g_sms[dev].store(sms, std::memory_order_relaxed);
  *out = sms;
  return 0;
}

ss_status check_sizes(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, bool need_len) {
  if (batch <= 0 || dim <= 0 || dstate <= 0 || (need_len && seqlen <= 0))
    return fail(SS_ERR_INVALID_ARG, "sizes must be positive (batch=%lld dim=%lld dstate=%lld seqlen=%lld)",
                (long long)batch, (long long)dim, (long long)dstate, (long long)seqlen);
  if (dstate != kN)
    return fail(SS_ERR_UNSUPPORTED, "dstate=%lld: only dstate=16 is implemented", (long long)dstate);
  if (batch > 65535 || dim > (1 << 26) || seqlen > (1 << 30))
    return fail(SS_ERR_UNSUPPORTED, "size out of supported range (batch<=65535, dim<=2^26, seqlen<=2^30)");
  if ((unsigned long long)batch * (unsigned long long)dim > (1ull << 31))
    return fail(SS_ERR_UNSUPPORTED, "batch*dim above 2^31");
  return SS_OK;
}

// Launch-failure injection, for testing callers' error paths without faulting
// a GPU: with the environment variable SS_FAIL_LAUNCH set (to anything but "0"),
// every entry point returns SS_ERR_CUDA at the point where it would launch,
// having enqueued nothing.
bool launch_injected() {
  const char* v = getenv("SS_FAIL_LAUNCH");
  return v && *v && strcmp(v, "0") != 0;
}

ss_status check_dtype(int dtype) {
  if (dtype != SS_F32 && dtype != SS_BF16 && dtype != SS_F16)
    return fail(SS_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  return SS_OK;
}

// Forward path: per-channel scan unless there are too few channels to occupy
// the GPU, then split L into segments (multiples of the checkpoint chunk).
void choose_segments(int64_t batch, int64_t dim, int64_t seqlen, int sms, int* nseg, int* seg_len) {
  const int64_t channels = batch * dim;
  const int64_t nchunk = (seqlen + kChunk - 1) / kChunk;
  int64_t ns = 1;
  if (channels < (int64_t)sms * 32) {
    ns = ((int64_t)sms * 128 + channels - 1) / channels;
    if (ns > nchunk) ns = nchunk;
    if (ns > 65535) ns = 65535;
  }
  if (ns <= 1) {
    *nseg = 1;
    *seg_len = (int)(nchunk * kChunk);
    return;
  }
  const int64_t chunks_per_seg = (nchunk + ns - 1) / ns;
  *seg_len = (int)(chunks_per_seg * kChunk);
  *nseg = (int)((nchunk + chunks_per_seg - 1) / chunks_per_seg);
}

size_t fwd_ws_bytes(int64_t batch, int64_t dim, int nseg) {
  if (nseg <= 1) return 0;
  return 3 * round_up((size_t)nseg * batch * dim * kN * sizeof(float), 256);
}

// Forward lanes per channel: 4 lanes x 4 states, or 8 lanes x 2 states.  Four
// lanes issue fewer instructions per token*channel; eight double the warps
// for problems too small to give every SM sub-partition one.
int choose_lanes(int64_t items, int64_t dim, int sms) {
#ifdef SS_FORCE_LANES
  (void)items; (void)dim; (void)sms;
  return SS_FORCE_LANES;
#else
  // 8 lanes (16-channel blocks) when 4 would leave most sub-partitions
  // without a warp, or when d_inner fills no more than half of a 4-lane
  // block's 32 channels
  const double w4 = (double)items * 4.0 / 32.0 / (4.0 * sms);
  return (w4 < 1.0 || dim <= 16) ? 8 : 4;
#endif
}

struct BwdLayout {
  size_t off_S, off_B, off_C, off_A, off_D, off_bias, off_E, off_P, off_G, total;
  int nblk, nsub, nchunk, gmax;
  // the one-channel-per-thread walk's layout (offsets from the workspace start)
  size_t ch_S, ch_B, ch_C, ch_A, ch_D, ch_bias, ch_E, ch_P, ch_G, ch_total;
  int nsub4, ncb, lpad, dpad, ch_gmax;
};

// Reverse-walk variant.  Problems whose rows are 16-byte aligned take the
// one-channel-per-thread walk (ss_bwd_ch.cu).  Other rows take the 4-lane
// walks: channel pairs halve the shared-memory traffic per token*channel but
// also halve the threads; they pay off once the pair blocks, times the chunk
// groups the walk can run in parallel, give every SM at least eight one-warp
// blocks.  Below that the one-channel-per-lane-group walk keeps more warps in
// flight.  The environment variable SS_BWD_VARIANT (0..3) forces a variant for
// testing; variant 3 is honoured only where the rows allow it.
int choose_bwd_variant(int64_t batch, int64_t dim, int64_t seqlen, int sms, bool vec) {
  if (const char* env = getenv("SS_BWD_VARIANT")) {
    const int v = atoi(env);
    if (v >= 0 && v <= 2) return v;
    if (v == ss::kBwdChannel && vec) return v;
  }
#ifdef SS_BWD_FORCE
  (void)batch; (void)dim; (void)seqlen; (void)sms; (void)vec;
  return SS_BWD_FORCE;
#else
  if (vec) return ss::kBwdChannel;
  const int64_t channels = batch * dim;
  if (channels >= (int64_t)sms * 128) return ss::kBwdPairs16;
  const int64_t nchunk = (seqlen + kChunk - 1) / kChunk;
  const int64_t groups = nchunk < ss::kMaxBwdGroups ? nchunk : ss::kMaxBwdGroups;
  const int64_t pair_blocks = batch * ((dim + 15) / 16);
  return pair_blocks * groups >= (int64_t)sms * 8 ? ss::kBwdPairs16 : ss::kBwdLanes;
#endif
}

// Workspace of the backward, sized for the most chunk groups the walk may use.
BwdLayout bwd_layout(int64_t batch, int64_t dim, int64_t seqlen) {
  BwdLayout l;
  l.nblk = (int)((dim + ss::kBwdMinBlockChannels - 1) / ss::kBwdMinBlockChannels);
  l.nsub = (int)((seqlen + ss::kSub - 1) / ss::kSub);
  l.nchunk = (int)((seqlen + kChunk - 1) / kChunk);
  l.gmax = l.nchunk < ss::kMaxBwdGroups ? l.nchunk : ss::kMaxBwdGroups;
  const size_t Lp = round_up((size_t)seqlen, 16);
  const size_t part = round_up((size_t)batch * l.nblk * kN * Lp * sizeof(float), 256);
  const size_t rows = (size_t)l.gmax * batch;                  // (group, batch row) partials
  const size_t chunk_maps = l.gmax > 1 ? round_up((size_t)batch * dim * l.nchunk * kN * sizeof(float), 256) : 0;
  l.off_S = 0;
  l.off_B = round_up((size_t)batch * dim * l.nsub * kN * sizeof(float), 256);
  l.off_C = l.off_B + part;
  l.off_A = l.off_C + part;
  l.off_D = l.off_A + round_up(rows * dim * kN * sizeof(float), 256);
  l.off_bias = l.off_D + round_up(rows * dim * sizeof(float), 256);
  l.off_E = l.off_bias + round_up(rows * dim * sizeof(float), 256);
  l.off_P = l.off_E + chunk_maps;
  l.off_G = l.off_P + chunk_maps;
  l.total = l.off_G + (l.gmax > 1 ? round_up((size_t)batch * dim * l.gmax * kN * sizeof(float), 256) : 0);
  // one-channel-per-thread walk
  l.nsub4 = (int)((seqlen + ss::kChSub - 1) / ss::kChSub);
  l.ncb = (int)((dim + ss::kChBlock - 1) / ss::kChBlock);
  l.lpad = l.nchunk * kChunk;
  l.dpad = (int)((dim + 3) / 4 * 4);
  l.ch_gmax = l.nchunk < ss::kMaxChGroups ? l.nchunk : ss::kMaxChGroups;
  const size_t ch_part = round_up((size_t)batch * l.ncb * l.lpad * kN * sizeof(float), 256);
  const size_t ch_rows = (size_t)l.ch_gmax * batch;
  const size_t ch_maps = l.nchunk > 1 ? round_up((size_t)batch * l.nchunk * l.dpad * kN * sizeof(float), 256) : 0;
  l.ch_S = 0;
  l.ch_B = round_up((size_t)batch * l.nsub4 * l.dpad * kN * sizeof(float), 256);
  l.ch_C = l.ch_B + ch_part;
  l.ch_A = l.ch_C + ch_part;
  l.ch_D = l.ch_A + round_up(ch_rows * dim * kN * sizeof(float), 256);
  l.ch_bias = l.ch_D + round_up(ch_rows * dim * sizeof(float), 256);
  l.ch_E = l.ch_bias + round_up(ch_rows * dim * sizeof(float), 256);
  l.ch_P = l.ch_E + ch_maps;
  l.ch_G = l.ch_P + ch_maps;
  l.ch_total = l.ch_G + (l.nchunk > 1 ? round_up((size_t)batch * l.ch_gmax * l.dpad * kN * sizeof(float), 256) : 0);
  if (l.ch_total > l.total) l.total = l.ch_total;
  return l;
}

bool rows_vec_ok(int64_t seqlen, int dtype, std::initializer_list<const void*> ptrs) {
  if (((size_t)seqlen * elt_size(dtype)) % 16 != 0) return false;
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return false;
  return true;
}

}  // namespace

extern "C" {

int ss_version(void) { return 1 * 10000 + 4 * 100 + 0; }

const char* ss_last_error(void) { return g_err; }

const char* ss_status_string(int status) {
  switch (status) {
    case SS_OK: return "SS_OK";
    case SS_ERR_INVALID_ARG: return "SS_ERR_INVALID_ARG";
    case SS_ERR_UNSUPPORTED: return "SS_ERR_UNSUPPORTED";
    case SS_ERR_ALIGNMENT: return "SS_ERR_ALIGNMENT";
    case SS_ERR_WORKSPACE: return "SS_ERR_WORKSPACE";
    case SS_ERR_CUDA: return "SS_ERR_CUDA";
    case SS_ERR_INTERNAL: return "SS_ERR_INTERNAL";
  }
  return "SS_UNKNOWN_STATUS";
}

int ss_fwd_path(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int64_t* num_segments) {
  if (check_sizes(batch, dim, dstate, seqlen, true) != SS_OK) return -1;
  int sms = 0;
  if (current_sm_count(&sms) != 0) {
    fail(SS_ERR_CUDA, "cannot query the current device's SM count");
    return -1;
  }
  int nseg = 1, seg_len = 0;
  choose_segments(batch, dim, seqlen, sms, &nseg, &seg_len);
  if (num_segments) *num_segments = nseg;
  return nseg > 1 ? 1 : 0;
}

size_t ss_fwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen) {
  if (check_sizes(batch, dim, dstate, seqlen, true) != SS_OK) return (size_t)-1;
  int sms = 0;
  if (current_sm_count(&sms) != 0) {
    fail(SS_ERR_CUDA, "cannot query the current device's SM count");
    return (size_t)-1;
  }
  int nseg = 1, seg_len = 0;
  choose_segments(batch, dim, seqlen, sms, &nseg, &seg_len);
  return fwd_ws_bytes(batch, dim, nseg);
}

ss_status ss_fwd_with_state(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                            const void* u, const void* delta, const void* z, const float* A,
                            const void* B, const void* C, const float* D, const float* delta_bias,
                            int delta_softplus, const float* h0, const int32_t* seq_idx, void* y,
                            float* final_state, float* checkpoints, void* workspace,
                            size_t workspace_bytes, void* stream) {
  ss_status st = check_sizes(batch, dim, dstate, seqlen, true);
  if (st != SS_OK) return st;
  if ((st = check_dtype(dtype)) != SS_OK) return st;
  if (!u || !delta || !A || !B || !C || !y)
    return fail(SS_ERR_INVALID_ARG, "ss_fwd: u, delta, A, B, C and y are required");
  const size_t es = elt_size(dtype);
  for (const void* p : {u, delta, z, B, C, (const void*)y})
    if (p && !aligned(p, es)) return fail(SS_ERR_ALIGNMENT, "ss_fwd: data pointer %p not aligned to %zu bytes", p, es);
  for (const void* p : {(const void*)A, (const void*)D, (const void*)delta_bias})
    if (p && !aligned(p, 4)) return fail(SS_ERR_ALIGNMENT, "ss_fwd: fp32 pointer %p not 4-byte aligned", p);
  for (const void* p : {(const void*)h0, (const void*)final_state, (const void*)checkpoints})
    if (p && !aligned(p, 16)) return fail(SS_ERR_ALIGNMENT, "ss_fwd: state pointer %p not 16-byte aligned", p);
  if (seq_idx && !aligned(seq_idx, 4)) return fail(SS_ERR_ALIGNMENT, "ss_fwd: seq_idx not 4-byte aligned");
  int sms = 0;
  if (current_sm_count(&sms) != 0) return fail(SS_ERR_CUDA, "ss_fwd: cannot query the device");
  int nseg = 1, seg_len = 0;
  choose_segments(batch, dim, seqlen, sms, &nseg, &seg_len);
  const size_t need = fwd_ws_bytes(batch, dim, nseg);
  if (need > 0) {
    if (!workspace || workspace_bytes < need)
      return fail(SS_ERR_WORKSPACE, "ss_fwd: chunk-parallel path needs %zu workspace bytes, got %zu", need,
                  workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, 16)) return fail(SS_ERR_ALIGNMENT, "ss_fwd: workspace not 16-byte aligned");
  }
  ss::FwdParams p{};
  p.batch = (int)batch;
  p.dim = (int)dim;
  p.seqlen = (int)seqlen;
  p.nseg = nseg;
  p.seg_len = seg_len;
  p.nchunk = (int)((seqlen + kChunk - 1) / kChunk);
  p.lanes = choose_lanes(batch * dim * nseg, dim, sms);
  p.sms = sms;
  p.u = u; p.delta = delta; p.z = z; p.B = B; p.C = C;
  p.A = A; p.D = D; p.bias = delta_bias;
  p.softplus = delta_softplus ? 1 : 0;
  p.y = y;
  p.h0 = h0;
  p.seq_idx = seq_idx;
  p.final_state = final_state;
  p.ckpt = checkpoints;
  if (need > 0) {
    const size_t one = need / 3;
    char* w = static_cast<char*>(workspace);
    p.seg_end = reinterpret_cast<float*>(w);
    p.seg_decay = reinterpret_cast<float*>(w + one);
    p.seg_hin = reinterpret_cast<float*>(w + 2 * one);
  }
  const bool vec = rows_vec_ok(seqlen, dtype, {u, delta, z, B, C, (const void*)y});
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  cudaError_t e = ss::launch_fwd(p, static_cast<ss::DType>(dtype), vec, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_fwd: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

ss_status ss_fwd(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                 const void* u, const void* delta, const void* z, const float* A,
                 const void* B, const void* C, const float* D, const float* delta_bias,
                 int delta_softplus, void* y, float* final_state, float* checkpoints,
                 void* workspace, size_t workspace_bytes, void* stream) {
  return ss_fwd_with_state(batch, dim, dstate, seqlen, dtype, u, delta, z, A, B, C, D, delta_bias,
                           delta_softplus, nullptr, nullptr, y, final_state, checkpoints, workspace,
                           workspace_bytes, stream);
}

int ss_bwd_path(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                int64_t* num_groups) {
  if (check_sizes(batch, dim, dstate, seqlen, true) != SS_OK) return -1;
  if (check_dtype(dtype) != SS_OK) return -1;
  int sms = 0;
  if (current_sm_count(&sms) != 0) {
    fail(SS_ERR_CUDA, "cannot query the current device's SM count");
    return -1;
  }
  const BwdLayout lay = bwd_layout(batch, dim, seqlen);
  ss::BwdParams p{};
  p.batch = (int)batch;
  p.dim = (int)dim;
  p.seqlen = (int)seqlen;
  p.nchunk = lay.nchunk;
  p.nsub = lay.nsub;
  p.sms = sms;
  const bool vec = ((size_t)seqlen * elt_size(dtype)) % 16 == 0;
  p.variant = choose_bwd_variant(batch, dim, seqlen, sms, vec);
  p.nblk = (int)((dim + ss::bwd_block_channels(p.variant) - 1) / ss::bwd_block_channels(p.variant));
  p.nsub4 = lay.nsub4;
  p.ncb = lay.ncb;
  p.lpad = lay.lpad;
  p.dpad = lay.dpad;
  const cudaError_t pe = p.variant == ss::kBwdChannel ? ss::plan_bwd_ch(p, static_cast<ss::DType>(dtype))
                                                      : ss::plan_bwd(p, static_cast<ss::DType>(dtype), vec);
  if (pe != cudaSuccess) {
    fail(SS_ERR_CUDA, "ss_bwd_path: cannot plan the walk");
    return -1;
  }
  if (num_groups) *num_groups = p.ngroups;
  return p.variant;
}

size_t ss_bwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen) {
  if (check_sizes(batch, dim, dstate, seqlen, true) != SS_OK) return (size_t)-1;
  return bwd_layout(batch, dim, seqlen).total;
}

ss_status ss_bwd_with_state(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                            const void* u, const void* delta, const void* z, const float* A,
                            const void* B, const void* C, const float* D, const float* delta_bias,
                            int delta_softplus, const float* h0, const int32_t* seq_idx,
                            const void* dy, const float* dfinal,
                            const float* checkpoints, void* du, void* ddelta, void* dz, float* dA,
                            float* dB, float* dC, float* dD, float* ddelta_bias, float* dh0,
                            void* workspace, size_t workspace_bytes, void* stream) {
  ss_status st = check_sizes(batch, dim, dstate, seqlen, true);
  if (st != SS_OK) return st;
  if ((st = check_dtype(dtype)) != SS_OK) return st;
  if (!u || !delta || !A || !B || !C || !dy || !checkpoints || !du || !ddelta || !dA || !dB || !dC)
    return fail(SS_ERR_INVALID_ARG,
                "ss_bwd: u, delta, A, B, C, dy, checkpoints, du, ddelta, dA, dB and dC are required");
  if (z && !dz) return fail(SS_ERR_INVALID_ARG, "ss_bwd: dz is required when z is given");
  const size_t es = elt_size(dtype);
  for (const void* p : {u, delta, z, B, C, dy, (const void*)du, (const void*)ddelta, (const void*)(z ? dz : nullptr)})
    if (p && !aligned(p, es)) return fail(SS_ERR_ALIGNMENT, "ss_bwd: data pointer %p not aligned to %zu bytes", p, es);
  for (const void* p : {(const void*)A, (const void*)D, (const void*)delta_bias, (const void*)dA, (const void*)dB,
                        (const void*)dC, (const void*)dD, (const void*)ddelta_bias})
    if (p && !aligned(p, 4)) return fail(SS_ERR_ALIGNMENT, "ss_bwd: fp32 pointer %p not 4-byte aligned", p);
  if (!aligned(checkpoints, 16)) return fail(SS_ERR_ALIGNMENT, "ss_bwd: checkpoints not 16-byte aligned");
  for (const void* p : {(const void*)h0, (const void*)dfinal, (const void*)dh0})
    if (p && !aligned(p, 16)) return fail(SS_ERR_ALIGNMENT, "ss_bwd: state pointer %p not 16-byte aligned", p);
  if (seq_idx && !aligned(seq_idx, 4)) return fail(SS_ERR_ALIGNMENT, "ss_bwd: seq_idx not 4-byte aligned");
  const BwdLayout lay = bwd_layout(batch, dim, seqlen);
  if (!workspace || workspace_bytes < lay.total)
    return fail(SS_ERR_WORKSPACE, "ss_bwd: needs %zu workspace bytes, got %zu", lay.total,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned(workspace, 16)) return fail(SS_ERR_ALIGNMENT, "ss_bwd: workspace not 16-byte aligned");
  ss::BwdParams p{};
  p.batch = (int)batch;
  p.dim = (int)dim;
  p.seqlen = (int)seqlen;
  p.nchunk = (int)((seqlen + kChunk - 1) / kChunk);
  int sms = 0;
  if (current_sm_count(&sms) != 0) return fail(SS_ERR_CUDA, "ss_bwd: cannot query the current device");
  const bool vec = rows_vec_ok(seqlen, dtype, {u, delta, z, B, C, dy, (const void*)du, (const void*)ddelta,
                                               (const void*)(z ? dz : nullptr)}) &&
                   aligned(A, 16);
  p.variant = choose_bwd_variant(batch, dim, seqlen, sms, vec);
  p.sms = sms;
  p.nblk = (int)((dim + ss::bwd_block_channels(p.variant) - 1) / ss::bwd_block_channels(p.variant));
  p.nsub = lay.nsub;
  p.nsub4 = lay.nsub4;
  p.ncb = lay.ncb;
  p.lpad = lay.lpad;
  p.dpad = lay.dpad;
  p.u = u; p.delta = delta; p.z = z; p.B = B; p.C = C; p.dy = dy;
  p.A = A; p.D = D; p.bias = delta_bias; p.ckpt = checkpoints;
  p.h0 = h0; p.dfinal = dfinal; p.dh0 = dh0; p.seq_idx = seq_idx;
  p.softplus = delta_softplus ? 1 : 0;
  p.du = du; p.ddelta = ddelta; p.dz = z ? dz : nullptr;
  p.dA = dA; p.dB = dB; p.dC = dC; p.dD = dD; p.dbias = ddelta_bias;
  char* w = static_cast<char*>(workspace);
  if (p.variant == ss::kBwdChannel) {
    p.ch_state = reinterpret_cast<float*>(w + lay.ch_S);
    p.ch_part_dB = reinterpret_cast<float*>(w + lay.ch_B);
    p.ch_part_dC = reinterpret_cast<float*>(w + lay.ch_C);
    p.part_dA = reinterpret_cast<float*>(w + lay.ch_A);
    p.part_dD = reinterpret_cast<float*>(w + lay.ch_D);
    p.part_dbias = reinterpret_cast<float*>(w + lay.ch_bias);
    p.ch_map_e = lay.nchunk > 1 ? reinterpret_cast<float*>(w + lay.ch_E) : nullptr;
    p.ch_map_P = lay.nchunk > 1 ? reinterpret_cast<float*>(w + lay.ch_P) : nullptr;
    p.ch_carry = lay.nchunk > 1 ? reinterpret_cast<float*>(w + lay.ch_G) : nullptr;
    if (launch_injected())
      return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
    cudaError_t e = ss::launch_bwd_ch(p, static_cast<ss::DType>(dtype), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_bwd: launch failed: %s", cudaGetErrorString(e));
    return SS_OK;
  }
  p.sub_state = reinterpret_cast<float*>(w + lay.off_S);
  p.part_dB = reinterpret_cast<float*>(w + lay.off_B);
  p.part_dC = reinterpret_cast<float*>(w + lay.off_C);
  p.part_dA = reinterpret_cast<float*>(w + lay.off_A);
  p.part_dD = reinterpret_cast<float*>(w + lay.off_D);
  p.part_dbias = reinterpret_cast<float*>(w + lay.off_bias);
  p.chunk_carry = lay.gmax > 1 ? reinterpret_cast<float*>(w + lay.off_E) : nullptr;
  p.chunk_decay = lay.gmax > 1 ? reinterpret_cast<float*>(w + lay.off_P) : nullptr;
  p.group_carry = lay.gmax > 1 ? reinterpret_cast<float*>(w + lay.off_G) : nullptr;
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  cudaError_t e = ss::launch_bwd(p, static_cast<ss::DType>(dtype), vec, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_bwd: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

ss_status ss_bwd(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                 const void* u, const void* delta, const void* z, const float* A,
                 const void* B, const void* C, const float* D, const float* delta_bias,
                 int delta_softplus, const void* dy, const float* checkpoints,
                 void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC,
                 float* dD, float* ddelta_bias, void* workspace, size_t workspace_bytes,
                 void* stream) {
  return ss_bwd_with_state(batch, dim, dstate, seqlen, dtype, u, delta, z, A, B, C, D, delta_bias,
                           delta_softplus, nullptr, nullptr, dy, nullptr, checkpoints, du, ddelta, dz, dA, dB,
                           dC, dD, ddelta_bias, nullptr, workspace, workspace_bytes, stream);
}

ss_status ss_state_update(int64_t batch, int64_t dim, int64_t dstate, int dtype, float* state,
                          const void* u, const void* delta, const void* z, const float* A,
                          const void* B, const void* C, const float* D, const float* delta_bias,
                          int delta_softplus, void* y, void* stream) {
  ss_status st = check_sizes(batch, dim, dstate, 1, false);
  if (st != SS_OK) return st;
  if ((st = check_dtype(dtype)) != SS_OK) return st;
  if (!state || !u || !delta || !A || !B || !C || !y)
    return fail(SS_ERR_INVALID_ARG, "ss_state_update: state, u, delta, A, B, C and y are required");
  const size_t es = elt_size(dtype);
  for (const void* p : {u, delta, z, B, C, (const void*)y})
    if (p && !aligned(p, es)) return fail(SS_ERR_ALIGNMENT, "ss_state_update: data pointer %p not aligned", p);
  for (const void* p : {(const void*)A, (const void*)D, (const void*)delta_bias})
    if (p && !aligned(p, 4)) return fail(SS_ERR_ALIGNMENT, "ss_state_update: fp32 pointer %p not aligned", p);
  if (!aligned(state, 16)) return fail(SS_ERR_ALIGNMENT, "ss_state_update: state not 16-byte aligned");
  ss::UpdateParams p{};
  p.batch = (int)batch;
  p.dim = (int)dim;
  p.state = state;
  p.u = u; p.delta = delta; p.z = z; p.B = B; p.C = C;
  p.A = A; p.D = D; p.bias = delta_bias;
  p.softplus = delta_softplus ? 1 : 0;
  p.y = y;
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  cudaError_t e = ss::launch_state_update(p, static_cast<ss::DType>(dtype), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_state_update: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

static ss_status check_conv(const char* fn, int64_t batch, int64_t dim, int64_t seqlen, int64_t width,
                            int dtype, bool need_len) {
  if (batch <= 0 || dim <= 0 || (need_len && seqlen <= 0))
    return fail(SS_ERR_INVALID_ARG, "%s: batch, dim and seqlen must be positive", fn);
  if (width < 1 || width > 4)
    return fail(SS_ERR_UNSUPPORTED, "%s: width=%lld (supported: 1..4)", fn, (long long)width);
  if (batch > 65535LL * 65535LL || dim > (1LL << 26) || seqlen > (1LL << 30) ||
      batch * dim > (int64_t)INT32_MAX)
    return fail(SS_ERR_UNSUPPORTED, "%s: sizes beyond the supported range (batch*dim must fit in 31 bits)", fn);
  if (dtype != SS_F32 && dtype != SS_BF16 && dtype != SS_F16)
    return fail(SS_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, dtype);
  return SS_OK;
}

ss_status ss_conv1d_fwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t width, int dtype,
                        const void* x, const float* w, const float* bias, const float* state_in,
                        const int32_t* seq_idx, int silu, void* u, float* state_out, void* stream) {
  ss_status st = check_conv("ss_conv1d_fwd", batch, dim, seqlen, width, dtype, true);
  if (st != SS_OK) return st;
  if (!x || !w || !u) return fail(SS_ERR_INVALID_ARG, "ss_conv1d_fwd: x, w and u are required");
  const size_t es = elt_size(dtype);
  for (const void* p : {x, (const void*)u})
    if (!aligned(p, es)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_fwd: data pointer %p not aligned to %zu bytes", p, es);
  for (const void* p : {(const void*)w, (const void*)bias, (const void*)state_in, (const void*)state_out})
    if (p && !aligned(p, 4)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_fwd: fp32 pointer %p not 4-byte aligned", p);
  if (seq_idx && !aligned(seq_idx, 4)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_fwd: seq_idx not 4-byte aligned");
  ss::ConvParams p{};
  p.batch = (int)batch; p.dim = (int)dim; p.seqlen = (int)seqlen; p.width = (int)width;
  p.silu = silu ? 1 : 0;
  p.x = x; p.w = w; p.bias = bias; p.state_in = state_in; p.u = u; p.state_out = state_out;
  p.seq_idx = seq_idx;
  const bool vec = rows_vec_ok(seqlen, dtype, {x, (const void*)u});
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  cudaError_t e = ss::launch_conv(p, 0, static_cast<ss::DType>(dtype), vec, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_conv1d_fwd: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

size_t ss_conv1d_bwd_workspace_size(int64_t batch, int64_t dim, int64_t seqlen, int64_t width) {
  if (check_conv("ss_conv1d_bwd_workspace_size", batch, dim, seqlen, width, SS_F32, true) != SS_OK)
    return (size_t)-1;
  return round_up((size_t)batch * dim * (width + 1) * sizeof(float), 256);
}

ss_status ss_conv1d_bwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t width, int dtype,
                        const void* x, const float* w, const float* bias, const float* state_in,
                        const int32_t* seq_idx, int silu, const void* du, const float* dstate_out,
                        void* dx, float* dw,
                        float* dbias, float* dstate_in, void* workspace, size_t workspace_bytes,
                        void* stream) {
  ss_status st = check_conv("ss_conv1d_bwd", batch, dim, seqlen, width, dtype, true);
  if (st != SS_OK) return st;
  if (!x || !w || !du || !dx || !dw)
    return fail(SS_ERR_INVALID_ARG, "ss_conv1d_bwd: x, w, du, dx and dw are required");
  const size_t es = elt_size(dtype);
  for (const void* p : {x, du, (const void*)dx})
    if (!aligned(p, es)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_bwd: data pointer %p not aligned to %zu bytes", p, es);
  for (const void* p : {(const void*)w, (const void*)bias, (const void*)state_in, (const void*)dstate_out,
                        (const void*)dw, (const void*)dbias, (const void*)dstate_in})
    if (p && !aligned(p, 4)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_bwd: fp32 pointer %p not 4-byte aligned", p);
  if (seq_idx && !aligned(seq_idx, 4)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_bwd: seq_idx not 4-byte aligned");
  const size_t need = round_up((size_t)batch * dim * (width + 1) * sizeof(float), 256);
  if (!workspace || workspace_bytes < need)
    return fail(SS_ERR_WORKSPACE, "ss_conv1d_bwd: needs %zu workspace bytes, got %zu", need,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned(workspace, 16)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_bwd: workspace not 16-byte aligned");
  ss::ConvParams p{};
  p.batch = (int)batch; p.dim = (int)dim; p.seqlen = (int)seqlen; p.width = (int)width;
  p.silu = silu ? 1 : 0;
  p.x = x; p.w = w; p.bias = bias; p.state_in = state_in; p.seq_idx = seq_idx;
  p.du = du; p.dstate_out = dstate_out; p.dx = dx; p.dw = dw; p.dbias = dbias; p.dstate_in = dstate_in;
  p.part = static_cast<float*>(workspace);
  const bool vec = rows_vec_ok(seqlen, dtype, {x, du, (const void*)dx});
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  cudaError_t e = ss::launch_conv(p, 1, static_cast<ss::DType>(dtype), vec, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_conv1d_bwd: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

ss_status ss_ssd_fwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t ngroups,
                     int64_t dstate, int dtype, const void* x, const void* dt, const float* A,
                     const void* B, const void* C, const float* D, const void* z,
                     const float* dt_bias, int dt_softplus, const float* h0, void* y,
                     float* final_state, void* stream) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || ngroups <= 0)
    return fail(SS_ERR_INVALID_ARG, "ss_ssd_fwd: batch, seqlen, nheads and ngroups must be positive");
  if (nheads % ngroups)
    return fail(SS_ERR_INVALID_ARG, "ss_ssd_fwd: ngroups=%lld does not divide nheads=%lld",
                (long long)ngroups, (long long)nheads);
  if (headdim != 64 || (dstate != 64 && dstate != 128))
    return fail(SS_ERR_UNSUPPORTED, "ss_ssd_fwd: headdim=%lld dstate=%lld (supported: headdim 64, dstate 64 or 128)",
                (long long)headdim, (long long)dstate);
  if (dtype != SS_BF16 && dtype != SS_F16)
    return fail(SS_ERR_UNSUPPORTED, "ss_ssd_fwd: dtype %d (supported: bf16, fp16 storage)", dtype);
  if (batch > 65535 || nheads > 65535 || seqlen > (1LL << 30))
    return fail(SS_ERR_UNSUPPORTED, "ss_ssd_fwd: sizes beyond the supported range");
  if (!x || !dt || !A || !B || !C || !y)
    return fail(SS_ERR_INVALID_ARG, "ss_ssd_fwd: x, dt, A, B, C and y are required");
  for (const void* p : {x, B, C, z, (const void*)y, (const void*)h0, (const void*)final_state})
    if (p && !aligned(p, 16)) return fail(SS_ERR_ALIGNMENT, "ss_ssd_fwd: pointer %p not 16-byte aligned", p);
  if (!aligned(dt, 2)) return fail(SS_ERR_ALIGNMENT, "ss_ssd_fwd: dt not 2-byte aligned");
  for (const void* p : {(const void*)A, (const void*)D, (const void*)dt_bias})
    if (p && !aligned(p, 4)) return fail(SS_ERR_ALIGNMENT, "ss_ssd_fwd: fp32 pointer %p not 4-byte aligned", p);
  ss::SsdParams p{};
  p.batch = (int)batch; p.seqlen = (int)seqlen; p.nheads = (int)nheads; p.headdim = (int)headdim;
  p.ngroups = (int)ngroups; p.dstate = (int)dstate; p.softplus = dt_softplus ? 1 : 0;
  p.x = x; p.dt = dt; p.B = B; p.C = C; p.z = z; p.A = A; p.D = D; p.dt_bias = dt_bias;
  p.h0 = h0; p.y = y; p.final_state = final_state;
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  p.inject_timeout = std::getenv("SS_INJECT_WAIT_TIMEOUT") != nullptr;
  const char* var = std::getenv("SS_SSD_VARIANT");
  const bool mma = var && std::strcmp(var, "mma") == 0;
  cudaError_t e = mma ? ss::launch_ssd_fwd_mma(p, static_cast<ss::DType>(dtype), static_cast<cudaStream_t>(stream))
                      : ss::launch_ssd_fwd_tc(p, static_cast<ss::DType>(dtype), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_ssd_fwd: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

ss_status ss_segment_decay(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                           const void* delta, const float* A, const float* delta_bias, int delta_softplus,
                           float* P, void* stream) {
  if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0)
    return fail(SS_ERR_INVALID_ARG, "ss_segment_decay: batch, dim, dstate and seqlen must be positive");
  if (dstate > 256) return fail(SS_ERR_UNSUPPORTED, "ss_segment_decay: dstate %lld > 256", (long long)dstate);
  if (dtype != SS_F32 && dtype != SS_BF16 && dtype != SS_F16)
    return fail(SS_ERR_UNSUPPORTED, "ss_segment_decay: dtype %d", dtype);
  if (batch * dim > INT32_MAX || seqlen > INT32_MAX)
    return fail(SS_ERR_UNSUPPORTED, "ss_segment_decay: sizes beyond the supported range");
  if (!delta || !A || !P) return fail(SS_ERR_INVALID_ARG, "ss_segment_decay: delta, A and P are required");
  if (!aligned(delta, elt_size(dtype)) || !aligned(A, 4) || !aligned(P, 4) || (delta_bias && !aligned(delta_bias, 4)))
    return fail(SS_ERR_ALIGNMENT, "ss_segment_decay: misaligned pointer");
  ss::SegmentDecayParams p{};
  p.batch = (int)batch; p.dim = (int)dim; p.dstate = (int)dstate; p.seqlen = (int)seqlen;
  p.softplus = delta_softplus ? 1 : 0; p.delta = delta; p.A = A; p.delta_bias = delta_bias; p.P = P;
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  cudaError_t e = ss::launch_segment_decay(p, static_cast<ss::DType>(dtype), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_segment_decay: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

ss_status ss_state_chain(int64_t count, int64_t nseg, const float* P, const float* E, const float* init,
                         int reverse, float* out, void* stream) {
  if (count <= 0 || nseg <= 0)
    return fail(SS_ERR_INVALID_ARG, "ss_state_chain: count and nseg must be positive");
  if (nseg > 65536 || count > (int64_t(1) << 38))  // grid: count / 256 blocks < 2^31
    return fail(SS_ERR_UNSUPPORTED, "ss_state_chain: sizes beyond the supported range");
  if (!P || !E || !out) return fail(SS_ERR_INVALID_ARG, "ss_state_chain: P, E and out are required");
  for (const void* q : {(const void*)P, (const void*)E, (const void*)init, (const void*)out})
    if (q && !aligned(q, 4)) return fail(SS_ERR_ALIGNMENT, "ss_state_chain: pointer %p not 4-byte aligned", q);
  ss::StateChainParams p{};
  p.count = count; p.nseg = (int)nseg; p.reverse = reverse ? 1 : 0;
  p.P = P; p.E = E; p.init = init; p.out = out;
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  cudaError_t e = ss::launch_state_chain(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_state_chain: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

int ss_ssd_fwd_path(void) {
  const char* var = std::getenv("SS_SSD_VARIANT");
  return var && std::strcmp(var, "mma") == 0 ? SS_SSD_PATH_MMA : SS_SSD_PATH_TCGEN05;
}

int ss_device_fault(int clear) {
  unsigned bits = 0;
  const cudaError_t e = ss::read_tc_fault(&bits, clear != 0);
  if (e != cudaSuccess) {
    fail(SS_ERR_CUDA, "ss_device_fault: %s", cudaGetErrorString(e));
    return -1;
  }
  return static_cast<int>(bits);
}

static ss_status check_ssd(const char* fn, int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                           int64_t ngroups, int64_t dstate, int dtype) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || ngroups <= 0)
    return fail(SS_ERR_INVALID_ARG, "%s: batch, seqlen, nheads and ngroups must be positive", fn);
  if (nheads % ngroups)
    return fail(SS_ERR_INVALID_ARG, "%s: ngroups=%lld does not divide nheads=%lld", fn, (long long)ngroups,
                (long long)nheads);
  if (headdim != 64 || (dstate != 64 && dstate != 128))
    return fail(SS_ERR_UNSUPPORTED, "%s: headdim=%lld dstate=%lld (supported: headdim 64, dstate 64 or 128)", fn,
                (long long)headdim, (long long)dstate);
  if (dtype != SS_BF16 && dtype != SS_F16)
    return fail(SS_ERR_UNSUPPORTED, "%s: dtype %d (supported: bf16, fp16 storage)", fn, dtype);
  if (batch > 65535 || nheads > 65535 || seqlen > (1LL << 30))
    return fail(SS_ERR_UNSUPPORTED, "%s: sizes beyond the supported range", fn);
  return SS_OK;
}

size_t ss_ssd_bwd_workspace_size(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                                 int64_t ngroups, int64_t dstate) {
  if (check_ssd("ss_ssd_bwd_workspace_size", batch, seqlen, nheads, headdim, ngroups, dstate, SS_BF16) != SS_OK)
    return (size_t)-1;
  return ss::ssd_bwd_layout(batch, seqlen, nheads, headdim, dstate).total;
}

ss_status ss_ssd_bwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t ngroups,
                     int64_t dstate, int dtype, const void* x, const void* dt, const float* A,
                     const void* B, const void* C, const float* D, const void* z,
                     const float* dt_bias, int dt_softplus, const float* h0, const void* dy,
                     const float* dfinal, void* dx, void* ddt, float* dA, float* dB, float* dC,
                     float* dD, void* dz, float* ddt_bias, float* dh0, void* workspace,
                     size_t workspace_bytes, void* stream) {
  ss_status st = check_ssd("ss_ssd_bwd", batch, seqlen, nheads, headdim, ngroups, dstate, dtype);
  if (st != SS_OK) return st;
  if (!x || !dt || !A || !B || !C || !dy || !dx || !ddt || !dA || !dB || !dC)
    return fail(SS_ERR_INVALID_ARG, "ss_ssd_bwd: x, dt, A, B, C, dy, dx, ddt, dA, dB and dC are required");
  if (dz && !z) return fail(SS_ERR_INVALID_ARG, "ss_ssd_bwd: dz given without z");
  for (const void* p : {x, B, C, z, dy, (const void*)dx, (const void*)dz, (const void*)h0, (const void*)dfinal,
                        (const void*)dh0})
    if (p && !aligned(p, 16)) return fail(SS_ERR_ALIGNMENT, "ss_ssd_bwd: pointer %p not 16-byte aligned", p);
  for (const void* p : {dt, (const void*)ddt})
    if (!aligned(p, 2)) return fail(SS_ERR_ALIGNMENT, "ss_ssd_bwd: dt/ddt pointer %p not 2-byte aligned", p);
  for (const void* p : {(const void*)A, (const void*)D, (const void*)dt_bias, (const void*)dA, (const void*)dB,
                        (const void*)dC, (const void*)dD, (const void*)ddt_bias})
    if (p && !aligned(p, 4)) return fail(SS_ERR_ALIGNMENT, "ss_ssd_bwd: fp32 pointer %p not 4-byte aligned", p);
  const ss::SsdBwdLayout lay = ss::ssd_bwd_layout(batch, seqlen, nheads, headdim, dstate);
  if (!workspace || workspace_bytes < lay.total)
    return fail(SS_ERR_WORKSPACE, "ss_ssd_bwd: needs %zu workspace bytes, got %zu", lay.total,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned(workspace, 256)) return fail(SS_ERR_ALIGNMENT, "ss_ssd_bwd: workspace not 256-byte aligned");
  ss::SsdBwdParams p{};
  p.batch = (int)batch; p.seqlen = (int)seqlen; p.nheads = (int)nheads; p.headdim = (int)headdim;
  p.ngroups = (int)ngroups; p.dstate = (int)dstate; p.softplus = dt_softplus ? 1 : 0;
  p.nchunk = (int)((seqlen + 63) / 64);
  p.x = x; p.dt = dt; p.B = B; p.C = C; p.z = z; p.dy = dy;
  p.A = A; p.D = D; p.dt_bias = dt_bias; p.h0 = h0; p.dfinal = dfinal;
  p.dx = dx; p.ddt = ddt; p.dz = dz;
  p.dA = dA; p.dB = dB; p.dC = dC; p.dD = dD; p.ddt_bias = ddt_bias; p.dh0 = dh0;
  ss::ssd_bwd_bind(p, workspace);
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  const char* var = std::getenv("SS_SSD_VARIANT");
  const bool mma = var && std::strcmp(var, "mma") == 0;
  p.hpc = 1;
  if (!mma) {
    int sms = 0;
    if (current_sm_count(&sms) != 0) return fail(SS_ERR_CUDA, "ss_ssd_bwd: cannot query the device");
    // SS_SSD_HEADS_PER_CTA (tests, tuning): "max", or a number, forces the
    // largest divisor up to it (capped at 8) whatever the grid
    const char* hv = std::getenv("SS_SSD_HEADS_PER_CTA");
    const int cap = !hv ? 8 : std::strcmp(hv, "max") == 0 ? 8 : std::atoi(hv);
    p.hpc = ss::ssd_heads_per_cta(p.batch, p.nchunk, p.nheads, p.ngroups, sms, cap, hv != nullptr);
  }
  cudaError_t e = ss::launch_ssd_bwd(p, static_cast<ss::DType>(dtype), !mma, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_ssd_bwd: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

ss_status ss_conv1d_step(int64_t batch, int64_t dim, int64_t width, int dtype, float* state,
                         const void* x, const float* w, const float* bias, int silu, void* u,
                         void* stream) {
  ss_status st = check_conv("ss_conv1d_step", batch, dim, 1, width, dtype, false);
  if (st != SS_OK) return st;
  if ((!state && width > 1) || !x || !w || !u)
    return fail(SS_ERR_INVALID_ARG, "ss_conv1d_step: state, x, w and u are required");
  const size_t es = elt_size(dtype);
  for (const void* p : {x, (const void*)u})
    if (!aligned(p, es)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_step: data pointer %p not aligned to %zu bytes", p, es);
  for (const void* p : {(const void*)state, (const void*)w, (const void*)bias})
    if (p && !aligned(p, 4)) return fail(SS_ERR_ALIGNMENT, "ss_conv1d_step: fp32 pointer %p not 4-byte aligned", p);
  ss::ConvParams p{};
  p.batch = (int)batch; p.dim = (int)dim; p.seqlen = 1; p.width = (int)width;
  p.silu = silu ? 1 : 0;
  p.x = x; p.w = w; p.bias = bias; p.u = u; p.state_out = state;
  if (launch_injected())
    return fail(SS_ERR_CUDA, "%s: launch failure injected by SS_FAIL_LAUNCH (nothing enqueued)", __func__);
  cudaError_t e = ss::launch_conv(p, 2, static_cast<ss::DType>(dtype), false, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SS_ERR_CUDA, "ss_conv1d_step: launch failed: %s", cudaGetErrorString(e));
  return SS_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// ss_fwd_noalloc: ss_fwd with its scratch in a file-scope device array, for
// callers that cannot allocate.  The array lives in every device's copy of
// this module; host code only sees a stand-in for its name, so its device
// address is looked up on every call, with the caller's device current, and
// passed to ss_fwd as the workspace.  The lookup allocates nothing, and a fresh
// lookup stays right after a device reset or on another context.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_fwd_noalloc_scratch[SS_FWD_NOALLOC_SCRATCH_BYTES];

}  // namespace

extern "C" ss_status ss_fwd_noalloc(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                    int dtype, const void* u, const void* delta, const void* z,
                                    const float* A, const void* B, const void* C, const float* D,
                                    const float* delta_bias, int delta_softplus, void* y,
                                    float* final_state, float* checkpoints, void* stream) {
  const size_t need = ss_fwd_workspace_size(batch, dim, dstate, seqlen);
  if (need == (size_t)-1) {
    const ss_status st = check_sizes(batch, dim, dstate, seqlen, true);
    return st != SS_OK ? st : fail(SS_ERR_CUDA, "ss_fwd_noalloc: cannot query the device");
  }
  if (need > SS_FWD_NOALLOC_SCRATCH_BYTES)
    return fail(SS_ERR_WORKSPACE,
                "ss_fwd_noalloc: this problem needs %zu bytes of scratch; the built-in area holds %u "
                "(use ss_fwd with a caller-provided workspace)",
                need, (unsigned)SS_FWD_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = cudaGetSymbolAddress(&scratch, g_fwd_noalloc_scratch);
    if (e != cudaSuccess)
      return fail(SS_ERR_CUDA, "ss_fwd_noalloc: scratch address lookup failed: %s", cudaGetErrorString(e));
  }
  return ss_fwd(batch, dim, dstate, seqlen, dtype, u, delta, z, A, B, C, D, delta_bias, delta_softplus, y,
                final_state, checkpoints, scratch, need > 0 ? (size_t)SS_FWD_NOALLOC_SCRATCH_BYTES : 0, stream);
}

