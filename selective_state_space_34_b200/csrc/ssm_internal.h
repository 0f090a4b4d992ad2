// ssm_internal.h -- launch parameters and launcher declarations shared by the kernel files and
// the C-ABI layer. Host/device plain data only; no torch types anywhere in the library.
#pragma once

#include <cuda.h>  // CUtensorMap

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ssm_scan.h"

namespace ssm {

constexpr int kThreads = 128;  // threads per CTA for the scan kernels
constexpr int kT = 32;         // time steps staged per CTA pipeline stage
constexpr int kSub = 16;       // recompute / state-save block (SSM_STATE_CHUNK)
constexpr int kPre = 8;        // conv halo prefix kept in front of each staged x row
constexpr int kMaxThreadsPerSM = 2048;  // resident threads per SM on sm_100

// Lane layout of the scan kernels: a channel's N states are spread over G adjacent lanes of one
// warp, NS states per lane (G * NS >= N, padded states are inert).
struct LaneLayout {
  int G;
  int NS;
};

struct FwdParams {
  const void *x, *dt, *z, *B, *C;
  const float *dt_bias, *A_log, *D, *conv_w, *conv_b;
  void *out, *u_out;
  float *chunk_states;
  int64_t Bt, Dn, N, L, n_ck;
  int K;
  int delta_softplus;
  int vec;  // 1: rows are 16-byte aligned, stage with cp.async and store with vector stores
  int euler;  // input discretisation: 0 exact ZOH, 1 Delta * B
  int chunked;  // one-pass scan layout: 0 states over lanes (ssm_fwd.cu), 1 chunked in time (ssm_fwd_tp.cu)
  int tma;      // set by the launcher: stage x, dt, z with TMA boxes (the kernel's tensor maps are valid)
  const float *h0;        // (Bt, Dn, N) or null
  const void *conv_hist;  // (Bt, Dn, K-1) in-dtype or null
  float *h_last;          // (Bt, Dn, N) or null
  void *conv_hist_out;    // (Bt, Dn, K-1) in-dtype or null
  // split-L: the sequence runs as n_seg segments of seg_len steps (n_seg = 1, seg_len = L: one pass)
  int64_t seg_len;
  int n_seg;
  const float *seg_h0;    // (n_seg, Bt, Dn, N): start state of every segment (pass 3), or null
  float *seg_hend;        // (n_seg, Bt, Dn, N): end state from a zero start (pass 1)
  float *seg_sdl;         // (n_seg, Bt, Dn): sum of Delta over the segment (pass 1)
};

// Mamba-2 state-space duality forward (ssm_ssd.cu).
struct SsdParams {
  const void *x, *dt, *B, *C;  // bf16: x (Bt, H, L, P), dt (Bt, H, L), B / C (Bt, L, N)
  const float *dt_bias, *A_log, *D;  // [H]
  const float *h0;             // (Bt, H, N, P) or null
  void *y;                     // (Bt, H, L, P), bf16 or fp32
  float *h_last;               // (Bt, H, N, P) or null
  int64_t Bt, H, L, P, N;
  int delta_softplus, euler;
  float *S;                    // workspace: chunk states (Bt, H, n_chunks, N, P) fp32
  __nv_bfloat16 *Hin;          // workspace: state entering each chunk, same shape, bf16
  float *cum_end;              // workspace: log-decay of each chunk (Bt, H, n_chunks)
  int *error;                  // workspace: set to 1 if a tensor-core wait timed out
  void *const *timing_events;  // optional: 2 cudaEvent_t around the output (or the fused) kernel
  int form;                    // ssm_ssd_form
};
cudaError_t launch_ssd(const SsdParams &p, int out_bf16, cudaStream_t stream);
// A tensor map for TMA tile loads of a 3-D (d0 innermost, d1, d2) row-major bf16 or fp32 tensor, in
// boxes of box0 x box1 x 1 elements with zero fill out of bounds (ssm_tma.cu); false when the driver
// declines it.
bool encode_tma_3d(CUtensorMap *m, bool bf16, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                   uint32_t box0, uint32_t box1);
// The fused one-launch form (ssm_ssd_fused.cu): P = 64, N = 64 or 128.
bool ssd_fused_supported(const SsdParams &p);
cudaError_t launch_ssd_fused(const SsdParams &p, int out_bf16, cudaStream_t stream);
size_t ssd_workspace_bytes(int64_t Bt, int64_t H, int64_t L, int64_t P, int64_t N);
// Byte offset of the SSD error word inside the workspace (its last 256-byte block).
size_t ssd_error_offset(int64_t Bt, int64_t H, int64_t L, int64_t P, int64_t N);
// One CTA waiting, with a bound of `polls`, on an mbarrier that gets one arrival iff `arrive`.
cudaError_t launch_wait_selftest(int arrive, int polls, int *error, cudaStream_t stream);

// Segmentation of a split-L forward: how many segments of which length, and the scratch it needs.
struct SegPlan {
  int n_seg;
  int64_t seg_len;
  size_t workspace_bytes;
};
// requested: 0/1 one pass, >= 2 up to that many segments, -1 chosen from sm_count and the shape.
SegPlan plan_segments(int64_t Bt, int64_t Dn, int64_t N, int64_t L, int requested, int sm_count);

struct StepParams {
  const void *x, *dt, *B, *C, *z;
  const float *dt_bias, *A_log, *D, *conv_w, *conv_b;
  float *h;
  void *conv_hist, *out;
  int64_t Bt, Dn, N;
  int K, delta_softplus, euler;
};

struct BwdParams {
  FwdParams f;
  const void *dout;
  const float *chunk_states;
  float *dx, *ddt, *dz, *dB, *dC;
  // per-(b, d) partial sums of the per-channel parameter gradients, reduced over b afterwards
  float *p_dA_log;   // (Bt, Dn, N)
  float *p_dD;       // (Bt, Dn)
  float *p_ddt_bias; // (Bt, Dn)
  float *p_dconv_w;  // (Bt, Dn, 4)
  float *p_dconv_b;  // (Bt, Dn)
  // per-tile partial sums of dB / dC: (n_ptiles, Bt, N, L) each; a tile is one channel tile, or
  // the `cluster` consecutive channel tiles of a thread-block cluster whose CTAs add their sums
  float *p_dB, *p_dC;
  int64_t n_dtiles;
  int64_t n_ptiles;
  int cluster;
  float *dA_log, *dD, *ddt_bias, *dconv_w, *dconv_b;
  void *const *timing_events;  // optional: 2 cudaEvent_t around the main backward kernel
  const float *dh_last;        // (Bt, Dn, N) or null
  float *dh0;                  // (Bt, Dn, N) or null
  float *dconv_hist;           // (Bt, Dn, K-1) or null
  // split-L (f stays a one-pass forward for the state recompute): n_seg segments of seg_len steps;
  // the per-(b, d) parameter partials above then hold n_seg * Bt rows
  int n_seg;
  int64_t seg_len;
  float *seg_G;                // (n_seg, Bt, Dn, N): gradient arriving at each segment's last state
  float *seg_gloc;             // (n_seg, Bt, Dn, N): A_bar_ts lambda_ts from a zero arrival (pass 1)
  float *seg_sdl;              // (n_seg, Bt, Dn): sum of Delta over each segment (pass 1)
  float *seg_dxh;              // (n_seg, Bt, Dn, 4): each segment's gradient w.r.t. the K-1 inputs
                               // before it, added into the previous segment's dx afterwards
};

// Maps a CUDA error to the C ABI's status and records it for ssm_last_cuda_error() on this host
// thread (SSM_OK for cudaSuccess). The status type is the ABI's, passed as int here.
int record_cuda_error_code(cudaError_t e);

LaneLayout choose_layout(int64_t N, int64_t channels);
int channels_per_cta(const LaneLayout &lay);

cudaError_t launch_fwd(const FwdParams &p, int in_bf16, int out_bf16, cudaStream_t stream);
// The time-parallel forward (ssm_fwd_tp.cu): one pass, the same outputs as launch_fwd.
cudaError_t launch_fwd_tp(const FwdParams &p, int in_bf16, int out_bf16, cudaStream_t stream);
cudaError_t launch_bwd(const BwdParams &p, int in_bf16, cudaStream_t stream);
// Backward scratch for a cluster size of at most max_cluster (see bwd_cluster).
size_t bwd_workspace_bytes(int64_t Bt, int64_t Dn, int64_t N, int64_t L, int need_states, int n_seg,
                           int max_cluster);
// CTAs per thread-block cluster of the backward, at most max_cluster: the CTAs of a cluster (4 or 8
// consecutive channel tiles) add their dB / dC stage sums through distributed shared memory before
// writing them, which divides the per-tile partials (scratch and traffic) by the cluster size at
// the price of one cluster barrier per stage (measured 6% slower on 4x4096x16x4096). 1 when the
// layout (4 lanes x 4 states) or the tile count does not allow max_cluster.
int bwd_cluster(const LaneLayout &lay, int64_t n_dtiles, int max_cluster);
// ssm_scan_bwd with clusters of up to max_cluster CTAs (ssm_scan_bwd itself uses 1), and the
// scratch it needs (ssm_bwd_workspace_size for max_cluster = 1).
ssm_status scan_bwd_clustered(const ssm_bwd_args *args, void *stream, int max_cluster);
size_t bwd_workspace_for(const ssm_bwd_args *args, int max_cluster);
cudaError_t launch_step(const StepParams &p, int in_bf16, int out_bf16, cudaStream_t stream);
cudaError_t launch_conv1d_silu(const void *x, void *u, const float *w, const float *b, int64_t Bt,
                               int64_t Dn, int64_t L, int K, int in_bf16, int out_bf16, int vec,
                               cudaStream_t stream);

}  // namespace ssm
