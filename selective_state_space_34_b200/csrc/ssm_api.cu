// ssm_api.cu -- the extern "C" boundary declared in include/ssm_scan.h: host-side validation
// (synchronous, before any launch), workspace carving, and dispatch to the kernel launchers. No
// exception crosses the ABI and these entry points allocate no device memory (scratch comes from
// the caller's workspace; ssm_noalloc.cu is the one entry point with a library-owned array).
#include <stdint.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "../../include/ssm_scan.h"
#include "ssm_internal.h"

namespace {

// An NVTX range named after the entry point around its host work and launches, so a profiler's
// timeline groups each call's kernels under the API call that issued them. Header-only NVTX v3:
// without an attached tool a push or pop is one predictable branch.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
#define SSM_RANGE(name) NvtxRange ssm_nvtx_range_(name)

thread_local int g_last_cuda_error = 0;

ssm_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SSM_OK;
  g_last_cuda_error = (int)e;
  return SSM_ERR_CUDA;
}

}  // namespace

namespace ssm {
int record_cuda_error_code(cudaError_t e) { return (int)cuda_status(e); }
}  // namespace ssm

namespace {

size_t dtype_size(int32_t dt) { return dt == SSM_BF16 ? 2 : 4; }
bool dtype_ok(int32_t dt) { return dt == SSM_F32 || dt == SSM_BF16; }
bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool mul_ok(int64_t a, int64_t b, int64_t *out) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > INT64_MAX / a) return false;
  *out = a * b;
  return true;
}

// Shape, dtype and pointer checks shared by forward and backward. Sets *empty for Bt = 0 or L = 0.
ssm_status check_fwd(const ssm_fwd_args *a, bool need_out, bool *empty) {
  if (!a) return SSM_ERR_NULL;
  if (!dtype_ok(a->in_dtype) || !dtype_ok(a->out_dtype)) return SSM_ERR_DTYPE;
  if (a->discretization != SSM_ZOH && a->discretization != SSM_EULER) return SSM_ERR_UNSUPPORTED;
  if (a->scan_form != SSM_SCAN_LANES && a->scan_form != SSM_SCAN_CHUNKED) return SSM_ERR_UNSUPPORTED;
  if (a->Bt < 0 || a->Dn < 0 || a->N < 0 || a->L < 0) return SSM_ERR_SHAPE;
  if (a->Dn == 0 || a->N == 0) return SSM_ERR_SHAPE;  // empty internal axes are rejected
  if (a->conv_w && a->K <= 0) return SSM_ERR_SHAPE;
  if (a->N > 64) return SSM_ERR_UNSUPPORTED;
  if (a->conv_w && a->K > 4) return SSM_ERR_UNSUPPORTED;
  int64_t rows, elems, bc;
  if (!mul_ok(a->Bt, a->Dn, &rows) || !mul_ok(rows, a->L, &elems) || !mul_ok(a->Bt, a->N, &bc) ||
      !mul_ok(bc, a->L, &bc) || elems > (INT64_C(1) << 50))
    return SSM_ERR_SHAPE;
  *empty = (a->Bt == 0 || a->L == 0);
  if (*empty) return SSM_OK;
  if (!a->x || !a->dt || !a->A_log || !a->B || !a->C || (need_out && !a->out)) return SSM_ERR_NULL;
  const size_t ei = dtype_size(a->in_dtype), eo = dtype_size(a->out_dtype);
  const void *in_ptrs[5] = {a->x, a->dt, a->z, a->B, a->C};
  for (const void *p : in_ptrs)
    if (p && !aligned(p, ei)) return SSM_ERR_ALIGN;
  if ((a->out && !aligned(a->out, eo)) || (a->u_out && !aligned(a->u_out, eo))) return SSM_ERR_ALIGN;
  const void *f32_ptrs[8] = {a->dt_bias, a->A_log, a->D, a->conv_w, a->conv_b, a->chunk_states,
                             a->h0, a->h_last};
  for (const void *p : f32_ptrs)
    if (p && !aligned(p, 4)) return SSM_ERR_ALIGN;
  if ((a->conv_hist && !aligned(a->conv_hist, ei)) || (a->conv_hist_out && !aligned(a->conv_hist_out, ei)))
    return SSM_ERR_ALIGN;
  return SSM_OK;
}

// An empty chunk keeps the carried state ("Selective Mamba", runArray): copy it through.
cudaError_t carry_through_empty(const ssm_fwd_args *a, cudaStream_t s) {
  if (a->Bt <= 0) return cudaSuccess;
  const size_t nh = sizeof(float) * (size_t)(a->Bt * a->Dn * a->N);
  cudaError_t e = cudaSuccess;
  if (a->h_last) {
    e = a->h0 ? (a->h0 == a->h_last ? cudaSuccess : cudaMemcpyAsync(a->h_last, a->h0, nh, cudaMemcpyDeviceToDevice, s))
              : cudaMemsetAsync(a->h_last, 0, nh, s);
    if (e != cudaSuccess) return e;
  }
  if (a->conv_w && a->K > 1 && a->conv_hist_out) {
    const size_t nc = dtype_size(a->in_dtype) * (size_t)(a->Bt * a->Dn * (a->K - 1));
    e = a->conv_hist ? (a->conv_hist == a->conv_hist_out ? cudaSuccess
                                                         : cudaMemcpyAsync(a->conv_hist_out, a->conv_hist, nc, cudaMemcpyDeviceToDevice, s))
                     : cudaMemsetAsync(a->conv_hist_out, 0, nc, s);
  }
  return e;
}

// 16-byte staging / vector stores are allowed when every row starts on a 16-byte boundary.
int vec_ok(const ssm_fwd_args *a, const void *const *extra, int n_extra) {
  if (a->L % 8 != 0) return 0;
  const void *ptrs[7] = {a->x, a->dt, a->z, a->B, a->C, a->out, a->u_out};
  for (const void *p : ptrs)
    if (p && !aligned(p, 16)) return 0;
  for (int i = 0; i < n_extra; i++)
    if (extra[i] && !aligned(extra[i], 16)) return 0;
  return 1;
}

ssm::FwdParams make_fwd_params(const ssm_fwd_args *a, int vec) {
  ssm::FwdParams p;
  memset(&p, 0, sizeof(p));
  p.x = a->x;
  p.dt = a->dt;
  p.z = a->z;
  p.B = a->B;
  p.C = a->C;
  p.dt_bias = a->dt_bias;
  p.A_log = a->A_log;
  p.D = a->D;
  p.conv_w = a->conv_w;
  p.conv_b = a->conv_w ? a->conv_b : nullptr;
  p.out = a->out;
  p.u_out = a->u_out;
  p.chunk_states = a->chunk_states;
  p.Bt = a->Bt;
  p.Dn = a->Dn;
  p.N = a->N;
  p.L = a->L;
  p.n_ck = ssm_num_state_chunks(a->L);
  p.K = a->conv_w ? a->K : 0;
  p.delta_softplus = a->delta_softplus ? 1 : 0;
  p.vec = vec;
  p.euler = a->discretization == SSM_EULER ? 1 : 0;
  p.chunked = a->scan_form == SSM_SCAN_CHUNKED ? 1 : 0;
  p.h0 = a->h0;
  p.conv_hist = a->conv_w ? a->conv_hist : nullptr;
  p.h_last = a->h_last;
  p.conv_hist_out = a->conv_w ? a->conv_hist_out : nullptr;
  p.n_seg = 1;  // one pass unless ssm_scan_fwd plans a split
  p.seg_len = a->L;
  return p;
}

int sm_count_or_zero() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// The split-L plan of a forward call (one pass when n_segments asks for none or the device's
// SM count cannot be read for an automatic choice).
ssm::SegPlan fwd_plan(const ssm_fwd_args *a) {
  const int sms = a->n_segments < 0 ? sm_count_or_zero() : 0;
  if (a->n_segments < 0 && sms <= 0) return ssm::SegPlan{1, a->L, 0};
  return ssm::plan_segments(a->Bt, a->Dn, a->N, a->L, a->n_segments, sms);
}

}  // namespace

extern "C" {

int64_t ssm_num_state_chunks(int64_t L) {
  return L <= 0 ? 0 : (L + SSM_STATE_CHUNK - 1) / SSM_STATE_CHUNK;
}

const char *ssm_status_string(ssm_status s) {
  switch (s) {
    case SSM_OK: return "SSM_OK: success";
    case SSM_ERR_NULL: return "SSM_ERR_NULL: a required pointer is NULL";
    case SSM_ERR_SHAPE: return "SSM_ERR_SHAPE: negative size, empty internal axis or size overflow";
    case SSM_ERR_ALIGN: return "SSM_ERR_ALIGN: a pointer is not aligned to its element type";
    case SSM_ERR_DTYPE: return "SSM_ERR_DTYPE: unknown dtype code";
    case SSM_ERR_UNSUPPORTED: return "SSM_ERR_UNSUPPORTED: d_state > 64 or conv taps > 4";
    case SSM_ERR_CUDA: return "SSM_ERR_CUDA: a CUDA call or launch failed";
    case SSM_ERR_WORKSPACE: return "SSM_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case SSM_ERR_TIMEOUT: return "SSM_ERR_TIMEOUT: a bounded device wait ran out";
  }
  return "unknown ssm_status";
}

int ssm_last_cuda_error(void) { return g_last_cuda_error; }

ssm_status ssm_scan_fwd(const ssm_fwd_args *args, void *stream) {
  SSM_RANGE("ssm_scan_fwd");
  bool empty = false;
  ssm_status st = check_fwd(args, true, &empty);
  if (st != SSM_OK) return st;
  if (args->n_segments < -1) return SSM_ERR_SHAPE;
  if (empty) return cuda_status(carry_through_empty(args, static_cast<cudaStream_t>(stream)));
  ssm::FwdParams p = make_fwd_params(args, vec_ok(args, nullptr, 0));
  const ssm::SegPlan plan = fwd_plan(args);
  if (plan.n_seg > 1) {
    if (!args->workspace || args->workspace_bytes < plan.workspace_bytes ||
        (reinterpret_cast<uintptr_t>(args->workspace) & 255))
      return SSM_ERR_WORKSPACE;
    auto rnd = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t bdn = (size_t)plan.n_seg * args->Bt * args->Dn * args->N;
    char *w = static_cast<char *>(args->workspace);
    p.n_seg = plan.n_seg;
    p.seg_len = plan.seg_len;
    p.seg_hend = reinterpret_cast<float *>(w);
    p.seg_h0 = reinterpret_cast<float *>(w + rnd(sizeof(float) * bdn));
    p.seg_sdl = reinterpret_cast<float *>(w + 2 * rnd(sizeof(float) * bdn));
  }
  return cuda_status(ssm::launch_fwd(p, args->in_dtype == SSM_BF16, args->out_dtype == SSM_BF16,
                                     static_cast<cudaStream_t>(stream)));
}

size_t ssm_fwd_workspace_size(const ssm_fwd_args *args) {
  bool empty = false;
  if (check_fwd(args, false, &empty) != SSM_OK || empty || args->n_segments < -1) return 0;
  return fwd_plan(args).workspace_bytes;
}

ssm_status ssm_conv1d_silu(const void *x, void *u, const float *w, const float *b, int64_t Bt,
                           int64_t Dn, int64_t L, int32_t K, int32_t in_dtype, int32_t out_dtype,
                           void *stream) {
  SSM_RANGE("ssm_conv1d_silu");
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return SSM_ERR_DTYPE;
  if (Bt < 0 || Dn < 0 || L < 0) return SSM_ERR_SHAPE;
  if (Dn == 0 || K <= 0) return SSM_ERR_SHAPE;
  if (K > 4) return SSM_ERR_UNSUPPORTED;
  int64_t rows, elems;
  if (!mul_ok(Bt, Dn, &rows) || !mul_ok(rows, L, &elems) || elems > (INT64_C(1) << 50))
    return SSM_ERR_SHAPE;
  if (Bt == 0 || L == 0) return SSM_OK;
  if (!x || !u || !w) return SSM_ERR_NULL;
  if (!aligned(x, dtype_size(in_dtype)) || !aligned(u, dtype_size(out_dtype)) || !aligned(w, 4) ||
      (b && !aligned(b, 4)))
    return SSM_ERR_ALIGN;
  return cuda_status(ssm::launch_conv1d_silu(x, u, w, b, Bt, Dn, L, K, in_dtype == SSM_BF16,
                                             out_dtype == SSM_BF16, 0,
                                             static_cast<cudaStream_t>(stream)));
}

ssm_status ssm_scan_step(const ssm_step_args *a, void *stream) {
  SSM_RANGE("ssm_scan_step");
  if (!a) return SSM_ERR_NULL;
  if (!dtype_ok(a->in_dtype) || !dtype_ok(a->out_dtype)) return SSM_ERR_DTYPE;
  if (a->discretization != SSM_ZOH && a->discretization != SSM_EULER) return SSM_ERR_UNSUPPORTED;
  if (a->Bt < 0 || a->Dn <= 0 || a->N <= 0) return SSM_ERR_SHAPE;
  if (a->conv_w && a->K <= 0) return SSM_ERR_SHAPE;
  if (a->N > 64 || (a->conv_w && a->K > 4)) return SSM_ERR_UNSUPPORTED;
  int64_t rows;
  if (!mul_ok(a->Bt, a->Dn, &rows) || rows > (INT64_C(1) << 40)) return SSM_ERR_SHAPE;
  if (a->Bt == 0) return SSM_OK;
  if (!a->x || !a->dt || !a->A_log || !a->B || !a->C || !a->h || !a->out) return SSM_ERR_NULL;
  if (a->conv_w && a->K > 1 && !a->conv_hist) return SSM_ERR_NULL;
  const size_t ei = dtype_size(a->in_dtype), eo = dtype_size(a->out_dtype);
  const void *in_ptrs[6] = {a->x, a->dt, a->z, a->B, a->C, a->conv_hist};
  for (const void *p : in_ptrs)
    if (p && !aligned(p, ei)) return SSM_ERR_ALIGN;
  if (!aligned(a->out, eo)) return SSM_ERR_ALIGN;
  const void *f32_ptrs[7] = {a->dt_bias, a->A_log, a->D, a->conv_w, a->conv_b, a->h, nullptr};
  for (const void *p : f32_ptrs)
    if (p && !aligned(p, 4)) return SSM_ERR_ALIGN;
  ssm::StepParams p;
  memset(&p, 0, sizeof(p));
  p.x = a->x;
  p.dt = a->dt;
  p.B = a->B;
  p.C = a->C;
  p.z = a->z;
  p.dt_bias = a->dt_bias;
  p.A_log = a->A_log;
  p.D = a->D;
  p.conv_w = a->conv_w;
  p.conv_b = a->conv_w ? a->conv_b : nullptr;
  p.h = a->h;
  p.conv_hist = a->conv_w ? a->conv_hist : nullptr;
  p.out = a->out;
  p.Bt = a->Bt;
  p.Dn = a->Dn;
  p.N = a->N;
  p.K = a->conv_w ? a->K : 0;
  p.delta_softplus = a->delta_softplus ? 1 : 0;
  p.euler = a->discretization == SSM_EULER ? 1 : 0;
  return cuda_status(ssm::launch_step(p, a->in_dtype == SSM_BF16, a->out_dtype == SSM_BF16,
                                      static_cast<cudaStream_t>(stream)));
}

size_t ssm_workspace_size(const ssm_fwd_args *args, int32_t for_bwd) {
  if (!args) return 0;
  if (!for_bwd) return ssm_fwd_workspace_size(args);
  ssm_bwd_args b;
  memset(&b, 0, sizeof(b));
  b.fwd = *args;
  b.chunk_states = args->chunk_states;
  return ssm_bwd_workspace_size(&b);
}

size_t ssm_bwd_workspace_size(const ssm_bwd_args *args) { return ssm::bwd_workspace_for(args, 1); }

ssm_status ssm_scan_bwd(const ssm_bwd_args *args, void *stream) {
  return ssm::scan_bwd_clustered(args, stream, 1);
}

}  // extern "C"

namespace ssm {

size_t bwd_workspace_for(const ssm_bwd_args *args, int max_cluster) {
  if (!args) return 0;
  const ssm_fwd_args *a = &args->fwd;
  if (a->Bt <= 0 || a->L <= 0 || a->Dn <= 0 || a->N <= 0 || a->n_segments < -1) return 0;
  return bwd_workspace_bytes(a->Bt, a->Dn, a->N, a->L, args->chunk_states == nullptr,
                             fwd_plan(a).n_seg, max_cluster);
}

ssm_status scan_bwd_clustered(const ssm_bwd_args *args, void *stream, int max_cluster) {
  SSM_RANGE("ssm_scan_bwd");
  if (!args) return SSM_ERR_NULL;
  bool empty = false;
  ssm_status st = check_fwd(&args->fwd, false, &empty);
  if (st != SSM_OK) return st;
  const ssm_fwd_args *a = &args->fwd;
  if (a->n_segments < -1) return SSM_ERR_SHAPE;
  if (empty) {
    // nothing flows: parameter gradients are zero, the carried-state gradient passes through
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t fz = sizeof(float);
    const int64_t BD = a->Bt * a->Dn;
    cudaError_t e = cudaSuccess;
    auto zero = [&](void *ptr, size_t bytes) {
      if (ptr && bytes && e == cudaSuccess) e = cudaMemsetAsync(ptr, 0, bytes, s);
    };
    zero(args->dA_log, fz * (size_t)(a->Dn * a->N));
    zero(args->dD, fz * (size_t)a->Dn);
    zero(args->ddt_bias, fz * (size_t)a->Dn);
    if (a->conv_w) {
      zero(args->dconv_w, fz * (size_t)(a->Dn * a->K));
      zero(args->dconv_b, fz * (size_t)a->Dn);
      if (a->K > 1) zero(args->dconv_hist, fz * (size_t)(BD * (a->K - 1)));
    }
    if (args->dh0 && BD > 0 && e == cudaSuccess)
      e = args->dh_last ? cudaMemcpyAsync(args->dh0, args->dh_last, fz * (size_t)(BD * a->N), cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(args->dh0, 0, fz * (size_t)(BD * a->N), s);
    return cuda_status(e);
  }
  if (!args->dout) return SSM_ERR_NULL;
  if (!aligned(args->dout, dtype_size(a->in_dtype))) return SSM_ERR_ALIGN;
  const void *g32[14] = {args->chunk_states, args->dx, args->ddt, args->dz, args->dA_log, args->dB,
                         args->dC, args->dD, args->ddt_bias, args->dconv_w, args->dconv_b,
                         args->dh_last, args->dh0, args->dconv_hist};
  for (const void *p : g32)
    if (p && !aligned(p, 4)) return SSM_ERR_ALIGN;
  const size_t need = bwd_workspace_for(args, max_cluster);
  if (need > 0 && (!args->workspace || args->workspace_bytes < need || !aligned(args->workspace, 256)))
    return SSM_ERR_WORKSPACE;

  const void *extra[5] = {args->dout, args->dx, args->ddt, args->dz, nullptr};
  ssm_fwd_args fa = *a;
  fa.out = nullptr;
  fa.u_out = nullptr;
  fa.chunk_states = nullptr;
  fa.h_last = nullptr;
  fa.conv_hist_out = nullptr;
  ssm::BwdParams p;
  memset(&p, 0, sizeof(p));
  p.f = make_fwd_params(&fa, vec_ok(&fa, extra, 4));
  p.dout = args->dout;
  p.chunk_states = args->chunk_states;
  p.dx = args->dx;
  p.ddt = args->ddt;
  p.dz = a->z ? args->dz : nullptr;
  p.dB = args->dB;
  p.dC = args->dC;
  p.dA_log = args->dA_log;
  p.dD = args->dD;
  p.ddt_bias = args->ddt_bias;
  p.dconv_w = a->conv_w ? args->dconv_w : nullptr;
  p.dconv_b = a->conv_w ? args->dconv_b : nullptr;
  p.timing_events = args->timing_events;
  p.dh_last = args->dh_last;
  p.dh0 = args->dh0;
  p.dconv_hist = (a->conv_w && a->K > 1) ? args->dconv_hist : nullptr;
  const ssm::SegPlan plan = fwd_plan(a);
  p.n_seg = plan.n_seg;
  p.seg_len = plan.seg_len;
  // carve the workspace (layout mirrored by ssm::bwd_workspace_bytes)
  char *ws = static_cast<char *>(args->workspace);
  auto take = [&](size_t bytes) {
    char *r = ws;
    ws += (bytes + 255) & ~size_t(255);
    return r;
  };
  const ssm::LaneLayout lay = ssm::choose_layout(a->N, a->Bt * a->Dn * p.n_seg);
  const int64_t ch = ssm::channels_per_cta(lay);
  p.n_dtiles = (a->Dn + ch - 1) / ch;
  p.cluster = ssm::bwd_cluster(lay, p.n_dtiles, max_cluster);
  p.n_ptiles = p.n_dtiles / p.cluster;
  const int64_t BD = a->Bt * a->Dn, PD = BD * p.n_seg;
  p.p_dA_log = reinterpret_cast<float *>(take(sizeof(float) * PD * a->N));
  p.p_dD = reinterpret_cast<float *>(take(sizeof(float) * PD));
  p.p_ddt_bias = reinterpret_cast<float *>(take(sizeof(float) * PD));
  p.p_dconv_w = reinterpret_cast<float *>(take(sizeof(float) * PD * 4));
  p.p_dconv_b = reinterpret_cast<float *>(take(sizeof(float) * PD));
  p.p_dB = reinterpret_cast<float *>(take(sizeof(float) * p.n_ptiles * a->Bt * a->N * a->L));
  p.p_dC = reinterpret_cast<float *>(take(sizeof(float) * p.n_ptiles * a->Bt * a->N * a->L));
  if (!args->chunk_states)
    p.f.chunk_states = reinterpret_cast<float *>(take(sizeof(float) * BD * p.f.n_ck * a->N));
  if (p.n_seg > 1) {
    p.seg_G = reinterpret_cast<float *>(take(sizeof(float) * PD * a->N));
    p.seg_gloc = reinterpret_cast<float *>(take(sizeof(float) * PD * a->N));
    p.seg_sdl = reinterpret_cast<float *>(take(sizeof(float) * PD));
    p.seg_dxh = reinterpret_cast<float *>(take(sizeof(float) * PD * 4));
  }
  return cuda_status(ssm::launch_bwd(p, a->in_dtype == SSM_BF16, static_cast<cudaStream_t>(stream)));
}

}  // namespace ssm

namespace {
ssm_status check_ssd(const ssm_ssd_args *a, bool *empty) {
  if (!a) return SSM_ERR_NULL;
  if (!dtype_ok(a->in_dtype) || !dtype_ok(a->out_dtype)) return SSM_ERR_DTYPE;
  if (a->discretization != SSM_ZOH && a->discretization != SSM_EULER) return SSM_ERR_UNSUPPORTED;
  if (a->Bt < 0 || a->H < 0 || a->L < 0 || a->P < 0 || a->N < 0) return SSM_ERR_SHAPE;
  if (a->H == 0 || a->P == 0 || a->N == 0) return SSM_ERR_SHAPE;
  if (a->in_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if ((a->P != 64 && a->P != 128) || (a->N != 64 && a->N != 128)) return SSM_ERR_UNSUPPORTED;
  if (a->form != SSM_SSD_AUTO && a->form != SSM_SSD_THREE_PASS && a->form != SSM_SSD_FUSED)
    return SSM_ERR_UNSUPPORTED;
  if (a->form == SSM_SSD_FUSED && a->P != 64) return SSM_ERR_UNSUPPORTED;
  int64_t bh, rows, elems;
  if (!mul_ok(a->Bt, a->H, &bh) || !mul_ok(bh, a->L, &rows) || !mul_ok(rows, a->P, &elems) ||
      elems > (INT64_C(1) << 50) || (bh > 0 && (a->L + 127) / 128 > (INT64_C(1) << 31) / bh))
    return SSM_ERR_SHAPE;
  *empty = (a->Bt == 0 || a->L == 0);
  if (*empty) return SSM_OK;
  if (!a->x || !a->dt || !a->A_log || !a->B || !a->C || !a->y) return SSM_ERR_NULL;
  const void *v16[4] = {a->x, a->B, a->C, a->y};
  for (const void *p : v16)
    if (!aligned(p, 16)) return SSM_ERR_ALIGN;
  if (!aligned(a->dt, 2)) return SSM_ERR_ALIGN;
  const void *f32[3] = {a->dt_bias, a->A_log, a->D};
  for (const void *p : f32)
    if (p && !aligned(p, 4)) return SSM_ERR_ALIGN;
  if ((a->h0 && !aligned(a->h0, 16)) || (a->h_last && !aligned(a->h_last, 16))) return SSM_ERR_ALIGN;
  return SSM_OK;
}

// Synchronise `s`, then read a device error word: non-zero means a bounded wait ran out.
ssm_status read_error_word(const void *word, cudaStream_t s) {
  int32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, word, sizeof(host), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  return host ? SSM_ERR_TIMEOUT : SSM_OK;
}
}  // namespace

extern "C" {

size_t ssm_ssd_workspace_size(const ssm_ssd_args *args) {
  bool empty = false;
  if (check_ssd(args, &empty) != SSM_OK || empty) return 0;
  return ssm::ssd_workspace_bytes(args->Bt, args->H, args->L, args->P, args->N);
}

ssm_status ssm_ssd_fwd(const ssm_ssd_args *args, void *stream) {
  SSM_RANGE("ssm_ssd_fwd");
  bool empty = false;
  ssm_status st = check_ssd(args, &empty);
  if (st != SSM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (empty) {
    // nothing to run: the state passes through
    if (args->h_last && args->Bt > 0) {
      const size_t nb = sizeof(float) * (size_t)(args->Bt * args->H * args->N * args->P);
      return cuda_status(args->h0 ? cudaMemcpyAsync(args->h_last, args->h0, nb, cudaMemcpyDeviceToDevice, s)
                                  : cudaMemsetAsync(args->h_last, 0, nb, s));
    }
    return SSM_OK;
  }
  const size_t need = ssm::ssd_workspace_bytes(args->Bt, args->H, args->L, args->P, args->N);
  if (!args->workspace || args->workspace_bytes < need || !aligned(args->workspace, 256))
    return SSM_ERR_WORKSPACE;
  auto rnd = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int64_t nC = (args->L + 127) / 128;
  const size_t chunks = (size_t)(args->Bt * args->H * nC), np = (size_t)(args->N * args->P);
  char *w = static_cast<char *>(args->workspace);
  ssm::SsdParams p;
  memset(&p, 0, sizeof(p));
  p.x = args->x;
  p.dt = args->dt;
  p.B = args->B;
  p.C = args->C;
  p.dt_bias = args->dt_bias;
  p.A_log = args->A_log;
  p.D = args->D;
  p.h0 = args->h0;
  p.y = args->y;
  p.h_last = args->h_last;
  p.Bt = args->Bt;
  p.H = args->H;
  p.L = args->L;
  p.P = args->P;
  p.N = args->N;
  p.delta_softplus = args->delta_softplus ? 1 : 0;
  p.euler = args->discretization == SSM_EULER ? 1 : 0;
  p.timing_events = args->timing_events;
  p.form = args->form;
  p.S = reinterpret_cast<float *>(w);
  w += rnd(sizeof(float) * chunks * np);
  p.Hin = reinterpret_cast<__nv_bfloat16 *>(w);
  w += rnd(sizeof(__nv_bfloat16) * chunks * np);
  p.cum_end = reinterpret_cast<float *>(w);
  w += rnd(sizeof(float) * chunks);
  p.error = reinterpret_cast<int *>(static_cast<char *>(args->workspace) +
                                     ssm::ssd_error_offset(args->Bt, args->H, args->L, args->P, args->N));
  cudaError_t e = cudaMemsetAsync(p.error, 0, sizeof(int), s);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(ssm::launch_ssd(p, args->out_dtype == SSM_BF16, s));
}

ssm_status ssm_ssd_check(const ssm_ssd_args *args, void *stream) {
  SSM_RANGE("ssm_ssd_check");
  bool empty = false;
  ssm_status st = check_ssd(args, &empty);
  if (st != SSM_OK) return st;
  if (empty) return SSM_OK;  // nothing ran, nothing to report
  if (!args->workspace || !aligned(args->workspace, 256) ||
      args->workspace_bytes < ssm::ssd_workspace_bytes(args->Bt, args->H, args->L, args->P, args->N))
    return SSM_ERR_WORKSPACE;
  return read_error_word(static_cast<const char *>(args->workspace) +
                             ssm::ssd_error_offset(args->Bt, args->H, args->L, args->P, args->N),
                         static_cast<cudaStream_t>(stream));
}

ssm_status ssm_wait_selftest(int32_t arrive, int32_t polls, int32_t *error_word, void *stream) {
  SSM_RANGE("ssm_wait_selftest");
  if (!error_word) return SSM_ERR_NULL;
  if (!aligned(error_word, 4)) return SSM_ERR_ALIGN;
  if (polls < 1 || polls > (1 << 22)) return SSM_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(error_word, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = ssm::launch_wait_selftest(arrive ? 1 : 0, polls, error_word, s);
  if (e != cudaSuccess) return cuda_status(e);
  return read_error_word(error_word, s);
}

}  // extern "C"
