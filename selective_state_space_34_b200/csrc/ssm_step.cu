// ssm_step.cu -- one-token decode step ("Selective Mamba", step): every channel advances its
// carried state by one token and emits one output, reading and rewriting the state in place.
//
// A warp takes 32 kStepRows consecutive (batch, channel) rows, handled as kStepRows slots of 32.
// Lane c forms the per-channel scalars (conv + SiLU, Delta, the gate) of row c of every slot once,
// and owns those rows' outputs and conv histories (read and rewritten by that lane alone). The
// states of a slot are updated in P passes, P lanes per row and 4 states per lane (P = ceil(N / 4)
// rounded up to a power of two, 4 at N = 16): pass q takes the slot's rows q R .. q R + R - 1
// (R = 32 / P rows per pass) and lane l row q R + l / P, states 4 (l % P) .. 4 (l % P) + 3. With N = 4 P the 16-byte state and A_log accesses of a pass then
// cover one contiguous span of the warp (a row-per-lane layout puts 16 rows, 16 cache lines, under
// every 16-byte access). A pass takes its row's u and Delta from the owning lane by shuffles, and
// the P partial readouts sum_n C_n h_n are added by shuffles and handed to the owning lane. Each
// state element is read and written by exactly one thread, so updating in place needs no
// synchronisation. B_t and C_t are shared by the channels of a batch element and hit in L1. With
// bf16 inputs A = -exp(A_log), A_bar and (A_bar - 1) / A come from the hardware exp2 (the last as
// (1 - A_bar) e^{-A_log}, without a division); with fp32 inputs they use the accurate library
// functions.
#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

// (batch, channel) rows per lane: 2 keeps the whole 64 x 4096 decode grid in one wave (1024 CTAs
// of 128 threads at up to 8 per SM) where one row per lane needed 1.4 waves.
#ifndef SSM_STEP_ROWS
#define SSM_STEP_ROWS 2
#endif
constexpr int kStepRows = SSM_STEP_ROWS;

template <typename Tin, typename Tout, bool EULER, int P>
__global__ void __launch_bounds__(128) ssm_step_kernel(const StepParams p) {
  constexpr int R = 32 / P;  // rows per pass
  constexpr bool PRECISE = sizeof(Tin) == 4;
  constexpr unsigned kFull = 0xffffffffu;
  const int64_t rows = p.Bt * p.Dn;
  const int lane = threadIdx.x & 31;
  const int64_t row0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x - lane) * kStepRows;  // the warp's first row
  const int64_t N = p.N;

  // -- this lane's rows row0 + 32 k + lane: the per-channel scalars
  float u[kStepRows], dl[kStepRows];
  int64_t bk[kStepRows], dk[kStepRows];
#pragma unroll
  for (int k = 0; k < kStepRows; k++) {
    const int64_t gi = row0 + 32 * k + lane;
    const bool live = gi < rows;
    const int64_t i = live ? gi : rows - 1;  // dead rows are computed on a valid row and not stored
    int64_t b, d;
    if (rows <= 0x7fffffffLL) {  // 32-bit division where it fits (always, in practice)
      const uint32_t i32 = (uint32_t)i, dn = (uint32_t)p.Dn;
      b = i32 / dn;
      d = i32 - (uint32_t)b * dn;
    } else {
      b = i / p.Dn;
      d = i % p.Dn;
    }
    bk[k] = b;
    dk[k] = d;
    const Tin xin = static_cast<const Tin *>(p.x)[i];
    float uk;
    if (p.conv_w) {
      const int K = p.K;
      float acc = (p.conv_b ? p.conv_b[d] : 0.f) + p.conv_w[d * K] * to_f32(xin);
      if (K > 1) {
        Tin *hist = static_cast<Tin *>(p.conv_hist) + i * (K - 1);
        Tin old[3];
#pragma unroll
        for (int j = 0; j < 3; j++)
          if (j < K - 1) old[j] = hist[j];
#pragma unroll
        for (int kk = 1; kk < 4; kk++)
          if (kk < K) acc = fmaf(p.conv_w[d * K + kk], to_f32(old[kk - 1]), acc);
        if (live) {  // the new token becomes the newest entry, the oldest one drops out
          hist[0] = xin;
#pragma unroll
          for (int j = 1; j < 3; j++)
            if (j < K - 1) hist[j] = old[j - 1];
        }
      }
      uk = acc * sigmoid<PRECISE>(acc);
    } else {
      uk = to_f32(xin);
    }
    u[k] = uk;
    const float v = to_f32(static_cast<const Tin *>(p.dt)[i]) + (p.dt_bias ? p.dt_bias[d] : 0.f);
    dl[k] = p.delta_softplus ? softplus<PRECISE>(v) : v;
  }

  // -- the states, in kStepRows * P passes of 4 states per lane
  const int sq = lane % P, rl = lane / P;
  const int64_t n0 = 4 * sq;
  const uintptr_t bc_align = PRECISE ? 15 : 7;  // 4 values of B_t / C_t as one access
  const bool vec = N == 4 * P && ((reinterpret_cast<uintptr_t>(p.h) | reinterpret_cast<uintptr_t>(p.A_log)) & 15) == 0 &&
                   ((reinterpret_cast<uintptr_t>(p.B) | reinterpret_cast<uintptr_t>(p.C)) & bc_align) == 0;
  float yown[kStepRows];  // this lane's row readouts, collected from the passes that update them
#pragma unroll
  for (int k = 0; k < kStepRows; k++) yown[k] = 0.f;
#pragma unroll
  for (int q = 0; q < kStepRows * P; q++) {
    const int k = q / P;                  // the slot of the pass's rows in their owners
    const int src = (q % P) * R + rl;     // the lane that owns this lane's row of the pass
    const float ur = __shfl_sync(kFull, u[k], src);
    const float dlr = __shfl_sync(kFull, dl[k], src);
    const int64_t br = __shfl_sync(kFull, (long long)bk[k], src);
    const int64_t dr = __shfl_sync(kFull, (long long)dk[k], src);
    const int64_t r = row0 + 32 * k + src;
    const bool rlive = r < rows;
    const int64_t rr = rlive ? r : rows - 1;
    float *h = p.h + rr * N + n0;
    const float *Al = p.A_log + dr * N + n0;
    const Tin *Bb = static_cast<const Tin *>(p.B) + br * N + n0;
    const Tin *Cb = static_cast<const Tin *>(p.C) + br * N + n0;
    float hv[4], av[4], Bv[4], Cv[4];
    if (vec) {
      const float4 h4 = *reinterpret_cast<const float4 *>(h);
      const float4 a4 = *reinterpret_cast<const float4 *>(Al);
      hv[0] = h4.x; hv[1] = h4.y; hv[2] = h4.z; hv[3] = h4.w;
      av[0] = a4.x; av[1] = a4.y; av[2] = a4.z; av[3] = a4.w;
      if constexpr (PRECISE) {
        const float4 b4 = *reinterpret_cast<const float4 *>(Bb);
        const float4 c4 = *reinterpret_cast<const float4 *>(Cb);
        Bv[0] = b4.x; Bv[1] = b4.y; Bv[2] = b4.z; Bv[3] = b4.w;
        Cv[0] = c4.x; Cv[1] = c4.y; Cv[2] = c4.z; Cv[3] = c4.w;
      } else {
        // 4 bf16 as 8 bytes; a bf16 is the top half of a float
        const uint2 bw = *reinterpret_cast<const uint2 *>(Bb);
        const uint2 cw = *reinterpret_cast<const uint2 *>(Cb);
        Bv[0] = __uint_as_float(bw.x << 16); Bv[1] = __uint_as_float(bw.x & 0xffff0000u);
        Bv[2] = __uint_as_float(bw.y << 16); Bv[3] = __uint_as_float(bw.y & 0xffff0000u);
        Cv[0] = __uint_as_float(cw.x << 16); Cv[1] = __uint_as_float(cw.x & 0xffff0000u);
        Cv[2] = __uint_as_float(cw.y << 16); Cv[3] = __uint_as_float(cw.y & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const bool in = n0 + j < N;
        hv[j] = in ? h[j] : 0.f;
        av[j] = in ? Al[j] : 0.f;
        Bv[j] = in ? to_f32(Bb[j]) : 0.f;
        Cv[j] = in ? to_f32(Cb[j]) : 0.f;
      }
    }
    float y = 0.f;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      if (n0 + j < N) {
        float a, kb;  // A_bar, and B_bar / B_n: (A_bar - 1) / A (exact ZOH) or Delta (Euler)
        if (PRECISE) {
          const float A = -expf(av[j]);
          const float em1 = expm1f(dlr * A);
          a = 1.f + em1;
          kb = EULER ? dlr : em1 / A;
        } else {
          // A = -e^{A_log}, so (A_bar - 1) / A = (1 - A_bar) e^{-A_log}: two exp2, no division
          const float lg = av[j] * kLog2e;
          a = ex2_approx(-dlr * ex2_approx(lg) * kLog2e);
          kb = EULER ? dlr : (1.f - a) * ex2_approx(-lg);
        }
        hv[j] = fmaf(a, hv[j], kb * Bv[j] * ur);
        y = fmaf(Cv[j], hv[j], y);
      }
    }
    if (rlive) {
      if (vec) {
        *reinterpret_cast<float4 *>(h) = make_float4(hv[0], hv[1], hv[2], hv[3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; j++)
          if (n0 + j < N) h[j] = hv[j];
      }
    }
    // the row's P partial readouts, then to the lane that owns the row
#pragma unroll
    for (int off = P / 2; off >= 1; off >>= 1) y += __shfl_xor_sync(kFull, y, off);
    const float yr = __shfl_sync(kFull, y, (lane % R) * P);
    if (lane / R == q % P) yown[k] = yr;
  }
#pragma unroll
  for (int k = 0; k < kStepRows; k++) {
    const int64_t gi = row0 + 32 * k + lane;
    if (gi < rows) {
      float y = fmaf(p.D ? p.D[dk[k]] : 0.f, u[k], yown[k]);
      if (p.z) {
        const float zz = to_f32(static_cast<const Tin *>(p.z)[gi]);
        y *= zz * sigmoid<PRECISE>(zz);
      }
      static_cast<Tout *>(p.out)[gi] = from_f32<Tout>(y);
    }
  }
}

template <typename Tin, typename Tout, int P>
static cudaError_t step_p(const StepParams &p, cudaStream_t s) {
  const int64_t warps = (p.Bt * p.Dn + 32 * kStepRows - 1) / (32 * kStepRows);  // 32 kStepRows rows each
  const int64_t blocks = (warps + 3) / 4;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (p.euler)
    ssm_step_kernel<Tin, Tout, true, P><<<(unsigned)blocks, 128, 0, s>>>(p);
  else
    ssm_step_kernel<Tin, Tout, false, P><<<(unsigned)blocks, 128, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
static cudaError_t step_t(const StepParams &p, cudaStream_t s) {
  if (p.N <= 4) return step_p<Tin, Tout, 1>(p, s);
  if (p.N <= 8) return step_p<Tin, Tout, 2>(p, s);
  if (p.N <= 16) return step_p<Tin, Tout, 4>(p, s);
  if (p.N <= 32) return step_p<Tin, Tout, 8>(p, s);
  return step_p<Tin, Tout, 16>(p, s);  // N <= 64 (checked by the caller)
}

cudaError_t launch_step(const StepParams &p, int in_bf16, int out_bf16, cudaStream_t stream) {
  if (in_bf16) {
    if (out_bf16) return step_t<__nv_bfloat16, __nv_bfloat16>(p, stream);
    return step_t<__nv_bfloat16, float>(p, stream);
  }
  if (out_bf16) return step_t<float, __nv_bfloat16>(p, stream);
  return step_t<float, float>(p, stream);
}

}  // namespace ssm
