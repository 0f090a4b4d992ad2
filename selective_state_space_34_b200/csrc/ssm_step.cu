// ssm_step.cu -- one-token decode step ("Selective Mamba", step): every channel advances its
// carried state by one token and emits one output, reading and rewriting the state in place.
//
// G lanes per (batch, channel), G = ceil(N / 16) rounded up to a power of two (1 at N = 16): lane l
// owns states 16l .. 16l+15, read and written as four 16-byte accesses, so the per-channel scalars
// (conv + SiLU, Delta, the gate, about a third of the instructions) are formed once per 16 states;
// with G > 1 every lane of the group forms them from the same addresses and the readout
// sum_n C_n h_n is a shuffle sum over the group. Lane 0 writes the output and the updated conv
// history. Each state element is read and written by exactly one thread, so
// updating in place needs no synchronisation. B_t and C_t are shared by the channels of a batch
// element and hit in L1. With bf16 inputs A = -exp(A_log), A_bar and (A_bar - 1) / A come from the
// hardware exp2 (the last as (1 - A_bar) e^{-A_log}, without a division); with fp32 inputs they
// use the accurate library functions.
#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

template <typename Tin, typename Tout, bool EULER, int G>
__global__ void __launch_bounds__(128) ssm_step_kernel(const StepParams p) {
  constexpr int NS = 16;  // states per lane
  const int64_t rows = p.Bt * p.Dn;
  const int64_t gi = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;  // b * Dn + d
  const int l = threadIdx.x % G;
  const bool live = gi < rows;  // the same for the G lanes of a channel
  const int64_t i = live ? gi : rows - 1;  // dead groups compute on a valid row and store nothing
  constexpr bool PRECISE = sizeof(Tin) == 4;
  int64_t b, d;
  if (rows <= 0x7fffffffLL) {  // 32-bit division where it fits (always, in practice)
    const uint32_t i32 = (uint32_t)i, dn = (uint32_t)p.Dn;
    b = i32 / dn;
    d = i32 - (uint32_t)b * dn;
  } else {
    b = i / p.Dn;
    d = i % p.Dn;
  }
  const int64_t N = p.N;
  const Tin xin = static_cast<const Tin *>(p.x)[i];
  float u;
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
      for (int k = 1; k < 4; k++)
        if (k < K) acc = fmaf(p.conv_w[d * K + k], to_f32(old[k - 1]), acc);
      // every lane has read the history before lane 0 rewrites it: the new token becomes the
      // newest entry, the oldest one drops out
      __syncwarp();
      if (live && l == 0) {
        hist[0] = xin;
#pragma unroll
        for (int j = 1; j < 3; j++)
          if (j < K - 1) hist[j] = old[j - 1];
      }
    }
    u = acc * sigmoid<PRECISE>(acc);
  } else {
    u = to_f32(xin);
  }
  const float v = to_f32(static_cast<const Tin *>(p.dt)[i]) + (p.dt_bias ? p.dt_bias[d] : 0.f);
  const float dl = p.delta_softplus ? softplus<PRECISE>(v) : v;
  const Tin *Bb = static_cast<const Tin *>(p.B) + b * N;
  const Tin *Cb = static_cast<const Tin *>(p.C) + b * N;
  float *h = p.h + i * N;
  const float *Al = p.A_log + d * N;
  const int64_t n0 = (int64_t)l * NS;
  // this lane's states: one 16-byte access where the row allows it
  float hv[NS], av[NS];
  const bool vec = N % NS == 0 && (reinterpret_cast<uintptr_t>(p.h) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(p.A_log) & 15) == 0 && n0 < N;
  if (vec) {
#pragma unroll
    for (int q = 0; q < NS / 4; q++) {
      const float4 h4 = *reinterpret_cast<const float4 *>(h + n0 + 4 * q);
      const float4 a4 = *reinterpret_cast<const float4 *>(Al + n0 + 4 * q);
      hv[4 * q] = h4.x; hv[4 * q + 1] = h4.y; hv[4 * q + 2] = h4.z; hv[4 * q + 3] = h4.w;
      av[4 * q] = a4.x; av[4 * q + 1] = a4.y; av[4 * q + 2] = a4.z; av[4 * q + 3] = a4.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < NS; j++) {
      hv[j] = n0 + j < N ? h[n0 + j] : 0.f;
      av[j] = n0 + j < N ? Al[n0 + j] : 0.f;
    }
  }
  float y = 0.f;
#pragma unroll
  for (int j = 0; j < NS; j++) {
    const int64_t n = n0 + j;
    if (n < N) {
      const float Bn = to_f32(Bb[n]);
      float a, kb;  // A_bar, and B_bar / B_n: (A_bar - 1) / A (exact ZOH) or Delta (Euler)
      if (PRECISE) {
        const float A = -expf(av[j]);
        const float em1 = expm1f(dl * A);
        a = 1.f + em1;
        kb = EULER ? dl : em1 / A;
      } else {
        // A = -e^{A_log}, so (A_bar - 1) / A = (1 - A_bar) e^{-A_log}: two exp2, no division
        const float lg = av[j] * kLog2e;
        a = ex2_approx(-dl * ex2_approx(lg) * kLog2e);
        kb = EULER ? dl : (1.f - a) * ex2_approx(-lg);
      }
      const float bbar = kb * Bn;
      hv[j] = fmaf(a, hv[j], bbar * u);
      y = fmaf(to_f32(Cb[n]), hv[j], y);
    }
  }
  if (live) {
    if (vec) {
#pragma unroll
      for (int q = 0; q < NS / 4; q++)
        *reinterpret_cast<float4 *>(h + n0 + 4 * q) = make_float4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < NS; j++)
        if (n0 + j < N) h[n0 + j] = hv[j];
    }
  }
#pragma unroll
  for (int off = G / 2; off >= 1; off >>= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
  if (live && l == 0) {
    y = fmaf(p.D ? p.D[d] : 0.f, u, y);
    if (p.z) {
      const float zz = to_f32(static_cast<const Tin *>(p.z)[i]);
      y *= zz * sigmoid<PRECISE>(zz);
    }
    static_cast<Tout *>(p.out)[i] = from_f32<Tout>(y);
  }
}

template <typename Tin, typename Tout, int G>
static cudaError_t step_g(const StepParams &p, cudaStream_t s) {
  const int64_t n = p.Bt * p.Dn * G;
  const int64_t blocks = (n + 127) / 128;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (p.euler)
    ssm_step_kernel<Tin, Tout, true, G><<<(unsigned)blocks, 128, 0, s>>>(p);
  else
    ssm_step_kernel<Tin, Tout, false, G><<<(unsigned)blocks, 128, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
static cudaError_t step_t(const StepParams &p, cudaStream_t s) {
  if (p.N <= 16) return step_g<Tin, Tout, 1>(p, s);
  if (p.N <= 32) return step_g<Tin, Tout, 2>(p, s);
  return step_g<Tin, Tout, 4>(p, s);  // N <= 64 (checked by the caller)
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
