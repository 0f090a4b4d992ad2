// ssm_step.cu -- one-token decode step ("Selective Mamba", step): every channel advances its
// carried state by one token and emits one output, reading and rewriting the state in place.
//
// One thread per (batch, channel): the conv history (K-1 values) and the N fp32 states are read,
// advanced and written back by the same thread, so updating in place needs no synchronisation.
// B_t and C_t are shared by the channels of a batch element and hit in L1.
#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

template <typename Tin, typename Tout, bool EULER>
__global__ void __launch_bounds__(128) ssm_step_kernel(const StepParams p) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // b * Dn + d
  if (i >= p.Bt * p.Dn) return;
  constexpr bool PRECISE = sizeof(Tin) == 4;
  const int64_t b = i / p.Dn, d = i % p.Dn, N = p.N;
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
      // the new token becomes the newest entry; the oldest one drops out
      hist[0] = xin;
#pragma unroll
      for (int j = 1; j < 3; j++)
        if (j < K - 1) hist[j] = old[j - 1];
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
  float y = 0.f;
  for (int64_t n = 0; n < N; n++) {
    const float A = -expf(p.A_log[d * N + n]);
    const float Bn = to_f32(Bb[n]);
    float a, em1;
    if (PRECISE) {
      em1 = expm1f(dl * A);
      a = 1.f + em1;
    } else {
      a = ex2_approx(dl * A * kLog2e);
      em1 = a - 1.f;
    }
    const float bbar = EULER ? dl * Bn : em1 / A * Bn;  // B_bar (Delta B, or the exact ZOH)
    const float hn = fmaf(a, h[n], bbar * u);
    h[n] = hn;
    y = fmaf(to_f32(Cb[n]), hn, y);
  }
  y = fmaf(p.D ? p.D[d] : 0.f, u, y);
  if (p.z) {
    const float zz = to_f32(static_cast<const Tin *>(p.z)[i]);
    y *= zz * sigmoid<PRECISE>(zz);
  }
  static_cast<Tout *>(p.out)[i] = from_f32<Tout>(y);
}

template <typename Tin, typename Tout>
static cudaError_t step_t(const StepParams &p, cudaStream_t s) {
  const int64_t n = p.Bt * p.Dn;
  const int64_t blocks = (n + 127) / 128;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (p.euler)
    ssm_step_kernel<Tin, Tout, true><<<(unsigned)blocks, 128, 0, s>>>(p);
  else
    ssm_step_kernel<Tin, Tout, false><<<(unsigned)blocks, 128, 0, s>>>(p);
  return cudaGetLastError();
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
