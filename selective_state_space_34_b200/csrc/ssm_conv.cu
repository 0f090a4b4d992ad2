// ssm_conv.cu -- standalone causal depthwise conv1d + SiLU ("Selective Mamba": convKernel with
// row zero on the current token, convBias added before the content SiLU; rustytorch commit log,
// "causal depthwise conv1d -> SiLU").
//
// Pure streaming: each thread produces EPT consecutive outputs of one channel from EPT + 3 inputs
// (the 3-step halo is re-read from global memory; it is served by L1/L2). HBM-bound by design.
#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

template <typename Tin, typename Tout, int EPT>
__global__ void __launch_bounds__(256)
conv1d_silu_kernel(const Tin *__restrict__ x, Tout *__restrict__ u, const float *__restrict__ w,
                   const float *__restrict__ bias, int64_t Dn, int64_t L, int K,
                   int64_t runs_per_row, int64_t total_runs) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total_runs) return;
  const int64_t row = i / runs_per_row;
  const int64_t t0 = (i % runs_per_row) * EPT;
  const int64_t d = row % Dn;
  float wk[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = 0; k < K; k++) wk[k] = w[d * K + k];
  const float b = bias ? bias[d] : 0.f;
  const Tin *xr = x + row * L;
  Tout *ur = u + row * L;
  float xv[EPT + 3];
#pragma unroll
  for (int j = 0; j < EPT + 3; j++) {
    const int64_t t = t0 - 3 + j;
    xv[j] = (t >= 0 && t < L) ? to_f32(xr[t]) : 0.0f;
  }
  constexpr bool PRECISE = sizeof(Tin) == 4;
#pragma unroll
  for (int j = 0; j < EPT; j++) {
    const int64_t t = t0 + j;
    if (t < L) {
      float acc = b;
#pragma unroll
      for (int k = 0; k < 4; k++) acc = fmaf(wk[k], xv[j + 3 - k], acc);
      ur[t] = from_f32<Tout>(acc * sigmoid<PRECISE>(acc));
    }
  }
}

template <typename Tin, typename Tout>
static cudaError_t conv_t(const void *x, void *u, const float *w, const float *b, int64_t Bt,
                          int64_t Dn, int64_t L, int K, cudaStream_t s) {
  constexpr int EPT = 8;
  const int64_t runs_per_row = (L + EPT - 1) / EPT;
  const int64_t total = Bt * Dn * runs_per_row;
  const int64_t blocks = (total + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  conv1d_silu_kernel<Tin, Tout, EPT><<<(unsigned)blocks, 256, 0, s>>>(
      static_cast<const Tin *>(x), static_cast<Tout *>(u), w, b, Dn, L, K, runs_per_row, total);
  return cudaGetLastError();
}

cudaError_t launch_conv1d_silu(const void *x, void *u, const float *w, const float *b, int64_t Bt,
                               int64_t Dn, int64_t L, int K, int in_bf16, int out_bf16, int vec,
                               cudaStream_t stream) {
  (void)vec;
  if (in_bf16) {
    if (out_bf16) return conv_t<__nv_bfloat16, __nv_bfloat16>(x, u, w, b, Bt, Dn, L, K, stream);
    return conv_t<__nv_bfloat16, float>(x, u, w, b, Bt, Dn, L, K, stream);
  }
  if (out_bf16) return conv_t<float, __nv_bfloat16>(x, u, w, b, Bt, Dn, L, K, stream);
  return conv_t<float, float>(x, u, w, b, Bt, Dn, L, K, stream);
}

}  // namespace ssm
