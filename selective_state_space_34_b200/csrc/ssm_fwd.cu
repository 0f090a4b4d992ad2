// ssm_fwd.cu -- fused selective-scan forward for sm_100a:
//   causal depthwise conv1d + SiLU  ->  softplus(dt + dt_bias)  ->  exact-ZOH diagonal scan
//   ->  y = C.h + D u  ->  y * SiLU(z)
// (rustytorch commit log, "Real S6 forward"; "Selective Mamba" step; exact zero-order hold of
// "Sequence and state-space models", state_space_models).
//
// Work decomposition. One CTA owns CH = 128 / G channels of one batch element and walks the whole
// sequence in stages of kT time steps. Inside a warp, the G lanes of a channel each hold NS of its
// states in fp32 registers and run the recurrence sequentially in time; B_t and C_t are shared by
// all channels, so every lane reads them as shared-memory broadcasts. Per-element work (conv,
// SiLU, softplus, gate, the D skip and the store) is split over the G lanes of a channel so that
// nothing is computed twice; u and Delta reach the other lanes through shared memory and the G
// partial readouts sum_n C h are combined through shared memory.
//
// Staging: each stage's x, dt, z rows and B, C rows are streamed global -> shared with 16-byte
// cp.async (double-buffered, one stage in flight while the previous one is computed). The conv
// halo of 3 steps is carried across stages in a prefix in front of each x row.
#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

template <typename T> __device__ __forceinline__ T zero_val() { return from_f32<T>(0.0f); }

// dst[r][i] = src[r][t0 + i] for r < rows_valid and t0 + i < L, else 0, for i in [0, kT).
template <typename T, int ROWS>
__device__ __forceinline__ void stage_rows(T *dst, int dst_stride, const T *src, int64_t src_stride,
                                           int rows_valid, int64_t t0, int64_t L, bool vec) {
  constexpr int EPV = 16 / sizeof(T);
  constexpr int VPR = kT / EPV;
  if (vec) {
    for (int idx = threadIdx.x; idx < ROWS * VPR; idx += kThreads) {
      const int r = idx / VPR, v = idx % VPR;
      const int64_t t = t0 + (int64_t)v * EPV;
      T *d = dst + r * dst_stride + v * EPV;
      if (r < rows_valid && t < L)
        cp_async16(d, src + (int64_t)r * src_stride + t);
      else
        *reinterpret_cast<uint4 *>(d) = make_uint4(0u, 0u, 0u, 0u);
    }
  } else {
    for (int idx = threadIdx.x; idx < ROWS * kT; idx += kThreads) {
      const int r = idx / kT, i = idx % kT;
      const int64_t t = t0 + i;
      dst[r * dst_stride + i] = (r < rows_valid && t < L) ? src[(int64_t)r * src_stride + t] : zero_val<T>();
    }
  }
}

template <typename T, int E> struct VecStore;
template <typename T> struct VecStore<T, 1> {
  static __device__ __forceinline__ void run(T *p, const float *v) { p[0] = from_f32<T>(v[0]); }
};
template <> struct VecStore<float, 2> {
  static __device__ __forceinline__ void run(float *p, const float *v) {
    *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
  }
};
template <> struct VecStore<float, 4> {
  static __device__ __forceinline__ void run(float *p, const float *v) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct VecStore<__nv_bfloat16, 2> {
  static __device__ __forceinline__ void run(__nv_bfloat16 *p, const float *v) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v[0], v[1]);
  }
};
template <> struct VecStore<__nv_bfloat16, 4> {
  static __device__ __forceinline__ void run(__nv_bfloat16 *p, const float *v) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t *>(&lo);
    pk.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = pk;
  }
};

// Store E consecutive outputs starting at time t (vector store when allowed, else per element
// with the L bound).
template <typename T, int E>
__device__ __forceinline__ void store_run(T *row, int64_t t, int64_t L, const float *v, bool vec) {
  if (vec) {
    if (t < L) VecStore<T, E>::run(row + t, v);
  } else {
#pragma unroll
    for (int j = 0; j < E; j++)
      if (t + j < L) row[t + j] = from_f32<T>(v[j]);
  }
}

// Shared-memory plan of one CTA (all offsets in bytes, 16-byte aligned).
template <int G, int NS, typename Tin> struct FwdSmem {
  static constexpr int CH = kThreads / G;    // channels per CTA
  static constexpr int NP = G * NS;          // padded state count
  static constexpr int XS = kPre + kT;       // x row length (elements)
  static constexpr int BS = NP + 4;          // Bs/Cs row stride (floats)
  static constexpr int US = kT + 4;          // us/dls/ss row stride (floats)
  static constexpr int YG = kSub + 8;        // y-partial stride between lanes of a channel
  static constexpr int YC = G * YG + 4;      // y-partial stride between channels
  static constexpr size_t x_off = 0;
  static constexpr size_t dt_off = x_off + sizeof(Tin) * 2 * CH * XS;
  static constexpr size_t z_off = dt_off + sizeof(Tin) * 2 * CH * kT;
  static constexpr size_t braw_off = z_off + sizeof(Tin) * 2 * CH * kT;
  static constexpr size_t craw_off = braw_off + sizeof(Tin) * 2 * NP * kT;
  static constexpr size_t bs_off = craw_off + sizeof(Tin) * 2 * NP * kT;
  static constexpr size_t cs_off = bs_off + sizeof(float) * kT * BS;
  static constexpr size_t us_off = cs_off + sizeof(float) * kT * BS;
  static constexpr size_t dls_off = us_off + sizeof(float) * CH * US;
  static constexpr size_t ss_off = dls_off + sizeof(float) * CH * US;
  static constexpr size_t yp_off = ss_off + sizeof(float) * CH * US;
  static constexpr size_t bytes = yp_off + sizeof(float) * CH * YC;
};

template <int G, int NS, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads)
ssm_fwd_kernel(const FwdParams p) {
  using S = FwdSmem<G, NS, Tin>;
  constexpr int CH = S::CH, NP = S::NP, EPL = kSub / G;
  constexpr bool PRECISE = sizeof(Tin) == 4;
  extern __shared__ __align__(16) unsigned char smem[];
  Tin *xs = reinterpret_cast<Tin *>(smem + S::x_off);
  Tin *dts = reinterpret_cast<Tin *>(smem + S::dt_off);
  Tin *zs = reinterpret_cast<Tin *>(smem + S::z_off);
  Tin *braw = reinterpret_cast<Tin *>(smem + S::braw_off);
  Tin *craw = reinterpret_cast<Tin *>(smem + S::craw_off);
  float *Bs = reinterpret_cast<float *>(smem + S::bs_off);
  float *Cs = reinterpret_cast<float *>(smem + S::cs_off);
  float *us = reinterpret_cast<float *>(smem + S::us_off);
  float *dls = reinterpret_cast<float *>(smem + S::dls_off);
  float *ss = reinterpret_cast<float *>(smem + S::ss_off);
  float *yp = reinterpret_cast<float *>(smem + S::yp_off);

  const int64_t n_dtiles = (p.Dn + CH - 1) / CH;
  const int64_t b = blockIdx.x / n_dtiles;
  const int64_t d0 = (blockIdx.x % n_dtiles) * CH;
  const int rows_valid = (int)imin64(CH, p.Dn - d0);
  const int tid = threadIdx.x, c = tid / G, g = tid % G;
  const int64_t d = d0 + c;
  const bool live = d < p.Dn;
  const bool has_conv = p.conv_w != nullptr, has_z = p.z != nullptr;
  const bool vec = p.vec != 0;
  const int64_t L = p.L, N = p.N;

  // per-lane constants
  float Acoef[NS], invA[NS], h[NS];
#pragma unroll
  for (int j = 0; j < NS; j++) {
    const int n = g * NS + j;
    h[j] = 0.0f;
    if (live && n < N) {
      const float A = -expf(p.A_log[d * N + n]);
      Acoef[j] = PRECISE ? A : A * kLog2e;
      invA[j] = 1.0f / A;
    } else {
      Acoef[j] = 0.0f;
      invA[j] = 0.0f;
    }
  }
  float w4[4] = {0.f, 0.f, 0.f, 0.f};
  float cbias = 0.f, Dd = 0.f, dtb = 0.f;
  if (live) {
    if (has_conv) {
      for (int k = 0; k < p.K; k++) w4[k] = p.conv_w[d * p.K + k];
      cbias = p.conv_b ? p.conv_b[d] : 0.f;
    }
    Dd = p.D ? p.D[d] : 0.f;
    dtb = p.dt_bias ? p.dt_bias[d] : 0.f;
  }

  const int64_t row0 = (b * p.Dn + d0) * L;  // first activation row of this CTA
  const Tin *gx = static_cast<const Tin *>(p.x) + row0;
  const Tin *gdt = static_cast<const Tin *>(p.dt) + row0;
  const Tin *gz = has_z ? static_cast<const Tin *>(p.z) + row0 : nullptr;
  const Tin *gB = static_cast<const Tin *>(p.B) + b * N * L;
  const Tin *gC = static_cast<const Tin *>(p.C) + b * N * L;
  const int n_rows = (int)imin64(NP, N);

  // zero the conv-halo prefixes of both x buffers (the sequence starts from zero history)
  for (int i = tid; i < 2 * CH * kPre; i += kThreads) {
    const int r = i / kPre, k = i % kPre;
    xs[r * S::XS + k] = zero_val<Tin>();
  }

  const int64_t n_stages = (L + kT - 1) / kT;
  auto issue = [&](int64_t stage, int buf) {
    const int64_t t0 = stage * kT;
    stage_rows<Tin, CH>(xs + buf * CH * S::XS + kPre, S::XS, gx, L, rows_valid, t0, L, vec);
    stage_rows<Tin, CH>(dts + buf * CH * kT, kT, gdt, L, rows_valid, t0, L, vec);
    if (has_z) stage_rows<Tin, CH>(zs + buf * CH * kT, kT, gz, L, rows_valid, t0, L, vec);
    stage_rows<Tin, NP>(braw + buf * NP * kT, kT, gB, L, n_rows, t0, L, vec);
    stage_rows<Tin, NP>(craw + buf * NP * kT, kT, gC, L, n_rows, t0, L, vec);
    cp_async_commit();
  };

  if (n_stages > 0) issue(0, 0);
  for (int64_t st = 0; st < n_stages; st++) {
    const int buf = (int)(st & 1), nbuf = buf ^ 1;
    const int64_t t0 = st * kT;
    cp_async_wait<0>();
    __syncthreads();  // stage st landed; everyone is done with stage st-1's buffers
    if (st + 1 < n_stages) issue(st + 1, nbuf);

    // B, C: raw (n, t) tile -> fp32 (t, n) rows for broadcast reads
    for (int i = tid; i < NP * kT; i += kThreads) {
      const int n = i / kT, t = i % kT;
      Bs[t * S::BS + n] = to_f32(braw[buf * NP * kT + i]);
      Cs[t * S::BS + n] = to_f32(craw[buf * NP * kT + i]);
    }

    // per-element phase: lane g of channel c owns EPL consecutive steps of every sub-block
    const Tin *xrow = xs + (buf * CH + c) * S::XS + kPre;
    const Tin *dtrow = dts + (buf * CH + c) * kT;
    const Tin *zrow = zs + (buf * CH + c) * kT;
#pragma unroll
    for (int sb = 0; sb < kT / kSub; sb++) {
      float uo[EPL];
#pragma unroll
      for (int j = 0; j < EPL; j++) {
        const int t = sb * kSub + g * EPL + j;
        float u;
        if (has_conv) {
          float acc = cbias;
#pragma unroll
          for (int k = 0; k < 4; k++) acc = fmaf(w4[k], to_f32(xrow[t - k]), acc);
          u = acc * sigmoid<PRECISE>(acc);
        } else {
          u = to_f32(xrow[t]);
        }
        const float v = to_f32(dtrow[t]) + dtb;
        float dl = p.delta_softplus ? softplus<PRECISE>(v) : v;
        float s = 1.0f;
        if (has_z) {
          const float zz = to_f32(zrow[t]);
          s = zz * sigmoid<PRECISE>(zz);
        }
        if (t0 + t >= L) {  // padded tail: an identity step
          u = 0.0f;
          dl = 0.0f;
        }
        us[c * S::US + t] = u;
        dls[c * S::US + t] = dl;
        ss[c * S::US + t] = s;
        uo[j] = u;
        if (t >= kT - 3)  // carry the conv halo into the next stage's prefix
          xs[(nbuf * CH + c) * S::XS + kPre + t - kT] = xrow[t];
      }
      if (p.u_out && live)
        store_run<Tout, EPL>(static_cast<Tout *>(p.u_out) + row0 + (int64_t)c * L,
                             t0 + sb * kSub + g * EPL, L, uo, vec);
    }
    __syncthreads();  // Bs/Cs complete (written by all threads); us/dls/ss visible

    // scan phase
#pragma unroll
    for (int sb = 0; sb < kT / kSub; sb++) {
      float ypart[kSub];
#pragma unroll
      for (int tt = 0; tt < kSub; tt++) {
        const int t = sb * kSub + tt;
        const float u = us[c * S::US + t];
        const float dl = dls[c * S::US + t];
        const float *brow = Bs + t * S::BS + g * NS;
        const float *crow = Cs + t * S::BS + g * NS;
        float y = 0.0f;
#pragma unroll
        for (int j = 0; j < NS; j++) {
          const float w = brow[j] * u * invA[j];  // B u / A
          if (PRECISE) {
            const float em1 = expm1f(dl * Acoef[j]);  // A_bar - 1
            h[j] = fmaf(em1, h[j] + w, h[j]);         // A_bar h + (A_bar - 1) B u / A
          } else {
            const float a = ex2_approx(dl * Acoef[j]);  // A_bar
            h[j] = fmaf(a, h[j] + w, -w);
          }
          y = fmaf(crow[j], h[j], y);
        }
        ypart[tt] = y;
      }
      // combine the G partial readouts of each step
      float *myp = yp + c * S::YC + g * S::YG;
#pragma unroll
      for (int tt = 0; tt < kSub; tt += 4)
        *reinterpret_cast<float4 *>(myp + tt) = make_float4(ypart[tt], ypart[tt + 1], ypart[tt + 2], ypart[tt + 3]);
      __syncwarp();
      float o[EPL];
#pragma unroll
      for (int j = 0; j < EPL; j++) {
        const int tl = g * EPL + j, t = sb * kSub + tl;
        float y = 0.0f;
#pragma unroll
        for (int gg = 0; gg < G; gg++) y += yp[c * S::YC + gg * S::YG + tl];
        y = fmaf(Dd, us[c * S::US + t], y);
        o[j] = y * ss[c * S::US + t];
      }
      if (live && p.out)
        store_run<Tout, EPL>(static_cast<Tout *>(p.out) + row0 + (int64_t)c * L,
                             t0 + sb * kSub + g * EPL, L, o, vec);
      if (p.chunk_states && live && t0 + sb * kSub < L) {
        const int64_t kk = (t0 + sb * kSub) / kSub;
        float *dst = p.chunk_states + ((b * p.Dn + d) * p.n_ck + kk) * N;
#pragma unroll
        for (int j = 0; j < NS; j++)
          if (g * NS + j < N) dst[g * NS + j] = h[j];
      }
      __syncwarp();
    }
  }
}

// ---- host side -----------------------------------------------------------------------------

LaneLayout choose_layout(int64_t N, int64_t channels) {
  // Prefer the most states per lane (least cross-lane work) that still gives about two CTAs
  // per SM on a 148-SM part; N decides which (G, NS) pairs can hold it.
  const int64_t want_ctas = 2 * 148;
  const int Gs[3] = {4, 8, 16};
  LaneLayout best = {16, 4};
  bool found = false;
  for (int i = 0; i < 3 && !found; i++) {
    const int G = Gs[i];
    int NS = 0;
    for (int cand : {1, 2, 4})
      if ((int64_t)G * cand >= N) {
        NS = cand;
        break;
      }
    if (NS == 0) continue;
    best = {G, NS};
    const int64_t ctas = (channels + (kThreads / G) - 1) / (kThreads / G);
    if (ctas >= want_ctas) found = true;
  }
  if (!found) {
    // few channels: take the widest layout that can still hold N
    for (int i = 2; i >= 0; i--) {
      const int G = Gs[i];
      for (int cand : {1, 2, 4})
        if ((int64_t)G * cand >= N) return LaneLayout{G, cand};
    }
  }
  return best;
}

int channels_per_cta(const LaneLayout &lay) { return kThreads / lay.G; }

template <int G, int NS, typename Tin, typename Tout>
static cudaError_t launch_fwd_t(const FwdParams &p, cudaStream_t stream) {
  using S = FwdSmem<G, NS, Tin>;
  auto kern = ssm_fwd_kernel<G, NS, Tin, Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::bytes);
  if (e != cudaSuccess) return e;
  const int64_t n_dtiles = (p.Dn + S::CH - 1) / S::CH;
  const int64_t grid = n_dtiles * p.Bt;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<(unsigned)grid, kThreads, S::bytes, stream>>>(p);
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
static cudaError_t dispatch_layout(const LaneLayout &lay, const FwdParams &p, cudaStream_t s) {
#define SSM_FWD_CASE(G_, NS_) \
  if (lay.G == G_ && lay.NS == NS_) return launch_fwd_t<G_, NS_, Tin, Tout>(p, s);
  SSM_FWD_CASE(4, 1) SSM_FWD_CASE(4, 2) SSM_FWD_CASE(4, 4)
  SSM_FWD_CASE(8, 1) SSM_FWD_CASE(8, 2) SSM_FWD_CASE(8, 4)
  SSM_FWD_CASE(16, 1) SSM_FWD_CASE(16, 2) SSM_FWD_CASE(16, 4)
#undef SSM_FWD_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd(const FwdParams &p, int in_bf16, int out_bf16, cudaStream_t stream) {
  const LaneLayout lay = choose_layout(p.N, p.Bt * p.Dn);
  if (in_bf16) {
    if (out_bf16) return dispatch_layout<__nv_bfloat16, __nv_bfloat16>(lay, p, stream);
    return dispatch_layout<__nv_bfloat16, float>(lay, p, stream);
  }
  if (out_bf16) return dispatch_layout<float, __nv_bfloat16>(lay, p, stream);
  return dispatch_layout<float, float>(lay, p, stream);
}

}  // namespace ssm
