// ssm_stage.cuh -- staging and vector load/store helpers shared by the scan kernels: global ->
// shared row staging with 16-byte cp.async (L2 256-byte prefetch), B/C staging through registers
// into transposed fp32 rows, and small vectorized shared-memory reads / global stores.
#pragma once

#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

template <typename T> __device__ __forceinline__ T zero_val() { return from_f32<T>(0.0f); }

// dst[r][i] = src[r][t0 + i] for r < rows_valid and 0 <= t0 + i < L, else 0, for i in [0, LEN).
template <typename T, int ROWS, int LEN = kT, int NT = kThreads>
__device__ __forceinline__ void stage_rows(T *dst, int dst_stride, const T *src, int64_t src_stride,
                                           int rows_valid, int64_t t0, int64_t L, bool vec) {
  constexpr int EPV = 16 / sizeof(T);
  constexpr int VPR = LEN / EPV;
  if (vec) {
    for (int idx = threadIdx.x; idx < ROWS * VPR; idx += NT) {
      const int r = idx / VPR, v = idx % VPR;
      const int64_t t = t0 + (int64_t)v * EPV;
      T *d = dst + r * dst_stride + v * EPV;
      if (r < rows_valid && t >= 0 && t < L)
        cp_async16_l2pf(d, src + (int64_t)r * src_stride + t);
      else
        *reinterpret_cast<uint4 *>(d) = make_uint4(0u, 0u, 0u, 0u);
    }
  } else {
    for (int idx = threadIdx.x; idx < ROWS * LEN; idx += NT) {
      const int r = idx / LEN, i = idx % LEN;
      const int64_t t = t0 + i;
      dst[r * dst_stride + i] =
          (r < rows_valid && t >= 0 && t < L) ? src[(int64_t)r * src_stride + t] : zero_val<T>();
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

// n consecutive activations from shared memory as fp32, read with the widest aligned vectors
// (the callers' offsets are multiples of 4 elements, so 8-byte loads for bf16, 16-byte for fp32).
template <typename T, int NE> __device__ __forceinline__ void load_window(float *dst, const T *src) {
  if (sizeof(T) == 2 && NE % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NE; i += 4) {
      const uint2 v = *reinterpret_cast<const uint2 *>(src + i);
      const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&v.x);
      const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&v.y);
      dst[i] = __low2float(lo);
      dst[i + 1] = __high2float(lo);
      dst[i + 2] = __low2float(hi);
      dst[i + 3] = __high2float(hi);
    }
  } else if (sizeof(T) == 4 && NE % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NE; i += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + i);
      dst[i] = v.x;
      dst[i + 1] = v.y;
      dst[i + 2] = v.z;
      dst[i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < NE; i++) dst[i] = to_f32(src[i]);
  }
}
template <int NE> __device__ __forceinline__ void load_floats(float *dst, const float *src) {
  if (NE % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NE; i += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + i);
      dst[i] = v.x;
      dst[i + 1] = v.y;
      dst[i + 2] = v.z;
      dst[i + 3] = v.w;
    }
  } else if (NE % 2 == 0) {
#pragma unroll
    for (int i = 0; i < NE; i += 2) {
      const float2 v = *reinterpret_cast<const float2 *>(src + i);
      dst[i] = v.x;
      dst[i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < NE; i++) dst[i] = src[i];
  }
}
template <int NS> __device__ __forceinline__ void load_states(float *dst, const float *src) {
  load_floats<NS>(dst, src);
}

// B and C of one stage (NP rows x LEN steps, row stride L in global memory) go global ->
// registers -> transposed fp32 rows [t][n] in shared memory, so that the scan reads all of a
// lane's states at one step with one 16-byte broadcast load. Loads for stage s+1 are issued one
// stage early into registers; the transposed stores happen after the next barrier-free point.
template <typename Tin, int NP, int NT = kThreads, int LEN = kT> struct BCStager {
  static constexpr int EPV = 16 / sizeof(Tin);               // elements per 16-byte vector
  static constexpr int VPR = LEN / EPV;                      // vectors per row
  static constexpr int NV = 2 * NP * VPR;                    // B and C vectors per stage
  static constexpr int PER = (NV + NT - 1) / NT;             // per thread
  uint4 v[PER];

  __device__ __forceinline__ void load(const Tin *gB, const Tin *gC, int n_rows, int64_t t0,
                                       int64_t L, bool vec) {
#pragma unroll
    for (int k = 0; k < PER; k++) {
      const int i = threadIdx.x + k * NT;
      v[k] = make_uint4(0u, 0u, 0u, 0u);
      if (i >= NV) continue;
      const int which = i / (NP * VPR), r = (i / VPR) % NP, q = i % VPR;
      const Tin *src = (which ? gC : gB) + (int64_t)r * L;
      const int64_t t = t0 + (int64_t)q * EPV;
      if (r >= n_rows) continue;
      if (vec) {
        if (t < L) v[k] = ld_global_l2pf(src + t);
      } else {
        Tin tmp[EPV];
#pragma unroll
        for (int e = 0; e < EPV; e++) tmp[e] = (t + e < L) ? src[t + e] : from_f32<Tin>(0.0f);
        v[k] = *reinterpret_cast<const uint4 *>(tmp);
      }
    }
  }
  __device__ __forceinline__ void store(float *Bs, float *Cs, int BS) const {
#pragma unroll
    for (int k = 0; k < PER; k++) {
      const int i = threadIdx.x + k * NT;
      if (i >= NV) continue;
      const int which = i / (NP * VPR), r = (i / VPR) % NP, q = i % VPR;
      float *dst = (which ? Cs : Bs) + (q * EPV) * BS + r;
      const Tin *e = reinterpret_cast<const Tin *>(&v[k]);
#pragma unroll
      for (int j = 0; j < EPV; j++) dst[j * BS] = to_f32(e[j]);
    }
  }
};

}  // namespace ssm
