// ssm_fwd_tp.cu -- time-parallel selective-scan forward for sm_100a: a chunked scan over L.
//
// The same operation as ssm_fwd.cu (causal depthwise conv1d + SiLU, softplus Delta, exact-ZOH or
// Euler diagonal scan, y = C.h + D u, SiLU(z) gate), decomposed over time instead of over states:
//
//  * A group of 8 lanes owns one channel; lane i of the group owns 8 consecutive steps of every
//    64-step chunk (steps 8i .. 8i+7), so a warp holds 4 channels and a 128-thread CTA 16
//    channels of one batch element. Each lane computes conv, SiLU, softplus and the gate of its
//    own steps once, in registers: nothing per-element is shared between lanes.
//  * For each pair of states the chunk is scanned in three moves ("state-space models", "One
//    recurrence, one convolution"; the glossary's Lab 3 associative combine of (A_bar, B_bar u)
//    pairs): (1) every lane runs its 8 steps from a zero state, keeping the local states h_i and
//    the running products P_i of A_bar; (2) an inclusive scan of the lanes' summaries (P, H) over
//    the group by warp shuffles, with (P1, H1) then (P2, H2) composing to (P2 P1, P2 H1 + H2),
//    gives each lane the state entering its steps from the chunk's carried state; (3) the lane
//    finishes its steps as h_i = h_local_i + P_i h_in and adds C_i h_i to its outputs. The last
//    lane's end state is the carry into the next chunk.
//  * B and C of a chunk (shared by the CTA's channels) are staged global -> registers -> fp32 rows
//    [n][64 steps] in shared memory, double-buffered, one chunk ahead.
//
// The arithmetic per element-state is that of the sequential kernel plus the second pass over
// the lane's steps; the scan costs O(log 8) shuffles per state pair and lane.
#include "ssm_common.cuh"
#include "ssm_internal.h"
#include "ssm_stage.cuh"

namespace ssm {

constexpr int kTpLanes = 8;                  // lanes per channel
constexpr int kTpT = 8;                      // steps per lane
constexpr int kTpChunk = kTpLanes * kTpT;    // steps per chunk
constexpr int kTpThreads = 128;
constexpr int kTpCh = kTpThreads / kTpLanes;  // channels per CTA

// Shared-memory plan (bytes, 16-byte aligned); NP = N rounded up to even.
struct TpSmem {
  static __host__ __device__ size_t bc_bytes(int NP) { return sizeof(float) * 2 * 2 * NP * kTpChunk; }
  static __host__ __device__ size_t coef_off(int NP) { return bc_bytes(NP); }
  static __host__ __device__ size_t carry_off(int NP) { return coef_off(NP) + sizeof(float) * 2 * kTpCh * NP; }
  static __host__ __device__ size_t bytes(int NP) { return carry_off(NP) + sizeof(float) * kTpCh * NP; }
};

// 8 consecutive activations of a row into fp32, as one or two 16-byte loads when aligned and in
// range, else element by element with zeros outside [0, L).
template <typename T>
__device__ __forceinline__ void load8(float *v, const T *row, int64_t t, int64_t L, bool vec) {
  if (vec && t + 7 < L) {
    if constexpr (sizeof(T) == 2) {
      const uint4 w = *reinterpret_cast<const uint4 *>(row + t);
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
    } else {
      const float4 a = *reinterpret_cast<const float4 *>(row + t);
      const float4 b = *reinterpret_cast<const float4 *>(row + t + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = (t + i >= 0 && t + i < L) ? to_f32(row[t + i]) : 0.0f;
  }
}

// 8 consecutive outputs from step t: one or two 16-byte stores when aligned and in range, else
// element by element below L.
template <typename T>
__device__ __forceinline__ void store8(T *row, int64_t t, int64_t L, const float *v, bool vec) {
  if (vec && t + 7 < L) {
    if constexpr (sizeof(T) == 2) {
      uint4 w;
      uint32_t *pw = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        pw[i] = *reinterpret_cast<const uint32_t *>(&h);
      }
      *reinterpret_cast<uint4 *>(row + t) = w;
    } else {
      *reinterpret_cast<float4 *>(row + t) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4 *>(row + t + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; i++)
      if (t + i < L) row[t + i] = from_f32<T>(v[i]);
  }
}

// B and C of one chunk: global (Bt, N, L) rows -> registers -> fp32 rows [n][kTpChunk] in shared
// memory (B rows, then C rows; rows from N to NP are zero). Loads for chunk c+1 are issued while
// chunk c is computed; the stores follow the next barrier. NPC: state pairs the kernel is built for.
template <typename Tin, int NPC> struct TpBCStager {
  static constexpr int EPV = 16 / sizeof(Tin);
  static constexpr int VPR = kTpChunk / EPV;
  static constexpr int NITEM = 2 * (2 * NPC) * VPR;
  static constexpr int PER = (NITEM + kTpThreads - 1) / kTpThreads;
  uint4 v[PER];

  __device__ __forceinline__ void load(const Tin *gB, const Tin *gC, int N, int NP, int64_t t0,
                                       int64_t L, bool vec) {
#pragma unroll
    for (int k = 0; k < PER; k++) {
      const int i = threadIdx.x + k * kTpThreads;
      v[k] = make_uint4(0u, 0u, 0u, 0u);
      const int which = i / (2 * NPC * VPR), r = (i / VPR) % (2 * NPC), q = i % VPR;
      if (i >= NITEM || r >= N) continue;
      const Tin *src = (which ? gC : gB) + (int64_t)r * L;
      const int64_t t = t0 + (int64_t)q * EPV;
      if (vec) {
        if (t < L) v[k] = ld_global_l2pf(src + t);  // aligned rows: all EPV steps lie in the row
      } else {
        Tin tmp[EPV];
#pragma unroll
        for (int e = 0; e < EPV; e++) tmp[e] = (t + e < L) ? src[t + e] : from_f32<Tin>(0.0f);
        v[k] = *reinterpret_cast<const uint4 *>(tmp);
      }
    }
  }
  __device__ __forceinline__ void store(float *sm, int NP) const {
#pragma unroll
    for (int k = 0; k < PER; k++) {
      const int i = threadIdx.x + k * kTpThreads;
      const int which = i / (2 * NPC * VPR), r = (i / VPR) % (2 * NPC), q = i % VPR;
      if (i >= NITEM || r >= NP) continue;
      float *dst = sm + ((int64_t)which * NP + r) * kTpChunk + q * EPV;
      const Tin *e = reinterpret_cast<const Tin *>(&v[k]);
#pragma unroll
      for (int j = 0; j < EPV; j += 4)
        *reinterpret_cast<float4 *>(dst + j) = make_float4(to_f32(e[j]), to_f32(e[j + 1]), to_f32(e[j + 2]), to_f32(e[j + 3]));
    }
  }
};

template <int NPC, typename Tin, typename Tout, bool EULER>
__global__ void __launch_bounds__(kTpThreads, 4) ssm_fwd_tp_kernel(const FwdParams p) {
  constexpr bool PRECISE = sizeof(Tin) == 4;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = (int)p.N, NP = (N + 1) & ~1, npair = NP / 2;
  float *bcs = reinterpret_cast<float *>(smem);                        // [2 buffers][B, C][NP][64]
  float *Acs = reinterpret_cast<float *>(smem + TpSmem::coef_off(NP));  // [CH][NP]: A (or A log2 e)
  float *nIAs = Acs + kTpCh * NP;                                      // [CH][NP]: -1/A
  float *carry = reinterpret_cast<float *>(smem + TpSmem::carry_off(NP));  // [CH][NP]: state entering the chunk

  const int tid = threadIdx.x, cl = tid / kTpLanes, li = tid % kTpLanes;
  const int64_t n_ct = (p.Dn + kTpCh - 1) / kTpCh;
  const int64_t b = blockIdx.x / n_ct, d0 = (blockIdx.x % n_ct) * kTpCh, d = d0 + cl;
  const bool live = d < p.Dn;
  const bool has_conv = p.conv_w != nullptr, has_z = p.z != nullptr, vec = p.vec != 0;
  const int64_t L = p.L;

  // per-channel coefficients (padded states inert: A_bar = 1, no input) and the carried state
  for (int i = tid; i < kTpCh * NP; i += kTpThreads) {
    const int c = i / NP, n = i % NP;
    const int64_t dd = d0 + c;
    float Ac = 0.f, nI = 0.f, h = 0.f;
    if (dd < p.Dn && n < N) {
      const float A = -expf(p.A_log[dd * N + n]);
      Ac = PRECISE ? A : A * kLog2e;
      nI = -1.0f / A;
      if (p.h0) h = p.h0[(b * p.Dn + dd) * N + n];
    }
    Acs[i] = Ac;
    nIAs[i] = nI;
    carry[i] = h;
  }
  float w4[4] = {0.f, 0.f, 0.f, 0.f};
  float cbias = 0.f, Dd = 0.f, dtb = 0.f;
  if (live) {
    if (has_conv) {
#pragma unroll
      for (int k = 0; k < 4; k++)
        if (k < p.K) w4[k] = p.conv_w[d * p.K + k];
      cbias = p.conv_b ? p.conv_b[d] : 0.f;
    }
    Dd = p.D ? p.D[d] : 0.f;
    dtb = p.dt_bias ? p.dt_bias[d] : 0.f;
  }
  // the 3 pre-conv inputs before the chunk (x_{t0-1}, x_{t0-2}, x_{t0-3}): the carried history
  // (newest-first), zero where there is none
  const Tin *hist = (has_conv && p.conv_hist && p.K > 1) ? static_cast<const Tin *>(p.conv_hist) : nullptr;
  float hx[3];
#pragma unroll
  for (int j = 0; j < 3; j++)
    hx[j] = (live && hist && j < p.K - 1) ? to_f32(hist[(b * p.Dn + d) * (p.K - 1) + j]) : 0.f;

  const int64_t row = (b * p.Dn + (live ? d : 0)) * L;
  const Tin *gx = static_cast<const Tin *>(p.x) + row;
  const Tin *gdt = static_cast<const Tin *>(p.dt) + row;
  const Tin *gz = has_z ? static_cast<const Tin *>(p.z) + row : nullptr;
  const Tin *gB = static_cast<const Tin *>(p.B) + b * p.N * L;
  const Tin *gC = static_cast<const Tin *>(p.C) + b * p.N * L;

  const int64_t nck = (L + kTpChunk - 1) / kTpChunk;
  TpBCStager<Tin, NPC> bc;
  bc.load(gB, gC, N, NP, 0, L, vec);
  bc.store(bcs, NP);
  if (nck > 1) bc.load(gB, gC, N, NP, kTpChunk, L, vec);

  for (int64_t ck = 0; ck < nck; ck++) {
    const int buf = (int)(ck & 1);
    __syncthreads();  // chunk ck's rows are in place; every thread is done with chunk ck-1's buffer
    if (ck + 1 < nck) {
      bc.store(bcs + (buf ^ 1) * 2 * NP * kTpChunk, NP);
      if (ck + 2 < nck) bc.load(gB, gC, N, NP, (ck + 2) * kTpChunk, L, vec);
    }
    const float *Bsm = bcs + buf * 2 * NP * kTpChunk, *Csm = Bsm + NP * kTpChunk;
    const int64_t tl = ck * kTpChunk + li * kTpT;  // this lane's first step

    // ---- per-element work of the lane's 8 steps, in registers
    float xv[kTpT], dv[kTpT], zv[kTpT];
    if (live) {
      load8(xv, gx, tl, L, vec);
      load8(dv, gdt, tl, L, vec);
      if (has_z) load8(zv, gz, tl, L, vec);
    } else {
#pragma unroll
      for (int i = 0; i < kTpT; i++) xv[i] = dv[i] = 0.f;
    }
    // x_{tl-3..tl-1}: the previous lane's last three, or the previous chunk's for the first lane
    float xe[kTpT + 3];
    xe[2] = __shfl_up_sync(FULL, xv[7], 1, kTpLanes);
    xe[1] = __shfl_up_sync(FULL, xv[6], 1, kTpLanes);
    xe[0] = __shfl_up_sync(FULL, xv[5], 1, kTpLanes);
    if (li == 0) {
      xe[2] = hx[0];
      xe[1] = hx[1];
      xe[0] = hx[2];
    }
    hx[0] = __shfl_sync(FULL, xv[7], kTpLanes - 1, kTpLanes);
    hx[1] = __shfl_sync(FULL, xv[6], kTpLanes - 1, kTpLanes);
    hx[2] = __shfl_sync(FULL, xv[5], kTpLanes - 1, kTpLanes);
#pragma unroll
    for (int i = 0; i < kTpT; i++) xe[i + 3] = xv[i];
    float u[kTpT], dl[kTpT];
#pragma unroll
    for (int i = 0; i < kTpT; i++) {
      if (has_conv) {
        float acc = cbias;
#pragma unroll
        for (int k = 0; k < 4; k++) acc = fmaf(w4[k], xe[i + 3 - k], acc);
        u[i] = acc * sigmoid<PRECISE>(acc);
      } else {
        u[i] = xv[i];
      }
      const float v = dv[i] + dtb;
      dl[i] = p.delta_softplus ? softplus<PRECISE>(v) : v;
      if (tl + i >= L) {  // padded tail: an identity step
        u[i] = 0.f;
        dl[i] = 0.f;
      }
    }

    // ---- the scan, one pair of states at a time
    float2 y2[kTpT];
#pragma unroll
    for (int i = 0; i < kTpT; i++) y2[i] = make_float2(0.f, 0.f);
#pragma unroll 1
    for (int q = 0; q < npair; q++) {
      const float2 Ac2 = *reinterpret_cast<const float2 *>(Acs + cl * NP + 2 * q);
      const float2 nI2 = *reinterpret_cast<const float2 *>(nIAs + cl * NP + 2 * q);
      const float *b0 = Bsm + (2 * q) * kTpChunk + li * kTpT, *b1 = b0 + kTpChunk;
      // (1) the lane's steps from a zero state: local states and running products of A_bar
      float2 hl[kTpT], cp[kTpT];
      float2 h2 = make_float2(0.f, 0.f), P2 = make_float2(1.f, 1.f);
#pragma unroll
      for (int i4 = 0; i4 < kTpT; i4 += 4) {
        const float4 bA = *reinterpret_cast<const float4 *>(b0 + i4);
        const float4 bB = *reinterpret_cast<const float4 *>(b1 + i4);
        const float ba[4] = {bA.x, bA.y, bA.z, bA.w}, bb[4] = {bB.x, bB.y, bB.z, bB.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
          const int i = i4 + k;
          const float2 Bi = make_float2(ba[k], bb[k]);
          if (PRECISE) {
            const float e0 = expm1f(dl[i] * Ac2.x), e1 = expm1f(dl[i] * Ac2.y);  // A_bar - 1
            if (EULER) {
              h2.x = fmaf(e0, h2.x, fmaf(dl[i] * Bi.x, u[i], h2.x));
              h2.y = fmaf(e1, h2.y, fmaf(dl[i] * Bi.y, u[i], h2.y));
            } else {
              const float w0 = Bi.x * u[i] * nI2.x, w1 = Bi.y * u[i] * nI2.y;  // -B u / A
              h2.x = fmaf(e0, h2.x - w0, h2.x);
              h2.y = fmaf(e1, h2.y - w1, h2.y);
            }
            P2.x = fmaf(e0, P2.x, P2.x);
            P2.y = fmaf(e1, P2.y, P2.y);
          } else {
            const float2 x2 = __fmul2_rn(make_float2(dl[i], dl[i]), Ac2);
            const float2 a2 = make_float2(ex2_approx(x2.x), ex2_approx(x2.y));
            const float2 u2 = make_float2(u[i], u[i]);
            if (EULER) {
              h2 = __ffma2_rn(a2, h2, __fmul2_rn(__fmul2_rn(Bi, u2), make_float2(dl[i], dl[i])));
            } else {
              const float2 nw = __fmul2_rn(__fmul2_rn(Bi, u2), nI2);                   // -B u / A
              h2 = __ffma2_rn(a2, __ffma2_rn(nw, make_float2(-1.f, -1.f), h2), nw);  // a (h + w) - w
            }
            P2 = __fmul2_rn(P2, a2);
          }
          hl[i] = h2;
          cp[i] = P2;
        }
      }
      // (2) inclusive scan of the lanes' (P, H) over the group: (P1, H1) then (P2, H2) is
      //     (P2 P1, P2 H1 + H2)
      float2 Hs = h2, Ps = P2;
#pragma unroll
      for (int off = 1; off < kTpLanes; off <<= 1) {
        const float2 Hp = make_float2(__shfl_up_sync(FULL, Hs.x, off, kTpLanes), __shfl_up_sync(FULL, Hs.y, off, kTpLanes));
        const float2 Pp = make_float2(__shfl_up_sync(FULL, Ps.x, off, kTpLanes), __shfl_up_sync(FULL, Ps.y, off, kTpLanes));
        if (li >= off) {
          Hs = __ffma2_rn(Ps, Hp, Hs);
          Ps = __fmul2_rn(Ps, Pp);
        }
      }
      float2 He = make_float2(__shfl_up_sync(FULL, Hs.x, 1, kTpLanes), __shfl_up_sync(FULL, Hs.y, 1, kTpLanes));
      float2 Pe = make_float2(__shfl_up_sync(FULL, Ps.x, 1, kTpLanes), __shfl_up_sync(FULL, Ps.y, 1, kTpLanes));
      if (li == 0) {
        He = make_float2(0.f, 0.f);
        Pe = make_float2(1.f, 1.f);
      }
      float2 *cq = reinterpret_cast<float2 *>(carry + cl * NP + 2 * q);
      const float2 hc = *cq;
      const float2 hin = __ffma2_rn(Pe, hc, He);  // state entering this lane's steps
      __syncwarp();                               // the group has read the carry
      if (li == kTpLanes - 1) *cq = __ffma2_rn(Ps, hc, Hs);  // state after the chunk
      // (3) the lane's states from the state entering them, and the readout
      const float *c0 = Csm + (2 * q) * kTpChunk + li * kTpT, *c1 = c0 + kTpChunk;
#pragma unroll
      for (int i4 = 0; i4 < kTpT; i4 += 4) {
        const float4 cA = *reinterpret_cast<const float4 *>(c0 + i4);
        const float4 cB = *reinterpret_cast<const float4 *>(c1 + i4);
        const float ca[4] = {cA.x, cA.y, cA.z, cA.w}, cb[4] = {cB.x, cB.y, cB.z, cB.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
          const int i = i4 + k;
          const float2 h = __ffma2_rn(cp[i], hin, hl[i]);
          y2[i] = __ffma2_rn(make_float2(ca[k], cb[k]), h, y2[i]);
        }
      }
      // saved states: after every SSM_STATE_CHUNK = 16 steps, i.e. at the end of odd lanes (the
      // last entry is the state after step L-1: padded steps are identity steps)
      if (p.chunk_states && live && (li & 1) && tl - kTpT < L) {
        const float2 he = __ffma2_rn(cp[kTpT - 1], hin, hl[kTpT - 1]);
        const int64_t kk = (tl - kTpT) / kSub;
        float *dst = p.chunk_states + ((b * p.Dn + d) * p.n_ck + kk) * N + 2 * q;
        dst[0] = he.x;
        if (2 * q + 1 < N) dst[1] = he.y;
      }
    }

    // ---- D skip, gate, store
    float o[kTpT];
#pragma unroll
    for (int i = 0; i < kTpT; i++) {
      const float s = has_z ? zv[i] * sigmoid<PRECISE>(zv[i]) : 1.f;
      o[i] = fmaf(Dd, u[i], y2[i].x + y2[i].y) * s;
    }
    if (live && p.out) store8<Tout>(static_cast<Tout *>(p.out) + row, tl, L, o, vec);
    if (live && p.u_out) store8<Tout>(static_cast<Tout *>(p.u_out) + row, tl, L, u, vec);
  }
  __syncthreads();  // the last chunk's carry is written
  if (live && p.h_last)
    for (int n = li; n < N; n += kTpLanes) p.h_last[(b * p.Dn + d) * N + n] = carry[cl * NP + n];
  // the K-1 newest pre-conv inputs, newest-first; read everything before writing (the output may
  // alias the input history)
  if (live && has_conv && p.conv_hist_out && p.K > 1 && li == 0) {
    const Tin *hr = hist ? hist + (b * p.Dn + d) * (p.K - 1) : nullptr;
    Tin v[3];
#pragma unroll
    for (int j = 0; j < 3; j++) {
      const int64_t t = L - 1 - j;
      v[j] = zero_val<Tin>();
      if (j < p.K - 1) v[j] = (t >= 0) ? gx[t] : (hr ? hr[j - L] : zero_val<Tin>());
    }
    Tin *o = static_cast<Tin *>(p.conv_hist_out) + (b * p.Dn + d) * (p.K - 1);
#pragma unroll
    for (int j = 0; j < 3; j++)
      if (j < p.K - 1) o[j] = v[j];
  }
}

// ---- host side -----------------------------------------------------------------------------

template <int NPC, typename Tin, typename Tout>
static cudaError_t launch_tp_t(const FwdParams &p, cudaStream_t stream) {
  auto kern = p.euler ? ssm_fwd_tp_kernel<NPC, Tin, Tout, true> : ssm_fwd_tp_kernel<NPC, Tin, Tout, false>;
  const int NP = (int)((p.N + 1) & ~int64_t(1));
  const size_t smem = TpSmem::bytes(NP);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (p.Dn + kTpCh - 1) / kTpCh * p.Bt;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<(unsigned)grid, kTpThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
static cudaError_t launch_tp_n(const FwdParams &p, cudaStream_t stream) {
  if (p.N <= 16) return launch_tp_t<8, Tin, Tout>(p, stream);
  return launch_tp_t<32, Tin, Tout>(p, stream);
}

// One pass of the time-parallel forward (no split-L fields are read).
cudaError_t launch_fwd_tp(const FwdParams &p, int in_bf16, int out_bf16, cudaStream_t stream) {
  if (in_bf16)
    return out_bf16 ? launch_tp_n<__nv_bfloat16, __nv_bfloat16>(p, stream) : launch_tp_n<__nv_bfloat16, float>(p, stream);
  return out_bf16 ? launch_tp_n<float, __nv_bfloat16>(p, stream) : launch_tp_n<float, float>(p, stream);
}

}  // namespace ssm
