// ssm_ssd.cu -- Mamba-2 state-space duality (SSD) forward on the sm_100a tensor cores.
//
// "state-space models" (aarnphm.xyz), "Mamba-2 and state-space duality": within a head the
// transition is a_t I, so y_t = sum_{s<=t} (C_t . B-bar_s)(prod_{k=s+1..t} a_k) x_s, i.e.
// Y = (L o Q K^T) V, computed by matrix products within chunks while a state is carried between
// chunks. With cum_t the running sum of log a over a chunk of Q steps and B-bar_s = beta_s B_s:
//
//   S_c      = sum_s e^{cum_end - cum_s} beta_s B_s x_s^T                  (N x P, chunk state)
//   H_c      = e^{cum_end} H_{c-1} + S_c                                   (state after chunk c)
//   Y_c[t]   = sum_{s<=t} (C_t . B_s) e^{cum_t - cum_s} beta_s x_s  +  e^{cum_t} C_t H_{c-1}
//              + D x_t
//
// Three kernels: ssd_state_kernel (S_c, one tcgen05 product per chunk and head), ssd_pass_kernel
// (the carry over chunks, fp32, CUDA cores), ssd_out_kernel (C B^T and C H_{c-1} on the tensor
// cores, the masked decay applied to C B^T in registers, then the product with X). The state and
// output kernels take a group of up to 8 heads per CTA, since B, C and C B^T do not depend on the
// head. Operands are bf16 in shared memory in the canonical no-swizzle layouts (8 x 16-byte core
// matrices); accumulators are fp32 in tensor memory with M = 128, so accumulator row i is TMEM
// lane i. A CTA has 256 threads: threads i and i + 128 (warps w and w + 4 reach the same 32 lanes)
// own row i and split its columns. One elected thread issues the MMAs; completion is signalled
// through an mbarrier whose wait is bounded (on a timeout the kernel records an error and still
// frees its tensor memory).
#include "ssm_common.cuh"
#include "ssm_internal.h"
#include "ssm_stage.cuh"
#include "ssm_tc.cuh"
#include "ssm_tmem.cuh"

namespace ssm {

namespace {

constexpr int kQ = 128;   // chunk length (steps)
constexpr int kNP = 128;  // padded state dimension (N = 64 runs with zero rows)
constexpr int kSsdHeader = 2048;  // bytes of small per-CTA data in front of the tiles
constexpr int kHGMax = 8;         // heads per CTA at most (they share B, C and C B^T)
constexpr int kCoefBytes = 3 * kHGMax * kQ * 4;  // output kernel: q, ct, e^{cum} of every head

// One 16-byte chunk of outputs into shared memory: 8 values as bf16, or 4 as fp32.
__device__ __forceinline__ void put16(unsigned char *dst, const float *v, __nv_bfloat16 *) {
  *reinterpret_cast<uint4 *>(dst) = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                               pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
}
__device__ __forceinline__ void put16(unsigned char *dst, const float *v, float *) {
  *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}

// Threads per CTA of the chunk-state and output kernels: two threads per tensor-memory lane (warps
// w and w + 4 reach the same 32 lanes), each taking half of the row's columns.
constexpr int kThr = 256;

// Cooperative asynchronous copy (cp.async, 16 bytes) of a tile of R rows x VPR 16-byte vectors
// (8 bf16 each) from a row-major source into an operand tile: vector (row, v) goes to
// smem_off(row, v). Row r of the source starts at src + r * rs elements; rows with valid(r) false,
// and vectors past vmax, are zero-filled with plain stores. A warp takes 8 rows x 4 vectors: 64
// contiguous bytes per row from global memory, and the 8 lanes of each shared-memory phase write 8
// different core-matrix rows (distinct banks). The caller commits, waits and fences.
template <int R, int VPR, typename Off, typename Valid>
__device__ __forceinline__ void coop_tile_async(unsigned char *tile, const __nv_bfloat16 *src,
                                                int64_t rs, int vmax, Off smem_off, Valid valid) {
  static_assert(R % 8 == 0 && (R * VPR) % kThr == 0, "tile shape");
#pragma unroll 4
  for (int it = 0; it < R * VPR / kThr; it++) {
    const int idx = it * kThr + threadIdx.x;
    const int r8 = idx & 7, v = (idx >> 3) % VPR, rg = (idx >> 3) / VPR;
    const int row = rg * 8 + r8;
    unsigned char *dst = tile + smem_off(row, v);
    if (valid(row) && v < vmax)
      cp_async16(dst, src + (int64_t)row * rs + v * 8);
    else
      *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// This thread's lane of the CTA's tensor memory: row (threadIdx.x mod 128), column 0.
__device__ __forceinline__ uint32_t ssd_lane_addr(uint32_t tbase) {
  return tbase + (static_cast<uint32_t>(threadIdx.x & 96) << 16);
}

}  // namespace

// ---- kernel 1: chunk states S_c = (w beta B)^T X -------------------------------------------
// One CTA per (batch, chunk, group of HG <= 8 heads). B_c is shared by the heads: every thread
// keeps its share of the raw tile in registers and, per head, writes it scaled by that head's
// row weights e^{cum_end - cum_s} beta_s as the A operand. X of the next head is copied into a
// second buffer while the current head's product runs. Thread t owns accumulator row t mod 128
// (state n) and half of its P columns.
template <int P>
__global__ void __launch_bounds__(kThr, 2) ssd_state_kernel(const SsdParams p, int HG) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float *scan_buf = reinterpret_cast<float *>(smem);  // header: kHGMax x 4 warp sums, cum_end per head
  float *cend_s = scan_buf + kHGMax * 4;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kSsdHeader - 16);
  uint32_t *slot = reinterpret_cast<uint32_t *>(smem + kSsdHeader - 8);
  float *scale_s = reinterpret_cast<float *>(smem + kSsdHeader);       // [head][step]
  unsigned char *sA = smem + kSsdHeader + kHGMax * kQ * 4;             // M = n (128), K = s, MN-major
  unsigned char *sX0 = sA + kNP * kQ * 2;                              // N = p (P), K = s, MN-major; x2

  constexpr uint32_t kCols = P < 32 ? 32u : (uint32_t)P;
  constexpr int VPR = kNP / 8;                   // 16-byte vectors per row of B
  constexpr int NV = kQ * VPR / kThr;            // vectors of B per thread
  constexpr int HH = kHGMax / 2;                 // heads per thread in the coefficient pass
  const int64_t nC = (p.L + kQ - 1) / kQ;
  const int64_t ngrp = p.H / HG;
  const int64_t c = blockIdx.x % nC, rest = blockIdx.x / nC;
  const int64_t hgrp = rest % ngrp, b = rest / ngrp;
  const int t = threadIdx.x, r = t & 127, hf = t >> 7, wq = (t >> 5) & 3;
  const int64_t rows_left = p.L - c * kQ;
  auto valid = [&](int row) { return row < rows_left; };
  auto load_x = [&](int hi) {
    const int64_t bh = b * p.H + hgrp * HG + hi;
    coop_tile_async<kQ, P / 8>(sX0 + (hi & 1) * P * kQ * 2,
                               static_cast<const __nv_bfloat16 *>(p.x) + (bh * p.L + c * kQ) * P, P, P / 8,
                               [](int row, int v) { return mnmaj_off(P, v * 8, row); }, valid);
    cp_async_commit();
  };

  const uint32_t tbase = tmem_alloc_cta(slot, kCols);
  if (t == 0) mbar_init(bar, 1);
  load_x(0);
  // row weights: thread (r, hf) takes step r of heads hf, hf + 2, ...
  {
    const int64_t tg = c * kQ + r;
    float beta[HH], sc[HH];
#pragma unroll
    for (int j = 0; j < HH; j++) {
      const int hi = 2 * j + hf;
      float la = 0.f;
      beta[j] = 0.f;
      if (hi < HG && tg < p.L) {
        const int64_t h = hgrp * HG + hi;
        const float A = -expf(p.A_log[h]);
        const float v = to_f32(static_cast<const __nv_bfloat16 *>(p.dt)[(b * p.H + h) * p.L + tg]) +
                        (p.dt_bias ? p.dt_bias[h] : 0.f);
        const float dl = p.delta_softplus ? softplus<false>(v) : v;
        la = dl * A;
        beta[j] = p.euler ? dl : expm1f(la) / A;  // 0 past the sequence end: identity steps
      }
      sc[j] = la;
    }
    const int lane = t & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
      for (int j = 0; j < HH; j++) {
        const float o = __shfl_up_sync(0xffffffffu, sc[j], off);
        if (lane >= off) sc[j] += o;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int j = 0; j < HH; j++) scan_buf[(2 * j + hf) * 4 + wq] = sc[j];
    }
    __syncthreads();
    if (t < HG) cend_s[t] = scan_buf[t * 4] + scan_buf[t * 4 + 1] + scan_buf[t * 4 + 2] + scan_buf[t * 4 + 3];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < HH; j++) {
      const int hi = 2 * j + hf;
      if (hi < HG) {
        float base = 0.f;
        for (int i = 0; i < wq; i++) base += scan_buf[hi * 4 + i];
        scale_s[hi * kQ + r] = beta[j] * __expf(cend_s[hi] - (sc[j] + base));  // e^{cum_end - cum_s} beta_s
      }
    }
    if (t < HG) p.cum_end[(b * p.H + hgrp * HG + t) * nC + c] = cend_s[t];
  }
  // this thread's vectors of the raw B tile (rows past the sequence end and n >= N read as zero)
  uint4 braw[NV];
  {
    const __nv_bfloat16 *Bsrc = static_cast<const __nv_bfloat16 *>(p.B) + (b * p.L + c * kQ) * p.N;
    const int vmax = (int)(p.N / 8);
#pragma unroll
    for (int it = 0; it < NV; it++) {
      const int idx = it * kThr + t;
      const int row = ((idx >> 3) / VPR) * 8 + (idx & 7), v = (idx >> 3) % VPR;
      braw[it] = (valid(row) && v < vmax) ? *reinterpret_cast<const uint4 *>(Bsrc + (int64_t)row * p.N + v * 8)
                                          : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __syncthreads();  // the row weights of every head are in place

  bool ok = true;
  const uint32_t lane_addr = ssd_lane_addr(tbase);
  for (int hi = 0; hi < HG; hi++) {
    const int64_t bh = b * p.H + hgrp * HG + hi;
    const unsigned char *sX = sX0 + (hi & 1) * P * kQ * 2;
    // A operand of this head: row s of B times its weight, MN-major along n
    {
      const float *wts = scale_s + hi * kQ;
#pragma unroll
      for (int it = 0; it < NV; it++) {
        const int idx = it * kThr + t;
        const int row = ((idx >> 3) / VPR) * 8 + (idx & 7), v = (idx >> 3) % VPR;
        const float sw = wts[row];
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&braw[it]);
        uint4 o;
        uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const float2 f = __bfloat1622float2(h2[i]);
          ow[i] = pack_bf16(f.x * sw, f.y * sw);
        }
        *reinterpret_cast<uint4 *>(sA + mnmaj_off(kNP, v * 8, row)) = o;
      }
    }
    cp_async_wait<0>();  // this thread's copies of this head's X landed
    tc_fence_before();
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
      constexpr uint32_t idesc = instr_desc(128, P, 1, 1);
#pragma unroll
      for (int ks = 0; ks < kQ / 16; ks++) {
        const uint64_t da = smem_desc(sA + ks * 2 * (kNP / 8) * 128, (kNP / 8) * 128, 128);
        const uint64_t db = smem_desc(sX + ks * 2 * (P / 8) * 128, (P / 8) * 128, 128);
        mma_bf16(tbase, da, db, idesc, ks > 0);
      }
      mma_commit(bar);
    }
    // the other X buffer was read by the previous head's product, which has completed
    if (hi + 1 < HG) load_x(hi + 1);
    ok = __all_sync(0xffffffffu, mbar_wait(bar, (uint32_t)(hi & 1))) && ok;
    tc_fence_after();
    // S_c leaves through the consumed A tile, 64 columns at a time: thread (r, hf) parks its 32
    // columns of row r as 16-byte chunks at slot (chunk ^ (r mod 16)) -- no bank conflicts -- and
    // the CTA then writes whole rows (256 contiguous bytes) to global memory; rows n >= N are padding
    {
      float *stage = reinterpret_cast<float *>(sA);  // 128 rows x 64 floats
      float *dst = p.S + (bh * nC + c) * p.N * P;
#pragma unroll 1
      for (int q0 = 0; q0 < P; q0 += 64) {
        float v[32];
        tmem_ld32(lane_addr + q0 + hf * 32, v);
#pragma unroll
        for (int i = 0; i < 8; i++) {
          const int slot = (hf * 8 + i) ^ (r & 15);
          *reinterpret_cast<float4 *>(stage + r * 64 + slot * 4) = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < 128 * 16 / kThr; it++) {
          const int idx = it * kThr + t, row = idx >> 4, j = idx & 15;
          if (ok && row < p.N)
            *reinterpret_cast<float4 *>(dst + (int64_t)row * P + q0 + j * 4) =
                *reinterpret_cast<const float4 *>(stage + row * 64 + ((j ^ (row & 15)) * 4));
        }
        __syncthreads();  // the stage (the A tile) is rewritten next
      }
    }
  }
  if (!ok && (t & 31) == 0) atomicExch(p.error, 1);
  tc_fence_before();
  tmem_free_cta(tbase, kCols);
}

// ---- kernel 2: carry over chunks ------------------------------------------------------------
// H_in[c] = state entering chunk c (bf16, the MMA operand of kernel 3); H_c = e^{cum_end} H + S_c.
template <int P>
__global__ void __launch_bounds__(256) ssd_pass_kernel(const SsdParams p) {
  // grid: (batch x head) x (N P / 1024); each thread carries 4 consecutive state entries
  const int64_t nC = (p.L + kQ - 1) / kQ;
  const int64_t NPs = p.N * P;
  const int64_t per = NPs / 1024;
  const int64_t bh = blockIdx.x / per;
  const int64_t e = (blockIdx.x % per) * 1024 + threadIdx.x * 4;
  float4 hcur = p.h0 ? *reinterpret_cast<const float4 *>(p.h0 + bh * NPs + e) : make_float4(0.f, 0.f, 0.f, 0.f);
  const float *S = p.S + bh * nC * NPs + e;
  __nv_bfloat16 *Hin = p.Hin + bh * nC * NPs + e;
  const float *ce = p.cum_end + bh * nC;
#pragma unroll 4
  for (int64_t c = 0; c < nC; c++) {
    const float4 sv = *reinterpret_cast<const float4 *>(S + c * NPs);
    const float a = __expf(ce[c]);
    uint2 pk;
    pk.x = pack_bf16(hcur.x, hcur.y);
    pk.y = pack_bf16(hcur.z, hcur.w);
    *reinterpret_cast<uint2 *>(Hin + c * NPs) = pk;
    hcur = make_float4(fmaf(a, hcur.x, sv.x), fmaf(a, hcur.y, sv.y), fmaf(a, hcur.z, sv.z), fmaf(a, hcur.w, sv.w));
  }
  if (p.h_last) *reinterpret_cast<float4 *>(p.h_last + bh * NPs + e) = hcur;
}

// ---- kernel 3: chunk outputs ------------------------------------------------------------------
// One CTA per (batch, chunk, group of HG <= 8 heads): C and B are shared by the heads, so they are
// staged once and G = C B^T is formed once; each head then applies its own decays to G.
//
// The decay of score (t, s) is written e^{cum_t - cum_s} beta_s = 2^{ct_t - q_s} with
// ct_t = cum_t log2 e and q_s = cum_s log2 e - log2 beta_s, both computed once per step and head
// (beta_s = 0 gives q_s = +inf and a zero score). The skip term D x_t is the diagonal of the
// product G' X, so it is added to G'[t][t] rather than re-reading x. Scores above the diagonal are
// zero for every head: those blocks are cleared once and never rewritten. Thread t owns row
// t mod 128 of every accumulator and half of its columns.
template <int P, typename Tout>
__global__ void __launch_bounds__(kThr, 2) ssd_out_kernel(const SsdParams p, int HG) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float *scan_buf = reinterpret_cast<float *>(smem);  // header: kHGMax x 4 warp sums, D per head
  float *Dh_s = scan_buf + kHGMax * 4;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kSsdHeader - 24);  // two barriers
  uint32_t *slot = reinterpret_cast<uint32_t *>(smem + kSsdHeader - 8);
  float *q_s = reinterpret_cast<float *>(smem + kSsdHeader);  // [head][step]
  float *ct_s = q_s + kHGMax * kQ;
  float *et_s = ct_s + kHGMax * kQ;
  unsigned char *sC = smem + kSsdHeader + kCoefBytes;  // C: M = t (128), K = n (128), K-major
  unsigned char *sB = sC + kQ * kNP * 2;  // B: N = s, K = n, K-major; then each head's G' (K = s)
  unsigned char *sX = sB + kQ * kNP * 2;  // X: N = p (P), K = s (128), MN-major
  unsigned char *sH = sX + P * kQ * 2;    // H_in: N = p (P), K = n (128), MN-major

  constexpr uint32_t kCols = (128 + 2 * P <= 256) ? 256u : 512u;  // G (128) + Y (P) + C H (P)
  constexpr int HH = kHGMax / 2;  // heads per thread in the coefficient pass
  const int64_t nC = (p.L + kQ - 1) / kQ;
  const int64_t ngrp = p.H / HG;
  const int64_t c = blockIdx.x % nC, rest = blockIdx.x / nC;
  const int64_t hgrp = rest % ngrp, b = rest / ngrp;
  const int t = threadIdx.x, r = t & 127, hf = t >> 7, wq = (t >> 5) & 3;
  const int64_t rows_left = p.L - c * kQ;
  auto valid = [&](int row) { return row < rows_left; };
  const int nks = (int)((p.N + 15) / 16);  // K slices of C H that are not all zero padding
  auto load_xh = [&](int hi) {  // this head's X and H_in tiles, asynchronously
    const int64_t bh = b * p.H + hgrp * HG + hi;
    const auto mnmaj = [](int row, int v) { return mnmaj_off(P, v * 8, row); };
    coop_tile_async<kQ, P / 8>(sX, static_cast<const __nv_bfloat16 *>(p.x) + (bh * p.L + c * kQ) * P, P, P / 8, mnmaj, valid);
    const int64_t nrows = p.N;
    coop_tile_async<kNP, P / 8>(sH, p.Hin + (bh * nC + c) * p.N * P, P, P / 8, mnmaj, [&](int row) { return row < nrows; });
    cp_async_commit();
  };

  const uint32_t tbase = tmem_alloc_cta(slot, kCols);
  if (t == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
  }
  {
    // C and B first (one group), then the first head's X and H_in (a second group): every copy is
    // in flight at once, and only the first group is waited for before C B^T
    const int64_t off = (b * p.L + c * kQ) * p.N;
    const auto kmaj = [](int row, int v) { return kmaj_off(kQ, row, v * 8); };
    coop_tile_async<kQ, kNP / 8>(sC, static_cast<const __nv_bfloat16 *>(p.C) + off, p.N, (int)(p.N / 8), kmaj, valid);
    coop_tile_async<kQ, kNP / 8>(sB, static_cast<const __nv_bfloat16 *>(p.B) + off, p.N, (int)(p.N / 8), kmaj, valid);
    cp_async_commit();
  }
  load_xh(0);
  cp_async_wait<1>();
  fence_async_smem();
  __syncthreads();
  tc_fence_after();
  const uint32_t tG = tbase, tY = tbase + 128, tCH = tbase + 128 + P;
  if (t == 0) {
#pragma unroll
    for (int ks = 0; ks < kNP / 16; ks++) {
      const uint64_t dc = smem_desc(sC + ks * 2 * (kQ / 8) * 128, (kQ / 8) * 128, 128);
      const uint64_t dbm = smem_desc(sB + ks * 2 * (kQ / 8) * 128, (kQ / 8) * 128, 128);
      mma_bf16(tG, dc, dbm, instr_desc(128, 128, 0, 0), ks > 0);
    }
    mma_commit(bar);
  }

  // while G is formed: the decay coefficients, thread (r, hf) taking step r of heads hf, hf + 2, ...
  {
    const int64_t tg = c * kQ + r;
    float beta[HH], sc[HH];
#pragma unroll
    for (int j = 0; j < HH; j++) {
      const int hi = 2 * j + hf;
      float la = 0.f;
      beta[j] = 0.f;
      if (hi < HG && tg < p.L) {
        const int64_t h = hgrp * HG + hi;
        const float A = -expf(p.A_log[h]);
        const float v = to_f32(static_cast<const __nv_bfloat16 *>(p.dt)[(b * p.H + h) * p.L + tg]) +
                        (p.dt_bias ? p.dt_bias[h] : 0.f);
        const float dl = p.delta_softplus ? softplus<false>(v) : v;
        la = dl * A;
        beta[j] = p.euler ? dl : expm1f(la) / A;  // 0 past the sequence end: identity steps
      }
      sc[j] = la;
    }
    // inclusive scan of log a over the chunk (the 4 warps of this thread's half)
    const int lane = t & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
      for (int j = 0; j < HH; j++) {
        const float o = __shfl_up_sync(0xffffffffu, sc[j], off);
        if (lane >= off) sc[j] += o;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int j = 0; j < HH; j++) scan_buf[(2 * j + hf) * 4 + wq] = sc[j];
    }
    if (t < HG) Dh_s[t] = p.D ? p.D[hgrp * HG + t] : 0.f;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < HH; j++) {
      const int hi = 2 * j + hf;
      if (hi < HG) {
        float base = 0.f;
        for (int i = 0; i < wq; i++) base += scan_buf[hi * 4 + i];
        const float cum = sc[j] + base;
        q_s[hi * kQ + r] = cum * kLog2e - lg2_approx(beta[j]);
        ct_s[hi * kQ + r] = cum * kLog2e;
        et_s[hi * kQ + r] = __expf(cum);
      }
    }
  }
  bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0));
  tc_fence_after();
  // B is consumed: clear this thread's half of the score blocks above the diagonal, once
#pragma unroll
  for (int kb = 1; kb < 4; kb++)
    if (kb > wq) {
      *reinterpret_cast<uint4 *>(sB + kmaj_off(kQ, r, kb * 32 + hf * 16)) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4 *>(sB + kmaj_off(kQ, r, kb * 32 + hf * 16 + 8)) = make_uint4(0u, 0u, 0u, 0u);
    }
  __syncthreads();  // the coefficients of every head are in place

  uint32_t phase = 0;  // of bar + 1, one completion per head
  const uint32_t lane_addr = ssd_lane_addr(tbase);
  for (int hi = 0; hi < HG; hi++) {
    const int64_t h = hgrp * HG + hi, bh = b * p.H + h;
    // G'[t][s] = G[t][s] 2^{ct_t - q_s} for s <= t (+ D on the diagonal): the A operand of G' X;
    // this thread: row r, the 16 columns hf*16.. of every block on or below the diagonal
    {
      const float ct = ct_s[hi * kQ + r], Dh = Dh_s[hi];
      const float *qh = q_s + hi * kQ;
#pragma unroll 1
      for (int kb = 0; kb < 4; kb++) {
        if (kb > wq) break;  // warp-uniform: the blocks above the diagonal stay zero
        const int s0 = kb * 32 + hf * 16;
        float g[16];
        tmem_ld2<8>(lane_addr + s0, g, lane_addr + s0 + 8, g + 8);
        const bool diag = kb == wq;
#pragma unroll
        for (int e = 0; e < 16; e += 8) {
          const float4 q0 = *reinterpret_cast<const float4 *>(qh + s0 + e);
          const float4 q1 = *reinterpret_cast<const float4 *>(qh + s0 + e + 4);
          const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
          float v[8];
#pragma unroll
          for (int j = 0; j < 8; j++) {
            const int s = s0 + e + j;
            const float sv = g[e + j] * ex2_approx(ct - qv[j]);
            v[j] = (!diag || s < r) ? sv : (s == r ? sv + Dh : 0.f);
          }
          const uint4 pk = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
          *reinterpret_cast<uint4 *>(sB + kmaj_off(kQ, r, s0 + e)) = pk;
        }
      }
    }
    cp_async_wait<0>();  // this thread's X / H_in copies landed
    tc_fence_before();
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
#pragma unroll
      for (int ks = 0; ks < kQ / 16; ks++) {
        const uint64_t dg = smem_desc(sB + ks * 2 * (kQ / 8) * 128, (kQ / 8) * 128, 128);
        const uint64_t dx = smem_desc(sX + ks * 2 * (P / 8) * 128, (P / 8) * 128, 128);
        mma_bf16(tY, dg, dx, instr_desc(128, P, 0, 1), ks > 0);
      }
      for (int ks = 0; ks < nks; ks++) {
        const uint64_t dc = smem_desc(sC + ks * 2 * (kQ / 8) * 128, (kQ / 8) * 128, 128);
        const uint64_t dh = smem_desc(sH + ks * 2 * (P / 8) * 128, (P / 8) * 128, 128);
        mma_bf16(tCH, dc, dh, instr_desc(128, P, 0, 1), ks > 0);
      }
      mma_commit(bar + 1);
    }
    ok = __all_sync(0xffffffffu, mbar_wait(bar + 1, phase)) && ok;
    phase ^= 1u;
    tc_fence_after();
    // the products have read X, H_in and G': the next head's tiles travel during this epilogue
    if (hi + 1 < HG) load_xh(hi + 1);
    // y = G'X + e^{cum_t} C H_in leaves through the consumed G' tile, W columns at a time (staged
    // rows of at most 256 bytes): thread (r, hf) parks its half of row r as 16-byte chunks at slot
    // (chunk ^ (r mod CPR)) -- no bank conflicts -- and the CTA then writes whole rows to global
    // memory. The zero blocks above the diagonal of G' are cleared again afterwards.
    {
      constexpr int ES = (int)sizeof(Tout);
      constexpr int W = P * ES <= 256 ? P : 256 / ES;  // columns per pass
      constexpr int CPR = W * ES / 16;                 // 16-byte chunks per staged row
      constexpr int EPC = 16 / ES;                     // elements per chunk
      const float et = et_s[hi * kQ + r];
      Tout *yblk = static_cast<Tout *>(p.y) + (bh * p.L + c * kQ) * P;
#pragma unroll 1
      for (int q0 = 0; q0 < P; q0 += W) {
#pragma unroll 1
        for (int q = 0; q < W / 2; q += 32) {
          const int col = q0 + hf * (W / 2) + q;
          float yv[32], cv[32];
          tmem_ld32(lane_addr + 128 + col, yv);
          tmem_ld32(lane_addr + 128 + P + col, cv);
#pragma unroll
          for (int j = 0; j < 32; j++) yv[j] = fmaf(et, cv[j], yv[j]);
#pragma unroll
          for (int i = 0; i < 32 / EPC; i++) {
            const int slot = ((hf * (W / 2) + q) / EPC + i) ^ (r & (CPR - 1));
            put16(sB + r * CPR * 16 + slot * 16, yv + i * EPC, static_cast<Tout *>(nullptr));
          }
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < kQ * CPR / kThr; it++) {
          const int idx = it * kThr + t, row = idx / CPR, j = idx % CPR;
          if (ok && row < rows_left)
            *reinterpret_cast<uint4 *>(yblk + (int64_t)row * P + q0 + j * EPC) =
                *reinterpret_cast<const uint4 *>(sB + row * CPR * 16 + (j ^ (row & (CPR - 1))) * 16);
        }
        __syncthreads();  // the stage is read out
      }
#pragma unroll
      for (int kb = 1; kb < 4; kb++)
        if (kb > wq) {
          *reinterpret_cast<uint4 *>(sB + kmaj_off(kQ, r, kb * 32 + hf * 16)) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4 *>(sB + kmaj_off(kQ, r, kb * 32 + hf * 16 + 8)) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
  }
  if (!ok && (t & 31) == 0) atomicExch(p.error, 1);
  tc_fence_before();
  tmem_free_cta(tbase, kCols);
}

// The timeout path of the bounded wait above, on its own: one CTA waits on an mbarrier that
// expects one arrival; with arrive = 0 nothing arrives, every poll fails, and the CTA records the
// same error word the SSD kernels record. No tensor memory or MMA is involved.
__global__ void __launch_bounds__(128) wait_selftest_kernel(int arrive, int polls, int *error) {
  __shared__ __align__(8) uint64_t bar;
  const int t = threadIdx.x;
  if (t == 0) mbar_init(&bar, 1);
  __syncthreads();
  if (arrive && t == 0) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}\n" ::"r"(a)
                 : "memory");
  }
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar, 0, polls));
  if (!ok && (t & 31) == 0) atomicExch(error, 1);
}

// ---- host ------------------------------------------------------------------------------------

// header + operand tiles, or header + the padded fp32 result rows staged over them
size_t ssd_smem_state(int P) {
  // header, the heads' row weights, the A operand, two X buffers
  return kSsdHeader + (size_t)kHGMax * kQ * 4 + (size_t)kNP * kQ * 2 + (size_t)2 * P * kQ * 2;
}
size_t ssd_smem_out(int P) {
  // header, the heads' decay coefficients, then C, B / G', X, H_in
  return kSsdHeader + kCoefBytes + (size_t)2 * kQ * kNP * 2 + (size_t)P * kQ * 2 + (size_t)P * kNP * 2;
}

template <int P, typename Tout>
static cudaError_t launch_ssd_t(const SsdParams &p, cudaStream_t s) {
  const int64_t nC = (p.L + kQ - 1) / kQ;
  const int64_t grid = p.Bt * p.H * nC;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const size_t s1 = ssd_smem_state(P), s3 = ssd_smem_out(P);
  cudaError_t e = cudaFuncSetAttribute(ssd_state_kernel<P>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(ssd_out_kernel<P, Tout>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3);
  if (e != cudaSuccess) return e;
  int HG = 1;  // heads per CTA: B (and C, C B^T) are shared by them
  for (int cand : {8, 4, 2})
    if (p.H % cand == 0) {
      HG = cand;
      break;
    }
  ssd_state_kernel<P><<<(unsigned)(grid / HG), kThr, s1, s>>>(p, HG);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ssd_pass_kernel<P><<<(unsigned)(p.Bt * p.H * (p.N * P / 1024)), 256, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p.timing_events && p.timing_events[0] &&
      (e = cudaEventRecord(static_cast<cudaEvent_t>(p.timing_events[0]), s)) != cudaSuccess)
    return e;
  ssd_out_kernel<P, Tout><<<(unsigned)(grid / HG), kThr, s3, s>>>(p, HG);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p.timing_events && p.timing_events[1])
    e = cudaEventRecord(static_cast<cudaEvent_t>(p.timing_events[1]), s);
  return e;
}

size_t ssd_workspace_bytes(int64_t Bt, int64_t H, int64_t L, int64_t P, int64_t N) {
  auto rnd = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int64_t nC = (L + kQ - 1) / kQ;
  const size_t chunks = (size_t)(Bt * H * nC);
  return rnd(sizeof(float) * chunks * N * P)               // S
         + rnd(sizeof(__nv_bfloat16) * chunks * N * P)     // H_in
         + rnd(sizeof(float) * chunks)                     // cum_end
         + 256;                                            // error flag
}

size_t ssd_error_offset(int64_t Bt, int64_t H, int64_t L, int64_t P, int64_t N) {
  return ssd_workspace_bytes(Bt, H, L, P, N) - 256;
}

cudaError_t launch_wait_selftest(int arrive, int polls, int *error, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 128, 0, stream>>>(arrive, polls, error);
  return cudaGetLastError();
}

cudaError_t launch_ssd(const SsdParams &p, int out_bf16, cudaStream_t stream) {
  if (p.form != SSM_SSD_THREE_PASS && ssd_fused_supported(p)) {
    const cudaError_t e = launch_ssd_fused(p, out_bf16, stream);
    // the automatic choice takes the three-pass form when the fused one cannot be set up
    if (e != cudaErrorNotSupported || p.form == SSM_SSD_FUSED) return e;
  } else if (p.form == SSM_SSD_FUSED) {
    return cudaErrorInvalidValue;
  }
  if (p.P == 64) return out_bf16 ? launch_ssd_t<64, __nv_bfloat16>(p, stream) : launch_ssd_t<64, float>(p, stream);
  if (p.P == 128) return out_bf16 ? launch_ssd_t<128, __nv_bfloat16>(p, stream) : launch_ssd_t<128, float>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ssm
