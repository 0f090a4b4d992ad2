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
// cores, the masked decay applied to C B^T in registers, then the product with X). Operands are
// bf16 in shared memory in the canonical no-swizzle layouts (8 x 16-byte core matrices);
// accumulators are fp32 in tensor memory with M = 128, so accumulator row i is TMEM lane i and
// thread i of the 128-thread CTA owns it. One elected thread issues the MMAs; completion is
// signalled through an mbarrier whose wait is bounded (on a timeout the kernel records an error
// and still frees its tensor memory).
#include "ssm_common.cuh"
#include "ssm_internal.h"
#include "ssm_stage.cuh"
#include "ssm_tmem.cuh"
#include "ssm_umma.cuh"

namespace ssm {

namespace {

constexpr int kQ = 128;   // chunk length (steps)
constexpr int kNP = 128;  // padded state dimension (N = 64 runs with zero rows)
constexpr int kSsdHeader = 2048;  // bytes of small per-CTA data in front of the tiles

// ---- tcgen05 plumbing ----------------------------------------------------------------------

// Shared-memory matrix descriptor of a no-swizzle operand tile (bit layout in ssm_umma.cuh).
__device__ __forceinline__ uint64_t smem_desc(const void *p, uint32_t lbo, uint32_t sbo) {
  return umma_smem_desc_bits(static_cast<uint32_t>(__cvta_generic_to_shared(p)), lbo, sbo);
}
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, int a_mn_major, int b_mn_major) {
  return umma_instr_desc_bf16_f32(M, N, a_mn_major, b_mn_major);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(a)
               : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");  // visible to the async proxy
}

// Wait for the phase with parity `phase`; gives up after max_polls polls. Returns false on timeout.
// A failed poll suspends the thread for a hardware-chosen time (about 4 us on B200, measured by
// the wait self-test), so the default bound of 2^18 polls gives up after about one second; a
// product completes in microseconds. The result is made warp-uniform by the caller before any
// warp-collective tcgen05 access.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t phase, int max_polls = 1 << 18) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
  for (int i = 0; i < max_polls; i++) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(a), "r"(phase)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t addr, float *v) {
  float a[16], b[16];
  tmem_ld2<16>(addr, a, addr + 16, b);
#pragma unroll
  for (int i = 0; i < 16; i++) {
    v[i] = a[i];
    v[16 + i] = b[i];
  }
}

// Byte offset of element (mn, k) in a no-swizzle operand tile with R rows along M/N; core
// matrices are laid out K-group-major: group (i, j) at (j * R/8 + i) * 128, so sbo = 128 and
// lbo = R / 8 * 128. K-major rows hold 8 consecutive k; MN-major rows hold 8 consecutive mn.
__device__ __forceinline__ uint32_t kmaj_off(int R, int mn, int k) {
  return (uint32_t)(((k >> 3) * (R >> 3) + (mn >> 3)) * 128 + (mn & 7) * 16 + (k & 7) * 2);
}
__device__ __forceinline__ uint32_t mnmaj_off(int R, int mn, int k) {
  return (uint32_t)(((k >> 3) * (R >> 3) + (mn >> 3)) * 128 + (k & 7) * 16 + (mn & 7) * 2);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Cooperative copy of a tile of R rows x VPR 16-byte vectors (8 bf16 each) from a row-major
// source into an operand tile: vector (row, v) goes to smem_off(row, v). Row r of the source
// starts at src + r * rs elements; rows with valid(r) false, and vectors past vmax, read as zero.
// A warp takes 8 rows x 4 vectors: 64 contiguous bytes per row from global memory, and the 8
// lanes of each shared-memory phase write 8 different core-matrix rows (distinct banks).
template <int R, int VPR, typename Off, typename Valid, typename Xform>
__device__ __forceinline__ void coop_tile(unsigned char *tile, const __nv_bfloat16 *src, int64_t rs,
                                          int vmax, Off smem_off, Valid valid, Xform xform) {
  static_assert(R % 8 == 0 && (R * VPR) % 128 == 0, "tile shape");
#pragma unroll 4
  for (int it = 0; it < R * VPR / 128; it++) {
    const int idx = it * 128 + threadIdx.x;
    const int r8 = idx & 7, v = (idx >> 3) % VPR, rg = (idx >> 3) / VPR;
    const int row = rg * 8 + r8;
    uint4 pk = make_uint4(0u, 0u, 0u, 0u);
    if (valid(row) && v < vmax) pk = *reinterpret_cast<const uint4 *>(src + (int64_t)row * rs + v * 8);
    *reinterpret_cast<uint4 *>(tile + smem_off(row, v)) = xform(row, pk);
  }
}
struct NoXform {
  __device__ __forceinline__ uint4 operator()(int, uint4 v) const { return v; }
};
// Same placement, copied asynchronously (cp.async, 16 bytes) with no transform; invalid rows are
// zero-filled with plain stores. The caller commits, waits and fences before the tile is read.
template <int R, int VPR, typename Off, typename Valid>
__device__ __forceinline__ void coop_tile_async(unsigned char *tile, const __nv_bfloat16 *src,
                                                int64_t rs, int vmax, Off smem_off, Valid valid) {
  static_assert(R % 8 == 0 && (R * VPR) % 128 == 0, "tile shape");
#pragma unroll 4
  for (int it = 0; it < R * VPR / 128; it++) {
    const int idx = it * 128 + threadIdx.x;
    const int r8 = idx & 7, v = (idx >> 3) % VPR, rg = (idx >> 3) / VPR;
    const int row = rg * 8 + r8;
    unsigned char *dst = tile + smem_off(row, v);
    if (valid(row) && v < vmax)
      cp_async16(dst, src + (int64_t)row * rs + v * 8);
    else
      *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Delta, log a = Delta A and beta of step t of the chunk (0 past the sequence end: an identity
// step), and the inclusive running sum of log a over the chunk (block-wide scan, 128 threads).
struct StepCoefs {
  float la, beta, cum;
};
__device__ __forceinline__ StepCoefs chunk_coefs(const SsdParams &p, int64_t bh, int64_t t_glob,
                                                 float A, float bias, float *scan_buf) {
  float la = 0.f, beta = 0.f;
  if (t_glob < p.L) {
    const float v = to_f32(static_cast<const __nv_bfloat16 *>(p.dt)[bh * p.L + t_glob]) + bias;
    const float dl = p.delta_softplus ? softplus<false>(v) : v;
    la = dl * A;
    beta = p.euler ? dl : expm1f(la) / A;
  }
  // inclusive scan of la over the 128 threads
  float s = la;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float o = __shfl_up_sync(0xffffffffu, s, off);
    if (lane >= off) s += o;
  }
  if (lane == 31) scan_buf[w] = s;
  __syncthreads();
  float base = 0.f;
  for (int i = 0; i < w; i++) base += scan_buf[i];
  __syncthreads();
  return StepCoefs{la, beta, s + base};
}

}  // namespace

// ---- kernel 1: chunk states S_c = (w beta B)^T X -------------------------------------------
template <int P>
__global__ void __launch_bounds__(128, 1) ssd_state_kernel(const SsdParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  // header (scan scratch, per-row scales, barrier, TMEM address), then the operand tiles; the
  // tiles' region is reused afterwards to stage the result rows
  float *scan_buf = reinterpret_cast<float *>(smem);                 // 8 + kQ floats
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kSsdHeader - 16);
  uint32_t *slot = reinterpret_cast<uint32_t *>(smem + kSsdHeader - 8);
  unsigned char *sA = smem + kSsdHeader;          // (w beta B)^T: M = n (128), K = s (128), MN-major
  unsigned char *sX = sA + kNP * kQ * 2;          // X: N = p (P), K = s (128), MN-major

  const int64_t nC = (p.L + kQ - 1) / kQ;
  const int64_t c = blockIdx.x % nC, bh = blockIdx.x / nC, b = bh / p.H, h = bh % p.H;
  const int t = threadIdx.x;
  const int64_t tg = c * kQ + t;

  const uint32_t tbase = tmem_alloc_cta(slot, (uint32_t)P);
  if (t == 0) mbar_init(bar, 1);

  const float A = -expf(p.A_log[h]);
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
  const StepCoefs k = chunk_coefs(p, bh, tg, A, bias, scan_buf);
  // total log-decay of the chunk = the last thread's inclusive sum
  if (t == kQ - 1) scan_buf[4] = k.cum;
  __syncthreads();
  const float cum_end = scan_buf[4];
  const float scale = k.beta * __expf(cum_end - k.cum);  // e^{cum_end - cum_s} beta_s

  // stage both operands: row s of B scaled by e^{cum_end - cum_s} beta_s (A operand, MN-major
  // along n), row s of X (B operand, MN-major along p)
  float *row_scale = scan_buf + 8;  // kQ floats after the scan scratch
  row_scale[t] = scale;
  __syncthreads();
  {
    const int64_t rows_left = p.L - c * kQ;
    auto valid = [&](int r) { return r < rows_left; };
    const __nv_bfloat16 *Bsrc = static_cast<const __nv_bfloat16 *>(p.B) + (b * p.L + c * kQ) * p.N;
    coop_tile<kQ, kNP / 8>(sA, Bsrc, p.N, (int)(p.N / 8),
                           [](int r, int v) { return mnmaj_off(kNP, v * 8, r); }, valid,
                           [&](int r, uint4 pk) {
                             const float sc = row_scale[r];
                             const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&pk);
                             uint4 o;
                             uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
                             for (int i = 0; i < 4; i++) {
                               const float2 f = __bfloat1622float2(h2[i]);
                               ow[i] = pack_bf16(f.x * sc, f.y * sc);
                             }
                             return o;
                           });
    const __nv_bfloat16 *Xsrc = static_cast<const __nv_bfloat16 *>(p.x) + (bh * p.L + c * kQ) * P;
    coop_tile<kQ, P / 8>(sX, Xsrc, P, P / 8, [](int r, int v) { return mnmaj_off(P, v * 8, r); },
                         valid, NoXform());
  }
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
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0));
  tc_fence_after();
  if (!ok && (t & 31) == 0) atomicExch(p.error, 1);
  // row n = t of S_c: TMEM -> registers -> shared (padded rows, over the consumed A tile) ->
  // coalesced global stores
  constexpr int SR = P + 4;  // padded row, floats
  float *stage = reinterpret_cast<float *>(sA);
  {
    const uint32_t lane_addr = tmem_lane_addr(tbase);
#pragma unroll
    for (int q = 0; q < P; q += 32) {
      float v[32];
      tmem_ld32(lane_addr + q, v);
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4 *>(stage + t * SR + q + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
  }
  __syncthreads();
  if (ok) {
    float *dst = p.S + (bh * nC + c) * p.N * P;
    for (int i = t; i < p.N * P / 4; i += 128) {
      const int r = i / (P / 4), q = (i % (P / 4)) * 4;
      *reinterpret_cast<float4 *>(dst + r * P + q) = *reinterpret_cast<const float4 *>(stage + r * SR + q);
    }
  }
  if (t == 0) p.cum_end[bh * nC + c] = cum_end;
  tc_fence_before();
  tmem_free_cta(tbase, (uint32_t)P);
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
// One CTA per (batch, chunk, group of HG heads): C and B are shared by the heads, so they are
// staged once and G = C B^T is formed once; each head then applies its own decays to G.
template <int P, typename Tout>
__global__ void __launch_bounds__(128, 1) ssd_out_kernel(const SsdParams p, int HG) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float *cum_s = reinterpret_cast<float *>(smem);  // header: 2 kQ + 8 floats, 2 barriers, slot
  float *beta_s = cum_s + kQ;
  float *scan_buf = beta_s + kQ;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kSsdHeader - 24);  // two barriers
  uint32_t *slot = reinterpret_cast<uint32_t *>(smem + kSsdHeader - 8);
  unsigned char *sC = smem + kSsdHeader;           // C: M = t (128), K = n (128), K-major
  unsigned char *sB = sC + kQ * kNP * 2;           // B: N = s, K = n, K-major; then each head's G'
  unsigned char *sX = sB + kQ * kNP * 2;           // X: N = p (P), K = s (128), MN-major
  unsigned char *sH = sX + P * kQ * 2;             // H_in: N = p (P), K = n (128), MN-major
  float *stage = reinterpret_cast<float *>(sB);    // result rows, over G' and X once consumed

  constexpr uint32_t kCols = (128 + 2 * P <= 256) ? 256u : 512u;  // G (128) + Y (P) + C H (P)
  const int64_t nC = (p.L + kQ - 1) / kQ;
  const int64_t ngrp = p.H / HG;
  const int64_t c = blockIdx.x % nC, rest = blockIdx.x / nC;
  const int64_t hgrp = rest % ngrp, b = rest / ngrp;
  const int t = threadIdx.x;
  const int64_t tg = c * kQ + t;
  const int64_t rows_left = p.L - c * kQ;
  auto valid = [&](int r) { return r < rows_left; };

  const uint32_t tbase = tmem_alloc_cta(slot, kCols);
  if (t == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
  }
  {
    const int64_t off = (b * p.L + c * kQ) * p.N;
    const auto kmaj = [](int r, int v) { return kmaj_off(kQ, r, v * 8); };
    coop_tile<kQ, kNP / 8>(sC, static_cast<const __nv_bfloat16 *>(p.C) + off, p.N, (int)(p.N / 8), kmaj, valid, NoXform());
    coop_tile<kQ, kNP / 8>(sB, static_cast<const __nv_bfloat16 *>(p.B) + off, p.N, (int)(p.N / 8), kmaj, valid, NoXform());
  }
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
  bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0));
  uint32_t phase = 0;  // of bar + 1, one completion per head
  const uint32_t lane_addr = tmem_lane_addr(tbase);
  for (int hi = 0; hi < HG; hi++) {
    const int64_t h = hgrp * HG + hi, bh = b * p.H + h;
    // this head's X and H_in tiles travel while the decays and G' are computed
    {
      const auto mnmaj = [](int r, int v) { return mnmaj_off(P, v * 8, r); };
      coop_tile_async<kQ, P / 8>(sX, static_cast<const __nv_bfloat16 *>(p.x) + (bh * p.L + c * kQ) * P, P, P / 8, mnmaj, valid);
      const int64_t nrows = p.N;
      coop_tile_async<kNP, P / 8>(sH, p.Hin + (bh * nC + c) * p.N * P, P, P / 8, mnmaj, [&](int r) { return r < nrows; });
      cp_async_commit();
    }
    const float A = -expf(p.A_log[h]);
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
    const StepCoefs k = chunk_coefs(p, bh, tg, A, bias, scan_buf);  // (synchronises the CTA)
    cum_s[t] = k.cum;
    beta_s[t] = k.beta;
    __syncthreads();  // cum_s / beta_s of this head
    tc_fence_after();
    // G'[t][s] = G[t][s] e^{cum_t - cum_s} beta_s for s <= t -> the A operand of G' X
    {
      const float ct = k.cum;
#pragma unroll 1
      for (int s0 = 0; s0 < kQ; s0 += 32) {
        float g[32];
        tmem_ld32(lane_addr + s0, g);
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          float v[8];
#pragma unroll
          for (int j = 0; j < 8; j++) {
            const int s = s0 + e + j;
            v[j] = (s <= t) ? g[e + j] * __expf(ct - cum_s[s]) * beta_s[s] : 0.f;
          }
          uint4 pk = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
          *reinterpret_cast<uint4 *>(sB + kmaj_off(kQ, t, s0 + e)) = pk;
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
        const uint64_t dc = smem_desc(sC + ks * 2 * (kQ / 8) * 128, (kQ / 8) * 128, 128);
        const uint64_t dh = smem_desc(sH + ks * 2 * (P / 8) * 128, (P / 8) * 128, 128);
        mma_bf16(tY, dg, dx, instr_desc(128, P, 0, 1), ks > 0);
        mma_bf16(tCH, dc, dh, instr_desc(128, P, 0, 1), ks > 0);
      }
      mma_commit(bar + 1);
    }
    ok = __all_sync(0xffffffffu, mbar_wait(bar + 1, phase)) && ok;
    phase ^= 1u;
    tc_fence_after();
    // y row t = G'X + e^{cum_t} C H_in -> shared (padded) -> coalesced stores with + D x
    constexpr int SR = P + 4;
    {
      const float et = __expf(k.cum);
#pragma unroll 1
      for (int q = 0; q < P; q += 32) {
        float yv[32], cv[32];
        tmem_ld32(lane_addr + 128 + q, yv);
        tmem_ld32(lane_addr + 128 + P + q, cv);
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4 *>(stage + t * SR + q + j) =
              make_float4(fmaf(et, cv[j], yv[j]), fmaf(et, cv[j + 1], yv[j + 1]),
                          fmaf(et, cv[j + 2], yv[j + 2]), fmaf(et, cv[j + 3], yv[j + 3]));
      }
    }
    tc_fence_before();
    __syncthreads();
    if (ok) {
      const float Dh = p.D ? p.D[h] : 0.f;
      const __nv_bfloat16 *xs = static_cast<const __nv_bfloat16 *>(p.x) + (bh * p.L + c * kQ) * P;
      Tout *ys = static_cast<Tout *>(p.y) + (bh * p.L + c * kQ) * P;
      for (int i = t; i < kQ * P / 4; i += 128) {
        const int r = i / (P / 4), q = (i % (P / 4)) * 4;
        if (r >= rows_left) continue;
        const float4 v = *reinterpret_cast<const float4 *>(stage + r * SR + q);
        const uint2 xv = *reinterpret_cast<const uint2 *>(xs + (int64_t)r * P + q);
        const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xv.x));
        const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xv.y));
        const float o[4] = {fmaf(Dh, x01.x, v.x), fmaf(Dh, x01.y, v.y), fmaf(Dh, x23.x, v.z), fmaf(Dh, x23.y, v.w)};
        VecStore<Tout, 4>::run(ys + (int64_t)r * P + q, o);
      }
    }
    __syncthreads();  // the staged rows, G' and X are rewritten by the next head
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
  const size_t tiles = (size_t)kNP * kQ * 2 + (size_t)P * kQ * 2, stage = (size_t)kNP * (P + 4) * 4;
  return kSsdHeader + (tiles > stage ? tiles : stage);
}
size_t ssd_smem_out(int P) {
  // C, B / G', X, H_in; the staged result rows overlay G' and X (kQ x (P + 4) floats)
  const size_t tiles = (size_t)2 * kQ * kNP * 2 + (size_t)P * kQ * 2 + (size_t)P * kNP * 2;
  const size_t stage_end = (size_t)kQ * kNP * 2 + (size_t)kQ * (P + 4) * 4;
  return kSsdHeader + (tiles > stage_end ? tiles : stage_end);
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
  ssd_state_kernel<P><<<(unsigned)grid, 128, s1, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ssd_pass_kernel<P><<<(unsigned)(p.Bt * p.H * (p.N * P / 1024)), 256, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int HG = 1;  // heads per CTA: C, B and C B^T are shared by them
  for (int cand : {8, 4, 2})
    if (p.H % cand == 0) {
      HG = cand;
      break;
    }
  ssd_out_kernel<P, Tout><<<(unsigned)(grid / HG), 128, s3, s>>>(p, HG);
  return cudaGetLastError();
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
  if (p.P == 64) return out_bf16 ? launch_ssd_t<64, __nv_bfloat16>(p, stream) : launch_ssd_t<64, float>(p, stream);
  if (p.P == 128) return out_bf16 ? launch_ssd_t<128, __nv_bfloat16>(p, stream) : launch_ssd_t<128, float>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ssm
