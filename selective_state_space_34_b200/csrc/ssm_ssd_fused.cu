// ssm_ssd_fused.cu -- Mamba-2 SSD forward in one launch on sm_100a: one CTA per (batch, head) walks
// the sequence chunk by chunk and keeps the N x P state in tensor memory, so neither the chunk
// states nor the state entering each chunk go through global memory.
//
// "state-space models" (aarnphm.xyz), "Mamba-2 and state-space duality": within a head the
// transition is a_t I, and with cum_t the running sum of log a_t over a chunk of Q steps,
// B-bar_s = beta_s B_s and w_s = beta_s e^{cum_end - cum_s}:
//
//   G        = C B^T                                       (Q x Q, K = N)
//   G'[t,s]  = G[t,s] e^{cum_t - cum_s} beta_s for s <= t, plus D on the diagonal
//   y        = G' X + diag(e^{cum_t}) C H_{c-1}            (Q x P)
//   H_c      = e^{cum_end} H_{c-1} + B^T diag(w) X          (N x P)
//
// Roles (576 threads): warp 0 loads the tiles with TMA (cp.async.bulk.tensor, completion counted
// on mbarriers), warp 1 issues the tcgen05 products from one thread, warps 2..17 do everything
// else -- four threads per accumulator row (warps w, w + 4, w + 8, w + 12 reach the same 32 TMEM
// lanes), each taking a quarter of the row's columns. Per chunk c the compute warps (1) form the
// decay coefficients, (2) copy H_{c-1} out of tensor memory as the bf16 operand of C H_{c-1},
// scale H in place by e^{cum_end}, and write diag(w) X, (3) finish chunk c-1's output from its two
// accumulators, and (4) turn G into G'. The MMA warp issues C H_{c-1} and the state product of
// chunk c after step (2), then G of chunk c+1 if its tiles have landed (else right after G' X),
// then G' X of chunk c after step (4), so the tensor core works on one chunk while the compute
// warps are on the other and the next chunk's G is usually ready before they need it. G is double-buffered in tensor memory, C, B and X in
// shared memory; the scaled X, the bf16 state and G' are single buffers whose reuse is ordered by
// the barriers below. Every wait is bounded; a wait that runs out records the error word and an
// abort flag, after which every role runs its loop to the end without issuing work, waits for its
// own copies and products in flight, and the CTA frees its tensor memory.
//
// Scores below the diagonal blocks: with cum_ref the running sum at the last step of the column's
// 32-step block, e^{cum_t - cum_s} beta_s = e^{cum_t - cum_ref} (beta_s e^{cum_ref - cum_s}); both
// factors are at most 1 (the second at most beta_s), so a score there costs one exp per row and
// block instead of one per score. The diagonal blocks keep one exp per score.
//
// Tile layouts in shared memory (bf16, no-swizzle canonical, 8 rows x 16 bytes per core matrix):
//   C, B  [n/8][t][n%8]   -- C is the K-major A operand (M = t, K = n) of G and of C H, B the K-major
//                            B operand (N = s, K = n) of G and the MN-major A operand (M = n, K = s)
//                            of the state product
//   X, XW [p/8][s][p%8]   -- MN-major B operands (N = p, K = s)
//   SH    [p/8][n][p%8]   -- MN-major B operand (N = p, K = n)
//   G'    [s/8][t][s%8]   -- K-major A operand (M = t, K = s)
#include "ssm_common.cuh"
#include "ssm_internal.h"
#include "ssm_tc.cuh"
#include "ssm_tmem.cuh"

namespace ssm {

namespace {

constexpr int kQ = 128;          // chunk length
constexpr int kP = 64;           // head dimension this kernel takes
constexpr int kFThreads = 576;   // producer warp, MMA warp, 16 compute warps
constexpr int kCompute = 512;
constexpr uint32_t kTmemCols = 512;
constexpr int kRowBytes = kQ * 16;  // one 8-column group of a Q-row tile

// shared-memory plan (byte offsets; operand tiles 1024-byte aligned)
constexpr int kOffC = 0;                       // 2 x (C 32 KB, B 32 KB): C in 16 KB and B's upper
constexpr int kCBStride = 65536;               //   half zero for N = 64
constexpr int kOffX = kOffC + 2 * kCBStride;   // 2 x 16 KB
constexpr int kOffXW = kOffX + 2 * 16384;      // 16 KB
constexpr int kOffSH = kOffXW + 16384;         // 16 KB
constexpr int kOffGP = kOffSH + 16384;         // 32 KB
constexpr int kOffQ = kOffGP + 32768;          // the chunk's q_s and v_s (score factors)
constexpr int kOffRef = kOffQ + 2 * kQ * 4;    // the chunk's block references (4 floats)
constexpr int kOffTot = kOffRef + 16;          // scan totals: 4 column quarters x 4 warps
constexpr int kOffBar = kOffTot + 64;          // mbarriers
constexpr int kNumBars = 17;
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // TMEM slot, abort flag
constexpr int kFusedSmem = kOffMisc + 16;
static_assert(kFusedSmem <= 232448, "shared memory per CTA");

// mbarrier indices
enum {
  FULL_CB = 0,   // C and B buffer i landed (TMA), 2 entries
  CBEMPTY = 2,   // C and B buffer i consumed by C H and the state product (commit), 2 entries
  FULL_X = 4,    // X buffer i landed (TMA), 2 entries
  XEMPTY = 6,    // X buffer i consumed by G' X (commit), 2 entries
  GFULL = 8,     // G buffer i written (commit), 2 entries
  GFREE = 10,    // G buffer i read out by the compute warps, 2 entries
  HX_READY = 12, // bf16 state, scaled state and diag(w) X in place (compute warps)
  S_DONE = 13,   // C H_{c-1} and the state product done (commit): SH, XW and the state reusable
  GP_READY = 14, // G' in place (compute warps)
  Y_FULL = 15,   // G' X done (commit): both output accumulators final, G' and X reusable
  Y_FREE = 16    // output accumulators read out (compute warps)
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}\n" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool poll_once(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait that gives up at once when another role has already given up. A wait that runs out
// (2^18 polls, about a second) raises the abort flag and the error word.
__device__ __forceinline__ bool fwait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *err) {
  for (int i = 0; i < (1 << 18); i++) {
    if (*abort_flag) return false;
    if (poll_once(bar, parity)) return true;
  }
  *abort_flag = 1;
  atomicExch(err, 1);
  return false;
}

// The same without the abort check: for the final wait on this thread's own copies or products,
// which complete whatever the other roles do.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, int *err) {
  for (int i = 0; i < (1 << 18); i++)
    if (poll_once(bar, parity)) return;
  atomicExch(err, 1);
}

// NK consecutive K-slices of one product: the descriptors of slice ks are the first slice's with
// the start address moved on by ks steps (the address field counts 16-byte units, and every tile
// lies below 256 KB, so the step is a plain add).
template <int NK>
__device__ __forceinline__ void mma_chain(uint32_t d_tmem, uint64_t da, uint32_t da_step, uint64_t db,
                                          uint32_t db_step, uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int ks = 0; ks < NK; ks++)
    mma_bf16(d_tmem, da + (uint64_t)(ks * da_step), db + (uint64_t)(ks * db_step), idesc, accumulate || ks > 0);
}

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

__device__ __forceinline__ void store_row16(float *dst, const float *v) {
#pragma unroll
  for (int i = 0; i < 4; i++)
    reinterpret_cast<float4 *>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
__device__ __forceinline__ void store_row16(__nv_bfloat16 *dst, const float *v) {
#pragma unroll
  for (int i = 0; i < 2; i++)
    reinterpret_cast<uint4 *>(dst)[i] =
        make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                   pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t v) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v));
}

}  // namespace

template <int NN, typename Tout>
__global__ void __launch_bounds__(kFThreads, 1)
ssd_fused_kernel(const SsdParams p, const __grid_constant__ CUtensorMap tmX,
                 const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char *sXW = smem + kOffXW;
  unsigned char *sSH = smem + kOffSH, *sGP = smem + kOffGP;
  float *qs = reinterpret_cast<float *>(smem + kOffQ);
  float *vs = qs + kQ, *rref = reinterpret_cast<float *>(smem + kOffRef);
  float *tot = reinterpret_cast<float *>(smem + kOffTot);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  constexpr int N = NN;  // 64 or 128
  const int64_t L = p.L, nC = (L + kQ - 1) / kQ;

  if (threadIdx.x == 0) {
    // the tiles are TMA destinations and descriptor bases: refuse to run on a misaligned window
    const bool aligned = (smem_u32(smem) & 1023u) == 0;
    *abort_flag = aligned ? 0 : 1;
    if (!aligned) atomicExch(p.error, 1);
    for (int i = 0; i < 2; i++) {
      mbar_init(bars + FULL_CB + i, 1);
      mbar_init(bars + CBEMPTY + i, 1);
      mbar_init(bars + FULL_X + i, 1);
      mbar_init(bars + XEMPTY + i, 1);
      mbar_init(bars + GFULL + i, 1);
      mbar_init(bars + GFREE + i, 16);

    }
    mbar_init(bars + HX_READY, 16);
    mbar_init(bars + S_DONE, 1);
    mbar_init(bars + GP_READY, 16);
    mbar_init(bars + Y_FULL, 1);
    mbar_init(bars + Y_FREE, 16);
  }
  // zero what no load or score ever writes: the B rows n >= N (read by the state product as
  // M rows) and the score blocks above the diagonal of G'
  if (warp >= 2) {
    const int ct = threadIdx.x - 64;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    if (N < 128)
      for (int i = ct; i < 2 * (128 - N) * kQ / 8; i += kCompute) {
        const int buf = i / ((128 - N) * kQ / 8), k = i % ((128 - N) * kQ / 8);
        reinterpret_cast<uint4 *>(smem + kOffC + buf * kCBStride + 32768 + N / 8 * kRowBytes)[k] = z;
      }
    // G' block (row block tb, column block sb) of 32 x 32, sb > tb: 4 column groups x 32 rows
    for (int i = ct; i < 6 * 4 * 32; i += kCompute) {
      const int blk = i / 128, rem = i % 128, grp = rem / 32, row = rem % 32;
      const int tb = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
      const int sb = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
      *reinterpret_cast<uint4 *>(sGP + (sb * 4 + grp) * kRowBytes + (tb * 32 + row) * 16) = z;
    }
    fence_async_smem();
  }
  const uint32_t tbase = tmem_alloc_cta(tslot, kTmemCols);  // includes a CTA barrier
  const uint32_t tG0 = tbase, tY1 = tbase + 256, tY2 = tbase + 320, tH = tbase + 384;

  if (warp == 0) {
    // ---- producer: C and B of chunk c once the state product of chunk c-2 released their buffer,
    //      then X once G' X of chunk c-2 released its buffer
    if (lane == 0 && !*abort_flag) {
      const uint32_t bytesX = (kP / 8) * kRowBytes;
      const uint32_t bytesCB = 2u * (uint32_t)(N / 8) * kRowBytes;
      uint32_t nX0 = 0u, nX1 = 0u, nCB0 = 0u, nCB1 = 0u;  // copies issued per buffer
      for (int64_t c = 0; c < nC; c++) {
        const int xb = (int)(c & 1);
        if (c < 2 || fwait(bars + CBEMPTY + xb, (uint32_t)(((c >> 1) - 1) & 1), abort_flag, p.error)) {
          unsigned char *sC = smem + kOffC + xb * kCBStride, *sB = sC + 32768;
          mbar_expect_tx(bars + FULL_CB + xb, bytesCB);
          for (int j = 0; j < N / 8; j++) {
            tma_load_3d(sC + j * kRowBytes, &tmC, j * 8, (int)(c * kQ), (int)b, bars + FULL_CB + xb);
            tma_load_3d(sB + j * kRowBytes, &tmB, j * 8, (int)(c * kQ), (int)b, bars + FULL_CB + xb);
          }
          (xb ? nCB1 : nCB0)++;
        }
        if (c < 2 || fwait(bars + XEMPTY + xb, (uint32_t)(((c >> 1) - 1) & 1), abort_flag, p.error)) {
          unsigned char *dst = smem + kOffX + xb * 16384;
          mbar_expect_tx(bars + FULL_X + xb, bytesX);
          for (int j = 0; j < kP / 8; j++)
            tma_load_3d(dst + j * kRowBytes, &tmX, j * 8, (int)(c * kQ), (int)bh, bars + FULL_X + xb);
          (xb ? nX1 : nX0)++;
        }
      }
      // every issued copy lands before the CTA may exit
      if (nCB0) drain_wait(bars + FULL_CB, (nCB0 - 1) & 1, p.error);
      if (nCB1) drain_wait(bars + FULL_CB + 1, (nCB1 - 1) & 1, p.error);
      if (nX0) drain_wait(bars + FULL_X, (nX0 - 1) & 1, p.error);
      if (nX1) drain_wait(bars + FULL_X + 1, (nX1 - 1) & 1, p.error);
    }
  } else if (warp == 1) {
    // ---- tensor-core issue, one thread
    if (lane == 0) {
      constexpr uint32_t idG = instr_desc(128, 128, 0, 0);
      constexpr uint32_t idY = instr_desc(128, kP, 0, 1);
      constexpr uint32_t idS = instr_desc(128, kP, 1, 1);
      uint64_t *last_bar = nullptr;  // the barrier of the latest commit, and its phase
      uint32_t last_phase = 0;
      // every operand descriptor, built once: C / B of either buffer as K-major operands (G, C H),
      // B as the MN-major A operand of the state product, X of either buffer, diag(w) X, the bf16
      // state and G'. Steps per K-slice of 16, in 16-byte units: 2 K-groups of a K-major tile
      // (2 x 2048 bytes), 2 of an MN-major one (2 x 128 bytes).
      constexpr uint32_t kKStep = 2 * kRowBytes / 16, kMStep = 256 / 16;
      const uint64_t dCk0 = smem_desc(smem + kOffC, kRowBytes, 128);
      const uint64_t dCk1 = smem_desc(smem + kOffC + kCBStride, kRowBytes, 128);
      const uint64_t dBk0 = smem_desc(smem + kOffC + 32768, kRowBytes, 128);
      const uint64_t dBk1 = smem_desc(smem + kOffC + kCBStride + 32768, kRowBytes, 128);
      const uint64_t dBm0 = smem_desc(smem + kOffC + 32768, 128, kRowBytes);
      const uint64_t dBm1 = smem_desc(smem + kOffC + kCBStride + 32768, 128, kRowBytes);
      const uint64_t dX0 = smem_desc(smem + kOffX, 128, kRowBytes);
      const uint64_t dX1 = smem_desc(smem + kOffX + 16384, 128, kRowBytes);
      const uint64_t dXW = smem_desc(sXW, 128, kRowBytes), dSH = smem_desc(sSH, 128, (uint32_t)N * 16);
      const uint64_t dGP = smem_desc(sGP, kRowBytes, 128);
      // G = C B^T of chunk cc into G buffer cc & 1, once its C and B landed and the compute warps
      // read out that buffer's previous G
      auto issue_g = [&](int64_t cc) {
        const int gb = (int)(cc & 1);
        if (fwait(bars + FULL_CB + gb, (uint32_t)((cc >> 1) & 1), abort_flag, p.error) &&
            (cc < 2 || fwait(bars + GFREE + gb, (uint32_t)(((cc >> 1) - 1) & 1), abort_flag, p.error))) {
          tc_fence_after();
          mma_chain<N / 16>(tG0 + gb * 128, gb ? dCk1 : dCk0, kKStep, gb ? dBk1 : dBk0, kKStep, idG, false);
          mma_commit(bars + GFULL + gb);
          last_bar = bars + GFULL + gb;
          last_phase = (uint32_t)((cc >> 1) & 1);
        }
      };
      issue_g(0);
      for (int64_t c = 0; c < nC; c++) {
        const int cb = (int)(c & 1);
        // C H_{c-1} into the second output accumulator; H += B^T diag(w) X
        if (fwait(bars + HX_READY, (uint32_t)(c & 1), abort_flag, p.error) &&
            (c < 1 || fwait(bars + Y_FREE, (uint32_t)((c - 1) & 1), abort_flag, p.error))) {
          tc_fence_after();
          mma_chain<N / 16>(tY2, cb ? dCk1 : dCk0, kKStep, dSH, kMStep, idY, false);
          mma_chain<kQ / 16>(tH, cb ? dBm1 : dBm0, kMStep, dXW, kMStep, idS, true);
          mma_commit(bars + S_DONE);
          mma_commit(bars + CBEMPTY + cb);
          last_bar = bars + CBEMPTY + cb;
          last_phase = (uint32_t)((c >> 1) & 1);
        }
        // the next chunk's C B^T now if its tiles and its G buffer are ready (so that its scores
        // do not wait for the tensor core), else right after G' X
        bool g_next = c + 1 < nC;
        if (g_next && poll_once(bars + FULL_CB + ((c + 1) & 1), (uint32_t)(((c + 1) >> 1) & 1)) &&
            (c + 1 < 2 || poll_once(bars + GFREE + ((c + 1) & 1), (uint32_t)((((c + 1) >> 1) - 1) & 1)))) {
          issue_g(c + 1);
          g_next = false;
        }
        // G' X into the first output accumulator
        if (fwait(bars + GP_READY, (uint32_t)(c & 1), abort_flag, p.error) &&
            fwait(bars + FULL_X + cb, (uint32_t)((c >> 1) & 1), abort_flag, p.error)) {
          tc_fence_after();
          mma_chain<kQ / 16>(tY1, dGP, kKStep, cb ? dX1 : dX0, kMStep, idY, false);
          mma_commit(bars + Y_FULL);
          mma_commit(bars + XEMPTY + cb);
          last_bar = bars + XEMPTY + cb;
          last_phase = (uint32_t)((c >> 1) & 1);
        }
        if (g_next) issue_g(c + 1);
      }
      // no product in flight when the CTA frees its tensor memory
      if (last_bar) drain_wait(last_bar, last_phase, p.error);
    }
  } else {
    // ---- compute warps: thread (row r, column quarter cq); row r is step t (outputs, scores, X) or
    //      state n, the quarter picks 16 of the P columns and 8 of every 32-column score block
    const int cq = (warp - 2) >> 2, q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int p0 = cq * 16;  // this thread's columns of X, H and y
    const float A = -expf(p.A_log[h]);
    const float dtb = p.dt_bias ? p.dt_bias[h] : 0.f, Dh = p.D ? p.D[h] : 0.f;
    const __nv_bfloat16 *dtrow = static_cast<const __nv_bfloat16 *>(p.dt) + bh * L;
    const bool has_h = r < N;  // warp-uniform: rows n >= N of the state stay zero
    Tout *yh = static_cast<Tout *>(p.y) + bh * L * kP;

    // the entering state (h0 or zero) into tensor memory
    if (has_h) {
      float hv[16];
      const float *src = p.h0 ? p.h0 + (bh * N + r) * kP + p0 : nullptr;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const float4 v = src ? reinterpret_cast<const float4 *>(src)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        hv[4 * i] = v.x;
        hv[4 * i + 1] = v.y;
        hv[4 * i + 2] = v.z;
        hv[4 * i + 3] = v.w;
      }
      tmem_st<16>(tH + lane_off + p0, hv);
      tmem_wait_st();
    }

    auto epilogue = [&](int64_t cc, float et) {
      bool ok = fwait(bars + Y_FULL, (uint32_t)(cc & 1), abort_flag, p.error);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        float y1[16], y2[16];
        tmem_ld2<16>(tY1 + lane_off + p0, y1, tY2 + lane_off + p0, y2);
#pragma unroll
        for (int i = 0; i < 16; i++) y1[i] = fmaf(et, y2[i], y1[i]);
        const int64_t t = cc * kQ + r;
        if (t < L) store_row16(yh + t * kP + p0, y1);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + Y_FREE);
    };

    float dt_next = r < L ? to_f32(dtrow[r]) : 0.f;
    float et_prev = 0.f;
    for (int64_t c = 0; c < nC; c++) {
      // (1) decay coefficients of step r: Delta, log a = Delta A, beta; the running sum of log a
      //     over the chunk by a warp scan plus the earlier warps' totals (each quarter on its own)
      const int64_t tg = c * kQ + r;
      const float v = dt_next + dtb;
      dt_next = (tg + kQ < L) ? to_f32(dtrow[tg + kQ]) : 0.f;  // the next chunk's, early
      float la = 0.f, beta = 0.f;
      if (tg < L) {
        const float dl = p.delta_softplus ? softplus<false>(v) : v;
        la = dl * A;
        beta = p.euler ? dl : expm1f(la) / A;  // padded steps: a = 1, beta = 0 (identity)
      }
      float cum = la;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, cum, off);
        if (lane >= off) cum += o;
      }
      if (lane == 31) tot[cq * 4 + q] = cum;
      compute_bar();
      float cend = 0.f;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const float s = tot[cq * 4 + i];
        if (i < q) cum += s;
        cend += s;
      }
      const float ct = cum * kLog2e;                // e^{cum_t} = 2^{ct}
      const float et = __expf(cum);
      const float wgt = beta * __expf(cend - cum);  // row weight of the state product
      const float a = __expf(cend);                 // decay of the whole chunk
      // score factors: q_s for the diagonal blocks, and for the blocks below the diagonal
      // v_s = beta_s e^{cum_ref - cum_s}, with cum_ref the running sum at the last step of s's
      // 32-step block (the last lane of this warp), so that a score there is
      // G[t,s] e^{cum_t - cum_ref} v_s with both factors at most 1 (and v_s at most beta_s)
      const float qv_r = ct - lg2_approx(beta);      // beta = 0: +inf, a zero score
      const float cref = __shfl_sync(0xffffffffu, ct, 31);
      if (cq == 0) {
        qs[r] = qv_r;
        vs[r] = ex2_approx(cref - qv_r);
        if (lane == 31) rref[q] = ct;
      }
      compute_bar();                                // every q_s, v_s and block reference in place

      // (2) H_{c-1} -> bf16 operand, H *= a; X -> diag(w) X
      const int xb = (int)(c & 1);
      bool ok = (c == 0 || fwait(bars + S_DONE, (uint32_t)((c - 1) & 1), abort_flag, p.error)) &&
                fwait(bars + FULL_X + xb, (uint32_t)((c >> 1) & 1), abort_flag, p.error);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        if (has_h) {
          float hv[16];
          tmem_ld2<8>(tH + lane_off + p0, hv, tH + lane_off + p0 + 8, hv + 8);
#pragma unroll
          for (int j = 0; j < 2; j++)
            *reinterpret_cast<uint4 *>(sSH + ((cq * 2 + j) * N + r) * 16) =
                make_uint4(pack_bf16(hv[8 * j], hv[8 * j + 1]), pack_bf16(hv[8 * j + 2], hv[8 * j + 3]),
                           pack_bf16(hv[8 * j + 4], hv[8 * j + 5]), pack_bf16(hv[8 * j + 6], hv[8 * j + 7]));
#pragma unroll
          for (int i = 0; i < 16; i++) hv[i] *= a;
          tmem_st<16>(tH + lane_off + p0, hv);
          tmem_wait_st();
        }
        const unsigned char *sX = smem + kOffX + xb * 16384;
#pragma unroll
        for (int j = cq * 2; j < cq * 2 + 2; j++) {
          const uint4 raw = *reinterpret_cast<const uint4 *>(sX + j * kRowBytes + r * 16);
          const float2 f0 = bf2_to_f2(raw.x), f1 = bf2_to_f2(raw.y), f2 = bf2_to_f2(raw.z), f3 = bf2_to_f2(raw.w);
          *reinterpret_cast<uint4 *>(sXW + j * kRowBytes + r * 16) =
              make_uint4(pack_bf16(f0.x * wgt, f0.y * wgt), pack_bf16(f1.x * wgt, f1.y * wgt),
                         pack_bf16(f2.x * wgt, f2.y * wgt), pack_bf16(f3.x * wgt, f3.y * wgt));
        }
      }
      tc_fence_before();
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + HX_READY);

      // (3) the previous chunk's output, while the tensor core runs this chunk's products
      if (c > 0) epilogue(c - 1, et_prev);

      // (4) G' = masked, decayed scores (+ D on the diagonal): row t = r, in every 32-column block
      //     on or below the diagonal the 8 columns of this quarter. All four blocks' columns are
      //     read in one go (the ones above the diagonal are not used).
      ok = fwait(bars + GFULL + xb, (uint32_t)((c >> 1) & 1), abort_flag, p.error);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const uint32_t tg_addr = tG0 + xb * 128 + lane_off + cq * 8;
        float g[32];
        tmem_ld2<8>(tg_addr, g, tg_addr + 32, g + 8);
        tmem_ld2<8>(tg_addr + 64, g + 16, tg_addr + 96, g + 24);
#pragma unroll
        for (int kb = 0; kb < 4; kb++) {
          if (kb > q) break;  // warp-uniform: the blocks above the diagonal stay zero
          const int s0 = kb * 32 + cq * 8;
          float o[8];
          if (kb < q) {
            // below the diagonal: G[t,s] e^{cum_t - cum_ref} v_s
            const float u = ex2_approx(ct - rref[kb]);
            const float4 v0 = *reinterpret_cast<const float4 *>(vs + s0);
            const float4 v1 = *reinterpret_cast<const float4 *>(vs + s0 + 4);
            const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int j = 0; j < 8; j++) o[j] = g[kb * 8 + j] * u * vv[j];
          } else {
            // the diagonal block: one exp per score, s <= t, D on the diagonal
            const float4 q0 = *reinterpret_cast<const float4 *>(qs + s0);
            const float4 q1 = *reinterpret_cast<const float4 *>(qs + s0 + 4);
            const float qq[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int j = 0; j < 8; j++) {
              const int s = s0 + j;
              const float sv = g[kb * 8 + j] * ex2_approx(ct - qq[j]);
              o[j] = s < r ? sv : (s == r ? sv + Dh : 0.f);
            }
          }
          *reinterpret_cast<uint4 *>(sGP + (s0 >> 3) * kRowBytes + r * 16) =
              make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                         pack_bf16(o[6], o[7]));
        }
      }
      tc_fence_before();
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bars + GFREE + xb);
        mbar_arrive(bars + GP_READY);
      }
      et_prev = et;
    }
    epilogue(nC - 1, et_prev);
    // the state after the last step (the last state product is done: it precedes G' X)
    if (p.h_last && has_h && __all_sync(0xffffffffu, *abort_flag == 0)) {
      float hv[16];
      tmem_ld2<8>(tH + lane_off + p0, hv, tH + lane_off + p0 + 8, hv + 8);
      float *dst = p.h_last + (bh * N + r) * kP + p0;
#pragma unroll
      for (int i = 0; i < 4; i++)
        reinterpret_cast<float4 *>(dst)[i] = make_float4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
    }
  }
  tmem_free_cta(tbase, kTmemCols);
}

// ---- host ------------------------------------------------------------------------------------

namespace {

// A (inner, rows, outer) bf16 tensor, row-major, loaded as boxes of 8 inner elements x 128 rows:
// one box is one 8-column group of a tile, [row][8], 16 bytes a row. Rows past `rows` read zero.
bool encode_rows_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t outer) {
  return encode_tma_3d(m, true, base, inner, rows, outer, 8, (uint32_t)kQ);
}

}  // namespace

bool ssd_fused_supported(const SsdParams &p) { return p.P == kP && (p.N == 64 || p.N == 128); }

cudaError_t launch_ssd_fused(const SsdParams &p, int out_bf16, cudaStream_t s) {
  if (!ssd_fused_supported(p)) return cudaErrorInvalidValue;
  if (p.Bt * p.H > 0x7fffffffLL || p.L > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  CUtensorMap mX, mB, mC;
  if (!encode_rows_map(&mX, p.x, (uint64_t)kP, (uint64_t)p.L, (uint64_t)(p.Bt * p.H)) ||
      !encode_rows_map(&mB, p.B, (uint64_t)p.N, (uint64_t)p.L, (uint64_t)p.Bt) ||
      !encode_rows_map(&mC, p.C, (uint64_t)p.N, (uint64_t)p.L, (uint64_t)p.Bt))
    return cudaErrorNotSupported;  // the driver declined a tensor map; nothing was launched
  auto kern = p.N == 64 ? (out_bf16 ? ssd_fused_kernel<64, __nv_bfloat16> : ssd_fused_kernel<64, float>)
                        : (out_bf16 ? ssd_fused_kernel<128, __nv_bfloat16> : ssd_fused_kernel<128, float>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmem);
  if (e != cudaSuccess) return e;
  if (p.timing_events && p.timing_events[0] &&
      (e = cudaEventRecord(static_cast<cudaEvent_t>(p.timing_events[0]), s)) != cudaSuccess)
    return e;
  kern<<<(unsigned)(p.Bt * p.H), kFThreads, kFusedSmem, s>>>(p, mX, mB, mC);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p.timing_events && p.timing_events[1])
    e = cudaEventRecord(static_cast<cudaEvent_t>(p.timing_events[1]), s);
  return e;
}

}  // namespace ssm
