// ssm_bwd.cu -- selective-scan backward (vector-Jacobian product) for sm_100a.
//
// The analytic VJP of the fused forward, run as a reverse-time recurrence over the states that
// are recomputed block by block from the saved chunk states (rustytorch commit log, "Hand-written
// VJP": reverse-time recurrence over the cached h trajectory; dA_log = dA * A). With
// x = Delta*A, a = exp(x), lambda_t = dL/dh_t:
//
//   lambda_t   = dy_t C_t + a_{t+1} lambda_{t+1}
//   dC_t[n]   += dy_t h_t[n]                        (summed over channels)
//   dB_t[n]   += lambda_t[n] u_t (a - 1) / A        (summed over channels)
//   dDelta_t   = sum_n lambda_t[n] (A h_t[n] + B_t[n] u_t)      [= a (A h_{t-1} + B u)]
//   du_t       = D dy_t + sum_n lambda_t[n] B_bar_t[n]
//   dA_log[n] += Delta_t * lambda (A h_t + B u) - u_t lambda B_bar
//
// The last line is A * dA (the chain rule through A = -exp(A_log)); it uses the identity
// A * d(h-update)/dA = Delta * d(h-update)/dDelta - u * B_bar, which avoids the cancelling
// difference x a - (a - 1) for small x.
//
// Decomposition mirrors the forward: a CTA owns CH = 128/G channels of one batch element, lanes
// hold NS states each, and the sequence is walked backwards in stages of 16 steps (one saved-state
// chunk each): recompute the stage forward from its saved start state, keeping h_t and a_t of
// every step (a_t - 1 on the precise path) in the thread's lane of tensor memory (TMEM, otherwise
// idle here) instead of registers, then run the adjoint backwards through it one 4-step group at a
// time. Moving that trajectory out of the register file is what lets four CTAs
// share an SM. dB and dC are summed over the CTA's channels (a warp butterfly per step and one
// cross-warp sum per stage, or a shared-memory sum after every 4 steps for the other lane layouts)
// and written as per-tile partials; one more launch adds the tiles (and the per-batch partials of
// the per-channel parameter gradients) in a fixed order, so the result is deterministic. The
// stage's x, dt, z and dout rows arrive by TMA boxes where rows are 16-byte aligned, else by
// 16-byte cp.async.
#include "ssm_common.cuh"
#include "ssm_internal.h"
#include "ssm_stage.cuh"
#include "ssm_tc.cuh"
#include "ssm_tmem.cuh"

namespace ssm {

// 1: the dB / dC channel sum of the 4-lane, 4-state layout runs as a warp butterfly (below).
#ifndef SSM_BWD_BFLY
#define SSM_BWD_BFLY 1
#endif
// Resident CTAs per SM the backward is compiled for (its register budget: 65536 / (128 x this)).
#ifndef SSM_BWD_MIN_CTAS
#define SSM_BWD_MIN_CTAS 4
#endif
// 1: the adjoint recomputes A_bar on the bf16 path instead of reading it back from TMEM (one
// more exp per element-state, 16 fewer live registers). Measured on 4x4096x16x4096: 2.63 -> 2.46 ms
// when the kernel spilled 60 bytes per thread; with the stages staged by TMA and the exp argument
// formed as (Delta log2 e) A, reading A_bar back is the faster one (2.300 against 2.337 ms).
#ifndef SSM_BWD_AREC
#define SSM_BWD_AREC 0
#endif

template <int G, int NS, typename Tin> struct BwdSmem {
  static constexpr int CH = kThreads / G;
  static constexpr int NP = G * NS;
  static constexpr int TS = kSub;                 // steps per stage = one saved-state chunk
  static constexpr int XS = kPre + TS;
  static constexpr int BS = NP + 4;
  static constexpr int ES = TS + 1;               // e3 / pe row stride
  static constexpr int YG = TS;
  static constexpr int YC = G * YG + 4;
  // with 4 lanes per channel the du / dDelta lane sums go through shuffles (no shared rows)
  static constexpr bool SHFL = (G == 4);
  // dc row: this stage, then the next stage's 3. With 4 lanes per channel each lane stores its 4
  // values and reads its 8-value window as 16-byte vectors; a stride of 48 floats (16 mod 32)
  // keeps those accesses free of bank conflicts
  static constexpr int DCS = (G == 4) ? 48 : TS + 8;
  static constexpr int RH = 4;                    // steps per cross-channel reduction
  static constexpr int CHH = CH / 2;
  static constexpr int RBC = CHH * NP + 16;       // half-tile of channels (+16 words: banks)
  static constexpr int RBT = 2 * RBC + 4;         // one step
  static constexpr int RBW = RH * RBT;            // one quantity (dB or dC)
  // With 4 lanes of 4 states per channel the channel sum runs as a warp butterfly (BFLY): each
  // lane ends each step with the 8-channel sum of one (quantity, state), parked in a row of
  // 4 warps x 32 lanes (+2 words: the per-stage cross-warp sum then reads without bank conflicts)
  static constexpr bool BFLY = (G == 4 && NS == 4 && SSM_BWD_BFLY);
  static constexpr int WPT = 4 * 32 + 2;
  // AREC (bf16 path): TMEM keeps only h of the stage's steps and the adjoint recomputes A_bar
  // from Delta (bitwise the same value: the same product and the same ex2); otherwise TMEM keeps
  // h and A_bar (A_bar - 1 on the precise path). At least 32 columns per allocation.
  static constexpr bool AREC = sizeof(Tin) == 2 && SSM_BWD_AREC;
  static constexpr uint32_t NCOLS = (AREC ? (16 * NS < 32 ? 32 : 16 * NS) : 32 * NS);
  static constexpr size_t x_off = 0;
  static constexpr size_t dt_off = x_off + sizeof(Tin) * 2 * CH * XS;
  static constexpr size_t z_off = dt_off + sizeof(Tin) * 2 * CH * TS;
  static constexpr size_t do_off = z_off + sizeof(Tin) * 2 * CH * TS;
  static constexpr size_t bs_off = do_off + sizeof(Tin) * 2 * CH * TS;
  static constexpr size_t cs_off = bs_off + sizeof(float) * 2 * TS * BS;
  static constexpr size_t e3_off = cs_off + sizeof(float) * 2 * TS * BS;   // (dl, u, dy, gc)
  static constexpr size_t pe_off = e3_off + sizeof(float4) * CH * ES;      // (sv, gz)
  static constexpr size_t y0_off = pe_off + sizeof(float2) * CH * ES;
  static constexpr size_t y1_off = y0_off + sizeof(float) * CH * YC;
  static constexpr size_t dcs_off = y1_off + (SHFL ? 0 : sizeof(float) * CH * YC);
  static constexpr size_t rb_off = dcs_off + sizeof(float) * CH * DCS;
  // cluster exchange: every thread's 4-step sums of the stage, two rows (one per stage parity)
  static constexpr size_t cx_off = rb_off + (BFLY ? sizeof(float) * TS * WPT : sizeof(float) * 2 * RBW);
  static constexpr size_t slot_off = cx_off + (BFLY ? sizeof(float4) * 2 * kThreads : 0);
  static constexpr size_t bar_off = slot_off + 16;  // 2 mbarriers of the TMA stage copies
  static constexpr size_t bytes = bar_off + 16;
  static_assert(dt_off % 128 == 0 && z_off % 128 == 0 && do_off % 128 == 0 &&
                (sizeof(Tin) * CH * XS) % 128 == 0 && (sizeof(Tin) * CH * TS) % 128 == 0,
                "TMA destinations are 128-byte aligned");
  __host__ __device__ static constexpr int rb_index(int which, int tt, int c, int n) {
    return which * RBW + tt * RBT + (c / CHH) * RBC + (c % CHH) * NP + n;
  }
};

// Thread-block cluster helpers: a full barrier of the cluster's CTAs (release / acquire, so shared
// memory written before it is visible to the other CTAs after it), this CTA's rank, and a 16-byte
// load from the same offset of another CTA's shared memory.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(const float4 *local, uint32_t rank) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local));
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(ra) : "memory");
  return v;
}

template <int NS> __device__ __forceinline__ void store_states(float *dst, const float *v) {
  if (NS % 4 == 0) {
#pragma unroll
    for (int j = 0; j < NS; j += 4)
      *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  } else if (NS % 2 == 0) {
#pragma unroll
    for (int j = 0; j < NS; j += 2) *reinterpret_cast<float2 *>(dst + j) = make_float2(v[j], v[j + 1]);
  } else {
#pragma unroll
    for (int j = 0; j < NS; j++) dst[j] = v[j];
  }
}

// SEG: split-L pass 3 (a grid of segments x batch x channel tiles); without it the segment is
// the whole sequence and its bounds are compile-time constants of the one-pass kernel.
template <int G, int NS, typename Tin, bool EULER, bool SEG>
__global__ void __launch_bounds__(kThreads, SSM_BWD_MIN_CTAS)
ssm_bwd_kernel(const BwdParams P, const __grid_constant__ CUtensorMap tmx,
               const __grid_constant__ CUtensorMap tmdt, const __grid_constant__ CUtensorMap tmz,
               const __grid_constant__ CUtensorMap tmdo) {
  using S = BwdSmem<G, NS, Tin>;
  constexpr int CH = S::CH, NP = S::NP, TS = S::TS, EPL = TS / G, RH = S::RH;
  constexpr int GV = 4 * NS;  // TMEM columns of one quantity over a 4-step group
  constexpr bool PRECISE = sizeof(Tin) == 4;
  constexpr bool PAIRS = !PRECISE && (NS % 2 == 0);
  static_assert(RH == 4 && TS % 4 == 0, "a reduction quarter is one 4-step TMEM group");
  const FwdParams &p = P.f;
  extern __shared__ __align__(16) unsigned char smem[];
  Tin *xs = reinterpret_cast<Tin *>(smem + S::x_off);
  Tin *dts = reinterpret_cast<Tin *>(smem + S::dt_off);
  Tin *zs = reinterpret_cast<Tin *>(smem + S::z_off);
  Tin *dos = reinterpret_cast<Tin *>(smem + S::do_off);
  float *Bs = reinterpret_cast<float *>(smem + S::bs_off);
  float *Cs = reinterpret_cast<float *>(smem + S::cs_off);
  float4 *e3 = reinterpret_cast<float4 *>(smem + S::e3_off);
  float2 *pe = reinterpret_cast<float2 *>(smem + S::pe_off);
  float *y0 = reinterpret_cast<float *>(smem + S::y0_off);
  float *y1 = reinterpret_cast<float *>(smem + S::y1_off);
  float *dcs = reinterpret_cast<float *>(smem + S::dcs_off);
  float *rb = reinterpret_cast<float *>(smem + S::rb_off);
  uint32_t *slot = reinterpret_cast<uint32_t *>(smem + S::slot_off);

  // h and A_bar (A_bar - 1 on the precise path) of the stage's steps live in this thread's TMEM
  // lane: column t*NS + j holds step t, state j
  const uint32_t tbase = tmem_alloc_cta(slot, S::NCOLS);
  const uint32_t th = tmem_lane_addr(tbase);
  const uint32_t ta = th + TS * NS;

  const int64_t n_dtiles = (p.Dn + CH - 1) / CH;
  const int64_t tile = blockIdx.x % n_dtiles;
  const int64_t b = SEG ? (blockIdx.x / n_dtiles) % p.Bt : blockIdx.x / n_dtiles;
  const int64_t seg = SEG ? blockIdx.x / (n_dtiles * p.Bt) : 0;  // segment of the sequence
  const int64_t d0 = tile * CH;
  const int rows_valid = (int)imin64(CH, p.Dn - d0);
  const int tid = threadIdx.x, c = tid / G, g = tid % G;
  const int64_t d = d0 + c;
  const bool live = d < p.Dn;
  const bool has_conv = p.conv_w != nullptr, has_z = p.z != nullptr;
  const bool vec = p.vec != 0;
  const int64_t L = p.L, N = p.N;
  // this CTA's steps: [ts, te). L stays the row length; steps from te on are padding here.
  const int64_t ts = SEG ? seg * P.seg_len : 0, te = SEG ? imin64(L, ts + P.seg_len) : L;
  const int64_t sbd = (seg * p.Bt + b) * p.Dn + d;  // row of the per-(segment, b, d) partials

  // A and -1/A per owned state (the fast path forms the exp argument as (Delta log2 e) A)
  constexpr int NH = (NS + 1) / 2;  // state pairs per lane
  float2 A2[NH], nIA2[NH], lam2[NH], aN2[NH], dAl2[NH];
  float *A = reinterpret_cast<float *>(A2);
  float *nIA = reinterpret_cast<float *>(nIA2);
  float *lam = reinterpret_cast<float *>(lam2);
  float *aN = reinterpret_cast<float *>(aN2);
  float *dAl = reinterpret_cast<float *>(dAl2);
#pragma unroll
  for (int j = 0; j < 2 * NH; j++) {
    const int n = g * NS + j;
    // gradient arriving at the last state: from the next segment, or dh_last
    const float *gin = (SEG && P.seg_G) ? P.seg_G + (seg * p.Bt * p.Dn) * N : P.dh_last;
    lam[j] = (gin && j < NS && live && n < N) ? gin[(b * p.Dn + d) * N + n] : 0.f;
    aN[j] = 1.f;
    dAl[j] = 0.f;
    if (j < NS && live && n < N) {
      A[j] = -expf(p.A_log[d * N + n]);
      nIA[j] = -1.0f / A[j];
    } else {
      A[j] = 0.f;
      nIA[j] = 0.f;
    }
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
  float accD = 0.f, accDtb = 0.f, accCb = 0.f, accW[4] = {0.f, 0.f, 0.f, 0.f};

  const int64_t row0 = (b * p.Dn + d0) * L;
  const Tin *gx = static_cast<const Tin *>(p.x) + row0;
  const Tin *gdt = static_cast<const Tin *>(p.dt) + row0;
  const Tin *gz = has_z ? static_cast<const Tin *>(p.z) + row0 : nullptr;
  const Tin *gdo = static_cast<const Tin *>(P.dout) + row0;
  const Tin *gB = static_cast<const Tin *>(p.B) + b * N * L;
  const Tin *gC = static_cast<const Tin *>(p.C) + b * N * L;
  const int n_rows = (int)imin64(NP, N);
  const float *states = P.chunk_states ? P.chunk_states : p.chunk_states;

  // dc of the (non-existent) steps after the sequence end are zero
  for (int i = tid; i < CH * S::DCS; i += kThreads) dcs[i] = 0.f;

  const int64_t n_stages = (te - ts + TS - 1) / TS;
  // TMA stage copies where the rows are 16-byte aligned: one box per tensor and stage, issued by
  // one thread, counted on the buffer's mbarrier (x from kPre steps before the stage: its halo)
  uint64_t *sbar = reinterpret_cast<uint64_t *>(smem + S::bar_off);
  const bool tma = P.f.tma && (static_cast<uint32_t>(__cvta_generic_to_shared(smem)) & 127u) == 0;
  if (tma && tid == 0) {
    mbar_init(sbar, 1);
    mbar_init(sbar + 1, 1);
  }
  if (tma) __syncthreads();  // the barriers are initialised before anyone polls them
  auto issue = [&](int64_t stage, int buf) {
    const int64_t t0 = ts + stage * TS;
    if (tma) {
      if (tid == 0) {
        const uint32_t bytes = (uint32_t)(sizeof(Tin) * CH * (S::XS + TS * (has_z ? 3 : 2)));
        mbar_expect_tx(sbar + buf, bytes);
        tma_load_3d(xs + buf * CH * S::XS, &tmx, (int)(t0 - kPre), (int)d0, (int)b, sbar + buf);
        tma_load_3d(dts + buf * CH * TS, &tmdt, (int)t0, (int)d0, (int)b, sbar + buf);
        if (has_z) tma_load_3d(zs + buf * CH * TS, &tmz, (int)t0, (int)d0, (int)b, sbar + buf);
        tma_load_3d(dos + buf * CH * TS, &tmdo, (int)t0, (int)d0, (int)b, sbar + buf);
      }
      return;
    }
    stage_rows<Tin, CH, kPre + TS>(xs + buf * CH * S::XS, S::XS, gx, L, rows_valid, t0 - kPre, L, vec);
    stage_rows<Tin, CH, TS>(dts + buf * CH * TS, TS, gdt, L, rows_valid, t0, L, vec);
    if (has_z) stage_rows<Tin, CH, TS>(zs + buf * CH * TS, TS, gz, L, rows_valid, t0, L, vec);
    stage_rows<Tin, CH, TS>(dos + buf * CH * TS, TS, gdo, L, rows_valid, t0, L, vec);
    cp_async_commit();
  };

  BCStager<Tin, NP, kThreads, TS> bc;
  if (n_stages > 0) {
    const int lbuf = (int)((n_stages - 1) & 1);
    issue(n_stages - 1, lbuf);
    bc.load(gB, gC, n_rows, ts + (n_stages - 1) * TS, L, vec);
    bc.store(Bs + lbuf * TS * S::BS, Cs + lbuf * TS * S::BS, S::BS);
    if (n_stages > 1) bc.load(gB, gC, n_rows, ts + (n_stages - 2) * TS, L, vec);
  }
  for (int64_t st = n_stages - 1; st >= 0; st--) {
    const int buf = (int)(st & 1), pbuf = buf ^ 1;
    const int64_t t0 = ts + st * TS;
    if (tma)  // buffers are used from the last stage down: use (n_stages - 1 - st) / 2 of buffer buf
      mbar_wait(sbar + buf, (uint32_t)(((n_stages - 1 - st) >> 1) & 1));  // bounded
    else
      cp_async_wait<0>();
    __syncthreads();  // stage st landed; B/C rows of stage st written; stage st+1's buffers free
    if (st > 0) {
      issue(st - 1, pbuf);
      bc.store(Bs + pbuf * TS * S::BS, Cs + pbuf * TS * S::BS, S::BS);
      if (st > 1) bc.load(gB, gC, n_rows, ts + (st - 2) * TS, L, vec);
    }
    const float *Bst = Bs + buf * TS * S::BS;
    const float *Cst = Cs + buf * TS * S::BS;
    const Tin *xrow = xs + (buf * CH + c) * S::XS + kPre;
    const Tin *dtrow = dts + (buf * CH + c) * TS;
    const Tin *zrow = zs + (buf * CH + c) * TS;
    const Tin *dorow = dos + (buf * CH + c) * TS;
    if (t0 == 0 && has_conv && p.conv_hist && p.K > 1) {
      // the carried inputs before step 0 (newest-first) replace the zero fill of the prefix
      if (live && g == 0) {
        const Tin *hr = static_cast<const Tin *>(p.conv_hist) + (b * p.Dn + d) * (p.K - 1);
        for (int j = 0; j < p.K - 1; j++) xs[(buf * CH + c) * S::XS + kPre - 1 - j] = hr[j];
      }
      __syncwarp();
    }
    const int tb = g * EPL;  // first owned step (stage-local)

    // the stage's saved start state, requested now so that phase A hides the load: the state
    // after the previous chunk of SSM_STATE_CHUNK = TS steps, h0 for the first, else zero; one
    // 16-byte load where base, row and lane offset allow it
    float2 hs2[NH];
    {
      float *hs = reinterpret_cast<float *>(hs2);
      const float *src = t0 > 0 ? states + ((b * p.Dn + d) * p.n_ck + (t0 / TS - 1)) * N
                                : (p.h0 ? p.h0 + (b * p.Dn + d) * N : nullptr);
      bool vec4 = false;
      if constexpr (NS == 4) {
        vec4 = N % 4 == 0 && src && live && g * NS < N &&
               (reinterpret_cast<uintptr_t>(t0 > 0 ? states : p.h0) & 15) == 0;
        if (vec4) {
          const float4 v = *reinterpret_cast<const float4 *>(src + g * NS);
          hs2[0] = make_float2(v.x, v.y);
          hs2[1] = make_float2(v.z, v.w);
        }
      }
      if (!vec4) {
#pragma unroll
        for (int j = 0; j < 2 * NH; j++) {
          const int n = g * NS + j;
          hs[j] = (j < NS && live && n < N && src) ? src[n] : 0.f;
        }
      }
    }

    // (A) per-element values of the owned steps: (Delta, u, dy, dSiLU/dc) -> e3, (dDelta/dv,
    //     dout/dz) -> pe
    {
      float xw[EPL + 4], dtw[EPL], zw[EPL], dow[EPL];
      load_window<Tin, EPL + 4>(xw, xrow + tb - 4);
      load_window<Tin, EPL>(dtw, dtrow + tb);
      load_window<Tin, EPL>(dow, dorow + tb);
      if (has_z) load_window<Tin, EPL>(zw, zrow + tb);
#pragma unroll
      for (int j = 0; j < EPL; j++) {
        // u = SiLU(c) with dSiLU/dc = s (1 + c (1 - s)); Delta = softplus(v) with dDelta/dv =
        // sigmoid(v); out = y SiLU(z) with dout/dz = y s_z (1 + z (1 - s_z))
        float u, gc = 1.f;
        if (has_conv) {
          float acc = cbias;
#pragma unroll
          for (int k = 0; k < 4; k++) acc = fmaf(w4[k], xw[j + 4 - k], acc);
          const float sc = sigmoid<PRECISE>(acc);
          u = acc * sc;
          gc = sc * fmaf(acc, 1.f - sc, 1.f);
        } else {
          u = xw[j + 4];
        }
        const float v = dtw[j] + dtb;
        float dl = v, sv = 1.f;
        if (p.delta_softplus) {
          dl = softplus<PRECISE>(v);
          sv = sigmoid<PRECISE>(v);
        }
        float dy = dow[j], gz = 0.f;
        if (has_z) {
          const float sz = sigmoid<PRECISE>(zw[j]);
          dy *= zw[j] * sz;
          gz = dow[j] * sz * fmaf(zw[j], 1.f - sz, 1.f);
        }
        if (t0 + tb + j >= te) {  // padded steps are identity steps with no inputs
          u = 0.f;
          dl = 0.f;
          dy = 0.f;
          gc = 0.f;
          sv = 0.f;
          gz = 0.f;
        }
        e3[c * S::ES + tb + j] = make_float4(dl, u, dy, gc);
        pe[c * S::ES + tb + j] = make_float2(sv, gz);
      }
    }
    __syncwarp();

    // (B) recompute the stage forward from its saved start state; h (and A_bar unless the
    //     adjoint recomputes it) of every step go to TMEM, the readout partials to y0
    {
      float2 h2[NH];
      float *h = reinterpret_cast<float *>(h2);
#pragma unroll
      for (int q = 0; q < NH; q++) h2[q] = hs2[q];
      float *my0 = y0 + c * S::YC + g * S::YG;
#pragma unroll
      for (int tq = 0; tq < TS; tq += 4) {
        float4 eq[4];
        float2 Bq[4][NH], Cq[4][NH];
#pragma unroll
        for (int tt = 0; tt < 4; tt++) {
          const int t = tq + tt;
          eq[tt] = e3[c * S::ES + t];
          load_states<NS>(reinterpret_cast<float *>(Bq[tt]), Bst + t * S::BS + g * NS);
          load_states<NS>(reinterpret_cast<float *>(Cq[tt]), Cst + t * S::BS + g * NS);
        }
        float hv[GV], av[GV], yq[4];
#pragma unroll
        for (int tt = 0; tt < 4; tt++) {
          if (PAIRS) {
            const float2 dl2 = make_float2(eq[tt].x, eq[tt].x), u2 = make_float2(eq[tt].y, eq[tt].y);
            const float dlg = eq[tt].x * kLog2e;
            float2 y2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < NH; q++) {
              const float2 x = __fmul2_rn(make_float2(dlg, dlg), A2[q]);
              float2 a;
              a.x = ex2_approx(x.x);
              a.y = ex2_approx(x.y);
              if (EULER) {
                h2[q] = __ffma2_rn(a, h2[q], __fmul2_rn(__fmul2_rn(Bq[tt][q], u2), dl2));  // a h + Delta B u
              } else {
                const float2 nw = __fmul2_rn(__fmul2_rn(Bq[tt][q], u2), nIA2[q]);  // -B u / A
                h2[q] = __ffma2_rn(a, __ffma2_rn(nw, make_float2(-1.f, -1.f), h2[q]), nw);
              }
              av[tt * NS + 2 * q] = a.x;
              av[tt * NS + 2 * q + 1] = a.y;
              hv[tt * NS + 2 * q] = h2[q].x;
              hv[tt * NS + 2 * q + 1] = h2[q].y;
              y2 = __ffma2_rn(Cq[tt][q], h2[q], y2);
            }
            yq[tt] = y2.x + y2.y;
          } else {
            const float *Bt = reinterpret_cast<const float *>(Bq[tt]);
            const float *Ct = reinterpret_cast<const float *>(Cq[tt]);
            float y = 0.f;
#pragma unroll
            for (int j = 0; j < NS; j++) {
              const float nw = Bt[j] * eq[tt].y * nIA[j];  // -B u / A
              if (PRECISE) {
                const float em1 = expm1f(eq[tt].x * A[j]);
                h[j] = EULER ? fmaf(em1, h[j], fmaf(eq[tt].x * Bt[j], eq[tt].y, h[j]))
                             : fmaf(em1, h[j] - nw, h[j]);
                av[tt * NS + j] = em1;
              } else {
                const float a = ex2_approx((eq[tt].x * kLog2e) * A[j]);
                h[j] = EULER ? fmaf(a, h[j], eq[tt].x * Bt[j] * eq[tt].y) : fmaf(a, h[j] - nw, nw);
                av[tt * NS + j] = a;
              }
              hv[tt * NS + j] = h[j];
              y = fmaf(Ct[j], h[j], y);
            }
            yq[tt] = y;
          }
        }
        *reinterpret_cast<float4 *>(my0 + tq) = make_float4(yq[0], yq[1], yq[2], yq[3]);
        __syncwarp();  // the TMEM stores are warp-collective
        tmem_st<GV>(th + tq * NS, hv);
        if constexpr (!S::AREC) tmem_st<GV>(ta + tq * NS, av);
      }
    }
    tmem_wait_st();
    __syncwarp();
    float yfin[EPL];
    {
      float o[EPL];
#pragma unroll
      for (int j = 0; j < EPL; j++) o[j] = 0.f;
#pragma unroll
      for (int gg = 0; gg < G; gg++) {
        float part[EPL];
        load_floats<EPL>(part, y0 + c * S::YC + gg * S::YG + tb);
#pragma unroll
        for (int j = 0; j < EPL; j++) o[j] += part[j];
      }
#pragma unroll
      for (int j = 0; j < EPL; j++) yfin[j] = fmaf(Dd, e3[c * S::ES + tb + j].y, o[j]);
    }
    __syncwarp();  // y0 is reused for the du partials

    // (C) the adjoint backwards through the stage, one 4-step TMEM group per quarter. The dB / dC
    //     partials are summed over the CTA's channels: with the butterfly, per step inside each
    //     warp and once per stage across the 4 warps; otherwise through shared memory after
    //     every quarter
    float duo[EPL], ddo[EPL];  // lane sums of du / dDelta of the owned steps (shuffle path)
#pragma unroll
    for (int j = 0; j < EPL; j++) {
      duo[j] = 0.f;
      ddo[j] = 0.f;
    }
#pragma unroll
    for (int hf = TS / RH - 1; hf >= 0; hf--) {
      const int tq = hf * RH;
      float hv[GV], av[GV];
      if constexpr (S::AREC)
        tmem_ld1<GV>(th + tq * NS, hv);
      else
        tmem_ld2<GV>(th + tq * NS, hv, ta + tq * NS, av);
      float duq[4], ddq[4];
#pragma unroll
      for (int tt = 3; tt >= 0; tt--) {
        const int tl = tq + tt;
        const float4 e = e3[c * S::ES + tl];  // (dl, u, dy, gc)
        float2 Bv[NH], Cv[NH];
        load_states<NS>(reinterpret_cast<float *>(Bv), Bst + tl * S::BS + g * NS);
        load_states<NS>(reinterpret_cast<float *>(Cv), Cst + tl * S::BS + g * NS);
        float2 nB2[NH], dC2[NH];
        float *nB = reinterpret_cast<float *>(nB2);
        float *dCv = reinterpret_cast<float *>(dC2);
        float ndu = 0.f, dd = 0.f;
        if (PAIRS) {
          float2 ndu2 = make_float2(0.f, 0.f), dd2 = make_float2(0.f, 0.f);
          const float2 dl2 = make_float2(e.x, e.x), u2 = make_float2(e.y, e.y), dy2 = make_float2(e.z, e.z);
#pragma unroll
          for (int q = 0; q < NH; q++) {
            float2 a2;
            if constexpr (S::AREC) {
              const float dlg = e.x * kLog2e;
              const float2 x = __fmul2_rn(make_float2(dlg, dlg), A2[q]);  // as in the recompute: same bits
              a2 = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            } else {
              a2 = make_float2(av[tt * NS + 2 * q], av[tt * NS + 2 * q + 1]);
            }
            const float2 hs = make_float2(hv[tt * NS + 2 * q], hv[tt * NS + 2 * q + 1]);
            lam2[q] = __ffma2_rn(aN2[q], lam2[q], __fmul2_rn(Cv[q], dy2));         // lambda_t
            aN2[q] = a2;
            // kb = -dB_bar/dB: (A_bar - 1)(-1/A) for the exact ZOH, -Delta for Euler
            // (A_bar - 1)(-1/A) as one fused multiply-add: A_bar - 1 is exact in fp32, so this is
            // the same single rounding as the product
            const float2 em1n = EULER ? make_float2(-e.x, -e.x)
                                      : __ffma2_rn(a2, nIA2[q], make_float2(-nIA2[q].x, -nIA2[q].y));
            const float2 k = __fmul2_rn(lam2[q], em1n);
            const float2 nlb = __fmul2_rn(k, Bv[q]);                                // -lambda B_bar
            ndu2 = __fadd2_rn(ndu2, nlb);
            nB2[q] = __fmul2_rn(k, u2);                                             // -dB partial
            dC2[q] = __fmul2_rn(hs, dy2);
            // dh_t/dDelta = A h_t + B u (ZOH) or A h_t + B u (1 - A Delta) (Euler)
            float2 bu = __fmul2_rn(Bv[q], u2);
            if (EULER) bu = __fmul2_rn(bu, __ffma2_rn(A2[q], make_float2(-e.x, -e.x), make_float2(1.f, 1.f)));
            const float2 dterm = __fmul2_rn(lam2[q], __ffma2_rn(A2[q], hs, bu));
            dd2 = __fadd2_rn(dd2, dterm);
            dAl2[q] = __ffma2_rn(u2, nlb, __ffma2_rn(dl2, dterm, dAl2[q]));       // A dA
          }
          ndu = ndu2.x + ndu2.y;
          dd = dd2.x + dd2.y;
        } else {
          const float *Bt = reinterpret_cast<const float *>(Bv);
          const float *Ct = reinterpret_cast<const float *>(Cv);
#pragma unroll
          for (int j = 0; j < NS; j++) {
            const float aj = S::AREC ? ex2_approx((e.x * kLog2e) * A[j]) : av[tt * NS + j];
            const float em1 = PRECISE ? aj : aj - 1.f;
            const float hs = hv[tt * NS + j];
            lam[j] = fmaf(aN[j], lam[j], Ct[j] * e.z);
            aN[j] = PRECISE ? 1.f + aj : aj;
            const float em1n = EULER ? -e.x : em1 * nIA[j];
            const float nlb = lam[j] * (em1n * Bt[j]);
            ndu += nlb;
            nB[j] = lam[j] * em1n * e.y;
            dCv[j] = hs * e.z;
            const float bu = EULER ? Bt[j] * e.y * fmaf(-A[j], e.x, 1.f) : Bt[j] * e.y;
            const float dterm = lam[j] * fmaf(A[j], hs, bu);
            dd += dterm;
            dAl[j] = fmaf(e.y, nlb, fmaf(e.x, dterm, dAl[j]));
          }
        }
        if constexpr (S::BFLY) {
          // reduce-scatter over the warp's 8 channels (lane bits 2, 3, 4): at each level a lane
          // keeps half of its values, sends the other half to its partner and adds what it gets.
          // Lane l ends with quantity l>>4 (0: -dB, 1: dC) of state g*4 + 2*bit3 + bit2.
          const int lane = tid & 31;
          const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
          float s4[4], s2[2];
#pragma unroll
          for (int k = 0; k < 4; k++) {
            const float send = b4 ? nB[k] : dCv[k], keep = b4 ? dCv[k] : nB[k];
            s4[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
          }
#pragma unroll
          for (int k = 0; k < 2; k++) {
            const float send = b3 ? s4[k] : s4[k + 2], keep = b3 ? s4[k + 2] : s4[k];
            s2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
          }
          const float send = b2 ? s2[0] : s2[1], keep = b2 ? s2[1] : s2[0];
          rb[tl * S::WPT + (tid >> 5) * 32 + lane] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        } else {
          store_states<NS>(rb + S::rb_index(0, tt, c, g * NS), nB);
          store_states<NS>(rb + S::rb_index(1, tt, c, g * NS), dCv);
        }
        if (S::SHFL) {
          // sum over the channel's G lanes; the step's owner keeps it
          float su = -ndu, sd = dd;
#pragma unroll
          for (int off = 1; off < G; off <<= 1) {
            su += __shfl_xor_sync(0xffffffffu, su, off);
            sd += __shfl_xor_sync(0xffffffffu, sd, off);
          }
          if (g == tl / EPL) {
            duo[tl % EPL] = su;
            ddo[tl % EPL] = sd;
          }
        } else {
          duq[tt] = -ndu;
          ddq[tt] = dd;
        }
      }
      if (!S::SHFL) {
        *reinterpret_cast<float4 *>(y0 + c * S::YC + g * S::YG + tq) = make_float4(duq[0], duq[1], duq[2], duq[3]);
        *reinterpret_cast<float4 *>(y1 + c * S::YC + g * S::YG + tq) = make_float4(ddq[0], ddq[1], ddq[2], ddq[3]);
      }
      if constexpr (!S::BFLY) {
        __syncthreads();  // the quarter's dB / dC partials of every channel are in place
        {
          // every thread runs the same number of rounds, so the shuffles below see whole warps
          // (threads without a column still take part in them)
          constexpr int NQ = NP / 4;
          constexpr int NGRP = 2 * RH * NQ;
          // two threads per column: fewer shuffles than a wider split, and half the CTA's warps
          // stay free (measured fastest on B200)
          constexpr int SPLIT = NGRP >= kThreads ? 1 : 2;
          constexpr int CPS = CH / SPLIT;
          constexpr int ROUNDS = (NGRP * SPLIT + kThreads - 1) / kThreads;
          const int part = tid % SPLIT;
  #pragma unroll
          for (int r = 0; r < ROUNDS; r++) {
            const int gi = (r * kThreads + tid) / SPLIT;
            const bool ok = gi < NGRP;
            const int which = gi / (RH * NQ), rem = gi % (RH * NQ), q = rem / RH, tt = rem % RH;
            float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
            if (ok) {
              if (SPLIT > 1) {
                // this thread's channels lie in one half: walk them with a fixed stride
                const float *src = rb + S::rb_index(which, tt, part * CPS, 4 * q);
  #pragma unroll 8
                for (int ci = 0; ci < CPS; ci++) {
                  const float4 v = *reinterpret_cast<const float4 *>(src + ci * NP);
                  a01 = __fadd2_rn(a01, make_float2(v.x, v.y));
                  a23 = __fadd2_rn(a23, make_float2(v.z, v.w));
                }
              } else {
  #pragma unroll 4
                for (int ci = 0; ci < CPS; ci++) {
                  const float4 v = *reinterpret_cast<const float4 *>(rb + S::rb_index(which, tt, ci, 4 * q));
                  a01 = __fadd2_rn(a01, make_float2(v.x, v.y));
                  a23 = __fadd2_rn(a23, make_float2(v.z, v.w));
                }
              }
            }
            float4 acc = make_float4(a01.x, a01.y, a23.x, a23.y);
  #pragma unroll
            for (int off = 1; off < SPLIT; off <<= 1) {
              acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
              acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
              acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
              acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
            }
            const int64_t t = t0 + tq + tt;
            if (ok && part == 0 && t < te) {
              float *dst = (which ? P.p_dC : P.p_dB) + ((tile * p.Bt + b) * N) * L + t;
              const float sg = which ? 1.f : -1.f;  // dB partials were kept negated
              const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
  #pragma unroll
              for (int k = 0; k < 4; k++)
                if (4 * q + k < N) dst[(int64_t)(4 * q + k) * L] = sg * vals[k];
            }
          }
        }
        __syncthreads();  // rb is rewritten by the next quarter
      }
    }
    if constexpr (S::BFLY) {
      // the stage's per-warp 8-channel sums -> this tile's dB / dC partials: thread (slot l, 4-step
      // group tq) adds the 4 warps in order and writes 4 consecutive steps of one (quantity, state)
      __syncthreads();
      const int l = tid >> 2, tq = tid & 3;
      float acc[4];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const float *src = rb + (4 * tq + i) * S::WPT + l;
        acc[i] = ((src[0] + src[32]) + src[64]) + src[96];
      }
      // with a cluster, the CTAs of the cluster (consecutive channel tiles of this batch element)
      // first add their sums in rank order: every thread parks its 4 values, and thread i of
      // rank r then adds item r * 128 / CL + i of every rank through distributed shared memory
      int item = tid, ptile = (int)tile;
      bool mine = true;
      if (P.cluster > 1) {
        float4 *cx = reinterpret_cast<float4 *>(smem + S::cx_off) + (st & 1) * kThreads;
        cx[tid] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        cluster_sync();  // every rank's sums of this stage are in place
        const uint32_t rank = cluster_rank();
        const int per = kThreads / P.cluster;
        mine = tid < per;
        item = (int)rank * per + tid;
        ptile = (int)(tile / P.cluster);
        if (mine) {
          float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int r = 0; r < P.cluster; r++) {
            const float4 v = ld_cluster_f4(cx + item, (uint32_t)r);
            tot.x += v.x;
            tot.y += v.y;
            tot.z += v.z;
            tot.w += v.w;
          }
          acc[0] = tot.x;
          acc[1] = tot.y;
          acc[2] = tot.z;
          acc[3] = tot.w;
        }
      }
      const int li = item >> 2, qi = item & 3;
      const int wi = li >> 4, ni = (li & 3) * 4 + ((li >> 3) & 1) * 2 + ((li >> 2) & 1);
      const int64_t t = t0 + 4 * qi;
      if (mine && ni < N && t < te) {
        const float sg = wi ? 1.f : -1.f;  // dB partials were kept negated
        float *dst = (wi ? P.p_dC : P.p_dB) + (((int64_t)ptile * p.Bt + b) * N + ni) * L + t;
        if (vec && t + 3 < te) {
          *reinterpret_cast<float4 *>(dst) = make_float4(sg * acc[0], sg * acc[1], sg * acc[2], sg * acc[3]);
        } else {
#pragma unroll
          for (int i = 0; i < 4; i++)
            if (t + i < te) dst[i] = sg * acc[i];
        }
      }
    }

    __syncwarp();  // the du / dDelta partial rows (shared-memory path) are complete
    // (D) per-element gradients of the owned steps
    {
      float dup[EPL], ddp[EPL];
      if (S::SHFL) {
#pragma unroll
        for (int j = 0; j < EPL; j++) {
          dup[j] = duo[j];
          ddp[j] = ddo[j];
        }
      } else {
#pragma unroll
        for (int j = 0; j < EPL; j++) {
          dup[j] = 0.f;
          ddp[j] = 0.f;
        }
#pragma unroll
        for (int gg = 0; gg < G; gg++) {
          float a0[EPL], a1[EPL];
          load_floats<EPL>(a0, y0 + c * S::YC + gg * S::YG + tb);
          load_floats<EPL>(a1, y1 + c * S::YC + gg * S::YG + tb);
#pragma unroll
          for (int j = 0; j < EPL; j++) {
            dup[j] += a0[j];
            ddp[j] += a1[j];
          }
        }
      }
      float xw[EPL + 4];
      if (has_conv) load_window<Tin, EPL + 4>(xw, xrow + tb - 4);
      float dzv[EPL], dtv[EPL], dcv[EPL];
#pragma unroll
      for (int j = 0; j < EPL; j++) {
        const float4 e = e3[c * S::ES + tb + j];  // (dl, u, dy, gc); zero past L
        const float2 f = pe[c * S::ES + tb + j];  // (sv, gz); zero past L
        const float du = fmaf(Dd, e.z, dup[j]);
        accD = fmaf(e.z, e.y, accD);
        dzv[j] = yfin[j] * f.y;
        dtv[j] = ddp[j] * f.x;
        accDtb += dtv[j];
        dcv[j] = du * e.w;
        if (has_conv) {
          if (EPL != 4) dcs[c * S::DCS + tb + j] = dcv[j];
          accCb += dcv[j];
#pragma unroll
          for (int k = 0; k < 4; k++) accW[k] = fmaf(dcv[j], xw[j + 4 - k], accW[k]);
        }
      }
      if (EPL == 4 && has_conv)
        *reinterpret_cast<float4 *>(dcs + c * S::DCS + tb) = make_float4(dcv[0], dcv[EPL > 1 ? 1 : 0],
                                                                         dcv[EPL > 2 ? 2 : 0], dcv[EPL > 3 ? 3 : 0]);
      if (live) {
        const int64_t roff = (b * p.Dn + d) * L;
        if (has_z && P.dz) store_run<float, EPL>(P.dz + roff, t0 + tb, te, dzv, vec);
        if (P.ddt) store_run<float, EPL>(P.ddt + roff, t0 + tb, te, dtv, vec);
        if (!has_conv && P.dx) store_run<float, EPL>(P.dx + roff, t0 + tb, te, dcv, vec);
      }
    }

    // conv backward for the stage: dx_t = sum_k w[k] dc_{t+k} (dc beyond the stage = halo).
    // dcs rows are written and read by the G lanes of their own channel only.
    if (has_conv) {
      __syncwarp();
      {
        float dxv[EPL];
        if constexpr (EPL == 4) {
          // dc of the owned steps and the 4 after them (the next lane's, or the halo)
          const float4 lo = *reinterpret_cast<const float4 *>(dcs + c * S::DCS + tb);
          const float4 hi = *reinterpret_cast<const float4 *>(dcs + c * S::DCS + tb + 4);
          const float dw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
          for (int j = 0; j < EPL; j++) {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < 4; k++) acc = fmaf(w4[k], dw[j + k], acc);
            dxv[j] = acc;
          }
        } else {
#pragma unroll
          for (int j = 0; j < EPL; j++) {
            const int t = tb + j;
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < 4; k++) acc = fmaf(w4[k], dcs[c * S::DCS + t + k], acc);
            dxv[j] = acc;
          }
        }
        if (live && P.dx) store_run<float, EPL>(P.dx + (b * p.Dn + d) * L, t0 + tb, te, dxv, vec);
      }
      __syncwarp();
      if (st == 0 && live && g == 0 && p.K > 1 && (seg > 0 ? P.seg_dxh != nullptr : P.dconv_hist != nullptr)) {
        // x_{ts-1-j} reaches c_t through tap k = t - ts + 1 + j: the carried history's gradient
        // for the first segment, else a term of the previous segment's dx (added afterwards)
        for (int j = 0; j < p.K - 1; j++) {
          float acc = 0.f;
          for (int k = j + 1; k < p.K; k++) acc = fmaf(w4[k], dcs[c * S::DCS + k - j - 1], acc);
          if (SEG && seg > 0)
            P.seg_dxh[sbd * 4 + j] = acc;
          else
            P.dconv_hist[(b * p.Dn + d) * (p.K - 1) + j] = acc;
        }
      }
      // this stage's first 3 dc values become the halo of the stage before it
      if (g == 0)
        for (int k = 0; k < 3; k++) dcs[c * S::DCS + TS + k] = dcs[c * S::DCS + k];
      __syncwarp();
    }
  }

  // per-channel parameter partials for this batch element; gradient of the carried state
  // (h_0 = A_bar_0 h0 + ..., so dh0 = A_bar_0 lambda_0)
  if (live) {
#pragma unroll
    for (int j = 0; j < NS; j++) {
      const int n = g * NS + j;
      if (n < N) {
        P.p_dA_log[sbd * N + n] = dAl[j];
        if (P.dh0 && seg == 0) P.dh0[(b * p.Dn + d) * N + n] = aN[j] * lam[j];
      }
    }
  }
#pragma unroll
  for (int off = 1; off < G; off <<= 1) {
    accD += __shfl_xor_sync(0xffffffffu, accD, off);
    accDtb += __shfl_xor_sync(0xffffffffu, accDtb, off);
    accCb += __shfl_xor_sync(0xffffffffu, accCb, off);
#pragma unroll
    for (int k = 0; k < 4; k++) accW[k] += __shfl_xor_sync(0xffffffffu, accW[k], off);
  }
  if (live && g == 0) {
    P.p_dD[sbd] = accD;
    P.p_ddt_bias[sbd] = accDtb;
    P.p_dconv_b[sbd] = accCb;
    for (int k = 0; k < 4; k++) P.p_dconv_w[sbd * 4 + k] = accW[k];
  }
  if (S::BFLY && P.cluster > 1) cluster_sync();  // no rank leaves while another may still read its rows
  tmem_free_cta(tbase, S::NCOLS);
}

// dB/dC: add the channel-tile partials in tile order.
__global__ void reduce_tiles_kernel(const float *__restrict__ pdB, const float *__restrict__ pdC,
                                    float *dB, float *dC, int64_t n_tiles, int64_t per_tile) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= per_tile) return;
  float sb = 0.f, sc = 0.f;
  for (int64_t k = 0; k < n_tiles; k++) {
    sb += pdB[k * per_tile + i];
    sc += pdC[k * per_tile + i];
  }
  if (dB) dB[i] = sb;
  if (dC) dC[i] = sc;
}

// per-channel parameters: add the (segment, batch) partials in order.
// The same sum, 4 consecutive elements per thread with 16-byte accesses and 8 tiles' loads in
// flight; the adds still run in tile order, so the result is bitwise that of the scalar kernel.
// dB / dC: thread i adds 4 consecutive floats of the channel-tile partials in tile order.
__device__ __forceinline__ void reduce_tiles_vec_at(const float4 *__restrict__ pdB, const float4 *__restrict__ pdC,
                                                    float4 *dB, float4 *dC, int64_t n_tiles, int64_t per_tile4,
                                                    int64_t i) {
  if (i >= per_tile4) return;
  float4 sb = make_float4(0.f, 0.f, 0.f, 0.f), sc = sb;
  constexpr int U = 8;
  for (int64_t k0 = 0; k0 < n_tiles; k0 += U) {
    float4 vb[U], vc[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      if (k0 + u < n_tiles) {
        vb[u] = pdB[(k0 + u) * per_tile4 + i];
        vc[u] = pdC[(k0 + u) * per_tile4 + i];
      }
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      if (k0 + u < n_tiles) {
        sb.x += vb[u].x; sb.y += vb[u].y; sb.z += vb[u].z; sb.w += vb[u].w;
        sc.x += vc[u].x; sc.y += vc[u].y; sc.z += vc[u].z; sc.w += vc[u].w;
      }
    }
  }
  if (dB) dB[i] = sb;
  if (dC) dC[i] = sc;
}

// per-channel parameters: thread j = d * N + n adds the (segment, batch) partials of dA_log[d, n]
// in order, and the thread of state 0 those of the channel's D, dt_bias, conv bias and taps.
__device__ __forceinline__ void reduce_params_at(const BwdParams &P, int64_t j) {
  const int64_t Dn = P.f.Dn, N = P.f.N, Bt = P.f.Bt * P.n_seg;
  if (j >= Dn * N) return;
  const int64_t d = j / N, n = j - d * N;
  if (P.dA_log) {
    float s = 0.f;
    for (int64_t b = 0; b < Bt; b++) s += P.p_dA_log[b * Dn * N + j];
    P.dA_log[j] = s;
  }
  if (n != 0) return;
  float sD = 0.f, sT = 0.f, sCb = 0.f, sW[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t b = 0; b < Bt; b++) {
    sD += P.p_dD[b * Dn + d];
    sT += P.p_ddt_bias[b * Dn + d];
    sCb += P.p_dconv_b[b * Dn + d];
    for (int k = 0; k < 4; k++) sW[k] += P.p_dconv_w[(b * Dn + d) * 4 + k];
  }
  if (P.dD) P.dD[d] = sD;
  if (P.ddt_bias) P.ddt_bias[d] = sT;
  if (P.dconv_b) P.dconv_b[d] = sCb;
  if (P.dconv_w)
    for (int k = 0; k < P.f.K; k++) P.dconv_w[d * P.f.K + k] = sW[k];
}

// Both reductions in one launch where the dB / dC rows are whole 16-byte vectors: blocks
// [0, n_tb) take the dB / dC tiles, the blocks after them the per-channel parameters.
__global__ void reduce_all_vec_kernel(const BwdParams P, int64_t n_tb, int64_t per_tile4) {
  if ((int64_t)blockIdx.x < n_tb) {
    reduce_tiles_vec_at(reinterpret_cast<const float4 *>(P.p_dB), reinterpret_cast<const float4 *>(P.p_dC),
                        reinterpret_cast<float4 *>(P.dB), reinterpret_cast<float4 *>(P.dC), P.n_ptiles,
                        per_tile4, (int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    return;
  }
  reduce_params_at(P, ((int64_t)blockIdx.x - n_tb) * blockDim.x + threadIdx.x);
}

__global__ void reduce_params_kernel(const BwdParams P) {
  reduce_params_at(P, (int64_t)blockIdx.x * blockDim.x + threadIdx.x);
}

// Split-L pass 1: for every segment but the first, the adjoint run backwards from a zero arrival
// -- lambda_t = dy_t C_t + A_bar_{t+1} lambda_{t+1} over [ts, te) -- needs only Delta, dy and C
// (no state recompute). Keeps A_bar_ts lambda_ts (what the segment hands to the one before it
// when nothing arrives) and the sum of Delta. One thread per (segment, b, d, group of SG states);
// the sequence is walked in 8-step blocks read as 16-byte vectors when rows are aligned.
template <typename Tin, int SG>
__global__ void seg_adjoint_kernel(const BwdParams P) {
  constexpr bool PRECISE = sizeof(Tin) == 4;
  const FwdParams &p = P.f;
  const int64_t L = p.L, N = p.N, NQ = (N + SG - 1) / SG, BD = p.Bt * p.Dn;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)(P.n_seg - 1) * BD * NQ) return;
  const int64_t q = i % NQ, sb = i / NQ, bd = sb % BD, seg = 1 + sb / BD;
  const int64_t b = bd / p.Dn, d = bd % p.Dn;
  const int64_t ts = seg * P.seg_len, te = imin64(L, ts + P.seg_len);
  float A[SG], Ac[SG], lam[SG], an[SG];
#pragma unroll
  for (int j = 0; j < SG; j++) {
    const int64_t n = SG * q + j;
    A[j] = n < N ? -expf(p.A_log[d * N + n]) : 0.f;
    Ac[j] = PRECISE ? A[j] : A[j] * kLog2e;
    lam[j] = 0.f;
    an[j] = 1.f;
  }
  const float dtb = p.dt_bias ? p.dt_bias[d] : 0.f;
  const Tin *dtr = static_cast<const Tin *>(p.dt) + bd * L;
  const Tin *zr = p.z ? static_cast<const Tin *>(p.z) + bd * L : nullptr;
  const Tin *dor = static_cast<const Tin *>(P.dout) + bd * L;
  const Tin *Cb = static_cast<const Tin *>(p.C) + (b * N + SG * q) * L;
  const int nv = (int)imin64(SG, N - SG * q);  // valid states of this group
  float sdl = 0.f;
  // one step t with the group's C_t values in cv
  auto step = [&](float dtv, float zv, float dov, const float *cv) {
    const float v = dtv + dtb;
    const float dl = p.delta_softplus ? softplus<PRECISE>(v) : v;
    float dy = dov;
    if (zr) dy *= zv * sigmoid<PRECISE>(zv);
    sdl += dl;
#pragma unroll
    for (int j = 0; j < SG; j++) {
      lam[j] = fmaf(an[j], lam[j], dy * cv[j]);
      an[j] = PRECISE ? expf(dl * A[j]) : ex2_approx(dl * Ac[j]);
    }
  };
  int64_t t = te - 1;
  // the ragged end first (te - ts need not be a multiple of 8), one step at a time
  for (int64_t k = 0; k < (te - ts) % 8; k++, t--) {
    float cv[SG];
#pragma unroll
    for (int j = 0; j < SG; j++) cv[j] = j < nv ? to_f32(Cb[(int64_t)j * L + t]) : 0.f;
    step(to_f32(dtr[t]), zr ? to_f32(zr[t]) : 0.f, to_f32(dor[t]), cv);
  }
  // then whole 8-step blocks [t - 7, t], ts a multiple of 64 so t - 7 is a multiple of 8
  for (; t >= ts; t -= 8) {
    const int64_t t0 = t - 7;
    float dtw[8], zw[8], dow[8], cw[SG][8];
    if (p.vec) {
      load_window<Tin, 8>(dtw, dtr + t0);
      load_window<Tin, 8>(dow, dor + t0);
      if (zr) load_window<Tin, 8>(zw, zr + t0);
#pragma unroll
      for (int j = 0; j < SG; j++) {
        if (j < nv)
          load_window<Tin, 8>(cw[j], Cb + (int64_t)j * L + t0);
        else
#pragma unroll
          for (int e = 0; e < 8; e++) cw[j][e] = 0.f;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; e++) {
        dtw[e] = to_f32(dtr[t0 + e]);
        dow[e] = to_f32(dor[t0 + e]);
        zw[e] = zr ? to_f32(zr[t0 + e]) : 0.f;
#pragma unroll
        for (int j = 0; j < SG; j++) cw[j][e] = j < nv ? to_f32(Cb[(int64_t)j * L + t0 + e]) : 0.f;
      }
    }
    if (!zr)
#pragma unroll
      for (int e = 0; e < 8; e++) zw[e] = 0.f;
#pragma unroll
    for (int e = 7; e >= 0; e--) {
      float cv[SG];
#pragma unroll
      for (int j = 0; j < SG; j++) cv[j] = cw[j][e];
      step(dtw[e], zw[e], dow[e], cv);
    }
  }
  const int64_t row = (seg * BD + bd) * N;
#pragma unroll
  for (int j = 0; j < SG; j++)
    if (j < nv) P.seg_gloc[row + SG * q + j] = an[j] * lam[j];
  if (q == 0) P.seg_sdl[seg * BD + bd] = sdl;
}

// Split-L pass 2: the gradient arriving at every segment's last state, from the end --
// G_last = dh_last, G_{s-1} = A_bar_ts lambda_ts (zero arrival) + exp(A * sum of Delta over s) G_s.
__global__ void seg_adjoint_carry_kernel(const BwdParams P) {
  const FwdParams &p = P.f;
  const int64_t BDN = p.Bt * p.Dn * p.N;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // (b, d, n)
  if (i >= BDN) return;
  const int64_t n = i % p.N, bd = i / p.N, d = bd % p.Dn;
  const float A = -expf(p.A_log[d * p.N + n]);
  float G = P.dh_last ? P.dh_last[i] : 0.f;
  for (int s = P.n_seg - 1; s >= 0; s--) {
    P.seg_G[s * BDN + i] = G;
    if (s > 0) G = fmaf(expf(A * P.seg_sdl[s * p.Bt * p.Dn + bd]), G, P.seg_gloc[s * BDN + i]);
  }
}

// After pass 3: each later segment's gradient w.r.t. the K-1 inputs before it belongs to the
// previous segment's last K-1 steps of dx.
__global__ void seg_dx_fixup_kernel(const BwdParams P) {
  const FwdParams &p = P.f;
  const int64_t BD = p.Bt * p.Dn;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // (segment >= 1, b, d)
  if (i >= (int64_t)(P.n_seg - 1) * BD) return;
  const int64_t bd = i % BD, seg = 1 + i / BD;
  const int64_t ts = seg * P.seg_len;
  for (int j = 0; j < p.K - 1; j++) P.dx[bd * p.L + ts - 1 - j] += P.seg_dxh[(seg * BD + bd) * 4 + j];
}

int bwd_cluster(const LaneLayout &lay, int64_t n_dtiles, int max_cluster) {
  if (lay.G != 4 || lay.NS != 4) return 1;
  for (int cl = 8; cl > 1; cl >>= 1)
    if (cl <= max_cluster && n_dtiles % cl == 0) return cl;
  return 1;
}

size_t bwd_workspace_bytes(int64_t Bt, int64_t Dn, int64_t N, int64_t L, int need_states, int n_seg,
                           int max_cluster) {
  auto rnd = [](size_t x) { return (x + 255) & ~size_t(255); };
  const LaneLayout lay = choose_layout(N, Bt * Dn * n_seg);
  const int64_t ch = channels_per_cta(lay);
  const int64_t n_dtiles = (Dn + ch - 1) / ch;
  const int64_t n_tiles = n_dtiles / bwd_cluster(lay, n_dtiles, max_cluster);  // partial tiles
  const int64_t BD = Bt * Dn, PD = BD * n_seg;  // parameter partials: one row per (segment, b, d)
  size_t s = 0;
  s += rnd(sizeof(float) * PD * N);
  s += rnd(sizeof(float) * PD);
  s += rnd(sizeof(float) * PD);
  s += rnd(sizeof(float) * PD * 4);
  s += rnd(sizeof(float) * PD);
  s += rnd(sizeof(float) * n_tiles * Bt * N * L);
  s += rnd(sizeof(float) * n_tiles * Bt * N * L);
  if (need_states) s += rnd(sizeof(float) * BD * ((L + kSub - 1) / kSub) * N);
  if (n_seg > 1) {
    s += 2 * rnd(sizeof(float) * PD * N);  // seg_G, seg_gloc
    s += rnd(sizeof(float) * PD);          // seg_sdl
    s += rnd(sizeof(float) * PD * 4);      // seg_dxh
  }
  return s;
}

template <int G, int NS, typename Tin>
static cudaError_t launch_bwd_t(const BwdParams &P, cudaStream_t stream) {
  using S = BwdSmem<G, NS, Tin>;
  auto kern = P.n_seg > 1 ? (P.f.euler ? ssm_bwd_kernel<G, NS, Tin, true, true> : ssm_bwd_kernel<G, NS, Tin, false, true>)
                           : (P.f.euler ? ssm_bwd_kernel<G, NS, Tin, true, false> : ssm_bwd_kernel<G, NS, Tin, false, false>);
  // Each resident CTA holds S::NCOLS of the SM's 512 TMEM columns. Ask for enough shared memory
  // that no more CTAs fit on an SM than the columns allow, so no allocation ever has to wait.
  int dev = 0, smem_sm = 0, reserved = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  size_t smem = S::bytes;
  const int max_ctas = 512 / (int)S::NCOLS;
  if (max_ctas < kMaxThreadsPerSM / kThreads) {
    const size_t floor_bytes = (size_t)smem_sm / (max_ctas + 1) + 16 - (size_t)reserved;
    if (smem < floor_bytes) smem = (floor_bytes + 15) & ~size_t(15);
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = P.n_dtiles * P.f.Bt * P.n_seg;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  // TMA boxes for x (the stage plus its kPre-step halo), dt, z and dout where rows are 16-byte aligned
  CUtensorMap mx, mdt, mz, mdo;
  memset(&mx, 0, sizeof(mx));
  memset(&mdt, 0, sizeof(mdt));
  memset(&mz, 0, sizeof(mz));
  memset(&mdo, 0, sizeof(mdo));
  BwdParams Q = P;
  {
    constexpr bool bf = sizeof(Tin) == 2;
    const FwdParams &f = P.f;
    const uint64_t Lq = (uint64_t)f.L, Dq = (uint64_t)f.Dn, Bq = (uint64_t)f.Bt;
    Q.f.tma = f.vec && f.L <= 0x7fffffffLL && f.Dn <= 0x7fffffffLL &&
              encode_tma_3d(&mx, bf, f.x, Lq, Dq, Bq, kPre + S::TS, S::CH) &&
              encode_tma_3d(&mdt, bf, f.dt, Lq, Dq, Bq, S::TS, S::CH) &&
              (!f.z || encode_tma_3d(&mz, bf, f.z, Lq, Dq, Bq, S::TS, S::CH)) &&
              encode_tma_3d(&mdo, bf, P.dout, Lq, Dq, Bq, S::TS, S::CH);
  }
  if (P.cluster > 1) {
    // consecutive blocks are consecutive channel tiles of one (segment, batch element), and the
    // tile count is a multiple of the cluster size, so a cluster never straddles two of them
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)P.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, Q, mx, mdt, mz, mdo);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  kern<<<(unsigned)grid, kThreads, smem, stream>>>(Q, mx, mdt, mz, mdo);
  return cudaGetLastError();
}

template <typename Tin>
static cudaError_t bwd_dispatch(const LaneLayout &lay, const BwdParams &P, cudaStream_t s) {
#define SSM_BWD_CASE(G_, NS_) \
  if (lay.G == G_ && lay.NS == NS_) return launch_bwd_t<G_, NS_, Tin>(P, s);
  SSM_BWD_CASE(4, 1) SSM_BWD_CASE(4, 2) SSM_BWD_CASE(4, 4)
  SSM_BWD_CASE(8, 1) SSM_BWD_CASE(8, 2) SSM_BWD_CASE(8, 4)
  SSM_BWD_CASE(16, 1) SSM_BWD_CASE(16, 2) SSM_BWD_CASE(16, 4)
#undef SSM_BWD_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd(const BwdParams &P, int in_bf16, cudaStream_t stream) {
  cudaError_t e;
  if (!P.chunk_states) {
    // states were not saved by the forward: recompute them (no outputs) into the workspace
    FwdParams f = P.f;
    f.out = nullptr;
    f.u_out = nullptr;
    e = launch_fwd(f, in_bf16, 0, stream);
    if (e != cudaSuccess) return e;
  }
  const LaneLayout lay = choose_layout(P.f.N, P.f.Bt * P.f.Dn * P.n_seg);
  if (P.n_seg > 1) {
    // split-L passes 1 and 2: what arrives at each segment's last state
    constexpr int SG = 8;  // states per thread
    const int64_t n1 = (int64_t)(P.n_seg - 1) * P.f.Bt * P.f.Dn * ((P.f.N + SG - 1) / SG);
    if (in_bf16)
      seg_adjoint_kernel<__nv_bfloat16, SG><<<(unsigned)((n1 + 127) / 128), 128, 0, stream>>>(P);
    else
      seg_adjoint_kernel<float, SG><<<(unsigned)((n1 + 127) / 128), 128, 0, stream>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t bdn = P.f.Bt * P.f.Dn * P.f.N;
    seg_adjoint_carry_kernel<<<(unsigned)((bdn + 255) / 256), 256, 0, stream>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (P.timing_events && P.timing_events[0]) {
    e = cudaEventRecord(static_cast<cudaEvent_t>(P.timing_events[0]), stream);
    if (e != cudaSuccess) return e;
  }
  e = in_bf16 ? bwd_dispatch<__nv_bfloat16>(lay, P, stream) : bwd_dispatch<float>(lay, P, stream);
  if (e != cudaSuccess) return e;
  if (P.timing_events && P.timing_events[1]) {
    e = cudaEventRecord(static_cast<cudaEvent_t>(P.timing_events[1]), stream);
    if (e != cudaSuccess) return e;
  }
  if (P.n_seg > 1 && P.dx && P.f.conv_w && P.f.K > 1) {
    const int64_t n = (int64_t)(P.n_seg - 1) * P.f.Bt * P.f.Dn;
    seg_dx_fixup_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t per_tile = P.f.Bt * P.f.N * P.f.L;
  const int64_t n_pb = (P.f.Dn * P.f.N + 255) / 256;  // blocks of the parameter reduction
  if (P.dB || P.dC) {
    const bool vec = per_tile % 4 == 0 && ((reinterpret_cast<uintptr_t>(P.p_dB) | reinterpret_cast<uintptr_t>(P.p_dC) |
                                             reinterpret_cast<uintptr_t>(P.dB) | reinterpret_cast<uintptr_t>(P.dC)) & 15) == 0;
    if (vec) {
      const int64_t n_tb = (per_tile / 4 + 255) / 256;
      if (n_tb + n_pb > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
      reduce_all_vec_kernel<<<(unsigned)(n_tb + n_pb), 256, 0, stream>>>(P, n_tb, per_tile / 4);
      return cudaGetLastError();
    }
    const int64_t blocks = (per_tile + 255) / 256;
    reduce_tiles_kernel<<<(unsigned)blocks, 256, 0, stream>>>(P.p_dB, P.p_dC, P.dB, P.dC, P.n_ptiles, per_tile);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  reduce_params_kernel<<<(unsigned)n_pb, 256, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace ssm
