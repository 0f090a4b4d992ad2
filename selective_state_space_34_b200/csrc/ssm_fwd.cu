// ssm_fwd.cu -- fused selective-scan forward for sm_100a:
//   causal depthwise conv1d + SiLU  ->  softplus(dt + dt_bias)  ->  exact-ZOH diagonal scan
//   ->  y = C.h + D u  ->  y * SiLU(z)
// (rustytorch commit log, "Real S6 forward"; "Selective Mamba" step; exact zero-order hold of
// "Sequence and state-space models", state_space_models).
//
// Work decomposition. One CTA owns CH = 128 / G channels of one batch element and walks the whole
// sequence (or, with split-L, one segment of it) in stages of kT time steps. Inside a warp, the G lanes of a channel each hold NS of its
// states in fp32 registers and run the recurrence sequentially in time; B_t and C_t are shared by
// all channels, so every lane reads them as shared-memory broadcasts. Per-element work (conv,
// SiLU, softplus, gate, the D skip and the store) is split over the G lanes of a channel so that
// nothing is computed twice; u and Delta reach the other lanes through shared memory and the G
// partial readouts sum_n C h are combined through shared memory.
//
// Staging: each stage's x, dt, z rows and B, C rows are streamed global -> shared (double-buffered,
// one stage in flight while the previous one is computed). Where rows are 16-byte aligned, x, dt and
// z arrive as one TMA box each (cp.async.bulk.tensor, issued by one thread, completion counted on
// the buffer's mbarrier): the x box starts kPre steps early, so it also brings the conv halo in
// front of each row. Otherwise every thread copies its share element by element and the halo of 3
// steps is carried across stages in the prefix. B and C go through registers (transposed, fp32).
#include "ssm_common.cuh"
#include "ssm_internal.h"
#include "ssm_stage.cuh"
#include "ssm_tc.cuh"

namespace ssm {

// Shared-memory plan of one CTA (all offsets in bytes, 16-byte aligned).
template <int G, int NS, typename Tin, int NT> struct FwdSmem {
  static constexpr int CH = NT / G;          // channels per CTA
  static constexpr int NP = G * NS;          // padded state count
  static constexpr int XS = kPre + kT;       // x row length (elements)
  static constexpr int BS = NP + 4;          // Bs/Cs row stride (floats)
  static constexpr int US = kSub + 2;        // ud row stride (float2 entries: dl, u)
  static constexpr int YG = kSub + 4;        // y-partial stride between lanes of a channel
  static constexpr int YC = G * YG + 4;      // y-partial stride between channels
  static constexpr size_t x_off = 0;
  static constexpr size_t dt_off = x_off + sizeof(Tin) * 2 * CH * XS;
  static constexpr size_t z_off = dt_off + sizeof(Tin) * 2 * CH * kT;
  static constexpr size_t bs_off = z_off + sizeof(Tin) * 2 * CH * kT;
  static constexpr size_t cs_off = bs_off + sizeof(float) * 2 * kT * BS;
  static constexpr size_t ud_off = cs_off + sizeof(float) * 2 * kT * BS;
  static constexpr size_t yp_off = ud_off + sizeof(float2) * CH * US;
  static constexpr size_t bar_off = (yp_off + sizeof(float) * CH * YC + 7) / 8 * 8;  // 2 mbarriers
  static constexpr size_t bytes = bar_off + 16;
  static_assert(dt_off % 128 == 0 && z_off % 128 == 0 && (sizeof(Tin) * CH * XS) % 128 == 0 &&
                (sizeof(Tin) * CH * kT) % 128 == 0, "TMA destinations are 128-byte aligned");
};

// SUMMARY: pass 1 of the split-L forward -- the segment's recurrence from a zero state, keeping
// only its end state and its sum of Delta (no readout, no outputs).
template <int G, int NS, typename Tin, typename Tout, int NT, bool EULER, bool SUMMARY>
__global__ void __launch_bounds__(NT, 512 / NT)
ssm_fwd_kernel(const FwdParams p, const __grid_constant__ CUtensorMap tmx,
               const __grid_constant__ CUtensorMap tmdt, const __grid_constant__ CUtensorMap tmz) {
  using S = FwdSmem<G, NS, Tin, NT>;
  constexpr int CH = S::CH, NP = S::NP, EPL = kSub / G;
  constexpr bool PRECISE = sizeof(Tin) == 4;
  extern __shared__ __align__(16) unsigned char smem[];
  Tin *xs = reinterpret_cast<Tin *>(smem + S::x_off);
  Tin *dts = reinterpret_cast<Tin *>(smem + S::dt_off);
  Tin *zs = reinterpret_cast<Tin *>(smem + S::z_off);
  float *Bs = reinterpret_cast<float *>(smem + S::bs_off);
  float *Cs = reinterpret_cast<float *>(smem + S::cs_off);
  float2 *ud = reinterpret_cast<float2 *>(smem + S::ud_off);
  float *yp = reinterpret_cast<float *>(smem + S::yp_off);
  uint64_t *sbar = reinterpret_cast<uint64_t *>(smem + S::bar_off);

  const int64_t n_dtiles = (p.Dn + CH - 1) / CH;
  const int64_t per_seg = n_dtiles * p.Bt;
  const int64_t seg = blockIdx.x / per_seg;  // segment of the sequence (0 without split-L)
  const int64_t b = (blockIdx.x % per_seg) / n_dtiles;
  const int64_t d0 = (blockIdx.x % n_dtiles) * CH;
  const int rows_valid = (int)imin64(CH, p.Dn - d0);
  const int tid = threadIdx.x, c = tid / G, g = tid % G;
  const int64_t d = d0 + c;
  const bool live = d < p.Dn;
  const bool has_conv = p.conv_w != nullptr, has_z = p.z != nullptr;
  const bool vec = p.vec != 0;
  const int64_t L = p.L, N = p.N;
  // this CTA's steps: [ts, te). L stays the row length; steps from te on are padding here.
  const int64_t ts = seg * p.seg_len, te = imin64(L, ts + p.seg_len);

  // per-lane constants: Acoef = A (precise) or A log2(e) (fast), nIA = -1/A; padded states are
  // inert (A_bar = 1, no input, no readout)
  float Acoef[NS], nIA[NS], h[NS];
  const float *hinit = p.seg_h0 ? p.seg_h0 + (seg * p.Bt * p.Dn) * N : p.h0;  // carried state
#pragma unroll
  for (int j = 0; j < NS; j++) {
    const int n = g * NS + j;
    h[j] = (!SUMMARY && hinit && live && n < N) ? hinit[(b * p.Dn + d) * N + n] : 0.0f;
    if (live && n < N) {
      const float A = -expf(p.A_log[d * N + n]);
      Acoef[j] = PRECISE ? A : A * kLog2e;
      nIA[j] = -1.0f / A;
    } else {
      Acoef[j] = 0.0f;
      nIA[j] = 0.0f;
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

  const int64_t row0 = (b * p.Dn + d0) * L;  // first activation row of this CTA
  const Tin *gx = static_cast<const Tin *>(p.x) + row0;
  const Tin *gdt = static_cast<const Tin *>(p.dt) + row0;
  const Tin *gz = has_z ? static_cast<const Tin *>(p.z) + row0 : nullptr;
  const Tin *gB = static_cast<const Tin *>(p.B) + b * N * L;
  const Tin *gC = static_cast<const Tin *>(p.C) + b * N * L;
  const int n_rows = (int)imin64(NP, N);

  // conv-halo prefixes of both x buffers: the kPre inputs before the first step -- from x itself
  // for a later segment, else the carried history (newest-first), zero where there is none
  const Tin *hist = (has_conv && p.conv_hist && p.K > 1) ? static_cast<const Tin *>(p.conv_hist) : nullptr;
  const bool tma = p.tma && (static_cast<uint32_t>(__cvta_generic_to_shared(smem)) & 127u) == 0;
  if (tma && tid == 0) {
    mbar_init(sbar, 1);
    mbar_init(sbar + 1, 1);
  }
  for (int i = tid; !tma && i < 2 * CH * kPre; i += NT) {
    const int r = i / kPre, k = i % kPre, j = kPre - 1 - k;  // x_{ts-1-j}
    Tin v = zero_val<Tin>();
    if (r < rows_valid) {
      if (ts > 0)
        v = gx[(int64_t)r * L + ts - 1 - j];
      else if (hist && j < p.K - 1)
        v = hist[(b * p.Dn + d0 + r) * (p.K - 1) + j];
    }
    xs[r * S::XS + k] = v;
  }

  const int64_t n_stages = (te - ts + kT - 1) / kT;
  auto issue = [&](int64_t stage, int buf) {
    const int64_t t0 = ts + stage * kT;
    if (tma) {
      // x from kPre steps before the stage (its halo; a negative start reads zeros), dt, z: one box
      // of (steps, channels) each; rows past Dn and steps past L read zeros
      if (tid == 0) {
        const uint32_t bytes = (uint32_t)(sizeof(Tin) * CH * (S::XS + kT * (has_z ? 2 : 1)));
        mbar_expect_tx(sbar + buf, bytes);
        tma_load_3d(xs + buf * CH * S::XS, &tmx, (int)(t0 - kPre), (int)d0, (int)b, sbar + buf);
        tma_load_3d(dts + buf * CH * kT, &tmdt, (int)t0, (int)d0, (int)b, sbar + buf);
        if (has_z) tma_load_3d(zs + buf * CH * kT, &tmz, (int)t0, (int)d0, (int)b, sbar + buf);
      }
      return;
    }
    stage_rows<Tin, CH, kT, NT>(xs + buf * CH * S::XS + kPre, S::XS, gx, L, rows_valid, t0, L, vec);
    stage_rows<Tin, CH, kT, NT>(dts + buf * CH * kT, kT, gdt, L, rows_valid, t0, L, vec);
    if (has_z) stage_rows<Tin, CH, kT, NT>(zs + buf * CH * kT, kT, gz, L, rows_valid, t0, L, vec);
    cp_async_commit();
  };

  BCStager<Tin, NP, NT> bc;
  float sdl = 0.0f;  // sum of Delta over the segment (SUMMARY)
  if (tma) __syncthreads();  // the barriers are initialised before anyone polls them
  if (n_stages > 0) {
    issue(0, 0);
    bc.load(gB, gC, n_rows, ts, L, vec);
    bc.store(Bs, Cs, S::BS);
    if (n_stages > 1) bc.load(gB, gC, n_rows, ts + kT, L, vec);
    if (tma && ts == 0 && hist) {
      // the carried inputs before step 0 (newest-first) replace the zeros of the first box's halo,
      // once it has landed (the wait at the top of stage 0 then returns at once)
      mbar_wait(sbar, 0u);
      for (int i = tid; i < CH * (p.K - 1); i += NT) {
        const int r = i / (p.K - 1), j = i % (p.K - 1);
        if (r < rows_valid) xs[r * S::XS + kPre - 1 - j] = hist[(b * p.Dn + d0 + r) * (p.K - 1) + j];
      }
    }
  }
  for (int64_t st = 0; st < n_stages; st++) {
    const int buf = (int)(st & 1), nbuf = buf ^ 1;
    const int64_t t0 = ts + st * kT;
    if (tma) {
      mbar_wait(sbar + buf, (uint32_t)((st >> 1) & 1));  // bounded; the copy completes on its own
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // stage st landed and Bs/Cs[buf] written; stage st-1's buffers are free
    if (st + 1 < n_stages) {
      issue(st + 1, nbuf);
      bc.store(Bs + nbuf * kT * S::BS, Cs + nbuf * kT * S::BS, S::BS);
      if (st + 2 < n_stages) bc.load(gB, gC, n_rows, ts + (st + 2) * kT, L, vec);
    }
    const float *Bst = Bs + buf * kT * S::BS;
    const float *Cst = Cs + buf * kT * S::BS;
    const Tin *xrow = xs + (buf * CH + c) * S::XS + kPre;
    const Tin *dtrow = dts + (buf * CH + c) * kT;
    const Tin *zrow = zs + (buf * CH + c) * kT;

#pragma unroll
    for (int sb = 0; sb < kT / kSub; sb++) {
      // -- per-element work of this block: lane g owns EPL consecutive steps of its channel.
      //    Its inputs (x over [t-3, t+EPL), dt, z) are read as one small vector each.
      const int tb = sb * kSub + g * EPL;  // first owned step (stage-local)
      float xw[EPL + 4], dtw[EPL], zw[EPL];
      load_window<Tin, EPL + 4>(xw, xrow + tb - 4);
      load_window<Tin, EPL>(dtw, dtrow + tb);
      if (has_z) load_window<Tin, EPL>(zw, zrow + tb);
      float gate[EPL], uown[EPL], dlown[EPL];
      const bool tail = t0 + kT > te;  // this stage runs past the end of the sequence
#pragma unroll
      for (int j = 0; j < EPL; j++) {
        const int t = tb + j;
        float u;
        if (has_conv) {
          float acc = cbias;
#pragma unroll
          for (int k = 0; k < 4; k++) acc = fmaf(w4[k], xw[j + 4 - k], acc);
          u = acc * sigmoid<PRECISE>(acc);
        } else {
          u = xw[j + 4];
        }
        const float v = dtw[j] + dtb;
        float dl = p.delta_softplus ? softplus<PRECISE>(v) : v;
        float s = 1.0f;
        if (has_z) s = zw[j] * sigmoid<PRECISE>(zw[j]);
        if (tail && t0 + t >= te) {  // padded tail: an identity step
          u = 0.0f;
          dl = 0.0f;
        }
        if constexpr (EPL % 2 != 0) ud[c * S::US + g * EPL + j] = make_float2(dl, u);
        dlown[j] = dl;
        gate[j] = s;
        uown[j] = u;
        if (!tma && t >= kT - 3)  // carry the conv halo into the next stage's prefix (TMA brings it)
          xs[(nbuf * CH + c) * S::XS + kPre + t - kT] = xrow[t];
      }
      if constexpr (EPL % 2 == 0) {
#pragma unroll
        for (int j = 0; j < EPL; j += 2)
          *reinterpret_cast<float4 *>(ud + c * S::US + g * EPL + j) = make_float4(dlown[j], uown[j], dlown[j + 1], uown[j + 1]);
      }
      if (!SUMMARY && p.u_out && live)
        store_run<Tout, EPL>(static_cast<Tout *>(p.u_out) + row0 + (int64_t)c * L,
                             t0 + tb, te, uown, vec);
      __syncwarp();

      // -- the recurrence over the block's kSub steps, in groups of 4 steps: all shared-memory
      //    reads of a group are issued together, then the group's exps, then its updates.
      float *myp = yp + c * S::YC + g * S::YG;
#pragma unroll
      for (int tq = 0; tq < kSub; tq += 4) {
        float dlq[4], uq[4], Bq[4][NS], Cq[4][NS];
        {
          // the group's (Delta, u) pairs as two 16-byte reads (rows and groups are 16-byte aligned)
          const float4 d01 = *reinterpret_cast<const float4 *>(ud + c * S::US + tq);
          const float4 d23 = *reinterpret_cast<const float4 *>(ud + c * S::US + tq + 2);
          dlq[0] = d01.x; uq[0] = d01.y; dlq[1] = d01.z; uq[1] = d01.w;
          dlq[2] = d23.x; uq[2] = d23.y; dlq[3] = d23.z; uq[3] = d23.w;
        }
#pragma unroll
        for (int tt = 0; tt < 4; tt++) {
          const int t = sb * kSub + tq + tt;
          if (SUMMARY) sdl += dlq[tt];
          load_states<NS>(Bq[tt], Bst + t * S::BS + g * NS);
          load_states<NS>(Cq[tt], Cst + t * S::BS + g * NS);
        }
        float yq[4];
        if (PRECISE) {
#pragma unroll
          for (int tt = 0; tt < 4; tt++) {
            float y = 0.0f;
#pragma unroll
            for (int j = 0; j < NS; j++) {
              const float em1 = expm1f(dlq[tt] * Acoef[j]);    // A_bar - 1
              if (EULER) {
                h[j] = fmaf(em1, h[j], fmaf(dlq[tt] * Bq[tt][j], uq[tt], h[j]));  // A_bar h + Delta B u
              } else {
                const float nw = Bq[tt][j] * uq[tt] * nIA[j];   // -B u / A
                h[j] = fmaf(em1, h[j] - nw, h[j]);               // A_bar h + (A_bar - 1) B u / A
              }
              y = fmaf(Cq[tt][j], h[j], y);
            }
            yq[tt] = y;
          }
        } else {
          float a[4][NS];
#pragma unroll
          for (int tt = 0; tt < 4; tt++) {
            if (NS % 2 == 0) {
#pragma unroll
              for (int j = 0; j < NS; j += 2) {
                const float2 x = __fmul2_rn(make_float2(dlq[tt], dlq[tt]), make_float2(Acoef[j], Acoef[j + 1]));
                a[tt][j] = ex2_approx(x.x);
                a[tt][j + 1] = ex2_approx(x.y);
              }
            } else {
#pragma unroll
              for (int j = 0; j < NS; j++) a[tt][j] = ex2_approx(dlq[tt] * Acoef[j]);
            }
          }
#pragma unroll
          for (int tt = 0; tt < 4; tt++) {
            if (NS % 2 == 0) {
              float2 y2 = make_float2(0.0f, 0.0f);
              const float2 u2 = make_float2(uq[tt], uq[tt]);
#pragma unroll
              for (int j = 0; j < NS; j += 2) {
                float2 hh = make_float2(h[j], h[j + 1]);
                if (EULER) {
                  const float2 bdu = __fmul2_rn(__fmul2_rn(make_float2(Bq[tt][j], Bq[tt][j + 1]), u2),
                                                make_float2(dlq[tt], dlq[tt]));  // Delta B u
                  hh = __ffma2_rn(make_float2(a[tt][j], a[tt][j + 1]), hh, bdu);
                } else {
                  const float2 nw = __fmul2_rn(__fmul2_rn(make_float2(Bq[tt][j], Bq[tt][j + 1]), u2),
                                               make_float2(nIA[j], nIA[j + 1]));  // -B u / A
                  const float2 sum = __ffma2_rn(nw, make_float2(-1.0f, -1.0f), hh);  // h + w
                  hh = __ffma2_rn(make_float2(a[tt][j], a[tt][j + 1]), sum, nw);     // a (h+w) - w
                }
                h[j] = hh.x;
                h[j + 1] = hh.y;
                y2 = __ffma2_rn(make_float2(Cq[tt][j], Cq[tt][j + 1]), hh, y2);
              }
              yq[tt] = y2.x + y2.y;
            } else {
              float y = 0.0f;
#pragma unroll
              for (int j = 0; j < NS; j++) {
                if (EULER) {
                  h[j] = fmaf(a[tt][j], h[j], dlq[tt] * Bq[tt][j] * uq[tt]);
                } else {
                  const float nw = Bq[tt][j] * uq[tt] * nIA[j];
                  h[j] = fmaf(a[tt][j], h[j] - nw, nw);
                }
                y = fmaf(Cq[tt][j], h[j], y);
              }
              yq[tt] = y;
            }
          }
        }
        if (!SUMMARY) *reinterpret_cast<float4 *>(myp + tq) = make_float4(yq[0], yq[1], yq[2], yq[3]);
      }
      __syncwarp();
      if constexpr (!SUMMARY) {  // pass 1 keeps only the state

        // -- combine the G partial readouts of the owned steps, D skip, gate, store
        float o[EPL];
#pragma unroll
        for (int j = 0; j < EPL; j++) o[j] = 0.0f;
#pragma unroll
        for (int gg = 0; gg < G; gg++) {
          float part[EPL];
          load_floats<EPL>(part, yp + c * S::YC + gg * S::YG + g * EPL);
#pragma unroll
          for (int j = 0; j < EPL; j++) o[j] += part[j];
        }
#pragma unroll
        for (int j = 0; j < EPL; j++) o[j] = fmaf(Dd, uown[j], o[j]) * gate[j];
        if (live && p.out)
          store_run<Tout, EPL>(static_cast<Tout *>(p.out) + row0 + (int64_t)c * L, t0 + tb, te, o, vec);
        if (p.chunk_states && live && t0 + sb * kSub < te) {
          const int64_t kk = (t0 + sb * kSub) / kSub;
          float *dst = p.chunk_states + ((b * p.Dn + d) * p.n_ck + kk) * N;
          if (NS == 4 && N % 4 == 0 && g * NS < N && (reinterpret_cast<uintptr_t>(p.chunk_states) & 15) == 0) {
            // 16-byte aligned: an aligned base, rows of N floats with N a multiple of 4, lane offset g * 4
            *reinterpret_cast<float4 *>(dst + g * NS) = make_float4(h[0], h[NS > 1 ? 1 : 0], h[NS > 2 ? 2 : 0], h[NS > 3 ? 3 : 0]);
          } else {
#pragma unroll
            for (int j = 0; j < NS; j++)
              if (g * NS + j < N) dst[g * NS + j] = h[j];
          }
        }
      }
      __syncwarp();  // ud / yp are rewritten by the next block
    }
  }
  if (SUMMARY) {
    // the segment's end state from a zero start, and its sum of Delta
    if (live) {
      const int64_t sbd = (seg * p.Bt + b) * p.Dn + d;
#pragma unroll
      for (int j = 0; j < NS; j++)
        if (g * NS + j < N) p.seg_hend[sbd * N + g * NS + j] = h[j];
      if (g == 0) p.seg_sdl[sbd] = sdl;
    }
    return;
  }
  if (te != L) return;  // only the last segment hands the state on
  // carried state after step L-1 (padded tail steps are identity steps)
  if (live && p.h_last) {
#pragma unroll
    for (int j = 0; j < NS; j++)
      if (g * NS + j < N) p.h_last[(b * p.Dn + d) * N + g * NS + j] = h[j];
  }
  // the K-1 newest pre-conv inputs, newest-first; read everything before writing (the output
  // may alias the input history)
  if (live && has_conv && p.conv_hist_out && p.K > 1 && g == 0) {
    const Tin *xr = static_cast<const Tin *>(p.x) + (b * p.Dn + d) * L;
    const Tin *hr = hist ? hist + (b * p.Dn + d) * (p.K - 1) : nullptr;
    Tin v[3];
#pragma unroll
    for (int j = 0; j < 3; j++) {
      const int64_t t = L - 1 - j;
      v[j] = zero_val<Tin>();
      if (j < p.K - 1) v[j] = (t >= 0) ? xr[t] : (hr ? hr[j - L] : zero_val<Tin>());
    }
    Tin *o = static_cast<Tin *>(p.conv_hist_out) + (b * p.Dn + d) * (p.K - 1);
#pragma unroll
    for (int j = 0; j < 3; j++)
      if (j < p.K - 1) o[j] = v[j];
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

// Threads per forward CTA (a template parameter of the kernel; 128 measured best on the
// 4x4096x16x4096 shape, 64 was no faster).
constexpr int kFwdThreads = 128;

template <int G, int NS, typename Tin, typename Tout, bool SUMMARY>
static cudaError_t launch_fwd_t(const FwdParams &p, int n_seg_launch, cudaStream_t stream) {
  constexpr int NT = kFwdThreads;
  using S = FwdSmem<G, NS, Tin, NT>;
  auto kern = p.euler ? ssm_fwd_kernel<G, NS, Tin, Tout, NT, true, SUMMARY>
                      : ssm_fwd_kernel<G, NS, Tin, Tout, NT, false, SUMMARY>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::bytes);
  if (e != cudaSuccess) return e;
  const int64_t n_dtiles = (p.Dn + S::CH - 1) / S::CH;
  const int64_t grid = n_dtiles * p.Bt * n_seg_launch;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  // TMA boxes for x (the stage plus its kPre-step halo), dt and z where the rows are 16-byte aligned
  CUtensorMap mx, mdt, mz;
  memset(&mx, 0, sizeof(mx));
  memset(&mdt, 0, sizeof(mdt));
  memset(&mz, 0, sizeof(mz));
  FwdParams q = p;
  constexpr bool bf = sizeof(Tin) == 2;
  q.tma = p.vec && p.L <= 0x7fffffffLL && p.Dn <= 0x7fffffffLL &&
          encode_tma_3d(&mx, bf, p.x, (uint64_t)p.L, (uint64_t)p.Dn, (uint64_t)p.Bt, kPre + kT, S::CH) &&
          encode_tma_3d(&mdt, bf, p.dt, (uint64_t)p.L, (uint64_t)p.Dn, (uint64_t)p.Bt, kT, S::CH) &&
          (!p.z || encode_tma_3d(&mz, bf, p.z, (uint64_t)p.L, (uint64_t)p.Dn, (uint64_t)p.Bt, kT, S::CH));
  kern<<<(unsigned)grid, NT, S::bytes, stream>>>(q, mx, mdt, mz);
  return cudaGetLastError();
}

template <typename Tin, typename Tout, bool SUMMARY>
static cudaError_t dispatch_layout(const LaneLayout &lay, const FwdParams &p, int n_seg_launch, cudaStream_t s) {
#define SSM_FWD_CASE(G_, NS_) \
  if (lay.G == G_ && lay.NS == NS_) return launch_fwd_t<G_, NS_, Tin, Tout, SUMMARY>(p, n_seg_launch, s);
  SSM_FWD_CASE(4, 1) SSM_FWD_CASE(4, 2) SSM_FWD_CASE(4, 4)
  SSM_FWD_CASE(8, 1) SSM_FWD_CASE(8, 2) SSM_FWD_CASE(8, 4)
  SSM_FWD_CASE(16, 1) SSM_FWD_CASE(16, 2) SSM_FWD_CASE(16, 4)
#undef SSM_FWD_CASE
  return cudaErrorInvalidValue;
}

template <bool SUMMARY>
static cudaError_t dispatch_types(const LaneLayout &lay, const FwdParams &p, int in_bf16, int out_bf16,
                                  int n_seg_launch, cudaStream_t stream) {
  if (in_bf16) {
    if (out_bf16 || SUMMARY) return dispatch_layout<__nv_bfloat16, __nv_bfloat16, SUMMARY>(lay, p, n_seg_launch, stream);
    return dispatch_layout<__nv_bfloat16, float, SUMMARY>(lay, p, n_seg_launch, stream);
  }
  if (out_bf16 && !SUMMARY) return dispatch_layout<float, __nv_bfloat16, SUMMARY>(lay, p, n_seg_launch, stream);
  return dispatch_layout<float, float, SUMMARY>(lay, p, n_seg_launch, stream);
}

// Pass 2 of the split-L forward: the start state of every segment, walking the segments in order
// -- h_in[s+1] = exp(A * sum of Delta over s) h_in[s] + (end state of s from a zero start). The
// product of a segment's A_bar is exp(A * its sum of Delta), for the ZOH and the Euler rule alike.
__global__ void seg_carry_kernel(const FwdParams p) {
  const int64_t BDN = p.Bt * p.Dn * p.N;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // (b, d, n)
  if (i >= BDN) return;
  const int64_t n = i % p.N, bd = i / p.N, d = bd % p.Dn;
  const float A = -expf(p.A_log[d * p.N + n]);
  float h = p.h0 ? p.h0[i] : 0.0f;
  float *hin = const_cast<float *>(p.seg_h0);
  for (int s = 0; s < p.n_seg; s++) {
    hin[s * BDN + i] = h;
    if (s + 1 < p.n_seg) h = fmaf(expf(A * p.seg_sdl[s * p.Bt * p.Dn + bd]), h, p.seg_hend[s * BDN + i]);
  }
}

SegPlan plan_segments(int64_t Bt, int64_t Dn, int64_t N, int64_t L, int requested, int sm_count) {
  SegPlan plan = {1, L, 0};
  constexpr int64_t kSegAlign = 64;  // a multiple of the stage and of the state chunk
  int64_t want = requested;
  if (requested < 0) {
    // automatic, from measurements on B200 (4 CTAs per SM): the one-pass 4-lane grid has
    // base = Bt ceil(Dn / 32) CTAs. From three quarters of a wave up, no split. When even the widest lane
    // layout leaves fewer than two CTAs per SM, aim the segments at one wave (1x512x16x65536:
    // 37 segments, 7.1x); otherwise at just under three waves, since a last wave that is only
    // partly filled costs nearly a whole one (1x5120x16x65536: 11 segments, 2.97 waves, 4.57 ms;
    // 8 segments, 2.16 waves, 4.96 ms; 2x1536x16x2048: 16 segments of 128 steps 0.113 ms, 8 of 256
    // steps 0.120 ms, one pass 0.136 ms). Segments of at least 1024 resp. 128 steps.
    const int64_t slots = 4 * (int64_t)sm_count;
    const int64_t base = Bt * ((Dn + 31) / 32);
    if (4 * base >= 3 * slots) return plan;  // three quarters of a wave or more (1.4B shape: 86%)
    const int64_t widest = Bt * ((Dn + 7) / 8);
    if (widest < 2 * (int64_t)sm_count)
      want = imin64(slots / (base > 0 ? base : 1), L / 1024);
    else
      want = imin64(3 * slots / (base > 0 ? base : 1), L / 128);
  }
  if (want < 2 || L < 2 * kSegAlign) return plan;
  int64_t len = (L + want - 1) / want;
  len = (len + kSegAlign - 1) / kSegAlign * kSegAlign;
  const int64_t n = (L + len - 1) / len;
  if (n < 2) return plan;
  auto rnd = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t bdn = (size_t)(n * Bt * Dn * N);
  plan.n_seg = (int)n;
  plan.seg_len = len;
  plan.workspace_bytes = 2 * rnd(sizeof(float) * bdn) + rnd(sizeof(float) * (size_t)(n * Bt * Dn));
  return plan;
}

cudaError_t launch_fwd(const FwdParams &p, int in_bf16, int out_bf16, cudaStream_t stream) {
  if (p.n_seg <= 1 && p.chunked) return launch_fwd_tp(p, in_bf16, out_bf16, stream);
  if (p.n_seg <= 1) {
    FwdParams q = p;
    q.n_seg = 1;
    q.seg_len = p.L;
    q.seg_h0 = nullptr;
    return dispatch_types<false>(choose_layout(p.N, p.Bt * p.Dn), q, in_bf16, out_bf16, 1, stream);
  }
  // split-L: the layout is chosen as if the segments were more channels
  const LaneLayout lay = choose_layout(p.N, p.Bt * p.Dn * p.n_seg);
  FwdParams s1 = p;  // pass 1: every segment but the last, from a zero state
  s1.seg_h0 = nullptr;
  s1.out = nullptr;
  s1.u_out = nullptr;
  s1.chunk_states = nullptr;
  cudaError_t e = dispatch_types<true>(lay, s1, in_bf16, out_bf16, p.n_seg - 1, stream);
  if (e != cudaSuccess) return e;
  const int64_t bdn = p.Bt * p.Dn * p.N;
  seg_carry_kernel<<<(unsigned)((bdn + 255) / 256), 256, 0, stream>>>(p);  // pass 2
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return dispatch_types<false>(lay, p, in_bf16, out_bf16, p.n_seg, stream);  // pass 3
}

}  // namespace ssm
