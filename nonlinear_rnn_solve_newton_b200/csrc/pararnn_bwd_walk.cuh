// pararnn_bwd_walk.cuh -- the backward pass as a TMA tile walker, for the case
// where 32-channel tiles alone fill the GPU.
//
// Same recursion and arithmetic as pararnn_bwd_kernel (the reverse-time adjoint
// mu_t = J_t^T mu_{t+1} + J_t^T g_t, lambda_t = g_t + mu_{t+1}), organised like
// the forward tile walker:
//   * one CTA per tile walks the time chunks of its tile from the last to the
//     first, carrying mu across chunks in shared memory;
//   * each chunk's inputs -- the projected gates P_t, the forward trajectory one
//     step behind (the state each step's Jacobian is taken at) and the upstream
//     gradients -- arrive by TMA tensor copies into the other half of a double
//     buffer while the current chunk is processed;
//   * the stage is free as soon as the per-step factors are in registers, so the
//     copy two chunks ahead is issued right after the combine barrier: one
//     __syncthreads per chunk.
// Chunks are aligned to the end of the sequence (chunk j covers times
// [L - (j+1) T, L - j T)); the last one may start before t = 0, where the rows
// read are either zero fill or another batch row's data, and are never used.
#pragma once

#include "pararnn_bwd.cuh"
#include "pararnn_walk.cuh"

namespace pararnn {

struct BwdMaps {
  CUtensorMap P;    // 3-D {D, G, B*L}, box {32, G, T}
  CUtensorMap x0;   // trajectory h (GRU) / c (LSTM), 2-D {D, B*L}, box {32, T}
  CUtensorMap x1;   // trajectory h (LSTM)
  CUtensorMap g0;   // dl/dh (GRU) / dl/dc (LSTM); unused when the pointer is NULL
  CUtensorMap g1;   // dl/dh (LSTM); unused when the pointer is NULL
};

// Shared-memory image of one chunk: P [T][G][32], then NS trajectory planes and
// NS gradient planes, each fp32 [T][32].
template <int OP, typename PT, int TCH> struct BwdStage {
  static constexpr int G = BwdT<OP>::G;
  static constexpr int NS = BwdT<OP>::NS;
  static constexpr unsigned kP = TCH * G * 32 * sizeof(PT);
  static constexpr unsigned kPlane = TCH * 32 * 4;
  static constexpr unsigned kBytes = kP + 2 * NS * kPlane;
  static constexpr unsigned kPadded = (kBytes + 1023u) / 1024u * 1024u;
};

template <bool B> struct BoolC {
  static constexpr bool value = B;
};

// One step's map of the adjoint scan, mu -> J^T mu + J^T g, composed onto agg
// (which holds the later steps); keeps J^T and the factors for the apply phase.
template <int OP>
__device__ __forceinline__ void bwd_step_map(const float* pin, const float* wv,
                                             const Vec<BwdT<OP>::NS>& xp,
                                             const Vec<BwdT<OP>::NS>& g,
                                             Map<BwdT<OP>::NS>& JT, float* fac,
                                             Map<BwdT<OP>::NS>& agg) {
  constexpr int NS = BwdT<OP>::NS;
  BwdStep<OP>::eval(pin, wv, xp, JT, fac);
  Map<NS> m = JT;
  const Vec<NS> jg = apply(JT, g);
#pragma unroll
  for (int q = 0; q < NS; ++q) m.v[q] = jg.x[q];
  agg = compose(m, agg);
}

template <int OP, typename PT, int S, int NW, int MINB>
__global__ void __launch_bounds__(NW * 32, MINB)
    pararnn_bwd_walk_kernel(const __grid_constant__ BwdParams p,
                            const __grid_constant__ BwdMaps tm) {
  using T_ = BwdT<OP>;
  constexpr int NS = T_::NS;
  constexpr int G = T_::G;
  constexpr int F = T_::F;
  constexpr int CW = 32;
  constexpr int NT = NW * 32;
  constexpr int TCH = NW * S;  // one segment of S steps per warp
  using St = BwdStage<OP, PT, TCH>;

  extern __shared__ __align__(1024) unsigned char dsmem[];
  __shared__ unsigned long long s_bar[2];
  __shared__ Map<NS> s_wagg[2][NW][CW];  // per-warp aggregates, by chunk parity
  __shared__ Vec<NS> s_mu[2][CW];            // mu leaving the chunk (into earlier times)
  __shared__ float s_da[G][CW];
  __shared__ int s_item;

  const WaitCtx wctx{p.ctrl, p.status_dev, p.timeout_ns};
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int c = tid & 31;
  const bool has_g0 = p.g0 != nullptr;
  const bool has_g1 = NS == 2 && p.g1 != nullptr;
  const unsigned stage_bytes =
      St::kP + NS * St::kPlane + (has_g0 ? St::kPlane : 0u) + (has_g1 ? St::kPlane : 0u);

  // A gradient that is not given is a plane of zeros that no copy overwrites.
  for (int st = 0; st < 2; ++st) {
    float* sg = reinterpret_cast<float*>(dsmem + st * St::kPadded + St::kP) + NS * TCH * 32;
    if (!has_g0)
      for (int i = tid; i < TCH * 32; i += NT) sg[i] = 0.0f;
    if (NS == 2 && !has_g1)
      for (int i = tid; i < TCH * 32; i += NT) sg[TCH * 32 + i] = 0.0f;
  }
  if (tid == 0) {
    mbar_init(&s_bar[0], 1);
    mbar_init(&s_bar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  unsigned phase = 0u;    // parity of the next wait, per stage (bit s)
  unsigned pending = 0u;  // stages with a copy in flight (thread 0's view)
  bool aborted = false;

  // Thread 0: copies of chunk jj of the tile starting at channel d0, batch row0.
  auto issue = [&](int jj, int d0, int row0, int st) {
    unsigned char* dst = dsmem + st * St::kPadded;
    const int row = row0 + (int)(p.L - (long long)(jj + 1) * TCH);
    mbar_expect_tx(&s_bar[st], stage_bytes);
    tma_load_3d(dst, &tm.P, d0, 0, row, &s_bar[st]);
    unsigned char* q = dst + St::kP;
    tma_load_2d(q, &tm.x0, d0, row - 1, &s_bar[st]);
    if constexpr (NS == 2) tma_load_2d(q + St::kPlane, &tm.x1, d0, row - 1, &s_bar[st]);
    q += NS * St::kPlane;
    if (has_g0) tma_load_2d(q, &tm.g0, d0, row, &s_bar[st]);
    if constexpr (NS == 2) {
      if (has_g1) tma_load_2d(q + St::kPlane, &tm.g1, d0, row, &s_bar[st]);
    }
    pending |= 1u << st;
  };

  for (;;) {  // tiles
    if (tid == 0) {
      int u = (int)atomicAdd(&p.ticket[0], 1u);
      if (ld_volatile(&p.ctrl->abort) != 0u) u = p.ntiles;
      s_item = u;
    }
    if (tid < G * CW) (&s_da[0][0])[tid] = 0.0f;
    __syncthreads();
    const int tile = s_item;
    if (tile >= p.ntiles) break;

    const long long b = tile / p.ntd;
    const int td = tile - (int)b * p.ntd;
    const int d0 = td * CW;
    const long long d = d0 + c;
    const bool cvalid = d < p.D;
    const long long bd = b * p.D + d;
    const int row0 = (int)(b * p.L);

    if (tid == 0) {
      for (int jj = 0; jj < 2 && jj < p.nchunks; ++jj) issue(jj, d0, row0, jj);
    }

    float wv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) wv[g] = cvalid ? __ldg(p.w + (long long)g * p.D + d) : 0.0f;
    Vec<NS> xinit;  // the state before t = 0
    xinit.x[0] = (cvalid && p.x0a) ? __ldg(p.x0a + bd) : 0.0f;
    if constexpr (NS == 2) xinit.x[1] = (cvalid && p.x0b) ? __ldg(p.x0b + bd) : 0.0f;
    float da[G];
#pragma unroll
    for (int g = 0; g < G; ++g) da[g] = 0.0f;

    for (int j = 0; j < p.nchunks; ++j) {
      const int st = j & 1;
      const unsigned char* stage = dsmem + st * St::kPadded;
      const bool ok = stage_wait(&s_bar[st], (phase >> st) & 1u, wctx);
      if (ok) {  // a copy that did not land stays pending for the final wait
        phase ^= 1u << st;
        if (tid == 0) pending &= ~(1u << st);
      }
      if (!__syncthreads_and(ok ? 1 : 0)) {
        if (tid == 0) raise_error(wctx, 4u);
        aborted = true;
        break;
      }
      const long long tlo = p.L - (long long)(j + 1) * TCH;
      // Two instantiations of the chunk: FULL when every step has t >= 1 (no
      // bounds, no initial state: all chunks but the earliest), else checked.
      auto chunk = [&](auto full_c) {
        constexpr bool FULL = decltype(full_c)::value;
        const int rtop = TCH - 1 - warp * S;  // row of this warp's first (latest) step
        const PT* sP = reinterpret_cast<const PT*>(stage) + rtop * G * 32 + c;
        const float* sx = reinterpret_cast<const float*>(stage + St::kP) + rtop * 32 + c;
        const float* sg = sx + NS * TCH * 32;
        const int tl = FULL ? 1 : (int)(tlo + rtop);  // time of step s = 0 (checked form)

        // ---- per step (scan order s runs backwards in time) ----------------
        Map<NS> JT[S];
        Vec<NS> gv[S];
        float fac[S][F];
        Map<NS> agg = map_identity<NS>();
#pragma unroll
        for (int s = 0; s < S; ++s) {
          if (FULL || (cvalid && tl - s >= 0)) {
            float pin[G];
#pragma unroll
            for (int g = 0; g < G; ++g) pin[g] = to_f(sP[(g - s * G) * 32]);
            Vec<NS> xp;
#pragma unroll
            for (int q = 0; q < NS; ++q) {
              xp.x[q] = sx[(q * TCH - s) * 32];
              gv[s].x[q] = sg[(q * TCH - s) * 32];
            }
            if (!FULL && tl - s == 0) xp = xinit;
            bwd_step_map<OP>(pin, wv, xp, gv[s], JT[s], fac[s], agg);
          } else {
            JT[s] = map_identity<NS>();
#pragma unroll
            for (int q = 0; q < NS; ++q) gv[s].x[q] = 0.0f;
#pragma unroll
            for (int f = 0; f < F; ++f) fac[s][f] = 0.0f;
          }
        }

        // ---- combine: one barrier; each warp composes the warps before it ----
        s_wagg[st][warp][c] = agg;
        __syncthreads();
        // the stage has been read by every warp: refill it two chunks ahead
        if (tid == 0 && j + 2 < p.nchunks) issue(j + 2, d0, row0, st);
        Map<NS> pre = map_identity<NS>();
#pragma unroll 4
        for (int w2 = 0; w2 < warp; ++w2) pre = compose(s_wagg[st][w2][c], pre);
        Vec<NS> carry;
        if (j == 0) {
#pragma unroll
          for (int q = 0; q < NS; ++q) carry.x[q] = 0.0f;  // mu_{L+1} = 0
        } else {
          carry = s_mu[(j - 1) & 1][c];
        }
        Vec<NS> mu = apply(pre, carry);
        if (warp == NW - 1) s_mu[st][c] = apply(agg, mu);

        // ---- apply: lambda_t = g_t + mu_{t+1}; dP_t, da; mu_t = J_t^T lambda_t --
        const int gd = G * (int)p.D;  // floats between consecutive steps of dP
        float* dst = p.dP + (b * p.L + tlo + rtop) * (long long)gd + d;  // step s = 0
#pragma unroll
        for (int s = 0; s < S; ++s) {
          if (FULL || (cvalid && tl - s >= 0)) {
            Vec<NS> lam;
#pragma unroll
            for (int q = 0; q < NS; ++q) lam.x[q] = gv[s].x[q] + mu.x[q];
            float dp[G];
            BwdStep<OP>::outputs(fac[s], lam, dp, da);
            if (FULL ? cvalid : true) {
#pragma unroll
              for (int g = 0; g < G; ++g) __stcs(dst - s * gd + g * (int)p.D, dp[g]);
            }
            Map<NS> jt = JT[s];
#pragma unroll
            for (int q = 0; q < NS; ++q) jt.v[q] = 0.0f;
            mu = apply(jt, lam);
            if (!FULL && tl - s == 0) {
              if (p.d0a) p.d0a[bd] = mu.x[0];
              if constexpr (NS == 2) {
                if (p.d0b) p.d0b[bd] = mu.x[1];
              }
            }
          }
        }
      };
      if (tlo >= 1)
        chunk(BoolC<true>{});
      else
        chunk(BoolC<false>{});
    }
    if (aborted) break;

    // ---- da: sum the warps of each channel, one atomic per (gate, channel) ----
    if (cvalid) {
#pragma unroll
      for (int g = 0; g < G; ++g) atomicAdd(&s_da[g][c], da[g]);
    }
    __syncthreads();
    if (tid < G * CW) {
      const int g = tid / CW, cc = tid % CW;
      const long long dd = (long long)d0 + cc;
      if (dd < p.D) atomicAdd(p.da + (long long)g * p.D + dd, s_da[g][cc]);
    }
    __syncthreads();
  }

  // never leave with copies in flight into this CTA's shared memory
  if (tid == 0 && pending) drain_stages(s_bar, pending, phase, wctx);
}

}  // namespace pararnn
