// pararnn_bwd.cuh -- gradients through the solved trajectory (backward pass).
//
// The forward solve returns h with h_t = f(h_{t-1}, P_t).  For a loss with
// upstream gradient g_t = dl/dh_t the total gradient lambda_t obeys the adjoint
// recursion lambda_t = g_t + J_{t+1}^T lambda_{t+1} (J_t = df/dh at step t), a
// block bi-diagonal system with the transposed Jacobians running backwards in
// time -- the transposed counterpart of the Newton step's solve (ParaRNN,
// TL;DR; DEER summary: forward plus gradients).  Written with
// mu_t = J_t^T lambda_t, it is the reverse-time affine recurrence
//     mu_t = J_t^T mu_{t+1} + J_t^T g_t,   mu_{L+1} = 0,   lambda_t = g_t + mu_{t+1},
// whose map at step t uses step t's own data only.  Then
//     dl/dP_t = lambda_t^T df/dP_t,   dl/da = sum_t lambda_t^T df/da,   dl/dh0 = mu_1.
//
// One kernel pass: the scan runs over positions tau = 0..L-1 with time
// t = L-1-tau, through the same machinery as the forward kernel (thread-serial
// composition, warp and shared-memory combine, chunks chained inside one CTA
// when tiles fill the GPU, else by windowed look-back).  The apply phase emits
// dP_t and accumulates da per thread; da is reduced per CTA in shared memory and
// added to global memory with one atomic per (gate, channel) and work item.
#pragma once

#include "pararnn_kernel.cuh"

namespace pararnn {

enum BwdKind : int { kGruBwd = 4, kLstmBwd = 5 };

template <int OP> struct BwdT;
template <> struct BwdT<kGruBwd> {
  static constexpr int NS = 1, G = 3, F = 5;  // F: per-step factors kept for the apply phase
};
template <> struct BwdT<kLstmBwd> {
  static constexpr int NS = 2, G = 4, F = 6;
};

struct BwdParams {
  const void* P;       // [B, L, G, D] fp32 or bf16
  const float* w;      // [G, D]
  const float* x0a;    // h0 (GRU) / c0 (LSTM), or NULL
  const float* x0b;    // h0 (LSTM), or NULL
  const float* tr0;    // forward trajectory h (GRU) / c (LSTM) [B, L, D]
  const float* tr1;    // forward trajectory h (LSTM)
  const float* g0;     // dl/dh (GRU) / dl/dc (LSTM) [B, L, D], may be NULL for LSTM
  const float* g1;     // dl/dh (LSTM), may be NULL
  float* dP;           // [B, L, G, D] fp32
  float* da;           // [G, D] fp32, zeroed by the host, accumulated atomically
  float* d0a;          // dl/dh0 (GRU) / dl/dc0 (LSTM) [B, D], or NULL
  float* d0b;          // dl/dh0 (LSTM), or NULL
  long long B, L, D;
  int ntd, ntiles, nchunks, nunits;
  Ctrl* ctrl;
  unsigned* ticket;
  unsigned long long* rec;
  int* status_dev;
  long long timeout_ns;
  long long stall_unit;
};

// Step of the backward pass at time t: the transposed Jacobian, the upstream
// gradient and the factors that turn lambda_t into dP_t and da.
template <int OP> struct BwdStep;

// GRU.  u_z = Pz + az h, z = sig(u_z); u_r = Pr + ar h, r = sig(u_r);
// u_c = Pc + ac r h, c = tanh(u_c); f = (1-z) h + z c.
//   df/dPz = (c - h) z (1-z),  df/dPc = z (1-c^2),  df/dPr = df/dPc ac h r (1-r),
//   df/da_z = df/dPz h,  df/da_r = df/dPr h,  df/da_c = df/dPc r h.
template <> struct BwdStep<kGruBwd> {
  __device__ static void eval(const float* p, const float* w, const Vec<1>& xp, Map<1>& JT,
                              float* fac) {
    const float h = xp.x[0];
    const float z = sigm(fmaf(w[0], h, p[0]));
    const float r = sigm(fmaf(w[1], h, p[1]));
    const float rh = r * h;
    const float c = tanh_f(fmaf(w[2], rh, p[2]));
    const float cmh = c - h;
    const float omz = 1.0f - z;
    const float zz = z * omz;
    const float dfdz = cmh * zz;
    const float dfdu = z * fmaf(-c, c, 1.0f);
    const float rr = r * (1.0f - r);
    const float dfdr = dfdu * w[2] * h * rr;
    // J = (1-z) + (c-h) z(1-z) az + z (1-c^2) ac (r + h r(1-r) ar)
    const float J = fmaf(dfdz, w[0], omz) + dfdu * w[2] * fmaf(h * rr, w[1], r);
    JT.m[0][0] = J;
    JT.v[0] = 0.0f;
    fac[0] = dfdz;
    fac[1] = dfdr;
    fac[2] = dfdu;
    fac[3] = h;
    fac[4] = rh;
  }
  // lambda -> dP (3 values), da += ...
  __device__ static void outputs(const float* fac, const Vec<1>& lam, float* dp, float* da) {
    const float l = lam.x[0];
    dp[0] = l * fac[0];
    dp[1] = l * fac[1];
    dp[2] = l * fac[2];
    da[0] = fmaf(dp[0], fac[3], da[0]);
    da[1] = fmaf(dp[1], fac[3], da[1]);
    da[2] = fmaf(dp[2], fac[4], da[2]);
  }
};

// LSTM, state (c, h).  With u_x = P_x + a_x h:
//   dc'/du_i = g i(1-i), dc'/du_f = c f(1-f), dc'/du_g = i(1-g^2), dc'/du_o = 0,
//   dh'/du_x = o(1 - tanh(c')^2) dc'/du_x (x = i, f, g), dh'/du_o = tanh(c') o(1-o),
//   dl/dP_x = lambda_c dc'/du_x + lambda_h dh'/du_x,  dl/da_x += dl/dP_x h.
template <> struct BwdStep<kLstmBwd> {
  __device__ static void eval(const float* p, const float* w, const Vec<2>& xp, Map<2>& JT,
                              float* fac) {
    const float c = xp.x[0], h = xp.x[1];
    const float ig = sigm(fmaf(w[0], h, p[0]));
    const float fg = sigm(fmaf(w[1], h, p[1]));
    const float gg = tanh_f(fmaf(w[2], h, p[2]));
    const float og = sigm(fmaf(w[3], h, p[3]));
    const float cn = fmaf(fg, c, ig * gg);
    const float tc = tanh_f(cn);
    const float dcdi = gg * ig * (1.0f - ig);   // dc'/du_i
    const float dcdf = c * fg * (1.0f - fg);    // dc'/du_f
    const float dcdg = ig * fmaf(-gg, gg, 1.0f);  // dc'/du_g
    const float dhdo = tc * og * (1.0f - og);   // dh'/du_o
    const float odtc = og * fmaf(-tc, tc, 1.0f);  // o (1 - tanh(c')^2)
    // J = [[dc'/dc, dc'/dh], [dh'/dc, dh'/dh]] with dc'/dh = sum_x dc'/du_x a_x
    const float dcn_dh = fmaf(dcdi, w[0], fmaf(dcdf, w[1], dcdg * w[2]));
    JT.m[0][0] = fg;                              // (dc'/dc)
    JT.m[1][0] = dcn_dh;                          // (dc'/dh)
    JT.m[0][1] = odtc * fg;                       // (dh'/dc)
    JT.m[1][1] = fmaf(dhdo, w[3], odtc * dcn_dh);  // (dh'/dh)
    JT.v[0] = 0.0f;
    JT.v[1] = 0.0f;
    fac[0] = dcdi;
    fac[1] = dcdf;
    fac[2] = dcdg;
    fac[3] = dhdo;
    fac[4] = odtc;
    fac[5] = h;
  }
  __device__ static void outputs(const float* fac, const Vec<2>& lam, float* dp, float* da) {
    const float kappa = fmaf(lam.x[1], fac[4], lam.x[0]);
    dp[0] = kappa * fac[0];
    dp[1] = kappa * fac[1];
    dp[2] = kappa * fac[2];
    dp[3] = lam.x[1] * fac[3];
#pragma unroll
    for (int g = 0; g < 4; ++g) da[g] = fmaf(dp[g], fac[5], da[g]);
  }
};

template <int OP, typename PT, int CW, int S, int MINB, bool WALK>
__global__ void __launch_bounds__(kThreads, MINB) pararnn_bwd_kernel(const BwdParams p) {
  using T_ = BwdT<OP>;
  constexpr int NS = T_::NS;
  constexpr int G = T_::G;
  constexpr int F = T_::F;
  constexpr int NSEG = kThreads / CW;
  constexpr int TCH = NSEG * S;

  __shared__ Map<NS> s_wagg[kWarps][CW];
  __shared__ Vec<NS> s_carry[CW];
  __shared__ Vec<NS> s_inc[2][CW];
  __shared__ float s_da[G][CW];
  __shared__ int s_unit;
  __shared__ int s_abort;

  const WaitCtx wctx{p.ctrl, p.status_dev, p.timeout_ns};
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int c = tid % CW;
  const int seg = tid / CW;
  const int nwork = WALK ? p.ntiles : p.nunits;
  const unsigned tag = 1u;

  if (tid == 0) s_abort = 0;
  __syncthreads();

  for (;;) {
    if (tid == 0) {
      int u = (int)atomicAdd(&p.ticket[0], 1u);
      if (ld_volatile(&p.ctrl->abort) != 0u) u = nwork;
      s_unit = u;
    }
    if (tid < G * CW) (&s_da[0][0])[tid] = 0.0f;
    __syncthreads();
    const int item = s_unit;
    if (item >= nwork) break;

    const int jbeg = WALK ? 0 : item / p.ntiles;
    const int jend = WALK ? p.nchunks : jbeg + 1;
    const int tile = WALK ? item : item - jbeg * p.ntiles;
    const long long b = tile / p.ntd;
    const int td = tile - (int)b * p.ntd;
    const long long d = (long long)td * CW + c;
    const bool cvalid = d < p.D;
    const long long bd = b * p.D + d;

    float wv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) wv[g] = cvalid ? __ldg(p.w + (long long)g * p.D + d) : 0.0f;
    float da[G];
#pragma unroll
    for (int g = 0; g < G; ++g) da[g] = 0.0f;

    for (int j = jbeg; j < jend; ++j) {
      const int u = j * p.ntiles + tile;
      const long long tau0 = (long long)j * TCH + (long long)seg * S;
      const bool publish = (long long)u != p.stall_unit;

      // ---- per step: transposed Jacobian, upstream gradient, factors ------
      Map<NS> JT[S];
      Vec<NS> gv[S];
      float fac[S][F];
      Map<NS> agg = map_identity<NS>();
#pragma unroll
      for (int s = 0; s < S; ++s) {
        const long long t = p.L - 1 - (tau0 + s);
        if (cvalid && t >= 0) {
          const long long i = (b * p.L + t) * p.D + d;
          float pin[G];
          const PT* P = reinterpret_cast<const PT*>(p.P) + (b * p.L + t) * G * p.D + d;
#pragma unroll
          for (int g = 0; g < G; ++g) pin[g] = to_f(__ldg(P + g * p.D));
          Vec<NS> xp;
          if (t == 0) {
            xp.x[0] = p.x0a ? __ldg(p.x0a + bd) : 0.0f;
            if constexpr (NS == 2) xp.x[1] = p.x0b ? __ldg(p.x0b + bd) : 0.0f;
          } else {
            xp.x[0] = __ldg(p.tr0 + i - p.D);
            if constexpr (NS == 2) xp.x[1] = __ldg(p.tr1 + i - p.D);
          }
          gv[s].x[0] = p.g0 ? __ldg(p.g0 + i) : 0.0f;
          if constexpr (NS == 2) gv[s].x[1] = p.g1 ? __ldg(p.g1 + i) : 0.0f;
          BwdStep<OP>::eval(pin, wv, xp, JT[s], fac[s]);
          // map of this step: mu -> J^T mu + J^T g
          Map<NS> m = JT[s];
          const Vec<NS> jg = apply(JT[s], gv[s]);
#pragma unroll
          for (int q = 0; q < NS; ++q) m.v[q] = jg.x[q];
          agg = compose(m, agg);
        } else {
          JT[s] = map_identity<NS>();
#pragma unroll
          for (int q = 0; q < NS; ++q) gv[s].x[q] = 0.0f;
#pragma unroll
          for (int f = 0; f < F; ++f) fac[s][f] = 0.0f;
        }
      }

      // ---- combine segments: warp (segments stride CW), then the 8 warps ----
      Map<NS> incl = agg;
      Map<NS> wexcl = map_identity<NS>();
      if constexpr (CW < 32) {
#pragma unroll
        for (int off = CW; off < 32; off <<= 1) {
          Map<NS> o = shfl_up_map(incl, off);
          if (lane >= off) incl = compose(incl, o);
        }
        Map<NS> e = shfl_up_map(incl, CW);
        if (lane >= CW) wexcl = e;
      }
      if (lane >= 32 - CW) s_wagg[warp][c] = incl;
      __syncthreads();

      if (warp == 0) {
        Map<NS> cta = map_identity<NS>();
        if (lane < CW) {
#pragma unroll
          for (int w2 = 0; w2 < kWarps; ++w2) cta = compose(s_wagg[w2][c], cta);
        }
        Vec<NS> carry;
#pragma unroll
        for (int q = 0; q < NS; ++q) carry.x[q] = 0.0f;  // mu_{L+1} = 0
        bool failed = false;
        if (j > 0) {
          if constexpr (WALK) {
            carry = s_inc[(j - 1) & 1][c];
          } else {
            constexpr int RW = Rec<NS>::kWords;
            if (publish && lane < CW)
              publish_agg<NS>(p.rec + ((size_t)u * CW + c) * RW, tag, cta);
            failed = !window_lookback<NS, CW>(p.rec, (size_t)CW * RW, u - p.ntiles, p.ntiles,
                                              tag, carry, wctx);
          }
        }
        const Vec<NS> xe = apply(cta, carry);
        if constexpr (WALK) {
          if (lane < CW) s_inc[j & 1][c] = xe;
        } else {
          constexpr int RW = Rec<NS>::kWords;
          if (publish && !failed && lane < CW)
            publish_inc<NS>(p.rec + ((size_t)u * CW + c) * RW, tag, xe);
        }
        if (lane < CW) s_carry[c] = carry;
        if (lane == 0 && failed) s_abort = 1;
      }
      Map<NS> wpre = map_identity<NS>();
      for (int w2 = 0; w2 < warp; ++w2) wpre = compose(s_wagg[w2][c], wpre);
      __syncthreads();

      // ---- apply: lambda_t = g_t + mu_{t+1}; outputs; mu_t = J_t^T lambda_t --
      Vec<NS> mu = apply(wexcl, apply(wpre, s_carry[c]));
#pragma unroll
      for (int s = 0; s < S; ++s) {
        const long long t = p.L - 1 - (tau0 + s);
        if (cvalid && t >= 0) {
          Vec<NS> lam;
#pragma unroll
          for (int q = 0; q < NS; ++q) lam.x[q] = gv[s].x[q] + mu.x[q];
          float dp[G];
          BwdStep<OP>::outputs(fac[s], lam, dp, da);
          float* dst = p.dP + (b * p.L + t) * G * p.D + d;
#pragma unroll
          for (int g = 0; g < G; ++g) __stcs(dst + g * p.D, dp[g]);
          Map<NS> jt = JT[s];
#pragma unroll
          for (int q = 0; q < NS; ++q) jt.v[q] = 0.0f;
          mu = apply(jt, lam);
          if (t == 0) {
            if (p.d0a) p.d0a[bd] = mu.x[0];
            if constexpr (NS == 2) {
              if (p.d0b) p.d0b[bd] = mu.x[1];
            }
          }
        }
      }
      if (s_abort) break;
      __syncthreads();  // s_wagg / s_carry are rewritten by the next chunk
    }

    // ---- da: sum the segments of each channel, one atomic per (gate, channel)
    if (!s_abort) {
      if (cvalid) {
#pragma unroll
        for (int g = 0; g < G; ++g) atomicAdd(&s_da[g][c], da[g]);
      }
      __syncthreads();
      if (tid < G * CW) {
        const int g = tid / CW, cc = tid % CW;
        const long long dd = (long long)td * CW + cc;
        if (dd < p.D) atomicAdd(p.da + (long long)g * p.D + dd, s_da[g][cc]);
      }
    }
    if (s_abort) break;
    __syncthreads();
  }
}

}  // namespace pararnn
