// pararnn_walk2.cuh -- the ParaGRU tile walker with two channels per thread in
// packed fp32x2 arithmetic.
//
// Same method, schedule and arithmetic as the GRU case of pararnn_walk_kernel
// (pararnn_walk.cuh): one CTA walks the time chunks of a tile of CW channels,
// each chunk staged by one tensor copy, all iterations of a sweep on chip, the
// carry between chunks in shared memory.  What differs is the thread mapping:
// a thread owns a PAIR of adjacent channels (2p, 2p + 1) and S steps, and
// evaluates the cell, the Jacobian, the residual and the affine maps of both
// channels with the packed f32x2 instructions of sm_100 (add/sub/mul/fma
// .rn.f32x2: two fp32 operations per issued instruction, each rounded as the
// scalar one).  The special-function operations (ex2, rcp) stay one per
// channel.  On the GRU cell this halves the issued arithmetic per channel, so
// the solve, bound by issue slots and the special-function pipe together,
// becomes bound by the latter alone.
//
// Lane = pair + (CW / 2) x (segment within the warp).  For bf16 gates a pair's
// two values are one 32-bit shared-memory word; with an odd S the warp's
// segments read different banks.
#pragma once

#include "pararnn_walk.cuh"

namespace pararnn {

// Two fp32 values in one 64-bit register pair.
struct F2 {
  unsigned long long v;
};
__device__ __forceinline__ F2 f2(float a, float b) {
  F2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float f2lo(F2 x) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(x.v));
  return a;
}
__device__ __forceinline__ float f2hi(F2 x) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(x.v));
  return b;
}
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c) {
  F2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.v) : "l"(a.v), "l"(b.v), "l"(c.v));
  return d;
}
__device__ __forceinline__ F2 mul2(F2 a, F2 b) {
  F2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
  return d;
}
__device__ __forceinline__ F2 add2(F2 a, F2 b) {
  F2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
  return d;
}
__device__ __forceinline__ F2 sub2(F2 a, F2 b) {
  F2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
  return d;
}
__device__ __forceinline__ F2 splat2(float a) { return f2(a, a); }
__device__ __forceinline__ F2 shfl_up2(F2 x, int d) {
  return f2(__shfl_up_sync(0xffffffffu, f2lo(x), d), __shfl_up_sync(0xffffffffu, f2hi(x), d));
}

// Affine map x -> m x + v of a channel pair.
struct Map2 {
  F2 m, v;
};
__device__ __forceinline__ Map2 map2_identity() { return Map2{splat2(1.0f), splat2(0.0f)}; }
// later o earlier
__device__ __forceinline__ Map2 compose2(const Map2& later, const Map2& earlier) {
  return Map2{mul2(later.m, earlier.m), fma2(later.m, earlier.v, later.v)};
}
__device__ __forceinline__ F2 apply2(const Map2& M, F2 x) { return fma2(M.m, x, M.v); }

// sigmoid and tanh of both halves from the identities of gru_cell: one ex2 and
// one rcp each (scale folded into the packed multiply).
__device__ __forceinline__ F2 sigm2(F2 u) {
  const F2 a = mul2(u, splat2(-kLog2e));
  const F2 d = add2(f2(ex2_approx(f2lo(a)), ex2_approx(f2hi(a))), splat2(1.0f));
  return f2(rcp_approx(f2lo(d)), rcp_approx(f2hi(d)));
}
__device__ __forceinline__ F2 tanh2(F2 u) {
  const F2 a = mul2(u, splat2(2.0f * kLog2e));
  const F2 d = add2(f2(ex2_approx(f2lo(a)), ex2_approx(f2hi(a))), splat2(1.0f));
  return fma2(splat2(-2.0f), f2(rcp_approx(f2lo(d)), rcp_approx(f2hi(d))), splat2(1.0f));
}

// One Newton linearisation of a pair at step t: the ParaGRU cell at h = h^k_{t-1},
// its derivative J, the residual against x = h^k_t (max into rmax) and the map
// h^{k+1}_t = J h^{k+1}_{t-1} + (f - J h^k_{t-1}).
__device__ __forceinline__ Map2 gru_newton2(F2 pz, F2 pr, F2 pc, F2 wz, F2 wr, F2 wc, F2 h, F2 x,
                                            float& rmax) {
  const F2 one = splat2(1.0f);
  const F2 z = sigm2(fma2(wz, h, pz));
  const F2 r = sigm2(fma2(wr, h, pr));
  const F2 c = tanh2(fma2(wc, mul2(r, h), pc));
  const F2 cmh = sub2(c, h);
  const F2 f = fma2(z, cmh, h);
  const F2 omz = sub2(one, z);
  const F2 dz = mul2(mul2(z, omz), wz);
  const F2 dr = mul2(mul2(r, sub2(one, r)), wr);
  const F2 du = mul2(wc, fma2(h, dr, r));
  const F2 dc = mul2(fma2(sub2(splat2(0.0f), c), c, one), du);
  const F2 J = fma2(z, dc, fma2(cmh, dz, omz));
  const F2 res = sub2(f, x);
  rmax = max_abs_nan(max_abs_nan(rmax, f2lo(res)), f2hi(res));
  return Map2{J, sub2(f, mul2(J, h))};
}

template <typename PT> struct PairIO;
template <> struct PairIO<float> {
  // gates z, r, c of the pair at staged step tl: [T][3][CW] fp32
  template <int CW>
  __device__ static void read(const unsigned char* s, int tl, int p, F2& z, F2& r, F2& c) {
    const float2* q = reinterpret_cast<const float2*>(s) + tl * 3 * (CW / 2) + p;
    const float2 a = q[0], b = q[CW / 2], e = q[CW];
    z = f2(a.x, a.y);
    r = f2(b.x, b.y);
    c = f2(e.x, e.y);
  }
};
template <> struct PairIO<__nv_bfloat16> {
  // [T][3][CW] bf16: a pair is one 32-bit word; bf16 -> fp32 puts the 16 bits on top
  template <int CW>
  __device__ static void read(const unsigned char* s, int tl, int p, F2& z, F2& r, F2& c) {
    const unsigned* q = reinterpret_cast<const unsigned*>(s) + tl * 3 * (CW / 2) + p;
    const unsigned a = q[0], b = q[CW / 2], e = q[CW];
    z = f2(__uint_as_float(a << 16), __uint_as_float(a & 0xffff0000u));
    r = f2(__uint_as_float(b << 16), __uint_as_float(b & 0xffff0000u));
    c = f2(__uint_as_float(e << 16), __uint_as_float(e & 0xffff0000u));
  }
};

__device__ __forceinline__ F2 ld_pair_cg(const float* p) {
  const float2 v = __ldcg(reinterpret_cast<const float2*>(p));
  return f2(v.x, v.y);
}
__device__ __forceinline__ void st_pair(float* p, F2 x) {
  *reinterpret_cast<float2*>(p) = make_float2(f2lo(x), f2hi(x));
}

// Requirements (host): D even, h and h0 8-byte aligned, TMA rules for P.
template <typename PT, int S, int NW, int MINB, int CW = 32>
__global__ void __launch_bounds__(NW * 32, MINB)
    pararnn_walk_gru2_kernel(const __grid_constant__ KParams p, const __grid_constant__ TmaMaps tm) {
  constexpr int CP = CW / 2;          // pairs per tile
  constexpr int SPL = 32 / CP;        // segments per warp
  constexpr int NSEG = NW * SPL;
  constexpr int TCH = NSEG * S;       // steps per chunk
  using St = Stage<kGru, PT, TCH, CW>;
  constexpr unsigned kStageBytes = (St::kBytes + 1023u) / 1024u * 1024u;
  constexpr int WM = kMaxWalkIters;
  static_assert(CW % 2 == 0 && 32 % CP == 0, "pairs per tile divide a warp");

  extern __shared__ __align__(1024) unsigned char dsmem[];
  __shared__ unsigned long long s_bar[2];
  __shared__ Map2 s_wagg[2][NW][CP];
  __shared__ F2 s_inc[2][WM][CP];
  __shared__ F2 s_pend[2][CP];
  __shared__ unsigned s_racc[WM];
  __shared__ int s_item;
  __shared__ int s_flag;

  const WaitCtx wctx{p.ctrl, p.status_dev, p.timeout_ns};
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int pi = lane % CP;       // pair within the tile
  const int sub = lane / CP;      // segment within the warp
  const int seg = warp * SPL + sub;
  const bool last_in_warp = sub == SPL - 1;

  if (tid == 0) {
    mbar_init(&s_bar[0], 1);
    mbar_init(&s_bar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  unsigned phase = 0u;
  unsigned pending = 0u;
  int k0 = 0;
  int q = 0;
  bool aborted = false;

  for (;; ++q) {
    const int m = sweep_len(q, k0, p.m_first, p.m_next, p.max_iters);

    for (;;) {  // tiles
      if (tid == 0) {
        int u = (int)atomicAdd(&p.ticket[q], 1u);
        if (ld_volatile(&p.ctrl->abort) != 0u) u = p.ntiles;
        s_item = u;
      }
      if (tid < WM) s_racc[tid] = 0u;
      __syncthreads();
      const int tile = s_item;
      if (tile >= p.ntiles) break;

      const long long b = tile / p.ntd;
      const int td = tile - (int)b * p.ntd;
      const int d0 = td * CW;
      const long long d = d0 + 2 * pi;     // the pair's first channel (D is even)
      const bool cvalid = d < p.D;
      const long long bd = b * p.D + d;
      const int row0 = (int)(b * p.L);

      F2 wz = splat2(0.0f), wr = splat2(0.0f), wc = splat2(0.0f);
      F2 x0v = splat2(0.0f);
      if (cvalid) {
        wz = f2(__ldg(p.w + d), __ldg(p.w + d + 1));
        wr = f2(__ldg(p.w + p.D + d), __ldg(p.w + p.D + d + 1));
        wc = f2(__ldg(p.w + 2 * p.D + d), __ldg(p.w + 2 * p.D + d + 1));
        if (p.x0a) x0v = f2(p.x0a[bd], p.x0a[bd + 1]);
      }

      if (tid == 0) {
        for (int jj = 0; jj < 2 && jj < p.nchunks; ++jj) {
          St::issue(dsmem + jj * kStageBytes, tm, d0, row0 + jj * TCH, &s_bar[jj]);
          pending |= 1u << jj;
        }
      }

      for (int j = 0; j < p.nchunks; ++j) {
        const int st = j & 1;
        const unsigned char* stage = dsmem + st * kStageBytes;
        const long long t0 = (long long)j * TCH + (long long)seg * S;
        const bool full = cvalid && (t0 + S) <= p.L;

        // ---- current iterate and the state before this segment -------------
        F2 x[S];
        F2 xb = splat2(0.0f);
        if (k0 == 0) {
#pragma unroll
          for (int s = 0; s < S; ++s) x[s] = splat2(0.0f);
          if (t0 == 0) xb = x0v;
        } else {
#pragma unroll
          for (int s = 0; s < S; ++s) {
            const long long t = t0 + s;
            x[s] = (cvalid && t < p.L) ? ld_pair_cg(p.out0 + (b * p.L + t) * p.D + d)
                                       : splat2(0.0f);
          }
          if (t0 == 0) {
            xb = x0v;
          } else if (seg == 0) {
            xb = s_pend[(j - 1) & 1][pi];
          } else if (cvalid && t0 - 1 < p.L) {
            xb = ld_pair_cg(p.out0 + (b * p.L + t0 - 1) * p.D + d);
          }
          if (seg == NSEG - 1) s_pend[j & 1][pi] = x[S - 1];
        }

        // ---- this chunk's inputs have landed --------------------------------
        const bool ok = stage_wait(&s_bar[st], (phase >> st) & 1u, wctx);
        if (ok) {
          phase ^= 1u << st;
          if (tid == 0) pending &= ~(1u << st);
        }
        if (!__syncthreads_and(ok ? 1 : 0)) {
          if (tid == 0) raise_error(wctx, 4u);
          aborted = true;
          break;
        }

        bool any_update = false;
        for (int kk = 0; kk < m; ++kk) {
          const int k = k0 + kk;
          const bool upd = k < p.max_iters;

          Map2 mp[S];
          Map2 agg = map2_identity();
          float rmax = 0.0f;
          F2 xp = xb;
#pragma unroll
          for (int s = 0; s < S; ++s) {
            if (full || (cvalid && t0 + s < p.L)) {
              F2 pz, pr, pc;
              PairIO<PT>::template read<CW>(stage, seg * S + s, pi, pz, pr, pc);
              mp[s] = gru_newton2(pz, pr, pc, wz, wr, wc, xp, x[s], rmax);
              xp = x[s];
            } else {
              mp[s] = map2_identity();
            }
            agg = compose2(mp[s], agg);
          }
          const unsigned rbits = __reduce_max_sync(0xffffffffu, __float_as_uint(rmax));
          if (lane == 0) atomicMax(&s_racc[kk], rbits);
          if (!upd) continue;  // residual-only iteration (k == max_iters)
          any_update = true;

          // ---- combine the segments: one barrier per iteration --------------
          const int buf = kk & 1;
          Map2 wincl = agg, wexcl = map2_identity();
          if constexpr (SPL > 1) {
#pragma unroll
            for (int off = CP; off < 32; off <<= 1) {
              const Map2 o{shfl_up2(wincl.m, off), shfl_up2(wincl.v, off)};
              if (lane >= off) wincl = compose2(wincl, o);
            }
            const Map2 e{shfl_up2(wincl.m, CP), shfl_up2(wincl.v, CP)};
            if (sub > 0) wexcl = e;
          }
          if (last_in_warp) s_wagg[buf][warp][pi] = wincl;
          __syncthreads();
          Map2 pre = map2_identity();
#pragma unroll 4
          for (int w2 = 0; w2 < warp; ++w2) pre = compose2(s_wagg[buf][w2][pi], pre);
          const F2 carry = (j == 0) ? x0v : s_inc[(j - 1) & 1][kk][pi];
          const F2 xin = apply2(wexcl, apply2(pre, carry));
          if (warp == NW - 1 && last_in_warp) s_inc[j & 1][kk][pi] = apply2(agg, xin);
          F2 xr = xin;
#pragma unroll
          for (int s = 0; s < S; ++s) {
            xr = apply2(mp[s], xr);
            x[s] = xr;
          }
          xb = xin;
        }

        // ---- write the chunk; refill its stage with chunk j + 2 -------------
        if (any_update || k0 == 0) {
#pragma unroll
          for (int s = 0; s < S; ++s) {
            const long long t = t0 + s;
            if (cvalid && t < p.L) st_pair(p.out0 + (b * p.L + t) * p.D + d, x[s]);
          }
        }
        __syncthreads();  // every warp is done reading this stage
        if (tid == 0 && j + 2 < p.nchunks) {
          St::issue(dsmem + st * kStageBytes, tm, d0, row0 + (j + 2) * TCH, &s_bar[st]);
          pending |= 1u << st;
        }
      }
      if (aborted) break;
      if (tid < m) atomicMax(&p.rho_bits[k0 + tid], s_racc[tid]);
      __syncthreads();
    }
    if (aborted) break;

    if (!grid_barrier(wctx)) {
      aborted = true;
      break;
    }
    if (tid == 0) {
      int done = 0;
      for (int kk = 0; kk < m; ++kk) {
        const float r = __uint_as_float(ld_volatile(&p.rho_bits[k0 + kk]));
        if (!(r <= 3.0e38f)) {
          done = 1;
          break;
        }
        if (r <= p.tol) done = 1;
      }
      if (k0 + m > p.max_iters) done = 1;
      s_flag = done;
    }
    __syncthreads();
    if (s_flag) break;
    k0 += m;
  }

  // No copy may still be writing this CTA's shared memory when it exits.
  if (tid == 0 && pending) drain_stages(s_bar, pending, phase, wctx);

  if (blockIdx.x == 0 && tid == 0) {
    struct Info {
      int iterations, converged, status, updates, passes, reserved;
      float max_residual;
      float rho[128];
    };
    Info* info = reinterpret_cast<Info*>(p.info);
    __threadfence();
    unsigned status = ld_volatile(&p.ctrl->status);
    const int last = k0 + sweep_len(q, k0, p.m_first, p.m_next, p.max_iters) - 1;
    int iters = p.max_iters, conv = 0, nonfinite = 0;
    float maxres = 0.0f;
    for (int k = 0; k <= last && k <= p.max_iters; ++k) {
      const float r = __uint_as_float(ld_volatile(&p.rho_bits[k]));
      info->rho[k] = r;
      if (!(r <= 3.0e38f)) nonfinite = 1;
    }
    for (int k = 0; k <= last && k <= p.max_iters; ++k) {
      const float r = __uint_as_float(ld_volatile(&p.rho_bits[k]));
      iters = k;
      maxres = r;
      if (!(r <= 3.0e38f)) break;
      if (r <= p.tol) {
        conv = 1;
        break;
      }
    }
    for (int k = last + 1; k <= p.max_iters; ++k) info->rho[k] = 0.0f;
    if (status == 0u && nonfinite) status = 5u;
    info->iterations = iters;
    info->converged = (status == 0u) ? conv : 0;
    info->status = (int)status;
    info->updates = last < p.max_iters ? last + 1 : p.max_iters;
    info->passes = q + 1;
    info->reserved = 0;
    info->max_residual = maxres;
  }
}

}  // namespace pararnn
