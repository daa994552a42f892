// pararnn_projsolve.cuh -- a ParaGRU layer from its inputs: the input projection
// P = x W^T + bias on the tensor cores feeding the Newton walk in one persistent
// kernel, so that P is never written to (or read back from) HBM.
//
// ParaRNN's language-model layers apply dense weights to the inputs and keep
// only diagonal weights in the recurrence (TL;DR, Abstract).  Run as two calls,
// the projection writes P [B, L, 3, D] to HBM and the Newton solve reads it
// back.  Here a CTA owns a work item = (batch row b, 32 consecutive channels)
// and walks its time chunks of 128 steps in order.  Items are numbered channel
// group first (item = g B + b), so the CTAs running at once are the batch rows
// of a few channel groups: they share those groups' rows of W in L2, and x is
// streamed once per wave of items:
//   * warp 0, one thread: TMA copies of each chunk's 64-deep k-blocks of x
//     (rows b*L + t0 .. + 127) and of the item's W rows -- the z, r and c
//     blocks of its 32 channels, one 3-D box -- into a ring of stages;
//   * warp 1, one thread: tcgen05.mma with M = 128 steps, N = 96 (3 gates x 32
//     channels), bf16 operands, fp32 accumulation, into one of two TMEM
//     accumulators;
//   * 16 walker warps (warps 2-17) in NG groups, each group walking its own
//     items: read the chunk's accumulator (a thread = one time step, a warp = a
//     quarter of the steps x a share of the 96 columns), add the bias and lay
//     the chunk out in shared memory as [step][gate][channel] fp32, free the
//     accumulator, and run the sweep's m Newton iterations on the chunk exactly
//     as the tensor-copy walker does (a thread = one channel x 128 / warps steps:
//     cell, Jacobian and residual, serial composition, cross-warp combine, the
//     carry of the previous chunk at the same iteration kept in shared memory).
// The MMAs of chunk j + 1 run on the tensor cores while a group iterates on
// chunk j on the CUDA cores.  With NG = 2 the CTA holds two items at once (two
// accumulators and one staged chunk per group, the copy and MMA threads
// alternating between the groups' chunks): one group computes while the other
// waits at its barriers, and 1.5-2 items per CTA run in one round instead of
// two.  A later sweep -- needed only when the first sweep's
// m iterations do not converge -- recomputes the projection.  Every wait is
// bounded; a wait that runs out sets the status and the CTA still waits for its
// copies and MMAs and frees its TMEM before it returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "pararnn_kernel.cuh"
#include "pararnn_proj.cuh"
#include "pararnn_walk.cuh"

namespace pararnn {

constexpr int kPsCW = 32;                         // channels per work item
constexpr int kPsN = 3 * kPsCW;                   // accumulator columns: gates z, r, c
constexpr int kPsBM = 128;                        // time steps per chunk (TMEM lanes)
constexpr int kPsWalkWarps = 16;                  // walker warps (all groups)
constexpr int kPsThreads = 32 * (2 + kPsWalkWarps);
constexpr unsigned kPsABytes = kPsBM * kProjBK * 2;         // x k-block: 128 rows x 128 B
constexpr unsigned kPsBBytes = kPsN * kProjBK * 2;          // W k-block: 96 rows x 128 B
constexpr unsigned kPsStageBytes = kPsABytes + kPsBBytes;   // 28 KB, a multiple of 1024
constexpr int kPsRow = kPsN + 4;                  // padded row of the staged chunk (words)
constexpr unsigned kPsPBytes = kPsBM * kPsRow * 4;          // one group's staged chunk
constexpr unsigned kPsAccCols = 128;              // TMEM columns per accumulator
// kind::f16: fp32 accumulator, bf16 A and B, both K-major, N = 96, M = 128.
constexpr unsigned kPsIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                              ((unsigned)(kPsN >> 3) << 17) | ((unsigned)(kPsBM >> 4) << 24);
static_assert(kPsStageBytes % 1024 == 0 && kPsABytes % 1024 == 0, "swizzle atoms stay aligned");
static_assert(kPsN % 16 == 0 && kPsN <= 256, "UMMA N for M = 128");

// The walker's shape for NG groups.
template <int NG> struct PsShape {
  static_assert(NG == 1 || NG == 2, "walker groups");
  static constexpr int NW = kPsWalkWarps / NG;   // walker warps per group = time segments
  static constexpr int S = kPsBM / NW;           // steps per walker thread
  static constexpr int PARTS = NW / 4;           // warps per TMEM lane quarter
  static constexpr int COLS = kPsN / PARTS;      // accumulator columns one warp drains
  static constexpr unsigned TMEM_COLS = NG == 1 ? 256u : 512u;  // two accumulators per group
  static_assert(COLS % 8 == 0, "columns are drained 8 at a time");
};

template <int ST, int NG> constexpr size_t ps_smem_bytes() {
  return (size_t)ST * kPsStageBytes + (size_t)NG * kPsPBytes + 1024;  // + alignment slack
}

struct PsParams {
  const float* bias;   // [3 D] or NULL
  const float* w;      // diagonal recurrence weights a [3, D]
  const float* h0;     // [B, D] or NULL (= 0)
  float* h;            // [B, L, D], t = 1..L
  long long B, L, D;
  int K;
  int ntd;             // 32-channel groups along D
  int nitems;          // B * ntd
  int nchunks;         // ceil(L / 128)
  float tol;
  int max_iters;
  int m_first, m_next;
  Ctrl* ctrl;
  unsigned* rho_bits;  // [max_iters + 1]
  void* info;          // pararnn_solve_info_t (device)
  long long timeout_ns;
};

struct PsMaps {
  CUtensorMap x;  // 2-D {K, B L}, box {64, 128}, 128-byte swizzle
  CUtensorMap w;  // 3-D {K, D, 3} (W viewed as gate blocks), box {64, 32, 3}, 128-byte swizzle
};

__device__ __forceinline__ void tma_load_3d_s(unsigned dst, const CUtensorMap* map, int x, int y,
                                              int z, unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Named barrier of one walker group (barrier 0 stays __syncthreads; group g
// uses barrier 1 + g).
template <int NG>
__device__ __forceinline__ void ps_walker_sync(int grp) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "n"(32 * PsShape<NG>::NW) : "memory");
}
// The same barrier, returning whether `ok` held for every thread of the group.
template <int NG>
__device__ __forceinline__ bool ps_walker_all(int grp, bool ok) {
  unsigned r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(ok ? 1u : 0u), "r"(1 + grp), "n"(32 * PsShape<NG>::NW)
      : "memory");
  return r != 0u;
}

// Item r of this CTA (r = 0, 1, ...) is blockIdx.x + r gridDim.x; it belongs to
// walker group r % NG and round r / NG.  The copy and MMA threads visit the
// jobs round by round, chunk by chunk, group by group; each group consumes its
// own jobs in that order.
template <int ST, int NG>
__global__ void __launch_bounds__(kPsThreads, 1)
    pararnn_projsolve_kernel(const __grid_constant__ PsParams p,
                             const __grid_constant__ PsMaps tm) {
  using Sh = PsShape<NG>;
  constexpr int S = Sh::S;
  constexpr int NW = Sh::NW;
  constexpr int CW = kPsCW;
  constexpr int WM = kMaxWalkIters;

  extern __shared__ __align__(1024) unsigned char dsmem[];
  __shared__ unsigned long long s_full[ST], s_empty[ST], s_tfull[NG][2], s_tempty[NG][2], s_mdone;
  __shared__ unsigned s_tmem;
  __shared__ unsigned s_mma_uses;      // stage uses the MMA thread consumed
  __shared__ int s_fail;
  __shared__ int s_flag;
  __shared__ Map<1> s_wagg[NG][2][NW][CW];
  __shared__ Vec<1> s_inc[NG][2][WM][CW];
  __shared__ Vec<1> s_pend[NG][2][CW];
  __shared__ unsigned s_racc[NG][WM];
  __shared__ __align__(16) float s_bias[NG][kPsN];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned sraw = smem_u32(dsmem);
  const unsigned sbase = (sraw + 1023u) & ~1023u;
  float* const Ps0 = reinterpret_cast<float*>(dsmem + (sbase - sraw) + ST * kPsStageBytes);
  const int nk = (p.K + kProjBK - 1) / kProjBK;
  const WaitCtx wctx{p.ctrl, nullptr, p.timeout_ns};
  // items of this CTA (the grid never exceeds the item count) and rounds
  const int nmine = (p.nitems - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  const int nrounds = (nmine + NG - 1) / NG;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
    }
    for (int g = 0; g < NG; ++g)
      for (int a = 0; a < 2; ++a) {
        mbar_init(&s_tfull[g][a], 1);
        mbar_init(&s_tempty[g][a], 32 * NW);  // every thread of the group arrives
      }
    mbar_init(&s_mdone, 1);
    s_fail = 0;
    s_mma_uses = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {  // the whole warp allocates the accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(Sh::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned tmem = s_tmem;

  unsigned pit = 0;           // producer: stage uses issued
  unsigned mit = 0;           // MMA: stage uses consumed
  unsigned mlt[NG];           // MMA: accumulators of each group filled
#pragma unroll
  for (int g = 0; g < NG; ++g) mlt[g] = 0;
  unsigned wlt = 0;           // walker: its group's accumulators drained
  int k0 = 0, q = 0;
  bool aborted = false;

  for (;; ++q) {
    const int m = sweep_len(q, k0, p.m_first, p.m_next, p.max_iters);

    if (warp == 0) {
      if (lane == 0) {
        // ---- producer: x and W k-blocks of every job ---------------------------------
        for (int R = 0; R < nrounds; ++R)
          for (int j = 0; j < p.nchunks; ++j)
            for (int grp = 0; grp < NG; ++grp) {
              const int r = R * NG + grp;
              if (r >= nmine) break;
              const int it = (int)blockIdx.x + r * (int)gridDim.x;
              const int g = it / (int)p.B;
              const long long b = it - (long long)g * p.B;
              const int row = (int)(b * p.L) + j * kPsBM;
              for (int kb = 0; kb < nk; ++kb, ++pit) {
                const int s = (int)(pit % ST);
                const unsigned ph = (pit / ST) & 1u;
                // a fresh barrier passes a wait on parity 1: the first ST stages are free
                if (*(volatile int*)&s_fail || !stage_wait(&s_empty[s], ph ^ 1u, wctx)) {
                  s_fail = 1;
                  goto produced;
                }
                const unsigned a = sbase + s * kPsStageBytes;
                mbar_expect_tx(&s_full[s], kPsStageBytes);
                tma_load_2d_s(a, &tm.x, kb * kProjBK, row, &s_full[s]);
                tma_load_3d_s(a + kPsABytes, &tm.w, kb * kProjBK, g * CW, 0, &s_full[s]);
              }
            }
      produced:;
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---- MMA issuer ------------------------------------------------------------------
        for (int R = 0; R < nrounds; ++R)
          for (int j = 0; j < p.nchunks; ++j)
            for (int grp = 0; grp < NG; ++grp) {
              if (R * NG + grp >= nmine) break;
              const unsigned acc = mlt[grp] & 1u, use = mlt[grp] >> 1;
              // the group has drained this accumulator (fresh: passes)
              if (*(volatile int*)&s_fail ||
                  !stage_wait(&s_tempty[grp][acc], (use & 1u) ^ 1u, wctx)) {
                s_fail = 1;
                goto issued;
              }
              tc_fence_after();
              const unsigned d = tmem + (unsigned)(grp * 2 + (int)acc) * kPsAccCols;
              for (int kb = 0; kb < nk; ++kb, ++mit) {
                const int s = (int)(mit % ST);
                const unsigned ph = (mit / ST) & 1u;
                if (!stage_wait(&s_full[s], ph, wctx)) {
                  s_fail = 1;
                  goto issued;
                }
                tc_fence_after();
                const unsigned a = sbase + s * kPsStageBytes;
                const unsigned bb = a + kPsABytes;
#pragma unroll
                for (int k = 0; k < kProjBK / 16; ++k)  // K = 16 per MMA: 32 bytes along a row
                  umma_f16_ss(d, umma_desc_sw128(a + 32u * k), umma_desc_sw128(bb + 32u * k),
                              kPsIdesc, (kb | k) != 0 ? 1u : 0u);
                umma_commit(&s_empty[s]);  // the stage is free once these MMAs have read it
              }
              umma_commit(&s_tfull[grp][acc]);  // the chunk's accumulator is final
              ++mlt[grp];
            }
      issued:
        s_mma_uses = mit;
      }
    } else {
      // ---- the walker groups (warps 2 .. 17) -------------------------------------------
      const int grp = (warp - 2) / NW;
      const int ww = (warp - 2) - grp * NW;       // time segment of the chunk
      const int tw = ww * 32 + lane;              // thread within the group
      const int c = lane;                         // channel within the item
      const int quarter = warp & 3;               // the TMEM lanes (time steps) this warp may read
      const int part = ww >> 2;                   // its Sh::COLS of the 96 accumulator columns
      float* const Ps = Ps0 + grp * (kPsBM * kPsRow);
      for (int r = grp; r < nmine && !aborted; r += NG) {
        const int it = (int)blockIdx.x + r * (int)gridDim.x;
        const int g = it / (int)p.B;
        const long long b = it - (long long)g * p.B;
        const long long d = (long long)g * CW + c;
        const bool cvalid = d < p.D;
        const long long bd = b * p.D + d;
        float wv[3];
#pragma unroll
        for (int gt = 0; gt < 3; ++gt)
          wv[gt] = cvalid ? __ldg(p.w + (long long)gt * p.D + d) : 0.0f;
        Vec<1> x0v;
        x0v.x[0] = (cvalid && p.h0) ? __ldg(p.h0 + bd) : 0.0f;
        if (tw < WM) s_racc[grp][tw] = 0u;
        if (tw < kPsN) {
          const long long dd = (long long)g * CW + (tw % CW);
          s_bias[grp][tw] = (p.bias && dd < p.D)
                                ? __ldg(p.bias + (long long)(tw / CW) * p.D + dd)
                                : 0.0f;
        }
        ps_walker_sync<NG>(grp);

        for (int j = 0; j < p.nchunks; ++j) {
          // ---- the chunk's projection: TMEM -> + bias -> shared memory ----------
          const unsigned acc = wlt & 1u, use = wlt >> 1;
          const bool ok = stage_wait(&s_tfull[grp][acc], use & 1u, wctx);
          if (!ps_walker_all<NG>(grp, ok && !*(volatile int*)&s_fail)) {
            if (tw == 0) {
              s_fail = 1;
              raise_error(wctx, 4u);
            }
            aborted = true;
            break;
          }
          ++wlt;
          tc_fence_after();
          {
            const unsigned taddr = tmem + (unsigned)(grp * 2 + (int)acc) * kPsAccCols +
                                   ((unsigned)(32 * quarter) << 16) + (unsigned)(Sh::COLS * part);
            unsigned rv[Sh::COLS];
#pragma unroll
            for (int i = 0; i < Sh::COLS; i += 8)
              asm volatile(
                  "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                  : "=r"(rv[i]), "=r"(rv[i + 1]), "=r"(rv[i + 2]), "=r"(rv[i + 3]), "=r"(rv[i + 4]),
                    "=r"(rv[i + 5]), "=r"(rv[i + 6]), "=r"(rv[i + 7])
                  : "r"(taddr + (unsigned)i));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            float* dst = Ps + (32 * quarter + lane) * kPsRow + Sh::COLS * part;
            const float* bsrc = s_bias[grp] + Sh::COLS * part;
#pragma unroll
            for (int i = 0; i < Sh::COLS; i += 4) {
              const float4 bb = *reinterpret_cast<const float4*>(bsrc + i);
              *reinterpret_cast<float4*>(dst + i) =
                  make_float4(__uint_as_float(rv[i]) + bb.x, __uint_as_float(rv[i + 1]) + bb.y,
                              __uint_as_float(rv[i + 2]) + bb.z, __uint_as_float(rv[i + 3]) + bb.w);
            }
          }
          tc_fence_before();
          mbar_arrive(&s_tempty[grp][acc]);  // the MMAs of a later chunk may use it
          ps_walker_sync<NG>(grp);           // the whole chunk is in shared memory

          // ---- the sweep's m Newton iterations on the chunk -------------------------
          const long long t0 = (long long)j * kPsBM + (long long)ww * S;
          const bool full = cvalid && (t0 + S) <= p.L;
          const float* prow = Ps + (ww * S) * kPsRow + c;
          Vec<1> x[S];
          Vec<1> xb;
          xb.x[0] = 0.0f;
          if (k0 == 0) {
#pragma unroll
            for (int s = 0; s < S; ++s) x[s].x[0] = 0.0f;
            if (t0 == 0) xb = x0v;
          } else {
#pragma unroll
            for (int s = 0; s < S; ++s) {
              const long long t = t0 + s;
              x[s].x[0] = (cvalid && t < p.L) ? ldcg(p.h + (b * p.L + t) * p.D + d) : 0.0f;
            }
            if (t0 == 0) {
              xb = x0v;
            } else if (ww == 0) {
              xb = s_pend[grp][(j - 1) & 1][c];
            } else if (cvalid && t0 - 1 < p.L) {
              xb.x[0] = ldcg(p.h + (b * p.L + t0 - 1) * p.D + d);
            }
            if (ww == NW - 1) s_pend[grp][j & 1][c] = x[S - 1];
          }

          bool any_update = false;
          for (int kk = 0; kk < m; ++kk) {
            const int k = k0 + kk;
            const bool upd = k < p.max_iters;
            Map<1> mp[S];
            Map<1> agg = map_identity<1>();
            float rmax = 0.0f;
            Vec<1> xp = xb;
#pragma unroll
            for (int s = 0; s < S; ++s) {
              if (full || (cvalid && t0 + s < p.L)) {
                const float vin[3] = {prow[s * kPsRow], prow[s * kPsRow + CW],
                                      prow[s * kPsRow + 2 * CW]};
                mp[s] = newton_step<kGru>(vin, wv, xp, x[s], rmax);
                xp = x[s];
              } else {
                mp[s] = map_identity<1>();
              }
              agg = compose(mp[s], agg);
            }
            const unsigned rbits = __reduce_max_sync(0xffffffffu, __float_as_uint(rmax));
            if (lane == 0) atomicMax(&s_racc[grp][kk], rbits);
            if (!upd) continue;  // residual-only iteration (k == max_iters)
            any_update = true;

            // one barrier per iteration: each warp composes the aggregates of the
            // warps before it (double-buffered by iteration parity) and applies the
            // prefix to the carry of the previous chunk at this iteration
            const int buf = kk & 1;
            s_wagg[grp][buf][ww][c] = agg;
            ps_walker_sync<NG>(grp);
            Map<1> pre = map_identity<1>();
#pragma unroll 4
            for (int w2 = 0; w2 < ww; ++w2) pre = compose(s_wagg[grp][buf][w2][c], pre);
            const Vec<1> carry = (j == 0) ? x0v : s_inc[grp][(j - 1) & 1][kk][c];
            const Vec<1> xin = apply(pre, carry);
            if (ww == NW - 1) s_inc[grp][j & 1][kk][c] = apply(agg, xin);
            Vec<1> xr = xin;
#pragma unroll
            for (int s = 0; s < S; ++s) {
              xr = apply(mp[s], xr);
              x[s] = xr;
            }
            xb = xin;
          }

          // ---- write the chunk's iterate ---------------------------------------------
          if (any_update || k0 == 0) {
#pragma unroll
            for (int s = 0; s < S; ++s) {
              const long long t = t0 + s;
              if (cvalid && t < p.L) p.h[(b * p.L + t) * p.D + d] = x[s].x[0];
            }
          }
          ps_walker_sync<NG>(grp);  // every warp of the group is done with the staged chunk
        }
        if (aborted) break;
        if (tw < m) atomicMax(&p.rho_bits[k0 + tw], s_racc[grp][tw]);
        ps_walker_sync<NG>(grp);
      }
    }

    // ---- end of the sweep: every role is done; the global stop decision ------------
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (s_fail) {
      aborted = true;
      break;
    }
    if (!grid_barrier(wctx)) {
      aborted = true;
      break;
    }
    if (threadIdx.x == 0) s_flag = sweep_stops(p.rho_bits, k0, m, p.max_iters, p.tol);
    __syncthreads();
    if (s_flag) break;
    k0 += m;
  }

  // ---- leave cleanly: no copy or MMA may still target this CTA's memory ----------
  if (warp == 0 && lane == 0) {
    WaitCtx wl = wctx;
    if (wl.timeout_ns < 2000000000LL) wl.timeout_ns = 2000000000LL;
    for (unsigned u = s_mma_uses; u < pit; ++u)  // issued copies the MMAs never consumed
      stage_wait(&s_full[u % ST], (u / ST) & 1u, wl);
  }
  if (warp == 1 && lane == 0) {
    WaitCtx wl = wctx;
    if (wl.timeout_ns < 2000000000LL) wl.timeout_ns = 2000000000LL;
    umma_commit(&s_mdone);  // arrives once every MMA this thread issued has completed
    stage_wait(&s_mdone, 0u, wl);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Sh::TMEM_COLS)
                 : "memory");
  }

  if (blockIdx.x == 0 && threadIdx.x == 0)
    write_solve_info(p.info, p.ctrl, p.rho_bits,
                     k0 + sweep_len(q, k0, p.m_first, p.m_next, p.max_iters) - 1, q + 1,
                     p.max_iters, p.tol, aborted ? 4u : 0u);
}

}  // namespace pararnn
