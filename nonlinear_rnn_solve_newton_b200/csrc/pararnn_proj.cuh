// pararnn_proj.cuh -- the input projection P = x W^T + bias on the tensor cores.
//
// ParaRNN's cells take the projected gate pre-activations P_t = W x_t (+ bias)
// as inputs (the recurrence itself only has diagonal weights; ParaRNN TL;DR and
// Figure 2 caption); for LM-width layers this dense projection is the one
// contraction on the path.  x is [M, K] bf16 (M = B*L rows, K input features),
// W is [N, K] bf16 (N = G*D output features, the nn.Linear layout), P is [M, N]
// fp32 or bf16 -- i.e. [B, L, G, D], the layout the Newton solve reads.
//
// A persistent CTA per SM computes 128 x 256 tiles of P with tcgen05:
//   * warp 0, one thread: TMA copies of the x and W k-blocks (64 deep, 128-byte
//     swizzle) into a ring of shared-memory stages (mbarrier completion); the
//     ring runs on from one tile to the next;
//   * warp 1, one thread: per stage, four tcgen05.mma (M=128, N=256, K=16, bf16
//     in, fp32 accumulate) into one of two 256-column TMEM accumulators, then
//     tcgen05.commit to release the stage (and, after the last k-block, to
//     hand the accumulator to the epilogue);
//   * warps 2-9: the epilogue reads an accumulator with tcgen05.ld (warp w owns
//     TMEM lanes = rows 32 (w mod 4) .. + 31 and one half of the columns),
//     adds the bias, writes P by tensor stores of 32-row boxes staged in
//     shared memory and frees the accumulator -- while the MMAs of the next
//     tile run.
// Every wait is bounded; a wait that runs out sets status 4 and the CTA still
// frees its TMEM before it returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "pararnn_walk.cuh"

namespace pararnn {

constexpr int kProjBM = 128;  // rows of P per CTA (TMEM lanes)
constexpr int kProjBN = 256;  // columns of P per CTA (TMEM columns, fp32)
constexpr int kProjBK = 64;   // k per stage: one 128-byte swizzle row of bf16
constexpr unsigned kProjABytes = kProjBM * kProjBK * 2;
constexpr unsigned kProjBBytes = kProjBN * kProjBK * 2;
constexpr unsigned kProjStageBytes = kProjABytes + kProjBBytes;

// Epilogue: 8 warps, two per TMEM lane quarter (each takes 128 of the 256
// columns), each staging one 32-row x 128-byte box at a time.
constexpr int kProjEpiWarps = 8;
constexpr int kProjThreads = 32 * (2 + kProjEpiWarps);
constexpr unsigned kProjEpiBox = 32 * 128;
constexpr unsigned kProjEpiBytes = kProjEpiWarps * kProjEpiBox;

template <int ST> constexpr size_t proj_smem_bytes() {
  // + alignment slack for the 1024-byte swizzle atoms
  return (size_t)ST * kProjStageBytes + kProjEpiBytes + 1024;
}

struct ProjParams {
  const float* bias;  // [N] or NULL
  void* out;          // [M, N], fp32 or bf16
  int M, N, K;
  int ntn;            // tiles along N
  int out_bf16;
  int* status_dev;    // 0 / 4, or NULL
  long long timeout_ns;
};

struct ProjMaps {
  CUtensorMap x;  // 2-D {K, M}, box {64, 128}, 128-byte swizzle
  CUtensorMap w;  // 2-D {K, N}, box {64, 256}, 128-byte swizzle
  CUtensorMap p;  // 2-D {N, M}, box {128 bytes of columns, 32 rows}, 128-byte swizzle
};

// Shared-memory matrix descriptor of a K-major operand tile written by TMA with
// the 128-byte swizzle: rows of 128 bytes, 8-row (1024-byte) swizzle atoms
// stacked densely.  Fields: start address >> 4 (bits 0-13), leading-dimension
// offset (unused for swizzled K-major; 1), stride between 8-row groups >> 4
// (bits 32-45), descriptor version 1 (bits 46-47), swizzle mode 2 = 128 B
// (bits 61-63).
__device__ __forceinline__ unsigned long long umma_desc_sw128(unsigned saddr) {
  return (unsigned long long)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) |
         ((unsigned long long)(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at
// bit 17, M >> 4 at bit 24.
constexpr unsigned kProjIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                ((unsigned)(kProjBN >> 3) << 17) |
                                ((unsigned)(kProjBM >> 4) << 24);

__device__ __forceinline__ void tma_load_2d_s(unsigned dst, const CUtensorMap* map, int x, int y,
                                              unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void umma_f16_ss(unsigned tmem_d, unsigned long long da,
                                            unsigned long long db, unsigned idesc,
                                            unsigned accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on bar once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(unsigned long long* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(unsigned taddr, float* v) {
  unsigned r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Tensor store of a 32-row x 128-byte box from shared memory (bulk group).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, unsigned src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<unsigned long long>(map)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// The TMEM columns of one box row: 32 (fp32 out) or 64 (bf16 out), loads
// issued without waiting (tcgen05.wait::ld completes them).
template <bool OB>
__device__ __forceinline__ void tmem_ld_box_async(unsigned taddr, unsigned* r) {
#define PARARNN_LD16(OFF, R)                                                                    \
  asm volatile(                                                                                 \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "   \
      "%11, %12, %13, %14, %15}, [%16];"                                                        \
      : "=r"(R[0]), "=r"(R[1]), "=r"(R[2]), "=r"(R[3]), "=r"(R[4]), "=r"(R[5]), "=r"(R[6]),     \
        "=r"(R[7]), "=r"(R[8]), "=r"(R[9]), "=r"(R[10]), "=r"(R[11]), "=r"(R[12]), "=r"(R[13]), \
        "=r"(R[14]), "=r"(R[15])                                                                \
      : "r"(taddr + (OFF)))
  PARARNN_LD16(0u, (r + 0));
  PARARNN_LD16(16u, (r + 16));
  if constexpr (OB) {
    PARARNN_LD16(32u, (r + 32));
    PARARNN_LD16(48u, (r + 48));
  }
#undef PARARNN_LD16
}

// Epilogue of one tile for one warp: TMEM columns [c_lo, c_lo + 128) of its
// 32 lanes (rows y0 .. y0 + 31) -> + bias -> 128-byte-swizzled box in shared
// memory (16-byte chunk j of row r at chunk j ^ (r mod 8): conflict-free) ->
// tensor store.  The next box's TMEM load is in flight while the current one
// is staged and stored; when this returns, every TMEM load of the tile is done.
template <bool OB>
__device__ __forceinline__ void proj_epilogue(const ProjParams& p, const CUtensorMap* pmap,
                                              unsigned taddr, unsigned ebuf, int y0, int n0,
                                              int c_lo, bool zero) {
  constexpr int CB = OB ? 64 : 32;  // columns per 128-byte box row
  const int lane = threadIdx.x & 31;
  int nb = 0;  // boxes of this tile for this warp
  while (nb * CB < 128 && n0 + c_lo + nb * CB < p.N) ++nb;
  if (nb == 0) return;
  unsigned cur[CB], nxt[CB];
  tmem_ld_box_async<OB>(taddr + (unsigned)c_lo, cur);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll 1
  for (int b = 0; b < nb; ++b) {
    const int col = n0 + c_lo + b * CB;
    if (zero) {
#pragma unroll
      for (int i = 0; i < CB; ++i) cur[i] = 0u;
    }
    if (p.bias) {
      // bias is 16-byte aligned and N a multiple of 8: groups of 4 are whole
#pragma unroll
      for (int i = 0; i < CB; i += 4) {
        if (col + i < p.N) {
          const float4 bb = __ldg(reinterpret_cast<const float4*>(p.bias + col + i));
          cur[i] = __float_as_uint(__uint_as_float(cur[i]) + bb.x);
          cur[i + 1] = __float_as_uint(__uint_as_float(cur[i + 1]) + bb.y);
          cur[i + 2] = __float_as_uint(__uint_as_float(cur[i + 2]) + bb.z);
          cur[i + 3] = __float_as_uint(__uint_as_float(cur[i + 3]) + bb.w);
        }
      }
    }
    if (b + 1 < nb) tmem_ld_box_async<OB>(taddr + (unsigned)(c_lo + (b + 1) * CB), nxt);
    // the previous tensor store has finished reading the staging box
    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    __syncwarp();
    const unsigned rowp = ebuf + (unsigned)lane * 128u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      unsigned w0, w1, w2, w3;
      if constexpr (OB) {
        __nv_bfloat162 t0 = __floats2bfloat162_rn(__uint_as_float(cur[8 * j]), __uint_as_float(cur[8 * j + 1]));
        __nv_bfloat162 t1 = __floats2bfloat162_rn(__uint_as_float(cur[8 * j + 2]), __uint_as_float(cur[8 * j + 3]));
        __nv_bfloat162 t2 = __floats2bfloat162_rn(__uint_as_float(cur[8 * j + 4]), __uint_as_float(cur[8 * j + 5]));
        __nv_bfloat162 t3 = __floats2bfloat162_rn(__uint_as_float(cur[8 * j + 6]), __uint_as_float(cur[8 * j + 7]));
        w0 = *reinterpret_cast<unsigned*>(&t0);
        w1 = *reinterpret_cast<unsigned*>(&t1);
        w2 = *reinterpret_cast<unsigned*>(&t2);
        w3 = *reinterpret_cast<unsigned*>(&t3);
      } else {
        w0 = cur[4 * j];
        w1 = cur[4 * j + 1];
        w2 = cur[4 * j + 2];
        w3 = cur[4 * j + 3];
      }
      const unsigned dst = rowp + ((unsigned)(j ^ (lane & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w0), "r"(w1),
                   "r"(w2), "r"(w3)
                   : "memory");
    }
    // make the generic-proxy writes visible to the tensor store, then issue it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) tma_store_2d(pmap, ebuf, col, y0);
    if (b + 1 < nb) {
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int i = 0; i < CB; ++i) cur[i] = nxt[i];
    }
  }
}

// Persistent: CTA c takes tiles c, c + grid, ... (row-block major, so CTAs
// running at once share x row blocks and all of W in L2).  Warp 0 = TMA
// producer, warp 1 = MMA issuer, warps 2-5 = epilogue; the shared-memory ring
// runs on across tiles and the accumulator is double-buffered in TMEM (2 x 256
// columns), so the epilogue of tile i overlaps the MMAs of tile i + 1.
template <int ST, bool OB>
__global__ void __launch_bounds__(kProjThreads, 1)
    pararnn_proj_kernel(const __grid_constant__ ProjParams p, const __grid_constant__ ProjMaps tm) {
  extern __shared__ __align__(1024) unsigned char dsmem[];
  __shared__ unsigned long long s_full[ST], s_empty[ST], s_tfull[2], s_tempty[2];
  __shared__ unsigned s_tmem;
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned sbase = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int nk = (p.K + kProjBK - 1) / kProjBK;
  const int ntiles = ((p.M + kProjBM - 1) / kProjBM) * p.ntn;
  const WaitCtx wctx{nullptr, p.status_dev, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&s_tfull[a], 1);
      mbar_init(&s_tempty[a], 32 * kProjEpiWarps);  // every epilogue thread arrives
    }
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {  // the whole warp allocates both accumulators (all 512 columns)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(2 * kProjBN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: k-blocks of every tile into the ring -----------------------
      unsigned it = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*(volatile int*)&s_fail; tile += gridDim.x) {
        const int m0 = (tile / p.ntn) * kProjBM, n0 = (tile % p.ntn) * kProjBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const unsigned ph = (it / ST) & 1u;
          // a fresh barrier passes a wait on parity 1: the first ST stages are free
          if (!stage_wait(&s_empty[s], ph ^ 1u, wctx)) {
            s_fail = 1;
            break;
          }
          const unsigned a = sbase + s * kProjStageBytes;
          mbar_expect_tx(&s_full[s], kProjStageBytes);
          tma_load_2d_s(a, &tm.x, kb * kProjBK, m0, &s_full[s]);
          tma_load_2d_s(a + kProjABytes, &tm.w, kb * kProjBK, n0, &s_full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ---------------------------------------------------------------
      unsigned it = 0, lt = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*(volatile int*)&s_fail; tile += gridDim.x, ++lt) {
        const unsigned acc = lt & 1u, use = lt >> 1;
        // the epilogue has drained this accumulator (fresh: passes)
        if (!stage_wait(&s_tempty[acc], (use & 1u) ^ 1u, wctx)) {
          s_fail = 1;
          break;
        }
        tc_fence_after();
        const unsigned d = tmem + acc * kProjBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const unsigned ph = (it / ST) & 1u;
          if (!stage_wait(&s_full[s], ph, wctx)) {
            s_fail = 1;
            break;
          }
          tc_fence_after();
          const unsigned a = sbase + s * kProjStageBytes;
          const unsigned b = a + kProjABytes;
#pragma unroll
          for (int k = 0; k < kProjBK / 16; ++k)  // K = 16 per MMA: 32 bytes along the row
            umma_f16_ss(d, umma_desc_sw128(a + 32u * k), umma_desc_sw128(b + 32u * k),
                        kProjIdesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&s_empty[s]);  // the stage is free once these MMAs have read it
        }
        umma_commit(&s_tfull[acc]);  // the tile's accumulator is final
      }
    }
  } else {
    // ---- epilogue (warps 2-9: TMEM lane quarter = warp % 4, column half) -------
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const unsigned ebuf = sbase + ST * kProjStageBytes + (unsigned)(warp - 2) * kProjEpiBox;
    unsigned lt = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
      const unsigned acc = lt & 1u, use = lt >> 1;
      const bool ok = stage_wait(&s_tfull[acc], use & 1u, wctx);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok) || *(volatile int*)&s_fail) {
        s_fail = 1;
        break;
      }
      tc_fence_after();
      const int m0 = (tile / p.ntn) * kProjBM, n0 = (tile % p.ntn) * kProjBN;
      proj_epilogue<OB>(p, &tm.p, tmem + acc * kProjBN + ((unsigned)(32 * q) << 16), ebuf,
                    m0 + 32 * q, n0, half * 128, nk == 0);
      tc_fence_before();
      mbar_arrive(&s_tempty[acc]);
    }
    // every tensor store of this warp has completed before the CTA exits
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && s_fail && p.status_dev) atomicCAS(p.status_dev, 0, 4);
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(2 * kProjBN)
                 : "memory");
  }
}

}  // namespace pararnn

// ===========================================================================
// CTA-pair variant: a cluster of two CTAs computes 256 x 256 tiles with
// tcgen05.mma.cta_group::2 (M = 256).  Each CTA loads its own 128 rows of x and
// its own 128 rows of W (half of N) per k-block -- 32 KB instead of 48 KB for
// the same tensor work, so six stages fit and each SM pulls a third less from
// L2.  Each CTA copies only into its own shared memory (plain tensor copies);
// the copies complete on the leader CTA's barrier (.cta_group::2).
//   * leader (rank 0), warp 1: issues the MMAs (A from both CTAs' stages, B
//     from both CTAs' stages, D rows 128 r .. 128 r + 127 in CTA r's TMEM) and
//     commits them to the stage and accumulator barriers of both CTAs;
//   * both CTAs: warp 0 produces, warps 2-9 drain their own TMEM; the leader's
//     accumulator-free barrier counts the epilogue threads of both CTAs.
// ===========================================================================
namespace pararnn {

constexpr unsigned kP2ABytes = kProjBM * kProjBK * 2;       // 128 rows of x
constexpr unsigned kP2BBytes = (kProjBN / 2) * kProjBK * 2;  // 128 rows of W
constexpr unsigned kP2StageBytes = kP2ABytes + kP2BBytes;
// M = 256 (both CTAs), N = 256, fp32 accumulate, bf16 A/B, K-major
constexpr unsigned kP2Idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                              ((unsigned)(kProjBN >> 3) << 17) | ((unsigned)(256 >> 4) << 24);

template <int ST> constexpr size_t proj2_smem_bytes() {
  return (size_t)ST * kP2StageBytes + kProjEpiBytes + 1024;
}

__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of this CTA's shared variable at `local` in CTA `rank`
__device__ __forceinline__ unsigned mapa_shared(unsigned local, unsigned rank) {
  unsigned r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(unsigned dst, const CUtensorMap* map, int x, int y,
                                                 unsigned bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void umma_f16_ss_pair(unsigned tmem_d, unsigned long long da,
                                                 unsigned long long db, unsigned idesc,
                                                 unsigned accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this offset in both CTAs of the pair when the
// MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(unsigned long long* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], m;\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(unsigned bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

template <int ST, bool OB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kProjThreads, 1)
    pararnn_proj2_kernel(const __grid_constant__ ProjParams p, const __grid_constant__ ProjMaps tm) {
  extern __shared__ __align__(1024) unsigned char dsmem[];
  __shared__ unsigned long long s_full[ST], s_empty[ST], s_tfull[2], s_tempty[2];
  __shared__ unsigned s_tmem;
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned rank = cluster_rank();
  const unsigned sbase = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int nk = (p.K + kProjBK - 1) / kProjBK;
  const int ntm = (p.M + 2 * kProjBM - 1) / (2 * kProjBM);
  const int ntiles = ntm * p.ntn;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const WaitCtx wctx{nullptr, p.status_dev, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&s_tfull[a], 1);
      mbar_init(&s_tempty[a], 2 * 32 * kProjEpiWarps);  // epilogue threads of both CTAs
    }
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {  // same warp in both CTAs: both accumulators of the pair
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(2 * kProjBN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const unsigned tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer (both CTAs): this CTA's halves of each k-block ------------------
      unsigned it = 0;
      for (int tile = pair; tile < ntiles && !*(volatile int*)&s_fail; tile += npairs) {
        const int m0 = (tile / p.ntn) * 2 * kProjBM + (int)rank * kProjBM;
        const int n0 = (tile % p.ntn) * kProjBN + (int)rank * (kProjBN / 2);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const unsigned ph = (it / ST) & 1u;
          if (!stage_wait(&s_empty[s], ph ^ 1u, wctx)) {
            s_fail = 1;
            break;
          }
          // the leader's barrier expects both CTAs' bytes of this stage
          if (rank == 0) mbar_expect_tx(&s_full[s], 2 * kP2StageBytes);
          const unsigned bar = mapa_shared(smem_u32(&s_full[s]), 0);
          const unsigned a = sbase + s * kP2StageBytes;
          tma_load_2d_pair(a, &tm.x, kb * kProjBK, m0, bar);
          tma_load_2d_pair(a + kP2ABytes, &tm.w, kb * kProjBK, n0, bar);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---- MMA issuer (leader CTA) ----------------------------------------------------
      unsigned it = 0, lt = 0;
      for (int tile = pair; tile < ntiles && !*(volatile int*)&s_fail; tile += npairs, ++lt) {
        const unsigned acc = lt & 1u, use = lt >> 1;
        if (!stage_wait(&s_tempty[acc], (use & 1u) ^ 1u, wctx)) {
          s_fail = 1;
          break;
        }
        tc_fence_after();
        const unsigned d = tmem + acc * kProjBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const unsigned ph = (it / ST) & 1u;
          if (!stage_wait(&s_full[s], ph, wctx)) {
            s_fail = 1;
            break;
          }
          tc_fence_after();
          const unsigned a = sbase + s * kP2StageBytes;
          const unsigned b = a + kP2ABytes;
#pragma unroll
          for (int k = 0; k < kProjBK / 16; ++k)
            umma_f16_ss_pair(d, umma_desc_sw128(a + 32u * k), umma_desc_sw128(b + 32u * k),
                             kP2Idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit_pair(&s_empty[s]);  // frees stage s in both CTAs
        }
        umma_commit_pair(&s_tfull[acc]);  // both CTAs' accumulators are final
      }
    }
  } else {
    // ---- epilogue (both CTAs, own TMEM: rows m0 + 128 rank + 32 q + lane) -------------
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const unsigned ebuf = sbase + ST * kP2StageBytes + (unsigned)(warp - 2) * kProjEpiBox;
    const unsigned tempty0 = mapa_shared(smem_u32(&s_tempty[0]), 0);
    const unsigned tempty1 = mapa_shared(smem_u32(&s_tempty[1]), 0);
    unsigned lt = 0;
    for (int tile = pair; tile < ntiles; tile += npairs, ++lt) {
      const unsigned acc = lt & 1u, use = lt >> 1;
      const bool ok = stage_wait(&s_tfull[acc], use & 1u, wctx);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok) || *(volatile int*)&s_fail) {
        s_fail = 1;
        break;
      }
      tc_fence_after();
      const int m0 = (tile / p.ntn) * 2 * kProjBM + (int)rank * kProjBM;
      const int n0 = (tile % p.ntn) * kProjBN;
      proj_epilogue<OB>(p, &tm.p, tmem + acc * kProjBN + ((unsigned)(32 * q) << 16), ebuf,
                        m0 + 32 * q, n0, half * 128, nk == 0);
      tc_fence_before();
      mbar_arrive_cluster(acc ? tempty1 : tempty0);
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // no CTA leaves while its peer may still signal it
  if (threadIdx.x == 0 && s_fail && p.status_dev) atomicCAS(p.status_dev, 0, 4);
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(2 * kProjBN)
                 : "memory");
  }
}

}  // namespace pararnn
