// pararnn_proj.cuh -- the input projection P = x W^T + bias on the tensor cores.
//
// ParaRNN's cells take the projected gate pre-activations P_t = W x_t (+ bias)
// as inputs (the recurrence itself only has diagonal weights; ParaRNN TL;DR and
// Figure 2 caption); for LM-width layers this dense projection is the one
// contraction on the path.  x is [M, K] bf16 (M = B*L rows, K input features),
// W is [N, K] bf16 (N = G*D output features, the nn.Linear layout), P is [M, N]
// fp32 or bf16 -- i.e. [B, L, G, D], the layout the Newton solve reads.
//
// One CTA computes one 128 x 256 tile of P with tcgen05:
//   * warp 0, one thread: TMA copies of the x and W k-blocks (64 deep, 128-byte
//     swizzle) into a ring of shared-memory stages (mbarrier completion);
//   * warp 1, one thread: per stage, four tcgen05.mma (M=128, N=256, K=16, bf16
//     in, fp32 accumulate) into a 256-column TMEM accumulator, then
//     tcgen05.commit to release the stage;
//   * all four warps: the epilogue reads the accumulator with tcgen05.ld (warp w
//     owns TMEM lanes = rows 32w..32w+31), adds the bias and stores P.
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

template <int ST> constexpr size_t proj_smem_bytes() {
  return (size_t)ST * kProjStageBytes + 1024;  // + alignment slack for the 1024-byte swizzle atoms
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

template <int ST>
__global__ void __launch_bounds__(128, 1)
    pararnn_proj_kernel(const __grid_constant__ ProjParams p, const __grid_constant__ ProjMaps tm) {
  extern __shared__ __align__(1024) unsigned char dsmem[];
  __shared__ unsigned long long s_full[ST], s_empty[ST], s_acc;
  __shared__ unsigned s_tmem;
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned sbase = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int nb = blockIdx.x % p.ntn, mb = blockIdx.x / p.ntn;
  const int m0 = mb * kProjBM, n0 = nb * kProjBN;
  const int nk = (p.K + kProjBK - 1) / kProjBK;
  const WaitCtx wctx{nullptr, p.status_dev, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
    }
    mbar_init(&s_acc, 1);
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {  // the whole warp allocates the accumulator's 256 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kProjBN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned tmem = s_tmem;

  if (warp == 0 && lane == 0) {
    // ---- producer: k-blocks into the ring ---------------------------------
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % ST;
      const unsigned ph = (unsigned)(kb / ST) & 1u;
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
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer -----------------------------------------------------------
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % ST;
      const unsigned ph = (unsigned)(kb / ST) & 1u;
      if (!stage_wait(&s_full[s], ph, wctx)) {
        s_fail = 1;
        break;
      }
      tc_fence_after();
      const unsigned a = sbase + s * kProjStageBytes;
      const unsigned b = a + kProjABytes;
#pragma unroll
      for (int k = 0; k < kProjBK / 16; ++k)  // K = 16 per MMA: 32 bytes along the swizzled row
        umma_f16_ss(tmem, umma_desc_sw128(a + 32u * k), umma_desc_sw128(b + 32u * k), kProjIdesc,
                    (kb | k) != 0 ? 1u : 0u);
      umma_commit(&s_empty[s]);  // the stage is free once these MMAs have read it
    }
    umma_commit(&s_acc);  // the accumulator is final once every MMA has completed
  }
  __syncwarp();

  // ---- epilogue: TMEM -> registers -> bias -> P ------------------------------------
  const bool ok = stage_wait(&s_acc, 0u, wctx);
  __syncwarp();
  tc_fence_after();
  const int row = m0 + warp * 32 + lane;
  if (!ok || s_fail) {
    if (lane == 0 && p.status_dev) atomicCAS(p.status_dev, 0, 4);
  } else {
#pragma unroll 1
    for (int c0 = 0; c0 < kProjBN && n0 + c0 < p.N; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + ((unsigned)(warp * 32) << 16) + (unsigned)c0, v);
      if (nk == 0) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.0f;
      }
      const int col = n0 + c0;
      if (p.bias) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] += col + i < p.N ? __ldg(p.bias + col + i) : 0.0f;
      }
      if (row < p.M) {
        const size_t o = (size_t)row * p.N + col;
        // N is a multiple of 8: the tile's tail is whole groups of 8 columns
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (col + 8 * h + 8 > p.N) break;
          if (p.out_bf16) {
            uint4 q;
            __nv_bfloat162 t[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              t[i] = __floats2bfloat162_rn(v[8 * h + 2 * i], v[8 * h + 2 * i + 1]);
            q.x = *reinterpret_cast<unsigned*>(&t[0]);
            q.y = *reinterpret_cast<unsigned*>(&t[1]);
            q.z = *reinterpret_cast<unsigned*>(&t[2]);
            q.w = *reinterpret_cast<unsigned*>(&t[3]);
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o + 8 * h) = q;
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o + 8 * h);
            dst[0] = make_float4(v[8 * h], v[8 * h + 1], v[8 * h + 2], v[8 * h + 3]);
            dst[1] = make_float4(v[8 * h + 4], v[8 * h + 5], v[8 * h + 6], v[8 * h + 7]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kProjBN)
                 : "memory");
  }
}

}  // namespace pararnn
