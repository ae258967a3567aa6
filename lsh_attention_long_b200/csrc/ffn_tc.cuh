// Chunked position-wise feed-forward on the 5th-generation tensor cores
// (bf16 in, fp32 accumulation, bf16 out).
//
// "Reformer explainer" (akshathtiwari.co.in/blog/reformer): beside LSH
// attention and reversible layers, Reformer runs its feed-forward in chunks;
// "Reformer Language Models (Korean)" (techvasolutions.com, Reformer
// overview): feed-forward activations can dominate memory, so the
// feed-forward is chunked to cut peak memory.  Per position
//   y = W2 max(0, W1 x + b1) + b2,
// evaluated `chunk` positions at a time: the hidden activation [chunk, d_ff]
// exists for one chunk only (and, at the sizes used, stays in L2 between its
// two products).
//
// Each product is one launch of gemm_tc_kernel:
//   C[M, N] = act(A[M, K] . B[N, K]^T + bias[N])
// with A and B row-major bf16 (both K-major), C row-major bf16.  Tiles of
// 128 x 256 outputs, K in steps of 64.  Warp roles (192 threads):
//   warp 0     one thread loads A and B tiles with TMA (tensor maps, 128-byte
//              swizzle) into a ring of four stages (full/empty mbarriers with
//              transaction counts);
//   warp 1     one thread issues tcgen05.mma (M = 128, N = 256, K = 16) into
//              one of two 256-column TMEM accumulators;
//   warps 2-5  epilogue: each thread reads its output row from TMEM (lane =
//              row), adds the bias, applies max(0, .) when asked, and stores
//              bf16; it frees the accumulator for the tile after next.
// CTAs are persistent and take tiles round-robin.
#pragma once

#include <cuda.h>

#include "tc.cuh"

namespace lsh {

constexpr int kGmBM = 128, kGmBN = 256, kGmBK = 64, kGmStages = 4;
constexpr int kGmThreads = 192;
constexpr int kGmABytes = kGmBM * kGmBK * 2;  // 16 KB
constexpr int kGmBBytes = kGmBN * kGmBK * 2;  // 32 KB

struct GemmArgs {
  int M, N, K;       // M % 128 == 0, N % 256 == 0, K % 64 == 0
  int a_row0;        // first row of A inside its tensor map
  const __nv_bfloat16* bias;  // [N]
  __nv_bfloat16* C;  // row-major, ldc elements per row
  int ldc;
  int relu;
  long long wait_limit;
};

struct GemmSmem {
  uint64_t full[kGmStages], empty[kGmStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ inline size_t gemm_tc_smem_bytes() {
  return 1024 + (size_t)kGmStages * (kGmABytes + kGmBBytes) + sizeof(GemmSmem);
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc::smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// 2-D tiled TMA load of the box at (x = inner coordinate, y = row) into
// shared memory, completing on `bar` with its byte count.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(tc::smem_u32(bar))
      : "memory");
}

// Waits for a phase unless the CTA aborted; false on abort or timeout.
__device__ __forceinline__ bool gm_wait(uint64_t* bar, uint32_t parity, int* abort,
                                        long long limit) {
  const long long t0 = clock64();
  while (!tc::mbar_test(bar, parity)) {
    if (*(volatile int*)abort) return false;
    if (clock64() - t0 > limit) {
      record_status(tc::kErrTimeout);
      *(volatile int*)abort = 1;
      return false;
    }
  }
  return true;
}

__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a,
                   const __grid_constant__ CUtensorMap map_b, GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_a = sm;
  uint8_t* stage_b = sm + kGmStages * kGmABytes;
  GemmSmem& S = *reinterpret_cast<GemmSmem*>(stage_b + kGmStages * kGmBBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long limit = g.wait_limit;

  if (tid == 0) {
    for (int s = 0; s < kGmStages; ++s) {
      tc::mbar_init(&S.full[s], 1);
      tc::mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&S.acc_full[b], 1);
      tc::mbar_init(&S.acc_empty[b], 128);
    }
    tc::mbar_init(&S.mma_done, 1);
    tc::mbar_init_fence();
    S.abort = 0;
  }
  if (warp == 1) {
    tc::tmem_alloc(&S.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  const int n_n = g.N / kGmBN;
  const int n_tiles = (g.M / kGmBM) * n_n;
  const int n_k = g.K / kGmBK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
      uint32_t q = 0;  // k-steps issued
      for (int t = blockIdx.x; t < n_tiles && !*(volatile int*)&S.abort; t += gridDim.x) {
        const int m0 = (t / n_n) * kGmBM, n0 = (t % n_n) * kGmBN;
        for (int ks = 0; ks < n_k; ++ks, ++q) {
          const int s = q % kGmStages;
          if (!gm_wait(&S.empty[s], ((q / kGmStages) & 1u) ^ 1u, &S.abort, limit)) break;
          mbar_expect_tx(&S.full[s], kGmABytes + kGmBBytes);
          tma_load_2d(tc::smem_u32(stage_a + s * kGmABytes), &map_a, ks * kGmBK, g.a_row0 + m0,
                      &S.full[s]);
          tma_load_2d(tc::smem_u32(stage_b + s * kGmBBytes), &map_b, ks * kGmBK, n0, &S.full[s]);
        }
      }
      // every load issued has landed before the CTA leaves
      const uint32_t first = q > (uint32_t)kGmStages ? q - kGmStages : 0;
      for (uint32_t p = first; p < q; ++p) {
        const long long t0 = clock64();
        while (!tc::mbar_test(&S.full[p % kGmStages], (p / kGmStages) & 1u)) {
          if (clock64() - t0 > limit) {
            record_status(tc::kErrTimeout);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(kGmBM, kGmBN, 0, 0);
      uint32_t q = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++i) {
        const int b = i & 1;
        if (!gm_wait(&S.acc_empty[b], ((i >> 1) & 1u) ^ 1u, &S.abort, limit)) break;
        tc::fence_after_sync();
        const uint32_t d = tmem + b * 256;
        for (int ks = 0; ks < n_k; ++ks, ++q) {
          const int s = q % kGmStages;
          if (!gm_wait(&S.full[s], (q / kGmStages) & 1u, &S.abort, limit)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t sa = tc::smem_u32(stage_a + s * kGmABytes);
          const uint32_t sb = tc::smem_u32(stage_b + s * kGmBBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(d, tc::sdesc_sw128(sa + kk * 32, 16, 1024),
                         tc::sdesc_sw128(sb + kk * 32, 16, 1024), idesc, (ks | kk) != 0);
          tc::mma_commit(&S.empty[s]);  // the stage is free once these MMAs are done
        }
        if (ok) tc::mma_commit(&S.acc_full[b]);
      }
      // every MMA issued has finished before tensor memory is freed
      tc::mma_commit(&S.mma_done);
      const long long t0 = clock64();
      while (!tc::mbar_test(&S.mma_done, 0)) {
        if (clock64() - t0 > limit) {
          record_status(tc::kErrTimeout);
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;  // TMEM lanes 32*sub .. 32*sub+31
    const int row_in_tile = sub * 32 + lane;
    uint32_t i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      const int m0 = (t / n_n) * kGmBM, n0 = (t % n_n) * kGmBN;
      const bool okw = gm_wait(&S.acc_full[b], (i >> 1) & 1u, &S.abort, limit);
      if (!__all_sync(0xffffffffu, okw)) break;
      tc::fence_after_sync();
      const uint32_t taddr = tmem + b * 256 + ((uint32_t)(sub * 32) << 16);
      __nv_bfloat16* crow = g.C + (size_t)(m0 + row_in_tile) * g.ldc + n0;
#pragma unroll 1
      for (int c = 0; c < kGmBN / 32; ++c) {
        float v[32];
        tc::tmem_ld32(taddr + 32 * c, v);
        tc::tmem_ld_wait();
        tc::tmem_pin<32>(v);
        if (c == kGmBN / 32 - 1) {  // the accumulator is read: free it
          tc::fence_before_sync();
          tc::mbar_arrive(&S.acc_empty[b]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float bias[8], o[8];
          load8(g.bias + n0 + 32 * c + 8 * q, bias);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x = v[8 * q + e] + bias[e];
            o[e] = g.relu ? fmaxf(x, 0.f) : x;
          }
          store8(crow + 32 * c + 8 * q, o);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace lsh
