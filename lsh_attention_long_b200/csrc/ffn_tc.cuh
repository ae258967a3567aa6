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
//   C[M, N] = epilogue(A[M, K] . B[N, K]^T)
// with A and B bf16, each stored either K-major (row-major [M or N][K]) or
// MN-major (row-major [K][M or N]: a transposed operand read in place, as the
// backward's products need).  Epilogues: bias and optional max(0, .) to bf16;
// a zero mask from a bf16 matrix (the derivative of max(0, .)) to bf16; fp32
// addition of a residual matrix; fp32 atomic accumulation (weight
// gradients, with K split over CTAs).  Tiles of 128 x 256 outputs, K in
// steps of 64.  Warp roles (192 threads):
//   warp 0     one thread loads A and B tiles with TMA (tensor maps, 128-byte
//              swizzle) into a ring of four stages (full/empty mbarriers with
//              transaction counts);
//   warp 1     one thread issues tcgen05.mma (M = 128, N = 256, K = 16) into
//              one of two 256-column TMEM accumulators;
//   warps 2-5  epilogue: each thread reads its output row from TMEM (lane =
//              row) and writes it through the epilogue; it frees the
//              accumulator for the work unit after next.
// CTAs are persistent and take work units (an output tile and a range of K)
// round-robin.
#pragma once

#include <cuda.h>

#include "tc.cuh"

namespace lsh {

constexpr int kGmBM = 128, kGmBN = 256, kGmBK = 64, kGmStages = 4;
constexpr int kGmThreads = 192;
constexpr int kGmABytes = kGmBM * kGmBK * 2;  // 16 KB
constexpr int kGmBBytes = kGmBN * kGmBK * 2;  // 32 KB

enum GemmEpi { kEpiBiasAct = 0, kEpiMask = 1, kEpiAddF32 = 2, kEpiAtomicF32 = 3 };

struct GemmArgs {
  int M, N, K;       // M % 128 == 0, N % 256 == 0, K % 64 == 0
  int a_mn, b_mn;    // operand stored MN-major ([K][M], [K][N]) rather than K-major
  int a_row0, b_row0;  // offset added to each operand's row (outer) coordinate
  int k_splits;      // K ranges per output tile (kEpiAtomicF32 only; else 1)
  int epi;           // GemmEpi
  const __nv_bfloat16* bias;  // kEpiBiasAct: [N]
  int relu;                   // kEpiBiasAct: max(0, .)
  const __nv_bfloat16* mask;  // kEpiMask: output zero where mask <= 0; [M][ldm]
  int ldm;
  __nv_bfloat16* C;  // bf16 output, ldc elements per row
  int ldc;
  float* C32;        // kEpiAddF32 (C32 = R + acc) and kEpiAtomicF32 (C32 += acc)
  int ldc32;
  const float* R;    // kEpiAddF32: [M][ldr], or NULL (C32 = acc)
  int ldr;
  long long wait_limit;
  // 1: the operands this launch loads are not written by the previous grid
  // in the stream (only its stores must follow that grid), so loads and MMAs
  // start at once and the epilogue waits; 0: every global access waits
  int late_wait;
};

constexpr int kGmStageOutBytes = 4 * 32 * 128;  // per epilogue warp: 32 rows of 128 B

struct GemmSmem {
  float bias[kGmBN];  // the output tile's bias columns (kEpiBiasAct)
  uint64_t full[kGmStages], empty[kGmStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ inline size_t gemm_tc_smem_bytes() {
  return 1024 + (size_t)kGmStages * (kGmABytes + kGmBBytes) + kGmStageOutBytes +
         sizeof(GemmSmem);
}

// OR of pred over the 128 epilogue threads (named barrier 2).
__device__ __forceinline__ bool epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
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
  uint8_t* stage_out = stage_b + kGmStages * kGmBBytes;
  GemmSmem& S = *reinterpret_cast<GemmSmem*>(stage_out + kGmStageOutBytes);
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
  // Launched as a programmatic dependent of the previous grid in the stream,
  // this CTA may have got here while that grid still runs: global accesses
  // wait for it to complete and for its writes to be visible (all of them,
  // or with late_wait only the epilogue's).  Then the next grid may start its
  // own set-up (it can only take SMs this grid has left: each CTA holds most
  // of an SM's shared memory).
  if (!g.late_wait) grid_dep_wait();
  grid_dep_launch();
  const uint32_t tmem = S.tmem_base;
  const int n_n = g.N / kGmBN;
  const int n_units = (g.M / kGmBM) * n_n * g.k_splits;
  const int n_k = g.K / kGmBK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
      uint32_t q = 0;  // k-steps issued
      for (int u = blockIdx.x; u < n_units && !*(volatile int*)&S.abort; u += gridDim.x) {
        const int t = u / g.k_splits, sp = u % g.k_splits;
        const int m0 = (t / n_n) * kGmBM, n0 = (t % n_n) * kGmBN;
        const int k_lo = sp * n_k / g.k_splits, k_hi = (sp + 1) * n_k / g.k_splits;
        for (int ks = k_lo; ks < k_hi; ++ks, ++q) {
          const int s = q % kGmStages;
          if (!gm_wait(&S.empty[s], ((q / kGmStages) & 1u) ^ 1u, &S.abort, limit)) break;
          tc::mbar_expect_tx(&S.full[s], kGmABytes + kGmBBytes);
          const uint32_t sa = tc::smem_u32(stage_a + s * kGmABytes);
          const uint32_t sb = tc::smem_u32(stage_b + s * kGmBBytes);
          if (!g.a_mn) {  // one box: 64 K x 128 rows
            tc::tma_load_2d(sa, &map_a, ks * kGmBK, g.a_row0 + m0, &S.full[s]);
          } else {        // two boxes: 64 M x 64 K rows each
            for (int h = 0; h < kGmBM / 64; ++h)
              tc::tma_load_2d(sa + h * 8192, &map_a, m0 + 64 * h, g.a_row0 + ks * kGmBK, &S.full[s]);
          }
          if (!g.b_mn) {
            tc::tma_load_2d(sb, &map_b, ks * kGmBK, g.b_row0 + n0, &S.full[s]);
          } else {
            for (int h = 0; h < kGmBN / 64; ++h)
              tc::tma_load_2d(sb + h * 8192, &map_b, n0 + 64 * h, g.b_row0 + ks * kGmBK, &S.full[s]);
          }
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
      const uint32_t idesc = tc::idesc_bf16(kGmBM, kGmBN, g.a_mn, g.b_mn);
      uint32_t q = 0, i = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++i) {
        const int sp = u % g.k_splits;
        const int k_lo = sp * n_k / g.k_splits, k_hi = (sp + 1) * n_k / g.k_splits;
        const int b = i & 1;
        if (!gm_wait(&S.acc_empty[b], ((i >> 1) & 1u) ^ 1u, &S.abort, limit)) break;
        tc::fence_after_sync();
        const uint32_t d = tmem + b * 256;
        for (int ks = k_lo; ks < k_hi; ++ks, ++q) {
          const int s = q % kGmStages;
          if (!gm_wait(&S.full[s], (q / kGmStages) & 1u, &S.abort, limit)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t sa = tc::smem_u32(stage_a + s * kGmABytes);
          const uint32_t sb = tc::smem_u32(stage_b + s * kGmBBytes);
          // K-major: 16 K = 32 bytes along the row; MN-major: 16 K rows of
          // 128 bytes, 64-element MN blocks 8 KB apart.  The address field
          // counts 16-byte units: a K step adds 2 (K-major) or 128 (MN-major).
          const uint64_t da0 = g.a_mn ? tc::sdesc_sw128(sa, 8192, 1024) : tc::sdesc_sw128(sa, 16, 1024);
          const uint64_t db0 = g.b_mn ? tc::sdesc_sw128(sb, 8192, 1024) : tc::sdesc_sw128(sb, 16, 1024);
          const uint32_t sta = g.a_mn ? 128u : 2u, stb = g.b_mn ? 128u : 2u;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(d, da0 + kk * sta, db0 + kk * stb, idesc, (ks > k_lo || kk > 0) ? 1u : 0u);
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
    if (g.late_wait) grid_dep_wait();
    // Each thread owns one output row (its TMEM lane) and works 32 columns
    // at a time.  Per-row operands (mask, residual) are loaded before the
    // TMEM load they are combined with; the bias of the tile sits in shared
    // memory.  Results go through this warp's staging rows (16-byte pieces
    // rotated by row) and leave eight lanes per 128-byte row: bf16 rows
    // every 64 columns, fp32 rows (stores or reductions) every 32.
    const int sub = warp & 3;  // TMEM lanes 32*sub .. 32*sub+31
    const int row_in_tile = sub * 32 + lane;
    const int et = tid - 64;   // 0..127 over the epilogue warps
    uint8_t* stg = stage_out + sub * (32 * 128);
    uint8_t* my_row = stg + lane * 128;
    const bool f32_out = g.epi == kEpiAddF32 || g.epi == kEpiAtomicF32;
    uint32_t i = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++i) {
      const int t = u / g.k_splits;
      const int b = i & 1;
      const int m0 = (t / n_n) * kGmBM, n0 = (t % n_n) * kGmBN;
      if (g.epi == kEpiBiasAct) {
        asm volatile("bar.sync 1, 128;" ::: "memory");  // the last tile's bias is read
        for (int c = et; c < kGmBN; c += 128) S.bias[c] = __bfloat162float(g.bias[n0 + c]);
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      const bool okw = gm_wait(&S.acc_full[b], (i >> 1) & 1u, &S.abort, limit);
      // all four epilogue warps leave together (they share named barriers)
      if (epi_any(!okw)) break;
      tc::fence_after_sync();
      const uint32_t taddr = tmem + b * 256 + ((uint32_t)(sub * 32) << 16);
      const size_t row = (size_t)(m0 + row_in_tile);
#pragma unroll 1
      for (int c = 0; c < kGmBN / 32; ++c) {
        const int col = n0 + 32 * c;
        uint4 mk[4];
        float4 rr[8];
        if (g.epi == kEpiMask) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mk[q] = *reinterpret_cast<const uint4*>(g.mask + row * g.ldm + col + 8 * q);
        } else if (g.epi == kEpiAddF32 && g.R) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            rr[q] = *reinterpret_cast<const float4*>(g.R + row * g.ldr + col + 4 * q);
        }
        float v[32];
        tc::tmem_ld32(taddr + 32 * c, v);
        tc::tmem_ld_wait();
        tc::tmem_pin<32>(v);
        if (c == kGmBN / 32 - 1) {  // the accumulator is read: free it
          tc::fence_before_sync();
          tc::mbar_arrive(&S.acc_empty[b]);
        }
        if (g.epi == kEpiBiasAct) {
          const float* bs = S.bias + 32 * c;
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = g.relu ? fmaxf(v[e] + bs[e], 0.f) : v[e] + bs[e];
        } else if (g.epi == kEpiMask) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __nv_bfloat16* m8 = reinterpret_cast<const __nv_bfloat16*>(&mk[q]);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              v[8 * q + e] = __bfloat162float(m8[e]) > 0.f ? v[8 * q + e] : 0.f;
          }
        } else if (g.epi == kEpiAddF32 && g.R) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            v[4 * q] += rr[q].x; v[4 * q + 1] += rr[q].y;
            v[4 * q + 2] += rr[q].z; v[4 * q + 3] += rr[q].w;
          }
        }
        if (!f32_out) {
          // 32 bf16 = 64 B: pieces 4(c&1) .. 4(c&1)+3 of the staging row
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int p = 4 * (c & 1) + q;
            *reinterpret_cast<uint4*>(my_row + ((p ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                           pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
          }
          if ((c & 1) == 0) continue;
          __syncwarp();
          const int col0 = n0 + 64 * (c >> 1);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int rl = 4 * k + (lane >> 3), p = lane & 7;
            const uint4 w = *reinterpret_cast<const uint4*>(stg + rl * 128 + ((p ^ (rl & 7)) << 4));
            *reinterpret_cast<uint4*>(g.C + (size_t)(m0 + sub * 32 + rl) * g.ldc + col0 + 8 * p) = w;
          }
          __syncwarp();
        } else {
          // 32 fp32 = 128 B: the whole staging row
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(my_row + ((q ^ (lane & 7)) << 4)) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int rl = 4 * k + (lane >> 3), p = lane & 7;
            const float4 w = *reinterpret_cast<const float4*>(stg + rl * 128 + ((p ^ (rl & 7)) << 4));
            float* dst = g.C32 + (size_t)(m0 + sub * 32 + rl) * g.ldc32 + col + 4 * p;
            if (g.epi == kEpiAddF32)
              *reinterpret_cast<float4*>(dst) = w;
            else
              asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(w.x),
                           "f"(w.y), "f"(w.z), "f"(w.w)
                           : "memory");
          }
          __syncwarp();
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

// Column sums of a bf16 matrix [rows][cols] added into fp32 out[cols] (bias
// gradients): thread x of block (y) sums its column over a slab of rows.
__global__ void colsum_add_kernel(const __nv_bfloat16* __restrict__ a, int rows, int cols,
                                  int rows_per_block, float* __restrict__ out) {
  grid_dep_wait();
  grid_dep_launch();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int r0 = blockIdx.y * rows_per_block;
  const int r1 = min(rows, r0 + rows_per_block);
  float s = 0.f;
  for (int r = r0; r < r1; ++r) s += __bfloat162float(a[(size_t)r * cols + c]);
  atomicAdd(out + c, s);
}

}  // namespace lsh
