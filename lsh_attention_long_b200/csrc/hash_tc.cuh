// Angular LSH hash on the 5th-generation tensor cores (bf16, d = 64).
//
// "Reformer explainer" (akshathtiwari.co.in/blog/reformer): a token's bucket
// is the angular sector it lands in after a random rotation.  With R_r of
// shape [d, nb/2], the sectors are the directions +R_r[:, j] and -R_r[:, j],
// and the bucket is the first index of the maximum of [q.R_r ; -q.R_r].
//
// The projection is a GEMM: P[tokens, R*nb/2] = Q[tokens, 64] x [R_0 | R_1 | ..].
// bf16 x bf16 products are exact in fp32, so only the fp32 accumulation order
// differs from an exact computation.  tcgen05.mma (M = 128 tokens, N <= 256
// rotation columns, K = 64) accumulates into tensor memory; two epilogue
// warpgroups read each token's row (one TMEM lane per thread, each warpgroup
// one 128-column half of the N-tile) and keep the signed argmax.
//
// Signed argmax, exactly as defined: the maximum of [p ; -p] is max_j |p_j|;
// among the entries reaching it the lowest index of the concatenation wins,
// i.e. the smallest "bucket candidate" b_j = j (p_j >= 0) or j + nb/2
// (p_j < 0).  Pass A takes max |p| per 32 columns with one FMNMX per value
// and parks the chunk holding the running maximum in shared memory; pass B
// scans that chunk for the index.  Exactly tied chunk maxima take a slow path
// that scans every candidate.
//
// Work split: CTAs are grouped by rounds; a group keeps its rounds' rotation
// columns resident in shared memory (transposed to K-major, 128B-swizzled,
// <= 128 KB) and streams 128-token Q tiles (cp.async, double-buffered).  Two
// TMEM buffers of 256 columns let the MMA of one N-tile run while the
// epilogue of the previous one reads its buffer.
#pragma once

#include "tc.cuh"

namespace lsh {

constexpr int kHashTcRotBytes = 128 * 1024;
constexpr int kHashTcThreads = 256;  // two epilogue warpgroups

struct HashTcArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* rot;
  uint32_t* keys;
  int32_t* buckets;
  int n_tok, L, half, R;
  int rounds_per_group, n_groups, ctas_per_group, n_mtiles;
};

__host__ __device__ inline size_t hash_tc_smem_bytes(int rounds_per_group, int half) {
  // alignment slack, rotation columns, two Q tiles, one 128-byte slot per
  // thread, the cross-warpgroup hand-off; at least 120 KB so that one CTA
  // (holding all 512 TMEM columns) runs per SM
  const size_t need = 1024 + (size_t)rounds_per_group * half * 128 + 2 * 16384 +
                      kHashTcThreads * 128 + 128 * 8;
  return need > 120 * 1024 ? need : 120 * 1024;
}

// Exact (max |p|, bucket) over `len` columns starting at TMEM address `ta`
// whose first column is column `jbase` of its round.
//
// Pass A: per CW columns, max |p| (one FMNMX per value); a chunk that raises
// the running maximum is copied to this thread's 128-byte slot in shared
// memory (16-byte pieces, swizzled by thread).  Pass B: the slot holds the
// chunk of the maximum; an exact scan there gives the lowest bucket
// candidate.  Chunks whose maxima tie exactly send the warp through a slow
// exact scan of every chunk.
template <int CW>
__device__ __forceinline__ void hash_segment(uint32_t ta, int len, int jbase, int half,
                                             uint8_t* slot, int sw, float& best_out,
                                             int& bkt_out) {
  float v[CW];
  float best = -1.f;
  int bc = -1;
  bool tie = false;
  for (int cc = 0; cc < len; cc += CW) {
    if (CW == 32) tc::tmem_ld32(ta + cc, v); else tc::tmem_ld16(ta + cc, v);
    tc::tmem_ld_wait();
    float m0 = fabsf(v[0]), m1 = fabsf(v[1]);
#pragma unroll
    for (int j = 2; j < CW; j += 2) {
      m0 = fmaxf(m0, fabsf(v[j]));
      m1 = fmaxf(m1, fabsf(v[j + 1]));
    }
    const float m = fmaxf(m0, m1);
    if (m > best) {
      best = m;
      bc = cc;
      tie = false;
#pragma unroll
      for (int q = 0; q < CW / 4; ++q)
        *reinterpret_cast<float4*>(slot + ((q ^ sw) << 4)) =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else if (m == best) {
      tie = true;
    }
  }
  int bkt = jbase;
  if (__any_sync(0xffffffffu, tie)) {
    // exact scan of every chunk for the lanes with a tie (warp-uniform loads)
    int b_all = 0x7fffffff;
    for (int cc = 0; cc < len; cc += CW) {
      if (CW == 32) tc::tmem_ld32(ta + cc, v); else tc::tmem_ld16(ta + cc, v);
      tc::tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int b = jbase + cc + j + (v[j] < 0.f ? half : 0);
        if (fabsf(v[j]) == best && b < b_all) b_all = b;
      }
    }
    if (tie) bkt = b_all;
  }
  if (!tie && bc >= 0) {
#pragma unroll
    for (int q = 0; q < CW / 4; ++q) {
      const float4 f = *reinterpret_cast<const float4*>(slot + ((q ^ sw) << 4));
      v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
    int b_min = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < CW; ++j) {
      const int b = j + (v[j] < 0.f ? half : 0);
      if (fabsf(v[j]) == best && b < b_min) b_min = b;
    }
    bkt = jbase + bc + b_min;  // b_min already carries + nb/2 for a negative maximum
  }
  best_out = best;
  bkt_out = bkt;
}

template <int CW>
__global__ void __launch_bounds__(kHashTcThreads, 1) hash_tc_kernel(HashTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tmem_base_s;
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tid = threadIdx.x, warp = tid >> 5;

  const int g = blockIdx.x % a.n_groups;
  const int c = blockIdx.x / a.n_groups;
  const int r0 = g * a.rounds_per_group;
  const int nr = min(a.rounds_per_group, a.R - r0);
  const int cols = nr * a.half;
  const int T = (cols + 255) / 256;  // N-tiles of <= 256 columns
  uint8_t* rot_s = sm;
  uint8_t* q_s = sm + (size_t)a.rounds_per_group * a.half * 128;
  uint8_t* slot = q_s + 2 * 16384 + threadIdx.x * 128;
  const int sw = threadIdx.x & 7;
  // warpgroup wg reads columns [128 wg, 128 wg + 128) of each N-tile for the
  // token in TMEM lane `row`; for rounds wider than 128 columns the two
  // halves meet here at the round's end
  float* comb_best = reinterpret_cast<float*>(q_s + 2 * 16384 + kHashTcThreads * 128);
  int* comb_bkt = reinterpret_cast<int*>(comb_best + 128);
  const int wg = threadIdx.x >> 7, row = threadIdx.x & 127;

  if (warp == 0) {
    tc::tmem_alloc(&tmem_base_s, 512);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(&bars[0], 1);
    tc::mbar_init(&bars[1], 1);
    tc::mbar_init_fence();
  }
  // Rotation columns of this group, transposed: smem row j holds the 64
  // values of column j (round r0 + j / half), 128B-swizzled.
  for (int row = tid; row < cols; row += blockDim.x) {
    const __nv_bfloat16* src = a.rot + (size_t)(r0 + row / a.half) * 64 * a.half + row % a.half;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = __bfloat16_as_ushort(src[(size_t)(ch * 8 + 2 * e) * a.half]);
        const uint32_t hi = __bfloat16_as_ushort(src[(size_t)(ch * 8 + 2 * e + 1) * a.half]);
        w[e] = lo | (hi << 16);
      }
      *reinterpret_cast<uint4*>(rot_s + tc::sw128_offset(row, ch)) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
  }

  const int n_items = (c < a.n_mtiles) ? (a.n_mtiles - c + a.ctas_per_group - 1) / a.ctas_per_group : 0;
  auto load_q = [&](int k) {  // Q rows of this CTA's k-th token tile -> buffer k & 1
    const int tok0 = (c + k * a.ctas_per_group) * 128;
    uint8_t* dst = q_s + (k & 1) * 16384;
    for (int e = tid; e < 128 * 8; e += blockDim.x) {
      const int row = e >> 3, ch = e & 7;
      const int tok = tok0 + row;
      if (tok < a.n_tok)
        tc::cp_async16(tc::smem_u32(dst + tc::sw128_offset(row, ch)),
                       a.Q + (size_t)tok * 64 + ch * 8);
      else
        *reinterpret_cast<uint4*>(dst + tc::sw128_offset(row, ch)) = make_uint4(0, 0, 0, 0);
    }
    tc::cp_async_commit();
  };
  if (n_items > 0) load_q(0);
  if (n_items > 1) load_q(1);

  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);

  float rbest = -1.f;
  int rbkt = 0;
  const int n_jobs = n_items * T;
  const int seg_len = min(a.half, 128);
  for (int n = 0; n <= n_jobs; ++n) {
    if (n < n_jobs) {
      const int k = n / T, t = n % T;
      if (t == 0) {  // this tile's Q rows must have landed
        // only at the first tile is a later tile (k = 1) already in flight
        if (k == 0 && n_items > 1) tc::cp_async_wait<1>(); else tc::cp_async_wait<0>();
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
      }
      if (tid == 0) {
        tc::fence_after_sync();  // the epilogue that read this buffer synced before
        const int nt = min(256, cols - t * 256);
        const uint32_t idesc = tc::idesc_bf16(128, nt, 0, 0);
        const uint32_t qa = tc::smem_u32(q_s + (k & 1) * 16384);
        const uint32_t ra = tc::smem_u32(rot_s + (size_t)t * 256 * 128);
        const uint32_t d = tmem + (n & 1) * 256;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::mma_bf16(d, tc::sdesc_sw128(qa + kk * 32, 16, 1024),
                       tc::sdesc_sw128(ra + kk * 32, 16, 1024), idesc, kk > 0);
        tc::mma_commit(&bars[n & 1]);
      }
    }
    if (n > 0) {  // epilogue of job m = n - 1
      const int m = n - 1;
      const int k = m / T, t = m % T;
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars[m & 1], (m >> 1) & 1));
      tc::fence_after_sync();
      const int tok = (c + k * a.ctas_per_group) * 128 + row;
      const int nt = min(256, cols - t * 256);
      if (ok) {
        for (int s0 = wg * 128; s0 < min(nt, wg * 128 + 128); s0 += seg_len) {
          const int gcol = t * 256 + s0;
          const int rl = gcol / a.half, jbase = gcol % a.half;
          // a round starts: at its first column, or (rounds wider than 128
          // columns) at this warpgroup's first columns of the round's first tile
          if (jbase == 0 || (s0 == wg * 128 && (t * 256) % a.half == 0)) {
            rbest = -1.f;
            rbkt = 0;
          }
          float sb;
          int sk;
          hash_segment<CW>(lane_base + (m & 1) * 256 + s0, seg_len, jbase, a.half, slot, sw, sb,
                           sk);
          if (sb > rbest || (sb == rbest && sk < rbkt)) { rbest = sb; rbkt = sk; }
          if (a.half <= 128 && jbase + seg_len == a.half && tok < a.n_tok) {
            const size_t o = (size_t)(r0 + rl) * a.n_tok + tok;
            a.keys[o] = (uint32_t)rbkt * (uint32_t)a.L + (uint32_t)(tok % a.L);
            if (a.buckets) a.buckets[o] = rbkt;
          }
        }
      }
      // rounds wider than 128 columns: the second warpgroup's half joins the
      // first's at the N-tile holding the round's last column
      if (a.half > 128 && ((t + 1) * 256) % a.half == 0) {
        if (wg == 1) { comb_best[row] = rbest; comb_bkt[row] = rbkt; }
        __syncthreads();
        if (wg == 0 && ok) {
          const float ob = comb_best[row];
          const int okk = comb_bkt[row];
          if (ob > rbest || (ob == rbest && okk < rbkt)) { rbest = ob; rbkt = okk; }
          const int rl = (t * 256) / a.half;
          if (tok < a.n_tok) {
            const size_t o = (size_t)(r0 + rl) * a.n_tok + tok;
            a.keys[o] = (uint32_t)rbkt * (uint32_t)a.L + (uint32_t)(tok % a.L);
            if (a.buckets) a.buckets[o] = rbkt;
          }
        }
      }
      tc::fence_before_sync();
      if (__syncthreads_or(!ok)) {
        if (tid == 0) record_status(tc::kErrTimeout);
        break;
      }
      // all MMAs of tile k are complete once its last job is consumed:
      // its Q buffer may take tile k + 2
      if (t == T - 1 && k + 2 < n_items) load_q(k + 2);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace lsh
