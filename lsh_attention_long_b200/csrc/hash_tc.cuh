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
// rotation columns, K = 64) accumulates into tensor memory; epilogue
// warpgroups read each token's row (one TMEM lane per thread) and keep the
// signed argmax.
//
// Signed argmax, exactly as defined: the maximum of [p ; -p] is max_j |p_j|;
// among the entries reaching it the lowest index of the concatenation wins,
// i.e. the smallest "bucket candidate" b_j = j (p_j >= 0) or j + nb/2
// (p_j < 0).  Each token's row is reduced in chunks of 32 columns: a tree of
// 3-input maxima gives the chunk's max |p|; the first chunk to reach the
// round's running maximum is parked in shared memory, and once per round an
// exact scan of the parked chunk gives the index.  A later chunk whose maximum
// ties the running one exactly is scanned on the spot.
//
// Work split: CTAs are grouped by rounds; a group keeps its rounds' rotation
// columns resident in shared memory (transposed to K-major, 128B-swizzled,
// <= 128 KB) and streams 128-token Q tiles.  Warp roles, synchronised only
// by mbarriers (no block-wide barrier in the steady state):
//   warp 9      loads Q tiles (one TMA copy each) into two buffers;
//   warp 8      one thread issues the MMAs of each N-tile (<= 256 columns)
//               into one of two 256-column TMEM buffers;
//   warps 0-7   two epilogue warpgroups; a whole round goes to one of them
//               (rounds alternate between the two), so rounds wider than one
//               N-tile never straddle warpgroups.
#pragma once

#include "tc.cuh"

namespace lsh {

constexpr int kHashTcRotBytes = 128 * 1024;
constexpr int kHashTcThreads = 320;  // two epilogue warpgroups, MMA warp, Q loader
constexpr int kHashBatch = 64;       // TMEM columns read per wait in the epilogue

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
  // epilogue thread; at least 120 KB so that one CTA (holding all 512 TMEM
  // columns) runs per SM
  const size_t need = 1024 + (size_t)rounds_per_group * half * 128 + 2 * 16384 + 256 * 128;
  return need > 120 * 1024 ? need : 120 * 1024;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max over N values as a tree of 3-input maxima (short dependency chains)
template <int N>
__device__ __forceinline__ float max_tree(const float* x) {
  if constexpr (N == 1) {
    return x[0];
  } else if constexpr (N == 2) {
    return fmaxf(x[0], x[1]);
  } else {
    constexpr int M = (N + 2) / 3;
    float y[M];
#pragma unroll
    for (int i = 0; i < N / 3; ++i) y[i] = max3f(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
    if constexpr (N % 3 == 1) y[M - 1] = x[N - 1];
    if constexpr (N % 3 == 2) y[M - 1] = fmaxf(x[N - 2], x[N - 1]);
    return max_tree<M>(y);
  }
}

// Running signed argmax of one token over one round, fed CW columns at a
// time.  `slot` (this thread's 128 bytes of shared memory, 16-byte pieces
// swizzled by `sw`) keeps the first chunk that reached the running maximum
// `best` and `bc` its first column; chunks arriving later whose maximum equals
// `best` exactly are resolved on the spot into `tie_cand`.
struct ArgmaxState {
  float best;
  int bc;
  int tie_cand;
  __device__ __forceinline__ void reset() {
    best = -1.f;
    bc = 0;
    tie_cand = 0x7fffffff;
  }
};

// lowest bucket candidate (column j -> j for p_j >= 0, j + nb/2 for p_j < 0)
// among the CW values of a chunk whose |p| equals m
template <int CW>
__device__ __forceinline__ int chunk_candidate(const float* v, float m, int base, int half) {
  int jp = 0x7fffffff, jn = 0x7fffffff;
#pragma unroll
  for (int j = CW - 1; j >= 0; --j) {
    if (v[j] == m) jp = j;
    if (v[j] == -m) jn = j;
  }
  return jp != 0x7fffffff ? base + jp : (jn != 0x7fffffff ? base + jn + half : 0x7fffffff);
}

template <int CW>
__device__ __forceinline__ void argmax_update(ArgmaxState& st, const float* v, int base, int half,
                                              uint8_t* slot, int sw) {
  float a[CW];
#pragma unroll
  for (int j = 0; j < CW; ++j) a[j] = fabsf(v[j]);
  const float m = max_tree<CW>(a);
  if (m > st.best) {
    st.best = m;
    st.bc = base;
    st.tie_cand = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < CW / 4; ++q)
      *reinterpret_cast<float4*>(slot + ((q ^ sw) << 4)) =
          make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else if (m == st.best) {  // exact tie with an earlier chunk: rare
    st.tie_cand = min(st.tie_cand, chunk_candidate<CW>(v, m, base, half));
  }
}

// bucket of the round: the parked chunk's lowest candidate, or a later tied one
template <int CW>
__device__ __forceinline__ int argmax_finish(const ArgmaxState& st, int half, const uint8_t* slot,
                                             int sw) {
  float v[CW];
#pragma unroll
  for (int q = 0; q < CW / 4; ++q) {
    const float4 f = *reinterpret_cast<const float4*>(slot + ((q ^ sw) << 4));
    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
  }
  return min(chunk_candidate<CW>(v, st.best, st.bc, half), st.tie_cand);
}

// Bounded mbarrier wait that also gives up once the CTA has aborted.
__device__ __forceinline__ bool hash_wait(uint64_t* bar, uint32_t parity, int* abort) {
  const long long t0 = clock64();
  while (!tc::mbar_test(bar, parity)) {
    if (*(volatile int*)abort) return false;
    if (clock64() - t0 > tc::kSpinCycles) {
      record_status(tc::kErrTimeout);
      *(volatile int*)abort = 1;
      return false;
    }
  }
  return true;
}

template <int CW>
__global__ void __launch_bounds__(kHashTcThreads, 1)
    hash_tc_kernel(const __grid_constant__ CUtensorMap map_q, HashTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // buf_full[w][b]: a job for warpgroup w landed in TMEM buffer b.  Each
  // warpgroup has its own pair, so it waits on every phase of the barriers
  // it uses (a barrier shared with jobs it skips could be two phases behind,
  // where a parity wait cannot tell the phases apart).
  __shared__ uint64_t buf_full[2][2], buf_empty[2], q_full[2], q_empty[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int g = blockIdx.x % a.n_groups;
  const int c = blockIdx.x / a.n_groups;
  const int r0 = g * a.rounds_per_group;
  const int nr = min(a.rounds_per_group, a.R - r0);
  const int cols = nr * a.half;
  const int T = (cols + 255) / 256;  // N-tiles of <= 256 columns per token tile
  uint8_t* rot_s = sm;
  uint8_t* q_s = sm + (size_t)a.rounds_per_group * a.half * 128;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&buf_full[0][b], 1);
      tc::mbar_init(&buf_full[1][b], 1);
      tc::mbar_init(&buf_empty[b], 128);
      tc::mbar_init(&q_full[b], 1);  // the TMA issuer's arrive
      tc::mbar_init(&q_empty[b], 1);
    }
    tc::mbar_init_fence();
    abort_s = 0;
  }
  if (warp == 8) {
    tc::tmem_alloc(&tmem_base_s, 512);
    tc::tmem_relinquish();
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
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;

  const int n_items = (c < a.n_mtiles) ? (a.n_mtiles - c + a.ctas_per_group - 1) / a.ctas_per_group : 0;
  const int n_jobs = n_items * T;
  // rounds alternate between the epilogue warpgroups; a round wider than one
  // N-tile keeps all of its N-tiles on one warpgroup
  const int tiles_per_round = a.half >= 256 ? a.half / 256 : 1;
  auto job_wg = [&](int n) {
    const int k = n / T, t = n % T;
    const int rr = a.half >= 256 ? t / tiles_per_round : t;
    return (k * (a.half >= 256 ? nr : T) + rr) & 1;
  };

  if (warp == 9) {
    // ------------------------------------------------------- Q tile loads
    // one TMA copy per 128-token tile (16 KB, 128B-swizzled: the MMA's
    // K-major layout); rows past the last token read as zeros
    if (lane == 0) {
      for (int k = 0; k < n_items; ++k) {
        const int b = k & 1;
        if (!hash_wait(&q_empty[b], ((k >> 1) & 1) ^ 1, &abort_s)) break;
        tc::mbar_expect_tx(&q_full[b], 16384);
        tc::tma_load_2d(tc::smem_u32(q_s + b * 16384), &map_q, 0,
                        (c + k * a.ctas_per_group) * 128, &q_full[b]);
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ------------------------------------------------------- MMA issue
    if (lane == 0) {
      for (int n = 0; n < n_jobs; ++n) {
        const int k = n / T, t = n % T, b = n & 1;
        if (t == 0 && !hash_wait(&q_full[k & 1], (k >> 1) & 1, &abort_s)) break;
        if (!hash_wait(&buf_empty[b], ((n >> 1) & 1) ^ 1, &abort_s)) break;
        tc::fence_after_sync();
        const int nt = min(256, cols - t * 256);
        const uint32_t idesc = tc::idesc_bf16(128, nt, 0, 0);
        const uint64_t dq = tc::sdesc_sw128(tc::smem_u32(q_s + (k & 1) * 16384), 16, 1024);
        const uint64_t dr = tc::sdesc_sw128(tc::smem_u32(rot_s + (size_t)t * 256 * 128), 16, 1024);
        const uint32_t d = tmem + b * 256;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K steps of 32 bytes: 2 units of the address field
          tc::mma_bf16(d, dq + 2 * kk, dr + 2 * kk, idesc, kk > 0);
        tc::mma_commit(&buf_full[job_wg(n)][b]);
        if (t == T - 1) tc::mma_commit(&q_empty[k & 1]);  // the Q buffer frees after these
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- epilogue
    const int wgi = warp >> 2, row = tid & 127;
    uint8_t* slot = q_s + 2 * 16384 + tid * 128;
    const int sw = tid & 7;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int bw = min(a.half, kHashBatch);  // columns per TMEM load batch; divides a round
    const int bw_shift = __ffs(bw) - 1, half_shift = __ffs(a.half) - 1;  // powers of two
    const int nch = bw / CW;
    ArgmaxState st;
    st.reset();
    uint32_t seen = 0;  // bit b: parity of this warpgroup's next job in buffer b
    for (int n = 0; n < n_jobs; ++n) {
      if (job_wg(n) != wgi) continue;
      const int k = n / T, t = n % T, b = n & 1;
      if (!__all_sync(0xffffffffu, hash_wait(&buf_full[wgi][b], (seen >> b) & 1u, &abort_s)))
        break;
      seen ^= 1u << b;
      tc::fence_after_sync();
      const int tok = (c + k * a.ctas_per_group) * 128 + row;
      const uint32_t pos = (uint32_t)(tok % a.L);
      const int nt = min(256, cols - t * 256);
      const int nbat = nt >> bw_shift;
      const uint32_t ta = lane_base + b * 256;
      auto load = [&](float* va, int i) {
#pragma unroll
        for (int ch = 0; ch < kHashBatch / CW; ++ch)
          if (ch < nch) {
            if (CW == 32) tc::tmem_ld32(ta + (i << bw_shift) + ch * CW, va + ch * CW);
            else tc::tmem_ld16(ta + (i << bw_shift) + ch * CW, va + ch * CW);
          }
      };
      auto process = [&](float* va, int i) {
        const int gcol = t * 256 + (i << bw_shift);
        const int rl = gcol >> half_shift, jb = gcol & (a.half - 1);
#pragma unroll
        for (int ch = 0; ch < kHashBatch / CW; ++ch)
          if (ch < nch) argmax_update<CW>(st, va + ch * CW, jb + ch * CW, a.half, slot, sw);
        if (jb + bw == a.half) {  // the round is complete
          const int bkt = argmax_finish<CW>(st, a.half, slot, sw);
          st.reset();
          if (tok < a.n_tok) {
            const size_t o = (size_t)(r0 + rl) * a.n_tok + tok;
            a.keys[o] = (uint32_t)bkt * (uint32_t)a.L + pos;
            if (a.buckets) a.buckets[o] = bkt;
          }
        }
      };
      for (int i = 0; i < nbat; ++i) {
        float va[kHashBatch];
        load(va, i);
        tc::tmem_ld_wait();
        tc::tmem_pin<kHashBatch>(va);
        process(va, i);
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&buf_empty[b]);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 8) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Four epilogue warpgroups (nb/2 = 128, 256 or 512; every N-tile 256 columns
// wide).  Each job (128 tokens x 256 columns in one of two TMEM buffers) is
// read by the two warpgroups of its buffer's pair, 128 columns each, so four
// epilogue warps share each SM sub-partition instead of two.  A round's
// columns then fall to one warpgroup (nb/2 = 128), to a pair (256) or to all
// four (512); each keeps the exact partial argmax of its columns (largest
// |p|, then its lowest bucket candidate), and the last warpgroup to finish a
// round merges the partials through shared memory: the largest |p| wins,
// equal ones go to the lowest candidate, the same first index of the maximum
// of [p ; -p] as one scan of the whole round.  Measured against the
// two-warpgroup kernel (same keys): 0.514 against 0.541 ms at 1024 buckets
// and 8 rounds, 0.039 against 0.051 ms at 256 buckets and 4 rounds.
// ---------------------------------------------------------------------------

constexpr int kHash4Threads = 576;  // four epilogue warpgroups, MMA warp, Q loader
constexpr int kHash4Batch = 32;     // TMEM columns read per wait
constexpr int kHash4Slots = 4;      // rounds whose partials may be in flight

// Per round slot and token row: the largest (|p| bits, ~candidate) pair of
// the pieces merged so far (non-negative floats order as their bits; a
// larger ~candidate is a smaller candidate), and how many pieces are in.
struct Hash4Merge {
  unsigned long long key[kHash4Slots][128];
  unsigned cnt[kHash4Slots][128];
};

__host__ __device__ inline size_t hash_tc4_smem_bytes(int rounds_per_group, int half) {
  // alignment slack, rotation columns, two Q tiles, 64 bytes of parking per
  // epilogue thread, the merge slots
  return 1024 + (size_t)rounds_per_group * half * 128 + 2 * 16384 + 512 * 64 + sizeof(Hash4Merge);
}

__global__ void __launch_bounds__(kHash4Threads, 1)
    hash_tc4_kernel(const __grid_constant__ CUtensorMap map_q, HashTcArgs a) {
  constexpr int CW = 16;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t buf_full[2], buf_empty[2], q_full[2], q_empty[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int g = blockIdx.x % a.n_groups;
  const int c = blockIdx.x / a.n_groups;
  const int r0 = g * a.rounds_per_group;
  const int nr = min(a.rounds_per_group, a.R - r0);
  const int cols = nr * a.half;
  const int T = cols / 256;  // N-tiles per token tile, all 256 wide
  uint8_t* rot_s = sm;
  uint8_t* q_s = sm + (size_t)a.rounds_per_group * a.half * 128;
  uint8_t* park = q_s + 2 * 16384;
  Hash4Merge& M = *reinterpret_cast<Hash4Merge*>(park + 512 * 64);

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&buf_full[b], 1);
      tc::mbar_init(&buf_empty[b], 256);  // both warpgroups of the buffer's pair
      tc::mbar_init(&q_full[b], 1);
      tc::mbar_init(&q_empty[b], 1);
    }
    tc::mbar_init_fence();
    abort_s = 0;
  }
  if (warp == 16) {
    tc::tmem_alloc(&tmem_base_s, 512);
    tc::tmem_relinquish();
  }
  for (int e = tid; e < kHash4Slots * 128; e += blockDim.x) {
    M.key[e / 128][e % 128] = 0ull;
    M.cnt[e / 128][e % 128] = 0u;
  }
  // rotation columns of this group, transposed: smem row j holds column j
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
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  const int n_items =
      (c < a.n_mtiles) ? (a.n_mtiles - c + a.ctas_per_group - 1) / a.ctas_per_group : 0;
  const int n_jobs = n_items * T;

  if (warp == 17) {
    // ------------------------------------------------------- Q tile loads
    if (lane == 0) {
      for (int k = 0; k < n_items; ++k) {
        const int b = k & 1;
        if (!hash_wait(&q_empty[b], ((k >> 1) & 1) ^ 1, &abort_s)) break;
        tc::mbar_expect_tx(&q_full[b], 16384);
        tc::tma_load_2d(tc::smem_u32(q_s + b * 16384), &map_q, 0,
                        (c + k * a.ctas_per_group) * 128, &q_full[b]);
      }
    }
    __syncwarp();
  } else if (warp == 16) {
    // ------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, 256, 0, 0);
      for (int n = 0; n < n_jobs; ++n) {
        const int k = n / T, t = n % T, b = n & 1;
        if (t == 0 && !hash_wait(&q_full[k & 1], (k >> 1) & 1, &abort_s)) break;
        if (!hash_wait(&buf_empty[b], ((n >> 1) & 1) ^ 1, &abort_s)) break;
        tc::fence_after_sync();
        const uint64_t dq = tc::sdesc_sw128(tc::smem_u32(q_s + (k & 1) * 16384), 16, 1024);
        const uint64_t dr = tc::sdesc_sw128(tc::smem_u32(rot_s + (size_t)t * 256 * 128), 16, 1024);
        const uint32_t d = tmem + b * 256;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K steps of 32 bytes: 2 units of the address field
          tc::mma_bf16(d, dq + 2 * kk, dr + 2 * kk, idesc, kk > 0);
        tc::mma_commit(&buf_full[b]);
        if (t == T - 1) tc::mma_commit(&q_empty[k & 1]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- epilogue
    const int w = warp >> 2, row = tid & 127;
    const int pb = w >> 1, h = w & 1;  // buffer of the pair, half of each job
    // 64-byte slots: the eight lanes of a quarter-warp take two slot bases
    // (tid & 1) and four piece rotations ((tid >> 1) & 3), so a 16-byte
    // store of piece q lands on eight distinct bank groups
    uint8_t* slot = park + tid * 64;
    const int sw = (tid >> 1) & 3;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int np = a.half / 128;           // 128-column pieces per round
    const int P = np < 4 ? np : 4;         // warpgroups that share a round
    const int half_shift = __ffs(a.half) - 1;
    uint32_t phase = 0;
    for (int n = pb; n < n_jobs; n += 2, phase ^= 1u) {
      const int k = n / T, t = n % T;
      if (!__all_sync(0xffffffffu, hash_wait(&buf_full[pb], phase, &abort_s))) break;
      tc::fence_after_sync();
      const int tok = (c + k * a.ctas_per_group) * 128 + row;
      const uint32_t pos = (uint32_t)(tok % a.L);
      const int gc0 = t * 256 + h * 128;  // first column of this piece in the group
      const int rl = gc0 >> half_shift, jb0 = gc0 & (a.half - 1);
      const uint32_t ta = lane_base + pb * 256 + h * 128;
      ArgmaxState st;
      st.reset();
#pragma unroll 1
      for (int i = 0; i < 128 / kHash4Batch; ++i) {
        float va[kHash4Batch];
        tc::tmem_ld32(ta + i * kHash4Batch, va);
        tc::tmem_ld_wait();
        tc::tmem_pin<kHash4Batch>(va);
        if (i == 128 / kHash4Batch - 1) {  // the piece is read: free the buffer half
          tc::fence_before_sync();
          tc::mbar_arrive(&buf_empty[pb]);
        }
#pragma unroll
        for (int ch = 0; ch < kHash4Batch / CW; ++ch)
          argmax_update<CW>(st, va + ch * CW, jb0 + i * kHash4Batch + ch * CW, a.half, slot, sw);
      }
      const int cand = argmax_finish<CW>(st, a.half, slot, sw);
      int bkt = cand;
      if (P > 1) {
        // merge this piece into the round's row; the last of its P pieces
        // takes the result (and clears the slot for a later round)
        const int gr = k * nr + rl, ms = gr % kHash4Slots;
        const unsigned long long mine =
            ((unsigned long long)__float_as_uint(st.best) << 32) | (uint32_t)~(uint32_t)cand;
        atomicMax(&M.key[ms][row], mine);
        __threadfence_block();
        if (atomicAdd(&M.cnt[ms][row], 1u) != (unsigned)(P - 1)) continue;
        __threadfence_block();
        const unsigned long long all = atomicExch(&M.key[ms][row], 0ull);
        M.cnt[ms][row] = 0;
        bkt = (int)~(uint32_t)(all & 0xffffffffull);
      }
      if (tok < a.n_tok) {
        const size_t o = (size_t)(r0 + rl) * a.n_tok + tok;
        a.keys[o] = (uint32_t)bkt * (uint32_t)a.L + pos;
        if (a.buckets) a.buckets[o] = bkt;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 16) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace lsh
