// Per-row stable counting sort of packed LSH keys.
//
// "Reformer explainer" (akshathtiwari.co.in/blog/reformer): after hashing,
// tokens are sorted by bucket.  Within every (round, batch, head) row the
// order is (bucket, position); since a row's keys arrive in position order,
// a stable counting sort on the bucket produces it.
//
// A row is sorted by one thread-block cluster of P CTAs (P = 1 or 2), CTA c
// taking the c-th part of the row.  Each warp owns a contiguous segment and a
// private histogram in shared memory:
//   pass 1  every key's bucket (key / L by a multiply-high with a
//           precomputed constant) is counted into the warp's histogram with a
//           shared-memory atomic (counts do not depend on order) and, when
//           the CTA's part fits, kept in shared memory as 16 bits;
//   scan    per-bucket totals of every CTA of the cluster meet through
//           distributed shared memory; bucket-major, CTA-minor, warp-minor
//           exclusive prefix sums give each warp's first output slot per
//           bucket;
//   pass 2  the same walk again over the kept bucket ids (or the keys); a
//           token's slot is its warp's offset for the bucket plus its rank
//           among equal-bucket lanes of lower index (__match_any_sync).
// CTAs, warps, steps and lanes visit positions in increasing order, so equal
// buckets keep position order: the sort is stable.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace lsh {

constexpr uint32_t kNoBucket = 0xffffffffu;

// floor(key / L) for key < 2^31 as umulhi(key, m) >> sh, with
// m = ceil(2^(31 + l) / L), l = ceil(log2 L), sh = l - 1 (the round-up
// method of division by an invariant integer); L == 1 is the identity.
struct DivL {
  uint32_t m;
  int sh;  // -1: L == 1
};
__host__ inline DivL make_divl(uint32_t L) {
  DivL d;
  int l = 0;
  while ((1ull << l) < L) ++l;
  if (l == 0) { d.m = 0; d.sh = -1; return d; }
  const unsigned __int128 num = (unsigned __int128)1 << (31 + l);
  d.m = (uint32_t)((num + L - 1) / L);
  d.sh = l - 1;
  return d;
}
__device__ __forceinline__ uint32_t div_l(uint32_t key, DivL d) {
  return d.sh < 0 ? key : __umulhi(key, d.m) >> d.sh;
}

// Bucket of the key at position t, or kNoBucket (and bad) when the key is
// not bucket * L + t with bucket < nb.
__device__ __forceinline__ uint32_t checked_bucket(uint32_t key, int t, int L, int nb, DivL dl,
                                                   bool& bad) {
  const uint32_t b = div_l(key, dl);
  if (b >= (uint32_t)nb || key - b * (uint32_t)L != (uint32_t)t) {
    bad = true;
    return kNoBucket;
  }
  return b;
}

__global__ void __launch_bounds__(1024)
sort_rows_kernel(const uint32_t* __restrict__ keys, int32_t* __restrict__ perm, int L, int nb,
                 DivL dl, int cache_ids) {
  namespace cg = cooperative_groups;
  extern __shared__ uint32_t cnt[];  // [nwarps][nb], (P > 1) this CTA's totals [nb], ids
  __shared__ uint32_t warp_sums[32];
  cg::cluster_group cluster = cg::this_cluster();
  const int P = (int)cluster.num_blocks(), crank = (int)cluster.block_rank();
  const int nwarps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = blockIdx.x / P;
  const uint32_t* k = keys + row * L;
  int32_t* out = perm + row * L;
  uint32_t* tot = cnt + (size_t)nwarps * nb;
  uint16_t* ids = reinterpret_cast<uint16_t*>(tot + (P > 1 ? nb : 0));  // this CTA's bucket ids

  for (int e = threadIdx.x; e < nwarps * nb; e += blockDim.x) cnt[e] = 0;
  __syncthreads();

  // this CTA's part of the row, then this warp's segment of it
  const int part = (((L + P - 1) / P) + 31) & ~31;
  const int cbeg = min(L, crank * part), cend = min(L, cbeg + part);
  const int seg = ((((cend - cbeg) + nwarps - 1) / nwarps) + 31) & ~31;
  const int begin = min(cend, cbeg + w * seg), end = min(cend, begin + seg);
  uint32_t* my = cnt + (size_t)w * nb;
  bool bad = false;

  // pass 1: per-warp histograms (counts do not depend on order: shared-
  // memory atomics), bucket ids kept for pass 2 when they fit; each lane
  // has four keys in flight before it counts them
  for (int base = begin; base < end; base += 128) {
    uint32_t kv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = base + 32 * j + lane;
      kv[j] = t < end ? __ldg(k + t) : 0u;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = base + 32 * j + lane;
      if (t < end) {
        const uint32_t b = checked_bucket(kv[j], t, L, nb, dl, bad);
        if (b != kNoBucket) atomicAdd(&my[b], 1u);
        if (cache_ids) ids[t - cbeg] = b != kNoBucket ? (uint16_t)b : (uint16_t)0xffffu;
      }
    }
  }
  if (bad) record_status(kErrBadKeys);
  __syncthreads();

  // this CTA's totals per bucket, visible to the cluster (a lone CTA sums
  // its histograms in place)
  if (P > 1)
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
      uint32_t s0 = 0;
      for (int ww = 0; ww < nwarps; ++ww) s0 += cnt[ww * nb + b];
      tot[b] = s0;
    }
  cluster.sync();
  auto total = [&](int c, int b) -> uint32_t {  // CTA c's tokens of bucket b
    if (P == 1) {
      uint32_t s0 = 0;
      for (int ww = 0; ww < nwarps; ++ww) s0 += cnt[ww * nb + b];
      return s0;
    }
    return cluster.map_shared_rank(tot, c)[b];
  };

  // scan: each thread owns a contiguous run of buckets; a bucket's slots
  // start after every smaller bucket of the row, then after the earlier
  // CTAs' tokens of the same bucket
  const int per = (nb + blockDim.x - 1) / blockDim.x;
  const int b0 = min(nb, threadIdx.x * per), b1 = min(nb, b0 + per);
  uint32_t local = 0;
  for (int b = b0; b < b1; ++b)
    for (int c = 0; c < P; ++c) local += total(c, b);
  uint32_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += x;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    uint32_t v = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += x;
    }
    if (lane < nwarps) warp_sums[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  uint32_t running = incl - local + (w > 0 ? warp_sums[w - 1] : 0);
  for (int b = b0; b < b1; ++b) {
    uint32_t all = 0, before = 0;
    for (int c = 0; c < P; ++c) {
      const uint32_t x = total(c, b);
      all += x;
      if (c < crank) before += x;
    }
    uint32_t r = running + before;
    for (int ww = 0; ww < nwarps; ++ww) {
      const uint32_t c = cnt[ww * nb + b];
      cnt[ww * nb + b] = r;
      r += c;
    }
    running += all;
  }
  cluster.sync();  // every CTA has read the others' totals

  // pass 2: stable scatter of positions
  for (int base = begin; base < end; base += 32) {
    const int t = base + lane;
    bool dummy = false;
    uint32_t b = kNoBucket;
    if (t < end) {
      if (cache_ids) {
        const uint32_t c = ids[t - cbeg];
        b = c == 0xffffu ? kNoBucket : c;
      } else {
        b = checked_bucket(k[t], t, L, nb, dl, dummy);
      }
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    if (b != kNoBucket) {
      const uint32_t rank = __popc(peers & ((1u << lane) - 1u));
      out[my[b] + rank] = t;
    }
    __syncwarp();
    if (b != kNoBucket && lane == __ffs(peers) - 1) my[b] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace lsh
