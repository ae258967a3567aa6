// Angular LSH hash, general kernel (any even n_buckets, f32 or bf16 input).
//
// "Reformer explainer" (akshathtiwari.co.in/blog/reformer): a vector goes to
// the bucket of the angular sector it lands in after a random rotation.  Per
// round r the rotation R_r is [d, nb/2]; the sectors are the nb directions
// +R_r[:, j] and -R_r[:, j], and the bucket is the first index of the maximum
// of [q.R_r ; -q.R_r].  The key packs bucket*L + position for the sort.
//
// This kernel is the FFMA path: one thread per (token, round), the query row
// in registers, rotation columns staged in shared memory 32 at a time and
// read as broadcasts.  It serves f32 inputs (no TF32 rounding is allowed in
// the projection) and n_buckets whose half is not a multiple of 16.
#pragma once

#include "common.cuh"

namespace lsh {

// Running state of the first-index argmax over [p ; -p].  Tracking the
// first maximum and the first minimum of p is enough: the maximum of -p is
// minus the minimum of p, and on equality the first half (+p) wins.
struct SignedArgmax {
  float maxv, minv;
  int maxi, mini;
  __device__ __forceinline__ void init() {
    maxv = -INFINITY;
    minv = INFINITY;
    maxi = 0;
    mini = 0;
  }
  __device__ __forceinline__ void push(float p, int j) {
    if (p > maxv) { maxv = p; maxi = j; }
    if (p < minv) { minv = p; mini = j; }
  }
  __device__ __forceinline__ int bucket(int half) const {
    return (maxv >= -minv) ? maxi : mini + half;
  }
};

template <typename T, int TOK>
__global__ void __launch_bounds__(TOK)
hash_simt_kernel(const T* __restrict__ Q, const T* __restrict__ rot, uint32_t* __restrict__ keys,
                 int32_t* __restrict__ buckets, int BHL, int L, int half) {
  constexpr int COLS = 32;
  __shared__ float rs[kHeadDim][COLS];
  const int r = blockIdx.y;
  const int tok = blockIdx.x * TOK + threadIdx.x;
  const bool valid = tok < BHL;

  float q[kHeadDim];
  if (valid) {
    const T* qp = Q + (size_t)tok * kHeadDim;
#pragma unroll
    for (int k = 0; k < kHeadDim; k += 8) load8(qp + k, q + k);
  }
  SignedArgmax am;
  am.init();
  const T* R = rot + (size_t)r * kHeadDim * half;
  for (int j0 = 0; j0 < half; j0 += COLS) {
    const int nc = min(COLS, half - j0);
    __syncthreads();
    for (int e = threadIdx.x; e < kHeadDim * COLS; e += TOK) {
      const int k = e / COLS, j = e % COLS;
      rs[k][j] = (j < nc) ? to_f32(R[(size_t)k * half + j0 + j]) : 0.f;
    }
    __syncthreads();
    if (valid) {
      for (int j = 0; j < nc; ++j) {
        float p = 0.f;
#pragma unroll
        for (int k = 0; k < kHeadDim; ++k) p = fmaf(q[k], rs[k][j], p);
        am.push(p, j0 + j);
      }
    }
  }
  if (valid) {
    const int bucket = half > 0 ? am.bucket(half) : 0;
    const int pos = tok % L;
    const size_t o = (size_t)r * BHL + tok;
    keys[o] = (uint32_t)bucket * (uint32_t)L + (uint32_t)pos;
    if (buckets) buckets[o] = bucket;
  }
}

}  // namespace lsh
