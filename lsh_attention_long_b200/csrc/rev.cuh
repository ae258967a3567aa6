// Element-wise steps of the reversible residual block around LSH attention.
//
// The Reformer abstract (codewithpapers.app listing) and the explainer
// (akshathtiwari.co.in/blog/reformer) replace standard residuals with
// reversible ones (RevNet): a block maps (X1, X2) to
//   Y1 = X1 + F(X2),   Y2 = X2 + G(Y1),
// and its inputs are recomputed from its outputs in the backward pass
// (X2 = Y2 - G(Y1), X1 = Y1 - F(X2)) instead of being stored.  Here F is LSH
// attention with each token's features as its query (= key) and value, and
// G the chunked feed-forward.  The residual stream is fp32, token-major
// [B, L, H*d]; the sublayers take bf16 inputs, the attention head-major
// [B, H, L, d].  These kernels move between the layouts and do the residual
// additions, 8 elements (one 16-byte piece of bf16) per thread.
#pragma once

#include "common.cuh"

namespace lsh {

struct RevDims {
  int B, H, L;  // d = 64, D = H * 64
};

// Token-major element index of head-major element (b, h, l, k8 .. k8+7).
__device__ __forceinline__ size_t rev_token_index(const RevDims& r, size_t g8) {
  const size_t per_head = (size_t)r.L * 8;  // 8-wide pieces per (b, h)
  const size_t bh = g8 / per_head;
  const size_t rem = g8 - bh * per_head;
  const size_t l = rem >> 3, k = (rem & 7) * 8;
  const size_t b = bh / r.H, h = bh - b * r.H;
  return ((b * r.L + l) * r.H + h) * kHeadDim + k;
}

// heads[b, h, l, :] = bf16(x[b, l, h, :])
__global__ void rev_to_heads_kernel(RevDims r, const float* __restrict__ x,
                                    __nv_bfloat16* __restrict__ heads) {
  const size_t g8 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g8 >= (size_t)r.B * r.H * r.L * 8) return;
  float v[8];
  load8(x + rev_token_index(r, g8), v);
  store8(heads + g8 * 8, v);
}

// out[b, l, h, :] = a[b, l, h, :] + sign * o[b, h, l, :] (fp32), and its bf16
// copy (token-major) when out16 is given
__global__ void rev_residual_heads_kernel(RevDims r, const float* __restrict__ a,
                                          const __nv_bfloat16* __restrict__ o, float sign,
                                          float* __restrict__ out,
                                          __nv_bfloat16* __restrict__ out16) {
  const size_t g8 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g8 >= (size_t)r.B * r.H * r.L * 8) return;
  const size_t t = rev_token_index(r, g8);
  float x[8], y[8];
  load8(a + t, x);
  load8(o + g8 * 8, y);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = fmaf(sign, y[e], x[e]);
  store8(out + t, x);
  if (out16) store8(out16 + t, x);
}

// out[i] = a[i] + sign * b[i] (fp32 + bf16, the same layout), and its bf16
// copy when out16 is given; b == NULL copies (bf16 rounding of a)
__global__ void rev_residual_kernel(size_t n8, const float* __restrict__ a,
                                    const __nv_bfloat16* __restrict__ b, float sign,
                                    float* __restrict__ out, __nv_bfloat16* __restrict__ out16) {
  const size_t g8 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g8 >= n8) return;
  float x[8];
  load8(a + g8 * 8, x);
  if (b) {
    float y[8];
    load8(b + g8 * 8, y);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = fmaf(sign, y[e], x[e]);
  }
  if (out) store8(out + g8 * 8, x);
  if (out16) store8(out16 + g8 * 8, x);
}

// dx2[b, l, h, :] = dy2[b, l, h, :] + dq[b, h, l, :] + dv[b, h, l, :]: the
// attention's input is both its query and its value
__global__ void rev_grad_x2_kernel(RevDims r, const float* __restrict__ dy2,
                                   const float* __restrict__ dq, const float* __restrict__ dv,
                                   float* __restrict__ dx2) {
  const size_t g8 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g8 >= (size_t)r.B * r.H * r.L * 8) return;
  const size_t t = rev_token_index(r, g8);
  float x[8], q[8], v[8];
  load8(dy2 + t, x);
  load8(dq + g8 * 8, q);
  load8(dv + g8 * 8, v);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] += q[e] + v[e];
  store8(dx2 + t, x);
}

}  // namespace lsh
