// Chunked shared-QK LSH attention, general kernels (f32 or bf16, chunk <= 64).
//
// "Reformer explainer" (akshathtiwari.co.in/blog/reformer): sorted tokens are
// processed in equal chunks, each attending to its bucket-mates; several
// hash rounds are unioned.  The arithmetic (steps 3-5 of the definition in
// include/lsh.h): chunk k of sorted slots attends to chunk k and chunk k-1
// (chunk 0 wraps to the last, a lone chunk sees itself once); keys are
// q/|q|, scores are scaled by 1/sqrt(d); another bucket or a later position
// (causal) scores -inf, the token itself scores -1e5; each round's output
// and logsumexp go back to original positions; rounds combine by their
// logsumexp weights.
//
// Mask test on packed keys (key = bucket*L + position): key_j lies in the
// query's bucket iff (key_j - bucket_i*L) < L as unsigned, and within a
// bucket key order is position order, so "later position" is key_j > key_i.
//
// One CTA per (row, chunk); 256 threads; four threads share a query and
// split the window's keys (scores) and the head dimension (outputs).
// These kernels serve f32 inputs and every shape the tensor-core kernels do
// not take; the forward also provides per-round partials for the parity
// tests.
#pragma once

#include "common.cuh"

namespace lsh {

struct AttnDims {
  int B, H, L, chunk, n_chunks, causal;
  int W;       // window length: 2*chunk, or chunk when the row is one chunk
  int BH;
};

__device__ __forceinline__ int window_slot(const AttnDims& a, int cur, int u) {
  if (a.n_chunks == 1) return cur * a.chunk + u;
  const int prev = (cur == 0) ? a.n_chunks - 1 : cur - 1;
  return (u < a.chunk) ? prev * a.chunk + u : cur * a.chunk + (u - a.chunk);
}

// Shared-memory carve-up of the forward kernel, in floats.
__host__ __device__ inline size_t simt_fwd_smem_bytes(int chunk, int W) {
  return sizeof(float) * ((size_t)W * 65 + (size_t)W * 64 + W + (size_t)chunk * W) +
         sizeof(uint32_t) * W + sizeof(int) * W;
}

// Gathers the window's rows: raw q (stride 65), v (stride 64), the key scale
// 1/(|q| sqrt(d)) (0 for a zero row), packed keys and original positions.
template <typename T>
__device__ __forceinline__ void load_window(const AttnDims& a, const T* Qbh, const T* Vbh,
                                            const uint32_t* krow, const int32_t* prow, int cur,
                                            float* qs, float* vs, int vstride, float* sc,
                                            uint32_t* ks, int* ps) {
  for (int u = threadIdx.x; u < a.W; u += blockDim.x) {
    int pos = prow[window_slot(a, cur, u)];
    if ((unsigned)pos >= (unsigned)a.L) {  // not a permutation of the row
      record_status(kErrBadKeys);
      pos = 0;
    }
    ps[u] = pos;
    ks[u] = krow[pos];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.W * 8; e += blockDim.x) {
    const int u = e >> 3, k = (e & 7) * 8;
    float tmp[8];
    const size_t off = (size_t)ps[u] * kHeadDim + k;
    load8(Qbh + off, tmp);
#pragma unroll
    for (int x = 0; x < 8; ++x) qs[u * 65 + k + x] = tmp[x];
    load8(Vbh + off, tmp);
#pragma unroll
    for (int x = 0; x < 8; ++x) vs[u * vstride + k + x] = tmp[x];
  }
  __syncthreads();
  for (int u = threadIdx.x; u < a.W; u += blockDim.x) {
    float ss = 0.f;
#pragma unroll 16
    for (int k = 0; k < kHeadDim; ++k) ss = fmaf(qs[u * 65 + k], qs[u * 65 + k], ss);
    const float n = sqrtf(ss);
    sc[u] = n > 0.f ? 1.f / (n * 8.f) : 0.f;  // 8 = sqrt(64)
  }
  __syncthreads();
}

// Score of query (key ki, raw q in registers) against window slot u.
// Returns -inf for another bucket / a later position, -1e5 for itself.
__device__ __forceinline__ float masked_score(const float* q, const float* qs, const float* sc,
                                              const uint32_t* ks, int u, uint32_t ki,
                                              uint32_t lo, uint32_t span, bool* live) {
  const uint32_t kj = ks[u];
  *live = false;
  if (kj - lo >= span) return -INFINITY;
  if (kj == ki) return kSelfScore;
  float dot = 0.f;
#pragma unroll 16
  for (int k = 0; k < kHeadDim; ++k) dot = fmaf(q[k], qs[u * 65 + k], dot);
  *live = true;
  return dot * sc[u];
}

// Forward for rounds [round0, round0 + gridDim.y / BH).  When `combine` is
// set the launch covers exactly the last round and folds the earlier rounds'
// partials (prev_o / prev_lse, rounds 0..R-2) into O and lse.
template <typename T>
__global__ void __launch_bounds__(256)
attend_fwd_simt_kernel(const T* __restrict__ Q, const T* __restrict__ V,
                       const uint32_t* __restrict__ keys, const int32_t* __restrict__ perm,
                       AttnDims a, int round0, float* __restrict__ o_part,
                       float* __restrict__ lse_r, int combine, int n_rounds,
                       const float* __restrict__ prev_o, const float* __restrict__ prev_lse,
                       T* __restrict__ O, float* __restrict__ lse) {
  extern __shared__ float smem[];
  const int W = a.W, c = a.chunk;
  float* qs = smem;                   // [W][65]
  float* vs = qs + (size_t)W * 65;    // [W][64]
  float* sc = vs + (size_t)W * 64;    // [W]
  float* pr = sc + W;                 // [c][W]
  uint32_t* ks = reinterpret_cast<uint32_t*>(pr + (size_t)c * W);  // [W]
  int* ps = reinterpret_cast<int*>(ks + W);                          // [W]

  const int cur = blockIdx.x;
  const int rl = blockIdx.y / a.BH, bh = blockIdx.y % a.BH;
  const int r = round0 + rl;
  const size_t row = (size_t)r * a.BH + bh;
  const T* Qbh = Q + (size_t)bh * a.L * kHeadDim;
  const T* Vbh = V + (size_t)bh * a.L * kHeadDim;
  load_window(a, Qbh, Vbh, keys + row * a.L, perm + row * a.L, cur, qs, vs, 64, sc, ks, ps);

  const int part = threadIdx.x & 3;
  const int qbase = (a.n_chunks > 1) ? c : 0;  // window index of the chunk's first query
  // The loop trip count is uniform across the block so that the group
  // shuffles below always run with every lane present.
  for (int q0 = 0; q0 < c; q0 += blockDim.x >> 2) {
    const int qi = q0 + (threadIdx.x >> 2);
    const bool act = qi < c;
    const int wq = qbase + (act ? qi : 0);
    float q[kHeadDim];
#pragma unroll
    for (int k = 0; k < kHeadDim; ++k) q[k] = qs[wq * 65 + k];
    const uint32_t ki = ks[wq];
    const uint32_t lo = ki - ki % (uint32_t)a.L;
    const uint32_t span = a.causal ? (ki - lo + 1) : (uint32_t)a.L;
    float* prow = pr + (size_t)(act ? qi : 0) * W;
    float m = -INFINITY;
    if (act)
      for (int u = part; u < W; u += 4) {
        bool live;
        const float s = masked_score(q, qs, sc, ks, u, ki, lo, span, &live);
        prow[u] = s;
        m = fmaxf(m, s);
      }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    float l = 0.f;
    if (act)
      for (int u = part; u < W; u += 4) {
        const float p = expf(prow[u] - m);
        prow[u] = p;
        l += p;
      }
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    __syncwarp();
    if (!act) continue;
    float acc[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) acc[x] = 0.f;
    for (int u = 0; u < W; ++u) {
      const float p = prow[u];
      const float* vr = vs + (size_t)u * 64 + part * 16;
#pragma unroll
      for (int x = 0; x < 16; ++x) acc[x] = fmaf(p, vr[x], acc[x]);
    }
    const float inv = 1.f / l;
#pragma unroll
    for (int x = 0; x < 16; ++x) acc[x] *= inv;
    const float my_lse = m + logf(l);

    const int i = ps[wq];
    const size_t tok = (size_t)bh * a.L + i;
    const size_t n_tok = (size_t)a.BH * a.L;
    if (o_part) {
      float* dst = o_part + ((size_t)r * n_tok + tok) * kHeadDim + part * 16;
      store8(dst, acc);
      store8(dst + 8, acc + 8);
    }
    if (lse_r && part == 0) lse_r[(size_t)r * n_tok + tok] = my_lse;
    if (combine) {
      float mx = my_lse;
      for (int rr = 0; rr < n_rounds - 1; ++rr) mx = fmaxf(mx, prev_lse[(size_t)rr * n_tok + tok]);
      float z = expf(my_lse - mx);
      for (int rr = 0; rr < n_rounds - 1; ++rr) z += expf(prev_lse[(size_t)rr * n_tok + tok] - mx);
      // weights relative to the maximum: near lse = -1e5 (a token alone in
      // every round) mx + log(z) is not representable to the needed precision
      const float rz = 1.f / z;
      const float tot = mx + logf(z);
      const float wl = expf(my_lse - mx) * rz;
      float o[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) o[x] = wl * acc[x];
      for (int rr = 0; rr < n_rounds - 1; ++rr) {
        const float wr = expf(prev_lse[(size_t)rr * n_tok + tok] - mx) * rz;
        const float* src = prev_o + ((size_t)rr * n_tok + tok) * kHeadDim + part * 16;
        float t8[8];
        load8(src, t8);
#pragma unroll
        for (int x = 0; x < 8; ++x) o[x] = fmaf(wr, t8[x], o[x]);
        load8(src + 8, t8);
#pragma unroll
        for (int x = 0; x < 8; ++x) o[8 + x] = fmaf(wr, t8[x], o[8 + x]);
      }
      T* dst = O + tok * kHeadDim + part * 16;
      store8(dst, o);
      store8(dst + 8, o + 8);
      if (lse && part == 0) lse[tok] = tot;
    }
  }
}

// ---------------------------------------------------------------------------
// Backward (buckets and permutations constant).
//
// With every round's window entries taken together, the combined output is
// one softmax over all entries (the round weights exp(lse_r - lse) times the
// per-round softmax give exp(s - lse)).  So for entry (i, j) of any round:
//   P = exp(s - lse_i),  dS = P (dO_i . v_j - G_i),  G_i = dO_i . O_i,
//   dv_j += P dO_i,  dq_i += dS khat_j / sqrt(d),  dkhat_j += dS q_i / sqrt(d),
// and dQ = dq + (dkhat - khat (khat . dkhat)) / |q| at the end.  Masked
// entries (another bucket, a later position, the token itself) have no dS.
// ---------------------------------------------------------------------------

__host__ __device__ inline size_t simt_bwd_smem_bytes(int chunk, int W) {
  return sizeof(float) * ((size_t)W * 65 * 2 + W + (size_t)chunk * 65 + 2 * (size_t)chunk +
                          2 * (size_t)chunk * W) +
         sizeof(uint32_t) * W + sizeof(int) * W;
}

// G_i = dO_i . O_i for every token (fp32).
template <typename T>
__global__ void bwd_dot_kernel(const T* __restrict__ O, const T* __restrict__ dO, size_t n_tok,
                               float* __restrict__ G) {
  const size_t tok = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tok >= n_tok) return;
  float s = 0.f;
  for (int k = 0; k < kHeadDim; k += 8) {
    float a[8], b[8];
    load8(O + tok * kHeadDim + k, a);
    load8(dO + tok * kHeadDim + k, b);
#pragma unroll
    for (int x = 0; x < 8; ++x) s = fmaf(a[x], b[x], s);
  }
  G[tok] = s;
}

template <typename T>
__global__ void __launch_bounds__(256)
attend_bwd_simt_kernel(const T* __restrict__ Q, const T* __restrict__ V, const T* __restrict__ dO,
                       const uint32_t* __restrict__ keys, const int32_t* __restrict__ perm,
                       const float* __restrict__ lse, const float* __restrict__ G, AttnDims a,
                       float inv_rounds, float* __restrict__ dq_acc, float* __restrict__ dk_acc,
                       float* __restrict__ dv_acc) {
  extern __shared__ float smem[];
  const int W = a.W, c = a.chunk;
  float* qs = smem;                     // [W][65] raw q
  float* vs = qs + (size_t)W * 65;      // [W][65] v
  float* sc = vs + (size_t)W * 65;      // [W] 1/(|q| sqrt d)
  float* dos = sc + W;                  // [c][65] dO of the chunk's queries
  float* gs = dos + (size_t)c * 65;     // [c] G
  float* ls = gs + c;                   // [c] lse
  float* pr = ls + c;                   // [c][W] P
  float* dsr = pr + (size_t)c * W;      // [c][W] dS
  uint32_t* ks = reinterpret_cast<uint32_t*>(dsr + (size_t)c * W);
  int* ps = reinterpret_cast<int*>(ks + W);

  const int cur = blockIdx.x;
  const int bh = blockIdx.y % a.BH;
  const int r = blockIdx.y / a.BH;
  const size_t row = (size_t)r * a.BH + bh;
  const T* Qbh = Q + (size_t)bh * a.L * kHeadDim;
  const T* Vbh = V + (size_t)bh * a.L * kHeadDim;
  load_window(a, Qbh, Vbh, keys + row * a.L, perm + row * a.L, cur, qs, vs, 65, sc, ks, ps);
  const int qbase = (a.n_chunks > 1) ? c : 0;
  const size_t tok0 = (size_t)bh * a.L;
  for (int e = threadIdx.x; e < c * 8; e += blockDim.x) {
    const int qi = e >> 3, k = (e & 7) * 8;
    float tmp[8];
    load8(dO + (tok0 + ps[qbase + qi]) * kHeadDim + k, tmp);
#pragma unroll
    for (int x = 0; x < 8; ++x) dos[qi * 65 + k + x] = tmp[x];
  }
  for (int qi = threadIdx.x; qi < c; qi += blockDim.x) {
    gs[qi] = G[tok0 + ps[qbase + qi]];
    ls[qi] = lse[tok0 + ps[qbase + qi]];
  }
  __syncthreads();

  const int part = threadIdx.x & 3;
  for (int qi = threadIdx.x >> 2; qi < c; qi += blockDim.x >> 2) {
    const int wq = qbase + qi;
    float q[kHeadDim];
#pragma unroll
    for (int k = 0; k < kHeadDim; ++k) q[k] = qs[wq * 65 + k];
    const uint32_t ki = ks[wq];
    const uint32_t lo = ki - ki % (uint32_t)a.L;
    const uint32_t span = a.causal ? (ki - lo + 1) : (uint32_t)a.L;
    const float li = ls[qi], gi = gs[qi];
    // A token alone in every round has lse = -1e5 + ln R, which fp32 stores
    // only to ~4e-3; its self weight in each round is exactly 1/R.
    const bool lone = li < kSelfScore + kLoneMargin;
    for (int u = part; u < W; u += 4) {
      bool live;
      const float s = masked_score(q, qs, sc, ks, u, ki, lo, span, &live);
      const float p = (lone && ks[u] == ki) ? inv_rounds : expf(s - li);
      float ds = 0.f;
      if (live) {
        float dp = 0.f;
#pragma unroll 16
        for (int k = 0; k < kHeadDim; ++k) dp = fmaf(dos[qi * 65 + k], vs[u * 65 + k], dp);
        ds = p * (dp - gi);
      }
      pr[(size_t)qi * W + u] = p;
      dsr[(size_t)qi * W + u] = ds;
    }
  }
  __syncthreads();

  // query side: dq_i = sum_u dS_iu q_u sc_u  (complete for this round)
  for (int qi = threadIdx.x >> 2; qi < c; qi += blockDim.x >> 2) {
    float acc[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) acc[x] = 0.f;
    for (int u = 0; u < W; ++u) {
      const float w = dsr[(size_t)qi * W + u] * sc[u];
      if (w == 0.f) continue;
#pragma unroll
      for (int x = 0; x < 16; ++x) acc[x] = fmaf(w, qs[u * 65 + part * 16 + x], acc[x]);
    }
    float* dst = dq_acc + (tok0 + ps[qbase + qi]) * kHeadDim + part * 16;
#pragma unroll
    for (int x = 0; x < 16; ++x) atomicAdd(dst + x, acc[x]);
  }
  // key side: dkhat_u = sum_i dS_iu q_i / sqrt(d);  dv_u = sum_i P_iu dO_i
  for (int task = threadIdx.x; task < W * 4; task += blockDim.x) {
    const int u = task >> 2, pt = task & 3;
    float dk[16], dv[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) { dk[x] = 0.f; dv[x] = 0.f; }
    for (int qi = 0; qi < c; ++qi) {
      const float ds = dsr[(size_t)qi * W + u] * 0.125f;  // 1/sqrt(64)
      const float p = pr[(size_t)qi * W + u];
      const float* qr = qs + (size_t)(qbase + qi) * 65 + pt * 16;
      const float* dr = dos + (size_t)qi * 65 + pt * 16;
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        dk[x] = fmaf(ds, qr[x], dk[x]);
        dv[x] = fmaf(p, dr[x], dv[x]);
      }
    }
    const size_t t = (tok0 + ps[u]) * kHeadDim + pt * 16;
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      atomicAdd(dk_acc + t + x, dk[x]);
      atomicAdd(dv_acc + t + x, dv[x]);
    }
  }
}

// dQ = dq + (dkhat - khat (khat . dkhat)) / |q|,  dV = dv, cast to T.  With
// dk_acc null the projection is already inside dq (dQ = dq).
template <typename T, typename OutT = T>
__global__ void bwd_finalize_kernel(const T* __restrict__ Q, const float* __restrict__ dq_acc,
                                    const float* __restrict__ dk_acc,
                                    const float* __restrict__ dv_acc, size_t n_tok,
                                    OutT* __restrict__ dQ, OutT* __restrict__ dV) {
  const size_t tok = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tok >= n_tok) return;
  if (!dk_acc) {
    for (int k = 0; k < kHeadDim; k += 8) {
      float dq[8], dv[8];
      load8(dq_acc + tok * kHeadDim + k, dq);
      load8(dv_acc + tok * kHeadDim + k, dv);
      store8(dQ + tok * kHeadDim + k, dq);
      store8(dV + tok * kHeadDim + k, dv);
    }
    return;
  }
  float q[kHeadDim], dk[kHeadDim];
  float ss = 0.f, proj = 0.f;
  for (int k = 0; k < kHeadDim; k += 8) {
    load8(Q + tok * kHeadDim + k, q + k);
    load8(dk_acc + tok * kHeadDim + k, dk + k);
  }
#pragma unroll
  for (int k = 0; k < kHeadDim; ++k) ss = fmaf(q[k], q[k], ss);
  const float n = sqrtf(ss);
  const float inv = n > 0.f ? 1.f / n : 0.f;
#pragma unroll
  for (int k = 0; k < kHeadDim; ++k) proj = fmaf(q[k] * inv, dk[k], proj);
  for (int k = 0; k < kHeadDim; k += 8) {
    float dq[8], dv[8];
    load8(dq_acc + tok * kHeadDim + k, dq);
    load8(dv_acc + tok * kHeadDim + k, dv);
#pragma unroll
    for (int x = 0; x < 8; ++x) dq[x] += (dk[k + x] - q[k + x] * inv * proj) * inv;
    store8(dQ + tok * kHeadDim + k, dq);
    store8(dV + tok * kHeadDim + k, dv);
  }
}

}  // namespace lsh
