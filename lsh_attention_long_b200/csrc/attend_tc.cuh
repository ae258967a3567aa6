// Chunked shared-QK LSH attention on the 5th-generation tensor cores
// (bf16 inputs, d = 64, chunk = 64).
//
// "Reformer explainer" (akshathtiwari.co.in/blog/reformer): sorted tokens are
// cut into equal chunks that attend to their bucket-mates, and several hash
// rounds are unioned.  Per round and chunk k of sorted slots: queries are the
// chunk's tokens, the window is chunk k and chunk k-1 (chunk 0 wraps to the
// last; a lone chunk sees itself once); scores are q_i . q_j / (|q_j| sqrt d);
// another bucket or (causal) a later position scores -inf; the token itself
// scores -1e5, so it only counts when nothing else is left.
//
// Tile = two consecutive chunks (128 query rows, one TMEM lane each); its
// window is three chunks (k-1, k, k+1), 192 keys, of which each query chunk
// uses two.  Per tile:
//   S  = Q[128 x 64] . K[192 x 64]^T   tcgen05.mma (N=192, the window's three
//                                       chunks contiguous in the slot) -> TMEM
//   P  = masked softmax numerators      CUDA cores, fp16, written over S in TMEM
//   O  = P[128 x 192] . V[192 x 64]     tcgen05.mma with A = P from TMEM
// The raw queries serve as keys in the MMA; 1/|q_j| (precomputed per token)
// and 1/sqrt(d) scale the scores in the softmax, so the MMA multiplies exact
// bf16 inputs.  P and V enter P.V as fp16 (V converted once per call, exactly
// for bf16 values in fp16's normal range): 11 significant bits of P instead
// of bf16's 8 keep the rounding of P well inside the bf16 output tolerance.  The softmax is referenced to the bound |q_i|/sqrt(d) of every
// score of row i (keys are unit vectors), so it takes one pass; a row whose
// bound exceeds kRefLimit takes an exact two-pass route.
//
// Mask on packed keys (key = bucket*L + position, ascending within a bucket
// in position order): key_j is in the query's bucket and allowed iff
// (key_j - bucket_i*L) < span as unsigned, with span = key_i - bucket_i*L
// (causal: strictly earlier positions, which also drops the token itself) or
// L (non-causal, where key_j == key_i is dropped separately).  The token's
// own entry enters only when a row has no other key in its round's window:
// then the round's output is its own value and lse = -1e5.
//
// Warp roles (480 threads):
//   warps 0-11   three softmax/epilogue warpgroups; warpgroup w takes the
//                CTA's tiles w, w+3, w+6, ... and always uses slot w.
//   warps 12-13  producers: warp 12 gathers the CTA's even tiles, warp 13 the
//                odd ones (perm, packed keys, key scales, q and v rows;
//                cp.async, 128B-swizzled) into the tile's slot.
//   warp 14      tensor-core issue: one thread issues S of tile n into TMEM
//                region n % 2 once the slot is full and the region free, and
//                P.V once P is written.
// Tensor memory holds two regions of 256 columns (S/P in the first 192, O in
// the last 64); a region is held from S to the load of O, about half of a
// warpgroup's work on a tile, so three warpgroups keep both regions busy.
// A slot is released as soon as P.V has read it: the epilogue keeps what it
// needs in registers.
//
// Tiles are dealt to CTAs statically: items of up to `tpi` consecutive tiles
// of one (round, head) row, item i to CTA i mod grid.  Items are ordered by
// blocks of heads, round by round within a block, so a block's q and v rows
// stay in L2 while its rounds run.  No tile depends on another.
//
// Output modes (per round, at original positions):
//   partial16  normalised o_r in fp16 and lse_r in fp32 (workspace); the
//              rounds are combined afterwards by combine_kernel.  fp16 keeps
//              11 significant bits of values bounded by max |v|, so the
//              combined O, rounded to bf16, stays within the bf16 tolerance;
//   partial32  normalised o_r in fp32 and lse_r (caller's buffers);
//   direct     one round: O in bf16 and lse written here.
#pragma once

#include <cuda_fp16.h>

#include "tc.cuh"

namespace lsh {

constexpr int kAtWG = 3;                          // softmax/epilogue warpgroups
constexpr int kAtSlots = kAtWG;                   // one gather slot per warpgroup
constexpr int kAtProducerWarp = 4 * kAtWG;        // warps 12, 13
constexpr int kAtMmaWarp = 4 * kAtWG + 2;         // warp 14
constexpr int kAtThreads = 32 * (4 * kAtWG + 3);  // 480
constexpr int kAtChunkBytes = 64 * 128;           // 64 rows of 128 B
constexpr int kAtSlotBytes = 6 * kAtChunkBytes;   // q then v of 3 chunks
constexpr int kAtStageBytes = 128 * 128;          // per warpgroup: 128 rows of 16-bit outputs
constexpr uint32_t kAtNoKey = 0xffffffffu;        // never inside a bucket range
constexpr float kLog2e = 1.4426950408889634f;
// Largest score bound |q_i|/sqrt(d) used directly as the softmax reference:
// every allowed score s >= -bound, so exp(s - bound) >= exp(-2 * 4) = 2^-11.5,
// above the smallest normal fp16 (2^-14), the type P enters P.V in.
constexpr float kRefLimit = 4.f;

enum AtMode { kAtPartial16 = 0, kAtPartial32 = 1, kAtDirect = 2 };

struct AtInfo {
  int r, bh;
  int nq;        // query chunks present: 1 or 2
  int has_prev;  // window has a previous chunk (the row has > 1 chunk)
};

struct AttnTcArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* V;
  const __half* V16;  // V in fp16, the P.V operand
  const uint32_t* keys;
  const int32_t* perm;
  const float* rn;   // [n_tok] log2(e) / (|q| sqrt(d)), 0 for a zero row
  int L, R, BH, n_chunks, causal;
  int n_tiles;       // tiles per row: ceil(n_chunks / 2)
  int tpi;           // tiles per item
  int ipr;           // items per (round, head) row
  int heads_per_block;
  long long n_items;
  int mode;          // AtMode
  __half* o16;       // partial16: [R][n_tok][64]
  float* o32;        // partial32: [R][n_tok][64]
  float* lse_r;      // partial modes (direct mode: optional): [R][n_tok]
  __nv_bfloat16* O;  // direct mode: [n_tok][64]
  float* lse;        // direct mode (optional): [n_tok]
  long long wait_limit;  // clock cycles a wait may take before the kernel gives up
  int hold_tile;         // test hook: producers stop before this tile of each CTA (-1: never)
};

struct AtSmem {
  uint32_t pos[kAtSlots][192];
  uint32_t key[kAtSlots][192];
  float rn[kAtSlots][192];
  AtInfo info[kAtSlots];
  uint32_t perm_stage[2][2][192];  // per producer, two tiles of perm entries
  uint64_t full[kAtSlots], empty[kAtSlots];
  uint64_t s_full[2], p_full[2], o_full[2], tm_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ inline size_t attend_tc_smem_bytes() {
  return 1024 + (size_t)kAtSlots * kAtSlotBytes + (size_t)kAtWG * kAtStageBytes + sizeof(AtSmem);
}

// Named barrier (id 1 + w) over the 128 threads of warpgroup w; OR of pred.
__device__ __forceinline__ bool wg_or(int w, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(1 + w)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Waits for a phase unless the CTA aborted; false on abort or after `limit`
// clock cycles (a timeout records LSH_ERR_TIMEOUT and sets the abort flag).
__device__ __forceinline__ bool at_wait(uint64_t* bar, uint32_t parity, int* abort,
                                        long long limit = tc::kSpinCycles) {
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

// Item -> (round, head row, first tile).  Order: blocks of heads; within a
// block round by round; within a round head by head, then items.
__device__ __forceinline__ void at_decode(const AttnTcArgs& a, long long item, int& r, int& bh,
                                          int& t0) {
  const long long per_full_block = (long long)a.R * a.heads_per_block * a.ipr;
  const int blk = (int)(item / per_full_block);
  const long long idx = item - (long long)blk * per_full_block;
  const int h0 = blk * a.heads_per_block;
  const int nh = min(a.heads_per_block, a.BH - h0);
  const long long per_round = (long long)nh * a.ipr;
  r = (int)(idx / per_round);
  const int rem = (int)(idx - (long long)r * per_round);
  bh = h0 + rem / a.ipr;
  t0 = (rem % a.ipr) * a.tpi;
}

// Masked, scaled scores (log2 units; -inf where masked) of 32 window
// columns whose packed keys and key scales are kw[0..31], rw[0..31].
__device__ __forceinline__ void mask32(float* v, const uint32_t* kw, const float* rw,
                                       uint32_t lo, uint32_t span, uint32_t ki, bool active,
                                       bool causal) {
#pragma unroll
  for (int jj = 0; jj < 32; jj += 4) {
    const uint4 k4 = *reinterpret_cast<const uint4*>(kw + jj);
    const float4 r4 = *reinterpret_cast<const float4*>(rw + jj);
    const uint32_t kj[4] = {k4.x, k4.y, k4.z, k4.w};
    const float rj[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      bool in = active && (kj[x] - lo) < span;
      if (!causal) in = in && kj[x] != ki;
      v[jj + x] = in ? v[jj + x] * rj[x] : -INFINITY;
    }
  }
}

// P (fp16 pairs into pk) for 32 window columns and their sum into ls: a
// column in the query's bucket and allowed gets exp2(s * r_j - ref2), any
// other column 0.  With `scaled` the scores are already masked and scaled
// (the exact route) and only ref2 is subtracted.  The block's packed keys are
// ascending (a piece of the sorted row), so a row can only have allowed
// columns in it if [kw[0], kw[31]] meets [lo, lo + span); when no row of the
// warp does, the block is all zeros and its exponentials are skipped.
__device__ __forceinline__ void softmax32(const float* v, const uint32_t* kw, const float* rw,
                                          uint32_t lo, uint32_t span, uint32_t ki, bool active,
                                          bool causal, bool scaled, float ref2, float* ls,
                                          uint32_t* pk) {
  const bool any = active && kw[31] >= lo && kw[0] < lo + span;  // lo + span <= nb * L < 2^31
  if (!__any_sync(0xffffffffu, any)) {
#pragma unroll
    for (int x = 0; x < 16; ++x) pk[x] = 0u;
    return;
  }
#pragma unroll
  for (int jj = 0; jj < 32; jj += 4) {
    const uint4 k4 = *reinterpret_cast<const uint4*>(kw + jj);
    const float4 r4 = *reinterpret_cast<const float4*>(rw + jj);
    const uint32_t kj[4] = {k4.x, k4.y, k4.z, k4.w};
    const float rj[4] = {r4.x, r4.y, r4.z, r4.w};
    float p[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      bool in = active && (kj[x] - lo) < span;
      if (!causal) in = in && kj[x] != ki;
      const float t = scaled ? v[jj + x] - ref2 : fmaf(v[jj + x], rj[x], -ref2);
      p[x] = ex2((scaled || in) ? t : -INFINITY);
    }
    ls[(jj >> 2) & 3] += (p[0] + p[1]) + (p[2] + p[3]);
    pk[jj / 2] = pack_f16(p[0], p[1]);
    pk[jj / 2 + 1] = pack_f16(p[2], p[3]);
  }
}

// Exact route for rows with a large score bound: writes the masked scores
// back over S and returns the row maximum (log2 units; 0 if all masked).
// Out of line: rarely taken, kept out of the hot loop's instruction cache.
__device__ __noinline__ float exact_row_max(uint32_t region, int qc, const uint32_t* key_s,
                                            const float* rn_s, uint32_t lo, uint32_t span,
                                            uint32_t ki, bool valid, bool has_prev, bool causal) {
  float mx2 = -INFINITY;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    const int kc = qc + (c >> 1);
    float v[32];
    tc::tmem_ld32(region + qc * 64 + 32 * c, v);
    tc::tmem_ld_wait();
    mask32(v, key_s + kc * 64 + 32 * (c & 1), rn_s + kc * 64 + 32 * (c & 1), lo, span, ki,
           valid && (kc != 0 || has_prev), causal);
#pragma unroll
    for (int x = 0; x < 32; ++x) mx2 = fmaxf(mx2, v[x]);
    tc::tmem_st32(region + qc * 64 + 32 * c, reinterpret_cast<const uint32_t*>(v));
  }
  tc::tmem_st_wait();
  return mx2 == -INFINITY ? 0.f : mx2;
}

// Per token, before the forward: the key scale log2(e)/(|q| sqrt(d)) (0 for a
// zero row) and the value row in fp16 for the P.V product.  Eight threads
// per token, 16 bytes of q and of v each.
__global__ void fwd_prep_kernel(const __nv_bfloat16* __restrict__ Q,
                                const __nv_bfloat16* __restrict__ V, size_t n_tok,
                                float* __restrict__ rn, __half* __restrict__ V16) {
  const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t tok = g >> 3;
  const int k = (int)(g & 7) * 8;
  const bool in = tok < n_tok;
  float ssq = 0.f;
  if (in) {
    float x[8];
    load8(Q + tok * kHeadDim + k, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) ssq = fmaf(x[e], x[e], ssq);
    load8(V + tok * kHeadDim + k, x);
    store8(V16 + tok * kHeadDim + k, x);
  }
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 1);
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 2);
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 4);
  if (in && k == 0) rn[tok] = ssq > 0.f ? rsqrtf(ssq) * (0.125f * kLog2e) : 0.f;
}

// Walks one CTA's tiles in order: items blockIdx.x, blockIdx.x + gridDim.x, ...
struct AtSeq {
  long long item;
  int r, bh, t, t_end;
  bool valid;
};
__device__ __forceinline__ void seq_load(const AttnTcArgs& a, AtSeq& q) {
  q.valid = q.item < a.n_items;
  if (!q.valid) return;
  at_decode(a, q.item, q.r, q.bh, q.t);
  q.t_end = min(q.t + a.tpi, a.n_tiles);
}
__device__ __forceinline__ void seq_start(const AttnTcArgs& a, AtSeq& q) {
  q.item = blockIdx.x;
  seq_load(a, q);
}
__device__ __forceinline__ void seq_next(const AttnTcArgs& a, AtSeq& q) {
  if (!q.valid) return;
  if (++q.t >= q.t_end) {
    q.item += gridDim.x;
    seq_load(a, q);
  }
}
// Tiles this CTA processes.
__device__ __forceinline__ uint32_t cta_tiles(const AttnTcArgs& a) {
  uint32_t n = 0;
  for (long long it = blockIdx.x; it < a.n_items; it += gridDim.x) {
    int r, bh, t0;
    at_decode(a, it, r, bh, t0);
    n += (uint32_t)(min(t0 + a.tpi, a.n_tiles) - t0);
  }
  return n;
}

__global__ void __launch_bounds__(kAtThreads, 1) attend_tc_kernel(AttnTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* slots = sm;
  uint8_t* stage = sm + kAtSlots * kAtSlotBytes;
  AtSmem& S = *reinterpret_cast<AtSmem*>(stage + kAtWG * kAtStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long limit = a.wait_limit;

  if (tid == 0) {
    for (int s = 0; s < kAtSlots; ++s) {
      tc::mbar_init(&S.full[s], 64);    // 32 producer lanes x (cp.async arrive + arrive)
      tc::mbar_init(&S.empty[s], 128);  // every thread of the slot's warpgroup
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&S.s_full[b], 1);
      tc::mbar_init(&S.p_full[b], 128);
      tc::mbar_init(&S.o_full[b], 1);
      tc::mbar_init(&S.tm_free[b], 128);
    }
    tc::mbar_init(&S.mma_done, 1);
    tc::mbar_init_fence();
    S.abort = 0;
  }
  if (warp == kAtMmaWarp) {
    tc::tmem_alloc(&S.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  const size_t n_tok = (size_t)a.BH * a.L;
  const uint32_t n_total = cta_tiles(a);

  if (warp == kAtProducerWarp || warp == kAtProducerWarp + 1) {
    // ------------------------------------------------------------ producers
    // Producer p takes tiles p, p+2, p+4, ... of this CTA.  The perm entries
    // of its next tile are staged (cp.async) while it gathers the current one.
    const int p = warp - kAtProducerWarp;
    AtSeq cur;
    seq_start(a, cur);
    if (p == 1) seq_next(a, cur);
    AtSeq nxt = cur;
    seq_next(a, nxt);
    seq_next(a, nxt);
    // window slot u: chunk u/64 of (prev, k0, k0+1); absent chunks read kAtNoKey
    auto stage_perm = [&](const AtSeq& q, int buf) {
      if (q.valid) {
        const size_t rowbase = ((size_t)q.r * a.BH + q.bh) * a.L;
        const int k0 = 2 * q.t;
        const int prev = (k0 == 0) ? a.n_chunks - 1 : k0 - 1;
        for (int piece = lane; piece < 48; piece += 32) {  // 16-byte pieces
          const int cw = piece >> 4;
          const int ch = cw == 0 ? prev : k0 + cw - 1;
          const bool present = (cw == 0) ? (a.n_chunks > 1) : (ch < a.n_chunks);
          uint32_t* dst = &S.perm_stage[p][buf][cw * 64 + (piece & 15) * 4];
          if (present)
            tc::cp_async16(tc::smem_u32(dst), a.perm + rowbase + (size_t)ch * 64 + (piece & 15) * 4);
          else
            *reinterpret_cast<uint4*>(dst) = make_uint4(kAtNoKey, kAtNoKey, kAtNoKey, kAtNoKey);
        }
      }
      tc::cp_async_commit();
    };
    stage_perm(cur, 0);
    stage_perm(nxt, 1);
    for (uint32_t n = p, j = 0; n < n_total; n += 2, ++j) {
      if ((int)n == a.hold_tile) break;  // test hook: the tile's slot is never filled
      const int s = n % kAtSlots;
      if (j == 0) tc::cp_async_wait<1>(); else tc::cp_async_wait<2>();  // perm of this tile
      __syncwarp();
      if (!__all_sync(0xffffffffu, at_wait(&S.empty[s], ((n / kAtSlots) & 1u) ^ 1u, &S.abort, limit)))
        break;
      uint32_t pos[6];
#pragma unroll
      for (int e = 0; e < 6; ++e) pos[e] = S.perm_stage[p][j & 1][lane + 32 * e];
      AtInfo inf;
      const int k0 = 2 * cur.t;
      inf.r = cur.r;
      inf.bh = cur.bh;
      inf.nq = (k0 + 1 < a.n_chunks) ? 2 : 1;
      inf.has_prev = a.n_chunks > 1 ? 1 : 0;
      const size_t rowbase = ((size_t)cur.r * a.BH + cur.bh) * a.L;
      uint8_t* slot = slots + (size_t)s * kAtSlotBytes;
      const __nv_bfloat16* Qbh = a.Q + (size_t)cur.bh * a.L * 64;
      const __half* Vbh = a.V16 + (size_t)cur.bh * a.L * 64;
      const float* rnbh = a.rn + (size_t)cur.bh * a.L;
      // slot metadata, lane-per-row: position, packed key, key scale
#pragma unroll
      for (int e = 0; e < 6; ++e) {
        const int u = lane + 32 * e;
        uint32_t q = pos[e];
        if (q != kAtNoKey && q >= (uint32_t)a.L) {  // not a permutation of the row
          record_status(kErrBadKeys);
          q = 0;
        }
        if (q != kAtNoKey) {
          S.pos[s][u] = q;
          cp_async4(tc::smem_u32(&S.key[s][u]), a.keys + rowbase + q);
          cp_async4(tc::smem_u32(&S.rn[s][u]), rnbh + q);
        } else {
          S.pos[s][u] = kAtNoKey;
          S.key[s][u] = kAtNoKey;
          S.rn[s][u] = 0.f;
        }
      }
      __syncwarp();
      // q and v rows, eight lanes per 128-byte row (coalesced per row): four
      // rows per warp instruction; lane group G takes window rows 48G..48G+47
      // and reads their positions four at a time
      {
        const int G = lane >> 3, c = lane & 7;
#pragma unroll 1
        for (int i0 = 0; i0 < 48; i0 += 4) {
          const uint4 p4 = *reinterpret_cast<const uint4*>(&S.pos[s][48 * G + i0]);
          const uint32_t pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int u = 48 * G + i0 + x;
            const int cw = u >> 6, row = u & 63;
            uint8_t* qd = slot + cw * kAtChunkBytes + tc::sw128_offset(row, c);
            uint8_t* vd = qd + 3 * kAtChunkBytes;
            const uint32_t q = pv[x];
            if (q != kAtNoKey) {
              tc::cp_async16(tc::smem_u32(qd), Qbh + (size_t)q * 64 + c * 8);
              tc::cp_async16(tc::smem_u32(vd), Vbh + (size_t)q * 64 + c * 8);
            } else {
              *reinterpret_cast<uint4*>(qd) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
            }
          }
        }
      }
      __syncwarp();
#pragma unroll
      for (int e = 0; e < 6; ++e)  // absent rows read as position 0 downstream
        if (S.pos[s][lane + 32 * e] == kAtNoKey) S.pos[s][lane + 32 * e] = 0;
      if (lane == 0) S.info[s] = inf;
      tc::cp_async_commit();  // this tile's gathers
      tc::fence_async_smem();
      cp_async_arrive_noinc(&S.full[s]);
      tc::mbar_arrive(&S.full[s]);
      // this producer's tile after next: its perm entries into the buffer
      // just read
      cur = nxt;
      seq_next(a, nxt);
      seq_next(a, nxt);
      stage_perm(nxt, j & 1);
    }
    tc::cp_async_wait_all();
  } else if (warp == kAtMmaWarp) {
    // ------------------------------------------------------ tensor-core issue
    if (lane == 0) {
      const uint32_t idesc_s = tc::idesc_bf16(128, 192, 0, 0);
      const uint32_t idesc_o = tc::idesc_f16(128, 64, 0, 1);
      uint32_t n_s = 0, n_p = 0;  // next S to issue, next P.V to issue
      long long idle_since = clock64();
      while (n_p < n_total) {
        bool progress = false;
        // S of tile n_s into region n_s % 2, once tile n_s - 2 (the region's
        // last user) has had its P.V issued and its O read
        if (n_s < n_total && n_s < n_p + 2) {
          const int s = n_s % kAtSlots, b = n_s & 1;
          if (tc::mbar_probe(&S.full[s], (n_s / kAtSlots) & 1u) &&
              tc::mbar_probe(&S.tm_free[b], ((n_s >> 1) & 1u) ^ 1u)) {
            tc::fence_after_sync();
            tc::fence_async_smem();  // cp.async rows of this slot -> tensor-core reads
            uint8_t* slot = slots + (size_t)s * kAtSlotBytes;
            // descriptors of the slot's first chunk; the address field counts
            // 16-byte units, so later pieces are constant offsets
            const uint64_t dk0 = tc::sdesc_sw128(tc::smem_u32(slot), 16, 1024);
            const uint64_t dq0 = dk0 + (kAtChunkBytes >> 4);  // chunks k0, k0+1
            const uint32_t d = tmem + b * 256;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // N = 192: the window's three chunks at once
              tc::mma_bf16(d, dq0 + 2 * kk, dk0 + 2 * kk, idesc_s, kk > 0);
            tc::mma_commit(&S.s_full[b]);
            ++n_s;
            progress = true;
          }
        }
        if (n_p < n_s) {
          const int s = n_p % kAtSlots, b = n_p & 1;
          if (tc::mbar_probe(&S.p_full[b], (n_p >> 1) & 1u)) {
            tc::fence_after_sync();
            uint8_t* slot = slots + (size_t)s * kAtSlotBytes;
            const uint32_t pa = tmem + b * 256;  // P over S: key block c at columns 32c
            const uint64_t dv0 = tc::sdesc_sw128(tc::smem_u32(slot + 3 * kAtChunkBytes), 8192, 1024);
#pragma unroll
            for (int c = 0; c < 3; ++c) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16_ts(tmem + b * 256 + 192, pa + c * 32 + kk * 8,
                                dv0 + ((c * kAtChunkBytes + kk * 2048) >> 4), idesc_o,
                                (c | kk) != 0);
            }
            tc::mma_commit(&S.o_full[b]);
            ++n_p;
            progress = true;
          }
        }
        if (progress) {
          idle_since = clock64();
        } else {
          __nanosleep(32);  // leave issue slots to the softmax warps on this SMSP
          if (*(volatile int*)&S.abort) break;
          if (clock64() - idle_since > limit) {
            record_status(tc::kErrTimeout);
            *(volatile int*)&S.abort = 1;
            break;
          }
        }
      }
      // every MMA issued above has finished before tensor memory is freed
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
  } else if (warp < 4 * kAtWG) {
    // --------------------------------------------- softmax and epilogue
    const int w = warp >> 2;            // warpgroup = slot
    const int m = tid & 127;            // query row = TMEM lane
    const int qc = m >> 6;              // query chunk within the tile
    const int wrow0 = (warp & 3) * 32;  // first row of this warp
    const int s = w;
    uint8_t* my_stage = stage + (size_t)w * kAtStageBytes;
    for (uint32_t n = w, j = 0; n < n_total; n += kAtWG, ++j) {
      const int b = n & 1;
      const uint32_t region = tmem + (uint32_t)b * 256 + ((uint32_t)wrow0 << 16);
      const bool okf = at_wait(&S.full[s], j & 1u, &S.abort, limit);
      if (wg_or(w, !okf)) break;
      const AtInfo inf = S.info[s];
      const bool valid = qc < inf.nq;
      const uint32_t ki = S.key[s][64 + m];
      const uint32_t my_pos = S.pos[s][64 + m];
      const size_t bhL = (size_t)inf.bh * a.L;
      const size_t tok = bhL + my_pos;

      // scores of this row's two window chunks (qc, qc + 1), 32 columns at a
      // time, referenced to the bound |q_i|/sqrt(d) (single pass), or to the
      // exact row maximum when a row of the warp has a bound above kRefLimit
      const bool oks = at_wait(&S.s_full[b], (n >> 1) & 1u, &S.abort, limit);
      if (wg_or(w, !oks)) break;
      tc::fence_after_sync();
      const uint32_t lo = ki - ki % (uint32_t)a.L;
      const uint32_t span = a.causal ? (ki - lo) : (uint32_t)a.L;
      const float rn_i = S.rn[s][64 + m];  // log2(e)/(|q_i| sqrt d)
      const float bound = rn_i > 0.f ? 1.f / (64.f * rn_i * (1.f / kLog2e)) : 0.f;
      const bool exact = __any_sync(0xffffffffu, bound > kRefLimit);
      float ref2 = bound * kLog2e;  // reference in log2 units
      if (exact)  // pass 1: masked scores back into S, exact row maximum
        ref2 = exact_row_max(region, qc, S.key[s], S.rn[s], lo, span, ki, valid, inf.has_prev,
                             a.causal != 0);
      float ls[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
      // P (bf16, two per column) over S: key block b at columns [32b, 32b+32).
      // Step c reads S columns qc*64 + 32c .. +32 (window chunk qc + c/2) and
      // writes P columns 32(qc + c/2) + 16(c&1) .. +16; every write lands on
      // columns already read and never on ones a later step reads.
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int kc = qc + (c >> 1);
        float v[32];
        tc::tmem_ld32(region + qc * 64 + 32 * c, v);
        tc::tmem_ld_wait();
        tc::tmem_pin<32>(v);
        uint32_t pk[16];
        softmax32(v, &S.key[s][kc * 64 + 32 * (c & 1)], &S.rn[s][kc * 64 + 32 * (c & 1)], lo, span,
                  ki, valid && (kc != 0 || inf.has_prev), a.causal != 0, exact, ref2, ls, pk);
        tc::tmem_st16(region + kc * 32 + 16 * (c & 1), pk);
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) pk[x] = 0u;
        tc::tmem_st32(region + (qc == 0 ? 2 : 0) * 32, pk);  // the block outside the window
      }
      tc::tmem_st_wait();
      tc::fence_before_sync();
      tc::mbar_arrive(&S.p_full[b]);
      const float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      const bool lone = !(lsum > 0.f);  // nothing but itself in this round
      const float mx = ref2 * (1.f / kLog2e);
      const float m_r = lone ? kSelfScore : mx;
      const float l_r = lone ? 1.f : lsum;
      const float scale = 1.f / l_r;

      const bool oko = at_wait(&S.o_full[b], (n >> 1) & 1u, &S.abort, limit);
      if (wg_or(w, !oko)) break;
      tc::fence_after_sync();
      tc::mbar_arrive(&S.empty[s]);  // P.V has read the slot's rows
      float o[64];
      tc::tmem_ld32(region + 192, o);
      tc::tmem_ld32(region + 224, o + 32);
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      tc::mbar_arrive(&S.tm_free[b]);  // this region of tensor memory is free again
      if (lone && valid) {
        const __nv_bfloat16* vs = a.V + tok * 64;
#pragma unroll
        for (int q = 0; q < 8; ++q) load8(vs + 8 * q, o + 8 * q);
      }
#pragma unroll
      for (int x = 0; x < 64; ++x) o[x] *= scale;
      const float lse_row = lone ? kSelfScore : m_r + logf(l_r);
      if (a.mode == kAtPartial32) {
        if (valid) {
          float* dst = a.o32 + ((size_t)inf.r * n_tok + tok) * 64;
#pragma unroll
          for (int q = 0; q < 16; ++q)
            *reinterpret_cast<float4*>(dst + 4 * q) =
                make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          a.lse_r[(size_t)inf.r * n_tok + tok] = lse_row;
        }
        continue;
      }
      // 16-bit rows through this warpgroup's staging rows (16-byte pieces
      // swizzled by row), then eight lanes per 128-byte row to their positions
      uint8_t* my_row = my_stage + (size_t)m * 128;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint4 u;
        if (a.mode == kAtPartial16) {
          const __half2 h0 = __floats2half2_rn(o[8 * q], o[8 * q + 1]);
          const __half2 h1 = __floats2half2_rn(o[8 * q + 2], o[8 * q + 3]);
          const __half2 h2 = __floats2half2_rn(o[8 * q + 4], o[8 * q + 5]);
          const __half2 h3 = __floats2half2_rn(o[8 * q + 6], o[8 * q + 7]);
          u = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                         *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
        } else {
          u = make_uint4(pack_bf16(o[8 * q], o[8 * q + 1]), pack_bf16(o[8 * q + 2], o[8 * q + 3]),
                         pack_bf16(o[8 * q + 4], o[8 * q + 5]), pack_bf16(o[8 * q + 6], o[8 * q + 7]));
        }
        *reinterpret_cast<uint4*>(my_row + ((q ^ (m & 7)) << 4)) = u;
      }
      if (valid) {
        if (a.mode == kAtPartial16) a.lse_r[(size_t)inf.r * n_tok + tok] = lse_row;
        else {
          if (a.lse) a.lse[tok] = lse_row;
          if (a.lse_r) a.lse_r[tok] = lse_row;
        }
      }
      __syncwarp();
      if (valid) {  // uniform per warp
        uint16_t* base = a.mode == kAtPartial16
                             ? reinterpret_cast<uint16_t*>(a.o16) + (size_t)inf.r * n_tok * 64
                             : reinterpret_cast<uint16_t*>(a.O);
#pragma unroll 2
        for (int i = 0; i < 8; ++i) {
          const int rl = 4 * i + (lane >> 3), q = lane & 7;
          const int rr = wrow0 + rl;
          const uint32_t pr = __shfl_sync(0xffffffffu, my_pos, rl);
          const uint4 u = *reinterpret_cast<const uint4*>(my_stage + (size_t)rr * 128 + ((q ^ (rr & 7)) << 4));
          *reinterpret_cast<uint4*>(base + (bhL + pr) * 64 + 8 * q) = u;
        }
      }
      __syncwarp();  // the staging rows are rewritten by the next tile
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kAtMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// O and lse from the per-round partials: lse = logsumexp_r lse_r,
// O = sum_r exp(lse_r - lse) o_r, with the weights formed as
// exp(lse_r - max) / sum (a token alone in every round has lse_r = -1e5 in
// each, whose logsumexp fp32 cannot resolve).  Eight threads per token.
template <typename P, typename T>
__global__ void combine_kernel(const P* __restrict__ o_part, const float* __restrict__ lse_r,
                               int n_rounds, size_t n_tok, T* __restrict__ O,
                               float* __restrict__ lse) {
  const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= n_tok * 8) return;
  const size_t tok = g >> 3;
  const int k = (int)(g & 7) * 8;
  float mx = -INFINITY;
  for (int r = 0; r < n_rounds; ++r) mx = fmaxf(mx, lse_r[(size_t)r * n_tok + tok]);
  float z = 0.f;
  for (int r = 0; r < n_rounds; ++r) z += expf(lse_r[(size_t)r * n_tok + tok] - mx);
  const float rz = 1.f / z;
  const float tot = mx + logf(z);
  float o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = 0; r < n_rounds; ++r) {
    const float w = expf(lse_r[(size_t)r * n_tok + tok] - mx) * rz;
    float t8[8];
    load8(o_part + ((size_t)r * n_tok + tok) * kHeadDim + k, t8);
#pragma unroll
    for (int x = 0; x < 8; ++x) o[x] = fmaf(w, t8[x], o[x]);
  }
  store8(O + tok * kHeadDim + k, o);
  if (lse && k == 0) lse[tok] = tot;
}

// The same for the fp16 partials with R a compile-time constant, so that all
// R partial rows of a token are in flight before they are weighed (same
// arithmetic, same order, as combine_kernel).
template <int R, typename T>
__global__ void combine16_kernel(const __half* __restrict__ o_part, const float* __restrict__ lse_r,
                                 size_t n_tok, T* __restrict__ O, float* __restrict__ lse) {
  const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= n_tok * 8) return;
  const size_t tok = g >> 3;
  const int k = (int)(g & 7) * 8;
  float l[R];
  uint4 raw[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    l[r] = lse_r[(size_t)r * n_tok + tok];
    raw[r] = *reinterpret_cast<const uint4*>(o_part + ((size_t)r * n_tok + tok) * kHeadDim + k);
  }
  float mx = l[0];
#pragma unroll
  for (int r = 1; r < R; ++r) mx = fmaxf(mx, l[r]);
  float w[R], z = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r) { w[r] = expf(l[r] - mx); z += w[r]; }
  const float rz = 1.f / z;
  float o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float wr = w[r] * rz;
    const __half2* h = reinterpret_cast<const __half2*>(&raw[r]);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float2 v = __half22float2(h[x]);
      o[2 * x] = fmaf(wr, v.x, o[2 * x]);
      o[2 * x + 1] = fmaf(wr, v.y, o[2 * x + 1]);
    }
  }
  store8(O + tok * kHeadDim + k, o);
  if (lse && k == 0) lse[tok] = mx + logf(z);
}

}  // namespace lsh
