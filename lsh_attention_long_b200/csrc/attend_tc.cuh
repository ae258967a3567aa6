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
//   S  = Q[128 x 64] . K[192 x 64]^T   tcgen05.mma (three N=64 MMAs) -> TMEM
//   P  = masked softmax numerators      CUDA cores, bf16, written over S in TMEM
//   O  = P[128 x 192] . V[192 x 64]     tcgen05.mma with A = P from TMEM
// The raw queries serve as keys in the MMA; 1/|q_j| (precomputed per token)
// and 1/sqrt(d) scale the scores in the softmax, so the MMA multiplies exact
// bf16 inputs.
//
// Mask on packed keys (key = bucket*L + position, ascending within a bucket
// in position order): key_j is in the query's bucket and allowed iff
// (key_j - bucket_i*L) < span as unsigned, with span = key_i - bucket_i*L
// (causal: strictly earlier positions, which also drops the token itself) or
// L (non-causal, where key_j == key_i is dropped separately).  The token's
// own entry enters only when a row has no other key in its round's window:
// then the round's output is its own value and lse = -1e5.
//
// Warp roles (352 threads):
//   warps 0-3, 4-7  two softmax/epilogue warpgroups; warpgroup w takes the
//                   CTA's tiles w, w+2, w+4, ... so one warpgroup's softmax
//                   overlaps the other's MMAs and epilogue.  Each owns half of
//                   tensor memory: S/P in columns [256w, 256w+192), O in
//                   [256w+192, 256w+256).
//   warp 8          producer: takes work tickets, gathers perm, packed keys,
//                   key scales and q, v rows (cp.async, 128B-swizzled) into a
//                   ring of 4 shared-memory slots (full/empty mbarriers).
//   warp 9          tensor-core issue: one thread polls the barriers and
//                   issues S for tile n+1 as soon as its data and TMEM half
//                   are free, and P.V for tile n as soon as P is written.
//   warp 10         publisher (online mode): fences and counts finished
//                   tiles so the compute warps never wait on store latency.
//
// Two output modes:
//   partial  every round's normalised o_r (fp32) and lse_r go to o_part /
//            lse_r at original positions (the combine runs afterwards);
//   online   each round folds its result into a running (max, sum,
//            unnormalised output) per token kept in the workspace; even
//            rounds fold into one running state and odd rounds into a second,
//            and online_merge_kernel joins the two into O (bf16) and lse.  A
//            tile of round r of a head waits (bounded spin) until every tile
//            of round r-2 of that head is done (per-head tile counters), so
//            consecutive rounds of a head overlap; tickets are handed out in
//            an order where that dependency always points to earlier
//            tickets, so the scheme cannot deadlock.  Heads are taken in
//            blocks sized so that a block's running states and q, v rows stay
//            resident in L2 while its rounds run.
#pragma once

#include "tc.cuh"

namespace lsh {

constexpr int kAtSlots = 3;
constexpr int kAtThreads = 352;
constexpr int kAtPubRing = 16;
constexpr int kAtChunkBytes = 64 * 128;          // 64 rows of 128 B
constexpr int kAtSlotBytes = 6 * kAtChunkBytes;  // q then v of 3 chunks
// Per warpgroup, the running state of its tile's 128 rows (online mode),
// staged by cp.async while the softmax runs: 64 fp32 per row (16-byte pieces
// swizzled by row) and the (max, sum) pair padded to 16 bytes.
constexpr int kAtAccBytes = 2 * 128 * 256;
constexpr int kAtMlBytes = 2 * 128 * 16;
constexpr uint32_t kAtNoKey = 0xffffffffu;       // never inside a bucket range
constexpr float kLog2e = 1.4426950408889634f;
// Largest score bound |q_i|/sqrt(d) used directly as the softmax reference:
// every allowed score s >= -bound, so exp(s - bound) >= exp(-2 * 30), far
// from fp32 / bf16 underflow.
constexpr float kRefLimit = 30.f;

struct AtInfo {
  int r, bh, t;
  int first, last;  // first / last tile of its item
  int done;
  int nq;           // query chunks present: 1 or 2
  int has_prev;     // window has a previous chunk (the row has > 1 chunk)
  int seq;          // tile sequence number the slot holds
};

struct AttnTcArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* V;
  const uint32_t* keys;
  const int32_t* perm;
  const float* rn;   // [n_tok] log2(e) / (|q| sqrt(d)), 0 for a zero row
  int L, R, BH, n_chunks, causal;
  int n_tiles;       // tiles per row: ceil(n_chunks / 2)
  int tpi;           // tiles per item
  int ipr;           // items per (round, head) row
  int heads_per_block;
  long long n_items;
  int online;
  float* o_part;     // partial mode
  float* lse_r;
  float* acc_o;      // online mode: [2][n_tok][64] unnormalised output (even, odd rounds)
  float4* acc_ml;    // online mode: [2][n_tok] (running max, running sum, -, -)
  unsigned* counters;  // [BH][R] tiles done; then one ticket counter
};

struct AtSmem {
  uint32_t pos[kAtSlots][192];
  uint32_t key[kAtSlots][192];
  float rn[kAtSlots][192];
  AtInfo info[kAtSlots];
  uint64_t full[kAtSlots], empty[kAtSlots];
  uint64_t s_full[2], p_full[2], o_full[2], tm_free[2];
  uint32_t perm_stage[kAtSlots][192];  // perm entries of the tile two ahead
  // completion ring (online mode): compute warpgroups post finished tiles,
  // the publisher warp makes them visible and counts them
  int pub_bh[kAtPubRing], pub_r[kAtPubRing];
  unsigned pub_seq[kAtPubRing];
  unsigned pub_head;  // tiles published so far
  unsigned n_total;   // tiles this CTA will process (set when known)
  uint32_t tmem_base;
  int abort;
  int dep_bh, dep_r;  // last (head, round) whose previous round was seen complete
};

__host__ __device__ inline size_t attend_tc_smem_bytes() {
  return 1024 + (size_t)kAtSlots * kAtSlotBytes + kAtAccBytes + kAtMlBytes + sizeof(AtSmem);
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
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_acquire_cta(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(v) : "r"(tc::smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_cta(unsigned* p, unsigned v) {
  asm volatile("st.release.cta.shared.u32 [%0], %1;" ::"r"(tc::smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Waits for a phase unless the CTA aborted; false on abort or timeout
// (timeouts record LSH_ERR_TIMEOUT and set the abort flag).
__device__ __forceinline__ bool at_wait(uint64_t* bar, uint32_t parity, int* abort) {
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

// Item `ticket` -> (round, head row, first tile).  Order: blocks of heads;
// within a block round by round; within a round head by head, then items.
__device__ __forceinline__ void at_decode(const AttnTcArgs& a, long long ticket, int& r, int& bh,
                                          int& t0) {
  const long long per_full_block = (long long)a.R * a.heads_per_block * a.ipr;
  const int blk = (int)(ticket / per_full_block);
  const long long idx = ticket - (long long)blk * per_full_block;
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

// P (bf16 pairs into pk) for 32 window columns and their sum into ls: a
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
    pk[jj / 2] = pack_bf16(p[0], p[1]);
    pk[jj / 2 + 1] = pack_bf16(p[2], p[3]);
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

// log2(e) / (|q| sqrt(d)) per token (0 for a zero row): the key
// normalisation and score scale, in the log2 units the softmax uses.
__global__ void key_scale_kernel(const __nv_bfloat16* __restrict__ Q, size_t n_tok,
                                 float* __restrict__ rn) {
  const size_t tok = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tok >= n_tok) return;
  float ssq = 0.f;
#pragma unroll
  for (int k = 0; k < kHeadDim; k += 8) {
    float x[8];
    load8(Q + tok * kHeadDim + k, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) ssq = fmaf(x[e], x[e], ssq);
  }
  rn[tok] = ssq > 0.f ? rsqrtf(ssq) * (0.125f * kLog2e) : 0.f;
}

__global__ void __launch_bounds__(kAtThreads, 1) attend_tc_kernel(AttnTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* slots = sm;
  uint8_t* acc_s = sm + kAtSlots * kAtSlotBytes;
  float4* ml_s = reinterpret_cast<float4*>(acc_s + kAtAccBytes);
  AtSmem& S = *reinterpret_cast<AtSmem*>(acc_s + kAtAccBytes + kAtMlBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kAtSlots; ++s) {
      tc::mbar_init(&S.full[s], 64);    // 32 producer lanes x (cp.async arrive + arrive)
      tc::mbar_init(&S.empty[s], 128);  // every thread of the warpgroup that used it
    }
    for (int w = 0; w < 2; ++w) {
      tc::mbar_init(&S.s_full[w], 1);
      tc::mbar_init(&S.p_full[w], 128);
      tc::mbar_init(&S.o_full[w], 1);
      tc::mbar_init(&S.tm_free[w], 128);
    }
    tc::mbar_init_fence();
    S.abort = 0;
    S.dep_bh = -1;
    S.dep_r = -1;
    S.pub_head = 0;
    S.n_total = 0xffffffffu;
    for (int i = 0; i < kAtPubRing; ++i) S.pub_seq[i] = 0;
  }
  if (warp == 9) {
    tc::tmem_alloc(&S.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  const size_t n_tok = (size_t)a.BH * a.L;
  unsigned* ticket_ctr = a.counters + (size_t)a.BH * a.R;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // The perm entries of tile n+2 are staged (cp.async) while tile n is
    // gathered, and the ticket of the next item is fetched one item ahead,
    // so neither latency sits on the gather path.
    struct Pt {
      long long item;
      int r, bh, t, t_end, done;
    };
    long long tk_pending = 0;  // lane 0: the ticket reserved for the next item
    if (lane == 0) tk_pending = (long long)atomicAdd(ticket_ctr, 1u);
    auto next_item = [&](Pt& p) {
      const long long tk = __shfl_sync(0xffffffffu, tk_pending, 0);
      if (lane == 0 && tk < a.n_items) tk_pending = (long long)atomicAdd(ticket_ctr, 1u);
      if (tk >= a.n_items) {
        p.done = 1;
        return;
      }
      p.item = tk;
      at_decode(a, tk, p.r, p.bh, p.t);
      p.t_end = min(p.t + a.tpi, a.n_tiles);
      p.done = 0;
    };
    auto advance = [&](const Pt& p) {
      Pt q = p;
      if (!p.done) {
        q.t = p.t + 1;
        if (q.t >= q.t_end) next_item(q);
      }
      return q;
    };
    // window slot u: chunk u/64 of (prev, k0, k0+1); absent chunks read kAtNoKey
    auto stage_perm = [&](const Pt& p, int st) {
      if (!p.done) {
        const size_t rowbase = ((size_t)p.r * a.BH + p.bh) * a.L;
        const int k0 = 2 * p.t;
        const int prev = (k0 == 0) ? a.n_chunks - 1 : k0 - 1;
        for (int piece = lane; piece < 48; piece += 32) {  // 16-byte pieces
          const int cw = piece >> 4;
          const int ch = cw == 0 ? prev : k0 + cw - 1;
          const bool present = (cw == 0) ? (a.n_chunks > 1) : (ch < a.n_chunks);
          uint32_t* dst = &S.perm_stage[st][cw * 64 + (piece & 15) * 4];
          if (present)
            tc::cp_async16(tc::smem_u32(dst), a.perm + rowbase + (size_t)ch * 64 + (piece & 15) * 4);
          else
            *reinterpret_cast<uint4*>(dst) = make_uint4(kAtNoKey, kAtNoKey, kAtNoKey, kAtNoKey);
        }
      }
      tc::cp_async_commit();
    };
    Pt q0;
    q0.item = 0; q0.r = 0; q0.bh = 0; q0.t = 0; q0.t_end = 0; q0.done = 0;
    next_item(q0);
    Pt q1 = advance(q0);
    stage_perm(q0, 0);
    stage_perm(q1, 1);
    int done_marks = 0;
    for (uint32_t n = 0;; ++n) {
      const int s = n % kAtSlots;
      const Pt cur = q0;
      if (n == 0) tc::cp_async_wait<1>(); else tc::cp_async_wait<2>();  // perm of tile n
      __syncwarp();
      const bool ok = __all_sync(0xffffffffu,
                                 at_wait(&S.empty[s], ((n / kAtSlots) & 1u) ^ 1u, &S.abort));
      if (!ok) break;
      if (cur.done) {
        // one end marker for each warpgroup (the issuing warp sees the first)
        if (lane == 0) {
          S.info[s].done = 1;
          S.info[s].seq = (int)n;
          if (done_marks == 0) st_release_cta(&S.n_total, n);
        }
        tc::fence_async_smem();
        cp_async_arrive_noinc(&S.full[s]);
        tc::mbar_arrive(&S.full[s]);
        tc::cp_async_commit();  // keep two groups per iteration
        tc::cp_async_commit();
        if (++done_marks == 2) break;
        continue;
      }
      uint32_t pos[6];
#pragma unroll
      for (int e = 0; e < 6; ++e) pos[e] = S.perm_stage[n % kAtSlots][lane + 32 * e];
      AtInfo inf;
      const int k0 = 2 * cur.t;
      inf.done = 0;
      inf.seq = (int)n;
      inf.r = cur.r;
      inf.bh = cur.bh;
      inf.t = cur.t;
      inf.first = (cur.t == (int)((cur.item % a.ipr) * a.tpi)) ? 1 : 0;
      inf.last = (cur.t + 1 == cur.t_end) ? 1 : 0;
      inf.nq = (k0 + 1 < a.n_chunks) ? 2 : 1;
      inf.has_prev = a.n_chunks > 1 ? 1 : 0;
      const size_t rowbase = ((size_t)cur.r * a.BH + cur.bh) * a.L;
      uint8_t* slot = slots + (size_t)s * kAtSlotBytes;
      const __nv_bfloat16* Qbh = a.Q + (size_t)cur.bh * a.L * 64;
      const __nv_bfloat16* Vbh = a.V + (size_t)cur.bh * a.L * 64;
      const float* rnbh = a.rn + (size_t)cur.bh * a.L;
      // slot metadata, lane-per-row: position, packed key, key scale
#pragma unroll
      for (int e = 0; e < 6; ++e) {
        const int u = lane + 32 * e;
        uint32_t p = pos[e];
        if (p != kAtNoKey && p >= (uint32_t)a.L) {  // not a permutation of the row
          record_status(kErrBadKeys);
          p = 0;
        }
        if (p != kAtNoKey) {
          S.pos[s][u] = p;
          cp_async4(tc::smem_u32(&S.key[s][u]), a.keys + rowbase + p);
          cp_async4(tc::smem_u32(&S.rn[s][u]), rnbh + p);
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
            const uint32_t p = pv[x];
            if (p != kAtNoKey) {
              tc::cp_async16(tc::smem_u32(qd), Qbh + (size_t)p * 64 + c * 8);
              tc::cp_async16(tc::smem_u32(vd), Vbh + (size_t)p * 64 + c * 8);
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
      // two tiles ahead: its ticket (if it starts an item) and perm entries
      q0 = q1;
      q1 = advance(q1);
      stage_perm(q1, (n + 2) % kAtSlots);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------ tensor-core issue
    if (lane == 0) {
      const uint32_t idesc_s = tc::idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_o = tc::idesc_bf16(128, 64, 0, 1);
      uint32_t n_s = 0, n_p = 0;  // next S to issue, next P.V to issue
      bool s_done = false;
      long long idle_since = clock64();
      for (;;) {
        bool progress = false;
        if (!s_done && n_s <= n_p + 1) {
          const int s = n_s % kAtSlots, w = n_s & 1;
          if (tc::mbar_probe(&S.full[s], (n_s / kAtSlots) & 1u)) {
            if (S.info[s].done) {
              s_done = true;
            } else if (tc::mbar_probe(&S.tm_free[w], ((n_s >> 1) & 1u) ^ 1u)) {
              tc::fence_after_sync();
              tc::fence_async_smem();  // cp.async rows of this slot -> tensor-core reads
              uint8_t* slot = slots + (size_t)s * kAtSlotBytes;
              const uint32_t qa = tc::smem_u32(slot + kAtChunkBytes);  // chunks k0, k0+1
              const uint32_t d = tmem + w * 256;
#pragma unroll
              for (int c = 0; c < 3; ++c) {
                const uint32_t kb = tc::smem_u32(slot + c * kAtChunkBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  tc::mma_bf16(d + c * 64, tc::sdesc_sw128(qa + kk * 32, 16, 1024),
                               tc::sdesc_sw128(kb + kk * 32, 16, 1024), idesc_s, kk > 0);
              }
              tc::mma_commit(&S.s_full[w]);
              ++n_s;
              progress = true;
            }
          }
        }
        if (n_p < n_s) {
          const int s = n_p % kAtSlots, w = n_p & 1;
          if (tc::mbar_probe(&S.p_full[w], (n_p >> 1) & 1u)) {
            tc::fence_after_sync();
            uint8_t* slot = slots + (size_t)s * kAtSlotBytes;
            const uint32_t pa = tmem + w * 256;  // P over S: key block c at columns 32c
#pragma unroll
            for (int c = 0; c < 3; ++c) {
              const uint32_t vb = tc::smem_u32(slot + (3 + c) * kAtChunkBytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16_ts(tmem + w * 256 + 192, pa + c * 32 + kk * 8,
                                tc::sdesc_sw128(vb + kk * 2048, 8192, 1024), idesc_o,
                                (c | kk) != 0);
            }
            tc::mma_commit(&S.o_full[w]);
            ++n_p;
            progress = true;
          }
        }
        if (s_done && n_p == n_s) break;
        if (progress) {
          idle_since = clock64();
        } else {
          __nanosleep(32);  // leave issue slots to the softmax warps on this SMSP
          if (*(volatile int*)&S.abort) break;
          if (clock64() - idle_since > tc::kSpinCycles) {
            record_status(tc::kErrTimeout);
            *(volatile int*)&S.abort = 1;
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 10) {
    // ------------------------------------------------------------ publisher
    // Online mode: makes each finished tile's stores visible device-wide and
    // counts it for its (head, round).  One fence covers every tile posted
    // since the last one, so fence latency never reaches the compute warps.
    if (a.online && lane == 0) {
      unsigned head = 0;
      long long idle_since = clock64();
      for (;;) {
        unsigned tail = head;
        while (ld_acquire_cta(&S.pub_seq[tail % kAtPubRing]) == tail + 1) ++tail;
        if (tail > head) {
          __threadfence();
          for (unsigned t = head; t < tail; ++t) {
            const int bh = S.pub_bh[t % kAtPubRing];
            if (bh >= 0) atomicAdd(a.counters + (size_t)bh * a.R + S.pub_r[t % kAtPubRing], 1u);
          }
          head = tail;
          st_release_cta(&S.pub_head, head);
          idle_since = clock64();
          continue;
        }
        if (head == ld_acquire_cta(&S.n_total)) break;  // every tile of this CTA published
        if (*(volatile int*)&S.abort) break;
        if (clock64() - idle_since > tc::kSpinCycles) {
          record_status(tc::kErrTimeout);
          *(volatile int*)&S.abort = 1;
          break;
        }
        __nanosleep(64);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------- softmax and epilogue
    const int w = warp >> 2;            // warpgroup
    const int m = tid & 127;            // query row = TMEM lane
    const int qc = m >> 6;              // query chunk within the tile
    const int wrow0 = (warp & 3) * 32;  // first row of this warp
    const uint32_t region = tmem + (uint32_t)w * 256 + ((uint32_t)wrow0 << 16);
    uint8_t* wg_acc = acc_s + (size_t)w * 128 * 256;  // this warpgroup's staging rows
    for (uint32_t j = 0;; ++j) {
      const uint32_t n = (uint32_t)w + 2 * j;
      const int s = n % kAtSlots;
      // slot s last held tile n - 3, the other warpgroup's: a parity wait
      // can pass on that older phase, so the slot's sequence number decides
      bool okf;
      const long long t_full = clock64();
      for (;;) {
        okf = at_wait(&S.full[s], (n / kAtSlots) & 1u, &S.abort);
        if (!okf || *(volatile int*)&S.info[s].seq == (int)n) break;
        if (clock64() - t_full > tc::kSpinCycles) {
          record_status(tc::kErrTimeout);
          *(volatile int*)&S.abort = 1;
          okf = false;
          break;
        }
      }
      const AtInfo inf = S.info[s];
      if (wg_or(w, !okf || inf.done)) break;

      if (a.online && inf.r >= 2) {
        // every tile of round r-2 of this head (the same running state) must
        // be folded in; the last (head, round) seen complete is cached so
        // later tiles skip the load
        bool waited = true;
        if (!(S.dep_bh == inf.bh && S.dep_r == inf.r)) {
          if (m == 0) {
            const unsigned* c = a.counters + (size_t)inf.bh * a.R + (inf.r - 2);
            const long long t0 = clock64();
            while (ld_acquire(c) < (unsigned)a.n_tiles) {
              if (*(volatile int*)&S.abort) { waited = false; break; }
              if (clock64() - t0 > tc::kSpinCycles) {
                record_status(tc::kErrTimeout);
                *(volatile int*)&S.abort = 1;
                waited = false;
                break;
              }
            }
            if (waited) { S.dep_bh = inf.bh; S.dep_r = inf.r; }
          }
        }
        if (wg_or(w, !waited)) break;
      }

      const bool valid = qc < inf.nq;
      const uint32_t ki = S.key[s][64 + m];
      const size_t tok = (size_t)inf.bh * a.L + S.pos[s][64 + m];
      const size_t bhL = (size_t)inf.bh * a.L;
      const bool fold = a.online && inf.r >= 2 && valid;  // uniform per warp
      // this round's running state (online mode)
      float* acc_o = a.acc_o + (size_t)(inf.r & 1) * n_tok * 64;
      float4* acc_ml = a.acc_ml + (size_t)(inf.r & 1) * n_tok;

      // running state of this warp's 32 rows: staged by cp.async while the
      // softmax runs, sixteen lanes per 256-byte row
      if (fold) {
#pragma unroll 2
        for (int i = 0; i < 16; ++i) {
          const int rr = wrow0 + 2 * i + (lane >> 4), q = lane & 15;
          const size_t t2 = bhL + S.pos[s][64 + rr];
          tc::cp_async16(tc::smem_u32(wg_acc + (size_t)rr * 256 + ((q ^ (rr & 15)) << 4)),
                         acc_o + t2 * 64 + 4 * q);
        }
        tc::cp_async16(tc::smem_u32(&ml_s[w * 128 + m]), acc_ml + tok);
      }
      tc::cp_async_commit();

      // scores of this row's two window chunks (qc, qc + 1), 64 columns at a
      // time.  Reference for the exponentials: the bound |q_i|/sqrt(d) on any
      // score (keys are unit vectors) instead of the row maximum, so one pass
      // suffices; a warp with a row whose bound exceeds kRefLimit (where
      // exp(score - bound) could underflow) takes the exact two-pass route.
      const bool oks = at_wait(&S.s_full[w], j & 1u, &S.abort);
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
      tc::mbar_arrive(&S.p_full[w]);
      const float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      const bool lone = !(lsum > 0.f);  // nothing but itself in this round
      const float mx = ref2 * (1.f / kLog2e);

      const bool oko = at_wait(&S.o_full[w], j & 1u, &S.abort);
      if (wg_or(w, !oko)) break;
      tc::fence_after_sync();
      tc::cp_async_wait<0>();  // this lane's staged pieces have landed
      __syncwarp();            // ... and the other lanes' (rows are shared)
      const float4 ml = fold ? ml_s[w * 128 + m] : make_float4(0.f, 0.f, 0.f, 0.f);

      // this round's (max, sum); a row with nothing but itself takes its value
      const float m_r = lone ? kSelfScore : mx;
      const float l_r = lone ? 1.f : lsum;
      float M = m_r, Lsum = l_r, ea = 0.f, eb = 1.f;
      if (fold) {
        M = fmaxf(ml.x, m_r);
        ea = __expf(ml.x - M);
        eb = __expf(m_r - M);
        Lsum = ml.y * ea + l_r * eb;
      }
      const float scale = !a.online ? 1.f / l_r : eb;
      const float scale_acc = ea;
      uint8_t* my_row = wg_acc + (size_t)m * 256;
      // O in two 32-column halves; the result goes back into this row's
      // staging space (fp32)
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        float o[32];
        tc::tmem_ld32(region + 192 + 32 * hh, o);
        tc::tmem_ld_wait();
        if (hh == 1) {  // this warpgroup's half of tensor memory is free again
          tc::fence_before_sync();
          tc::mbar_arrive(&S.tm_free[w]);
        }
        if (!valid) continue;
        if (lone) {
          const __nv_bfloat16* vs = a.V + tok * 64 + 32 * hh;
#pragma unroll
          for (int q = 0; q < 4; ++q) load8(vs + 8 * q, o + 8 * q);
        }
#pragma unroll
        for (int x = 0; x < 32; ++x) o[x] *= scale;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint8_t* piece = my_row + (((8 * hh + q) ^ (m & 15)) << 4);
          if (fold) {
            const float4 f = *reinterpret_cast<const float4*>(piece);
            o[4 * q] = fmaf(f.x, scale_acc, o[4 * q]);
            o[4 * q + 1] = fmaf(f.y, scale_acc, o[4 * q + 1]);
            o[4 * q + 2] = fmaf(f.z, scale_acc, o[4 * q + 2]);
            o[4 * q + 3] = fmaf(f.w, scale_acc, o[4 * q + 3]);
          }
          *reinterpret_cast<float4*>(piece) =
              make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
      }
      if (valid) {
        if (!a.online)
          a.lse_r[(size_t)inf.r * n_tok + tok] = lone ? kSelfScore : m_r + logf(l_r);
        else
          __stcg(acc_ml + tok, make_float4(M, Lsum, 0.f, 0.f));
      }
      __syncwarp();
      // the warp's 32 result rows (fp32) to their original positions,
      // sixteen lanes per 256-byte row
      if (valid) {
        float* base = !a.online ? a.o_part + (size_t)inf.r * n_tok * 64 : acc_o;
#pragma unroll 2
        for (int i = 0; i < 16; ++i) {
          const int rr = wrow0 + 2 * i + (lane >> 4), q = lane & 15;
          const size_t t2 = bhL + S.pos[s][64 + rr];
          const float4 f =
              *reinterpret_cast<const float4*>(wg_acc + (size_t)rr * 256 + ((q ^ (rr & 15)) << 4));
          if (!a.online) *reinterpret_cast<float4*>(base + t2 * 64 + 4 * q) = f;
          else __stcg(reinterpret_cast<float4*>(base + t2 * 64 + 4 * q), f);
        }
      }
      tc::mbar_arrive(&S.empty[s]);
      if (a.online) {
        // hand the finished tile to the publisher: every thread's stores are
        // ordered before the release below by this barrier
        if (wg_or(w, false)) break;
        if (m == 0) {
          const int k = n % kAtPubRing;
          bool room = true;
          const long long t0 = clock64();
          while (ld_acquire_cta(&S.pub_head) + kAtPubRing <= n) {  // ring full (never in practice)
            if (*(volatile int*)&S.abort || clock64() - t0 > tc::kSpinCycles) { room = false; break; }
          }
          if (!room) {
            record_status(tc::kErrTimeout);
            *(volatile int*)&S.abort = 1;
          }
          S.pub_bh[k] = inf.r + 2 < a.R ? (int)inf.bh : -1;  // rounds without a waiter
          S.pub_r[k] = inf.r;
          st_release_cta(&S.pub_seq[k], n + 1);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) tc::tmem_dealloc(tmem, 512);
}

// O and lse from the running states of the even and the odd rounds (online
// mode): M = max(M_0, M_1), L = sum_b L_b e^(M_b - M),
// O = sum_b acc_b e^(M_b - M) / L, lse = M + ln L.  Eight threads per token.
__global__ void online_merge_kernel(const float* __restrict__ acc_o,
                                    const float4* __restrict__ acc_ml, int nbuf, size_t n_tok,
                                    __nv_bfloat16* __restrict__ O, float* __restrict__ lse) {
  const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= n_tok * 8) return;
  const size_t tok = g >> 3;
  const int k = (int)(g & 7) * 8;
  const float4 m0 = acc_ml[tok];
  const float4 m1 = nbuf > 1 ? acc_ml[n_tok + tok] : make_float4(-INFINITY, 0.f, 0.f, 0.f);
  const float M = fmaxf(m0.x, m1.x);
  const float e0 = __expf(m0.x - M), e1 = nbuf > 1 ? __expf(m1.x - M) : 0.f;
  const float Lsum = m0.y * e0 + m1.y * e1;
  const float r = 1.f / Lsum;
  float a0[8], a1[8] = {0, 0, 0, 0, 0, 0, 0, 0}, o[8];
  load8(acc_o + tok * kHeadDim + k, a0);
  if (nbuf > 1) load8(acc_o + (n_tok + tok) * kHeadDim + k, a1);
#pragma unroll
  for (int x = 0; x < 8; ++x) o[x] = (a0[x] * e0 + a1[x] * e1) * r;
  store8(O + tok * kHeadDim + k, o);
  if (lse && k == 0) lse[tok] = M + logf(Lsum);
}

}  // namespace lsh
