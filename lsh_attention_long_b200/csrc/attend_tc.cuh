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
//   S  = Q[128 x 64] . K[192 x 64]^T   tcgen05.mma, three N=64 MMAs -> TMEM
//   P  = masked softmax numerators      CUDA cores, bf16 into shared memory
//   O  = P[128 x 192] . V[192 x 64]     tcgen05.mma -> TMEM
// The raw (unnormalised) queries serve as keys in the MMA; the key
// normalisation 1/|q_j| and 1/sqrt(d) scale the scores in the softmax, so
// the MMA multiplies exact bf16 inputs.
//
// Mask on packed keys (key = bucket*L + position, ascending within a bucket
// in position order): key_j is in the query's bucket and allowed iff
// (key_j - bucket_i*L) < span as unsigned, with span = key_i - bucket_i*L
// (causal: strictly earlier positions, which also drops the token itself) or
// L (non-causal, where key_j == key_i is dropped separately).  The token's
// own entry enters only when a row has no other key in any of its round's
// chunks: then the round's output is its own value and lse = -1e5.
//
// Warp roles: warps 0-7 (256 threads) compute; thread (wg, m) owns query row
// m and the window chunk kc = m/64 + wg, i.e. 64 of the row's 128 window
// columns; the two halves of a row meet through shared memory for the row
// max and sum.  Warp 8 gathers: row indices (perm), packed keys, and q, v
// rows (cp.async, 128B-swizzled) of the next tiles into a ring of 3 slots,
// signalling full/empty mbarriers.  Work comes from a global ticket
// (dynamic scheduling) in items of up to 4 tiles of one (round, head) row.
//
// Two output modes:
//   partial  every round's normalised o_r (fp32) and lse_r go to o_part /
//            lse_r at original positions (the combine runs afterwards);
//   online   rounds of a head are taken in order; each round's tile folds its
//            result into a running (max, sum, unnormalised output) per token
//            kept in the workspace, and the last round writes O (bf16) and
//            lse.  Items of round r of a head wait (bounded spin) until all
//            items of round r-1 of that head are done; tickets are taken in
//            an order where that dependency always points to earlier
//            tickets, so the scheme cannot deadlock.  Heads are processed in
//            blocks sized so that a block's accumulators and q, v rows stay
//            resident in L2 while its rounds run.
#pragma once

#include "tc.cuh"

namespace lsh {

constexpr int kAtSlots = 3;
constexpr int kAtConsumers = 256;
constexpr int kAtThreads = kAtConsumers + 32;
constexpr int kAtChunkBytes = 64 * 128;              // 64 rows of 128 B
constexpr int kAtSlotBytes = 6 * kAtChunkBytes;      // q then v of 3 chunks
constexpr int kAtPBytes = 3 * 128 * 128;             // P: 3 key blocks of 128 rows
constexpr uint32_t kAtNoKey = 0xffffffffu;           // never inside a bucket range
constexpr float kLog2e = 1.4426950408889634f;

struct AtInfo {
  int r, bh, t;
  int first, last;  // first / last tile of its item
  int done;
  int nq;           // query chunks present: 1 or 2
  int has_prev;     // window has a previous chunk (the row has > 1 chunk)
};

struct AttnTcArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* V;
  const uint32_t* keys;
  const int32_t* perm;
  int L, R, BH, n_chunks, causal;
  int n_tiles;       // tiles per row: ceil(n_chunks / 2)
  int tpi;           // tiles per item
  int ipr;           // items per (round, head) row
  int heads_per_block;
  long long n_items;
  int online;
  float* o_part;     // partial mode
  float* lse_r;
  float* acc_o;      // online mode: [n_tok][64] unnormalised output
  float2* acc_ml;    // online mode: [n_tok] (running max, running sum)
  __nv_bfloat16* O;  // online mode, last round
  float* lse;
  unsigned* counters;  // [BH][R] items done; then one ticket counter
};

// Shared memory beyond the 1024-aligned base.
struct AtSmem {
  uint32_t pos[kAtSlots][192];
  uint32_t key[kAtSlots][192];
  AtInfo info[kAtSlots];
  float rn[192];
  float red_max[2][128];
  float red_sum[2][128];
  uint64_t full[kAtSlots], empty[kAtSlots], bar_s, bar_o;
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ inline size_t attend_tc_smem_bytes() {
  return 1024 + (size_t)kAtSlots * kAtSlotBytes + kAtPBytes + sizeof(AtSmem);
}

// Named barrier over the 256 compute threads; returns the OR of `pred`.
__device__ __forceinline__ bool consumers_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, 256;" ::: "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar))
               : "memory");
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

__global__ void __launch_bounds__(kAtThreads, 1) attend_tc_kernel(AttnTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* slots = sm;
  uint8_t* pbuf = sm + kAtSlots * kAtSlotBytes;
  AtSmem& S = *reinterpret_cast<AtSmem*>(pbuf + kAtPBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kAtSlots; ++s) {
      tc::mbar_init(&S.full[s], 64);  // 32 producer lanes x (cp.async arrive + arrive)
      tc::mbar_init(&S.empty[s], 1);
    }
    tc::mbar_init(&S.bar_s, 1);
    tc::mbar_init(&S.bar_o, 1);
    tc::mbar_init_fence();
    S.abort = 0;
  }
  if (warp == 0) {
    tc::tmem_alloc(&S.tmem_base, 256);
    tc::tmem_relinquish();
  }
  // structural zeros of P: key block 0 for rows 64..127, block 2 for rows 0..63
  for (int e = tid; e < 64 * 8 * 2; e += blockDim.x) {
    const int half = e / 512, row = (e % 512) / 8 + (half ? 0 : 64), ch = e % 8;
    uint8_t* blk = pbuf + (half ? 2 : 0) * 16384;
    *reinterpret_cast<uint4*>(blk + tc::sw128_offset(row, ch)) = make_uint4(0, 0, 0, 0);
  }
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  const size_t n_tok = (size_t)a.BH * a.L;
  unsigned* ticket_ctr = a.counters + (size_t)a.BH * a.R;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    int s = 0;
    uint32_t empty_phase = 0;  // bit s: parity to wait for on empty[s]
    long long item = -1;
    int r = 0, bh = 0, t = 0, t_end = 0;
    for (;;) {
      int done = 0;
      if (t >= t_end) {  // next item
        long long tk = 0;
        if (lane == 0) tk = (long long)atomicAdd(ticket_ctr, 1u);
        tk = __shfl_sync(0xffffffffu, tk, 0);
        if (tk >= a.n_items) {
          done = 1;
        } else {
          item = tk;
          at_decode(a, item, r, bh, t);
          t_end = min(t + a.tpi, a.n_tiles);
        }
      }
      // wait until the consumers released this slot (first pass: free)
      const bool ok = __all_sync(0xffffffffu,
                                 tc::mbar_wait(&S.empty[s], ((empty_phase >> s) & 1u) ^ 1u));
      empty_phase ^= 1u << s;
      if (!ok || *(volatile int*)&S.abort) {
        if (lane == 0) { record_status(tc::kErrTimeout); S.abort = 1; }
        // still release the consumers waiting on this slot
        if (lane == 0) S.info[s].done = 1;
        tc::mbar_arrive(&S.full[s]);
        cp_async_arrive_noinc(&S.full[s]);
        break;
      }
      AtInfo inf;
      inf.done = done;
      if (!done) {
        const int k0 = 2 * t;
        inf.r = r; inf.bh = bh; inf.t = t;
        inf.first = (t == (int)((item % a.ipr) * a.tpi)) ? 1 : 0;
        inf.last = (t + 1 == t_end) ? 1 : 0;
        inf.nq = (k0 + 1 < a.n_chunks) ? 2 : 1;
        inf.has_prev = a.n_chunks > 1 ? 1 : 0;
        const size_t rowbase = ((size_t)r * a.BH + bh) * a.L;
        const int prev = (k0 == 0) ? a.n_chunks - 1 : k0 - 1;
        // window slot u in [0,192): chunk u/64 of (prev, k0, k0+1)
        uint32_t pos[6];
        bool present[6];
#pragma unroll
        for (int e = 0; e < 6; ++e) {
          const int u = lane + 32 * e;
          const int cw = u >> 6;
          const int ch = cw == 0 ? prev : k0 + cw - 1;
          present[e] = (cw == 0) ? (inf.has_prev != 0) : (ch < a.n_chunks);
          uint32_t p = 0;
          if (present[e]) {
            p = (uint32_t)a.perm[rowbase + (size_t)ch * 64 + (u & 63)];
            if (p >= (uint32_t)a.L) { record_status(kErrBadKeys); p = 0; }
          }
          pos[e] = p;
        }
        uint8_t* slot = slots + (size_t)s * kAtSlotBytes;
        const __nv_bfloat16* Qbh = a.Q + (size_t)bh * a.L * 64;
        const __nv_bfloat16* Vbh = a.V + (size_t)bh * a.L * 64;
#pragma unroll
        for (int e = 0; e < 6; ++e) {
          const int u = lane + 32 * e;
          const int cw = u >> 6, row = u & 63;
          S.pos[s][u] = pos[e];
          S.key[s][u] = present[e] ? a.keys[rowbase + pos[e]] : kAtNoKey;
          uint8_t* qd = slot + cw * kAtChunkBytes;
          uint8_t* vd = slot + (3 + cw) * kAtChunkBytes;
          if (present[e]) {
            const __nv_bfloat16* qs = Qbh + (size_t)pos[e] * 64;
            const __nv_bfloat16* vs = Vbh + (size_t)pos[e] * 64;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              tc::cp_async16(tc::smem_u32(qd + tc::sw128_offset(row, c)), qs + c * 8);
              tc::cp_async16(tc::smem_u32(vd + tc::sw128_offset(row, c)), vs + c * 8);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              *reinterpret_cast<uint4*>(qd + tc::sw128_offset(row, c)) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(vd + tc::sw128_offset(row, c)) = make_uint4(0, 0, 0, 0);
            }
          }
        }
        if (lane == 0) S.info[s] = inf;
        ++t;
      } else if (lane == 0) {
        S.info[s].done = 1;
      }
      tc::fence_async_smem();
      cp_async_arrive_noinc(&S.full[s]);
      tc::mbar_arrive(&S.full[s]);
      s = (s + 1 == kAtSlots) ? 0 : s + 1;
      if (done) break;
    }
  } else {
    // ------------------------------------------------------------ compute
    const int wg = tid >> 7;      // which half of the row's window
    const int m = tid & 127;      // query row = TMEM lane
    const int qc = m >> 6;        // query chunk within the tile
    const int kc = qc + wg;       // window chunk this thread scores
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t idesc_s = tc::idesc_bf16(128, 64, 0, 0);
    const uint32_t idesc_o = tc::idesc_bf16(128, 64, 0, 1);
    int s = 0;
    uint32_t full_phase = 0;
    uint32_t tile_n = 0;
    for (;;) {
      bool ok = tc::mbar_wait(&S.full[s], (full_phase >> s) & 1u);
      full_phase ^= 1u << s;
      if (consumers_or(!ok)) {
        if (tid == 0) { record_status(tc::kErrTimeout); S.abort = 1; }
        break;
      }
      const AtInfo inf = S.info[s];
      if (consumers_or(inf.done || *(volatile int*)&S.abort)) break;
      uint8_t* slot = slots + (size_t)s * kAtSlotBytes;

      // online mode: rounds of a head run in order
      if (a.online && inf.first && inf.r > 0) {
        bool waited = true;
        if (tid == 0) {
          const unsigned* c = a.counters + (size_t)inf.bh * a.R + (inf.r - 1);
          const long long t0 = clock64();
          while (ld_acquire(c) < (unsigned)a.ipr) {
            if (clock64() - t0 > tc::kSpinCycles) { waited = false; break; }
          }
        }
        if (consumers_or(!waited)) {
          if (tid == 0) { record_status(tc::kErrTimeout); S.abort = 1; }
          break;
        }
      }

      // S = Q . K^T (three window chunks)
      if (tid == 0) {
        tc::fence_after_sync();
        tc::fence_async_smem();  // cp.async rows of this slot -> tensor-core reads
        const uint32_t qa = tc::smem_u32(slot + kAtChunkBytes);  // chunks k0, k0+1
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const uint32_t kb = tc::smem_u32(slot + c * kAtChunkBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + c * 64, tc::sdesc_sw128(qa + kk * 32, 16, 1024),
                         tc::sdesc_sw128(kb + kk * 32, 16, 1024), idesc_s, kk > 0);
        }
        tc::mma_commit(&S.bar_s);
      }

      const bool valid = qc < inf.nq;
      const uint32_t my_pos = S.pos[s][64 + m];
      const uint32_t ki = S.key[s][64 + m];
      const size_t tok = (size_t)inf.bh * a.L + my_pos;

      // online mode: fetch this row's running state early (L2, not L1)
      float acc[32];
      float2 ml = make_float2(0.f, 0.f);
      if (a.online && inf.r > 0 && valid) {
        const float4* src = reinterpret_cast<const float4*>(a.acc_o + tok * 64 + wg * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 f = __ldcg(src + q);
          acc[4 * q] = f.x; acc[4 * q + 1] = f.y; acc[4 * q + 2] = f.z; acc[4 * q + 3] = f.w;
        }
        ml = __ldcg(a.acc_ml + tok);
      }

      // key scale 1 / (|q_j| sqrt(d)) of the 192 window rows
      if (tid < 192) {
        const uint8_t* qrow = slot + (tid >> 6) * kAtChunkBytes;
        const int row = tid & 63;
        float ssq = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(qrow + tc::sw128_offset(row, c));
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float2 f = __bfloat1622float2(h[x]);
            ssq = fmaf(f.x, f.x, ssq);
            ssq = fmaf(f.y, f.y, ssq);
          }
        }
        S.rn[tid] = ssq > 0.f ? rsqrtf(ssq) * 0.125f : 0.f;
      }
      consumers_sync();

      bool okw = tc::mbar_wait(&S.bar_s, tile_n & 1u);
      if (consumers_or(!okw)) {
        if (tid == 0) { record_status(tc::kErrTimeout); S.abort = 1; }
        break;
      }
      tc::fence_after_sync();

      // masked, scaled scores of this thread's 64 window columns
      float sv[64];
      tc::tmem_ld32(lane_addr + kc * 64, sv);
      tc::tmem_ld32(lane_addr + kc * 64 + 32, sv + 32);
      tc::tmem_ld_wait();
      const bool active = valid && (kc != 0 || inf.has_prev);
      const uint32_t lo = ki - ki % (uint32_t)a.L;
      const uint32_t span = a.causal ? (ki - lo) : (uint32_t)a.L;
      const uint32_t* kw = &S.key[s][kc * 64];
      const float* rw = &S.rn[kc * 64];
      float mloc = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; j += 4) {
        const uint4 k4 = *reinterpret_cast<const uint4*>(kw + j);
        const float4 r4 = *reinterpret_cast<const float4*>(rw + j);
        const uint32_t kj[4] = {k4.x, k4.y, k4.z, k4.w};
        const float rj[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          bool in = active && (kj[x] - lo) < span;
          if (!a.causal) in = in && kj[x] != ki;
          const float v = in ? sv[j + x] * rj[x] : -INFINITY;
          sv[j + x] = v;
          mloc = fmaxf(mloc, v);
        }
      }
      S.red_max[wg][m] = mloc;
      consumers_sync();
      const float mrow = fmaxf(S.red_max[0][m], S.red_max[1][m]);
      const bool lone = mrow == -INFINITY;  // nothing but itself in this round
      const float mb = lone ? 0.f : mrow * kLog2e;
      float lsum = 0.f;
      uint8_t* pblk = pbuf + kc * 16384;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float p0 = ex2(fmaf(sv[8 * c + 2 * x], kLog2e, -mb));
          const float p1 = ex2(fmaf(sv[8 * c + 2 * x + 1], kLog2e, -mb));
          lsum += p0 + p1;
          const __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
          w[x] = *reinterpret_cast<const uint32_t*>(&b);
        }
        *reinterpret_cast<uint4*>(pblk + tc::sw128_offset(m, c)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      S.red_sum[wg][m] = lsum;
      tc::fence_async_smem();
      tc::fence_before_sync();
      consumers_sync();
      const float lrow = S.red_sum[0][m] + S.red_sum[1][m];

      // O = P . V (192 keys)
      if (tid == 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const uint32_t pa = tc::smem_u32(pbuf + c * 16384);
          const uint32_t vb = tc::smem_u32(slot + (3 + c) * kAtChunkBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + 192, tc::sdesc_sw128(pa + kk * 32, 16, 1024),
                         tc::sdesc_sw128(vb + kk * 2048, 8192, 1024), idesc_o,
                         (c | kk) != 0);
        }
        tc::mma_commit(&S.bar_o);
      }
      okw = tc::mbar_wait(&S.bar_o, tile_n & 1u);
      if (consumers_or(!okw)) {
        if (tid == 0) { record_status(tc::kErrTimeout); S.abort = 1; }
        break;
      }
      tc::fence_after_sync();
      float o[32];
      tc::tmem_ld32(lane_addr + 192 + wg * 32, o);
      tc::tmem_ld_wait();

      if (valid) {
        // this round: max m_r, sum l_r, unnormalised output o (or the lone case)
        float m_r = mrow, l_r = lrow;
        if (lone) {
          m_r = kSelfScore;
          l_r = 1.f;
          const __nv_bfloat16* vs = a.V + tok * 64 + wg * 32;
#pragma unroll
          for (int q = 0; q < 4; ++q) load8(vs + 8 * q, o + 8 * q);
        }
        if (!a.online) {
          const size_t pr = (size_t)inf.r * n_tok + tok;
          const float inv = 1.f / l_r;
          float* dst = a.o_part + pr * 64 + wg * 32;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(dst + 4 * q) =
                make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv, o[4 * q + 3] * inv);
          if (wg == 0) a.lse_r[pr] = lone ? kSelfScore : m_r + logf(l_r);
        } else {
          float M = m_r, Lsum = l_r;
          if (inf.r > 0) {  // fold into the running state
            M = fmaxf(ml.x, m_r);
            const float ea = __expf(ml.x - M), eb = __expf(m_r - M);
            Lsum = ml.y * ea + l_r * eb;
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = fmaf(acc[x], ea, o[x] * eb);
          }
          if (inf.r + 1 < a.R) {
            float4* dst = reinterpret_cast<float4*>(a.acc_o + tok * 64 + wg * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              __stcg(dst + q, make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]));
            if (wg == 0) __stcg(a.acc_ml + tok, make_float2(M, Lsum));
          } else {
            const float inv = 1.f / Lsum;
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] *= inv;
            __nv_bfloat16* dst = a.O + tok * 64 + wg * 32;
#pragma unroll
            for (int q = 0; q < 4; ++q) store8(dst + 8 * q, o + 8 * q);
            if (wg == 0 && a.lse) a.lse[tok] = M + logf(Lsum);
          }
        }
      }
      tc::fence_before_sync();
      consumers_sync();
      if (tid == 0) {
        tc::mbar_arrive(&S.empty[s]);
        if (a.online && inf.last) {
          __threadfence();
          atomicAdd(a.counters + (size_t)inf.bh * a.R + inf.r, 1u);
        }
      }
      s = (s + 1 == kAtSlots) ? 0 : s + 1;
      ++tile_n;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

}  // namespace lsh
