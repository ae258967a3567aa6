// Backward of chunked shared-QK LSH attention on the 5th-generation tensor
// cores (bf16 inputs, d = 64, chunk = 64).  Buckets and permutations are
// constants of the backward pass.
//
// "Reformer explainer" (akshathtiwari.co.in/blog/reformer), chunked attention
// over sorted buckets and the union of hash rounds: every round's window
// entries taken together form one softmax per query over all rounds, so with
// the combined logsumexp lse_i of the forward pass and G_i = dO_i . O_i,
// entry (i, j) of any round has
//   P = exp(s_ij - lse_i),  dS = P (dO_i . v_j - G_i),
//   dv_j += P dO_i,  dq_i += dS khat_j / sqrt(d),  dkhat_j += dS q_i / sqrt(d),
// where khat_j = q_j / |q_j| (the shared-QK keys) and dQ = dq + (dkhat -
// khat (khat . dkhat)) / |q| per token.  Masked entries (another
// bucket, a later position, the token itself) have no dS; a token alone in
// every round gives its own value the weight 1/R in each round.
//
// Tile = two consecutive chunks k0, k0+1 of one (round, head) row: 128 query
// rows against a window of three chunks, 192 keys, as in the forward kernel.
// The window chunks are held in the order [w0, w2, w1] = [k0-1, k0+1, k0]
// (window column c, chunk c/64); the queries are columns 64..191, so TMEM
// lane m holds query column 64 + m: chunk k0+1 (q1) for m < 64, k0 (q0) for
// m >= 64.  Per tile (TMEM columns in brackets):
//   S   = Q[cols 64..191] . Q[cols 0..191]^T    [0, 192)      tcgen05.mma
//   dP  = dO[128 x 64] . V[cols 0..191]^T       [192, 384)    tcgen05.mma
//   P, dS per entry on the CUDA cores (one TMEM lane = one query row); P^T
//   and dS^T go to shared memory as MN-major operands, dS scaled by the key
//   normalisation goes to TMEM columns [416, 512) (bf16 pairs);
//   dQ  = dS' [128 x 192] . Q[cols 0..191]      [0, 64)       A from TMEM
//   dV1 = P^T[w0 ; w1 | q0] . dO[q0]            [64, 128)
//   dK1 = dS^T[w0 ; w1 | q0] . Q[q0]            [128, 192)
//   dV2 = P^T[w2 ; w1 | q1] . dO[q1]            [192, 256)
//   dK2 = dS^T[w2 ; w1 | q1] . Q[q1]            [256, 320)
// q0 sees w0, w1 and q1 sees w1, w2.  With this order every accumulator row
// of a token sits on one TMEM lane: lanes 64..127 hold w1 in dQ, dV1, dK1,
// dV2 and dK2, lanes 0..63 hold w2 in dQ, dV2, dK2 and w0 in dV1, dK1.  So
// the drain merges per lane, projects the key gradient onto the query
// (dq += (dkhat - khat (khat . dkhat)) / |q|, linear, so it can be applied
// per contribution) and adds two rows per token and tile (dq, dv) into the
// fp32 gradient buffers with vector reductions; they sum over tiles and
// rounds.
//
// Warp roles (352 threads):
//   warps 0-3, 4-7  two compute warpgroups; warpgroup 1 takes the w1 columns
//                   of every query row, warpgroup 0 the row's other window
//                   chunk (w0 for q0, w2 for q1); in the drain warpgroup 0
//                   forms the dq rows and warpgroup 1 the dv rows of the
//                   column-64+m tokens, and the other way round for the w0
//                   tokens of lanes 0..63.
//   warps 8, 9      producers: warp 8 + p gathers the CTA's tiles p, p + 2,
//                   ... (window q, v rows, packed keys, key scales; the
//                   queries' dO rows, lse and G) into shared-memory slot p.
//   warp 10         one thread issues the MMAs.
#pragma once

#include "attend_tc.cuh"

namespace lsh {

constexpr int kBwThreads = 352;
constexpr int kBwProducerWarp = 8;  // warps 8, 9
constexpr int kBwMmaWarp = 10;
constexpr int kBwSlots = 2;
constexpr int kBwChunkBytes = 64 * 128;                 // 64 rows of 128 B
constexpr int kBwSlotBytes = 8 * kBwChunkBytes;         // q x3, v x3, dO x2
constexpr int kBwOpBytes = 2 * 2 * kBwChunkBytes;       // one MN-major operand pair
// TMEM columns: S and dP during the softmax, dS' (bf16 pairs, A of the dQ
// product) in columns no softmax read touches, the five accumulators over S
// and dP once both are consumed.
constexpr uint32_t kBwColS = 0, kBwColDP = 192, kBwColDS = 416;
constexpr uint32_t kBwColDQ = 0, kBwColDV1 = 64, kBwColDK1 = 128, kBwColDV2 = 192,
                   kBwColDK2 = 256;

struct BwInfo {
  int r, bh, nq, has_prev, done;
};

struct BwSmem {
  uint32_t pos[kBwSlots][192];
  uint32_t key[kBwSlots][192];
  float rn[kBwSlots][192];
  float lse[kBwSlots][128];
  float G[kBwSlots][128];
  BwInfo info[kBwSlots];
  uint64_t full[kBwSlots], empty[kBwSlots];
  uint64_t s_full, p_full, o_full, tm_free;
  uint32_t tmem_base;
  int abort;
};

struct AttnBwdTcArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* V;
  const __nv_bfloat16* dO;
  const uint32_t* keys;
  const int32_t* perm;
  const float* rn;   // [n_tok] log2(e) / (|q| sqrt(d)), 0 for a zero row
  const float* lse;  // [n_tok] combined logsumexp of the forward pass
  const float* G;    // [n_tok] dO . O
  int L, R, BH, n_chunks, causal;
  int n_tiles;       // tiles per (round, head) row
  long long total_tiles;
  float inv_rounds;
  float* dq_acc;     // [n_tok][64] fp32, zeroed: dq with the dkhat projection added
  float* dv_acc;
};

__host__ __device__ inline size_t attend_bwd_tc_smem_bytes() {
  return 1024 + (size_t)kBwSlots * kBwSlotBytes + 2 * (size_t)kBwOpBytes + sizeof(BwSmem);
}

// OR of pred over the 256 compute threads (named barrier 1).
__device__ __forceinline__ bool bw_or(bool pred) {
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

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// dq row of one token from its accumulator rows on this lane:
//   dQ (query side, if has_q) + P(dK1 (if k1) + dK2 (if k2)),
//   P(x) = (x - khat (khat . x)) / |q| with khat = q / |q|,
// q = the token's bf16 row in shared memory (128B-swizzled), inv = 1/|q|.
// Sixteen columns at a time: two passes (the projection needs khat . x).
// Every accumulator is loaded and the absent ones are selected away (a
// conditional tcgen05.ld costs registers).
__device__ __forceinline__ void drain_dq(uint32_t region, bool has_q, bool k1, bool k2,
                                         const uint8_t* qrow, uint32_t qr, float inv, float* dst) {
  float dot = 0.f;  // q . (dK1 + dK2)
#pragma unroll 1
  for (int h = 0; h < 4; ++h) {
    float x[16], y[16];
    tc::tmem_ld16(region + kBwColDK1 + 16 * h, x);
    tc::tmem_ld16(region + kBwColDK2 + 16 * h, y);
    tc::tmem_ld_wait();
    tc::tmem_pin<16>(x);
    tc::tmem_pin<16>(y);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 w = *reinterpret_cast<const uint4*>(qrow + tc::sw128_offset(qr, 2 * h + q));
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
        const int j = 8 * q + 2 * e;
        const float a0 = (k1 ? x[j] : 0.f) + (k2 ? y[j] : 0.f);
        const float a1 = (k1 ? x[j + 1] : 0.f) + (k2 ? y[j + 1] : 0.f);
        dot = fmaf(f.x, a0, fmaf(f.y, a1, dot));
      }
    }
  }
  const float c = dot * inv * inv;  // khat (khat . x) = q (q . x) / |q|^2
#pragma unroll 1
  for (int h = 0; h < 4; ++h) {
    float x[16], y[16], z[16];
    tc::tmem_ld16(region + kBwColDK1 + 16 * h, x);
    tc::tmem_ld16(region + kBwColDK2 + 16 * h, y);
    tc::tmem_ld16(region + kBwColDQ + 16 * h, z);
    tc::tmem_ld_wait();
    tc::tmem_pin<16>(x);
    tc::tmem_pin<16>(y);
    tc::tmem_pin<16>(z);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 w = *reinterpret_cast<const uint4*>(qrow + tc::sw128_offset(qr, 2 * h + q));
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
      float o[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
        const int j = 8 * q + 2 * e;
        const float a0 = (k1 ? x[j] : 0.f) + (k2 ? y[j] : 0.f);
        const float a1 = (k1 ? x[j + 1] : 0.f) + (k2 ? y[j + 1] : 0.f);
        o[2 * e] = (has_q ? z[j] : 0.f) + (a0 - f.x * c) * inv;
        o[2 * e + 1] = (has_q ? z[j + 1] : 0.f) + (a1 - f.y * c) * inv;
      }
      red_add_v4(dst + 16 * h + 8 * q, o[0], o[1], o[2], o[3]);
      red_add_v4(dst + 16 * h + 8 * q + 4, o[4], o[5], o[6], o[7]);
    }
  }
}

// dv row of one token: dV1 (if v1) + dV2 (if v2) on this lane
__device__ __forceinline__ void drain_dv(uint32_t region, bool v1, bool v2, float* dst) {
#pragma unroll 1
  for (int h = 0; h < 4; ++h) {
    float x[16], y[16];
    tc::tmem_ld16(region + kBwColDV1 + 16 * h, x);
    tc::tmem_ld16(region + kBwColDV2 + 16 * h, y);
    tc::tmem_ld_wait();
    tc::tmem_pin<16>(x);
    tc::tmem_pin<16>(y);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = (v1 ? x[4 * q + e] : 0.f) + (v2 ? y[4 * q + e] : 0.f);
      red_add_v4(dst + 16 * h + 4 * q, o[0], o[1], o[2], o[3]);
    }
  }
}

// Per token, before the backward: G = dO . O, the key scale log2(e)/(|q|
// sqrt(d)) (0 for a zero row) and zeroed fp32 gradient rows.  Eight threads
// per token: 16 bytes of each input row, 32 bytes of each gradient row.
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ Q,
                                const __nv_bfloat16* __restrict__ O,
                                const __nv_bfloat16* __restrict__ dO, size_t n_tok,
                                float* __restrict__ G, float* __restrict__ rn,
                                float* __restrict__ dq_acc, float* __restrict__ dv_acc) {
  const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t tok = g >> 3;
  const int k = (int)(g & 7) * 8;
  const bool in = tok < n_tok;
  float ssq = 0.f, dot = 0.f;
  if (in) {
    float x[8], y[8];
    load8(Q + tok * kHeadDim + k, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) ssq = fmaf(x[e], x[e], ssq);
    load8(O + tok * kHeadDim + k, x);
    load8(dO + tok * kHeadDim + k, y);
#pragma unroll
    for (int e = 0; e < 8; ++e) dot = fmaf(x[e], y[e], dot);
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    store8(dq_acc + tok * kHeadDim + k, z);
    store8(dv_acc + tok * kHeadDim + k, z);
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
  }
  if (in && k == 0) {
    rn[tok] = ssq > 0.f ? rsqrtf(ssq) * (0.125f * kLog2e) : 0.f;
    G[tok] = dot;
  }
}

// dQ and dV from the fp32 gradient rows, eight consecutive values per thread.
template <typename OutT>
__global__ void bwd_cast_kernel(const float* __restrict__ dq_acc, const float* __restrict__ dv_acc,
                                size_t n, OutT* __restrict__ dQ, OutT* __restrict__ dV) {
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  float x[8];
  load8(dq_acc + i, x);
  store8(dQ + i, x);
  load8(dv_acc + i, x);
  store8(dV + i, x);
}

__global__ void __launch_bounds__(kBwThreads, 1) attend_bwd_tc_kernel(AttnBwdTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* slots = sm;
  uint8_t* opP = sm + kBwSlots * kBwSlotBytes;  // P^T: [query chunk][window atom][64 rows]
  uint8_t* opD = opP + kBwOpBytes;              // dS^T / sqrt(d), same layout
  BwSmem& S = *reinterpret_cast<BwSmem*>(opD + kBwOpBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kBwSlots; ++s) {
      tc::mbar_init(&S.full[s], 32);    // producer lanes
      tc::mbar_init(&S.empty[s], 256);  // compute threads
    }
    tc::mbar_init(&S.s_full, 1);
    tc::mbar_init(&S.p_full, 256);
    tc::mbar_init(&S.o_full, 1);
    tc::mbar_init(&S.tm_free, 256);
    tc::mbar_init_fence();
    S.abort = 0;
  }
  if (warp == kBwMmaWarp) {
    tc::tmem_alloc(&S.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;

  if (warp == kBwProducerWarp || warp == kBwProducerWarp + 1) {
    // ------------------------------------------------------------ producers
    // producer p fills slot p with the CTA's tiles p, p + 2, ...
    for (uint32_t n = (uint32_t)(warp - kBwProducerWarp);; n += kBwSlots) {
      const int s = n % kBwSlots;
      const long long tile = (long long)blockIdx.x + (long long)n * gridDim.x;
      if (!__all_sync(0xffffffffu, at_wait(&S.empty[s], ((n / kBwSlots) & 1u) ^ 1u, &S.abort)))
        break;
      if (tile >= a.total_tiles) {
        if (lane == 0) S.info[s].done = 1;
        tc::mbar_arrive(&S.full[s]);
        break;
      }
      // head-major order: the rounds of a head follow one another, so the
      // head's gradient rows stay in L2 while its rounds add into them
      const int per_head = a.R * a.n_tiles;
      const int bh = (int)(tile / per_head);
      const int rem = (int)(tile - (long long)bh * per_head);
      const int r = rem / a.n_tiles, t = rem % a.n_tiles;
      const int k0 = 2 * t;
      const int prev = (k0 == 0) ? a.n_chunks - 1 : k0 - 1;
      const int has_prev = a.n_chunks > 1 ? 1 : 0;
      const int nq = (k0 + 1 < a.n_chunks) ? 2 : 1;
      const size_t rowbase = ((size_t)r * a.BH + bh) * a.L;
      const size_t bhL = (size_t)bh * a.L;
      uint8_t* slot = slots + (size_t)s * kBwSlotBytes;
      // window column u: chunk u/64 of (prev, k0+1, k0); absent chunks read kAtNoKey
      uint32_t pe[6];  // all six loads in flight together
#pragma unroll
      for (int e = 0; e < 6; ++e) {
        const int u = lane + 32 * e, cw = u >> 6;
        const int ch = cw == 0 ? prev : (cw == 1 ? k0 + 1 : k0);
        const bool present = cw == 0 ? has_prev != 0 : (cw == 2 || nq == 2);
        pe[e] = present ? (uint32_t)__ldg(a.perm + rowbase + (size_t)ch * 64 + (u & 63)) : kAtNoKey;
      }
#pragma unroll
      for (int e = 0; e < 6; ++e) {
        const int u = lane + 32 * e;
        uint32_t p = pe[e];
        if (p != kAtNoKey && p >= (uint32_t)a.L) {  // not a permutation of the row
          record_status(kErrBadKeys);
          p = 0;
        }
        pe[e] = p;
        S.pos[s][u] = p;
        if (p != kAtNoKey) {
          cp_async4(tc::smem_u32(&S.key[s][u]), a.keys + rowbase + p);
          cp_async4(tc::smem_u32(&S.rn[s][u]), a.rn + bhL + p);
          if (u >= 64) {
            cp_async4(tc::smem_u32(&S.lse[s][u - 64]), a.lse + bhL + p);
            cp_async4(tc::smem_u32(&S.G[s][u - 64]), a.G + bhL + p);
          }
        } else {
          S.key[s][u] = kAtNoKey;
          S.rn[s][u] = 0.f;
          if (u >= 64) {
            S.lse[s][u - 64] = 0.f;
            S.G[s][u - 64] = 0.f;
          }
        }
      }
      __syncwarp();
      // q and v rows of the window, dO rows of the queries: eight lanes per
      // 128-byte row, four rows per warp instruction
      const __nv_bfloat16* Qbh = a.Q + bhL * 64;
      const __nv_bfloat16* Vbh = a.V + bhL * 64;
      const __nv_bfloat16* dObh = a.dO + bhL * 64;
      // window column u's position is pe[u / 32] of lane u % 32
#pragma unroll
      for (int i = 0; i < 48; ++i) {
        const int u = 4 * i + (lane >> 3), c = lane & 7;
        const uint32_t p = __shfl_sync(0xffffffffu, pe[i >> 3], u & 31);
        uint8_t* qd = slot + tc::sw128_offset(u, c);
        uint8_t* vd = slot + 3 * kBwChunkBytes + tc::sw128_offset(u, c);
        uint8_t* dd = slot + 6 * kBwChunkBytes + tc::sw128_offset(u - 64, c);
        if (p != kAtNoKey) {
          tc::cp_async16(tc::smem_u32(qd), Qbh + (size_t)p * 64 + c * 8);
          tc::cp_async16(tc::smem_u32(vd), Vbh + (size_t)p * 64 + c * 8);
          if (u >= 64) tc::cp_async16(tc::smem_u32(dd), dObh + (size_t)p * 64 + c * 8);
        } else {
          *reinterpret_cast<uint4*>(qd) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
          if (u >= 64) *reinterpret_cast<uint4*>(dd) = make_uint4(0, 0, 0, 0);
        }
      }
      if (lane == 0) {
        BwInfo inf;
        inf.r = r;
        inf.bh = bh;
        inf.nq = nq;
        inf.has_prev = has_prev;
        inf.done = 0;
        S.info[s] = inf;
      }
      // the rows land, become visible to the tensor cores' (async proxy)
      // reads, then the slot is published
      tc::cp_async_commit();
      tc::cp_async_wait<0>();
      tc::fence_async_smem();
      __syncwarp();
      tc::mbar_arrive(&S.full[s]);
    }
  } else if (warp == kBwMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_bf16(128, 192, 0, 0);
      const uint32_t id_q = tc::idesc_bf16(128, 64, 0, 1);
      const uint32_t id_k = tc::idesc_bf16(128, 64, 1, 1);
      for (uint32_t n = 0;; ++n) {
        const int s = n % kBwSlots;
        if (!at_wait(&S.full[s], (n / kBwSlots) & 1u, &S.abort)) break;
        if (S.info[s].done) break;
        const int nq = S.info[s].nq;
        if (!at_wait(&S.tm_free, (n & 1u) ^ 1u, &S.abort)) break;
        tc::fence_after_sync();
        const uint32_t sq = tc::smem_u32(slots + (size_t)s * kBwSlotBytes);
        // descriptors built once; the address field counts 16-byte units, so
        // the other pieces of an operand are constant offsets (C(x) = x / 16)
        const uint64_t kq = tc::sdesc_sw128(sq, 16, 1024);        // K-major rows of the slot
        const uint64_t mq = tc::sdesc_sw128(sq, 8192, 1024);      // MN-major view of the slot
        constexpr uint32_t CH = kBwChunkBytes >> 4, SV = 3 * CH, SDO = 6 * CH;
        // S = Q(window rows 64..191) . Qw^T,  dP = dO . Vw^T  (K-major, K = 64)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::mma_bf16(tmem + kBwColS, kq + CH + 2 * kk, kq + 2 * kk, id_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::mma_bf16(tmem + kBwColDP, kq + SDO + 2 * kk, kq + SV + 2 * kk, id_s, kk > 0);
        tc::mma_commit(&S.s_full);
        if (!at_wait(&S.p_full, n & 1u, &S.abort)) break;
        tc::fence_after_sync();
        // dQ = dS' (TMEM, 192 keys = 96 columns) . Qw (MN-major)
#pragma unroll
        for (int kk = 0; kk < 12; ++kk)
          tc::mma_bf16_ts(tmem + kBwColDQ, tmem + kBwColDS + kk * 8,
                          mq + (kk >> 2) * CH + (kk & 3) * 128, id_q, kk > 0);
        // key side: A = P^T / dS^T of one query chunk (two 64-key atoms,
        // MN-major), B = that chunk's dO / q rows (MN-major), K = 64 queries.
        // q0 = columns 128..191 (dO rows 64..127), q1 = columns 64..127.
        const uint64_t mp = tc::sdesc_sw128(tc::smem_u32(opP), kBwChunkBytes, 1024);
        const uint64_t md = tc::sdesc_sw128(tc::smem_u32(opD), kBwChunkBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          tc::mma_bf16(tmem + kBwColDV1, mp + 128 * kk, mq + SDO + CH + 128 * kk, id_k, kk > 0);
          tc::mma_bf16(tmem + kBwColDK1, md + 128 * kk, mq + 2 * CH + 128 * kk, id_k, kk > 0);
        }
        if (nq == 2) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            tc::mma_bf16(tmem + kBwColDV2, mp + 2 * CH + 128 * kk, mq + SDO + 128 * kk, id_k,
                         kk > 0);
            tc::mma_bf16(tmem + kBwColDK2, md + 2 * CH + 128 * kk, mq + CH + 128 * kk, id_k,
                         kk > 0);
          }
        }
        tc::mma_commit(&S.o_full);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ compute warpgroups
    const int g = warp >> 2;            // 1: the w1 columns; 0: the row's other chunk
    const int m = tid & 127;            // query row = TMEM lane = window column 64 + m
    const int qb = m >= 64 ? 0 : 1;     // query chunk: q0 (k0) or q1 (k0+1)
    const int qi = m & 63;              // K-row in that chunk's key-side operands
    const int cb = g == 1 ? 128 : (qb == 0 ? 0 : 64);  // first window column of this thread
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t region = tmem + lane_off;
    for (uint32_t n = 0;; ++n) {
      const int s = n % kBwSlots;
      const bool okf = at_wait(&S.full[s], (n / kBwSlots) & 1u, &S.abort);
      const BwInfo inf = S.info[s];
      if (bw_or(!okf || inf.done)) break;
      const bool valid = qb == 0 || inf.nq == 2;
      const bool active = valid && (g == 1 || qb == 1 || inf.has_prev);
      const uint32_t ki = S.key[s][64 + m];
      const uint32_t lo = ki - ki % (uint32_t)a.L;
      const uint32_t span = a.causal ? (ki - lo) : (uint32_t)a.L;
      const float lse_i = S.lse[s][m];
      const float lse2 = lse_i * kLog2e;
      const float G_i = S.G[s][m];
      const bool lone = valid && lse_i < kSelfScore + kLoneMargin;
      const bool oks = at_wait(&S.s_full, n & 1u, &S.abort);
      if (bw_or(!oks)) break;
      tc::fence_after_sync();

      // P^T / dS^T operand row: query chunk qb, atom g (w1 is atom 1), K-row qi
      uint8_t* prow = opP + qb * 2 * kBwChunkBytes + g * kBwChunkBytes;
      uint8_t* drow = opD + qb * 2 * kBwChunkBytes + g * kBwChunkBytes;
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        const int u0 = cb + 16 * blk;  // first window column of the block
        float sv[16], dp[16];
        tc::tmem_ld16(region + kBwColS + u0, sv);
        tc::tmem_ld16(region + kBwColDP + u0, dp);
        tc::tmem_ld_wait();
        tc::tmem_pin<16>(sv);
        tc::tmem_pin<16>(dp);
        uint32_t pp[8], pd[8], dsq[8];  // P, dS / sqrt(d), dS / (|q_j| sqrt(d)): bf16 pairs
        // the block's packed keys ascend: a row can have allowed columns in it
        // only if [key[u0], key[u0+15]] meets [lo, lo + span) (or its own
        // column is here and it is alone); a block no row of the warp uses is zero
        const bool any = (active && S.key[s][u0 + 15] >= lo && S.key[s][u0] < lo + span) ||
                         (lone && (uint32_t)(64 + m - u0) < 16u);
        const bool skip = !__any_sync(0xffffffffu, any);
#pragma unroll
        for (int x = 0; x < 8; ++x) { pp[x] = 0u; pd[x] = 0u; dsq[x] = 0u; }
#pragma unroll
        for (int jj = 0; jj < 16; jj += 4) {
          if (skip) break;
          const uint4 k4 = *reinterpret_cast<const uint4*>(&S.key[s][u0 + jj]);
          const float4 r4 = *reinterpret_cast<const float4*>(&S.rn[s][u0 + jj]);
          const uint32_t kj[4] = {k4.x, k4.y, k4.z, k4.w};
          const float rj[4] = {r4.x, r4.y, r4.z, r4.w};
          float pv[4], dv[4], qv[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            bool in = active && (kj[x] - lo) < span;
            if (!a.causal) in = in && kj[x] != ki;
            const float p = in ? ex2(sv[jj + x] * rj[x] - lse2) : 0.f;
            const float ds = p * (dp[jj + x] - G_i);
            pv[x] = p;
            dv[x] = ds * 0.125f;                    // dkhat side: dS / sqrt(d)
            qv[x] = ds * (rj[x] * (1.f / kLog2e));  // dq side: dS / (|q_j| sqrt(d))
          }
          if (lone) {  // only its own entry, with weight 1/R and no dS
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              pv[x] = (u0 + jj + x == 64 + m) ? a.inv_rounds : 0.f;
              dv[x] = 0.f;
              qv[x] = 0.f;
            }
          }
          pp[jj / 2] = pack_bf16(pv[0], pv[1]);
          pp[jj / 2 + 1] = pack_bf16(pv[2], pv[3]);
          pd[jj / 2] = pack_bf16(dv[0], dv[1]);
          pd[jj / 2 + 1] = pack_bf16(dv[2], dv[3]);
          dsq[jj / 2] = pack_bf16(qv[0], qv[1]);
          dsq[jj / 2 + 1] = pack_bf16(qv[2], qv[3]);
        }
        tc::tmem_st8(region + kBwColDS + u0 / 2, dsq);
        // 16-byte pieces 2blk, 2blk+1 of the 128-byte operand row
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t off = tc::sw128_offset(qi, 2 * blk + q);
          *reinterpret_cast<uint4*>(prow + off) =
              make_uint4(pp[4 * q], pp[4 * q + 1], pp[4 * q + 2], pp[4 * q + 3]);
          *reinterpret_cast<uint4*>(drow + off) =
              make_uint4(pd[4 * q], pd[4 * q + 1], pd[4 * q + 2], pd[4 * q + 3]);
        }
      }
      if (g == 1) {  // zeros for the window chunk outside the row's window (w2 / w0)
        uint32_t z[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) z[x] = 0u;
        tc::tmem_st32(region + kBwColDS + (qb == 0 ? 32 : 0), z);
      }
      tc::tmem_st_wait();
      tc::fence_async_smem();  // P^T, dS^T rows -> tensor-core reads
      tc::fence_before_sync();
      tc::mbar_arrive(&S.p_full);

      const bool oko = at_wait(&S.o_full, n & 1u, &S.abort);
      if (bw_or(!oko)) break;
      tc::fence_after_sync();
      // drain, merged per lane: lanes 64..127 hold the w1 token of column
      // 64 + m, lanes 0..63 the w2 token of column 64 + m and the w0 token of
      // column m
      const size_t bhL = (size_t)inf.bh * a.L;
      const bool two = inf.nq == 2;
      const uint8_t* qrows = slots + (size_t)s * kBwSlotBytes;
      const float inv_scale = 8.f / kLog2e;  // rn * 8 / log2(e) = 1 / |q|
#pragma unroll 1
      for (int rr = 0; rr < 2; ++rr) {  // at most two tokens per lane (warp-uniform)
        // rr 0: column 64 + m (w1 for q0 lanes, w2 for q1 lanes); rr 1: w0, column m
        const bool w1row = qb == 0;
        if (rr == 0 ? (!w1row && !two) : (w1row || !inf.has_prev)) continue;
        const uint32_t c = rr == 0 ? 64 + m : m;
        // accumulators holding this token on this lane
        const bool acc1 = rr == 1 || w1row;       // dV1 / dK1
        const bool acc2 = rr == 0 && (!w1row || two);  // dV2 / dK2
        // lanes 0..63 drain two tokens: warpgroup 0 takes the dq row of the
        // first and the dv row of the second, warpgroup 1 the others, so both
        // do one dq and one dv row there
        const bool dq_row = (g == 0) == (rr == 0);
        float* dst = (dq_row ? a.dq_acc : a.dv_acc) + (bhL + S.pos[s][c]) * 64;
        if (dq_row) drain_dq(region, rr == 0, acc1, acc2, qrows, c, S.rn[s][c] * inv_scale, dst);
        else drain_dv(region, acc1, acc2, dst);
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&S.tm_free);
      tc::mbar_arrive(&S.empty[s]);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kBwMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace lsh
