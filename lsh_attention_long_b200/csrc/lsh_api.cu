// C ABI of the LSH attention library (declared in include/lsh.h): argument
// checks, workspace carve-up and kernel dispatch.  The whole library is this
// one translation unit; the kernels live in the included headers.
#include "lsh.h"

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "attend_bwd_tc.cuh"
#include "attend_simt.cuh"
#include "attend_tc.cuh"
#include "common.cuh"
#include "ffn_tc.cuh"
#include "hash_simt.cuh"
#include "hash_tc.cuh"
#include "rev.cuh"
#include "sort.cuh"

// Scratch of lsh_attend_fwd_static: the per-round partials of rounds
// 0..R-2 for callers that cannot hand the library a workspace.  It is sized
// once, here, and shared by every call on the device.
static __device__ __align__(256) unsigned char g_static_scratch[LSH_STATIC_SCRATCH_BYTES];

namespace {

using lsh::kHeadDim;

constexpr size_t kAlign = 256;
constexpr int kMaxBuckets = 32768;
constexpr int kMaxChunk = 64;

inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

inline bool misaligned(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u); }

struct Dims {
  int B, H, L, d, nb, R, c, causal, dtype;
  size_t n_tok;  // B*H*L
  bool empty;
};

lsh_status check_shape(const lsh_shape* s, Dims* o) {
  if (!s) return LSH_ERR_INVALID_ARG;
  if (s->B < 0 || s->H < 0 || s->L < 0 || s->d <= 0 || s->n_rounds < 1 || s->chunk < 1)
    return LSH_ERR_INVALID_ARG;
  if (s->n_buckets < 1 || (s->n_buckets > 1 && (s->n_buckets & 1))) return LSH_ERR_INVALID_ARG;
  if (s->dtype != LSH_F32 && s->dtype != LSH_BF16) return LSH_ERR_INVALID_ARG;
  o->B = s->B; o->H = s->H; o->L = s->L; o->d = s->d; o->nb = s->n_buckets;
  o->R = s->n_rounds; o->c = s->chunk; o->causal = s->causal ? 1 : 0; o->dtype = s->dtype;
  o->n_tok = (size_t)s->B * s->H * s->L;
  o->empty = o->n_tok == 0;
  if (!o->empty && s->L % s->chunk) return LSH_ERR_INVALID_ARG;
  if (s->d != kHeadDim) return LSH_ERR_UNSUPPORTED;
  if (s->n_buckets > kMaxBuckets) return LSH_ERR_UNSUPPORTED;
  if (s->chunk > kMaxChunk) return LSH_ERR_UNSUPPORTED;
  if ((int64_t)s->n_buckets * s->L >= (int64_t(1) << 31)) return LSH_ERR_UNSUPPORTED;
  if ((int64_t)o->n_tok * s->n_rounds >= (int64_t(1) << 31)) return LSH_ERR_UNSUPPORTED;
  if ((int64_t)s->n_rounds * s->B * s->H > 65535) return LSH_ERR_UNSUPPORTED;  // grid.y
  return LSH_OK;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline lsh_status last_launch() {
  return cudaGetLastError() == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}

// Launches a kernel as a programmatic dependent of the previous grid in the
// stream: it may be scheduled while that grid finishes, and waits for it
// (grid_dep_wait) before the global accesses that depend on it.
template <typename... KArgs, typename... Args>
lsh_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess)
    return LSH_ERR_CUDA;
  return last_launch();
}

// Opt a kernel into more than 48 KB of dynamic shared memory.
template <typename K>
lsh_status allow_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return LSH_OK;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
                 cudaSuccess
             ? LSH_OK
             : LSH_ERR_CUDA;
}

// Tensor-core attention: bf16, d = 64, chunk = 64.
bool attend_tc_supported(const Dims& D) { return D.dtype == LSH_BF16 && D.c == 64; }

// Workspace of one lsh_attend_fwd call, given which optional outputs the
// caller supplies.
size_t attend_fwd_ws_bytes(const Dims& D, bool has_o_part, bool has_lse_r, bool has_O) {
  if (attend_tc_supported(D)) {
    // per-token key scales and fp16 values, then per-round partials the
    // caller does not take: fp16 outputs and fp32 logsumexps when the rounds
    // are combined here, none for a single combined round (written as O
    // directly)
    size_t b = align_up(D.n_tok * sizeof(float)) + align_up(D.n_tok * kHeadDim * sizeof(__half));
    if (has_O && !has_o_part && D.R == 1) return b;
    const size_t all = (size_t)D.R * D.n_tok;
    if (has_O && !has_o_part) b += align_up(all * kHeadDim * sizeof(__half));
    if (!has_lse_r) b += align_up(all * sizeof(float));
    return b;
  }
  if (!has_O) return 0;
  const size_t prev = (size_t)(D.R - 1) * D.n_tok;
  return (has_o_part ? 0 : align_up(prev * kHeadDim * sizeof(float))) +
         (has_lse_r ? 0 : align_up(prev * sizeof(float)));
}

size_t fwd_ws_bytes(const Dims& D) {
  size_t m = 0;
  for (int i = 0; i < 8; ++i) {
    const size_t b = attend_fwd_ws_bytes(D, i & 1, i & 2, i & 4);
    m = b > m ? b : m;
  }
  return m;
}

// G = dO . O and the key scales per token, then the dq, dkhat, dv accumulators
size_t bwd_ws_bytes(const Dims& D) {
  return 2 * align_up(D.n_tok * sizeof(float)) + 3 * align_up(D.n_tok * kHeadDim * sizeof(float));
}

lsh::AttnDims attn_dims(const Dims& D) {
  lsh::AttnDims a;
  a.B = D.B; a.H = D.H; a.L = D.L; a.chunk = D.c; a.n_chunks = D.L / D.c;
  a.causal = D.causal;
  a.W = a.n_chunks > 1 ? 2 * D.c : D.c;
  a.BH = D.B * D.H;
  return a;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

// cuTensorMapEncodeTiled, reached through the runtime so that the library
// does not link the driver library itself.
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_tiled() {
  static std::once_flag once;
  static EncodeTiled fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  });
  return fn;
}

// Row-major bf16 matrix [rows, cols] read in boxes of 64 columns x box_rows
// rows, 128-byte swizzled (the K-major operand layout of the MMA).
bool bf16_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
              uint32_t box_rows) {
  const EncodeTiled f = encode_tiled();
  if (!f) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t elem[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
           elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor-core hash: bf16, nb/2 a power of two in [16, 1024].
bool hash_tc_supported(const Dims& D) {
  const int half = D.nb / 2;
  return D.dtype == LSH_BF16 && half >= 16 && half <= 1024 && (half & (half - 1)) == 0;
}

lsh_status hash_tc_launch(const Dims& D, const void* Q, const void* rot, uint32_t* keys,
                          int32_t* buckets, cudaStream_t st) {
  lsh::HashTcArgs a;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.rot = static_cast<const __nv_bfloat16*>(rot);
  a.keys = keys;
  a.buckets = buckets;
  a.n_tok = (int)D.n_tok;
  a.L = D.L;
  a.half = D.nb / 2;
  a.R = D.R;
  // rounds whose rotation columns fit the shared-memory budget; when they
  // span more than one 256-column N-tile they must fill whole N-tiles
  int rg = lsh::kHashTcRotBytes / (a.half * 128);
  if (rg > D.R) rg = D.R;
  if (rg * a.half > 256) rg = (rg * a.half / 256) * 256 / a.half;
  if (rg < 1) rg = 1;
  a.rounds_per_group = rg;
  a.n_groups = (D.R + rg - 1) / rg;
  a.n_mtiles = (int)((D.n_tok + 127) / 128);
  int per = num_sms() / a.n_groups;
  if (per < 1) per = 1;
  if (per > a.n_mtiles) per = a.n_mtiles;
  a.ctas_per_group = per;
  const unsigned grid = (unsigned)(a.n_groups * per);
  // Q as [n_tok, 64] rows, read in 128-token boxes
  CUtensorMap mq;
  if (!bf16_map(&mq, Q, (uint64_t)D.n_tok, 64, 128)) return LSH_ERR_CUDA;
  // four epilogue warpgroups when every N-tile is 256 columns wide: rounds
  // of 256 or 512 columns, or of 128 in groups of an even number of rounds
  // (R even makes rg and the last group even)
  if ((a.half == 256 || a.half == 512 || (a.half == 128 && D.R % 2 == 0 && rg % 2 == 0)) &&
      rg * a.half >= 256) {
    const size_t smem4 = lsh::hash_tc4_smem_bytes(rg, a.half);
    lsh_status s0 = allow_smem(lsh::hash_tc4_kernel, smem4);
    if (s0 != LSH_OK) return s0;
    lsh::hash_tc4_kernel<<<grid, lsh::kHash4Threads, smem4, st>>>(mq, a);
    return last_launch();
  }
  const size_t smem = lsh::hash_tc_smem_bytes(rg, a.half);
  if (a.half >= 32) {
    lsh_status s0 = allow_smem(lsh::hash_tc_kernel<32>, smem);
    if (s0 != LSH_OK) return s0;
    lsh::hash_tc_kernel<32><<<grid, lsh::kHashTcThreads, smem, st>>>(mq, a);
  } else {
    lsh_status s0 = allow_smem(lsh::hash_tc_kernel<16>, smem);
    if (s0 != LSH_OK) return s0;
    lsh::hash_tc_kernel<16><<<grid, lsh::kHashTcThreads, smem, st>>>(mq, a);
  }
  return last_launch();
}

template <typename T>
lsh_status hash_launch(const Dims& D, const void* Q, const void* rot, uint32_t* keys,
                       int32_t* buckets, cudaStream_t st) {
  if (hash_tc_supported(D)) return hash_tc_launch(D, Q, rot, keys, buckets, st);
  constexpr int TOK = 128;
  const int half = D.nb / 2;
  const dim3 grid((unsigned)((D.n_tok + TOK - 1) / TOK), (unsigned)D.R);
  lsh::hash_simt_kernel<T, TOK><<<grid, TOK, 0, st>>>(
      static_cast<const T*>(Q), static_cast<const T*>(rot), keys, buckets, (int)D.n_tok, D.L, half);
  return last_launch();
}

lsh_status sort_launch(const Dims& D, const uint32_t* keys, int32_t* perm, cudaStream_t st) {
  const size_t budget = 200 * 1024;
  const size_t hist = (size_t)D.nb * sizeof(uint32_t);
  const size_t rows = (size_t)D.R * D.B * D.H;
  // two CTAs per row (a cluster) when the rows alone would leave most SMs
  // idle; the pair exchanges per-bucket totals, one more histogram of memory
  const int P = (rows * 2 <= (size_t)num_sms() && D.L >= 4096 && 2 * hist <= budget) ? 2 : 1;
  int nwarps = (int)((budget - (P > 1 ? hist : 0)) / hist);
  nwarps = nwarps > 32 ? 32 : nwarps;
  const int by_len = (D.L / P + 127) / 128;  // at least 4 steps of 32 per warp
  nwarps = nwarps > by_len ? by_len : nwarps;
  if (nwarps < 1) nwarps = 1;
  size_t smem = (size_t)(nwarps + (P > 1 ? 1 : 0)) * hist;
  // this CTA's bucket ids (u16), so that pass 2 reads no keys, when they fit
  const size_t part = ((((size_t)D.L + P - 1) / P) + 31) & ~(size_t)31;
  const int cache_ids = smem + part * 2 <= 220 * 1024 ? 1 : 0;
  if (cache_ids) smem += part * 2;
  lsh_status st0 = allow_smem(lsh::sort_rows_kernel, smem);
  if (st0 != LSH_OK) return st0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * P));
  cfg.blockDim = dim3((unsigned)(nwarps * 32));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, lsh::sort_rows_kernel, keys, perm, D.L, D.nb,
                         lsh::make_divl((uint32_t)D.L), cache_ids) != cudaSuccess)
    return LSH_ERR_CUDA;
  return last_launch();
}

// Test hook state (lsh_set_wait_test): the wait limit of the tensor-core
// attention kernel and the tile its producers withhold.
long long g_wait_limit = lsh::tc::kSpinCycles;
int g_hold_tile = -1;

lsh_status attend_tc_launch(const Dims& D, const void* Q, const void* V, const uint32_t* keys,
                            const int32_t* perm, float* o_part, float* lse_r, void* O,
                            float* lse, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (ws_bytes < attend_fwd_ws_bytes(D, o_part != nullptr, lse_r != nullptr, O != nullptr) ||
      !ws)
    return LSH_ERR_WORKSPACE;
  lsh::AttnTcArgs a;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.keys = keys;
  a.perm = perm;
  a.L = D.L;
  a.R = D.R;
  a.BH = D.B * D.H;
  a.n_chunks = D.L / 64;
  a.causal = D.causal;
  a.n_tiles = (a.n_chunks + 1) / 2;
  // items head by head, every round of a head before the next head: tiles
  // do not depend on one another, so the CTAs in flight share one or a few
  // heads' q and v rows, which stay in L2 across the rounds
  const int sms = num_sms();
  // tiles per item: a run of consecutive tiles shares window chunks, so
  // eight beat four unless they lengthen the tail (items go to CTAs
  // round-robin; the busiest CTA runs ceil(items / CTAs) of them)
  const auto busiest = [&](int t) {
    const long long items = (long long)D.R * a.BH * ((a.n_tiles + t - 1) / t);
    return (items + sms - 1) / sms * t;
  };
  a.tpi = busiest(8) <= busiest(4) ? 8 : 4;
  if (a.tpi > a.n_tiles) a.tpi = a.n_tiles;
  a.ipr = (a.n_tiles + a.tpi - 1) / a.tpi;
  a.heads_per_block = 1;
  a.n_items = (long long)a.R * a.BH * a.ipr;
  a.wait_limit = g_wait_limit;
  a.hold_tile = g_hold_tile;
  char* w = static_cast<char*>(ws);
  float* rn = reinterpret_cast<float*>(w);
  a.rn = rn;
  w += align_up(D.n_tok * sizeof(float));
  __half* v16 = reinterpret_cast<__half*>(w);
  a.V16 = v16;
  w += align_up(D.n_tok * kHeadDim * sizeof(__half));
  a.o16 = nullptr;
  a.o32 = o_part;
  a.lse_r = lse_r;
  a.O = nullptr;
  a.lse = nullptr;
  const size_t all = (size_t)D.R * D.n_tok;
  if (O && !o_part && D.R == 1) {  // one round: O and lse directly
    a.mode = lsh::kAtDirect;
    a.O = static_cast<__nv_bfloat16*>(O);
    a.lse = lse;
  } else {
    a.mode = o_part ? lsh::kAtPartial32 : lsh::kAtPartial16;
    if (!o_part) {
      a.o16 = reinterpret_cast<__half*>(w);
      w += align_up(all * kHeadDim * sizeof(__half));
    }
    if (!a.lse_r) a.lse_r = reinterpret_cast<float*>(w);
  }
  lsh::fwd_prep_kernel<<<(unsigned)((D.n_tok * 8 + 255) / 256), 256, 0, st>>>(
      a.Q, a.V, D.n_tok, rn, v16);
  if (last_launch() != LSH_OK) return LSH_ERR_CUDA;
  const size_t smem = lsh::attend_tc_smem_bytes();
  lsh_status s0 = allow_smem(lsh::attend_tc_kernel, smem);
  if (s0 != LSH_OK) return s0;
  const long long grid = a.n_items < sms ? a.n_items : sms;
  lsh::attend_tc_kernel<<<(unsigned)grid, lsh::kAtThreads, smem, st>>>(a);
  if (last_launch() != LSH_OK) return LSH_ERR_CUDA;
  if (O && a.mode != lsh::kAtDirect) {
    const size_t n8 = D.n_tok * 8;
    if (a.mode == lsh::kAtPartial16)
      {
        const unsigned nb8 = (unsigned)((n8 + 255) / 256);
        __nv_bfloat16* Ob = static_cast<__nv_bfloat16*>(O);
        switch (D.R) {
          case 2: lsh::combine16_kernel<2><<<nb8, 256, 0, st>>>(a.o16, a.lse_r, D.n_tok, Ob, lse); break;
          case 3: lsh::combine16_kernel<3><<<nb8, 256, 0, st>>>(a.o16, a.lse_r, D.n_tok, Ob, lse); break;
          case 4: lsh::combine16_kernel<4><<<nb8, 256, 0, st>>>(a.o16, a.lse_r, D.n_tok, Ob, lse); break;
          case 5: lsh::combine16_kernel<5><<<nb8, 256, 0, st>>>(a.o16, a.lse_r, D.n_tok, Ob, lse); break;
          case 6: lsh::combine16_kernel<6><<<nb8, 256, 0, st>>>(a.o16, a.lse_r, D.n_tok, Ob, lse); break;
          case 7: lsh::combine16_kernel<7><<<nb8, 256, 0, st>>>(a.o16, a.lse_r, D.n_tok, Ob, lse); break;
          case 8: lsh::combine16_kernel<8><<<nb8, 256, 0, st>>>(a.o16, a.lse_r, D.n_tok, Ob, lse); break;
          default:
            lsh::combine_kernel<__half, __nv_bfloat16><<<nb8, 256, 0, st>>>(a.o16, a.lse_r, D.R,
                                                                            D.n_tok, Ob, lse);
        }
      }
    else
      lsh::combine_kernel<float, __nv_bfloat16><<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(
          a.o32, a.lse_r, D.R, D.n_tok, static_cast<__nv_bfloat16*>(O), lse);
    return last_launch();
  }
  return LSH_OK;
}

template <typename T>
lsh_status attend_fwd_launch(const Dims& D, const void* Q, const void* V, const uint32_t* keys,
                             const int32_t* perm, float* o_part, float* lse_r, void* O, float* lse,
                             void* ws, size_t ws_bytes, cudaStream_t st) {
  if (attend_tc_supported(D))
    return attend_tc_launch(D, Q, V, keys, perm, o_part, lse_r, O, lse, ws, ws_bytes, st);
  const lsh::AttnDims a = attn_dims(D);
  const size_t smem = lsh::simt_fwd_smem_bytes(a.chunk, a.W);
  lsh_status s0 = allow_smem(lsh::attend_fwd_simt_kernel<T>, smem);
  if (s0 != LSH_OK) return s0;
  const T* q = static_cast<const T*>(Q);
  const T* v = static_cast<const T*>(V);
  if (!O) {
    const dim3 grid((unsigned)a.n_chunks, (unsigned)(D.R * a.BH));
    lsh::attend_fwd_simt_kernel<T><<<grid, 256, smem, st>>>(
        q, v, keys, perm, a, 0, o_part, lse_r, 0, D.R, nullptr, nullptr, nullptr, nullptr);
    return last_launch();
  }
  // partial buffers for rounds 0..R-2
  float* po = o_part;
  float* pl = lse_r;
  if (D.R > 1 && (!po || !pl)) {
    if (!ws || ws_bytes < attend_fwd_ws_bytes(D, po != nullptr, pl != nullptr, true))
      return LSH_ERR_WORKSPACE;
    char* w = static_cast<char*>(ws);
    const size_t prev = (size_t)(D.R - 1) * D.n_tok;
    if (!po) po = reinterpret_cast<float*>(w);
    if (!pl) pl = reinterpret_cast<float*>(w + align_up(prev * kHeadDim * sizeof(float)));
  }
  if (D.R > 1) {
    const dim3 grid((unsigned)a.n_chunks, (unsigned)((D.R - 1) * a.BH));
    lsh::attend_fwd_simt_kernel<T><<<grid, 256, smem, st>>>(
        q, v, keys, perm, a, 0, po, pl, 0, D.R, nullptr, nullptr, nullptr, nullptr);
    if (last_launch() != LSH_OK) return LSH_ERR_CUDA;
  }
  const dim3 grid((unsigned)a.n_chunks, (unsigned)a.BH);
  lsh::attend_fwd_simt_kernel<T><<<grid, 256, smem, st>>>(
      q, v, keys, perm, a, D.R - 1, o_part, lse_r, 1, D.R, po, pl, static_cast<T*>(O), lse);
  return last_launch();
}

template <typename T>
lsh_status combine_launch(const Dims& D, const float* o_part, const float* lse_r, void* O,
                          float* lse, cudaStream_t st) {
  const size_t n = D.n_tok * 8;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  lsh::combine_kernel<float, T><<<blocks, 256, 0, st>>>(o_part, lse_r, D.R, D.n_tok,
                                                        static_cast<T*>(O), lse);
  return last_launch();
}

// f32_out: dQ and dV are written as fp32 (for callers inside the library
// that add them up before any rounding), else in the shape's dtype.
template <typename T>
lsh_status attend_bwd_launch(const Dims& D, const void* Q, const void* V, const void* O,
                             const void* dO, const uint32_t* keys, const int32_t* perm,
                             const float* lse, void* dQ, void* dV, void* ws, size_t ws_bytes,
                             cudaStream_t st, bool f32_out = false) {
  if (!ws || ws_bytes < bwd_ws_bytes(D)) return LSH_ERR_WORKSPACE;
  const lsh::AttnDims a = attn_dims(D);
  char* w = static_cast<char*>(ws);
  const size_t tok_bytes = align_up(D.n_tok * sizeof(float));
  const size_t acc_bytes = align_up(D.n_tok * kHeadDim * sizeof(float));
  float* G = reinterpret_cast<float*>(w);
  float* rn = reinterpret_cast<float*>(w + tok_bytes);
  float* dq = reinterpret_cast<float*>(w + 2 * tok_bytes);
  float* dv = reinterpret_cast<float*>(reinterpret_cast<char*>(dq) + acc_bytes);
  float* dk = reinterpret_cast<float*>(reinterpret_cast<char*>(dv) + acc_bytes);
  // the tensor-core kernel projects dkhat into dq itself: no dk accumulator
  const bool tc_path = attend_tc_supported(D);
  const T* q = static_cast<const T*>(Q);
  const unsigned tb = (unsigned)((D.n_tok + 255) / 256);
  const unsigned tb8 = (unsigned)((D.n_tok * 8 + 255) / 256);  // eight threads per token
  if (tc_path) {
    // G, key scales and zeroed dq, dv rows in one pass
    lsh::bwd_prep_kernel<<<tb8, 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(Q), reinterpret_cast<const __nv_bfloat16*>(O),
        reinterpret_cast<const __nv_bfloat16*>(dO), D.n_tok, G, rn, dq, dv);
    if (last_launch() != LSH_OK) return LSH_ERR_CUDA;
    lsh::AttnBwdTcArgs b;
    b.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
    b.V = static_cast<const __nv_bfloat16*>(V);
    b.dO = static_cast<const __nv_bfloat16*>(dO);
    b.keys = keys;
    b.perm = perm;
    b.rn = rn;
    b.lse = lse;
    b.G = G;
    b.L = D.L;
    b.R = D.R;
    b.BH = D.B * D.H;
    b.n_chunks = D.L / D.c;
    b.causal = D.causal;
    b.n_tiles = (b.n_chunks + 1) / 2;
    b.total_tiles = (long long)D.R * b.BH * b.n_tiles;
    b.inv_rounds = 1.f / (float)D.R;
    b.dq_acc = dq;
    b.dv_acc = dv;
    const size_t smem = lsh::attend_bwd_tc_smem_bytes();
    lsh_status s0 = allow_smem(lsh::attend_bwd_tc_kernel, smem);
    if (s0 != LSH_OK) return s0;
    const long long sms = num_sms();
    const unsigned grid = (unsigned)(b.total_tiles < sms ? b.total_tiles : sms);
    lsh::attend_bwd_tc_kernel<<<grid, lsh::kBwThreads, smem, st>>>(b);
  } else {
    if (cudaMemsetAsync(dq, 0, 3 * acc_bytes, st) != cudaSuccess) return LSH_ERR_CUDA;
    lsh::bwd_dot_kernel<T><<<tb, 256, 0, st>>>(static_cast<const T*>(O),
                                               static_cast<const T*>(dO), D.n_tok, G);
    if (last_launch() != LSH_OK) return LSH_ERR_CUDA;
    const size_t smem = lsh::simt_bwd_smem_bytes(a.chunk, a.W);
    lsh_status s0 = allow_smem(lsh::attend_bwd_simt_kernel<T>, smem);
    if (s0 != LSH_OK) return s0;
    const dim3 grid((unsigned)a.n_chunks, (unsigned)(D.R * a.BH));
    lsh::attend_bwd_simt_kernel<T><<<grid, 256, smem, st>>>(
        q, static_cast<const T*>(V), static_cast<const T*>(dO), keys, perm, lse, G, a,
        1.f / (float)D.R, dq, dk, dv);
  }
  if (last_launch() != LSH_OK) return LSH_ERR_CUDA;
  if (tc_path) {  // the tensor-core kernel has already projected dkhat into dq
    const size_t n = D.n_tok * kHeadDim;
    if (f32_out)
      lsh::bwd_cast_kernel<float><<<tb8, 256, 0, st>>>(dq, dv, n, static_cast<float*>(dQ),
                                                       static_cast<float*>(dV));
    else
      lsh::bwd_cast_kernel<T><<<tb8, 256, 0, st>>>(dq, dv, n, static_cast<T*>(dQ),
                                                   static_cast<T*>(dV));
  } else if (f32_out) {
    lsh::bwd_finalize_kernel<T, float><<<tb, 256, 0, st>>>(q, dq, dk, dv, D.n_tok,
                                                           static_cast<float*>(dQ),
                                                           static_cast<float*>(dV));
  } else {
    lsh::bwd_finalize_kernel<T><<<tb, 256, 0, st>>>(q, dq, dk, dv, D.n_tok, static_cast<T*>(dQ),
                                                    static_cast<T*>(dV));
  }
  return last_launch();
}

// Device address of g_static_scratch per device, looked up on first use.
// In host code the symbol is only a handle; kernels must get this address.
constexpr int kMaxDevices = 64;
std::mutex g_static_mutex;
void* g_static_ptr[kMaxDevices] = {};

lsh_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LSH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return LSH_ERR_CUDA;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return LSH_OK;
}

}  // namespace

extern "C" {

size_t lsh_workspace_size(const lsh_shape* shape) {
  Dims D;
  if (check_shape(shape, &D) != LSH_OK || D.empty) return 0;
  const size_t f = fwd_ws_bytes(D), b = bwd_ws_bytes(D);
  return f > b ? f : b;
}

lsh_status lsh_hash(const lsh_shape* shape, const void* Q, const void* rot, uint32_t* keys,
                    int32_t* buckets, void* stream) {
  Dims D;
  lsh_status s = check_shape(shape, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!Q || !keys || (D.nb > 1 && !rot)) return LSH_ERR_INVALID_ARG;
  if (misaligned(Q) || misaligned(rot) || misaligned(keys) || misaligned(buckets))
    return LSH_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  return D.dtype == LSH_BF16 ? hash_launch<__nv_bfloat16>(D, Q, rot, keys, buckets, st)
                             : hash_launch<float>(D, Q, rot, keys, buckets, st);
}

lsh_status lsh_sort(const lsh_shape* shape, const uint32_t* keys, int32_t* perm, void* ws,
                    size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  Dims D;
  lsh_status s = check_shape(shape, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!keys || !perm || misaligned(keys) || misaligned(perm)) return LSH_ERR_INVALID_ARG;
  return sort_launch(D, keys, perm, as_stream(stream));
}

lsh_status lsh_attend_fwd(const lsh_shape* shape, const void* Q, const void* V,
                          const uint32_t* keys, const int32_t* perm, float* o_part, float* lse_r,
                          void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  Dims D;
  lsh_status s = check_shape(shape, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!Q || !V || !keys || !perm) return LSH_ERR_INVALID_ARG;
  if (!O && (!o_part || !lse_r)) return LSH_ERR_INVALID_ARG;
  if (misaligned(Q) || misaligned(V) || misaligned(keys) || misaligned(perm) ||
      misaligned(o_part) || misaligned(lse_r) || misaligned(O) || misaligned(lse) ||
      misaligned(ws))
    return LSH_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  return D.dtype == LSH_BF16
             ? attend_fwd_launch<__nv_bfloat16>(D, Q, V, keys, perm, o_part, lse_r, O, lse, ws,
                                                ws_bytes, st)
             : attend_fwd_launch<float>(D, Q, V, keys, perm, o_part, lse_r, O, lse, ws, ws_bytes,
                                        st);
}

lsh_status lsh_combine(const lsh_shape* shape, const float* o_part, const float* lse_r, void* O,
                       float* lse, void* stream) {
  Dims D;
  lsh_status s = check_shape(shape, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!o_part || !lse_r || !O) return LSH_ERR_INVALID_ARG;
  if (misaligned(o_part) || misaligned(lse_r) || misaligned(O) || misaligned(lse))
    return LSH_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  return D.dtype == LSH_BF16 ? combine_launch<__nv_bfloat16>(D, o_part, lse_r, O, lse, st)
                             : combine_launch<float>(D, o_part, lse_r, O, lse, st);
}

lsh_status lsh_forward(const lsh_shape* shape, const void* Q, const void* V, const void* rot,
                       uint32_t* keys, int32_t* buckets, int32_t* perm, void* O, float* lse,
                       void* ws, size_t ws_bytes, void* stream) {
  Dims D;
  lsh_status s = check_shape(shape, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!O || !lse || !perm) return LSH_ERR_INVALID_ARG;
  s = lsh_hash(shape, Q, rot, keys, buckets, stream);
  if (s != LSH_OK) return s;
  s = lsh_sort(shape, keys, perm, ws, ws_bytes, stream);
  if (s != LSH_OK) return s;
  return lsh_attend_fwd(shape, Q, V, keys, perm, nullptr, nullptr, O, lse, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// Forward from host buffers, pipelined over groups of heads
// ---------------------------------------------------------------------------

namespace {

// Heads per group: at least three groups when there are heads enough, so
// that copies in, kernels and copies out of neighbouring groups overlap.
int host_group_heads(const Dims& D) {
  const int BH = D.B * D.H;
  const int groups = BH >= 4 ? 4 : BH;
  return (BH + groups - 1) / groups;
}

// Heads of the group that starts at head h0.  Groups hold G heads, except the
// last G heads, which form two groups of half the size: what runs after the
// last copy in (its kernels and its copy out) is then half as long.
int host_group_size(int BH, int G, int h0) {
  const int tail = BH < G ? BH : G;
  const int tail_start = BH - tail;
  if (h0 < tail_start) return (tail_start - h0) < G ? tail_start - h0 : G;
  if (h0 == tail_start && tail >= 2) return (tail + 1) / 2;
  return BH - h0;
}

// Device buffer sets the groups rotate through: with three, the copy in of
// group i+1 never waits for the copy out of group i-1.
constexpr int kHostBufs = 3;

// One group's device buffers: Q, V, O, lse, keys, perm, the forward workspace.
struct HostGroupLayout {
  size_t q, v, o, lse, keys, perm, ws, ws_bytes, total;
};

HostGroupLayout host_group_layout(const Dims& D, int G) {
  Dims g = D;
  g.B = 1;
  g.H = G;
  g.n_tok = (size_t)G * D.L;
  const size_t elt = D.dtype == LSH_BF16 ? 2 : 4;
  HostGroupLayout l;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off += align_up(bytes); return at; };
  l.q = take(g.n_tok * D.d * elt);
  l.v = take(g.n_tok * D.d * elt);
  l.o = take(g.n_tok * D.d * elt);
  l.lse = take(g.n_tok * sizeof(float));
  l.keys = take((size_t)D.R * g.n_tok * sizeof(uint32_t));
  l.perm = take((size_t)D.R * g.n_tok * sizeof(int32_t));
  l.ws_bytes = fwd_ws_bytes(g);
  l.ws = take(l.ws_bytes);
  l.total = off;
  return l;
}

size_t rot_bytes(const Dims& D) {
  return D.nb > 1 ? (size_t)D.R * D.d * (D.nb / 2) * (D.dtype == LSH_BF16 ? 2 : 4) : 0;
}

// Two copy streams and the events of the pipeline, made once per device.
struct HostPipe {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t q_done[kHostBufs] = {}, v_done[kHostBufs] = {}, comp_done[kHostBufs] = {},
              out_done[kHostBufs] = {}, rot_done = nullptr;
  bool ready = false;
  // held while one call enqueues its copies, waits and kernels, so that the
  // events of concurrent calls from several host threads do not interleave
  std::mutex enqueue;
};
std::mutex g_pipe_mutex;
HostPipe g_pipe[kMaxDevices];

HostPipe* host_pipe() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  HostPipe& p = g_pipe[dev];
  if (!p.ready) {
    bool ok = cudaStreamCreateWithFlags(&p.up, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.down, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.rot_done, cudaEventDisableTiming) == cudaSuccess;
    for (int b = 0; b < kHostBufs && ok; ++b)
      ok = cudaEventCreateWithFlags(&p.q_done[b], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.v_done[b], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.comp_done[b], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.out_done[b], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return nullptr;
    p.ready = true;
  }
  return &p;
}

}  // namespace

size_t lsh_forward_host_ws_size(const lsh_shape* shape) {
  Dims D;
  if (check_shape(shape, &D) != LSH_OK || D.empty) return 0;
  const HostGroupLayout l = host_group_layout(D, host_group_heads(D));
  return align_up(rot_bytes(D)) + kHostBufs * l.total;
}

lsh_status lsh_forward_host(const lsh_shape* shape, const void* Q, const void* V, const void* rot,
                            void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  Dims D;
  lsh_status s = check_shape(shape, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!Q || !V || !O || (D.nb > 1 && !rot) || !ws) return LSH_ERR_INVALID_ARG;
  if (misaligned(ws)) return LSH_ERR_INVALID_ARG;
  const int G = host_group_heads(D);
  const HostGroupLayout l = host_group_layout(D, G);
  if (ws_bytes < align_up(rot_bytes(D)) + kHostBufs * l.total) return LSH_ERR_WORKSPACE;
  HostPipe* p = host_pipe();
  if (!p) return LSH_ERR_CUDA;
  std::lock_guard<std::mutex> hold(p->enqueue);
  cudaStream_t st = as_stream(stream);
  char* base = static_cast<char*>(ws) + align_up(rot_bytes(D));
  void* rot_d = ws;
  const size_t elt = D.dtype == LSH_BF16 ? 2 : 4;
  const size_t head_elems = (size_t)D.L * D.d;
  const int BH = D.B * D.H;
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // the copy streams start after the work already on `stream`
  if (!ok(cudaEventRecord(p->rot_done, st)) || !ok(cudaStreamWaitEvent(p->up, p->rot_done, 0)))
    return LSH_ERR_CUDA;
  if (rot_bytes(D) &&
      !ok(cudaMemcpyAsync(rot_d, rot, rot_bytes(D), cudaMemcpyHostToDevice, p->up)))
    return LSH_ERR_CUDA;
  int i = 0;
  for (int h0 = 0; h0 < BH; ++i) {
    const int b = i % kHostBufs;
    const int gh = host_group_size(BH, G, h0);
    char* d = base + (size_t)b * l.total;
    lsh_shape gs = *shape;
    gs.B = 1;
    gs.H = gh;
    const size_t bytes = gh * head_elems * elt;
    // copies in, after the copy out of the group that last used this buffer
    // set; q first, so that hashing and sorting overlap the copy of v
    if (i >= kHostBufs && !ok(cudaStreamWaitEvent(p->up, p->out_done[b], 0)))
      return LSH_ERR_CUDA;
    if (!ok(cudaMemcpyAsync(d + l.q, static_cast<const char*>(Q) + h0 * head_elems * elt, bytes,
                            cudaMemcpyHostToDevice, p->up)) ||
        !ok(cudaEventRecord(p->q_done[b], p->up)) ||
        !ok(cudaMemcpyAsync(d + l.v, static_cast<const char*>(V) + h0 * head_elems * elt, bytes,
                            cudaMemcpyHostToDevice, p->up)) ||
        !ok(cudaEventRecord(p->v_done[b], p->up)))
      return LSH_ERR_CUDA;
    // kernels on `stream`: the same calls as lsh_forward
    uint32_t* keys = reinterpret_cast<uint32_t*>(d + l.keys);
    int32_t* perm = reinterpret_cast<int32_t*>(d + l.perm);
    if (!ok(cudaStreamWaitEvent(st, p->q_done[b], 0))) return LSH_ERR_CUDA;
    s = lsh_hash(&gs, d + l.q, rot_d, keys, nullptr, st);
    if (s == LSH_OK) s = lsh_sort(&gs, keys, perm, d + l.ws, l.ws_bytes, st);
    if (s != LSH_OK) return s;
    if (!ok(cudaStreamWaitEvent(st, p->v_done[b], 0))) return LSH_ERR_CUDA;
    s = lsh_attend_fwd(&gs, d + l.q, d + l.v, keys, perm, nullptr, nullptr, d + l.o,
                       reinterpret_cast<float*>(d + l.lse), d + l.ws, l.ws_bytes, st);
    if (s != LSH_OK) return s;
    if (!ok(cudaEventRecord(p->comp_done[b], st))) return LSH_ERR_CUDA;
    // copies out
    if (!ok(cudaStreamWaitEvent(p->down, p->comp_done[b], 0)) ||
        !ok(cudaMemcpyAsync(static_cast<char*>(O) + h0 * head_elems * elt, d + l.o, bytes,
                            cudaMemcpyDeviceToHost, p->down)))
      return LSH_ERR_CUDA;
    if (lse && !ok(cudaMemcpyAsync(lse + (size_t)h0 * D.L, d + l.lse, gh * D.L * sizeof(float),
                                   cudaMemcpyDeviceToHost, p->down)))
      return LSH_ERR_CUDA;
    if (!ok(cudaEventRecord(p->out_done[b], p->down))) return LSH_ERR_CUDA;
    h0 += gh;
  }
  // the end of the work on `stream` waits for the last copies out
  for (int b = 0; b < kHostBufs && b < i; ++b)
    if (!ok(cudaStreamWaitEvent(st, p->out_done[b], 0))) return LSH_ERR_CUDA;
  return LSH_OK;
}

lsh_status lsh_attend_bwd(const lsh_shape* shape, const void* Q, const void* V, const void* O,
                          const void* dO, const uint32_t* keys, const int32_t* perm,
                          const float* lse, void* dQ, void* dV, void* ws, size_t ws_bytes,
                          void* stream) {
  Dims D;
  lsh_status s = check_shape(shape, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!Q || !V || !O || !dO || !keys || !perm || !lse || !dQ || !dV) return LSH_ERR_INVALID_ARG;
  if (misaligned(Q) || misaligned(V) || misaligned(O) || misaligned(dO) || misaligned(keys) ||
      misaligned(perm) || misaligned(lse) || misaligned(dQ) || misaligned(dV) || misaligned(ws))
    return LSH_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  return D.dtype == LSH_BF16
             ? attend_bwd_launch<__nv_bfloat16>(D, Q, V, O, dO, keys, perm, lse, dQ, dV, ws,
                                                ws_bytes, st)
             : attend_bwd_launch<float>(D, Q, V, O, dO, keys, perm, lse, dQ, dV, ws, ws_bytes,
                                        st);
}

lsh_status lsh_attend_fwd_static(const lsh_shape* shape, const void* Q, const void* V,
                                 const uint32_t* keys, const int32_t* perm, void* O, float* lse,
                                 void* stream) {
  Dims D;
  lsh_status s = check_shape(shape, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!Q || !V || !keys || !perm || !O) return LSH_ERR_INVALID_ARG;
  if (misaligned(Q) || misaligned(V) || misaligned(keys) || misaligned(perm) || misaligned(O) ||
      misaligned(lse))
    return LSH_ERR_INVALID_ARG;
  if (attend_fwd_ws_bytes(D, false, false, true) > LSH_STATIC_SCRATCH_BYTES)
    return LSH_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  s = static_scratch(&scratch);
  if (s != LSH_OK) return s;
  cudaStream_t st = as_stream(stream);
  return D.dtype == LSH_BF16
             ? attend_fwd_launch<__nv_bfloat16>(D, Q, V, keys, perm, nullptr, nullptr, O, lse,
                                                scratch, LSH_STATIC_SCRATCH_BYTES, st)
             : attend_fwd_launch<float>(D, Q, V, keys, perm, nullptr, nullptr, O, lse, scratch,
                                        LSH_STATIC_SCRATCH_BYTES, st);
}

// ---------------------------------------------------------------------------
// Chunked feed-forward
// ---------------------------------------------------------------------------

namespace {

lsh_status ffn_check(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk) {
  if (tokens < 0 || d_model <= 0 || d_ff <= 0 || chunk <= 0) return LSH_ERR_INVALID_ARG;
  if (d_model % lsh::kGmBN || d_ff % lsh::kGmBN || tokens % lsh::kGmBM || chunk % lsh::kGmBM)
    return LSH_ERR_UNSUPPORTED;
  if ((int64_t)tokens * d_model >= (int64_t(1) << 31) ||
      (int64_t)chunk * d_ff >= (int64_t(1) << 31))
    return LSH_ERR_UNSUPPORTED;
  return LSH_OK;
}

lsh::GemmArgs gemm_args(int M, int N, int K, int epi) {
  lsh::GemmArgs g = {};
  g.M = M; g.N = N; g.K = K; g.epi = epi; g.k_splits = 1;
  g.wait_limit = g_wait_limit;
  return g;
}

lsh_status gemm_launch(const CUtensorMap& ma, const CUtensorMap& mb, const lsh::GemmArgs& g,
                       cudaStream_t st) {
  const size_t smem = lsh::gemm_tc_smem_bytes();
  lsh_status s0 = allow_smem(lsh::gemm_tc_kernel, smem);
  if (s0 != LSH_OK) return s0;
  const int units = (g.M / lsh::kGmBM) * (g.N / lsh::kGmBN) * g.k_splits;
  const int sms = num_sms();
  return launch_pdl(lsh::gemm_tc_kernel, dim3((unsigned)(units < sms ? units : sms)),
                    dim3(lsh::kGmThreads), smem, st, ma, mb, g);
}

// K ranges per output tile for a weight-gradient product: enough work units
// to fill the SMs, each at least four K steps long.
int k_splits_for(int tiles, int K) {
  const int sms = num_sms();
  int ks = (sms + tiles - 1) / tiles;
  const int max_ks = (K / lsh::kGmBK) / 4;
  if (ks > max_ks) ks = max_ks;
  return ks < 1 ? 1 : ks;
}

}  // namespace

size_t lsh_ffn_ws_size(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk) {
  if (ffn_check(tokens, d_model, d_ff, chunk) != LSH_OK || tokens == 0) return 0;
  return align_up((size_t)chunk * d_ff * sizeof(__nv_bfloat16));
}

lsh_status lsh_ffn_forward(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk,
                           const void* X, const void* W1, const void* b1, const void* W2,
                           const void* b2, void* Y, void* ws, size_t ws_bytes, void* stream) {
  lsh_status s = ffn_check(tokens, d_model, d_ff, chunk);
  if (s != LSH_OK) return s;
  if (tokens == 0) return LSH_OK;
  if (!X || !W1 || !b1 || !W2 || !b2 || !Y || !ws) return LSH_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(W1) || misaligned(b1) || misaligned(W2) || misaligned(b2) ||
      misaligned(Y) || misaligned(ws))
    return LSH_ERR_INVALID_ARG;
  if (ws_bytes < (size_t)chunk * d_ff * sizeof(__nv_bfloat16)) return LSH_ERR_WORKSPACE;
  CUtensorMap mx, mw1, mh, mw2;
  if (!bf16_map(&mx, X, (uint64_t)tokens, (uint64_t)d_model, lsh::kGmBM) ||
      !bf16_map(&mw1, W1, (uint64_t)d_ff, (uint64_t)d_model, lsh::kGmBN) ||
      !bf16_map(&mh, ws, (uint64_t)chunk, (uint64_t)d_ff, lsh::kGmBM) ||
      !bf16_map(&mw2, W2, (uint64_t)d_model, (uint64_t)d_ff, lsh::kGmBN))
    return LSH_ERR_CUDA;
  cudaStream_t st = as_stream(stream);
  __nv_bfloat16* H = static_cast<__nv_bfloat16*>(ws);
  for (int c0 = 0; c0 < tokens; c0 += chunk) {
    const int n = tokens - c0 < chunk ? tokens - c0 : chunk;
    // H = max(0, X[c0 : c0+n] W1^T + b1): the chunk's hidden activation
    lsh::GemmArgs g1 = gemm_args(n, d_ff, d_model, lsh::kEpiBiasAct);
    g1.a_row0 = c0;
    g1.bias = static_cast<const __nv_bfloat16*>(b1);
    g1.relu = 1;
    g1.C = H; g1.ldc = d_ff;
    // after the first chunk, the grid before this one is the previous
    // chunk's second product, which reads H but writes nothing this product
    // loads (X and W1 were complete before the first chunk's wait returned):
    // only the stores into H must wait for it
    g1.late_wait = c0 > 0 ? 1 : 0;
    s = gemm_launch(mx, mw1, g1, st);
    if (s != LSH_OK) return s;
    // Y[c0 : c0+n] = H W2^T + b2
    lsh::GemmArgs g2 = gemm_args(n, d_model, d_ff, lsh::kEpiBiasAct);
    g2.bias = static_cast<const __nv_bfloat16*>(b2);
    g2.C = static_cast<__nv_bfloat16*>(Y) + (size_t)c0 * d_model; g2.ldc = d_model;
    s = gemm_launch(mh, mw2, g2, st);
    if (s != LSH_OK) return s;
  }
  return LSH_OK;
}

size_t lsh_ffn_bwd_ws_size(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk) {
  if (ffn_check(tokens, d_model, d_ff, chunk) != LSH_OK || tokens == 0) return 0;
  return 2 * align_up((size_t)chunk * d_ff * sizeof(__nv_bfloat16));
}

lsh_status lsh_ffn_backward(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk,
                            const void* X, const void* W1, const void* b1, const void* W2,
                            const void* dY, const float* R, float* dX, float* dW1, float* db1,
                            float* dW2, float* db2, void* ws, size_t ws_bytes, void* stream) {
  lsh_status s = ffn_check(tokens, d_model, d_ff, chunk);
  if (s != LSH_OK) return s;
  if (!X || !W1 || !b1 || !W2 || !dY || !dX || !dW1 || !db1 || !dW2 || !db2 || !ws)
    return LSH_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(W1) || misaligned(b1) || misaligned(W2) || misaligned(dY) ||
      misaligned(R) || misaligned(dX) || misaligned(dW1) || misaligned(db1) || misaligned(dW2) ||
      misaligned(db2) || misaligned(ws))
    return LSH_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  // the weight and bias gradients are sums over every position
  if (cudaMemsetAsync(dW1, 0, (size_t)d_ff * d_model * sizeof(float), st) != cudaSuccess ||
      cudaMemsetAsync(db1, 0, (size_t)d_ff * sizeof(float), st) != cudaSuccess ||
      cudaMemsetAsync(dW2, 0, (size_t)d_model * d_ff * sizeof(float), st) != cudaSuccess ||
      cudaMemsetAsync(db2, 0, (size_t)d_model * sizeof(float), st) != cudaSuccess)
    return LSH_ERR_CUDA;
  if (tokens == 0) return LSH_OK;
  const size_t hbytes = align_up((size_t)chunk * d_ff * sizeof(__nv_bfloat16));
  if (ws_bytes < 2 * hbytes) return LSH_ERR_WORKSPACE;
  __nv_bfloat16* H = static_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* dA = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + hbytes);
  // K-major operands read rows of K in 128-row (A) or 256-row (B) boxes;
  // MN-major operands read 64 x 64 boxes of [K][MN] storage
  CUtensorMap mx, mw1, mdy, mda, mw2_mn, mw1_mn, mdy_mn, mh_mn, mda_mn, mx_mn;
  const uint64_t T = (uint64_t)tokens, C = (uint64_t)chunk, D = (uint64_t)d_model,
                 F = (uint64_t)d_ff;
  if (!bf16_map(&mx, X, T, D, lsh::kGmBM) || !bf16_map(&mw1, W1, F, D, lsh::kGmBN) ||
      !bf16_map(&mdy, dY, T, D, lsh::kGmBM) || !bf16_map(&mda, dA, C, F, lsh::kGmBM) ||
      !bf16_map(&mw2_mn, W2, D, F, 64) || !bf16_map(&mw1_mn, W1, F, D, 64) ||
      !bf16_map(&mdy_mn, dY, T, D, 64) || !bf16_map(&mh_mn, H, C, F, 64) ||
      !bf16_map(&mda_mn, dA, C, F, 64) || !bf16_map(&mx_mn, X, T, D, 64))
    return LSH_ERR_CUDA;
  // Every launch below is a programmatic dependent of the one before.  A
  // grid completes only after its wait has returned, so when a grid is
  // launched every grid two or more launches back has completed, and a grid
  // whose loads read only inputs or such grids' outputs may load and multiply
  // at once and wait in its epilogue (late_wait).  Only dX = R + dA W1 loads
  // what its immediate predecessor writes.
  for (int c0 = 0; c0 < tokens; c0 += chunk) {
    const int n = tokens - c0 < chunk ? tokens - c0 : chunk;
    // H = max(0, X W1^T + b1), recomputed for the chunk
    lsh::GemmArgs g1 = gemm_args(n, d_ff, d_model, lsh::kEpiBiasAct);
    g1.a_row0 = c0;
    g1.bias = static_cast<const __nv_bfloat16*>(b1);
    g1.relu = 1;
    g1.C = H; g1.ldc = d_ff;
    g1.late_wait = c0 > 0 ? 1 : 0;  // its stores into H wait for the last chunk's readers
    if ((s = gemm_launch(mx, mw1, g1, st)) != LSH_OK) return s;
    // dA = (dY W2) where H > 0: the gradient at the pre-activation
    lsh::GemmArgs g2 = gemm_args(n, d_ff, d_model, lsh::kEpiMask);
    g2.a_row0 = c0;
    g2.b_mn = 1;  // W2 [d_model][d_ff] is [K][N]
    g2.mask = H; g2.ldm = d_ff;
    g2.C = dA; g2.ldc = d_ff;
    g2.late_wait = 1;  // loads dY and W2; its epilogue reads the mask H
    if ((s = gemm_launch(mdy, mw2_mn, g2, st)) != LSH_OK) return s;
    // dX = R + dA W1
    lsh::GemmArgs g3 = gemm_args(n, d_model, d_ff, lsh::kEpiAddF32);
    g3.b_mn = 1;  // W1 [d_ff][d_model] is [K][N]
    g3.C32 = dX + (size_t)c0 * d_model; g3.ldc32 = d_model;
    g3.R = R ? R + (size_t)c0 * d_model : nullptr; g3.ldr = d_model;
    if ((s = gemm_launch(mda, mw1_mn, g3, st)) != LSH_OK) return s;
    // dW2 += dY^T H, dW1 += dA^T X (positions are K, split over CTAs)
    lsh::GemmArgs g4 = gemm_args(d_model, d_ff, n, lsh::kEpiAtomicF32);
    g4.a_mn = 1; g4.b_mn = 1; g4.a_row0 = c0;
    g4.k_splits = k_splits_for((d_model / lsh::kGmBM) * (d_ff / lsh::kGmBN), n);
    g4.C32 = dW2; g4.ldc32 = d_ff;
    g4.late_wait = 1;  // loads dY and H (two launches back)
    if ((s = gemm_launch(mdy_mn, mh_mn, g4, st)) != LSH_OK) return s;
    lsh::GemmArgs g5 = gemm_args(d_ff, d_model, n, lsh::kEpiAtomicF32);
    g5.a_mn = 1; g5.b_mn = 1; g5.b_row0 = c0;
    g5.k_splits = k_splits_for((d_ff / lsh::kGmBM) * (d_model / lsh::kGmBN), n);
    g5.C32 = dW1; g5.ldc32 = d_model;
    g5.late_wait = 1;  // loads dA (three launches back) and X
    if ((s = gemm_launch(mda_mn, mx_mn, g5, st)) != LSH_OK) return s;
    // db2 += column sums of dY, db1 += column sums of dA
    const int rpb = 256;
    const dim3 gb2((unsigned)((d_model + 255) / 256), (unsigned)((n + rpb - 1) / rpb));
    if ((s = launch_pdl(lsh::colsum_add_kernel, gb2, dim3(256), 0, st,
                        static_cast<const __nv_bfloat16*>(dY) + (size_t)c0 * d_model, n,
                        d_model, rpb, db2)) != LSH_OK)
      return s;
    const dim3 gb1((unsigned)((d_ff + 255) / 256), (unsigned)((n + rpb - 1) / rpb));
    if ((s = launch_pdl(lsh::colsum_add_kernel, gb1, dim3(256), 0, st,
                        static_cast<const __nv_bfloat16*>(dA), n, d_ff, rpb, db1)) != LSH_OK)
      return s;
  }
  return LSH_OK;
}

// ---------------------------------------------------------------------------
// Reversible residual block around LSH attention
// ---------------------------------------------------------------------------

namespace {

struct RevLayout {
  size_t x2h, o, lse, y1b, g, dyb, dO, dq, dv, attn, ffn, total;
  size_t attn_bytes, ffn_bytes;
};

lsh_status rev_check(const lsh_shape* shape, int32_t d_ff, int32_t ffn_chunk, Dims* D) {
  lsh_status s = check_shape(shape, D);
  if (s != LSH_OK) return s;
  if (D->dtype != LSH_BF16) return LSH_ERR_UNSUPPORTED;
  return ffn_check(D->B * D->L, D->H * kHeadDim, d_ff, ffn_chunk);
}

RevLayout rev_layout(const lsh_shape* shape, const Dims& D, int32_t d_ff, int32_t ffn_chunk) {
  RevLayout l;
  const size_t n = D.n_tok * kHeadDim;  // elements of one activation
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off += align_up(bytes); return at; };
  l.x2h = take(n * 2);
  l.o = take(n * 2);
  l.lse = take(D.n_tok * sizeof(float));
  l.y1b = take(n * 2);
  l.g = take(n * 2);
  l.dyb = take(n * 2);
  l.dO = take(n * 2);
  l.dq = take(n * 4);  // the attention's input gradients in fp32
  l.dv = take(n * 4);
  l.attn_bytes = lsh_workspace_size(shape);
  l.attn = take(l.attn_bytes);
  const int T = D.B * D.L, Dm = D.H * kHeadDim;
  const size_t f = lsh_ffn_ws_size(T, Dm, d_ff, ffn_chunk),
               b = lsh_ffn_bwd_ws_size(T, Dm, d_ff, ffn_chunk);
  l.ffn_bytes = f > b ? f : b;
  l.ffn = take(l.ffn_bytes);
  l.total = off;
  return l;
}

inline unsigned blocks8(size_t n8) { return (unsigned)((n8 + 255) / 256); }

}  // namespace

size_t lsh_rev_ws_size(const lsh_shape* shape, int32_t d_ff, int32_t ffn_chunk) {
  Dims D;
  if (rev_check(shape, d_ff, ffn_chunk, &D) != LSH_OK || D.empty) return 0;
  return rev_layout(shape, D, d_ff, ffn_chunk).total;
}

lsh_status lsh_rev_forward(const lsh_shape* shape, int32_t d_ff, int32_t ffn_chunk,
                           const float* X1, const float* X2, const void* rot, const void* W1,
                           const void* b1, const void* W2, const void* b2, float* Y1, float* Y2,
                           uint32_t* keys, int32_t* perm, void* ws, size_t ws_bytes,
                           void* stream) {
  Dims D;
  lsh_status s = rev_check(shape, d_ff, ffn_chunk, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!X1 || !X2 || !Y1 || !Y2 || !keys || !perm || !ws || (D.nb > 1 && !rot))
    return LSH_ERR_INVALID_ARG;
  if (misaligned(X1) || misaligned(X2) || misaligned(Y1) || misaligned(Y2) || misaligned(ws))
    return LSH_ERR_INVALID_ARG;
  const RevLayout l = rev_layout(shape, D, d_ff, ffn_chunk);
  if (ws_bytes < l.total) return LSH_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  char* w = static_cast<char*>(ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(w + off); };
  const lsh::RevDims r{D.B, D.H, D.L};
  const size_t n8 = D.n_tok * 8;
  const int T = D.B * D.L, Dm = D.H * kHeadDim;
  // F: LSH attention of X2 (its own query, key and value), head-major bf16
  lsh::rev_to_heads_kernel<<<blocks8(n8), 256, 0, st>>>(r, X2, bf(l.x2h));
  if ((s = last_launch()) != LSH_OK) return s;
  s = lsh_forward(shape, bf(l.x2h), bf(l.x2h), rot, keys, nullptr, perm, bf(l.o),
                  reinterpret_cast<float*>(w + l.lse), w + l.attn, l.attn_bytes, stream);
  if (s != LSH_OK) return s;
  // Y1 = X1 + F(X2), and Y1 in bf16 for G
  lsh::rev_residual_heads_kernel<<<blocks8(n8), 256, 0, st>>>(r, X1, bf(l.o), 1.f, Y1, bf(l.y1b));
  if ((s = last_launch()) != LSH_OK) return s;
  // G: the chunked feed-forward of Y1; Y2 = X2 + G(Y1)
  s = lsh_ffn_forward(T, Dm, d_ff, ffn_chunk, bf(l.y1b), W1, b1, W2, b2, bf(l.g), w + l.ffn,
                      l.ffn_bytes, stream);
  if (s != LSH_OK) return s;
  lsh::rev_residual_kernel<<<blocks8(n8), 256, 0, st>>>(n8, X2, bf(l.g), 1.f, Y2, nullptr);
  return last_launch();
}

lsh_status lsh_rev_backward(const lsh_shape* shape, int32_t d_ff, int32_t ffn_chunk,
                            const float* Y1, const float* Y2, const float* dY1, const float* dY2,
                            const uint32_t* keys, const int32_t* perm, const void* W1,
                            const void* b1, const void* W2, const void* b2, float* X1, float* X2,
                            float* dX1, float* dX2, float* dW1, float* db1, float* dW2, float* db2,
                            void* ws, size_t ws_bytes, void* stream) {
  Dims D;
  lsh_status s = rev_check(shape, d_ff, ffn_chunk, &D);
  if (s != LSH_OK) return s;
  if (D.empty) return LSH_OK;
  if (!Y1 || !Y2 || !dY1 || !dY2 || !keys || !perm || !X1 || !X2 || !dX1 || !dX2 || !ws)
    return LSH_ERR_INVALID_ARG;
  if (misaligned(Y1) || misaligned(Y2) || misaligned(dY1) || misaligned(dY2) || misaligned(X1) ||
      misaligned(X2) || misaligned(dX1) || misaligned(dX2) || misaligned(ws))
    return LSH_ERR_INVALID_ARG;
  const RevLayout l = rev_layout(shape, D, d_ff, ffn_chunk);
  if (ws_bytes < l.total) return LSH_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  char* w = static_cast<char*>(ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(w + off); };
  float* lse = reinterpret_cast<float*>(w + l.lse);
  const lsh::RevDims r{D.B, D.H, D.L};
  const size_t n8 = D.n_tok * 8;
  const int T = D.B * D.L, Dm = D.H * kHeadDim;
  // X2 = Y2 - G(Y1), G recomputed from Y1
  lsh::rev_residual_kernel<<<blocks8(n8), 256, 0, st>>>(n8, Y1, nullptr, 0.f, nullptr, bf(l.y1b));
  if ((s = last_launch()) != LSH_OK) return s;
  s = lsh_ffn_forward(T, Dm, d_ff, ffn_chunk, bf(l.y1b), W1, b1, W2, b2, bf(l.g), w + l.ffn,
                      l.ffn_bytes, stream);
  if (s != LSH_OK) return s;
  lsh::rev_residual_kernel<<<blocks8(n8), 256, 0, st>>>(n8, Y2, bf(l.g), -1.f, X2, nullptr);
  lsh::rev_to_heads_kernel<<<blocks8(n8), 256, 0, st>>>(r, X2, bf(l.x2h));
  // dX1 = dY1 + G'(Y1)^T dY2, with G's parameter gradients
  lsh::rev_residual_kernel<<<blocks8(n8), 256, 0, st>>>(n8, dY2, nullptr, 0.f, nullptr, bf(l.dyb));
  if ((s = last_launch()) != LSH_OK) return s;
  s = lsh_ffn_backward(T, Dm, d_ff, ffn_chunk, bf(l.y1b), W1, b1, W2, bf(l.dyb), dY1, dX1, dW1,
                       db1, dW2, db2, w + l.ffn, l.ffn_bytes, stream);
  if (s != LSH_OK) return s;
  // X1 = Y1 - F(X2), F recomputed with the forward's buckets
  s = lsh_attend_fwd(shape, bf(l.x2h), bf(l.x2h), keys, perm, nullptr, nullptr, bf(l.o), lse,
                     w + l.attn, l.attn_bytes, stream);
  if (s != LSH_OK) return s;
  lsh::rev_residual_heads_kernel<<<blocks8(n8), 256, 0, st>>>(r, Y1, bf(l.o), -1.f, X1, nullptr);
  // dX2 = dY2 + F'(X2)^T dX1: the attention's query and value gradients
  lsh::rev_to_heads_kernel<<<blocks8(n8), 256, 0, st>>>(r, dX1, bf(l.dO));
  if ((s = last_launch()) != LSH_OK) return s;
  s = attend_bwd_launch<__nv_bfloat16>(D, bf(l.x2h), bf(l.x2h), bf(l.o), bf(l.dO), keys, perm,
                                       lse, w + l.dq, w + l.dv, w + l.attn, l.attn_bytes, st,
                                       true);
  if (s != LSH_OK) return s;
  lsh::rev_grad_x2_kernel<<<blocks8(n8), 256, 0, st>>>(r, dY2, reinterpret_cast<float*>(w + l.dq),
                                                       reinterpret_cast<float*>(w + l.dv), dX2);
  return last_launch();
}

lsh_status lsh_set_wait_test(int32_t hold_tile, int64_t wait_cycles) {
  if (wait_cycles < 0) return LSH_ERR_INVALID_ARG;
  g_wait_limit = wait_cycles > 0 ? (long long)wait_cycles : lsh::tc::kSpinCycles;
  g_hold_tile = hold_tile >= 0 ? hold_tile : -1;
  return LSH_OK;
}

lsh_status lsh_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return LSH_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, lsh::g_status, sizeof(int)) != cudaSuccess) return LSH_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(lsh::g_status, &zero, sizeof(int)) != cudaSuccess) return LSH_ERR_CUDA;
  return static_cast<lsh_status>(v);
}

const char* lsh_status_string(lsh_status status) {
  switch (status) {
    case LSH_OK: return "ok";
    case LSH_ERR_INVALID_ARG: return "invalid argument";
    case LSH_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case LSH_ERR_CUDA: return "CUDA error";
    case LSH_ERR_WORKSPACE: return "workspace missing or too small";
    case LSH_ERR_TIMEOUT: return "device wait timed out";
    case LSH_ERR_BAD_KEYS: return "keys are not bucket*L + position";
    case LSH_ERR_SCRATCH_LIMIT: return "problem exceeds the built-in scratch of lsh_attend_fwd_static";
  }
  return "unknown status";
}

}  // extern "C"
