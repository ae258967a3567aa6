/*
 * lsh.h -- C ABI of the B200 (sm_100a) shared-QK LSH attention library.
 *
 * The library implements Reformer's LSH attention as described in
 * "Reformer explainer" (akshathtiwari.co.in/blog/reformer, its single
 * section) and "Reformer: The Efficient Transformer" (codewithpapers.app
 * listing, abstract): tokens are hashed by the angular sector they fall
 * into after a random rotation, queries and keys are tied (shared-QK), tokens
 * are sorted by bucket and cut into equal chunks that attend to their
 * bucket-mates, and several hash rounds are unioned.  The exact arithmetic
 * is the five-step definition below:
 *
 *   1. hash     bucket = argmax([q.R_r ; -q.R_r]), R_r of shape [d, nb/2]
 *               (lowest index wins a tie), key = bucket*L + position;
 *   2. sort     stable sort of every (round, batch, head) row by
 *               (bucket, position);
 *   3. attend   chunks of `chunk` sorted slots attend to themselves and to the
 *               previous chunk (chunk 0 wraps to the last; a single chunk
 *               attends to itself once); keys are q/|q|, scores are scaled by
 *               1/sqrt(d); another bucket or (causal) a later position
 *               scores -inf, the token itself scores -1e5 (replacing its
 *               score), so it is used only when nothing else is left;
 *   4. scatter  each round's output o_r and logsumexp lse_r land at the
 *               token's original position;
 *   5. combine  lse = logsumexp_r lse_r,  O = sum_r exp(lse_r - lse) o_r.
 *
 * Conventions shared by every entry point
 *   - All tensors are dense, row-major DEVICE pointers owned by the caller.
 *     The library allocates nothing; scratch memory comes from the caller's
 *     workspace `ws` of `ws_bytes` bytes (see lsh_workspace_size).
 *   - Layouts: Q, V, O, dO, dQ, dV are [B, H, L, d] in the shape's dtype;
 *     rot is [n_rounds, d, n_buckets/2] in the same dtype; keys, buckets and
 *     perm are [n_rounds, B, H, L]; o_part is [n_rounds, B, H, L, d] fp32;
 *     lse_r is [n_rounds, B, H, L] fp32; lse is [B, H, L] fp32.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call is asynchronous on it.  Argument errors are returned before any
 *     launch; a launch failure returns LSH_ERR_CUDA.  Errors found by a
 *     kernel (malformed keys) are recorded in a device status word that
 *     lsh_device_status() reads.
 *   - Supported: d == 64; dtype LSH_F32 or LSH_BF16; n_buckets == 1 or an
 *     even number 2..32768; n_buckets * L < 2^31; B*H*L*n_rounds < 2^31;
 *     n_rounds*B*H <= 65535; chunk >= 1 divides L; chunk <= 64.  B, H or L
 *     equal to 0 is an empty call that returns LSH_OK without launching.
 *   - On the tensor-core path of the attention (bf16 and chunk == 64) the
 *     softmax weights and V enter the weights-times-values product in fp16:
 *     |V| must stay below 65504, and values below 2^-24 in magnitude count
 *     as zero there.
 *   - Every buffer must be 16-byte aligned.
 */
#ifndef LSH_ATTENTION_LSH_H_
#define LSH_ATTENTION_LSH_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LSH_API __attribute__((visibility("default")))
#else
#define LSH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LSH_OK = 0,
  LSH_ERR_INVALID_ARG = 1, /* null pointer, negative size, chunk not dividing L, ... */
  LSH_ERR_UNSUPPORTED = 2, /* valid but outside the supported set above */
  LSH_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
  LSH_ERR_WORKSPACE = 4,   /* ws is NULL or smaller than lsh_workspace_size() */
  LSH_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
  LSH_ERR_BAD_KEYS = 6,    /* keys not of the form bucket*L + position, bucket < n_buckets */
  LSH_ERR_SCRATCH_LIMIT = 7 /* problem too large for the library's built-in scratch array */
} lsh_status;

typedef enum { LSH_F32 = 0, LSH_BF16 = 1 } lsh_dtype;

typedef struct lsh_shape {
  int32_t B;         /* batch */
  int32_t H;         /* heads */
  int32_t L;         /* sequence length */
  int32_t d;         /* head dimension (64) */
  int32_t n_buckets; /* buckets per hash round */
  int32_t n_rounds;  /* hash rounds R */
  int32_t chunk;     /* chunk length c in sorted slots */
  int32_t causal;    /* nonzero: a later original position is masked */
  int32_t dtype;     /* lsh_dtype of Q, V, rot, O, dO, dQ, dV */
} lsh_shape;

/* Bytes of workspace that covers any call below for this shape (the largest
 * need: the per-round partials of lsh_attend_fwd when the caller passes no
 * o_part / lse_r, or the fp32 gradient accumulators of lsh_attend_bwd).
 * Returns 0 for an invalid or empty shape. */
LSH_API size_t lsh_workspace_size(const lsh_shape* shape);

/* Step 1 (hash).  For every round r and token (b, h, i):
 *   p = Q[b,h,i,:] . rot[r,:,:]   (fp32 accumulation of exact products for
 *                                  bf16; fp32 FMA for f32),
 *   bucket = first index of the maximum of [p ; -p],
 *   keys[r,b,h,i] = bucket*L + i.
 * Q: [B,H,L,d]; rot: [R,d,n_buckets/2] (ignored, may be NULL, when
 * n_buckets == 1); keys: [R,B,H,L] u32 (required); buckets: [R,B,H,L] i32
 * or NULL. */
LSH_API lsh_status lsh_hash(const lsh_shape* shape, const void* Q, const void* rot, uint32_t* keys,
                    int32_t* buckets, void* stream);

/* Step 2 (sort).  For every row (r, b, h), perm[r,b,h,t] = original position
 * at sorted slot t, with slots in ascending (bucket, position) order: a
 * stable counting sort on the bucket.  keys must be as lsh_hash writes them;
 * a malformed key records LSH_ERR_BAD_KEYS in the device status word.
 * ws is not used by the current kernels (may be NULL). */
LSH_API lsh_status lsh_sort(const lsh_shape* shape, const uint32_t* keys, int32_t* perm, void* ws,
                    size_t ws_bytes, void* stream);

/* Steps 3-5 (gather -> chunk attention -> scatter, with the combine).
 * Q, V: [B,H,L,d]; keys, perm: from lsh_hash / lsh_sort.
 * o_part: [R,B,H,L,d] fp32 or NULL; lse_r: [R,B,H,L] fp32 or NULL.
 * O: [B,H,L,d] in dtype, or NULL to skip the combine (then o_part and lse_r
 * are required and receive every round).  lse: [B,H,L] fp32 or NULL.
 * When O is given, the rounds are combined into O and lse (fp32 o_part
 * and lse_r receive every round when given).  Scratch comes from ws
 * (ws_bytes >= lsh_workspace_size()): on the tensor-core path (bf16, chunk
 * 64) the per-token key scales, the values in fp16 and, unless the caller
 * takes o_part or there is one round, every round's fp16 output and fp32
 * logsumexp, which a combine kernel then reads; on the CUDA-core path the
 * partials of rounds 0..R-2, combined in the epilogue of the last round. */
LSH_API lsh_status lsh_attend_fwd(const lsh_shape* shape, const void* Q, const void* V,
                          const uint32_t* keys, const int32_t* perm, float* o_part,
                          float* lse_r, void* O, float* lse, void* ws, size_t ws_bytes,
                          void* stream);

/* Step 5 alone: O = sum_r exp(lse_r - lse) o_part[r], lse = logsumexp_r lse_r.
 * o_part [R,B,H,L,d] fp32, lse_r [R,B,H,L] fp32 -> O [B,H,L,d] dtype,
 * lse [B,H,L] fp32 (or NULL). */
LSH_API lsh_status lsh_combine(const lsh_shape* shape, const float* o_part, const float* lse_r, void* O,
                       float* lse, void* stream);

/* Whole forward in one call: lsh_hash -> lsh_sort -> lsh_attend_fwd with the
 * combine.  keys and perm are outputs (they are also what the backward
 * needs); buckets may be NULL; lse [B,H,L] fp32 is required (the backward
 * needs it).  ws_bytes >= lsh_workspace_size(). */
LSH_API lsh_status lsh_forward(const lsh_shape* shape, const void* Q, const void* V, const void* rot,
                       uint32_t* keys, int32_t* buckets, int32_t* perm, void* O, float* lse,
                       void* ws, size_t ws_bytes, void* stream);

/* Whole forward from host memory: Q, V [B,H,L,d] and rot [R,d,n_buckets/2]
 * (dtype) are host buffers; O [B,H,L,d] (dtype) and lse [B,H,L] fp32 (or
 * NULL) are written to host buffers.  Page-locked host buffers let the
 * copies run asynchronously: the heads are processed in groups (the last
 * group split in two), rotating through three device buffer sets, and the
 * host-to-device copy of one group, the kernels of the one before and the
 * device-to-host copy of the one before that overlap; a group's hashing and
 * sorting start once its Q has arrived, while its V is still in flight (two
 * internal streams, made once per device; every step is ordered before the
 * end of the work on `stream`, so synchronising `stream` covers the copies
 * too).  Same
 * arithmetic as lsh_forward, head by head.  ws is device scratch of at least
 * lsh_forward_host_ws_size() bytes, owned by the caller; nothing is
 * allocated.  Keys and permutations are not returned.  The internal streams
 * and events are shared by every call on a device: calls from several host
 * threads take turns to enqueue their work (a per-device lock), and the
 * copies of all calls on a device run in call order on those streams.  Calls
 * that run at the same time need separate ws and output buffers. */
LSH_API size_t lsh_forward_host_ws_size(const lsh_shape* shape);
LSH_API lsh_status lsh_forward_host(const lsh_shape* shape, const void* Q, const void* V,
                            const void* rot, void* O, float* lse, void* ws, size_t ws_bytes,
                            void* stream);

/* Backward of steps 3-5 with buckets and permutations held constant.
 * Given the forward's O [B,H,L,d] and lse [B,H,L] and the upstream gradient
 * dO [B,H,L,d], writes dQ and dV [B,H,L,d] in dtype.  dQ includes the path
 * through the key normalisation q/|q|.  Masked entries (another bucket, a
 * later position, the token itself) carry no score gradient; the token's own
 * value still receives the weight it was given.  ws_bytes >=
 * lsh_workspace_size(). */
LSH_API lsh_status lsh_attend_bwd(const lsh_shape* shape, const void* Q, const void* V, const void* O,
                          const void* dO, const uint32_t* keys, const int32_t* perm,
                          const float* lse, void* dQ, void* dV, void* ws, size_t ws_bytes,
                          void* stream);

/* lsh_attend_fwd with the combine, for callers that cannot allocate memory.
 *
 * No passage of the pages corresponds to this entry point; it exists for
 * deployment.  Some callers may not call cudaMalloc at the moment they run
 * attention: a host framework whose memory planner owns every device buffer,
 * a plugin inside another runtime's execution phase, or a latency-critical
 * loop where an allocation would synchronise the device.  This call takes
 * the same inputs and outputs as lsh_attend_fwd with O given (Q, V, keys,
 * perm -> O, lse) but no workspace: the attention's scratch lives in an
 * array of LSH_STATIC_SCRATCH_BYTES (64 MiB) that the library defines at
 * file scope in device memory.  Every GPU that loads the library holds that
 * array until the process exits.  It allocates nothing itself: no
 * cudaMalloc, no cudaFree, no allocating library call.
 *   - Capacity.  With n = B * H * L tokens, and every part below rounded up
 *     to a multiple of 256 bytes, the scratch a call needs is
 *       tensor-core path (dtype LSH_BF16 and chunk == 64):
 *         n * 4                        per-token key scales
 *       + n * 64 * 2                   the values in fp16
 *       + n_rounds * n * 64 * 2        fp16 outputs of every round
 *       + n_rounds * n * 4             logsumexps of every round,
 *       the last two only when n_rounds > 1; so 132 bytes per token for
 *       one round, 396 for two, 660 for four, 1188 for eight;
 *       CUDA-core path (every other supported case):
 *         (n_rounds - 1) * n * d * 4 + (n_rounds - 1) * n * 4
 *                                      partials of rounds 0 .. n_rounds-2,
 *       none for one round.
 *     A call whose need exceeds LSH_STATIC_SCRATCH_BYTES returns
 *     LSH_ERR_SCRATCH_LIMIT before any launch.
 *   - Set-up: the first call on a device, with that device current, looks up
 *     the array's device address (cudaGetSymbolAddress) and caches it; make
 *     that first call outside any stream capture.  The cached address
 *     belongs to the device's primary context as it was then: after
 *     cudaDeviceReset the process must not call this entry point again.
 *   - Sharing: all calls in the process on a device use the same array and
 *     it keeps whatever the last call left there.  Every element a call reads
 *     is written earlier in the same call, so nothing needs clearing, but
 *     two calls whose kernels overlap on the GPU (different streams, no
 *     ordering between them) race on the array and give wrong results.
 *     Order such calls on one stream or with events.
 * Results are those of lsh_attend_fwd(shape, Q, V, keys, perm, NULL, NULL,
 * O, lse, ws, ws_bytes, stream). */
#define LSH_STATIC_SCRATCH_BYTES ((size_t)64 << 20)
LSH_API lsh_status lsh_attend_fwd_static(const lsh_shape* shape, const void* Q, const void* V,
                                         const uint32_t* keys, const int32_t* perm, void* O,
                                         float* lse, void* stream);

/* Chunked position-wise feed-forward, the companion of LSH attention in a
 * Reformer layer ("Reformer explainer", its single section: a chunked
 * feed-forward beside LSH attention and reversible layers; "Reformer Language
 * Models (Korean)", Reformer overview: feed-forward activations can dominate
 * memory, so the feed-forward is chunked to cut peak memory).  Per position
 *   Y[t] = W2 max(0, W1 X[t] + b1) + b2,
 * taken `chunk` positions at a time, so the hidden activation exists for one
 * chunk only (in ws).  Chunking does not change the result.
 *   X, Y: [tokens, d_model] bf16;  W1: [d_ff, d_model] bf16;  b1: [d_ff]
 *   bf16;  W2: [d_model, d_ff] bf16;  b2: [d_model] bf16 (row-major, device).
 * Both products run on the tensor cores with fp32 accumulation; the hidden
 * activation is rounded to bf16 between them.  Supported: d_model and d_ff
 * multiples of 256, tokens and chunk multiples of 128, tokens * d_model and
 * chunk * d_ff below 2^31; else LSH_ERR_UNSUPPORTED.  ws: at least
 * lsh_ffn_ws_size() bytes of device scratch (chunk * d_ff * 2), caller-owned.
 * Asynchronous on `stream`; nothing is allocated. */
LSH_API size_t lsh_ffn_ws_size(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk);
LSH_API lsh_status lsh_ffn_forward(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk,
                                   const void* X, const void* W1, const void* b1, const void* W2,
                                   const void* b2, void* Y, void* ws, size_t ws_bytes,
                                   void* stream);

/* Backward of the chunked feed-forward (gradients of sum(dY * Y)):
 *   dA[t] = (W2^T dY[t]) where W1 X[t] + b1 > 0 (max(0, .)' = 0 at 0),
 *   dX[t] = R[t] + W1^T dA[t]            (R: fp32 [tokens, d_model] or NULL),
 *   dW1 = sum_t dA[t] X[t]^T,  db1 = sum_t dA[t],
 *   dW2 = sum_t dY[t] H[t]^T,  db2 = sum_t dY[t],  H[t] = max(0, W1 X[t] + b1),
 * the hidden activation recomputed chunk by chunk (ws holds one chunk's H
 * and dA, lsh_ffn_bwd_ws_size() bytes).  X, W1, b1, W2, dY bf16 as in
 * lsh_ffn_forward; dX [tokens, d_model], dW1 [d_ff, d_model], db1 [d_ff],
 * dW2 [d_model, d_ff], db2 [d_model] fp32 (the four parameter gradients are
 * overwritten).  The products run on the tensor cores: the transposed
 * operands are read in place (MN-major), the parameter gradients accumulate
 * with fp32 atomics over positions split across thread blocks, so their
 * summation order varies from call to call. */
LSH_API size_t lsh_ffn_bwd_ws_size(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk);
LSH_API lsh_status lsh_ffn_backward(int32_t tokens, int32_t d_model, int32_t d_ff, int32_t chunk,
                                    const void* X, const void* W1, const void* b1, const void* W2,
                                    const void* dY, const float* R, float* dX, float* dW1,
                                    float* db1, float* dW2, float* db2, void* ws, size_t ws_bytes,
                                    void* stream);

/* Reversible residual block around LSH attention.  The Reformer abstract
 * (codewithpapers.app listing) and the explainer (its single section) use
 * reversible residual layers (RevNet) so that a layer's inputs are
 * recomputed from its outputs in the backward pass instead of being stored:
 *   Y1 = X1 + F(X2),   Y2 = X2 + G(Y1),
 * with F = LSH attention of X2 (each token's features, split into H heads of
 * d = 64, are its query = key and its value; shape's B, H, L, n_buckets,
 * n_rounds, chunk, causal; dtype must be LSH_BF16) and G = the chunked
 * feed-forward (d_model = H * 64, d_ff, ffn_chunk; see lsh_ffn_forward).
 *   X1, X2, Y1, Y2, dY1, dY2, dX1, dX2: fp32 [B, L, H * 64] (the residual
 *   stream); the sublayers take bf16 copies of their inputs.
 *   rot [n_rounds, 64, n_buckets / 2] bf16; W1, b1, W2, b2 bf16 as in
 *   lsh_ffn_forward; dW1, db1, dW2, db2 fp32 (overwritten).
 * lsh_rev_forward writes Y1, Y2 and the keys and permutations of X2's hash
 * ([n_rounds, B, H, L]), which the backward holds constant.
 * lsh_rev_backward takes only the outputs: it recomputes X2 = Y2 - G(Y1) and
 * X1 = Y1 - F(X2) (written to X1, X2), and writes
 *   dX1 = dY1 + G'(Y1)^T dY2,   dX2 = dY2 + F'(X2)^T dX1,
 * (F'(X2)^T g is the sum of the attention's query and value gradients for
 * the upstream gradient g) and G's parameter gradients.  ws: at least
 * lsh_rev_ws_size() bytes of device scratch, caller-owned.  Every step runs
 * in this library's kernels; nothing is allocated.  Supported: H a multiple
 * of 4, B * L a multiple of 128, and the limits of lsh_forward and
 * lsh_ffn_forward. */
LSH_API size_t lsh_rev_ws_size(const lsh_shape* shape, int32_t d_ff, int32_t ffn_chunk);
LSH_API lsh_status lsh_rev_forward(const lsh_shape* shape, int32_t d_ff, int32_t ffn_chunk,
                                   const float* X1, const float* X2, const void* rot,
                                   const void* W1, const void* b1, const void* W2, const void* b2,
                                   float* Y1, float* Y2, uint32_t* keys, int32_t* perm, void* ws,
                                   size_t ws_bytes, void* stream);
LSH_API lsh_status lsh_rev_backward(const lsh_shape* shape, int32_t d_ff, int32_t ffn_chunk,
                                    const float* Y1, const float* Y2, const float* dY1,
                                    const float* dY2, const uint32_t* keys, const int32_t* perm,
                                    const void* W1, const void* b1, const void* W2,
                                    const void* b2, float* X1, float* X2, float* dX1, float* dX2,
                                    float* dW1, float* db1, float* dW2, float* db2, void* ws,
                                    size_t ws_bytes, void* stream);

/* Test hook for the failure path of the bounded device waits.  No passage of
 * the pages corresponds to it.  Every wait in the kernels gives up after a
 * limit of clock cycles (about 2 s by default), records LSH_ERR_TIMEOUT in
 * the device status word, stops its thread block cleanly (in-flight copies and
 * tensor-core operations finish, tensor memory is freed) and returns.
 *   wait_cycles > 0   the limit of the waits of the tensor-core attention and
 *                     feed-forward kernels for the calls that follow; 0
 *                     restores the default;
 *   hold_tile >= 0    in the calls that follow, the tensor-core attention
 *                     kernel's producers stop before tile `hold_tile` of each
 *                     thread block, so the waits for that tile's data run out
 *                     (their outputs are then undefined); -1 restores normal
 *                     operation.
 * The setting is process-wide and not synchronised with calls on other host
 * threads.  LSH_ERR_INVALID_ARG for wait_cycles < 0. */
LSH_API lsh_status lsh_set_wait_test(int32_t hold_tile, int64_t wait_cycles);

/* Synchronises `stream`, returns the first error a kernel recorded since the
 * last call (LSH_OK if none) and clears it.  LSH_ERR_CUDA if the
 * synchronisation itself fails. */
LSH_API lsh_status lsh_device_status(void* stream);

/* Static text for a status code. */
LSH_API const char* lsh_status_string(lsh_status status);

#ifdef __cplusplus
}
#endif

#endif /* LSH_ATTENTION_LSH_H_ */
