// CPU oracle for shared-QK LSH attention -- TEST INFRASTRUCTURE ONLY.
//
// Only the test suite, the smoke check and the benchmark's CPU-baseline leg
// load this library.  The product path (lsh_attention_long_b200 and its CUDA
// library) never calls, links or imports anything here, and this file shares
// no code, header, table or constant with it.
//
// It is a plain, slow, single-threaded restatement of the method in fp64:
// every input is upcast exactly (fp32 and bf16 values are exact in fp64) and
// every loop follows the definition without blocking, fusion or reordering.
//
// Sources it follows:
//   * "Reformer explainer" (akshathtiwari.co.in/blog/reformer), its single
//     section: angular LSH by a random rotation and the sector a vector falls
//     into; shared-QK (a token's query and key hash together); sort by
//     bucket; equal chunks attending to bucket-mates; several hash rounds
//     whose buckets are unioned.
//   * "Reformer: The Efficient Transformer" (codewithpapers.app listing),
//     abstract: LSH attention replaces dot-product attention.
//   * The five-step definition this library implements, which fixes what the
//     pages leave open:
//       1. hash: h = argmax([x.R_r ; -x.R_r]) per round r, R_r of shape
//          [d, n_buckets/2];
//       2. a stable sort of every (batch, head, round) row by
//          (bucket, position);
//       3. chunks of c sorted slots; each chunk attends to itself and the
//          previous chunk (chunk 0 wraps to the last); keys are the unit-
//          normalised queries; scores are scaled by 1/sqrt(d); a different
//          bucket or (if causal) a later position gets -inf, the token
//          itself gets -1e5;
//       4. results are scattered back to original positions with each
//          round's logsumexp;
//       5. rounds combine as o = sum_r softmax_r(lse_r) * o_r.
//
// Readings taken where the pages are silent (the same list is kept with the
// design notes of the library):
//   - n_buckets == 1: every bucket is 0 and the rotation is not read.
//   - argmax ties: the lowest index of the concatenation wins, so +p_j beats
//     -p_k on exact equality.
//   - a query of zero norm has a zero unit key.
//   - masks replace the score (they are not added to it); a replaced entry
//     carries no gradient.
//   - a single chunk (c == L) attends to itself once.
//   - near tie: the top two entries z1 >= z2 of [p ; -p] satisfy
//     z1 - z2 <= 1e-5 * |z1|.
//
// Also here: the chunked position-wise feed-forward that sits beside LSH
// attention in a Reformer layer ("Reformer explainer": a chunked feed-forward
// with the reversible layers; "Reformer Language Models (Korean)", its
// Reformer overview: feed-forward activations can dominate memory, so the
// feed-forward runs in chunks to cut peak memory).  Readings taken: the
// standard Transformer feed-forward y = W2 relu(W1 x + b1) + b2 at every
// position; chunking evaluates `chunk` positions at a time, so the hidden
// activation exists for one chunk only, and does not change the result.
//
// Parity pins for every function live in tests/test_oracle_pins.py.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

namespace {

const double kSelfScore = -1e5;   // the score that replaces a token's own entry
const double kNearTieRel = 1e-5;  // relative gap below which a hash is a near tie

inline size_t row_index(int r, int b, int h, int B, int H) {
  return ((size_t)r * B + b) * H + h;
}

}  // namespace

extern "C" {

// Step 1 -- angular LSH.  For every round r, batch b, head h and position i:
//   p_j = sum_k Q[b,h,i,k] * rot[r,k,j]          (j < n_buckets/2)
//   z   = (p_0 .. p_{nb/2-1}, -p_0 .. -p_{nb/2-1})
//   bucket = lowest index j with z_j == max(z)
//   key    = bucket * L + i
// Outputs are laid out [R, B, H, L].  `buckets` and `near_tie` may be NULL.
// Returns 0, or 1 on an invalid argument.
int oracle_lsh_hash(int B, int H, int L, int d, int n_buckets, int n_rounds,
                    const double* Q, const double* rot, uint32_t* keys,
                    int32_t* buckets, uint8_t* near_tie) {
  if (B < 0 || H < 0 || L < 0 || d <= 0 || n_rounds < 0) return 1;
  if (n_buckets < 1 || (n_buckets > 1 && n_buckets % 2 != 0)) return 1;
  const int half = n_buckets / 2;
  std::vector<double> z(n_buckets);
  for (int r = 0; r < n_rounds; ++r)
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h)
        for (int i = 0; i < L; ++i) {
          const double* q = Q + (((size_t)b * H + h) * L + i) * d;
          int bucket = 0;
          bool tie = false;
          if (n_buckets > 1) {
            for (int j = 0; j < half; ++j) {
              double p = 0.0;
              for (int k = 0; k < d; ++k) p += q[k] * rot[((size_t)r * d + k) * half + j];
              z[j] = p;
              z[j + half] = -p;
            }
            // argmax with the first index winning
            for (int j = 1; j < n_buckets; ++j)
              if (z[j] > z[bucket]) bucket = j;
            double z1 = z[bucket];
            double z2 = -std::numeric_limits<double>::infinity();
            for (int j = 0; j < n_buckets; ++j)
              if (j != bucket && z[j] > z2) z2 = z[j];
            tie = (z1 - z2) <= kNearTieRel * std::fabs(z1);
          }
          size_t o = row_index(r, b, h, B, H) * L + i;
          keys[o] = (uint32_t)((uint64_t)bucket * (uint64_t)L + (uint64_t)i);
          if (buckets) buckets[o] = bucket;
          if (near_tie) near_tie[o] = tie ? 1 : 0;
        }
  return 0;
}

// Step 2 -- per-row stable sort by (bucket, position).  `keys` holds `rows`
// rows of L packed keys bucket*L + position (position == index in the row).
// perm[row, t] is the original position at sorted slot t.
int oracle_lsh_sort(int rows, int L, const uint32_t* keys, int32_t* perm) {
  if (rows < 0 || L < 0) return 1;
  std::vector<int32_t> idx(L);
  for (int row = 0; row < rows; ++row) {
    const uint32_t* k = keys + (size_t)row * L;
    for (int i = 0; i < L; ++i) idx[i] = i;
    // stable sort of positions by bucket: ties keep ascending position
    std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) {
      return k[a] / (uint32_t)L < k[b] / (uint32_t)L;
    });
    std::memcpy(perm + (size_t)row * L, idx.data(), sizeof(int32_t) * L);
  }
  return 0;
}

// Steps 3-4 -- chunked shared-QK attention for every round, scattered back to
// original positions.  o_part is [R, B, H, L, d], lse_r is [R, B, H, L].
// The bucket of position j in row (r, b, h) is keys[r,b,h,j] / L.
// Only the queries of chunks [chunk_begin, chunk_end) of every row are
// computed (their outputs land at those queries' positions); the plain
// entry point below takes every chunk.
int oracle_lsh_attend_fwd_range(int B, int H, int L, int d, int n_rounds, int chunk, int causal,
                                const double* Q, const double* V, const uint32_t* keys,
                                const int32_t* perm, int chunk_begin, int chunk_end,
                                double* o_part, double* lse_r) {
  if (B < 0 || H < 0 || L < 0 || d <= 0 || n_rounds < 0 || chunk <= 0) return 1;
  if (L % chunk != 0) return 1;
  const int n_chunks = L / chunk;
  if (chunk_begin < 0 || chunk_end > n_chunks || chunk_begin > chunk_end) return 1;
  const double scale = 1.0 / std::sqrt((double)d);
  const double neg_inf = -std::numeric_limits<double>::infinity();
  std::vector<double> khat((size_t)L * d);
  std::vector<double> s(2 * (size_t)chunk);
  std::vector<int32_t> win(2 * (size_t)chunk);
  for (int r = 0; r < n_rounds; ++r)
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h) {
        const size_t row = row_index(r, b, h, B, H);
        const double* q = Q + ((size_t)b * H + h) * L * d;
        const double* v = V + ((size_t)b * H + h) * L * d;
        const uint32_t* key = keys + row * L;
        const int32_t* pm = perm + row * L;
        // keys are the unit-normalised queries (shared-QK)
        for (int j = 0; j < L; ++j) {
          double nrm = 0.0;
          for (int k = 0; k < d; ++k) nrm += q[(size_t)j * d + k] * q[(size_t)j * d + k];
          nrm = std::sqrt(nrm);
          for (int k = 0; k < d; ++k)
            khat[(size_t)j * d + k] = nrm > 0.0 ? q[(size_t)j * d + k] / nrm : 0.0;
        }
        for (int c = chunk_begin; c < chunk_end; ++c) {
          // window: the previous chunk (wrapping) then this chunk; one chunk
          // only once when the row is a single chunk
          int nw = 0;
          if (n_chunks > 1) {
            int prev = (c - 1 + n_chunks) % n_chunks;
            for (int t = 0; t < chunk; ++t) win[nw++] = pm[prev * chunk + t];
          }
          for (int t = 0; t < chunk; ++t) win[nw++] = pm[c * chunk + t];
          for (int t = 0; t < chunk; ++t) {
            const int i = pm[c * chunk + t];
            const uint32_t bi = key[i] / (uint32_t)L;
            double m = neg_inf;
            for (int u = 0; u < nw; ++u) {
              const int j = win[u];
              double sc;
              if (key[j] / (uint32_t)L != bi) {
                sc = neg_inf;
              } else if (causal && j > i) {
                sc = neg_inf;
              } else if (j == i) {
                sc = kSelfScore;
              } else {
                sc = 0.0;
                for (int k = 0; k < d; ++k) sc += q[(size_t)i * d + k] * khat[(size_t)j * d + k];
                sc *= scale;
              }
              s[u] = sc;
              if (sc > m) m = sc;
            }
            double sum = 0.0;
            for (int u = 0; u < nw; ++u) sum += std::exp(s[u] - m);
            const double lse = m + std::log(sum);
            double* o = o_part + (row * L + i) * d;
            for (int k = 0; k < d; ++k) o[k] = 0.0;
            for (int u = 0; u < nw; ++u) {
              const double p = std::exp(s[u] - lse);
              if (p == 0.0) continue;
              const double* vj = v + (size_t)win[u] * d;
              for (int k = 0; k < d; ++k) o[k] += p * vj[k];
            }
            lse_r[row * L + i] = lse;
          }
        }
      }
  return 0;
}

int oracle_lsh_attend_fwd(int B, int H, int L, int d, int n_rounds, int chunk, int causal,
                          const double* Q, const double* V, const uint32_t* keys,
                          const int32_t* perm, double* o_part, double* lse_r) {
  if (chunk <= 0 || L < 0) return 1;
  return oracle_lsh_attend_fwd_range(B, H, L, d, n_rounds, chunk, causal, Q, V, keys, perm, 0,
                                     L / chunk, o_part, lse_r);
}

// Step 5 -- combine rounds: lse = logsumexp_r lse_r, o = sum_r exp(lse_r - lse) o_r.
// o_part [R, B, H, L, d], lse_r [R, B, H, L] -> O [B, H, L, d], lse [B, H, L].
int oracle_lsh_combine(int n_rounds, int B, int H, int L, int d, const double* o_part,
                       const double* lse_r, double* O, double* lse) {
  if (n_rounds < 1 || B < 0 || H < 0 || L < 0 || d <= 0) return 1;
  const size_t n = (size_t)B * H * L;
  for (size_t t = 0; t < n; ++t) {
    double m = -std::numeric_limits<double>::infinity();
    for (int r = 0; r < n_rounds; ++r) m = std::max(m, lse_r[(size_t)r * n + t]);
    double sum = 0.0;
    for (int r = 0; r < n_rounds; ++r) sum += std::exp(lse_r[(size_t)r * n + t] - m);
    const double l = m + std::log(sum);
    for (int k = 0; k < d; ++k) O[t * d + k] = 0.0;
    for (int r = 0; r < n_rounds; ++r) {
      const double w = std::exp(lse_r[(size_t)r * n + t] - l);
      for (int k = 0; k < d; ++k) O[t * d + k] += w * o_part[((size_t)r * n + t) * d + k];
    }
    if (lse) lse[t] = l;
  }
  return 0;
}

// Backward of steps 3-5 with buckets and permutations held constant, for an
// upstream gradient dO on the combined output O.  It recomputes the forward,
// then follows the chain rule term by term:
//   w_r = exp(lse_r - lse),  do_r = w_r dO,  g_r = dO . o_r,
//   dlse_r = w_r (g_r - sum_s w_s g_s);
//   per round and window entry (unmasked only):
//     P = exp(s - lse_r),  dP = do_r . v_j,  D = do_r . o_r,
//     dS = P (dP - D + dlse_r);
//   dv_j += P do_r (every entry with P > 0, the token itself included),
//   dq_i += dS khat_j / sqrt(d),  dkhat_j += dS q_i / sqrt(d);
//   finally dQ_j = dq_j + (dkhat_j - khat_j (khat_j . dkhat_j)) / |q_j|.
// Q, V, dO, dQ, dV are [B, H, L, d].
int oracle_lsh_attend_bwd(int B, int H, int L, int d, int n_rounds, int chunk, int causal,
                          const double* Q, const double* V, const double* dO,
                          const uint32_t* keys, const int32_t* perm,
                          double* dQ, double* dV) {
  if (B < 0 || H < 0 || L < 0 || d <= 0 || n_rounds < 1 || chunk <= 0) return 1;
  if (L % chunk != 0) return 1;
  const size_t n = (size_t)B * H * L;
  std::vector<double> o_part((size_t)n_rounds * n * d), lse_r((size_t)n_rounds * n);
  std::vector<double> O(n * d), lse(n);
  int rc = oracle_lsh_attend_fwd(B, H, L, d, n_rounds, chunk, causal, Q, V, keys, perm,
                                 o_part.data(), lse_r.data());
  if (rc) return rc;
  oracle_lsh_combine(n_rounds, B, H, L, d, o_part.data(), lse_r.data(), O.data(), lse.data());

  const int n_chunks = L / chunk;
  const double scale = 1.0 / std::sqrt((double)d);
  const double neg_inf = -std::numeric_limits<double>::infinity();
  std::vector<double> dq(n * d, 0.0), dkhat(n * d, 0.0), dv(n * d, 0.0);
  std::vector<double> w((size_t)n_rounds * n), dlse((size_t)n_rounds * n);
  for (size_t t = 0; t < n; ++t) {
    double gbar = 0.0;
    std::vector<double> g(n_rounds);
    for (int r = 0; r < n_rounds; ++r) {
      w[(size_t)r * n + t] = std::exp(lse_r[(size_t)r * n + t] - lse[t]);
      double acc = 0.0;
      for (int k = 0; k < d; ++k) acc += dO[t * d + k] * o_part[((size_t)r * n + t) * d + k];
      g[r] = acc;
      gbar += w[(size_t)r * n + t] * acc;
    }
    for (int r = 0; r < n_rounds; ++r)
      dlse[(size_t)r * n + t] = w[(size_t)r * n + t] * (g[r] - gbar);
  }

  std::vector<double> khat((size_t)L * d), nrm(L);
  std::vector<double> s(2 * (size_t)chunk);
  std::vector<int32_t> win(2 * (size_t)chunk);
  std::vector<double> do_r(d);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = (size_t)b * H + h;
      const double* q = Q + bh * L * d;
      const double* v = V + bh * L * d;
      for (int j = 0; j < L; ++j) {
        double a = 0.0;
        for (int k = 0; k < d; ++k) a += q[(size_t)j * d + k] * q[(size_t)j * d + k];
        nrm[j] = std::sqrt(a);
        for (int k = 0; k < d; ++k)
          khat[(size_t)j * d + k] = nrm[j] > 0.0 ? q[(size_t)j * d + k] / nrm[j] : 0.0;
      }
      for (int r = 0; r < n_rounds; ++r) {
        const size_t row = row_index(r, b, h, B, H);
        const uint32_t* key = keys + row * L;
        const int32_t* pm = perm + row * L;
        for (int c = 0; c < n_chunks; ++c) {
          int nw = 0;
          if (n_chunks > 1) {
            int prev = (c - 1 + n_chunks) % n_chunks;
            for (int t = 0; t < chunk; ++t) win[nw++] = pm[prev * chunk + t];
          }
          for (int t = 0; t < chunk; ++t) win[nw++] = pm[c * chunk + t];
          for (int t = 0; t < chunk; ++t) {
            const int i = pm[c * chunk + t];
            const size_t ti = bh * L + i;             // token index in [B, H, L]
            const uint32_t bi = key[i] / (uint32_t)L;
            const double lr = lse_r[(size_t)r * n + ti];
            const double wr = w[(size_t)r * n + ti];
            for (int k = 0; k < d; ++k) do_r[k] = wr * dO[ti * d + k];
            double D = 0.0;
            for (int k = 0; k < d; ++k) D += do_r[k] * o_part[((size_t)r * n + ti) * d + k];
            const double dl = dlse[(size_t)r * n + ti];
            for (int u = 0; u < nw; ++u) {
              const int j = win[u];
              const size_t tj = bh * L + j;
              bool masked = false;  // replaced by -inf or by the self score
              double sc;
              if (key[j] / (uint32_t)L != bi) {
                sc = neg_inf; masked = true;
              } else if (causal && j > i) {
                sc = neg_inf; masked = true;
              } else if (j == i) {
                sc = kSelfScore; masked = true;
              } else {
                sc = 0.0;
                for (int k = 0; k < d; ++k) sc += q[(size_t)i * d + k] * khat[(size_t)j * d + k];
                sc *= scale;
              }
              const double P = std::exp(sc - lr);
              if (P != 0.0)
                for (int k = 0; k < d; ++k) dv[tj * d + k] += P * do_r[k];
              if (masked) continue;
              double dP = 0.0;
              for (int k = 0; k < d; ++k) dP += do_r[k] * v[(size_t)j * d + k];
              const double dS = P * (dP - D + dl);
              for (int k = 0; k < d; ++k) {
                dq[ti * d + k] += dS * khat[(size_t)j * d + k] * scale;
                dkhat[tj * d + k] += dS * q[(size_t)i * d + k] * scale;
              }
            }
          }
        }
      }
      // through the normalisation khat = q / |q|
      for (int j = 0; j < L; ++j) {
        const size_t tj = bh * L + j;
        double proj = 0.0;
        for (int k = 0; k < d; ++k) proj += khat[(size_t)j * d + k] * dkhat[tj * d + k];
        for (int k = 0; k < d; ++k) {
          double g = 0.0;
          if (nrm[j] > 0.0) g = (dkhat[tj * d + k] - khat[(size_t)j * d + k] * proj) / nrm[j];
          dQ[tj * d + k] = dq[tj * d + k] + g;
          dV[tj * d + k] = dv[tj * d + k];
        }
      }
    }
  return 0;
}

// Chunked feed-forward, forward.  X [T, d_model], W1 [d_ff, d_model],
// b1 [d_ff], W2 [d_model, d_ff], b2 [d_model] -> Y [T, d_model].  Positions
// are taken `chunk` at a time; for each chunk the hidden activation
//   h[t, j] = max(0, b1[j] + sum_k W1[j, k] X[t, k])
// is formed, then
//   Y[t, i] = b2[i] + sum_j W2[i, j] h[t, j].
// Returns 0, or 1 on an invalid argument.
int oracle_ffn_forward(int T, int d_model, int d_ff, int chunk, const double* X, const double* W1,
                       const double* b1, const double* W2, const double* b2, double* Y) {
  if (T < 0 || d_model <= 0 || d_ff <= 0 || chunk <= 0) return 1;
  std::vector<double> h((size_t)chunk * d_ff);
  for (int c0 = 0; c0 < T; c0 += chunk) {
    const int n = std::min(chunk, T - c0);
    for (int t = 0; t < n; ++t) {
      const double* x = X + (size_t)(c0 + t) * d_model;
      for (int j = 0; j < d_ff; ++j) {
        double a = b1[j];
        for (int k = 0; k < d_model; ++k) a += W1[(size_t)j * d_model + k] * x[k];
        h[(size_t)t * d_ff + j] = a > 0.0 ? a : 0.0;
      }
    }
    for (int t = 0; t < n; ++t) {
      double* y = Y + (size_t)(c0 + t) * d_model;
      for (int i = 0; i < d_model; ++i) {
        double s = b2[i];
        for (int j = 0; j < d_ff; ++j) s += W2[(size_t)i * d_ff + j] * h[(size_t)t * d_ff + j];
        y[i] = s;
      }
    }
  }
  return 0;
}

// Chunked feed-forward, backward: gradients of sum(dY * Y) with respect to
// X, W1, b1, W2, b2 (the weight and bias gradients summed over every
// position).  Per chunk the pre-activation a = b1 + W1 x and h = max(0, a)
// are recomputed, then
//   dW2[i, j] += dY[t, i] h[t, j],   db2[i] += dY[t, i],
//   dh[t, j] = sum_i W2[i, j] dY[t, i],   da = dh where a > 0, else 0,
//   dW1[j, k] += da[t, j] X[t, k],   db1[j] += da[t, j],
//   dX[t, k] = sum_j W1[j, k] da[t, j].
// The derivative of max(0, a) at a = 0 is taken as 0.
int oracle_ffn_backward(int T, int d_model, int d_ff, int chunk, const double* X, const double* W1,
                        const double* b1, const double* W2, const double* dY, double* dX,
                        double* dW1, double* db1, double* dW2, double* db2) {
  if (T < 0 || d_model <= 0 || d_ff <= 0 || chunk <= 0) return 1;
  std::fill(dW1, dW1 + (size_t)d_ff * d_model, 0.0);
  std::fill(db1, db1 + d_ff, 0.0);
  std::fill(dW2, dW2 + (size_t)d_model * d_ff, 0.0);
  std::fill(db2, db2 + d_model, 0.0);
  std::vector<double> a((size_t)d_ff), h((size_t)d_ff), da((size_t)d_ff);
  for (int c0 = 0; c0 < T; c0 += chunk) {
    const int n = std::min(chunk, T - c0);
    for (int t = 0; t < n; ++t) {
      const double* x = X + (size_t)(c0 + t) * d_model;
      const double* dy = dY + (size_t)(c0 + t) * d_model;
      for (int j = 0; j < d_ff; ++j) {
        double s = b1[j];
        for (int k = 0; k < d_model; ++k) s += W1[(size_t)j * d_model + k] * x[k];
        a[j] = s;
        h[j] = s > 0.0 ? s : 0.0;
      }
      for (int i = 0; i < d_model; ++i) {
        db2[i] += dy[i];
        for (int j = 0; j < d_ff; ++j) dW2[(size_t)i * d_ff + j] += dy[i] * h[j];
      }
      for (int j = 0; j < d_ff; ++j) {
        double dh = 0.0;
        for (int i = 0; i < d_model; ++i) dh += W2[(size_t)i * d_ff + j] * dy[i];
        da[j] = a[j] > 0.0 ? dh : 0.0;
        db1[j] += da[j];
        for (int k = 0; k < d_model; ++k) dW1[(size_t)j * d_model + k] += da[j] * x[k];
      }
      double* dx = dX + (size_t)(c0 + t) * d_model;
      for (int k = 0; k < d_model; ++k) {
        double s = 0.0;
        for (int j = 0; j < d_ff; ++j) s += W1[(size_t)j * d_model + k] * da[j];
        dx[k] = s;
      }
    }
  }
  return 0;
}

}  // extern "C"
