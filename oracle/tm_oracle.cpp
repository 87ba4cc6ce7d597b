// TriangleMix CPU oracle: plain, slow, fp64, explicit mask.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or
// call this file: only the tests, the smoke check and the benchmark's CPU
// baseline leg do. It shares no code with the CUDA library.
//
// What it computes (TriangleMix blog post by He Zhiyuan, section 介绍 and the
// "Middle Q-K" discussion in section 缘由; 36kr interview with Yang Yuqing,
// lead paragraphs on the streaming region and the last Q-K region):
//
//   keep_tri(i, j)    = j <= i  and  (j < S  or  i - j < W  or  i >= N - L)
//   keep_causal(i, j) = j <= i
//
//   s_ij = scale * sum_d q[b,i,hq,d] * k[b,j,g,d]          (j kept, fp64)
//   p_ij = exp(s_ij - max_j s_ij),  l_i = sum_j p_ij
//   o_i  = sum_j p_ij * v[b,j,g,:] / l_i
//
// with g = hq / (Hq / Hkv) (consecutive q heads share a kv head). The
// pages give the pattern in words only; the exact set (sink tokens j < S, a
// window of W positions ending at and including i, and the last L query
// rows seeing every causal key) is the plainest reading of that wording and
// is the one used everywhere here. Inputs are bf16 bit patterns converted
// exactly to double; all sums are fp64; every mask row is materialised as an
// explicit boolean vector before it is used.
//
// parity pins (checked by the CPU tests, not by this file):
//   * kept count per row equals min(i+1,W) + max(0, min(S, i+1-W)) for
//     i < N-L and i+1 otherwise;
//   * L = N or S + W >= N gives causal attention;
//   * the last L rows equal the causal rows; rows sum to 1;
//   * S=0, W=1, L=0 gives o_i = v_i; q = 0 gives the mean of v over K_i;
//   * causal and masked rows match a library softmax-attention routine;
//   * block-sparse: every causal block listed gives causal attention exactly;
//     q = 0 gives the mean of v over the kept keys; rows match the library
//     routine under a block mask built independently; empty lists give 0;
//   * discovery scores: q = 0 gives 1 / (I + 1); one probe on one head gives
//     a plain softmax (a worked example with closed-form values);
//   * per-head bands: every head equals the single-pattern oracle run with
//     that head's sinks and window; equal bands give the shared-band result.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

inline double bf16_to_double(uint16_t h) {
  uint32_t u = uint32_t(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

struct Pattern {
  long long N, S, W, L;
  bool causal;
};

// One mask entry, straight from the definition above.
inline bool keep(const Pattern& p, long long i, long long j) {
  if (j > i) return false;
  if (p.causal) return true;
  return j < p.S || i - j < p.W || i >= p.N - p.L;
}

bool make_pattern(int N, int causal, int S, int W, int L, Pattern* out) {
  if (N < 1) return false;
  if (!causal && (S < 0 || L < 0 || W < 1)) return false;
  out->N = N;
  out->causal = causal != 0;
  out->S = std::min<long long>(std::max(S, 0), N);
  out->W = std::min<long long>(std::max(W, 1), N);
  out->L = std::min<long long>(std::max(L, 0), N);
  return true;
}

// Explicit boolean mask row i.
void mask_row(const Pattern& p, long long i, std::vector<unsigned char>& m) {
  m.assign(size_t(p.N), 0);
  for (long long j = 0; j < p.N; ++j) m[size_t(j)] = keep(p, i, j) ? 1 : 0;
}

template <class F>
void parallel_for(long long n, int nthreads, F&& f) {
  if (nthreads < 1) nthreads = 1;
  if (n < nthreads) nthreads = int(std::max<long long>(n, 1));
  if (nthreads == 1) {
    f(0LL, n);
    return;
  }
  std::vector<std::thread> th;
  long long chunk = (n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    long long b = t * chunk, e = std::min(n, b + chunk);
    if (b >= e) break;
    th.emplace_back([=, &f] { f(b, e); });
  }
  for (auto& x : th) x.join();
}

}  // namespace

extern "C" {

// 1 if (i, j) is kept, 0 if not, -1 on a bad pattern.
int oracle_keep(int N, int causal, int S, int W, int L, long long i, long long j) {
  Pattern p;
  if (!make_pattern(N, causal, S, W, L, &p)) return -1;
  return keep(p, i, j) ? 1 : 0;
}

// Writes the explicit mask row i (N bytes of 0/1). Returns 0 or -1.
int oracle_mask_row(int N, int causal, int S, int W, int L, long long i, unsigned char* out) {
  Pattern p;
  if (!make_pattern(N, causal, S, W, L, &p) || !out || i < 0 || i >= N) return -1;
  std::vector<unsigned char> m;
  mask_row(p, i, m);
  std::memcpy(out, m.data(), size_t(N));
  return 0;
}

// |K_i| counted from the explicit mask row; -1 on a bad argument.
long long oracle_kept_count_row(int N, int causal, int S, int W, int L, long long i) {
  Pattern p;
  if (!make_pattern(N, causal, S, W, L, &p) || i < 0 || i >= N) return -1;
  std::vector<unsigned char> m;
  mask_row(p, i, m);
  long long c = 0;
  for (unsigned char x : m) c += x;
  return c;
}

// sum_i |K_i| over all rows (explicit masks); -1 on a bad argument.
long long oracle_kept_pairs(int N, int causal, int S, int W, int L, int nthreads) {
  Pattern p;
  if (!make_pattern(N, causal, S, W, L, &p)) return -1;
  std::vector<long long> acc(size_t(N), 0);
  parallel_for(N, nthreads, [&](long long b, long long e) {
    std::vector<unsigned char> m;
    for (long long i = b; i < e; ++i) {
      mask_row(p, i, m);
      long long c = 0;
      for (unsigned char x : m) c += x;
      acc[size_t(i)] = c;
    }
  });
  long long total = 0;
  for (long long c : acc) total += c;
  return total;
}

// Masked softmax attention in fp64.
//   q: [B, N, Hq, D], k, v: [B, N, Hkv, D], bf16 bit patterns, contiguous.
//   rows: nrows query indices (NULL = every row 0..N-1, nrows ignored).
//   out: [B, nrows, Hq, D] fp64.   rowsum (optional): [B, nrows, Hq] = sum_j p_ij / l_i.
// Returns 0, or -1 on a bad argument.
int oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                     int Hkv, int N, int D, double scale, int causal, int S, int W, int L,
                     const long long* rows, long long nrows, double* out, double* rowsum,
                     int nthreads) {
  Pattern p;
  if (!q || !k || !v || !out || B < 1 || Hq < 1 || Hkv < 1 || D < 1 || Hq % Hkv != 0) return -1;
  if (!make_pattern(N, causal, S, W, L, &p)) return -1;
  if (!rows) nrows = N;
  if (nrows < 0) return -1;
  for (long long r = 0; rows && r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= N) return -1;
  const int G = Hq / Hkv;
  const long long units = (long long)B * nrows;  // one unit = one (b, row), all heads
  parallel_for(units, nthreads, [&](long long ub, long long ue) {
    std::vector<unsigned char> m;
    std::vector<long long> idx;
    std::vector<double> s, qrow(static_cast<size_t>(D)), o(static_cast<size_t>(D));
    for (long long u = ub; u < ue; ++u) {
      const long long b = u / nrows, r = u % nrows;
      const long long i = rows ? rows[r] : r;
      mask_row(p, i, m);  // explicit mask row, shared by all heads
      idx.clear();
      for (long long j = 0; j < N; ++j)
        if (m[size_t(j)]) idx.push_back(j);
      s.resize(idx.size());
      for (int hq = 0; hq < Hq; ++hq) {
        const int g = hq / G;
        const uint16_t* qp = q + ((b * N + i) * Hq + hq) * (long long)D;
        for (int d = 0; d < D; ++d) qrow[size_t(d)] = bf16_to_double(qp[d]);
        double mx = -std::numeric_limits<double>::infinity();
        for (size_t t = 0; t < idx.size(); ++t) {
          const uint16_t* kp = k + ((b * N + idx[t]) * Hkv + g) * (long long)D;
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += qrow[size_t(d)] * bf16_to_double(kp[d]);
          s[t] = scale * acc;
          mx = std::max(mx, s[t]);
        }
        double l = 0.0;
        for (size_t t = 0; t < idx.size(); ++t) {
          s[t] = std::exp(s[t] - mx);
          l += s[t];
        }
        std::fill(o.begin(), o.end(), 0.0);
        for (size_t t = 0; t < idx.size(); ++t) {
          const uint16_t* vp = v + ((b * N + idx[t]) * Hkv + g) * (long long)D;
          for (int d = 0; d < D; ++d) o[size_t(d)] += s[t] * bf16_to_double(vp[d]);
        }
        double* op = out + ((b * nrows + r) * Hq + hq) * (long long)D;
        for (int d = 0; d < D; ++d) op[d] = o[size_t(d)] / l;
        if (rowsum) {
          double sum = 0.0;
          for (size_t t = 0; t < idx.size(); ++t) sum += s[t] / l;
          rowsum[(b * nrows + r) * Hq + hq] = sum;
        }
      }
    }
  });
  return 0;
}

// Block-sparse causal attention in fp64 (the shallow-layer counterpart the
// TriangleMix blog post, section 介绍, leaves to dynamic sparse methods; the
// block index is the input format of the FlashPrefill summary, section 2.3):
//
//   keep(i, j) = j <= i  and  j / BS is listed for (b, g, i / BM)
//
// with the list of (b, kv head g, q-block qb) = the entries
// indices[offsets[r] .. offsets[r+1]), r = (b * Hkv + g) * nqb + qb,
// nqb = ceil(N / BM), read as a set of k-block numbers (entries that name no
// block of keys j <= i keep nothing). Each mask row is built explicitly from
// that definition; the attention is the same fp64 computation as above, and a
// row that keeps no key is 0. Returns 0, or -1 on a bad argument (offsets
// decreasing or outside [0, nnz]).
int oracle_block_sparse_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B,
                                  int Hq, int Hkv, int N, int D, double scale, int BM, int BS,
                                  const int* offsets, const int* indices, long long nnz,
                                  const long long* rows, long long nrows, double* out,
                                  int nthreads) {
  if (!q || !k || !v || !out || !offsets || B < 1 || Hq < 1 || Hkv < 1 || N < 1 || D < 1 ||
      Hq % Hkv != 0 || BM < 1 || BS < 1 || nnz < 0 || (nnz > 0 && !indices))
    return -1;
  const long long nqb = (N + BM - 1) / BM, nrec = (long long)B * Hkv * nqb;
  for (long long r = 0; r <= nrec; ++r)
    if (offsets[r] < 0 || offsets[r] > nnz || (r > 0 && offsets[r] < offsets[r - 1])) return -1;
  if (!rows) nrows = N;
  if (nrows < 0) return -1;
  for (long long r = 0; rows && r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= N) return -1;
  const int G = Hq / Hkv;
  const long long units = (long long)B * nrows;
  parallel_for(units, nthreads, [&](long long ub, long long ue) {
    std::vector<unsigned char> listed, m(static_cast<size_t>(N));
    std::vector<long long> idx;
    std::vector<double> s, qrow(static_cast<size_t>(D)), o(static_cast<size_t>(D));
    for (long long u = ub; u < ue; ++u) {
      const long long b = u / nrows, r = u % nrows;
      const long long i = rows ? rows[r] : r;
      for (int g = 0; g < Hkv; ++g) {
        // explicit mask row of (b, g, i)
        const long long rec = (b * Hkv + g) * nqb + i / BM;
        listed.assign(static_cast<size_t>((N + BS - 1) / BS), 0);
        for (long long e = offsets[rec]; e < offsets[rec + 1]; ++e)
          if (indices[e] >= 0 && indices[e] < (long long)listed.size()) listed[size_t(indices[e])] = 1;
        for (long long j = 0; j < N; ++j) m[size_t(j)] = (j <= i && listed[size_t(j / BS)]) ? 1 : 0;
        idx.clear();
        for (long long j = 0; j < N; ++j)
          if (m[size_t(j)]) idx.push_back(j);
        s.resize(idx.size());
        for (int hq = g * G; hq < (g + 1) * G; ++hq) {
          double* op = out + ((b * nrows + r) * Hq + hq) * (long long)D;
          if (idx.empty()) {
            for (int d = 0; d < D; ++d) op[d] = 0.0;
            continue;
          }
          const uint16_t* qp = q + ((b * N + i) * Hq + hq) * (long long)D;
          for (int d = 0; d < D; ++d) qrow[size_t(d)] = bf16_to_double(qp[d]);
          double mx = -std::numeric_limits<double>::infinity();
          for (size_t t = 0; t < idx.size(); ++t) {
            const uint16_t* kp = k + ((b * N + idx[t]) * Hkv + g) * (long long)D;
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += qrow[size_t(d)] * bf16_to_double(kp[d]);
            s[t] = scale * acc;
            mx = std::max(mx, s[t]);
          }
          double l = 0.0;
          for (size_t t = 0; t < idx.size(); ++t) {
            s[t] = std::exp(s[t] - mx);
            l += s[t];
          }
          std::fill(o.begin(), o.end(), 0.0);
          for (size_t t = 0; t < idx.size(); ++t) {
            const uint16_t* vp = v + ((b * N + idx[t]) * Hkv + g) * (long long)D;
            for (int d = 0; d < D; ++d) o[size_t(d)] += s[t] * bf16_to_double(vp[d]);
          }
          for (int d = 0; d < D; ++d) op[d] = o[size_t(d)] / l;
        }
      }
    }
  });
  return 0;
}

// Block pattern discovery (FlashPrefill summary, section 2.1: probe queries
// spread evenly over each query block, keys average-pooled per block;
// section 2.2: keep the key blocks whose score reaches alpha times the best
// score of the query block). In fp64, step by step, for batch b, kv head g
// and query block I with rows [r0, r1):
//   kbar_J      = mean of k[b, j, g, :] over the keys j of block J
//   probe rows  max(r0, r0 + ((p + 1) (r1 - r0)) / P - 1), p = 0 .. P-1, in each
//               q head h of g's group (a block shorter than P repeats rows)
//   pi_{h,p}(J) = softmax over J in [0, I] of scale * q[b, row, h, :] . kbar_J
//   Score(I, J) = mean over (h, p) of pi_{h,p}(J)
// scores: [B * Hkv, nqb, nqb] (J > I left 0). Block size BS for both queries
// and keys. Returns 0, or -1 on a bad argument.
int oracle_flashprefill_scores(const uint16_t* q, const uint16_t* k, int B, int Hq, int Hkv, int N,
                               int D, double scale, int P, int BS, double* scores, int nthreads) {
  if (!q || !k || !scores || B < 1 || Hq < 1 || Hkv < 1 || N < 1 || D < 1 || Hq % Hkv != 0 ||
      P < 1 || BS < 1)
    return -1;
  const int G = Hq / Hkv;
  const long long nb = (N + BS - 1) / BS;
  std::vector<double> kbar(size_t(B) * Hkv * nb * D, 0.0);
  for (long long b = 0; b < B; ++b)
    for (int g = 0; g < Hkv; ++g)
      for (long long J = 0; J < nb; ++J) {
        const long long j0 = J * BS, j1 = std::min<long long>(N, j0 + BS);
        double* kb = &kbar[size_t(((b * Hkv + g) * nb + J) * D)];
        for (long long j = j0; j < j1; ++j)
          for (int d = 0; d < D; ++d) kb[d] += bf16_to_double(k[((b * N + j) * Hkv + g) * D + d]);
        for (int d = 0; d < D; ++d) kb[d] /= double(j1 - j0);
      }
  parallel_for((long long)B * Hkv * nb, nthreads, [&](long long ub, long long ue) {
    std::vector<double> logit, mean;
    for (long long u = ub; u < ue; ++u) {
      const long long bg = u / nb, I = u % nb, b = bg / Hkv, g = bg % Hkv;
      const long long r0 = I * BS, r1 = std::min<long long>(N, r0 + BS);
      logit.assign(size_t(I + 1), 0.0);
      mean.assign(size_t(I + 1), 0.0);
      for (int h = 0; h < G; ++h)
        for (int pi = 0; pi < P; ++pi) {
          const long long row = std::max(r0, r0 + ((pi + 1) * (r1 - r0)) / P - 1);
          const uint16_t* qp = q + ((b * N + row) * Hq + g * G + h) * (long long)D;
          double mx = -std::numeric_limits<double>::infinity();
          for (long long J = 0; J <= I; ++J) {
            const double* kb = &kbar[size_t((bg * nb + J) * D)];
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += bf16_to_double(qp[d]) * kb[d];
            logit[size_t(J)] = scale * acc;
            mx = std::max(mx, logit[size_t(J)]);
          }
          double z = 0.0;
          for (long long J = 0; J <= I; ++J) z += std::exp(logit[size_t(J)] - mx);
          for (long long J = 0; J <= I; ++J) mean[size_t(J)] += std::exp(logit[size_t(J)] - mx) / z;
        }
      double* out = scores + (bg * nb + I) * nb;
      for (long long J = 0; J < nb; ++J) out[J] = J <= I ? mean[size_t(J)] / double(G * P) : 0.0;
    }
  });
  return 0;
}

// Triangle attention with a band per q head (the bf16 reading of the
// TriAttention page's per-head regions bounded by diagonal distances): head h
// keeps j <= i and (j < S_h or i - j < W_h or i >= N - L). For every (b, i, h)
// the mask row is built explicitly from head h's pattern and the attention is
// the same fp64 computation as oracle_attention. S_h, W_h: Hq ints each.
// Returns 0, or -1 on a bad argument.
int oracle_attention_heads(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                           int Hkv, int N, int D, double scale, const int* S_h, const int* W_h,
                           int L, const long long* rows, long long nrows, double* out,
                           int nthreads) {
  if (!q || !k || !v || !out || !S_h || !W_h || B < 1 || Hq < 1 || Hkv < 1 || D < 1 ||
      Hq % Hkv != 0)
    return -1;
  std::vector<Pattern> pats(static_cast<size_t>(Hq));
  for (int h = 0; h < Hq; ++h)
    if (!make_pattern(N, 0, S_h[h], W_h[h], L, &pats[size_t(h)])) return -1;
  if (!rows) nrows = N;
  if (nrows < 0) return -1;
  for (long long r = 0; rows && r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= N) return -1;
  const int G = Hq / Hkv;
  parallel_for((long long)B * nrows, nthreads, [&](long long ub, long long ue) {
    std::vector<unsigned char> m;
    std::vector<long long> idx;
    std::vector<double> s, qrow(static_cast<size_t>(D)), o(static_cast<size_t>(D));
    for (long long u = ub; u < ue; ++u) {
      const long long b = u / nrows, r = u % nrows;
      const long long i = rows ? rows[r] : r;
      for (int hq = 0; hq < Hq; ++hq) {
        const int g = hq / G;
        mask_row(pats[size_t(hq)], i, m);  // explicit mask row of this head
        idx.clear();
        for (long long j = 0; j < N; ++j)
          if (m[size_t(j)]) idx.push_back(j);
        s.resize(idx.size());
        const uint16_t* qp = q + ((b * N + i) * Hq + hq) * (long long)D;
        for (int d = 0; d < D; ++d) qrow[size_t(d)] = bf16_to_double(qp[d]);
        double mx = -std::numeric_limits<double>::infinity();
        for (size_t t = 0; t < idx.size(); ++t) {
          const uint16_t* kp = k + ((b * N + idx[t]) * Hkv + g) * (long long)D;
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += qrow[size_t(d)] * bf16_to_double(kp[d]);
          s[t] = scale * acc;
          mx = std::max(mx, s[t]);
        }
        double l = 0.0;
        for (size_t t = 0; t < idx.size(); ++t) {
          s[t] = std::exp(s[t] - mx);
          l += s[t];
        }
        std::fill(o.begin(), o.end(), 0.0);
        for (size_t t = 0; t < idx.size(); ++t) {
          const uint16_t* vp = v + ((b * N + idx[t]) * Hkv + g) * (long long)D;
          for (int d = 0; d < D; ++d) o[size_t(d)] += s[t] * bf16_to_double(vp[d]);
        }
        double* op = out + ((b * nrows + r) * Hq + hq) * (long long)D;
        for (int d = 0; d < D; ++d) op[d] = o[size_t(d)] / l;
      }
    }
  });
  return 0;
}

// Kept tiles at tile shape (BM, BN) by brute force over every (i, j) pair.
// Records are (qb, kb, flag), qb ascending then kb ascending; flag = 1 (full)
// iff every pair of the tile's existing rows and columns is kept, else 0
// (partial). Tiles with no kept pair are not listed. Writes at most cap
// records; *count gets the total. Returns 0, or -1 on a bad argument.
int oracle_tile_list_bruteforce(int N, int causal, int S, int W, int L, int BM, int BN, int* out,
                                long long cap, long long* count) {
  Pattern p;
  if (!make_pattern(N, causal, S, W, L, &p) || BM < 1 || BN < 1 || !count) return -1;
  const long long nqb = (N + BM - 1) / BM, nkb = (N + BN - 1) / BN;
  long long n = 0;
  for (long long qb = 0; qb < nqb; ++qb) {
    const long long r0 = qb * BM, r1 = std::min<long long>(N, r0 + BM);
    for (long long kb = 0; kb < nkb; ++kb) {
      const long long c0 = kb * BN, c1 = std::min<long long>(N, c0 + BN);
      long long kept = 0;
      for (long long i = r0; i < r1; ++i)
        for (long long j = c0; j < c1; ++j) kept += keep(p, i, j) ? 1 : 0;
      if (kept == 0) continue;
      if (out && n < cap) {
        out[3 * n + 0] = int(qb);
        out[3 * n + 1] = int(kb);
        out[3 * n + 2] = kept == (r1 - r0) * (c1 - c0) ? 1 : 0;
      }
      ++n;
    }
  }
  *count = n;
  return 0;
}

// Same list by the row-interval method: K_i is [0, i] for causal rows and
// last-L rows, else the union of the sink interval [0, min(S, i+1)) and the
// window [max(0, i-W+1), i]. Per tile the kept count is the sum over its rows
// of |K_i intersected with the tile's columns|. Usable at N = 128K.
int oracle_tile_list_rows(int N, int causal, int S, int W, int L, int BM, int BN, int* out,
                          long long cap, long long* count) {
  Pattern p;
  if (!make_pattern(N, causal, S, W, L, &p) || BM < 1 || BN < 1 || !count) return -1;
  auto overlap = [](long long a0, long long a1, long long b0, long long b1) {  // half-open
    return std::max(0LL, std::min(a1, b1) - std::max(a0, b0));
  };
  const long long nqb = (N + BM - 1) / BM, nkb = (N + BN - 1) / BN;
  long long n = 0;
  for (long long qb = 0; qb < nqb; ++qb) {
    const long long r0 = qb * BM, r1 = std::min<long long>(N, r0 + BM);
    for (long long kb = 0; kb < nkb; ++kb) {
      const long long c0 = kb * BN, c1 = std::min<long long>(N, c0 + BN);
      long long kept = 0;
      for (long long i = r0; i < r1; ++i) {
        if (p.causal || i >= p.N - p.L) {
          kept += overlap(0, i + 1, c0, c1);
        } else {
          const long long se = std::min(p.S, i + 1);          // sinks [0, se)
          const long long wb = std::max(0LL, i - p.W + 1);    // window [wb, i]
          kept += overlap(0, se, c0, c1) + overlap(wb, i + 1, c0, c1) -
                  overlap(std::max(0LL, wb), std::min(se, i + 1), c0, c1);
        }
      }
      if (kept == 0) continue;
      if (out && n < cap) {
        out[3 * n + 0] = int(qb);
        out[3 * n + 1] = int(kb);
        out[3 * n + 2] = kept == (r1 - r0) * (c1 - c0) ? 1 : 0;
      }
      ++n;
    }
  }
  *count = n;
  return 0;
}

int oracle_hardware_threads(void) {
  unsigned n = std::thread::hardware_concurrency();
  return n ? int(n) : 1;
}

}  // extern "C"
