// Infini-attention layer forward: plain, slow, double-precision CPU oracle.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or
// load this file; only the tests, the smoke check and the CPU-baseline leg of
// the benchmark do. It shares no code, header, table or helper with the CUDA
// library: every step below is written out from the method's definition.
//
// Sources (web pages on the method; cited by title and section):
//  [HF]  "Hugging Face Infini-Attention reproduction analysis", section
//        "Infini-Attention mechanism", steps Segmentation, Local Attention,
//        Memory Retrieval, Integration, Memory Update, State Transfer.
//  [KV]  "KV linear-addition Infini-attention" (forum summary of "Leave No
//        Context Behind"): masked local attention plus long-term *linear*
//        attention in one block; standard scaled dot-product attention;
//        causal dot-product attention inside each segment.
// The pages give the steps in prose only. The formulas below are the plain
// reading of those steps that the layer's specification fixes:
//   A_dot = softmax(Q K^T / sqrt(d), causal incl. diagonal) V   (per segment)
//   A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}),  A_mem = 0 where the
//           denominator is 0,  sigma(x) = ELU(x) + 1 (alpha = 1)
//   A     = sigmoid(beta_h) A_mem + (1 - sigmoid(beta_h)) A_dot
//   M_s   = M_{s-1} + sigma(K)^T V,   z_s = z_{s-1} + sum_t sigma(K_t)
// Only (M, z) crosses segment and call boundaries [HF State Transfer].
//
// Every accumulation is in double; inputs arrive as fp32, bf16 bit patterns or
// double and are widened exactly. No blocking, fusion or reordering beyond the
// definition: for each query row the scores, the softmax, the retrieval and
// the gate are computed in the order written above; the memory update is
// applied token by token after the whole segment has been read.
//
// The decode step (one new token at position pos of its segment, attending to
// the segment's cached keys 0..pos and to the memory of earlier segments; the
// cached segment is folded into (M, z) after its last token) is the same
// definition taken one query row at a time [HF State Transfer; KV streaming].
//
// Parity status: pinned (see the oracle self-tests): causal softmax attention
// against a library SDPA, the memory-only output against a brute-force sum
// that never forms M, the final state against a library matmul, streaming
// identity, constant-V and linearity invariants, a hand-computed d=1 case and
// permutation invariance of earlier segments.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

enum { IN_F32 = 0, IN_BF16 = 1, IN_F64 = 2 };

// Widen one stored element to double. bf16 is the top 16 bits of an IEEE
// binary32 value, so shifting the bits up by 16 recovers it exactly.
double widen(const void* base, int dtype, int64_t idx) {
  if (dtype == IN_F64) return static_cast<const double*>(base)[idx];
  if (dtype == IN_F32) return static_cast<double>(static_cast<const float*>(base)[idx]);
  uint32_t bits = static_cast<uint32_t>(static_cast<const uint16_t*>(base)[idx]) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return static_cast<double>(f);
}

// sigma(x) = ELU(x) + 1 with alpha = 1 [HF Memory Retrieval: "ELU + 1"].
double sigma(double x) { return x > 0.0 ? x + 1.0 : std::exp(x); }

// sigmoid gate [HF Integration]; beta = +inf -> 1, -inf -> 0 by IEEE rules.
double sigmoid(double b) { return 1.0 / (1.0 + std::exp(-b)); }

struct Problem {
  int64_t B, H, L, d, N;
  const void *q, *k, *v;
  int dtype;
  const double* beta;   // [H]
  const double* M_in;   // [B,H,d,d] or null (zero state)
  const double* z_in;   // [B,H,d]   or null
  // Output rows: either all segments (seg_list == null) or the listed ones.
  const int64_t* seg_list;
  int64_t n_seg_out;
  double* out;          // [B,H,L,d] or [B,H,n_seg_out,N,d]
  double* M_out;        // [B,H,d,d]
  double* z_out;        // [B,H,d]
};

// One (b, h) pair: walk the segments in order [HF Segmentation].
void run_head(const Problem& P, int64_t b, int64_t h) {
  const int64_t d = P.d, N = P.N, L = P.L, S = L / N;
  const int64_t bh = b * P.H + h;
  const int64_t row0 = bh * L;  // first token row of this (b, h) in [B,H,L,d]
  const double inv_sqrt_d = 1.0 / std::sqrt(static_cast<double>(d));
  const double g = sigmoid(P.beta[h]);

  std::vector<double> M(d * d, 0.0), z(d, 0.0);
  if (P.M_in) {
    for (int64_t i = 0; i < d * d; ++i) M[i] = P.M_in[bh * d * d + i];
    for (int64_t i = 0; i < d; ++i) z[i] = P.z_in[bh * d + i];
  }

  // Which output slot (if any) each segment writes.
  std::vector<int64_t> slot(S, -1);
  if (P.seg_list) {
    for (int64_t i = 0; i < P.n_seg_out; ++i)
      if (P.seg_list[i] >= 0 && P.seg_list[i] < S) slot[P.seg_list[i]] = i;
  } else {
    for (int64_t s = 0; s < S; ++s) slot[s] = s;
  }

  std::vector<double> qrow(d), score(N), adot(d), sq(d), num(d);
  std::vector<double> kseg(N * d), vseg(N * d);  // the segment's keys and values, widened
  for (int64_t s = 0; s < S; ++s) {
    const int64_t base = row0 + s * N;  // first token row of segment s
    for (int64_t e = 0; e < N * d; ++e) {
      kseg[e] = widen(P.k, P.dtype, base * d + e);
      vseg[e] = widen(P.v, P.dtype, base * d + e);
    }
    if (slot[s] >= 0) {
      double* out_seg = P.seg_list
          ? P.out + ((bh * P.n_seg_out + slot[s]) * N) * d
          : P.out + (row0 + s * N) * d;
      for (int64_t i = 0; i < N; ++i) {
        for (int64_t c = 0; c < d; ++c) qrow[c] = widen(P.q, P.dtype, (base + i) * d + c);

        // Local causal dot-product attention inside the segment, keys j <= i
        // [HF Local Attention; KV: scaled dot-product, causal per segment].
        double mx = -INFINITY;
        for (int64_t j = 0; j <= i; ++j) {
          double acc = 0.0;
          for (int64_t c = 0; c < d; ++c) acc += qrow[c] * kseg[j * d + c];
          score[j] = acc * inv_sqrt_d;
          if (score[j] > mx) mx = score[j];
        }
        double den_soft = 0.0;
        for (int64_t c = 0; c < d; ++c) adot[c] = 0.0;
        for (int64_t j = 0; j <= i; ++j) {
          const double p = std::exp(score[j] - mx);
          den_soft += p;
          for (int64_t c = 0; c < d; ++c) adot[c] += p * vseg[j * d + c];
        }
        for (int64_t c = 0; c < d; ++c) adot[c] /= den_soft;

        // Memory retrieval from M_{s-1}, z_{s-1} with sigma(Q) [HF Memory
        // Retrieval]; A_mem = 0 where the normaliser is 0.
        double den = 0.0;
        for (int64_t c = 0; c < d; ++c) {
          sq[c] = sigma(qrow[c]);
          den += sq[c] * z[c];
        }
        for (int64_t j = 0; j < d; ++j) num[j] = 0.0;
        for (int64_t c = 0; c < d; ++c)
          for (int64_t j = 0; j < d; ++j) num[j] += sq[c] * M[c * d + j];

        // Gate [HF Integration].
        for (int64_t j = 0; j < d; ++j) {
          const double amem = (den == 0.0) ? 0.0 : num[j] / den;
          out_seg[i * d + j] = g * amem + (1.0 - g) * adot[j];
        }
      }
    }
    // Memory update after the segment [HF Memory Update; KV linear addition]:
    // M += sigma(k_t) v_t^T, z += sigma(k_t), token by token.
    for (int64_t i = 0; i < N; ++i) {
      for (int64_t c = 0; c < d; ++c) {
        const double sk = sigma(kseg[i * d + c]);
        z[c] += sk;
        for (int64_t j = 0; j < d; ++j) M[c * d + j] += sk * vseg[i * d + j];
      }
    }
  }
  // State transfer: only (M, z) leaves the call [HF State Transfer].
  for (int64_t i = 0; i < d * d; ++i) P.M_out[bh * d * d + i] = M[i];
  for (int64_t i = 0; i < d; ++i) P.z_out[bh * d + i] = z[i];
}

void run_all(const Problem& P, int nthreads) {
  const int64_t units = P.B * P.H;
  if (nthreads <= 1 || units == 1) {
    for (int64_t u = 0; u < units; ++u) run_head(P, u / P.H, u % P.H);
    return;
  }
  // Independent (b, h) pairs split over threads; each pair is computed exactly
  // as in the sequential loop, so the result does not depend on nthreads.
  std::vector<std::thread> pool;
  for (int t = 0; t < nthreads; ++t) {
    pool.emplace_back([&P, t, nthreads, units]() {
      for (int64_t u = t; u < units; u += nthreads) run_head(P, u / P.H, u % P.H);
    });
  }
  for (auto& th : pool) th.join();
}

// One decode step for one (b, h): the query row at position pos of the current
// segment. Keys and values 0..pos-1 come from the cache, key/value pos is this
// token's. Output, then (after the segment's last token) the memory update of
// the whole segment in token order, exactly as run_head does it.
void decode_head(int64_t H, int64_t d, int64_t N, int64_t pos, int64_t b, int64_t h, const void* q,
                 const void* k, const void* v, const void* kc, const void* vc, int dtype, const double* beta,
                 double* M, double* z, double* out) {
  const int64_t bh = b * H + h;
  const double inv_sqrt_d = 1.0 / std::sqrt(static_cast<double>(d));
  const double g = sigmoid(beta[h]);
  double* Mh = M + bh * d * d;
  double* zh = z + bh * d;
  // The segment's keys and values seen so far, widened; row pos is this token.
  std::vector<double> kseg((pos + 1) * d), vseg((pos + 1) * d), qrow(d);
  for (int64_t j = 0; j < pos; ++j)
    for (int64_t c = 0; c < d; ++c) {
      kseg[j * d + c] = widen(kc, dtype, (bh * N + j) * d + c);
      vseg[j * d + c] = widen(vc, dtype, (bh * N + j) * d + c);
    }
  for (int64_t c = 0; c < d; ++c) {
    kseg[pos * d + c] = widen(k, dtype, bh * d + c);
    vseg[pos * d + c] = widen(v, dtype, bh * d + c);
    qrow[c] = widen(q, dtype, bh * d + c);
  }
  // Local causal attention over keys 0..pos [HF Local Attention].
  std::vector<double> score(pos + 1), adot(d, 0.0), sq(d), num(d, 0.0);
  double mx = -INFINITY;
  for (int64_t j = 0; j <= pos; ++j) {
    double acc = 0.0;
    for (int64_t c = 0; c < d; ++c) acc += qrow[c] * kseg[j * d + c];
    score[j] = acc * inv_sqrt_d;
    if (score[j] > mx) mx = score[j];
  }
  double den_soft = 0.0;
  for (int64_t j = 0; j <= pos; ++j) {
    const double p = std::exp(score[j] - mx);
    den_soft += p;
    for (int64_t c = 0; c < d; ++c) adot[c] += p * vseg[j * d + c];
  }
  for (int64_t c = 0; c < d; ++c) adot[c] /= den_soft;
  // Retrieval from the memory of earlier segments [HF Memory Retrieval].
  double den = 0.0;
  for (int64_t c = 0; c < d; ++c) {
    sq[c] = sigma(qrow[c]);
    den += sq[c] * zh[c];
  }
  for (int64_t c = 0; c < d; ++c)
    for (int64_t j = 0; j < d; ++j) num[j] += sq[c] * Mh[c * d + j];
  for (int64_t j = 0; j < d; ++j) {
    const double amem = (den == 0.0) ? 0.0 : num[j] / den;
    out[bh * d + j] = g * amem + (1.0 - g) * adot[j];
  }
  // The segment is complete: fold it into the memory [HF Memory Update].
  if (pos == N - 1) {
    for (int64_t i = 0; i < N; ++i)
      for (int64_t c = 0; c < d; ++c) {
        const double sk = sigma(kseg[i * d + c]);
        zh[c] += sk;
        for (int64_t j = 0; j < d; ++j) Mh[c * d + j] += sk * vseg[i * d + j];
      }
  }
}

// Backward of the forward above for one (b, h), derived from its definition
// by the chain rule (the pages give no gradient; every formula below follows
// from the forward's steps):
//   out_t = g A_mem,t + (1 - g) A_dot,t,   g = sigmoid(beta)
//     d beta += g (1 - g) sum_c dout_tc (A_mem,tc - A_dot,tc)
//   A_dot,t = sum_{j<=t} P_tj v_j,  P_t = softmax(q_t . k_j / sqrt(d))
//     with dA = (1 - g) dout_t:  dv_j += P_tj dA,  dP_tj = dA . v_j,
//     dS_tj = P_tj (dP_tj - sum_j' P_tj' dP_tj'),
//     dq_t += sum_j dS_tj k_j / sqrt(d),  dk_j += dS_tj q_t / sqrt(d)
//   A_mem,t = num / den, num = sigma(q_t)^T M_{s-1}, den = sigma(q_t) . z_{s-1}
//     (A_mem = 0 where den = 0: no gradient flows there)
//     with dA' = g dout_t: dnum = dA' / den, dden = -(dA' . A_mem) / den,
//     dsigma(q_t) = M_{s-1} dnum + z_{s-1} dden,  dq_t += dsigma(q_t) sigma'(q_t),
//     dM_{s-1} += sigma(q_t) dnum^T,  dz_{s-1} += sigma(q_t) dden
//   M_s = M_{s-1} + sum_{t in s} sigma(k_t) v_t^T (and z): with G_s the
//     gradient reaching M_s (dM_out plus every later segment's dM_{s'-1}),
//     dv_t += G_s^T sigma(k_t), dsigma(k_t) = G_s v_t + Gz_s,
//     dk_t += dsigma(k_t) sigma'(k_t); dM_in = G reaching M_in.
// sigma'(x) = 1 for x > 0, exp(x) otherwise.
struct BwdProblem {
  int64_t B, H, L, d, N;
  const void *q, *k, *v;
  int dtype;
  const double* beta;
  const double *M_in, *z_in;     // null = zero state
  const double* dout;            // [B,H,L,d]
  const double *dM_out, *dz_out; // null = zero
  double *dq, *dk, *dv;          // [B,H,L,d]
  double* dbeta;                 // [B,H]: per (b, h) share; the caller sums over b
  double *dM_in, *dz_in;         // [B,H,d,d], [B,H,d]
};

double dsigma(double x) { return x > 0.0 ? 1.0 : std::exp(x); }

void backward_head(const BwdProblem& P, int64_t b, int64_t h) {
  const int64_t d = P.d, N = P.N, L = P.L, S = L / N;
  const int64_t bh = b * P.H + h;
  const int64_t row0 = bh * L;
  const double inv_sqrt_d = 1.0 / std::sqrt(static_cast<double>(d));
  const double g = sigmoid(P.beta[h]);
  auto Q = [&](int64_t t, int64_t c) { return widen(P.q, P.dtype, (row0 + t) * d + c); };
  auto K = [&](int64_t t, int64_t c) { return widen(P.k, P.dtype, (row0 + t) * d + c); };
  auto V = [&](int64_t t, int64_t c) { return widen(P.v, P.dtype, (row0 + t) * d + c); };

  // Forward state chain: Mprev[s] = M_{s-1}, zprev[s] = z_{s-1}.
  std::vector<double> Mprev(S * d * d), zprev(S * d);
  {
    std::vector<double> M(d * d, 0.0), z(d, 0.0);
    if (P.M_in) {
      for (int64_t i = 0; i < d * d; ++i) M[i] = P.M_in[bh * d * d + i];
      for (int64_t i = 0; i < d; ++i) z[i] = P.z_in[bh * d + i];
    }
    for (int64_t s = 0; s < S; ++s) {
      for (int64_t i = 0; i < d * d; ++i) Mprev[s * d * d + i] = M[i];
      for (int64_t i = 0; i < d; ++i) zprev[s * d + i] = z[i];
      for (int64_t i = 0; i < N; ++i)
        for (int64_t c = 0; c < d; ++c) {
          const double sk = sigma(K(s * N + i, c));
          z[c] += sk;
          for (int64_t j = 0; j < d; ++j) M[c * d + j] += sk * V(s * N + i, j);
        }
    }
  }
  for (int64_t e = 0; e < L * d; ++e) {
    P.dq[row0 * d + e] = 0.0;
    P.dk[row0 * d + e] = 0.0;
    P.dv[row0 * d + e] = 0.0;
  }
  double dbeta = 0.0;
  // Gradient reaching M_{s-1} from segment s's queries.
  std::vector<double> dMprev(S * d * d, 0.0), dzprev(S * d, 0.0);
  std::vector<double> qrow(d), score(N), p(N), dp(N), adot(d), sq(d), num(d), amem(d), dA(d), dAm(d);
  for (int64_t s = 0; s < S; ++s) {
    const double* Ms = &Mprev[s * d * d];
    const double* zs = &zprev[s * d];
    for (int64_t i = 0; i < N; ++i) {
      const int64_t t = s * N + i;
      for (int64_t c = 0; c < d; ++c) qrow[c] = Q(t, c);
      // Local attention, recomputed.
      double mx = -INFINITY;
      for (int64_t j = 0; j <= i; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) acc += qrow[c] * K(s * N + j, c);
        score[j] = acc * inv_sqrt_d;
        if (score[j] > mx) mx = score[j];
      }
      double den_soft = 0.0;
      for (int64_t j = 0; j <= i; ++j) {
        p[j] = std::exp(score[j] - mx);
        den_soft += p[j];
      }
      for (int64_t j = 0; j <= i; ++j) p[j] /= den_soft;
      for (int64_t c = 0; c < d; ++c) {
        adot[c] = 0.0;
        for (int64_t j = 0; j <= i; ++j) adot[c] += p[j] * V(s * N + j, c);
      }
      // Retrieval, recomputed.
      double den = 0.0;
      for (int64_t c = 0; c < d; ++c) {
        sq[c] = sigma(qrow[c]);
        den += sq[c] * zs[c];
      }
      for (int64_t j = 0; j < d; ++j) {
        num[j] = 0.0;
        for (int64_t c = 0; c < d; ++c) num[j] += sq[c] * Ms[c * d + j];
        amem[j] = den == 0.0 ? 0.0 : num[j] / den;
      }
      const double* go = P.dout + (row0 + t) * d;
      // Gate.
      for (int64_t c = 0; c < d; ++c) {
        dbeta += g * (1.0 - g) * go[c] * (amem[c] - adot[c]);
        dA[c] = (1.0 - g) * go[c];
        dAm[c] = g * go[c];
      }
      // Local attention backward.
      double pdp = 0.0;
      for (int64_t j = 0; j <= i; ++j) {
        dp[j] = 0.0;
        for (int64_t c = 0; c < d; ++c) dp[j] += dA[c] * V(s * N + j, c);
        pdp += p[j] * dp[j];
      }
      for (int64_t j = 0; j <= i; ++j) {
        const double ds = p[j] * (dp[j] - pdp);
        for (int64_t c = 0; c < d; ++c) {
          P.dv[(row0 + s * N + j) * d + c] += p[j] * dA[c];
          P.dq[(row0 + t) * d + c] += ds * K(s * N + j, c) * inv_sqrt_d;
          P.dk[(row0 + s * N + j) * d + c] += ds * qrow[c] * inv_sqrt_d;
        }
      }
      // Retrieval backward.
      if (den != 0.0) {
        double dden = 0.0;
        for (int64_t j = 0; j < d; ++j) dden -= dAm[j] * amem[j];
        dden /= den;
        for (int64_t c = 0; c < d; ++c) {
          double dsq = zs[c] * dden;
          for (int64_t j = 0; j < d; ++j) {
            const double dnum = dAm[j] / den;
            dsq += Ms[c * d + j] * dnum;
            dMprev[s * d * d + c * d + j] += sq[c] * dnum;
          }
          dzprev[s * d + c] += sq[c] * dden;
          P.dq[(row0 + t) * d + c] += dsq * dsigma(qrow[c]);
        }
      }
    }
  }
  // State chain backward: G = gradient reaching M_s, from the last segment down.
  std::vector<double> G(d * d, 0.0), Gz(d, 0.0);
  if (P.dM_out) {
    for (int64_t i = 0; i < d * d; ++i) G[i] = P.dM_out[bh * d * d + i];
    for (int64_t i = 0; i < d; ++i) Gz[i] = P.dz_out[bh * d + i];
  }
  for (int64_t s = S - 1; s >= 0; --s) {
    // Keys and values of segment s enter M_s.
    for (int64_t i = 0; i < N; ++i) {
      const int64_t t = s * N + i;
      for (int64_t c = 0; c < d; ++c) {
        double dsk = Gz[c];
        for (int64_t j = 0; j < d; ++j) dsk += G[c * d + j] * V(t, j);
        P.dk[(row0 + t) * d + c] += dsk * dsigma(K(t, c));
      }
      for (int64_t j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) acc += sigma(K(t, c)) * G[c * d + j];
        P.dv[(row0 + t) * d + j] += acc;
      }
    }
    // M_{s-1} feeds M_s and segment s's retrieval.
    for (int64_t e = 0; e < d * d; ++e) G[e] += dMprev[s * d * d + e];
    for (int64_t e = 0; e < d; ++e) Gz[e] += dzprev[s * d + e];
  }
  for (int64_t e = 0; e < d * d; ++e) P.dM_in[bh * d * d + e] = G[e];
  for (int64_t e = 0; e < d; ++e) P.dz_in[bh * d + e] = Gz[e];
  P.dbeta[bh] = dbeta;
}

int check(int64_t B, int64_t H, int64_t L, int64_t d, int64_t N, int dtype) {
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || N <= 0) return -2;
  if (L % N != 0) return -2;
  if (dtype != IN_F32 && dtype != IN_BF16 && dtype != IN_F64) return -3;
  return 0;
}

}  // namespace

extern "C" {

// Full forward. q, k, v: [B,H,L,d] in `dtype` (0 fp32, 1 bf16 bits, 2 double).
// beta [H], M_in [B,H,d,d], z_in [B,H,d] in double (M_in/z_in may be null for
// the zero state). out [B,H,L,d], M_out, z_out in double. Returns 0, or -2 for
// a bad shape (including L % N != 0), -3 for a bad dtype, -1 for a null.
int oracle_infini_forward(int64_t B, int64_t H, int64_t L, int64_t d, int64_t N,
                          const void* q, const void* k, const void* v, int dtype,
                          const double* beta, const double* M_in, const double* z_in,
                          double* out, double* M_out, double* z_out, int nthreads) {
  int rc = check(B, H, L, d, N, dtype);
  if (rc) return rc;
  if (!q || !k || !v || !beta || !out || !M_out || !z_out) return -1;
  if ((M_in == nullptr) != (z_in == nullptr)) return -1;
  Problem P{B, H, L, d, N, q, k, v, dtype, beta, M_in, z_in, nullptr, 0, out, M_out, z_out};
  run_all(P, nthreads);
  return 0;
}

// Same computation, but output rows are produced only for the listed segments
// (out: [B,H,n_seg,N,d]); the state chain still covers every segment.
int oracle_infini_forward_segments(int64_t B, int64_t H, int64_t L, int64_t d, int64_t N,
                                   const void* q, const void* k, const void* v, int dtype,
                                   const double* beta, const double* M_in, const double* z_in,
                                   const int64_t* seg_list, int64_t n_seg,
                                   double* out, double* M_out, double* z_out, int nthreads) {
  int rc = check(B, H, L, d, N, dtype);
  if (rc) return rc;
  if (!q || !k || !v || !beta || !M_out || !z_out || (n_seg > 0 && (!seg_list || !out))) return -1;
  if ((M_in == nullptr) != (z_in == nullptr)) return -1;
  Problem P{B, H, L, d, N, q, k, v, dtype, beta, M_in, z_in, seg_list, n_seg, out, M_out, z_out};
  run_all(P, nthreads);
  return 0;
}

// Backward. Inputs as for oracle_infini_forward plus dout [B,H,L,d] and the
// gradient of the output state dM_out [B,H,d,d], dz_out [B,H,d] (both null =
// zero), all double. Outputs (double): dq, dk, dv [B,H,L,d], dbeta [B,H] (the
// (b, h) shares; d loss / d beta_h is their sum over b), dM_in [B,H,d,d],
// dz_in [B,H,d]. Returns as the forward does.
int oracle_infini_backward(int64_t B, int64_t H, int64_t L, int64_t d, int64_t N, const void* q, const void* k,
                           const void* v, int dtype, const double* beta, const double* M_in, const double* z_in,
                           const double* dout, const double* dM_out, const double* dz_out, double* dq, double* dk,
                           double* dv, double* dbeta, double* dM_in, double* dz_in, int nthreads) {
  int rc = check(B, H, L, d, N, dtype);
  if (rc) return rc;
  if (!q || !k || !v || !beta || !dout || !dq || !dk || !dv || !dbeta || !dM_in || !dz_in) return -1;
  if ((M_in == nullptr) != (z_in == nullptr) || (dM_out == nullptr) != (dz_out == nullptr)) return -1;
  BwdProblem P{B, H, L, d, N, q, k, v, dtype, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv, dbeta, dM_in, dz_in};
  const int64_t units = B * H;
  if (nthreads <= 1 || units == 1) {
    for (int64_t u = 0; u < units; ++u) backward_head(P, u / H, u % H);
  } else {
    std::vector<std::thread> pool;
    for (int t = 0; t < nthreads; ++t)
      pool.emplace_back([&P, t, nthreads, units, H]() {
        for (int64_t u = t; u < units; u += nthreads) backward_head(P, u / H, u % H);
      });
    for (auto& th : pool) th.join();
  }
  return 0;
}

// One decode step. q, k, v: [B,H,d] (this token) and k_cache, v_cache:
// [B,H,N,d] (rows 0..pos-1 used) in `dtype`; beta [H]; M [B,H,d,d] and z
// [B,H,d] in double, in/out (the memory of earlier segments; the segment is
// folded in when pos == N - 1); out [B,H,d] in double. Returns 0, -2 for a bad
// shape or position, -3 for a bad dtype, -1 for a null.
int oracle_infini_decode_step(int64_t B, int64_t H, int64_t d, int64_t N, int64_t pos, const void* q,
                              const void* k, const void* v, const void* k_cache, const void* v_cache,
                              int dtype, const double* beta, double* M, double* z, double* out) {
  int rc = check(B, H, N, d, N, dtype);
  if (rc) return rc;
  if (pos < 0 || pos >= N) return -2;
  if (!q || !k || !v || !beta || !M || !z || !out || (pos > 0 && (!k_cache || !v_cache))) return -1;
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < H; ++h)
      decode_head(H, d, N, pos, b, h, q, k, v, k_cache, v_cache, dtype, beta, M, z, out);
  return 0;
}

}  // extern "C"
