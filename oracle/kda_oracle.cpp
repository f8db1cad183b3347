// KDA oracle -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, fp64 CPU implementation of the Kimi Delta Attention (KDA)
// forward pass. It exists to check the CUDA path: only the tests, the smoke
// check and the bench's CPU-baseline leg may load it. It shares no code,
// header, table or helper with the CUDA library.
//
// What it computes (per sequence of a cu_seqlens-packed batch, per head):
//
//   S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
//   o_t = scale * S_t^T q_t
//
// S is dk x dv (rows = key channels, columns = value channels), g_t is a
// natural-log decay per key channel, beta_t a scalar per token and head.
// Sources: KDA refines Gated DeltaNet by giving every channel its own decay
// instead of one scalar decay for the whole state, and keeps the history in a
// fixed-size recurrent state (page "Kimi K3 开源满月…", section
// "KDA 内核到底难在哪"; page "FlashKDA: CUTLASS Kernel من Moonshot لـ Kimi",
// section "سياق Kimi Linear"). Variable-length packing follows the
// FlashAttention cu_seqlens convention (same FlashKDA page, section
// "تكامل مباشر مع flash-linear-attention").
//
// Readings taken where the pages are silent:
//   * g_t scales the KEY rows of S (Diag multiplies S from the left).
//   * decay first, then erase, then write -- exactly the order of the formula.
//   * o_t reads S_t, i.e. after token t's own decay and write.
//   * every sequence starts from its initial state (or zero) and its cumulative
//     decay restarts at the sequence start.
//   * inputs are widened exactly to fp64 (bf16 bit patterns, fp32 values);
//     all arithmetic is fp64 with std::exp.
//
// Entry points (extern "C", called through ctypes by the tests):
//   kda_oracle_scan_bf16   -- the token-by-token recurrence on library-format
//                             inputs (bf16 q/k/v, fp32 g/beta/state).
//   kda_oracle_scan_f64    -- the same recurrence on fp64 inputs.
//   kda_oracle_chunked_f64 -- a naive chunked (WY-form) rewrite of the same
//                             recurrence; the blueprint of the CUDA algorithm,
//                             checked against the scan.
//   kda_oracle_unit_lower_inverse -- (I + L)^{-1} for strictly lower L, by
//                             forward substitution or by the Neumann/doubling
//                             product (page "Kimi K3 开源满月…", section
//                             "KDA 内核到底难在哪": L^16 = 0 for 16x16 L).
//   kda_oracle_backward_*  -- the reverse-mode derivative of the recurrence
//                             (gradients of q, k, v, g, beta and the initial
//                             state for given output and final-state
//                             gradients), token by token.
//   kda_oracle_preprocess  -- the gate preprocessing that precedes the
//                             recurrence in a layer: q, k L2-normalised per
//                             (token, head); g = max(log sigmoid(x), lower_bound)
//                             from gate logits x (the lower bound that keeps
//                             the decay range bounded, page "Kimi K3 开源满月…",
//                             section "KDA 内核到底难在哪"); beta = sigmoid(b)
//                             from logits b.
//
// Parity status: the scan is pinned by closed forms and invariants in
// tests/test_oracle_pins.py; the chunked rewrite is pinned by agreement with
// the scan. No function here is "parity unpinned".

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

inline double widen(uint16_t bf16_bits) {
  uint32_t u = static_cast<uint32_t>(bf16_bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof(f));
  return static_cast<double>(f);
}
inline double widen(float x) { return static_cast<double>(x); }
inline double widen(double x) { return x; }

// Element types: TV for q/k/v (uint16 bf16 bits or double), TG for g, beta and
// the initial state (float or double).
template <class TV, class TG>
struct ScanProblem {
  const TV* q;
  const TV* k;
  const TV* v;
  const TG* g;
  const TG* beta;
  int64_t T;
  int32_t H, dk, dv;
  const int32_t* cu;      // [nseq + 1]
  int32_t nseq;
  double scale;
  const TG* init;         // [nseq, H, dk, dv] or nullptr (zero state)
  double* out;            // [T, H, dv] or nullptr
  double* fin;            // [nseq, H, dk, dv] or nullptr
  int32_t erase;          // 1: the KDA recurrence; 0: drop the erase term
  int32_t col_begin, col_end;  // value columns computed
};

// One (sequence, head, value-column block). Columns of S evolve independently
// (the recurrence multiplies S only from the left), so a block of columns is
// computed with exactly the arithmetic of the full matrix, column by column.
template <class TV, class TG>
void scan_block(const ScanProblem<TV, TG>& P, int seq, int h, int c0, int c1) {
  const int dk = P.dk, dv = P.dv, nb = c1 - c0, H = P.H;
  const int64_t t0 = P.cu[seq], t1 = P.cu[seq + 1];
  std::vector<double> S(static_cast<size_t>(dk) * nb), kS(nb);
  auto Sat = [&](int r, int c) -> double& { return S[static_cast<size_t>(r) * nb + c]; };

  for (int r = 0; r < dk; ++r)
    for (int c = 0; c < nb; ++c)
      Sat(r, c) = P.init ? widen(P.init[((static_cast<size_t>(seq) * H + h) * dk + r) * dv + c0 + c])
                         : 0.0;

  for (int64_t t = t0; t < t1; ++t) {
    const size_t bk = (static_cast<size_t>(t) * H + h) * dk;
    const size_t bv = (static_cast<size_t>(t) * H + h) * dv;
    const double b = widen(P.beta[static_cast<size_t>(t) * H + h]);

    // (1) decay: S <- Diag(exp g_t) S  (row r = key channel r)
    for (int r = 0; r < dk; ++r) {
      const double d = std::exp(widen(P.g[bk + r]));
      for (int c = 0; c < nb; ++c) Sat(r, c) *= d;
    }
    // (2) erase and write: S <- S - b k (k^T S) + b k v^T
    for (int c = 0; c < nb; ++c) kS[c] = 0.0;
    for (int r = 0; r < dk; ++r) {
      const double kr = widen(P.k[bk + r]);
      for (int c = 0; c < nb; ++c) kS[c] += kr * Sat(r, c);
    }
    for (int r = 0; r < dk; ++r) {
      const double kr = widen(P.k[bk + r]);
      for (int c = 0; c < nb; ++c) {
        const double vc = widen(P.v[bv + c0 + c]);
        if (P.erase)
          Sat(r, c) = Sat(r, c) - b * kr * kS[c] + b * kr * vc;
        else
          Sat(r, c) = Sat(r, c) + b * kr * vc;
      }
    }
    // (3) output: o_t = scale * S^T q_t
    if (P.out) {
      for (int c = 0; c < nb; ++c) kS[c] = 0.0;  // reused as the output accumulator
      for (int r = 0; r < dk; ++r) {
        const double qr = widen(P.q[bk + r]);
        for (int c = 0; c < nb; ++c) kS[c] += qr * Sat(r, c);
      }
      for (int c = 0; c < nb; ++c) P.out[bv + c0 + c] = P.scale * kS[c];
    }
  }
  if (P.fin)
    for (int r = 0; r < dk; ++r)
      for (int c = 0; c < nb; ++c)
        P.fin[((static_cast<size_t>(seq) * H + h) * dk + r) * dv + c0 + c] = Sat(r, c);
}

template <class F>
void parallel_for(int64_t n, int nthreads, F&& f) {
  if (nthreads <= 0) nthreads = static_cast<int>(std::thread::hardware_concurrency());
  if (nthreads <= 0) nthreads = 1;
  if (nthreads > n) nthreads = static_cast<int>(n > 0 ? n : 1);
  std::atomic<int64_t> next(0);
  auto worker = [&]() {
    for (;;) {
      const int64_t i = next.fetch_add(1);
      if (i >= n) break;
      f(i);
    }
  };
  if (nthreads == 1) {
    worker();
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(nthreads);
  for (int i = 0; i < nthreads; ++i) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
}

int check_common(int64_t T, int32_t H, int32_t dk, int32_t dv, const int32_t* cu, int32_t nseq,
                 int32_t col_begin, int32_t col_end) {
  if (T < 0 || H <= 0 || dk <= 0 || dv <= 0 || nseq < 0 || !cu) return 1;
  if (cu[0] != 0 || cu[nseq] != T) return 2;
  for (int i = 0; i < nseq; ++i)
    if (cu[i + 1] < cu[i]) return 3;
  if (col_begin < 0 || col_end > dv || col_begin > col_end) return 4;
  return 0;
}

template <class TV, class TG>
int run_scan(const ScanProblem<TV, TG>& P, int32_t col_block, int32_t nthreads) {
  int rc = check_common(P.T, P.H, P.dk, P.dv, P.cu, P.nseq, P.col_begin, P.col_end);
  if (rc) return rc;
  const int ncols = P.col_end - P.col_begin;
  if (ncols == 0) return 0;
  if (col_block <= 0 || col_block > ncols) col_block = ncols;
  const int nblk = (ncols + col_block - 1) / col_block;
  // Longest sequences first so the thread pool drains evenly.
  std::vector<int> order(P.nseq);
  for (int i = 0; i < P.nseq; ++i) order[i] = i;
  for (int i = 1; i < P.nseq; ++i)
    for (int j = i; j > 0 && (P.cu[order[j] + 1] - P.cu[order[j]]) >
                                 (P.cu[order[j - 1] + 1] - P.cu[order[j - 1]]);
         --j)
      std::swap(order[j], order[j - 1]);
  const int64_t items = static_cast<int64_t>(P.nseq) * P.H * nblk;
  parallel_for(items, nthreads, [&](int64_t i) {
    const int b = static_cast<int>(i % nblk);
    const int h = static_cast<int>((i / nblk) % P.H);
    const int s = order[static_cast<int>(i / (static_cast<int64_t>(nblk) * P.H))];
    const int c0 = P.col_begin + b * col_block;
    const int c1 = c0 + col_block < P.col_end ? c0 + col_block : P.col_end;
    scan_block(P, s, h, c0, c1);
  });
  return 0;
}

// ---------------------------------------------------------------------------
// Naive chunked rewrite (fp64, all value columns, one thread per (seq, head)).
//
// Within a chunk of m tokens starting from state S0, with G_i the inclusive
// cumulative sum of g over the chunk (i = 0..m-1):
//   A[i][j]   = sum_r k_i[r] k_j[r] exp(G_i[r] - G_j[r])        (j < i)
//   T         = (I + diag(beta) A)^{-1}                          (unit lower)
//   W         = T diag(beta) (k_j * exp(G_j))_j                  (m x dk)
//   U         = T diag(beta) V                                   (m x dv)
//   Vnew      = U - W S0                                         (the delta-rule
//               writes u_i = beta_i (v_i - (D_i S_{i-1})^T k_i) of the chunk)
//   Aqk[i][j] = sum_r q_i[r] k_j[r] exp(G_i[r] - G_j[r])        (j <= i)
//   O         = scale (Qd S0 + Aqk Vnew),  Qd_i = q_i * exp(G_i)
//   S         = Diag(exp G_{m-1}) S0 + Kend^T Vnew,  Kend_j = k_j * exp(G_{m-1} - G_j)
// This is the chunk-local "small dense matrix" form of the recurrence that the
// FlashKDA description relies on (page "Kimi K3 开源满月…", section
// "KDA 内核到底难在哪": 16-token chunks rewritten as small matrix products with
// one state chain across chunks). The exponentials are evaluated directly from
// differences of G, which fp64 range allows at any chunk size used here.
// ---------------------------------------------------------------------------
void forward_substitution_inverse(const std::vector<double>& L, int n, std::vector<double>& X) {
  // Solve (I + L) X = I column by column; L strictly lower, row-major n x n.
  X.assign(static_cast<size_t>(n) * n, 0.0);
  for (int col = 0; col < n; ++col) {
    for (int i = 0; i < n; ++i) {
      double acc = (i == col) ? 1.0 : 0.0;
      for (int j = 0; j < i; ++j) acc -= L[static_cast<size_t>(i) * n + j] * X[static_cast<size_t>(j) * n + col];
      X[static_cast<size_t>(i) * n + col] = acc;
    }
  }
}

void matmul(const std::vector<double>& A, const std::vector<double>& B, std::vector<double>& C, int n) {
  C.assign(static_cast<size_t>(n) * n, 0.0);
  for (int i = 0; i < n; ++i)
    for (int k = 0; k < n; ++k) {
      const double a = A[static_cast<size_t>(i) * n + k];
      for (int j = 0; j < n; ++j) C[static_cast<size_t>(i) * n + j] += a * B[static_cast<size_t>(k) * n + j];
    }
}

// (I + L)^{-1} = sum_{p<n} (-L)^p = (I - L)(I + L^2)(I + L^4)...(I + L^{2^s}), 2^{s+1} >= n.
void doubling_inverse(const std::vector<double>& L, int n, std::vector<double>& X) {
  X.assign(static_cast<size_t>(n) * n, 0.0);
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j)
      X[static_cast<size_t>(i) * n + j] = (i == j ? 1.0 : 0.0) - L[static_cast<size_t>(i) * n + j];
  std::vector<double> Q = L, Q2, F, tmp;
  for (int span = 2; span < n; span *= 2) {
    matmul(Q, Q, Q2, n);  // Q = L^span
    Q.swap(Q2);
    F = Q;
    for (int i = 0; i < n; ++i) F[static_cast<size_t>(i) * n + i] += 1.0;
    matmul(X, F, tmp, n);
    X.swap(tmp);
  }
}

void chunked_one(const double* q, const double* k, const double* v, const double* g, const double* beta,
                 int H, int dk, int dv, int64_t t0, int64_t t1, int h, double scale, const double* init,
                 double* out, double* fin, int C) {
  std::vector<double> S(static_cast<size_t>(dk) * dv, 0.0);
  if (init) std::memcpy(S.data(), init, sizeof(double) * dk * dv);
  auto K = [&](int64_t t, int r) { return k[(static_cast<size_t>(t) * H + h) * dk + r]; };
  auto Qv = [&](int64_t t, int r) { return q[(static_cast<size_t>(t) * H + h) * dk + r]; };
  auto V = [&](int64_t t, int c) { return v[(static_cast<size_t>(t) * H + h) * dv + c]; };
  auto Gin = [&](int64_t t, int r) { return g[(static_cast<size_t>(t) * H + h) * dk + r]; };
  auto B = [&](int64_t t) { return beta[static_cast<size_t>(t) * H + h]; };

  for (int64_t s0 = t0; s0 < t1; s0 += C) {
    const int m = static_cast<int>((t1 - s0) < C ? (t1 - s0) : C);
    std::vector<double> G(static_cast<size_t>(m) * dk);
    for (int r = 0; r < dk; ++r) {
      double acc = 0.0;
      for (int i = 0; i < m; ++i) {
        acc += Gin(s0 + i, r);
        G[static_cast<size_t>(i) * dk + r] = acc;
      }
    }
    auto Gat = [&](int i, int r) { return G[static_cast<size_t>(i) * dk + r]; };
    std::vector<double> L(static_cast<size_t>(m) * m, 0.0), Aqk(static_cast<size_t>(m) * m, 0.0);
    for (int i = 0; i < m; ++i)
      for (int j = 0; j <= i; ++j) {
        double a = 0.0, aq = 0.0;
        for (int r = 0; r < dk; ++r) {
          const double e = std::exp(Gat(i, r) - Gat(j, r));
          a += K(s0 + i, r) * K(s0 + j, r) * e;
          aq += Qv(s0 + i, r) * K(s0 + j, r) * e;
        }
        if (j < i) L[static_cast<size_t>(i) * m + j] = B(s0 + i) * a;
        Aqk[static_cast<size_t>(i) * m + j] = aq;
      }
    std::vector<double> Tm;
    forward_substitution_inverse(L, m, Tm);
    // W = T diag(beta) Kd,  U = T diag(beta) V
    std::vector<double> W(static_cast<size_t>(m) * dk, 0.0), U(static_cast<size_t>(m) * dv, 0.0);
    for (int i = 0; i < m; ++i)
      for (int j = 0; j <= i; ++j) {
        const double tb = Tm[static_cast<size_t>(i) * m + j] * B(s0 + j);
        for (int r = 0; r < dk; ++r) W[static_cast<size_t>(i) * dk + r] += tb * K(s0 + j, r) * std::exp(Gat(j, r));
        for (int c = 0; c < dv; ++c) U[static_cast<size_t>(i) * dv + c] += tb * V(s0 + j, c);
      }
    // Vnew = U - W S
    std::vector<double> Vn(static_cast<size_t>(m) * dv);
    for (int i = 0; i < m; ++i)
      for (int c = 0; c < dv; ++c) {
        double acc = U[static_cast<size_t>(i) * dv + c];
        for (int r = 0; r < dk; ++r) acc -= W[static_cast<size_t>(i) * dk + r] * S[static_cast<size_t>(r) * dv + c];
        Vn[static_cast<size_t>(i) * dv + c] = acc;
      }
    // O = scale (Qd S + Aqk Vnew)
    if (out)
      for (int i = 0; i < m; ++i)
        for (int c = 0; c < dv; ++c) {
          double acc = 0.0;
          for (int r = 0; r < dk; ++r) acc += Qv(s0 + i, r) * std::exp(Gat(i, r)) * S[static_cast<size_t>(r) * dv + c];
          for (int j = 0; j <= i; ++j) acc += Aqk[static_cast<size_t>(i) * m + j] * Vn[static_cast<size_t>(j) * dv + c];
          out[(static_cast<size_t>(s0 + i) * H + h) * dv + c] = scale * acc;
        }
    // S = Diag(exp G_{m-1}) S + Kend^T Vnew
    for (int r = 0; r < dk; ++r) {
      const double gam = std::exp(Gat(m - 1, r));
      for (int c = 0; c < dv; ++c) {
        double acc = gam * S[static_cast<size_t>(r) * dv + c];
        for (int j = 0; j < m; ++j)
          acc += K(s0 + j, r) * std::exp(Gat(m - 1, r) - Gat(j, r)) * Vn[static_cast<size_t>(j) * dv + c];
        S[static_cast<size_t>(r) * dv + c] = acc;
      }
    }
  }
  if (fin) std::memcpy(fin, S.data(), sizeof(double) * dk * dv);
}

// ------------------------------------------------------------------ backward
// Reverse-mode derivative of the token recurrence for one (sequence, head).
// Per token t (S_{t-1} -> S_t), with S' = Diag(exp g) S_{t-1}, u = v - S'^T k:
//   S_t = S' + beta k u^T = (I - beta k k^T) S' + beta k v^T,  o_t = scale S_t^T q.
// Walking t backwards with L = dLoss/dS_t (the final-state gradient at t = T):
//   L   += scale q dO^T            dq = scale S_t dO
//   lk   = L^T k                   dv = beta lk,   dbeta = lk . u
//   dk   = beta L u - beta S' lk   (through the write and through u = v - S'^T k)
//   dS'  = L - beta k lk^T         dg_r = sum_c dS'_rc S'_rc
//   L    = Diag(exp g) dS'         (dLoss/dS_{t-1}); at the start, d initial state = L.
// The states of a sequence are recomputed segment by segment from checkpoints
// taken every kCheckpoint tokens of a first forward pass.
template <class TV, class TG>
struct BackwardProblem {
  const TV* q;
  const TV* k;
  const TV* v;
  const TG* g;
  const TG* beta;
  int64_t T;
  int32_t H, dk, dv;
  const int32_t* cu;
  int32_t nseq;
  double scale;
  const TG* init;    // [nseq, H, dk, dv] or nullptr
  const TV* dout;    // [T, H, dv]
  const TG* dfin;    // [nseq, H, dk, dv] or nullptr
  double *dq, *dk_out, *dv_out, *dg, *dbeta;  // [T, H, dk], [T, H, dk], [T, H, dv], [T, H, dk], [T, H]
  double* dinit;     // [nseq, H, dk, dv] or nullptr
};

constexpr int kCheckpoint = 64;

template <class TV, class TG>
void backward_one(const BackwardProblem<TV, TG>& P, int seq, int h) {
  const int dk = P.dk, dv = P.dv, H = P.H;
  const int64_t t0 = P.cu[seq], t1 = P.cu[seq + 1], len = t1 - t0;
  const size_t SS = static_cast<size_t>(dk) * dv;
  const size_t so = (static_cast<size_t>(seq) * H + h) * SS;
  auto kat = [&](int64_t t, int r) { return widen(P.k[(static_cast<size_t>(t) * H + h) * dk + r]); };
  auto qat = [&](int64_t t, int r) { return widen(P.q[(static_cast<size_t>(t) * H + h) * dk + r]); };
  auto vat = [&](int64_t t, int c) { return widen(P.v[(static_cast<size_t>(t) * H + h) * dv + c]); };
  auto gat = [&](int64_t t, int r) { return widen(P.g[(static_cast<size_t>(t) * H + h) * dk + r]); };
  auto bat = [&](int64_t t) { return widen(P.beta[static_cast<size_t>(t) * H + h]); };
  // one forward step S <- (I - b k k^T) Diag(exp g) S + b k v^T (the scan's arithmetic)
  std::vector<double> kS(dv);
  auto step = [&](std::vector<double>& S, int64_t t) {
    for (int r = 0; r < dk; ++r) {
      const double d = std::exp(gat(t, r));
      for (int c = 0; c < dv; ++c) S[r * dv + c] *= d;
    }
    for (int c = 0; c < dv; ++c) kS[c] = 0.0;
    for (int r = 0; r < dk; ++r)
      for (int c = 0; c < dv; ++c) kS[c] += kat(t, r) * S[r * dv + c];
    const double b = bat(t);
    for (int r = 0; r < dk; ++r)
      for (int c = 0; c < dv; ++c) S[r * dv + c] += b * kat(t, r) * (vat(t, c) - kS[c]);
  };
  std::vector<double> S(SS, 0.0);
  if (P.init)
    for (size_t i = 0; i < SS; ++i) S[i] = widen(P.init[so + i]);
  const int64_t nck = len / kCheckpoint + 1;
  std::vector<double> ck(static_cast<size_t>(nck) * SS);
  for (int64_t t = t0; t < t1; ++t) {
    if ((t - t0) % kCheckpoint == 0) std::copy(S.begin(), S.end(), ck.begin() + ((t - t0) / kCheckpoint) * SS);
    step(S, t);
  }
  std::vector<double> L(SS, 0.0), Sp(SS), lk(dv), u(dv);
  if (P.dfin)
    for (size_t i = 0; i < SS; ++i) L[i] = widen(P.dfin[so + i]);
  std::vector<double> seg(static_cast<size_t>(kCheckpoint + 1) * SS);
  for (int64_t m = (len - 1) / kCheckpoint; m >= 0 && len > 0; --m) {
    const int64_t ts = t0 + m * kCheckpoint, te = std::min<int64_t>(ts + kCheckpoint, t1);
    // seg[j] = the state before token ts + j (j = 0 .. te - ts)
    std::copy(ck.begin() + m * SS, ck.begin() + (m + 1) * SS, seg.begin());
    for (int64_t t = ts; t < te; ++t) {
      const size_t j = static_cast<size_t>(t - ts);
      std::copy(seg.begin() + j * SS, seg.begin() + (j + 1) * SS, seg.begin() + (j + 1) * SS);
      std::vector<double> tmp(seg.begin() + (j + 1) * SS, seg.begin() + (j + 2) * SS);
      step(tmp, t);
      std::copy(tmp.begin(), tmp.end(), seg.begin() + (j + 1) * SS);
    }
    for (int64_t t = te - 1; t >= ts; --t) {
      const size_t j = static_cast<size_t>(t - ts);
      const double* Sprev = &seg[j * SS];
      const double* St = &seg[(j + 1) * SS];
      const size_t rk = (static_cast<size_t>(t) * H + h) * dk, rv = (static_cast<size_t>(t) * H + h) * dv;
      const double b = bat(t);
      // output t: L += scale q dO^T, dq = scale S_t dO
      for (int r = 0; r < dk; ++r) {
        double acc = 0.0;
        for (int c = 0; c < dv; ++c) {
          const double dov = widen(P.dout[rv + c]);
          L[r * dv + c] += P.scale * qat(t, r) * dov;
          acc += St[r * dv + c] * dov;
        }
        P.dq[rk + r] = P.scale * acc;
      }
      // S' = Diag(exp g) S_{t-1}, u = v - S'^T k
      for (int r = 0; r < dk; ++r) {
        const double d = std::exp(gat(t, r));
        for (int c = 0; c < dv; ++c) Sp[r * dv + c] = d * Sprev[r * dv + c];
      }
      for (int c = 0; c < dv; ++c) {
        double w = 0.0, l = 0.0;
        for (int r = 0; r < dk; ++r) {
          w += Sp[r * dv + c] * kat(t, r);
          l += L[r * dv + c] * kat(t, r);
        }
        u[c] = vat(t, c) - w;
        lk[c] = l;
      }
      double db = 0.0;
      for (int c = 0; c < dv; ++c) {
        P.dv_out[rv + c] = b * lk[c];
        db += lk[c] * u[c];
      }
      P.dbeta[static_cast<size_t>(t) * H + h] = db;
      for (int r = 0; r < dk; ++r) {
        double lu = 0.0, sl = 0.0;
        for (int c = 0; c < dv; ++c) {
          lu += L[r * dv + c] * u[c];
          sl += Sp[r * dv + c] * lk[c];
        }
        P.dk_out[rk + r] = b * lu - b * sl;
      }
      // dS' = L - b k lk^T; dg; L <- Diag(exp g) dS'
      for (int r = 0; r < dk; ++r) {
        const double kr = kat(t, r), d = std::exp(gat(t, r));
        double dgr = 0.0;
        for (int c = 0; c < dv; ++c) {
          const double dsp = L[r * dv + c] - b * kr * lk[c];
          dgr += dsp * Sp[r * dv + c];
          L[r * dv + c] = d * dsp;
        }
        P.dg[rk + r] = dgr;
      }
    }
  }
  if (P.dinit)
    for (size_t i = 0; i < SS; ++i) P.dinit[so + i] = L[i];
}

template <class TV, class TG>
int run_backward(const BackwardProblem<TV, TG>& P, int32_t nthreads) {
  int rc = check_common(P.T, P.H, P.dk, P.dv, P.cu, P.nseq, 0, P.dv);
  if (rc) return rc;
  if (!P.dout || !P.dq || !P.dk_out || !P.dv_out || !P.dg || !P.dbeta) return 1;
  parallel_for(static_cast<int64_t>(P.nseq) * P.H, nthreads, [&](int64_t i) {
    backward_one(P, static_cast<int>(i / P.H), static_cast<int>(i % P.H));
  });
  return 0;
}

}  // namespace

extern "C" {

// Token-by-token recurrence on library-format inputs.
//   q, k: uint16 bf16 bit patterns [T, H, dk]; v: [T, H, dv]
//   g: float32 [T, H, dk]; beta: float32 [T, H]
//   cu: int32 [nseq + 1] (cu[0] = 0, non-decreasing, cu[nseq] = T)
//   init: float32 [nseq, H, dk, dv] or NULL (zero state)
//   out: fp64 [T, H, dv] or NULL; fin: fp64 [nseq, H, dk, dv] or NULL
//   Only value columns [col_begin, col_end) are computed and written.
//   col_block: value columns per work item (<= 0: all); nthreads <= 0: all cores.
// Returns 0 on success, non-zero for invalid arguments (nothing written).
int kda_oracle_scan_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* g,
                         const float* beta, int64_t T, int32_t H, int32_t dk, int32_t dv,
                         const int32_t* cu, int32_t nseq, double scale, const float* init, double* out,
                         double* fin, int32_t erase, int32_t col_begin, int32_t col_end, int32_t col_block,
                         int32_t nthreads) {
  if (!q || !k || !v || !g || !beta) return 1;
  ScanProblem<uint16_t, float> P{q, k, v, g, beta, T, H, dk, dv, cu, nseq, scale, init, out, fin, erase,
                                 col_begin, col_end};
  return run_scan(P, col_block, nthreads);
}

// Same recurrence with every input in fp64.
int kda_oracle_scan_f64(const double* q, const double* k, const double* v, const double* g, const double* beta,
                        int64_t T, int32_t H, int32_t dk, int32_t dv, const int32_t* cu, int32_t nseq,
                        double scale, const double* init, double* out, double* fin, int32_t erase,
                        int32_t col_begin, int32_t col_end, int32_t col_block, int32_t nthreads) {
  if (!q || !k || !v || !g || !beta) return 1;
  ScanProblem<double, double> P{q, k, v, g, beta, T, H, dk, dv, cu, nseq, scale, init, out, fin, erase,
                                col_begin, col_end};
  return run_scan(P, col_block, nthreads);
}

// Naive chunked rewrite, fp64 inputs, chunk size C >= 1 (chunks restart at
// every sequence start; the last chunk of a sequence may be shorter).
int kda_oracle_chunked_f64(const double* q, const double* k, const double* v, const double* g,
                           const double* beta, int64_t T, int32_t H, int32_t dk, int32_t dv, const int32_t* cu,
                           int32_t nseq, double scale, const double* init, double* out, double* fin, int32_t C,
                           int32_t nthreads) {
  if (!q || !k || !v || !g || !beta || C <= 0) return 1;
  int rc = check_common(T, H, dk, dv, cu, nseq, 0, dv);
  if (rc) return rc;
  parallel_for(static_cast<int64_t>(nseq) * H, nthreads, [&](int64_t i) {
    const int s = static_cast<int>(i / H), h = static_cast<int>(i % H);
    const size_t so = (static_cast<size_t>(s) * H + h) * dk * dv;
    chunked_one(q, k, v, g, beta, H, dk, dv, cu[s], cu[s + 1], h, scale, init ? init + so : nullptr, out,
                fin ? fin + so : nullptr, C);
  });
  return 0;
}

// (I + L)^{-1} for a strictly lower-triangular n x n L (row-major; entries on
// or above the diagonal are ignored). method 0: forward substitution;
// method 1: Neumann series by repeated squaring (doubling).
int kda_oracle_unit_lower_inverse(const double* L, int32_t n, double* X, int32_t method) {
  if (!L || !X || n <= 0) return 1;
  std::vector<double> Lm(static_cast<size_t>(n) * n, 0.0), Xm;
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < i; ++j) Lm[static_cast<size_t>(i) * n + j] = L[static_cast<size_t>(i) * n + j];
  if (method == 0)
    forward_substitution_inverse(Lm, n, Xm);
  else if (method == 1)
    doubling_inverse(Lm, n, Xm);
  else
    return 2;
  std::memcpy(X, Xm.data(), sizeof(double) * n * n);
  return 0;
}

// Gate preprocessing, fp64, elementwise except for the per-(token, head)
// norms:
//   q_hat = q / max(||q||_2, eps), k_hat likewise   (q, k: bf16 bit patterns [T, H, dk])
//   g     = max(log(sigmoid(x)), lower_bound)      (x: fp32 gate logits [T, H, dk])
//   beta  = sigmoid(b)                             (b: fp32 logits [T, H])
// log(sigmoid(x)) is evaluated as -log1p(exp(-x)) for x >= 0 and
// x - log1p(exp(x)) for x < 0 (no overflow for any x).
int kda_oracle_preprocess(const uint16_t* q, const uint16_t* k, const float* x, const float* b, int64_t T,
                          int32_t H, int32_t dk, double lower_bound, double eps, double* q_out, double* k_out,
                          double* g_out, double* beta_out) {
  if (!q || !k || !x || !b || !q_out || !k_out || !g_out || !beta_out || T < 0 || H < 1 || dk < 1) return 1;
  for (int64_t t = 0; t < T; ++t)
    for (int32_t h = 0; h < H; ++h) {
      const size_t row = (static_cast<size_t>(t) * H + h) * dk;
      double nq = 0.0, nk = 0.0;
      for (int32_t c = 0; c < dk; ++c) {
        nq += widen(q[row + c]) * widen(q[row + c]);
        nk += widen(k[row + c]) * widen(k[row + c]);
      }
      const double dq = std::max(std::sqrt(nq), eps), dkn = std::max(std::sqrt(nk), eps);
      for (int32_t c = 0; c < dk; ++c) {
        q_out[row + c] = widen(q[row + c]) / dq;
        k_out[row + c] = widen(k[row + c]) / dkn;
        const double xv = widen(x[row + c]);
        const double ls = xv >= 0.0 ? -std::log1p(std::exp(-xv)) : xv - std::log1p(std::exp(xv));
        g_out[row + c] = std::max(ls, lower_bound);
      }
      const double bv = widen(b[static_cast<size_t>(t) * H + h]);
      beta_out[static_cast<size_t>(t) * H + h] = 1.0 / (1.0 + std::exp(-bv));
    }
  return 0;
}

// Derivatives of the loss sum(dout * o) + sum(dfin * S_final) with respect to
// q, k, v, g, beta and the initial state (reverse mode of the token
// recurrence; see backward_one). Library-format inputs (bf16 bits for q, k, v
// and dout; float32 for g, beta, init and dfin); every output fp64.
// init, dfin and dinit may be NULL (zero initial state / no final-state
// gradient / not written).
int kda_oracle_backward_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* g,
                             const float* beta, int64_t T, int32_t H, int32_t dk, int32_t dv, const int32_t* cu,
                             int32_t nseq, double scale, const float* init, const uint16_t* dout, const float* dfin,
                             double* dq, double* dkk, double* dvv, double* dg, double* dbeta, double* dinit,
                             int32_t nthreads) {
  if (!q || !k || !v || !g || !beta) return 1;
  BackwardProblem<uint16_t, float> P{q, k, v, g, beta, T, H, dk, dv, cu, nseq, scale, init, dout, dfin,
                                     dq, dkk, dvv, dg, dbeta, dinit};
  return run_backward(P, nthreads);
}

// Same with every input in fp64.
int kda_oracle_backward_f64(const double* q, const double* k, const double* v, const double* g, const double* beta,
                            int64_t T, int32_t H, int32_t dk, int32_t dv, const int32_t* cu, int32_t nseq,
                            double scale, const double* init, const double* dout, const double* dfin, double* dq,
                            double* dkk, double* dvv, double* dg, double* dbeta, double* dinit, int32_t nthreads) {
  if (!q || !k || !v || !g || !beta) return 1;
  BackwardProblem<double, double> P{q, k, v, g, beta, T, H, dk, dv, cu, nseq, scale, init, dout, dfin,
                                    dq, dkk, dvv, dg, dbeta, dinit};
  return run_backward(P, nthreads);
}

int kda_oracle_abi_version(void) { return 1; }

}  // extern "C"
