// GPTQ weight rounding on the host, in fp64 (the pages' LLM pack builds its
// 4-bit weights with GPTQ on the composite-rotated weights: block 128,
// damping 0.05; "Omega-QVLA: Nen VLA W4A4 tren Edge", "Build LLM pack").
//
// The rotated weight columns are quantised one at a time with the RTN rule
// and per-row RTN scale; each column's rounding error, divided by the
// diagonal of U, is subtracted from every later column in proportion to the
// row of U, where U is the upper Cholesky factor of the inverse of the damped
// Hessian H = X'^T X' of the rotated calibration inputs.  The block size of
// the pages only groups those updates (it does not change the result); here
// every element still takes its updates in column order, one IEEE multiply
// and one subtract each (no fused operations), so the codes follow from
// (W', U) alone, whatever the grouping of rows or threads.
//
// The inverse factor never forms H^-1: with J the exchange matrix and
// J A J = L L^T (lower Cholesky), A = V V^T for the upper V = J L J, so
// A^-1 = V^-T V^-1 and, the Cholesky factor being unique, U = V^-1 =
// J L^-1 J.  One factorisation and one triangular inverse.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <condition_variable>
#include <cstring>
#include <mutex>
#include <thread>
#include <vector>

#include "qvla_internal.h"

namespace qvla {
namespace {

unsigned host_threads() {
  return std::max(1u, std::min(32u, std::thread::hardware_concurrency()));
}

// Dot product of two contiguous fp64 runs, four partial sums.
double dot4(const double* a, const double* b, int n) {
  double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
  int k = 0;
  for (; k + 4 <= n; k += 4) {
    s0 += a[k] * b[k];
    s1 += a[k + 1] * b[k + 1];
    s2 += a[k + 2] * b[k + 2];
    s3 += a[k + 3] * b[k + 3];
  }
  for (; k < n; ++k) s0 += a[k] * b[k];
  return (s0 + s1) + (s2 + s3);
}

// Reusable barrier for a fixed set of threads.
class Barrier {
 public:
  explicit Barrier(unsigned n) : n_(n) {}
  void wait() {
    std::unique_lock<std::mutex> lk(m_);
    const unsigned gen = gen_;
    if (++count_ == n_) {
      count_ = 0;
      ++gen_;
      cv_.notify_all();
    } else {
      cv_.wait(lk, [&] { return gen != gen_; });
    }
  }

 private:
  std::mutex m_;
  std::condition_variable cv_;
  unsigned n_, count_ = 0, gen_ = 0;
};

// In-place lower Cholesky factor of the SPD matrix A (K x K, row-major, only
// the lower triangle read); the strict upper triangle is zeroed.  Column by
// column; the rows below the pivot are shared out over threads.  False if a
// pivot is not positive.
bool cholesky_lower(std::vector<double>& A, int K) {
  const unsigned nt = std::min<unsigned>(host_threads(), std::max(1, K / 64));
  Barrier bar(nt);
  std::atomic<bool> ok{true};
  auto worker = [&](unsigned t) {
    for (int j = 0; j < K; ++j) {
      double* rj = &A[static_cast<size_t>(j) * K];
      // every thread computes the pivot itself (same arithmetic, same value)
      const double d = rj[j] - dot4(rj, rj, j);
      if (!(d > 0.0)) {
        ok = false;
        return;                                        // all threads see the same d
      }
      const double ljj = std::sqrt(d);
      for (int i = j + 1 + static_cast<int>(t); i < K; i += static_cast<int>(nt)) {
        double* ri = &A[static_cast<size_t>(i) * K];
        ri[j] = (ri[j] - dot4(ri, rj, j)) / ljj;
      }
      bar.wait();                                      // column j complete
      if (t == 0) rj[j] = ljj;
      bar.wait();
    }
  };
  std::vector<std::thread> pool;
  for (unsigned t = 0; t < nt; ++t) pool.emplace_back(worker, t);
  for (auto& th : pool) th.join();
  if (!ok) return false;
  for (int i = 0; i < K; ++i)
    std::fill(A.begin() + static_cast<size_t>(i) * K + i + 1, A.begin() + static_cast<size_t>(i + 1) * K, 0.0);
  return true;
}

}  // namespace

void gptq_hessian(const float* xr, int T, int K, std::vector<double>& H) {
  // columns of X' made contiguous (fp64), then one dot product per H entry
  std::vector<double> Xt(static_cast<size_t>(K) * T);
  for (int r = 0; r < T; ++r)
    for (int k = 0; k < K; ++k)
      Xt[static_cast<size_t>(k) * T + r] = static_cast<double>(xr[static_cast<size_t>(r) * K + k]);
  H.assign(static_cast<size_t>(K) * K, 0.0);
  std::atomic<int> next{0};
  auto worker = [&]() {
    for (int i; (i = next.fetch_add(1)) < K;)
      for (int j = 0; j <= i; ++j) {
        const double v = dot4(&Xt[static_cast<size_t>(i) * T], &Xt[static_cast<size_t>(j) * T], T);
        H[static_cast<size_t>(i) * K + j] = v;
        H[static_cast<size_t>(j) * K + i] = v;
      }
  };
  std::vector<std::thread> pool;
  for (unsigned t = 0; t < host_threads(); ++t) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
}

bool gptq_inverse_factor(const double* H, int K, double damp, std::vector<double>& U,
                         std::vector<char>& dead) {
  dead.assign(K, 0);
  std::vector<double> diag(K);
  double mean = 0.0;
  for (int i = 0; i < K; ++i) {
    diag[i] = H[static_cast<size_t>(i) * K + i];
    if (diag[i] == 0.0) {
      dead[i] = 1;
      diag[i] = 1.0;
    }
    mean += diag[i];
  }
  mean /= K;
  // B = J A J with A the damped Hessian: B[a][b] = A[K-1-a][K-1-b]
  std::vector<double> B(static_cast<size_t>(K) * K);
  for (int a = 0; a < K; ++a)
    for (int b = 0; b < K; ++b)
      B[static_cast<size_t>(a) * K + b] =
          a == b ? diag[K - 1 - a] + damp * mean
                 : H[static_cast<size_t>(K - 1 - a) * K + (K - 1 - b)];
  if (!cholesky_lower(B, K)) return false;             // B = L L^T
  // X = L^-1 by columns (independent), kept transposed: Xt[j][i] = X[i][j]
  std::vector<double> Xt(static_cast<size_t>(K) * K, 0.0);
  std::atomic<int> next{0};
  auto worker = [&]() {
    for (int j; (j = next.fetch_add(1)) < K;) {
      double* xj = &Xt[static_cast<size_t>(j) * K];
      xj[j] = 1.0 / B[static_cast<size_t>(j) * K + j];
      for (int i = j + 1; i < K; ++i) {
        const double* li = &B[static_cast<size_t>(i) * K];
        xj[i] = -dot4(li + j, xj + j, i - j) / li[i];
      }
    }
  };
  std::vector<std::thread> pool;
  for (unsigned t = 0; t < host_threads(); ++t) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
  // U = J X J: U[a][b] = X[K-1-a][K-1-b] = Xt[K-1-b][K-1-a]
  U.assign(static_cast<size_t>(K) * K, 0.0);
  for (int a = 0; a < K; ++a)
    for (int b = a; b < K; ++b)
      U[static_cast<size_t>(a) * K + b] = Xt[static_cast<size_t>(K - 1 - b) * K + (K - 1 - a)];
  return true;
}

void gptq_quantize_rows(const float* Wr, int N, int K, const double* U, const char* dead, int qmax,
                        int8_t* q, float* s) {
  // Rows in groups of kR: each row of U is read once per group and applied to
  // all kR rows while it is in cache.
  constexpr int kR = 16;
  const int groups = (N + kR - 1) / kR;
  std::atomic<int> next{0};
  auto worker = [&]() {
    std::vector<double> w(static_cast<size_t>(kR) * K);
    double s64[kR], safe[kR], e[kR];
    for (int g; (g = next.fetch_add(1)) < groups;) {
      const int n0 = g * kR, R = std::min(kR, N - n0);
      for (int r = 0; r < R; ++r) {
        const float* src = Wr + static_cast<size_t>(n0 + r) * K;
        float amax = 0.f;
        for (int k = 0; k < K; ++k) amax = std::max(amax, std::fabs(src[k]));
        const float sf = amax / static_cast<float>(qmax);
        s[n0 + r] = sf;
        s64[r] = sf;
        safe[r] = s64[r] == 0.0 ? 1.0 : s64[r];
        double* wr = &w[static_cast<size_t>(r) * K];
        for (int k = 0; k < K; ++k) wr[k] = (dead && dead[k]) ? 0.0 : static_cast<double>(src[k]);
      }
      for (int j = 0; j < K; ++j) {
        const double* uj = U + static_cast<size_t>(j) * K;
        for (int r = 0; r < R; ++r) {
          double* wr = &w[static_cast<size_t>(r) * K];
          double qd = 0.0;
          if (s64[r] != 0.0) {
            qd = std::nearbyint(wr[j] / safe[r]);
            qd = std::min(std::max(qd, -static_cast<double>(qmax)), static_cast<double>(qmax));
          }
          q[static_cast<size_t>(n0 + r) * K + j] = static_cast<int8_t>(qd);
          const double prod = qd * s64[r];
          e[r] = (wr[j] - prod) / uj[j];
        }
        for (int r = 0; r < R; ++r) {
          double* wr = &w[static_cast<size_t>(r) * K];
          const double er = e[r];
          for (int k = j + 1; k < K; ++k) {
            const double t = er * uj[k];
            wr[k] = wr[k] - t;
          }
        }
      }
    }
  };
  const unsigned nt = std::min<unsigned>(host_threads(), static_cast<unsigned>(groups));
  std::vector<std::thread> pool;
  for (unsigned t = 0; t < nt; ++t) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
}

}  // namespace qvla
