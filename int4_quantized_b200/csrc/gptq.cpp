// gptq.cpp -- the GPTQ host quantizer (host code, fp64): codes chosen to keep a layer's
// output, in the same payload format as qpack ("Huit bits, puis quatre", section "Arrondir
// mieux : GPTQ").
//
// With H = sum over calibration samples of x^T x ([K, K]) and U the upper triangular
// factor of (H + damping)^-1 = U^T U, the input components k (the columns of W [N, K])
// are quantized in order; the error of column k, divided by U[k][k], is taken off every
// later column j in proportion to U[k][j]. A group's scale is fixed when its first column
// is reached, from the weights corrected so far, by the rounding rule of qpack (scale =
// max|w| / qmax in fp32, 0 -> 1; code = clip(rint(w / scale)) with an IEEE fp32 divide).
// Each output row only ever reads its own weights, so rows run on separate threads; the
// operations on every weight are those of the definition, in its order.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <condition_variable>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <thread>
#include <vector>

#include "../../include/q4.h"

namespace {

inline bool finite_all(const float *p, int64_t n) {
    for (int64_t i = 0; i < n; ++i)
        if (!std::isfinite(p[i])) return false;
    return true;
}

inline int qmax_of(int bits) { return bits == 4 ? 7 : 127; }

// Run f(lo, hi) over [0, n) split into contiguous parts, one per thread.
template <typename F>
void parallel_rows(int64_t n, int threads, F f) {
    int t = threads > 0 ? threads : (int)std::thread::hardware_concurrency();
    if (t < 1) t = 1;
    if (t > n) t = (int)std::max<int64_t>(n, 1);
    if (t == 1) {
        f((int64_t)0, n);
        return;
    }
    std::vector<std::thread> pool;
    for (int i = 0; i < t; ++i) {
        const int64_t lo = n * i / t, hi = n * (i + 1) / t;
        pool.emplace_back([=] { f(lo, hi); });
    }
    for (auto &th : pool) th.join();
}

int thread_count(int threads, int64_t work_items) {
    int t = threads > 0 ? threads : (int)std::thread::hardware_concurrency();
    if (t < 1) t = 1;
    if (t > work_items) t = (int)std::max<int64_t>(work_items, 1);
    return t;
}

// A reusable barrier for a fixed set of threads (C++17 has none).
class Barrier {
  public:
    explicit Barrier(int n) : n_(n) {}
    void wait() {
        std::unique_lock<std::mutex> lk(mu_);
        const uint64_t gen = gen_;
        if (++count_ == n_) {
            count_ = 0;
            ++gen_;
            cv_.notify_all();
        } else {
            cv_.wait(lk, [&] { return gen_ != gen; });
        }
    }

  private:
    std::mutex mu_;
    std::condition_variable cv_;
    int n_, count_ = 0;
    uint64_t gen_ = 0;
};

// In place lower Cholesky factor of the symmetric [K, K] matrix A (A = L L^T), column by
// column; the strict upper triangle is set to zero. False when A is not positive definite.
// Rows below the diagonal are shared cyclically among the threads, one barrier per column;
// every thread forms the column's diagonal itself (the same operations on the same
// values), so the factor is the same for any thread count.
bool cholesky_lower(std::vector<double> &A, int64_t K, int threads) {
    const int T = thread_count(threads, K / 64);
    std::vector<double> diag((size_t)K);
    bool ok = true;
    Barrier bar(T);
    auto work = [&](int tid) {
        for (int64_t j = 0; j < K; ++j) {
            const double *aj = &A[j * K];
            double d = aj[j];
            for (int64_t p = 0; p < j; ++p) d -= aj[p] * aj[p];
            const bool pd = d > 0.0 && std::isfinite(d);
            if (!pd) {
                if (tid == 0) ok = false;
                return;  // every thread sees the same d and leaves at the same column
            }
            const double ljj = std::sqrt(d);
            if (j % T == tid) diag[j] = ljj;
            int64_t i0 = j + 1 + ((tid - (j + 1)) % T + T) % T;  // first row > j owned by tid
            for (int64_t i = i0; i < K; i += T) {
                double *ai = &A[i * K];
                double s = ai[j];
                for (int64_t p = 0; p < j; ++p) s -= ai[p] * aj[p];
                ai[j] = s / ljj;
            }
            if (T > 1) bar.wait();
        }
    };
    if (T == 1) {
        work(0);
    } else {
        std::vector<std::thread> pool;
        for (int t = 0; t < T; ++t) pool.emplace_back(work, t);
        for (auto &th : pool) th.join();
    }
    if (!ok) return false;
    for (int64_t j = 0; j < K; ++j) {
        A[j * K + j] = diag[j];
        for (int64_t i = j + 1; i < K; ++i) A[j * K + i] = 0.0;
    }
    return true;
}

}  // namespace

extern "C" {

q4_status q4_gptq_hessian(const float *x, int64_t rows, int64_t K, double *H, int threads) {
    if (rows < 0 || K < 1 || !H || (rows > 0 && !x)) return Q4_ERR_ARG;
    if (!finite_all(x, rows * K)) return Q4_ERR_NONFINITE;
    // thread i owns rows [lo, hi) of H; samples are added in order
    parallel_rows(K, threads, [&](int64_t lo, int64_t hi) {
        for (int64_t r = 0; r < rows; ++r) {
            const float *xr = x + r * K;
            for (int64_t i = lo; i < hi; ++i) {
                const double xi = (double)xr[i];
                double *hi_row = H + i * K;
                for (int64_t j = 0; j < K; ++j) hi_row[j] += xi * (double)xr[j];
            }
        }
    });
    return Q4_OK;
}

q4_status q4_gptq_prepare(const double *H, int64_t K, double damp, double *U, int threads) {
    if (!H || !U || K < 1 || !(damp >= 0.0)) return Q4_ERR_ARG;
    double mean = 0.0;
    for (int64_t i = 0; i < K; ++i) mean += H[i * K + i];
    mean /= (double)K;
    if (!(mean > 0.0) || !std::isfinite(mean)) return Q4_ERR_ARG;
    // (H + d I)^-1 = U^T U with U upper  <=>  H + d I = V V^T with V = U^-1 upper. With J the
    // order reversal, J (H + d I) J = (J V J)(J V J)^T is a lower Cholesky factorisation, so
    // U = J L^-1 J for L = chol(J (H + d I) J).
    std::vector<double> A((size_t)(K * K));
    for (int64_t i = 0; i < K; ++i)
        for (int64_t j = 0; j < K; ++j) {
            const double h = 0.5 * (H[i * K + j] + H[j * K + i]);
            A[(K - 1 - i) * K + (K - 1 - j)] = h + (i == j ? damp * mean : 0.0);
        }
    if (!cholesky_lower(A, K, threads)) return Q4_ERR_ARG;
    // column c of L^-1 by forward substitution (x_c = 1 / L[c][c]; x_i for i > c), written
    // straight into U[K-1-i][K-1-c]; the columns are independent, shared cyclically
    std::fill(U, U + K * K, 0.0);
    const int T = thread_count(threads, K / 64);
    auto columns = [&](int tid) {
        std::vector<double> x((size_t)K);
        for (int64_t c = tid; c < K; c += T) {
            x[c] = 1.0 / A[c * K + c];
            for (int64_t i = c + 1; i < K; ++i) {
                const double *li = &A[i * K];
                double s = 0.0;
                for (int64_t p = c; p < i; ++p) s += li[p] * x[p];
                x[i] = -s / li[i];
            }
            for (int64_t i = c; i < K; ++i) U[(K - 1 - i) * K + (K - 1 - c)] = x[i];
        }
    };
    if (T == 1) {
        columns(0);
    } else {
        std::vector<std::thread> pool;
        for (int t = 0; t < T; ++t) pool.emplace_back(columns, t);
        for (auto &th : pool) th.join();
    }
    return Q4_OK;
}

q4_status q4_gptq_quantize(const float *w, int64_t N, int64_t K, const double *U, int bits, int64_t group,
                           uint8_t *payload, float *scales, int threads) {
    if (bits != 4 && bits != 8) return Q4_ERR_ARG;
    if (N < 0 || K < 1 || group < 1 || K % group != 0) return Q4_ERR_ARG;
    if (bits == 4 && (N * K) % 2 != 0) return Q4_ERR_ARG;
    if (N == 0) return Q4_OK;
    if (!w || !U || !payload || !scales) return Q4_ERR_ARG;
    for (int64_t k = 0; k < K; ++k)
        if (!(U[k * K + k] != 0.0) || !std::isfinite(U[k * K + k])) return Q4_ERR_ARG;
    if (!finite_all(w, N * K)) return Q4_ERR_NONFINITE;
    const int qmax = qmax_of(bits);
    const int64_t spr = K / group;
    std::vector<int8_t> codes((size_t)(N * K));
    // scales are kept here until the whole walk is known to be finite: an ill-conditioned U
    // can push a corrected weight past the fp32 range, and then nothing is written
    std::vector<float> sc((size_t)(N * spr));
    std::atomic<bool> nonfinite{false};
    // rows go through the columns in batches of kRowBatch, so that row k of U is read from
    // cache by the whole batch; every weight still sees its own updates in k order
    constexpr int kRowBatch = 8;
    parallel_rows(N, threads, [&](int64_t lo, int64_t hi) {
        std::vector<double> Wb((size_t)(kRowBatch * K));
        double err[kRowBatch];
        float s[kRowBatch];
        for (int64_t n0 = lo; n0 < hi; n0 += kRowBatch) {
            const int nb = (int)std::min<int64_t>(kRowBatch, hi - n0);
            for (int r = 0; r < nb; ++r)
                for (int64_t k = 0; k < K; ++k) Wb[r * K + k] = (double)w[(n0 + r) * K + k];
            for (int64_t k = 0; k < K; ++k) {
                const double *uk = U + k * K;
                for (int r = 0; r < nb; ++r) {
                    double *W = &Wb[r * K];
                    const int64_t n = n0 + r;
                    if (k % group == 0) {
                        float a = 0.0f;
                        bool ok = true;
                        for (int64_t j = k; j < k + group; ++j) {
                            const float v = (float)W[j];
                            ok = ok && std::isfinite(v);
                            a = std::max(a, std::fabs(v));
                        }
                        if (!ok) nonfinite.store(true, std::memory_order_relaxed);
                        s[r] = a / (float)qmax;
                        if (s[r] == 0.0f) s[r] = 1.0f;
                        sc[n * spr + k / group] = s[r];
                    }
                    const float t = (float)W[k] / s[r];
                    float c = std::nearbyint(t);
                    c = std::min(std::max(c, (float)-qmax), (float)qmax);
                    codes[n * K + k] = (int8_t)c;
                    const double wq = (double)(c * s[r]);
                    err[r] = (W[k] - wq) / uk[k];
                }
                for (int r = 0; r < nb; ++r) {
                    double *W = &Wb[r * K];
                    const double e = err[r];
                    for (int64_t j = k + 1; j < K; ++j) W[j] -= e * uk[j];
                }
            }
        }
    });
    if (nonfinite.load()) return Q4_ERR_NONFINITE;
    std::memcpy(scales, sc.data(), sc.size() * sizeof(float));
    const int64_t n = N * K;
    if (bits == 8) {
        std::memcpy(payload, codes.data(), (size_t)n);
    } else {
        for (int64_t t = 0; t < n / 2; ++t)
            payload[t] = (uint8_t)((codes[2 * t] + 8) | ((codes[2 * t + 1] + 8) << 4));
    }
    return Q4_OK;
}

}  // extern "C"
