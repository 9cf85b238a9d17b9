// GSPN fp64 CPU oracle -- TEST INFRASTRUCTURE ONLY.
//
// Only the test suite, the smoke check and the benchmark's CPU-baseline leg
// may load this library.  The product path (the CUDA library) never calls it
// and shares no code, header or constant with it.
//
// What it computes (Generalized Spatial Propagation Network, "Parallel
// Sequence Modeling via Generalized Spatial Propagation Network", arXiv
// 2501.12381, as summarised by the CSDN walkthrough of the paper):
//
//   * Section "方法" (method), linear recurrence:
//         h_i = w_i h_{i-1} + lambda_i (.) x_i ,   y_i = u_i (.) h_i
//     with the first line h_0 = lambda_0 (.) x_0 (the diagonal block
//     G_ii = lambda_i of the unrolled matrix G in the same section).
//   * Section "如何设计一个高效的传播层" (efficient propagation layer): w_i is
//     tridiagonal -- every pixel links to the three pixels of the previous
//     line at orthogonal offsets -1, 0, +1 -- and the scan runs in four
//     directions.
//   * Section "行随机矩阵" (row-stochastic matrix): each non-zero is
//     sigmoid(logit) divided by the sum of sigmoids over the m_i non-zeros of
//     its row, so a border pixel normalises over its two existing neighbours.
//   * Section "全局与局部GSPN" (global and local GSPN): the local variant
//     splits the scan axis into non-overlapping groups and propagates inside
//     each group only.
//   * The four directions are merged as y = sum_d u_d (.) h_d.
//
// Conventions (the pages leave them open; these are the library's):
//   direction d: 0 top->bottom, 1 bottom->top, 2 left->right, 3 right->left.
//   All logits, lambda and u are stored at the pixel being computed, in
//   original image coordinates; logit slot s = 0,1,2 is the neighbour at
//   orthogonal offset s-1 (row offset for d=2,3, column offset for d=0,1).
//   Local groups are blocks [s*g, (s+1)*g) of the ORIGINAL scan-axis
//   coordinate; the scan restarts (h = lambda*x) on the first line of each
//   block in scan order.
//
// Layouts (contiguous, row-major): x, lam[d], u[d], y: [B][C][H][W];
// wlogit[d]: [B][C][3][H][W].  All arrays are double.

#include <cmath>
#include <cstdint>
#include <thread>
#include <vector>

namespace {

struct Dir {
    int d;
    int64_t H, W;
    int64_t L() const { return d < 2 ? H : W; }   // scan length
    int64_t K() const { return d < 2 ? W : H; }   // orthogonal length
    // flat pixel index r*W + c of scan line i, orthogonal position k
    int64_t pixel(int64_t i, int64_t k) const {
        switch (d) {
            case 0: return i * W + k;
            case 1: return (H - 1 - i) * W + k;
            case 2: return k * W + i;
            default: return k * W + (W - 1 - i);
        }
    }
    // coordinate of scan line i along the scan axis, in original coordinates
    int64_t axis_coord(int64_t i) const {
        return (d == 0 || d == 2) ? i : L() - 1 - i;
    }
};

double logistic(double z) { return 1.0 / (1.0 + std::exp(-z)); }

// Is scan line i the first line of a propagation group?
bool group_start(const Dir& dir, int64_t i, int64_t g) {
    if (i == 0) return true;
    if (g <= 0) return false;
    return dir.axis_coord(i) / g != dir.axis_coord(i - 1) / g;
}

// Normalised tridiagonal weights of one pixel: w[s] for neighbour offset s-1.
void pixel_weights(const double* z_plane3, int64_t HW, int64_t p, int64_t k, int64_t K,
                   double w[3]) {
    double s[3] = {0.0, 0.0, 0.0};
    double total = 0.0;
    for (int slot = 0; slot < 3; ++slot) {
        int64_t kn = k + slot - 1;
        if (kn < 0 || kn >= K) continue;          // missing neighbour: dropped
        s[slot] = logistic(z_plane3[slot * HW + p]);
        total += s[slot];
    }
    for (int slot = 0; slot < 3; ++slot) w[slot] = s[slot] / total;
}

// h for one plane and one direction (h has H*W entries, original layout).
void plane_hidden(const Dir& dir, const double* x, const double* z3, const double* lam,
                  int64_t g, double* h) {
    const int64_t L = dir.L(), K = dir.K(), HW = dir.H * dir.W;
    std::vector<double> prev(K), cur(K);
    for (int64_t i = 0; i < L; ++i) {
        const bool start = group_start(dir, i, g);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t p = dir.pixel(i, k);
            const double drive = lam[p] * x[p];
            if (start) {
                cur[k] = drive;
            } else {
                double w[3];
                pixel_weights(z3, HW, p, k, K, w);
                double acc = 0.0;
                for (int slot = 0; slot < 3; ++slot) {
                    int64_t kn = k + slot - 1;
                    if (kn < 0 || kn >= K) continue;
                    acc += w[slot] * prev[kn];
                }
                cur[k] = acc + drive;
            }
            h[p] = cur[k];
        }
        prev.swap(cur);
    }
}

template <class F>
void parallel_planes(int64_t planes, int nthreads, F&& body) {
    if (nthreads <= 0) nthreads = (int)std::thread::hardware_concurrency();
    if (nthreads <= 0) nthreads = 1;
    if (nthreads > planes) nthreads = (int)(planes > 0 ? planes : 1);
    std::vector<std::thread> pool;
    for (int t = 0; t < nthreads; ++t)
        pool.emplace_back([&, t] {
            for (int64_t q = t; q < planes; q += nthreads) body(q);
        });
    for (auto& th : pool) th.join();
}

bool bad_shape(int64_t B, int64_t C, int64_t H, int64_t W) {
    return B <= 0 || C <= 0 || H <= 0 || W <= 0;
}

}  // namespace

extern "C" {

// Number of host threads the oracle uses when asked for 0 (all cores).
int gspn_oracle_default_threads() {
    int n = (int)std::thread::hardware_concurrency();
    return n > 0 ? n : 1;
}

// Hidden state h_d of one direction for every plane: h[B][C][H][W].
// Returns 0, or -1 on a bad argument.
int gspn_oracle_hidden(const double* x, const double* wlogit, const double* lam, int64_t B,
                       int64_t C, int64_t H, int64_t W, int64_t group_len, int d,
                       int nthreads, double* h) {
    if (!x || !wlogit || !lam || !h || bad_shape(B, C, H, W) || d < 0 || d > 3 ||
        group_len < 0)
        return -1;
    const int64_t HW = H * W;
    const Dir dir{d, H, W};
    parallel_planes(B * C, nthreads, [&](int64_t q) {
        plane_hidden(dir, x + q * HW, wlogit + q * 3 * HW, lam + q * HW, group_len, h + q * HW);
    });
    return 0;
}

// Normalised weights of one direction: w[B][C][3][H][W] (slot s = offset s-1).
// Entries for a missing neighbour are 0.  Returns 0, or -1 on a bad argument.
int gspn_oracle_weights(const double* wlogit, int64_t B, int64_t C, int64_t H, int64_t W,
                        int d, double* w_out) {
    if (!wlogit || !w_out || bad_shape(B, C, H, W) || d < 0 || d > 3) return -1;
    const int64_t HW = H * W;
    const Dir dir{d, H, W};
    for (int64_t q = 0; q < B * C; ++q) {
        const double* z3 = wlogit + q * 3 * HW;
        double* o3 = w_out + q * 3 * HW;
        for (int64_t i = 0; i < dir.L(); ++i)
            for (int64_t k = 0; k < dir.K(); ++k) {
                const int64_t p = dir.pixel(i, k);
                double w[3];
                pixel_weights(z3, HW, p, k, dir.K(), w);
                for (int s = 0; s < 3; ++s) o3[s * HW + p] = w[s];
            }
    }
    return 0;
}

// Full four-direction output y = sum_d u_d (.) h_d, y[B][C][H][W].
// wlogit, lam, u are arrays of four pointers, indexed by direction.
// Returns 0, or -1 on a bad argument.
int gspn_oracle_forward(const double* x, const double* const* wlogit, const double* const* lam,
                        const double* const* u, int64_t B, int64_t C, int64_t H, int64_t W,
                        int64_t group_len, int nthreads, double* y) {
    if (!x || !wlogit || !lam || !u || !y || bad_shape(B, C, H, W) || group_len < 0) return -1;
    for (int d = 0; d < 4; ++d)
        if (!wlogit[d] || !lam[d] || !u[d]) return -1;
    const int64_t HW = H * W;
    parallel_planes(B * C, nthreads, [&](int64_t q) {
        std::vector<double> h(HW);
        double* yq = y + q * HW;
        for (int64_t p = 0; p < HW; ++p) yq[p] = 0.0;
        for (int d = 0; d < 4; ++d) {
            const Dir dir{d, H, W};
            plane_hidden(dir, x + q * HW, wlogit[d] + q * 3 * HW, lam[d] + q * HW, group_len,
                         h.data());
            const double* ud = u[d] + q * HW;
            for (int64_t p = 0; p < HW; ++p) yq[p] += ud[p] * h[p];
        }
    });
    return 0;
}

}  // extern "C"
