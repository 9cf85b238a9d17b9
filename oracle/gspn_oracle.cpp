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
//
// Backward (section "反向传播" of the same walkthrough: the gradient flows
// into each line's hidden state from the later lines of the scan, and the
// input and gate gradients follow from it and the previous hidden state).
// For L = sum(gy (.) y) the adjoint a_i = dL/dh_i of one direction obeys
//     a_i = u_i (.) gy_i + w_{i+1}^T a_{i+1}      (no second term when line
//                                                   i+1 starts a group)
// and  dx = sum_d lambda_d (.) a_d,  dlambda_d = x (.) a_d,  du_d = gy (.) h_d,
//      dW_i[k,o] = a_i[k] h_{i-1}[k+o]  (lines that do not start a group),
// and, through w_o = s_o / sum_p s_p with s = sigmoid(z) over the existing
// neighbours,  dz_p = w_p (1 - s_p) (dW_p - sum_o dW_o w_o)  (0 for a missing
// neighbour and on a group's first line).  This is the chain rule on the
// forward definition above; the pages' own backward stops at the gates.

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

// Gradients of L = sum(gy (.) y) with respect to the inputs of one plane and
// one direction: dx is accumulated, dz3, dlam and du are written.  h is
// scratch of H*W doubles.
void plane_backward(const Dir& dir, const double* x, const double* z3, const double* lam,
                    const double* u, const double* gy, int64_t g, double* dx, double* dz3,
                    double* dlam, double* du, double* h) {
    const int64_t L = dir.L(), K = dir.K(), HW = dir.H * dir.W;
    plane_hidden(dir, x, z3, lam, g, h);
    std::vector<double> a(K), carry(K, 0.0);
    for (int64_t i = L - 1; i >= 0; --i) {
        const bool start = group_start(dir, i, g);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t p = dir.pixel(i, k);
            a[k] = u[p] * gy[p] + carry[k];
            du[p] = gy[p] * h[p];
            dlam[p] = x[p] * a[k];
            dx[p] += lam[p] * a[k];
        }
        for (int64_t k = 0; k < K; ++k) carry[k] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const int64_t p = dir.pixel(i, k);
            if (start) {
                for (int slot = 0; slot < 3; ++slot) dz3[slot * HW + p] = 0.0;
                continue;
            }
            double w[3];
            pixel_weights(z3, HW, p, k, K, w);
            double dw[3] = {0.0, 0.0, 0.0};
            double dw_dot_w = 0.0;
            for (int slot = 0; slot < 3; ++slot) {
                const int64_t kn = k + slot - 1;
                if (kn < 0 || kn >= K) continue;
                dw[slot] = a[k] * h[dir.pixel(i - 1, kn)];
                dw_dot_w += dw[slot] * w[slot];
                carry[kn] += w[slot] * a[k];
            }
            for (int slot = 0; slot < 3; ++slot) {
                const int64_t kn = k + slot - 1;
                if (kn < 0 || kn >= K) {
                    dz3[slot * HW + p] = 0.0;
                    continue;
                }
                const double sg = logistic(z3[slot * HW + p]);
                dz3[slot * HW + p] = w[slot] * (1.0 - sg) * (dw[slot] - dw_dot_w);
            }
        }
    }
}

// ---- wider neighbourhoods ---------------------------------------------------
// Section "如何设计一个高效的传播层" first states a direct method -- every pixel
// links to all n pixels of the previous line, with weights normalised to sum
// to 1 -- and sets it aside for its feature cost in favour of the three
// neighbours above.  The banded form links pixel k to the previous line's
// pixels k + o for |o| <= r: r = 1 is the tridiagonal layer, r >= K - 1 links
// every pixel to the whole previous line (the direct method, a dense
// row-stochastic w_i).  Logit slot s = 0 .. 2r is orthogonal offset s - r;
// neighbours outside the line are dropped from the normaliser, as in section
// "行随机矩阵".  Layout of the logits: [B][C][2r + 1][H][W].
void plane_hidden_band(const Dir& dir, const double* x, const double* zb, const double* lam,
                       int64_t g, int64_t r, double* h) {
    const int64_t L = dir.L(), K = dir.K(), HW = dir.H * dir.W;
    const int64_t nslot = 2 * r + 1;
    std::vector<double> before(K), now(K), sig(nslot);
    for (int64_t i = 0; i < L; ++i) {
        const bool restart = group_start(dir, i, g);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t p = dir.pixel(i, k);
            double v = lam[p] * x[p];
            if (!restart) {
                double norm = 0.0;
                for (int64_t s = 0; s < nslot; ++s) {
                    const int64_t src = k + (s - r);
                    sig[s] = (src >= 0 && src < K) ? logistic(zb[s * HW + p]) : 0.0;
                    norm += sig[s];
                }
                double mix = 0.0;
                for (int64_t s = 0; s < nslot; ++s) {
                    const int64_t src = k + (s - r);
                    if (src >= 0 && src < K) mix += (sig[s] / norm) * before[src];
                }
                v += mix;
            }
            now[k] = v;
            h[p] = v;
        }
        before.swap(now);
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

// Hidden state of one direction with a (2 * radius + 1)-neighbour band:
// wlogit[B][C][2 * radius + 1][H][W], h[B][C][H][W].  radius = 1 is
// gspn_oracle_hidden.  Returns 0, or -1 on a bad argument.
int gspn_oracle_hidden_band(const double* x, const double* wlogit, const double* lam, int64_t B,
                            int64_t C, int64_t H, int64_t W, int64_t radius, int64_t group_len,
                            int d, int nthreads, double* h) {
    if (!x || !wlogit || !lam || !h || bad_shape(B, C, H, W) || d < 0 || d > 3 ||
        group_len < 0 || radius < 0)
        return -1;
    const int64_t HW = H * W;
    const int64_t nslot = 2 * radius + 1;
    const Dir dir{d, H, W};
    parallel_planes(B * C, nthreads, [&](int64_t q) {
        plane_hidden_band(dir, x + q * HW, wlogit + q * nslot * HW, lam + q * HW, group_len,
                          radius, h + q * HW);
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

// Gradients of L = sum(gy (.) y) for the four-direction operation:
// dx[B][C][H][W]; dwlogit[d][B][C][3][H][W]; dlam[d], du[d][B][C][H][W].
// Returns 0, or -1 on a bad argument.
int gspn_oracle_backward(const double* x, const double* const* wlogit, const double* const* lam,
                         const double* const* u, const double* gy, int64_t B, int64_t C,
                         int64_t H, int64_t W, int64_t group_len, int nthreads, double* dx,
                         double* const* dwlogit, double* const* dlam, double* const* du) {
    if (!x || !wlogit || !lam || !u || !gy || !dx || !dwlogit || !dlam || !du ||
        bad_shape(B, C, H, W) || group_len < 0)
        return -1;
    for (int d = 0; d < 4; ++d)
        if (!wlogit[d] || !lam[d] || !u[d] || !dwlogit[d] || !dlam[d] || !du[d]) return -1;
    const int64_t HW = H * W;
    parallel_planes(B * C, nthreads, [&](int64_t q) {
        std::vector<double> h(HW);
        double* dxq = dx + q * HW;
        for (int64_t p = 0; p < HW; ++p) dxq[p] = 0.0;
        for (int d = 0; d < 4; ++d) {
            const Dir dir{d, H, W};
            plane_backward(dir, x + q * HW, wlogit[d] + q * 3 * HW, lam[d] + q * HW,
                           u[d] + q * HW, gy + q * HW, group_len, dxq, dwlogit[d] + q * 3 * HW,
                           dlam[d] + q * HW, du[d] + q * HW, h.data());
        }
    });
    return 0;
}

}  // extern "C"
