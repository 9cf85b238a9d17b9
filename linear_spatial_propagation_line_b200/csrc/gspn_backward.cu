// Backward pass of the GSPN propagation (any plane size).
//
// For L = sum(gy (.) y) the adjoint of one direction's hidden state runs the
// scan in reverse (CSDN walkthrough "GSPN——在convolution基础上并行序列建模",
// section "反向传播": the gradient reaches each line from the later lines):
//     a_i = u_i (.) gy_i + w_{i+1}^T a_{i+1}   (no second term when line i+1
//                                              starts a group)
//     dx += lambda_i (.) a_i,  dlambda_i = x_i (.) a_i,  du_i = gy_i (.) h_i
//     dz_i[k,o] = w_o (1 - s_o) (a_i[k] h_{i-1}[k+o] - sum_p w_p a_i[k] h_{i-1}[k+p])
// with s = sigmoid(z) and w the border-aware normalised weights; the logits
// of a group's first line and of missing neighbours get zero gradient.
//
// Two kernels per call: hidden_kernel stores every direction's h (fp32) in
// the workspace; backward_kernel runs the reverse scan, one CTA per (plane,
// direction), with the adjoint line in shared memory.  The adjoint carried to
// the previous line is a gather of the neighbours' weighted adjoints:
//     carry[k] = w[k+1,0] a[k+1] + w[k,1] a[k] + w[k-1,2] a[k-1].
// dx sums four directions and is accumulated in fp32, then rounded once.
#include <utility>

#include "gspn_internal.h"

namespace gspn {
namespace {

// Calls f(std::integral_constant<int, I>{}) for I = 0..N-1, so that array
// indices inside f are compile-time constants.
template <class F, int... Is>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, Is...>) {
    (f(std::integral_constant<int, Is>{}), ...);
}
template <int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

constexpr int kThreads = 512;
constexpr int kPer = 4;  // positions per thread whose loads are issued together

template <class T>
__device__ __forceinline__ float ld(const T* p) {
    return to_f32(*p);
}

// h_d of every line of one (plane, direction): hbuf[d][plane][H*W].  Each
// thread takes up to kPer positions of a line at once and issues all their
// loads before any store, so a step costs one round of memory latency.
template <class T, bool kRefine>
__global__ void __launch_bounds__(kThreads)
    hidden_kernel(const T* __restrict__ x, Ptr4 zp, Ptr4 lp, int H, int W, int g, int64_t planes,
                  float* __restrict__ hbuf) {
    extern __shared__ __align__(16) float hb[];
    const int d = (int)blockIdx.y;
    const int64_t plane = blockIdx.x;
    const int HW = H * W;
    const int L = d < 2 ? H : W, K = d < 2 ? W : H;
    const T* __restrict__ xq = x + plane * HW;
    const T* __restrict__ zq = static_cast<const T*>(zp.p[d]) + plane * 3 * HW;
    const T* __restrict__ lq = static_cast<const T*>(lp.p[d]) + plane * HW;
    float* __restrict__ hq = hbuf + ((int64_t)d * planes + plane) * HW;
    float* hcur = hb;
    float* hnxt = hb + K + 2;
    for (int k = threadIdx.x; k < K + 2; k += kThreads) hcur[k] = hnxt[k] = 0.0f;
    __syncthreads();
    for (int i = 0; i < L; ++i) {
        const bool start = group_start(d, L, g, i);
        for (int kb = threadIdx.x; kb < K; kb += kPer * kThreads) {
            float lx[kPer], z0[kPer], z1[kPer], z2[kPer];
            int pix[kPer];
            static_for<kPer>([&](auto jc) {
                constexpr int j = decltype(jc)::value;
                const int k = kb + j * kThreads;
                const int p = pixel_of(d, H, W, i, k < K ? k : K - 1);
                pix[j] = p;
                lx[j] = ld(lq + p) * ld(xq + p);
                z0[j] = ld(zq + p);
                z1[j] = ld(zq + HW + p);
                z2[j] = ld(zq + 2 * HW + p);
            });
            static_for<kPer>([&](auto jc) {
                constexpr int j = decltype(jc)::value;
                const int k = kb + j * kThreads;
                if (k < K) {
                    float hv = lx[j];
                    if (!start) {
                        float w0, w1, w2;
                        tri_weights<kRefine>(z0[j], z1[j], z2[j], k > 0, k < K - 1, w0, w1, w2);
                        hv = fmaf(w0, hcur[k], fmaf(w1, hcur[k + 1], fmaf(w2, hcur[k + 2], hv)));
                    }
                    hnxt[k + 1] = hv;
                    hq[pix[j]] = hv;
                }
            });
        }
        __syncthreads();
        float* t = hcur;
        hcur = hnxt;
        hnxt = t;
    }
}

struct MutPtr4 {
    void* p[4];
};

// Sigmoid s and 1 - s of one logit from e = exp(-z) (exact complement).
__device__ __forceinline__ void sigmoid_pair(float z, float& s, float& one_minus_s) {
    const float e = __expf(-fminf(fmaxf(z, -80.0f), 80.0f));
    const float r = 1.0f / (1.0f + e);
    s = r;
    one_minus_s = e * r;
}

// Reverse adjoint scan of one (plane, direction).  As in hidden_kernel, a
// thread issues the loads of up to kPer positions (inputs, gy, the stored
// states of the line and of its neighbours on the previous line) before it
// computes and stores their gradients.
template <class T, bool kRefine>
__global__ void __launch_bounds__(kThreads)
    backward_kernel(const T* __restrict__ x, Ptr4 zp, Ptr4 lp, Ptr4 up, const T* __restrict__ gy,
                    int H, int W, int g, int64_t planes, const float* __restrict__ hbuf,
                    float* __restrict__ dxacc, MutPtr4 dzp, MutPtr4 dlp, MutPtr4 dup) {
    extern __shared__ __align__(16) float sm[];
    const int d = (int)blockIdx.y;
    const int64_t plane = blockIdx.x;
    const int HW = H * W;
    const int L = d < 2 ? H : W, K = d < 2 ? W : H;
    const T* __restrict__ xq = x + plane * HW;
    const T* __restrict__ gq = gy + plane * HW;
    const T* __restrict__ zq = static_cast<const T*>(zp.p[d]) + plane * 3 * HW;
    const T* __restrict__ lq = static_cast<const T*>(lp.p[d]) + plane * HW;
    const T* __restrict__ uq = static_cast<const T*>(up.p[d]) + plane * HW;
    T* __restrict__ dzq = static_cast<T*>(dzp.p[d]) + plane * 3 * HW;
    T* __restrict__ dlq = static_cast<T*>(dlp.p[d]) + plane * HW;
    T* __restrict__ duq = static_cast<T*>(dup.p[d]) + plane * HW;
    const float* __restrict__ hq = hbuf + ((int64_t)d * planes + plane) * HW;
    float* __restrict__ dxq = dxacc + plane * HW;
    float* carry = sm;          // [K]
    float* c0 = sm + K;         // [K] w[k,0] a[k]
    float* c1 = sm + 2 * K;     // [K] w[k,1] a[k]
    float* c2 = sm + 3 * K;     // [K] w[k,2] a[k]
    for (int k = threadIdx.x; k < K; k += kThreads) carry[k] = 0.0f;
    __syncthreads();
    for (int i = L - 1; i >= 0; --i) {
        const bool start = group_start(d, L, g, i);
        const int ip = i > 0 ? i - 1 : 0;  // previous line (unused on a group's first line)
        for (int kb = threadIdx.x; kb < K; kb += kPer * kThreads) {
            float gyv[kPer], uv[kPer], xv[kPer], lv[kPer], z0[kPer], z1[kPer], z2[kPer];
            float hv[kPer], hl[kPer], hs[kPer], hr[kPer];
            int pix[kPer];
            static_for<kPer>([&](auto jc) {
                constexpr int j = decltype(jc)::value;
                const int kk = kb + j * kThreads;
                const int k = kk < K ? kk : K - 1;
                const int p = pixel_of(d, H, W, i, k);
                pix[j] = p;
                gyv[j] = ld(gq + p);
                uv[j] = ld(uq + p);
                xv[j] = ld(xq + p);
                lv[j] = ld(lq + p);
                z0[j] = ld(zq + p);
                z1[j] = ld(zq + HW + p);
                z2[j] = ld(zq + 2 * HW + p);
                hv[j] = hq[p];
                hl[j] = hq[pixel_of(d, H, W, ip, k > 0 ? k - 1 : 0)];
                hs[j] = hq[pixel_of(d, H, W, ip, k)];
                hr[j] = hq[pixel_of(d, H, W, ip, k < K - 1 ? k + 1 : K - 1)];
            });
            static_for<kPer>([&](auto jc) {
                constexpr int j = decltype(jc)::value;
                const int k = kb + j * kThreads;
                if (k >= K) return;
                const int p = pix[j];
                const float a = fmaf(uv[j], gyv[j], carry[k]);
                duq[p] = from_f32<T>(gyv[j] * hv[j]);
                dlq[p] = from_f32<T>(xv[j] * a);
                atomicAdd(dxq + p, lv[j] * a);
                float dz0 = 0.0f, dz1 = 0.0f, dz2 = 0.0f, w0 = 0.0f, w1 = 0.0f, w2 = 0.0f;
                if (!start) {
                    const bool lo = k > 0, hi = k < K - 1;
                    tri_weights<kRefine>(z0[j], z1[j], z2[j], lo, hi, w0, w1, w2);
                    const float dw0 = lo ? a * hl[j] : 0.0f, dw1 = a * hs[j];
                    const float dw2 = hi ? a * hr[j] : 0.0f;
                    const float dot = fmaf(dw0, w0, fmaf(dw1, w1, dw2 * w2));
                    float s, oms;
                    if (lo) {
                        sigmoid_pair(z0[j], s, oms);
                        dz0 = w0 * oms * (dw0 - dot);
                    }
                    sigmoid_pair(z1[j], s, oms);
                    dz1 = w1 * oms * (dw1 - dot);
                    if (hi) {
                        sigmoid_pair(z2[j], s, oms);
                        dz2 = w2 * oms * (dw2 - dot);
                    }
                }
                dzq[p] = from_f32<T>(dz0);
                dzq[HW + p] = from_f32<T>(dz1);
                dzq[2 * HW + p] = from_f32<T>(dz2);
                c0[k] = w0 * a;
                c1[k] = w1 * a;
                c2[k] = w2 * a;
            });
        }
        __syncthreads();
        for (int k = threadIdx.x; k < K; k += kThreads)
            carry[k] = c1[k] + (k + 1 < K ? c0[k + 1] : 0.0f) + (k > 0 ? c2[k - 1] : 0.0f);
        __syncthreads();
    }
}

template <class T>
__global__ void round_kernel(const float* __restrict__ acc, int64_t n, T* __restrict__ out) {
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < n;
         p += (int64_t)gridDim.x * blockDim.x)
        out[p] = from_f32<T>(acc[p]);
}

template <class T, bool kRefine>
cudaError_t launch_typed(const BackwardProblem& bp, float* ws, int* launches) {
    const Problem& pb = bp.fwd;
    const int H = (int)pb.H, W = (int)pb.W;
    const int K = H > W ? H : W;
    const int64_t planes = pb.planes();
    const int64_t n = pb.pixch();
    float* hbuf = ws;               // [4][planes][HW]
    float* dxacc = ws + 4 * n;      // [planes][HW]
    cudaError_t e = cudaMemsetAsync(dxacc, 0, sizeof(float) * (size_t)n, pb.stream);
    if (e != cudaSuccess) return e;
    const size_t smem_h = sizeof(float) * 2 * (size_t)(K + 2);
    const size_t smem_b = sizeof(float) * 4 * (size_t)K;
    auto hk = hidden_kernel<T, kRefine>;
    auto bk = backward_kernel<T, kRefine>;
    if ((e = cudaFuncSetAttribute(hk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_h)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(bk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b)) !=
        cudaSuccess)
        return e;
    const dim3 grid((unsigned)planes, 4);
    const T* x = static_cast<const T*>(pb.x);
    hk<<<grid, kThreads, smem_h, pb.stream>>>(x, pb.z, pb.lam, H, W, (int)pb.g, planes, hbuf);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    MutPtr4 dz, dl, du;
    for (int d = 0; d < 4; ++d) {
        dz.p[d] = bp.dz[d];
        dl.p[d] = bp.dlam[d];
        du.p[d] = bp.du[d];
    }
    if (pb.ev_begin) cudaEventRecord(pb.ev_begin, pb.stream);
    bk<<<grid, kThreads, smem_b, pb.stream>>>(x, pb.z, pb.lam, pb.u,
                                              static_cast<const T*>(bp.gy), H, W, (int)pb.g,
                                              planes, hbuf, dxacc, dz, dl, du);
    if (pb.ev_end) cudaEventRecord(pb.ev_end, pb.stream);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    round_kernel<T><<<148 * 8, 256, 0, pb.stream>>>(dxacc, n, static_cast<T*>(bp.dx));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    *launches += 3;
    return cudaSuccess;
}

}  // namespace

size_t backward_workspace_bytes(const Problem& pb) {
    return sizeof(float) * 5 * (size_t)pb.pixch();
}

cudaError_t launch_backward(BackwardProblem& bp, float* ws, int* launches) {
    bp.fwd.kernel_name = "backward_kernel";
    return bp.fwd.dtype == 0 ? launch_typed<float, true>(bp, ws, launches)
                             : launch_typed<__nv_bfloat16, false>(bp, ws, launches);
}

}  // namespace gspn
