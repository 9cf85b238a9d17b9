// Generic GSPN line-chain path (any plane size).
//
// One CTA runs one (plane, direction) chain: the whole current line h_{i-1}
// lives in shared memory (double-buffered, zero-padded at both ends so a
// missing neighbour reads 0 with weight 0), every thread advances positions
// k = t, t + blockDim, ... of line i, and one barrier per line separates the
// steps of the recurrence h_i = w_i h_{i-1} + lambda_i x_i (CSDN walkthrough
// "GSPN——在convolution基础上并行序列建模", section "方法").  Each chain adds its
// u_d * h_d into an fp32 workspace with atomic adds; a conversion kernel then
// rounds the workspace to the output dtype once.
#include "gspn_internal.h"

namespace gspn {
namespace {

constexpr int kThreads = 512;

template <class T, bool kRefine>
__global__ void __launch_bounds__(kThreads)
    chain_kernel(const T* __restrict__ x, Ptr4 zp, Ptr4 lp, Ptr4 up, int H, int W, int g,
                 int d0, int z_div, float* __restrict__ ws) {
    extern __shared__ __align__(16) float hb[];
    const int d = d0 + (int)blockIdx.y;
    const int64_t plane = blockIdx.x;
    const int HW = H * W;
    const bool vert = d < 2;
    const int L = vert ? H : W;
    const int K = vert ? W : H;
    const T* xq = x + plane * HW;
    const T* zq = static_cast<const T*>(zp.p[d]) + (plane / z_div) * 3 * HW;
    const T* lq = static_cast<const T*>(lp.p[d]) + plane * HW;
    const T* uq = static_cast<const T*>(up.p[d]) + plane * HW;
    float* wq = ws + plane * HW;

    float* hcur = hb;
    float* hnxt = hb + K + 2;
    for (int k = threadIdx.x; k < K + 2; k += kThreads) {
        hcur[k] = 0.0f;
        hnxt[k] = 0.0f;
    }
    __syncthreads();

    for (int i = 0; i < L; ++i) {
        const bool start = group_start(d, L, g, i);
        for (int k = threadIdx.x; k < K; k += kThreads) {
            const int p = pixel_of(d, H, W, i, k);
            const float lx = to_f32(lq[p]) * to_f32(xq[p]);
            float hv = lx;
            if (!start) {
                float w0, w1, w2;
                tri_weights<kRefine>(to_f32(zq[p]), to_f32(zq[HW + p]), to_f32(zq[2 * HW + p]),
                                     k > 0, k < K - 1, w0, w1, w2);
                hv = fmaf(w0, hcur[k], fmaf(w1, hcur[k + 1], fmaf(w2, hcur[k + 2], lx)));
            }
            hnxt[k + 1] = hv;
            atomicAdd(wq + p, to_f32(uq[p]) * hv);
        }
        __syncthreads();
        float* t = hcur;
        hcur = hnxt;
        hnxt = t;
    }
}

template <class T>
__global__ void convert_kernel(const float* __restrict__ ws, int64_t n, T* __restrict__ y) {
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < n;
         p += (int64_t)gridDim.x * blockDim.x)
        y[p] = from_f32<T>(ws[p]);
}

template <class T, bool kRefine>
cudaError_t launch_typed(Problem& pb, float* ws, int* launches) {
    const int H = (int)pb.H, W = (int)pb.W;
    const int K = H > W ? H : W;
    const size_t smem = sizeof(float) * 2 * (size_t)(K + 2);
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(float) * (size_t)pb.pixch(), pb.stream);
    if (e != cudaSuccess) return e;
    auto kernel = chain_kernel<T, kRefine>;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)pb.planes(), (unsigned)(pb.d1 - pb.d0));
    if (pb.ev_begin) cudaEventRecord(pb.ev_begin, pb.stream);
    kernel<<<grid, kThreads, smem, pb.stream>>>(static_cast<const T*>(pb.x), pb.z, pb.lam, pb.u,
                                                H, W, (int)pb.g, pb.d0, (int)pb.z_div, ws);
    if (pb.ev_end) cudaEventRecord(pb.ev_end, pb.stream);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    convert_kernel<T><<<148 * 8, 256, 0, pb.stream>>>(ws, pb.pixch(), static_cast<T*>(pb.y));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    *launches += 2;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_chain(Problem& pb, float* ws, int* launches) {
    pb.kernel_name = "chain_kernel";
    return pb.dtype == 0 ? launch_typed<float, true>(pb, ws, launches)
                         : launch_typed<__nv_bfloat16, false>(pb, ws, launches);
}

}  // namespace gspn
