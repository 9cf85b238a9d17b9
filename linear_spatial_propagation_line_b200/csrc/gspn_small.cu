// Whole-plane GSPN kernel for small planes (max(H, W) <= 64).
//
// One CTA owns one (b, c) plane.  It keeps the plane's fp32 output
// accumulator in shared memory for all four directions, so y is written to
// HBM exactly once.  For each direction:
//   phase 1 (all threads, fully parallel over pixels): read the three logits,
//     lambda, u and x of every pixel, form the row-stochastic weights
//     (sigmoid + normalisation over existing neighbours, CSDN walkthrough
//     "GSPN——在convolution基础上并行序列建模", section "行随机矩阵") and
//     lambda*x, and store them in scan-line order (line i, position k) with an
//     odd line pitch, so both the row-wise writes of the vertical directions
//     and the transposed writes of the horizontal directions are free of
//     shared-memory bank conflicts;
//   phase 2 (one warp): the sequential line recurrence h_i = w_i h_{i-1} +
//     lambda_i x_i (section "方法") with position k held by lane k % 32,
//     neighbours exchanged with warp shuffles, and u_d * h_d added to the
//     accumulator.  Local groups restart the recurrence (section
//     "全局与局部GSPN").
#include "gspn_internal.h"

namespace gspn {
namespace {

constexpr int kThreads = 256;

struct SmallLayout {
    int pitch_y;  // odd row pitch of the fp32 accumulator
    int kp_v;     // line pitch when K = W (vertical directions)
    int kp_h;     // line pitch when K = H (horizontal directions)
    int scr;      // floats per scratch array (multiple of 4)
    size_t bytes;
};

SmallLayout small_layout(int H, int W) {
    SmallLayout s;
    s.pitch_y = W | 1;
    s.kp_v = W | 1;
    s.kp_h = H | 1;
    int a = H * s.kp_v, b = W * s.kp_h;
    s.scr = ((a > b ? a : b) + 3) & ~3;
    s.bytes = sizeof(float) * ((size_t)((H * s.pitch_y + 3) & ~3) + 5 * (size_t)s.scr);
    return s;
}

template <class T, bool kRefine, int V>
__global__ void __launch_bounds__(kThreads)
    small_plane_kernel(const T* __restrict__ x, Ptr4 zp, Ptr4 lp, Ptr4 up, int H, int W, int g,
                       int d0, int d1, int pitch_y, int kp_v, int kp_h, int scr, int z_div,
                       T* __restrict__ y) {
    extern __shared__ __align__(16) float smem[];
    float* yacc = smem;
    float* sw0 = smem + ((H * pitch_y + 3) & ~3);
    float* sw1 = sw0 + scr;
    float* sw2 = sw1 + scr;
    float* slx = sw2 + scr;
    float* su = slx + scr;

    const int HW = H * W;
    const int64_t plane = blockIdx.x;
    const T* xq = x + plane * HW;
    for (int p = threadIdx.x; p < H * pitch_y; p += kThreads) yacc[p] = 0.0f;

    for (int d = d0; d < d1; ++d) {
        const T* zq = static_cast<const T*>(zp.p[d]) + (plane / z_div) * 3 * HW;
        const T* lq = static_cast<const T*>(lp.p[d]) + plane * HW;
        const T* uq = static_cast<const T*>(up.p[d]) + plane * HW;
        const bool vert = d < 2;
        const int L = vert ? H : W;
        const int K = vert ? W : H;
        const int KP = vert ? kp_v : kp_h;

        // ---- phase 1: per-pixel weights, lambda*x and u in scan-line order
        for (int p = threadIdx.x; p < HW; p += kThreads) {
            const int r = p / W, c = p - r * W;
            int i, k;
            switch (d) {
                case 0: i = r; k = c; break;
                case 1: i = H - 1 - r; k = c; break;
                case 2: i = c; k = r; break;
                default: i = W - 1 - c; k = r; break;
            }
            float w0, w1, w2;
            tri_weights<kRefine>(to_f32(zq[p]), to_f32(zq[HW + p]), to_f32(zq[2 * HW + p]), k > 0,
                                 k < K - 1, w0, w1, w2);
            const int s = i * KP + k;
            sw0[s] = w0;
            sw1[s] = w1;
            sw2[s] = w2;
            slx[s] = to_f32(lq[p]) * to_f32(xq[p]);
            su[s] = to_f32(uq[p]);
        }
        __syncthreads();

        // ---- phase 2: the recurrence, one warp, position k on lane k % 32
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            const unsigned full = 0xffffffffu;
            float h[V];
#pragma unroll
            for (int v = 0; v < V; ++v) h[v] = 0.0f;
            for (int i = 0; i < L; ++i) {
                const bool start = group_start(d, L, g, i);
                float hl[V], hr[V], hn[V];
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    // left neighbour of k = 32v + lane is k-1: lane-1, or lane 31 of slot v-1
                    const float send_l = (lane == 31) ? (v > 0 ? h[v > 0 ? v - 1 : 0] : 0.0f) : h[v];
                    hl[v] = __shfl_sync(full, send_l, (lane + 31) & 31);
                    // right neighbour k+1: lane+1, or lane 0 of slot v+1
                    const float send_r =
                        (lane == 0) ? (v + 1 < V ? h[v + 1 < V ? v + 1 : v] : 0.0f) : h[v];
                    hr[v] = __shfl_sync(full, send_r, (lane + 1) & 31);
                }
                if (lane == 0) hl[0] = 0.0f;
                if (lane == 31) hr[V - 1] = 0.0f;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int k = 32 * v + lane;
                    hn[v] = 0.0f;
                    if (k < K) {
                        const int s = i * KP + k;
                        const float lx = slx[s];
                        float hv = lx;
                        if (!start)
                            hv = fmaf(sw0[s], hl[v], fmaf(sw1[s], h[v], fmaf(sw2[s], hr[v], lx)));
                        hn[v] = hv;
                        int r, c;
                        switch (d) {
                            case 0: r = i; c = k; break;
                            case 1: r = H - 1 - i; c = k; break;
                            case 2: r = k; c = i; break;
                            default: r = k; c = W - 1 - i; break;
                        }
                        yacc[r * pitch_y + c] += su[s] * hv;
                    }
                }
#pragma unroll
                for (int v = 0; v < V; ++v) h[v] = hn[v];
            }
        }
        __syncthreads();
    }

    T* yq = y + plane * HW;
    for (int p = threadIdx.x; p < HW; p += kThreads) {
        const int r = p / W, c = p - r * W;
        yq[p] = from_f32<T>(yacc[r * pitch_y + c]);
    }
}

template <class T, bool kRefine>
cudaError_t launch_typed(const Problem& pb) {
    const int H = (int)pb.H, W = (int)pb.W;
    const SmallLayout s = small_layout(H, W);
    const int V = ((H > W ? H : W) + 31) / 32;
    auto run = [&](auto kernel) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)s.bytes);
        if (e != cudaSuccess) return e;
        if (pb.ev_begin) cudaEventRecord(pb.ev_begin, pb.stream);
        kernel<<<(unsigned)pb.planes(), kThreads, s.bytes, pb.stream>>>(
            static_cast<const T*>(pb.x), pb.z, pb.lam, pb.u, H, W, (int)pb.g, pb.d0, pb.d1,
            s.pitch_y, s.kp_v, s.kp_h, s.scr, (int)pb.z_div, static_cast<T*>(pb.y));
        if (pb.ev_end) cudaEventRecord(pb.ev_end, pb.stream);
        return cudaGetLastError();
    };
    if (V <= 1) return run(small_plane_kernel<T, kRefine, 1>);
    return run(small_plane_kernel<T, kRefine, 2>);
}

}  // namespace

bool small_plane_fits(const Problem& pb, size_t* smem_bytes) {
    if (pb.H > 64 || pb.W > 64) return false;
    if (pb.planes() > 0x7fffffffLL) return false;
    const SmallLayout s = small_layout((int)pb.H, (int)pb.W);
    if (smem_bytes) *smem_bytes = s.bytes;
    return s.bytes <= 200 * 1024;
}

cudaError_t launch_small_plane(Problem& pb, int* launches) {
    pb.kernel_name = "small_plane_kernel";
    cudaError_t e = pb.dtype == 0 ? launch_typed<float, true>(pb)
                                  : launch_typed<__nv_bfloat16, false>(pb);
    if (e == cudaSuccess) *launches += 1;
    return e;
}

}  // namespace gspn
