// Device helpers shared by the GSPN kernels (sm_100a).
//
// Weight arithmetic follows the CSDN walkthrough "GSPN——在convolution基础上并行
// 序列建模", section "行随机矩阵": w_o = sigmoid(z_o) / sum over the row's existing
// neighbours of sigmoid(z_o').  With a_o = 1 + exp(-z_o) (so sigmoid = 1/a_o) the
// same ratio is
//     w_o = prod_{o' != o} a_o' / sum_o prod_{o' != o} a_o'
// over the existing neighbours, which needs three exponentials and one
// reciprocal per pixel instead of three sigmoids plus a normalising divide.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gspn {

struct Ptr4 {
    const void* p[4];
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <class T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// PTX approximate base-2 exponential and reciprocal (single MUFU instructions).
__device__ __forceinline__ float ex2_approx(float t) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
    return r;
}
__device__ __forceinline__ float rcp_approx(float s) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}

// a = 1 + exp(-z).  The exponent is capped at 2^62 so that the product of two
// denominators stays finite in fp32; this only changes the result when every
// existing neighbour of a pixel has a logit below about -43.
__device__ __forceinline__ float sig_denominator(float z) {
    const float t = fminf(z * -1.4426950408889634f, 62.0f);
    return 1.0f + ex2_approx(t);
}

// Normalised three-neighbour weights of one pixel.  has_lo / has_hi say whether
// the neighbours at orthogonal offset -1 / +1 exist; a missing one gets weight 0
// and is left out of the normaliser.  kRefine adds one Newton step to the
// reciprocal so the weights sum to 1 to within an fp32 rounding (used when the
// storage dtype is fp32).
template <bool kRefine>
__device__ __forceinline__ void tri_weights(float z0, float z1, float z2, bool has_lo,
                                            bool has_hi, float& w0, float& w1, float& w2) {
    const float a0 = has_lo ? sig_denominator(z0) : 1.0f;
    const float a1 = sig_denominator(z1);
    const float a2 = has_hi ? sig_denominator(z2) : 1.0f;
    const float p0 = has_lo ? a1 * a2 : 0.0f;
    const float p1 = a0 * a2;
    const float p2 = has_hi ? a0 * a1 : 0.0f;
    const float s = p0 + p1 + p2;
    float r = rcp_approx(s);
    if (kRefine) {
        const float e = fmaf(-s, r, 1.0f);
        r = fmaf(r, e, r);
    }
    w0 = p0 * r;
    w1 = p1 * r;
    w2 = p2 * r;
}

// Original-image pixel of scan line i, orthogonal position k, direction d.
__device__ __forceinline__ int pixel_of(int d, int H, int W, int i, int k) {
    switch (d) {
        case 0: return i * W + k;
        case 1: return (H - 1 - i) * W + k;
        case 2: return k * W + i;
        default: return k * W + (W - 1 - i);
    }
}

// Does scan line i start a propagation group?  Groups are blocks
// [s*g, (s+1)*g) of the original scan-axis coordinate.
__device__ __forceinline__ bool group_start(int d, int L, int g, int i) {
    if (i == 0) return true;
    if (g <= 0) return false;
    const bool fwd = (d == 0 || d == 2);
    const int a = fwd ? i : L - 1 - i;
    const int b = fwd ? i - 1 : L - i;
    return (a / g) != (b / g);
}

}  // namespace gspn
