// Line-sweep GSPN kernel for large planes (sm_100a): the scan line lives in
// registers and neighbouring positions meet through warp shuffles.
//
// What it computes (the same operation as the other kernels): for every (b, c)
// plane and direction d, the line recurrence
//   h_i = w_i h_{i-1} + lambda_i (.) x_i,   h = lambda (.) x on a group's first line
// with three-neighbour row-stochastic weights (sigmoid, then normalisation over
// the existing neighbours), and y = sum_d u_d (.) h_d -- CSDN walkthrough
// "GSPN——在convolution基础上并行序列建模", sections "方法", "如何设计一个高效的
// 传播层", "行随机矩阵" and "全局与局部GSPN".
//
// How (B200 design):
//  * A chain (plane, direction) runs on So CTAs of one thread block cluster;
//    CTA sr owns positions [sr*Kc, (sr+1)*Kc) of the line.
//  * Inside a CTA every consumer warp keeps a segment of 32 kP consecutive
//    line positions in registers, kP (2) per lane as one packed fp32 pair.  A
//    step needs the neighbours' previous states, which adjacent lanes trade by
//    warp shuffles, so no block-wide barrier separates two steps.
//  * Segments of adjacent warps overlap by one lane (kP positions) on each
//    side.  A copy of a position stays exact for as many steps as it lies away
//    from the end of the segment holding it, so warps refresh their edge lanes
//    from the neighbouring warp through shared memory only every kP steps (one
//    named barrier), and the interior positions of a segment are always exact.
//    Between CTAs of a chain the same holds with 16-position halos refreshed
//    through DSMEM `st.async` every 16 steps.
//  * Vertical scans (along H): a lane's positions are adjacent columns, one
//    shared load per tensor and step.  Horizontal scans (along W): a lane's
//    positions are the rows lane + 32 j of its segment, so one 8-byte load of
//    a row covers several steps and a warp's loads cover consecutive rows; the
//    scan runs along W with no transposition.
//  * Inputs stream through a shared-memory ring filled by TMA tensor loads (no
//    multicast) from a producer warp; one stage is 32 bytes of steps (16 bf16
//    or 8 fp32 lines).  Horizontal maps use the 32-byte swizzle, so that the
//    16-byte halves of consecutive rows fall in different banks.  u_d * h_d of the four directions accumulates in an fp32
//    "slot" per plane kept L2-resident (evict_last reductions); the team that
//    finishes a plane's last chain rounds the slot into y, re-zeroes it and
//    releases it to the plane n_slots later in the work queue.
//  * Every wait (TMA stage, slot release, halo) is bounded by a global-timer
//    limit; on expiry the kernel records an error word and winds down.
//
// Weights: with a_o = 1 + exp(-z_o) scaled by 2^-32, w_o = prod_{o' != o} a_o' /
// sum_o prod_{o' != o} a_o' over the existing neighbours (3 exponentials and 1
// reciprocal per pixel).  A missing neighbour's logit is replaced by +inf (its
// exponential is 0, so its a is finite) and its product by 0.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdio.h>
#include <stdlib.h>

#include <type_traits>
#include <utility>

#include "gspn_internal.h"
#include "gspn_ptx.cuh"

namespace gspn {
namespace {

using ptx::f2;

constexpr int kP = 2;           // line positions per lane (one packed pair)
constexpr int kSegLen = 32 * kP;  // positions per warp segment
constexpr int kStride = kSegLen - 2 * kP;  // segment spacing: interior positions of a segment
constexpr int kEpoch = kP;      // steps between warp refreshes (one lane of halo)
constexpr int kXHalo = 16;      // halo between CTAs == steps between CTA refreshes
constexpr int kEdge = 8;        // window margin at the ends of the line
constexpr int kMaxWarps = 10;   // consumer warps per CTA
constexpr int kMaxOwned = 544;  // owned positions per CTA: two stages of the window fit
constexpr int kMaxStages = 4;
constexpr int kMaxSlots = 64;
constexpr int kMaxItems = 4;    // work items per plane

// Control block in global memory (the first bytes of the workspace); the
// layout matches the fused kernel's so that both share the workspace handling.
struct SweepCtrl {
    int sticky_error;  // kept across calls until the host reads it
    int pad0[3];
    int call_error;    // this call: nonzero stops every team (1 TMA, 2 slot, 3 halo, 4 stale, 6 ring)
    int next_item;
    int pad1[10];
    int slot_epoch[kMaxSlots];
    // int plane_done[planes] follows
};
constexpr size_t kCtrlResetOffset = 16;  // bytes before this survive the per-call reset

struct __align__(64) SweepParams {
    CUtensorMap tm_xv, tm_xh;  // x with vertical / horizontal boxes
    CUtensorMap tm_z[4];       // logits of direction d (boxes of d's orientation)
    CUtensorMap tm_l[4];
    CUtensorMap tm_u[4];
    void* y;
    float* slots;
    SweepCtrl* ctrl;
    int* plane_done;
    unsigned long long timeout_ns;
    int H, W, planes, g;
    int S;                 // CTAs per cluster (team)
    int So[2];             // CTAs per chain: [0] vertical scans, [1] horizontal scans
    int Kc[2];             // owned positions per CTA
    int nw;                // consumer warps per CTA
    int nb[2], bw[2];      // boxes per tensor and stage, box width in line positions
    int tile_bytes;        // one tensor's tile in one stage
    int stages;            // depth of the shared-memory ring
    int z_div;             // logits of plane q are logit plane q / z_div
    int n_slots;
    int n_items;
    int ipp;               // work items per plane
    int item_dir[kMaxItems][2];  // directions run by the two halves of a team (-1: idle)
    int force_stale;       // test hook: expect a slot epoch that never comes
};

// Shared-memory carve-up.
struct View {
    uint32_t ring;      // [stages][6 tensors][tile_bytes]
    uint32_t xb;        // warp refresh buffer: float [2 parity][kMaxWarps][2 sides][kP]
    uint32_t rx;        // CTA halo receive buffer: float [2 parity][2 sides][kXHalo]
    uint32_t full;      // uint64 [kMaxStages]: TMA completion
    uint32_t empty;     // uint64 [kMaxStages]: stage released (one arrival per consumer warp)
    uint32_t halo;      // uint64 [2]: CTA halo data arrived
    int* cell;          // [0] item, [1] convert decision
};

__host__ __device__ inline size_t smem_bytes_for(int tile_bytes, int stages, size_t* off_xb,
                                                 size_t* off_rx, size_t* off_bar) {
    size_t off = (size_t)stages * 6 * tile_bytes;
    *off_xb = off;
    off += sizeof(float) * 2 * kMaxWarps * 2 * kP;
    *off_rx = off;
    off += sizeof(float) * 2 * 2 * kXHalo;
    off = (off + 7) & ~(size_t)7;
    *off_bar = off;
    off += sizeof(uint64_t) * (2 * kMaxStages + 2) + 4 * sizeof(int);
    return off;
}

__device__ __forceinline__ View carve(char* base, const SweepParams& p) {
    size_t oxb, orx, obar;
    smem_bytes_for(p.tile_bytes, p.stages, &oxb, &orx, &obar);
    View v;
    v.ring = ptx::smem_addr(base);
    v.xb = v.ring + (uint32_t)oxb;
    v.rx = v.ring + (uint32_t)orx;
    v.full = v.ring + (uint32_t)obar;
    v.empty = v.full + 8u * kMaxStages;
    v.halo = v.empty + 8u * kMaxStages;
    v.cell = reinterpret_cast<int*>(base + obar + sizeof(uint64_t) * (2 * kMaxStages + 2));
    return v;
}

template <class F, int... Is>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, Is...>) {
    (f(std::integral_constant<int, Is>{}), ...);
}
template <int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

// Barrier phases seen by the consumer threads (identical in all of them).
struct Phases {
    uint32_t full;  // bit s: parity to wait for on full[s]
    uint32_t halo;  // bit p: parity to wait for on halo[p]
    bool abort;     // a bounded wait expired: skip further waits
};

__device__ __forceinline__ void report_error(SweepCtrl* ctrl, int code) {
    atomicCAS(&ctrl->call_error, 0, code);
    atomicCAS(&ctrl->sticky_error, 0, code);
}

__device__ __forceinline__ void wait_bounded(const SweepParams& p, bool& abort, uint32_t bar,
                                             uint32_t parity, int code) {
    if (abort) return;
    if (!ptx::wait_parity_bounded(bar, parity, p.timeout_ns)) {
        abort = true;
        report_error(p.ctrl, code);
    }
}

// ------------------------------------------------------------------ weights
constexpr float kScale = 2.3283064365386963e-10f;  // 2^-32
constexpr float kNegLog2e = -1.4426950408889634f;

__device__ __forceinline__ f2 splat(float v) { return ptx::pk(v, v); }

// Inputs of one step for a pair of positions (low half: first position).
struct PairIn {
    f2 x, z0, z1, z2, lam, u;
};
// What the state update of a pair needs: h = w0 hl + w1 hs + w2 hr + lx.
struct PairW {
    f2 w0, w1, w2, lx, u;
};

__device__ __forceinline__ f2 bf16x2_pair(uint32_t w) {
    return ptx::pk(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Weights of a pair.  lo0 / lo1: the first / second position has no
// neighbour at offset -1; hi0 / hi1: none at offset +1.
template <bool kRefine>
__device__ __forceinline__ PairW pair_weights(const PairIn& in, bool lo0, bool lo1, bool hi0,
                                              bool hi1) {
    const float inf = __int_as_float(0x7f800000);
    float z0a, z0b, z2a, z2b;
    ptx::upk(in.z0, z0a, z0b);
    ptx::upk(in.z2, z2a, z2b);
    const f2 z0 = ptx::pk(lo0 ? inf : z0a, lo1 ? inf : z0b);
    const f2 z2 = ptx::pk(hi0 ? inf : z2a, hi1 ? inf : z2b);
    const f2 kL = splat(kNegLog2e), kO = splat(-32.0f), kS = splat(kScale);
    f2 t0 = ptx::fma2(z0, kL, kO), t1 = ptx::fma2(in.z1, kL, kO), t2 = ptx::fma2(z2, kL, kO);
    float u0, v0, u1, v1, u2, v2;
    ptx::upk(t0, u0, v0);
    ptx::upk(t1, u1, v1);
    ptx::upk(t2, u2, v2);
    const f2 a0 = ptx::add2(ptx::pk(ex2_approx(u0), ex2_approx(v0)), kS);
    const f2 a1 = ptx::add2(ptx::pk(ex2_approx(u1), ex2_approx(v1)), kS);
    const f2 a2 = ptx::add2(ptx::pk(ex2_approx(u2), ex2_approx(v2)), kS);
    PairW W;
    W.lx = ptx::mul2(in.lam, in.x);
    W.u = in.u;
    f2 p0 = ptx::mul2(a1, a2);
    f2 p2 = ptx::mul2(a0, a1);
    const f2 p1 = ptx::mul2(a0, a2);
    {
        float pa, pb;
        ptx::upk(p0, pa, pb);
        p0 = ptx::pk(lo0 ? 0.0f : pa, lo1 ? 0.0f : pb);
        ptx::upk(p2, pa, pb);
        p2 = ptx::pk(hi0 ? 0.0f : pa, hi1 ? 0.0f : pb);
    }
    const f2 sum = ptx::add2(ptx::add2(p0, p1), p2);
    float s0, s1;
    ptx::upk(sum, s0, s1);
    f2 r = ptx::pk(rcp_approx(s0), rcp_approx(s1));
    if (kRefine) {  // one Newton step: r += r (1 - s r)
        const f2 e = ptx::fma2(ptx::mul2(sum, splat(-1.0f)), r, splat(1.0f));
        r = ptx::fma2(r, e, r);
    }
    W.w0 = ptx::mul2(p0, r);
    W.w1 = ptx::mul2(p1, r);
    W.w2 = ptx::mul2(p2, r);
    return W;
}

__device__ __forceinline__ f2 pair_state(const PairW& W, f2 hl, f2 hs, f2 hr) {
    return ptx::fma2(W.w2, hr, ptx::fma2(W.w1, hs, ptx::fma2(W.w0, hl, W.lx)));
}

// Element e of a 16-byte vector of bf16 (e < 8) or fp32 (e < 4).
template <class T>
__device__ __forceinline__ float vec_elem(const uint4& v, int e) {
    if constexpr (sizeof(T) == 4) {
        return __uint_as_float(e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w);
    } else {
        const int q = e >> 1;
        const uint32_t w = q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
        return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
    }
}

// Element e of an 8-byte vector of bf16 (e < 4) or fp32 (e < 2).
template <class T>
__device__ __forceinline__ float vec2_elem(const uint2& v, int e) {
    if constexpr (sizeof(T) == 4) {
        return __uint_as_float(e == 0 ? v.x : v.y);
    } else {
        const uint32_t w = (e >> 1) ? v.y : v.x;
        return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
    }
}

// First step > 0 at which a local group restarts (INT_MAX if none); later
// restarts follow every g steps.
__device__ __forceinline__ int first_restart(int g, int L, bool fwd) {
    if (g <= 0) return 0x7fffffff;
    return fwd ? g : ((L - 1) % g) + 1;
}

__device__ __forceinline__ const CUtensorMap* tensor_map(const SweepParams& p, bool vert, int d,
                                                         int tensor) {
    if (tensor == 0) return vert ? &p.tm_xv : &p.tm_xh;
    return tensor <= 3 ? &p.tm_z[d] : tensor == 4 ? &p.tm_l[d] : &p.tm_u[d];
}
__device__ __forceinline__ int tensor_plane(const SweepParams& p, int q, int tensor) {
    return tensor == 0 ? q : tensor <= 3 ? 3 * (q / p.z_div) + tensor - 1 : q;
}

// ------------------------------------------------------------------ producer
// The producer warp fills the ring: it waits for a slot's release (one arrival
// per consumer warp per use) before reusing it, sets the expected bytes and
// spreads the stage's boxes over its lanes.
struct ProducerState {
    uint32_t used;   // bit s: slot s has been filled before
    uint32_t phase;  // bit s: parity of the next release of slot s
    uint32_t fill;   // bit s: parity of the next fill of slot s
    bool abort;
};

template <class T, bool VERT, bool FWD>
__device__ __forceinline__ void produce(const SweepParams& p, const View& sm, ProducerState& ps,
                                        int q, int d, int ws) {
    constexpr int J = 32 / (int)sizeof(T);
    const int o = VERT ? 0 : 1;
    const int L = VERT ? p.H : p.W;
    const int nst = (L + J - 1) / J;
    const int nb = p.nb[o], bw = p.bw[o];
    const uint32_t box_bytes = 32u * (uint32_t)bw;  // bw positions x 32 bytes of steps
    const uint32_t stage_bytes = 6u * nb * box_bytes;
    const int lane = threadIdx.x & 31;
    const uint64_t pol_in = ptx::policy_evict_first();
    for (int st = 0; st < nst; ++st) {
        const int sl = st % p.stages;
        if (ps.used & (1u << sl)) {
            if (!ps.abort && !ptx::wait_parity_bounded(sm.empty + 8u * sl, (ps.phase >> sl) & 1u,
                                                       p.timeout_ns)) {
                ps.abort = true;
                report_error(p.ctrl, 6);
            }
            ps.phase ^= 1u << sl;
        }
        ps.used |= 1u << sl;
        ps.fill ^= 1u << sl;
        const uint32_t bar = sm.full + 8u * sl;
        if (lane == 0) ptx::mbar_arrive_expect_tx(bar, stage_bytes);
        __syncwarp();
        const int step0 = FWD ? st * J : L - J - st * J;  // first line of the stage box
        for (int b = lane; b < 6 * nb; b += 32) {
            const int tensor = b / nb, bi = b % nb;
            const uint32_t dst =
                sm.ring + (uint32_t)(sl * 6 + tensor) * p.tile_bytes + bi * box_bytes;
            const CUtensorMap* map = tensor_map(p, VERT, d, tensor);
            const int zc = tensor_plane(p, q, tensor);
            const int pos = ws + bi * bw;
            const int cx = VERT ? pos : step0, cy = VERT ? step0 : pos;
            if (tensor == 0)  // x is read by all four directions: default L2 policy
                ptx::tma_load_3d_normal(dst, map, cx, cy, zc, bar);
            else
                ptx::tma_load_3d(dst, map, cx, cy, zc, bar, pol_in);
        }
        __syncwarp();
    }
    // No load of this chain may still be landing when the CTA moves on (or
    // exits): wait for the last fill of every slot, also after an abort, when
    // the consumers may have stopped waiting for them.
    for (int sl = 0; sl < p.stages && sl < nst; ++sl) {
        if (!ptx::wait_parity_bounded(sm.full + 8u * sl, ((ps.fill >> sl) & 1u) ^ 1u,
                                      p.timeout_ns)) {
            ps.abort = true;
            report_error(p.ctrl, 1);
        }
    }
}

// CTA halo refresh after step s (every kXHalo steps of a chain on several
// CTAs): a CTA's first and last kXHalo owned positions go to its neighbours'
// halo buffers through DSMEM stores that complete transaction bytes on their
// halo barrier; the lanes holding halo positions then read what arrived.
// Thread 0 re-arms the barrier for the exchange two blocks later.
__device__ __forceinline__ void cta_refresh(const SweepParams& p, const View& sm, Phases& ph,
                                            float (&v)[kP], const int (&a)[kP],
                                            const bool (&core)[kP], int own0, int Kc, int So,
                                            int sr, int rank0, int s, int L) {
    const int t = threadIdx.x;
    const bool has_left = sr > 0, has_right = sr < So - 1;
    const int blk = (s + 1) / kXHalo - 1;
    const int par = blk & 1;
    const uint32_t bar = sm.halo + 8u * par;
    const uint32_t rxl = sm.rx + 4u * (par * 2 + 0) * kXHalo;  // left halo
    const uint32_t rxr = sm.rx + 4u * (par * 2 + 1) * kXHalo;  // right halo
    const int r0 = own0 + Kc - kXHalo;
#pragma unroll
    for (int j = 0; j < kP; ++j) {
        // first owned positions -> left neighbour's right halo
        if (!ph.abort && has_left && core[j] && a[j] >= own0 && a[j] < own0 + kXHalo)
            ptx::st_async_f32(ptx::map_shared(rxr + 4u * (a[j] - own0), rank0 + sr - 1), v[j],
                              ptx::map_shared(bar, rank0 + sr - 1));
        // last owned positions -> right neighbour's left halo
        if (!ph.abort && has_right && core[j] && a[j] >= r0 && a[j] < own0 + Kc)
            ptx::st_async_f32(ptx::map_shared(rxl + 4u * (a[j] - r0), rank0 + sr + 1), v[j],
                              ptx::map_shared(bar, rank0 + sr + 1));
    }
    bool recv = t == 0;
#pragma unroll
    for (int j = 0; j < kP; ++j)
        recv = recv || (has_left && a[j] >= own0 - kXHalo && a[j] < own0) ||
               (has_right && a[j] >= own0 + Kc && a[j] < own0 + Kc + kXHalo);
    if (recv) {
        wait_bounded(p, ph.abort, bar, (ph.halo >> par) & 1u, 3);
#pragma unroll
        for (int j = 0; j < kP; ++j) {
            if (has_left && a[j] >= own0 - kXHalo && a[j] < own0)
                v[j] = ptx::lds_f32(rxl + 4u * (a[j] - (own0 - kXHalo)));
            if (has_right && a[j] >= own0 + Kc && a[j] < own0 + Kc + kXHalo)
                v[j] = ptx::lds_f32(rxr + 4u * (a[j] - (own0 + Kc)));
        }
    }
    if (t == 0 && blk * kXHalo + 3 * kXHalo < L) {
        const uint32_t bytes =
            sizeof(float) * kXHalo * ((has_left ? 1u : 0u) + (has_right ? 1u : 0u));
        ptx::mbar_arrive_expect_tx(bar, bytes);  // block blk + 2
    }
    ph.halo ^= 1u << par;
}

// Warp refresh after an epoch: every warp publishes the states of its first
// and last interior lane's positions; after one named barrier over the
// consumer warps, the edge lanes take over their neighbours' values (the
// window's outer edges keep theirs: they are refreshed by the CTA exchange or
// lie outside the line).  Vertically a lane's positions are contiguous, so
// the edges are whole lanes (lanes 1 and 30 send, lanes 0 and 31 receive);
// horizontally position j of lane l is l + 32 j, so the edges are the first
// and last kP rows of the segment, one value per lane.  Predicated accesses,
// no divergence.
template <bool VERT>
__device__ __forceinline__ void warp_refresh(const View& sm, float (&v)[kP], int epoch, int warp,
                                             int lane, int nw, uint32_t nthr) {
    const int par = epoch & 1;
    const uint32_t xw = sm.xb + 4u * kP * 2 * (par * kMaxWarps + warp);
    const uint32_t xprev_r = xw - 4u * kP * 2 + 4u * kP;  // previous warp, right edge
    const uint32_t xnext_l = xw + 4u * kP * 2;            // next warp, left edge
    if constexpr (VERT) {
        if constexpr (kP == 4) {
            ptx::sts_v4_f32_if(lane == 1, xw, v[0], v[1], v[2], v[3]);
            ptx::sts_v4_f32_if(lane == 30, xw + 4u * kP, v[0], v[1], v[2], v[3]);
        } else {
            ptx::sts_v2_f32_if(lane == 1, xw, v[0], v[1]);
            ptx::sts_v2_f32_if(lane == 30, xw + 4u * kP, v[0], v[1]);
        }
        ptx::named_barrier(1, nthr);
        const bool take_l = lane == 0 && warp > 0;
        const bool take_r = lane == 31 && warp < nw - 1;
        const uint32_t src = take_l ? xprev_r : take_r ? xnext_l : xw;
        if constexpr (kP == 4) {
            const uint4 r4 = ptx::lds_v4(src);
            const bool tk = take_l || take_r;
            v[0] = tk ? __uint_as_float(r4.x) : v[0];
            v[1] = tk ? __uint_as_float(r4.y) : v[1];
            v[2] = tk ? __uint_as_float(r4.z) : v[2];
            v[3] = tk ? __uint_as_float(r4.w) : v[3];
        } else {
            const uint2 r2 = ptx::lds_v2(src);
            const bool tk = take_l || take_r;
            v[0] = tk ? __uint_as_float(r2.x) : v[0];
            v[1] = tk ? __uint_as_float(r2.y) : v[1];
        }
    } else {
        const int lo = lane & (kP - 1);
        ptx::sts_f32_if(lane >= kP && lane < 2 * kP, xw + 4u * lo, v[0]);
        ptx::sts_f32_if(lane >= 32 - 2 * kP && lane < 32 - kP, xw + 4u * kP + 4u * lo, v[kP - 1]);
        ptx::named_barrier(1, nthr);
        const bool take0 = lane < kP && warp > 0;
        const bool take1 = lane >= 32 - kP && warp < nw - 1;
        const float r1 = ptx::lds_f32((take0 ? xprev_r : take1 ? xnext_l : xw) + 4u * lo);
        v[0] = take0 ? r1 : v[0];
        v[kP - 1] = take1 ? r1 : v[kP - 1];
    }
}

// ------------------------------------------------------------------ consumers
// Runs one chain on this CTA (chain rank sr of So; cluster rank of chain rank 0
// is rank0).  Window position 0 is line position ws = sr*Kc - (left margin).
// A lane's kP positions travel as kNP packed pairs.  Software pipeline: during
// step w a lane issues the shared loads of step w + 2 (vertical), computes the
// weights of step w + 1 and finishes step w with the weights computed one step
// earlier, so the dependent state chain of a step (three fused multiply-adds
// after the shuffles) overlaps the exponentials of the next.
template <class T, bool kRefine, bool VERT, bool FWD>
__device__ __forceinline__ void consume(const SweepParams& p, const View& sm, Phases& ph, int q,
                                        int sr, int So, int rank0, int ws, uint64_t pol_acc) {
    constexpr int J = 32 / (int)sizeof(T);  // steps per stage
    constexpr int kNP = kP / 2;             // pairs per lane
    const int H = p.H, W = p.W;
    const int L = VERT ? H : W, K = VERT ? W : H;
    const int o = VERT ? 0 : 1;
    const int Kc = p.Kc[o];
    const int own0 = sr * Kc;
    const int own1 = min(K, own0 + Kc);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int nw = p.nw;
    const uint32_t nthr = 32u * (uint32_t)nw;
    const int nst = (L + J - 1) / J;
    const int seg0 = warp * kStride;  // window position of this warp's segment
    const uint32_t tb = (uint32_t)p.tile_bytes;
    const int stages = p.stages;
    const int tile_pos = p.nb[o] * p.bw[o];  // window positions held by a tile

    // This lane's positions: vertical seg0 + kP lane + j, horizontal seg0 + lane + 32 j.
    int rel[kP], a[kP];
    bool own[kP], core[kP], hi[kP];
#pragma unroll
    for (int j = 0; j < kP; ++j) {
        rel[j] = VERT ? kP * lane + j : lane + 32 * j;
        a[j] = ws + seg0 + rel[j];
        core[j] = rel[j] >= kP && rel[j] < kSegLen - kP;
        own[j] = core[j] && a[j] >= own0 && a[j] < own1;
        // missing neighbour at offset +1: vertically only the last position of
        // a lane can be column W - 1 (W is a multiple of kP)
        hi[j] = (VERT && j != kP - 1) ? false : a[j] == K - 1;
    }
    // missing neighbour at offset -1: only position j = 0 can be line position 0
    const bool lo0 = a[0] == 0;

    // Shared-memory offsets of this lane's inputs inside a tensor's tile.
    // Window positions past the tile (beyond every halo) read the tile's last
    // ones: any finite inputs do, their results are never used.
    uint32_t voff = 0, vpitch = 0;  // vertical: this lane's columns, row pitch
    uint32_t hrow[kP], hswz[kP];    // horizontal: row offsets, 16-byte half swap of the row
    if constexpr (VERT) {
        const int bw = p.bw[0];
        int c = seg0 + kP * lane;
        if (c > tile_pos - kP) c = tile_pos - kP;
        voff = (uint32_t)(c / bw) * (32u * bw) + (uint32_t)(c % bw) * sizeof(T);
        vpitch = (uint32_t)bw * sizeof(T);
    } else {
#pragma unroll
        for (int j = 0; j < kP; ++j) {
            int r = seg0 + rel[j];
            if (r > tile_pos - 1) r = tile_pos - 1;
            hrow[j] = 32u * (uint32_t)r;
            hswz[j] = (uint32_t)(r >> 2) & 1u;  // the maps' 32-byte swizzle
        }
    }
    float* const slot = p.slots + (size_t)(q % p.n_slots) * H * W;

    int lsl = 0;  // slot of the next stage to acquire
    auto acquire = [&]() {
        wait_bounded(p, ph.abort, sm.full + 8u * lsl, (ph.full >> lsl) & 1u, 1);
        ph.full ^= 1u << lsl;
        lsl = (lsl + 1 == stages) ? 0 : lsl + 1;
    };
    auto release = [&](int sl) {
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(sm.empty + 8u * sl);
    };

    // vertical: the inputs of box row r of a stage, kP elements per tensor
    constexpr int kVW = kP * (int)sizeof(T) / 4;  // 32-bit words per tensor and step
    struct VRaw {
        uint32_t w[6][kVW];
    };
    auto vfetch = [&](int sl, int r, VRaw& v) {
        const uint32_t b = sm.ring + (uint32_t)sl * 6u * tb + voff + (uint32_t)r * vpitch;
#pragma unroll
        for (int k6 = 0; k6 < 6; ++k6) {
            if constexpr (kVW == 4) {
                const uint4 x = ptx::lds_v4(b + k6 * tb);
                v.w[k6][0] = x.x, v.w[k6][1] = x.y, v.w[k6][2] = x.z, v.w[k6][3] = x.w;
            } else if constexpr (kVW == 2) {
                const uint2 x = ptx::lds_v2(b + k6 * tb);
                v.w[k6][0] = x.x, v.w[k6][1] = x.y;
            } else {
                v.w[k6][0] = ptx::lds_u32(b + k6 * tb);
            }
        }
    };
    auto vweights = [&](const VRaw& v, PairW (&Wp)[kNP]) {
#pragma unroll
        for (int k = 0; k < kNP; ++k) {
            f2 qv[6];
#pragma unroll
            for (int k6 = 0; k6 < 6; ++k6) {
                if constexpr (sizeof(T) == 4)
                    qv[k6] = ptx::pk(__uint_as_float(v.w[k6][2 * k]),
                                     __uint_as_float(v.w[k6][2 * k + 1]));
                else
                    qv[k6] = bf16x2_pair(v.w[k6][k]);
            }
            Wp[k] = pair_weights<kRefine>(PairIn{qv[0], qv[1], qv[2], qv[3], qv[4], qv[5]},
                                          k == 0 && lo0, false, hi[2 * k], hi[2 * k + 1]);
        }
    };
    // horizontal: one 8-byte chunk (JC steps) of this lane's rows in a stage;
    // chunk c of a 32-byte row lies in 16-byte half c / 2, swapped by the swizzle
    constexpr int JC = 8 / (int)sizeof(T);
    uint2 hraw[6][kP];
    auto hfetch = [&](int sl, int c) {
        const uint32_t b = sm.ring + (uint32_t)sl * 6u * tb + 8u * (uint32_t)(c & 1);
#pragma unroll
        for (int k6 = 0; k6 < 6; ++k6)
#pragma unroll
            for (int j = 0; j < kP; ++j)
                hraw[k6][j] =
                    ptx::lds_v2(b + k6 * tb + hrow[j] + 16u * ((uint32_t)(c >> 1) ^ hswz[j]));
    };
    auto hweights = [&](int e, PairW (&Wp)[kNP]) {
#pragma unroll
        for (int k = 0; k < kNP; ++k) {
            f2 qv[6];
#pragma unroll
            for (int k6 = 0; k6 < 6; ++k6)
                qv[k6] = ptx::pk(vec2_elem<T>(hraw[k6][2 * k], e),
                                 vec2_elem<T>(hraw[k6][2 * k + 1], e));
            Wp[k] = pair_weights<kRefine>(PairIn{qv[0], qv[1], qv[2], qv[3], qv[4], qv[5]},
                                          k == 0 && lo0, false, hi[2 * k], hi[2 * k + 1]);
        }
    };

    const bool has_left = sr > 0, has_right = sr < So - 1;
    auto arm_halo = [&](int blk) {
        if (blk * kXHalo + kXHalo < L) {
            const uint32_t bytes =
                sizeof(float) * kXHalo * ((has_left ? 1u : 0u) + (has_right ? 1u : 0u));
            ptx::mbar_arrive_expect_tx(sm.halo + 8u * (blk & 1), bytes);
        }
    };
    if (So > 1 && t == 0) {
        arm_halo(0);
        arm_halo(1);
    }

    f2 h[kNP];      // this lane's states, pair k = positions (2k, 2k + 1)
    f2 acc[kP][2];  // horizontal: u*h of the last 4 steps per row
#pragma unroll
    for (int k = 0; k < kNP; ++k) h[k] = splat(0.0f);
#pragma unroll
    for (int j = 0; j < kP; ++j) acc[j][0] = acc[j][1] = splat(0.0f);

    int next_rs = first_restart(p.g, L, FWD);
    int epoch = 0;
    int cur_sl = 0;
    PairW Wt[kNP];  // weights of the current step
    VRaw vnext;     // vertical: raw inputs of the next step
    acquire();
    if constexpr (VERT) {
        VRaw v0;
        vfetch(cur_sl, FWD ? 0 : J - 1, v0);
        vfetch(cur_sl, FWD ? 1 : J - 2, vnext);
        vweights(v0, Wt);
    } else {
        // step w of a stage is column FWD ? w : J - 1 - w of its box
        hfetch(cur_sl, FWD ? 0 : (J - 1) / JC);
        hweights(FWD ? 0 : JC - 1, Wt);
    }
    for (int st = 0; st < nst; ++st) {
        const int nxt_sl = (cur_sl + 1 == stages) ? 0 : cur_sl + 1;
        const bool more = st + 1 < nst;
        uint32_t starts = st == 0 ? 1u : 0u;  // bit w: step w of the stage starts a group
        while (next_rs < (st + 1) * J) {
            starts |= 1u << (next_rs - st * J);
            next_rs += p.g;
        }
        static_for<J>([&](auto wc) {
            constexpr int w = decltype(wc)::value;
            const int s = st * J + w;
            // 1. weights of step w + 1 (inputs fetched a step earlier)
            PairW Wn[kNP];
            if constexpr (VERT) {
                VRaw vfar;  // inputs of step w + 2
                constexpr int w2 = w + 2;
                if constexpr (w2 < J) {
                    vfetch(cur_sl, FWD ? w2 : J - 1 - w2, vfar);
                } else {
                    if (more) {
                        if constexpr (w2 == J) acquire();
                        vfetch(nxt_sl, FWD ? w2 - J : 2 * J - 1 - w2, vfar);
                    }
                }
                vweights(vnext, Wn);
                vnext = vfar;
            } else {
                constexpr int w1 = (w + 1) % J;             // step w + 1 within its stage
                constexpr int col = FWD ? w1 : J - 1 - w1;  // its column in the stage box
                if constexpr (w + 1 == J) {
                    if (more) {
                        acquire();
                        hfetch(nxt_sl, col / JC);
                    }
                } else if constexpr (w1 % JC == 0) {
                    hfetch(cur_sl, col / JC);
                }
                hweights(col % JC, Wn);
            }
            // 2. neighbours' previous states
            float hv[kP];
#pragma unroll
            for (int k = 0; k < kNP; ++k) ptx::upk(h[k], hv[2 * k], hv[2 * k + 1]);
            float hl[kP], hr[kP];
            if constexpr (VERT) {
                const float left = __shfl_up_sync(0xffffffffu, hv[kP - 1], 1);
                const float right = __shfl_down_sync(0xffffffffu, hv[0], 1);
#pragma unroll
                for (int j = 0; j < kP; ++j) {
                    hl[j] = j == 0 ? left : hv[j - 1];
                    hr[j] = j == kP - 1 ? right : hv[j + 1];
                }
            } else {
                // left of (lane, j) is (lane - 1, j), or (31, j - 1) on lane 0;
                // right is (lane + 1, j), or (0, j + 1) on lane 31
                const int lu = (lane + 31) & 31, ld = (lane + 1) & 31;
                float up[kP], dn[kP];
#pragma unroll
                for (int j = 0; j < kP; ++j) {
                    up[j] = __shfl_sync(0xffffffffu, hv[j], lu);
                    dn[j] = __shfl_sync(0xffffffffu, hv[j], ld);
                }
                const bool first = lane == 0, last = lane == 31;
#pragma unroll
                for (int j = 0; j < kP; ++j) {
                    hl[j] = (j > 0 && first) ? up[j - 1] : up[j];
                    hr[j] = (j < kP - 1 && last) ? dn[j + 1] : dn[j];
                }
            }
            // 3. this step's states
            const bool start = (starts >> w) & 1u;
            float uh[kP];
#pragma unroll
            for (int k = 0; k < kNP; ++k) {
                h[k] = ptx::sel64(start, Wt[k].lx,
                                  pair_state(Wt[k], ptx::pk(hl[2 * k], hl[2 * k + 1]), h[k],
                                             ptx::pk(hr[2 * k], hr[2 * k + 1])));
                ptx::upk(ptx::mul2(Wt[k].u, h[k]), uh[2 * k], uh[2 * k + 1]);
                Wt[k] = Wn[k];
            }
            if constexpr (VERT) {
                const int row = FWD ? s : L - 1 - s;
                float* const dst = slot + (size_t)row * W + a[0];
                if constexpr (kP == 4)
                    ptx::red_add_v4_f32_if(own[0] && s < L, dst, uh[0], uh[1], uh[2], uh[3],
                                           pol_acc);
                else
                    ptx::red_add_v2_f32_if(own[0] && s < L, dst, uh[0], uh[1], pol_acc);
            } else {
                // acc[j][0] holds columns c0, c0 + 1, acc[j][1] columns c0 + 2, c0 + 3
                constexpr int kc = FWD ? (w & 3) : 3 - (w & 3);
#pragma unroll
                for (int j = 0; j < kP; ++j) {
                    float x0, x1;
                    ptx::upk(acc[j][kc >> 1], x0, x1);
                    acc[j][kc >> 1] = (kc & 1) ? ptx::pk(x0, uh[j]) : ptx::pk(uh[j], x1);
                }
                if constexpr ((w & 3) == 3) {
                    // The last stage may run past the line (W a multiple of 4,
                    // not of the stage): such groups of 4 steps are not added.
                    const bool in = s < L;
                    const int c0 = in ? (FWD ? s - 3 : L - 1 - s) : 0;
#pragma unroll
                    for (int j = 0; j < kP; ++j) {
                        float x0, x1, x2, x3;
                        ptx::upk(acc[j][0], x0, x1);
                        ptx::upk(acc[j][1], x2, x3);
                        ptx::red_add_v4_f32_if(own[j] && in,
                                               slot + (size_t)(own[j] ? a[j] : 0) * W + c0, x0, x1,
                                               x2, x3, pol_acc);
                    }
                }
            }
            // 4. end of an epoch: refresh halos (CTA every kXHalo steps, warps every kEpoch)
            if constexpr ((w % kEpoch) == kEpoch - 1) {
                if (s + 1 < L) {
                    float v[kP];
#pragma unroll
                    for (int k = 0; k < kNP; ++k) ptx::upk(h[k], v[2 * k], v[2 * k + 1]);
                    if (So > 1 && (s + 1) % kXHalo == 0)
                        cta_refresh(p, sm, ph, v, a, core, own0, Kc, So, sr, rank0, s, L);
                    warp_refresh<VERT>(sm, v, epoch, warp, lane, nw, nthr);
#pragma unroll
                    for (int k = 0; k < kNP; ++k) h[k] = ptx::pk(v[2 * k], v[2 * k + 1]);
                    ++epoch;
                }
            }
        });
        // the stage has been read completely (vertical reads of it ended two
        // steps ago; horizontal chunks are in registers)
        release(cur_sl);
        cur_sl = nxt_sl;
    }
    // After an abort, halo stores of the neighbours may still be in flight to
    // this CTA: give the phases it stopped waiting for a short bounded wait
    // before the CTA reuses (or releases) its shared memory.
    if (So > 1 && t == 0 && ph.abort) {
        for (int par = 0; par < 2; ++par)
            ptx::wait_parity_bounded(sm.halo + 8u * par, (ph.halo >> par) & 1u, 2000000ull);
    }
}

template <class T, bool kRefine, bool VERT, bool FWD>
__device__ __forceinline__ void run_chain(const SweepParams& p, const View& sm, Phases& ph,
                                          ProducerState& ps, int q, int d, int sr, int So,
                                          int rank0, uint64_t pol_acc) {
    const int o = VERT ? 0 : 1;
    const int ws = sr * p.Kc[o] - (sr > 0 ? kXHalo : kEdge);
    const int warp = threadIdx.x >> 5;
    if (warp == p.nw)
        produce<T, VERT, FWD>(p, sm, ps, q, d, ws);
    else if (warp < p.nw)
        consume<T, kRefine, VERT, FWD>(p, sm, ph, q, sr, So, rank0, ws, pol_acc);
    __syncthreads();
}

// Rounds the finished slot of plane q to the output dtype, writes y, re-zeroes
// the slot.  CTA `rank` of the team takes a contiguous 1/S share; every thread
// keeps kUnroll 16-byte loads in flight.
template <class T>
__device__ __forceinline__ void convert_plane(const SweepParams& p, int q, int rank) {
    constexpr int kUnroll = 8;
    const size_t HW = (size_t)p.H * p.W;
    float4* slot = reinterpret_cast<float4*>(p.slots + (size_t)(q % p.n_slots) * HW);
    T* yq = static_cast<T*>(p.y) + (size_t)q * HW;
    const size_t nvec = HW / 4;  // HW is a multiple of 4 (W * sizeof(T) % 16 == 0)
    const size_t per = (nvec + p.S - 1) / p.S;
    const size_t v0 = per * rank, v1 = min(nvec, v0 + per);
    const size_t stride = blockDim.x;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (size_t base = v0 + threadIdx.x; base < v1; base += kUnroll * stride) {
        float4 r[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            const size_t v = base + j * stride;
            if (v < v1) r[j] = __ldcg(slot + v);
        }
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            const size_t v = base + j * stride;
            if (v >= v1) continue;
            __stcg(slot + v, zero);
            if constexpr (sizeof(T) == 4) {
                __stcs(reinterpret_cast<float4*>(yq) + v, r[j]);
            } else {
                __nv_bfloat162 lo = __floats2bfloat162_rn(r[j].x, r[j].y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(r[j].z, r[j].w);
                uint2 packed;
                packed.x = *reinterpret_cast<uint32_t*>(&lo);
                packed.y = *reinterpret_cast<uint32_t*>(&hi);
                __stcs(reinterpret_cast<uint2*>(yq) + v, packed);
            }
        }
    }
}

__device__ __forceinline__ void team_sync(int S) {
    if (S > 1)
        ptx::cluster_sync();
    else
        __syncthreads();
}

// Leader writes `v` into cell `c` of every CTA of the team.
__device__ __forceinline__ void team_broadcast(const View& sm, int S, int c, int v) {
    if (S > 1) {
        for (int r = 0; r < S; ++r)
            ptx::st_cluster_s32(ptx::map_shared(ptx::smem_addr(sm.cell + c), r), v);
    } else {
        sm.cell[c] = v;
    }
}

template <class T, bool kRefine>
__global__ void __launch_bounds__(32 * (kMaxWarps + 1), 1)
    sweep_kernel(const __grid_constant__ SweepParams p) {
    extern __shared__ __align__(128) char smem_raw[];
    // TMA destinations sit on 1024-byte boundaries
    char* const base = smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u);
    const View sm = carve(base, p);
    const int rank = p.S > 1 ? (int)ptx::cluster_ctarank() : 0;
    const int t = threadIdx.x;

    if (t == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            ptx::mbar_init(sm.full + 8u * s, 1);
            ptx::mbar_init(sm.empty + 8u * s, (uint32_t)p.nw);
        }
        for (int s = 0; s < 2; ++s) ptx::mbar_init(sm.halo + 8u * s, 1);
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&p.tm_xv);
        ptx::prefetch_tensormap(&p.tm_xh);
    }
    team_sync(p.S);

    const uint64_t pol_acc = ptx::policy_evict_last();
    Phases ph{0u, 0u, false};
    ProducerState ps{0u, 0u, 0u, false};

    while (true) {
        if (rank == 0 && t == 0) {
            int it = -1;
            if (ptx::ld_acquire_gpu(&p.ctrl->sticky_error) != 0) {
                // a previous launch aborted: its slots may be dirty
                atomicCAS(&p.ctrl->call_error, 0, 4);
            } else if (ptx::ld_acquire_gpu(&p.ctrl->call_error) == 0) {
                it = atomicAdd(&p.ctrl->next_item, 1);
                if (it >= p.n_items) {
                    it = -1;
                } else {
                    const int q = it / p.ipp;
                    const int s = q % p.n_slots;
                    const int want = q / p.n_slots + (p.force_stale ? 1000000 : 0);
                    if (ptx::ld_acquire_gpu(&p.ctrl->slot_epoch[s]) != want) {
                        const uint64_t t0 = ptx::global_timer_ns();
                        while (ptx::ld_acquire_gpu(&p.ctrl->slot_epoch[s]) != want) {
                            if (ptx::ld_acquire_gpu(&p.ctrl->call_error) != 0 ||
                                ptx::global_timer_ns() - t0 > p.timeout_ns) {
                                report_error(p.ctrl, 2);
                                it = -1;
                                break;
                            }
                            __nanosleep(256);
                        }
                    }
                }
            }
            team_broadcast(sm, p.S, 0, it);
        }
        team_sync(p.S);
        const int it = sm.cell[0];
        if (it < 0) break;
        const int q = it / p.ipp;
        const int k = it % p.ipp;
        const bool vert = p.item_dir[k][0] < 2;
        const int So = p.So[vert ? 0 : 1];
        const int sub = rank / So, sr = rank % So;
        const int d = sub < 2 ? p.item_dir[k][sub] : -1;
        const int rank0 = sub * So;
        if (d == 0)
            run_chain<T, kRefine, true, true>(p, sm, ph, ps, q, d, sr, So, rank0, pol_acc);
        else if (d == 1)
            run_chain<T, kRefine, true, false>(p, sm, ph, ps, q, d, sr, So, rank0, pol_acc);
        else if (d == 2)
            run_chain<T, kRefine, false, true>(p, sm, ph, ps, q, d, sr, So, rank0, pol_acc);
        else if (d == 3)
            run_chain<T, kRefine, false, false>(p, sm, ph, ps, q, d, sr, So, rank0, pol_acc);

        // Publish this item, decide whether this team closes the plane.
        __threadfence();
        team_sync(p.S);
        if (rank == 0 && t == 0) {
            const int old = ptx::atom_add_acq_rel_gpu(p.plane_done + q, 1);
            team_broadcast(sm, p.S, 1, (old == p.ipp - 1) ? 1 : 0);
        }
        team_sync(p.S);
        if (sm.cell[1]) {
            convert_plane<T>(p, q, rank);
            __threadfence();
            team_sync(p.S);
            if (rank == 0 && t == 0)
                ptx::st_release_gpu(&p.ctrl->slot_epoch[q % p.n_slots], q / p.n_slots + 1);
        }
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult qr;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool encode_map(CUtensorMap* m, const void* ptr, int dtype, int W, int H, int64_t depth, int box_x,
                int box_y, bool swizzle32) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const size_t es = dtype == 0 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)depth};
    cuuint64_t strides[2] = {(cuuint64_t)(W * es), (cuuint64_t)((size_t)H * W * es)};
    cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)box_y, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     3, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int round_up(int a, int b) { return (a + b - 1) / b * b; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }

template <class T, bool kRefine>
cudaError_t set_attributes(const SweepPlan& sp) {
    auto kernel = sweep_kernel<T, kRefine>;
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.smem);
    if (e == cudaSuccess && sp.S > 1)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

void fill_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, const SweepPlan& sp,
                 int clusters, cudaStream_t stream) {
    memset(cfg, 0, sizeof(*cfg));
    cfg->gridDim = dim3(clusters * sp.S, 1, 1);
    cfg->blockDim = dim3(sp.threads, 1, 1);
    cfg->dynamicSmemBytes = sp.smem;
    cfg->stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = sp.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg->attrs = attr;
    cfg->numAttrs = 1;
}

template <class T, bool kRefine>
int max_teams(const SweepPlan& sp) {
    if (set_attributes<T, kRefine>(sp) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    fill_config(&cfg, attr, sp, 1, 0);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, sweep_kernel<T, kRefine>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

template <class T, bool kRefine>
cudaError_t launch_typed(Problem& pb, const SweepPlan& sp, void* ws) {
    cudaError_t e = set_attributes<T, kRefine>(sp);
    if (e != cudaSuccess) return e;
    const int H = (int)pb.H, W = (int)pb.W;
    constexpr int J = 32 / (int)sizeof(T);  // steps per stage: 32-byte row segments
    SweepParams prm;
    memset(&prm, 0, sizeof(prm));
    const int64_t planes = pb.planes();
    if (!encode_map(&prm.tm_xv, pb.x, pb.dtype, W, H, planes, sp.bw[0], J, false) ||
        !encode_map(&prm.tm_xh, pb.x, pb.dtype, W, H, planes, J, sp.bw[1], true))
        return cudaErrorInvalidValue;
    for (int d = pb.d0; d < pb.d1; ++d) {
        const bool vert = d < 2;
        const int bx = vert ? sp.bw[0] : J;
        const int by = vert ? J : sp.bw[1];
        if (!encode_map(&prm.tm_z[d], pb.z.p[d], pb.dtype, W, H, 3 * (planes / pb.z_div), bx, by,
                        !vert) ||
            !encode_map(&prm.tm_l[d], pb.lam.p[d], pb.dtype, W, H, planes, bx, by, !vert) ||
            !encode_map(&prm.tm_u[d], pb.u.p[d], pb.dtype, W, H, planes, bx, by, !vert))
            return cudaErrorInvalidValue;
    }
    char* base = static_cast<char*>(ws);
    prm.y = pb.y;
    prm.ctrl = reinterpret_cast<SweepCtrl*>(base);
    prm.plane_done = reinterpret_cast<int*>(base + sizeof(SweepCtrl));
    prm.slots = reinterpret_cast<float*>(base + sp.ctrl_bytes);
    prm.timeout_ns = sp.timeout_ns;
    prm.H = H;
    prm.W = W;
    prm.planes = (int)planes;
    prm.g = (int)pb.g;
    prm.S = sp.S;
    for (int o = 0; o < 2; ++o) {
        prm.So[o] = sp.So[o];
        prm.Kc[o] = sp.Kc[o];
        prm.nb[o] = sp.nb[o];
        prm.bw[o] = sp.bw[o];
    }
    prm.nw = sp.nw;
    prm.tile_bytes = sp.tile_bytes;
    prm.stages = sp.stages;
    prm.z_div = (int)pb.z_div;
    prm.n_slots = sp.n_slots;
    prm.ipp = sp.ipp;
    for (int k = 0; k < kMaxItems; ++k) {
        prm.item_dir[k][0] = sp.item_dir[k][0];
        prm.item_dir[k][1] = sp.item_dir[k][1];
    }
    prm.n_items = (int)(planes * sp.ipp);
    prm.force_stale = sp.force_stale;

    // Reset the per-call part of the control block (not the sticky error).
    e = cudaMemsetAsync(base + kCtrlResetOffset, 0, sp.ctrl_bytes - kCtrlResetOffset, pb.stream);
    if (e != cudaSuccess) return e;
    if (sp.zero_slots) {
        e = cudaMemsetAsync(prm.slots, 0, sp.slot_bytes * sp.n_slots, pb.stream);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    fill_config(&cfg, attr, sp, sp.n_teams, pb.stream);
    if (pb.ev_begin) cudaEventRecord(pb.ev_begin, pb.stream);
    e = cudaLaunchKernelEx(&cfg, sweep_kernel<T, kRefine>, prm);
    if (pb.ev_end) cudaEventRecord(pb.ev_end, pb.stream);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Window of a chain rank: margins kEdge at the ends of the line, kXHalo
// towards a neighbouring CTA; warps needed to cover it.
int window_span(int So, int Kc) {
    int span = 0;
    for (int sr = 0; sr < So; ++sr) {
        const int left = sr > 0 ? kXHalo : kEdge;
        const int right = sr < So - 1 ? kXHalo : kEdge;
        if (left + Kc + right > span) span = left + Kc + right;
    }
    return span;
}

}  // namespace

size_t sweep_ctrl_bytes(int64_t planes) {
    return ((sizeof(SweepCtrl) + sizeof(int) * (size_t)planes) + 255) & ~(size_t)255;
}

bool sweep_plan(const Problem& pb, SweepPlan* sp) {
    const int es = pb.dtype == 0 ? 4 : 2;
    if (pb.H > 0x7fffffff / pb.W) return false;
    // 16-byte rows (TMA strides, whole 4-step output groups); a horizontal
    // stage (32 bytes of columns) may run past W on zero-filled columns
    if ((pb.W * es) % 16 != 0) return false;
    if (pb.planes() * 3 > 0x7fffffffLL) return false;
    if (pb.H < 2 * kP || pb.W < 2 * kP) return false;
    const int H = (int)pb.H, W = (int)pb.W;
    const int K[2] = {W, H};

    // Items: the directions of one orientation run together on one team when
    // a chain of that orientation needs only half of the team's CTAs.
    int dirs[2][2], nd[2] = {0, 0};
    for (int d = pb.d0; d < pb.d1; ++d) dirs[d < 2 ? 0 : 1][nd[d < 2 ? 0 : 1]++] = d;

    const size_t slot_bytes = sizeof(float) * (size_t)H * W;
    const size_t l2_budget = (size_t)96 << 20;
    {
        const int kc_max = kMaxOwned;
        SweepPlan plan;
        memset(&plan, 0, sizeof(plan));
        int So[2];
        bool ok = true;
        for (int o = 0; o < 2; ++o) {
            So[o] = 1;
            while (So[o] <= 8 && round_up(ceil_div(K[o], So[o]), 8) > kc_max) So[o] *= 2;
            if (So[o] > 8) ok = false;
        }
        if (!ok) return false;
        int S = 1;
        for (int o = 0; o < 2; ++o)
            if (nd[o] > 0 && So[o] > S) S = So[o];
        // a team runs one chain per item, or two when a chain needs half of it
        for (int o = 0; o < 2; ++o)
            if (So[o] < S / 2 || nd[o] == 0) So[o] = S > 1 ? S / 2 : 1;
        plan.S = S;
        int span = 0;  // window positions that must be exact (margins + owned)
        for (int o = 0; o < 2; ++o) {
            plan.So[o] = So[o];
            plan.Kc[o] = round_up(ceil_div(K[o], So[o]), 8);
            if (nd[o] == 0) continue;
            // a CTA sends its first and last kXHalo owned positions to its
            // neighbours: it must own at least that many
            if (So[o] > 1 && plan.Kc[o] < kXHalo) ok = false;
            const int sp_o = window_span(So[o], plan.Kc[o]);
            if (sp_o > span) span = sp_o;
        }
        const int nw = ceil_div(span - 2 * kP, kStride);
        if (!ok || nw > kMaxWarps) return false;
        plan.nw = nw;
        plan.threads = 32 * (nw + 1);
        // A stage holds the exact span (rounded to 32 positions, so that every
        // box is a whole number of KB) in at most 256-position boxes of 32
        // bytes of steps per position; lanes past it read its last positions.
        const int tile_pos = round_up(span, 32);
        for (int o = 0; o < 2; ++o) {
            plan.nb[o] = ceil_div(tile_pos, 256);
            plan.bw[o] = round_up(ceil_div(tile_pos, plan.nb[o]), 32);
            if (plan.bw[o] > 256) return false;
        }
        plan.tile_bytes = plan.nb[0] * plan.bw[0] * 32;
        plan.stages = 0;
        for (int st = kMaxStages; st >= 2; --st) {
            size_t a, b, c;
            const size_t need = smem_bytes_for(plan.tile_bytes, st, &a, &b, &c) + 1024;
            if (need <= 227 * 1024) {
                plan.stages = st;
                plan.smem = need;
                break;
            }
        }
        if (plan.stages == 0) return false;
        // work items of one plane
        int ipp = 0;
        for (int o = 0; o < 2; ++o) {
            const int per = S / So[o];  // chains of orientation o per item (1 or 2)
            for (int i = 0; i < nd[o]; i += per) {
                plan.item_dir[ipp][0] = dirs[o][i];
                plan.item_dir[ipp][1] = (per == 2 && i + 1 < nd[o]) ? dirs[o][i + 1] : -1;
                ++ipp;
            }
        }
        plan.ipp = ipp;
        int teams = pb.dtype == 0 ? max_teams<float, true>(plan)
                                  : max_teams<__nv_bfloat16, false>(plan);
        if (teams <= 0) return false;
        const int64_t items = pb.planes() * ipp;
        if (teams > items) teams = (int)items;
        const int64_t want_slots = (teams + ipp - 1) / ipp + 2;
        int64_t cap = (int64_t)(l2_budget / slot_bytes);
        if (cap < 1) cap = 1;
        int64_t slots = want_slots < cap ? want_slots : cap;
        if (slots > kMaxSlots) slots = kMaxSlots;
        if (slots > pb.planes()) slots = pb.planes();
        plan.n_teams = teams;
        plan.n_slots = (int)slots;
        plan.slot_bytes = slot_bytes;
        plan.ctrl_bytes = sweep_ctrl_bytes(pb.planes());
        plan.ws_bytes = plan.ctrl_bytes + slot_bytes * (size_t)slots;
        plan.timeout_ns = 4000000000ull;
        plan.zero_slots = false;
        plan.force_stale = 0;
        *sp = plan;
        return true;
    }
    return false;
}

cudaError_t launch_sweep(Problem& pb, const SweepPlan& sp, void* ws, int* launches) {
    pb.kernel_name = "sweep_kernel";
    if (getenv("GSPN_DEBUG_PLAN"))
        fprintf(stderr,
                "gspn sweep plan: S=%d So=%d,%d Kc=%d,%d nw=%d nb=%d,%d bw=%d,%d tile=%d "
                "stages=%d smem=%zu teams=%d slots=%d ipp=%d\n",
                sp.S, sp.So[0], sp.So[1], sp.Kc[0], sp.Kc[1], sp.nw, sp.nb[0], sp.nb[1], sp.bw[0],
                sp.bw[1], sp.tile_bytes, sp.stages, sp.smem, sp.n_teams, sp.n_slots, sp.ipp);
    cudaError_t e = pb.dtype == 0 ? launch_typed<float, true>(pb, sp, ws)
                                  : launch_typed<__nv_bfloat16, false>(pb, sp, ws);
    if (e == cudaSuccess) *launches += 1;
    return e;
}

}  // namespace gspn
