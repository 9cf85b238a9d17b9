// Fused persistent GSPN kernel for large planes (sm_100a).
//
// What it computes: for every (b, c) plane and direction d, the line recurrence
//   h_i = w_i h_{i-1} + lambda_i (.) x_i,   h = lambda (.) x on a group's first line
// with three-neighbour row-stochastic weights (sigmoid, then normalisation over
// the existing neighbours), and y = sum_d u_d (.) h_d -- CSDN walkthrough
// "GSPN——在convolution基础上并行序列建模", sections "方法", "如何设计一个高效的
// 传播层", "行随机矩阵" and "全局与局部GSPN".
//
// How (B200 design):
//  * Work item = one (plane, direction) chain.  A team of S CTAs (one thread
//    block cluster, one CTA per SM) runs a chain; CTA j owns positions
//    [j*Kc, (j+1)*Kc) of the line and also recomputes a halo of kHalo positions
//    on each side.  A halo value stays exact for kHalo steps after a refresh,
//    so neighbouring CTAs exchange their edge states only every kHalo steps,
//    through DSMEM `st.async` stores that complete transaction bytes on the
//    receiver's mbarrier.
//  * Each consumer thread owns one position.  The previous line lives in a
//    double-buffered shared-memory line; one named barrier over the consumer
//    warps separates two steps.  The weights are software-pipelined: in the
//    interval between two barriers a thread finishes step i, completes the
//    products and reciprocal of step i+1 and issues the exponentials of step
//    i+2, so the dependent chain between barriers stays short.
//  * Inputs stream through a 2-3 stage shared-memory ring filled by TMA tensor
//    loads (no multicast) from a dedicated producer warp.  A stage is one
//    32-byte segment of steps (16 bf16 or 8 fp32 lines): vertical scans load
//    that many rows x (Kc + 2*kHalo) columns; horizontal scans load
//    (Kc + 2*kHalo) rows x 32 bytes, and each thread copies its row segment
//    to registers 16 bytes at a time, so the scan runs along W with no
//    transposition.  The stage loop is unrolled at compile time and a halo
//    block (32 steps) is a whole number of stages, so the exchange runs
//    between stages.  Warps with no border position run a variant without
//    border selects.
//  * The four chains of a plane accumulate u_d * h_d into an fp32 "slot" kept
//    L2-resident (evict_last reductions; streaming inputs use evict_first).
//    The team that finishes a plane's last chain rounds the slot to the output
//    dtype once, writes y, re-zeroes the slot and releases it.  A ring of
//    n_slots slots bounds the L2 footprint; teams take items from a global
//    queue in plane-major order, so every plane a team waits for has already
//    been handed to running teams (no deadlock).
//  * Every wait (TMA stage, halo, slot release) is bounded by a global-timer
//    limit; on expiry the kernel records an error word and winds down.
//
// Weights: with a_o = 1 + exp(-z_o), w_o = prod_{o' != o} a_o' / sum_o prod_{o'
// != o} a_o' over the existing neighbours (3 exponentials + 1 reciprocal per
// pixel).  Every a_o is computed scaled by 2^-32, which cancels in the ratio and
// keeps the products finite unless two neighbour logits of one pixel sum to
// less than about -133.
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

constexpr int kMaxStages = 3;
constexpr int kMaxSlots = 64;
constexpr int kHalo = 32;        // halo width == steps between exchanges
constexpr int kMaxThreads = 320; // two positions per consumer thread + one producer warp

// Control block in global memory (the first bytes of the fused workspace).
struct FusedCtrl {
    int sticky_error;  // kept across calls until the host reads it
    int pad0[3];
    int call_error;    // this call: nonzero stops every team (1 TMA, 2 slot, 3 halo, 4 stale)
    int next_item;
    int pad1[10];
    int slot_epoch[kMaxSlots];
    // int plane_done[planes] follows
};
constexpr size_t kCtrlResetOffset = 16;  // bytes before this survive the per-call reset

struct __align__(64) FusedParams {
    CUtensorMap tm_xv;     // x with vertical boxes
    CUtensorMap tm_xh;     // x with horizontal boxes
    CUtensorMap tm_z[4];   // logits of direction d (boxes of d's orientation)
    CUtensorMap tm_l[4];
    CUtensorMap tm_u[4];
    void* y;
    float* slots;
    FusedCtrl* ctrl;
    int* plane_done;
    unsigned long long timeout_ns;
    int H, W, planes, g;
    int d0, nd;            // directions [d0, d0 + nd)
    int S;                 // team size (CTAs per cluster)
    int Kc_v, Kc_h;        // owned positions per CTA (vertical / horizontal scans)
    int np_v, np_h;        // positions handled per CTA (owned + halos)
    int nb_v;              // vertical: 64-column boxes per stage (one per consumer warp)
    int nb_h, bh_h;        // horizontal: row boxes, box height (multiple of 8)
    int tile_bytes;        // one tensor's tile in one stage
    int stages;            // depth of the shared-memory ring (2 or 3)
    int z_div;             // logits of plane q are logit plane q / z_div
    int n_slots;
    int n_items;
    int force_stale;       // test hook: expect a slot epoch that never comes
};

// Shared-memory carve-up (dynamic shared memory).
struct SmemView {
    char* ring;
    float* hb;   // 2 lines of (np_max + 4) floats; position p at index p + 2
    float* rx;   // [2 parity][2 side][kHalo]
    uint64_t* full_bar;   // [stages] TMA completion (expect_tx by the producer warp)
    uint64_t* empty_bar;  // [stages] slot released by the consumers (one arrival)
    uint64_t* halo_bar;   // [2] halo data arrived from the neighbour CTAs
    int* cell;   // [0] item, [1] convert decision, [2] full phases, [3] halo phases
    int line;    // floats per line buffer
    int tile_bytes;
    __device__ char* tile(int stage, int tensor) const {
        return ring + (size_t)(stage * 6 + tensor) * tile_bytes;
    }
};

__host__ __device__ inline size_t smem_layout(int tile_bytes, int stages, int npmax,
                                              size_t* off_hb, size_t* off_rx, size_t* off_bar) {
    size_t off = (size_t)stages * 6 * tile_bytes;
    *off_hb = off;
    off += sizeof(float) * 2 * (size_t)(npmax + 4);
    *off_rx = off;
    off += sizeof(float) * 2 * 2 * kHalo;
    off = (off + 7) & ~(size_t)7;
    *off_bar = off;
    off += sizeof(uint64_t) * (2 * kMaxStages + 2) + 4 * sizeof(int);
    return off;
}

__device__ __forceinline__ SmemView carve(char* base, const FusedParams& p) {
    const int npmax = p.np_v > p.np_h ? p.np_v : p.np_h;
    size_t ohb, orx, obar;
    smem_layout(p.tile_bytes, p.stages, npmax, &ohb, &orx, &obar);
    SmemView v;
    v.tile_bytes = p.tile_bytes;
    v.ring = base;
    v.line = npmax + 4;
    v.hb = reinterpret_cast<float*>(base + ohb);
    v.rx = reinterpret_cast<float*>(base + orx);
    v.full_bar = reinterpret_cast<uint64_t*>(base + obar);
    v.empty_bar = v.full_bar + kMaxStages;
    v.halo_bar = v.empty_bar + kMaxStages;
    v.cell = reinterpret_cast<int*>(v.halo_bar + 2);
    return v;
}

// Calls f(std::integral_constant<int, I>{}) for I = 0..N-1 (compile-time indices).
template <class F, int... Is>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, Is...>) {
    (f(std::integral_constant<int, Is>{}), ...);
}
template <int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

// Per-thread view of the mbarrier phases (identical in every active thread;
// thread 0 publishes them in shared memory between chains).
struct Phases {
    uint32_t full;  // bit s: parity to wait for on full_bar[s]
    uint32_t halo;  // bit p: parity to wait for on halo_bar[p]
    bool abort;     // a bounded wait expired: skip further waits
};

__device__ __forceinline__ void report_error(const FusedParams& p, int code) {
    atomicCAS(&p.ctrl->call_error, 0, code);
    atomicCAS(&p.ctrl->sticky_error, 0, code);
}

__device__ __forceinline__ void wait_bar(const FusedParams& p, Phases& ph, uint64_t* bar,
                                         uint32_t parity, int code) {
    if (ph.abort) return;
    if (!ptx::wait_parity_bounded(ptx::smem_addr(bar), parity, p.timeout_ns)) {
        ph.abort = true;
        report_error(p, code);
    }
}

// What a chain's consumer loop needs from the launch parameters and the
// shared-memory carve-up, as plain values.  The consumer copies them once so
// that no parameter is re-read after each shared-memory access.
struct ChainEnv {
    uint32_t full_s, empty_s, halo_s, rx_s;  // shared addresses of the barriers and halo buffer
    unsigned long long timeout_ns;
    FusedCtrl* ctrl;
    int S;
};

__device__ __forceinline__ void wait_env(const ChainEnv& env, Phases& ph, uint32_t bar,
                                         uint32_t parity, int code) {
    if (ph.abort) return;
    if (!ptx::wait_parity_bounded(bar, parity, env.timeout_ns)) {
        ph.abort = true;
        atomicCAS(&env.ctrl->call_error, 0, code);
        atomicCAS(&env.ctrl->sticky_error, 0, code);
    }
}

// Element e of a 16-byte vector of bf16 (e < 8) or fp32 (e < 4); e folds to a
// constant inside fully unrolled loops.
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

// Thread 0 arms halo barrier (blk & 1) for block blk if that block ends in an
// exchange (block blk covers steps [blk*kHalo, (blk+1)*kHalo) and exchanges
// after its last step when more steps follow).  Blocks 0 and 1 are armed at
// chain start; block b+2 right after block b's exchange completed on this CTA,
// which is before any neighbour can send block b+2's data.
__device__ __forceinline__ void arm_halo_block(const FusedParams& p, const SmemView& sm, int rank,
                                               int blk, int L) {
    if ((blk + 1) * kHalo < L) {
        const uint32_t bytes =
            sizeof(float) * kHalo * ((rank > 0 ? 1 : 0) + (rank < p.S - 1 ? 1 : 0));
        ptx::mbar_arrive_expect_tx(ptx::smem_addr(sm.halo_bar + (blk & 1)), bytes);
    }
}

__device__ __forceinline__ void arm_halo_env(const ChainEnv& env, int rank, int blk, int L) {
    if ((blk + 1) * kHalo < L) {
        const uint32_t bytes =
            sizeof(float) * kHalo * ((rank > 0 ? 1 : 0) + (rank < env.S - 1 ? 1 : 0));
        ptx::mbar_arrive_expect_tx(env.halo_s + 8u * (blk & 1), bytes);
    }
}

// First step > 0 at which a local group restarts (INT_MAX if none); later
// restarts follow every g steps.
__device__ __forceinline__ int first_restart(int g, int L, bool fwd) {
    if (g <= 0) return 0x7fffffff;
    return fwd ? g : ((L - 1) % g) + 1;
}

// ------------------------------------------------------------------ pair math
// A consumer thread owns two positions of the line; their values travel as
// packed fp32 pairs.  A step's weights are computed in two pipelined halves,
// each in a different barrier interval, so that no instruction of an interval
// waits for an exponential or a reciprocal issued in the same interval:
//   begin:    e_o = 2^-32 exp(-z_o) for the three neighbours, lambda*x, u
//   complete: a_o = e_o + 2^-32, p_o = product of the other two a's (0 for a
//             missing neighbour), r = 1 / (p_0 + p_1 + p_2)
// so that h = (p_0 h_left + p_1 h_self + p_2 h_right) r + lambda*x.
struct PairA {
    f2 e0, e1, e2, lx, u;  // exp(-z_o) * 2^-32 (0 for a missing neighbour), lambda*x, u
};
struct PairW {
    f2 p0, p1, p2, r, lx, u;
};
// Border handling without branches.  A neighbour outside the plane is
// dropped: its a is the neutral scaled 1 and its product is 0.  Per thread
// and half, m_lo / m_hi are 1 where the neighbour at offset -1 / +1 exists and
// 0 where it does not; the exponent of a missing neighbour is forced to -inf
// (ex2 gives 0, so a = 2^-32 exactly and no overflow can reach the masks).
// Positions outside the plane need no forcing: their inputs are the zeros
// the tensor maps fill in, their neighbours give them zero weight, and their
// results are never accumulated.
struct PairMask {
    f2 m_lo, m_hi;        // 1 / 0
    f2 kl_lo, ko_lo;      // exponent coefficients of slot 0: (-log2 e, -32) or (0, -inf)
    f2 kl_hi, ko_hi;      // ... of slot 2
};

constexpr float kScale = 2.3283064365386963e-10f;  // 2^-32
constexpr float kNegLog2e = -1.4426950408889634f;

__device__ __forceinline__ f2 splat(float v) { return ptx::pk(v, v); }
__device__ __forceinline__ float lo_of(f2 v) {
    float a, b;
    ptx::upk(v, a, b);
    return a;
}
__device__ __forceinline__ float hi_of(f2 v) {
    float a, b;
    ptx::upk(v, a, b);
    return b;
}
__device__ __forceinline__ f2 ex2_pair(f2 t) {
    float a, b;
    ptx::upk(t, a, b);
    return ptx::pk(ex2_approx(a), ex2_approx(b));
}

__device__ __forceinline__ PairMask make_mask(bool lo0, bool lo1, bool hi0, bool hi1) {
    const float ninf = __int_as_float(0xff800000);
    PairMask m;
    m.m_lo = ptx::pk(lo0 ? 1.0f : 0.0f, lo1 ? 1.0f : 0.0f);
    m.m_hi = ptx::pk(hi0 ? 1.0f : 0.0f, hi1 ? 1.0f : 0.0f);
    m.kl_lo = ptx::pk(lo0 ? kNegLog2e : 0.0f, lo1 ? kNegLog2e : 0.0f);
    m.ko_lo = ptx::pk(lo0 ? -32.0f : ninf, lo1 ? -32.0f : ninf);
    m.kl_hi = ptx::pk(hi0 ? kNegLog2e : 0.0f, hi1 ? kNegLog2e : 0.0f);
    m.ko_hi = ptx::pk(hi0 ? -32.0f : ninf, hi1 ? -32.0f : ninf);
    return m;
}

__device__ __forceinline__ f2 bf16x2_pair(uint32_t w) {
    return ptx::pk(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// The six inputs of one step for this thread's pair.
struct PairIn {
    f2 x, z0, z1, z2, lam, u;
};

// The six inputs as loaded from a vertical tile: one 32-bit word (two bf16)
// or two floats per tensor; unpacked only when they are used.
template <class T>
struct RawIn {
    typename std::conditional<sizeof(T) == 4, uint2, uint32_t>::type v[6];
};
template <class T>
__device__ __forceinline__ PairIn unpack_raw(const RawIn<T>& r) {
    f2 q[6];
#pragma unroll
    for (int k6 = 0; k6 < 6; ++k6) {
        if constexpr (sizeof(T) == 4)
            q[k6] = ptx::pk(__uint_as_float(r.v[k6].x), __uint_as_float(r.v[k6].y));
        else
            q[k6] = bf16x2_pair(r.v[k6]);
    }
    PairIn in;
    in.x = q[0];
    in.z0 = q[1];
    in.z1 = q[2];
    in.z2 = q[3];
    in.lam = q[4];
    in.u = q[5];
    return in;
}

__device__ __forceinline__ PairA begin_pair(const PairIn& in, const PairMask& m) {
    const f2 kL = splat(kNegLog2e), kO = splat(-32.0f);
    PairA A;
    A.lx = ptx::mul2(in.lam, in.x);
    A.u = in.u;
    A.e0 = ex2_pair(ptx::fma2(in.z0, m.kl_lo, m.ko_lo));
    A.e1 = ex2_pair(ptx::fma2(in.z1, kL, kO));
    A.e2 = ex2_pair(ptx::fma2(in.z2, m.kl_hi, m.ko_hi));
    return A;
}

template <bool kRefine>
__device__ __forceinline__ PairW complete_pair(const PairA& A, const PairMask& m) {
    const f2 kS = splat(kScale);
    const f2 a0 = ptx::add2(A.e0, kS), a1 = ptx::add2(A.e1, kS), a2 = ptx::add2(A.e2, kS);
    PairW W;
    W.lx = A.lx;
    W.u = A.u;
    W.p0 = ptx::mul2(ptx::mul2(a1, a2), m.m_lo);
    W.p1 = ptx::mul2(a0, a2);
    W.p2 = ptx::mul2(ptx::mul2(a0, a1), m.m_hi);
    const f2 sum = ptx::add2(ptx::add2(W.p0, W.p1), W.p2);
    float s0, s1;
    ptx::upk(sum, s0, s1);
    W.r = ptx::pk(rcp_approx(s0), rcp_approx(s1));
    if (kRefine) {  // one Newton step: r += r (1 - s r)
        const f2 e = ptx::fma2(ptx::mul2(sum, splat(-1.0f)), W.r, splat(1.0f));
        W.r = ptx::fma2(W.r, e, W.r);
    }
    return W;
}

// h of the pair from the previous states of the left neighbours (hl), the
// positions themselves (hs) and the right neighbours (hr).
__device__ __forceinline__ f2 finish_pair(const PairW& W, f2 hl, f2 hs, f2 hr) {
    return ptx::fma2(ptx::fma2(W.p2, hr, ptx::fma2(W.p1, hs, ptx::mul2(W.p0, hl))), W.r, W.lx);
}


// Halo exchange after the last step of block blk.  Senders push their exact
// pair to a neighbour CTA; halo threads return the received pair (others
// return h unchanged).  Window position of this thread's pair: 2 * threadIdx.x.
__device__ __forceinline__ f2 halo_exchange(const ChainEnv& env, Phases& ph, int rank, int Kc,
                                            int blk, int L, f2 h) {
    const int t = threadIdx.x;
    const int pos = 2 * t;
    const int par = blk & 1;
    const uint32_t rx_side0 = env.rx_s + 4u * (par * 2 + 0) * kHalo;  // left halo of a CTA
    const uint32_t rx_side1 = env.rx_s + 4u * (par * 2 + 1) * kHalo;  // right halo of a CTA
    const uint32_t bar = env.halo_s + 8u * par;
    float a, b;
    ptx::upk(h, a, b);
    if (rank > 0 && pos >= kHalo && pos < 2 * kHalo)  // first owned -> left neighbour's right halo
        ptx::st_async_f32x2(ptx::map_shared(rx_side1 + 4u * (pos - kHalo), rank - 1), a, b,
                            ptx::map_shared(bar, rank - 1));
    if (rank < env.S - 1 && pos >= Kc && pos < Kc + kHalo)  // last owned -> right neighbour's left halo
        ptx::st_async_f32x2(ptx::map_shared(rx_side0 + 4u * (pos - Kc), rank + 1), a, b,
                            ptx::map_shared(bar, rank + 1));
    const bool recv_l = rank > 0 && pos < kHalo;
    const bool recv_r = rank < env.S - 1 && pos >= kHalo + Kc && pos < 2 * kHalo + Kc;
    if (recv_l || recv_r || t == 0) {
        wait_env(env, ph, bar, (ph.halo >> par) & 1u, 3);
        uint2 v = make_uint2(0u, 0u);
        if (recv_l) v = ptx::lds_v2(rx_side0 + 4u * pos);
        if (recv_r) v = ptx::lds_v2(rx_side1 + 4u * (pos - kHalo - Kc));
        if (recv_l || recv_r) h = ptx::pk(__uint_as_float(v.x), __uint_as_float(v.y));
    }
    if (t == 0) arm_halo_env(env, rank, blk + 2, L);
    ph.halo ^= 1u << par;
    return h;
}

// The same exchange for the horizontal thread mapping, where window position p
// is half p / nthr of thread p % nthr: the owned edges and the halos are whole
// low or high halves, so every sender or receiver moves one float.
__device__ __forceinline__ f2 halo_exchange_split(const ChainEnv& env, Phases& ph, int rank,
                                                  int Kc, int nthr, int blk, int L, f2 h) {
    const int t = threadIdx.x;
    const int par = blk & 1;
    const uint32_t rx_side0 = env.rx_s + 4u * (par * 2 + 0) * kHalo;  // left halo of a CTA
    const uint32_t rx_side1 = env.rx_s + 4u * (par * 2 + 1) * kHalo;  // right halo of a CTA
    const uint32_t bar = env.halo_s + 8u * par;
    float a, b;
    ptx::upk(h, a, b);
    const int pa = t, pb = t + nthr;  // window positions of the low and high halves
    if (rank > 0 && pa >= kHalo && pa < 2 * kHalo)  // first owned -> left neighbour's right halo
        ptx::st_async_f32(ptx::map_shared(rx_side1 + 4u * (pa - kHalo), rank - 1), a,
                          ptx::map_shared(bar, rank - 1));
    if (rank < env.S - 1 && pb >= Kc && pb < Kc + kHalo)  // last owned -> right neighbour's left halo
        ptx::st_async_f32(ptx::map_shared(rx_side0 + 4u * (pb - Kc), rank + 1), b,
                          ptx::map_shared(bar, rank + 1));
    const bool recv_l = rank > 0 && pa < kHalo;
    const bool recv_r = rank < env.S - 1 && pb >= kHalo + Kc && pb < 2 * kHalo + Kc;
    if (recv_l || recv_r || t == 0) {
        wait_env(env, ph, bar, (ph.halo >> par) & 1u, 3);
        if (recv_l) a = ptx::lds_f32(rx_side0 + 4u * pa);
        if (recv_r) b = ptx::lds_f32(rx_side1 + 4u * (pb - kHalo - Kc));
        h = ptx::pk(a, b);
    }
    if (t == 0) arm_halo_env(env, rank, blk + 2, L);
    ph.halo ^= 1u << par;
    return h;
}

// The producer warp (the warp after the consumer threads) issues the chain's
// stages into the ring.  It waits for a slot's release (empty barrier, one
// consumer arrival per use) before reusing it and never joins the consumers'
// per-step barrier, so the time a TMA instruction blocks its issuing warp is
// hidden from the recurrence.  Lane 0 sets the expected bytes; the boxes of a
// stage (6 tensors x nb boxes) are spread over the lanes.
struct ProducerState {
    uint32_t used;   // bit s: slot s has been filled before
    uint32_t phase;  // bit s: parity of the next release of slot s
    bool abort;
};

template <class BoxFn>
__device__ __forceinline__ void producer_run(const FusedParams& p, const SmemView& sm,
                                             ProducerState& ps, int nst, int nb,
                                             uint32_t stage_bytes, BoxFn&& box) {
    const int lane = threadIdx.x & 31;
    for (int st = 0; st < nst; ++st) {
        const int sl = st % p.stages;
        if (ps.used & (1u << sl)) {
            if (!ps.abort && !ptx::wait_parity_bounded(ptx::smem_addr(sm.empty_bar + sl),
                                                       (ps.phase >> sl) & 1u, p.timeout_ns)) {
                ps.abort = true;
                report_error(p, 6);
            }
            ps.phase ^= 1u << sl;
        }
        ps.used |= 1u << sl;
        const uint32_t bar = ptx::smem_addr(sm.full_bar + sl);
        if (lane == 0) ptx::mbar_arrive_expect_tx(bar, stage_bytes);
        __syncwarp();
        for (int b = lane; b < 6 * nb; b += 32) box(st, sl, b / nb, b % nb, bar);
        __syncwarp();
    }
}

__device__ __forceinline__ const CUtensorMap* tensor_map(const FusedParams& p,
                                                         const CUtensorMap* xmap, int d,
                                                         int tensor) {
    return tensor == 0 ? xmap : tensor <= 3 ? &p.tm_z[d] : tensor == 4 ? &p.tm_l[d] : &p.tm_u[d];
}
__device__ __forceinline__ int tensor_z(const FusedParams& p, int q, int tensor) {
    return tensor == 0 ? q : tensor <= 3 ? 3 * (q / p.z_div) + tensor - 1 : q;
}

// ------------------------------------------------------------------- one chain
// Runs one (plane, direction) chain segment on this CTA, two positions per
// consumer thread.  VERT: scan along H (positions are columns; a stage holds
// kSeg rows of 64-column boxes, one box per warp, read straight from the
// tile); otherwise scan along W (positions are rows; a stage holds each row's
// 32-byte segment, copied to registers 16 bytes at a time).  Every stage
// covers kSeg = 32 / sizeof(T) steps, so a halo block (32 steps) is a whole
// number of stages and the exchange runs between stages.  Horizontal chains
// need W to be a multiple of kSeg (every stage full); a vertical chain's last
// stage may run past the plane on zero-filled rows, whose results are not
// accumulated.
template <class T, bool kRefine, bool VERT, bool FWD>
__device__ __forceinline__ Phases chain_consume(const FusedParams& p, const SmemView& sm, Phases ph,
                                                int q, int rank, uint64_t pol_acc) {
    ChainEnv env;
    env.full_s = ptx::smem_addr(sm.full_bar);
    env.empty_s = ptx::smem_addr(sm.empty_bar);
    env.halo_s = ptx::smem_addr(sm.halo_bar);
    env.rx_s = ptx::smem_addr(sm.rx);
    env.timeout_ns = p.timeout_ns;
    env.ctrl = p.ctrl;
    env.S = p.S;
    constexpr int kSeg = 32 / sizeof(T);
    constexpr int kPer = kSeg / 2;                   // steps per 16-byte half segment
    constexpr uint32_t kRowB = 64u * sizeof(T);      // vertical box row pitch
    constexpr uint32_t kBoxB = kRowB * kSeg;         // vertical box bytes (2 KB)
    const int H = p.H, W = p.W;
    const int L = VERT ? H : W, K = VERT ? W : H;
    const int Kc = VERT ? p.Kc_v : p.Kc_h, np = VERT ? p.np_v : p.np_h;
    const int k0 = rank * Kc, kb = k0 - (p.S > 1 ? kHalo : 0);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int nthr = np >> 1;
    const int nst = (L + kSeg - 1) / kSeg;
    const int stages = p.stages, g_len = p.g;
    const bool multi = p.S > 1;

    // This thread's two positions: vertical k, k+1 (adjacent columns);
    // horizontal k, k + nthr (rows in the two halves of the window), so that a
    // warp's rows are consecutive and its neighbour pairs are the adjacent
    // entries of the line buffer.
    const int kA = VERT ? kb + 2 * t : kb + t;
    const int kB = VERT ? kA + 1 : kA + nthr;
    const bool ownA = kA >= k0 && kA < k0 + Kc && kA < K;
    const bool ownB = kB >= k0 && kB < k0 + Kc && kB < K;
    const PairMask fl = make_mask(kA != 0, kB != 0, kA != K - 1, kB != K - 1);

    const uint32_t ring_s = ptx::smem_addr(sm.ring);
    const uint32_t tb = p.tile_bytes;
    // vertical: the pair's bytes in its warp's 64-column box; horizontal: row
    // t of the row tile (32-byte rows, 16-byte halves swapped on every other
    // group of four rows by the map's 32-byte swizzle); row t + nthr follows
    // at 32 * nthr bytes with the same swizzle phase (nthr % 32 == 0)
    // vertical: a stage holds, per warp, the six tensors' 64-column boxes
    // back to back ([warp][tensor][row][64 columns]), so every input load of a
    // step is this base plus a compile-time offset
    const uint32_t col_byte =
        VERT ? warp * (6u * kBoxB) + lane * (2u * (uint32_t)sizeof(T)) : 32u * t;
    const uint32_t swz = VERT ? 0u : (uint32_t)((t >> 2) & 1);
    // line buffers: 8-byte entry e at byte 8 (e + 1); this thread's entry is
    // e = t, its neighbours e = t - 1 and t + 1 (vertical: the floats of the
    // adjacent pairs; horizontal: whole entries)
    const uint32_t hb_line0 = ptx::smem_addr(sm.hb);
    const uint32_t hb_line1 = hb_line0 + sm.line * 4;
    const uint32_t hb0 = hb_line0 + 8u * t;
    const uint32_t hb1 = hb_line1 + 8u * t;
    float* const slot = p.slots + (size_t)(q % p.n_slots) * H * W;
    float* const out_rowA = slot + (size_t)(ownA ? kA : 0) * W;                  // horizontal
    float* const out_rowB = slot + (size_t)(ownB ? kB : 0) * W;
    float* out_px = slot + (FWD ? 0 : (size_t)(H - 1) * W) + (ownA ? kA : 0);  // vertical
    const ptrdiff_t out_step = FWD ? W : -W;

    uint4 v0[6], v1[6];  // horizontal: the current 16-byte half segment of rows kA, kB
    float acc0[4], acc1[4];
    int lsl = 0;         // slot of the next stage to acquire
    int rel_sl = 0;      // slot of the next stage to release
    int released = 0;
    auto acquire = [&]() {
        wait_env(env, ph, env.full_s + 8u * lsl, (ph.full >> lsl) & 1u, 1);
        ph.full ^= 1u << lsl;
        lsl = (lsl + 1 == stages) ? 0 : lsl + 1;
    };
    auto release = [&]() {
        if (t == 0) ptx::mbar_arrive(env.empty_s + 8u * rel_sl);
        rel_sl = (rel_sl + 1 == stages) ? 0 : rel_sl + 1;
        ++released;
    };
    auto tile_base = [&](int sl) -> uint32_t { return ring_s + sl * 6 * tb + col_byte; };
    // horizontal: load logical half jl (steps jl*kPer ..) of the stage in slot sl
    auto load_half = [&](int sl, int jl) {
        const uint32_t b = tile_base(sl) + 16u * ((uint32_t)(FWD ? jl : 1 - jl) ^ swz);
#pragma unroll
        for (int k6 = 0; k6 < 6; ++k6) {
            v0[k6] = ptx::lds_v4(b + k6 * tb);
            v1[k6] = ptx::lds_v4(b + k6 * tb + 32u * nthr);
        }
    };
    // vertical: raw inputs of step w of the stage in slot sl
    auto fetch_raw = [&](uint32_t base, int w) -> RawIn<T> {
        RawIn<T> r;
        const uint32_t b = base + (FWD ? w : kSeg - 1 - w) * kRowB;
#pragma unroll
        for (int k6 = 0; k6 < 6; ++k6) {
            if constexpr (sizeof(T) == 4)
                r.v[k6] = ptx::lds_v2(b + k6 * kBoxB);
            else
                r.v[k6] = ptx::lds_u32(b + k6 * kBoxB);
        }
        return r;
    };
    // inputs of step w (0 <= w < kSeg) of the stage in slot sl
    auto fetch = [&](int sl, int w) -> PairIn {
        if constexpr (VERT) return unpack_raw<T>(fetch_raw(tile_base(sl), w));
        PairIn in;
        f2 r[6];
        const int e = FWD ? (w % kPer) : (kPer - 1 - (w % kPer));
#pragma unroll
        for (int k6 = 0; k6 < 6; ++k6) r[k6] = ptx::pk(vec_elem<T>(v0[k6], e), vec_elem<T>(v1[k6], e));
        in.x = r[0];
        in.z0 = r[1];
        in.z1 = r[2];
        in.z2 = r[3];
        in.lam = r[4];
        in.u = r[5];
        return in;
    };

    // Software pipeline.  In the barrier interval of step w a thread
    //   issues the loads of the neighbour state of step w (the critical path)
    //   and, vertically, the inputs of step w + 3;
    //   completes the weights of step w + 1 and begins those of step w + 2
    //   (inputs loaded one interval earlier), which covers the load latency;
    //   finishes step w, stores its state and accumulates u * h.
    // Vertical stage reads end at step kSeg - 4 (inputs of row kSeg - 1), so
    // the stage is released after the barrier of step kSeg - 3; horizontal
    // stages are copied to registers, the second half at step kPer - 2.
    int cur_sl = 0;
    acquire();
    if constexpr (!VERT) load_half(cur_sl, 0);
    PairW Wt = complete_pair<kRefine>(begin_pair(fetch(cur_sl, 0), fl), fl);
    PairA A = begin_pair(fetch(cur_sl, 1), fl);
    RawIn<T> raw2;  // vertical: inputs of step w + 2
    if constexpr (VERT) raw2 = fetch_raw(tile_base(cur_sl), 2);
    f2 h = splat(0.0f);
    int next_rs = first_restart(g_len, L, FWD);
    for (int st = 0; st < nst; ++st) {
        const int nxt_sl = (cur_sl + 1 == stages) ? 0 : cur_sl + 1;
        const bool more = st + 1 < nst;
        // vertical: steps of this stage inside the plane (0 if not owned)
        const int wl = !ownA ? 0 : more ? kSeg : L - st * kSeg;
        const uint32_t cur_base = tile_base(cur_sl), nxt_base = tile_base(nxt_sl);
        // steps of this stage that start a group (bit w)
        uint32_t starts = st == 0 ? 1u : 0u;
        while (next_rs < (st + 1) * kSeg) {
            starts |= 1u << (next_rs - st * kSeg);
            next_rs += g_len;
        }
        static_for<kSeg>([&](auto wc) {
            constexpr int w = decltype(wc)::value;
            const bool start = (starts >> w) & 1u;
            if (w > 0 || st > 0) {
                ptx::named_barrier(1, nthr);
                if constexpr (w == (VERT ? kSeg - 3 : kPer - 1)) release();
            }
            const uint32_t hprev = (w & 1) ? hb0 : hb1;
            const uint32_t hcur = (w & 1) ? hb1 : hb0;
            // 1. neighbour state of step w
            const uint2 lp = ptx::lds_v2(hprev);
            const uint2 rp = ptx::lds_v2(hprev + 16u);
            // 2. shared-memory inputs: vertical step w + 3; horizontal the half
            //    segment that step w + 2 starts, if it starts one
            constexpr bool kNext2 = w + 2 >= kSeg;  // step w + 2 is in the next stage
            constexpr int w2 = kNext2 ? w + 2 - kSeg : w + 2;
            const bool have2 = !kNext2 || more;
            RawIn<T> raw3;
            if constexpr (VERT) {
                constexpr bool kNext3 = w + 3 >= kSeg;
                constexpr int w3 = kNext3 ? w + 3 - kSeg : w + 3;
                if constexpr (!kNext3) {
                    raw3 = fetch_raw(cur_base, w3);
                } else {
                    if (more) {
                        if constexpr (w3 == 0) acquire();
                        raw3 = fetch_raw(nxt_base, w3);
                    }
                }
            } else {
                if constexpr (kNext2 && w2 == 0) {
                    if (more) {
                        acquire();
                        load_half(nxt_sl, 0);
                    }
                }
                if constexpr (!kNext2 && w2 == kPer) load_half(cur_sl, 1);
            }
            // 3. weights of step w + 1 (registers) and first half of step w + 2's
            const PairW Wn = complete_pair<kRefine>(A, fl);
            if (have2) {
                if constexpr (VERT)
                    A = begin_pair(unpack_raw<T>(raw2), fl);
                else
                    A = begin_pair(fetch(kNext2 ? nxt_sl : cur_sl, w2), fl);
            }
            // 4. this step's state
            f2 hl, hr;
            if constexpr (VERT) {
                hl = ptx::pk(__uint_as_float(lp.y), lo_of(h));
                hr = ptx::pk(hi_of(h), __uint_as_float(rp.x));
            } else {
                hl = ptx::pk(__uint_as_float(lp.x), __uint_as_float(lp.y));
                hr = ptx::pk(__uint_as_float(rp.x), __uint_as_float(rp.y));
            }
            h = ptx::sel64(start, Wt.lx, finish_pair(Wt, hl, h, hr));
            {
                float a, b;
                ptx::upk(h, a, b);
                ptx::sts_v2_f32(hcur + 8u, a, b);
                if constexpr (!VERT) {  // the seam between the window's two halves
                    const uint32_t line = (w & 1) ? hb_line1 : hb_line0;
                    ptx::sts_f32_if(t == nthr - 1, line + 4u, a);           // left of kB(0)
                    ptx::sts_f32_if(t == 0, line + 8u * (nthr + 1), b);   // right of kA(nthr-1)
                }
            }
            const f2 uh = ptx::mul2(Wt.u, h);
            if constexpr (VERT) {
                {
                    float a, b;
                    ptx::upk(uh, a, b);
                    ptx::red_add_v2_f32_if(w < wl, out_px, a, b, pol_acc);
                }
                out_px += out_step;
            } else {
                float a, b;
                ptx::upk(uh, a, b);
                acc0[FWD ? (w & 3) : 3 - (w & 3)] = a;
                acc1[FWD ? (w & 3) : 3 - (w & 3)] = b;
                if constexpr ((w & 3) == 3) {
                    const int c0 = FWD ? st * kSeg + (w - 3) : W - st * kSeg - (w + 1);
                    ptx::red_add_v4_f32_if(ownA, out_rowA + c0, acc0[0], acc0[1], acc0[2], acc0[3],
                                           pol_acc);
                    ptx::red_add_v4_f32_if(ownB, out_rowB + c0, acc1[0], acc1[1], acc1[2], acc1[3],
                                           pol_acc);
                }
            }
            Wt = Wn;
            if constexpr (VERT) raw2 = raw3;
        });
        cur_sl = nxt_sl;
        // halo exchange at the end of every 32-step block that has a successor
        if (multi && ((st + 1) * kSeg) % kHalo == 0 && (st + 1) * kSeg < L) {
            const int blk = (st + 1) * kSeg / kHalo - 1;
            const f2 hx = VERT ? halo_exchange(env, ph, rank, Kc, blk, L, h)
                               : halo_exchange_split(env, ph, rank, Kc, nthr, blk, L, h);
            if (hx != h) {
                h = hx;
                float a, b;
                ptx::upk(h, a, b);
                ptx::sts_v2_f32(hb1 + 8u, a, b);  // the last step (odd) wrote line 1
            }
        }
    }
    // release the stages still held (read in the last steps)
    ptx::named_barrier(1, nthr);
    while (released < nst) release();
    if (t == 0) {
        sm.cell[2] = (int)ph.full;
        sm.cell[3] = (int)ph.halo;
    }
    return ph;
}

// Zero the two line buffers and arm the first two halo blocks.
__device__ __forceinline__ void chain_begin(const FusedParams& p, const SmemView& sm, int rank,
                                            int L) {
    const int t = threadIdx.x;
    for (int e = t; e < 2 * sm.line; e += blockDim.x) sm.hb[e] = 0.0f;
    if (t == 0 && p.S > 1) {
        arm_halo_block(p, sm, rank, 0, L);
        arm_halo_block(p, sm, rank, 1, L);
    }
    __syncthreads();
}

template <class T, bool kRefine, bool VERT, bool FWD>
__device__ __forceinline__ void run_chain(const FusedParams& p, const SmemView& sm, Phases& ph,
                                          ProducerState& ps, int q, int rank, int producer_warp,
                                          uint64_t pol_in, uint64_t pol_acc) {
    constexpr int kSeg = 32 / sizeof(T);
    constexpr int d = VERT ? (FWD ? 0 : 1) : (FWD ? 2 : 3);
    const int H = p.H, W = p.W;
    const int L = VERT ? H : W, K = VERT ? W : H;
    const int Kc = VERT ? p.Kc_v : p.Kc_h, np = VERT ? p.np_v : p.np_h;
    const int kb = rank * Kc - (p.S > 1 ? kHalo : 0);
    const int t = threadIdx.x;
    const int nthr = np >> 1;
    const int nst = (L + kSeg - 1) / kSeg;
    chain_begin(p, sm, rank, L);
    if ((t >> 5) == producer_warp) {
        if constexpr (VERT) {
            const int nb = p.nb_v;
            producer_run(p, sm, ps, nst, nb, 6u * nb * 64u * kSeg * sizeof(T),
                         [&](int st, int sl, int tensor, int b, uint32_t bar) {
                             const int row0 = FWD ? st * kSeg : H - kSeg - st * kSeg;
                             constexpr uint32_t kBox = 64u * kSeg * (uint32_t)sizeof(T);
                             const uint32_t dst = ptx::smem_addr(sm.tile(sl, 0)) +
                                                  (b * 6u + tensor) * kBox;
                             const CUtensorMap* map = tensor_map(p, &p.tm_xv, d, tensor);
                             if (tensor == 0)
                                 ptx::tma_load_3d_normal(dst, map, kb + 64 * b, row0,
                                                         tensor_z(p, q, tensor), bar);
                             else
                                 ptx::tma_load_3d(dst, map, kb + 64 * b, row0, tensor_z(p, q, tensor),
                                                  bar, pol_in);
                         });
        } else {
            const int nb = p.nb_h, bh = p.bh_h;
            producer_run(p, sm, ps, nst, nb, 6u * nb * bh * 32u,
                         [&](int st, int sl, int tensor, int b, uint32_t bar) {
                             const int col0 = FWD ? st * kSeg : W - kSeg - st * kSeg;
                             const uint32_t dst = ptx::smem_addr(sm.tile(sl, tensor)) + b * bh * 32;
                             ptx::tma_load_3d_normal(dst, tensor_map(p, &p.tm_xh, d, tensor), col0,
                                                     kb + b * bh, tensor_z(p, q, tensor), bar);
                         });
        }
    } else if (t < nthr) {
        ph = chain_consume<T, kRefine, VERT, FWD>(p, sm, ph, q, rank, pol_acc);
    }
    __syncthreads();
}

// Rounds the finished slot of plane q to the output dtype, writes y, re-zeroes
// the slot.  CTA `rank` of the team takes a contiguous 1/S share; every thread
// keeps kUnroll 16-byte loads in flight so the pass runs at L2 bandwidth, not
// at one load latency per thread.
template <class T>
__device__ __forceinline__ void convert_plane(const FusedParams& p, int q, int rank) {
    constexpr int kUnroll = 8;
    const size_t HW = (size_t)p.H * p.W;
    float4* slot = reinterpret_cast<float4*>(p.slots + (size_t)(q % p.n_slots) * HW);
    T* yq = static_cast<T*>(p.y) + (size_t)q * HW;
    const size_t nvec = HW / 4;  // HW is a multiple of 4 (W * sizeof(T) % 32 == 0)
    const size_t per = (nvec + p.S - 1) / p.S;
    const size_t v0 = per * rank, v1 = min(nvec, v0 + per);
    const size_t stride = blockDim.x;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (size_t base = v0 + threadIdx.x; base < v1; base += kUnroll * stride) {
        float4 a[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            const size_t v = base + j * stride;
            if (v < v1) a[j] = __ldcg(slot + v);
        }
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            const size_t v = base + j * stride;
            if (v >= v1) continue;
            __stcg(slot + v, zero);
            if constexpr (sizeof(T) == 4) {
                __stcs(reinterpret_cast<float4*>(yq) + v, a[j]);
            } else {
                __nv_bfloat162 lo = __floats2bfloat162_rn(a[j].x, a[j].y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(a[j].z, a[j].w);
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
__device__ __forceinline__ void team_broadcast(const SmemView& sm, int S, int c, int v) {
    if (S > 1) {
        for (int r = 0; r < S; ++r)
            ptx::st_cluster_s32(ptx::map_shared(ptx::smem_addr(sm.cell + c), r), v);
    } else {
        sm.cell[c] = v;
    }
}

template <class T, bool kRefine>
__global__ void __launch_bounds__(kMaxThreads, 1)
    fused_kernel(const __grid_constant__ FusedParams p) {
    extern __shared__ __align__(128) char smem_raw[];
    // TMA destinations sit on 1024-byte boundaries (the horizontal maps are swizzled)
    char* const smem_base = smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u);
    const SmemView sm = carve(smem_base, p);
    const int rank = p.S > 1 ? (int)ptx::cluster_ctarank() : 0;
    const int t = threadIdx.x;

    const int producer_warp = (blockDim.x >> 5) - 1;
    if (t == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            ptx::mbar_init(ptx::smem_addr(sm.full_bar + s), 1);
            ptx::mbar_init(ptx::smem_addr(sm.empty_bar + s), 1);
        }
        for (int s = 0; s < 2; ++s) ptx::mbar_init(ptx::smem_addr(sm.halo_bar + s), 1);
        sm.cell[2] = 0;
        sm.cell[3] = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&p.tm_xv);
        ptx::prefetch_tensormap(&p.tm_xh);
    }
    team_sync(p.S);

    const uint64_t pol_in = ptx::policy_evict_first();
    const uint64_t pol_acc = ptx::policy_evict_last();
    bool abort = false;
    ProducerState ps{0u, 0u, false};

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
                    const int q = it / p.nd;
                    const int s = q % p.n_slots;
                    const int want = q / p.n_slots + (p.force_stale ? 1000000 : 0);
                    if (ptx::ld_acquire_gpu(&p.ctrl->slot_epoch[s]) != want) {
                        const uint64_t t0 = ptx::global_timer_ns();
                        while (ptx::ld_acquire_gpu(&p.ctrl->slot_epoch[s]) != want) {
                            if (ptx::ld_acquire_gpu(&p.ctrl->call_error) != 0 ||
                                ptx::global_timer_ns() - t0 > p.timeout_ns) {
                                report_error(p, 2);
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
        const int q = it / p.nd;
        const int d = p.d0 + it % p.nd;

        Phases ph{(uint32_t)sm.cell[2], (uint32_t)sm.cell[3], abort};
        if (d == 0)
            run_chain<T, kRefine, true, true>(p, sm, ph, ps, q, rank, producer_warp, pol_in, pol_acc);
        else if (d == 1)
            run_chain<T, kRefine, true, false>(p, sm, ph, ps, q, rank, producer_warp, pol_in, pol_acc);
        else if (d == 2)
            run_chain<T, kRefine, false, true>(p, sm, ph, ps, q, rank, producer_warp, pol_in, pol_acc);
        else
            run_chain<T, kRefine, false, false>(p, sm, ph, ps, q, rank, producer_warp, pol_in, pol_acc);
        abort = abort || ph.abort || ps.abort;

        // Publish this chain, decide whether this team closes the plane.
        __threadfence();
        team_sync(p.S);
        if (rank == 0 && t == 0) {
            const int old = ptx::atom_add_acq_rel_gpu(p.plane_done + q, 1);
            team_broadcast(sm, p.S, 1, (old == p.nd - 1) ? 1 : 0);
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
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool encode_map(CUtensorMap* m, const void* ptr, int dtype, int W, int H, int64_t depth, int box_x,
                int box_y, bool swizzle32 = false) {
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

// Geometry of one team size S; false if it does not fit.  Owned ranges are
// multiples of 64 positions (one vertical box per consumer warp).
bool geometry_for(int S, int H, int W, int es, FusedPlan* gm) {
    FusedPlan g;
    memset(&g, 0, sizeof(g));
    g.S = S;
    g.T = S > 1 ? kHalo : 0;
    const int seg = 32 / es;  // steps per stage
    if (S == 1) {
        g.Kc_v = round_up(W, 64);
        g.Kc_h = round_up(H, 64);
        g.np_v = g.Kc_v;
        g.np_h = g.Kc_h;
    } else {
        g.Kc_v = round_up((W + S - 1) / S, 64);
        g.Kc_h = round_up((H + S - 1) / S, 64);
        // (on narrow planes the last CTAs may own no position of one
        // orientation: they compute out-of-plane positions and exchange zeros)
        g.np_v = g.Kc_v + 2 * g.T;
        g.np_h = g.Kc_h + 2 * g.T;
    }
    const int npmax = g.np_v > g.np_h ? g.np_v : g.np_h;
    g.threads = npmax / 2 + 32;  // consumers (two positions each) + the producer warp
    if (g.threads > kMaxThreads) return false;
    // vertical tile: np_v / 64 boxes of seg rows x 64 columns
    g.nb_v = g.np_v / 64;
    const int tile_v = g.nb_v * 64 * seg * es;
    // horizontal tile: np_h rows x 32 bytes in boxes of <= 256 rows (multiple of 8)
    g.nb_h = (g.np_h + 255) / 256;
    g.bh_h = round_up((g.np_h + g.nb_h - 1) / g.nb_h, 32);  // boxes on 1024-byte boundaries
    if (g.bh_h > 256) return false;
    const int tile_h = g.nb_h * g.bh_h * 32;
    g.tile_bytes = round_up(tile_h > tile_v ? tile_h : tile_v, 1024);
    size_t a, b, c;
    g.stages = 0;
    for (int st = kMaxStages; st >= 2; --st) {
        g.smem = smem_layout(g.tile_bytes, st, npmax, &a, &b, &c) + 1024;  // + base alignment
        if (g.smem <= 227 * 1024) {
            g.stages = st;
            break;
        }
    }
    if (g.stages == 0) return false;
    *gm = g;
    return true;
}

template <class T, bool kRefine>
cudaError_t set_attributes(const FusedPlan& fp) {
    auto kernel = fused_kernel<T, kRefine>;
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fp.smem);
    if (e == cudaSuccess && fp.S > 1)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

void fill_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, const FusedPlan& fp,
                 int clusters, cudaStream_t stream) {
    memset(cfg, 0, sizeof(*cfg));
    cfg->gridDim = dim3(clusters * fp.S, 1, 1);
    cfg->blockDim = dim3(fp.threads, 1, 1);
    cfg->dynamicSmemBytes = fp.smem;
    cfg->stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = fp.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg->attrs = attr;
    cfg->numAttrs = 1;
}

template <class T, bool kRefine>
int max_teams(const FusedPlan& fp) {
    if (set_attributes<T, kRefine>(fp) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    fill_config(&cfg, attr, fp, 1, 0);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fused_kernel<T, kRefine>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

template <class T, bool kRefine>
cudaError_t launch_typed(Problem& pb, const FusedPlan& fp, void* ws) {
    cudaError_t e = set_attributes<T, kRefine>(fp);
    if (e != cudaSuccess) return e;
    const int H = (int)pb.H, W = (int)pb.W;
    const int nd = pb.d1 - pb.d0;
    constexpr int J = 32 / (int)sizeof(T);  // steps per stage: 32-byte row segments
    FusedParams prm;
    memset(&prm, 0, sizeof(prm));
    const int64_t planes = pb.planes();
    if (!encode_map(&prm.tm_xv, pb.x, pb.dtype, W, H, planes, 64, J) ||
        !encode_map(&prm.tm_xh, pb.x, pb.dtype, W, H, planes, J, fp.bh_h, true))
        return cudaErrorInvalidValue;
    for (int d = pb.d0; d < pb.d1; ++d) {
        const bool vert = d < 2;
        const int bx = vert ? 64 : J;
        const int by = vert ? J : fp.bh_h;
        if (!encode_map(&prm.tm_z[d], pb.z.p[d], pb.dtype, W, H, 3 * (planes / pb.z_div), bx, by,
                        !vert) ||
            !encode_map(&prm.tm_l[d], pb.lam.p[d], pb.dtype, W, H, planes, bx, by, !vert) ||
            !encode_map(&prm.tm_u[d], pb.u.p[d], pb.dtype, W, H, planes, bx, by, !vert))
            return cudaErrorInvalidValue;
    }
    char* base = static_cast<char*>(ws);
    prm.y = pb.y;
    prm.ctrl = reinterpret_cast<FusedCtrl*>(base);
    prm.plane_done = reinterpret_cast<int*>(base + sizeof(FusedCtrl));
    prm.slots = reinterpret_cast<float*>(base + fp.ctrl_bytes);
    prm.timeout_ns = fp.timeout_ns;
    prm.H = H;
    prm.W = W;
    prm.planes = (int)planes;
    prm.g = (int)pb.g;
    prm.d0 = pb.d0;
    prm.nd = nd;
    prm.S = fp.S;
    prm.Kc_v = fp.Kc_v;
    prm.Kc_h = fp.Kc_h;
    prm.np_v = fp.np_v;
    prm.np_h = fp.np_h;
    prm.nb_v = fp.nb_v;
    prm.nb_h = fp.nb_h;
    prm.bh_h = fp.bh_h;
    prm.tile_bytes = fp.tile_bytes;
    prm.stages = fp.stages;
    prm.n_slots = fp.n_slots;
    prm.n_items = (int)(planes * nd);
    prm.z_div = (int)pb.z_div;
    prm.force_stale = fp.force_stale;

    // Reset the per-call part of the control block (not the sticky error).
    e = cudaMemsetAsync(base + kCtrlResetOffset, 0, fp.ctrl_bytes - kCtrlResetOffset, pb.stream);
    if (e != cudaSuccess) return e;
    if (fp.zero_slots) {
        e = cudaMemsetAsync(prm.slots, 0, fp.slot_bytes * fp.n_slots, pb.stream);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    fill_config(&cfg, attr, fp, fp.n_teams, pb.stream);
    if (pb.ev_begin) cudaEventRecord(pb.ev_begin, pb.stream);
    e = cudaLaunchKernelEx(&cfg, fused_kernel<T, kRefine>, prm);
    if (pb.ev_end) cudaEventRecord(pb.ev_end, pb.stream);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

size_t fused_ctrl_bytes(int64_t planes) {
    return ((sizeof(FusedCtrl) + sizeof(int) * (size_t)planes) + 255) & ~(size_t)255;
}

bool fused_plan(const Problem& pb, FusedPlan* fp) {
    const int es = pb.dtype == 0 ? 4 : 2;
    if (pb.H > 0x7fffffff / pb.W) return false;
    if ((pb.W * es) % 32 != 0) return false;  // whole 32-byte horizontal stages (and TMA strides)
    if (pb.planes() * 3 > 0x7fffffffLL) return false;
    const int H = (int)pb.H, W = (int)pb.W;
    const int nd = pb.d1 - pb.d0;
    const size_t slot_bytes = sizeof(float) * (size_t)H * W;
    const size_t l2_budget = (size_t)96 << 20;
    for (int S : {1, 2, 4, 8}) {
        FusedPlan plan;
        if (!geometry_for(S, H, W, es, &plan)) continue;
        int teams = pb.dtype == 0 ? max_teams<float, true>(plan)
                                  : max_teams<__nv_bfloat16, false>(plan);
        if (teams <= 0) continue;
        const int64_t items = pb.planes() * nd;
        if (teams > items) teams = (int)items;
        // planes that can be in flight at once, plus two for the ones closing
        const int64_t want_slots = (teams + nd - 1) / nd + 2;
        int64_t cap = (int64_t)(l2_budget / slot_bytes);
        if (cap < 1) cap = 1;
        int64_t slots = want_slots < cap ? want_slots : cap;
        if (slots > kMaxSlots) slots = kMaxSlots;
        if (slots > pb.planes()) slots = pb.planes();
        // Prefer a larger team when the slot budget, not the SM count, would
        // leave teams idle.
        const bool starved = (int64_t)slots * nd < teams && S < 8;
        if (starved) {
            FusedPlan g2;
            if (geometry_for(S * 2, H, W, es, &g2)) continue;
        }
        plan.n_teams = teams;
        plan.n_slots = (int)slots;
        plan.slot_bytes = slot_bytes;
        plan.ctrl_bytes = fused_ctrl_bytes(pb.planes());
        plan.ws_bytes = plan.ctrl_bytes + slot_bytes * (size_t)slots;
        plan.timeout_ns = 4000000000ull;
        plan.zero_slots = false;
        plan.force_stale = 0;
        *fp = plan;
        return true;
    }
    return false;
}

cudaError_t launch_fused(Problem& pb, const FusedPlan& fp, void* ws, int* launches) {
    pb.kernel_name = "fused_kernel";
    if (getenv("GSPN_DEBUG_PLAN"))
        fprintf(stderr,
                "gspn fused plan: S=%d T=%d Kc_v=%d Kc_h=%d np_v=%d np_h=%d nb_v=%d nb_h=%d "
                "bh_h=%d tile=%d stages=%d threads=%d smem=%zu teams=%d slots=%d\n",
                fp.S, fp.T, fp.Kc_v, fp.Kc_h, fp.np_v, fp.np_h, fp.nb_v, fp.nb_h, fp.bh_h,
                fp.tile_bytes, fp.stages, fp.threads, fp.smem, fp.n_teams, fp.n_slots);
    cudaError_t e = pb.dtype == 0 ? launch_typed<float, true>(pb, fp, ws)
                                  : launch_typed<__nv_bfloat16, false>(pb, fp, ws);
    if (e == cudaSuccess) *launches += 1;
    return e;
}

}  // namespace gspn
