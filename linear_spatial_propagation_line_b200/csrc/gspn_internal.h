// Internal launch interface between the C ABI (gspn_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string.h>

#include "../../include/gspn.h"
#include "gspn_common.cuh"

namespace gspn {

// One validated call: directions [d0, d1) of the four-direction operation.
// For a single-direction call the pointer arrays hold the tensors at index d0.
struct Problem {
    const void* x;
    Ptr4 z;    // wlogit[d]: [B][C][3][H][W]
    Ptr4 lam;  // [B][C][H][W]
    Ptr4 u;    // [B][C][H][W]
    int64_t B, C, H, W, g;
    int64_t z_div = 1;  // logits of plane q are logit plane q / z_div (C: shared by channels)
    int dtype;  // GSPN_F32 / GSPN_BF16
    int d0, d1;
    cudaStream_t stream;
    void* y;
    cudaEvent_t ev_begin = nullptr;  // recorded around the dominant kernel if set
    cudaEvent_t ev_end = nullptr;
    const char* kernel_name = "";   // set by the launcher: the dominant kernel
    int64_t planes() const { return B * C; }
    int64_t pixch() const { return B * C * H * W; }
};

// Whole-plane kernel: one CTA keeps a plane's fp32 output and one direction's
// weights in shared memory.  Used when max(H, W) <= 64 and the plane fits.
bool small_plane_fits(const Problem& pb, size_t* smem_bytes);
cudaError_t launch_small_plane(Problem& pb, int* launches);

// Generic line-chain path for any plane size: one CTA per (plane, direction)
// scans with the whole line in shared memory and adds u_d * h_d into the fp32
// workspace `ws` (B*C*H*W floats, zeroed here), then a conversion kernel
// writes y.
cudaError_t launch_chain(Problem& pb, float* ws, int* launches);

// Backward pass: gradients of L = sum(gy * y) for every input of a forward
// call.  Workspace: backward_workspace_bytes(fwd) bytes of fp32 (every
// direction's hidden state and the dx accumulator).
struct BackwardProblem {
    Problem fwd;          // the forward call's inputs (all four directions)
    const void* gy;       // dL/dy [B][C][H][W]
    void* dx;             // [B][C][H][W]
    void* dz[4];          // [B][C][3][H][W]
    void* dlam[4];        // [B][C][H][W]
    void* du[4];          // [B][C][H][W]
};
size_t backward_workspace_bytes(const Problem& pb);
cudaError_t launch_backward(BackwardProblem& bp, float* ws, int* launches);

// Fixed-scratch variant of the line-chain path (gspn_forward_noalloc): the
// fp32 accumulator is a static device array of kNoAllocMaxPixch floats.
// noalloc_scratch returns its address on `device` (which must be current),
// looking it up on the first call for that device.
constexpr int64_t kNoAllocMaxPixch = GSPN_NOALLOC_MAX_ELEMENTS;
cudaError_t noalloc_scratch(int device, float** scratch);

// Fused persistent path (large planes whose rows are 16-byte multiples): one
// launch computes all directions, accumulating in L2-resident fp32 slots.
struct FusedPlan {
    int S, T;                 // CTAs per team (cluster), halo width
    int Kc_v, Kc_h, np_v, np_h;
    int nb_v, nb_h, bh_h;
    int tile_bytes, threads, stages;
    size_t smem;
    int n_teams, n_slots;
    size_t slot_bytes, ctrl_bytes, ws_bytes;
    unsigned long long timeout_ns;
    bool zero_slots;          // clear the slot area before the launch
    int force_stale;          // test hook: make the slot wait expire
};
bool fused_plan(const Problem& pb, FusedPlan* fp);
cudaError_t launch_fused(Problem& pb, const FusedPlan& fp, void* ws, int* launches);
// Line-sweep persistent path (large planes whose rows are 16-byte multiples):
// the scan line lives in registers, four positions per lane; one launch
// computes all directions into the same workspace layout as the fused path.
struct SweepPlan {
    int S;                    // CTAs per team (cluster)
    int So[2], Kc[2];         // CTAs per chain and owned positions per CTA (vertical, horizontal)
    int nw, threads;          // consumer warps, threads per CTA
    int nb[2], bw[2];         // boxes per tensor and stage, box width in line positions
    int tile_bytes, stages;
    size_t smem;
    int ipp;                  // work items per plane
    int item_dir[4][2];       // directions of each item (-1: that half of the team idles)
    int n_teams, n_slots;
    size_t slot_bytes, ctrl_bytes, ws_bytes;
    unsigned long long timeout_ns;
    bool zero_slots;
    int force_stale;
};
bool sweep_plan(const Problem& pb, SweepPlan* sp);
cudaError_t launch_sweep(Problem& pb, const SweepPlan& sp, void* ws, int* launches);

// Offset of the sticky device error word inside the fused workspace.
constexpr size_t kFusedStickyErrorOffset = 0;

}  // namespace gspn
