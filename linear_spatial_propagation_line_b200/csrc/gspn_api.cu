// C ABI of the GSPN propagation library: argument validation, kernel choice,
// the per-device workspace and the host-buffer entry point.  See
// include/gspn.h for the contract of every function.
#include <cuda_runtime.h>

#include <mutex>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "../../include/gspn.h"
#include "gspn_internal.h"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceBuffers {
    void* ws = nullptr;  // fp32 accumulator of the line-chain path
    size_t ws_bytes = 0;
    void* fused = nullptr;  // control block + L2 slots of the fused path (kept zeroed)
    size_t fused_bytes = 0;
    bool fused_dirty = false;    // slots may hold leftovers of an aborted launch
    bool pending_error = false;  // a device error seen while replacing the workspace
    void* staging = nullptr;
    size_t staging_bytes = 0;
    void* bws = nullptr;  // backward: hidden states and the dx accumulator
    size_t bws_bytes = 0;
};

std::mutex g_mutex;
DeviceBuffers g_dev[kMaxDevices];

thread_local char t_cuda_error[256] = "no error";
thread_local int t_last_launches = 0;
thread_local cudaEvent_t t_ev_begin = nullptr;
thread_local cudaEvent_t t_ev_end = nullptr;
thread_local const char* t_last_kernel = "";
thread_local bool t_force_timeout = false;
thread_local unsigned long long t_force_timeout_ns = 0;
thread_local int t_large_path = GSPN_PATH_AUTO;

int cuda_fail(cudaError_t e) {
    snprintf(t_cuda_error, sizeof(t_cuda_error), "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return GSPN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Grow-only buffer for the current device.
int ensure_buffer(void** ptr, size_t* have, size_t need) {
    if (*have >= need) return GSPN_OK;
    if (*ptr) {
        cudaError_t e = cudaFree(*ptr);
        *ptr = nullptr;
        *have = 0;
        if (e != cudaSuccess) return cuda_fail(e);
    }
    cudaError_t e = cudaMalloc(ptr, need);
    if (e != cudaSuccess) {
        *ptr = nullptr;
        return cuda_fail(e);
    }
    *have = need;
    return GSPN_OK;
}

int current_device(int* dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (*dev < 0 || *dev >= kMaxDevices) {
        snprintf(t_cuda_error, sizeof(t_cuda_error), "device ordinal %d out of range", *dev);
        return GSPN_ERR_CUDA;
    }
    return GSPN_OK;
}

// Shape checks shared by every entry point.  Per-plane indices are 32-bit in
// the kernels, so 3*H*W must fit in int32; the plane count must fit too.
int check_shape(int64_t B, int64_t C, int64_t H, int64_t W) {
    if (B <= 0 || C <= 0 || H <= 0 || W <= 0) return GSPN_ERR_SHAPE;
    if (H > 0x7fffffffLL / W) return GSPN_ERR_SHAPE;
    if (3 * H * W > 0x7fffffffLL) return GSPN_ERR_SHAPE;
    if (B > 0x7fffffffLL / C) return GSPN_ERR_SHAPE;
    const int64_t planes = B * C;
    if (planes > (int64_t)1 << 40 || H * W > ((int64_t)1 << 62) / planes / 3 / 4)
        return GSPN_ERR_SHAPE;
    return GSPN_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// Validates a call of directions [d0, d1) whose tensors sit at index d of the
// pointer arrays, and fills the problem description.
int validate(const void* x, const void* const* wlogit, const void* const* lam,
             const void* const* u, int64_t B, int64_t C, int64_t H, int64_t W,
             int64_t group_len, int dtype, int d0, int d1, bool need_align, void* y,
             gspn::Problem* pb, bool shared_logits = false) {
    if (!x || !wlogit || !lam || !u || !y) return GSPN_ERR_NULL;
    for (int d = d0; d < d1; ++d)
        if (!wlogit[d] || !lam[d] || !u[d]) return GSPN_ERR_NULL;
    int s = check_shape(B, C, H, W);
    if (s != GSPN_OK) return s;
    if (dtype != GSPN_F32 && dtype != GSPN_BF16) return GSPN_ERR_DTYPE;
    if (group_len < 0) return GSPN_ERR_GROUP;
    if (need_align) {
        if (!aligned16(x) || !aligned16(y)) return GSPN_ERR_ALIGN;
        for (int d = d0; d < d1; ++d)
            if (!aligned16(wlogit[d]) || !aligned16(lam[d]) || !aligned16(u[d]))
                return GSPN_ERR_ALIGN;
    }
    const size_t es = dtype == GSPN_F32 ? 4 : 2;
    const size_t n = (size_t)(B * C * H * W) * es;
    if (overlaps(y, n, x, n)) return GSPN_ERR_ALIAS;
    const size_t nz = shared_logits ? (size_t)(B * H * W) * es : n;  // one logit plane set per b
    for (int d = d0; d < d1; ++d)
        if (overlaps(y, n, wlogit[d], 3 * nz) || overlaps(y, n, lam[d], n) ||
            overlaps(y, n, u[d], n))
            return GSPN_ERR_ALIAS;
    pb->x = x;
    for (int d = 0; d < 4; ++d) {
        const bool in = d >= d0 && d < d1;
        pb->z.p[d] = in ? wlogit[d] : nullptr;
        pb->lam.p[d] = in ? lam[d] : nullptr;
        pb->u.p[d] = in ? u[d] : nullptr;
    }
    pb->B = B;
    pb->C = C;
    pb->H = H;
    pb->W = W;
    pb->g = group_len > 0x7fffffffLL ? 0x7fffffffLL : group_len;
    pb->z_div = shared_logits ? C : 1;
    pb->dtype = dtype;
    pb->d0 = d0;
    pb->d1 = d1;
    pb->y = y;
    return GSPN_OK;
}

// The fused workspace: grown on demand, zero-filled when (re)allocated.
int ensure_fused(DeviceBuffers& db, size_t need, cudaStream_t stream) {
    if (db.fused_bytes >= need) return GSPN_OK;
    if (db.fused) {
        int sticky = 0;
        cudaError_t e = cudaMemcpy(&sticky, static_cast<char*>(db.fused) +
                                                gspn::kFusedStickyErrorOffset,
                                   sizeof(int), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e);
        if (sticky) db.pending_error = true;
        e = cudaFree(db.fused);
        db.fused = nullptr;
        db.fused_bytes = 0;
        if (e != cudaSuccess) return cuda_fail(e);
    }
    cudaError_t e = cudaMalloc(&db.fused, need);
    if (e != cudaSuccess) {
        db.fused = nullptr;
        return cuda_fail(e);
    }
    db.fused_bytes = need;
    e = cudaMemsetAsync(db.fused, 0, need, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    db.fused_dirty = false;
    return GSPN_OK;
}

int run(gspn::Problem& pb) {
    int launches = 0;
    pb.ev_begin = t_ev_begin;
    pb.ev_end = t_ev_end;
    cudaError_t e;
    gspn::FusedPlan fp;
    gspn::SweepPlan sp;
    if (gspn::small_plane_fits(pb, nullptr)) {
        e = gspn::launch_small_plane(pb, &launches);
    } else if (t_large_path == GSPN_PATH_SWEEP && gspn::sweep_plan(pb, &sp)) {
        int dev;
        int s = current_device(&dev);
        if (s != GSPN_OK) return s;
        std::lock_guard<std::mutex> lock(g_mutex);
        DeviceBuffers& db = g_dev[dev];
        s = ensure_fused(db, sp.ws_bytes, pb.stream);
        if (s != GSPN_OK) return s;
        sp.zero_slots = db.fused_dirty;
        db.fused_dirty = false;
        if (t_force_timeout) {
            sp.force_stale = 1;
            sp.timeout_ns = t_force_timeout_ns;
            t_force_timeout = false;
        }
        e = gspn::launch_sweep(pb, sp, db.fused, &launches);
    } else if (t_large_path != GSPN_PATH_SWEEP && gspn::fused_plan(pb, &fp)) {
        int dev;
        int s = current_device(&dev);
        if (s != GSPN_OK) return s;
        std::lock_guard<std::mutex> lock(g_mutex);
        DeviceBuffers& db = g_dev[dev];
        s = ensure_fused(db, fp.ws_bytes, pb.stream);
        if (s != GSPN_OK) return s;
        fp.zero_slots = db.fused_dirty;
        db.fused_dirty = false;
        if (t_force_timeout) {
            fp.force_stale = 1;
            fp.timeout_ns = t_force_timeout_ns;
            t_force_timeout = false;
        }
        e = gspn::launch_fused(pb, fp, db.fused, &launches);
    } else {
        int dev;
        int s = current_device(&dev);
        if (s != GSPN_OK) return s;
        std::lock_guard<std::mutex> lock(g_mutex);
        DeviceBuffers& db = g_dev[dev];
        s = ensure_buffer(&db.ws, &db.ws_bytes, sizeof(float) * (size_t)pb.pixch());
        if (s != GSPN_OK) return s;
        e = gspn::launch_chain(pb, static_cast<float*>(db.ws), &launches);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    t_last_launches = launches;
    t_last_kernel = pb.kernel_name;
    return GSPN_OK;
}

}  // namespace

extern "C" {

int gspn_forward(const void* x, const void* const wlogit[4], const void* const lam[4],
                 const void* const u[4], int64_t B, int64_t C, int64_t H, int64_t W,
                 int64_t group_len, int dtype, void* stream, void* y) {
    gspn::Problem pb;
    int s = validate(x, wlogit, lam, u, B, C, H, W, group_len, dtype, 0, 4, true, y, &pb);
    if (s != GSPN_OK) return s;
    pb.stream = static_cast<cudaStream_t>(stream);
    return run(pb);
}

int gspn_forward_shared(const void* x, const void* const wlogit[4], const void* const lam[4],
                        const void* const u[4], int64_t B, int64_t C, int64_t H, int64_t W,
                        int64_t group_len, int dtype, void* stream, void* y) {
    gspn::Problem pb;
    int s = validate(x, wlogit, lam, u, B, C, H, W, group_len, dtype, 0, 4, true, y, &pb, true);
    if (s != GSPN_OK) return s;
    pb.stream = static_cast<cudaStream_t>(stream);
    return run(pb);
}

int gspn_forward_dir(const void* x, const void* wlogit, const void* lam, const void* u,
                     int64_t B, int64_t C, int64_t H, int64_t W, int64_t group_len, int d,
                     int dtype, void* stream, void* y) {
    if (d < 0 || d > 3) return GSPN_ERR_DIR;
    const void* zs[4] = {nullptr, nullptr, nullptr, nullptr};
    const void* ls[4] = {nullptr, nullptr, nullptr, nullptr};
    const void* us[4] = {nullptr, nullptr, nullptr, nullptr};
    zs[d] = wlogit;
    ls[d] = lam;
    us[d] = u;
    gspn::Problem pb;
    int s = validate(x, zs, ls, us, B, C, H, W, group_len, dtype, d, d + 1, true, y, &pb);
    if (s != GSPN_OK) return s;
    pb.stream = static_cast<cudaStream_t>(stream);
    return run(pb);
}

int gspn_forward_host(const void* x, const void* const wlogit[4], const void* const lam[4],
                      const void* const u[4], int64_t B, int64_t C, int64_t H, int64_t W,
                      int64_t group_len, int dtype, void* stream, void* y) {
    gspn::Problem hp;
    int s = validate(x, wlogit, lam, u, B, C, H, W, group_len, dtype, 0, 4, false, y, &hp);
    if (s != GSPN_OK) return s;
    int dev;
    if ((s = current_device(&dev)) != GSPN_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t es = dtype == GSPN_F32 ? 4 : 2;
    const size_t n = (size_t)(B * C * H * W) * es;
    const size_t slot = (n + 255) & ~(size_t)255;  // 256-byte aligned sub-buffers
    char* base;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        DeviceBuffers& db = g_dev[dev];
        s = ensure_buffer(&db.staging, &db.staging_bytes, 22 * slot);
        if (s != GSPN_OK) return s;
        base = static_cast<char*>(db.staging);
    }
    // device layout: x | y | z0 (3 slots) | lam0 | u0 | z1 ...
    char* dx = base;
    char* dy = base + slot;
    const void* dz[4];
    const void* dl[4];
    const void* du[4];
    cudaError_t e = cudaMemcpyAsync(dx, x, n, cudaMemcpyHostToDevice, st);
    for (int d = 0; d < 4 && e == cudaSuccess; ++d) {
        char* zd = base + (2 + 5 * d) * slot;
        char* ld = zd + 3 * slot;
        char* ud = ld + slot;
        dz[d] = zd;
        dl[d] = ld;
        du[d] = ud;
        e = cudaMemcpyAsync(zd, wlogit[d], 3 * n, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(ld, lam[d], n, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(ud, u[d], n, cudaMemcpyHostToDevice, st);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    s = gspn_forward(dx, dz, dl, du, B, C, H, W, group_len, dtype, stream, dy);
    if (s != GSPN_OK) return s;
    e = cudaMemcpyAsync(y, dy, n, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    return GSPN_OK;
}

int gspn_forward_noalloc(const void* x, const void* const wlogit[4], const void* const lam[4],
                         const void* const u[4], int64_t B, int64_t C, int64_t H, int64_t W,
                         int64_t group_len, int dtype, void* stream, void* y) {
    gspn::Problem pb;
    int s = validate(x, wlogit, lam, u, B, C, H, W, group_len, dtype, 0, 4, true, y, &pb);
    if (s != GSPN_OK) return s;
    if (pb.pixch() > gspn::kNoAllocMaxPixch) return GSPN_ERR_SCRATCH;
    int dev;
    if ((s = current_device(&dev)) != GSPN_OK) return s;
    float* scratch = nullptr;
    cudaError_t e = gspn::noalloc_scratch(dev, &scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    pb.stream = static_cast<cudaStream_t>(stream);
    pb.ev_begin = t_ev_begin;
    pb.ev_end = t_ev_end;
    int launches = 0;
    e = gspn::launch_chain(pb, scratch, &launches);  // zeroes scratch[0, B*C*H*W) first
    if (e != cudaSuccess) return cuda_fail(e);
    t_last_launches = launches;
    t_last_kernel = pb.kernel_name;
    return GSPN_OK;
}

int gspn_backward(const void* x, const void* const wlogit[4], const void* const lam[4],
                  const void* const u[4], const void* gy, int64_t B, int64_t C, int64_t H,
                  int64_t W, int64_t group_len, int dtype, void* stream, void* dx,
                  void* const dwlogit[4], void* const dlam[4], void* const du[4]) {
    if (!gy || !dx || !dwlogit || !dlam || !du) return GSPN_ERR_NULL;
    for (int d = 0; d < 4; ++d)
        if (!dwlogit[d] || !dlam[d] || !du[d]) return GSPN_ERR_NULL;
    gspn::BackwardProblem bp;
    // validate the forward inputs; dx stands in for y in the alias checks
    int s = validate(x, wlogit, lam, u, B, C, H, W, group_len, dtype, 0, 4, true, dx, &bp.fwd);
    if (s != GSPN_OK) return s;
    if (!aligned16(gy)) return GSPN_ERR_ALIGN;
    for (int d = 0; d < 4; ++d)
        if (!aligned16(dwlogit[d]) || !aligned16(dlam[d]) || !aligned16(du[d]))
            return GSPN_ERR_ALIGN;
    // no output may overlap an input or another output
    const size_t es = dtype == GSPN_F32 ? 4 : 2;
    const size_t n = (size_t)(B * C * H * W) * es;
    const void* in_p[14];
    size_t in_n[14];
    int ni = 0;
    in_p[ni] = x; in_n[ni++] = n;
    in_p[ni] = gy; in_n[ni++] = n;
    for (int d = 0; d < 4; ++d) {
        in_p[ni] = wlogit[d]; in_n[ni++] = 3 * n;
        in_p[ni] = lam[d]; in_n[ni++] = n;
        in_p[ni] = u[d]; in_n[ni++] = n;
    }
    const void* out_p[13];
    size_t out_n[13];
    int no = 0;
    out_p[no] = dx; out_n[no++] = n;
    for (int d = 0; d < 4; ++d) {
        out_p[no] = dwlogit[d]; out_n[no++] = 3 * n;
        out_p[no] = dlam[d]; out_n[no++] = n;
        out_p[no] = du[d]; out_n[no++] = n;
    }
    for (int o = 0; o < no; ++o) {
        for (int i = 0; i < ni; ++i)
            if (overlaps(out_p[o], out_n[o], in_p[i], in_n[i])) return GSPN_ERR_ALIAS;
        for (int o2 = o + 1; o2 < no; ++o2)
            if (overlaps(out_p[o], out_n[o], out_p[o2], out_n[o2])) return GSPN_ERR_ALIAS;
    }
    bp.gy = gy;
    bp.dx = dx;
    for (int d = 0; d < 4; ++d) {
        bp.dz[d] = dwlogit[d];
        bp.dlam[d] = dlam[d];
        bp.du[d] = du[d];
    }
    bp.fwd.stream = static_cast<cudaStream_t>(stream);
    bp.fwd.ev_begin = t_ev_begin;
    bp.fwd.ev_end = t_ev_end;
    int dev;
    if ((s = current_device(&dev)) != GSPN_OK) return s;
    int launches = 0;
    cudaError_t e;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        DeviceBuffers& db = g_dev[dev];
        s = ensure_buffer(&db.bws, &db.bws_bytes, gspn::backward_workspace_bytes(bp.fwd));
        if (s != GSPN_OK) return s;
        e = gspn::launch_backward(bp, static_cast<float*>(db.bws), &launches);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    t_last_launches = launches;
    t_last_kernel = bp.fwd.kernel_name;
    return GSPN_OK;
}

int gspn_last_launch_count(void) { return t_last_launches; }

int gspn_check_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    int dev;
    int s = current_device(&dev);
    if (s != GSPN_OK) return s;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceBuffers& db = g_dev[dev];
    bool failed = db.pending_error;
    db.pending_error = false;
    if (db.fused) {
        int sticky = 0;
        char* word = static_cast<char*>(db.fused) + gspn::kFusedStickyErrorOffset;
        e = cudaMemcpy(&sticky, word, sizeof(int), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e);
        if (sticky) {
            e = cudaMemset(word, 0, sizeof(int));
            if (e != cudaSuccess) return cuda_fail(e);
            failed = true;
        }
    }
    if (failed) {
        db.fused_dirty = true;
        return GSPN_ERR_TIMEOUT;
    }
    return GSPN_OK;
}

int gspn_debug_force_timeout(int64_t timeout_ns) {
    if (timeout_ns <= 0) return GSPN_ERR_SHAPE;
    t_force_timeout = true;
    t_force_timeout_ns = (unsigned long long)timeout_ns;
    return GSPN_OK;
}

int gspn_debug_select_path(int path) {
    if (path != GSPN_PATH_AUTO && path != GSPN_PATH_FUSED && path != GSPN_PATH_SWEEP)
        return GSPN_ERR_DIR;
    t_large_path = path;
    return GSPN_OK;
}

int gspn_set_timing_events(void* begin, void* end) {
    t_ev_begin = static_cast<cudaEvent_t>(begin);
    t_ev_end = static_cast<cudaEvent_t>(end);
    return GSPN_OK;
}

const char* gspn_last_kernel_name(void) { return t_last_kernel; }

int gspn_release(void) {
    int dev;
    int s = current_device(&dev);
    if (s != GSPN_OK) return s;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceBuffers& db = g_dev[dev];
    cudaError_t e = cudaSuccess;
    if (db.ws) e = cudaFree(db.ws);
    if (db.fused) {
        cudaError_t e2 = cudaFree(db.fused);
        if (e == cudaSuccess) e = e2;
    }
    if (db.staging) {
        cudaError_t e2 = cudaFree(db.staging);
        if (e == cudaSuccess) e = e2;
    }
    if (db.bws) {
        cudaError_t e2 = cudaFree(db.bws);
        if (e == cudaSuccess) e = e2;
    }
    db = DeviceBuffers();
    return e == cudaSuccess ? GSPN_OK : cuda_fail(e);
}

const char* gspn_status_string(int status) {
    switch (status) {
        case GSPN_OK: return "ok";
        case GSPN_ERR_NULL: return "a required pointer is NULL";
        case GSPN_ERR_SHAPE: return "bad shape: a dimension <= 0 or an element count overflows";
        case GSPN_ERR_DTYPE: return "unknown dtype";
        case GSPN_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case GSPN_ERR_GROUP: return "group_len < 0";
        case GSPN_ERR_CUDA: return "CUDA error (see gspn_last_cuda_error)";
        case GSPN_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        case GSPN_ERR_DIR: return "direction outside 0..3";
        case GSPN_ERR_ALIAS: return "output overlaps an input";
        case GSPN_ERR_SCRATCH: return "B*C*H*W exceeds the fixed scratch of gspn_forward_noalloc";
        default: return "unknown status";
    }
}

const char* gspn_last_cuda_error(void) { return t_cuda_error; }

int gspn_version(void) { return 100; }

}  // extern "C"
