/*
 * gspn.h -- C ABI of the B200 (sm_100a) GSPN line-scan propagation library.
 *
 * The operation (Generalized Spatial Propagation Network, arXiv 2501.12381,
 * as walked through on the CSDN page "GSPN——在convolution基础上并行序列建模"):
 *
 *   For each plane (b, c) and each of four scan directions d, with lines i
 *   taken along the scan axis and positions k along the orthogonal axis,
 *
 *     h_i[k] = sum_{o in {-1,0,+1}} w_i[k,o] * h_{i-1}[k+o] + lam_i[k] * x_i[k]
 *     h_0[k] = lam_0[k] * x_0[k]                       (section "方法")
 *
 *   with w_i[k,o] = sigmoid(z[o]) / sum over EXISTING neighbours o' of
 *   sigmoid(z[o']): a missing (outside-the-plane) neighbour is dropped before
 *   normalising, so every row of w_i is stochastic (section "行随机矩阵").
 *   The four directions are merged as y = sum_d u_d (.) h_d (section "方法",
 *   y_i = u_i (.) h_i; four-direction scan in "如何设计一个高效的传播层").
 *   With group_len = g > 0 (local GSPN, section "全局与局部GSPN") the scan
 *   axis is cut into blocks [s*g, (s+1)*g) of the original coordinate and the
 *   recurrence restarts (h = lam * x) on the first line of every block in
 *   scan order.
 *
 * Directions: 0 top->bottom, 1 bottom->top (scan along H, positions along W);
 *             2 left->right, 3 right->left (scan along W, positions along H).
 * Logit slots: wlogit[d][b][c][s][r][col] is the logit of the neighbour at
 *   orthogonal offset s-1 (column offset for d = 0,1; row offset for
 *   d = 2,3) of pixel (r, col) -- all parameters sit at the pixel being
 *   computed, in original image coordinates.
 *
 * Layouts: contiguous row-major.  x, lam[d], u[d], y: [B][C][H][W];
 *   wlogit[d]: [B][C][3][H][W].  One dtype for every tensor of a call.
 * Arithmetic: fp32 throughout (state, weights, accumulation); y is rounded
 *   once to the storage dtype (round-to-nearest-even for bf16).
 *
 * Ownership and concurrency: every pointer of gspn_forward / gspn_forward_dir
 *   is DEVICE memory owned by the caller, on the current CUDA device.  The
 *   calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and return after the launches.  Inputs are read only; y is
 *   overwritten completely and must not overlap any input.  Every pointer
 *   must be 16-byte aligned.  The library keeps one lazily created,
 *   per-device workspace for large planes (freed by gspn_release); calls
 *   that use it must not run concurrently on different streams of the same
 *   device.
 *
 * Errors: every entry point validates its arguments before any launch and
 *   returns a negative GSPN_ERR_* with nothing launched.  A CUDA launch
 *   failure returns GSPN_ERR_CUDA (text from gspn_last_cuda_error()).  The
 *   library never aborts the process.
 */
#ifndef GSPN_B200_H
#define GSPN_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* storage dtypes */
#define GSPN_F32 0
#define GSPN_BF16 1

/* status codes */
#define GSPN_OK 0
#define GSPN_ERR_NULL (-1)     /* a required pointer is NULL */
#define GSPN_ERR_SHAPE (-2)    /* a dimension <= 0, or an element count overflows */
#define GSPN_ERR_DTYPE (-3)    /* dtype is not GSPN_F32 / GSPN_BF16 */
#define GSPN_ERR_ALIGN (-4)    /* a pointer is not 16-byte aligned */
#define GSPN_ERR_GROUP (-5)    /* group_len < 0 */
#define GSPN_ERR_CUDA (-6)     /* a CUDA call failed; see gspn_last_cuda_error() */
#define GSPN_ERR_TIMEOUT (-7)  /* a bounded device-side wait gave up */
#define GSPN_ERR_DIR (-8)      /* direction index outside 0..3 */
#define GSPN_ERR_ALIAS (-9)    /* y overlaps an input */
#define GSPN_ERR_SCRATCH (-10) /* B*C*H*W > GSPN_NOALLOC_MAX_ELEMENTS (gspn_forward_noalloc) */

/*
 * Four-direction GSPN propagation (the operation above):
 *   y = sum_{d=0..3} u[d] (.) h_d(x; wlogit[d], lam[d], group_len).
 * x, y: [B][C][H][W]; wlogit[d]: [B][C][3][H][W]; lam[d], u[d]: [B][C][H][W];
 * group_len: 0 = global scan, g >= 1 = local groups of g lines (g >= the
 * scan length is the global scan); dtype: GSPN_F32 or GSPN_BF16;
 * stream: cudaStream_t.  Returns GSPN_OK or a negative GSPN_ERR_*.
 */
int gspn_forward(const void* x, const void* const wlogit[4], const void* const lam[4],
                 const void* const u[4], int64_t B, int64_t C, int64_t H, int64_t W,
                 int64_t group_len, int dtype, void* stream, void* y);

/*
 * gspn_forward with channel-shared neighbour logits: wlogit[d] is
 * [B][1][3][H][W] and every channel c of batch entry b uses the logits of b.
 * lam[d], u[d], x and y keep their [B][C][H][W] layout.  This is the plain
 * reading of the walkthrough's section "局限性" (the feature dimension of the
 * propagation weights set to 1 to fit memory); it moves 10 + 12/C elements per
 * pixel-channel instead of 22.  Same rules and errors as gspn_forward.
 */
int gspn_forward_shared(const void* x, const void* const wlogit[4], const void* const lam[4],
                        const void* const u[4], int64_t B, int64_t C, int64_t H, int64_t W,
                        int64_t group_len, int dtype, void* stream, void* y);

/*
 * One direction only: y = u (.) h_d(x; wlogit, lam, group_len), with the
 * same layouts, rules and errors as gspn_forward (d in 0..3, else
 * GSPN_ERR_DIR).  Used to test each scan direction on its own.
 */
int gspn_forward_dir(const void* x, const void* wlogit, const void* lam, const void* u,
                     int64_t B, int64_t C, int64_t H, int64_t W, int64_t group_len, int d,
                     int dtype, void* stream, void* y);

/*
 * gspn_forward on HOST buffers: the same operation and layouts, but every
 * pointer is host memory (page-locked memory makes the copies asynchronous).
 * The call copies the inputs to a library-owned device staging area on
 * `stream` (one cudaMemcpyAsync per tensor), runs gspn_forward there, copies
 * y back, and synchronises `stream` before returning, so y is ready on
 * return.  The staging area grows to the largest call and is freed by
 * gspn_release.  Pointers need no alignment.
 */
int gspn_forward_host(const void* x, const void* const wlogit[4], const void* const lam[4],
                      const void* const u[4], int64_t B, int64_t C, int64_t H, int64_t W,
                      int64_t group_len, int dtype, void* stream, void* y);

/*
 * Backward pass (walkthrough section "反向传播"): the gradients of
 * L = sum(gy (.) y) with respect to every input of gspn_forward, where y is
 * gspn_forward's output for the same arguments.
 *   dx[B][C][H][W]; dwlogit[d][B][C][3][H][W] (through the sigmoid and the
 *   border-aware normalisation; 0 for a missing neighbour and on a group's
 *   first line); dlam[d], du[d][B][C][H][W].
 * Same layouts, dtype, alignment and stream rules as gspn_forward; outputs
 * are device memory owned by the caller, overwritten completely, and must
 * not overlap any input or each other (GSPN_ERR_ALIAS).  Arithmetic is fp32;
 * each output is rounded once to the storage dtype.  The library keeps a
 * per-device fp32 workspace of 5 * B*C*H*W floats for it (freed by
 * gspn_release).
 */
int gspn_backward(const void* x, const void* const wlogit[4], const void* const lam[4],
                  const void* const u[4], const void* gy, int64_t B, int64_t C, int64_t H,
                  int64_t W, int64_t group_len, int dtype, void* stream, void* dx,
                  void* const dwlogit[4], void* const dlam[4], void* const du[4]);

/*
 * gspn_forward without any device allocation.  The operation has no
 * counterpart in the GSPN papers or pages: it is a deployment variant of the
 * same computation for callers that cannot call cudaMalloc when they run it
 * -- a process whose device memory is owned by another allocator (a caching
 * allocator or a pool that reserved the GPU up front), or a latency-bound
 * loop that cannot take the device-wide synchronisation of cudaMalloc /
 * cudaFree.
 *
 * Same operation, arguments, layouts, alignment and errors as gspn_forward.
 * It always runs the line-chain kernel (one CTA per plane and direction),
 * accumulating in a fixed fp32 scratch array that is part of the library
 * image (one per device) instead of an allocated workspace; the scratch is
 * zeroed on `stream` at the start of every call.  Limit: B*C*H*W must not
 * exceed GSPN_NOALLOC_MAX_ELEMENTS, else GSPN_ERR_SCRATCH with nothing
 * launched.
 *
 * Concurrency: all calls on one device share that scratch, so calls must not
 * overlap on the GPU -- issue them on one stream, or order them with events.
 * The first call on each device looks the scratch up (and may load the
 * library's device code); make it before any stream capture begins.
 */
#define GSPN_NOALLOC_MAX_ELEMENTS (((int64_t)1) << 23) /* 32 MiB of fp32 */
int gspn_forward_noalloc(const void* x, const void* const wlogit[4], const void* const lam[4],
                         const void* const u[4], int64_t B, int64_t C, int64_t H, int64_t W,
                         int64_t group_len, int dtype, void* stream, void* y);

/* Kernels launched by the most recent successful gspn_forward on this thread. */
int gspn_last_launch_count(void);

/*
 * Profiling hook: while set, every later gspn_forward / gspn_forward_dir call
 * on this thread records `begin` and `end` (cudaEvent_t, owned by the caller)
 * on its stream immediately before and after its dominant kernel, so the
 * caller can time that kernel alone with cudaEventElapsedTime.  Pass NULL,
 * NULL to stop.  Returns GSPN_OK.
 */
int gspn_set_timing_events(void* begin, void* end);

/* Name of the dominant kernel of the most recent successful call on this
 * thread (static storage; "" before the first call). */
const char* gspn_last_kernel_name(void);

/*
 * Synchronises `stream` and reports whether a kernel of this library on the
 * current device gave up a bounded device-side wait (a TMA stage, a halo
 * exchange or a slot hand-over that did not arrive within its time limit).
 * Returns GSPN_OK, or GSPN_ERR_TIMEOUT once per such event (the word is then
 * cleared).  After such an event the large-plane kernel refuses further work
 * (its calls leave y unwritten) until this function has been called; the
 * next call after it starts from a cleared workspace.
 */
int gspn_check_device_status(void* stream);

/*
 * Test hook: the next large-plane launch on this thread waits for a slot
 * hand-over that never happens, gives up after `timeout_ns` nanoseconds and
 * records GSPN_ERR_TIMEOUT for gspn_check_device_status.  No GPU fault is
 * involved.  Returns GSPN_OK, or GSPN_ERR_SHAPE if timeout_ns <= 0.
 */
int gspn_debug_force_timeout(int64_t timeout_ns);

/*
 * Test hook: which kernel takes large planes on this thread from now on.
 * GSPN_PATH_AUTO (the default) and GSPN_PATH_FUSED use the fused kernel and
 * fall back to the line-chain kernel when a plane does not fit its
 * constraints; GSPN_PATH_SWEEP uses the line-sweep kernel (scan line in
 * registers, warp-shuffle neighbours) instead of the fused kernel.  Results
 * agree within the tolerances of the storage dtype.  Returns GSPN_OK, or
 * GSPN_ERR_DIR for an unknown path.
 */
#define GSPN_PATH_AUTO 0
#define GSPN_PATH_FUSED 1
#define GSPN_PATH_SWEEP 2
int gspn_debug_select_path(int path);

/* Frees the current device's workspace and staging area.  Not thread safe
 * against concurrent gspn_* calls on the same device. */
int gspn_release(void);

/* Human-readable text of a status code (static storage). */
const char* gspn_status_string(int status);

/* Text of the last CUDA error seen by the library on this thread. */
const char* gspn_last_cuda_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int gspn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GSPN_B200_H */
