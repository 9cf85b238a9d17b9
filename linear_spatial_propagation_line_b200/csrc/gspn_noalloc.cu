// Fixed scratch of gspn_forward_noalloc: the line-chain path's fp32
// accumulator, held in a statically sized device array instead of a buffer
// from cudaMalloc.
//
// Some callers cannot allocate device memory at the moment they run the
// operation: a process whose device memory is owned by another allocator
// (a caching allocator or a memory pool that reserved the GPU up front, so a
// cudaMalloc here would fail or fragment it), or a latency-bound loop that
// cannot take the implicit device-wide synchronisation of cudaMalloc /
// cudaFree.  For them the accumulator lives in this file's static array,
// created with the module, so no call of this path allocates.
//
// The array is one per device (one per CUDA context).  Its address is looked
// up once per device, with that device current, and cached; that first
// look-up may load this module, so a caller should make its first call before
// any stream capture begins.  Calls that use the array must not overlap on
// the GPU (two streams, or two host threads on the same device): they would
// share one accumulator.
#include <cuda_runtime.h>

#include <mutex>

#include "gspn_internal.h"

// Largest B*C*H*W a call may use: GSPN_NOALLOC_MAX_ELEMENTS = 2^23 fp32 values
// (32 MiB).
static __device__ __align__(256) float g_noalloc_scratch[gspn::kNoAllocMaxPixch];

namespace gspn {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[kMaxDevices] = {};

}  // namespace

cudaError_t noalloc_scratch(int device, float** scratch) {
    if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[device]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[device] = static_cast<float*>(p);
    }
    *scratch = g_noalloc_ptr[device];
    return cudaSuccess;
}

}  // namespace gspn
