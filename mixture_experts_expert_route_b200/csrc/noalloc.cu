// noalloc.cu -- moe_align_permute_noalloc: the token permutation for callers
// that cannot allocate device memory or hand over a workspace.
//
// Some callers of a library like this one cannot call cudaMalloc while they
// enqueue work: plugins of an inference runtime that passes them no workspace
// buffer, or latency-critical threads where an allocation (and its possible
// failure) is not allowed.  This entry point needs no workspace: the
// per-chunk expert counts that moe_align_permute keeps in the caller's
// workspace live here in a fixed device array that the library itself holds.
//
// Properties a caller must know:
//   * the array holds kScratchInts int32 counters (256 KB) on every GPU that
//     loads the library, until the process exits;
//   * it bounds the problem: up to T*k = 2048 one CTA does the whole
//     permutation and needs no scratch; above that the assignments are cut
//     into chunks of 512 and ceil(T*k / 512) * E <= kScratchInts must hold,
//     i.e. T*k <= 512 * floor(65536 / E); larger problems return
//     MOE_ERR_WORKSPACE and launch nothing;
//   * the first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) once for that device; make that first call before
//     any stream capture;
//   * every call shares the one array and leaves its contents behind; each
//     call overwrites every counter it reads, so nothing needs clearing, but
//     calls whose work overlaps on the GPU (e.g. on two streams) race.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kScratchInts = 65536;
constexpr int kMaxDevices = 64;

// In host code this name is only a host-side stand-in for the symbol; kernels
// get the device address looked up below.
static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

int32_t* g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

// Device address of the array on the current device (looked up once per device).
cudaError_t scratch_for_current_device(int32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(g_scratch_once[dev], [dev] {
        void* p = nullptr;
        g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_permute_scratch);
        g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    });
    if (g_scratch_err[dev] != cudaSuccess) return g_scratch_err[dev];
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" MOE_API moe_status moe_align_permute_noalloc(
    const int32_t* ids, int T, int k, int E, int block_m, int32_t* counts, int32_t* offsets,
    int32_t* sorted_ids, int32_t* inv_perm, int32_t* tiles, int32_t* num_tiles, int capacity,
    moe_stream_t stream) {
    using namespace moe;
    if (T < 0 || E < 1 || k < 1 || k > E || block_m < 1) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if (!counts || !offsets || !num_tiles || (T > 0 && (!ids || !inv_perm)))
        return MOE_ERR_INVALID_ARG;
    const int need = moe_permute_capacity(T, k, E, block_m);
    if (need < 0) return MOE_ERR_UNSUPPORTED;
    if (capacity < need) return MOE_ERR_WORKSPACE;
    if (capacity > 0 && (!sorted_ids || !tiles)) return MOE_ERR_INVALID_ARG;
    const long A = static_cast<long>(T) * k;
    const long nch = permute_chunks(A);
    if (nch > 1 && nch * E > kScratchInts) return MOE_ERR_WORKSPACE;
    int32_t* scratch = nullptr;
    if (nch > 1 && scratch_for_current_device(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    const cudaError_t e = launch_align_permute(ids, T, k, E, block_m, capacity, counts, offsets,
                                               sorted_ids, inv_perm, tiles, num_tiles, scratch,
                                               nullptr, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
