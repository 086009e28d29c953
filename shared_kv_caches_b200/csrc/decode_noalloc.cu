// kvattn_decode_noalloc: decode attention for callers that cannot allocate
// device memory.
//
// Some callers have no way to provide the scratch workspace kvattn_decode
// needs: a serving engine that has already reserved all of HBM for its own
// cache pool and owns every further byte, a plugin host that hands a library
// only its input and output buffers, or a latency-critical path where a
// cudaMalloc (which can synchronise the device) is not acceptable.  This entry
// point runs the same split pass and combine pass with their scratch (device
// error word, per-part lse and outputs) in one file-scope device array of
// kNoallocScratchBytes.  The array belongs to the library image: every GPU
// that loads the library holds it until the process exits.
//
// Set-up: the first call on a device, with that device current, looks up the
// array's device address with cudaGetSymbolAddress (in host code the array's
// name is only a host-side stand-in, not a device address) and keeps it for
// that device.  Make that first call before any stream capture.  With lazy
// module loading (the CUDA default since 12.2) that same first call is also
// when the driver loads this code onto the device and reserves the array, so
// make it before the caller takes the rest of HBM for itself.  The cached
// address is stale after cudaDeviceReset; the library does not notice a reset.
// No call allocates: there is no cudaMalloc, cudaFree or allocating library
// routine on this path.  All calls share the one array and it keeps the last call's
// contents, so calls that overlap on the GPU (different streams, no ordering
// between them) race on it; calls on one stream are ordered and safe.
#include <mutex>

#include "kvattn_internal.cuh"

namespace kvattn {
namespace {

constexpr size_t kNoallocScratchBytes = KVATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once).
int scratch_for_current_device(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return KVATTN_ERR_CUDA;
    if (dev >= kMaxDevices)
        return KVATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return KVATTN_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KVATTN_OK;
}

}  // namespace
}  // namespace kvattn

extern "C" int kvattn_decode_noalloc(int32_t variant, const kvattn_params *p, const void *q_nope,
                                     const void *q_rope, const void *kv_cache,
                                     const int32_t *block_table, const int32_t *seq_lens,
                                     float sm_scale, void *out, float *lse, int32_t *device_error,
                                     void *stream)
{
    using namespace kvattn;
    if (!p)
        return KVATTN_ERR_INVALID_ARG;
    if (device_error && (reinterpret_cast<uintptr_t>(device_error) % 4))
        return KVATTN_ERR_MISALIGNED;
    // Fit the split count into the scratch array: keep the caller's forced
    // count if it fits, else (automatic choice) use fewer parts per context.
    kvattn_params q = *p;
    kvattn_plan plan;
    int st = kvattn_get_plan(variant, &q, &plan);
    if (st)
        return st;
    if (plan.workspace_bytes > kNoallocScratchBytes) {
        if (p->num_splits > 0)
            return KVATTN_ERR_WORKSPACE_TOO_SMALL;
        int splits = plan.num_splits;
        while (plan.workspace_bytes > kNoallocScratchBytes && splits > 1) {
            q.num_splits = --splits;
            st = kvattn_get_plan(variant, &q, &plan);
            if (st)
                return st;
        }
        if (plan.workspace_bytes > kNoallocScratchBytes)
            return KVATTN_ERR_WORKSPACE_TOO_SMALL;
    }
    void *scratch = nullptr;
    st = scratch_for_current_device(&scratch);
    if (st)
        return st;
    // every argument check kvattn_decode makes, before the scratch is touched,
    // so that a refused call enqueues nothing
    Problem pr;
    st = validate_call(variant, &q, q_nope, q_rope, kv_cache, block_table, seq_lens, sm_scale, out, lse,
                       scratch, &pr);
    if (st)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the device error word and the part counters are the only parts of the
    // scratch that must start at zero
    if (cudaMemsetAsync(scratch, 0, (size_t)plan.header_bytes, s) != cudaSuccess)
        return KVATTN_ERR_CUDA;
    st = kvattn_decode(variant, &q, q_nope, q_rope, kv_cache, block_table, seq_lens, sm_scale, out,
                       lse, scratch, kNoallocScratchBytes, stream);
    if (st)
        return st;
    if (device_error &&
        cudaMemcpyAsync(device_error, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return KVATTN_ERR_CUDA;
    return KVATTN_OK;
}
