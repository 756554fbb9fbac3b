// Dynamic NVFP4 quantization for callers that cannot allocate device memory.
//
// nvfp4_quantize_dynamic needs a 32-byte device workspace from its caller.
// Some callers have no way to provide one: an inference-engine plugin whose
// execute step is not allowed to allocate, a runtime that hands out all
// device memory from its own arena and exposes no allocator to extensions,
// or a latency-critical loop that must not call cudaMalloc/cudaFree because
// they can synchronise the device.  This entry point keeps the workspace in
// a file-scope device array instead, so the caller passes only its inputs and
// outputs and nothing is allocated, here or in anything it calls.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "api_checks.h"
#include "gemm.h"
#include "nvfp4.h"

namespace {

// Scratch shared by every call on a device; every GPU that loads this
// library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// A host object whose only use is to be a non-NULL workspace argument of the
// shared argument check.
const char g_noalloc_scratch_tag[1] = {0};

static_assert(sizeof(nvfp4::DynWorkspace) <= kNoAllocScratchBytes,
              "the dynamic-quantize workspace must fit the scratch array");

constexpr int kMaxDevices = 64;
// Per device, the array's device address once taken (atomic: host threads
// may make their first calls at the same time; they all store the same value).
std::atomic<void *> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is taken once
// per device with that device current and checked before any kernel sees it.
nvfp4_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return NVFP4_ERR_UNSUPPORTED_DEVICE;
    }
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return NVFP4_ERR_LAUNCH;
        }
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_dynamic_noalloc(const void *x_bf16, int64_t rows,
                                                       int64_t cols, uint8_t *q_out,
                                                       uint8_t *sf_out, float *s_dec_out,
                                                       float *amax_out, nvfp4_stream_t stream) {
    // The same argument and device checks as nvfp4_quantize_dynamic, done
    // first, so a call it would refuse is refused here before anything is
    // enqueued on the shared array (the workspace argument those checks want
    // non-NULL is this library's own array, so any non-NULL stand-in does).
    nvfp4_status st = nvfp4::check_quantize_args(x_bf16, rows, cols, g_noalloc_scratch_tag,
                                                 q_out, sf_out);
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = nvfp4::current_device(&sms);
    if (st != NVFP4_OK) return st;
    // The workspace this call needs does not grow with the tensor; a request
    // for more than the array holds is refused rather than overrunning it.
    if (nvfp4_quantize_dynamic_workspace_bytes() > kNoAllocScratchBytes)
        return NVFP4_ERR_INVALID_ARG;
    void *scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != NVFP4_OK) return st;
    // The array keeps whatever the previous call left; the barrier counter and
    // the amax words must start at zero, so clear them on this stream first.
    if (cudaMemsetAsync(scratch, 0, nvfp4_quantize_dynamic_workspace_bytes(), stream) !=
        cudaSuccess)
        return NVFP4_ERR_LAUNCH;
    return nvfp4_quantize_dynamic(x_bf16, rows, cols, q_out, sf_out, s_dec_out, amax_out, scratch,
                                  stream);
}
