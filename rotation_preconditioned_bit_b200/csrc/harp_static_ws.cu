// harp_static_ws.cu -- harp_rotate_quantize_static: the fused two-sided
// forward path with its fp32 intermediate in a library-owned device array,
// for callers that cannot allocate device memory themselves.
//
// Who needs it: code that runs inside a host framework which owns all device
// memory (a fixed pool reserved at start-up, an allocator that rejects or
// cannot service further requests), and code on a latency-critical path that
// must not call cudaMalloc, which can synchronise the device. Such a caller
// still passes its input and output tensors; only the scratch intermediate
// moves into this file.
//
// The scratch is one file-scope __device__ array of HARP_STATIC_WORKSPACE_BYTES.
// Every device on which the library's module is loaded holds it until the
// process exits. In host code its name only stands for the symbol; the
// device address is fetched once per device with cudaGetSymbolAddress (with
// that device current) and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "harp.h"
#include "harp_internal.h"

namespace {

constexpr size_t kScratchBytes = HARP_STATIC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float harp_static_scratch[kScratchBytes / sizeof(float)];

std::mutex g_setup_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call per device). Returns a harp_status.
int scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return HARP_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return HARP_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, harp_static_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return HARP_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return HARP_OK;
}

}  // namespace

extern "C" {

int harp_rotate_quantize_static(harp_plan_t left, harp_plan_t right, harp_codebook_t cb,
                                const void *in, int in_dtype, int64_t rows, int64_t cols,
                                uint8_t *codes, uint16_t *scales, float *rotated_out,
                                void *stream) {
    if (!right || !cb) return HARP_ERR_INVALID_ARG;
    // the plans must belong to the current device before its scratch array is picked
    int st = harp::plans_on_current_device(left, right);
    if (st) return st;
    size_t need = 0;
    st = harp_workspace_size(left, right, rows, cols, &need);
    if (st) return st;
    if (need > kScratchBytes) return HARP_ERR_WORKSPACE;
    void *ws = nullptr;
    if (need > 0) {
        st = scratch_address(&ws);
        if (st) return st;
    }
    // The column pass writes every element of the intermediate before the
    // row pass reads it, so the array's previous contents never leak into a
    // result and nothing needs clearing.
    return harp_rotate_quantize(left, right, cb, in, in_dtype, rows, cols, codes, scales,
                                rotated_out, ws, need ? kScratchBytes : 0, stream);
}

}  // extern "C"
