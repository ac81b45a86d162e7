// milo_host.h -- host-side helpers of libmilo: error reporting and checks.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "../../include/milo.h"

namespace milo {

void clear_error();
void set_error(const std::string& msg);

inline milo_status fail(milo_status s, const std::string& msg) {
    set_error(msg);
    return s;
}

inline bool aligned(const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline milo_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(MILO_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return MILO_OK;
}

inline milo_status check_cuda(cudaError_t e, const char* what) {
    if (e != cudaSuccess)
        return fail(MILO_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return MILO_OK;
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Weight rows whose count padded to whole 64-row tiles (the blob's layout)
// still fits the 32-bit row counts of the kernels.
constexpr int32_t kMaxWeightRows = 0x7FFFFFFF - 63;

// Largest K (input features) of a projection the forward calls take: the
// planning's chunk, slice and byte counts of a row stay far inside 32 bits.
constexpr int32_t kMaxProjK = 1 << 24;

// Launch with programmatic stream serialization (see grid_dep_wait in
// milo_device.cuh): the kernel may be scheduled while the previous kernel of
// the stream drains.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace milo
