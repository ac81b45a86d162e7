// milo_host.h -- host-side helpers of libmilo: error reporting and checks.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

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

}  // namespace milo
