// noalloc.cu -- milo_grouped_linear for callers that cannot allocate device
// memory (see milo_grouped_linear_noalloc in milo.h).
//
// The scratch of the grouped linear lives in a file-scope device buffer of
// MILO_NOALLOC_SCRATCH_BYTES.  Host code cannot use the buffer's name as a
// device address (on the host it is only a stand-in), so the first call on
// each device asks the runtime for the address with that device current and
// caches it; later calls reuse it.  The call then runs the ordinary
// milo_grouped_linear with that buffer as its workspace.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "milo_host.h"

namespace {

constexpr size_t kScratchBytes = MILO_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

using namespace milo;

extern "C" milo_status milo_grouped_linear_noalloc(const milo_linear* lin, const void* x,
                                                   milo_dtype x_dt, int32_t T, int32_t k,
                                                   const int32_t* expert_offsets,
                                                   const int32_t* perm, void* y, milo_dtype y_dt,
                                                   int32_t* dev_status, void* stream) {
    clear_error();
    if (!lin) return fail(MILO_ERR_INVALID_ARG, "milo_grouped_linear_noalloc: NULL layer");
    size_t need = 0;
    milo_status s = milo_linear_workspace_bytes(lin, T, k, &need);
    if (s != MILO_OK) return s;
    if (need > kScratchBytes)
        return fail(MILO_ERR_WORKSPACE,
                    "milo_grouped_linear_noalloc: this call needs " + std::to_string(need) +
                        " bytes of scratch; the built-in buffer holds " + std::to_string(kScratchBytes) +
                        " (use milo_grouped_linear with a caller workspace)");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return check_cuda(e, "milo_grouped_linear_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return fail(MILO_ERR_INVALID_ARG, "milo_grouped_linear_noalloc: device index out of range");
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_addr[dev]) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess || !p)
                return check_cuda(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                                  "milo_grouped_linear_noalloc: cudaGetSymbolAddress");
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return milo_grouped_linear(lin, x, x_dt, T, k, expert_offsets, perm, y, y_dt, scratch, kScratchBytes,
                               dev_status, stream);
}
