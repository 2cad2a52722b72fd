// moe_permute_noalloc: the permutation step for callers that cannot hand the
// library a workspace. Some callers are not allowed to allocate device memory
// at all: code running while a CUDA graph is being captured, servers that
// fix their memory budget up front and forbid allocations on the request
// path (cudaMalloc can synchronise the device and fragment memory), and
// plugin hosts whose memory is owned by another allocator. For them this
// entry point takes its scratch from a fixed array in the library's own
// device memory instead of from the caller.
//
// The source pages have no counterpart of this entry point; it computes
// exactly what moe_permute computes, with the same kernels.
//
// The scratch array is a file-scope __device__ array, so every GPU that
// loads the library holds MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES of it until
// the process exits. Host code must not pass the array's name to a kernel:
// on the host that name is only a stand-in, not a device address. The first
// call on each device looks the real address up with cudaGetSymbolAddress
// (with that device current) and caches it; later calls reuse it.
#include <mutex>

#include "../../include/moe_fp8.h"
#include "common.cuh"

namespace moe {

size_t permute_scratch_bytes(int T, int E);
cudaError_t launch_permute(const uint16_t* x, const int32_t* topk_idx, int T, int H, int k, int E, int64_t cap,
                           int masked_max_m, int ld_rows, uint8_t* Aq, float* As, int32_t* counts, int32_t* kept,
                           int32_t* offsets, int32_t* row_src, int32_t* slot_row, void* scratch, int* status,
                           int num_sms, cudaStream_t s);
int* device_status_word();   // api.cu: the status word of the current device, or nullptr
// api.cu: the configuration rules, capacity and row count that moe_permute applies
moe_status_t check_cfg(const moe_config_t* c);
int64_t capacity_of(const moe_config_t* c);
size_t rows_of(const moe_config_t* c);

static __device__ __align__(256) int32_t g_noalloc_scratch[MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES / sizeof(int32_t)];

namespace {

struct NoAllocDevice {
    bool ready = false;
    bool supported = false;
    int num_sms = 0;
    void* scratch = nullptr;   // device address of g_noalloc_scratch on this device
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[64];

moe_status_t noalloc_device(NoAllocDevice** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocDevice& d = g_noalloc_dev[dev];
    if (!d.ready) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
        d.supported = prop.major == 10 && prop.minor == 0;
        d.num_sms = prop.multiProcessorCount;
        if (d.supported) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
            d.scratch = p;
        }
        d.ready = true;
    }
    if (!d.supported) return MOE_ERR_UNSUPPORTED_DEVICE;
    *out = &d;
    return MOE_OK;
}

inline bool ptr16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_permute_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                            uint8_t* Aq, float* As, int32_t* counts, int32_t* kept,
                                            int32_t* offsets, int32_t* row_src, int32_t* slot_row, void* stream) {
    // the same configuration rules as moe_permute (one validator serves both entry points)
    moe_status_t st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    const moe_config_t& c = *cfg;
    const bool masked = c.layout == MOE_LAYOUT_MASKED;
    // the fixed scratch must hold this call's per-chunk counts and bases
    if (permute_scratch_bytes(c.T, c.E) > MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED_SHAPE;
    NoAllocDevice* dev;
    if ((st = noalloc_device(&dev)) != MOE_OK) return st;
    // the status word receives MOE_ERR_CAPACITY from the kernels; without it an overflow would go
    // unreported, so refuse to launch
    int* status = device_status_word();
    if (status == nullptr) return MOE_ERR_CUDA;
    if (!ptr16(x) || !ptr16(topk_idx) || !ptr16(Aq) || !ptr16(As) || !ptr16(counts) || !ptr16(kept) ||
        !ptr16(offsets) || !ptr16(row_src) || !ptr16(slot_row))
        return MOE_ERR_INVALID_ARG;
    if (c.T == 0) return MOE_OK;
    const int64_t cap = capacity_of(cfg);
    const int rows = static_cast<int>(rows_of(cfg));
    // Nothing in the scratch has to start at zero: the count kernel writes every
    // count it holds before the scan reads them, and the scan writes every base.
    const cudaError_t e = launch_permute(static_cast<const uint16_t*>(x), topk_idx, c.T, c.H, c.k, c.E, cap,
                                         masked ? c.masked_max_m : 0, rows, Aq, As, counts, kept, offsets, row_src,
                                         slot_row, dev->scratch, status, dev->num_sms,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
