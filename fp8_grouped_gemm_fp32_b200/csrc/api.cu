// The C ABI (include/moe_fp8.h): argument validation on the host, workspace
// carving, the per-device status word and the launch sequence of moe_forward.
// Nothing here allocates device memory or synchronises the host, except
// moe_get_device_status, whose job is to synchronise and read the status.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "../../include/moe_fp8.h"
#include "backward.cuh"
#include "common.cuh"

namespace moe {
cudaError_t launch_router_softmax(const uint16_t* x, const float* Wg, const float* bias, float* logits, int T, int H,
                                  int E, int k, int32_t* topk_idx, float* topk_w, int* status, uint64_t wait_ns,
                                  int num_sms, cudaStream_t s);
cudaError_t launch_router_hash(const int32_t* token_ids, int T, int E, int32_t* topk_idx, float* topk_w,
                               cudaStream_t s);
size_t permute_scratch_bytes(int T, int E);
cudaError_t launch_permute(const uint16_t* x, const int32_t* topk_idx, int T, int H, int k, int E, int64_t cap,
                           int masked_max_m, int ld_rows, uint8_t* Aq, float* As, int32_t* counts, int32_t* kept,
                           int32_t* offsets, int32_t* row_src, int32_t* slot_row, void* scratch, int* status,
                           int num_sms, cudaStream_t s);
cudaError_t launch_grouped_gemm(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                                const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs, int epilogue,
                                void* D, float* Ds, int* status, uint64_t wait_ns, int num_sms, cudaStream_t s,
                                uint16_t* save_ab = nullptr);
cudaError_t launch_grouped_gemm_w4(int E, int N, int K, const uint8_t* A, const float* As, const int32_t* masked_m,
                                   int M_rows, const uint8_t* B, const float* Bs, int epilogue, void* D, float* Ds,
                                   int* status, uint64_t wait_ns, int num_sms, cudaStream_t s);
cudaError_t launch_combine(const uint16_t* O, const int32_t* slot_row, const float* topk_w, int T, int k, int H,
                           uint16_t* y, cudaStream_t s);
cudaError_t launch_selftest_wait(int* status, uint64_t wait_ns, cudaStream_t s);
void set_contig_mode(int mode);
cudaError_t launch_grouped_gemm_kgroup(int E, int M, int N, const uint8_t* A, const float* As, const int32_t* offsets,
                                       int rows_fwd, const uint8_t* B, const float* Bs, void* D, int* status,
                                       uint64_t wait_ns, int num_sms, cudaStream_t s);
cudaError_t launch_slot_lists(const int32_t* topk_idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
                              int32_t* list, int32_t* slot_tmp, void* scratch, int* status, cudaStream_t s);
size_t ep_scratch_bytes(int T, int E);
cudaError_t launch_bwd_dl(const uint16_t* dy, const uint16_t* O, const int32_t* slot_row, const float* topk_w, int T,
                          int k, int H, float* dl, cudaStream_t s);
cudaError_t launch_bwd_dout(const uint16_t* dy, const float* topk_w, const int32_t* row_src, int rows, int k, int H,
                            uint8_t* q, float* sc, cudaStream_t s);
cudaError_t launch_bwd_swiglu(const uint16_t* ab, const uint16_t* dh, const int32_t* row_src, int rows, int I,
                              uint16_t* g, uint8_t* gq, float* gs, cudaStream_t s);
cudaError_t launch_bwd_tquant(int src, bool rows_mode, const TqArgs& a, uint8_t* out, float* os, cudaStream_t s);
cudaError_t launch_bwd_dx(const uint16_t* dxr, const int32_t* slot_row, const int32_t* topk_idx, const float* dl,
                          const float* Wg, int T, int k, int H, uint16_t* dx, cudaStream_t s);
cudaError_t launch_bwd_gate(const uint16_t* x, const float* dl, const int32_t* offsets, const int32_t* list, int E, int k,
                            int H, float* dWg, float* db, cudaStream_t s);
cudaError_t launch_balance_bias(int E, const int32_t* counts, int64_t* load, float* bias, float gamma, int update,
                                cudaStream_t s);

// The device status word (one per device that loads the library).
__device__ int g_status;

// Configuration rules shared by every entry point that takes a moe_config_t (moe_permute and its
// workspace-free twin included), the capacity they imply and the rows of the permuted buffers.
moe_status_t check_cfg(const moe_config_t* c) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->T < 0 || c->H <= 0 || c->I <= 0 || c->E <= 0 || c->k <= 0) return MOE_ERR_INVALID_ARG;
    if (c->H % kGroup || c->I % kGroup || c->H > 16384 || c->I > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->E > MOE_MAX_EXPERTS || c->k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->k > c->E) return MOE_ERR_INVALID_ARG;
    if (c->routing != MOE_ROUTE_SOFTMAX_TOPK && c->routing != MOE_ROUTE_HASH) return MOE_ERR_INVALID_ARG;
    if (c->routing == MOE_ROUTE_HASH && c->k != 1) return MOE_ERR_INVALID_ARG;
    if (c->cap_num < 0 || c->cap_den < 0 || ((c->cap_num == 0) != (c->cap_den == 0))) return MOE_ERR_INVALID_ARG;
    if (c->layout != MOE_LAYOUT_CONTIGUOUS && c->layout != MOE_LAYOUT_MASKED) return MOE_ERR_INVALID_ARG;
    if (c->layout == MOE_LAYOUT_MASKED && (c->masked_max_m <= 0 || c->masked_max_m % 32)) return MOE_ERR_INVALID_ARG;
    if (c->weights != MOE_WEIGHTS_FP8 && c->weights != MOE_WEIGHTS_W4) return MOE_ERR_INVALID_ARG;
    const int64_t rows = c->layout == MOE_LAYOUT_MASKED
                             ? static_cast<int64_t>(c->E) * c->masked_max_m
                             : static_cast<int64_t>(c->T) * c->k + static_cast<int64_t>(c->E) * (kGroup - 1);
    if (rows >= (1ll << 31) / kGroup) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

int64_t capacity_of(const moe_config_t* c) {
    if (c->cap_num == 0) return -1;
    const int64_t R = static_cast<int64_t>(c->T) * c->k;
    return (R + c->E - 1) / c->E * c->cap_num / c->cap_den;
}

size_t rows_of(const moe_config_t* c) {
    if (c->layout == MOE_LAYOUT_MASKED) return static_cast<size_t>(c->E) * c->masked_max_m;
    const size_t r = static_cast<size_t>(c->T) * c->k + static_cast<size_t>(c->E) * (kGroup - 1);
    return (r + kGroup - 1) / kGroup * kGroup;
}


namespace {

constexpr uint64_t kWaitNs = 4000000000ull;   // a legitimate wait never comes near 4 s
constexpr size_t kAlign = 256;

struct DeviceInfo {
    bool ready = false;
    bool supported = false;
    int num_sms = 0;
    int* status = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[64];

moe_status_t device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
        d.supported = prop.major == 10 && prop.minor == 0;
        d.num_sms = prop.multiProcessorCount;
        if (d.supported) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return MOE_ERR_CUDA;
            d.status = static_cast<int*>(p);
        }
        d.ready = true;
    }
    if (!d.supported) return MOE_ERR_UNSUPPORTED_DEVICE;
    *out = &d;
    return MOE_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

size_t route_scratch(const moe_config_t* c) {
    return c->routing == MOE_ROUTE_SOFTMAX_TOPK ? align_up(sizeof(float) * static_cast<size_t>(c->T) * c->E) : 0;
}

// moe_forward's scratch, in carving order
struct FwdWs {
    uint8_t* Aq;
    float* As;
    uint8_t* Hq;
    float* Hs;
    uint16_t* O;
    int32_t* kept;
    int32_t* offsets;
    int32_t* row_src;
    void* step;   // route / permute scratch
    uint16_t* ab; // training workspace only: the up GEMM's gate and up values, bf16 [rows, 2I]
    size_t total;
};

FwdWs carve(const moe_config_t* c, void* base, bool train = false) {
    FwdWs w;
    const size_t rows = rows_of(c);
    uint8_t* p = static_cast<uint8_t*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* q = p ? p + off : nullptr;
        off += align_up(bytes);
        return q;
    };
    w.Aq = take(rows * c->H);
    w.As = reinterpret_cast<float*>(take(sizeof(float) * rows * (c->H / kGroup)));
    w.Hq = take(rows * c->I);
    w.Hs = reinterpret_cast<float*>(take(sizeof(float) * rows * (c->I / kGroup)));
    w.O = reinterpret_cast<uint16_t*>(take(sizeof(uint16_t) * rows * c->H));
    w.kept = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * c->E));
    w.offsets = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (c->E + 1)));
    w.row_src = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * rows));
    w.step = take(std::max(route_scratch(c), align_up(moe::permute_scratch_bytes(c->T, c->E))));
    w.ab = train ? reinterpret_cast<uint16_t*>(take(sizeof(uint16_t) * rows * 2 * c->I)) : nullptr;
    w.total = off;
    return w;
}

inline moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// moe_backward's scratch, in carving order (rows = the forward's contiguous rows, tiles = rows / 128)
struct BwdWs {
    uint8_t* dOq; float* dOs;             // w * dy on kept rows, 1x128 FP8 along H
    uint16_t* dh;                         // dO W2, bf16 [rows, I]
    uint16_t* ab;                         // x W13^T recomputed, bf16 [rows, 2I]
    uint16_t* g; uint8_t* gq; float* gs;  // SwiGLU backward, bf16 and 1x128 FP8 along 2I
    uint16_t* dxr;                        // g W13, bf16 [rows, H]
    float* dl;                            // [T k]
    uint8_t* A2; float* A2s; uint8_t* B2; float* B2s;        // weight-gradient operands of W2
    uint8_t* A13; float* A13s; uint8_t* B13; float* B13s;    // ... and of W13
    int32_t* counts; int32_t* offs; int32_t* list; int32_t* slot_tmp; void* scratch;
    size_t total;
};

BwdWs carve_bwd(const moe_config_t* c, void* base) {
    BwdWs w;
    const size_t rows = rows_of(c), tiles = rows / kGroup, H = c->H, I = c->I, R = static_cast<size_t>(c->T) * c->k;
    uint8_t* p = static_cast<uint8_t*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* q = p ? p + off : nullptr;
        off += align_up(bytes);
        return q;
    };
    w.dOq = take(rows * H);
    w.dOs = reinterpret_cast<float*>(take(4 * rows * (H / kGroup)));
    w.dh = reinterpret_cast<uint16_t*>(take(2 * rows * I));
    w.ab = reinterpret_cast<uint16_t*>(take(2 * rows * 2 * I));
    w.g = reinterpret_cast<uint16_t*>(take(2 * rows * 2 * I));
    w.gq = take(rows * 2 * I);
    w.gs = reinterpret_cast<float*>(take(4 * rows * (2 * I / kGroup)));
    w.dxr = reinterpret_cast<uint16_t*>(take(2 * rows * H));
    w.dl = reinterpret_cast<float*>(take(4 * R));
    w.A2 = take(rows * H);
    w.A2s = reinterpret_cast<float*>(take(4 * tiles * H));
    w.B2 = take(rows * I);
    w.B2s = reinterpret_cast<float*>(take(4 * tiles * (I / kGroup)));
    w.A13 = take(rows * 2 * I);
    w.A13s = reinterpret_cast<float*>(take(4 * tiles * 2 * I));
    w.B13 = take(rows * H);
    w.B13s = reinterpret_cast<float*>(take(4 * tiles * (H / kGroup)));
    w.counts = reinterpret_cast<int32_t*>(take(4 * static_cast<size_t>(c->E)));
    w.offs = reinterpret_cast<int32_t*>(take(4 * (static_cast<size_t>(c->E) + 1)));
    w.list = reinterpret_cast<int32_t*>(take(4 * R));
    w.slot_tmp = reinterpret_cast<int32_t*>(take(4 * R));
    w.scratch = take(ep_scratch_bytes(c->T, c->E));
    w.total = off;
    return w;
}

}  // namespace

// The current device's status word (for moe_permute_noalloc in its own file); nullptr if unavailable.
int* device_status_word() {
    DeviceInfo* dev;
    return device_info(&dev) == MOE_OK ? dev->status : nullptr;
}

// The current device's SM count and status word, for entry points defined in other files.
moe_status_t current_device(int* num_sms, int** status) {
    DeviceInfo* dev;
    const moe_status_t st = device_info(&dev);
    if (st != MOE_OK) return st;
    *num_sms = dev->num_sms;
    *status = dev->status;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_rows_capacity(const moe_config_t* cfg) {
    if (check_cfg(cfg) != MOE_OK) return 0;
    return rows_of(cfg);
}

size_t moe_workspace_size(const moe_config_t* cfg, int for_forward) {
    if (check_cfg(cfg) != MOE_OK || for_forward < 0 || for_forward > 2) return 0;
    // the training forward takes what the backward takes: contiguous layout, E4M3 weights, softmax routing
    if (for_forward == 2 && (cfg->layout != MOE_LAYOUT_CONTIGUOUS || cfg->weights != MOE_WEIGHTS_FP8 ||
                             cfg->routing != MOE_ROUTE_SOFTMAX_TOPK))
        return 0;
    if (for_forward) return carve(cfg, nullptr, for_forward == 2).total;
    return std::max(route_scratch(cfg), align_up(permute_scratch_bytes(cfg->T, cfg->E)));
}

moe_status_t moe_route(const moe_config_t* cfg, const void* x, const float* Wg, const float* bias,
                       const int32_t* token_ids, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                       void* stream) {
    moe_status_t st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    if (cfg->T == 0) return MOE_OK;                       // no tokens: nothing is read or written
    if (!ptr_ok(topk_idx) || !ptr_ok(topk_w)) return MOE_ERR_INVALID_ARG;
    if (cfg->routing == MOE_ROUTE_HASH) {
        if (!ptr_ok(token_ids)) return MOE_ERR_INVALID_ARG;
    } else {
        if (!ptr_ok(x) || !ptr_ok(Wg) || (bias && !aligned16(bias)) || !ptr_ok(ws)) return MOE_ERR_INVALID_ARG;
        if (ws_bytes < route_scratch(cfg)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    }
    if (cfg->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cfg->routing == MOE_ROUTE_HASH)
        return cuda_status(launch_router_hash(token_ids, cfg->T, cfg->E, topk_idx, topk_w, s));
    return cuda_status(launch_router_softmax(static_cast<const uint16_t*>(x), Wg, bias, static_cast<float*>(ws),
                                             cfg->T, cfg->H, cfg->E, cfg->k, topk_idx, topk_w, dev->status, kWaitNs,
                                             dev->num_sms, s));
}

moe_status_t moe_permute(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, uint8_t* Aq, float* As,
                         int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_src, int32_t* slot_row,
                         void* ws, size_t ws_bytes, void* stream) {
    moe_status_t st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    if (!ptr_ok(x) || !ptr_ok(topk_idx) || !ptr_ok(Aq) || !ptr_ok(As) || !ptr_ok(counts) || !ptr_ok(kept) ||
        !ptr_ok(offsets) || !ptr_ok(row_src) || !ptr_ok(slot_row) || !ptr_ok(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < permute_scratch_bytes(cfg->T, cfg->E)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (cfg->T == 0) return MOE_OK;
    const bool masked = cfg->layout == MOE_LAYOUT_MASKED;
    return cuda_status(launch_permute(static_cast<const uint16_t*>(x), topk_idx, cfg->T, cfg->H, cfg->k, cfg->E,
                                      capacity_of(cfg), masked ? cfg->masked_max_m : 0,
                                      static_cast<int>(rows_of(cfg)), Aq, As, counts, kept, offsets, row_src,
                                      slot_row, ws, dev->status, dev->num_sms, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_gemm_fp8(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                                  const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                                  int epilogue, void* D, float* Ds, void* stream) {
    if (layout != MOE_LAYOUT_CONTIGUOUS && layout != MOE_LAYOUT_MASKED) return MOE_ERR_INVALID_ARG;
    if (epilogue != MOE_EPI_BF16 && epilogue != MOE_EPI_SWIGLU_FP8) return MOE_ERR_INVALID_ARG;
    if (E <= 0 || N <= 0 || K <= 0 || M_rows <= 0) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS || N % kGroup || K % kGroup) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (epilogue == MOE_EPI_SWIGLU_FP8 && N % (2 * kGroup)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (K > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (layout == MOE_LAYOUT_MASKED && M_rows % 32) return MOE_ERR_INVALID_ARG;
    if (layout == MOE_LAYOUT_CONTIGUOUS && M_rows % 4) return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(E) * N >= (1ll << 31) || static_cast<int64_t>(E) * M_rows >= (1ll << 31))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!ptr_ok(A) || !ptr_ok(As) || !ptr_ok(group_info) || !ptr_ok(B) || !ptr_ok(Bs) || !ptr_ok(D))
        return MOE_ERR_INVALID_ARG;
    if (epilogue == MOE_EPI_SWIGLU_FP8 && !ptr_ok(Ds)) return MOE_ERR_INVALID_ARG;
    moe_status_t st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    return cuda_status(launch_grouped_gemm(layout, E, N, K, A, As, group_info, M_rows, B, Bs, epilogue, D, Ds,
                                           dev->status, kWaitNs, dev->num_sms, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_gemm_w4(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                                 const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                                 int epilogue, void* D, float* Ds, void* stream) {
    if (layout != MOE_LAYOUT_CONTIGUOUS && layout != MOE_LAYOUT_MASKED) return MOE_ERR_INVALID_ARG;
    if (epilogue != MOE_EPI_BF16 && epilogue != MOE_EPI_SWIGLU_FP8) return MOE_ERR_INVALID_ARG;
    if (E <= 0 || N <= 0 || K <= 0 || M_rows <= 0) return MOE_ERR_INVALID_ARG;
    if (layout != MOE_LAYOUT_MASKED) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (E > MOE_MAX_EXPERTS || N % kGroup || K % kGroup) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (epilogue == MOE_EPI_SWIGLU_FP8 && N % (2 * kGroup)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (K > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (M_rows % 32) return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(E) * N >= (1ll << 31) || static_cast<int64_t>(E) * M_rows >= (1ll << 31))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!ptr_ok(A) || !ptr_ok(As) || !ptr_ok(group_info) || !ptr_ok(B) || !ptr_ok(Bs) || !ptr_ok(D))
        return MOE_ERR_INVALID_ARG;
    if (epilogue == MOE_EPI_SWIGLU_FP8 && !ptr_ok(Ds)) return MOE_ERR_INVALID_ARG;
    moe_status_t st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    return cuda_status(launch_grouped_gemm_w4(E, N, K, A, As, group_info, M_rows, B, Bs, epilogue, D, Ds, dev->status,
                                              kWaitNs, dev->num_sms, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_combine(const moe_config_t* cfg, const void* O, const int32_t* slot_row, const float* topk_w,
                         void* y, void* stream) {
    moe_status_t st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    if (cfg->T == 0) return MOE_OK;                       // no tokens: nothing is read or written
    if (!ptr_ok(O) || !ptr_ok(slot_row) || !ptr_ok(topk_w) || !ptr_ok(y)) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_combine(static_cast<const uint16_t*>(O), slot_row, topk_w, cfg->T, cfg->k, cfg->H,
                                      static_cast<uint16_t*>(y), static_cast<cudaStream_t>(stream)));
}

static moe_status_t forward_impl(const moe_config_t* cfg, const void* x, const float* Wg, const float* bias,
                                 const int32_t* token_ids, const uint8_t* W13, const float* S13, const uint8_t* W2,
                                 const float* S2, void* y, int32_t* topk_idx, float* topk_w, int32_t* counts,
                                 int32_t* slot_row, void* ws, size_t ws_bytes, void* stream, bool train) {
    moe_status_t st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    if (train && (cfg->layout != MOE_LAYOUT_CONTIGUOUS || cfg->weights != MOE_WEIGHTS_FP8 ||
                  cfg->routing != MOE_ROUTE_SOFTMAX_TOPK))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    if (!ptr_ok(x) || !ptr_ok(W13) || !ptr_ok(S13) || !ptr_ok(W2) || !ptr_ok(S2) || !ptr_ok(y) || !ptr_ok(topk_idx) ||
        !ptr_ok(topk_w) || !ptr_ok(counts) || !ptr_ok(slot_row) || !ptr_ok(ws) || (ws && (reinterpret_cast<uintptr_t>(ws) % kAlign)))
        return MOE_ERR_INVALID_ARG;
    if (cfg->routing == MOE_ROUTE_SOFTMAX_TOPK && (!ptr_ok(Wg) || (bias && !aligned16(bias))))
        return MOE_ERR_INVALID_ARG;
    if (cfg->routing == MOE_ROUTE_HASH && !ptr_ok(token_ids)) return MOE_ERR_INVALID_ARG;
    if (cfg->weights == MOE_WEIGHTS_W4 && cfg->layout != MOE_LAYOUT_MASKED) return MOE_ERR_UNSUPPORTED_SHAPE;
    const FwdWs w = carve(cfg, ws, train);
    if (ws_bytes < w.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (cfg->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool masked = cfg->layout == MOE_LAYOUT_MASKED;
    const int rows = static_cast<int>(rows_of(cfg));
    const int M_rows = masked ? cfg->masked_max_m : rows;
    const int32_t* group = masked ? w.kept : w.offsets;
    cudaError_t e;
    if (cfg->routing == MOE_ROUTE_HASH)
        e = launch_router_hash(token_ids, cfg->T, cfg->E, topk_idx, topk_w, s);
    else
        e = launch_router_softmax(static_cast<const uint16_t*>(x), Wg, bias, static_cast<float*>(w.step), cfg->T,
                                  cfg->H, cfg->E, cfg->k, topk_idx, topk_w, dev->status, kWaitNs, dev->num_sms, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_permute(static_cast<const uint16_t*>(x), topk_idx, cfg->T, cfg->H, cfg->k, cfg->E, capacity_of(cfg),
                       masked ? cfg->masked_max_m : 0, rows, w.Aq, w.As, counts, w.kept, w.offsets, w.row_src,
                       slot_row, w.step, dev->status, dev->num_sms, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (cfg->weights == MOE_WEIGHTS_W4) {
        e = launch_grouped_gemm_w4(cfg->E, 2 * cfg->I, cfg->H, w.Aq, w.As, group, M_rows, W13, S13, MOE_EPI_SWIGLU_FP8,
                                   w.Hq, w.Hs, dev->status, kWaitNs, dev->num_sms, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        e = launch_grouped_gemm_w4(cfg->E, cfg->H, cfg->I, w.Hq, w.Hs, group, M_rows, W2, S2, MOE_EPI_BF16, w.O,
                                   nullptr, dev->status, kWaitNs, dev->num_sms, s);
    } else {
        e = launch_grouped_gemm(cfg->layout, cfg->E, 2 * cfg->I, cfg->H, w.Aq, w.As, group, M_rows, W13, S13,
                                MOE_EPI_SWIGLU_FP8, w.Hq, w.Hs, dev->status, kWaitNs, dev->num_sms, s, w.ab);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        e = launch_grouped_gemm(cfg->layout, cfg->E, cfg->H, cfg->I, w.Hq, w.Hs, group, M_rows, W2, S2, MOE_EPI_BF16,
                                w.O, nullptr, dev->status, kWaitNs, dev->num_sms, s);
    }
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_combine(w.O, slot_row, topk_w, cfg->T, cfg->k, cfg->H, static_cast<uint16_t*>(y), s);
    return cuda_status(e);
}

moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const float* Wg, const float* bias,
                         const int32_t* token_ids, const uint8_t* W13, const float* S13, const uint8_t* W2,
                         const float* S2, void* y, int32_t* topk_idx, float* topk_w, int32_t* counts,
                         int32_t* slot_row, void* ws, size_t ws_bytes, void* stream) {
    return forward_impl(cfg, x, Wg, bias, token_ids, W13, S13, W2, S2, y, topk_idx, topk_w, counts, slot_row, ws,
                        ws_bytes, stream, false);
}

moe_status_t moe_forward_train(const moe_config_t* cfg, const void* x, const float* Wg, const float* bias,
                               const int32_t* token_ids, const uint8_t* W13, const float* S13, const uint8_t* W2,
                               const float* S2, void* y, int32_t* topk_idx, float* topk_w, int32_t* counts,
                               int32_t* slot_row, void* ws, size_t ws_bytes, void* stream) {
    return forward_impl(cfg, x, Wg, bias, token_ids, W13, S13, W2, S2, y, topk_idx, topk_w, counts, slot_row, ws,
                        ws_bytes, stream, true);
}

// What moe_backward takes beyond a valid configuration: contiguous layout, E4M3 weights, softmax routing, and
// K of the weight-gradient GEMMs (an expert's rows; 2I for g W13) within the 128 K blocks they stage.
static moe_status_t check_backward_shape(const moe_config_t* cfg) {
    if (cfg->layout != MOE_LAYOUT_CONTIGUOUS || cfg->weights != MOE_WEIGHTS_FP8 ||
        cfg->routing != MOE_ROUTE_SOFTMAX_TOPK)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    const int64_t most = cfg->cap_num ? std::min<int64_t>(cfg->T, capacity_of(cfg)) : cfg->T;
    if (most > 16384 || 2 * cfg->I > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

size_t moe_backward_workspace_size(const moe_config_t* cfg) {
    if (check_cfg(cfg) != MOE_OK || check_backward_shape(cfg) != MOE_OK) return 0;
    return carve_bwd(cfg, nullptr).total;
}

moe_status_t moe_backward(const moe_config_t* cfg, const void* x, const float* Wg, const uint8_t* W13, const float* S13,
                          const uint8_t* W13T, const float* S13T, const uint8_t* W2T, const float* S2T,
                          const int32_t* topk_idx, const float* topk_w, const int32_t* slot_row, const void* fwd_ws,
                          int fwd_train, const void* dy, void* dx, float* dWg, float* db, void* dW13, void* dW2,
                          void* ws, size_t ws_bytes, void* stream) {
    moe_status_t st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_backward_shape(cfg)) != MOE_OK) return st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    if (cfg->T == 0) return MOE_OK;
    if (!ptr_ok(x) || !ptr_ok(Wg) || !ptr_ok(W13) || !ptr_ok(S13) || !ptr_ok(W13T) || !ptr_ok(S13T) || !ptr_ok(W2T) ||
        !ptr_ok(S2T) || !ptr_ok(topk_idx) || !ptr_ok(topk_w) || !ptr_ok(slot_row) || !ptr_ok(fwd_ws) || !ptr_ok(dy) ||
        !ptr_ok(dx) || !ptr_ok(dWg) || !ptr_ok(db) || !ptr_ok(dW13) || !ptr_ok(dW2) || !ptr_ok(ws) ||
        (reinterpret_cast<uintptr_t>(ws) % kAlign) || (reinterpret_cast<uintptr_t>(fwd_ws) % kAlign))
        return MOE_ERR_INVALID_ARG;
    const BwdWs b = carve_bwd(cfg, ws);
    if (ws_bytes < b.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (fwd_train != 0 && fwd_train != 1) return MOE_ERR_INVALID_ARG;
    const FwdWs f = carve(cfg, const_cast<void*>(fwd_ws), fwd_train != 0);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = cfg->T, k = cfg->k, H = cfg->H, I = cfg->I, E = cfg->E;
    const int rows = static_cast<int>(rows_of(cfg));
    const uint16_t* dy16 = static_cast<const uint16_t*>(dy);
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    // gate: dw, dl; expert path: dO, dh, a|b, g, dx rows, dx
    if (!ok(launch_bwd_dl(dy16, f.O, slot_row, topk_w, T, k, H, b.dl, s))) return MOE_ERR_CUDA;
    if (!ok(launch_bwd_dout(dy16, topk_w, f.row_src, rows, k, H, b.dOq, b.dOs, s))) return MOE_ERR_CUDA;
    if (!ok(launch_grouped_gemm(MOE_LAYOUT_CONTIGUOUS, E, I, H, b.dOq, b.dOs, f.offsets, rows, W2T, S2T, MOE_EPI_BF16,
                                b.dh, nullptr, dev->status, kWaitNs, dev->num_sms, s)))
        return MOE_ERR_CUDA;
    // a | b: saved by moe_forward_train, else recomputed (the same kernel arithmetic, so the same values)
    const uint16_t* ab = f.ab;
    if (!fwd_train) {
        if (!ok(launch_grouped_gemm(MOE_LAYOUT_CONTIGUOUS, E, 2 * I, H, f.Aq, f.As, f.offsets, rows, W13, S13,
                                    MOE_EPI_BF16, b.ab, nullptr, dev->status, kWaitNs, dev->num_sms, s)))
            return MOE_ERR_CUDA;
        ab = b.ab;
    }
    if (!ok(launch_bwd_swiglu(ab, b.dh, f.row_src, rows, I, b.g, b.gq, b.gs, s))) return MOE_ERR_CUDA;
    if (!ok(launch_grouped_gemm(MOE_LAYOUT_CONTIGUOUS, E, H, 2 * I, b.gq, b.gs, f.offsets, rows, W13T, S13T,
                                MOE_EPI_BF16, b.dxr, nullptr, dev->status, kWaitNs, dev->num_sms, s)))
        return MOE_ERR_CUDA;
    if (!ok(launch_bwd_dx(b.dxr, slot_row, topk_idx, b.dl, Wg, T, k, H, static_cast<uint16_t*>(dx), s)))
        return MOE_ERR_CUDA;
    // gate gradients over every slot of each expert, in token order
    if (!ok(launch_slot_lists(topk_idx, T, k, E, b.counts, b.offs, b.list, b.slot_tmp, b.scratch, dev->status, s)))
        return MOE_ERR_CUDA;
    if (!ok(launch_bwd_gate(static_cast<const uint16_t*>(x), b.dl, b.offs, b.list, E, k, H, dWg, db, s)))
        return MOE_ERR_CUDA;
    // weight gradients: per forward row tile, the transposed operands, then the K-grouped GEMMs
    TqArgs a{dy16, topk_w, nullptr, nullptr, nullptr, f.row_src, rows, k, H};
    if (!ok(launch_bwd_tquant(0, true, a, b.A2, b.A2s, s))) return MOE_ERR_CUDA;
    a.codes = f.Hq; a.scales = f.Hs; a.C = I;
    if (!ok(launch_bwd_tquant(1, false, a, b.B2, b.B2s, s))) return MOE_ERR_CUDA;
    a.bf = b.g; a.C = 2 * I;
    if (!ok(launch_bwd_tquant(2, true, a, b.A13, b.A13s, s))) return MOE_ERR_CUDA;
    a.codes = f.Aq; a.scales = f.As; a.C = H;
    if (!ok(launch_bwd_tquant(1, false, a, b.B13, b.B13s, s))) return MOE_ERR_CUDA;
    if (!ok(launch_grouped_gemm_kgroup(E, H, I, b.A2, b.A2s, f.offsets, rows, b.B2, b.B2s, dW2, dev->status, kWaitNs,
                                       dev->num_sms, s)))
        return MOE_ERR_CUDA;
    if (!ok(launch_grouped_gemm_kgroup(E, 2 * I, H, b.A13, b.A13s, f.offsets, rows, b.B13, b.B13s, dW13, dev->status,
                                       kWaitNs, dev->num_sms, s)))
        return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status_t moe_balance_bias(int E, const int32_t* counts, int64_t* load, float* bias, float gamma, int update,
                              void* stream) {
    if (E <= 0) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!ptr_ok(counts) || !ptr_ok(load) || !ptr_ok(bias) || !isfinite(gamma)) return MOE_ERR_INVALID_ARG;
    moe_status_t st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    return cuda_status(launch_balance_bias(E, counts, load, bias, gamma, update != 0, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_set_contig_kernel(int form) {
    if (form != MOE_CONTIG_AUTO && form != MOE_CONTIG_SINGLE && form != MOE_CONTIG_PAIR) return MOE_ERR_INVALID_ARG;
    set_contig_mode(form);
    return MOE_OK;
}

moe_status_t moe_get_device_status(void* stream) {
    moe_status_t st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    const int zero = 0;
    if (cudaMemcpy(&v, dev->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(dev->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    return static_cast<moe_status_t>(v);
}

moe_status_t moe_selftest_wait_timeout(int limit_us, void* stream) {
    if (limit_us < 0) return MOE_ERR_INVALID_ARG;
    moe_status_t st;
    DeviceInfo* dev;
    if ((st = device_info(&dev)) != MOE_OK) return st;
    return cuda_status(launch_selftest_wait(dev->status, static_cast<uint64_t>(limit_us) * 1000ull,
                                            static_cast<cudaStream_t>(stream)));
}

const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MOE_ERR_UNSUPPORTED_DEVICE: return "FP8 not supported on this GPU (needs sm_100)";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_CAPACITY: return "a group had more rows than its bound (masked_max_m or M_rows)";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    }
    return "unknown status";
}

}  // extern "C"
