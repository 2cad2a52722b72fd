// Expert parallelism: the layer's dispatch and combine across GPUs, one process per GPU (TP-MoE page,
// sections 3.3 and 4.1 step 3: each card routes its own tokens and all-to-all carries them to the card
// that holds their expert and back; MegaMoE page, 3.4: dispatch and combine as the two primitives;
// TP-MoE page, 6.2: FP8 payload). The collectives themselves are the caller's (NCCL through
// torch.distributed); this file holds the exchange plan and the device steps around them:
//
//   moe_ep_plan      (host) from every rank's per-expert counts: what each rank keeps, sends and
//                    receives, and where each received block lands in the owner's grouped layout;
//   moe_ep_count     per-expert counts and in-chunk ranks of this rank's slots (permute.cu kernels);
//   moe_ep_dispatch  FP8 send rows, one per kept slot, quantised once per token (permute.cu kernels);
//   moe_ep_receive   received rows -> the contiguous grouped layout of the local experts;
//   moe_ep_return    the local experts' output rows -> receive order, for the way back.
//
// Ranks within an expert follow the global token order (rank 0's tokens first), so the capacity drop
// and every row's place equal those of one GPU running the concatenated batch.
#include <string.h>

#include <algorithm>
#include <vector>

#include "../../include/moe_fp8.h"
#include "common.cuh"

namespace moe {

moe_status_t check_cfg(const moe_config_t* c);
moe_status_t current_device(int* num_sms, int** status);
size_t ep_scratch_bytes(int T, int E);
int64_t ep_row_bytes(int H);
cudaError_t launch_ep_count(const int32_t* topk_idx, int T, int k, int E, int32_t* counts, void* scratch,
                            int* status, cudaStream_t s);
cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* topk_idx, int T, int H, int k, int E,
                               const int32_t* kept_mine, const int32_t* send_off, uint8_t* send, int32_t* slot_row,
                               void* scratch, int num_sms, cudaStream_t s);

// One warp per received row: the block b (source, local expert) that holds it (binary search over the
// blocks' first receive rows, which rise in receive order), its grouped row = the block's first grouped
// row + its place in the block; codes are copied in 16-byte pieces, scales to the K-block-major layout.
// Warps then fill the padding rows of each local expert (code 0, scale 1). chunk < 0: every row and
// expert (rows_recv must be the plan's); otherwise the rows and experts of that chunk, offsets written
// less the chunk's first expert's. A plan whose sizes disagree with the call's is reported
// (MOE_ERR_CAPACITY) and nothing is written.
__global__ void __launch_bounds__(256) ep_receive_kernel(const moe_ep_plan_t* __restrict__ plan, int H, int rows_recv,
                                                         int chunk, const uint8_t* __restrict__ recv, int64_t row_bytes,
                                                         uint8_t* __restrict__ Aq, float* __restrict__ As,
                                                         int M_rows, int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ group_row, int* status) {
    __shared__ int32_t rs[kMaxE + 1];
    __shared__ int32_t gs[kMaxE];
    __shared__ int32_t off_s[kMaxE + 1];
    __shared__ int32_t kept_s[kMaxE];
    const int El = plan->E_local, G = plan->G;
    const int nb = G * El;
    const int C = plan->chunks;
    bool bad = plan->rows_group > M_rows || nb > kMaxE || El > kMaxE || C < 1 || C > MOE_EP_MAX_CHUNKS;
    int64_t r0 = 0, r1 = plan->rows_recv;
    int e0 = 0, e1 = El;
    if (chunk < 0) {
        bad |= plan->rows_recv != rows_recv;
    } else if (chunk >= C) {
        bad = true;
    } else if (!bad) {
        r0 = plan->recv_chunk[chunk];
        r1 = plan->recv_chunk[chunk + 1];
        e0 = plan->chunk_first[chunk];
        e1 = plan->chunk_first[chunk + 1];
        bad |= r0 < 0 || r1 < r0 || r1 > plan->rows_recv || e0 < 0 || e1 < e0 || e1 > El;
    }
    if (bad) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, kStatusCapacity);
        return;
    }
    for (int b = threadIdx.x; b <= nb; b += blockDim.x) {
        rs[b] = plan->recv_start[b];
        if (b < nb) gs[b] = plan->group_start[b];
    }
    for (int e = threadIdx.x; e <= El; e += blockDim.x) {
        off_s[e] = plan->offsets[e];
        if (e < El) kept_s[e] = plan->kept[e];
    }
    __syncthreads();
    if (blockIdx.x == 0)
        for (int e = e0 + threadIdx.x; e <= e1; e += blockDim.x) offsets[e - e0] = off_s[e] - off_s[e0];
    const int lane = threadIdx.x & 31;
    const int G128 = H / kGroup;
    const int64_t wid = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t i = r0 + wid; i < r1; i += nw) {
        int lo = 0, hi = nb - 1;              // largest b with rs[b] <= i
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (rs[mid] <= i) lo = mid; else hi = mid - 1;
        }
        const int64_t gr = gs[lo] + (i - rs[lo]);
        const uint4* src = reinterpret_cast<const uint4*>(recv + i * row_bytes);
        uint4* dst = reinterpret_cast<uint4*>(Aq + gr * H);
        for (int c = lane; c < H / 16; c += 32) dst[c] = src[c];
        const float* ssrc = reinterpret_cast<const float*>(recv + i * row_bytes + H);
        for (int g = lane; g < G128; g += 32) As[static_cast<int64_t>(g) * M_rows + gr] = ssrc[g];
        if (lane == 0) group_row[i] = static_cast<int32_t>(gr);
    }
    // padding rows: (expert, row within its last tile) items, at most 127 per expert
    for (int64_t w = wid; w < static_cast<int64_t>(e1 - e0) * kGroup; w += nw) {
        const int e = e0 + static_cast<int>(w / kGroup);
        const int64_t r = off_s[e] + kept_s[e] + (w % kGroup);
        if (r >= off_s[e + 1]) continue;
        uint4* dst = reinterpret_cast<uint4*>(Aq + r * H);
        for (int c = lane; c < H / 16; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
        for (int g = lane; g < G128; g += 32) As[static_cast<int64_t>(g) * M_rows + r] = 1.0f;
    }
}

// ret[i] = O[group_row[i]] (bf16 rows of H), one warp per row, 16-byte pieces.
__global__ void __launch_bounds__(256) ep_return_kernel(int H, int rows, const uint16_t* __restrict__ O,
                                                        const int32_t* __restrict__ group_row,
                                                        uint16_t* __restrict__ ret) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t i = wid; i < rows; i += nw) {
        const uint4* src = reinterpret_cast<const uint4*>(O + static_cast<int64_t>(group_row[i]) * H);
        uint4* dst = reinterpret_cast<uint4*>(ret + i * H);
        for (int c = lane; c < H / 8; c += 32) dst[c] = src[c];
    }
}

namespace {
inline bool ptr16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int warp_blocks(int64_t warps, int num_sms) {
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((warps + 7) / 8, static_cast<int64_t>(num_sms) * 8)));
}
}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status_t moe_ep_plan_chunked(int G, int rank, int E, int64_t T_total, int k, int cap_num, int cap_den,
                                 const int32_t* counts_all, int chunks, moe_ep_plan_t* plan) {
    if (!plan || !counts_all) return MOE_ERR_INVALID_ARG;
    if (G < 1 || G > MOE_EP_MAX_RANKS || rank < 0 || rank >= G) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > MOE_MAX_EXPERTS || E % G) return MOE_ERR_INVALID_ARG;
    if (T_total < 0 || k < 1 || k > MOE_MAX_TOPK || k > E) return MOE_ERR_INVALID_ARG;
    if (cap_num < 0 || cap_den < 0 || ((cap_num == 0) != (cap_den == 0))) return MOE_ERR_INVALID_ARG;
    const int El = E / G;
    if (chunks < 1 || chunks > MOE_EP_MAX_CHUNKS || chunks > El) return MOE_ERR_INVALID_ARG;
    // per expert, slot counts of all ranks; keep[s][e] = rank s's kept slots of e (global token order)
    int64_t cap = -1;
    if (cap_num) cap = (T_total * k + E - 1) / E * cap_num / cap_den;
    std::vector<int32_t> keep(static_cast<size_t>(G) * E);
    for (int e = 0; e < E; ++e) {
        int64_t prefix = 0;
        for (int s = 0; s < G; ++s) {
            const int64_t c = counts_all[static_cast<size_t>(s) * E + e];
            if (c < 0) return MOE_ERR_INVALID_ARG;
            const int64_t kk = cap < 0 ? c : std::min<int64_t>(c, std::max<int64_t>(0, cap - prefix));
            keep[static_cast<size_t>(s) * E + e] = static_cast<int32_t>(kk);
            prefix += c;
        }
    }
    memset(plan, 0, sizeof(*plan));
    plan->G = G;
    plan->rank = rank;
    plan->E = E;
    plan->E_local = El;
    plan->cap = cap < 0 ? -1 : static_cast<int32_t>(std::min<int64_t>(cap, (1ll << 31) - 1));
    plan->chunks = chunks;
    for (int c = 0; c <= chunks; ++c) plan->chunk_first[c] = c * El / chunks;
    const int64_t limit = (1ll << 31) / kGroup;
    for (int e = 0; e < E; ++e) plan->kept_mine[e] = keep[static_cast<size_t>(rank) * E + e];
    // send rows in (chunk, destination, expert, token) order
    int64_t send = 0;
    for (int c = 0; c < chunks; ++c) {
        plan->send_chunk[c] = static_cast<int32_t>(send);
        for (int d = 0; d < G; ++d)
            for (int l = plan->chunk_first[c]; l < plan->chunk_first[c + 1]; ++l) {
                const int e = d * El + l;
                plan->send_off[e] = static_cast<int32_t>(send);
                plan->send_rows_c[c][d] += plan->kept_mine[e];
                plan->send_rows[d] += plan->kept_mine[e];
                send += plan->kept_mine[e];
            }
        if (send >= limit) return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    plan->send_chunk[chunks] = static_cast<int32_t>(send);
    // grouped rows in (local expert, source, token) order, each expert padded to whole 128-row tiles
    std::vector<int32_t> gstart(static_cast<size_t>(G) * El);
    int64_t grow = 0;
    for (int l = 0; l < El; ++l) {
        int64_t tot = 0;
        for (int s = 0; s < G; ++s) tot += keep[static_cast<size_t>(s) * E + rank * El + l];
        plan->kept[l] = static_cast<int32_t>(tot);
        plan->offsets[l] = static_cast<int32_t>(grow);
        int64_t g = grow;
        for (int s = 0; s < G; ++s) {
            gstart[static_cast<size_t>(s) * El + l] = static_cast<int32_t>(g);
            g += keep[static_cast<size_t>(s) * E + rank * El + l];
        }
        grow += (tot + kGroup - 1) / kGroup * kGroup;
        if (grow >= limit) return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    plan->offsets[El] = static_cast<int32_t>(grow);
    // blocks (source, local expert) in receive order: (chunk, source, local expert, token)
    int64_t rrow = 0;
    int b = 0;
    for (int c = 0; c < chunks; ++c) {
        plan->recv_chunk[c] = static_cast<int32_t>(rrow);
        for (int s = 0; s < G; ++s)
            for (int l = plan->chunk_first[c]; l < plan->chunk_first[c + 1]; ++l, ++b) {
                const int32_t n = keep[static_cast<size_t>(s) * E + rank * El + l];
                plan->recv_start[b] = static_cast<int32_t>(rrow);
                plan->group_start[b] = gstart[static_cast<size_t>(s) * El + l];
                plan->recv_rows_c[c][s] += n;
                plan->recv_rows[s] += n;
                rrow += n;
            }
        if (rrow >= limit) return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    plan->recv_chunk[chunks] = static_cast<int32_t>(rrow);
    plan->recv_start[G * El] = static_cast<int32_t>(rrow);
    plan->rows_send = static_cast<int32_t>(send);
    plan->rows_recv = static_cast<int32_t>(rrow);
    plan->rows_group = static_cast<int32_t>(grow);
    return MOE_OK;
}

moe_status_t moe_ep_plan(int G, int rank, int E, int64_t T_total, int k, int cap_num, int cap_den,
                         const int32_t* counts_all, moe_ep_plan_t* plan) {
    return moe_ep_plan_chunked(G, rank, E, T_total, k, cap_num, cap_den, counts_all, 1, plan);
}

size_t moe_ep_workspace_size(const moe_config_t* cfg) {
    if (check_cfg(cfg) != MOE_OK) return 0;
    return ep_scratch_bytes(cfg->T, cfg->E);
}

moe_status_t moe_ep_count(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts, void* ws,
                          size_t ws_bytes, void* stream) {
    moe_status_t st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    int num_sms = 0;
    int* status = nullptr;
    if ((st = current_device(&num_sms, &status)) != MOE_OK) return st;
    if (!ptr16(counts)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cfg->T == 0) return cuda_status(cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->E, s));   // all zero
    if (!ptr16(topk_idx) || !ptr16(ws)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < ep_scratch_bytes(cfg->T, cfg->E)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    return cuda_status(launch_ep_count(topk_idx, cfg->T, cfg->k, cfg->E, counts, ws, status, s));
}

moe_status_t moe_ep_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                             const moe_ep_plan_t* plan_dev, uint8_t* send, int32_t* slot_row, void* ws,
                             size_t ws_bytes, void* stream) {
    moe_status_t st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    int num_sms = 0;
    int* status = nullptr;
    if ((st = current_device(&num_sms, &status)) != MOE_OK) return st;
    if (cfg->T == 0) return MOE_OK;                       // no tokens: no send rows, no slots
    if (!ptr16(x) || !ptr16(topk_idx) || !ptr16(plan_dev) || !ptr16(slot_row) || !ptr16(ws)) return MOE_ERR_INVALID_ARG;
    if (send && !ptr16(send)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < ep_scratch_bytes(cfg->T, cfg->E)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    const uint8_t* pb = reinterpret_cast<const uint8_t*>(plan_dev);
    const int32_t* kept_mine = reinterpret_cast<const int32_t*>(pb + offsetof(moe_ep_plan_t, kept_mine));
    const int32_t* send_off = reinterpret_cast<const int32_t*>(pb + offsetof(moe_ep_plan_t, send_off));
    return cuda_status(launch_ep_dispatch(static_cast<const uint16_t*>(x), topk_idx, cfg->T, cfg->H, cfg->k, cfg->E,
                                          kept_mine, send_off, send, slot_row, ws, num_sms,
                                          static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_receive(int H, const moe_ep_plan_t* plan_dev, int rows_recv, const uint8_t* recv, uint8_t* Aq,
                            float* As, int M_rows, int32_t* offsets, int32_t* group_row, void* stream) {
    if (H <= 0 || H % kGroup || H > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows_recv < 0 || M_rows <= 0 || M_rows % 4) return MOE_ERR_INVALID_ARG;
    if (!ptr16(plan_dev) || !ptr16(Aq) || !ptr16(As) || !ptr16(offsets)) return MOE_ERR_INVALID_ARG;
    if (rows_recv > 0 && (!ptr16(recv) || !ptr16(group_row))) return MOE_ERR_INVALID_ARG;
    moe_status_t st;
    int num_sms = 0;
    int* status = nullptr;
    if ((st = current_device(&num_sms, &status)) != MOE_OK) return st;
    const int64_t warps = std::max<int64_t>(rows_recv, static_cast<int64_t>(kGroup) * 8);
    ep_receive_kernel<<<warp_blocks(warps, num_sms), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        plan_dev, H, rows_recv, -1, recv, ep_row_bytes(H), Aq, As, M_rows, offsets, group_row, status);
    return cuda_status(cudaGetLastError());
}

moe_status_t moe_ep_receive_chunk(int H, const moe_ep_plan_t* plan_dev, int chunk, const uint8_t* recv, uint8_t* Aq,
                                  float* As, int M_rows, int32_t* offsets, int32_t* group_row, void* stream) {
    if (H <= 0 || H % kGroup || H > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (chunk < 0 || chunk >= MOE_EP_MAX_CHUNKS || M_rows <= 0 || M_rows % 4) return MOE_ERR_INVALID_ARG;
    if (!ptr16(plan_dev) || !ptr16(Aq) || !ptr16(As) || !ptr16(offsets) || !ptr16(recv) || !ptr16(group_row))
        return MOE_ERR_INVALID_ARG;
    moe_status_t st;
    int num_sms = 0;
    int* status = nullptr;
    if ((st = current_device(&num_sms, &status)) != MOE_OK) return st;
    // the chunk's row count lives in the device copy of the plan: a grid of a few blocks per SM strides it
    ep_receive_kernel<<<num_sms * 4, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        plan_dev, H, 0, chunk, recv, ep_row_bytes(H), Aq, As, M_rows, offsets, group_row, status);
    return cuda_status(cudaGetLastError());
}

moe_status_t moe_ep_return(int H, int rows_recv, const void* O, const int32_t* group_row, void* ret, void* stream) {
    if (H <= 0 || H % kGroup || H > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows_recv < 0) return MOE_ERR_INVALID_ARG;
    if (rows_recv == 0) return MOE_OK;
    // group_row is read one int32 at a time (a chunk's rows start anywhere in it); rows move in 16 bytes
    if (!ptr16(O) || !group_row || (reinterpret_cast<uintptr_t>(group_row) & 3) || !ptr16(ret))
        return MOE_ERR_INVALID_ARG;
    moe_status_t st;
    int num_sms = 0;
    int* status = nullptr;
    if ((st = current_device(&num_sms, &status)) != MOE_OK) return st;
    ep_return_kernel<<<warp_blocks(rows_recv, num_sms), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        H, rows_recv, static_cast<const uint16_t*>(O), group_row, static_cast<uint16_t*>(ret));
    return cuda_status(cudaGetLastError());
}

}  // extern "C"
