// Permutation of token slots into expert groups with optional capacity drop,
// fused with the 1x128 FP8 quantisation of x.
//
// Sources: all T_i concatenated into one matrix for one grouped GEMM
// (MegaMoE page, section 2.1) over the flattened M of all groups (3.2);
// capacity ceil(top-k * N / E) * alpha, overflow dropped in token order
// (DeepSeek MoE page, section 2.5); x_fp8 = clamp(round(x / scale), -448, 448)
// (MegaMoE page, 3.3) with one fp32 scale per 1x128 group; FP16/BF16 input
// quantised to FP8 on the fly (section 4.2).
//
// Ranks are deterministic without any ordering of atomics: tokens are cut
// into 32-token chunks; for each chunk and expert a 32-bit mask records which
// of the chunk's tokens chose the expert (atomicOr commutes). A slot's rank
// in its expert = the expert's count in earlier chunks (an exclusive scan
// over chunks) + the popcount of the mask bits below the token's lane.
#include <algorithm>

#include "common.cuh"

namespace moe {

constexpr int kChunk = 32;

// masks of one chunk per warp; cnt[e * nchunks + c] = tokens of chunk c that chose e
__global__ void __launch_bounds__(256) permute_count_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E,
                                                            int nchunks, int32_t* __restrict__ cnt) {
    extern __shared__ uint32_t masks[];   // [8][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x * 8 + warp;
    uint32_t* m = masks + warp * E;
    for (int e = lane; e < E; e += 32) m[e] = 0u;
    __syncwarp();
    const int t = c * kChunk + lane;
    if (c < nchunks && t < T)
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[static_cast<int64_t>(t) * k + j];
            if (e >= 0 && e < E) atomicOr(&m[e], 1u << lane);
        }
    __syncwarp();
    if (c < nchunks)
        for (int e = lane; e < E; e += 32) cnt[static_cast<int64_t>(e) * nchunks + c] = __popc(m[e]);
}

// One block per expert: base[e*nchunks + c] = sum of cnt over chunks < c;
// counts[e] = total; kept[e] = min(total, cap, masked_max_m).
__global__ void __launch_bounds__(256) permute_scan_kernel(const int32_t* __restrict__ cnt, int nchunks, int64_t cap,
                                                           int masked_max_m, int32_t* __restrict__ base,
                                                           int32_t* __restrict__ counts, int32_t* __restrict__ kept,
                                                           int* status) {
    __shared__ int32_t warp_sums[8];
    const int e = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seg = (nchunks + 255) / 256;
    const int c0 = tid * seg, c1 = min(nchunks, c0 + seg);
    const int32_t* ce = cnt + static_cast<int64_t>(e) * nchunks;
    int32_t local = 0;
    for (int c = c0; c < c1; ++c) local += ce[c];
    // exclusive scan of `local` across the block
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int32_t warp_off = 0, total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        if (w < warp) warp_off += warp_sums[w];
        total += warp_sums[w];
    }
    int32_t run = warp_off + incl - local;
    int32_t* be = base + static_cast<int64_t>(e) * nchunks;
    for (int c = c0; c < c1; ++c) {
        be[c] = run;
        run += ce[c];
    }
    if (tid == 0) {
        int64_t kk = total;
        if (cap >= 0 && kk > cap) kk = cap;
        if (masked_max_m > 0 && kk > masked_max_m) {
            kk = masked_max_m;
            set_status(status, kStatusCapacity);
        }
        counts[e] = total;
        kept[e] = static_cast<int32_t>(kk);
    }
}

// Block-wide exclusive scan of per-expert row counts, each rounded up to a multiple of `pad` (the tile
// M, or 1 for unpadded send rows), into off_s[0..E].
__device__ void group_offsets(const int32_t* __restrict__ kept, int E, int masked_max_m, int pad, int32_t* off_s,
                              int32_t* kept_s) {
    __shared__ int32_t wsum[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // each thread owns experts 2*tid, 2*tid+1 (E <= 512)
    int32_t a = 0, b = 0;
    const int e0 = 2 * tid, e1 = 2 * tid + 1;
    if (e0 < E) { kept_s[e0] = kept[e0]; a = (kept_s[e0] + pad - 1) / pad * pad; }
    if (e1 < E) { kept_s[e1] = kept[e1]; b = (kept_s[e1] + pad - 1) / pad * pad; }
    const int32_t local = a + b;
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int32_t off = 0, total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        if (w < warp) off += wsum[w];
        total += wsum[w];
    }
    const int32_t ex = off + incl - local;
    if (masked_max_m > 0) {
        if (e0 <= E) off_s[e0] = e0 * masked_max_m;
        if (e1 <= E) off_s[e1] = e1 * masked_max_m;
        if (tid == 0) off_s[E] = E * masked_max_m;
    } else {
        if (e0 <= E) off_s[e0] = ex;
        if (e1 <= E) off_s[e1] = ex + a;
        if (tid == 0) off_s[E] = total;
    }
    __syncthreads();
}

// Scale and codes of one 1x128 group without a division per value. Markstein's correction step
// (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Dev. 34(1), 1990): with y = 1/b correctly rounded and q0 = a * y rounded, the
// remainder a - q0 * b is exact in one fused multiply-add and q0 + remainder * y, rounded once, is
// the correctly rounded quotient a / b, as long as no intermediate leaves the normal range. It
// gives s = amax / 448 (y = 1/448 rounded, a compile-time constant) and each v / s (y = 1/s from the
// correctly rounded reciprocal). For amax in [2^-60, 2^128) every quotient that can reach an E4M3
// code (|v / s| >= 2^-10) has v >= 2^-79, far inside the normal range; smaller quotients round to a
// signed zero code, and their sign is v's, which is restored explicitly (the correction would turn
// -0 into +0). Checked against C's correctly rounded division on 4e8 bf16 value / scale pairs with
// amax over 2^-100 .. 2^126 (the only difference needs amax near 2^-100) and by the bit-exact parity
// tests. Groups outside that range take the correctly rounded division, out of line (its arguments
// and results pass by value, so the common path keeps its values in registers).
struct GroupCodes {
    uint2 code;     // 8 E4M3 codes, the first value in the lowest byte
    float scale;
};

__device__ __forceinline__ uint2 pack_e4m3x8(const float (&v)[8]) {
    return make_uint2(f32x2_to_e4m3x2(v[0], v[1]) | (static_cast<uint32_t>(f32x2_to_e4m3x2(v[2], v[3])) << 16),
                      f32x2_to_e4m3x2(v[4], v[5]) | (static_cast<uint32_t>(f32x2_to_e4m3x2(v[6], v[7])) << 16));
}

__device__ __forceinline__ void unpack_bf16x8(uint4 raw, float (&v)[8]) {
    const uint32_t q[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(q[i] << 16);
        v[2 * i + 1] = __uint_as_float(q[i] & 0xffff0000u);
    }
}

__device__ __noinline__ GroupCodes quantise_group_div(uint4 raw, float amax) {
    float v[8];
    unpack_bf16x8(raw, v);
    const float s = __fdiv_rn(amax, 448.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __fdiv_rn(v[i], s);
    return GroupCodes{pack_e4m3x8(v), s};
}

// Codes and scale of a lane's 8 values (bf16, packed in raw) of a group whose max |value| is amax.
__device__ __forceinline__ GroupCodes quantise_group(uint4 raw, float amax) {
    float v[8];
    unpack_bf16x8(raw, v);
    if (amax == 0.0f) return GroupCodes{pack_e4m3x8(v), 1.0f};   // all (signed) zeros: codes of v itself
    if (!(amax >= 0x1p-60f && amax < 0x1p128f)) return quantise_group_div(raw, amax);
    constexpr float kInv448 = 1.0f / 448.0f;
    const float s0 = amax * kInv448;
    const float s = fmaf(fmaf(-s0, 448.0f, amax), kInv448, s0);
    const float r = __frcp_rn(s);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float q0 = v[i] * r;
        const float q = fmaf(fmaf(-q0, s, v[i]), r, q0);
        v[i] = __uint_as_float((__float_as_uint(q) & 0x7fffffffu) | (__float_as_uint(v[i]) & 0x80000000u));
    }
    return GroupCodes{pack_e4m3x8(v), s};
}

// blockIdx.x < nchunks: the slot maps of one 32-token chunk (slot_row, row_src);
// blockIdx.x >= nchunks (contiguous layout only): the padding rows of one expert, one slice of
// pad_slices of its 128-groups (codes 0, scale 1, row_src -1), and (the last expert's first slice)
// row_src -1 for the rows past the last group. Block 0 also writes offsets.
// row_base (nullable): each expert's first row, in place of the scan of kept (an expert-parallel
// plan's send rows, which run in chunk order).
__global__ void __launch_bounds__(256) permute_map_kernel(
    const int32_t* __restrict__ topk_idx, int T, int H, int k, int E, int nchunks, int pad, int pad_slices,
    int masked_max_m, int ld_rows, const int32_t* __restrict__ base, const int32_t* __restrict__ kept,
    uint8_t* __restrict__ Aq, float* __restrict__ As, int32_t* __restrict__ offsets, int32_t* __restrict__ row_src,
    int32_t* __restrict__ slot_row, const int32_t* __restrict__ row_base) {
    extern __shared__ int32_t sm[];
    int32_t* off_s = sm;                    // [E + 1]
    int32_t* kept_s = off_s + (E + 1);      // [E]
    uint32_t* masks = reinterpret_cast<uint32_t*>(kept_s + E);   // [E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = H / kGroup;

    group_offsets(kept, E, masked_max_m, pad, off_s, kept_s);
    if (row_base) {
        for (int e = tid; e < E; e += blockDim.x) off_s[e] = row_base[e];
        __syncthreads();
    }
    if (blockIdx.x == 0 && offsets)
        for (int e = tid; e <= E; e += blockDim.x) offsets[e] = off_s[e];

    if (blockIdx.x >= nchunks) {            // padding rows of one expert (contiguous layout)
        const int e = (blockIdx.x - nchunks) / pad_slices, sl = (blockIdx.x - nchunks) % pad_slices;
        const int gps = (G + pad_slices - 1) / pad_slices;
        const int g0 = sl * gps, g1 = min(G, g0 + gps);
        if (g0 >= g1) return;
        const int r0 = off_s[e] + kept_s[e], r1 = off_s[e + 1];
        const int per_row = (g1 - g0) * (kGroup / 16);           // 16-byte pieces per row slice
        for (int i = tid; i < (r1 - r0) * per_row; i += blockDim.x) {
            const int r = r0 + i / per_row, p = i % per_row;
            reinterpret_cast<uint4*>(Aq + static_cast<int64_t>(r) * H + g0 * kGroup)[p] = make_uint4(0, 0, 0, 0);
        }
        for (int i = tid; i < (r1 - r0) * (g1 - g0); i += blockDim.x) {
            const int r = r0 + i / (g1 - g0), g = g0 + i % (g1 - g0);
            As[static_cast<int64_t>(g) * ld_rows + r] = 1.0f;
        }
        if (sl == 0)
            for (int r = r0 + tid; r < r1; r += blockDim.x) row_src[r] = -1;
        // the rows past the last group, up to ld_rows, belong to no group: marked as padding too, so that a
        // step that walks every row (the backward pass) reads no stale source slot there
        if (sl == 0 && e == E - 1 && row_src)
            for (int r = off_s[E] + tid; r < ld_rows; r += blockDim.x) row_src[r] = -1;
        return;
    }

    const int c = blockIdx.x;
    for (int e = tid; e < E; e += blockDim.x) masks[e] = 0u;
    __syncthreads();
    const int t_lane = c * kChunk + lane;
    if (warp == 0 && t_lane < T)
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[static_cast<int64_t>(t_lane) * k + j];
            if (e >= 0 && e < E) atomicOr(&masks[e], 1u << lane);
        }
    __syncthreads();
    if (warp == 0 && t_lane < T) {
        for (int j = 0; j < k; ++j) {
            int32_t row = -1;
            const int e = topk_idx[static_cast<int64_t>(t_lane) * k + j];
            if (e >= 0 && e < E) {   // an out-of-range expert index is treated as dropped
                const int32_t rank =
                    base[static_cast<int64_t>(e) * nchunks + c] + __popc(masks[e] & ((1u << lane) - 1u));
                if (rank < kept_s[e]) row = off_s[e] + rank;
            }
            const int64_t s = static_cast<int64_t>(t_lane) * k + j;
            slot_row[s] = row;
            if (row >= 0 && row_src) row_src[row] = static_cast<int32_t>(s);
        }
    }
}

// Quantise x once per token and 1x128 group and write the codes and the scale to every kept
// destination row of the token (slot_row). A warp takes one token and up to 8 of its groups, a
// half-warp per group with 8 values (one 16-byte load) per lane, all four loads of a lane in flight
// together; warps stride over (token, 8-group slice) items.
// Scales go to As in the grouped layouts ([G][ld_rows], or [E][G][masked_max_m] when masked), or, with
// `trailer`, right after the row's codes (row stride row_bytes = H + 4 G: the send rows of expert
// parallelism, one contiguous record per row).
__global__ void __launch_bounds__(256, 4) permute_quant_kernel(
    const uint16_t* __restrict__ x, int T, int H, int k, int masked_max_m, int ld_rows, int64_t row_bytes,
    bool trailer, const int32_t* __restrict__ slot_row, uint8_t* __restrict__ Aq, float* __restrict__ As) {
    constexpr int U = 4;
    const int lane = threadIdx.x & 31, hl = lane & 15, hw = lane >> 4;
    const int G = H / kGroup;
    const int nsl = (G + 2 * U - 1) / (2 * U);
    const bool masked = masked_max_m > 0;
    const int64_t items = static_cast<int64_t>(T) * nsl;
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < items;
         w += static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5)) {
        const int t = static_cast<int>(w / nsl);
        const int g0 = static_cast<int>(w % nsl) * 2 * U;
        const uint16_t* xrow = x + static_cast<int64_t>(t) * H;
        // the token's destination rows load alongside its values (up to 8 here; more in the store loop)
        constexpr int KR = 8;
        int32_t rows[KR];
#pragma unroll
        for (int j = 0; j < KR; ++j) rows[j] = j < k ? slot_row[static_cast<int64_t>(t) * k + j] : -1;
        uint4 raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int g = g0 + 2 * u + hw;
            raw[u] = g < G ? *reinterpret_cast<const uint4*>(xrow + g * kGroup + hl * 8) : make_uint4(0, 0, 0, 0);
        }
        float amax[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t q[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                m = fmaxf(m, fmaxf(fabsf(__uint_as_float(q[i] << 16)), fabsf(__uint_as_float(q[i] & 0xffff0000u))));
            amax[u] = m;
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1)
#pragma unroll
            for (int u = 0; u < U; ++u) amax[u] = fmaxf(amax[u], __shfl_xor_sync(0xffffffffu, amax[u], o));
        float sc[U];
        uint2 code[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const GroupCodes gc = quantise_group(raw[u], amax[u]);
            code[u] = gc.code;
            sc[u] = gc.scale;
        }
        for (int j = 0; j < k; ++j) {
            int32_t row = -1;
#pragma unroll
            for (int i = 0; i < KR; ++i)
                if (i == j) row = rows[i];
            if (j >= KR) row = slot_row[static_cast<int64_t>(t) * k + j];
            if (row < 0) continue;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int g = g0 + 2 * u + hw;
                if (g >= G) continue;
                *reinterpret_cast<uint2*>(Aq + static_cast<int64_t>(row) * row_bytes + g * kGroup + hl * 8) = code[u];
                if (hl == 0) {
                    if (trailer) {
                        reinterpret_cast<float*>(Aq + static_cast<int64_t>(row) * row_bytes + H)[g] = sc[u];
                    } else if (masked) {
                        const int e = row / masked_max_m, rr = row - e * masked_max_m;
                        As[(static_cast<int64_t>(e) * G + g) * masked_max_m + rr] = sc[u];
                    } else {
                        As[static_cast<int64_t>(g) * ld_rows + row] = sc[u];
                    }
                }
            }
        }
    }
}

size_t permute_scratch_bytes(int T, int E) {
    const int nchunks = (T + kChunk - 1) / kChunk;
    return 2 * sizeof(int32_t) * static_cast<size_t>(nchunks) * E;
}

cudaError_t launch_permute(const uint16_t* x, const int32_t* topk_idx, int T, int H, int k, int E, int64_t cap,
                           int masked_max_m, int ld_rows, uint8_t* Aq, float* As, int32_t* counts, int32_t* kept,
                           int32_t* offsets, int32_t* row_src, int32_t* slot_row, void* scratch, int* status,
                           int num_sms, cudaStream_t s) {
    const int nchunks = (T + kChunk - 1) / kChunk;
    int32_t* cnt = static_cast<int32_t*>(scratch);
    int32_t* base = cnt + static_cast<size_t>(nchunks) * E;
    permute_count_kernel<<<(nchunks + 7) / 8, 256, 8 * E * sizeof(uint32_t), s>>>(topk_idx, T, k, E, nchunks, cnt);
    permute_scan_kernel<<<E, 256, 0, s>>>(cnt, nchunks, cap, masked_max_m, base, counts, kept, status);
    const int G = H / kGroup;
    // padding blocks: slices of four 128-groups per expert, so a block fills about 32 KB (64 rows)
    const int pad_slices = masked_max_m > 0 ? 1 : (G + 3) / 4;
    const int gx = nchunks + (masked_max_m > 0 ? 0 : E * pad_slices);
    const size_t smem = sizeof(int32_t) * (3 * static_cast<size_t>(E) + 1);
    permute_map_kernel<<<gx, 256, smem, s>>>(topk_idx, T, H, k, E, nchunks, kGroup, pad_slices, masked_max_m, ld_rows,
                                             base, kept, Aq, As, offsets, row_src, slot_row, nullptr);
    // one warp per (token, 8-group slice); enough blocks to keep every SM full, striding beyond that
    const int64_t warps = static_cast<int64_t>(T) * ((G + 7) / 8);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_quant_kernel, 256, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t cap_blocks = static_cast<int64_t>(per_sm) * num_sms * 4;
    const int blocks = static_cast<int>(std::min<int64_t>((warps + 7) / 8, cap_blocks));
    if (blocks > 0)
        permute_quant_kernel<<<blocks, 256, 0, s>>>(x, T, H, k, masked_max_m, ld_rows, H, false, slot_row, Aq, As);
    return cudaGetLastError();
}

int64_t ep_row_bytes(int H);

// Expert parallelism, first half (before the counts are exchanged): per-chunk masks and the per-expert
// exclusive scan over chunks, as for moe_permute; counts [E] out, ranks kept in `scratch`.
cudaError_t launch_ep_count(const int32_t* topk_idx, int T, int k, int E, int32_t* counts, void* scratch,
                            int* status, cudaStream_t s) {
    const int nchunks = (T + kChunk - 1) / kChunk;
    int32_t* cnt = static_cast<int32_t*>(scratch);
    int32_t* base = cnt + static_cast<size_t>(nchunks) * E;
    int32_t* unused_kept = base + static_cast<size_t>(nchunks) * E;   // no capacity here: kept = counts
    permute_count_kernel<<<(nchunks + 7) / 8, 256, 8 * E * sizeof(uint32_t), s>>>(topk_idx, T, k, E, nchunks, cnt);
    permute_scan_kernel<<<E, 256, 0, s>>>(cnt, nchunks, -1, 0, base, counts, unused_kept, status);
    return cudaGetLastError();
}

// Every slot of every expert, dropped ones included, in token order: counts [E], offsets [E + 1] (unpadded
// prefix) and list [T * k] (list[offsets[e] + r] = the slot t * k + j of expert e's r-th token); slot_tmp
// [T * k] receives each slot's position. Scratch as launch_ep_count's.
cudaError_t launch_slot_lists(const int32_t* topk_idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
                              int32_t* list, int32_t* slot_tmp, void* scratch, int* status, cudaStream_t s) {
    const int nchunks = (T + kChunk - 1) / kChunk;
    int32_t* cnt = static_cast<int32_t*>(scratch);
    int32_t* base = cnt + static_cast<size_t>(nchunks) * E;
    int32_t* unused_kept = base + static_cast<size_t>(nchunks) * E;
    permute_count_kernel<<<(nchunks + 7) / 8, 256, 8 * E * sizeof(uint32_t), s>>>(topk_idx, T, k, E, nchunks, cnt);
    permute_scan_kernel<<<E, 256, 0, s>>>(cnt, nchunks, -1, 0, base, counts, unused_kept, status);
    const size_t smem = sizeof(int32_t) * (3 * static_cast<size_t>(E) + 1);
    permute_map_kernel<<<nchunks, 256, smem, s>>>(topk_idx, T, 0, k, E, nchunks, 1, 1, 0, 0, base, counts, nullptr,
                                                  nullptr, offsets, list, slot_tmp, nullptr);
    return cudaGetLastError();
}

size_t ep_scratch_bytes(int T, int E) { return permute_scratch_bytes(T, E) + sizeof(int32_t) * static_cast<size_t>(E); }

// Bytes of one send / receive row: H codes, H/128 fp32 scales, padded to 16 bytes.
int64_t ep_row_bytes(int H) { return (static_cast<int64_t>(H) + 4 * (H / kGroup) + 15) / 16 * 16; }

// Second half: send rows for the kept slots. kept_mine [E] (device, from the plan) bounds each expert's
// ranks exactly as the capacity does in moe_permute; rows are unpadded (pad 1), in expert order, which
// is destination-rank order since each rank's experts are contiguous.
cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* topk_idx, int T, int H, int k, int E,
                               const int32_t* kept_mine, const int32_t* send_off, uint8_t* send, int32_t* slot_row,
                               void* scratch, int num_sms, cudaStream_t s) {
    const int nchunks = (T + kChunk - 1) / kChunk;
    int32_t* base = static_cast<int32_t*>(scratch) + static_cast<size_t>(nchunks) * E;
    const size_t smem = sizeof(int32_t) * (3 * static_cast<size_t>(E) + 1);
    permute_map_kernel<<<nchunks, 256, smem, s>>>(topk_idx, T, H, k, E, nchunks, 1, 1, 0, 0, base, kept_mine,
                                                  nullptr, nullptr, nullptr, nullptr, slot_row, send_off);
    const int G = H / kGroup;
    const int64_t warps = static_cast<int64_t>(T) * ((G + 7) / 8);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_quant_kernel, 256, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t cap_blocks = static_cast<int64_t>(per_sm) * num_sms * 4;
    const int blocks = static_cast<int>(std::min<int64_t>((warps + 7) / 8, cap_blocks));
    if (blocks > 0)
        permute_quant_kernel<<<blocks, 256, 0, s>>>(x, T, H, k, 0, 0, ep_row_bytes(H), true, slot_row, send, nullptr);
    return cudaGetLastError();
}

}  // namespace moe
