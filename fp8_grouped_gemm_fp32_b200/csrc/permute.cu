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

// Block-wide exclusive scan of per-expert row counts into off_s[0..E].
__device__ void group_offsets(const int32_t* __restrict__ kept, int E, int masked_max_m, int32_t* off_s,
                              int32_t* kept_s) {
    __shared__ int32_t wsum[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // each thread owns experts 2*tid, 2*tid+1 (E <= 512)
    int32_t a = 0, b = 0;
    const int e0 = 2 * tid, e1 = 2 * tid + 1;
    if (e0 < E) { kept_s[e0] = kept[e0]; a = (kept_s[e0] + kGroup - 1) / kGroup * kGroup; }
    if (e1 < E) { kept_s[e1] = kept[e1]; b = (kept_s[e1] + kGroup - 1) / kGroup * kGroup; }
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
// tests. Groups outside that range take the correctly rounded division, out of line.
__device__ __noinline__ float quantise_group_div(float (&v)[8], float amax) {
    const float s = __fdiv_rn(amax, 448.0f);
    for (int i = 0; i < 8; ++i) v[i] = __fdiv_rn(v[i], s);
    return s;
}

__device__ __forceinline__ float quantise_group(float (&v)[8], float amax) {
    if (amax == 0.0f) return 1.0f;                       // all values are (signed) zeros: codes of v itself
    if (!(amax >= 0x1p-60f && amax < 0x1p128f)) return quantise_group_div(v, amax);
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
    return s;
}

// blockIdx.x < nchunks: scatter one 32-token chunk (slot maps + quantised rows);
// blockIdx.x >= nchunks (contiguous layout only): fill expert (x - nchunks)'s padding rows.
// blockIdx.y selects a slice of the H/128 quantisation groups.
__global__ void __launch_bounds__(256, 3) permute_scatter_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx, int T, int H, int k, int E, int nchunks,
    int masked_max_m, int ld_rows, const int32_t* __restrict__ base, const int32_t* __restrict__ kept,
    uint8_t* __restrict__ Aq, float* __restrict__ As, int32_t* __restrict__ offsets, int32_t* __restrict__ row_src,
    int32_t* __restrict__ slot_row) {
    extern __shared__ int32_t sm[];
    int32_t* off_s = sm;                    // [E + 1]
    int32_t* kept_s = off_s + (E + 1);      // [E]
    uint32_t* masks = reinterpret_cast<uint32_t*>(kept_s + E);   // [E]
    int32_t* dest = reinterpret_cast<int32_t*>(masks + E);        // [32][k]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = H / kGroup;
    const int gpy = (G + gridDim.y - 1) / gridDim.y;
    const int g0 = blockIdx.y * gpy, g1 = min(G, g0 + gpy);
    const bool masked = masked_max_m > 0;

    group_offsets(kept, E, masked_max_m, off_s, kept_s);
    if (blockIdx.x == 0 && blockIdx.y == 0)
        for (int e = tid; e <= E; e += blockDim.x) offsets[e] = off_s[e];

    if (blockIdx.x >= nchunks) {            // padding rows of one expert (contiguous layout)
        const int e = blockIdx.x - nchunks;
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
        if (blockIdx.y == 0)
            for (int r = r0 + tid; r < r1; r += blockDim.x) row_src[r] = -1;
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
    if (warp == 0) {
        for (int j = 0; j < k; ++j) {
            int32_t row = -1;
            if (t_lane < T) {
                const int e = topk_idx[static_cast<int64_t>(t_lane) * k + j];
                if (e >= 0 && e < E) {   // an out-of-range expert index is treated as dropped
                    const int32_t rank =
                        base[static_cast<int64_t>(e) * nchunks + c] + __popc(masks[e] & ((1u << lane) - 1u));
                    if (rank < kept_s[e]) row = off_s[e] + rank;
                }
                if (blockIdx.y == 0) {
                    const int64_t s = static_cast<int64_t>(t_lane) * k + j;
                    slot_row[s] = row;
                    if (row >= 0) row_src[row] = static_cast<int32_t>(s);
                }
            }
            dest[lane * k + j] = row;
        }
    }
    __syncthreads();

    // quantise: warp w takes the (token, group) items of tokens w, w + 8, w + 16, w + 24 of the chunk,
    // 2U per pass: a half-warp per item, 8 values (16 bytes) per lane. Each phase runs over all
    // U items of a lane before the next, so the loads, the max butterflies, the divisions and
    // the stores of different items overlap.
    constexpr int U = 4;
    const int hl = lane & 15, hw = lane >> 4;
    const int gs = g1 - g0;
    const int ntok = min(kChunk, T - c * kChunk);
    const int my_tok = ntok > warp ? (ntok - warp + 7) / 8 : 0;
    const int my_items = my_tok * gs;
    const uint32_t inv_gs = (65536u + gs - 1) / gs;          // it / gs == (it * inv_gs) >> 16 for it < 2^16 / 64
    for (int p0 = 0; p0 < my_items; p0 += 2 * U) {
        uint4 raw[U];
        int row_r[U], grp[U];
        bool live[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int it = p0 + 2 * u + hw;
            const int q = static_cast<int>((static_cast<uint32_t>(it) * inv_gs) >> 16);
            live[u] = it < my_items;
            row_r[u] = warp + 8 * q;
            grp[u] = g0 + it - q * gs;
            raw[u] = live[u] ? *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(c * kChunk + row_r[u]) * H +
                                                               grp[u] * kGroup + hl * 8)
                             : make_uint4(0, 0, 0, 0);
        }
        float amax[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xffff0000u))));
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
            const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __uint_as_float(w[i] << 16);
                v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            }
            sc[u] = quantise_group(v, amax[u]);
            code[u].x = f32x2_to_e4m3x2(v[0], v[1]) | (static_cast<uint32_t>(f32x2_to_e4m3x2(v[2], v[3])) << 16);
            code[u].y = f32x2_to_e4m3x2(v[4], v[5]) | (static_cast<uint32_t>(f32x2_to_e4m3x2(v[6], v[7])) << 16);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (!live[u]) continue;
            for (int j = 0; j < k; ++j) {
                const int32_t row = dest[row_r[u] * k + j];
                if (row < 0) continue;
                *reinterpret_cast<uint2*>(Aq + static_cast<int64_t>(row) * H + grp[u] * kGroup + hl * 8) = code[u];
                if (hl == 0) {
                    if (masked) {
                        const int e = row / masked_max_m, rr = row - e * masked_max_m;
                        As[(static_cast<int64_t>(e) * G + grp[u]) * masked_max_m + rr] = sc[u];
                    } else {
                        As[static_cast<int64_t>(grp[u]) * ld_rows + row] = sc[u];
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
    const int gx = nchunks + (masked_max_m > 0 ? 0 : E);
    const size_t smem = sizeof(int32_t) * (3 * static_cast<size_t>(E) + 1 + kChunk * k);
    // as many group slices per chunk as keep every block resident at once (one wave)
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_scatter_kernel, 256, smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    int gy = per_sm * num_sms / gx;
    gy = gy < 1 ? 1 : (gy > G ? G : gy);
    gy = (G + (G + gy - 1) / gy - 1) / ((G + gy - 1) / gy);   // no empty group slices
    permute_scatter_kernel<<<dim3(gx, gy), 256, smem, s>>>(x, topk_idx, T, H, k, E, nchunks, masked_max_m, ld_rows,
                                                           base, kept, Aq, As, offsets, row_src, slot_row);
    return cudaGetLastError();
}

}  // namespace moe
