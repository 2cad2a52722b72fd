// The layer's backward pass (TP-MoE page, section 4.1, step 5: the gradients go back along the dispatch
// path and the gate network is updated as well). The expert path runs on the forward's FP8 grouped GEMM:
//
//   dO    = w * dy on every kept slot's row (fp32), 1x128 FP8 along H;
//   dh    = dO W2       grouped GEMM with the transposed W2 (bf16 out);
//   a | b = x W13^T     grouped GEMM, recomputed (bf16 out);
//   g     = SwiGLU backward: da = dh b s (1 + a (1 - s)), db = dh a s with s = sigmoid(a) (bf16), then 1x128
//           FP8 along 2I;
//   dx    = sum_j dx_rows + sum_j dl_j W_g[e_j],   dx_rows = g W13 (grouped GEMM, transposed W13);
//   dW2   = sum over each expert's rows dO^T h,  dW13 = sum g^T x: the K-grouped GEMM over the expert's
//           128-row tiles, its first operand (dO, g) in 1x128 groups along the rows, the second (h, x)
//           in 128 x 128 blocks, both transposed per tile by bwd_tquant_kernel;
//   gate  = dw_j = <dy, o_j>, dl_j = w_j (dw_j - sum_i w_i dw_i), dW_g[e] = sum of dl x over the slots of e,
//           db[e] = sum of dl, all in token order (dropped slots included: their logits still moved w).
// The quantisation steps of the forward pass pass the gradient through; selection and capacity are held.
#include "../../include/moe_fp8.h"
#include "backward.cuh"
#include "common.cuh"

#include <type_traits>

namespace moe {

constexpr int kTq = 128;        // transposed-quantisation tile: 128 rows x 128 columns
constexpr int kTqS = kTq + 4;   // its row stride in shared memory (4 mod 32 words)

// The scale of a group with largest magnitude amax (amax / 448 correctly rounded; 1 for an all-zero group)
// and what the quotients v / s need: r = 1 / s correctly rounded where Markstein's correction applies
// (P. Markstein, IBM J. Res. Dev. 34(1), 1990: with r = 1/s correctly rounded and q0 = v r rounded, the
// remainder v - q0 s is exact in one fused multiply-add and q0 + remainder * r, rounded once, is the
// correctly rounded quotient while no intermediate leaves the normal range). For amax in [2^-60, 2^128)
// every quotient that can reach a nonzero E4M3 code (|v / s| >= 2^-10) has |v| >= 2^-79, well inside the
// normal range; smaller quotients give a zero code whose sign, v's, is set explicitly. Other groups divide.
struct GroupScale {
    float s, r;
    bool fast;
};

__device__ __forceinline__ GroupScale group_scale(float amax) {
    if (amax == 0.0f) return GroupScale{1.0f, 1.0f, true};     // signed zeros keep their codes
    const float s = __fdiv_rn(amax, 448.0f);
    const bool fast = amax >= 0x1p-60f && amax < 0x1p128f;
    return GroupScale{s, fast ? __frcp_rn(s) : 0.0f, fast};
}

// v / s correctly rounded (the E4M3 conversion then rounds it to nearest even, saturating).
__device__ __forceinline__ float group_quot(float v, const GroupScale& g) {
    if (!g.fast) return __fdiv_rn(v, g.s);
    const float q0 = v * g.r;
    const float q = fmaf(fmaf(-q0, g.s, v), g.r, q0);
    return __uint_as_float((__float_as_uint(q) & 0x7fffffffu) | (__float_as_uint(v) & 0x80000000u));
}

// Four codes (v[0] in the lowest byte) of one group.
__device__ __forceinline__ uint32_t group_codes4(const float* v, const GroupScale& g) {
    return f32x2_to_e4m3x2(group_quot(v[0], g), group_quot(v[1], g)) |
           (static_cast<uint32_t>(f32x2_to_e4m3x2(group_quot(v[2], g), group_quot(v[3], g))) << 16);
}

// One warp per token: dw_j = <dy_t, o_j> over H (fp32; 0 for a dropped slot) and
// dl_j = w_j (dw_j - sum_i w_i dw_i).
__global__ void __launch_bounds__(256) bwd_dl_kernel(const uint16_t* __restrict__ dy, const uint16_t* __restrict__ O,
                                                     const int32_t* __restrict__ slot_row,
                                                     const float* __restrict__ topk_w, int T, int k, int H,
                                                     float* __restrict__ dl) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    float dw_mine = 0.0f;                     // lane j keeps dw_j
    for (int j = 0; j < k; ++j) {
        const int32_t r = slot_row[static_cast<int64_t>(t) * k + j];
        float acc = 0.0f;
        if (r >= 0)
#pragma unroll 4
            for (int h = lane * 8; h < H; h += 256) {
                const uint4 a = *reinterpret_cast<const uint4*>(dy + static_cast<int64_t>(t) * H + h);
                const uint4 b = *reinterpret_cast<const uint4*>(O + static_cast<int64_t>(r) * H + h);
                const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc = fmaf(__uint_as_float(av[i] << 16), __uint_as_float(bv[i] << 16), acc);
                    acc = fmaf(__uint_as_float(av[i] & 0xffff0000u), __uint_as_float(bv[i] & 0xffff0000u), acc);
                }
            }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == j) dw_mine = acc;
    }
    const float w = lane < k ? topk_w[static_cast<int64_t>(t) * k + lane] : 0.0f;
    float wdw = w * dw_mine;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) wdw += __shfl_xor_sync(0xffffffffu, wdw, o);
    if (lane < k) dl[static_cast<int64_t>(t) * k + lane] = w * (dw_mine - wdw);
}

// Eight lanes per (row, 128-group), a warp covering four groups of a row: dO = w * dy of the row's slot,
// quantised (1x128, scale max|v| / 448); padding rows get code 0, scale 1. Scales K-block-major
// [H/128][rows]. Lane part p of a group holds its columns 16 p .. 16 p + 15 (two 16-byte loads).
__global__ void __launch_bounds__(256) bwd_dout_quant_kernel(const uint16_t* __restrict__ dy,
                                                             const float* __restrict__ topk_w,
                                                             const int32_t* __restrict__ row_src, int rows, int k, int H,
                                                             uint8_t* __restrict__ q, float* __restrict__ s) {
    const int lane = threadIdx.x & 31;
    const int G = H / kGroup, NQ = (G + 3) / 4;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (item >= static_cast<int64_t>(rows) * NQ) return;
    const int r = static_cast<int>(item / NQ);
    const int g = static_cast<int>(item % NQ) * 4 + (lane >> 3), part = lane & 7;
    const bool act = g < G;
    const int32_t src = row_src[r];
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    if (act && src >= 0) {
        const float w = topk_w[src];
        const uint4* p = reinterpret_cast<const uint4*>(dy + static_cast<int64_t>(src / k) * H + g * kGroup + part * 16);
        const uint4 r0 = p[0], r1 = p[1];
        const uint32_t u[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = w * __uint_as_float(u[i] << 16);
            v[2 * i + 1] = w * __uint_as_float(u[i] & 0xffff0000u);
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const GroupScale gs = group_scale(amax);
    if (act) {
        *reinterpret_cast<uint4*>(q + static_cast<int64_t>(r) * H + g * kGroup + part * 16) =
            make_uint4(group_codes4(v, gs), group_codes4(v + 4, gs), group_codes4(v + 8, gs), group_codes4(v + 12, gs));
        if (part == 0) s[static_cast<int64_t>(g) * rows + r] = gs.s;
    }
}

// Eight lanes per (row, 128-wide block j of I), a warp covering four blocks of a row: a, b (bf16, the up
// GEMM's interleaved a | b columns of block j) and dh -> da, db (fp32, rounded to bf16) into g in the same
// interleaving, then each 128-group of g quantised (1x128 along 2I, scales K-block-major [2I/128][rows]).
// Padding rows: zeros, scale 1. Lane part p holds columns 16 p .. 16 p + 15 of the block.
__global__ void __launch_bounds__(256) bwd_swiglu_kernel(const uint16_t* __restrict__ ab, const uint16_t* __restrict__ dh,
                                                         const int32_t* __restrict__ row_src, int rows, int I,
                                                         uint16_t* __restrict__ g, uint8_t* __restrict__ gq,
                                                         float* __restrict__ gs) {
    const int lane = threadIdx.x & 31;
    const int NJ = I / kGroup, NQ = (NJ + 3) / 4;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (item >= static_cast<int64_t>(rows) * NQ) return;
    const int r = static_cast<int>(item / NQ);
    const int j = static_cast<int>(item % NQ) * 4 + (lane >> 3), part = lane & 7;
    const bool act = j < NJ;
    const bool valid = act && row_src[r] >= 0;
    const int64_t base = static_cast<int64_t>(r) * 2 * I + j * 2 * kGroup + part * 16;
    uint4 ra[2] = {}, rb[2] = {}, rd[2] = {};
    if (valid) {
        const uint4* pa = reinterpret_cast<const uint4*>(ab + base);
        const uint4* pb = reinterpret_cast<const uint4*>(ab + base + kGroup);
        const uint4* pd = reinterpret_cast<const uint4*>(dh + static_cast<int64_t>(r) * I + j * kGroup + part * 16);
        ra[0] = pa[0]; ra[1] = pa[1];
        rb[0] = pb[0]; rb[1] = pb[1];
        rd[0] = pd[0]; rd[1] = pd[1];
    }
    const uint32_t wa[8] = {ra[0].x, ra[0].y, ra[0].z, ra[0].w, ra[1].x, ra[1].y, ra[1].z, ra[1].w};
    const uint32_t wb[8] = {rb[0].x, rb[0].y, rb[0].z, rb[0].w, rb[1].x, rb[1].y, rb[1].z, rb[1].w};
    const uint32_t wd[8] = {rd[0].x, rd[0].y, rd[0].z, rd[0].w, rd[1].x, rd[1].y, rd[1].z, rd[1].w};
    float da[16], db[16];
    uint32_t ga[8], gb[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int sh = (i & 1) ? 0 : 16;
        const float a = __uint_as_float((wa[i >> 1] << sh) & 0xffff0000u);
        const float b = __uint_as_float((wb[i >> 1] << sh) & 0xffff0000u);
        const float d = __uint_as_float((wd[i >> 1] << sh) & 0xffff0000u);
        float dav = 0.0f, dbv = 0.0f;
        if (valid) {
            const float sg = 1.0f / (1.0f + expf(-a));
            dav = d * b * sg * (1.0f + a * (1.0f - sg));
            dbv = d * a * sg;
        }
        const uint32_t ua = __bfloat16_as_ushort(__float2bfloat16_rn(dav));
        const uint32_t ub = __bfloat16_as_ushort(__float2bfloat16_rn(dbv));
        da[i] = __uint_as_float(ua << 16);
        db[i] = __uint_as_float(ub << 16);
        if (i & 1) {
            ga[i >> 1] |= ua << 16;
            gb[i >> 1] |= ub << 16;
        } else {
            ga[i >> 1] = ua;
            gb[i >> 1] = ub;
        }
    }
    if (act) {
        uint4* oa = reinterpret_cast<uint4*>(g + base);
        uint4* ob = reinterpret_cast<uint4*>(g + base + kGroup);
        oa[0] = make_uint4(ga[0], ga[1], ga[2], ga[3]);
        oa[1] = make_uint4(ga[4], ga[5], ga[6], ga[7]);
        ob[0] = make_uint4(gb[0], gb[1], gb[2], gb[3]);
        ob[1] = make_uint4(gb[4], gb[5], gb[6], gb[7]);
    }
    // the two 128-groups of g: da (group 2j) and db (group 2j + 1), each over the block's eight lanes
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float* v = h == 0 ? da : db;
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const GroupScale q = group_scale(amax);
        if (act) {
            *reinterpret_cast<uint4*>(gq + base + h * kGroup) =
                make_uint4(group_codes4(v, q), group_codes4(v + 4, q), group_codes4(v + 8, q), group_codes4(v + 12, q));
            if (part == 0) gs[static_cast<int64_t>(2 * j + h) * rows + r] = q.s;
        }
    }
}

// For forward row tile m (blockIdx.x) and column block cb (blockIdx.y): the transposed 128 x 128 block
// quantised. ROWS: one scale per transposed row (column c over the tile's 128 rows), out scales [tiles][C];
// otherwise one scale for the block, out scales [tiles][C/128]. Codes [tiles * C, 128]: transposed row
// m * C + c holds the 128 rows of the tile.
//
// Loads: pieces of 8 columns (16 bytes of bf16, 8 of codes), a warp covering two rows with 16 pieces each.
// Shared memory holds the fp32 values with row stride kTqS and column c at c + c / 32, which puts the 32
// lanes' stores of one step (16 pieces x 2 rows) and the column reads of a warp (32 consecutive columns)
// in 32 different banks. Then thread (c = tid % 128, half = tid / 128) owns column c over rows
// 64 half .. 64 half + 63: their maximum, the scale, and 64 codes written as four 16-byte pieces.
template <int SRC, bool ROWS>
__global__ void __launch_bounds__(256, 3) bwd_tquant_kernel(TqArgs a, uint8_t* __restrict__ out, float* __restrict__ os) {
    extern __shared__ float tq_smem[];                     // [kTq][kTqS] values, [2][kTq] half maxima, [8]
    float (*tile)[kTqS] = reinterpret_cast<float (*)[kTqS]>(tq_smem);
    float* part = tq_smem + kTq * kTqS;
    float* red = part + 2 * kTq;
    const int m = blockIdx.x, cb = blockIdx.y;
    const int tid = threadIdx.x;
    constexpr int kIt = kTq * 16 / 256;                    // pieces per thread (the block has 256 threads)
    // every load of the thread first (raw bytes), then the conversion and the shared-memory stores
    using Raw = typename std::conditional<SRC == kTqFp8, uint2, uint4>::type;
    Raw raw[kIt];
    int32_t src[kIt];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int i = tid + it * 256;
        const int rr = i >> 4, p = i & 15;
        const int row = m * kTq + rr, col = cb * kTq + p * 8;
        src[it] = a.row_src[row];
        if constexpr (SRC == kTqFp8) {
            raw[it] = src[it] >= 0 ? *reinterpret_cast<const uint2*>(a.codes + static_cast<int64_t>(row) * a.C + col)
                                   : make_uint2(0u, 0u);
        } else {
            const uint16_t* rowp = SRC == kTqDout ? a.dy + static_cast<int64_t>(max(src[it], 0) / a.k) * a.C
                                                  : a.bf + static_cast<int64_t>(row) * a.C;
            raw[it] = src[it] >= 0 ? *reinterpret_cast<const uint4*>(rowp + col) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int i = tid + it * 256;
        const int rr = i >> 4, p = i & 15;
        const int row = m * kTq + rr, col = cb * kTq + p * 8;
        float v[8];
        if constexpr (SRC == kTqFp8) {
            const float sc = src[it] >= 0 ? a.scales[static_cast<int64_t>(col / kGroup) * a.rows + row] : 0.0f;
            const uint32_t w[2] = {raw[it].x, raw[it].y};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                    static_cast<__nv_fp8x2_storage_t>((w[h >> 1] >> (16 * (h & 1))) & 0xffffu), __NV_E4M3);
                const float2 f = __half22float2(__half2(hr));
                v[2 * h] = f.x * sc;
                v[2 * h + 1] = f.y * sc;
            }
        } else {
            const uint32_t w[4] = {raw[it].x, raw[it].y, raw[it].z, raw[it].w};
            const float wt = SRC == kTqDout && src[it] >= 0 ? a.topk_w[src[it]] : 1.0f;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                v[2 * h] = __uint_as_float(w[h] << 16);
                v[2 * h + 1] = __uint_as_float(w[h] & 0xffff0000u);
                if constexpr (SRC == kTqDout) {
                    v[2 * h] *= wt;
                    v[2 * h + 1] *= wt;
                }
            }
        }
        const int c0 = p * 8 + (p >> 2);          // column p * 8 at p * 8 + p / 4
#pragma unroll
        for (int j = 0; j < 8; ++j) tile[rr][c0 + j] = v[j];
    }
    __syncthreads();
    const int c = tid & (kTq - 1), half = tid >> 7;
    const int cs = c + (c >> 5);
    float amax = 0.0f;
#pragma unroll 16
    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(tile[half * 64 + i][cs]));
    if constexpr (ROWS) {
        part[half * kTq + c] = amax;
        __syncthreads();
        amax = fmaxf(part[c], part[kTq + c]);
    } else {
        amax = warp_max(amax);
        if ((tid & 31) == 0) red[tid >> 5] = amax;
        __syncthreads();
        amax = red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    }
    const GroupScale q = group_scale(amax);
    uint8_t* dst = out + (static_cast<int64_t>(m) * a.C + cb * kTq + c) * kTq + half * 64;
#pragma unroll
    for (int pc = 0; pc < 4; ++pc) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = tile[half * 64 + pc * 16 + i][cs];
        *reinterpret_cast<uint4*>(dst + pc * 16) =
            make_uint4(group_codes4(v, q), group_codes4(v + 4, q), group_codes4(v + 8, q), group_codes4(v + 12, q));
    }
    if constexpr (ROWS) {
        if (half == 0) os[static_cast<int64_t>(m) * a.C + cb * kTq + c] = q.s;
    } else {
        if (tid == 0) os[static_cast<int64_t>(m) * (a.C / kTq) + cb] = q.s;
    }
}

// One block per token: dx = sum over kept slots of dx_rows + sum over all slots of dl * W_g[e] (fp32), bf16.
// A thread takes 8 consecutive columns at a time (16-byte loads of the bf16 rows).
__global__ void __launch_bounds__(256) bwd_dx_kernel(const uint16_t* __restrict__ dxr, const int32_t* __restrict__ slot_row,
                                                     const int32_t* __restrict__ topk_idx, const float* __restrict__ dl,
                                                     const float* __restrict__ Wg, int k, int H,
                                                     uint16_t* __restrict__ dx) {
    const int t = blockIdx.x;
    for (int h = threadIdx.x * 8; h < H; h += blockDim.x * 8) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int32_t r = slot_row[static_cast<int64_t>(t) * k + j];
            if (r < 0) continue;
            const uint4 raw = *reinterpret_cast<const uint4*>(dxr + static_cast<int64_t>(r) * H + h);
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] += __uint_as_float(w[i] << 16);
                acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
            }
        }
        for (int j = 0; j < k; ++j) {
            const int64_t sl = static_cast<int64_t>(t) * k + j;
            const float d = dl[sl];
            const float4* wg = reinterpret_cast<const float4*>(Wg + static_cast<int64_t>(topk_idx[sl]) * H + h);
            const float4 w0 = wg[0], w1 = wg[1];
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(d, wv[i], acc[i]);
        }
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            o[i] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i]))) |
                   (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1]))) << 16);
        *reinterpret_cast<uint4*>(dx + static_cast<int64_t>(t) * H + h) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Block (expert e, chunk of kGateCols columns): dW_g[e, h] = sum over e's slots in token order of dl * x[t, h],
// a thread taking 8 consecutive columns (16-byte loads, four slots' rows in flight); db[e] = sum of dl in
// the same order (the chunk-0 block's first warp: 32 values loaded at once, added in order).
constexpr int kGateCols = 256 * 8;

__global__ void __launch_bounds__(256) bwd_gate_grad_kernel(const uint16_t* __restrict__ x, const float* __restrict__ dl,
                                                            const int32_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ list, int k, int H,
                                                            float* __restrict__ dWg, float* __restrict__ db) {
    const int e = blockIdx.x;
    const int h = blockIdx.y * kGateCols + threadIdx.x * 8;
    const int i0 = offsets[e], i1 = offsets[e + 1];
    if (h < H) {
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
        int i = i0;
        for (; i + 4 <= i1; i += 4) {
            uint4 raw[4];
            float d[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int32_t sl = list[i + u];
                d[u] = dl[sl];
                raw[u] = *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(sl / k) * H + h);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[2 * j] = fmaf(d[u], __uint_as_float(w[j] << 16), acc[2 * j]);
                    acc[2 * j + 1] = fmaf(d[u], __uint_as_float(w[j] & 0xffff0000u), acc[2 * j + 1]);
                }
            }
        }
        for (; i < i1; ++i) {
            const int32_t sl = list[i];
            const float d = dl[sl];
            const uint4 r = *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(sl / k) * H + h);
            const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[2 * j] = fmaf(d, __uint_as_float(w[j] << 16), acc[2 * j]);
                acc[2 * j + 1] = fmaf(d, __uint_as_float(w[j] & 0xffff0000u), acc[2 * j + 1]);
            }
        }
        float4* out = reinterpret_cast<float4*>(dWg + static_cast<int64_t>(e) * H + h);
        out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    if (blockIdx.y == 0 && threadIdx.x < 32) {
        const int lane = threadIdx.x;
        float acc = 0.0f;
        for (int b = i0; b < i1; b += 32) {
            const float v = b + lane < i1 ? dl[list[b + lane]] : 0.0f;
            const int n = min(32, i1 - b);
            for (int j = 0; j < n; ++j) acc += __shfl_sync(0xffffffffu, v, j);
        }
        if (lane == 0) db[e] = acc;
    }
}

static int blocks_for_warps(int64_t warps) { return static_cast<int>((warps + 7) / 8); }

cudaError_t launch_bwd_dl(const uint16_t* dy, const uint16_t* O, const int32_t* slot_row, const float* topk_w, int T,
                          int k, int H, float* dl, cudaStream_t s) {
    bwd_dl_kernel<<<blocks_for_warps(T), 256, 0, s>>>(dy, O, slot_row, topk_w, T, k, H, dl);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dout(const uint16_t* dy, const float* topk_w, const int32_t* row_src, int rows, int k, int H,
                            uint8_t* q, float* sc, cudaStream_t s) {
    bwd_dout_quant_kernel<<<blocks_for_warps(static_cast<int64_t>(rows) * ((H / kGroup + 3) / 4)), 256, 0, s>>>(
        dy, topk_w, row_src, rows, k, H, q, sc);
    return cudaGetLastError();
}

cudaError_t launch_bwd_swiglu(const uint16_t* ab, const uint16_t* dh, const int32_t* row_src, int rows, int I,
                              uint16_t* g, uint8_t* gq, float* gs, cudaStream_t s) {
    bwd_swiglu_kernel<<<blocks_for_warps(static_cast<int64_t>(rows) * ((I / kGroup + 3) / 4)), 256, 0, s>>>(ab, dh, row_src,
                                                                                                rows, I, g, gq, gs);
    return cudaGetLastError();
}

// src: 0 = w * dy, 1 = FP8 codes with 1x128 scales, 2 = bf16; rows: one scale per transposed row.
template <int SRC, bool ROWS>
static cudaError_t launch_tq(const TqArgs& a, uint8_t* out, float* os, cudaStream_t s) {
    constexpr size_t kSmem = sizeof(float) * (kTq * kTqS + 2 * kTq + 8);
    auto kern = bwd_tquant_kernel<SRC, ROWS>;
    const cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
    if (err != cudaSuccess) return err;
    kern<<<dim3(a.rows / kTq, a.C / kTq), 256, kSmem, s>>>(a, out, os);
    return cudaGetLastError();
}

cudaError_t launch_bwd_tquant(int src, bool rows_mode, const TqArgs& a, uint8_t* out, float* os, cudaStream_t s) {
    if (src == kTqDout && rows_mode) return launch_tq<kTqDout, true>(a, out, os, s);
    if (src == kTqFp8 && !rows_mode) return launch_tq<kTqFp8, false>(a, out, os, s);
    if (src == kTqBf16 && rows_mode) return launch_tq<kTqBf16, true>(a, out, os, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dx(const uint16_t* dxr, const int32_t* slot_row, const int32_t* topk_idx, const float* dl,
                          const float* Wg, int T, int k, int H, uint16_t* dx, cudaStream_t s) {
    bwd_dx_kernel<<<T, 256, 0, s>>>(dxr, slot_row, topk_idx, dl, Wg, k, H, dx);
    return cudaGetLastError();
}

cudaError_t launch_bwd_gate(const uint16_t* x, const float* dl, const int32_t* offsets, const int32_t* list, int E, int k,
                            int H, float* dWg, float* db, cudaStream_t s) {
    bwd_gate_grad_kernel<<<dim3(E, (H + kGateCols - 1) / kGateCols), 256, 0, s>>>(x, dl, offsets, list, k, H, dWg, db);
    return cudaGetLastError();
}

}  // namespace moe
