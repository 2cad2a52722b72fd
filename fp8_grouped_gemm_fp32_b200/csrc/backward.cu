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
#include "common.cuh"

namespace moe {

constexpr int kTq = 128;   // transposed-quantisation tile: 128 rows x 128 columns

// E4M3 code of v / s (the quotient correctly rounded, then round-to-nearest-even, saturating).
__device__ __forceinline__ uint8_t e4m3_of(float v, float s) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(__fdiv_rn(v, s), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float e4m3_value(uint8_t c) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
    return __half2float(__half(h));
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

// One warp per (row, 128-group): dO = w * dy of the row's slot, quantised (1x128, scale max|v| / 448);
// padding rows get code 0, scale 1. Scales K-block-major [H/128][rows].
__global__ void __launch_bounds__(256) bwd_dout_quant_kernel(const uint16_t* __restrict__ dy,
                                                             const float* __restrict__ topk_w,
                                                             const int32_t* __restrict__ row_src, int rows, int k, int H,
                                                             uint8_t* __restrict__ q, float* __restrict__ s) {
    const int lane = threadIdx.x & 31;
    const int G = H / kGroup;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (item >= static_cast<int64_t>(rows) * G) return;
    const int r = static_cast<int>(item / G), g = static_cast<int>(item % G);
    const int32_t src = row_src[r];
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (src >= 0) {
        const float w = topk_w[src];
        const uint2 raw = *reinterpret_cast<const uint2*>(dy + static_cast<int64_t>(src / k) * H + g * kGroup + lane * 4);
        v[0] = w * __uint_as_float(raw.x << 16);
        v[1] = w * __uint_as_float(raw.x & 0xffff0000u);
        v[2] = w * __uint_as_float(raw.y << 16);
        v[3] = w * __uint_as_float(raw.y & 0xffff0000u);
    }
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    amax = warp_max(amax);
    const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) packed |= static_cast<uint32_t>(amax == 0.0f ? 0u : e4m3_of(v[i], sc)) << (8 * i);
    if (amax == 0.0f)          // all zeros: the codes of the (signed) zeros themselves
        packed = f32x2_to_e4m3x2(v[0], v[1]) | (static_cast<uint32_t>(f32x2_to_e4m3x2(v[2], v[3])) << 16);
    *reinterpret_cast<uint32_t*>(q + static_cast<int64_t>(r) * H + g * kGroup + lane * 4) = packed;
    if (lane == 0) s[static_cast<int64_t>(g) * rows + r] = sc;
}

// One warp per (row, 128-wide block j of I): a, b (bf16, the up GEMM's interleaved a | b columns of block j)
// and dh -> da, db (fp32, rounded to bf16) into g in the same interleaving, then each 128-group of g
// quantised (1x128 along 2I, scales K-block-major [2I/128][rows]). Padding rows: zeros, scale 1.
__global__ void __launch_bounds__(256) bwd_swiglu_kernel(const uint16_t* __restrict__ ab, const uint16_t* __restrict__ dh,
                                                         const int32_t* __restrict__ row_src, int rows, int I,
                                                         uint16_t* __restrict__ g, uint8_t* __restrict__ gq,
                                                         float* __restrict__ gs) {
    const int lane = threadIdx.x & 31;
    const int NJ = I / kGroup;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (item >= static_cast<int64_t>(rows) * NJ) return;
    const int r = static_cast<int>(item / NJ), j = static_cast<int>(item % NJ);
    const bool valid = row_src[r] >= 0;
    const int64_t base = static_cast<int64_t>(r) * 2 * I + j * 2 * kGroup;
    float da[4], db[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int c = lane * 4 + i;
        float dav = 0.0f, dbv = 0.0f;
        if (valid) {
            const float a = bf16_bits_to_f32(ab[base + c]);
            const float b = bf16_bits_to_f32(ab[base + kGroup + c]);
            const float d = bf16_bits_to_f32(dh[static_cast<int64_t>(r) * I + j * kGroup + c]);
            const float sg = 1.0f / (1.0f + expf(-a));
            dav = d * b * sg * (1.0f + a * (1.0f - sg));
            dbv = d * a * sg;
        }
        da[i] = __bfloat162float(__float2bfloat16_rn(dav));
        db[i] = __bfloat162float(__float2bfloat16_rn(dbv));
        g[base + c] = __bfloat16_as_ushort(__float2bfloat16_rn(dav));
        g[base + kGroup + c] = __bfloat16_as_ushort(__float2bfloat16_rn(dbv));
    }
    // the two 128-groups of g this warp wrote: da (group 2j) and db (group 2j + 1)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float* v = h == 0 ? da : db;
        float amax = warp_max(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
        const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
        uint32_t packed = 0;
        if (amax == 0.0f)
            packed = f32x2_to_e4m3x2(v[0], v[1]) | (static_cast<uint32_t>(f32x2_to_e4m3x2(v[2], v[3])) << 16);
        else
#pragma unroll
            for (int i = 0; i < 4; ++i) packed |= static_cast<uint32_t>(e4m3_of(v[i], sc)) << (8 * i);
        *reinterpret_cast<uint32_t*>(gq + base + h * kGroup + lane * 4) = packed;
        if (lane == 0) gs[static_cast<int64_t>(2 * j + h) * rows + r] = sc;
    }
}

// Sources of the transposed quantisation: the value of row r, column c of an activation-like matrix.
enum TqSource { kTqDout = 0, kTqFp8 = 1, kTqBf16 = 2 };

struct TqArgs {
    const uint16_t* dy;       // kTqDout: w * dy of the row's slot
    const float* topk_w;
    const uint8_t* codes;     // kTqFp8: codes [rows, C] with scales [C/128][rows]
    const float* scales;
    const uint16_t* bf;       // kTqBf16: [rows, C]
    const int32_t* row_src;   // the forward layout's rows: slot, or -1 for padding (value 0)
    int rows, k, C;
};

// For forward row tile m (blockIdx.x) and column block cb (blockIdx.y): the transposed 128 x 128 block
// quantised. ROWS: one scale per transposed row (column c over the tile's 128 rows), out scales [tiles][C];
// otherwise one scale for the block, out scales [tiles][C/128]. Codes [tiles * C, 128]: transposed row
// m * C + c holds the 128 rows of the tile.
template <int SRC, bool ROWS>
__global__ void __launch_bounds__(256) bwd_tquant_kernel(TqArgs a, uint8_t* __restrict__ out, float* __restrict__ os) {
    extern __shared__ float tq_smem[];                     // [kTq][kTq + 1] values, then 8 partial maxima
    float (*tile)[kTq + 1] = reinterpret_cast<float (*)[kTq + 1]>(tq_smem);
    float* red = tq_smem + kTq * (kTq + 1);
    const int m = blockIdx.x, cb = blockIdx.y;
    const int tid = threadIdx.x;
    // load: thread (rr, cc) with 2 rows per pass
    for (int i = tid; i < kTq * kTq; i += blockDim.x) {
        const int rr = i / kTq, cc = i % kTq;
        const int row = m * kTq + rr, col = cb * kTq + cc;
        const int32_t src = a.row_src[row];
        float v = 0.0f;
        if (src >= 0) {
            if constexpr (SRC == kTqDout) {
                v = a.topk_w[src] * bf16_bits_to_f32(a.dy[static_cast<int64_t>(src / a.k) * a.C + col]);
            } else if constexpr (SRC == kTqFp8) {
                v = e4m3_value(a.codes[static_cast<int64_t>(row) * a.C + col]) *
                    a.scales[static_cast<int64_t>(col / kGroup) * a.rows + row];
            } else {
                v = bf16_bits_to_f32(a.bf[static_cast<int64_t>(row) * a.C + col]);
            }
        }
        tile[rr][cc] = v;
    }
    __syncthreads();
    // thread (c, half): column c, rows half * 64 .. half * 64 + 63
    const int c = tid >> 1, half = tid & 1;
    float amax = 0.0f;
    for (int rr = half * 64; rr < half * 64 + 64; ++rr) amax = fmaxf(amax, fabsf(tile[rr][c]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    if constexpr (!ROWS) {
        amax = warp_max(amax);
        if ((tid & 31) == 0) red[tid >> 5] = amax;
        __syncthreads();
        amax = red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    }
    const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
    uint8_t* dst = out + (static_cast<int64_t>(m) * a.C + cb * kTq + c) * kTq + half * 64;
    for (int p = 0; p < 4; ++p) {
        uint32_t w4[4];
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float v = tile[half * 64 + p * 16 + qd * 4 + i][c];
                const uint32_t code = amax == 0.0f ? static_cast<uint32_t>(f32x2_to_e4m3x2(v, 0.0f) & 0xff)
                                                   : static_cast<uint32_t>(e4m3_of(v, sc));
                packed |= code << (8 * i);
            }
            w4[qd] = packed;
        }
        *reinterpret_cast<uint4*>(dst + p * 16) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    if constexpr (ROWS) {
        if (half == 0) os[static_cast<int64_t>(m) * a.C + cb * kTq + c] = sc;
    } else {
        if (tid == 0) os[static_cast<int64_t>(m) * (a.C / kTq) + cb] = sc;
    }
}

// One block per token: dx = sum over kept slots of dx_rows + sum over all slots of dl * W_g[e] (fp32), bf16.
__global__ void __launch_bounds__(256) bwd_dx_kernel(const uint16_t* __restrict__ dxr, const int32_t* __restrict__ slot_row,
                                                     const int32_t* __restrict__ topk_idx, const float* __restrict__ dl,
                                                     const float* __restrict__ Wg, int k, int H,
                                                     uint16_t* __restrict__ dx) {
    const int t = blockIdx.x;
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        float acc = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int64_t s = static_cast<int64_t>(t) * k + j;
            const int32_t r = slot_row[s];
            if (r >= 0) acc += bf16_bits_to_f32(dxr[static_cast<int64_t>(r) * H + h]);
        }
        for (int j = 0; j < k; ++j) {
            const int64_t s = static_cast<int64_t>(t) * k + j;
            acc = fmaf(dl[s], Wg[static_cast<int64_t>(topk_idx[s]) * H + h], acc);
        }
        dx[static_cast<int64_t>(t) * H + h] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
    }
}

// Block (expert e, 256-column chunk): dW_g[e, h] = sum over e's slots in token order of dl * x[t, h];
// db[e] = sum of dl (the chunk-0 block).
__global__ void __launch_bounds__(256) bwd_gate_grad_kernel(const uint16_t* __restrict__ x, const float* __restrict__ dl,
                                                            const int32_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ list, int k, int H,
                                                            float* __restrict__ dWg, float* __restrict__ db) {
    const int e = blockIdx.x;
    const int h = blockIdx.y * blockDim.x + threadIdx.x;
    const int i0 = offsets[e], i1 = offsets[e + 1];
    if (h < H) {
        float acc = 0.0f;
        for (int i = i0; i < i1; ++i) {
            const int32_t s = list[i];
            acc = fmaf(dl[s], bf16_bits_to_f32(x[static_cast<int64_t>(s / k) * H + h]), acc);
        }
        dWg[static_cast<int64_t>(e) * H + h] = acc;
    }
    if (blockIdx.y == 0 && threadIdx.x == 0) {
        float acc = 0.0f;
        for (int i = i0; i < i1; ++i) acc += dl[list[i]];
        db[e] = acc;
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
    bwd_dout_quant_kernel<<<blocks_for_warps(static_cast<int64_t>(rows) * (H / kGroup)), 256, 0, s>>>(
        dy, topk_w, row_src, rows, k, H, q, sc);
    return cudaGetLastError();
}

cudaError_t launch_bwd_swiglu(const uint16_t* ab, const uint16_t* dh, const int32_t* row_src, int rows, int I,
                              uint16_t* g, uint8_t* gq, float* gs, cudaStream_t s) {
    bwd_swiglu_kernel<<<blocks_for_warps(static_cast<int64_t>(rows) * (I / kGroup)), 256, 0, s>>>(ab, dh, row_src,
                                                                                                rows, I, g, gq, gs);
    return cudaGetLastError();
}

// src: 0 = w * dy, 1 = FP8 codes with 1x128 scales, 2 = bf16; rows: one scale per transposed row.
template <int SRC, bool ROWS>
static cudaError_t launch_tq(const TqArgs& a, uint8_t* out, float* os, cudaStream_t s) {
    constexpr size_t kSmem = sizeof(float) * (kTq * (kTq + 1) + 8);
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
    bwd_gate_grad_kernel<<<dim3(E, (H + 255) / 256), 256, 0, s>>>(x, dl, offsets, list, k, H, dWg, db);
    return cudaGetLastError();
}

}  // namespace moe
