// Router: s = softmax(W_g x + b) in fp32 with top-k selection and weights
// renormalised over the selected experts (MegaMoE page, section 2.2;
// DeepSeek-V4 lecture page, section 2.3; DeepSeek MoE page, chapter 1), and
// hash routing expert = hash(token_id) % E (DeepSeek-V4 lecture page, 2.2).
//
// Logits use one fixed fp32 order so the selected experts are reproducible
// bit for bit: lane j of a warp owns h = j, j+32, j+64, ... and runs one
// fused multiply-add chain over them in ascending h from +0; the 32 partial
// sums are combined by an xor butterfly (j with j^16, then ^8, ^4, ^2, ^1),
// which pairs j with j+16 first, then j+8, ... exactly; the bias is added last.
//
// The logits kernel tiles tokens x experts so each W_g / x element staged in
// shared memory feeds TR x ER register accumulators per lane (CUDA cores: the
// fixed order rules out the tensor cores); logits go to scratch, and a
// warp-per-token kernel selects the top-k and computes the weights in fp64.
// W_g (7.3 MB at the largest size) stays L2-resident across token tiles.
#include "common.cuh"

namespace moe {

constexpr int kRouterHS = 128;     // h values per stage
constexpr int kPlaneRows = kRouterHS;
constexpr int kPlaneBytes = kPlaneRows * 16;   // one plane: 128 rows x 16 bytes

// Operands are staged h-major in "planes" of 16 bytes per h: 8 tokens (bf16) or 4
// experts (fp32) per plane, so a lane fetches all the tokens (experts) it needs for
// its h with one 16-byte load per plane. Rows are XOR-swizzled within each 8-row
// group, and W planes are padded by 32 bytes, so both the transposing stores and the
// 16-byte loads are free of bank conflicts.
__device__ __forceinline__ int swz_row(int row) { return row ^ ((row >> 3) & 7); }

template <int TR, int ER, int WT, int WE>
struct RouterTile {
    static constexpr int TT = TR * WT;               // tokens per CTA
    static constexpr int EC = ER * WE;               // experts per CTA
    static constexpr int kThreads = 32 * WT * WE;
    static constexpr int kXPlanes = TT / 8;
    static constexpr int kWPlanes = EC / 4;
    static constexpr int kWPlaneStride = kPlaneBytes + 32;
    static constexpr int kXBytes = kXPlanes * kPlaneBytes;
    static constexpr int kStageBytes = kXBytes + kWPlanes * kWPlaneStride;
    static constexpr int kSmem = 2 * kStageBytes;
    // global -> register chunks per thread per stage (16 bytes each)
    static constexpr int kXChunks = TT * (kRouterHS / 8) / kThreads;     // 8 h of one token
    static constexpr int kWChunks = EC * (kRouterHS / 4) / kThreads;     // 4 h of one expert
    static_assert(TR % 8 == 0 && ER % 4 == 0, "register tile must cover whole planes");
    static_assert(TT * (kRouterHS / 8) % kThreads == 0 && EC * (kRouterHS / 4) % kThreads == 0, "chunking");
};

template <int TR, int ER, int WT, int WE>
__global__ void __launch_bounds__(RouterTile<TR, ER, WT, WE>::kThreads, 1)
router_logits_kernel(const uint16_t* __restrict__ x, const float* __restrict__ Wg, const float* __restrict__ bias,
                     float* __restrict__ logits, int T, int H, int E) {
    using Tile = RouterTile<TR, ER, WT, WE>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int t_base = blockIdx.x * Tile::TT;
    const int e_base = blockIdx.y * Tile::EC;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int wt = warp / WE, we = warp % WE;
    const int nst = H / kRouterHS;

    // Chunk c of a stage: x chunks are (token, 8-h piece) with 4 pieces of one token per
    // 4 consecutive threads and 8 tokens per warp; W chunks are (expert, 4-h piece) alike.
    uint4 xr[Tile::kXChunks], wr[Tile::kWChunks];
    auto load_stage = [&](int st) {
        const int h0 = st * kRouterHS;
#pragma unroll
        for (int i = 0; i < Tile::kXChunks; ++i) {
            const int c = tid + i * Tile::kThreads;          // 0 .. TT*16
            const int grp = c >> 5, l = c & 31;               // 32 chunks: 8 tokens x 4 pieces
            const int tok = (grp % (Tile::TT / 8)) * 8 + (l >> 2);
            const int piece = (grp / (Tile::TT / 8)) * 4 + (l & 3);
            const int t = t_base + tok;
            xr[i] = t < T ? *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * H + h0 + piece * 8)
                          : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < Tile::kWChunks; ++i) {
            const int c = tid + i * Tile::kThreads;          // 0 .. EC*32
            const int grp = c >> 5, l = c & 31;               // 32 chunks: 8 experts x 4 pieces
            const int ex = (grp % (Tile::EC / 8)) * 8 + (l >> 2);
            const int piece = (grp / (Tile::EC / 8)) * 4 + (l & 3);
            const int e = e_base + ex;
            wr[i] = e < E ? *reinterpret_cast<const uint4*>(Wg + static_cast<int64_t>(e) * H + h0 + piece * 4)
                          : make_uint4(0, 0, 0, 0);
        }
    };
    auto store_stage = [&](int buf) {
        uint8_t* sx = smem + buf * Tile::kStageBytes;
        uint8_t* sw = sx + Tile::kXBytes;
#pragma unroll
        for (int i = 0; i < Tile::kXChunks; ++i) {
            const int c = tid + i * Tile::kThreads;
            const int grp = c >> 5, l = c & 31;
            const int tok = (grp % (Tile::TT / 8)) * 8 + (l >> 2);
            const int piece = (grp / (Tile::TT / 8)) * 4 + (l & 3);
            uint8_t* plane = sx + (tok >> 3) * kPlaneBytes + (tok & 7) * 2;
            const uint32_t u[4] = {xr[i].x, xr[i].y, xr[i].z, xr[i].w};
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int row = piece * 8 + r;
                *reinterpret_cast<uint16_t*>(plane + swz_row(row) * 16) =
                    static_cast<uint16_t>(r & 1 ? u[r >> 1] >> 16 : u[r >> 1] & 0xffffu);
            }
        }
#pragma unroll
        for (int i = 0; i < Tile::kWChunks; ++i) {
            const int c = tid + i * Tile::kThreads;
            const int grp = c >> 5, l = c & 31;
            const int ex = (grp % (Tile::EC / 8)) * 8 + (l >> 2);
            const int piece = (grp / (Tile::EC / 8)) * 4 + (l & 3);
            uint8_t* plane = sw + (ex >> 2) * Tile::kWPlaneStride + (ex & 3) * 4;
            const uint32_t u[4] = {wr[i].x, wr[i].y, wr[i].z, wr[i].w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = piece * 4 + r;
                *reinterpret_cast<uint32_t*>(plane + swz_row(row) * 16) = u[r];
            }
        }
    };

    float acc[TR][ER];
#pragma unroll
    for (int i = 0; i < TR; ++i)
#pragma unroll
        for (int q = 0; q < ER; ++q) acc[i][q] = 0.0f;

    load_stage(0);
    store_stage(0);
    if (nst > 1) load_stage(1);
    __syncthreads();
    for (int st = 0; st < nst; ++st) {
        const uint8_t* sx = smem + (st & 1) * Tile::kStageBytes;
        const uint8_t* sxw = sx + (wt * (TR / 8)) * kPlaneBytes;
        const uint8_t* sww = sx + Tile::kXBytes + (we * (ER / 4)) * Tile::kWPlaneStride;
#pragma unroll
        for (int s = 0; s < kRouterHS / 32; ++s) {
            const int row16 = swz_row(s * 32 + lane) * 16;
            float2 xv[TR / 2];
            float wv[ER];
#pragma unroll
            for (int p = 0; p < TR / 8; ++p) {
                const uint4 v = *reinterpret_cast<const uint4*>(sxw + p * kPlaneBytes + row16);
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    xv[p * 4 + i] = make_float2(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u));
            }
#pragma unroll
            for (int p = 0; p < ER / 4; ++p) {
                const float4 v = *reinterpret_cast<const float4*>(sww + p * Tile::kWPlaneStride + row16);
                wv[p * 4] = v.x; wv[p * 4 + 1] = v.y; wv[p * 4 + 2] = v.z; wv[p * 4 + 3] = v.w;
            }
            // lane j runs the chains for h = j (mod 32), ascending h
#pragma unroll
            for (int i = 0; i < TR / 2; ++i)
#pragma unroll
                for (int q = 0; q < ER; ++q) {
                    acc[2 * i][q] = fmaf(xv[i].x, wv[q], acc[2 * i][q]);
                    acc[2 * i + 1][q] = fmaf(xv[i].y, wv[q], acc[2 * i + 1][q]);
                }
        }
        if (st + 1 < nst) {
            store_stage((st + 1) & 1);       // the buffer read at st - 1; every warp passed the barrier since
            if (st + 2 < nst) load_stage(st + 2);
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < TR; ++i) {
#pragma unroll
        for (int q = 0; q < ER; ++q) {
            float v = acc[i][q];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v = v + __shfl_xor_sync(0xffffffffu, v, o);
            const int t = t_base + wt * TR + i, e = e_base + we * ER + q;
            if (lane == ((i * ER + q) & 31) && t < T && e < E)
                logits[static_cast<int64_t>(t) * E + e] = bias ? v + bias[e] : v;
        }
    }
}

// One warp per token: the k largest logits (ties to the lower expert index),
// in descending order; w_j = exp(l_j - m) / sum_{top-k} exp(l_i - m) in fp64.
template <int EPL>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                          int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    float v[EPL];
    bool taken[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        taken[i] = e >= E;
        v[i] = taken[i] ? 0.0f : logits[static_cast<int64_t>(t) * E + e];
    }
    float sel_l = 0.0f;     // lane j keeps the j-th selected logit
    int sel_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int be = 0x7fffffff;
        bool have = false;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (!taken[i] && (!have || v[i] > bv || (v[i] == bv && e < be))) {
                bv = v[i];
                be = e;
                have = true;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const bool oh = __shfl_xor_sync(0xffffffffu, have ? 1 : 0, o) != 0;
            if (oh && (!have || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
                have = true;
            }
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (be == lane + 32 * i) taken[i] = true;    // every lane agrees on (bv, be)
        if (lane == j) {
            sel_l = bv;
            sel_e = be;
        }
    }
    const double m = static_cast<double>(__shfl_sync(0xffffffffu, sel_l, 0));
    const double ex = lane < k ? exp(static_cast<double>(sel_l) - m) : 0.0;
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += __shfl_sync(0xffffffffu, ex, j);   // j = 0..k-1 in order
    if (lane < k) {
        topk_idx[static_cast<int64_t>(t) * k + lane] = sel_e;
        topk_w[static_cast<int64_t>(t) * k + lane] = static_cast<float>(ex / den);
    }
}

__global__ void router_hash_kernel(const int32_t* __restrict__ token_ids, int T, int E, int32_t* __restrict__ topk_idx,
                                   float* __restrict__ topk_w) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const uint32_t h = static_cast<uint32_t>(token_ids[t]) * 2654435761u;   // wraps mod 2^32
    topk_idx[t] = static_cast<int32_t>(h % static_cast<uint32_t>(E));
    topk_w[t] = 1.0f;
}

template <int TR, int ER, int WT, int WE>
static cudaError_t launch_logits(const uint16_t* x, const float* Wg, const float* bias, float* logits, int T, int H,
                                 int E, cudaStream_t s) {
    using Tile = RouterTile<TR, ER, WT, WE>;
    auto kern = router_logits_kernel<TR, ER, WT, WE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tile::kSmem);
    if (err != cudaSuccess) return err;
    dim3 grid((T + Tile::TT - 1) / Tile::TT, (E + Tile::EC - 1) / Tile::EC);
    kern<<<grid, Tile::kThreads, Tile::kSmem, s>>>(x, Wg, bias, logits, T, H, E);
    return cudaGetLastError();
}

cudaError_t launch_router_softmax(const uint16_t* x, const float* Wg, const float* bias, float* logits, int T, int H,
                                  int E, int k, int32_t* topk_idx, float* topk_w, int num_sms, cudaStream_t s) {
    cudaError_t err;
    // the largest register tile whose CTAs still cover the GPU at least once
    const long ctas_big = static_cast<long>((T + 31) / 32) * ((E + 31) / 32);
    const long ctas_mid = static_cast<long>((T + 15) / 16) * ((E + 15) / 16);
    if (ctas_big >= num_sms)
        err = launch_logits<16, 8, 2, 4>(x, Wg, bias, logits, T, H, E, s);      // 32 tokens x 32 experts
    else if (ctas_mid >= num_sms)
        err = launch_logits<8, 4, 2, 4>(x, Wg, bias, logits, T, H, E, s);       // 16 tokens x 16 experts
    else
        err = launch_logits<8, 4, 1, 4>(x, Wg, bias, logits, T, H, E, s);       // 8 tokens x 16 experts
    if (err != cudaSuccess) return err;
    const int blocks = (T + 7) / 8;
    if (E <= 64)
        router_topk_kernel<2><<<blocks, 256, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    else if (E <= 256)
        router_topk_kernel<8><<<blocks, 256, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    else
        router_topk_kernel<16><<<blocks, 256, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    return cudaGetLastError();
}

cudaError_t launch_router_hash(const int32_t* token_ids, int T, int E, int32_t* topk_idx, float* topk_w,
                               cudaStream_t s) {
    router_hash_kernel<<<(T + 255) / 256, 256, 0, s>>>(token_ids, T, E, topk_idx, topk_w);
    return cudaGetLastError();
}

}  // namespace moe
