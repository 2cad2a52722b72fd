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
#include "common.cuh"

namespace moe {

constexpr int kRouterHS = 128;     // h values per pipeline stage
constexpr int kRouterStages = 3;

template <int TR, int ER, int WT, int WE>
struct RouterTile {
    static constexpr int TT = TR * WT;       // tokens per CTA
    static constexpr int EC = ER * WE;       // experts per CTA
    static constexpr int kThreads = 32 * WT * WE;
    static constexpr int kXBytes = TT * kRouterHS * 2;
    static constexpr int kWBytes = EC * kRouterHS * 4;
    static constexpr int kStageBytes = kXBytes + kWBytes;
    static constexpr int kSmem = kRouterStages * kStageBytes;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
    const uint32_t s = smem_u32(smem);
    const int bytes = valid ? 16 : 0;   // 0 source bytes -> the 16 bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int TR, int ER, int WT, int WE>
__global__ void __launch_bounds__(RouterTile<TR, ER, WT, WE>::kThreads, 1)
router_logits_kernel(const uint16_t* __restrict__ x, const float* __restrict__ Wg, const float* __restrict__ bias,
                     float* __restrict__ logits, int T, int H, int E) {
    using Tile = RouterTile<TR, ER, WT, WE>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int t_base = blockIdx.x * Tile::TT;
    const int e_base = blockIdx.y * Tile::EC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wt = warp / WE, we = warp % WE;
    const int nst = H / kRouterHS;

    auto issue_stage = [&](int st) {
        uint8_t* sx = smem + (st % kRouterStages) * Tile::kStageBytes;
        uint8_t* sw = sx + Tile::kXBytes;
        const int h0 = st * kRouterHS;
        // x tile: TT rows x 256 bytes = TT*16 chunks; W tile: EC rows x 512 bytes = EC*32 chunks
        for (int c = threadIdx.x; c < Tile::TT * 16; c += Tile::kThreads) {
            const int r = c >> 4, q = c & 15;
            const int t = t_base + r;
            const bool ok = t < T;
            const uint16_t* src = x + static_cast<int64_t>(ok ? t : 0) * H + h0 + q * 8;
            cp_async16(sx + r * 256 + q * 16, src, ok);
        }
        for (int c = threadIdx.x; c < Tile::EC * 32; c += Tile::kThreads) {
            const int r = c >> 5, q = c & 31;
            const int e = e_base + r;
            const bool ok = e < E;
            const float* src = Wg + static_cast<int64_t>(ok ? e : 0) * H + h0 + q * 4;
            cp_async16(sw + r * 512 + q * 16, src, ok);
        }
    };

    float acc[TR][ER];
#pragma unroll
    for (int i = 0; i < TR; ++i)
#pragma unroll
        for (int q = 0; q < ER; ++q) acc[i][q] = 0.0f;

#pragma unroll
    for (int st = 0; st < kRouterStages - 1; ++st) {
        if (st < nst) issue_stage(st);
        cp_async_commit();
    }
    for (int st = 0; st < nst; ++st) {
        cp_async_wait<kRouterStages - 2>();
        __syncthreads();
        if (st + kRouterStages - 1 < nst) issue_stage(st + kRouterStages - 1);
        cp_async_commit();
        const uint8_t* sx = smem + (st % kRouterStages) * Tile::kStageBytes;
        const uint16_t* xs = reinterpret_cast<const uint16_t*>(sx) + (wt * TR) * kRouterHS;
        const float* ws = reinterpret_cast<const float*>(sx + Tile::kXBytes) + (we * ER) * kRouterHS;
#pragma unroll
        for (int s = 0; s < kRouterHS / 32; ++s) {
            const int h = s * 32 + lane;
            float xv[TR], wv[ER];
#pragma unroll
            for (int i = 0; i < TR; ++i) xv[i] = bf16_bits_to_f32(xs[i * kRouterHS + h]);
#pragma unroll
            for (int q = 0; q < ER; ++q) wv[q] = ws[q * kRouterHS + h];
#pragma unroll
            for (int i = 0; i < TR; ++i)
#pragma unroll
                for (int q = 0; q < ER; ++q) acc[i][q] = fmaf(xv[i], wv[q], acc[i][q]);
        }
    }
    cp_async_wait<0>();

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
    // large token x expert tiles when they still give a couple of waves, small ones otherwise
    const long big_ctas = static_cast<long>((T + 31) / 32) * ((E + 31) / 32);
    if (big_ctas >= 2L * num_sms)
        err = launch_logits<8, 16, 4, 2>(x, Wg, bias, logits, T, H, E, s);
    else
        err = launch_logits<2, 4, 4, 2>(x, Wg, bias, logits, T, H, E, s);
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
