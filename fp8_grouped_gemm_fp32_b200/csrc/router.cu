// Router: s = softmax(W_g x + b) in fp32 with top-k selection and weights
// renormalised over the selected experts (MegaMoE page, section 2.2;
// DeepSeek-V4 lecture page, section 2.3; DeepSeek MoE page, chapter 1), and
// hash routing expert = hash(token_id) % E (DeepSeek-V4 lecture page, 2.2).
//
// Logits use one fixed fp32 order so the selected experts are reproducible
// bit for bit: lane j of a warp owns h = 128 s + 4 j + i (i = 0..3, every
// 128-wide block s of H) and runs one fused multiply-add chain over them in
// ascending h from +0; the 32 partial sums are combined by an xor butterfly
// (j with j^16, then ^8, ^4, ^2, ^1), which pairs j with j+16 first, then
// j+8, ... exactly; the bias is added last.
//
// The logits kernel tiles tokens x experts: one thread streams 128-wide
// blocks of x ([tokens, h], bf16) and W_g ([experts, h], fp32) with TMA into a
// ring of shared-memory stages, row-major as they lie in global memory, and
// each compute warp keeps a TR x ER register tile per lane, so every 16-byte
// W_g load feeds 4 * TR and every 8-byte x load 4 * ER multiply-adds (CUDA
// cores: the fixed order rules out the tensor cores). Logits go to scratch,
// and a warp-per-token kernel selects the top-k and computes the weights in
// fp64. W_g (7.3 MB at the largest size) stays L2-resident across token tiles.
#include <algorithm>

#include "common.cuh"

namespace moe {

constexpr int kRouterHS = 128;     // h values per stage: lane j takes h = 4j .. 4j+3 of each

// DP: a dedicated producer warp issues the loads (small tiles, where the compute warps are few and
// quick); otherwise thread 0, a compute thread, refills each stage's slot as soon as every warp is done.
template <int TR, int ER, int WT, int WE, bool DP>
struct RouterCfg {
    static constexpr int TT = TR * WT;                  // tokens per CTA
    static constexpr int EC = ER * WE;                  // experts per CTA
    static constexpr int kWarps = WT * WE;              // compute warps
    static constexpr int kThreads = 32 * (kWarps + (DP ? 1 : 0));
    static constexpr int kXBytes = TT * kRouterHS * 2;
    static constexpr int kWBytes = EC * kRouterHS * 4;
    static constexpr int kStageBytes = kXBytes + kWBytes;
    // a power of two (slot and phase of a stage by mask and shift), up to 8, within 200 KB
    static constexpr int kStages = 8 * kStageBytes <= 200 * 1024 ? 8 : 4 * kStageBytes <= 200 * 1024 ? 4 : 2;
    static constexpr int kSmem = kStages * kStageBytes + 2 * kStages * 8 + 16 + 1024;
};

template <int TR, int ER, int WT, int WE, bool DP>
__global__ void __launch_bounds__(RouterCfg<TR, ER, WT, WE, DP>::kThreads, 1)
router_logits_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const float* __restrict__ bias, float* __restrict__ logits, int T, int H, int E, int* status,
                     uint64_t wait_ns) {
    using C = RouterCfg<TR, ER, WT, WE, DP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
    uint64_t* empty = full + C::kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::kStages);
    const int lane = threadIdx.x & 31;
    const int warp = (threadIdx.x >> 5) - (DP ? 1 : 0);             // compute warp index; -1: producer warp
    const int wt = warp / WE, we = warp % WE;
    const int nst = H / kRouterHS;
    const bool producer = threadIdx.x == 0;
    // Persistent: the CTA takes tiles blockIdx.x, blockIdx.x + gridDim.x, ... of (token tile, expert tile),
    // the expert tile varying fastest so that the CTAs running together share each x tile through L2.
    // The stage ring runs on across tiles: global stage g = (the CTA's i-th tile) * nst + stage in tile.
    const int ET = (E + C::EC - 1) / C::EC;
    const int tiles = ((T + C::TT - 1) / C::TT) * ET;
    const int my_tiles = static_cast<int>(blockIdx.x) < tiles ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const uint32_t stages_total = static_cast<uint32_t>(my_tiles) * nst;

    auto fail = [&]() {
        set_status(status, kStatusTimeout);
        *abort_flag = 1;
    };
    // Stages are issued strictly in order (only thread 0 issues): the next one's tile (the CTA's pf_it-th)
    // and stage within it are kept as running counters, so issuing costs no division by the stage count.
    int pf_it = 0, pf_st = 0, pf_t0 = 0, pf_e0 = 0;
    auto pf_tile = [&]() {
        const int tile = blockIdx.x + pf_it * gridDim.x;
        pf_t0 = (tile / ET) * C::TT;
        pf_e0 = (tile % ET) * C::EC;
    };
    auto issue = [&](uint32_t g) {      // global stage g (the next in order) into slot g % kStages
        const int s = static_cast<int>(g % C::kStages);
        uint8_t* stage = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        tma_load_2d(stage, &tmX, &full[s], pf_st * kRouterHS, pf_t0);
        tma_load_2d(stage + C::kXBytes, &tmW, &full[s], pf_st * kRouterHS, pf_e0);
        if (++pf_st == nst) {
            pf_st = 0;
            ++pf_it;
            pf_tile();
        }
    };
    if (producer) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::kWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmW);
        pf_tile();
        for (uint32_t g = 0; g < C::kStages && g < stages_total; ++g) issue(g);
    }
    __syncthreads();

    if (DP && warp < 0) {
        // dedicated producer: refill each slot as soon as every compute warp has finished with it
        if (producer)
            for (uint32_t g = C::kStages; g < stages_total && !*abort_flag; ++g) {
                const uint32_t u = g / C::kStages - 1;
                if (!mbar_wait(&empty[g % C::kStages], u & 1, wait_ns)) { fail(); break; }
                issue(g);
            }
        __syncthreads();
        if (*abort_flag) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 200000) __nanosleep(1000);
        }
        return;
    }
    bool ok = true;
    uint32_t g = 0;
    for (int it = 0; it < my_tiles && ok; ++it) {
    const int tile = blockIdx.x + it * gridDim.x;
    const int t_base = (tile / ET) * C::TT, e_base = (tile % ET) * C::EC;
    // acc2[p][q] holds the chains of tokens 2p and 2p + 1 with expert q: one packed fp32x2 multiply-add
    // advances both (each half rounds exactly as a scalar fused multiply-add) for half the issue slots
    static_assert(TR % 2 == 0, "tokens are paired");
    float2 acc2[TR / 2][ER];
#pragma unroll
    for (int i = 0; i < TR / 2; ++i)
#pragma unroll
        for (int q = 0; q < ER; ++q) acc2[i][q] = make_float2(0.0f, 0.0f);
    for (int st = 0; st < nst; ++st, ++g) {
        // the slot of stage g - 1 takes stage g - 1 + kStages once every warp has finished with it
        if (!DP && producer && g > 0 && g - 1 + C::kStages < stages_total) {
            if (!mbar_wait(&empty[(g - 1) % C::kStages], ((g - 1) / C::kStages) & 1, wait_ns))
                fail();
            else
                issue(g - 1 + C::kStages);
        }
        const int s = static_cast<int>(g % C::kStages);
        if (*abort_flag || !mbar_wait(&full[s], (g / C::kStages) & 1, wait_ns)) {
            fail();
            ok = false;
            break;
        }
        const uint8_t* stage = smem + s * C::kStageBytes;
        const uint16_t* xs = reinterpret_cast<const uint16_t*>(stage) + (wt * TR) * kRouterHS + 4 * lane;
        const float* ws = reinterpret_cast<const float*>(stage + C::kXBytes) + (we * ER) * kRouterHS + 4 * lane;
        float4 wv[ER];
#pragma unroll
        for (int q = 0; q < ER; ++q) wv[q] = *reinterpret_cast<const float4*>(ws + q * kRouterHS);
#pragma unroll
        for (int i = 0; i < TR / 2; ++i) {
            const uint2 xa = *reinterpret_cast<const uint2*>(xs + (2 * i) * kRouterHS);
            const uint2 xb = *reinterpret_cast<const uint2*>(xs + (2 * i + 1) * kRouterHS);
            const float2 x0 = make_float2(__uint_as_float(xa.x << 16), __uint_as_float(xb.x << 16));
            const float2 x1 = make_float2(__uint_as_float(xa.x & 0xffff0000u), __uint_as_float(xb.x & 0xffff0000u));
            const float2 x2 = make_float2(__uint_as_float(xa.y << 16), __uint_as_float(xb.y << 16));
            const float2 x3 = make_float2(__uint_as_float(xa.y & 0xffff0000u), __uint_as_float(xb.y & 0xffff0000u));
            // lane j's chain for (token, expert) runs over h = 4j, 4j+1, 4j+2, 4j+3 of this block in order
#pragma unroll
            for (int q = 0; q < ER; ++q) {
                acc2[i][q] = __ffma2_rn(x0, make_float2(wv[q].x, wv[q].x), acc2[i][q]);
                acc2[i][q] = __ffma2_rn(x1, make_float2(wv[q].y, wv[q].y), acc2[i][q]);
                acc2[i][q] = __ffma2_rn(x2, make_float2(wv[q].z, wv[q].z), acc2[i][q]);
                acc2[i][q] = __ffma2_rn(x3, make_float2(wv[q].w, wv[q].w), acc2[i][q]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (ok) {
        // The 32 chains of each (token, expert) meet in the canonical halving tree: lanes j and j ^ 16,
        // then j ^ 8, ^4, ^2, ^1. As a reduce-scatter: at each level a lane keeps half of its remaining
        // values, adds its partner's copy of them (the same pair of partial sums, so the same fp32
        // sums as the full butterfly: addition is commutative) and sends the other half, so the
        // TR * ER sums cost TR * ER - TR * ER / 32 shuffles instead of 5 per sum; each lane ends with
        // TR * ER / 32 finished logits.
        constexpr int NV = TR * ER;
        static_assert(NV % 32 == 0, "the register tile must spread evenly over the lanes");
        float* v = &acc2[0][0].x;             // value n: token 2 (n / (2 ER)) + (n & 1), expert (n / 2) % ER
        int base = 0;
#pragma unroll
        for (int lvl = 0; lvl < 5; ++lvl) {
            const int w = 16 >> lvl;
            constexpr int kC0 = NV;
            const int half = (kC0 >> lvl) >> 1;
            const bool upper = (lane & w) != 0;
#pragma unroll
            for (int m = 0; m < (NV >> 1); ++m) {
                if (m < half) {
                    const float send = upper ? v[m] : v[m + half];
                    const float recv = __shfl_xor_sync(0xffffffffu, send, w);
                    v[m] = (upper ? v[m + half] : v[m]) + recv;
                }
            }
            base += upper ? half : 0;
        }
#pragma unroll
        for (int m = 0; m < NV / 32; ++m) {
            const int n = base + m;
            const int t = t_base + wt * TR + 2 * (n / (2 * ER)) + (n & 1), e = e_base + we * ER + (n >> 1) % ER;
            if (t < T && e < E) logits[static_cast<int64_t>(t) * E + e] = bias ? v[m] + bias[e] : v[m];
        }
    }
    }
    __syncthreads();
    if (*abort_flag) {
        // let TMA copies that were already issued land before the shared memory is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000) __nanosleep(1000);
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

// 2-D map over a row-major matrix [rows, cols] of 2- or 4-byte elements, read in boxes of 128 columns x
// box_rows rows without swizzling; rows past the end read as zeros.
static bool make_router_map(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                            uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * elem_bytes};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kRouterHS), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int TR, int ER, int WT, int WE, bool DP>
static cudaError_t launch_logits(const uint16_t* x, const float* Wg, const float* bias, float* logits, int T, int H,
                                 int E, int* status, uint64_t wait_ns, int num_sms, cudaStream_t s) {
    using C = RouterCfg<TR, ER, WT, WE, DP>;
    CUtensorMap mx, mw;
    if (!make_router_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, H, T, C::TT) ||
        !make_router_map(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, Wg, H, E, C::EC))
        return cudaErrorInvalidValue;
    auto kern = router_logits_kernel<TR, ER, WT, WE, DP>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (err != cudaSuccess) return err;
    const long tiles = static_cast<long>((T + C::TT - 1) / C::TT) * ((E + C::EC - 1) / C::EC);
    const int grid = static_cast<int>(std::min<long>(tiles, num_sms));     // one CTA per SM, persistent
    kern<<<grid, C::kThreads, C::kSmem, s>>>(mx, mw, bias, logits, T, H, E, status, wait_ns);
    return cudaGetLastError();
}

cudaError_t launch_router_softmax(const uint16_t* x, const float* Wg, const float* bias, float* logits, int T, int H,
                                  int E, int k, int32_t* topk_idx, float* topk_w, int* status, uint64_t wait_ns,
                                  int num_sms, cudaStream_t s) {
    cudaError_t err;
    // the largest register tile whose CTAs still cover the GPU at least once
    const long ctas_big = static_cast<long>((T + 31) / 32) * ((E + 31) / 32);
    const long ctas_mid = static_cast<long>((T + 15) / 16) * ((E + 15) / 16);
    if (ctas_big >= num_sms)
        // 32 tokens x 32 experts in 8 warps of 16 x 8: 224 registers a thread and no spills (16 warps of
        // 8 x 8 must fit in 128 and spill), twice the multiply-adds per shared-memory load; 6-11 % faster
        err = launch_logits<16, 8, 2, 4, false>(x, Wg, bias, logits, T, H, E, status, wait_ns, num_sms, s);
    else if (ctas_mid >= num_sms)
        err = launch_logits<8, 4, 2, 4, true>(x, Wg, bias, logits, T, H, E, status, wait_ns, num_sms, s);   // 16 tokens x 16 experts
    else
        err = launch_logits<8, 4, 1, 4, true>(x, Wg, bias, logits, T, H, E, status, wait_ns, num_sms, s);   // 8 tokens x 16 experts
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
