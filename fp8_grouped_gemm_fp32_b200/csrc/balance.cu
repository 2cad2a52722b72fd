// Auxiliary-loss-free load balancing of the routing bias (MegaMoE page,
// section 2.2): every expert keeps a bias b_e inside the router softmax; over
// an update interval the slots routed to each expert are tallied, and when
// the interval ends an expert above the mean load has its bias lowered by a
// fixed step, one below it raised, one at the mean left alone (the page
// recommends a step of order 1e-3 every 100 steps). The comparison with the
// mean is exact, E * load[e] against the total in 64-bit integers, and the
// step is one fp32 round-to-nearest addition.
//
// E <= 512 experts fit one block: one thread per expert, a shuffle and
// shared-memory sum of the tally, then each thread updates its own expert.
#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(512) balance_bias_kernel(int E, const int32_t* __restrict__ counts,
                                                           int64_t* __restrict__ load, float* __restrict__ bias,
                                                           float gamma, int update) {
    __shared__ long long warp_sum[16];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    long long l = 0;
    if (e < E) l = static_cast<long long>(load[e]) + counts[e];
    if (!update) {   // uniform across the block
        if (e < E) load[e] = l;
        return;
    }
    long long s = l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) warp_sum[warp] = s;
    __syncthreads();
    long long total = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) total += warp_sum[w];
    if (e < E) {
        const long long scaled = static_cast<long long>(E) * l;
        float b = bias[e];
        if (scaled > total)
            b = __fsub_rn(b, gamma);   // above the mean: lower
        else if (scaled < total)
            b = __fadd_rn(b, gamma);   // below the mean: raise
        bias[e] = b;
        load[e] = 0;
    }
}

cudaError_t launch_balance_bias(int E, const int32_t* counts, int64_t* load, float* bias, float gamma, int update,
                                cudaStream_t s) {
    const int threads = (E + 31) / 32 * 32;
    balance_bias_kernel<<<1, threads, 0, s>>>(E, counts, load, bias, gamma, update);
    return cudaGetLastError();
}

}  // namespace moe
