// Combine: y[t, :] = sum_{j < k, slot kept} w[t, j] * O[slot_row[t*k + j], :]
// (MegaMoE page, section 2.1: y = sum_{i in TopK} G(x)_i * E_i(x)), summed in
// fp32 in slot order and rounded to bf16 to nearest even (section 3.3).
// Dropped slots contribute nothing and the other weights are not rescaled.
//
// HBM-bound: each block streams whole rows with 16-byte vector loads; a row
// of y is produced by one block and written once.
#include "common.cuh"

namespace moe {

template <int VPT>   // 16-byte vectors per thread per row
__global__ void __launch_bounds__(128) combine_kernel(const uint16_t* __restrict__ O, const int32_t* __restrict__ slot_row,
                                                      const float* __restrict__ topk_w, int T, int k, int H,
                                                      uint16_t* __restrict__ y) {
    const int t = blockIdx.x;
    const int nvec = H / 8;
    float acc[VPT][8];
#pragma unroll
    for (int v = 0; v < VPT; ++v)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[v][i] = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int32_t row = slot_row[static_cast<int64_t>(t) * k + j];
        if (row < 0) continue;
        const float w = topk_w[static_cast<int64_t>(t) * k + j];
        const uint4* src = reinterpret_cast<const uint4*>(O + static_cast<int64_t>(row) * H);
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            const int idx = threadIdx.x + v * 128;
            if (idx < nvec) {
                const uint4 q = src[idx];
                const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[v][2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[v][2 * i]);
                    acc[v][2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xffff0000u), acc[v][2 * i + 1]);
                }
            }
        }
    }
    uint4* dst = reinterpret_cast<uint4*>(y + static_cast<int64_t>(t) * H);
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        const int idx = threadIdx.x + v * 128;
        if (idx < nvec) {
            uint32_t u[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(acc[v][2 * i], acc[v][2 * i + 1]);
                u[i] = *reinterpret_cast<const uint32_t*>(&b);
            }
            dst[idx] = make_uint4(u[0], u[1], u[2], u[3]);
        }
    }
}

cudaError_t launch_combine(const uint16_t* O, const int32_t* slot_row, const float* topk_w, int T, int k, int H,
                           uint16_t* y, cudaStream_t s) {
    const int nvec = H / 8;
    const int vpt = (nvec + 127) / 128;
    if (vpt <= 2)
        combine_kernel<2><<<T, 128, 0, s>>>(O, slot_row, topk_w, T, k, H, y);
    else if (vpt <= 4)
        combine_kernel<4><<<T, 128, 0, s>>>(O, slot_row, topk_w, T, k, H, y);
    else if (vpt <= 8)
        combine_kernel<8><<<T, 128, 0, s>>>(O, slot_row, topk_w, T, k, H, y);
    else if (vpt <= 16)
        combine_kernel<16><<<T, 128, 0, s>>>(O, slot_row, topk_w, T, k, H, y);
    else
        return cudaErrorInvalidValue;   // H > 16384 is rejected before launch
    return cudaGetLastError();
}

}  // namespace moe
