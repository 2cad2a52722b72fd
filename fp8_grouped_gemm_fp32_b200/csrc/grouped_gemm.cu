// FP8 grouped GEMM on the sm_100a tensor cores (tcgen05 + tensor memory).
//
// Problem (MegaMoE page, sections 2.1 and 3.2): one GEMM per expert group;
// every group has its own M (tokens), all groups share N and K; A is the
// groups' rows concatenated, B = [E, N, K] ("nt": both K-major). FP8 E4M3
// operands with fine-grained fp32 scales: one per 1x128 activation group and
// one per 128x128 weight block (DeepSeek open-source week page, "Day 3").
// FP8 tensor-core partial sums are promoted to fp32 on the CUDA cores, where
// the scales are applied (same page: two-level accumulation), and the fp32
// accumulator is converted to bf16 with round-to-nearest-even only at the end
// (MegaMoE page, 3.3). The up projection fuses SwiGLU and the 1x128 FP8
// requantisation of h into its epilogue (3.2: epilogue fusion).
//
// Two kernels, both persistent (one CTA per SM) and warp-specialised:
//
// * contiguous layout (prefill): tiles of 128 rows x 256 columns over the
//   flattened, 128-padded M of all groups (the pages' global tile scheduler,
//   3.2). Warp 0 issues TMA loads into a 3- or 4-stage shared-memory ring,
//   bulk copies of each K block's 128 activation scales into a ring of their
//   own, and stages each tile's weight-block scales; warp 1 issues
//   tcgen05.mma (kind::f8f6f4, M=128, N=256, K=32) for each 128-wide K block
//   into one of two tensor-memory buffers; 8 promotion warps read each
//   finished block with tcgen05.ld and fold it into fp32 register
//   accumulators scaled by sa[row] * sw[block], then run the epilogue, whose
//   output leaves through shared memory and TMA stores. Tiles are ordered
//   expert -> N tile -> M tile, so the CTAs working at the same time share
//   one weight tile through L2.
// * masked layout (decode, few tokens per expert): swap-AB. The weight block
//   is the MMA's M=128 operand and up to 32 tokens are its N, so weights
//   stream from HBM in 16 KB (or 2 x 16 KB) stages while the token tile is
//   tiny; experts with no tokens produce no tiles. A second weight format,
//   4-bit levels -7..7 with one fp32 scale per weight row per 128-wide K
//   block (DeepSeek-V4 lecture page, 3.1), runs through the same kernel:
//   TMA brings the packed levels into a deep ring, four converter warps
//   expand them to E4M3 codes (every level is exact in E4M3) and write them
//   into tensor memory, from where the MMA reads its A operand (no expanded
//   copy passes through shared memory), and each promotion thread applies its
//   own row's scale.
//
// Every wait on an mbarrier is bounded; a wait that runs out records
// MOE_ERR_DEVICE_TIMEOUT, the CTA stops issuing work, lets copies and MMAs in
// flight land, frees its tensor memory and returns.
#include "common.cuh"

namespace moe {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kSaSlots = 8;                   // ring of per-K-block activation scales (128 rows each)
constexpr int kMaxKB = 128;                   // K <= 16384
constexpr int kABytes = kBM * kBK;            // 16 KB
constexpr int kBBytes = kBN * kBK;            // 32 KB
constexpr int kThreadsC = 384;                // 12 warps
// setmaxnreg split: 4 warps give registers up, 8 promotion warps take them.
constexpr int kRegsLow = 40, kRegsHigh = 232;
constexpr int kRegsSplit = 128 * kRegsLow + 256 * kRegsHigh;   // must fit the launch allocation
constexpr int kDrainNs = 200000;              // settle time after an abort

// Outputs leave through shared memory and TMA stores in boxes of 32 rows x 64 bytes (64-byte
// swizzle): bf16 (EPI 0) as four 32 x 32 boxes per promotion warp (its 32 rows x 128 columns;
// one fewer operand stage makes room for them), FP8 h (EPI 1) as one 32 x 64 box per warp.
constexpr int kOutBox = 32;
constexpr int kOutBoxBytes = kOutBox * kOutBox * 2;            // 2 KB
constexpr int kOutStageBytes = 8 * 4 * kOutBoxBytes;           // 64 KB

// PAIR: the two CTAs of a cluster compute one 256-row x 256-column tile with pair MMAs; each holds its
// 128 A rows and its 128-row half of the B tile, so a stage is 32 KB instead of 48 KB.
template <int EPI, bool PAIR = false>
struct SmemC {
    static constexpr int kBStage = PAIR ? kBBytes / 2 : kBBytes;
    static constexpr int kStages = PAIR ? (EPI == 0 ? 4 : 6) : (EPI == 0 ? 3 : 4);
    uint8_t a[kStages][kABytes];
    uint8_t b[kStages][kBStage];
    uint8_t out[EPI == 0 ? kOutStageBytes : 8 * kOutBoxBytes];
    float sa[kSaSlots][kBM];    // activation scales of one K block for the tile's 128 rows
    float wsc[2][2][kMaxKB];    // weight-block scales of a tile (two tiles in flight): [tile & 1][block][kb]
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t wfull[2];
    uint64_t wempty[2];
    uint64_t sfull[kSaSlots];
    uint64_t sempty[kSaSlots];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t red_bar[2];
    float red[2][2][kBM];
    uint32_t tmem_base;
    volatile int abort_flag;
    int32_t P[kMaxE + 1];
    int32_t Q[PAIR ? kMaxE + 1 : 1];     // PAIR: prefix of the pair tiles per expert, ceil(M tiles / 2)
};

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Largest e in [0, E) with P[e] <= q (P non-decreasing, P[0] = 0 <= q).
__device__ __forceinline__ int find_group(const int32_t* P, int E, int q) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P[mid] <= q) lo = mid; else hi = mid - 1;
    }
    return lo;
}

struct TileC {
    int e, m0, n0, width;
    bool store;      // false for the idle half of a lone pair tile: computed, not written
    int kb0, nkb;    // the tile's K blocks: kb0 .. kb0 + nkb - 1 (K-grouped: the expert's forward row tiles)
    int am0;         // K-grouped: the tile's first row within each K block's operand block
};

__device__ __forceinline__ TileC decode_tile_c(const int32_t* P, int E, int NT, int N, int tile) {
    TileC t;
    const int q = tile / NT;
    t.e = find_group(P, E, q);
    const int mt_e = P[t.e + 1] - P[t.e];
    const int local = tile - NT * P[t.e];
    const int nt = local / mt_e;
    t.m0 = (P[t.e] + local % mt_e) * kBM;
    t.n0 = nt * kBN;
    t.width = min(kBN, N - t.n0);
    t.store = true;
    return t;
}

// Pair tiles: an expert's M tiles are taken two at a time (the leader the first, the other CTA the second);
// with an odd count the last pair is lone: both CTAs load the leader's rows and only the leader stores.
// Order: expert -> N tile -> pair, so the pairs running at the same time share a weight tile through L2.
__device__ __forceinline__ TileC decode_tile_pair(const int32_t* P, const int32_t* Q, int E, int NT, int tile,
                                                  uint32_t rank) {
    TileC t;
    const int q = tile / NT;
    t.e = find_group(Q, E, q);
    const int mt_e = P[t.e + 1] - P[t.e];
    const int pr_e = Q[t.e + 1] - Q[t.e];
    const int local = tile - NT * Q[t.e];
    const int nt = local / pr_e;
    const int pp = local % pr_e;
    const bool lone = 2 * pp + 1 == mt_e;
    t.m0 = (P[t.e] + 2 * pp + (lone ? 0 : static_cast<int>(rank))) * kBM;
    t.n0 = nt * kBN;
    t.width = kBN;
    t.store = !(lone && rank == 1);
    return t;
}

__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

// KG (K-grouped, the weight gradients of the backward pass): expert e's output is its own M_rows x N
// matrix (rows e * M_rows ...); its K blocks are the expert's 128-row tiles of a forward contiguous layout
// (offsets, kg_rows rows in all), and K block m of the A operand is the [M_rows, 128] block at rows
// m * M_rows of A (of B: rows m * N); A's scales are [tiles][M_rows] (one per row per K block), B's
// [tiles][N / 128] (one per 128-row block per K block).
template <int EPI, bool PAIR, bool KG = false>
__global__ void __launch_bounds__(kThreadsC, 1)
gg_contig_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmD, const float* __restrict__ As, const int32_t* __restrict__ offsets, int M_rows,
                 const float* __restrict__ Bs, int E, int N, int K, void* __restrict__ D, float* __restrict__ Ds,
                 int* status, uint64_t wait_ns, int kg_rows, uint16_t* __restrict__ save_ab) {
    static_assert(!KG || (EPI == 0 && !PAIR), "K-grouped tiles run on single CTAs with the bf16 epilogue");
    extern __shared__ uint8_t smem_raw[];
    using SC = SmemC<EPI, PAIR>;
    constexpr int kStagesC = SC::kStages;
    SC& sm = *reinterpret_cast<SC*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / kBK;
    const int NB = N / kBM;                 // 128-wide weight blocks along N
    const int NT = (N + kBN - 1) / kBN;
    // PAIR: this CTA's rank in its cluster of two (0 = leader, which issues the MMAs), the cluster's index
    // and count (the persistent tile loop runs over clusters); otherwise each CTA works alone
    const uint32_t rank = PAIR ? cluster_ctarank() : 0;
    const int tile0 = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
    const int tstep = PAIR ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);

    // group prefix in M tiles: P[e] = offsets[e] / 128. Offsets that are not non-decreasing multiples of
    // 128 within [0, M_rows] (P[0] = 0) are forced into that shape by a running maximum of the clamped
    // values and reported, so that no tile reads or writes past row M_rows
    if (warp == 0) {
        int carry = 0;
        bool bad = false;
        for (int b = 0; b <= E; b += 32) {
            const int e = b + lane;
            const int o = e <= E ? offsets[e] : 0;
            int v = e == 0 ? 0 : min(max(o, 0), KG ? kg_rows : M_rows) / kBM;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, d);
                if (lane >= d) v = max(v, u);
            }
            v = max(v, carry);
            if (e <= E) {
                sm.P[e] = v;
                bad |= o != v * kBM;
            }
            carry = __shfl_sync(0xffffffffu, v, 31);
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, kStatusCapacity);
        if constexpr (KG) {
            // a K-grouped tile stages at most kMaxKB weight-block scales: longer experts are reported
            __syncwarp();
            bool longk = false;
            for (int e = lane; e < E; e += 32) longk |= sm.P[e + 1] - sm.P[e] > kMaxKB;
            if (__any_sync(0xffffffffu, longk) && lane == 0) set_status(status, kStatusCapacity);
        }
        if constexpr (PAIR) {
            // pair tiles per expert: Q[e + 1] - Q[e] = ceil((P[e + 1] - P[e]) / 2)
            __syncwarp();
            int qc = 0;
            if (lane == 0) sm.Q[0] = 0;
            for (int b = 0; b < E; b += 32) {
                const int e = b + lane;
                int v = e < E ? (sm.P[e + 1] - sm.P[e] + 1) >> 1 : 0;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, v, d);
                    if (lane >= d) v += u;
                }
                if (e < E) sm.Q[e + 1] = qc + v;
                qc += __shfl_sync(0xffffffffu, v, 31);
            }
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesC; ++s) {
            mbar_init(&sm.full[s], 1);
            // a stage is free once this CTA's eight promotion warps have seen its K block's accumulator
            // complete (the MMA commits once per K block, to the accumulator buffer only)
            mbar_init(&sm.empty[s], 8);
        }
        for (int j = 0; j < kSaSlots; ++j) {
            mbar_init(&sm.sfull[j], 1);
            mbar_init(&sm.sempty[j], 8);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            // PAIR: the leader's accumulator buffer is free when both CTAs' promotion warps have read it
            mbar_init(&sm.tempty[b], PAIR ? 16 : 8);
            mbar_init(&sm.red_bar[b], 256);
            mbar_init(&sm.wfull[b], 1);
            mbar_init(&sm.wempty[b], 8);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(&sm.tmem_base, 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&sm.tmem_base, 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if constexpr (PAIR) cluster_sync(); else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int MTd = M_rows / kBM;             // K-grouped: M tiles of each expert's output
    const int total = KG ? E * MTd * NT : (PAIR ? sm.Q[E] : sm.P[E]) * NT;
    auto decode = [&](int tile) -> TileC {
        TileC t;
        if constexpr (KG) {
            // expert -> N tile -> M tile: the tiles running together share the expert's B blocks
            t.e = tile / (NT * MTd);
            const int rem = tile - t.e * NT * MTd;
            const int nt = rem / MTd;
            t.am0 = (rem - nt * MTd) * kBM;
            t.m0 = t.e * M_rows + t.am0;
            t.n0 = nt * kBN;
            t.width = min(kBN, N - t.n0);
            t.store = true;
            t.kb0 = sm.P[t.e];
            t.nkb = min(sm.P[t.e + 1] - sm.P[t.e], kMaxKB);
            return t;
        } else {
            if constexpr (PAIR) t = decode_tile_pair(sm.P, sm.Q, E, NT, tile, rank);
            else t = decode_tile_c(sm.P, E, NT, N, tile);
            t.kb0 = 0;
            t.nkb = KB;
            t.am0 = t.m0;
            return t;
        }
    };

    // A wait that runs out stops this CTA and (PAIR) its partner, whose waits on this CTA would otherwise
    // only end at their own limits.
    auto fail = [&]() {
        set_status(status, kStatusTimeout);
        sm.abort_flag = 1;
        if constexpr (PAIR) st_shared_cluster_u32(mapa_shared(smem_u32((const void*)&sm.abort_flag), rank ^ 1u), 1u);
    };

    // Register split (launch: 384 threads x 168 = 64512): the TMA/MMA warpgroup gives up
    // registers to the two promotion warpgroups, 128 x 40 + 256 x 232 = 64512.
    if (warp < 4) {
      setmaxnreg_dec<kRegsLow>();
      if (warp == 0) {
        // ---------------- producer: TMA loads (lane 0) and, per tile, the weight-block scales (all lanes)
        if (lane == 0) {
            prefetch_tensormap(&tmA);
            prefetch_tensormap(&tmB);
        }
        // A tile's 2 x KB weight-block scales go to slot (tile index) & 1, freed when the promotion warps
        // finish the tile two before. The next tile's scales are read into registers while this tile's
        // loads are issued, so their latency stays off the TMA stream.
        float wr0[4], wr1[4];
        auto read_scales = [&](const TileC& u) {
            if constexpr (KG) {
                // K block kb of the tile is forward row tile u.kb0 + kb; B's scales are [tiles][N / 128]
                const float* b0 = Bs + static_cast<int64_t>(u.kb0) * NB + u.n0 / kBM;
                const int d1 = u.width == kBN ? 1 : 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kb = lane + 32 * i;
                    wr0[i] = kb < u.nkb ? b0[static_cast<int64_t>(kb) * NB] : 0.0f;
                    wr1[i] = kb < u.nkb ? b0[static_cast<int64_t>(kb) * NB + d1] : 0.0f;
                }
            } else {
                const float* b0 = Bs + (static_cast<int64_t>(u.e) * NB + u.n0 / kBM) * KB;
                const float* b1 = u.width == kBN ? b0 + KB : b0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kb = lane + 32 * i;
                    wr0[i] = kb < KB ? b0[kb] : 0.0f;
                    wr1[i] = kb < KB ? b1[kb] : 0.0f;
                }
            }
        };
        auto publish_scales = [&](uint32_t ti) -> bool {
            const int ws = ti & 1;
            int ok = 1;
            if (lane == 0) ok = !sm.abort_flag && mbar_wait(&sm.wempty[ws], ((ti >> 1) & 1) ^ 1, wait_ns);
            if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
            // K-grouped tiles have their own K block count (at most kMaxKB; read_scales zeroed the rest)
            const int lim = KG ? kMaxKB : KB;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kb = lane + 32 * i;
                if (kb < lim) {
                    sm.wsc[ws][0][kb] = wr0[i];
                    sm.wsc[ws][1][kb] = wr1[i];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.wfull[ws]);
            return true;
        };
        uint32_t it = 0, ti = 0;
        TileC t{};
        t.e = -1;                                    // no tile (a CTA past the last tile decodes nothing)
        if (tile0 < total) {
            t = decode(tile0);
            read_scales(t);
            if (!publish_scales(0)) {
                if (lane == 0 && !sm.abort_flag) fail();
                t.e = -1;
            }
        }
        for (int tile = tile0; tile < total && t.e >= 0; tile += tstep, ++ti) {
            const int nxt = tile + tstep;
            TileC tn = t;
            if (nxt < total) {
                tn = decode(nxt);
                read_scales(tn);
            }
            int ok = 1;
            if (lane == 0) {
                // PAIR: both CTAs' loads count on the leader's full barrier, which the leader arms with the
                // bytes of both (its MMA reads both CTAs' stages); each CTA loads its A rows and its half of B
                const uint32_t bytes = PAIR ? 2u * (kABytes + SC::kBStage)
                                            : kABytes + (t.width == kBN ? kBBytes : kBBytes / 2);
                for (int kb = 0; kb < t.nkb; ++kb, ++it) {
                    const int s = it % kStagesC;
                    const uint32_t ph = (it / kStagesC) & 1;
                    if (!mbar_wait(&sm.empty[s], ph ^ 1, wait_ns)) { fail(); ok = 0; break; }
                    if constexpr (KG) {
                        // operand blocks of forward row tile kb0 + kb: A rows (kb0 + kb) * M_rows + am0,
                        // B rows (kb0 + kb) * N + n0, each 128 bytes of K
                        const int m = t.kb0 + kb;
                        mbar_arrive_expect_tx(&sm.full[s], bytes);
                        tma_load_2d(sm.a[s], &tmA, &sm.full[s], 0, m * M_rows + t.am0);
                        tma_load_2d(sm.b[s], &tmB, &sm.full[s], 0, m * N + t.n0);
                        if (t.width == kBN) tma_load_2d(sm.b[s] + kBBytes / 2, &tmB, &sm.full[s], 0, m * N + t.n0 + 128);
                    } else if constexpr (PAIR) {
                        const uint32_t fb = mapa_shared(smem_u32(&sm.full[s]), 0);
                        if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], bytes);
                        tma_load_2d_pair(sm.a[s], &tmA, fb, kb * kBK, t.m0);
                        tma_load_2d_pair(sm.b[s], &tmB, fb, kb * kBK, t.e * N + t.n0 + static_cast<int>(rank) * 128);
                    } else {
                        mbar_arrive_expect_tx(&sm.full[s], bytes);
                        tma_load_2d(sm.a[s], &tmA, &sm.full[s], kb * kBK, t.m0);
                        tma_load_2d(sm.b[s], &tmB, &sm.full[s], kb * kBK, t.e * N + t.n0);
                        if (t.width == kBN)
                            tma_load_2d(sm.b[s] + kBBytes / 2, &tmB, &sm.full[s], kb * kBK, t.e * N + t.n0 + 128);
                    }
                    // the 128 activation scales of this K block, into the scale ring
                    const int j = it % kSaSlots;
                    if (!mbar_wait(&sm.sempty[j], ((it / kSaSlots) & 1) ^ 1, wait_ns)) { fail(); ok = 0; break; }
                    mbar_arrive_expect_tx(&sm.sfull[j], kBM * sizeof(float));
                    bulk_load(sm.sa[j], As + static_cast<int64_t>(t.kb0 + kb) * M_rows + t.am0, kBM * sizeof(float),
                              &sm.sfull[j]);
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if (nxt < total && !publish_scales(ti + 1)) {
                if (lane == 0 && !sm.abort_flag) fail();
                break;
            }
            t = tn;
        }
      } else if (warp == 1) {
        // ---------------- MMA issuer (PAIR: the leader only, for both CTAs)
        if (lane == 0 && rank == 0) {
            uint32_t it = 0, kbt = 0;
            for (int tile = tile0; tile < total && !sm.abort_flag; tile += tstep) {
                const TileC t = decode(tile);
                const uint32_t idesc = PAIR ? f8_idesc(2 * kBM, kBN) : f8_idesc(kBM, t.width);
                for (int kb = 0; kb < t.nkb; ++kb, ++it, ++kbt) {
                    const int s = it % kStagesC;
                    const uint32_t ph = (it / kStagesC) & 1;
                    const int buf = kbt & 1;
                    const uint32_t bph = (kbt >> 1) & 1;
                    if (!mbar_wait(&sm.full[s], ph, wait_ns)) { fail(); break; }
                    if (!mbar_wait(&sm.tempty[buf], bph ^ 1, wait_ns)) { fail(); break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
                    const uint32_t d = tmem + buf * kBN;
                    if constexpr (PAIR) {
#pragma unroll
                        for (int kk = 0; kk < kBK / 32; ++kk)
                            umma_f8_pair(d, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc,
                                         kk > 0);
                        umma_commit_pair(&sm.tfull[buf], 0x3);   // both CTAs' accumulator buffer is ready
                    } else {
#pragma unroll
                        for (int kk = 0; kk < kBK / 32; ++kk)
                            umma_f8(d, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc,
                                    kk > 0);
                        umma_commit(&sm.tfull[buf]);
                    }
                }
            }
        }
      }
    } else {
        setmaxnreg_inc<kRegsHigh>();
        // ---------------- promotion + epilogue (256 threads)
        const int q = warp & 3;                 // tensor-memory lane quadrant
        const int half = (warp - 4) >> 2;       // which 64 columns of each 128-column half
        const int row = q * 32 + lane;          // row within the tile
        uint32_t kbt = 0, ep = 0;
        uint32_t ti = 0;
        // PAIR: the accumulator buffer is released on the leader's barrier, which counts both CTAs' warps
        const uint32_t tempty_leader0 = PAIR ? mapa_shared(smem_u32(&sm.tempty[0]), 0) : 0u;
        for (int tile = tile0; tile < total; tile += tstep, ++ti) {
            if (sm.abort_flag) break;
            const TileC t = decode(tile);
            const bool full = t.width == kBN;
            // the tile's weight-block scales, staged by the producer warp
            const int ws = ti & 1;
            if (!mbar_wait(&sm.wfull[ws], (ti >> 1) & 1, wait_ns)) { fail(); break; }
            // acc2[i] holds columns (2i, 2i+1) of this thread's 128 (64 from each 128-column half)
            float2 acc2[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) acc2[i] = make_float2(0.0f, 0.0f);
            float* acc = reinterpret_cast<float*>(acc2);
            bool ok = true;
            for (int kb = 0; kb < t.nkb; ++kb, ++kbt) {
                const int buf = kbt & 1;
                const uint32_t bph = (kbt >> 1) & 1;
                // scales: sa from the ring (the producer copied it several K blocks ago), the weight
                // block scales from the registers of the lane that holds them
                const int j = kbt % kSaSlots;
                if (!mbar_wait(&sm.sfull[j], (kbt / kSaSlots) & 1, wait_ns)) { fail(); ok = false; break; }
                const float sa = sm.sa[j][row];
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sempty[j]);
                const float w0 = sm.wsc[ws][0][kb];
                const float w1 = sm.wsc[ws][1][kb];
                const float f0 = sa * w0;
                const float f1 = sa * w1;
                if (!mbar_wait(&sm.tfull[buf], bph, wait_ns)) { fail(); ok = false; break; }
                // the K block's MMAs are done, so its operand stage (this CTA's; in a pair the leader's MMA
                // read both CTAs' stages, and the commit reached both) can be refilled
                if (lane == 0) mbar_arrive(&sm.empty[kbt % kStagesC]);
                tc_fence_after();
                const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * kBN + half * 64;
                // The buffer is handed back to the MMA warp as soon as the last of its columns is in
                // registers; the multiply-adds of the second weight block run after the release.
                auto release = [&]() {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (PAIR && rank != 0)
                            mbar_arrive_cluster(tempty_leader0 + buf * static_cast<uint32_t>(sizeof(uint64_t)));
                        else
                            mbar_arrive(&sm.tempty[buf]);
                    }
                };
                auto fold = [&](float2* dst, const float (&v)[32], float f) {
                    const float2 ff = make_float2(f, f);
#pragma unroll
                    for (int i = 0; i < 16; ++i) dst[i] = __ffma2_rn(make_float2(v[2 * i], v[2 * i + 1]), ff, dst[i]);
                };
                float va[32], vb[32];
                tmem_ld32(taddr, va);
                tmem_ld32(taddr + 32, vb);
                tmem_ld_wait();
                if (full) {
                    fold(acc2, va, f0);
                    tmem_ld32(taddr + 128, va);
                    fold(acc2 + 16, vb, f0);
                    tmem_ld32(taddr + 160, vb);
                    tmem_ld_wait();
                    release();
                    fold(acc2 + 32, va, f1);
                    fold(acc2 + 48, vb, f1);
                } else {
                    release();
                    fold(acc2, va, f0);
                    fold(acc2 + 16, vb, f0);
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.wempty[ws]);          // the tile's weight scales are no longer read
            const int64_t grow = t.m0 + row;
            if (!t.store) {
                // the idle half of a lone pair tile: its rows belong to the leader, which stores them; the
                // SwiGLU epilogue's barrier phase still advances so both halves stay in step
                if constexpr (EPI == 1) {
                    const int p = ep & 1;
                    mbar_arrive(&sm.red_bar[p]);
                    if (!mbar_wait(&sm.red_bar[p], (ep >> 1) & 1, wait_ns)) { fail(); break; }
                    ++ep;
                }
            } else if constexpr (EPI == 0) {
                // this warp's 32 rows x 128 columns as four 32 x 32 boxes: box (r, c) holds columns
                // n0 + r * 128 + half * 64 + c * 32 + [0, 32); 16-byte pieces are placed with the
                // 64-byte swizzle (piece p of row l at p ^ ((l >> 1) & 3)), which the store undoes
                const uint32_t stage = smem_u32(sm.out) + (warp - 4) * 4 * kOutBoxBytes;
                if (lane == 0) bulk_wait_read_all();          // the previous tile's stores have read it
                __syncwarp();
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    if (r == 1 && !full) break;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t box = stage + (r * 2 + c) * kOutBoxBytes + lane * 64;
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            uint32_t u[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int col = r * 64 + c * 32 + p * 8 + 2 * i;
                                const __nv_bfloat162 b = __floats2bfloat162_rn(acc[col], acc[col + 1]);
                                u[i] = *reinterpret_cast<const uint32_t*>(&b);
                            }
                            st_shared_v4(box + ((p ^ ((lane >> 1) & 3)) << 4), u[0], u[1], u[2], u[3]);
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        if (r == 1 && !full) break;
#pragma unroll
                        for (int c = 0; c < 2; ++c)
                            tma_store_2d(&tmD, sm.out + (warp - 4) * 4 * kOutBoxBytes + (r * 2 + c) * kOutBoxBytes,
                                         t.n0 + r * 128 + half * 64 + c * 32, t.m0 + q * 32);
                    }
                    bulk_commit();
                }
            } else {
                if (save_ab) {
                    // training: the gate and up values themselves, rounded to bf16, kept for the backward
                    // pass ([M_rows, N] in W13's interleaved column order, as a bf16-output GEMM writes them)
                    uint16_t* dst = save_ab + grow * N + t.n0 + half * 64;
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb)
#pragma unroll
                        for (int p = 0; p < 8; ++p) {
                            uint32_t u[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const __nv_bfloat162 b2 =
                                    __floats2bfloat162_rn(acc[hb * 64 + p * 8 + 2 * i], acc[hb * 64 + p * 8 + 2 * i + 1]);
                                u[i] = *reinterpret_cast<const uint32_t*>(&b2);
                            }
                            *reinterpret_cast<uint4*>(dst + hb * kBM + p * 8) = make_uint4(u[0], u[1], u[2], u[3]);
                        }
                }
                // SwiGLU on (a = acc[0..63], b = acc[64..127]) for h columns n0/2 + half*64 + [0, 64)
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    acc[i] = silu_f(acc[i]) * acc[64 + i];
                    amax = fmaxf(amax, fabsf(acc[i]));
                }
                const int p = ep & 1;
                sm.red[p][half][row] = amax;
                mbar_arrive(&sm.red_bar[p]);
                if (!mbar_wait(&sm.red_bar[p], (ep >> 1) & 1, wait_ns)) { fail(); break; }
                ++ep;
                amax = fmaxf(sm.red[p][0][row], sm.red[p][1][row]);
                const float s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
                // h / s as h * (1 / s): the correctly rounded reciprocal keeps the quotient within one
                // ulp of the division, below the resolution of the E4M3 code it is rounded to
                const float rs = amax == 0.0f ? 1.0f : __frcp_rn(s);
                // this warp's 32 rows x 64 codes leave as one 32 x 64-byte box through shared memory
                // (64-byte swizzle: 16-byte piece p of row l at p ^ ((l >> 1) & 3))
                const uint32_t box = smem_u32(sm.out) + (warp - 4) * kOutBoxBytes;
                if (lane == 0) bulk_wait_read_all();          // the previous tile's store has read it
                __syncwarp();
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    uint32_t u[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = p * 16 + i * 4;
                        u[i] = f32x2_to_e4m3x2(acc[c] * rs, acc[c + 1] * rs) |
                               (static_cast<uint32_t>(f32x2_to_e4m3x2(acc[c + 2] * rs, acc[c + 3] * rs)) << 16);
                    }
                    st_shared_v4(box + lane * 64 + ((p ^ ((lane >> 1) & 3)) << 4), u[0], u[1], u[2], u[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmD, sm.out + (warp - 4) * kOutBoxBytes, t.n0 / 2 + half * 64, t.m0 + q * 32);
                    bulk_commit();
                }
                if (half == 0) Ds[static_cast<int64_t>(t.n0 / kBN) * M_rows + grow] = s;
            }
        }
    }

    if (warp >= 4 && lane == 0) bulk_wait_all();   // the output stores have completed
    tc_fence_before();
    // PAIR: neither CTA leaves while the leader's MMAs may still read the other's shared memory or write its
    // tensor memory; after this barrier both abort flags are final
    if constexpr (PAIR) cluster_sync(); else __syncthreads();
    if (sm.abort_flag) {
        // let TMA copies and MMAs that were already issued land before the memory is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < kDrainNs) __nanosleep(1000);
    }
    if constexpr (PAIR) cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

// ====================================================================== masked layout, swap-AB
constexpr int kBT = 32;                       // tokens per tile (the MMA's N)
constexpr int kXBytes = kBT * kBK;            // 4 KB
constexpr int kWBlk = kBM * kBK;              // 16 KB: 128 weight rows x 128 K bytes
// threads: warp 0 TMA, warp 1 MMA, then the promotion warps: four for SwiGLU (a thread holds a weight
// row's 32 gate and 32 up columns), eight for the bf16 output (two warps per lane quadrant, 16 token
// columns each, so two warps share each scheduler's promotion work)
// With 4-bit weights (W4) more warps, one per tensor-memory lane quadrant and K-block parity, expand each
// stage's packed levels to E4M3 codes and write them into tensor memory, where the MMA reads its A operand:
// eight for the bf16 output (two sets of four take alternate K blocks, so one set's load, expansion and
// store latency overlaps the other's), four for SwiGLU (whose promotion threads need the registers).
template <int EPI, bool W4 = false>
__host__ __device__ constexpr int conv_warps() { return W4 ? (EPI == 1 ? 4 : 8) : 0; }
template <int EPI, bool W4 = false>
__host__ __device__ constexpr int masked_threads() { return (EPI == 1 ? 192 : 320) + 32 * conv_warps<EPI, W4>(); }

__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Eight 4-bit weight levels of consecutive k (one 32-bit word of the packed row: level i < 4 has its
// magnitude in bits 4i..4i+2 and its sign in bit 8i+7, level 4+i its magnitude in bits 16+4i..16+4i+2
// and its sign in bit 8i+3) to eight E4M3 codes, k order, two words. A byte permute looks the magnitudes'
// codes up (0..7 are exact in E4M3: 0x00 38 40 44 48 4a 4c 4e) and the sign bits, already at bit 7 of
// their bytes (after a 4-bit shift for the upper four), are or-ed in: E4M3's sign is its top bit.
__device__ __forceinline__ void w4x8_to_e4m3x8(uint32_t w, uint32_t& lo, uint32_t& hi) {
    lo = prmt_b32(0x44403800u, 0x4e4c4a48u, w & 0x7777u) | (w & 0x80808080u);
    hi = prmt_b32(0x44403800u, 0x4e4c4a48u, (w >> 16) & 0x7777u) | ((w << 4) & 0x80808080u);
}

// WIDE (bf16 output only): a tile takes two consecutive 128-row weight blocks, so that each K block's fixed
// cost (barriers, the commit, the promotion round trip) is spread over twice the weight bytes.
template <int EPI, bool W4 = false, bool WIDE = false>
struct SmemM {
    static constexpr bool kTwo = EPI == 1 || WIDE;              // two 128-row weight blocks per tile
    static constexpr int kW = kTwo ? 2 * kWBlk : kWBlk;        // weight bytes per stage: 256 rows (a|b, or two) or 128
    // W4: a deep ring of packed stages (8 or 16 KB of levels + the 4 KB token tile each); the expanded
    // codes live in tensor memory (kA slots) instead of shared memory
    static constexpr int kStages = W4 ? (kTwo ? 8 : 16) : (EPI == 1 ? 4 : WIDE ? 5 : 10);
    static constexpr int kWS = W4 ? 16 : kW;                   // expanded codes in shared memory (FP8 only)
    static constexpr int kWP = W4 ? kW / 2 : 16;               // packed 4-bit levels per stage (W4 only)
    static constexpr int kCols = kTwo ? 2 * kBT : kBT;         // tensor-memory columns per accumulator buffer
    static constexpr int kBufs = 4;                            // MMA runs up to 3 K blocks ahead of promotion
    static constexpr int kSaSlots = 16;                        // scale ring deeper than the stage ring
    static constexpr int kACols = kW / kBM / 4;                // W4: tensor-memory columns of one A slot (32 or 64)
    // W4: A slots after the accumulators, as many as the accumulator buffers: the MMA of K block j uses
    // slot and buffer j % 4, so the buffer's completion also frees the slot
    static constexpr int kA = W4 ? kBufs : 1;
    static constexpr uint32_t kTmemCols = W4 ? 512u : static_cast<uint32_t>(kBufs * kCols);
    static_assert(!W4 || kBufs * kCols + kA * kACols <= 512, "tensor memory holds the accumulators and A slots");
    alignas(1024) uint8_t x[kStages][kXBytes];                  // 128-byte swizzled tiles: 1024-byte aligned
    alignas(1024) uint8_t w[kStages][kWS];
    alignas(1024) uint8_t wp[kStages][kWP];                     // packed levels (W4), 64 bytes per row, 64-byte swizzle
    float hs[EPI == 1 ? 2 : 1][EPI == 1 ? kBT : 1][kBM];       // SwiGLU output staged for the requant
    float sa[kSaSlots][kBT];                                    // activation scales of one K block, 32 tokens
    // W4: the tile's weight-row scales of the same K block (128 rows, or the 256 gate and up rows), copied
    // with the activation scales and released with them, so the promotion warps read no global memory
    float wrs[W4 ? kSaSlots : 1][W4 ? kW / kBK : 1];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t afull[kA];                                         // W4: A slot written by the converter warps
    uint64_t sfull[kSaSlots];
    uint64_t sempty[kSaSlots];
    uint64_t tfull[kBufs];
    uint64_t tempty[kBufs];
    uint64_t red_bar[2];
    uint32_t tmem_base;
    volatile int abort_flag;
    int32_t P[kMaxE + 1];
    int32_t M[kMaxE];                                           // tokens per expert (masked_m)
};

// every layout, plus the 1 KB the kernels spend aligning it, within the 227 KB a CTA may use
constexpr size_t kSmemLimit = 232448;
static_assert(sizeof(SmemC<0, false>) + 1024 <= kSmemLimit && sizeof(SmemC<1, false>) + 1024 <= kSmemLimit &&
              sizeof(SmemC<0, true>) + 1024 <= kSmemLimit && sizeof(SmemC<1, true>) + 1024 <= kSmemLimit,
              "contiguous kernel shared memory");
static_assert(sizeof(SmemM<0, false>) + 1024 <= kSmemLimit && sizeof(SmemM<1, false>) + 1024 <= kSmemLimit &&
              sizeof(SmemM<0, true>) + 1024 <= kSmemLimit && sizeof(SmemM<1, true>) + 1024 <= kSmemLimit &&
              sizeof(SmemM<0, false, true>) + 1024 <= kSmemLimit && sizeof(SmemM<0, true, true>) + 1024 <= kSmemLimit,
              "masked kernel shared memory");

template <int EPI, bool W4, bool WIDE = false>
__global__ void __launch_bounds__(masked_threads<EPI, W4>(), 1)
gg_masked_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const float* __restrict__ As, const int32_t* __restrict__ masked_m, int Mmax,
                 const float* __restrict__ Bs, int E, int N, int K, void* __restrict__ D, float* __restrict__ Ds,
                 int* status, uint64_t wait_ns) {
    static_assert(!WIDE || EPI == 0, "two output blocks per tile: bf16 epilogue only");
    using S = SmemM<EPI, W4, WIDE>;
    constexpr bool kTwo = S::kTwo;
    extern __shared__ uint8_t smem_raw[];
    S& sm = *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kPW = EPI == 1 ? 4 : 8;                      // promotion warps (2 .. 2 + kPW - 1)
    constexpr int kConvWarp0 = 2 + kPW;                        // W4: converter warps (conv_warps of them)
    constexpr int kConvSets = conv_warps<EPI, W4>() / 4;       // sets of four, taking alternate K blocks
    const int KB = K / kBK;
    const int NB = N / kBM;                          // 128-row weight blocks per expert
    const int NBt = kTwo ? NB / 2 : NB;              // weight tiles per expert
    constexpr uint32_t kTmemCols = S::kTmemCols;
    constexpr uint32_t kA0 = S::kBufs * S::kCols;              // W4: first column of the A slots

    if (warp == 0) {
        // tile prefix over experts: tiles_e = NBt * ceil(m_e / 32)
        int32_t carry = 0;
        if (lane == 0) sm.P[0] = 0;
        for (int b = 0; b < E; b += 32) {
            const int e = b + lane;
            // a block holds at most Mmax rows: a count outside [0, Mmax] is clamped (and reported) so
            // that no tile reads or writes past its expert's block
            const int32_t m_in = e < E ? masked_m[e] : 0;
            const int32_t m = min(max(m_in, 0), Mmax);
            if (m != m_in) set_status(status, kStatusCapacity);
            if (e < E) sm.M[e] = m;
            int32_t v = NBt * ((m + kBT - 1) / kBT);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (e < E) sm.P[e + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < S::kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            // a stage is free once the promotion warps have seen its K block's accumulator complete (the MMA
            // has read its token tile) and, W4, the four converter warps have read its levels
            mbar_init(&sm.empty[s], W4 ? 4 + kPW : kPW);
        }
        for (int a = 0; a < S::kA; ++a) {
            mbar_init(&sm.afull[a], 4);
        }
        for (int j = 0; j < S::kSaSlots; ++j) {
            mbar_init(&sm.sfull[j], 1);
            mbar_init(&sm.sempty[j], kPW);
        }
        for (int b = 0; b < S::kBufs; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], kPW);
        }
        for (int b = 0; b < 2; ++b) mbar_init(&sm.red_bar[b], 128);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int total = sm.P[E];

    auto fail = [&]() {
        set_status(status, kStatusTimeout);
        sm.abort_flag = 1;
    };
    auto decode = [&](int tile, int& e, int& nb, int& tt, int& m_e) {
        e = find_group(sm.P, E, tile);
        m_e = sm.M[e];
        const int ntt = (m_e + kBT - 1) / kBT;
        const int local = tile - sm.P[e];
        nb = local / ntt;
        tt = local % ntt;
    };

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&tmX);
            prefetch_tensormap(&tmW);
            uint32_t it = 0;
            for (int tile = blockIdx.x; tile < total && !sm.abort_flag; tile += gridDim.x) {
                int e, nb, tt, m_e;
                decode(tile, e, nb, tt, m_e);
                const int wrow = e * N + nb * (kTwo ? 2 * kBM : kBM);
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % S::kStages;
                    const uint32_t ph = (it / S::kStages) & 1;
                    if (!mbar_wait(&sm.empty[s], ph ^ 1, wait_ns)) { fail(); break; }
                    if constexpr (W4) {
                        mbar_arrive_expect_tx(&sm.full[s], S::kWP + kXBytes);
                        tma_load_2d(sm.wp[s], &tmW, &sm.full[s], kb * (kBK / 2), wrow);
                        if (kTwo) tma_load_2d(sm.wp[s] + kWBlk / 2, &tmW, &sm.full[s], kb * (kBK / 2), wrow + kBM);
                    } else {
                        mbar_arrive_expect_tx(&sm.full[s], S::kW + kXBytes);
                        tma_load_2d(sm.w[s], &tmW, &sm.full[s], kb * kBK, wrow);
                        if (kTwo) tma_load_2d(sm.w[s] + kWBlk, &tmW, &sm.full[s], kb * kBK, wrow + kBM);
                    }
                    tma_load_2d(sm.x[s], &tmX, &sm.full[s], kb * kBK, e * Mmax + tt * kBT);
                    // the token tile's 32 activation scales of this K block, into the scale ring
                    const int j = it % S::kSaSlots;
                    if (!mbar_wait(&sm.sempty[j], ((it / S::kSaSlots) & 1) ^ 1, wait_ns)) { fail(); break; }
                    constexpr uint32_t kWrsBytes = W4 ? static_cast<uint32_t>(sizeof(sm.wrs[0])) : 0u;
                    mbar_arrive_expect_tx(&sm.sfull[j], kBT * sizeof(float) + kWrsBytes);
                    bulk_load(sm.sa[j], As + (static_cast<int64_t>(e) * KB + kb) * Mmax + tt * kBT, kBT * sizeof(float),
                              &sm.sfull[j]);
                    if constexpr (W4)       // row scales [E, K/128, N]: the tile's rows are consecutive
                        bulk_load(sm.wrs[j], Bs + (static_cast<int64_t>(e) * KB + kb) * N + (wrow - e * N), kWrsBytes,
                                  &sm.sfull[j]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = f8_idesc(kBM, kBT);
            uint32_t it = 0, kbt = 0;
            for (int tile = blockIdx.x; tile < total && !sm.abort_flag; tile += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb, ++it, ++kbt) {
                    const int s = it % S::kStages;
                    const uint32_t ph = (it / S::kStages) & 1;
                    const int buf = kbt % S::kBufs;
                    const uint32_t bph = (kbt / S::kBufs) & 1;
                    if (!mbar_wait(&sm.full[s], ph, wait_ns)) { fail(); break; }
                    const int a = it % S::kA;
                    if (W4 && !mbar_wait(&sm.afull[a], (it / S::kA) & 1, wait_ns)) { fail(); break; }
                    if (!mbar_wait(&sm.tempty[buf], bph ^ 1, wait_ns)) { fail(); break; }
                    tc_fence_after();
                    const uint32_t x0 = smem_u32(sm.x[s]);
                    const uint32_t d = tmem + buf * S::kCols;
                    if constexpr (W4) {
                        // A (the expanded weight rows) from tensor memory: 8 columns per 32-wide K slice
                        const uint32_t a0 = tmem + kA0 + a * S::kACols;
#pragma unroll
                        for (int kk = 0; kk < kBK / 32; ++kk) {
                            const uint64_t xd = sw128_kmajor_desc(x0 + kk * 32);
                            umma_f8_ta(d, a0 + kk * 8, xd, idesc, kk > 0);
                            if (kTwo) umma_f8_ta(d + kBT, a0 + 32 + kk * 8, xd, idesc, kk > 0);
                        }
                    } else {
                        const uint32_t w0 = smem_u32(sm.w[s]);
#pragma unroll
                        for (int kk = 0; kk < kBK / 32; ++kk) {
                            const uint64_t xd = sw128_kmajor_desc(x0 + kk * 32);
                            umma_f8(d, sw128_kmajor_desc(w0 + kk * 32), xd, idesc, kk > 0);
                            if (kTwo) umma_f8(d + kBT, sw128_kmajor_desc(w0 + kWBlk + kk * 32), xd, idesc, kk > 0);
                        }
                    }
                    umma_commit(&sm.tfull[buf]);     // the one commit of the K block
                }
            }
        }
    } else if (W4 && warp >= kConvWarp0) {
        // Expansion: thread = tensor-memory lane = weight row r of the tile (warp % 4 is the lane quadrant
        // it may write). The row's packed levels of a K block (64 bytes per 128-row block, 64-byte
        // swizzled by TMA: 16-byte piece c of row r at c ^ ((r >> 1) & 3), conflict-free across eight
        // rows) go to registers, which frees the stage's levels; the 128 codes go to the row's 32 columns
        // of an A slot (64 for the gate and up blocks), whose completion the MMA waits on.
        const int q = warp & 3;
        const int set = (warp - kConvWarp0) >> 2;          // this warp expands the K blocks it % kConvSets == set
        const int r = q * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb, ++it) {
                if (kConvSets > 1 && static_cast<int>(it % (kConvSets > 1 ? kConvSets : 1)) != set) continue;
                if (sm.abort_flag) { ok = false; break; }
                const int s = it % S::kStages;
                const uint32_t ph = (it / S::kStages) & 1;
                const int a = it % S::kA;
                if (!mbar_wait(&sm.full[s], ph, wait_ns)) { fail(); ok = false; break; }
                uint4 pk[kTwo ? 2 : 1][4];
#pragma unroll
                for (int b = 0; b < (kTwo ? 2 : 1); ++b)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        pk[b][c] = *reinterpret_cast<const uint4*>(sm.wp[s] + b * (kWBlk / 2) + r * (kBK / 2) +
                                                                   ((c ^ ((r >> 1) & 3)) << 4));
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);
                // slot a was last read by the MMA of K block it - kA, whose accumulator buffer is a
                if (!mbar_wait(&sm.tfull[a], ((it / S::kA) & 1) ^ 1, wait_ns)) { fail(); ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int b = 0; b < (kTwo ? 2 : 1); ++b) {
                    uint32_t codes[32];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t wv[4] = {pk[b][c].x, pk[b][c].y, pk[b][c].z, pk[b][c].w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) w4x8_to_e4m3x8(wv[j], codes[8 * c + 2 * j], codes[8 * c + 2 * j + 1]);
                    }
                    tmem_st32(tmem + lane_base + kA0 + a * S::kACols + b * 32, codes);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.afull[a]);
            }
        }
    } else {
        // promotion + epilogue: thread = tensor-memory lane = weight row; for the bf16 output two warps
        // per lane quadrant take token columns [16 * hh, 16 * hh + 16)
        const int q = warp & 3;
        const int pw = warp - 2;                 // 0..3 (SwiGLU) or 0..7
        const int r = q * 32 + lane;
        constexpr int kC = EPI == 1 ? kBT : kBT / 2;     // token columns per thread
        const int cof = EPI == 1 ? 0 : (pw >> 2) * kC;  // its first token column
        uint32_t kbt = 0, ep = 0;
        // lane l holds the weight-block scales of K blocks l, l + 32, l + 64, l + 96 of the tile's
        // weight block(s) (K <= 16384), loaded one tile ahead so their latency hides behind a tile
        float wa[4], wb[4];
        auto load_w = [&](int tile) {
            if (tile >= total) return;
            int e, nb, tt, m_e;
            decode(tile, e, nb, tt, m_e);
            const float* pa = Bs + (static_cast<int64_t>(e) * NB + (kTwo ? 2 * nb : nb)) * KB;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kb = lane + 32 * i;
                wa[i] = kb < KB ? pa[kb] : 0.0f;
                wb[i] = kTwo && kb < KB ? pa[KB + kb] : 0.0f;
            }
        };
        if constexpr (!W4) load_w(blockIdx.x);
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            if (sm.abort_flag) break;
            int e, nb, tt, m_e;
            decode(tile, e, nb, tt, m_e);
            // EPI 1: 32 gate then 32 up token columns; EPI 0: kC token columns of each weight block
            constexpr int kAcc = EPI == 1 ? 2 * kBT : (WIDE ? 2 * kC : kC);
            float acc[kAcc];
#pragma unroll
            for (int i = 0; i < kAcc; ++i) acc[i] = 0.0f;
            const float wta[4] = {wa[0], wa[1], wa[2], wa[3]};
            const float wtb[4] = {wb[0], wb[1], wb[2], wb[3]};
            if constexpr (!W4) load_w(tile + gridDim.x);
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb, ++kbt) {
                const int buf = kbt % S::kBufs;
                const uint32_t bph = (kbt / S::kBufs) & 1;
                // scales: the token tile's 32 from the ring, the weight block's from the lane holding it
                const int j = kbt % S::kSaSlots;
                if (!mbar_wait(&sm.sfull[j], (kbt / S::kSaSlots) & 1, wait_ns)) { fail(); ok = false; break; }
                float sa[kC];
#pragma unroll
                for (int i = 0; i < kC / 4; ++i) {
                    const float4 v4 = *reinterpret_cast<const float4*>(&sm.sa[j][cof + 4 * i]);
                    sa[4 * i] = v4.x; sa[4 * i + 1] = v4.y; sa[4 * i + 2] = v4.z; sa[4 * i + 3] = v4.w;
                }
                float swa, swb;
                if constexpr (W4) {            // this thread's weight row (and its up row) scale for the K block
                    swa = sm.wrs[j][r];
                    swb = kTwo ? sm.wrs[j][kBM + r] : 0.0f;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sempty[j]);
                if constexpr (!W4) {
                    const int wi = kb >> 5;
                    swa = __shfl_sync(0xffffffffu, wi == 0 ? wta[0] : wi == 1 ? wta[1] : wi == 2 ? wta[2] : wta[3],
                                      kb & 31);
                    swb = kTwo ? __shfl_sync(0xffffffffu, wi == 0 ? wtb[0] : wi == 1 ? wtb[1]
                                                              : wi == 2 ? wtb[2] : wtb[3], kb & 31)
                                   : 0.0f;
                }
                if (!mbar_wait(&sm.tfull[buf], bph, wait_ns)) { fail(); ok = false; break; }
                if (lane == 0) mbar_arrive(&sm.empty[kbt % S::kStages]);     // the MMA has read the stage
                tc_fence_after();
                const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * S::kCols;
                if constexpr (EPI == 0) {
                    float v[16], v2[16];
                    tmem_ld16(taddr + cof, v);
                    if constexpr (WIDE) tmem_ld16(taddr + kBT + cof, v2);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < kC; ++c) acc[c] = fmaf(v[c], sa[c] * swa, acc[c]);
                    if constexpr (WIDE) {
#pragma unroll
                        for (int c = 0; c < kC; ++c) acc[kC + c] = fmaf(v2[c], sa[c] * swb, acc[kC + c]);
                    }
                } else {
                    float v[32];
                    tmem_ld32(taddr, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < kBT; ++c) acc[c] = fmaf(v[c], sa[c] * swa, acc[c]);
                }
                if (EPI == 1) {
                    float v[32];
                    tmem_ld32(taddr + kBT, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < kBT; ++c) acc[kBT + c] = fmaf(v[c], sa[c] * swb, acc[kBT + c]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.tempty[buf]);
            }
            if (!ok) break;
            const int nv = min(kBT, m_e - tt * kBT);       // valid tokens in this tile
            const int64_t row0 = static_cast<int64_t>(e) * Mmax + tt * kBT;
            if constexpr (EPI == 0) {
                uint16_t* out = static_cast<uint16_t*>(D) + (row0 + cof) * N + nb * (WIDE ? 2 * kBM : kBM) + r;
#pragma unroll
                for (int c = 0; c < kC; ++c)
                    if (cof + c < nv) {
                        out[static_cast<int64_t>(c) * N] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[c]));
                        if constexpr (WIDE)
                            out[static_cast<int64_t>(c) * N + kBM] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[kC + c]));
                    }
            } else {
                const int I = N / 2;
                const int p = ep & 1;
#pragma unroll
                for (int c = 0; c < kBT; ++c) sm.hs[p][c][r] = silu_f(acc[c]) * acc[kBT + c];
                mbar_arrive(&sm.red_bar[p]);
                if (!mbar_wait(&sm.red_bar[p], (ep >> 1) & 1, wait_ns)) { fail(); break; }
                ++ep;
                for (int i = 0; i < kBT / 4; ++i) {
                    const int c = pw * (kBT / 4) + i;
                    if (c >= nv) break;
                    const float4 h4 = *reinterpret_cast<const float4*>(&sm.hs[p][c][lane * 4]);
                    const float amax = warp_max(fmaxf(fmaxf(fabsf(h4.x), fabsf(h4.y)), fmaxf(fabsf(h4.z), fabsf(h4.w))));
                    uint32_t packed;
                    float s = 1.0f;
                    if (amax == 0.0f) {
                        packed = f32x2_to_e4m3x2(h4.x, h4.y) | (static_cast<uint32_t>(f32x2_to_e4m3x2(h4.z, h4.w)) << 16);
                    } else {
                        s = __fdiv_rn(amax, 448.0f);
                        packed = f32x2_to_e4m3x2(__fdiv_rn(h4.x, s), __fdiv_rn(h4.y, s)) |
                                 (static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(h4.z, s), __fdiv_rn(h4.w, s))) << 16);
                    }
                    uint8_t* hq = static_cast<uint8_t*>(D) + (row0 + c) * I + nb * kBM + lane * 4;
                    *reinterpret_cast<uint32_t*>(hq) = packed;
                    if (lane == 0) Ds[(static_cast<int64_t>(e) * (I / kBM) + nb) * Mmax + tt * kBT + c] = s;
                }
            }
        }
    }

    __syncthreads();
    if (sm.abort_flag) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < kDrainNs) __nanosleep(1000);
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ====================================================================== host side
// 2-D map over a row-major byte matrix [rows, cols] read in boxes of 128 bytes x box_rows, 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a row-major matrix [rows, cols] of bf16 (elem_bytes 2) or bytes (1) written in boxes of
// 32 rows x 64 bytes, 64-byte swizzle.
static bool make_out_map(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows, int elem_bytes) {
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * elem_bytes};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(64 / elem_bytes), static_cast<cuuint32_t>(kOutBox)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <typename Kern>
static cudaError_t set_smem(Kern k, size_t bytes) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

// A setmaxnreg.inc can only draw on the registers the block was launched with; if the
// compiled kernel's launch allocation were smaller than the split, the increase would
// never be granted. Refuse to launch such a build instead of starting it.
template <typename Kern>
static cudaError_t check_reg_split(Kern k) {
    cudaFuncAttributes a;
    cudaError_t err = cudaFuncGetAttributes(&a, k);
    if (err != cudaSuccess) return err;
    return a.numRegs * kThreadsC >= kRegsSplit ? cudaSuccess : cudaErrorInvalidConfiguration;
}

// Contiguous kernel in one of its two forms: one CTA per tile, or (PAIR) clusters of two CTAs sharing
// 256 x 256 tiles, as many clusters as fit on the device at once (queried once per device).
template <int EPI, bool PAIR, bool KG = false>
static cudaError_t launch_contig(const CUtensorMap& mapA, const CUtensorMap& mapB, const CUtensorMap& mapD,
                                 const float* As, const int32_t* offsets, int M_rows, const float* Bs, int E, int N,
                                 int K, void* D, float* Ds, int* status, uint64_t wait_ns, int num_sms,
                                 cudaStream_t s, int kg_rows = 0, uint16_t* save_ab = nullptr) {
    auto kern = gg_contig_kernel<EPI, PAIR, KG>;
    const size_t smem = sizeof(SmemC<EPI, PAIR>) + 1024;
    cudaError_t err = set_smem(kern, smem);
    if (err == cudaSuccess) err = check_reg_split(kern);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(kThreadsC);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    if constexpr (PAIR) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        static int clusters[64] = {0};
        int dev = 0;
        if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
        if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        if (clusters[dev] == 0) {
            cfg.gridDim = dim3(2 * (num_sms / 2));
            int n = 0;
            if ((err = cudaOccupancyMaxActiveClusters(&n, kern, &cfg)) != cudaSuccess) return err;
            if (n <= 0) return cudaErrorInvalidConfiguration;
            clusters[dev] = n;
        }
        cfg.gridDim = dim3(2 * clusters[dev]);
    } else {
        cfg.gridDim = dim3(num_sms);
        cfg.attrs = nullptr;
        cfg.numAttrs = 0;
    }
    return cudaLaunchKernelEx(&cfg, kern, mapA, mapB, mapD, As, offsets, M_rows, Bs, E, N, K, D, Ds, status, wait_ns,
                              kg_rows, save_ab);
}

// K-grouped grouped GEMM (the backward pass's weight gradients): D [E * M, N] bf16, expert e's rows
// e * M .. : sum over the expert's 128-row tiles m of the forward contiguous layout (offsets [E + 1],
// rows_fwd rows) of A_m [M, 128] x B_m [N, 128]^T, with A = [tiles * M, 128] codes, As = [tiles][M]
// (one scale per row per tile), B = [tiles * N, 128] codes, Bs = [tiles][N / 128].
cudaError_t launch_grouped_gemm_kgroup(int E, int M, int N, const uint8_t* A, const float* As, const int32_t* offsets,
                                       int rows_fwd, const uint8_t* B, const float* Bs, void* D, int* status,
                                       uint64_t wait_ns, int num_sms, cudaStream_t s) {
    const uint64_t tiles = static_cast<uint64_t>(rows_fwd) / kBM;
    CUtensorMap mapA, mapB, mapD;
    if (!make_map(&mapA, A, kBK, tiles * M, kBM)) return cudaErrorInvalidValue;
    if (!make_map(&mapB, B, kBK, tiles * N, 128)) return cudaErrorInvalidValue;
    if (!make_out_map(&mapD, D, N, static_cast<uint64_t>(E) * M, 2)) return cudaErrorInvalidValue;
    return launch_contig<0, false, true>(mapA, mapB, mapD, As, offsets, M, Bs, E, N, kBK, D, nullptr, status, wait_ns,
                                         num_sms, s, rows_fwd);
}

// Which form of the contiguous kernel runs (moe_set_contig_kernel): 0 chooses by shape, 1 forces single
// CTAs, 2 forces CTA pairs (where N allows them).
static int g_contig_mode = 0;

void set_contig_mode(int mode) { __atomic_store_n(&g_contig_mode, mode, __ATOMIC_RELAXED); }

// CTA pairs need whole 256-column tiles; they run only when asked for (the default is single CTAs, the
// faster form as measured on the prefill and skewed workloads).
static bool use_pairs(int E, int N, int M_rows) {
    (void)E;
    (void)M_rows;
    if (N % kBN) return false;
    return __atomic_load_n(&g_contig_mode, __ATOMIC_RELAXED) == 2;
}

// save_ab (contiguous layout, SwiGLU epilogue only; nullable): also write the gate and up values, bf16
// [M_rows, N], for the backward pass.
cudaError_t launch_grouped_gemm(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                                const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs, int epilogue,
                                void* D, float* Ds, int* status, uint64_t wait_ns, int num_sms, cudaStream_t s,
                                uint16_t* save_ab) {
    CUtensorMap mapA, mapB, mapD;
    if (layout == 0) {
        if (!make_map(&mapA, A, K, static_cast<uint64_t>(M_rows), kBM)) return cudaErrorInvalidValue;
        if (!make_map(&mapB, B, K, static_cast<uint64_t>(E) * N, 128)) return cudaErrorInvalidValue;
        const bool pair = use_pairs(E, N, M_rows);
        if (epilogue == 0) {
            if (!make_out_map(&mapD, D, N, static_cast<uint64_t>(M_rows), 2)) return cudaErrorInvalidValue;
            return pair ? launch_contig<0, true>(mapA, mapB, mapD, As, group_info, M_rows, Bs, E, N, K, D, Ds, status,
                                                 wait_ns, num_sms, s)
                        : launch_contig<0, false>(mapA, mapB, mapD, As, group_info, M_rows, Bs, E, N, K, D, Ds, status,
                                                  wait_ns, num_sms, s);
        }
        if (!make_out_map(&mapD, D, N / 2, static_cast<uint64_t>(M_rows), 1)) return cudaErrorInvalidValue;
        return pair ? launch_contig<1, true>(mapA, mapB, mapD, As, group_info, M_rows, Bs, E, N, K, D, Ds, status,
                                             wait_ns, num_sms, s, 0, save_ab)
                    : launch_contig<1, false>(mapA, mapB, mapD, As, group_info, M_rows, Bs, E, N, K, D, Ds, status,
                                              wait_ns, num_sms, s, 0, save_ab);
    } else {
        if (save_ab) return cudaErrorInvalidValue;
        if (!make_map(&mapA, A, K, static_cast<uint64_t>(E) * M_rows, kBT)) return cudaErrorInvalidValue;
        if (!make_map(&mapB, B, K, static_cast<uint64_t>(E) * N, 128)) return cudaErrorInvalidValue;
        if (epilogue == 0 && N % (2 * kBM) == 0) {
            const size_t smem = sizeof(SmemM<0, false, true>) + 1024;
            cudaError_t err = set_smem(gg_masked_kernel<0, false, true>, smem);
            if (err != cudaSuccess) return err;
            gg_masked_kernel<0, false, true><<<num_sms, masked_threads<0>(), smem, s>>>(
                mapA, mapB, As, group_info, M_rows, Bs, E, N, K, D, Ds, status, wait_ns);
        } else if (epilogue == 0) {
            const size_t smem = sizeof(SmemM<0>) + 1024;
            cudaError_t err = set_smem(gg_masked_kernel<0, false>, smem);
            if (err != cudaSuccess) return err;
            gg_masked_kernel<0, false><<<num_sms, masked_threads<0>(), smem, s>>>(mapA, mapB, As, group_info, M_rows, Bs, E, N, K, D,
                                                                  Ds, status, wait_ns);
        } else {
            const size_t smem = sizeof(SmemM<1>) + 1024;
            cudaError_t err = set_smem(gg_masked_kernel<1, false>, smem);
            if (err != cudaSuccess) return err;
            gg_masked_kernel<1, false><<<num_sms, masked_threads<1>(), smem, s>>>(mapA, mapB, As, group_info, M_rows, Bs, E, N, K, D,
                                                                  Ds, status, wait_ns);
        }
    }
    return cudaGetLastError();
}

// 2-D map over a row-major byte matrix [rows, cols] read in boxes of 64 bytes x box_rows with the 64-byte
// swizzle (4-bit weights: 64 bytes hold a row's 128 levels of one K block; 16-byte piece c of row r lands
// at c ^ ((r >> 1) & 3), so eight consecutive rows read at the same piece hit distinct banks).
static bool make_packed_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK / 2), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Masked layout with 4-bit weights: B = [E, N, K/2] packed levels, Bs = [E, K/128, N] row scales.
cudaError_t launch_grouped_gemm_w4(int E, int N, int K, const uint8_t* A, const float* As, const int32_t* masked_m,
                                   int M_rows, const uint8_t* B, const float* Bs, int epilogue, void* D, float* Ds,
                                   int* status, uint64_t wait_ns, int num_sms, cudaStream_t s) {
    CUtensorMap mapA, mapB;
    if (!make_map(&mapA, A, K, static_cast<uint64_t>(E) * M_rows, kBT)) return cudaErrorInvalidValue;
    if (!make_packed_map(&mapB, B, K / 2, static_cast<uint64_t>(E) * N, 128)) return cudaErrorInvalidValue;
    if (epilogue == 0 && N % (2 * kBM) == 0) {
        const size_t smem = sizeof(SmemM<0, true, true>) + 1024;
        cudaError_t err = set_smem(gg_masked_kernel<0, true, true>, smem);
        if (err != cudaSuccess) return err;
        gg_masked_kernel<0, true, true><<<num_sms, masked_threads<0, true>(), smem, s>>>(
            mapA, mapB, As, masked_m, M_rows, Bs, E, N, K, D, Ds, status, wait_ns);
    } else if (epilogue == 0) {
        const size_t smem = sizeof(SmemM<0, true>) + 1024;
        cudaError_t err = set_smem(gg_masked_kernel<0, true>, smem);
        if (err != cudaSuccess) return err;
        gg_masked_kernel<0, true><<<num_sms, masked_threads<0, true>(), smem, s>>>(mapA, mapB, As, masked_m, M_rows, Bs,
                                                                                 E, N, K, D, Ds, status, wait_ns);
    } else {
        const size_t smem = sizeof(SmemM<1, true>) + 1024;
        cudaError_t err = set_smem(gg_masked_kernel<1, true>, smem);
        if (err != cudaSuccess) return err;
        gg_masked_kernel<1, true><<<num_sms, masked_threads<1, true>(), smem, s>>>(mapA, mapB, As, masked_m, M_rows, Bs,
                                                                                 E, N, K, D, Ds, status, wait_ns);
    }
    return cudaGetLastError();
}

// One block waits on a barrier nothing completes; the bounded wait must give up and record a timeout.
__global__ void selftest_wait_kernel(int* status, uint64_t wait_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (!mbar_wait(&bar, 0, wait_ns)) set_status(status, kStatusTimeout);
    }
}

cudaError_t launch_selftest_wait(int* status, uint64_t wait_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(status, wait_ns);
    return cudaGetLastError();
}

}  // namespace moe
