/*
 * moe_fp8.h -- C ABI of a single-GPU FP8 Mixture-of-Experts expert layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (MegaMoE/DeepGEMM page, "2.1 From standard MoE to MegaMoE"):
 *     y = sum_{i in TopK} G(x)_i * E_i(x),   E_i(x) = W2_i (silu(W1_i x) * W3_i x)
 * computed as five steps, each an entry point below:
 *   moe_route            router scores s = softmax(W_g x + b) in fp32, top-k
 *                        (or hash routing), renormalised weights
 *   moe_permute          per-expert counts, optional capacity drop, expert-
 *                        contiguous (or masked per-expert) rows, and the 1x128
 *                        FP8 quantisation of x written into those rows
 *   moe_grouped_gemm_fp8 FP8 grouped GEMM: every group has its own M, all groups
 *                        share N and K; fine-grained fp32 block scales applied
 *                        in fp32 promotion; epilogue bf16 or SwiGLU + FP8 requant
 *   moe_combine          weighted un-permute y = sum_j w_j * o_j
 *   moe_forward          all of the above on one stream, no host sync
 * and, for training, moe_balance_bias: the auxiliary-loss-free update of the
 * routing bias b from the per-expert counts moe_permute reports; and
 * moe_grouped_gemm_w4: the grouped GEMM with 4-bit expert weights (masked
 * layout).
 *
 * Conventions (every entry point):
 *  - Every array argument is a DEVICE pointer owned by the caller, except the
 *    moe_config_t, which is read on the host during the call. The library
 *    allocates no memory; scratch comes from the caller's `ws` buffer.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream) and never synchronise the host.
 *  - Argument and shape errors are returned before anything is launched;
 *    launch failures return MOE_ERR_CUDA. Device-side conditions (a masked
 *    group overflowing its rows, a bounded wait that ran out) set a status
 *    word that moe_get_device_status() reports.
 *  - Device pointers must be 16-byte aligned. H and I must be multiples of 128,
 *    H at most 16384; the masked layout needs masked_max_m a multiple of 32.
 *  - bf16 arrays are raw 16-bit words (torch.bfloat16 layout); FP8 arrays are
 *    E4M3FN codes (torch.float8_e4m3fn layout), one byte each.
 *  - The group padding (tile M) is fixed at 128 rows.
 */
#ifndef MOE_FP8_H
#define MOE_FP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,        /* null/misaligned pointer, bad enum, k > E, ... */
    MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* H or I not a multiple of 128, E or k above the limits */
    MOE_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not sm_100 ("FP8 not supported on this GPU",
                                       MegaMoE page, section 5.1, problem three) */
    MOE_ERR_WORKSPACE_TOO_SMALL = 4,
    MOE_ERR_CAPACITY = 5,           /* device status: a group had more rows than its bound (masked_max_m, M_rows) */
    MOE_ERR_CUDA = 6,               /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = 7      /* device status: a bounded wait inside a kernel ran out */
} moe_status_t;

typedef enum { MOE_ROUTE_SOFTMAX_TOPK = 0, MOE_ROUTE_HASH = 1 } moe_routing_t;
typedef enum { MOE_LAYOUT_CONTIGUOUS = 0, MOE_LAYOUT_MASKED = 1 } moe_layout_t;
typedef enum { MOE_EPI_BF16 = 0, MOE_EPI_SWIGLU_FP8 = 1 } moe_epilogue_t;
typedef enum { MOE_CONTIG_AUTO = 0, MOE_CONTIG_SINGLE = 1, MOE_CONTIG_PAIR = 2 } moe_contig_kernel_t;
/* Expert weights: E4M3 with one fp32 scale per 128x128 block, or 4-bit levels with one fp32 scale per
 * weight row per 128-wide K block (moe_grouped_gemm_w4; masked layout only). */
typedef enum { MOE_WEIGHTS_FP8 = 0, MOE_WEIGHTS_W4 = 1 } moe_weights_t;

/* Limits checked by every entry point. */
#define MOE_MAX_EXPERTS 512
#define MOE_MAX_TOPK 32
#define MOE_TILE_M 128

typedef struct {
    int T;              /* tokens (0 allowed: nothing is launched and the per-token buffers may be
                           empty; moe_ep_count still zeroes its counts) */
    int H;              /* hidden size, multiple of 128 */
    int E;              /* experts, 1..MOE_MAX_EXPERTS */
    int I;              /* expert intermediate size, multiple of 128, at most 16384 */
    int k;              /* experts per token (1..min(E, MOE_MAX_TOPK)); hash routing needs k = 1 */
    int routing;        /* moe_routing_t */
    int cap_num;        /* capacity factor alpha = cap_num / cap_den; 0 / 0 = dropless */
    int cap_den;
    int layout;         /* moe_layout_t */
    int masked_max_m;   /* rows per expert in the masked layout (ignored when contiguous) */
    int weights;        /* moe_weights_t: the expert weights' format (moe_forward) */
} moe_config_t;

/* Rows of the permuted buffers (Aq, As, Hq, Hs, O, row_src) for `cfg`:
 * contiguous: roundup(T*k + E*127, 128) (every kept slot plus at most 127
 * padding rows per expert); masked: E * masked_max_m. 0 on a bad config. */
size_t moe_rows_capacity(const moe_config_t* cfg);

/* Scratch bytes moe_route and moe_permute need (ws_bytes >= this); with
 * for_forward = 1 the bytes moe_forward needs, with for_forward = 2 those of
 * moe_forward_train (the same plus the saved gate and up values, 4 I bytes per
 * row). 0 on a bad config, on for_forward outside 0..2, and with for_forward = 2
 * on a configuration moe_forward_train does not take (masked layout, 4-bit
 * weights or hash routing). */
size_t moe_workspace_size(const moe_config_t* cfg, int for_forward);

/*
 * Router. Source: s_i = softmax(W_g x + b_i) (MegaMoE page, section 2.2),
 * softmax in fp32 even for bf16 activations (DeepSeek-V4 lecture page,
 * section 2.3), top-k of the scores renormalised over the k selected experts
 * (DeepSeek MoE architecture page, chapter 1 pseudo-code; TP-MoE page,
 * section 3.1 names renormalisation as one of its two options).
 *   x         [T, H] bf16, row-major
 *   Wg        [E, H] fp32, row-major (softmax routing)
 *   bias      [E] fp32, nullable (no bias)
 *   token_ids [T] int32 (hash routing only; else ignored, nullable)
 *   topk_idx  [T, k] int32 out: experts in descending score, ties to the lower index
 *   topk_w    [T, k] fp32 out: w_j = exp(l_j - m) / sum_{top-k} exp(l_i - m)
 *   ws        scratch of at least moe_workspace_size(cfg, 0) bytes (holds the T x E logits)
 * Logits are fp32 with one fixed summation order: 32 fused multiply-add
 * chains, chain j over h = 128 s + 4 j + i (i = 0..3, every 128-wide block s
 * in order), halved pairwise (j with j+16, then j+8, 4, 2, 1), then + b. Hash routing (DeepSeek-V4 lecture page,
 * section 2.2, hash(token_id) % num_experts): expert =
 * (uint32)(token_id * 2654435761) % E, k = 1, weight 1.
 */
moe_status_t moe_route(const moe_config_t* cfg, const void* x, const float* Wg, const float* bias,
                       const int32_t* token_ids, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * Permutation and activation quantisation. Sources: Concat(E_1(T_1), ...,
 * E_E(T_E)) as one grouped GEMM (MegaMoE page, section 2.1); a global tile
 * scheduler over the flattened M of all groups (section 3.2); capacity
 * ceil(top-k * N / E) * alpha with overflow dropped silently in token order
 * (DeepSeek MoE page, section 2.5); x_fp8 = clamp(round(x / scale), -448, 448)
 * (MegaMoE page, section 3.3) with one scale per 1x128 group.
 *   x          [T, H] bf16
 *   topk_idx   [T, k] int32 (from moe_route)
 *   Aq         [rows, H] u8 out (rows = moe_rows_capacity); masked: [E, masked_max_m, H]
 *   As         [H/128][rows] fp32 out, K-block-major; masked: [E][H/128][masked_max_m]
 *   counts     [E] int32 out: slots routed to each expert
 *   kept       [E] int32 out: min(counts, capacity, masked_max_m)
 *   offsets    [E+1] int32 out: first row of each group; contiguous groups are
 *              padded to 128 rows, masked offsets[e] = e * masked_max_m
 *   row_src    [rows] int32 out: slot t*k+j that a row holds, -1 for padding
 *              (written for rows < offsets[E] in the contiguous layout and for
 *              the first kept[e] rows of each masked group)
 *   slot_row   [T*k] int32 out: row of slot t*k+j, or -1 if dropped
 * Within a group, rows follow token index. Padding rows get code 0 and
 * scale 1.0. Scale = max|x| / 448 in fp32 (1.0 for an all-zero group);
 * code = E4M3 round-to-nearest-even, saturating, of the fp32 quotient x / scale.
 * A masked group with more kept slots than masked_max_m keeps the first
 * masked_max_m and sets the device status MOE_ERR_CAPACITY.
 */
moe_status_t moe_permute(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                         uint8_t* Aq, float* As, int32_t* counts, int32_t* kept, int32_t* offsets,
                         int32_t* row_src, int32_t* slot_row, void* ws, size_t ws_bytes, void* stream);

/*
 * FP8 grouped GEMM, D_g = A_g * B_g^T per group g. Sources: every group has
 * its own M, all share N and K (MegaMoE page, sections 2.1 and 3.2); the
 * "nt" FP8 x FP8 -> bf16 grouped call with per-group sizes (section 3.2);
 * fp32 accumulation converted to bf16 with round-to-nearest-even only at the
 * end (section 3.3); FP8 partial sums promoted to fp32 on the CUDA cores with
 * fine-grained scales (DeepSeek open-source week page, "Day 3"); bias,
 * activation and quantisation fused into the epilogue (MegaMoE page, 3.2).
 *   layout      MOE_LAYOUT_CONTIGUOUS: group_info = offsets [E+1] (multiples of
 *               128, offsets[E] <= M_rows), rows [offsets[e], offsets[e+1]) use
 *               expert e; A is [M_rows, K]. MOE_LAYOUT_MASKED: group_info =
 *               masked_m [E], A is [E, M_rows, K] and rows [0, masked_m[e])
 *               of block e use expert e.
 *   A           u8 E4M3 codes, K-major
 *   As          fp32 1x128 scales, [K/128][M_rows] (masked: [E][K/128][M_rows])
 *   B           [E, N, K] u8 E4M3 codes, K-major ("nt")
 *   Bs          [E, N/128, K/128] fp32, one scale per 128x128 block
 *   epilogue    MOE_EPI_BF16: D = bf16 [rows, N] (RNE); Ds unused.
 *               MOE_EPI_SWIGLU_FP8: N = 2I and B's 128-row blocks alternate
 *               W1 block j, W3 block j; h = silu(a) * b in fp32 is quantised
 *               per 1x128 group: D = u8 [rows, I], Ds = fp32 [I/128][M_rows]
 *               (masked: [E][I/128][M_rows]), the A/As layout of the next GEMM.
 * N and K must be multiples of 128 (256 for N with the SwiGLU epilogue) and
 * K at most 16384 (MOE_ERR_UNSUPPORTED_SHAPE otherwise). Contiguous layout:
 * M_rows must be a multiple of 4, so that each K block's row of As starts on
 * a 16-byte boundary (MOE_ERR_INVALID_ARG otherwise).
 * Contiguous rows outside [0, offsets[E]) and masked rows at or past
 * masked_m[e] are neither read into any stored result nor written.
 * Group bounds are checked on the device: offsets must start at 0, be
 * non-decreasing multiples of 128 and stay within M_rows, and each masked_m[e]
 * must lie in [0, M_rows]. Values outside these bounds are clamped into them
 * (offsets by a running maximum of the clamped values), so that no read or
 * write leaves the caller's buffers, and the device status MOE_ERR_CAPACITY is
 * set (moe_get_device_status); the results of the offending groups are then
 * unspecified.
 */
moe_status_t moe_grouped_gemm_fp8(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                                  const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                                  int epilogue, void* D, float* Ds, void* stream);

/*
 * The same grouped GEMM with 4-bit expert weights, masked layout. Source:
 * DeepSeek-V4 lecture page, section 3.1: expert weights cut into per-channel
 * blocks, each scaled by its max-abs, stored as the integer levels
 * round((w / max|w|) * (2^3 - 1)) in 4 bits.
 *   layout      MOE_LAYOUT_MASKED only (MOE_ERR_UNSUPPORTED_SHAPE otherwise);
 *               A, As, group_info (masked_m), M_rows, epilogue, D and Ds as in
 *               moe_grouped_gemm_fp8
 *   B           [E, N, K/2] u8: levels -7..7 as a sign and a 3-bit magnitude,
 *               eight consecutive k per little-endian 32-bit word; level i
 *               (i = 0..3) of a word has its magnitude in bits 4i..4i+2 and
 *               its sign in bit 8i+7, level 4+i its magnitude in bits
 *               16+4i..16+4i+2 and its sign in bit 8i+3
 *   Bs          [E, K/128, N] fp32 (K-block-major): the scale of weight row n
 *               for K block kb, max-abs / 7 of its 128 weights; a weight is
 *               level * scale
 * N, K and M_rows follow moe_grouped_gemm_fp8's masked-layout rules. The
 * levels are expanded to E4M3 codes on the chip (all of -7..7 are exact), so
 * the arithmetic is the FP8 GEMM's with per-row weight scales.
 */
moe_status_t moe_grouped_gemm_w4(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                                 const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                                 int epilogue, void* D, float* Ds, void* stream);

/*
 * Combine. Source: y = sum_{i in TopK} G(x)_i * E_i(x) (MegaMoE page,
 * section 2.1); bf16 output rounded to nearest even (section 3.3).
 *   O         [rows, H] bf16 expert outputs (row = slot_row[t*k+j])
 *   slot_row  [T*k] int32; -1 = dropped slot (contributes nothing; the
 *             other weights are not renormalised; all dropped -> y = 0)
 *   topk_w    [T, k] fp32
 *   y         [T, H] bf16 out: fp32 sum over j = 0..k-1 in order, then RNE
 */
moe_status_t moe_combine(const moe_config_t* cfg, const void* O, const int32_t* slot_row,
                         const float* topk_w, void* y, void* stream);

/*
 * The whole layer on one stream: route -> permute -> grouped GEMM with W13
 * (SwiGLU + FP8 requant epilogue) -> grouped GEMM with W2 (bf16) -> combine.
 * cfg->weights = MOE_WEIGHTS_FP8:
 *   W13 [E, 2I, H] u8 with 128-row blocks alternating W1 block j, W3 block j
 *   S13 [E, 2I/128, H/128] fp32 in the same block order
 *   W2  [E, H, I] u8, S2 [E, H/128, I/128] fp32
 * cfg->weights = MOE_WEIGHTS_W4 (masked layout only; MOE_ERR_UNSUPPORTED_SHAPE
 * otherwise), the 4-bit format of moe_grouped_gemm_w4:
 *   W13 [E, 2I, H/2] u8, rows in the same W1/W3 block alternation
 *   S13 [E, H/128, 2I] fp32, W2 [E, H, I/2] u8, S2 [E, I/128, H] fp32
 *   y [T, H] bf16 out; topk_idx, topk_w, counts, slot_row as in the calls above
 *   ws  scratch of at least moe_workspace_size(cfg, 1) bytes, 256-byte aligned
 */
moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const float* Wg, const float* bias,
                         const int32_t* token_ids, const uint8_t* W13, const float* S13,
                         const uint8_t* W2, const float* S2, void* y, int32_t* topk_idx, float* topk_w,
                         int32_t* counts, int32_t* slot_row, void* ws, size_t ws_bytes, void* stream);

/* moe_forward for training: the same step and outputs, and the up GEMM also
 * keeps each row's gate and up values (a | b, bf16, W13's column order) in the
 * workspace, for moe_backward with fwd_train = 1 (which then needs no second
 * x W13^T GEMM). ws: moe_workspace_size(cfg, 2) bytes. Contiguous layout, E4M3
 * weights and softmax routing only (MOE_ERR_UNSUPPORTED_SHAPE otherwise), as
 * for moe_backward. */
moe_status_t moe_forward_train(const moe_config_t* cfg, const void* x, const float* Wg, const float* bias,
                               const int32_t* token_ids, const uint8_t* W13, const float* S13,
                               const uint8_t* W2, const float* S2, void* y, int32_t* topk_idx, float* topk_w,
                               int32_t* counts, int32_t* slot_row, void* ws, size_t ws_bytes, void* stream);

/*
 * Permutation without a workspace, for callers that may not allocate device
 * memory (code running during CUDA graph capture, servers that fix their
 * memory budget up front and forbid cudaMalloc on the request path, plugin
 * hosts whose memory belongs to another allocator). The source pages have no
 * counterpart: it computes exactly what moe_permute computes, with the same
 * kernels and the same arguments minus ws / ws_bytes.
 * Its scratch is a fixed array of MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES in the
 * library's own device memory, which every GPU that loads the library holds
 * until the process exits. The call needs 8 * ceil(T / 32) * E bytes of it
 * (e.g. T = 16384 with E = 512, or T = 32768 with E = 256) and returns
 * MOE_ERR_UNSUPPORTED_SHAPE, launching nothing, when that exceeds the array.
 * The first call on each device looks the array's device address up (a
 * runtime call), so make that first call before any stream capture. Every
 * call shares the one array: calls whose kernels overlap on the GPU (other
 * streams, other host threads) race and corrupt each other's results; order
 * them on one stream. It allocates nothing and calls no allocating routine.
 */
#define MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES (2u * 1024u * 1024u)
moe_status_t moe_permute_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                 uint8_t* Aq, float* As, int32_t* counts, int32_t* kept, int32_t* offsets,
                                 int32_t* row_src, int32_t* slot_row, void* stream);

/*
 * The layer's backward pass. Source: TP-MoE page, section 4.1, step 5 (the
 * gradients run back along the dispatch path and the gate network is updated
 * too). Given dy = dL/dy [T, H] bf16 of one moe_forward call, computes
 *   dx   [T, H] bf16     = sum over kept slots of (g W13)[row] + sum over all
 *                          slots of dl_j W_g[e_j]
 *   dWg  [E, H] fp32, db [E] fp32: sum over the slots of each expert, in token
 *                          order (dropped slots included), of dl x and of dl
 *   dW13 [E, 2I, H] bf16 (rows in W13's W1/W3 128-row block alternation) and
 *   dW2  [E, H, I] bf16: per expert, sums over its kept rows of g^T x and
 *                          dO^T h
 * with dw_j = <dy_t, o_j> (0 for a dropped slot), dl_j = w_j (dw_j -
 * sum_i w_i dw_i), dO = w dy (fp32) on each kept row, dh = dO W2, a | b = x
 * W13^T (saved by moe_forward_train, else recomputed with the same kernel, so
 * the same values), g = (dh b s (1 + a (1 - s)), dh a s), s = sigmoid(a).
 * The forward's quantisation steps pass the gradient straight through; the
 * selection and the capacity drop are held fixed. Every GEMM is FP8 with fp32
 * scales and fp32 promotion: dO, g and x in 1x128 groups along the
 * contraction (the weight gradients group along the expert's rows), h and x
 * in 128x128 blocks as the second weight-gradient operand; dh, a, b, g and
 * the GEMM outputs are bf16.
 *   x, Wg, W13, S13         the forward's inputs
 *   W13T [E, H, 2I], S13T [E, H/128, 2I/128], W2T [E, I, H], S2T [E, I/128,
 *                          H/128]: W13 and W2 transposed with their block
 *                          scales (a layout step done once, like the weights'
 *                          quantisation)
 *   topk_idx, topk_w, slot_row: the forward's outputs
 *   fwd_ws                  the workspace of that moe_forward (fwd_train = 0)
 *                          or moe_forward_train (fwd_train = 1) call,
 *                          unchanged since (it holds the quantised x and h
 *                          rows, the expert outputs and the row maps, and with
 *                          fwd_train = 1 the gate and up values)
 *   ws                      scratch, moe_backward_workspace_size(cfg) bytes,
 *                          256-byte aligned
 * Contiguous layout, E4M3 weights and softmax routing only
 * (MOE_ERR_UNSUPPORTED_SHAPE otherwise), I at most 8192, and at most 16384
 * rows per expert (T, or the capacity when smaller).
 * moe_backward_workspace_size gives 0 on a bad configuration and on one that
 * moe_backward rejects.
 */
size_t moe_backward_workspace_size(const moe_config_t* cfg);
moe_status_t moe_backward(const moe_config_t* cfg, const void* x, const float* Wg, const uint8_t* W13, const float* S13,
                          const uint8_t* W13T, const float* S13T, const uint8_t* W2T, const float* S2T,
                          const int32_t* topk_idx, const float* topk_w, const int32_t* slot_row, const void* fwd_ws,
                          int fwd_train, const void* dy, void* dx, float* dWg, float* db, void* dW13, void* dW2,
                          void* ws, size_t ws_bytes, void* stream);

/*
 * Auxiliary-loss-free load balancing. Source: MegaMoE page, section 2.2: each
 * expert keeps a bias b_e inside the router softmax (moe_route's `bias`); while
 * training, the bias of an expert with high load goes down and of one with low
 * load goes up, by a step of order 1e-3, once every 100 or so steps. One call
 * per training step:
 *   counts  [E] int32: slots routed to each expert this step (moe_permute's
 *           `counts`, before any capacity drop); must be >= 0
 *   load    [E] int64 in/out: the tally since the last update; zero it once
 *           before the first step
 *   bias    [E] fp32 in/out
 *   gamma   the step, finite (a negative step reverses the direction)
 *   update  0: load += counts only. Nonzero (the last step of an interval):
 *           load += counts; then b_e -= gamma where E * load[e] > sum(load),
 *           b_e += gamma where E * load[e] < sum(load), unchanged where equal
 *           (the mean compared exactly in 64-bit integers; one fp32
 *           round-to-nearest-even addition per expert); then load = 0.
 * E in 1..MOE_MAX_EXPERTS (MOE_ERR_UNSUPPORTED_SHAPE above it). One block of
 * one thread per expert; the tally must stay below 2^63 / E.
 */
moe_status_t moe_balance_bias(int E, const int32_t* counts, int64_t* load, float* bias, float gamma, int update,
                              void* stream);

/*
 * Chooses how the contiguous-layout grouped GEMM (moe_grouped_gemm_fp8 and
 * moe_forward) is run, for every later call in this process. The grouped
 * GEMM of the pages (MegaMoE page, 3.2) is one tile scheduler over the
 * flattened M of all groups; on B200 it has two forms:
 *   MOE_CONTIG_SINGLE  one CTA per 128-row x 256-column tile
 *   MOE_CONTIG_PAIR    clusters of two CTAs, each pair computing a 256-row x
 *                      256-column tile with paired tensor-core MMAs (each CTA
 *                      loads its 128 rows and half of the weight tile, which
 *                      halves the shared-memory traffic per MMA); an expert
 *                      with an odd number of 128-row tiles computes its last
 *                      one on one CTA of a pair while the other idles. Needs N
 *                      a multiple of 256 (otherwise the single form runs).
 *   MOE_CONTIG_AUTO    (the default) the faster form as measured on this
 *                      build's workloads: single CTAs.
 * Both forms compute the same products and the same fp32 promotion, in the
 * same order. Returns MOE_ERR_INVALID_ARG for any other value.
 */
moe_status_t moe_set_contig_kernel(int form);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: MOE_OK, MOE_ERR_CAPACITY or MOE_ERR_DEVICE_TIMEOUT. */
moe_status_t moe_get_device_status(void* stream);

/* Test hook for the bounded-wait machinery every kernel uses: launches one
 * block that waits, for at most `limit_us` microseconds, on a shared-memory
 * barrier that nothing completes; the wait gives up, records
 * MOE_ERR_DEVICE_TIMEOUT in the device status word and the kernel returns. */
moe_status_t moe_selftest_wait_timeout(int limit_us, void* stream);

/*
 * ---------------------------------------------------------------- expert parallelism
 * The layer across G GPUs, one process per GPU, experts split evenly: rank r
 * holds experts [r E/G, (r+1) E/G) and its own batch of tokens. Sources:
 * TP-MoE page, section 3.3 (experts placed on several cards; tokens travel to
 * their expert's card by all-to-all and back) and 4.1 step 3 (each card routes
 * its own tokens, then sends them by all-to-all); MegaMoE page, section 3.4
 * (dispatch and combine as the two communication primitives); TP-MoE page,
 * section 6.2 (the all-to-all payload compressed to FP8) and 5.3 (a send and
 * a receive buffer of the payload). The layer's result on
 * every rank equals that of one GPU on the ranks' batches concatenated in rank
 * order: routing is per token, ranks within an expert (and so the capacity
 * drop) follow that global token order, and capacity uses the global T.
 *
 * One step of rank r:
 *   moe_route                   its own tokens (all E experts)
 *   moe_ep_count                counts[E] of its slots per expert
 *   (collective)                all-gather of counts -> [G][E] on every rank
 *   moe_ep_plan (host)          the exchange plan below, from the gathered
 *                               counts; the same counts give every rank a
 *                               consistent plan
 *   moe_ep_dispatch             quantises x (1x128, as moe_permute) once per
 *                               token and writes one send row per kept slot,
 *                               ordered by destination rank, then expert, then
 *                               token; slot_row maps slot t*k+j to its send row
 *                               (-1 if the capacity drops it)
 *   (collective)                all-to-all of the send rows (send_rows[d] to d)
 *   moe_ep_receive              places the received rows into the contiguous
 *                               grouped layout of its E/G experts (padding rows
 *                               filled) and remembers each row's place
 *   moe_grouped_gemm_fp8 x 2    the local experts, contiguous layout
 *   moe_ep_return               gathers each received row's expert output into
 *                               receive order
 *   (collective)                all-to-all back (recv_rows[s] to s)
 *   moe_combine                 y from the returned rows (slot_row into them)
 *
 * A send/receive row is H bytes of E4M3 codes followed by H/128 fp32 scales,
 * padded to a multiple of 16 bytes (row stride MOE_EP_ROW_BYTES(H)).
 *
 * Chunked overlap (MegaMoE page, section 2.3: with the work cut into C chunks
 * of compute time T_comp and exchange time T_comm each, the exchange of one
 * chunk runs while another is computed, and a step takes T_comp + T_comm +
 * (C - 1) max(T_comp, T_comm) instead of C (T_comp + T_comm)): a
 * plan made with C chunks (moe_ep_plan_chunked) splits every rank's local
 * experts into C consecutive groups and orders the send and receive rows by
 * chunk first, so that chunk c is one contiguous slice of each buffer, with its
 * own per-rank row counts. The caller then runs, per chunk, the all-to-all of
 * its slice, moe_ep_receive_chunk, the two grouped GEMMs on the chunk's experts
 * (pointer offsets into the grouped layout, offsets from moe_ep_receive_chunk)
 * and moe_ep_return on its rows, with the collectives on a stream of their own;
 * results equal those of C = 1 bit for bit.
 */
#define MOE_EP_MAX_RANKS 64
#define MOE_EP_MAX_CHUNKS 8
#define MOE_EP_ROW_BYTES(H) (((size_t)(H) + 4u * ((size_t)(H) / 128u) + 15u) / 16u * 16u)

/* The exchange plan of one rank (host memory; the device steps read a device
 * copy of it, which the caller makes with one copy of sizeof(moe_ep_plan_t)). */
typedef struct {
    int32_t G, rank, E, E_local;   /* E_local = E / G experts on each rank */
    int32_t cap;                   /* per-expert capacity from the global T, -1 if none */
    int32_t rows_send;             /* rows this rank sends: sum of send_rows */
    int32_t rows_recv;             /* rows it receives: sum of recv_rows */
    int32_t rows_group;            /* rows of its grouped layout: offsets[E_local] */
    int32_t kept_mine[MOE_MAX_EXPERTS];      /* per expert e: this rank's slots of e kept */
    int32_t send_rows[MOE_EP_MAX_RANKS];     /* rows for each destination rank */
    int32_t recv_rows[MOE_EP_MAX_RANKS];     /* rows from each source rank */
    /* blocks (source s, local expert l) in receive order, which is (chunk, s, l, token): with one chunk
     * block b = s * E_local + l */
    int32_t recv_start[MOE_MAX_EXPERTS + 1]; /* block b: first receive row; [G * E_local] = rows_recv */
    int32_t group_start[MOE_MAX_EXPERTS];    /* block b: its first row in the grouped layout */
    int32_t offsets[MOE_MAX_EXPERTS + 1];    /* grouped layout of the local experts, multiples of 128 */
    int32_t kept[MOE_MAX_EXPERTS];           /* rows of each local expert (all sources) */
    int32_t chunks;                                     /* C, 1 .. MOE_EP_MAX_CHUNKS */
    int32_t chunk_first[MOE_EP_MAX_CHUNKS + 1];         /* chunk c = local experts [chunk_first[c], [c+1]) */
    int32_t send_off[MOE_MAX_EXPERTS];                  /* per expert e: its first send row */
    int32_t send_chunk[MOE_EP_MAX_CHUNKS + 1];          /* first send row of each chunk */
    int32_t recv_chunk[MOE_EP_MAX_CHUNKS + 1];          /* first receive row of each chunk */
    int32_t send_rows_c[MOE_EP_MAX_CHUNKS][MOE_EP_MAX_RANKS];   /* chunk c: rows for each destination */
    int32_t recv_rows_c[MOE_EP_MAX_CHUNKS][MOE_EP_MAX_RANKS];   /* chunk c: rows from each source */
} moe_ep_plan_t;

/* Host-only, no GPU needed. counts_all [G][E] int32 (host): counts_all[s][e] =
 * slots of rank s routed to expert e (moe_ep_count on rank s). T_total = the
 * tokens of all ranks; k, cap_num and cap_den as in moe_config_t (0/0 =
 * dropless). Capacity C = floor(ceil(T_total k / E) * cap_num / cap_den)
 * (DeepSeek MoE page, 2.5); expert e keeps its first C slots in global token
 * order, so rank s keeps clamp(C - sum_{s' < s} counts_all[s'][e], 0,
 * counts_all[s][e]). Errors: G outside 1..MOE_EP_MAX_RANKS, E not a multiple
 * of G or above MOE_MAX_EXPERTS, rank outside [0, G), negative counts,
 * MOE_ERR_UNSUPPORTED_SHAPE when a row count would pass 2^31 / 128. Send rows
 * are ordered by chunk, destination rank, expert, token; received rows by
 * chunk, source rank, local expert, token. moe_ep_plan is the one-chunk plan. */
moe_status_t moe_ep_plan(int G, int rank, int E, int64_t T_total, int k, int cap_num, int cap_den,
                         const int32_t* counts_all, moe_ep_plan_t* plan);
/* chunks: 1 .. min(MOE_EP_MAX_CHUNKS, E / G) (MOE_ERR_INVALID_ARG otherwise); chunk c holds local experts
 * [c E_local / C, (c + 1) E_local / C). */
moe_status_t moe_ep_plan_chunked(int G, int rank, int E, int64_t T_total, int k, int cap_num, int cap_den,
                                 const int32_t* counts_all, int chunks, moe_ep_plan_t* plan);

/* Per-expert counts of this rank's slots: counts [E] int32 out. cfg as for
 * moe_route on this rank's batch (cfg->T its tokens; capacity fields unused
 * here). ws: moe_ep_workspace_size(cfg) bytes; it must be passed unchanged to
 * the moe_ep_dispatch of the same step (it holds the slots' ranks). */
size_t moe_ep_workspace_size(const moe_config_t* cfg);
moe_status_t moe_ep_count(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts, void* ws,
                          size_t ws_bytes, void* stream);

/* Send rows of this rank: send [plan.rows_send rows x MOE_EP_ROW_BYTES(H)] u8
 * out; slot_row [T*k] out: the send row of each slot, -1 if dropped. x [T, H]
 * bf16; plan_dev: device copy of this rank's plan; ws as moe_ep_count left it.
 * Codes and scales are moe_permute's, bit for bit. */
moe_status_t moe_ep_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                             const moe_ep_plan_t* plan_dev, uint8_t* send, int32_t* slot_row, void* ws,
                             size_t ws_bytes, void* stream);

/* Received rows (recv: plan.rows_recv rows x MOE_EP_ROW_BYTES(H), in the
 * plan's receive order) into the grouped layout of the local experts: Aq
 * [M_rows, H] u8 and As [H/128][M_rows] fp32 (moe_permute's contiguous layout;
 * padding rows code 0, scale 1), offsets [E_local + 1] out (the plan's),
 * group_row [plan.rows_recv] int32 out: the grouped row of each received row.
 * M_rows >= plan.rows_group, a multiple of 4. A plan whose sizes disagree with
 * the call's is reported (MOE_ERR_CAPACITY in the device status) and nothing
 * is written. */
moe_status_t moe_ep_receive(int H, const moe_ep_plan_t* plan_dev, int rows_recv, const uint8_t* recv, uint8_t* Aq,
                            float* As, int M_rows, int32_t* offsets, int32_t* group_row, void* stream);
/* The same for chunk `chunk` of the plan only: its receive rows (recv is the
 * whole receive buffer; the chunk's rows are [plan.recv_chunk[chunk],
 * plan.recv_chunk[chunk + 1])) and the padding rows of its experts; offsets
 * [E_c + 1] out: the chunk's experts' offsets less that of its first expert, for
 * a grouped GEMM over the chunk's rows (A = Aq + plan.offsets[first] * H, As +
 * plan.offsets[first], M_rows unchanged as the scales' row stride); group_row
 * entries of the chunk's rows. chunk outside [0, plan.chunks) is reported like a
 * plan that disagrees. */
moe_status_t moe_ep_receive_chunk(int H, const moe_ep_plan_t* plan_dev, int chunk, const uint8_t* recv, uint8_t* Aq,
                                  float* As, int M_rows, int32_t* offsets, int32_t* group_row, void* stream);

/* ret [rows_recv, H] bf16 out: row i = O [group_row[i]] (the local experts'
 * output rows, moe_grouped_gemm_fp8's bf16 epilogue) in receive order.
 * group_row needs 4-byte alignment only, so that a chunk's rows can be passed
 * as group_row + plan.recv_chunk[c], ret + plan.recv_chunk[c] * H. */
moe_status_t moe_ep_return(int H, int rows_recv, const void* O, const int32_t* group_row, void* ret, void* stream);

const char* moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_FP8_H */
