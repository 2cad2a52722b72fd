/*
 * CPU oracle for the FP8 MoE expert layer -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously-correct C. Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it; the product library never
 * does, and the two share no code.
 *
 * Sources (page title, section):
 *  [P1] "MegaMoE math model + DeepGEMM source walk-through" (discosf.com),
 *       2.1 (y formula, Concat grouping, grouped shape contract),
 *       2.2 (biased softmax router), 3.2 (grouped call, group sizes),
 *       3.3 (E4M3 quantisation formula with the 448 clamp; fp32 accumulator,
 *       round-to-nearest-even conversion to BF16).
 *  [P2] "Dense GEMM -> TP MoE" (cf-1.com), 3.1 (linear + softmax + top-k,
 *       renormalisation inside the top-k), 3.2 / 4.2 (capacity, dropping).
 *  [P3] "DeepSeek-V4 lecture 4: routing, FP4 experts, parallelism"
 *       (tqpw.cn), 2.2 (hash routing hash(token_id) % num_experts),
 *       2.3 (fp32 softmax even for a bf16 model), 3.1 (4-bit expert
 *       weights: per-channel blocks scaled by their max-abs, 7 levels a side).
 *  [P4] "DeepSeek MoE architecture" (mooersco.com), chapter 1 (top-2
 *       pseudo-code: top-k of the logits, softmax over the selected ones),
 *       2.5 (capacity = ceil(top-k * N / E) * alpha, worked example -> 76;
 *       overflow tokens dropped silently, no re-route).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - router logits are fp32 with one canonical summation order
 *    (orc_router_logits); bf16 x converts exactly to fp32;
 *  - top-k selects on logits, ties to the lowest expert index, output in
 *    descending order; weights are renormalised over the top-k;
 *  - hash multiplier 2654435761 (uint32 wrap-around), k = 1, weight 1.0;
 *  - capacity C = floor(ceil(T*k/E) * cap_num / cap_den) in integers; ranks
 *    within an expert follow token index; dropped slots contribute zero and
 *    the surviving weights are not renormalised;
 *  - activation quantisation: one fp32 scale per 1x128 group, scale =
 *    max|v| / 448 (1.0 when max|v| = 0), code = E4M3 RNE (saturating) of the
 *    fp32-rounded v / scale;
 *  - dequantisation to fp32 (code * scale rounded to fp32), fp64 sums,
 *    h = silu(a) * b in fp64 rounded to fp32 and requantised as above,
 *    o rounded to bf16 (RNE), y = fp64 weighted sum rounded to bf16;
 *  - 4-bit expert weights ([P3] 3.1 gives the formula, not the block): the
 *    block is one weight row (output channel) by 128 consecutive k, the
 *    granularity of the activation scales and of the GEMM's K blocks; the
 *    level rounds half to even; the stored scale is max-abs / 7 in fp32;
 *  - bias balancing ([P1] 2.2 gives the direction, the step size and the
 *    interval): an expert's load is the number of slots routed to it (before
 *    any capacity drop), summed over the interval; above the mean -> bias
 *    minus gamma, below -> plus gamma, at the mean -> unchanged.
 *
 * Parity pins live in tests/ (run with -m "not gpu").
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* E4M3 (E4M3FN) codec, written from the format definition. */
double   orc_e4m3_decode(uint8_t code);
uint8_t  orc_e4m3_encode(float v);
float    orc_bf16_to_f32(uint16_t b);
uint16_t orc_f64_to_bf16(double v);

/* Router logits l[t,e] = (x[t,:] . Wg[e,:]) + bias[e] in fp32, canonical order. */
void orc_router_logits(int T, int H, int E, const uint16_t* x, const float* Wg,
                       const float* bias /* nullable */, float* logits, int nthreads);
/* Top-k of the logits + renormalised softmax weights over the selected k. */
void orc_topk_softmax(int T, int E, int k, const float* logits, int32_t* topk_idx, float* topk_w);
/* Hash routing: expert = (uint32)(token_id * 2654435761) % E, weight 1. */
void orc_route_hash(int T, int E, const int32_t* token_ids, int32_t* topk_idx, float* topk_w);
/* Capacity; returns -1 for dropless (cap_num == 0). */
int64_t orc_capacity(int T, int k, int E, int cap_num, int cap_den);
/* Dispatch: counts, kept, row offsets and the row <-> slot maps.
 * layout 0 = contiguous (groups padded to `pad` rows), 1 = masked (E x masked_max_m).
 * row_src has rows_cap entries (-1 where no slot); slot_row has T*k entries (-1 = dropped).
 * Returns 0, or 1 if a masked group overflowed masked_max_m (extra slots dropped). */
int orc_dispatch(int T, int k, int E, const int32_t* topk_idx, int64_t cap, int layout, int pad,
                 int masked_max_m, int64_t rows_cap, int32_t* counts, int32_t* kept,
                 int32_t* offsets, int32_t* row_src, int32_t* slot_row);
/* 1x128 group quantisation of fp32 rows: q [rows, K], s [rows, K/128] (row-major). */
void orc_quant_rows(int64_t rows, int K, const float* v, uint8_t* q, float* s);
/* One expert's SwiGLU FFN on n rows of quantised activations:
 * xq [n,H], xs [n,H/128] -> hq [n,I], hs [n,I/128], o [n,H] (bf16 bits). */
void orc_expert_rows(int n, int H, int I, const uint8_t* xq, const float* xs,
                     const uint8_t* W1q, const float* S1, const uint8_t* W3q, const float* S3,
                     const uint8_t* W2q, const float* S2,
                     uint8_t* hq, float* hs, uint16_t* o, int nthreads);
/* Grouped GEMM with the boundary's semantics (see include/moe_fp8.h):
 * layout 0: rows [offsets[e], offsets[e+1]) use expert e; layout 1: rows
 * e*M_rows + [0, masked_m[e]). As/Ds are K-block-major [K/128][ld].
 * epilogue 0: D bf16 [rows, N]; epilogue 1: N = 2I with 128-row blocks
 * alternating W1/W3, D = Hq u8 [rows, I], Ds = Hs [I/128][ld]. */
void orc_grouped_gemm(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                      const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                      int epilogue, void* D, float* Ds, int nthreads);
/* The same grouped GEMM with 4-bit weights ([P3] 3.1): B = [E, N, K/2] bytes,
 * two codes each (even k in the low nibble, 4-bit two's complement, levels
 * -7..7), Bs = [E, K/128, N] fp32 (one scale per weight row per 128-wide K
 * block: max-abs / 7, K-block-major); a weight dequantises to code * scale in
 * fp32. With the
 * SwiGLU epilogue the rows of B follow the same W1/W3 128-row alternation. */
void orc_grouped_gemm_w4(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                         const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                         int epilogue, void* D, float* Ds, int nthreads);
/* The 4-bit weight level (-7..7) of element k of a packed row: sign and 3-bit
 * magnitude, eight consecutive k per little-endian 32-bit word; level i of a
 * word (i = 0..3): magnitude in bits 4i..4i+2, sign in bit 8i+7; level 4+i:
 * magnitude in bits 16+4i..16+4i+2, sign in bit 8i+3. */
int orc_w4_decode(const uint8_t* row, int k);
/* One group of n values quantised with one scale: max|v| / 448 (1 for all
 * zeros), codes E4M3 of v / scale (the 1x128 rule applied to any group). */
void orc_quant_group(int64_t n, const float* v, uint8_t* q, float* s);
/* Combine: y[t,:] = sum_j [kept] w[t,j] * O[slot_row[t*k+j], :], fp64, -> bf16. */
void orc_combine(int T, int k, int H, const int32_t* slot_row, const float* topk_w,
                 const uint16_t* O, uint16_t* y);
/* Auxiliary-loss-free bias balancing: load += counts; if update, each bias
 * moves by -gamma / +gamma / 0 as E*load[e] is above / below / equal to
 * sum(load) (fp32 arithmetic), and load is cleared. */
void orc_balance_bias(int E, const int32_t* counts, int64_t* load, float* bias, float gamma, int update);

#ifdef __cplusplus
}
#endif
#endif
