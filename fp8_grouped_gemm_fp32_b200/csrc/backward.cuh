// Arguments of the backward's transposed quantisation (backward.cu), shared with its caller (api.cu).
#pragma once
#include <stdint.h>

namespace moe {

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

}  // namespace moe
