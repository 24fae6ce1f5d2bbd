// Arguments and small helpers of the grouped (many-token) dequantize-GEMM kernels.
//
// Swap-AB: the (dequantized) weight rows are the 128-row A operand and the tokens routed to an expert the B
// operand, so an expert with few tokens is not padded to 128 rows.  GATEUP mode runs gate and up together and
// applies SwiGLU in the epilogue; DOWN mode scales by the routing weight.
#pragma once
#include "common.cuh"

namespace ds4 {

struct GroupedArgs {
    const uint8_t *a0;  // gate (GATEUP) or down matrix of expert 0; dense bf16 matrix for the shared expert
    const uint8_t *a1;  // up matrix of expert 0 (GATEUP)
    uint64_t a_stride;  // bytes between experts (a0)
    uint64_t a1_stride; // bytes between experts (a1)
    int n_mats;         // experts (matrices) behind a0 / a1
    Planes pa;
    int rows;  // rows of one A matrix
    int K;
    const uint8_t *codebook;
    const void *b_src;         // B rows: [*, K] fp16
    const int32_t *b_rowidx;   // B row of each position (token gather) or NULL = position itself
    const float *b_colscale;   // per-B-row factor applied to the accumulator, or NULL
    const int32_t *tile_e, *tile_pos0, *tile_cnt, *n_tiles;  // device tile list; NULL = identity tiles
    int n_pos;                 // positions for identity tiles
    const float *pos_weight;   // DOWN: factor per position, or NULL
    void *out;                 // GATEUP: [pos][rows] fp16;  DOWN: [pos][rows] fp32
    int ldo;
    // Power-of-two exponents of the fp16 SwiGLU output, one per (token tile, 128-row tile of h): GATEUP writes
    // h_exp_out[tile * (rows / 128) + row tile] = e >= 0 and stores h * 2^-e (e = 0 unless |h| > 65504); DOWN
    // multiplies the weights of K range [128 i, 128 i + 128) by 2^h_exp_in[tile * (K / 128) + i], so each
    // product, and the result, is unchanged.  NULL: no scaling.
    int32_t *h_exp_out;
    const int32_t *h_exp_in;
    // DOWN: when set, row p of the result is added (red.global.add) into out row out_row[p] instead of being
    // stored at row p: the weighted combine of the layer fused into the epilogue
    const int32_t *out_row;
};

// 128-byte swizzle of a K-major fp16 tile: 16-byte chunk `chunk` of row `row`
__device__ __forceinline__ int swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

// 6-bit field at bit `pos` of the 96-bit little-endian Q4K scale string (s0 | s1 << 32 | s2 << 64)
__device__ __forceinline__ int q4k_field(uint32_t s0, uint32_t s1, uint32_t s2, int pos) {
    uint64_t lo = uint64_t(s0) | (uint64_t(s1) << 32);
    if (pos + 6 <= 64) return int((lo >> pos) & 63u);
    if (pos >= 64) return int((s2 >> (pos - 64)) & 63u);
    return int(((lo >> pos) | (uint64_t(s2) << (64 - pos))) & 63u);
}

}  // namespace ds4
