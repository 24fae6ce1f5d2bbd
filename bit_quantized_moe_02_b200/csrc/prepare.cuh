// Canonical -> prepared repacking, and the exact fp32 dequantization export.
//
// Block formats: up/gate IQ2_XXS-style, down Q2_K-style (ds4 news summary,
// "model weights"; upppp.jp, "asymmetric 2-bit quantization"), Q4_K-style for
// the 4-bit "q4" experts (ds4 news summary, "speed benchmarks").  The byte
// layouts of both forms are documented in include/ds4moe.h.
#pragma once
#include "common.cuh"

namespace ds4 {

__device__ __forceinline__ uint32_t rd_u32_bytes(const uint8_t *p) {
    return uint32_t(p[0]) | (uint32_t(p[1]) << 8) | (uint32_t(p[2]) << 16) | (uint32_t(p[3]) << 24);
}

// IQ2X: one thread per canonical block.  The 7 stored sign bits of each
// 8-vector are expanded with their parity bit and re-laid so that the mask for
// element pair p of vector j is (W << (4j+p)) & 0x80008000.
__global__ void prepare_iq2x_kernel(const uint8_t *__restrict__ canon, uint8_t *__restrict__ prep,
                                    uint64_t nblk, int n_mats, uint64_t stride) {
    uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= nblk * uint64_t(n_mats)) return;
    uint64_t m = i / nblk, b = i % nblk;
    const uint8_t *src = canon + m * nblk * 66 + b * 66;
    uint8_t *dst = prep + m * stride;
    Planes P = plane_layout(DS4MOE_FMT_IQ2X, nblk);
    uint32_t *idx = reinterpret_cast<uint32_t *>(dst + P.off[0]) + b * 8;
    uint32_t *sgn = reinterpret_cast<uint32_t *>(dst + P.off[1]) + b * 8;
    uint32_t *scl = reinterpret_cast<uint32_t *>(dst + P.off[2]) + b;
    uint16_t *dd = reinterpret_cast<uint16_t *>(dst + P.off[3]) + b;
    *dd = uint16_t(src[0] | (src[1] << 8));
    uint32_t scales = 0;
    for (int g = 0; g < 8; g++) {
        const uint8_t *gp = src + 2 + 8 * g;
        idx[g] = rd_u32_bytes(gp);
        uint32_t aux = rd_u32_bytes(gp + 4);
        scales |= (aux >> 28) << (4 * g);
        uint32_t W = 0;
        for (int j = 0; j < 4; j++) {
            uint32_t b7 = (aux >> (7 * j)) & 0x7Fu;
            uint32_t s8 = b7 | ((uint32_t(__popc(b7)) & 1u) << 7);
            for (int p = 0; p < 4; p++) {
                int sh = 4 * j + p;
                W |= ((s8 >> (2 * p)) & 1u) << (15 - sh);
                W |= ((s8 >> (2 * p + 1)) & 1u) << (31 - sh);
            }
        }
        sgn[g] = W;
    }
    *scl = scales;
}

__global__ void prepare_kquant_kernel(const uint8_t *__restrict__ canon, uint8_t *__restrict__ prep, uint64_t nblk,
                                      int n_mats, uint64_t stride, int fmt) {
    uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= nblk * uint64_t(n_mats)) return;
    uint64_t m = i / nblk, b = i % nblk;
    int bb = canonical_block_bytes(fmt);
    const uint8_t *src = canon + m * nblk * bb + b * bb;
    uint8_t *dst = prep + m * stride;
    Planes P = plane_layout(fmt, nblk);
    if (fmt == DS4MOE_FMT_Q2K) {
        uint8_t *qs = dst + P.off[0] + b * 64;
        uint8_t *sc = dst + P.off[1] + b * 16;
        uint32_t *dm = reinterpret_cast<uint32_t *>(dst + P.off[2]) + b;
        for (int t = 0; t < 16; t++) sc[t] = src[t];
        for (int t = 0; t < 64; t++) qs[t] = src[16 + t];
        *dm = rd_u32_bytes(src + 80);  // d | dmin << 16
    } else {
        uint8_t *qs = dst + P.off[0] + b * 128;
        uint8_t *sc = dst + P.off[1] + b * 12;
        uint32_t *dm = reinterpret_cast<uint32_t *>(dst + P.off[2]) + b;
        *dm = rd_u32_bytes(src);
        for (int t = 0; t < 12; t++) sc[t] = src[4 + t];
        for (int t = 0; t < 128; t++) qs[t] = src[16 + t];
    }
}

// ---- exact fp32 dequantization from the prepared planes -------------------

// Sign of element i (0..7) of vector j (0..3) in a prepared group sign word.
__device__ __forceinline__ uint32_t iq2x_sign_bit(uint32_t W, int j, int i) {
    int sh = 4 * j + (i >> 1);
    return (W >> ((i & 1) ? (31 - sh) : (15 - sh))) & 1u;
}

// One thread per (row, 8-vector).
__global__ void dequant_iq2x_kernel(const uint8_t *__restrict__ prep, const uint8_t *__restrict__ codebook, int rows,
                                    int cols, float *__restrict__ out) {
    uint64_t nvec_row = cols / 8;
    uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= uint64_t(rows) * nvec_row) return;
    uint64_t r = i / nvec_row, v = i % nvec_row;
    uint64_t nsb = cols / QK;
    Planes P = plane_layout(DS4MOE_FMT_IQ2X, uint64_t(rows) * nsb);
    uint64_t b = r * nsb + v / 32;
    int g8 = int((v / 4) % 8), j = int(v % 4);
    uint32_t ib = prep[P.off[0] + r * nvec_row + v];
    uint32_t W = reinterpret_cast<const uint32_t *>(prep + P.off[1])[r * (cols / 32) + v / 4];
    uint32_t s = (reinterpret_cast<const uint32_t *>(prep + P.off[2])[b] >> (4 * g8)) & 15u;
    float d = half_bits_to_float(reinterpret_cast<const uint16_t *>(prep + P.off[3])[b]);
    float dl = __fmul_rn(__fmul_rn(d, __fadd_rn(0.5f, float(s))), 0.25f);
    for (int e = 0; e < 8; e++) {
        float w = __fmul_rn(dl, float(codebook[ib * 8 + e]));
        out[r * cols + v * 8 + e] = iq2x_sign_bit(W, j, e) ? -w : w;
    }
}

// One thread per (row, 16-weight sub-block) for Q2K, per (row, 32-weight sub-block) for Q4K.
__global__ void dequant_kquant_kernel(const uint8_t *__restrict__ prep, int rows, int cols, int fmt,
                                      float *__restrict__ out) {
    int sub_w = fmt == DS4MOE_FMT_Q2K ? 16 : 32;
    uint64_t nsub_row = cols / sub_w;
    uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= uint64_t(rows) * nsub_row) return;
    uint64_t r = i / nsub_row, sbk = i % nsub_row;
    uint64_t nsb = cols / QK;
    Planes P = plane_layout(fmt, uint64_t(rows) * nsb);
    uint64_t b = r * nsb + (sbk * sub_w) / QK;
    int sub = int(sbk % (QK / sub_w));
    uint32_t dm = reinterpret_cast<const uint32_t *>(prep + P.off[2])[b];
    float d = half_bits_to_float(uint16_t(dm & 0xFFFF)), dmin = half_bits_to_float(uint16_t(dm >> 16));
    int sc, m;
    if (fmt == DS4MOE_FMT_Q2K) {
        uint8_t scb = prep[P.off[1] + b * 16 + sub];
        sc = scb & 15; m = scb >> 4;
    } else {
        const uint8_t *s12 = prep + P.off[1] + b * 12;
        uint64_t bits = 0;
        for (int t = 0; t < 12 && t < 8; t++) bits |= uint64_t(s12[t]) << (8 * t);
        uint32_t hi = uint32_t(s12[8]) | (uint32_t(s12[9]) << 8) | (uint32_t(s12[10]) << 16) | (uint32_t(s12[11]) << 24);
        // 96-bit string = bits (low 64) | hi << 64
        auto field = [&](int pos) -> int {
            if (pos + 6 <= 64) return int((bits >> pos) & 63u);
            if (pos >= 64) return int((hi >> (pos - 64)) & 63u);
            return int(((bits >> pos) | (uint64_t(hi) << (64 - pos))) & 63u);
        };
        sc = field(6 * sub); m = field(48 + 6 * sub);
    }
    float a = __fmul_rn(d, float(sc)), c = __fmul_rn(dmin, float(m));
    for (int e = 0; e < sub_w; e++) {
        int q;
        if (fmt == DS4MOE_FMT_Q2K) {
            uint8_t byte = prep[P.off[0] + b * 64 + (sub * 16 + e) / 4];
            q = (byte >> (2 * ((sub * 16 + e) & 3))) & 3;
        } else {
            uint8_t byte = prep[P.off[0] + b * 128 + (sub * 32 + e) / 2];
            q = ((sub * 32 + e) & 1) ? (byte >> 4) : (byte & 15);
        }
        out[r * cols + sbk * sub_w + e] = __fsub_rn(__fmul_rn(a, float(q)), c);
    }
}

}  // namespace ds4
