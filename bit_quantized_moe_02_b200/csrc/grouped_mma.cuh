// Grouped dequantize-GEMM for many tokens, warp-level mma.sync version.
//
// Swap-AB: the (dequantized) weight rows are the 128-row A operand, the tokens
// routed to the expert the 64-column B operand, so an expert with few tokens
// is not padded to 128.  Every K-chunk of packed weights is dequantized once
// per CTA straight into a swizzled fp16 shared-memory tile; token rows are
// gathered with cp.async.  GATEUP mode interleaves gate and up rows so each
// thread holds matching gate/up accumulators and applies SwiGLU in the
// epilogue; DOWN mode scales by the routing weight.  Operands are fp16 (bf16
// shared-expert weights are converted on their way into shared memory).  This is the portable
// tensor-core path; the tcgen05 path in grouped_tc.cuh supersedes it on sm_100a
// where available.
#pragma once
#include "common.cuh"
#include "permute.cuh"

namespace ds4 {

constexpr int GM_M = 128, GM_N = TILE_N, GM_K = 64, GM_THREADS = 256;
constexpr int GM_A_BYTES = GM_M * GM_K * 2;  // 16 KB
constexpr int GM_B_BYTES = GM_N * GM_K * 2;  // 8 KB
constexpr int GM_TABLE_BYTES = 256 * 16;     // plain codebook table: 256 x 8 fp16
constexpr int GM_SMEM = 2 * GM_A_BYTES + 2 * GM_B_BYTES + GM_TABLE_BYTES;

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
};

__device__ __forceinline__ int swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// bf16 pair -> fp16 pair; sets *inf when a value leaves the fp16 range.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t u, bool &inf) {
    const __half2 h = __floats2half2_rn(bf16_lo(u), bf16_hi(u));
    inf |= __hisinf(__low2half(h)) | __hisinf(__high2half(h));
    return half2_as_u32(h);
}

// ---- A-tile producers: 32 consecutive weights of one row -> 4 x 16 B of the swizzled tile -------------

// Raw packed data of 32 weights (one IQ2X group / two Q2K sub-blocks / one Q4K sub-block / 32 bf16).
struct APack {
    uint32_t w[16];
};

template <int AFMT>
__device__ __forceinline__ void a_load(APack &pk, const uint8_t *__restrict__ mat, const Planes &P, int row, int K,
                                       int k0) {
    const int nsb = K / QK;
    if constexpr (AFMT == DS4MOE_FMT_IQ2X) {
        const int gg = k0 / 32;
        pk.w[0] = ldg_nc_u32(mat + P.off[0] + size_t(row) * (K / 8) + gg * 4);
        pk.w[1] = ldg_nc_u32(mat + P.off[1] + (size_t(row) * (K / 32) + gg) * 4);
        pk.w[2] = ldg_nc_u32(mat + P.off[2] + (size_t(row) * nsb + gg / 8) * 4);
        pk.w[3] = *reinterpret_cast<const uint16_t *>(mat + P.off[3] + (size_t(row) * nsb + gg / 8) * 2);
        pk.w[4] = gg % 8;
    } else if constexpr (AFMT == DS4MOE_FMT_Q2K) {
        const size_t b = size_t(row) * nsb + k0 / QK;
        const int sub = (k0 % QK) / 16;
        const uint2 q = *reinterpret_cast<const uint2 *>(mat + P.off[0] + b * 64 + sub * 4);
        pk.w[0] = q.x;
        pk.w[1] = q.y;
        pk.w[2] = *reinterpret_cast<const uint16_t *>(mat + P.off[1] + b * 16 + sub);
        pk.w[3] = ldg_nc_u32(mat + P.off[2] + b * 4);
    } else if constexpr (AFMT == DS4MOE_FMT_Q4K) {
        const size_t b = size_t(row) * nsb + k0 / QK;
        const int sub = (k0 % QK) / 32;
        const uint4 q = ldg_nc_v4(mat + P.off[0] + b * 128 + sub * 16);
        pk.w[0] = q.x; pk.w[1] = q.y; pk.w[2] = q.z; pk.w[3] = q.w;
        const uint32_t *s = reinterpret_cast<const uint32_t *>(mat + P.off[1] + b * 12);
        pk.w[4] = s[0]; pk.w[5] = s[1]; pk.w[6] = s[2];
        pk.w[7] = ldg_nc_u32(mat + P.off[2] + b * 4);
    } else {  // dense bf16 row: 32 elements = 64 bytes, copied as is
        const uint8_t *p = mat + (size_t(row) * K + k0) * 2;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const uint4 v = ldg_nc_v4(p + 16 * i);
            pk.w[4 * i] = v.x; pk.w[4 * i + 1] = v.y; pk.w[4 * i + 2] = v.z; pk.w[4 * i + 3] = v.w;
        }
    }
}

__device__ __forceinline__ int q4k_field(uint32_t s0, uint32_t s1, uint32_t s2, int pos) {
    uint64_t lo = uint64_t(s0) | (uint64_t(s1) << 32);
    if (pos + 6 <= 64) return int((lo >> pos) & 63u);
    if (pos >= 64) return int((s2 >> (pos - 64)) & 63u);
    return int(((lo >> pos) | (uint64_t(s2) << (64 - pos))) & 63u);
}

// Dequantize 32 weights into 4 uint4 (8 fp16 each, consecutive k).  The IQ2X codebook table holds entry i
// at tbl + i * TSTRIDE (8 fp16 values); bf16 rows are converted, setting *inf if a value leaves fp16 range.
template <int AFMT, int TSTRIDE = 16>
__device__ __forceinline__ void a_dequant(const APack &pk, const uint8_t *tbl, int k0, uint4 (&o)[4],
                                          bool &inf) {
    constexpr uint32_t M = 0x80008000u;
    if constexpr (AFMT == DS4MOE_FMT_BF16) {
#pragma unroll
        for (int j = 0; j < 4; j++)
            o[j] = make_uint4(bf16x2_to_f16x2(pk.w[4 * j], inf), bf16x2_to_f16x2(pk.w[4 * j + 1], inf),
                              bf16x2_to_f16x2(pk.w[4 * j + 2], inf), bf16x2_to_f16x2(pk.w[4 * j + 3], inf));
    } else if constexpr (AFMT == DS4MOE_FMT_IQ2X) {
        const float dv = half_bits_to_float(uint16_t(pk.w[3]));
        const float s = float((pk.w[2] >> (4 * pk.w[4])) & 15u);
        const __half2 D2 = __float2half2_rn((dv * (0.5f + s)) * 0.25f);
        const uint32_t W = pk.w[1];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t ib = (pk.w[0] >> (8 * j)) & 0xFFu;
            const uint4 cb = *reinterpret_cast<const uint4 *>(tbl + ib * TSTRIDE);
            const uint32_t Wj = W << (4 * j);
            o[j].x = half2_as_u32(__hmul2(u32_as_half2(cb.x ^ (Wj & M)), D2));
            o[j].y = half2_as_u32(__hmul2(u32_as_half2(cb.y ^ ((Wj << 1) & M)), D2));
            o[j].z = half2_as_u32(__hmul2(u32_as_half2(cb.z ^ ((Wj << 2) & M)), D2));
            o[j].w = half2_as_u32(__hmul2(u32_as_half2(cb.w ^ ((Wj << 3) & M)), D2));
        }
    } else if constexpr (AFMT == DS4MOE_FMT_Q2K) {
        const float dv = half_bits_to_float(uint16_t(pk.w[3] & 0xFFFF));
        const float dm = half_bits_to_float(uint16_t(pk.w[3] >> 16));
        const __half2 k1024 = __float2half2_rn(1024.f);
#pragma unroll
        for (int sb = 0; sb < 2; sb++) {
            const uint32_t scb = (pk.w[2] >> (8 * sb)) & 0xFFu;
            const __half2 a2 = __float2half2_rn(dv * float(scb & 15u));
            const __half2 c2 = __float2half2_rn(-(dm * float(scb >> 4)));
            __half2 P[8];
#pragma unroll
            for (int p = 0; p < 8; p++) {
                const uint32_t v = ((pk.w[sb] >> (2 * p)) & 0x00030003u) | 0x64006400u;
                P[p] = __hfma2(__hsub2(u32_as_half2(v), k1024), a2, c2);  // (w_p, w_{p+8})
            }
            uint32_t *oo = reinterpret_cast<uint32_t *>(&o[2 * sb]);
#pragma unroll
            for (int p = 0; p < 4; p++) {
                oo[p] = half2_as_u32(__lows2half2(P[2 * p], P[2 * p + 1]));       // (w_2p, w_2p+1)
                oo[4 + p] = half2_as_u32(__highs2half2(P[2 * p], P[2 * p + 1]));  // (w_2p+8, w_2p+9)
            }
        }
    } else if constexpr (AFMT == DS4MOE_FMT_Q4K) {
        const int sub = (k0 % QK) / 32;
        const float dv = half_bits_to_float(uint16_t(pk.w[7] & 0xFFFF));
        const float dm = half_bits_to_float(uint16_t(pk.w[7] >> 16));
        const int sc = q4k_field(pk.w[4], pk.w[5], pk.w[6], 6 * sub);
        const int mn = q4k_field(pk.w[4], pk.w[5], pk.w[6], 48 + 6 * sub);
        const __half2 a2 = __float2half2_rn(dv * float(sc));
        const __half2 c2 = __float2half2_rn(-(dm * float(mn)));
        const __half2 k1024 = __float2half2_rn(1024.f);
#pragma unroll
        for (int w = 0; w < 4; w++) {  // word w: weights 8w..8w+7, nibble n at bits 4n
            __half2 P[4];
#pragma unroll
            for (int n = 0; n < 4; n++) {
                const uint32_t v = ((pk.w[w] >> (4 * n)) & 0x000F000Fu) | 0x64006400u;
                P[n] = __hfma2(__hsub2(u32_as_half2(v), k1024), a2, c2);  // (w_n, w_{n+4})
            }
            o[w].x = half2_as_u32(__lows2half2(P[0], P[1]));
            o[w].y = half2_as_u32(__lows2half2(P[2], P[3]));
            o[w].z = half2_as_u32(__highs2half2(P[0], P[1]));
            o[w].w = half2_as_u32(__highs2half2(P[2], P[3]));
        }
    }
}

// ---- the kernel -------------------------------------------------------------------------------------------

template <int AFMT, bool GATEUP>
__global__ void __launch_bounds__(GM_THREADS) grouped_mma_kernel(GroupedArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *As = smem;
    uint8_t *Bs = smem + 2 * GM_A_BYTES;
    uint8_t *tbl = smem + 2 * GM_A_BYTES + 2 * GM_B_BYTES;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    int e = 0, pos0, cnt;
    if (a.tile_e) {
        if (int(blockIdx.y) >= *a.n_tiles) return;
        e = a.tile_e[blockIdx.y];
        pos0 = a.tile_pos0[blockIdx.y];
        cnt = a.tile_cnt[blockIdx.y];
    } else {
        pos0 = blockIdx.y * GM_N;
        if (pos0 >= a.n_pos) return;
        cnt = min(GM_N, a.n_pos - pos0);
    }
    if constexpr (AFMT == DS4MOE_FMT_IQ2X) {
        for (int i = tid; i < 256; i += GM_THREADS) {
            const uint8_t *cb = a.codebook + i * 8;
            __half2 h[4];
#pragma unroll
            for (int p = 0; p < 4; p++) h[p] = __floats2half2_rn(float(cb[2 * p]), float(cb[2 * p + 1]));
            *reinterpret_cast<uint4 *>(tbl + i * 16) = *reinterpret_cast<uint4 *>(h);
        }
    }

    // A job of this thread: tile row R, 32-weight half hh of each K-chunk
    const int R = tid >> 1, hh = tid & 1;
    const uint8_t *amat;
    int arow;
    if constexpr (GATEUP) {
        const int q = R >> 4, w = R & 15;
        amat = w < 8 ? a.a0 + size_t(e) * a.a_stride : a.a1 + size_t(e) * a.a1_stride;
        arow = blockIdx.x * 64 + 8 * q + (w & 7);
    } else {
        amat = a.a0 + size_t(e) * a.a_stride;
        arow = blockIdx.x * GM_M + R;
    }
    __shared__ int32_t s_brow[GM_N];
    __shared__ float s_colsc[GM_N];
    if (tid < GM_N) {
        float sc = 1.f;
        int brow = 0;
        if (tid < cnt) {
            const int pos = pos0 + tid;
            brow = a.b_rowidx ? a.b_rowidx[pos] : pos;
            if (a.b_colscale) sc *= a.b_colscale[brow];
            if (a.pos_weight) sc *= a.pos_weight[pos];
        }
        s_brow[tid] = brow;
        s_colsc[tid] = sc;
    }
    __syncthreads();
    const int nk = a.K / GM_K;
    const int elem_b = 2;
    const uint8_t *bsrc = reinterpret_cast<const uint8_t *>(a.b_src);

    auto issue_b = [&](int kc, int stage) {
#pragma unroll
        for (int i = 0; i < 2; i++) {
            const int job = tid + GM_THREADS * i;
            const int n = job >> 3, c = job & 7;
            const uint32_t dst = smem_u32(Bs + stage * GM_B_BYTES + swz(n, c));
            if (n < cnt) {
                cp_async16(dst, bsrc + (size_t(s_brow[n]) * a.K + kc * GM_K + c * 8) * elem_b, 16);
            } else {
                cp_async16(dst, bsrc, 0);
            }
        }
        cp_async_commit();
    };
    auto store_a = [&](const APack &pk, int kc, int stage) {
        uint8_t *dst = As + stage * GM_A_BYTES;
        uint4 o[4];
        bool inf = false;
        a_dequant<AFMT>(pk, tbl, kc * GM_K + hh * 32, o, inf);
#pragma unroll
        for (int j = 0; j < 4; j++) *reinterpret_cast<uint4 *>(dst + swz(R, hh * 4 + j)) = o[j];
        if (inf) set_device_error(DS4MOE_EDEVICE);
    };

    float acc[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; i++)
#pragma unroll
        for (int j = 0; j < 4; j++)
#pragma unroll
            for (int t = 0; t < 4; t++) acc[i][j][t] = 0.f;

    const int wm = warp & 3, wn = warp >> 2;
    APack pk;
    issue_b(0, 0);
    a_load<AFMT>(pk, amat, a.pa, arow, a.K, hh * 32);
    __syncthreads();  // codebook table
    store_a(pk, 0, 0);
    cp_async_wait0();
    __syncthreads();

    for (int kc = 0; kc < nk; kc++) {
        const int st = kc & 1;
        const bool more = kc + 1 < nk;
        if (more) {
            issue_b(kc + 1, st ^ 1);
            a_load<AFMT>(pk, amat, a.pa, arow, a.K, (kc + 1) * GM_K + hh * 32);
        }
        const uint32_t abase = smem_u32(As + st * GM_A_BYTES), bbase = smem_u32(Bs + st * GM_B_BYTES);
#pragma unroll
        for (int ks = 0; ks < GM_K / 16; ks++) {
            uint32_t af[2][4], bf[4][2];
#pragma unroll
            for (int mi = 0; mi < 2; mi++) {
                const int row = wm * 32 + mi * 16 + (lane & 15);
                const int ch = ks * 2 + (lane >> 4);
                ldsm_x4(abase + swz(row, ch), af[mi][0], af[mi][1], af[mi][2], af[mi][3]);
            }
#pragma unroll
            for (int nj = 0; nj < 2; nj++) {
                const int row = wn * 32 + nj * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int ch = ks * 2 + ((lane >> 3) & 1);
                uint32_t r0, r1, r2, r3;
                ldsm_x4(bbase + swz(row, ch), r0, r1, r2, r3);
                bf[2 * nj][0] = r0; bf[2 * nj][1] = r1;
                bf[2 * nj + 1][0] = r2; bf[2 * nj + 1][1] = r3;
            }
#pragma unroll
            for (int mi = 0; mi < 2; mi++)
#pragma unroll
                for (int ni = 0; ni < 4; ni++) mma16816(acc[mi][ni], af[mi], bf[ni][0], bf[ni][1]);
        }
        if (more) store_a(pk, kc + 1, st ^ 1);
        cp_async_wait0();
        __syncthreads();
    }

    // ---- epilogue ----
    const int g = lane >> 2, t4 = lane & 3;
    if constexpr (GATEUP) {
        // h(o, n) = silu(gate) * up  staged as [n][64] then written as 128-byte rows
        uint16_t *Hs = reinterpret_cast<uint16_t *>(smem);
        bool overflow = false;
#pragma unroll
        for (int mi = 0; mi < 2; mi++) {
            const int o = 8 * (2 * wm + mi) + g;
#pragma unroll
            for (int ni = 0; ni < 4; ni++) {
#pragma unroll
                for (int cc = 0; cc < 2; cc++) {
                    const int n = wn * 32 + ni * 8 + 2 * t4 + cc;
                    const float sc = s_colsc[n];
                    const float gv = acc[mi][ni][cc] * sc, uv = acc[mi][ni][2 + cc] * sc;
                    const float hv = silu(gv) * uv;
                    overflow |= !(fabsf(hv) <= 65504.f) && n < cnt;
                    Hs[n * 64 + o] = __half_as_ushort(__float2half(hv));
                }
            }
        }
        if (overflow) set_device_error(DS4MOE_EDEVICE);
        __syncthreads();
        uint16_t *out = reinterpret_cast<uint16_t *>(a.out);
        for (int i = tid; i < GM_N * 8; i += GM_THREADS) {
            const int n = i >> 3, c = i & 7;
            if (n < cnt)
                *reinterpret_cast<uint4 *>(out + size_t(pos0 + n) * a.ldo + blockIdx.x * 64 + c * 8) =
                    *reinterpret_cast<const uint4 *>(Hs + n * 64 + c * 8);
        }
    } else {
        float *Ys = reinterpret_cast<float *>(smem);  // [n][128 + 4]
        constexpr int LDY = GM_M + 4;
#pragma unroll
        for (int mi = 0; mi < 2; mi++) {
#pragma unroll
            for (int ni = 0; ni < 4; ni++) {
#pragma unroll
                for (int cc = 0; cc < 2; cc++) {
                    const int n = wn * 32 + ni * 8 + 2 * t4 + cc;
                    const float sc = s_colsc[n];
                    const int r = wm * 32 + mi * 16 + g;
                    Ys[n * LDY + r] = acc[mi][ni][cc] * sc;
                    Ys[n * LDY + r + 8] = acc[mi][ni][2 + cc] * sc;
                }
            }
        }
        __syncthreads();
        float *out = reinterpret_cast<float *>(a.out);
        for (int i = tid; i < GM_N * (GM_M / 4); i += GM_THREADS) {
            const int n = i / (GM_M / 4), c = (i % (GM_M / 4)) * 4;
            if (n < cnt)
                *reinterpret_cast<float4 *>(out + size_t(pos0 + n) * a.ldo + blockIdx.x * GM_M + c) =
                    *reinterpret_cast<const float4 *>(Ys + n * LDY + c);
        }
    }
}

}  // namespace ds4
