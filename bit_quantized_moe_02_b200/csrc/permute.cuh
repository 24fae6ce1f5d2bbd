// Token permutation by expert id (prefill / batched decode), activation
// conversion for the fp16 tensor-core operands, and the final combine.
//
// The (token, slot) pairs routed to each expert are gathered into contiguous
// position ranges (stable: increasing token, then slot) so that the grouped
// GEMM reads every expert's packed weights once per token tile; the combine
// step adds each token's k weighted expert outputs back in slot order.  The
// MoE structure (router -> experts -> combine) is the ds4 news summary's
// "model weights" description; the permutation scheme is this library's own.
#pragma once
#include "common.cuh"

namespace ds4 {

constexpr int PERM_BLOCK = 1024;

// x16[t] = fp16(x[t] * 2^e_t) with max|x16[t]| in [2^13, 2^14); xinv[t] = 2^-e_t.
__global__ void __launch_bounds__(256) prep_x_kernel(const __nv_bfloat16 *__restrict__ x, int d,
                                                     __half *__restrict__ x16, float *__restrict__ xinv) {
    __shared__ float red[8];
    const int t = blockIdx.x;
    const __nv_bfloat16 *row = x + size_t(t) * d;
    float m = 0.f;
    for (int i = threadIdx.x * 8; i < d; i += blockDim.x * 8) {
        uint4 v = *reinterpret_cast<const uint4 *>(row + i);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; j++) m = fmaxf(m, fmaxf(fabsf(bf16_lo(u[j])), fabsf(bf16_hi(u[j]))));
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    float v = (threadIdx.x & 31) < (blockDim.x >> 5) ? red[threadIdx.x & 31] : 0.f;
    v = warp_max(v);
    const int e = pow2_exponent_for(v, 14);
    const float s = ldexpf(1.f, e);
    if (threadIdx.x == 0) xinv[t] = ldexpf(1.f, -e);
    for (int i = threadIdx.x * 8; i < d; i += blockDim.x * 8) {
        uint4 vv = *reinterpret_cast<const uint4 *>(row + i);
        const uint32_t u[4] = {vv.x, vv.y, vv.z, vv.w};
        uint4 o;
        uint32_t *ou = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int j = 0; j < 4; j++) ou[j] = half2_as_u32(__floats2half2_rn(bf16_lo(u[j]) * s, bf16_hi(u[j]) * s));
        *reinterpret_cast<uint4 *>(x16 + size_t(t) * d + i) = o;
    }
}

// Permuted activations for the routed gate/up GEMM: x_perm[p] = x16[perm_tok[p]], so that every expert's
// token rows are contiguous and one tensor copy moves a whole token tile.  One warp per row.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __half *__restrict__ x16, int d,
                                                          const int32_t *__restrict__ perm_tok, int N,
                                                          __half *__restrict__ x_perm) {
    const int p = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (p >= N) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x16 + size_t(perm_tok[p]) * d);
    uint4 *dst = reinterpret_cast<uint4 *>(x_perm + size_t(p) * d);
    for (int i = lane; i < d / 8; i += 32) dst[i] = src[i];
}

// Per-block expert histogram of the T*k routed pairs.
__global__ void __launch_bounds__(PERM_BLOCK) perm_count_kernel(const int32_t *__restrict__ ids, int N, int E,
                                                                int32_t *__restrict__ blk_counts) {
    extern __shared__ int32_t hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int i = blockIdx.x * PERM_BLOCK + threadIdx.x;
    if (i < N) {
        const int e = ids[i];
        if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
        else set_device_error(DS4MOE_EDEVICE);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blk_counts[size_t(blockIdx.x) * E + e] = hist[e];
}

// Single CTA: expert offsets, per-block scatter bases, and the token-tile list.
// meta = {n_tiles, n_used_experts}; counts/offsets [E].
__global__ void __launch_bounds__(1024) perm_scan_kernel(int32_t *__restrict__ blk_counts, int nblk, int E, int tile_n,
                                                         int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                                                         int32_t *__restrict__ tile_e, int32_t *__restrict__ tile_pos0,
                                                         int32_t *__restrict__ tile_cnt, int32_t *__restrict__ meta) {
    __shared__ int32_t s_tot[1024], s_nt[1024];
    __shared__ int32_t s_scan_a[1024], s_scan_b[1024];
    const int e = threadIdx.x;
    int tot = 0;
    if (e < E)
        for (int b = 0; b < nblk; b++) tot += blk_counts[size_t(b) * E + e];
    const int nt = (tot + tile_n - 1) / tile_n;
    s_tot[e] = e < E ? tot : 0;
    s_nt[e] = e < E ? nt : 0;
    __syncthreads();
    // inclusive Hillis-Steele scans of s_tot and s_nt
    s_scan_a[e] = s_tot[e];
    s_scan_b[e] = s_nt[e];
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        int a = e >= o ? s_scan_a[e - o] : 0;
        int b = e >= o ? s_scan_b[e - o] : 0;
        __syncthreads();
        s_scan_a[e] += a;
        s_scan_b[e] += b;
        __syncthreads();
    }
    if (e < E) {
        const int off = s_scan_a[e] - tot;
        const int toff = s_scan_b[e] - nt;
        counts[e] = tot;
        offsets[e] = off;
        int run = off;
        for (int b = 0; b < nblk; b++) {
            const int c = blk_counts[size_t(b) * E + e];
            blk_counts[size_t(b) * E + e] = run;  // becomes the block's scatter base
            run += c;
        }
        for (int i = 0; i < nt; i++) {
            tile_e[toff + i] = e;
            tile_pos0[toff + i] = off + i * tile_n;
            tile_cnt[toff + i] = min(tile_n, tot - i * tile_n);
        }
    }
    if (e == 1023) {
        meta[0] = s_scan_b[1023];
    }
    __syncthreads();
    if (e == 0) {
        int used = 0;
        for (int q = 0; q < E; q++) used += s_tot[q] > 0;
        meta[1] = used;
    }
}

// Stable scatter: position of pair i = base[blk][e] + (# earlier pairs of the block with the same expert).
__global__ void __launch_bounds__(PERM_BLOCK) perm_scatter_kernel(const int32_t *__restrict__ ids,
                                                                  const float *__restrict__ weights, int N, int k,
                                                                  int E, const int32_t *__restrict__ blk_base,
                                                                  int32_t *__restrict__ perm_tok,
                                                                  float *__restrict__ perm_w,
                                                                  int32_t *__restrict__ inv_perm) {
    extern __shared__ int32_t run[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = blk_base[size_t(blockIdx.x) * E + e];
    __syncthreads();
    const int i = blockIdx.x * PERM_BLOCK + threadIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int e = -1;
    if (i < N) {
        e = ids[i];
        if (e < 0 || e >= E) e = -1;
    }
    const int key = e >= 0 ? e : -1 - lane;  // invalid entries never share a key
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const bool leader = rank == 0;
    for (int w = 0; w < PERM_BLOCK / 32; w++) {
        if (warp == w && e >= 0) {
            const int base = run[e];
            __syncwarp(peers);
            const int pos = base + rank;
            if (leader) run[e] = base + __popc(peers);
            perm_tok[pos] = i / k;
            perm_w[pos] = weights[i];
            inv_perm[i] = pos;
        }
        __syncthreads();
    }
    if (i < N && e < 0) inv_perm[i] = -1;
}

// out[t] = y_shared[t] + sum_j y_perm[inv[t*k+j]], fp32 in slot order.
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ y_perm,
                                                      const int32_t *__restrict__ inv, const float *__restrict__ ys,
                                                      int T, int d, int k, float *__restrict__ out) {
    const int d4 = d / 4;
    const size_t total = size_t(T) * d4;
    for (size_t q = size_t(blockIdx.x) * blockDim.x + threadIdx.x; q < total; q += size_t(gridDim.x) * blockDim.x) {
        const int t = int(q / d4), c = int(q % d4) * 4;
        float4 acc = ys ? *reinterpret_cast<const float4 *>(ys + size_t(t) * d + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; j++) {
            const int p = inv[size_t(t) * k + j];
            if (p < 0) continue;
            const float4 v = *reinterpret_cast<const float4 *>(y_perm + size_t(p) * d + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        *reinterpret_cast<float4 *>(out + size_t(t) * d + c) = acc;
    }
}

}  // namespace ds4
