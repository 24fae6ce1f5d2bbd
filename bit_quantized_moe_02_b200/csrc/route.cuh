// Router: fp16 W_r x bf16 x logits (exact products, fp32 accumulation), then
// sigmoid scores, top-k (descending, ties to the smaller id) and renormalised
// gates.  The pages leave the routing function open beyond "routing is not
// quantized" (ds4 news summary, "model weights"); this is the sigmoid /
// top-k / renormalise gate of the layer definition in include/ds4moe.h.
#pragma once
#include "common.cuh"

namespace ds4 {

// ---- small T (decode): one CTA per pair of experts, 4 warps split K per expert.
constexpr int ROUTE_SMALL_T = 8;

__global__ void __launch_bounds__(256) route_logits_small_kernel(const __nv_bfloat16 *__restrict__ x, int T, int d,
                                                                 const __half *__restrict__ wr,
                                                                 const float *__restrict__ bias, int E,
                                                                 float *__restrict__ logits) {
    __shared__ float part[8][ROUTE_SMALL_T];
    pdl_launch_dependents();  // top-k may launch now; it waits for these logits before reading them
    int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int e = blockIdx.x * 2 + (warp >> 2);
    int q = warp & 3;
    float acc[ROUTE_SMALL_T];
#pragma unroll
    for (int t = 0; t < ROUTE_SMALL_T; t++) acc[t] = 0.f;
    if (e < E) {
        int kq = d / 4;  // multiple of 64
        const __half *row = wr + size_t(e) * d + q * kq;
#pragma unroll 4
        for (int c = lane * 8; c < kq; c += 256) {
            uint4 wv = *reinterpret_cast<const uint4 *>(row + c);
            float wf[8];
            const __half2 *wh = reinterpret_cast<const __half2 *>(&wv);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                float2 f2 = __half22float2(wh[i]);
                wf[2 * i] = f2.x; wf[2 * i + 1] = f2.y;
            }
#pragma unroll
            for (int t = 0; t < ROUTE_SMALL_T; t++) {
                if (t < T) {
                    uint4 xv = *reinterpret_cast<const uint4 *>(x + size_t(t) * d + q * kq + c);
                    const uint32_t *xu = reinterpret_cast<const uint32_t *>(&xv);
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        acc[t] = fmaf(wf[2 * i], bf16_lo(xu[i]), acc[t]);
                        acc[t] = fmaf(wf[2 * i + 1], bf16_hi(xu[i]), acc[t]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < ROUTE_SMALL_T; t++) {
        float v = warp_sum(acc[t]);
        if (lane == 0) part[warp][t] = v;
    }
    __syncthreads();
    int tid = threadIdx.x;
    if (tid < 2 * ROUTE_SMALL_T) {
        int h = tid / ROUTE_SMALL_T, t = tid % ROUTE_SMALL_T;
        int ee = blockIdx.x * 2 + h;
        if (ee < E && t < T) {
            float v = ((part[4 * h][t] + part[4 * h + 1][t]) + part[4 * h + 2][t]) + part[4 * h + 3][t];
            if (bias) v += bias[ee];
            logits[size_t(t) * E + ee] = v;
        }
    }
}

// ---- large T without a tensor-core tiling (E not a multiple of 128): 64 tokens x 64 experts per CTA.
__global__ void __launch_bounds__(256) route_logits_tiled_kernel(const __nv_bfloat16 *__restrict__ x, int T, int d,
                                                                 const __half *__restrict__ wr,
                                                                 const float *__restrict__ bias, int E,
                                                                 float *__restrict__ logits) {
    __shared__ float xs[32][68];
    __shared__ float ws[32][68];
    pdl_launch_dependents();
    int t0 = blockIdx.x * 64, e0 = blockIdx.y * 64;
    int tid = threadIdx.x;
    int tx = tid % 16, ty = tid / 16;  // thread computes tokens ty*4.., experts tx*4..
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; a++)
#pragma unroll
        for (int b = 0; b < 4; b++) acc[a][b] = 0.f;
    for (int k0 = 0; k0 < d; k0 += 32) {
        // load 64 rows x 32 k of x and of wr; each thread: 8 elements of each
        for (int i = tid; i < 64 * 4; i += 256) {
            int r = i / 4, c8 = (i % 4) * 8;
            int t = t0 + r, e = e0 + r;
            uint4 xv = make_uint4(0, 0, 0, 0), wv = make_uint4(0, 0, 0, 0);
            if (t < T) xv = *reinterpret_cast<const uint4 *>(x + size_t(t) * d + k0 + c8);
            if (e < E) wv = *reinterpret_cast<const uint4 *>(wr + size_t(e) * d + k0 + c8);
            const uint32_t *xu = reinterpret_cast<const uint32_t *>(&xv);
            const __half2 *wh = reinterpret_cast<const __half2 *>(&wv);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                xs[c8 + 2 * j][r] = bf16_lo(xu[j]);
                xs[c8 + 2 * j + 1][r] = bf16_hi(xu[j]);
                float2 f2 = __half22float2(wh[j]);
                ws[c8 + 2 * j][r] = f2.x;
                ws[c8 + 2 * j + 1][r] = f2.y;
            }
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; kk++) {
            float4 xa = *reinterpret_cast<const float4 *>(&xs[kk][ty * 4]);
            float4 wb = *reinterpret_cast<const float4 *>(&ws[kk][tx * 4]);
            float xv[4] = {xa.x, xa.y, xa.z, xa.w}, wv[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int a = 0; a < 4; a++)
#pragma unroll
                for (int b = 0; b < 4; b++) acc[a][b] = fmaf(xv[a], wv[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; a++) {
        int t = t0 + ty * 4 + a;
        if (t >= T) continue;
#pragma unroll
        for (int b = 0; b < 4; b++) {
            int e = e0 + tx * 4 + b;
            if (e < E) logits[size_t(t) * E + e] = acc[a][b] + (bias ? bias[e] : 0.f);
        }
    }
}

// ---- top-k: one warp per token, E <= 32 * PER logits spread over the lanes.
// late_bias: added here when the logits kernel did not add it (tensor-core path), else NULL.
// logits is written by the preceding grid and read after griddepcontrol.wait: a plain pointer, not
// const __restrict__ (which would allow non-coherent or hoisted loads).
template <int PER>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *logits, int T, int E, int k,
                                                         const float *__restrict__ late_bias,
                                                         int32_t *__restrict__ ids, float *__restrict__ weights) {
    // launched with programmatic dependent launch: the expert kernels that follow may start their own
    // prologues now, and this grid waits for the logits
    pdl_launch_dependents();
    pdl_wait();
    int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= T) return;
    const float *lg = logits + size_t(warp) * E;
    float v[PER];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < PER; i++)
        v[i] = (lane + 32 * i < E) ? lg[lane + 32 * i] + (late_bias ? late_bias[lane + 32 * i] : 0.f) : -INFINITY;
    uint32_t valid = 0;
#pragma unroll
    for (int i = 0; i < PER; i++)
        if (lane + 32 * i < E) valid |= 1u << i;
    float ssum = 0.f, s_mine = 0.f;
    int id_mine = -1;
    for (int j = 0; j < k; j++) {
        // lane-local best: largest logit, smallest id among equals (ids grow with i)
        float bv = -INFINITY;
        int bid = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PER; i++) {
            bool ok = ((valid & ~taken) >> i) & 1u;
            if (ok && (v[i] > bv || bid == 0x7fffffff)) { bv = v[i]; bid = lane + 32 * i; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oid = __shfl_xor_sync(0xffffffffu, bid, o);
            if (oid != 0x7fffffff && (bid == 0x7fffffff || ov > bv || (ov == bv && oid < bid))) { bv = ov; bid = oid; }
        }
        if (bid != 0x7fffffff && (bid & 31) == lane) taken |= 1u << (bid >> 5);
        float s = 1.f / (1.f + expf(-bv));
        ssum += s;
        if (lane == j) { s_mine = s; id_mine = bid; }
    }
    if (lane < k) {
        ids[size_t(warp) * k + lane] = id_mine;
        weights[size_t(warp) * k + lane] = s_mine / ssum;
    }
}

}  // namespace ds4
