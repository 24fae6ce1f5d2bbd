// Single-token decode, TMA-staged versions for the common shapes (d = 2048 or 4096 gate/up contraction,
// f = 2048 down contraction).
//
// Each warp streams its rows through a private ring of shared-memory slots.  One lane fills a slot with a
// few bulk copies (cp.async.bulk, the TMA engine) of whole contiguous row pieces -- the packed index,
// sign, scale and d planes of a row, or a 1 KB piece of a bf16 shared-expert row -- and arms the slot's
// mbarrier with the byte count; the warp dequantizes the row in the oldest slot while the next
// SLOTS-1 rows are in flight.  Whole-row bulk copies keep the number of memory requests per byte low,
// which is what limits per-lane copies at these rates.  Every mbarrier wait is bounded.
//
// Table lookups take one instruction to address: the tables sit at a 64 KB-aligned shared-memory address,
// one 256-byte row per entry, so __byte_perm splices a packed index byte between the lane's slot offset and
// the table base (slot | index << 8 | base).
//
//  * gate/up: IQ2X codebook table, 256 entries x 16 lane slots x 8 fp16 (64 KB); fp16 sign masks from the
//    prepared sign words; packed fp16 FMAs within a 32-weight group, fp32 across groups.  The shared
//    expert's bf16 rows are ring items too, taken before the grid-dependency wait so they overlap the
//    router.
//  * down: Q2K byte table, 256 entries x 32 lane slots x 4 fp16 (one lookup = 4 weights); h_j staged as
//    scaled fp16 pairs; per row the k routed items and the shared-expert items accumulate in a fixed order
//    (deterministic, no atomics).
#pragma once
#include "common.cuh"
#include "decode.cuh"
#include "grouped_tc.cuh"

namespace ds4 {

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     bar),
                 "r"(bytes)
                 : "memory");
}
// one bulk copy global -> shared, completion counted on `bar` (16-byte aligned addresses, size % 16 == 0)
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Bounded wait of every lane of a warp on a ring slot; false after a timeout (recorded on the device).
__device__ __forceinline__ bool ring_wait(uint32_t bar, uint32_t parity) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = tc::globaltimer();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (tc::globaltimer() - t0 > uint64_t(tc::WAIT_NS)) {
            set_device_error(DS4MOE_ETIMEOUT);
            return false;
        }
    }
    return true;
}

// After a timed-out wait: wait (bounded) for the slots of items [from, to) that were armed but not consumed,
// so no bulk copy lands in shared memory after the CTA has exited.
__device__ __forceinline__ void ring_drain(uint32_t bar0, int nslots, int from, int to) {
    const uint64_t t0 = tc::globaltimer();
    for (int i = from; i < to; i++)
        while (!tc::mbar_try_wait(bar0 + 8 * (i % nslots), uint32_t(i / nslots) & 1u) &&
               tc::globaltimer() - t0 < uint64_t(tc::WAIT_NS)) {
        }
}

// ============================================================================ gate / up

constexpr int GR_THREADS = 384;
constexpr int GR_WARPS = GR_THREADS / 32;
constexpr int GR_SLOTS = 4;
constexpr int GR_SLOT_BYTES = 2304;              // a gate/up row pair (2 x 1152 B at d = 4096) or a shared chunk (2 KB)
constexpr uint32_t GR_TABLE_ABS = 0x20000;       // absolute shared address of the codebook table
constexpr int GR_DYN = int(GR_TABLE_ABS) + 65536 + 16384;  // + fp32 copy of x (d <= 4096)

template <int VPL>  // 8-vectors per lane: 8 (d = 2048) or 16 (d = 4096)
__global__ void __launch_bounds__(GR_THREADS, 1)
    decode_gateup_ring_kernel(ExpertsDev ex, const __nv_bfloat16 *__restrict__ x, const int32_t *__restrict__ ids,
                              int k, float *__restrict__ h_out, float *__restrict__ sh_part) {
    static_assert(VPL == 8 || VPL == 16, "ring kernel covers d = 2048 and 4096");
    constexpr int D = VPL * 256;
    constexpr int IDXB = D / 8, SGNB = D / 8, SCLB = D / 64, DB = D / 128;  // bytes per row per plane
    constexpr int ROWB = ((IDXB + SGNB + SCLB + DB + 127) / 128) * 128;
    static_assert(2 * ROWB <= GR_SLOT_BYTES, "slot too small");
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[GR_WARPS * GR_SLOTS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t sbase = smem_u32(smem);
    uint8_t *tbl = smem + (GR_TABLE_ABS - sbase);
    float4 *xsh = reinterpret_cast<float4 *>(tbl + 65536);
    uint8_t *ring = smem + warp * (GR_SLOTS * GR_SLOT_BYTES);
    const uint32_t ring_s = sbase + warp * (GR_SLOTS * GR_SLOT_BYTES);
    const uint32_t bar0 = smem_u32(&bars[warp * GR_SLOTS]);

    if (lane == 0)
        for (int s = 0; s < GR_SLOTS; s++) tc::mbar_init(bar0 + 8 * s, 1);
    // codebook table: entry e, lane slot s at GR_TABLE_ABS + e*256 + s*16 (8 fp16); one entry per thread
    if (threadIdx.x < 256) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(ex.codebook + threadIdx.x * 8);
        const uint32_t b[2] = {raw.x, raw.y};
        __half2 hv[4];
#pragma unroll
        for (int p = 0; p < 4; p++)
            hv[p] = __floats2half2_rn(float((b[p >> 1] >> (16 * (p & 1))) & 0xFF),
                                      float((b[p >> 1] >> (16 * (p & 1) + 8)) & 0xFF));
        const uint4 v = *reinterpret_cast<uint4 *>(hv);
#pragma unroll
        for (int s = 0; s < 16; s++) *reinterpret_cast<uint4 *>(tbl + threadIdx.x * 256 + s * 16) = v;
    }
    // activations: every warp loads the lane slices of x (128-bit loads), takes the max over the warp, and
    // keeps its slice as scaled fp16 pairs; warp 0 also writes the fp32 copy the shared-expert items use.
    uint4 raw[VPL];
#pragma unroll
    for (int v = 0; v < VPL; v++) raw[v] = *reinterpret_cast<const uint4 *>(x + size_t(lane * VPL + v) * 8);
    // shared-expert chunks: lane covers EL = 16 consecutive elements of a CS = 512 element chunk;
    // element c*CS + l*EL + 4i + q sits at float4 slot (c*4 + i)*32 + l, component q
    constexpr int EL = 16, CS = 512;
    constexpr int nch = D / CS;
    if (warp == 0) {
#pragma unroll
        for (int v = 0; v < VPL; v++) {
            const int e0 = lane * VPL * 8 + v * 8;  // 8 elements e0 .. e0+7
            const int c = e0 / CS, l = (e0 % CS) / EL, i = (e0 % EL) / 4;
            xsh[(c * 4 + i) * 32 + l] = make_float4(bf16_lo(raw[v].x), bf16_hi(raw[v].x), bf16_lo(raw[v].y), bf16_hi(raw[v].y));
            xsh[(c * 4 + i + 1) * 32 + l] =
                make_float4(bf16_lo(raw[v].z), bf16_hi(raw[v].z), bf16_lo(raw[v].w), bf16_hi(raw[v].w));
        }
    }
    float m = 0.f;
#pragma unroll
    for (int v = 0; v < VPL; v++) {
        const uint32_t rw[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
#pragma unroll
        for (int i = 0; i < 4; i++) m = fmaxf(m, fmaxf(fabsf(bf16_lo(rw[i])), fabsf(bf16_hi(rw[i]))));
    }
    const int xe = pow2_exponent_for(warp_max(m), 6);
    const float xs = ldexpf(1.f, xe), inv_xs = ldexpf(1.f, -xe);
    uint32_t xh[VPL][4];
#pragma unroll
    for (int v = 0; v < VPL; v++) {
        const uint32_t rw[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
#pragma unroll
        for (int i = 0; i < 4; i++) xh[v][i] = half2_as_u32(__floats2half2_rn(bf16_lo(rw[i]) * xs, bf16_hi(rw[i]) * xs));
    }
    tc::fence_mbar_init();
    __syncthreads();

    const int nwt = gridDim.x * GR_WARPS, gw = blockIdx.x * GR_WARPS + warp;
    const int n_sh = ex.fs > 0 ? ex.fs * nch : 0;
    const int n_rt = k * ex.f;
    const int ns_w = n_sh > gw ? (n_sh - gw + nwt - 1) / nwt : 0;
    const int nr_w = n_rt > gw ? (n_rt - gw + nwt - 1) / nwt : 0;
    const int n_w = ns_w + nr_w;
    constexpr int nsb = D / QK;
    const uint32_t lane_tbl = GR_TABLE_ABS | uint32_t((lane & 15) * 16);
    bool waited = false;

    // lane 0 fills the slot of item i (one use of its barrier per fill)
    auto issue = [&](int i) {
        const int slot = i % GR_SLOTS;
        const uint32_t sd = ring_s + slot * GR_SLOT_BYTES, bar = bar0 + 8 * slot;
        if (i < ns_w) {
            const int s = gw + i * nwt;
            const size_t off = size_t(s / nch) * D + size_t(s % nch) * CS;
            mbar_arrive_tx(bar, 2048);
            bulk_g2s(sd, ex.sh_gate + off, 1024, bar);
            bulk_g2s(sd + 1024, ex.sh_up + off, 1024, bar);
            return;
        }
        const int q = gw + (i - ns_w) * nwt;
        const int j = q / ex.f, r = q % ex.f;
        const int e = ids[j];
        if (e < 0 || e >= ex.E) {
            set_device_error(DS4MOE_EDEVICE);
            mbar_arrive_tx(bar, 0);  // completes the phase with nothing to copy
            return;
        }
        mbar_arrive_tx(bar, 2 * (IDXB + SGNB + SCLB + DB));
#pragma unroll
        for (int mm = 0; mm < 2; mm++) {
            const uint8_t *mat = mm ? ex.up + size_t(e) * ex.up_stride : ex.gate + size_t(e) * ex.gate_stride;
            const uint32_t rd = sd + mm * ROWB;
            bulk_g2s(rd, mat + ex.pg.off[0] + size_t(r) * IDXB, IDXB, bar);
            bulk_g2s(rd + IDXB, mat + ex.pg.off[1] + size_t(r) * SGNB, SGNB, bar);
            bulk_g2s(rd + IDXB + SGNB, mat + ex.pg.off[2] + size_t(r) * SCLB, SCLB, bar);
            bulk_g2s(rd + IDXB + SGNB + SCLB, mat + ex.pg.off[3] + size_t(r) * DB, DB, bar);
        }
    };

    // one IQ2X row from a slot: this lane's VPL vectors, dotted with its activations
    auto row_dot = [&](const uint8_t *rs) -> float {
        constexpr uint32_t M = 0x80008000u;
        constexpr int NG = VPL / 4;
        uint32_t idx[NG], sgn[NG];
        if constexpr (VPL == 16) {
            const uint4 a = *reinterpret_cast<const uint4 *>(rs + lane * 16);
            const uint4 b = *reinterpret_cast<const uint4 *>(rs + IDXB + lane * 16);
            idx[0] = a.x; idx[1] = a.y; idx[2] = a.z; idx[3] = a.w;
            sgn[0] = b.x; sgn[1] = b.y; sgn[2] = b.z; sgn[3] = b.w;
        } else {
            const uint2 a = *reinterpret_cast<const uint2 *>(rs + lane * 8);
            const uint2 b = *reinterpret_cast<const uint2 *>(rs + IDXB + lane * 8);
            idx[0] = a.x; idx[1] = a.y;
            sgn[0] = b.x; sgn[1] = b.y;
        }
        const int sbi = (lane * VPL) / 32;
        const uint32_t scl = *reinterpret_cast<const uint32_t *>(rs + IDXB + SGNB + sbi * 4);
        const uint16_t dbits = *reinterpret_cast<const uint16_t *>(rs + IDXB + SGNB + SCLB + sbi * 2);
        const float dv = half_bits_to_float(dbits);
        const float dv4 = dv * 0.25f, dv8 = dv * 0.125f;
        const int g0 = ((lane * VPL) / 4) % 8;
        float acc = 0.f;
#pragma unroll
        for (int gi = 0; gi < NG; gi++) {
            const uint32_t W = sgn[gi];
            const float Dg = fmaf(float((scl >> (4 * (g0 + gi))) & 15u), dv4, dv8);  // d * (0.5 + s) / 4, exact
            __half2 a0 = __float2half2_rn(0.f), a1 = __float2half2_rn(0.f);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int v = gi * 4 + j;
                const uint4 cb = lds128(__byte_perm(idx[gi], lane_tbl, 0x7604 | (j << 4)));
                const uint32_t Wj = W << (4 * j);
                a0 = __hfma2(u32_as_half2(cb.x ^ (Wj & M)), u32_as_half2(xh[v][0]), a0);
                a1 = __hfma2(u32_as_half2(cb.y ^ ((Wj << 1) & M)), u32_as_half2(xh[v][1]), a1);
                a0 = __hfma2(u32_as_half2(cb.z ^ ((Wj << 2) & M)), u32_as_half2(xh[v][2]), a0);
                a1 = __hfma2(u32_as_half2(cb.w ^ ((Wj << 3) & M)), u32_as_half2(xh[v][3]), a1);
            }
            const float2 f = __half22float2(__hadd2(a0, a1));
            acc = fmaf(Dg, f.x + f.y, acc);
        }
        return acc;
    };

    // Items of this warp: its shared-expert chunks, then (after the grid dependency) its routed row pairs.
    auto item_valid = [&](int i) -> bool {  // same answer on every lane
        if (i < ns_w) return true;
        const int e = ids[(gw + (i - ns_w) * nwt) / ex.f];
        return e >= 0 && e < ex.E;
    };
    int issued = 0, i = 0;
    for (; issued < GR_SLOTS - 1 && issued < n_w; issued++) {
        if (issued >= ns_w && !waited) {
            pdl_wait();
            waited = true;
        }
        if (lane == 0) issue(issued);
    }
    for (; i < n_w; i++) {
        const int nxt = i + GR_SLOTS - 1;
        if (nxt < n_w) {
            if (nxt >= ns_w && !waited) {
                pdl_wait();
                waited = true;
            }
            __syncwarp();  // every lane is done with the slot about to be refilled
            if (lane == 0) {
                tc::fence_proxy_async();
                issue(nxt);
            }
            issued = nxt + 1;
        }
        const int slot = i % GR_SLOTS;
        if (!ring_wait(bar0 + 8 * slot, uint32_t(i / GR_SLOTS) & 1u)) break;
        const uint8_t *sl = ring + slot * GR_SLOT_BYTES;
        if (i < ns_w) {
            const int s = gw + i * nwt;
            const int r = s / nch, c = s % nch;
            const uint4 g0 = *reinterpret_cast<const uint4 *>(sl + lane * 32);
            const uint4 g1 = *reinterpret_cast<const uint4 *>(sl + lane * 32 + 16);
            const uint4 u0 = *reinterpret_cast<const uint4 *>(sl + 1024 + lane * 32);
            const uint4 u1 = *reinterpret_cast<const uint4 *>(sl + 1024 + lane * 32 + 16);
            const uint32_t gwv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const uint32_t uwv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            float ag = 0.f, au = 0.f;
#pragma unroll
            for (int t = 0; t < 4; t++) {
                const float4 xv = xsh[(c * 4 + t) * 32 + lane];
                ag = fmaf(bf16_lo(gwv[2 * t]), xv.x, ag);
                ag = fmaf(bf16_hi(gwv[2 * t]), xv.y, ag);
                ag = fmaf(bf16_lo(gwv[2 * t + 1]), xv.z, ag);
                ag = fmaf(bf16_hi(gwv[2 * t + 1]), xv.w, ag);
                au = fmaf(bf16_lo(uwv[2 * t]), xv.x, au);
                au = fmaf(bf16_hi(uwv[2 * t]), xv.y, au);
                au = fmaf(bf16_lo(uwv[2 * t + 1]), xv.z, au);
                au = fmaf(bf16_hi(uwv[2 * t + 1]), xv.w, au);
            }
            ag = warp_sum(ag);
            au = warp_sum(au);
            if (lane == 0) {
                sh_part[size_t(2 * c) * ex.fs + r] = ag;
                sh_part[size_t(2 * c + 1) * ex.fs + r] = au;
            }
        } else if (item_valid(i)) {
            const int q = gw + (i - ns_w) * nwt;
            float ag = row_dot(sl);
            float au = row_dot(sl + ROWB);
            ag = warp_sum(ag);
            au = warp_sum(au);
            if (lane == 0) {
                const float g = ag * inv_xs, u = au * inv_xs;
                h_out[q] = silu(g) * u;  // q = j * f + r
            }
        }
    }
    if (i < n_w) ring_drain(bar0, GR_SLOTS, i, issued);  // a wait timed out
}

// ============================================================================ down + combine

constexpr int DR_THREADS = 256;
constexpr int DR_WARPS = DR_THREADS / 32;
constexpr int DR_SLOTS = 7;
constexpr int DR_SLOT_BYTES = 1024;
constexpr uint32_t DR_TABLE_ABS = 0x10000;
constexpr int DR_WPL = 4;  // f = 2048: 4 Q2K sub-blocks (16 weights each) per lane

struct DownRingSmem {
    int hq, hsum, hsl, wsc, eid, hmax, total;  // offsets from the table base (= DR_TABLE_ABS - smem start)
};
__host__ __device__ __forceinline__ DownRingSmem down_ring_layout(int k, int fs) {
    DownRingSmem s;
    s.hq = 65536;                                // k * 4 * 2 * 32 uint4
    s.hsum = s.hq + k * DR_WPL * 2 * 32 * 16;    // k * 4 * 32 floats
    s.hsl = s.hsum + k * DR_WPL * 32 * 4;        // fs floats
    s.wsc = s.hsl + ((fs * 4 + 15) / 16) * 16;
    s.eid = s.wsc + ((k * 4 + 15) / 16) * 16;
    s.hmax = s.eid + ((k * 4 + 15) / 16) * 16;
    s.total = int(DR_TABLE_ABS) + s.hmax + ((k * 4 + 15) / 16) * 16;  // dynamic bytes to request
    return s;
}

__global__ void __launch_bounds__(DR_THREADS, 1)
    decode_down_ring_kernel(ExpertsDev ex, const float *__restrict__ h, const float *__restrict__ sh_part, int nchp,
                            const int32_t *__restrict__ ids, const float *__restrict__ wts, int k,
                            float *__restrict__ out) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[DR_WARPS * DR_SLOTS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int f = ex.f, fs = ex.fs, d = ex.d;
    const uint32_t sbase = smem_u32(smem);
    uint8_t *tb = smem + (DR_TABLE_ABS - sbase);  // table, then the staged activations
    const DownRingSmem L = down_ring_layout(k, fs);
    uint4 *hq = reinterpret_cast<uint4 *>(tb + L.hq);
    float *hsum = reinterpret_cast<float *>(tb + L.hsum);
    float *hsl = reinterpret_cast<float *>(tb + L.hsl);
    float *wsc = reinterpret_cast<float *>(tb + L.wsc);
    int *eid = reinterpret_cast<int *>(tb + L.eid);
    int *hmax = reinterpret_cast<int *>(tb + L.hmax);
    uint8_t *ring = smem + warp * (DR_SLOTS * DR_SLOT_BYTES);
    const uint32_t ring_s = sbase + warp * (DR_SLOTS * DR_SLOT_BYTES);
    const uint32_t bar0 = smem_u32(&bars[warp * DR_SLOTS]);

    if (lane == 0)
        for (int s = 0; s < DR_SLOTS; s++) tc::mbar_init(bar0 + 8 * s, 1);
    // byte -> 4 fp16 table: entry b (weights q_i = (b >> 2i) & 3), lane slot s at DR_TABLE_ABS + b*256 + s*8
    for (int i = threadIdx.x; i < 256 * 32; i += DR_THREADS) {
        const int b = i >> 5;
        const __half2 lo = __floats2half2_rn(float(b & 3), float((b >> 2) & 3));
        const __half2 hi = __floats2half2_rn(float((b >> 4) & 3), float((b >> 6) & 3));
        *reinterpret_cast<uint2 *>(tb + b * 256 + (i & 31) * 8) = make_uint2(half2_as_u32(lo), half2_as_u32(hi));
    }
    for (int j = threadIdx.x; j < k; j += DR_THREADS) hmax[j] = 0;
    tc::fence_mbar_init();

    pdl_wait();
    __syncthreads();
    // stage h_j: per 16-float sub-block, max |h| per expert, then scaled fp16 pairs (h[16s+2p], h[16s+2p+1]) of
    // sub-block s at lane s / 4, slot s % 4.  Sub-blocks are taken four per thread with all loads in flight.
    const int nsub = f / 16;
    const int ntot = k * nsub;
    constexpr int SB = 4;
    for (int q0 = threadIdx.x * SB; q0 < ntot; q0 += DR_THREADS * SB) {
        float4 v[SB][4];
#pragma unroll
        for (int u = 0; u < SB; u++)
#pragma unroll
            for (int t = 0; t < 4; t++)
                v[u][t] = q0 + u < ntot ? reinterpret_cast<const float4 *>(h + size_t(q0 + u) * 16)[t]
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < SB; u++) {
            if (q0 + u >= ntot) break;
            float m = 0.f;
#pragma unroll
            for (int t = 0; t < 4; t++)
                m = fmaxf(m, fmaxf(fmaxf(fabsf(v[u][t].x), fabsf(v[u][t].y)), fmaxf(fabsf(v[u][t].z), fabsf(v[u][t].w))));
            atomicMax(&hmax[(q0 + u) / nsub], __float_as_int(m));
        }
    }
    // shared expert: hs = silu(sum_c g_c) * sum_c u_c; element r at item r / 512, lane (r % 512) / 16,
    // float4 slot ((r / 512) * 4 + (r % 16) / 4) * 32 + lane
    for (int r4 = threadIdx.x * 4; r4 < fs; r4 += DR_THREADS * 4) {
        float4 gc[16], uc[16];
#pragma unroll
        for (int c = 0; c < 16; c++)
            if (c < nchp) {
                gc[c] = *reinterpret_cast<const float4 *>(sh_part + size_t(2 * c) * fs + r4);
                uc[c] = *reinterpret_cast<const float4 *>(sh_part + size_t(2 * c + 1) * fs + r4);
            }
        float4 g = make_float4(0.f, 0.f, 0.f, 0.f), u = g;
#pragma unroll
        for (int c = 0; c < 16; c++)
            if (c < nchp) {
                g.x += gc[c].x; g.y += gc[c].y; g.z += gc[c].z; g.w += gc[c].w;
                u.x += uc[c].x; u.y += uc[c].y; u.z += uc[c].z; u.w += uc[c].w;
            }
        const int c = r4 / 512, ln = (r4 % 512) / 16, t = (r4 % 16) / 4;
        reinterpret_cast<float4 *>(hsl)[(c * 4 + t) * 32 + ln] =
            make_float4(silu(g.x) * u.x, silu(g.y) * u.y, silu(g.z) * u.z, silu(g.w) * u.w);
    }
    __syncthreads();
    for (int q0 = threadIdx.x * SB; q0 < ntot; q0 += DR_THREADS * SB) {
        float4 v[SB][4];
#pragma unroll
        for (int u = 0; u < SB; u++)
#pragma unroll
            for (int t = 0; t < 4; t++)
                v[u][t] = q0 + u < ntot ? reinterpret_cast<const float4 *>(h + size_t(q0 + u) * 16)[t]
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < SB; u++) {
            const int q = q0 + u;
            if (q >= ntot) break;
            const int j = q / nsub, sbk = q % nsub;
            const int ln = sbk / DR_WPL, i = sbk % DR_WPL;
            const float sc = ldexpf(1.f, pow2_exponent_for(__int_as_float(hmax[j]), 6));
            __half2 pr[8];
            float ssum = 0.f;
#pragma unroll
            for (int t = 0; t < 4; t++) {
                pr[2 * t] = __floats2half2_rn(v[u][t].x * sc, v[u][t].y * sc);
                pr[2 * t + 1] = __floats2half2_rn(v[u][t].z * sc, v[u][t].w * sc);
                const float2 b0 = __half22float2(pr[2 * t]), b1 = __half22float2(pr[2 * t + 1]);
                ssum += (b0.x + b0.y) + (b1.x + b1.y);
            }
            hq[((j * DR_WPL + i) * 2 + 0) * 32 + ln] = *reinterpret_cast<uint4 *>(&pr[0]);
            hq[((j * DR_WPL + i) * 2 + 1) * 32 + ln] = *reinterpret_cast<uint4 *>(&pr[4]);
            hsum[(j * DR_WPL + i) * 32 + ln] = ssum;
        }
    }
    for (int j = threadIdx.x; j < k; j += DR_THREADS) {
        wsc[j] = wts[j] * ldexpf(1.f, -pow2_exponent_for(__int_as_float(hmax[j]), 6));
        eid[j] = ids[j];
    }
    __syncthreads();

    // items: for each of this warp's rows, k routed rows then NSH shared-expert pieces of 512 elements
    const int rpc = (d + gridDim.x - 1) / gridDim.x;
    const int n0 = blockIdx.x * rpc, n1 = min(d, n0 + rpc);
    const int nrows_w = n1 - (n0 + warp) > 0 ? (n1 - (n0 + warp) + DR_WARPS - 1) / DR_WARPS : 0;
    const int nsh = fs / 512;
    const int ipr = k + nsh;
    const int n_w = nrows_w * ipr;
    const int nsbf = f / QK;
    const uint32_t lane_tbl = DR_TABLE_ABS | uint32_t(lane * 8);

    auto issue = [&](int i) {  // lane 0
        const int n = n0 + warp + (i / ipr) * DR_WARPS;
        const int it = i % ipr;
        const uint32_t sd = ring_s + (i % DR_SLOTS) * DR_SLOT_BYTES, bar = bar0 + 8 * (i % DR_SLOTS);
        if (it < k) {
            const int e = eid[it];
            if (e < 0 || e >= ex.E) {
                mbar_arrive_tx(bar, 0);
                return;
            }
            const uint8_t *base = ex.down + size_t(e) * ex.down_stride;
            mbar_arrive_tx(bar, 512 + 128 + 32);
            bulk_g2s(sd, base + ex.pd.off[0] + size_t(n) * nsbf * 64, 512, bar);
            bulk_g2s(sd + 512, base + ex.pd.off[1] + size_t(n) * nsbf * 16, 128, bar);
            bulk_g2s(sd + 640, base + ex.pd.off[2] + size_t(n) * nsbf * 4, 32, bar);
        } else {
            mbar_arrive_tx(bar, 1024);
            bulk_g2s(sd, ex.sh_down + size_t(n) * fs + (it - k) * 512, 1024, bar);
        }
    };

    int issued = n_w < DR_SLOTS - 1 ? n_w : DR_SLOTS - 1, i = 0;
    if (lane == 0)
        for (int p = 0; p < issued; p++) issue(p);
    float acc = 0.f;
    for (; i < n_w; i++) {
        const int nxt = i + DR_SLOTS - 1;
        if (nxt < n_w) {
            __syncwarp();
            if (lane == 0) {
                tc::fence_proxy_async();
                issue(nxt);
            }
            issued = nxt + 1;
        }
        const int slot = i % DR_SLOTS;
        if (!ring_wait(bar0 + 8 * slot, uint32_t(i / DR_SLOTS) & 1u)) break;
        const uint8_t *sl = ring + slot * DR_SLOT_BYTES;
        const int it = i % ipr;
        if (it < k) {
            const int e = eid[it];
            if (e >= 0 && e < ex.E) {
                const uint4 qv = *reinterpret_cast<const uint4 *>(sl + lane * 16);
                const uint32_t scw = *reinterpret_cast<const uint32_t *>(sl + 512 + lane * 4);
                const uint32_t dm = *reinterpret_cast<const uint32_t *>(sl + 640 + (lane / 4) * 4);
                const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                const float dd = half_bits_to_float(uint16_t(dm & 0xFFFF));
                const float dmin = half_bits_to_float(uint16_t(dm >> 16));
                float part = 0.f;
#pragma unroll
                for (int w = 0; w < DR_WPL; w++) {
                    const uint4 hA = hq[((it * DR_WPL + w) * 2 + 0) * 32 + lane];
                    const uint4 hB = hq[((it * DR_WPL + w) * 2 + 1) * 32 + lane];
                    const uint32_t hp[8] = {hA.x, hA.y, hA.z, hA.w, hB.x, hB.y, hB.z, hB.w};
                    __half2 a2 = __float2half2_rn(0.f), b2 = __float2half2_rn(0.f);
#pragma unroll
                    for (int b = 0; b < 4; b++) {
                        const uint2 qq = lds64(__byte_perm(qw[w], lane_tbl, 0x7604 | (b << 4)));
                        a2 = __hfma2(u32_as_half2(qq.x), u32_as_half2(hp[2 * b]), a2);
                        b2 = __hfma2(u32_as_half2(qq.y), u32_as_half2(hp[2 * b + 1]), b2);
                    }
                    const float2 fs2 = __half22float2(__hadd2(a2, b2));
                    const uint32_t scb = (scw >> (8 * w)) & 0xFFu;
                    part += (dd * float(scb & 15u)) * (fs2.x + fs2.y) -
                            (dmin * float(scb >> 4)) * hsum[(it * DR_WPL + w) * 32 + lane];
                }
                acc = fmaf(wsc[it], part, acc);
            } else if (lane == 0) {
                set_device_error(DS4MOE_EDEVICE);
            }
        } else {
            const uint4 w0 = *reinterpret_cast<const uint4 *>(sl + lane * 32);
            const uint4 w1 = *reinterpret_cast<const uint4 *>(sl + lane * 32 + 16);
            const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            const float4 *h4 = reinterpret_cast<const float4 *>(hsl);
            const int c = it - k;
#pragma unroll
            for (int t = 0; t < 4; t++) {
                const float4 hv = h4[(c * 4 + t) * 32 + lane];
                acc = fmaf(bf16_lo(wv[2 * t]), hv.x, acc);
                acc = fmaf(bf16_hi(wv[2 * t]), hv.y, acc);
                acc = fmaf(bf16_lo(wv[2 * t + 1]), hv.z, acc);
                acc = fmaf(bf16_hi(wv[2 * t + 1]), hv.w, acc);
            }
        }
        if (it == ipr - 1) {
            const float tot = warp_sum(acc);
            if (lane == 0) out[n0 + warp + (i / ipr) * DR_WARPS] = tot;
            acc = 0.f;
        }
    }
    if (i < n_w) ring_drain(bar0, DR_SLOTS, i, issued);  // a wait timed out
}

}  // namespace ds4
