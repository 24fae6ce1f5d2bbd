// Single-token decode: GEMV over the k selected experts' packed rows and the
// shared expert's bf16 rows, SwiGLU, and the weighted combine, in two kernels
// (gate/up, then down + combine), each one persistent CTA of 16 warps per SM.
//
// Work is cut into warp-sized units of a few rows (8 gate/up row pairs, or 2
// output rows of the down projection over all k experts).  The 32 lanes of a
// warp split the contraction dimension: in each pass every lane owns a fixed
// slice, holds that slice of the activations in registers (loaded once per
// pass from shared memory) and walks the unit's rows, so consecutive lanes read
// consecutive bytes of a row's packed planes (coalesced) and the only shared-
// memory stream per weight is the dequantization table.  The packed data of
// the next few rows is kept in flight in a small register ring.  A unit ends
// with one butterfly reduce-scatter of its row sums over the 32 lanes: no
// partial sums leave the SM and the summation order is fixed.
//
//  * gate/up (IQ2X): codebook table in shared memory with 16 lane slots per
//    entry (128-bit lookups without bank conflicts, addressed with one byte
//    permute); signs XORed onto the fp16 sign bits; packed fp16 FMAs inside a
//    32-weight group (one scale), fp32 across groups; the row's first lane
//    writes h_j = silu(g) * u.  Shared-expert row pairs are units as well (one
//    row pair each for IQ2X, so the bf16 rows spread over all warps) and run
//    before the grid-dependency wait (they need neither ids nor the router).
//  * down (Q2K): byte -> 4 x fp16 table (32 lane slots); h_j staged per expert
//    as fp16 scaled by a power of two, with sums of every 8 staged values for
//    the min term; a unit is 2 output rows over all k experts and the shared
//    expert, accumulated as out[r] = sum_j w_j (D_j h_j)[r] + (Ds hs)[r].
//
// Both kernels are launched with programmatic dependent launch and may start
// while the preceding grid still runs: inputs that grid writes (ids, routing
// weights, h) are read only after griddepcontrol.wait, through plain pointers
// (never const __restrict__, which would let the compiler treat them as
// read-only for the kernel's lifetime: non-coherent loads, or loads hoisted
// above the wait).
//
// The method (routed experts quantized, IQ2_XXS-style gate/up, Q2_K-style
// down, shared expert unquantized) is the ds4 news summary's "model weights"
// section; the kernel design is this library's own.
#pragma once
#include "common.cuh"
#include "grouped_common.cuh"  // q4k_field

#include <type_traits>

namespace ds4 {

struct ExpertsDev {
    int d, f, E, fs;
    int fmt_gate, fmt_down;
    const uint8_t *gate, *up, *down;
    uint64_t gate_stride, up_stride, down_stride;
    const uint8_t *codebook;
    const __nv_bfloat16 *sh_gate, *sh_up, *sh_down;
    Planes pg;  // planes of one gate/up matrix [f x d]
    Planes pd;  // planes of one down matrix [d x f]
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 ldg_nc_v2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ldg_nc_u16(const void *p) {
    unsigned short r;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ldg_nc_u8(const void *p) {
    unsigned short r;
    asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(r) : "l"(p));
    return r & 0xFFu;
}

// Fire-and-forget bulk prefetch of [p, p + bytes) into L2 (16-byte aligned address and size).  A warp issues
// these for its next unit, so the bytes in flight are not limited by the registers that hold loaded data.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}


// Staged activations are stored in 16-byte chunks at swizzled positions: chunk c at c ^ ((c >> 3) & 7).  A lane
// that reads its slice of 1, 2, 4 or 8 consecutive chunks (lane stride 16 to 128 bytes) then meets no bank
// conflict within a quarter-warp.
__host__ __device__ __forceinline__ int swz16(int c) { return c ^ ((c >> 3) & 7); }

// Butterfly reduce-scatter over the 32 lanes of N per-lane partial sums (N a power of two <= 16): afterwards the
// 32 / N lanes lane = v * (32 / N) + i (i < 32 / N) all hold the full sum of value v.
template <int N>
__device__ __forceinline__ float reduce_scatter(float (&v)[N], int lane) {
#pragma unroll
    for (int n = N / 2, o = 16; n >= 1; n >>= 1, o >>= 1) {
        const bool hi = lane & o;
#pragma unroll
        for (int i = 0; i < n; i++) {
            const float send = hi ? v[i] : v[i + n], keep = hi ? v[i + n] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float r = v[0];
#pragma unroll
    for (int o = 16 / N; o >= 1; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
    return r;
}

// ============================================================================ gate / up

constexpr int DG_WARPS = 16;
constexpr int DG_THREADS = DG_WARPS * 32;
constexpr uint32_t DG_TABLE_ABS = 0x10000;  // absolute shared address of the 64 KB codebook table
constexpr int DG_ROWS = 4;                  // gate/up row pairs per unit (routed and shared): 4 or 8
constexpr int DG_MAX_D = 8192;
// Row slices whose packed data is in flight per lane (divides 2 DG_ROWS): all eight row-matrices of a unit for
// IQ2X (its slices are 22 bytes a lane); four for Q4K, whose larger slices would otherwise spill at 128 registers.
template <int FMT>
__host__ __device__ constexpr int dg_ring() { return FMT == DS4MOE_FMT_Q4K ? 4 : 8; }

// Contraction lengths the gate/up kernel takes: d = 256 * nblk with nblk in {1, 2, 4, 8, 16, 32}.  A lane owns
// VPP = min(nblk, 8) consecutive 8-vectors of a row per pass; nblk / VPP passes.
__host__ __device__ __forceinline__ bool dg_supported_d(int d) {
    const int nblk = d / QK;
    return d % QK == 0 && nblk >= 1 && nblk <= 32 && (nblk & (nblk - 1)) == 0;
}
// dynamic shared memory: everything up to the table's end, then x as fp16 (2d bytes) and fp32 (4d bytes) and the
// sums of every 8 fp16 activations (d / 2 bytes, Q4K rows only)
__host__ __device__ __forceinline__ int dg_smem_bytes(int d) { return int(DG_TABLE_ABS) + 65536 + d * 6 + d / 2; }

template <int VPP>
struct IqRp {  // a lane's slice of one IQ2X row in one pass: VPP 8-vectors
    static constexpr int NW = (VPP + 3) / 4;
    uint32_t idx[NW];  // codebook indices, one byte per vector
    uint32_t sgn[NW];  // sign words of the groups the slice touches
    uint32_t scl, d;   // the block's 4-bit group scales and fp16 scale
};

// v0: first vector of the slice within the row (a multiple of VPP)
template <int VPP>
__device__ __forceinline__ void iq_rp_load(IqRp<VPP> &R, const uint8_t *W, const Planes &P, size_t row, int nblk,
                                           int v0) {
    const size_t rb = row * size_t(nblk) * 32;  // bytes of one row in the index and sign planes
    const uint8_t *ip = W + P.off[0] + rb + v0;
    const uint8_t *sp = W + P.off[1] + rb + (v0 & ~3);
    if constexpr (VPP == 8) {
        const uint2 a = ldg_nc_v2(ip), b = ldg_nc_v2(sp);
        R.idx[0] = a.x; R.idx[1] = a.y; R.sgn[0] = b.x; R.sgn[1] = b.y;
    } else {
        R.idx[0] = VPP == 4 ? ldg_nc_u32(ip) : VPP == 2 ? ldg_nc_u16(ip) : ldg_nc_u8(ip);
        R.sgn[0] = ldg_nc_u32(sp);
    }
    const size_t blk = row * size_t(nblk) + v0 / 32;
    R.scl = ldg_nc_u32(W + P.off[2] + blk * 4);
    R.d = ldg_nc_u16(W + P.off[3] + blk * 2);
}

// Dot product of a lane's row slice with its activations xr (fp16 pairs, VPP vectors).  Group g of a block
// (vectors 4g..4g+3) has weights (d * (0.5 + s_g) / 4) * grid * sign; fp16 FMAs inside a group, fp32 across.
template <int VPP>
__device__ __forceinline__ float iq_rp_dot(const IqRp<VPP> &R, const uint4 (&xr)[VPP], int v0, uint32_t lane_tbl) {
    constexpr uint32_t M = 0x80008000u;
    constexpr int NG = VPP >= 4 ? VPP / 4 : 1, VG = VPP >= 4 ? 4 : VPP;
    const int pos0 = v0 & 3;          // position of the first vector inside its group (0 when VPP >= 4)
    const int g0 = (v0 >> 2) & 7;     // group of the first vector inside its block
    const float dv = half_bits_to_float(uint16_t(R.d));
    const float d4 = dv * 0.25f, d8 = dv * 0.125f;
    float acc = 0.f;
#pragma unroll
    for (int g = 0; g < NG; g++) {
        const uint32_t W = R.sgn[g];
        __half2 a0 = __float2half2_rn(0.f), a1 = a0;
#pragma unroll
        for (int j = 0; j < VG; j++) {
            const int v = g * 4 + j;
            const uint4 cb = lds128(__byte_perm(R.idx[v >> 2], lane_tbl, 0x7604 | ((v & 3) << 4)));
            const uint32_t Wj = W << (4 * (pos0 + j));
            a0 = __hfma2(u32_as_half2(cb.x ^ (Wj & M)), u32_as_half2(xr[v].x), a0);
            a1 = __hfma2(u32_as_half2(cb.y ^ ((Wj << 1) & M)), u32_as_half2(xr[v].y), a1);
            a0 = __hfma2(u32_as_half2(cb.z ^ ((Wj << 2) & M)), u32_as_half2(xr[v].z), a0);
            a1 = __hfma2(u32_as_half2(cb.w ^ ((Wj << 3) & M)), u32_as_half2(xr[v].w), a1);
        }
        const float Dg = fmaf(float((R.scl >> (4 * (g0 + g))) & 15u), d4, d8);  // d * (0.5 + s) / 4, exact
        const float2 fa = __half22float2(__hadd2(a0, a1));
        acc = fmaf(Dg, fa.x + fa.y, acc);
    }
    return acc;
}


// Q4K rows (gate/up Q4K-style layout): a lane's slice of one row in one pass is 8 VPP weights (VPP words of 8
// 4-bit codes), inside one 256-weight block, with that block's 12 scale bytes and its d | dmin << 16.
template <int VPP>
struct Q4Rp {
    uint32_t qs[VPP];
    uint32_t sc[3];
    uint32_t dm;
};

// v0: first 8-vector of the slice within the row (a multiple of VPP)
template <int VPP>
__device__ __forceinline__ void q4_rp_load(Q4Rp<VPP> &R, const uint8_t *W, const Planes &P, size_t row, int nblk,
                                           int v0) {
    const size_t blk = row * size_t(nblk) + v0 / 32;
    const uint8_t *qp = W + P.off[0] + blk * 128 + (v0 % 32) * 4;
    if constexpr (VPP == 8) {
        const uint4 a = ldg_nc_v4(qp), b = ldg_nc_v4(qp + 16);
        R.qs[0] = a.x; R.qs[1] = a.y; R.qs[2] = a.z; R.qs[3] = a.w;
        R.qs[4] = b.x; R.qs[5] = b.y; R.qs[6] = b.z; R.qs[7] = b.w;
    } else if constexpr (VPP == 4) {
        const uint4 a = ldg_nc_v4(qp);
        R.qs[0] = a.x; R.qs[1] = a.y; R.qs[2] = a.z; R.qs[3] = a.w;
    } else if constexpr (VPP == 2) {
        const uint2 a = ldg_nc_v2(qp);
        R.qs[0] = a.x; R.qs[1] = a.y;
    } else {
        R.qs[0] = ldg_nc_u32(qp);
    }
    const uint8_t *sp = W + P.off[1] + blk * 12;
    R.sc[0] = ldg_nc_u32(sp);
    R.sc[1] = ldg_nc_u32(sp + 4);
    R.sc[2] = ldg_nc_u32(sp + 8);
    R.dm = ldg_nc_u32(W + P.off[2] + blk * 4);
}

// Dot product of a lane's Q4K row slice with its activations xr (fp16 pairs, natural order) and their sums over
// 8-weight pieces xs8: w = d * sc * q - dmin * m per 32-weight sub-block, so the slice contributes
// d * sum_sb sc * (q . x) - dmin * sum_sb m * (sum x).  q comes from a byte -> (low nibble, high nibble) fp16-pair
// table (one 4-byte lane slot per lane: conflict-free); q . x in fp16 inside a sub-block (each half adds at most
// 16 products of q <= 15 and |x| < 64), the rest in fp32.
template <int VPP>
__device__ __forceinline__ float q4_rp_dot(const Q4Rp<VPP> &R, const uint4 (&xr)[VPP], const float (&xs8)[VPP], int v0,
                                           uint32_t lane_tbl) {
    constexpr int NSB = VPP >= 4 ? VPP / 4 : 1, VS = VPP >= 4 ? 4 : VPP;
    const int sb0 = (v0 % 32) / 4;  // first sub-block of the slice inside its block
    float A = 0.f, B = 0.f;
#pragma unroll
    for (int i = 0; i < NSB; i++) {
        __half2 a = __float2half2_rn(0.f), b = a;
        float xsum = 0.f;
#pragma unroll
        for (int j = 0; j < VS; j++) {
            const int v = i * 4 + j;
            const uint32_t t0 = lds32(__byte_perm(R.qs[v], lane_tbl, 0x7604));
            const uint32_t t1 = lds32(__byte_perm(R.qs[v], lane_tbl, 0x7614));
            const uint32_t t2 = lds32(__byte_perm(R.qs[v], lane_tbl, 0x7624));
            const uint32_t t3 = lds32(__byte_perm(R.qs[v], lane_tbl, 0x7634));
            a = __hfma2(u32_as_half2(t0), u32_as_half2(xr[v].x), a);
            b = __hfma2(u32_as_half2(t1), u32_as_half2(xr[v].y), b);
            a = __hfma2(u32_as_half2(t2), u32_as_half2(xr[v].z), a);
            b = __hfma2(u32_as_half2(t3), u32_as_half2(xr[v].w), b);
            xsum += xs8[v];
        }
        const int sb = sb0 + i;
        const float sc = float(q4k_field(R.sc[0], R.sc[1], R.sc[2], 6 * sb));
        const float mn = float(q4k_field(R.sc[0], R.sc[1], R.sc[2], 48 + 6 * sb));
        const float2 s2 = __half22float2(__hadd2(a, b));
        A = fmaf(sc, s2.x + s2.y, A);
        B = fmaf(mn, xsum, B);
    }
    return half_bits_to_float(uint16_t(R.dm & 0xFFFF)) * A - half_bits_to_float(uint16_t(R.dm >> 16)) * B;
}

__device__ __forceinline__ float bf16x8_dot(const uint4 w, const float4 a, const float4 b) {
    float s = bf16_lo(w.x) * a.x;
    s = fmaf(bf16_hi(w.x), a.y, s);
    s = fmaf(bf16_lo(w.y), a.z, s);
    s = fmaf(bf16_hi(w.y), a.w, s);
    s = fmaf(bf16_lo(w.z), b.x, s);
    s = fmaf(bf16_hi(w.z), b.y, s);
    s = fmaf(bf16_lo(w.w), b.z, s);
    s = fmaf(bf16_hi(w.w), b.w, s);
    return s;
}

// Units: shared-expert units first (NRS row pairs of Gs, Us each, see below), then routed units of NR row pairs
// (expert slot j, rows NR i ..).  Row-matrix index rr = 2 * (row - first row) + (0 gate, 1 up).
template <int FMT, int VPP, int NR>
__global__ void __launch_bounds__(DG_THREADS, 1)
    decode_gateup_kernel(const ExpertsDev ex, const __nv_bfloat16 *__restrict__ x, const int32_t *ids, int k,
                         float *__restrict__ h_out, float *__restrict__ hs_out) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ float s_red[DG_WARPS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = ex.d, f = ex.f, fs = ex.fs;
    const int nblk = d / QK;
    const int npass = nblk / VPP;
    const uint32_t sbase = smem_u32(smem);
    uint8_t *tbl = smem + (DG_TABLE_ABS - sbase);
    __half *x16 = reinterpret_cast<__half *>(tbl + 65536);
    float *x32 = reinterpret_cast<float *>(tbl + 65536 + d * 2);
    float *xs8 = reinterpret_cast<float *>(tbl + 65536 + d * 6);  // Q4K: sums of every 8 fp16 activations
    const uint32_t x16_s = DG_TABLE_ABS + 65536;
    constexpr bool Q4 = FMT == DS4MOE_FMT_Q4K;

    constexpr int NRR = 2 * NR;      // row-matrices per unit
    constexpr int LPV = 32 / NRR;    // lanes that hold one row-matrix sum after the reduce-scatter
    // Shared-expert units: one row pair for IQ2X rows of d >= 2048 (VPP = 8: d / 256 passes, a multiple of 4),
    // which spreads the bf16 rows over all warps; Q4K and shorter rows keep NR row pairs (one pass per ring turn).
    // Either way every pass and ring slot below is in range without run-time guards.
    constexpr int NRS = FMT == DS4MOE_FMT_Q4K || VPP < 8 ? NR : 1;
    const int n_sh = fs / NRS;
    const int upe = f / NR;  // routed units per expert
    const int n_all = n_sh + k * upe;
    const int nW = gridDim.x * DG_WARPS;
    const int u_first = warp * gridDim.x + blockIdx.x;
    // the shared expert's rows of this warp's first unit go to L2 while the tables are built
    if (u_first < n_sh && lane < 2 * NRS)
        prefetch_l2((lane & 1 ? ex.sh_up : ex.sh_gate) + size_t(u_first * NRS + (lane >> 1)) * d, uint32_t(d * 2));

    // prologue, one global round trip: every thread loads its codebook entry and its 8 activations together,
    // then writes the codebook table (entry e, lane slot s at DG_TABLE_ABS + e * 256 + s * 16: 8 grid values as
    // fp16), the fp32 activations, and after the block-wide max the fp16 activations scaled by the power of two
    // that puts max |x| in [32, 64)
    static_assert(DG_THREADS >= 512, "two threads per codebook entry");
    const int e_cb = tid >> 1;  // threads 0 .. 511 build the table
    const uint2 raw = !Q4 && tid < 512 ? *reinterpret_cast<const uint2 *>(ex.codebook + e_cb * 8) : make_uint2(0, 0);
    constexpr int XPT = (DG_MAX_D + DG_THREADS * 8 - 1) / (DG_THREADS * 8);  // 8-element chunks per thread
    uint4 xv[XPT];
#pragma unroll
    for (int c = 0; c < XPT; c++) {
        const int i = (tid + c * DG_THREADS) * 8;
        if (i < d) xv[c] = *reinterpret_cast<const uint4 *>(x + i);
    }
    if constexpr (Q4) {
        // byte -> (low nibble, high nibble) as an fp16 pair: entry b, lane slot s at DG_TABLE_ABS + b * 256 + s * 4
        for (int i = tid; i < 256 * 32; i += DG_THREADS) {
            const int b = i >> 5;
            *reinterpret_cast<uint32_t *>(tbl + b * 256 + (i & 31) * 4) =
                half2_as_u32(__floats2half2_rn(float(b & 15), float(b >> 4)));
        }
    } else if (tid < 512) {
        const uint32_t b[2] = {raw.x, raw.y};
        __half2 hv[4];
#pragma unroll
        for (int p = 0; p < 4; p++)
            hv[p] = __floats2half2_rn(float((b[p >> 1] >> (16 * (p & 1))) & 0xFF),
                                      float((b[p >> 1] >> (16 * (p & 1) + 8)) & 0xFF));
        const uint4 v = *reinterpret_cast<uint4 *>(hv);
#pragma unroll
        for (int s = 0; s < 8; s++) {  // slot order rotated so a quarter-warp's 8 stores hit 8 bank groups
            const int slot = ((s + 2 * (e_cb & 3) + (tid & 1)) & 7) + (tid & 1) * 8;
            *reinterpret_cast<uint4 *>(tbl + e_cb * 256 + slot * 16) = v;
        }
    }
    float m = 0.f;
#pragma unroll
    for (int c = 0; c < XPT; c++) {
        const int i = (tid + c * DG_THREADS) * 8;
        if (i < d) {
            const uint4 v = xv[c];
            const float4 a = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
            const float4 cc = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
            reinterpret_cast<float4 *>(x32)[swz16(i / 4)] = a;
            reinterpret_cast<float4 *>(x32)[swz16(i / 4 + 1)] = cc;
            m = fmaxf(m, fmaxf(fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))),
                               fmaxf(fmaxf(fabsf(cc.x), fabsf(cc.y)), fmaxf(fabsf(cc.z), fabsf(cc.w)))));
        }
    }
    m = warp_max(m);
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    m = warp_max(lane < DG_WARPS ? s_red[lane] : 0.f);
    const int xe = pow2_exponent_for(m, 6);
    const float xs = ldexpf(1.f, xe), inv_xs = ldexpf(1.f, -xe);
#pragma unroll
    for (int c = 0; c < XPT; c++) {
        const int i = (tid + c * DG_THREADS) * 8;
        if (i < d) {
            const uint4 v = xv[c];
            const __half2 h0 = __floats2half2_rn(bf16_lo(v.x) * xs, bf16_hi(v.x) * xs);
            const __half2 h1 = __floats2half2_rn(bf16_lo(v.y) * xs, bf16_hi(v.y) * xs);
            const __half2 h2 = __floats2half2_rn(bf16_lo(v.z) * xs, bf16_hi(v.z) * xs);
            const __half2 h3 = __floats2half2_rn(bf16_lo(v.w) * xs, bf16_hi(v.w) * xs);
            reinterpret_cast<uint4 *>(x16)[swz16(i / 8)] =
                make_uint4(half2_as_u32(h0), half2_as_u32(h1), half2_as_u32(h2), half2_as_u32(h3));
            if constexpr (Q4) {
                const float2 f0 = __half22float2(h0), f1 = __half22float2(h1), f2 = __half22float2(h2),
                             f3 = __half22float2(h3);
                xs8[i / 8] = ((f0.x + f0.y) + (f1.x + f1.y)) + ((f2.x + f2.y) + (f3.x + f3.y));
            }
        }
    }
    __syncthreads();

    // the down kernel may launch as CTAs of this grid finish (it waits for the whole grid before reading h)
    pdl_launch_dependents();
    const uint32_t lane_tbl = DG_TABLE_ABS | uint32_t(Q4 ? lane * 4 : (lane & 15) * 16);
    bool waited = false;
    for (int u = u_first; u < n_all; u += nW) {
        float acc[NRR];
#pragma unroll
        for (int i = 0; i < NRR; i++) acc[i] = 0.f;
        if (u < n_sh) {
            // shared expert (bf16), NRS row pairs: pass p covers elements [256 p, 256 p + 256), lane slice 8
            // elements; a ring of the next 8 row slices t = p * NRRS + rr (slot t % 8)
            constexpr int NRRS = 2 * NRS, PU = 8 / NRRS, LPVS = 32 / NRRS;
            const size_t r0 = size_t(u) * NRS;
            const int ns = d / 256, T = ns * NRRS;
            auto wptr = [&](int t) {
                const int rr = t % NRRS;
                return (rr & 1 ? ex.sh_up : ex.sh_gate) + (r0 + (rr >> 1)) * d + (t / NRRS) * 256 + lane * 8;
            };
            float sacc[NRRS];
#pragma unroll
            for (int i = 0; i < NRRS; i++) sacc[i] = 0.f;
            uint4 ring[8];
#pragma unroll
            for (int s = 0; s < 8; s++) ring[s] = ldg_nc_v4(wptr(s));
            for (int p0 = 0; p0 < ns; p0 += PU) {
#pragma unroll
                for (int q = 0; q < PU; q++) {
                    const int p = p0 + q;
                    const float4 xa = reinterpret_cast<const float4 *>(x32)[swz16(p * 64 + 2 * lane)];
                    const float4 xb = reinterpret_cast<const float4 *>(x32)[swz16(p * 64 + 2 * lane + 1)];
#pragma unroll
                    for (int rr = 0; rr < NRRS; rr++) {
                        sacc[rr] += bf16x8_dot(ring[q * NRRS + rr], xa, xb);
                        const int tn = p * NRRS + rr + 8;
                        if (tn < T) ring[q * NRRS + rr] = ldg_nc_v4(wptr(tn));
                    }
                }
            }
            const float v = reduce_scatter<NRRS>(sacc, lane);
            const float up = __shfl_xor_sync(0xffffffffu, v, LPVS);  // gate of row i on lane 2 i LPVS, up next
            if (lane % (2 * LPVS) == 0) hs_out[r0 + lane / (2 * LPVS)] = silu(v) * up;
            continue;
        }
        if (!waited) {
            pdl_wait();  // ids come from the router
            waited = true;
        }
        const int uu = u - n_sh;
        const int j = uu / upe;
        const size_t r0 = size_t(uu % upe) * NR;
        const int e = ids[j];
        if (e < 0 || e >= ex.E) {
            if (lane == 0) set_device_error(DS4MOE_EDEVICE);
            continue;
        }
        const uint8_t *G = ex.gate + size_t(e) * ex.gate_stride, *U = ex.up + size_t(e) * ex.up_stride;
        const int T = npass * NRR;
        using Rp = typename std::conditional<Q4, Q4Rp<VPP>, IqRp<VPP>>::type;
        auto load = [&](Rp &R, int t) {
            const int rr = t % NRR;
            if constexpr (Q4)
                q4_rp_load<VPP>(R, rr & 1 ? U : G, ex.pg, r0 + (rr >> 1), nblk, (t / NRR) * 32 * VPP + lane * VPP);
            else
                iq_rp_load<VPP>(R, rr & 1 ? U : G, ex.pg, r0 + (rr >> 1), nblk, (t / NRR) * 32 * VPP + lane * VPP);
        };
        constexpr int RING = dg_ring<FMT>();
        Rp ring[RING];
#pragma unroll
        for (int s = 0; s < RING; s++) load(ring[s], s);
        for (int p = 0; p < npass; p++) {
            const int v0 = p * 32 * VPP + lane * VPP;
            uint4 xr[VPP];
            float xsv[VPP];
#pragma unroll
            for (int v = 0; v < VPP; v++) xr[v] = lds128(x16_s + swz16(v0 + v) * 16);
            if constexpr (Q4) {
#pragma unroll
                for (int v = 0; v < VPP; v++) xsv[v] = xs8[v0 + v];
            }
#pragma unroll
            for (int rr = 0; rr < NRR; rr++) {
                if constexpr (Q4) acc[rr] += q4_rp_dot<VPP>(ring[rr % RING], xr, xsv, v0, lane_tbl);
                else acc[rr] += iq_rp_dot<VPP>(ring[rr % RING], xr, v0, lane_tbl);
                const int tn = p * NRR + rr + RING;
                if (tn < T) load(ring[rr % RING], tn);
            }
        }
        const float v = reduce_scatter<NRR>(acc, lane);
        const float up = __shfl_xor_sync(0xffffffffu, v, LPV);
        if (lane % (2 * LPV) == 0)
            h_out[size_t(j) * f + r0 + lane / (2 * LPV)] = silu(v * inv_xs) * (up * inv_xs);
    }
    // every warp waits once, so this grid completes only after the router's grid: the down kernel's wait on
    // this grid then covers the routing results too
    if (!waited) pdl_wait();
}

// ============================================================================ down + combine

constexpr int DD_WARPS = 16;
constexpr int DD_THREADS = DD_WARPS * 32;
constexpr uint32_t DD_TABLE_ABS = 0x10000;  // absolute shared address of the 64 KB byte table
constexpr int DD_ROWS = 2;                  // output rows per unit

// Contraction lengths (f) the down kernel takes: f = 256 * 2^i up to 8192.  A lane owns EPL = min(64, f / 32)
// consecutive weights of a row per pass for Q2K, min(32, f / 32) for Q4K (whose 64-weight slices, 32 bytes of
// codes plus 16 of scales per row, spill at 128 registers); f / (32 EPL) passes.
__host__ __device__ __forceinline__ bool dd_supported_f(int f) {
    const int nblk = f / QK;
    return f % QK == 0 && nblk >= 1 && nblk <= 32 && (nblk & (nblk - 1)) == 0;
}
__host__ __device__ __forceinline__ int dd_epl(int f, int fmt) {
    const int cap = fmt == DS4MOE_FMT_Q4K ? 32 : 64;
    return f / 32 < cap ? f / 32 : cap;
}

// Staged h is stored per lane slice (the EPL weights one lane owns in one pass), each slice padded by 16 bytes
// when that keeps the 8 lanes of a quarter-warp on distinct banks; the lane then reads its slice with
// immediate offsets.  hq: fp16 h * 2^e_j, slice stride hq_sb; hsum: fp32 sums of 8 staged values, stride hs_sb.
struct DownSmemLayout {
    int hq, hq_sb, hq_eb, hsum, hs_sb, hs_eb, hs, wsc, eid, total;  // byte offsets from the table base / strides
};
__host__ __device__ __forceinline__ DownSmemLayout dd_layout(int k, int f, int fs, int fmt) {
    DownSmemLayout L;
    const int epl = dd_epl(f, fmt);
    const int nsl = f / epl;                           // lane slices per expert (32 per pass)
    L.hq_sb = epl * 2 + (epl >= 16 ? 16 : 0);
    L.hq_eb = nsl * L.hq_sb;
    L.hs_sb = epl / 8 * 4 + (epl == 64 ? 16 : 0);
    L.hs_eb = nsl * L.hs_sb;
    L.hq = 65536;
    L.hsum = L.hq + ((k * L.hq_eb + 15) & ~15);
    L.hs = L.hsum + ((k * L.hs_eb + 15) & ~15);        // fs floats: shared-expert h (16-byte chunks swizzled)
    L.wsc = L.hs + ((fs * 4 + 15) & ~15);              // k floats: w_j * 2^-e_j
    L.eid = L.wsc + ((k * 4 + 15) & ~15);              // k ints: expert ids
    L.total = int(DD_TABLE_ABS) + L.eid + ((k * 4 + 15) & ~15);
    return L;
}

template <int EPL>
struct QkRp {  // a lane's slice of one Q2K row in one pass: EPL weights
    static constexpr int NQ = EPL >= 16 ? EPL / 16 : 1;
    uint32_t qs[NQ];  // 2-bit codes, one byte per 4 weights (word = 16 weights = one sub-block)
    uint32_t sc;      // sub-block bytes: low nibble scale, high nibble min
    uint32_t dm;      // block d | dmin << 16 (fp16)
};

// p: the row's bytes in the code plane at the slice (row * f / 4 + e0 / 4); the scale and d/dmin planes follow
// from the same slice position
template <int EPL>
__device__ __forceinline__ void qk_rp_load(QkRp<EPL> &R, const uint8_t *W, const Planes &P, size_t row, int nblkf,
                                           int e0) {
    const uint8_t *qp = W + P.off[0] + row * size_t(nblkf) * 64 + e0 / 4;
    const uint8_t *sp = W + P.off[1] + row * size_t(nblkf) * 16 + e0 / 16;
    if constexpr (EPL == 64) {
        const uint4 a = ldg_nc_v4(qp);
        R.qs[0] = a.x; R.qs[1] = a.y; R.qs[2] = a.z; R.qs[3] = a.w;
        R.sc = ldg_nc_u32(sp);
    } else if constexpr (EPL == 32) {
        const uint2 a = ldg_nc_v2(qp);
        R.qs[0] = a.x; R.qs[1] = a.y;
        R.sc = ldg_nc_u16(sp);
    } else if constexpr (EPL == 16) {
        R.qs[0] = ldg_nc_u32(qp);
        R.sc = ldg_nc_u8(sp);
    } else {
        R.qs[0] = ldg_nc_u16(qp);
        R.sc = ldg_nc_u8(sp);
    }
    R.dm = ldg_nc_u32(W + P.off[2] + (row * size_t(nblkf) + e0 / 256) * 4);
}

// sum over the slice of w_i * hh_i with w = d * sc * q - dmin * m per sub-block of 16:
// d * sum_sb sc * (q . hh) - dmin * sum_sb m * (sum hh); hh = the lane's staged h (fp16 pairs), hs8 = sums of 8
template <int EPL>
__device__ __forceinline__ float qk_rp_dot(const QkRp<EPL> &R, const uint32_t (&hh)[EPL / 2],
                                           const float (&hs8)[EPL / 8], uint32_t lane_tbl) {
    constexpr int NSB = EPL >= 16 ? EPL / 16 : 1, NB = EPL >= 16 ? 4 : 2;  // sub-blocks, code bytes per sub-block
    float A = 0.f, B = 0.f;
#pragma unroll
    for (int sb = 0; sb < NSB; sb++) {
        __half2 a = __float2half2_rn(0.f), b = a;
#pragma unroll
        for (int bb = 0; bb < NB; bb++) {
            const uint2 t = lds64(__byte_perm(R.qs[sb], lane_tbl, 0x7604 | (bb << 4)));
            a = __hfma2(u32_as_half2(t.x), u32_as_half2(hh[sb * 8 + 2 * bb]), a);
            b = __hfma2(u32_as_half2(t.y), u32_as_half2(hh[sb * 8 + 2 * bb + 1]), b);
        }
        const float2 s = __half22float2(__hadd2(a, b));
        const uint32_t scb = (R.sc >> (8 * sb)) & 0xFFu;
        const float hsum = EPL >= 16 ? hs8[2 * sb] + hs8[2 * sb + 1] : hs8[0];
        A = fmaf(float(scb & 15u), s.x + s.y, A);
        B = fmaf(float(scb >> 4), hsum, B);
    }
    const float dd = half_bits_to_float(uint16_t(R.dm & 0xFFFF));
    const float dmin = half_bits_to_float(uint16_t(R.dm >> 16));
    return dd * A - dmin * B;
}


// Q4K down rows: a lane's slice of one row in one pass is EPL weights (EPL / 8 words of 4-bit codes) inside one
// 256-weight block, with that block's 12 scale bytes and d | dmin << 16.
template <int EPL>
struct Q4DRp {
    static constexpr int NQ = EPL / 8;
    uint32_t qs[NQ];
    uint32_t sc[3];
    uint32_t dm;
};

template <int EPL>
__device__ __forceinline__ void q4d_rp_load(Q4DRp<EPL> &R, const uint8_t *W, const Planes &P, size_t row, int nblkf,
                                            int e0) {
    const size_t blk = row * size_t(nblkf) + e0 / 256;
    const uint8_t *qp = W + P.off[0] + blk * 128 + (e0 % 256) / 2;
    if constexpr (EPL == 64) {
        const uint4 a = ldg_nc_v4(qp), b = ldg_nc_v4(qp + 16);
        R.qs[0] = a.x; R.qs[1] = a.y; R.qs[2] = a.z; R.qs[3] = a.w;
        R.qs[4] = b.x; R.qs[5] = b.y; R.qs[6] = b.z; R.qs[7] = b.w;
    } else if constexpr (EPL == 32) {
        const uint4 a = ldg_nc_v4(qp);
        R.qs[0] = a.x; R.qs[1] = a.y; R.qs[2] = a.z; R.qs[3] = a.w;
    } else if constexpr (EPL == 16) {
        const uint2 a = ldg_nc_v2(qp);
        R.qs[0] = a.x; R.qs[1] = a.y;
    } else {
        R.qs[0] = ldg_nc_u32(qp);
    }
    const uint8_t *sp = W + P.off[1] + blk * 12;
    R.sc[0] = ldg_nc_u32(sp);
    R.sc[1] = ldg_nc_u32(sp + 4);
    R.sc[2] = ldg_nc_u32(sp + 8);
    R.dm = ldg_nc_u32(W + P.off[2] + blk * 4);
}

// sum over the slice of w_i * hh_i with w = d * sc * q - dmin * m per 32-weight sub-block (hh: the lane's staged
// h, fp16 pairs in natural order; hs8: sums of every 8 staged values); q from the byte -> fp16-pair table
template <int EPL>
__device__ __forceinline__ float q4d_rp_dot(const Q4DRp<EPL> &R, const uint32_t (&hh)[EPL / 2],
                                            const float (&hs8)[EPL / 8], int e0, uint32_t lane_tbl) {
    constexpr int NSB = EPL >= 32 ? EPL / 32 : 1, WS = EPL >= 32 ? 4 : EPL / 8;  // sub-blocks, words per sub-block
    const int sb0 = (e0 % 256) / 32;
    float A = 0.f, B = 0.f;
#pragma unroll
    for (int i = 0; i < NSB; i++) {
        __half2 a = __float2half2_rn(0.f), b = a;
        float hsum = 0.f;
#pragma unroll
        for (int j = 0; j < WS; j++) {
            const int w = i * 4 + j;  // word: weights 8 w .. 8 w + 7
            const uint32_t t0 = lds32(__byte_perm(R.qs[w], lane_tbl, 0x7604));
            const uint32_t t1 = lds32(__byte_perm(R.qs[w], lane_tbl, 0x7614));
            const uint32_t t2 = lds32(__byte_perm(R.qs[w], lane_tbl, 0x7624));
            const uint32_t t3 = lds32(__byte_perm(R.qs[w], lane_tbl, 0x7634));
            a = __hfma2(u32_as_half2(t0), u32_as_half2(hh[4 * w]), a);
            b = __hfma2(u32_as_half2(t1), u32_as_half2(hh[4 * w + 1]), b);
            a = __hfma2(u32_as_half2(t2), u32_as_half2(hh[4 * w + 2]), a);
            b = __hfma2(u32_as_half2(t3), u32_as_half2(hh[4 * w + 3]), b);
            hsum += hs8[w];
        }
        const int sb = sb0 + i;
        const float sc = float(q4k_field(R.sc[0], R.sc[1], R.sc[2], 6 * sb));
        const float mn = float(q4k_field(R.sc[0], R.sc[1], R.sc[2], 48 + 6 * sb));
        const float2 s2 = __half22float2(__hadd2(a, b));
        A = fmaf(sc, s2.x + s2.y, A);
        B = fmaf(mn, hsum, B);
    }
    return half_bits_to_float(uint16_t(R.dm & 0xFFFF)) * A - half_bits_to_float(uint16_t(R.dm >> 16)) * B;
}

// the lane's staged slice (EPL fp16 and EPL / 8 sums) at shared addresses hq_addr, hs_addr
template <int EPL>
__device__ __forceinline__ void dd_slice_load(uint32_t hq_addr, uint32_t hs_addr, uint32_t (&hh)[EPL / 2],
                                              float (&hs8)[EPL / 8]) {
#pragma unroll
    for (int i = 0; i < EPL / 8; i++) {
        const uint4 v = lds128(hq_addr + 16 * i);
        hh[4 * i] = v.x; hh[4 * i + 1] = v.y; hh[4 * i + 2] = v.z; hh[4 * i + 3] = v.w;
    }
    if constexpr (EPL >= 32) {
#pragma unroll
        for (int i = 0; i < EPL / 32; i++) {
            const uint4 v = lds128(hs_addr + 16 * i);
            hs8[4 * i] = __uint_as_float(v.x); hs8[4 * i + 1] = __uint_as_float(v.y);
            hs8[4 * i + 2] = __uint_as_float(v.z); hs8[4 * i + 3] = __uint_as_float(v.w);
        }
    } else if constexpr (EPL == 16) {
        const uint2 v = lds64(hs_addr);
        hs8[0] = __uint_as_float(v.x); hs8[1] = __uint_as_float(v.y);
    } else {
        uint32_t v;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(hs_addr));
        hs8[0] = __uint_as_float(v);
    }
}

template <int FMT, int EPL>
__global__ void __launch_bounds__(DD_THREADS, 1)
    decode_down_kernel(const ExpertsDev ex, const float *h, const float *hs_in, const int32_t *ids, const float *wts,
                       int k, float *__restrict__ out) {
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr bool Q4 = FMT == DS4MOE_FMT_Q4K;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = ex.d, f = ex.f, fs = ex.fs;
    const int nblkf = f / QK;
    const int npass = f / (32 * EPL);
    const uint32_t sbase = smem_u32(smem);
    uint8_t *tb = smem + (DD_TABLE_ABS - sbase);
    const DownSmemLayout L = dd_layout(k, f, fs, FMT);
    float *hsl = reinterpret_cast<float *>(tb + L.hs);
    float *wsc = reinterpret_cast<float *>(tb + L.wsc);
    int *eid = reinterpret_cast<int *>(tb + L.eid);
    const int n_units = d / DD_ROWS;
    const int nW = gridDim.x * DD_WARPS;
    const int u_first = warp * gridDim.x + blockIdx.x;
    // the shared expert's rows of this warp's first unit go to L2 while the table is built
    if (fs > 0 && u_first < n_units && lane == 0)
        prefetch_l2(ex.sh_down + size_t(u_first) * DD_ROWS * fs, uint32_t(DD_ROWS * fs * 2));

    // Q2K: byte -> 4 fp16 table, entry b holds q_i = (b >> 2i) & 3, lane slot s at DD_TABLE_ABS + b * 256 + s * 8;
    // Q4K: byte -> (low nibble, high nibble) as an fp16 pair, lane slot s at DD_TABLE_ABS + b * 256 + s * 4
    for (int i = tid; i < 256 * 32; i += DD_THREADS) {
        const int b = i >> 5;
        if constexpr (Q4) {
            *reinterpret_cast<uint32_t *>(tb + b * 256 + (i & 31) * 4) =
                half2_as_u32(__floats2half2_rn(float(b & 15), float(b >> 4)));
        } else {
            const __half2 lo = __floats2half2_rn(float(b & 3), float((b >> 2) & 3));
            const __half2 hi = __floats2half2_rn(float((b >> 4) & 3), float((b >> 6) & 3));
            *reinterpret_cast<uint2 *>(tb + b * 256 + (i & 31) * 8) = make_uint2(half2_as_u32(lo), half2_as_u32(hi));
        }
    }

    pdl_wait();  // h and hs come from the gate/up kernel, ids and weights from the router

    const int NS = npass * k;  // routed steps: (pass p, expert slot j), both rows of the unit
    const int nsp = fs / 256;  // shared passes: lane slice 8 weights of [256 p, 256 p + 256)
    // Rings of the unit in progress: routed steps n and n + 1 (both rows), shared passes p .. p + 3 (both rows).
    // (Filling the first unit's rings before the staging below was measured slower: those loads then compete
    // with the staging's reads of h, which every warp waits for.)
    using Rp = typename std::conditional<Q4, Q4DRp<EPL>, QkRp<EPL>>::type;
    Rp rg[2][2];
    uint4 sr[4][2];
    int pn = 0, jn = 0;  // next routed step to load
    auto rload = [&](Rp &R, int e, size_t row, int p) {
        if (e >= 0 && e < ex.E) {
            if constexpr (Q4)
                q4d_rp_load<EPL>(R, ex.down + size_t(e) * ex.down_stride, ex.pd, row, nblkf, p * 32 * EPL + lane * EPL);
            else
                qk_rp_load<EPL>(R, ex.down + size_t(e) * ex.down_stride, ex.pd, row, nblkf, p * 32 * EPL + lane * EPL);
        }
    };
    auto prime = [&](int u, const int *idv) {
        const size_t r0 = size_t(u) * DD_ROWS;
        pn = 0;
        jn = 0;
#pragma unroll
        for (int s = 0; s < 2; s++)
            if (s < NS) {
                const int e = idv[jn];
                rload(rg[s][0], e, r0, pn);
                rload(rg[s][1], e, r0 + 1, pn);
                if (++jn == k) { jn = 0; pn++; }
            }
        const __nv_bfloat16 *s0 = ex.sh_down + r0 * fs + lane * 8;
#pragma unroll
        for (int s = 0; s < 4; s++)
            if (s < nsp) {
                sr[s][0] = ldg_nc_v4(s0 + s * 256);
                sr[s][1] = ldg_nc_v4(s0 + fs + s * 256);
            }
    };

    // Stage h_j: fp16 of h * 2^e_j with max |h_j| * 2^e_j in [32, 64), and the fp32 sums of every 8 staged values,
    // both in per-lane-slice order.  With k <= 8 experts and f <= 2048 two warps share an expert and hold their
    // halves in registers (one round of loads, all 16 warps busy); otherwise one warp per expert loads its chunks
    // twice (for the maximum, then to convert), 4 per lane at a time.  The result is the same either way.
    const int nc = f / 128;  // float4 chunks of h_j per lane (a multiple of 2)
    // h_j -> fp16 slice of one chunk c (weights 4c .. 4c + 3 of lane slice order), and its sums of 8
    auto stage_chunk = [&](int j, int c, float4 v, float sc) {
        const __half2 p0 = __floats2half2_rn(v.x * sc, v.y * sc);
        const __half2 p1 = __floats2half2_rn(v.z * sc, v.w * sc);
        const int el = 4 * c, slice = el / EPL, o = el % EPL;  // slice = pass * 32 + lane
        *reinterpret_cast<uint2 *>(tb + L.hq + j * L.hq_eb + slice * L.hq_sb + o * 2) =
            make_uint2(half2_as_u32(p0), half2_as_u32(p1));
        const float2 a = __half22float2(p0), b = __half22float2(p1);
        float s = (a.x + a.y) + (b.x + b.y);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        if ((lane & 1) == 0)
            *reinterpret_cast<float *>(tb + L.hsum + j * L.hs_eb + slice * L.hs_sb + (o / 8) * 4) = s;
    };
    auto expert_meta = [&](int j, int e) {
        wsc[j] = wts[j] * ldexpf(1.f, -e);
        const int id = ids[j];
        eid[j] = id;
        if (id < 0 || id >= ex.E) set_device_error(DS4MOE_EDEVICE);
    };
    const bool two_warps = 2 * k <= DD_WARPS && nc <= 16;  // uniform over the block
    if (two_warps) {
        // two warps per expert, each holding its half of h_j's chunks in registers (one round of loads); the
        // halves' maxima meet in shared memory
        __shared__ float s_hmax[DD_WARPS];
        const int j = warp >> 1, hf = warp & 1, nh = nc / 2;
        float4 v[8];
        if (j < k) {
            const float4 *hj = reinterpret_cast<const float4 *>(h + size_t(j) * f) + hf * nh * 32;
#pragma unroll
            for (int i = 0; i < 8; i++)
                if (i < nh) v[i] = hj[i * 32 + lane];
            float m = 0.f;
#pragma unroll
            for (int i = 0; i < 8; i++)
                if (i < nh) m = fmaxf(m, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
            m = warp_max(m);
            if (lane == 0) s_hmax[warp] = m;
        }
        __syncthreads();
        if (j < k) {
            const int e = pow2_exponent_for(fmaxf(s_hmax[2 * j], s_hmax[2 * j + 1]), 6);
            const float sc = ldexpf(1.f, e);
#pragma unroll
            for (int i = 0; i < 8; i++)
                if (i < nh) stage_chunk(j, (hf * nh + i) * 32 + lane, v[i], sc);
            if (hf == 0 && lane == 0) expert_meta(j, e);
        }
    }
    for (int j = warp; j < k && !two_warps; j += DD_WARPS) {
        const float4 *hj = reinterpret_cast<const float4 *>(h + size_t(j) * f);
        float m = 0.f;
        for (int c0 = 0; c0 < nc; c0 += 4) {
            float4 v[4];
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (c0 + i < nc) v[i] = hj[(c0 + i) * 32 + lane];
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (c0 + i < nc)
                    m = fmaxf(m, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
        }
        const int e = pow2_exponent_for(warp_max(m), 6);
        const float sc = ldexpf(1.f, e);
        for (int c0 = 0; c0 < nc; c0 += 4) {
            float4 v[4];
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (c0 + i < nc) v[i] = hj[(c0 + i) * 32 + lane];
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (c0 + i < nc) stage_chunk(j, (c0 + i) * 32 + lane, v[i], sc);
        }
        if (lane == 0) expert_meta(j, e);
    }
    for (int i = tid * 4; i < fs; i += DD_THREADS * 4)
        reinterpret_cast<float4 *>(hsl)[swz16(i / 4)] = *reinterpret_cast<const float4 *>(hs_in + i);
    __syncthreads();

    const uint32_t lane_tbl = DD_TABLE_ABS | uint32_t(lane * (Q4 ? 4 : 8));
    const uint32_t hq_lane = DD_TABLE_ABS + uint32_t(L.hq + lane * L.hq_sb);
    const uint32_t hs_lane = DD_TABLE_ABS + uint32_t(L.hsum + lane * L.hs_sb);
    for (int u = u_first; u < n_units; u += nW) {
        const size_t r0 = size_t(u) * DD_ROWS;
        prime(u, eid);
        if (u + nW < n_units && fs > 0 && lane == 0)
            prefetch_l2(ex.sh_down + (r0 + size_t(nW) * DD_ROWS) * fs, uint32_t(DD_ROWS * fs * 2));
        // shared expert first (bf16 rows, fp32 hs): it covers the latency of the routed ring's first loads
        float acc0 = 0.f, acc1 = 0.f;
        if (nsp > 0) {
            const __nv_bfloat16 *s0 = ex.sh_down + r0 * fs + lane * 8, *s1 = s0 + fs;
            for (int p0 = 0; p0 < nsp; p0 += 4) {
#pragma unroll
                for (int s = 0; s < 4; s++) {
                    const int p = p0 + s;
                    if (p < nsp) {
                        const float4 xa = reinterpret_cast<const float4 *>(hsl)[swz16(p * 64 + 2 * lane)];
                        const float4 xb = reinterpret_cast<const float4 *>(hsl)[swz16(p * 64 + 2 * lane + 1)];
                        acc0 += bf16x8_dot(sr[s][0], xa, xb);
                        acc1 += bf16x8_dot(sr[s][1], xa, xb);
                        if (p + 4 < nsp) {
                            sr[s][0] = ldg_nc_v4(s0 + (p + 4) * 256);
                            sr[s][1] = ldg_nc_v4(s1 + (p + 4) * 256);
                        }
                    }
                }
            }
        }
        // routed experts
        int p = 0, j = 0;  // step being consumed
        for (int n0 = 0; n0 < NS; n0 += 2) {
#pragma unroll
            for (int s = 0; s < 2; s++) {
                if (n0 + s < NS) {
                    uint32_t hh[EPL / 2];
                    float hs8[EPL / 8];
                    const int sl = p * 32;  // slice offset of this pass
                    dd_slice_load<EPL>(hq_lane + j * L.hq_eb + sl * L.hq_sb, hs_lane + j * L.hs_eb + sl * L.hs_sb, hh,
                                       hs8);
                    const int e = eid[j];
                    if (e >= 0 && e < ex.E) {
                        const float w = wsc[j];
                        if constexpr (Q4) {
                            const int e0 = p * 32 * EPL + lane * EPL;
                            acc0 = fmaf(w, q4d_rp_dot<EPL>(rg[s][0], hh, hs8, e0, lane_tbl), acc0);
                            acc1 = fmaf(w, q4d_rp_dot<EPL>(rg[s][1], hh, hs8, e0, lane_tbl), acc1);
                        } else {
                            acc0 = fmaf(w, qk_rp_dot<EPL>(rg[s][0], hh, hs8, lane_tbl), acc0);
                            acc1 = fmaf(w, qk_rp_dot<EPL>(rg[s][1], hh, hs8, lane_tbl), acc1);
                        }
                    }
                    if (n0 + s + 2 < NS) {
                        const int en = eid[jn];
                        rload(rg[s][0], en, r0, pn);
                        rload(rg[s][1], en, r0 + 1, pn);
                        if (++jn == k) { jn = 0; pn++; }
                    }
                    if (++j == k) { j = 0; p++; }
                }
            }
        }
        // reduce: lanes 0..15 end with row 0, lanes 16..31 with row 1
        const bool hi = lane & 16;
        float v = (hi ? acc1 : acc0) + __shfl_xor_sync(0xffffffffu, hi ? acc0 : acc1, 16);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((lane & 15) == 0) out[r0 + (lane >> 4)] = v;
    }
}

}  // namespace ds4
