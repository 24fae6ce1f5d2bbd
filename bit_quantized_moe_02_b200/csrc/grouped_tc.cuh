// Grouped dequantize-GEMM on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// One CTA computes one (expert, 128-row weight tile, <=128-token tile) work item
// of the permuted MoE experts (swap-AB: weights are the M=128 operand, tokens
// the N operand, N rounded up to a multiple of 16 per tile):
//
//   warp 0      allocates TMEM and, from one lane, issues tcgen05.mma
//               (kind::f16, fp32 accumulators in TMEM) for every K-chunk;
//               tcgen05.commit releases the shared-memory stage back to the
//               producers and finally signals the epilogue.
//   warp 1      loads the tile's token rows (permuted fp16 activations or
//               SwiGLU outputs, contiguous per expert) with one 2D TMA tensor
//               copy per stage into a 128B-swizzled K-major stage; for dense
//               formats (router fp16, shared-expert bf16) it loads the A tiles
//               the same way.
//   warp 2      streams the packed IQ2X / Q2K planes of the tile's rows, one
//               256-wide K block at a time, with 3D TMA copies into a 2-slot
//               shared-memory ring (Q4K and bf16 producers load into registers).
//   warps 4-11  dequantize the packed blocks in registers (shared-memory
//               codebook / sign-bit XOR / fp16 scale) and store the fp16 A
//               tiles to tensor memory (tcgen05.st, row = TMEM lane); the MMA
//               reads A from there, which keeps the A tiles out of shared
//               memory (the MMA's operand reads, the producers' stores and the
//               codebook lookups would otherwise share its bandwidth).  All
//               eight then run the epilogue, splitting the token columns:
//               tcgen05.ld the accumulators, SwiGLU (gate/up) or
//               routing-weight scaling (down), stores.
//
// The packed down kernels need 256 TMEM columns and ~90 KB of shared memory,
// so two CTAs share an SM and one's prologue and epilogue overlap the other's
// main loop.
//
// Gate and up share one work item: two accumulators (TMEM columns [0,128) and
// [128,256)) hold matching rows, so each epilogue thread owns a gate/up pair.
// Every wait on an mbarrier is bounded; a timeout records DS4MOE_ETIMEOUT,
// stops the CTA's roles, lets its TMA copies in flight land and still frees
// TMEM before returning.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "grouped_common.cuh"

namespace ds4 {
namespace tc {

// Internal A formats.  Dense operands skip the dequantizing producers: the A tiles come by 2D TMA like the
// token tiles, and the MMA reads both as they are (A and B of one MMA have the same type).
constexpr int FMT_F16 = 4;    // fp16 rows (router weights) with fp16 tokens
constexpr int FMT_BF16D = 5;  // bf16 rows (shared expert) with bf16 tokens
template <int AFMT>
__host__ __device__ constexpr bool is_dense() { return AFMT == FMT_F16 || AFMT == FMT_BF16D; }

constexpr int M = 128;          // weight rows per accumulator
constexpr int BK = 64;          // K per pipeline stage (one 128-byte swizzle row of fp16)
constexpr int NT = 128;         // max tokens per work item
constexpr int THREADS = 384;    // 12 warps
constexpr int W_B0 = 1, N_WB = 3;
constexpr int W_A0 = 4, N_WA = 8;
constexpr int A_TILE = M * BK * 2;   // 16 KB
constexpr int B_TILE = NT * BK * 2;  // 16 KB
constexpr int TABLE_BYTES = 256 * 8 * 16;
constexpr long long WAIT_NS = 2000000000LL;  // 2 s bound on any single wait
constexpr int MAX_K = 16384;                 // longest contraction of a packed DOWN operand (f)

// Packed A planes streamed by TMA (3D maps: plane bytes x rows x experts) into a 2-slot shared-memory ring, one
// slot per 256-wide K block of the tile's 128 rows: IQ2X gate/up (index and sign planes of both matrices, 16 KB)
// and Q2K down (code and scale planes, 10 KB).  The producers read them there; the few per-block scalars
// (group scales, d, dmin) stay plain global loads.  Other formats load their packed data into registers.
template <int AFMT, bool GATEUP>
struct PackTma {
    static constexpr bool ON = (AFMT == DS4MOE_FMT_IQ2X && GATEUP) || (AFMT == DS4MOE_FMT_Q2K && !GATEUP);
    static constexpr int SLOT = AFMT == DS4MOE_FMT_IQ2X ? 4 * M * 32 : M * 64 + M * 16;
    static constexpr int NSLOT = ON ? 2 : 0;
};

template <int AFMT, bool GATEUP>
struct Cfg {
    // ATM: the dequantized A tiles live in tensor memory (tcgen05.st by the producers, MMA with A from TMEM);
    // the shared-memory stages then hold only the token tile.  Every packed format does this; dense A tiles
    // come by TMA into shared memory.
    static constexpr bool ATM = !is_dense<AFMT>();
    // the packed down kernels then fit twice per SM (shared memory, TMEM, registers), so one CTA's prologue and
    // epilogue overlap the other's main loop
    static constexpr int MIN_BLOCKS = (ATM && !GATEUP) ? 2 : 1;
    // K per pipeline step: 128 for the packed kernels (two 64-wide sub-steps: two token-tile boxes, two A parts
    // per producer), which halves the per-step barrier, fence and commit work; 64 for the dense ones
    static constexpr int KS = ATM ? 2 * BK : BK;
    static constexpr int SUB = KS / BK;
    static constexpr int STAGES = ATM ? 2 : 4;
    static constexpr int A_SMEM = ATM ? 0 : (GATEUP ? 2 : 1) * A_TILE;  // A bytes per shared-memory stage
    static constexpr int STAGE = A_SMEM + SUB * B_TILE;
    static constexpr int ACC_COLS = GATEUP ? 256 : 128;                  // fp32 accumulators
    static constexpr int A_COLS = ATM ? (GATEUP ? 2 : 1) * (KS / 2) : 0;  // TMEM columns of one stage's A tiles
    static constexpr int TMEM_COLS = ATM ? (GATEUP ? 512 : 256) : ACC_COLS;
    static_assert(ACC_COLS + STAGES * A_COLS <= TMEM_COLS, "tensor memory");
    static constexpr int PRING_OFF = STAGES * STAGE;
    static constexpr int TABLE_OFF = PRING_OFF + PackTma<AFMT, GATEUP>::NSLOT * PackTma<AFMT, GATEUP>::SLOT;
    static constexpr int TBL = AFMT == DS4MOE_FMT_IQ2X ? TABLE_BYTES : 0;  // only IQ2X dequantizes via a table
    static constexpr int SMEM = TABLE_OFF + TBL + 1024;  // + alignment slack
    static_assert(SMEM <= 232448, "shared memory");
};

// ---- PTX wrappers -----------------------------------------------------------------------------------------

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, "
        "p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false (and records a timeout, raises the
// CTA abort flag) if it did not complete within WAIT_NS, or if another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > uint64_t(WAIT_NS)) {
            set_device_error(DS4MOE_ETIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row x 128-byte atoms stacked every 1024 bytes.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
    uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t(1) << 16;            // leading byte offset (unused for swizzled K-major)
    d |= uint64_t(1024 >> 4) << 32;    // stride byte offset: next 8-row group
    d |= uint64_t(1) << 46;            // descriptor version
    d |= uint64_t(2) << 61;            // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: A and B K-major, both fp16 (or both bf16), fp32 accumulator, M = 128, N = n.
__device__ __forceinline__ uint32_t instr_desc(int n, bool bf16 = false) {
    return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | (uint32_t(n >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Same MMA with A read from tensor memory (a_tmem: lane 0, first column of a 128 x 16 fp16 tile).
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(
            d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// 32 consecutive 32-bit columns of this thread's TMEM lane (warp-collective), then wait for the stores.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// The wait sits in the same asm statement as the load: the registers are undefined until tcgen05.wait::ld, and
// outputs of a separate statement would let the compiler schedule their uses before the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
        "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 2D TMA tensor load (tile mode, no multicast): box at (c0 = inner element, c1 = row) into shared memory,
// completion counted on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
// 3D TMA tensor load (tile mode, no multicast): box at (c0 = byte, c1 = row, c2 = expert)
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     bar),
                 "r"(bytes)
                 : "memory");
}

// ---- A producers: packed data for a "super-stage" of SS pipeline stages is loaded one super-stage ahead ------
//
// GATEUP: thread t owns matrix m = t / 128 (gate, up) and tile row R = t % 128 and writes all 64 weights of
// its row per stage.  DOWN: thread t owns row R = t / 2 and half h = t % 2 (32 weights per stage).

template <int AFMT, bool GATEUP>
struct SPackCfg;
template <> struct SPackCfg<DS4MOE_FMT_IQ2X, true> { static constexpr int SS = 4, NW = 18; };   // one super-block
template <> struct SPackCfg<DS4MOE_FMT_Q4K, true> { static constexpr int SS = 2, NW = 20; };    // half super-block
template <> struct SPackCfg<DS4MOE_FMT_Q2K, false> { static constexpr int SS = 4, NW = 13; };
template <> struct SPackCfg<DS4MOE_FMT_Q4K, false> { static constexpr int SS = 4, NW = 20; };

template <int AFMT, bool GATEUP>
struct SPack {
    uint32_t w[SPackCfg<AFMT, GATEUP>::NW];
};

__device__ __forceinline__ void ld4(uint32_t *w, const uint8_t *p) {
    const uint4 v = ldg_nc_v4(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
}

// Load super-stage `ss` (K range [ss*SS*64, (ss+1)*SS*64)) of row `row` (half h for DOWN).
template <int AFMT, bool GATEUP>
__device__ __forceinline__ void sp_load(SPack<AFMT, GATEUP> &pk, const uint8_t *__restrict__ mat, const Planes &P,
                                        int row, int h, int K, int ss) {
    const int nsb = K / QK;
    if constexpr (AFMT == DS4MOE_FMT_IQ2X) {  // GATEUP, super-block ss
        const size_t b = size_t(row) * nsb + ss;
        ld4(pk.w + 0, mat + P.off[0] + b * 32);
        ld4(pk.w + 4, mat + P.off[0] + b * 32 + 16);
        ld4(pk.w + 8, mat + P.off[1] + b * 32);
        ld4(pk.w + 12, mat + P.off[1] + b * 32 + 16);
        pk.w[16] = ldg_nc_u32(mat + P.off[2] + b * 4);
        pk.w[17] = *reinterpret_cast<const uint16_t *>(mat + P.off[3] + b * 2);
    } else if constexpr (AFMT == DS4MOE_FMT_Q4K && GATEUP) {  // half super-block ss
        const size_t b = size_t(row) * nsb + ss / 2;
        const uint8_t *q = mat + P.off[0] + b * 128 + (ss & 1) * 64;
#pragma unroll
        for (int i = 0; i < 4; i++) ld4(pk.w + 4 * i, q + 16 * i);
        const uint32_t *sc = reinterpret_cast<const uint32_t *>(mat + P.off[1] + b * 12);
        pk.w[16] = sc[0]; pk.w[17] = sc[1]; pk.w[18] = sc[2];
        pk.w[19] = ldg_nc_u32(mat + P.off[2] + b * 4);
    } else if constexpr (AFMT == DS4MOE_FMT_Q2K) {  // DOWN, super-block ss; stage j uses sub-blocks 4j+2h, +1
        const size_t b = size_t(row) * nsb + ss;
        const uint8_t *q = mat + P.off[0] + b * 64 + h * 8;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint2 v = *reinterpret_cast<const uint2 *>(q + 16 * j);
            pk.w[2 * j] = v.x; pk.w[2 * j + 1] = v.y;
        }
        ld4(pk.w + 8, mat + P.off[1] + b * 16);
        pk.w[12] = ldg_nc_u32(mat + P.off[2] + b * 4);
    } else if constexpr (AFMT == DS4MOE_FMT_Q4K) {  // DOWN, super-block ss; stage j uses sub-block 2j+h
        const size_t b = size_t(row) * nsb + ss;
#pragma unroll
        for (int j = 0; j < 4; j++) ld4(pk.w + 4 * j, mat + P.off[0] + b * 128 + (2 * j + h) * 16);
        const uint32_t *sc = reinterpret_cast<const uint32_t *>(mat + P.off[1] + b * 12);
        pk.w[16] = sc[0]; pk.w[17] = sc[1]; pk.w[18] = sc[2];
        pk.w[19] = ldg_nc_u32(mat + P.off[2] + b * 4);
    } else {
        static_assert(AFMT == DS4MOE_FMT_IQ2X, "packed formats only: dense rows come by TMA");
    }
}

__device__ __forceinline__ void q4k_pairs(uint32_t word, __half2 a2, __half2 c2, uint4 &o) {
    const __half2 k1024 = __float2half2_rn(1024.f);
    __half2 P[4];
#pragma unroll
    for (int n = 0; n < 4; n++) {
        const uint32_t v = ((word >> (4 * n)) & 0x000F000Fu) | 0x64006400u;
        P[n] = __hfma2(__hsub2(u32_as_half2(v), k1024), a2, c2);  // (w_n, w_{n+4})
    }
    o.x = half2_as_u32(__lows2half2(P[0], P[1]));
    o.y = half2_as_u32(__lows2half2(P[2], P[3]));
    o.z = half2_as_u32(__highs2half2(P[0], P[1]));
    o.w = half2_as_u32(__highs2half2(P[2], P[3]));
}

// Dequantize stage j (compile-time) of a super-stage: GATEUP -> 8 uint4 (64 weights), DOWN -> 4 uint4 (32).
// hsc: power-of-two factor on the DOWN weights (the inverse of the SwiGLU output's scale for this K range);
// `inf` is raised when a scaled weight could leave the fp16 range.
template <int AFMT, bool GATEUP, int J>
__device__ __forceinline__ void sp_dequant(const SPack<AFMT, GATEUP> &pk, int h, int ss, const uint8_t *tbl_lane,
                                           uint4 *o, bool &inf, float hsc = 1.f) {
    constexpr uint32_t M = 0x80008000u;
    if constexpr (AFMT == DS4MOE_FMT_IQ2X) {
        const float dv = half_bits_to_float(uint16_t(pk.w[17]));
#pragma unroll
        for (int gg = 0; gg < 2; gg++) {
            constexpr int dummy = 0;
            (void)dummy;
            const int g = 2 * J + gg;
            const float s = float((pk.w[16] >> (4 * g)) & 15u);
            const __half2 D2 = __float2half2_rn((dv * (0.5f + s)) * 0.25f);
            const uint32_t W = pk.w[8 + g];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t ib = (pk.w[g] >> (8 * j)) & 0xFFu;
                const uint4 cb = *reinterpret_cast<const uint4 *>(tbl_lane + ib * 128);
                const uint32_t Wj = W << (4 * j);
                uint4 &r = o[gg * 4 + j];
                r.x = half2_as_u32(__hmul2(u32_as_half2(cb.x ^ (Wj & M)), D2));
                r.y = half2_as_u32(__hmul2(u32_as_half2(cb.y ^ ((Wj << 1) & M)), D2));
                r.z = half2_as_u32(__hmul2(u32_as_half2(cb.z ^ ((Wj << 2) & M)), D2));
                r.w = half2_as_u32(__hmul2(u32_as_half2(cb.w ^ ((Wj << 3) & M)), D2));
            }
        }
    } else if constexpr (AFMT == DS4MOE_FMT_Q4K) {
        const float dv = half_bits_to_float(uint16_t(pk.w[19] & 0xFFFF));
        const float dm = half_bits_to_float(uint16_t(pk.w[19] >> 16));
        constexpr int NSUB = GATEUP ? 2 : 1;
#pragma unroll
        for (int u = 0; u < NSUB; u++) {
            // sub-block within the super-block
            const int sub = GATEUP ? ((ss & 1) * 4 + 2 * J + u) : (2 * J + h);
            const int sc = q4k_field(pk.w[16], pk.w[17], pk.w[18], 6 * sub);
            const int mn = q4k_field(pk.w[16], pk.w[17], pk.w[18], 48 + 6 * sub);
            float av = dv * float(sc), cv = dm * float(mn);
            if constexpr (!GATEUP) {
                av *= hsc;
                cv *= hsc;
                inf |= !(fmaf(15.f, av, cv) <= 65504.f);
            }
            const __half2 a2 = __float2half2_rn(av);
            const __half2 c2 = __float2half2_rn(-cv);
            const uint32_t *q = pk.w + (GATEUP ? (2 * J + u) * 4 : J * 4);
#pragma unroll
            for (int w = 0; w < 4; w++) q4k_pairs(q[w], a2, c2, o[u * 4 + w]);
        }
    } else if constexpr (AFMT == DS4MOE_FMT_Q2K) {
        const float dv = half_bits_to_float(uint16_t(pk.w[12] & 0xFFFF));
        const float dm = half_bits_to_float(uint16_t(pk.w[12] >> 16));
        const __half2 k1024 = __float2half2_rn(1024.f);
        const uint32_t scw = (pk.w[8 + J] >> (16 * h)) & 0xFFFFu;  // bytes of sub-blocks 4J+2h, 4J+2h+1
#pragma unroll
        for (int sb = 0; sb < 2; sb++) {
            const uint32_t scb = (scw >> (8 * sb)) & 0xFFu;
            const float av = dv * float(scb & 15u) * hsc, cv = dm * float(scb >> 4) * hsc;
            inf |= !(fmaf(3.f, av, cv) <= 65504.f);
            const __half2 a2 = __float2half2_rn(av);
            const __half2 c2 = __float2half2_rn(-cv);
            __half2 P[8];
#pragma unroll
            for (int p = 0; p < 8; p++) {
                const uint32_t v = ((pk.w[2 * J + sb] >> (2 * p)) & 0x00030003u) | 0x64006400u;
                P[p] = __hfma2(__hsub2(u32_as_half2(v), k1024), a2, c2);  // (w_p, w_{p+8})
            }
            uint32_t *oo = reinterpret_cast<uint32_t *>(&o[2 * sb]);
#pragma unroll
            for (int p = 0; p < 4; p++) {
                oo[p] = half2_as_u32(__lows2half2(P[2 * p], P[2 * p + 1]));
                oo[4 + p] = half2_as_u32(__highs2half2(P[2 * p], P[2 * p + 1]));
            }
        }
    } else {
        static_assert(AFMT == DS4MOE_FMT_IQ2X, "packed formats only: dense rows come by TMA");
    }
}

// ---- the kernel -------------------------------------------------------------------------------------------

template <int AFMT, bool GATEUP>
__global__ void __launch_bounds__(THREADS, Cfg<AFMT, GATEUP>::MIN_BLOCKS)
    grouped_tc_kernel(GroupedArgs a, const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_a0,
                      const __grid_constant__ CUtensorMap tmap_a1, const __grid_constant__ CUtensorMap pmap0,
                      const __grid_constant__ CUtensorMap pmap1, const __grid_constant__ CUtensorMap pmap2,
                      const __grid_constant__ CUtensorMap pmap3) {
    constexpr bool DENSE = is_dense<AFMT>();
    using PT = PackTma<AFMT, GATEUP>;
    using C = Cfg<AFMT, GATEUP>;
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *tbl = smem + C::TABLE_OFF;
    __shared__ __align__(8) uint64_t bars[3 * 4 + 1 + 4];  // (unused)[S], full[S], empty[S], accum, packed ring
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float s_colsc[NT];
    __shared__ int s_orow[NT];      // DOWN with a fused combine: output row (token) of each position
    __shared__ uint32_t s_hmax;     // GATEUP: largest |h| of the tile (float bits; non-finite sorts above +inf)
    __shared__ float s_hsc[MAX_K / 128];  // DOWN: weight factor 2^e of each 128-wide K range

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    int e = 0, pos0, cnt;
    if (a.tile_e) {
        if (int(blockIdx.y) >= *a.n_tiles) return;
        e = a.tile_e[blockIdx.y];
        pos0 = a.tile_pos0[blockIdx.y];
        cnt = a.tile_cnt[blockIdx.y];
    } else {
        pos0 = blockIdx.y * NT;
        if (pos0 >= a.n_pos) return;
        cnt = min(NT, a.n_pos - pos0);
    }
    const int n_eff = max(16, (cnt + 15) & ~15);
    const int nk = a.K / C::KS;  // pipeline steps

    // One "stage full" barrier per stage: the token-tile TMA (its expect-tx arrival and bytes) and, for packed
    // formats, every producer thread (its A part) arrive on it, so the MMA issuer waits once per stage.
    auto full_b = [&](int s) { return smem_u32(&bars[4 + s]); };
    auto full_a = full_b;
    auto empty = [&](int s) { return smem_u32(&bars[8 + s]); };
    const uint32_t accum_bar = smem_u32(&bars[12]);
    auto full_p = [&](int s) { return smem_u32(&bars[13 + s]); };
    auto empty_p = [&](int s) { return smem_u32(&bars[15 + s]); };
    const int nss_p = a.K / QK;  // packed-ring blocks

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(full_b(s), DENSE ? 1 : N_WA * 32 + 1);  // TMA arrival + every producer thread
            mbar_init(empty(s), 1);
        }
        mbar_init(accum_bar, 1);
        for (int s = 0; s < 2; s++) {
            mbar_init(full_p(s), 1);
            mbar_init(empty_p(s), N_WA * 32);
        }
        s_abort = 0;
        s_hmax = 0;
        fence_mbar_init();
    }
    if (!GATEUP && !DENSE && tid < a.K / 128)
        s_hsc[tid] = a.h_exp_in ? ldexpf(1.f, a.h_exp_in[int(blockIdx.y) * (a.K / 128) + tid]) : 1.f;
    if (warp == 0) {
        tmem_alloc(smem_u32(&s_tmem), C::TMEM_COLS);
        tc_fence_before();
    }
    if (tid < NT) {
        // per-token column scale: the activation's power-of-two scale (indexed by token) times the gate weight
        float sc = 1.f;
        if (tid < cnt) {
            const int pos = pos0 + tid;
            if (a.b_colscale) sc *= a.b_colscale[a.b_rowidx ? a.b_rowidx[pos] : pos];
            if (a.pos_weight) sc *= a.pos_weight[pos];
            if (a.out_row) s_orow[tid] = a.out_row[pos];
        }
        s_colsc[tid] = sc;
    }
    if constexpr (AFMT == DS4MOE_FMT_IQ2X) {
        // lane-slot interleaved codebook table: entry i, slot s at (i*8 + s)*16
        for (int i = tid; i < 256 * 8; i += THREADS) {
            const uint8_t *cb = a.codebook + (i >> 3) * 8;
            __half2 h[4];
#pragma unroll
            for (int p = 0; p < 4; p++) h[p] = __floats2half2_rn(float(cb[2 * p]), float(cb[2 * p + 1]));
            *reinterpret_cast<uint4 *>(tbl + i * 16) = *reinterpret_cast<uint4 *>(h);
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort_flag = &s_abort;

    if (warp == 0) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = instr_desc(n_eff, AFMT == FMT_BF16D);
            bool ok = true;
            for (int kc = 0; kc < nk && ok; kc++) {
                const int s = kc % S;
                const uint32_t par = (kc / S) & 1;
                ok = mbar_wait(full_b(s), par, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * C::STAGE);
                const uint32_t a0 = st, a1 = st + A_TILE, b0 = st + C::A_SMEM;
                const uint32_t at0 = tmem + C::ACC_COLS + s * C::A_COLS;  // ATM: gate A columns, up at +KS/2
#pragma unroll
                for (int kk = 0; kk < C::KS / 16; kk++) {
                    const uint32_t acc = (kc > 0 || kk > 0) ? 1u : 0u;
                    if constexpr (C::ATM) {
                        const uint64_t bd = smem_desc(b0 + (kk / 4) * B_TILE + (kk % 4) * 32);  // 64-wide sub-tile, 16-wide slice
                        mma_f16_ta(tmem, at0 + kk * 8, bd, idesc, acc);
                        if constexpr (GATEUP) mma_f16_ta(tmem + NT, at0 + C::KS / 2 + kk * 8, bd, idesc, acc);
                    } else {
                        mma_f16(tmem, smem_desc(a0 + kk * 32), smem_desc(b0 + kk * 32), idesc, acc);
                        if constexpr (GATEUP) mma_f16(tmem + NT, smem_desc(a1 + kk * 32), smem_desc(b0 + kk * 32), idesc, acc);
                    }
                }
                mma_commit(empty(s));
            }
            mma_commit(accum_bar);  // also covers an aborted loop: the epilogue / teardown waits on it
        }
        __syncwarp();
    } else if (warp < W_B0 + N_WB) {
        // ------------------------------------------------------------------ token rows: one 2D TMA copy per stage
        if (warp == W_B0 && lane == 0) {
            int issued = 0;
            for (int kc = 0; kc < nk; kc++) {
                const int s = kc % S;
                const uint32_t par = ((kc / S) & 1) ^ 1;
                if (!mbar_wait(empty(s), par, abort_flag)) break;
                const uint32_t st = smem_u32(smem + s * C::STAGE), bst = st + C::A_SMEM;
                // full boxes: rows past a tensor's end are zero-filled and still counted
                mbar_expect_tx(full_b(s), C::SUB * B_TILE + (DENSE ? (GATEUP ? 2 : 1) * A_TILE : 0));
                if constexpr (DENSE) {
                    tma_load_2d(st, &tmap_a0, kc * BK, blockIdx.x * M, full_b(s));
                    if constexpr (GATEUP) tma_load_2d(st + A_TILE, &tmap_a1, kc * BK, blockIdx.x * M, full_b(s));
                }
#pragma unroll
                for (int sub = 0; sub < C::SUB; sub++)
                    tma_load_2d(bst + sub * B_TILE, &tmap_b, kc * C::KS + sub * BK, pos0, full_b(s));
                issued = kc + 1;
            }
            if (*abort_flag) {
                // let this CTA's copies still in flight land before its shared memory is released (bounded: the
                // stage barrier also counts the producers, so after an abort this may run to its time limit)
                const uint64_t t0 = globaltimer();
                for (int kc = max(0, issued - S); kc < issued; kc++)
                    while (!mbar_try_wait(full_b(kc % S), (kc / S) & 1) && globaltimer() - t0 < uint64_t(WAIT_NS)) {
                    }
            }
        }
        if constexpr (PT::ON) {
            // ------------------------------------------------------------------ packed A planes: 3D TMA copies
            if (warp == W_B0 + 1 && lane == 0) {
                int issued = 0;
                const int row0 = blockIdx.x * M;
                for (int ss = 0; ss < nss_p; ss++) {
                    const int sl = ss & 1;
                    if (!mbar_wait(empty_p(sl), ((ss >> 1) & 1) ^ 1, abort_flag)) break;
                    const uint32_t dst = smem_u32(smem + C::PRING_OFF + sl * PT::SLOT);
                    mbar_expect_tx(full_p(sl), PT::SLOT);
                    if constexpr (AFMT == DS4MOE_FMT_IQ2X) {  // gate idx, gate sgn, up idx, up sgn: 32 B x 128 rows
                        tma_load_3d(dst, &pmap0, ss * 32, row0, e, full_p(sl));
                        tma_load_3d(dst + M * 32, &pmap1, ss * 32, row0, e, full_p(sl));
                        tma_load_3d(dst + 2 * M * 32, &pmap2, ss * 32, row0, e, full_p(sl));
                        tma_load_3d(dst + 3 * M * 32, &pmap3, ss * 32, row0, e, full_p(sl));
                    } else {  // Q2K codes 64 B x 128 rows, scales 16 B x 128 rows
                        tma_load_3d(dst, &pmap0, ss * 64, row0, e, full_p(sl));
                        tma_load_3d(dst + M * 64, &pmap1, ss * 16, row0, e, full_p(sl));
                    }
                    issued = ss + 1;
                }
                if (*abort_flag) {  // let copies in flight land before the shared memory is released (bounded)
                    const uint64_t t0 = globaltimer();
                    for (int ss = max(0, issued - 2); ss < issued; ss++)
                        while (!mbar_try_wait(full_p(ss & 1), (ss >> 1) & 1) && globaltimer() - t0 < uint64_t(WAIT_NS)) {
                        }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ dequantizing producers
        // Hands this thread's dequantized part of stage s (row R of matrix m, or K half h of a DOWN row) to the
        // MMA through tensor memory, then arrives on the stage's barrier: row R is TMEM lane R (a warp may store
        // only to its lane quarter, warp & 3), fp16 K pairs in 32-bit columns.  The writing thread waits for its
        // own stores (tcgen05.wait::st) and releases them itself.
        // A step's A tile is C::KS / 2 columns per matrix; 64-wide sub-step js takes columns [32 js, 32 js + 32),
        // of which a DOWN thread's K half h writes [32 js + 16 h, 32 js + 16 h + 16).
        auto begin_a = [&]() {
            __syncwarp();
            tc_fence_after();  // after the stage-release wait: the MMA that read these columns is done
        };
        auto st_a = [&](int s, int m, int h, int js, const auto &o) {
            constexpr int NOUT = GATEUP ? 8 : 4;
            uint32_t wv[NOUT * 4];
#pragma unroll
            for (int c = 0; c < NOUT; c++) {
                wv[4 * c] = o[c].x; wv[4 * c + 1] = o[c].y; wv[4 * c + 2] = o[c].z; wv[4 * c + 3] = o[c].w;
            }
            const uint32_t ta = tmem + (uint32_t((warp & 3) * 32) << 16) + C::ACC_COLS + s * C::A_COLS + js * (BK / 2);
            if constexpr (GATEUP) tmem_st32(ta + m * (C::KS / 2), wv);
            else tmem_st16(ta + h * (BK / 4), wv);
        };
        auto end_a = [&](int s) {
            tc_fence_before();
            mbar_arrive(full_a(s));
        };
        if constexpr (PT::ON) {
            constexpr int NOUT = GATEUP ? 8 : 4;
            const int at = tid - W_A0 * 32;  // 0 .. 255
            const int m = GATEUP ? at >> 7 : 0;
            // DOWN with A in TMEM: a warp may store only to its TMEM lane quarter (warp & 3), so warps 4-7 take
            // the first K half of rows 32q..32q+31 and warps 8-11 the second
            const int R = GATEUP ? at & 127 : (C::ATM ? (warp & 3) * 32 + lane : at >> 1);
            const int h = GATEUP ? 0 : (C::ATM ? (warp - W_A0) >> 2 : at & 1);
            const uint8_t *mat = GATEUP && m ? a.a1 + size_t(e) * a.a1_stride : a.a0 + size_t(e) * a.a_stride;
            const size_t rowb = size_t(blockIdx.x * M + R) * nss_p;  // block index of the row's first block
            const uint8_t *tbl_lane = tbl + (lane & 7) * 16;
            // per-block scalars two blocks ahead: IQ2X group scales and d, Q2K d | dmin << 16
            auto sload = [&](uint32_t &w0, uint32_t &w1, int ss) {
                if (ss >= nss_p) return;
                if constexpr (AFMT == DS4MOE_FMT_IQ2X) {
                    w0 = ldg_nc_u32(mat + a.pa.off[2] + (rowb + ss) * 4);
                    w1 = *reinterpret_cast<const uint16_t *>(mat + a.pa.off[3] + (rowb + ss) * 2);
                } else {
                    w0 = ldg_nc_u32(mat + a.pa.off[2] + (rowb + ss) * 4);
                    w1 = 0;
                }
            };
            uint32_t s00 = 0, s01 = 0, s10 = 0, s11 = 0, s20 = 0, s21 = 0;
            sload(s00, s01, 0);
            sload(s10, s11, 1);
            bool inf = false, run = true;
            for (int ss = 0; ss < nss_p && run; ss++) {
                sload(s20, s21, ss + 2);
                const int sl = ss & 1;
                if (!mbar_wait(full_p(sl), (ss >> 1) & 1, abort_flag)) break;
                const uint8_t *slot = smem + C::PRING_OFF + sl * PT::SLOT;
                SPack<AFMT, GATEUP> cur;
                if constexpr (AFMT == DS4MOE_FMT_IQ2X) {
                    const uint4 *ip = reinterpret_cast<const uint4 *>(slot + m * 2 * M * 32 + R * 32);
                    const uint4 *sp = reinterpret_cast<const uint4 *>(slot + m * 2 * M * 32 + M * 32 + R * 32);
                    const uint4 i0 = ip[0], i1 = ip[1], g0 = sp[0], g1 = sp[1];
                    cur.w[0] = i0.x; cur.w[1] = i0.y; cur.w[2] = i0.z; cur.w[3] = i0.w;
                    cur.w[4] = i1.x; cur.w[5] = i1.y; cur.w[6] = i1.z; cur.w[7] = i1.w;
                    cur.w[8] = g0.x; cur.w[9] = g0.y; cur.w[10] = g0.z; cur.w[11] = g0.w;
                    cur.w[12] = g1.x; cur.w[13] = g1.y; cur.w[14] = g1.z; cur.w[15] = g1.w;
                    cur.w[16] = s00; cur.w[17] = s01;
                } else {
                    const uint8_t *q = slot + R * 64 + h * 8;
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const uint2 v = *reinterpret_cast<const uint2 *>(q + 16 * j);
                        cur.w[2 * j] = v.x; cur.w[2 * j + 1] = v.y;
                    }
                    const uint4 sc = *reinterpret_cast<const uint4 *>(slot + M * 64 + R * 16);
                    cur.w[8] = sc.x; cur.w[9] = sc.y; cur.w[10] = sc.z; cur.w[11] = sc.w;
                    cur.w[12] = s00;
                }
                // The slot is refilled by TMA (async proxy) as soon as every thread has arrived, and the words
                // just loaded are used only later: the proxy fence orders this thread's shared-memory reads
                // before that copy (without it, the last thread to arrive could see the next block's bytes).
                fence_proxy_async();
                mbar_arrive(empty_p(sl));
                s00 = s10; s01 = s11; s10 = s20; s11 = s21;
                constexpr int SPB = 4 / C::SUB;  // pipeline steps per 256-wide block
#pragma unroll
                for (int jj = 0; jj < SPB; jj++) {
                    const int kc = ss * SPB + jj;
                    const int s = kc % S;
                    const uint32_t par = ((kc / S) & 1) ^ 1;
                    if (!mbar_wait(empty(s), par, abort_flag)) {
                        run = false;
                        break;
                    }
                    begin_a();
#pragma unroll
                    for (int js = 0; js < C::SUB; js++) {
                        const int J = jj * C::SUB + js;  // 64-wide stage of the block
                        uint4 o[NOUT];
                        const float hsc = GATEUP ? 1.f : s_hsc[(kc * C::KS + js * BK) >> 7];
                        if (J == 0) sp_dequant<AFMT, GATEUP, 0>(cur, h, ss, tbl_lane, o, inf, hsc);
                        else if (J == 1) sp_dequant<AFMT, GATEUP, 1>(cur, h, ss, tbl_lane, o, inf, hsc);
                        else if (J == 2) sp_dequant<AFMT, GATEUP, 2>(cur, h, ss, tbl_lane, o, inf, hsc);
                        else sp_dequant<AFMT, GATEUP, 3>(cur, h, ss, tbl_lane, o, inf, hsc);
                        st_a(s, m, h, js, o);
                    }
                    end_a(s);
                }
            }
            if (inf) set_device_error(DS4MOE_EDEVICE);
        } else if constexpr (!DENSE) {
            constexpr int SS = SPackCfg<AFMT, GATEUP>::SS;
            constexpr int NOUT = GATEUP ? 8 : 4;
            const int at = tid - W_A0 * 32;  // 0 .. 255
            const int m = GATEUP ? at >> 7 : 0;
            const int R = GATEUP ? at & 127 : (C::ATM ? (warp & 3) * 32 + lane : at >> 1);  // as in the path above
            const int h = GATEUP ? 0 : (C::ATM ? (warp - W_A0) >> 2 : at & 1);
            const uint8_t *mat = GATEUP && m ? a.a1 + size_t(e) * a.a1_stride : a.a0 + size_t(e) * a.a_stride;
            const int row = blockIdx.x * M + R;
            const uint8_t *tbl_lane = tbl + (lane & 7) * 16;
            constexpr int SPP = SS / C::SUB;  // pipeline steps per packed super-stage
            static_assert(SS % C::SUB == 0, "a super-stage holds whole pipeline steps");
            const int nss = nk / SPP;
            // packed data of PF super-stages is in flight: super-stage ss+PF-1 is requested while ss is consumed
            // (two when two CTAs share the SM: their warps hide the latency, and the registers are halved)
            constexpr int PF = SPackCfg<AFMT, GATEUP>::NW <= 20 && C::MIN_BLOCKS == 1 ? 3 : 2;
            SPack<AFMT, GATEUP> pf[PF];
    #pragma unroll
            for (int p = 0; p < PF - 1; p++)
                if (p < nss) sp_load<AFMT, GATEUP>(pf[p], mat, a.pa, row, h, a.K, p);
            bool inf = false;
            bool run = true;
            for (int base = 0; base < nss && run; base += PF) {
    #pragma unroll
                for (int q = 0; q < PF; q++) {
                    const int ss = base + q;
                    if (ss >= nss || !run) break;
                    if (ss + PF - 1 < nss) sp_load<AFMT, GATEUP>(pf[(q + PF - 1) % PF], mat, a.pa, row, h, a.K, ss + PF - 1);
                    const SPack<AFMT, GATEUP> &cur = pf[q];
    #pragma unroll
                    for (int jj = 0; jj < SPP; jj++) {
                        const int kc = ss * SPP + jj;
                        const int s = kc % S;
                        const uint32_t par = ((kc / S) & 1) ^ 1;
                        if (!mbar_wait(empty(s), par, abort_flag)) {
                            run = false;
                            break;
                        }
                        begin_a();
    #pragma unroll
                        for (int js = 0; js < C::SUB; js++) {
                            const int J = jj * C::SUB + js;  // 64-wide stage of the super-stage
                            uint4 o[NOUT];
                            if constexpr (SS == 4) {
                                const float hsc = GATEUP ? 1.f : s_hsc[(kc * C::KS + js * BK) >> 7];
                                if (J == 0) sp_dequant<AFMT, GATEUP, 0>(cur, h, ss, tbl_lane, o, inf, hsc);
                                else if (J == 1) sp_dequant<AFMT, GATEUP, 1>(cur, h, ss, tbl_lane, o, inf, hsc);
                                else if (J == 2) sp_dequant<AFMT, GATEUP, 2>(cur, h, ss, tbl_lane, o, inf, hsc);
                                else sp_dequant<AFMT, GATEUP, 3>(cur, h, ss, tbl_lane, o, inf, hsc);
                            } else if constexpr (SS == 2) {
                                if (J == 0) sp_dequant<AFMT, GATEUP, 0>(cur, h, ss, tbl_lane, o, inf);
                                else sp_dequant<AFMT, GATEUP, 1>(cur, h, ss, tbl_lane, o, inf);
                            } else {
                                sp_dequant<AFMT, GATEUP, 0>(cur, h, ss, tbl_lane, o, inf);
                            }
                            st_a(s, m, h, js, o);
                        }
                        end_a(s);
                    }
                }
            }
            if (inf) set_device_error(DS4MOE_EDEVICE);
        }

        // ------------------------------------------------------------------ epilogue (warps 4..11)
        // Warps 4-7 and 8-11 cover the same TMEM lane quarters (warp & 3); they split the tile's token columns
        // in 32-wide chunks, so that two warps per scheduler hide each other's latencies.
        {
            const int q = warp & 3;  // TMEM lane quarter
            const int r = q * 32 + lane;
            const int c_first = ((warp - W_A0) >> 2) * 32;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(accum_bar, 0, abort_flag) && !*abort_flag);
            tc_fence_after();
            const uint32_t tq = tmem + (uint32_t(q * 32) << 16);
            if constexpr (GATEUP) {
                // h = silu(g) * u of the tile's rows and tokens.  fp16 h is stored as h * 2^-e with one e >= 0
                // per tile: e = 0 unless the tile's largest |h| exceeds the fp16 range, in which case the tile is
                // written again with max |h| * 2^-e in [2^14, 2^15) (bf16 output for the dense shared expert
                // needs no scale).  The down GEMM multiplies this K range of its weights by 2^e.
                constexpr bool F16OUT = AFMT != FMT_BF16D;
                auto store_pass = [&](float osc, uint32_t &amax_bits) {
                    for (int c0 = c_first; c0 < n_eff; c0 += 64) {
                        uint32_t g[32], u[32];
                        tmem_ld32(tq + c0, g);
                        tmem_ld32(tq + NT + c0, u);
#pragma unroll
                        for (int i = 0; i < 32; i++) {
                            const int n = c0 + i;
                            if (n < cnt) {
                                const float sc = s_colsc[n];
                                const float gv = __uint_as_float(g[i]) * sc, uv = __uint_as_float(u[i]) * sc;
                                const float hv = silu(gv) * uv;
                                amax_bits = max(amax_bits, __float_as_uint(hv) & 0x7FFFFFFFu);
                                const size_t o = size_t(pos0 + n) * a.ldo + blockIdx.x * M + r;
                                if constexpr (F16OUT) reinterpret_cast<__half *>(a.out)[o] = __float2half(hv * osc);
                                else reinterpret_cast<__nv_bfloat16 *>(a.out)[o] = __float2bfloat16_rn(hv);
                            }
                        }
                    }
                };
                uint32_t amax_bits = 0;  // |h| as float bits: NaN sorts above +inf
                if (ok) store_pass(1.f, amax_bits);
                amax_bits = __reduce_max_sync(0xffffffffu, amax_bits);
                if (lane == 0) atomicMax(&s_hmax, amax_bits);
                asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight epilogue warps
                const uint32_t tmax = *reinterpret_cast<volatile uint32_t *>(&s_hmax);
                int he = 0;
                if (tmax >= 0x7F800000u) {
                    if (ok && r == 0) set_device_error(DS4MOE_EDEVICE);  // inf / NaN in the tile
                } else if (F16OUT && tmax > 0x477FE000u) {                 // beyond 65504
                    int qe;
                    frexpf(__uint_as_float(tmax), &qe);
                    he = qe - 15;
                    uint32_t unused = 0;
                    if (ok) store_pass(ldexpf(1.f, -he), unused);
                }
                if (ok && r == 0 && c_first == 0 && a.h_exp_out) a.h_exp_out[int(blockIdx.y) * gridDim.x + blockIdx.x] = he;
            } else {
                if (ok) {
                    float *out = reinterpret_cast<float *>(a.out);
                    for (int c0 = c_first; c0 < n_eff; c0 += 64) {
                        uint32_t g[32];
                        tmem_ld32(tq + c0, g);
                        if (a.out_row) {
                            // fused combine: each warp adds 32 consecutive rows of one token (coalesced reductions)
#pragma unroll
                            for (int i = 0; i < 32; i++) {
                                const int n = c0 + i;
                                if (n < cnt) {
                                    float *dst = out + size_t(s_orow[n]) * a.ldo + blockIdx.x * M + r;
                                    const float v = __uint_as_float(g[i]) * s_colsc[n];
                                    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(dst), "f"(v) : "memory");
                                }
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; i++) {
                                const int n = c0 + i;
                                if (n < cnt) out[size_t(pos0 + n) * a.ldo + blockIdx.x * M + r] = __uint_as_float(g[i]) * s_colsc[n];
                            }
                        }
                    }
                }
            }
            tc_fence_before();
        }
    }

    __syncthreads();
    if (warp == 0) {
        // every MMA this CTA issued has completed once accum_bar flipped; after an abort wait (bounded) for it
        if (*abort_flag) {
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(accum_bar, 0) && globaltimer() - t0 < uint64_t(WAIT_NS)) {
            }
        }
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace ds4
