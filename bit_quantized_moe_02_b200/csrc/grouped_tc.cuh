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
//   warps 1-3   gather the tile's token rows (fp16 activations or SwiGLU
//               outputs) with cp.async into 128B-swizzled K-major stages.
//   warps 4-11  stream the packed 2-bit (or 4-bit) blocks, dequantize them in
//               registers (shared-memory codebook / sign-bit XOR / fp16 scale)
//               and write fp16 tiles in the same swizzled K-major layout the
//               MMA descriptor describes.  Warps 4-7 then run the epilogue:
//               tcgen05.ld the accumulators, SwiGLU (gate/up) or routing-weight
//               scaling (down), coalesced stores.
//
// Gate and up share one work item: two accumulators (TMEM columns [0,128) and
// [128,256)) hold matching rows, so each epilogue thread owns a gate/up pair.
// Every wait on an mbarrier is bounded; a timeout records DS4MOE_ETIMEOUT,
// stops the CTA's roles and still frees TMEM before returning.
#pragma once
#include "common.cuh"
#include "grouped_mma.cuh"

namespace ds4 {
namespace tc {

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

template <bool GATEUP>
struct Cfg {
    static constexpr int STAGES = GATEUP ? 3 : 4;
    static constexpr int STAGE = (GATEUP ? 2 : 1) * A_TILE + B_TILE;
    static constexpr int TMEM_COLS = GATEUP ? 256 : 128;
    static constexpr int TABLE_OFF = STAGES * STAGE;
    static constexpr int SMEM = TABLE_OFF + TABLE_BYTES + 1024;  // + alignment slack
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

// Instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 accumulator, M = 128, N = n.
__device__ __forceinline__ uint32_t instr_desc(int n) {
    return (1u << 4) | (uint32_t(n >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
        "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_le(int n) {
    // n is small and uniform; branch to the immediate forms
    if (n <= 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
    else if (n == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else if (n == 2) asm volatile("cp.async.wait_group 2;" ::: "memory");
    else asm volatile("cp.async.wait_group 3;" ::: "memory");
}

// ---- the kernel -------------------------------------------------------------------------------------------

template <int AFMT, bool GATEUP>
__global__ void __launch_bounds__(THREADS, 1) grouped_tc_kernel(GroupedArgs a) {
    using C = Cfg<GATEUP>;
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *tbl = smem + C::TABLE_OFF;
    __shared__ __align__(8) uint64_t bars[3 * 4 + 1];  // full_a[S], full_b[S], empty[S], accum
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int32_t s_brow[NT];
    __shared__ float s_colsc[NT];

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
    const int nk = a.K / BK;

    auto full_a = [&](int s) { return smem_u32(&bars[s]); };
    auto full_b = [&](int s) { return smem_u32(&bars[4 + s]); };
    auto empty = [&](int s) { return smem_u32(&bars[8 + s]); };
    const uint32_t accum_bar = smem_u32(&bars[12]);

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(full_a(s), N_WA);
            mbar_init(full_b(s), N_WB);
            mbar_init(empty(s), 1);
        }
        mbar_init(accum_bar, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&s_tmem), C::TMEM_COLS);
        tc_fence_before();
    }
    if (tid < NT) {
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
            const uint32_t idesc = instr_desc(n_eff);
            bool ok = true;
            for (int kc = 0; kc < nk && ok; kc++) {
                const int s = kc % S;
                const uint32_t par = (kc / S) & 1;
                ok = mbar_wait(full_a(s), par, abort_flag) && mbar_wait(full_b(s), par, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * C::STAGE);
                const uint32_t a0 = st, a1 = st + A_TILE, b0 = st + (GATEUP ? 2 : 1) * A_TILE;
#pragma unroll
                for (int kk = 0; kk < BK / 16; kk++) {
                    const uint32_t acc = (kc > 0 || kk > 0) ? 1u : 0u;
                    mma_f16(tmem, smem_desc(a0 + kk * 32), smem_desc(b0 + kk * 32), idesc, acc);
                    if constexpr (GATEUP) mma_f16(tmem + NT, smem_desc(a1 + kk * 32), smem_desc(b0 + kk * 32), idesc, acc);
                }
                mma_commit(empty(s));
            }
            mma_commit(accum_bar);  // also covers an aborted loop: the epilogue / teardown waits on it
        }
        __syncwarp();
    } else if (warp < W_B0 + N_WB) {
        // ------------------------------------------------------------------ token-row loaders (cp.async)
        const int bt = tid - W_B0 * 32;  // 0 .. 95
        const uint8_t *bsrc = reinterpret_cast<const uint8_t *>(a.b_src);
        const int nrow = cnt;
        int lag_arrive = 0;  // next stage index whose arrival is pending
        for (int kc = 0; kc < nk; kc++) {
            const int s = kc % S;
            const uint32_t par = ((kc / S) & 1) ^ 1;
            if (!mbar_wait(empty(s), par, abort_flag)) break;
            const uint32_t bst = smem_u32(smem + s * C::STAGE + (GATEUP ? 2 : 1) * A_TILE);
            for (int job = bt; job < nrow * 8; job += N_WB * 32) {
                const int n = job >> 3, c = job & 7;
                cp_async16(bst + swz(n, c), bsrc + (size_t(s_brow[n]) * a.K + kc * BK + c * 8) * 2, 16);
            }
            cp_async_commit();
            if (kc - lag_arrive >= S - 1) {
                cp_async_wait_le(S - 1);
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(full_b(lag_arrive % S));
                lag_arrive++;
            }
        }
        cp_async_wait_le(0);
        fence_proxy_async();
        __syncwarp();
        for (; lag_arrive < nk; lag_arrive++)
            if (lane == 0) mbar_arrive(full_b(lag_arrive % S));
    } else {
        // ------------------------------------------------------------------ dequantizing producers
        const int at = tid - W_A0 * 32;  // 0 .. 255
        const int R = at >> 1, hh = at & 1;
        const uint8_t *mat0 = a.a0 + size_t(e) * a.a_stride;
        const uint8_t *mat1 = GATEUP ? a.a1 + size_t(e) * a.a_stride : nullptr;
        const int row = (GATEUP ? blockIdx.x * M : blockIdx.x * M) + R;
        const uint8_t *tbl_lane = tbl + (lane & 7) * 16;
        APack p0, p1;
        a_load<AFMT>(p0, mat0, a.pa, row, a.K, hh * 32);
        if constexpr (GATEUP) a_load<AFMT>(p1, mat1, a.pa, row, a.K, hh * 32);
        for (int kc = 0; kc < nk; kc++) {
            const int s = kc % S;
            const uint32_t par = ((kc / S) & 1) ^ 1;
            if (!mbar_wait(empty(s), par, abort_flag)) break;
            uint8_t *ast = smem + s * C::STAGE;
            uint4 o[4];
            bool inf = false;
            a_dequant<AFMT, 128>(p0, tbl_lane, kc * BK + hh * 32, o, inf);
#pragma unroll
            for (int j = 0; j < 4; j++) *reinterpret_cast<uint4 *>(ast + swz(R, hh * 4 + j)) = o[j];
            if constexpr (GATEUP) {
                a_dequant<AFMT, 128>(p1, tbl_lane, kc * BK + hh * 32, o, inf);
#pragma unroll
                for (int j = 0; j < 4; j++) *reinterpret_cast<uint4 *>(ast + A_TILE + swz(R, hh * 4 + j)) = o[j];
            }
            if (inf) set_device_error(DS4MOE_EDEVICE);
            if (kc + 1 < nk) {
                a_load<AFMT>(p0, mat0, a.pa, row, a.K, (kc + 1) * BK + hh * 32);
                if constexpr (GATEUP) a_load<AFMT>(p1, mat1, a.pa, row, a.K, (kc + 1) * BK + hh * 32);
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(full_a(s));
        }

        // ------------------------------------------------------------------ epilogue (warps 4..7)
        if (warp < W_A0 + 4) {
            const int q = warp - W_A0;  // TMEM lane quarter
            const int r = q * 32 + lane;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(accum_bar, 0, abort_flag) && !*abort_flag);
            tc_fence_after();
            if (ok) {
                const uint32_t tq = tmem + (uint32_t(q * 32) << 16);
                for (int c0 = 0; c0 < n_eff; c0 += 32) {
                    uint32_t g[32];
                    tmem_ld32(tq + c0, g);
                    if constexpr (GATEUP) {
                        uint32_t u[32];
                        tmem_ld32(tq + NT + c0, u);
                        __half *out = reinterpret_cast<__half *>(a.out);
                        bool overflow = false;
#pragma unroll
                        for (int i = 0; i < 32; i++) {
                            const int n = c0 + i;
                            if (n < cnt) {
                                const float sc = s_colsc[n];
                                const float gv = __uint_as_float(g[i]) * sc, uv = __uint_as_float(u[i]) * sc;
                                const float hv = silu(gv) * uv;
                                overflow |= !(fabsf(hv) <= 65504.f);
                                out[size_t(pos0 + n) * a.ldo + blockIdx.x * M + r] = __float2half(hv);
                            }
                        }
                        if (overflow) set_device_error(DS4MOE_EDEVICE);
                    } else {
                        float *out = reinterpret_cast<float *>(a.out);
#pragma unroll
                        for (int i = 0; i < 32; i++) {
                            const int n = c0 + i;
                            if (n < cnt) out[size_t(pos0 + n) * a.ldo + blockIdx.x * M + r] = __uint_as_float(g[i]) * s_colsc[n];
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
