// ds4moe C ABI (include/ds4moe.h): argument checks, workspace carving and
// kernel launches.  One translation unit: the kernels live in the headers
// included below.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "decode_gemv.cuh"
#include "grouped_common.cuh"
#include "grouped_tc.cuh"
#include "permute.cuh"
#include "prepare.cuh"
#include "route.cuh"

using namespace ds4;

namespace {

#define DS4_CHECK_LAUNCH()                                          \
    do {                                                            \
        if (cudaGetLastError() != cudaSuccess) return DS4MOE_ECUDA; \
    } while (0)

inline cudaStream_t cs(ds4moe_stream s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }
inline uint64_t a256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 64 && cache[dev]) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cache[dev] = n;
    return n;
}

// Opt in to the dynamic shared memory a kernel needs (static + dynamic above 48 KB needs the attribute).  The
// attribute is per function and device and stays set, so each (kernel, device) pair is configured once for the
// largest size asked so far: a per-launch cudaFuncSetAttribute is a measurable share of a decode call.
template <typename Kern>
bool set_smem(Kern k, int bytes) {
    struct Entry {
        const void *fn;
        int dev, bytes;
    };
    static Entry cache[256];
    static int n = 0;
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const void *fn = reinterpret_cast<const void *>(k);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; i++)
        if (cache[i].fn == fn && cache[i].dev == dev) {
            if (cache[i].bytes >= bytes) return true;
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
            cache[i].bytes = bytes;
            return true;
        }
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    if (n < 256) cache[n++] = Entry{fn, dev, bytes};
    return true;
}

// Launch with programmatic dependent launch enabled (the kernel calls pdl_wait before consuming
// the previous kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- TMA tensor maps ----------------------------------------------------------------------------------------
//
// The tcgen05 kernels load their token operand (a row-major fp16 matrix, rows x cols) with 2D tensor copies:
// box = 64 columns (128 bytes, the swizzle span) x 128 rows, 128-byte swizzle, zero fill past the last row.
// The encoder comes from the driver through the runtime's entry-point query (no link against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        tried = true;
    }
    return fn;
}

// Row-major 16-bit matrix [rows x cols] (cols a multiple of 64) as a 2D TMA map with a 64 x 128 box.
bool make_tile_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, bool bf16) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc || !base || rows == 0 || cols % 64 || !aligned16(base)) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {uint32_t(tc::BK), uint32_t(tc::NT)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// One plane of E prepared matrices as a 3D byte map: (row_bytes, rows, E), expert stride in bytes; box
// (box_bytes, 128 rows, 1 expert), no swizzle.
bool make_plane_map(CUtensorMap *m, const void *base, uint64_t row_bytes, uint64_t rows, uint64_t E,
                    uint64_t expert_stride, uint32_t box_bytes) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc || !base || !aligned16(base) || row_bytes % 16 || expert_stride % 16 || box_bytes % 16) return false;
    const cuuint64_t dims[3] = {row_bytes, rows, E};
    const cuuint64_t strides[2] = {row_bytes, expert_stride};
    const cuuint32_t box[3] = {box_bytes, uint32_t(tc::M), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool fmt_quant(int f) { return f == DS4MOE_FMT_IQ2X || f == DS4MOE_FMT_Q2K || f == DS4MOE_FMT_Q4K; }

// The permutation's offset scan (perm_scan_kernel) is one CTA of 1024 threads, one per expert: the grouped path
// takes at most this many experts, and expert intermediate sizes f up to tc::MAX_K (the down GEMM keeps one
// scale per 128-wide K range on chip).
constexpr int MAX_E_GROUPED = 1024;
bool grouped_supported(const ds4moe_experts *ex) { return ex->E <= MAX_E_GROUPED && ex->f <= tc::MAX_K; }

ds4moe_status check_experts(const ds4moe_experts *ex) {
    if (!ex) return DS4MOE_EINVAL;
    if (ex->d <= 0 || ex->f <= 0 || ex->E <= 0 || ex->d % QK || ex->f % QK || ex->f_shared < 0 ||
        ex->f_shared % QK)
        return DS4MOE_EINVAL;
    if (!fmt_quant(ex->fmt_gate) || !fmt_quant(ex->fmt_down) || ex->fmt_up != ex->fmt_gate) return DS4MOE_EUNSUPPORTED;
    if (ex->fmt_gate == DS4MOE_FMT_Q2K) return DS4MOE_EUNSUPPORTED;  // gate/up: IQ2X or Q4K
    if (ex->fmt_down == DS4MOE_FMT_IQ2X) return DS4MOE_EUNSUPPORTED;  // down: Q2K or Q4K
    if (!ex->gate || !ex->up || !ex->down) return DS4MOE_EINVAL;
    if (!aligned256(ex->gate) || !aligned256(ex->up) || !aligned256(ex->down)) return DS4MOE_EINVAL;
    const uint64_t gb = ds4moe_prepared_bytes(ds4moe_fmt(ex->fmt_gate), ex->f, ex->d);
    const uint64_t db = ds4moe_prepared_bytes(ds4moe_fmt(ex->fmt_down), ex->d, ex->f);
    if (ex->gate_stride < gb || ex->up_stride < gb || ex->down_stride < db) return DS4MOE_EINVAL;
    if (ex->gate_stride % 256 || ex->up_stride % 256 || ex->down_stride % 256) return DS4MOE_EINVAL;
    if (ex->fmt_gate == DS4MOE_FMT_IQ2X && (!ex->codebook || !aligned16(ex->codebook))) return DS4MOE_EINVAL;
    if (ex->f_shared > 0) {
        if (!ex->sh_gate || !ex->sh_up || !ex->sh_down) return DS4MOE_EINVAL;
        if (!aligned16(ex->sh_gate) || !aligned16(ex->sh_up) || !aligned16(ex->sh_down)) return DS4MOE_EINVAL;
    }
    return DS4MOE_OK;
}

ExpertsDev to_dev(const ds4moe_experts *ex) {
    ExpertsDev e;
    e.d = ex->d; e.f = ex->f; e.E = ex->E; e.fs = ex->f_shared;
    e.fmt_gate = ex->fmt_gate; e.fmt_down = ex->fmt_down;
    e.gate = static_cast<const uint8_t *>(ex->gate);
    e.up = static_cast<const uint8_t *>(ex->up);
    e.down = static_cast<const uint8_t *>(ex->down);
    e.gate_stride = ex->gate_stride; e.up_stride = ex->up_stride; e.down_stride = ex->down_stride;
    e.codebook = ex->codebook;
    e.sh_gate = static_cast<const __nv_bfloat16 *>(ex->sh_gate);
    e.sh_up = static_cast<const __nv_bfloat16 *>(ex->sh_up);
    e.sh_down = static_cast<const __nv_bfloat16 *>(ex->sh_down);
    e.pg = plane_layout(ex->fmt_gate, uint64_t(ex->f) * (ex->d / QK));
    e.pd = plane_layout(ex->fmt_down, uint64_t(ex->d) * (ex->f / QK));
    return e;
}

// ---- workspace layouts -----------------------------------------------------------------------------

// The single-token GEMV kernels cover IQ2X gate/up with Q2K down, d <= 8192, and a down-kernel staging area
// that fits in shared memory; everything else runs the grouped path with one token.
bool decode_gemv_supported(const ds4moe_experts *ex, int k) {
    const bool iq = ex->fmt_gate == DS4MOE_FMT_IQ2X && ex->fmt_down == DS4MOE_FMT_Q2K;
    const bool q4 = ex->fmt_gate == DS4MOE_FMT_Q4K && ex->fmt_down == DS4MOE_FMT_Q4K;
    if (!(iq || q4) || k > 32) return false;
    if (!dg_supported_d(ex->d) || !dd_supported_f(ex->f)) return false;
    return dd_layout(k, ex->f, ex->f_shared, ex->fmt_down).total <= 200 * 1024;
}

// Decode batches of up to this many tokens run the single-token GEMV pair once per token (each pass streams its
// token's experts at the GEMV path's rate; see ds4moe_expert_ffn_decode), larger ones the grouped path.
constexpr int DECODE_GEMV_MAX_B = 16;

struct DecodeWs {
    uint64_t h, hs, total;  // h_j = silu(G_j x) * (U_j x) for the k experts [k x f]; shared expert's h [f_shared]
};
DecodeWs decode_ws(const ds4moe_experts *ex, int k) {
    DecodeWs w;
    w.h = 0;
    w.hs = a256(uint64_t(k) * ex->f * 4);
    w.total = w.hs + a256(uint64_t(ex->f_shared > 0 ? ex->f_shared : 1) * 4);
    return w;
}

struct GroupedWs {
    uint64_t x16, xinv, blk, counts, offsets, tile_e, tile_pos0, tile_cnt, meta, perm_tok, perm_w, x_perm, h16, hexp, hs;
    uint64_t inv;                    // inverse map of the fused-combine call (the caller's buffer otherwise)
    uint64_t y_perm, y_shared;       // only used when decode B > 16 runs through the grouped path
    uint64_t total_grouped, total_fused, total_decode;
    int nblk, max_tiles;
};
GroupedWs grouped_ws(const ds4moe_experts *ex, int T, int k) {
    GroupedWs w;
    const uint64_t N = uint64_t(T) * k;
    w.nblk = int((N + PERM_BLOCK - 1) / PERM_BLOCK);
    w.max_tiles = int(ex->E + (N + 63) / 64);  // >= the sum over experts of ceil(count / NT)
    uint64_t o = 0;
    auto take = [&](uint64_t bytes) {
        uint64_t r = o;
        o += a256(bytes > 0 ? bytes : 1);
        return r;
    };
    w.x16 = take(uint64_t(T) * ex->d * 2);
    w.xinv = take(uint64_t(T) * 4);
    w.blk = take(uint64_t(w.nblk > 0 ? w.nblk : 1) * ex->E * 4);
    w.counts = take(uint64_t(ex->E) * 4);
    w.offsets = take(uint64_t(ex->E) * 4);
    w.tile_e = take(uint64_t(w.max_tiles) * 4);
    w.tile_pos0 = take(uint64_t(w.max_tiles) * 4);
    w.tile_cnt = take(uint64_t(w.max_tiles) * 4);
    w.meta = take(16);
    w.perm_tok = take(N * 4);
    w.perm_w = take(N * 4);
    w.x_perm = take(N * ex->d * 2);
    w.h16 = take(N * ex->f * 2);
    w.hexp = take(uint64_t(w.max_tiles) * (ex->f / tc::M) * 4);  // fp16 h exponent per (token tile, row tile)
    w.hs = take(uint64_t(T) * (ex->f_shared > 0 ? ex->f_shared : 1) * 2);
    w.total_grouped = o;
    w.inv = take(N * 4);
    w.total_fused = o;
    w.y_perm = take(N * ex->d * 4);
    w.y_shared = take(uint64_t(T) * ex->d * 4);
    w.total_decode = o;
    return w;
}

// ---- grouped launch sequence --------------------------------------------------------------------------

// row_units: rows of one A matrix (f for gate/up, d for down); col_tiles: token tiles (upper bound).
// b_tma / b_rows: the token operand as the tcgen05 kernel reads it (row-major 16-bit, b_rows x ga.K).
// Dense A formats (tc::FMT_F16, tc::FMT_BF16D) also take their A matrices (ga.a0, ga.a1: row_units x ga.K) by TMA.
template <int AFMT, bool GATEUP>
ds4moe_status launch_grouped(const GroupedArgs &ga, int row_units, int col_tiles, const void *b_tma, uint64_t b_rows,
                             cudaStream_t st) {
    if (row_units <= 0 || col_tiles <= 0) return DS4MOE_OK;
    {
        constexpr bool bf16 = AFMT == tc::FMT_BF16D;
        CUtensorMap tb, ta0 = {}, ta1 = {};
        if (!make_tile_map(&tb, b_tma, b_rows, uint64_t(ga.K), bf16)) return DS4MOE_ECUDA;
        if (tc::is_dense<AFMT>()) {
            if (!make_tile_map(&ta0, ga.a0, uint64_t(row_units), uint64_t(ga.K), bf16)) return DS4MOE_ECUDA;
            if (GATEUP && !make_tile_map(&ta1, ga.a1, uint64_t(row_units), uint64_t(ga.K), bf16)) return DS4MOE_ECUDA;
        }
        CUtensorMap p0 = {}, p1 = {}, p2 = {}, p3 = {};
        if constexpr (tc::PackTma<AFMT, GATEUP>::ON) {
            const uint64_t K = uint64_t(ga.K), R = uint64_t(row_units), E = uint64_t(ga.n_mats);
            bool ok;
            if constexpr (AFMT == DS4MOE_FMT_IQ2X) {  // index and sign planes (K / 8 bytes per row) of gate and up
                ok = make_plane_map(&p0, ga.a0 + ga.pa.off[0], K / 8, R, E, ga.a_stride, 32) &&
                     make_plane_map(&p1, ga.a0 + ga.pa.off[1], K / 8, R, E, ga.a_stride, 32) &&
                     make_plane_map(&p2, ga.a1 + ga.pa.off[0], K / 8, R, E, ga.a1_stride, 32) &&
                     make_plane_map(&p3, ga.a1 + ga.pa.off[1], K / 8, R, E, ga.a1_stride, 32);
            } else {  // Q2K codes (K / 4 bytes per row) and scales (K / 16)
                ok = make_plane_map(&p0, ga.a0 + ga.pa.off[0], K / 4, R, E, ga.a_stride, 64) &&
                     make_plane_map(&p1, ga.a0 + ga.pa.off[1], K / 16, R, E, ga.a_stride, 16);
            }
            if (!ok) return DS4MOE_ECUDA;
        }
        auto kern = tc::grouped_tc_kernel<AFMT, GATEUP>;
        constexpr int smem = tc::Cfg<AFMT, GATEUP>::SMEM;
        if (!set_smem(kern, smem)) return DS4MOE_ECUDA;
        kern<<<dim3(row_units / tc::M, col_tiles), tc::THREADS, smem, st>>>(ga, tb, ta0, ta1, p0, p1, p2, p3);
    }
    DS4_CHECK_LAUNCH();
    return DS4MOE_OK;
}

// fused_out == NULL: routed rows to y_perm (position order) and the shared expert to y_shared, for ds4moe_combine.
// fused_out != NULL: the shared expert's output is stored into fused_out first (zeros without one), then the
// routed down GEMM adds each weighted row into its token's row of fused_out (y_perm, y_shared unused).
ds4moe_status run_grouped(const ds4moe_experts *ex, const void *x, int T, const int32_t *ids, const float *weights,
                          int k, float *y_perm, int32_t *inv_perm, float *y_shared, uint8_t *ws, cudaStream_t st,
                          float *fused_out = nullptr) {
    const GroupedWs W = grouped_ws(ex, T, k);
    const ExpertsDev D = to_dev(ex);
    const int N = T * k;
    __half *x16 = reinterpret_cast<__half *>(ws + W.x16);
    float *xinv = reinterpret_cast<float *>(ws + W.xinv);
    int32_t *blk = reinterpret_cast<int32_t *>(ws + W.blk);
    int32_t *counts = reinterpret_cast<int32_t *>(ws + W.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(ws + W.offsets);
    int32_t *tile_e = reinterpret_cast<int32_t *>(ws + W.tile_e);
    int32_t *tile_pos0 = reinterpret_cast<int32_t *>(ws + W.tile_pos0);
    int32_t *tile_cnt = reinterpret_cast<int32_t *>(ws + W.tile_cnt);
    int32_t *meta = reinterpret_cast<int32_t *>(ws + W.meta);
    int32_t *perm_tok = reinterpret_cast<int32_t *>(ws + W.perm_tok);
    float *perm_w = reinterpret_cast<float *>(ws + W.perm_w);
    __half *x_perm = reinterpret_cast<__half *>(ws + W.x_perm);
    __half *h16 = reinterpret_cast<__half *>(ws + W.h16);
    int32_t *hexp = reinterpret_cast<int32_t *>(ws + W.hexp);
    __half *hs = reinterpret_cast<__half *>(ws + W.hs);
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);

    prep_x_kernel<<<T, 256, 0, st>>>(xb, ex->d, x16, xinv);
    DS4_CHECK_LAUNCH();
    const size_t hist_smem = size_t(ex->E) * 4;
    perm_count_kernel<<<W.nblk, PERM_BLOCK, hist_smem, st>>>(ids, N, ex->E, blk);
    DS4_CHECK_LAUNCH();
    const int tile_n = tc::NT;
    perm_scan_kernel<<<1, 1024, 0, st>>>(blk, W.nblk, ex->E, tile_n, counts, offsets, tile_e, tile_pos0, tile_cnt,
                                         meta);
    DS4_CHECK_LAUNCH();
    perm_scatter_kernel<<<W.nblk, PERM_BLOCK, hist_smem, st>>>(ids, weights, N, k, ex->E, blk, perm_tok, perm_w,
                                                               inv_perm);
    DS4_CHECK_LAUNCH();
    gather_rows_kernel<<<(N + 7) / 8, 256, 0, st>>>(x16, ex->d, perm_tok, N, x_perm);
    DS4_CHECK_LAUNCH();

    auto shared_expert = [&](float *dst) -> ds4moe_status {
        const int ct = (T + tile_n - 1) / tile_n;
        // Shared expert, a dense bf16 SwiGLU: A and the tokens both come by TMA as bf16 (x as given, hs written
        // as bf16)
        GroupedArgs s1 = {};
        s1.a0 = static_cast<const uint8_t *>(ex->sh_gate); s1.a1 = static_cast<const uint8_t *>(ex->sh_up);
        s1.a_stride = 0; s1.rows = ex->f_shared; s1.K = ex->d;
        s1.b_src = x16; s1.b_colscale = nullptr; s1.n_pos = T; s1.out = hs; s1.ldo = ex->f_shared;
        const ds4moe_status r = launch_grouped<tc::FMT_BF16D, true>(s1, ex->f_shared, ct, xb, T, st);
        if (r != DS4MOE_OK) return r;
        GroupedArgs s2 = {};
        s2.a0 = static_cast<const uint8_t *>(ex->sh_down); s2.a_stride = 0; s2.rows = ex->d; s2.K = ex->f_shared;
        s2.b_src = hs; s2.n_pos = T; s2.out = dst; s2.ldo = ex->d;
        return launch_grouped<tc::FMT_BF16D, false>(s2, ex->d, ct, hs, T, st);
    };
    ds4moe_status s;
    if (fused_out) {  // the shared expert's rows (or zeros) first: the routed rows are added on top
        if (ex->f_shared > 0) s = shared_expert(fused_out);
        else s = cudaMemsetAsync(fused_out, 0, size_t(T) * ex->d * 4, st) == cudaSuccess ? DS4MOE_OK : DS4MOE_ECUDA;
        if (s != DS4MOE_OK) return s;
    }

    // routed GEMM-1: gate/up -> h16
    GroupedArgs g1 = {};
    g1.a0 = D.gate; g1.a1 = D.up; g1.a_stride = D.gate_stride; g1.a1_stride = D.up_stride; g1.pa = D.pg;
    g1.n_mats = ex->E;
    g1.rows = ex->f; g1.K = ex->d; g1.codebook = ex->codebook;
    g1.b_src = x16; g1.b_rowidx = perm_tok; g1.b_colscale = xinv;
    g1.tile_e = tile_e; g1.tile_pos0 = tile_pos0; g1.tile_cnt = tile_cnt; g1.n_tiles = meta;
    g1.out = h16; g1.ldo = ex->f; g1.h_exp_out = hexp;
    if (ex->fmt_gate == DS4MOE_FMT_IQ2X) s = launch_grouped<DS4MOE_FMT_IQ2X, true>(g1, ex->f, W.max_tiles, x_perm, N, st);
    else s = launch_grouped<DS4MOE_FMT_Q4K, true>(g1, ex->f, W.max_tiles, x_perm, N, st);
    if (s != DS4MOE_OK) return s;

    // routed GEMM-2: down -> y_perm (scaled by the routing weight)
    GroupedArgs g2 = {};
    g2.a0 = D.down; g2.a_stride = D.down_stride; g2.pa = D.pd; g2.rows = ex->d; g2.K = ex->f; g2.n_mats = ex->E;
    g2.b_src = h16; g2.b_rowidx = nullptr; g2.b_colscale = nullptr;
    g2.tile_e = tile_e; g2.tile_pos0 = tile_pos0; g2.tile_cnt = tile_cnt; g2.n_tiles = meta;
    g2.pos_weight = perm_w; g2.out = fused_out ? fused_out : y_perm; g2.ldo = ex->d; g2.h_exp_in = hexp;
    g2.out_row = fused_out ? perm_tok : nullptr;
    if (ex->fmt_down == DS4MOE_FMT_Q2K) s = launch_grouped<DS4MOE_FMT_Q2K, false>(g2, ex->d, W.max_tiles, h16, N, st);
    else s = launch_grouped<DS4MOE_FMT_Q4K, false>(g2, ex->d, W.max_tiles, h16, N, st);
    if (s != DS4MOE_OK) return s;
    if (!fused_out && ex->f_shared > 0) return shared_expert(y_shared);

    return DS4MOE_OK;
}

// ---- failure-path self-test: one thread waits, through the tensor-core kernel's bounded wait, on an mbarrier
// that nothing arrives at; the wait gives up after tc::WAIT_NS and records DS4MOE_ETIMEOUT.
__global__ void selftest_wait_timeout_kernel() {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)tc::mbar_wait(smem_u32(&bar), 0, &abort_flag);
}

// ---- scratch for the allocation-free decode entry point ------------------------------------------------
//
// Some callers cannot hand the library a workspace: code that must not call cudaMalloc at all
// (an engine whose memory planner already owns all of HBM and forbids any further allocation, a
// plugin host that exposes no allocator).  ds4moe_expert_ffn_decode_noalloc serves them from this
// fixed array instead.  Every GPU that loads the library holds it until the process exits.
constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(1) << 20;  // 1 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device.  The host-side symbol is only a stand-in, so the
// address is looked up once per device, with that device current, and cached.  Entries are atomics:
// host threads making their first call on a device at the same time may both look the address up (the
// same value), but never race on the entry.  A cached address does not survive cudaDeviceReset.
void *noalloc_scratch_on_current_device(ds4moe_status *st) {
    static std::atomic<void *> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();
        *st = DS4MOE_ECUDA;
        return nullptr;
    }
    void *p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            *st = DS4MOE_ECUDA;
            return nullptr;
        }
        cache[dev].store(p, std::memory_order_release);
    }
    *st = DS4MOE_OK;
    return p;
}

}  // namespace

// =======================================================================================================
extern "C" {

const char *ds4moe_status_string(ds4moe_status s) {
    switch (s) {
    case DS4MOE_OK: return "ok";
    case DS4MOE_EINVAL: return "invalid argument";
    case DS4MOE_EUNSUPPORTED: return "unsupported format or shape";
    case DS4MOE_ECUDA: return "CUDA error";
    case DS4MOE_ENOWORKSPACE: return "workspace too small";
    case DS4MOE_ETIMEOUT: return "device wait timed out";
    case DS4MOE_EDEVICE: return "device-side data error";
    }
    return "unknown status";
}

size_t ds4moe_prepared_bytes(ds4moe_fmt fmt, int rows, int cols) {
    if (!fmt_quant(fmt) || rows <= 0 || cols <= 0 || cols % QK) return 0;
    return plane_layout(fmt, uint64_t(rows) * (cols / QK)).total;
}

ds4moe_status ds4moe_prepare(ds4moe_fmt fmt, const void *canonical, void *prepared, int rows, int cols, int n_mats,
                             uint64_t prepared_stride, ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    if (!fmt_quant(fmt)) return DS4MOE_EUNSUPPORTED;
    if (!canonical || !prepared || rows <= 0 || cols <= 0 || cols % QK || n_mats < 0) return DS4MOE_EINVAL;
    if (!aligned256(prepared) || prepared_stride % 256 || prepared_stride < ds4moe_prepared_bytes(fmt, rows, cols))
        return DS4MOE_EINVAL;
    if (n_mats == 0) return DS4MOE_OK;
    const uint64_t nblk = uint64_t(rows) * (cols / QK);
    const uint64_t total = nblk * n_mats;
    const unsigned grid = unsigned((total + 255) / 256);
    if (fmt == DS4MOE_FMT_IQ2X)
        prepare_iq2x_kernel<<<grid, 256, 0, cs(stream)>>>(static_cast<const uint8_t *>(canonical),
                                                          static_cast<uint8_t *>(prepared), nblk, n_mats,
                                                          prepared_stride);
    else
        prepare_kquant_kernel<<<grid, 256, 0, cs(stream)>>>(static_cast<const uint8_t *>(canonical),
                                                            static_cast<uint8_t *>(prepared), nblk, n_mats,
                                                            prepared_stride, fmt);
    DS4_CHECK_LAUNCH();
    return DS4MOE_OK;
}

ds4moe_status ds4moe_dequant(ds4moe_fmt fmt, const void *prepared, const uint8_t *codebook, int rows, int cols,
                             float *out, ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    if (!fmt_quant(fmt)) return DS4MOE_EUNSUPPORTED;
    if (!prepared || !out || rows <= 0 || cols <= 0 || cols % QK || !aligned256(prepared)) return DS4MOE_EINVAL;
    if (fmt == DS4MOE_FMT_IQ2X && !codebook) return DS4MOE_EINVAL;
    const uint8_t *p = static_cast<const uint8_t *>(prepared);
    if (fmt == DS4MOE_FMT_IQ2X) {
        const uint64_t n = uint64_t(rows) * (cols / 8);
        dequant_iq2x_kernel<<<unsigned((n + 255) / 256), 256, 0, cs(stream)>>>(p, codebook, rows, cols, out);
    } else {
        const uint64_t n = uint64_t(rows) * (cols / (fmt == DS4MOE_FMT_Q2K ? 16 : 32));
        dequant_kquant_kernel<<<unsigned((n + 255) / 256), 256, 0, cs(stream)>>>(p, rows, cols, fmt, out);
    }
    DS4_CHECK_LAUNCH();
    return DS4MOE_OK;
}

// Router workspace: logits [T x E] fp32; for the tensor-core path (T > ROUTE_SMALL_T, E a multiple of 128)
// also the per-token scaled fp16 copy of x and its scales.
static bool route_tc(int T, int d, int E) { return T > ROUTE_SMALL_T && E % tc::M == 0 && d % QK == 0; }

size_t ds4moe_route_workspace_size(int T, int d, int E) {
    if (T < 0 || E <= 0 || d <= 0) return 0;
    const uint64_t TT = T > 0 ? T : 1;
    uint64_t n = a256(TT * E * 4);
    if (route_tc(T, d, E)) n += a256(TT * d * 2) + a256(TT * 4);
    return n;
}

ds4moe_status ds4moe_route(const void *x_bf16, int T, int d, const void *w_router_f16, const float *bias, int E,
                           int k, int32_t *ids, float *weights, void *ws, size_t ws_bytes, ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    if (T < 0 || d <= 0 || d % QK || E <= 0 || E > 1024 || k < 1 || k > E || k > 32) return DS4MOE_EINVAL;
    if (T == 0) return DS4MOE_OK;
    if (!x_bf16 || !w_router_f16 || !ids || !weights || !ws) return DS4MOE_EINVAL;
    if (!aligned16(x_bf16) || !aligned16(w_router_f16) || !aligned256(ws)) return DS4MOE_EINVAL;
    if (ws_bytes < ds4moe_route_workspace_size(T, d, E)) return DS4MOE_ENOWORKSPACE;
    float *logits = static_cast<float *>(ws);
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(x_bf16);
    const __half *wr = static_cast<const __half *>(w_router_f16);
    cudaStream_t st = cs(stream);
    const float *late_bias = nullptr;
    if (T <= ROUTE_SMALL_T) {
        route_logits_small_kernel<<<(E + 1) / 2, 256, 0, st>>>(x, T, d, wr, bias, E, logits);
    } else if (route_tc(T, d, E)) {
        // fp16 x fp16 products are exact on the tensor cores (W_r is fp16; x is scaled per token by a power of
        // two into fp16 range), accumulation in fp32: logits[t][e] = (W_r x16[t])[e] * 2^-e_t
        uint8_t *w8 = static_cast<uint8_t *>(ws);
        __half *x16 = reinterpret_cast<__half *>(w8 + a256(uint64_t(T) * E * 4));
        float *xinv = reinterpret_cast<float *>(w8 + a256(uint64_t(T) * E * 4) + a256(uint64_t(T) * d * 2));
        prep_x_kernel<<<T, 256, 0, st>>>(x, d, x16, xinv);
        DS4_CHECK_LAUNCH();
        GroupedArgs g = {};
        g.a0 = static_cast<const uint8_t *>(w_router_f16);
        g.a_stride = 0; g.rows = E; g.K = d;
        g.b_src = x16; g.b_colscale = xinv; g.n_pos = T;
        g.out = logits; g.ldo = E;
        const ds4moe_status rs = launch_grouped<tc::FMT_F16, false>(g, E, (T + tc::NT - 1) / tc::NT, x16, T, st);
        if (rs != DS4MOE_OK) return rs;
        late_bias = bias;
    } else {
        route_logits_tiled_kernel<<<dim3((T + 63) / 64, (E + 63) / 64), 256, 0, st>>>(x, T, d, wr, bias, E, logits);
    }
    DS4_CHECK_LAUNCH();
    const unsigned tg = unsigned((T + 7) / 8);
    cudaError_t err;
    const int per = E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : E <= 256 ? 8 : E <= 512 ? 16 : 32;
    switch (per) {
#define TOPK_CASE(P)                                                                                             \
    case P:                                                                                                      \
        err = launch_pdl(route_topk_kernel<P>, dim3(tg), dim3(256), 0, st, static_cast<const float *>(logits), T, \
                         E, k, late_bias, ids, weights);                                                         \
        break;
        TOPK_CASE(1) TOPK_CASE(2) TOPK_CASE(4) TOPK_CASE(8) TOPK_CASE(16) TOPK_CASE(32)
#undef TOPK_CASE
    default: return DS4MOE_EINVAL;
    }
    if (err != cudaSuccess) {
        (void)cudaGetLastError();
        return DS4MOE_ECUDA;
    }
    DS4_CHECK_LAUNCH();
    return DS4MOE_OK;
}

size_t ds4moe_workspace_size(const ds4moe_experts *ex, int T, int k) {
    if (check_experts(ex) != DS4MOE_OK || T < 0 || k < 1 || k > ex->E) return 0;
    const int TT = T > 0 ? T : 1;
    const bool gemv = decode_gemv_supported(ex, k);
    // the GEMV path gives each token of a decode batch its own h region
    const uint64_t gemv_need = gemv && TT <= DECODE_GEMV_MAX_B ? uint64_t(TT) * decode_ws(ex, k).total : 0;
    if (!grouped_supported(ex)) return gemv_need;  // no grouped path: only the GEMV path's batches
    uint64_t need = grouped_ws(ex, TT, k).total_decode;
    return need > gemv_need ? need : gemv_need;
}

ds4moe_status ds4moe_expert_ffn_decode(const ds4moe_experts *ex, const void *x_bf16, int B, const int32_t *ids,
                                       const float *weights, int k, float *out, void *ws, size_t ws_bytes,
                                       ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    ds4moe_status s = check_experts(ex);
    if (s != DS4MOE_OK) return s;
    if (B < 0 || k < 1 || k > ex->E) return DS4MOE_EINVAL;
    if (B == 0) return DS4MOE_OK;
    if (!x_bf16 || !ids || !weights || !out || !ws || !aligned16(x_bf16) || !aligned256(ws) || !aligned16(out))
        return DS4MOE_EINVAL;
    if (ws_bytes < ds4moe_workspace_size(ex, B, k)) return DS4MOE_ENOWORKSPACE;
    cudaStream_t st = cs(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    if (B <= DECODE_GEMV_MAX_B && decode_gemv_supported(ex, k)) {
        // token by token through the GEMV pair, each token with its own h region (256-byte aligned slices)
        const uint64_t per = decode_ws(ex, k).total;
        for (int t = 0; t < B; t++) {
            uint8_t *wt = w8 + uint64_t(t) * per;
            const void *xt = static_cast<const uint8_t *>(x_bf16) + size_t(t) * ex->d * 2;
            s = ds4moe_decode_gateup(ex, xt, ids + size_t(t) * k, k, wt, per, stream);
            if (s != DS4MOE_OK) return s;
            s = ds4moe_decode_down(ex, ids + size_t(t) * k, weights + size_t(t) * k, k, out + size_t(t) * ex->d, wt, per,
                                   stream);
            if (s != DS4MOE_OK) return s;
        }
        return DS4MOE_OK;
    }
    // B > 1 (or a format without a GEMV kernel): grouped path, then combine
    if (!grouped_supported(ex)) return ex->E > MAX_E_GROUPED ? DS4MOE_EINVAL : DS4MOE_EUNSUPPORTED;
    const GroupedWs W = grouped_ws(ex, B, k);
    float *y_perm = reinterpret_cast<float *>(w8 + W.y_perm);
    int32_t *inv = reinterpret_cast<int32_t *>(w8 + W.inv);
    float *y_sh = ex->f_shared > 0 ? reinterpret_cast<float *>(w8 + W.y_shared) : nullptr;
    s = run_grouped(ex, x_bf16, B, ids, weights, k, y_perm, inv, y_sh, w8, st);
    if (s != DS4MOE_OK) return s;
    return ds4moe_combine(y_perm, inv, y_sh, B, ex->d, k, out, stream);
}

ds4moe_status ds4moe_decode_gateup(const ds4moe_experts *ex, const void *x_bf16, const int32_t *ids, int k, void *ws,
                                   size_t ws_bytes, ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    ds4moe_status s = check_experts(ex);
    if (s != DS4MOE_OK) return s;
    if (k < 1 || k > ex->E) return DS4MOE_EINVAL;
    if (!decode_gemv_supported(ex, k)) return DS4MOE_EUNSUPPORTED;
    if (!x_bf16 || !ids || !ws || !aligned16(x_bf16) || !aligned256(ws)) return DS4MOE_EINVAL;
    const DecodeWs W = decode_ws(ex, k);
    if (ws_bytes < W.total) return DS4MOE_ENOWORKSPACE;
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    const ExpertsDev D = to_dev(ex);
    float *h = reinterpret_cast<float *>(w8 + W.h);
    float *hs = reinterpret_cast<float *>(w8 + W.hs);
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(x_bf16);
    const int smem = dg_smem_bytes(ex->d);
    const int vpp = ex->d / QK < 8 ? ex->d / QK : 8;  // 8-vectors of a row per lane and pass
    using GK = void (*)(const ExpertsDev, const __nv_bfloat16 *, const int32_t *, int, float *, float *);
    GK kern;
    if (ex->fmt_gate == DS4MOE_FMT_Q4K)
        kern = vpp == 8 ? decode_gateup_kernel<DS4MOE_FMT_Q4K, 8, DG_ROWS> : vpp == 4 ? decode_gateup_kernel<DS4MOE_FMT_Q4K, 4, DG_ROWS>
             : vpp == 2 ? decode_gateup_kernel<DS4MOE_FMT_Q4K, 2, DG_ROWS> : decode_gateup_kernel<DS4MOE_FMT_Q4K, 1, DG_ROWS>;
    else
        kern = vpp == 8 ? decode_gateup_kernel<DS4MOE_FMT_IQ2X, 8, DG_ROWS> : vpp == 4 ? decode_gateup_kernel<DS4MOE_FMT_IQ2X, 4, DG_ROWS>
             : vpp == 2 ? decode_gateup_kernel<DS4MOE_FMT_IQ2X, 2, DG_ROWS> : decode_gateup_kernel<DS4MOE_FMT_IQ2X, 1, DG_ROWS>;
    if (!set_smem(kern, smem)) return DS4MOE_ECUDA;
    const cudaError_t err =
        launch_pdl(kern, dim3(num_sms()), dim3(DG_THREADS), size_t(smem), cs(stream), D, x, ids, k, h, hs);
    if (err != cudaSuccess) {
        (void)cudaGetLastError();
        return DS4MOE_ECUDA;
    }
    return DS4MOE_OK;
}

ds4moe_status ds4moe_decode_down(const ds4moe_experts *ex, const int32_t *ids, const float *weights, int k, float *out,
                                 void *ws, size_t ws_bytes, ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    ds4moe_status s = check_experts(ex);
    if (s != DS4MOE_OK) return s;
    if (k < 1 || k > ex->E) return DS4MOE_EINVAL;
    if (!decode_gemv_supported(ex, k)) return DS4MOE_EUNSUPPORTED;
    if (!ids || !weights || !out || !ws || !aligned16(out) || !aligned256(ws)) return DS4MOE_EINVAL;
    const DecodeWs W = decode_ws(ex, k);
    if (ws_bytes < W.total) return DS4MOE_ENOWORKSPACE;
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    const ExpertsDev D = to_dev(ex);
    const float *h = reinterpret_cast<const float *>(w8 + W.h);
    const float *hs = reinterpret_cast<const float *>(w8 + W.hs);
    const int smem = dd_layout(k, ex->f, ex->f_shared, ex->fmt_down).total;
    const int epl = dd_epl(ex->f, ex->fmt_down);  // weights of a row per lane and pass
    using DK = void (*)(const ExpertsDev, const float *, const float *, const int32_t *, const float *, int, float *);
    DK kern;
    if (ex->fmt_down == DS4MOE_FMT_Q4K)
        kern = epl == 32 ? decode_down_kernel<DS4MOE_FMT_Q4K, 32> : epl == 16 ? decode_down_kernel<DS4MOE_FMT_Q4K, 16>
                         : decode_down_kernel<DS4MOE_FMT_Q4K, 8>;
    else
        kern = epl == 64 ? decode_down_kernel<DS4MOE_FMT_Q2K, 64> : epl == 32 ? decode_down_kernel<DS4MOE_FMT_Q2K, 32>
             : epl == 16 ? decode_down_kernel<DS4MOE_FMT_Q2K, 16> : decode_down_kernel<DS4MOE_FMT_Q2K, 8>;
    if (!set_smem(kern, smem)) return DS4MOE_ECUDA;
    const cudaError_t err = launch_pdl(kern, dim3(num_sms()), dim3(DD_THREADS), size_t(smem), cs(stream), D, h, hs,
                                       ids, weights, k, out);
    if (err != cudaSuccess) {
        (void)cudaGetLastError();
        return DS4MOE_ECUDA;
    }
    return DS4MOE_OK;
}

ds4moe_status ds4moe_expert_ffn_decode_noalloc(const ds4moe_experts *ex, const void *x_bf16, const int32_t *ids,
                                               const float *weights, int k, float *out, ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    ds4moe_status s = check_experts(ex);
    if (s != DS4MOE_OK) return s;
    if (k < 1 || k > ex->E) return DS4MOE_EINVAL;
    if (!decode_gemv_supported(ex, k)) return DS4MOE_EUNSUPPORTED;
    if (!x_bf16 || !ids || !weights || !out || !aligned16(x_bf16) || !aligned16(out)) return DS4MOE_EINVAL;
    const uint64_t need = decode_ws(ex, k).total;
    if (need > NOALLOC_SCRATCH_BYTES) return DS4MOE_ENOWORKSPACE;  // layer too large for the fixed scratch
    void *scratch = noalloc_scratch_on_current_device(&s);
    if (s != DS4MOE_OK) return s;
    // the gate/up kernel overwrites every scratch word the down kernel reads: nothing to clear
    s = ds4moe_decode_gateup(ex, x_bf16, ids, k, scratch, NOALLOC_SCRATCH_BYTES, stream);
    if (s != DS4MOE_OK) return s;
    return ds4moe_decode_down(ex, ids, weights, k, out, scratch, NOALLOC_SCRATCH_BYTES, stream);
}

ds4moe_status ds4moe_expert_ffn_grouped(const ds4moe_experts *ex, const void *x_bf16, int T, const int32_t *ids,
                                        const float *weights, int k, float *y_perm, int32_t *inv_perm,
                                        float *y_shared, void *ws, size_t ws_bytes, ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    ds4moe_status s = check_experts(ex);
    if (s != DS4MOE_OK) return s;
    if (T < 0 || k < 1 || k > ex->E || ex->E > MAX_E_GROUPED) return DS4MOE_EINVAL;
    if (!grouped_supported(ex)) return DS4MOE_EUNSUPPORTED;
    if (T == 0) return DS4MOE_OK;
    if (!x_bf16 || !ids || !weights || !y_perm || !inv_perm || !ws || !aligned16(x_bf16) || !aligned256(ws) ||
        !aligned16(y_perm))
        return DS4MOE_EINVAL;
    if (ex->f_shared > 0 && (!y_shared || !aligned16(y_shared))) return DS4MOE_EINVAL;
    if (ws_bytes < grouped_ws(ex, T, k).total_grouped) return DS4MOE_ENOWORKSPACE;
    return run_grouped(ex, x_bf16, T, ids, weights, k, y_perm, inv_perm, ex->f_shared > 0 ? y_shared : nullptr,
                       static_cast<uint8_t *>(ws), cs(stream));
}

ds4moe_status ds4moe_expert_ffn_grouped_fused(const ds4moe_experts *ex, const void *x_bf16, int T, const int32_t *ids,
                                              const float *weights, int k, float *out, void *ws, size_t ws_bytes,
                                              ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launches
    ds4moe_status s = check_experts(ex);
    if (s != DS4MOE_OK) return s;
    if (T < 0 || k < 1 || k > ex->E || ex->E > MAX_E_GROUPED) return DS4MOE_EINVAL;
    if (!grouped_supported(ex)) return DS4MOE_EUNSUPPORTED;
    if (T == 0) return DS4MOE_OK;
    if (!x_bf16 || !ids || !weights || !out || !ws || !aligned16(x_bf16) || !aligned256(ws) || !aligned16(out))
        return DS4MOE_EINVAL;
    const GroupedWs W = grouped_ws(ex, T, k);
    if (ws_bytes < W.total_fused) return DS4MOE_ENOWORKSPACE;
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    return run_grouped(ex, x_bf16, T, ids, weights, k, nullptr, reinterpret_cast<int32_t *>(w8 + W.inv), nullptr, w8,
                       cs(stream), out);
}

ds4moe_status ds4moe_combine(const float *y_perm, const int32_t *inv_perm, const float *y_shared, int T, int d, int k,
                             float *out, ds4moe_stream stream) {
    if (T < 0 || d <= 0 || d % 4 || k < 1) return DS4MOE_EINVAL;
    if (T == 0) return DS4MOE_OK;
    if (!y_perm || !inv_perm || !out || !aligned16(y_perm) || !aligned16(out)) return DS4MOE_EINVAL;
    if (y_shared && !aligned16(y_shared)) return DS4MOE_EINVAL;
    const uint64_t total = uint64_t(T) * (d / 4);
    const unsigned grid = unsigned(std::min<uint64_t>((total + 255) / 256, uint64_t(num_sms()) * 16));
    combine_kernel<<<grid, 256, 0, cs(stream)>>>(y_perm, inv_perm, y_shared, T, d, k, out);
    DS4_CHECK_LAUNCH();
    return DS4MOE_OK;
}

ds4moe_status ds4moe_selftest_wait_timeout(ds4moe_stream stream) {
    (void)cudaGetLastError();  // report only errors raised by this call's launch
    selftest_wait_timeout_kernel<<<1, 32, 0, cs(stream)>>>();
    DS4_CHECK_LAUNCH();
    return DS4MOE_OK;
}

ds4moe_status ds4moe_last_device_error(ds4moe_stream stream, int32_t *code) {
    if (!code) return DS4MOE_EINVAL;
    if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return DS4MOE_ECUDA;
    int32_t v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return DS4MOE_ECUDA;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return DS4MOE_ECUDA;
    *code = v;
    return DS4MOE_OK;
}

}  // extern "C"
