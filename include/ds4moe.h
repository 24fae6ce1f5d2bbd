/*
 * ds4moe — routed Mixture-of-Experts FFN with 2-bit block-quantized experts,
 * for NVIDIA B200 (sm_100a).  C ABI.
 *
 * What it computes (ds4 news summary, "model weights" section; upppp.jp,
 * "asymmetric 2-bit quantization" section): a MoE FFN layer in which only the
 * routed experts are quantized -- gate/up in an IQ2_XXS-style codebook layout,
 * down in a Q2_K-style layout (a Q4_K-style 4-bit variant is the pages' "q4"
 * model, ds4 news summary "speed benchmarks") -- while the shared expert and
 * the router stay in high precision (bf16 shared expert, fp16 router).
 *
 *   l_e  = sum_i W_r[e,i] x_i + b_e            (router logit)
 *   s_e  = 1 / (1 + exp(-l_e))                 (sigmoid score)
 *   S    = the k largest s_e, descending, ties -> smaller e
 *   w_j  = s_{S_j} / sum_j' s_{S_j'}           (renormalised gate)
 *   y_j  = D_e (silu(G_e x) * (U_e x))         (SwiGLU expert, e = S_j)
 *   y_s  = Ds (silu(Gs x) * (Us x))            (shared expert, weight 1)
 *   out  = y_s + sum_j w_j y_j
 *
 * Conventions for every call:
 *  - All pointers are DEVICE pointers owned by the caller unless stated; the
 *    library never allocates device or pinned memory.  Scratch comes from a
 *    caller-provided workspace whose size the *_workspace_size calls return.
 *  - Calls are asynchronous on the given stream (NULL = legacy default
 *    stream) and never block, throw or abort.  Host-side argument checks
 *    (shapes, null pointers, 16-byte alignment, formats) return
 *    DS4MOE_EINVAL / DS4MOE_EUNSUPPORTED before anything is launched; a failed
 *    launch returns DS4MOE_ECUDA.
 *  - Data errors found on the device do not trap: they set a per-device
 *    error word that ds4moe_last_device_error() reads and clears.  What each
 *    kernel checks:
 *      DS4MOE_EDEVICE  an expert id outside [0, E): the decode gate/up and
 *                      down kernels (that expert's rows are skipped) and the
 *                      permutation of the grouped path (the pair is dropped);
 *                      a non-finite SwiGLU output, or a scaled weight that
 *                      would leave the fp16 range, in the grouped path's
 *                      tensor-core kernels (see ds4moe_expert_ffn_grouped);
 *      DS4MOE_ETIMEOUT a bounded wait (2 s) that ran out in the grouped
 *                      path's tensor-core kernels (producer/consumer
 *                      mbarrier pipeline).
 *    The decode kernels need no fp16 range check: their fp16 sums are
 *    bounded for any finite input (activations are scaled per token by a
 *    power of two so that max |x| lies in [32, 64); an fp16 lane adds at
 *    most 16 products of a codebook value <= 43 and |x| < 64, i.e. less than
 *    44,032, or 4 products of q <= 3 and |h| < 64).
 *  - Matrices are [out x in], row-major; quantization blocks of 256 weights
 *    run along the input (contraction) dimension, so d and f are multiples of
 *    256.  Activations x are bf16 [T x d]; the layer output is fp32 [T x d]
 *    (a bf16 output could not carry the layer to its accuracy bar: rounding
 *    the exact result to bf16 alone moves the largest outputs by up to
 *    ~3% of the output rms).
 */
#ifndef DS4MOE_H
#define DS4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *ds4moe_stream; /* the same type as cudaStream_t */

typedef enum {
    DS4MOE_OK = 0,
    DS4MOE_EINVAL = 1,        /* bad shape, null pointer, misalignment */
    DS4MOE_EUNSUPPORTED = 2,  /* format or shape combination not implemented */
    DS4MOE_ECUDA = 3,         /* a CUDA launch or runtime call failed */
    DS4MOE_ENOWORKSPACE = 4,  /* workspace smaller than *_workspace_size() */
    DS4MOE_ETIMEOUT = 5,      /* (device error word) a bounded wait gave up */
    DS4MOE_EDEVICE = 6        /* (device error word) bad id / fp16 overflow */
} ds4moe_status;

/* Weight formats.
 *
 * CANONICAL block layouts (little endian; 256 weights per block; what the
 * caller hands to ds4moe_prepare):
 *   IQ2X, 66 B: fp16 d (bytes 0-1), then 8 groups of 32 weights, each
 *        { idx[4] u8, aux u32 }.  aux bits 7j..7j+6 = signs of elements 0..6
 *        of 8-vector j (1 = negative); the sign of element 7 is the parity of
 *        those 7 bits (every 8-vector has an even number of negatives); aux
 *        bits 28..31 = scale s.  Weight 32g+8j+i =
 *        ((d * (0.5 + s)) * 0.25) * codebook[idx[j]][i] * sign.
 *   Q2K, 84 B: scales[16] (low nibble sc, high nibble m; one per 16 weights),
 *        qs[64] (weight i in byte i>>2, bits 2*(i&3)), fp16 d, fp16 dmin.
 *        w = d*sc*q - dmin*m.
 *   Q4K, 144 B: fp16 d, fp16 dmin, 12 scale bytes forming a 96-bit little
 *        endian bit string (sc_j at bits 6j..6j+5, m_j at 48+6j..48+6j+5, one
 *        pair per 32 weights), qs[128] (weight i in byte i>>1, low nibble
 *        first).  w = d*sc*q - dmin*m.
 *   BF16: plain row-major bfloat16 (shared expert only; never prepared).
 *
 * PREPARED layout (what the compute calls read; written by ds4moe_prepare):
 * one matrix [rows x cols], nblk = rows*cols/256 blocks numbered row-major,
 * split into planes; each plane starts at a 256-byte aligned offset from the
 * matrix base, in the order listed:
 *   IQ2X: IDX  nblk*32 B  (one codebook index per 8-vector)
 *         SGN  nblk*32 B  (u32 per 32-weight group: all 32 signs, the
 *                          parity sign made explicit; sign of element 2p of
 *                          vector j at bit 15-(4j+p), of element 2p+1 at bit
 *                          31-(4j+p))
 *         SCL  nblk*4 B   (u32 per block: nibble g = scale s of group g)
 *         D    nblk*2 B   (fp16 d)                  -> 70 B per block
 *   Q2K:  QS nblk*64 B | SC nblk*16 B | DM nblk*4 B (d, dmin)  -> 84 B per block
 *   Q4K:  QS nblk*128 B | SC nblk*12 B | DM nblk*4 B           -> 144 B per block
 */
typedef enum {
    DS4MOE_FMT_IQ2X = 0,
    DS4MOE_FMT_Q2K = 1,
    DS4MOE_FMT_Q4K = 2,
    DS4MOE_FMT_BF16 = 3
} ds4moe_fmt;

/* One layer's experts.  All pointers are device pointers owned by the caller
 * and must stay valid while calls using this struct run.  Routed expert e's
 * prepared gate matrix [f x d] starts at gate + e * gate_stride (bytes), and
 * likewise up [f x d] and down [d x f].  Strides must be multiples of 256.
 * codebook: 256 x 8 uint8 values (entries in {8, 25, 43} in the reference
 * workloads), required when any format is IQ2X.  sh_gate / sh_up: bf16
 * [f_shared x d]; sh_down: bf16 [d x f_shared]; all NULL (and f_shared = 0)
 * when the layer has no shared expert. */
typedef struct ds4moe_experts {
    int32_t d, f, E, f_shared;
    int32_t fmt_gate, fmt_up, fmt_down; /* ds4moe_fmt; gate and up must match */
    const void *gate, *up, *down;
    uint64_t gate_stride, up_stride, down_stride;
    const uint8_t *codebook;
    const void *sh_gate, *sh_up, *sh_down;
} ds4moe_experts;

/* Human-readable name of a status code (static storage). */
const char *ds4moe_status_string(ds4moe_status s);

/* Bytes of one prepared matrix [rows x cols] in `fmt` (0 if unsupported or
 * cols is not a multiple of 256). */
size_t ds4moe_prepared_bytes(ds4moe_fmt fmt, int rows, int cols);

/* Repack n_mats canonical matrices (each rows*cols/256 consecutive blocks,
 * matrix m at canonical + m*rows*(cols/256)*block_bytes) into the prepared
 * layout at prepared + m*prepared_stride.  prepared_stride >=
 * ds4moe_prepared_bytes() and a multiple of 256; prepared 256-byte aligned.
 * The block layouts are defined above; the repacking is lossless.
 * Passage: the IQ2_XXS / Q2_K / Q4_K-style expert formats (ds4 news summary,
 * "model weights"; upppp.jp, "asymmetric 2-bit quantization"); the prepared
 * plane split is this library's own layout, with no counterpart there. */
ds4moe_status ds4moe_prepare(ds4moe_fmt fmt, const void *canonical, void *prepared, int rows, int cols, int n_mats,
                             uint64_t prepared_stride, ds4moe_stream stream);

/* Exact fp32 dequantization of one prepared matrix into out[rows x cols]
 * (row-major).  Every value equals the block definition evaluated in fp32:
 * all products are exact and the Q2K/Q4K subtraction rounds once, so the
 * result is bit-exact whatever the evaluation order.  Test / export call.
 * Passage: the same expert formats as ds4moe_prepare. */
ds4moe_status ds4moe_dequant(ds4moe_fmt fmt, const void *prepared, const uint8_t *codebook, int rows, int cols,
                             float *out, ds4moe_stream stream);

/* Router (gating).  x: bf16 [T x d]; w_router: fp16 [E x d]; bias: fp32 [E]
 * or NULL (added to the logit before the sigmoid).  Writes ids int32 [T x k]
 * (descending score, ties to the smaller id) and weights fp32 [T x k]
 * (renormalised to sum 1).  Products fp16 x bf16 are exact in fp32 and the
 * dot products accumulate in fp32: on CUDA cores for T <= 8 (and for E not a
 * multiple of 128), otherwise on the tensor cores with x scaled per token by
 * a power of two into fp16 (exact products, fp32 accumulation).  The top-k
 * kernel is launched with programmatic dependent launch after the logits.
 * 1 <= k <= min(E, 32), E <= 1024, d multiple of 256.  The workspace
 * (ds4moe_route_workspace_size bytes, 256-byte aligned) holds the logits and,
 * on the tensor-core path, the scaled activations; a smaller one is refused
 * with DS4MOE_ENOWORKSPACE.  Passage: the router is one of the parts left
 * unquantized (ds4 news summary, "model weights"); the pages do not give its
 * function, and this library reads it as the sigmoid -> top-k -> renormalise
 * rule written at the top of this file.
 * ds4moe_route_workspace_size: bytes of the router's workspace for T tokens (a
 * library detail with no counterpart in the pages; 0 for invalid sizes). */
size_t ds4moe_route_workspace_size(int T, int d, int E);
ds4moe_status ds4moe_route(const void *x_bf16, int T, int d, const void *w_router_f16, const float *bias, int E,
                           int k, int32_t *ids, float *weights, void *ws, size_t ws_bytes, ds4moe_stream stream);

/* Workspace for ds4moe_expert_ffn_decode / ds4moe_expert_ffn_grouped with T
 * tokens (B for decode) and top-k.  Alignment: 256 bytes.  Returns 0 when the
 * layer or sizes are invalid, or when the call would need the grouped path
 * and the layer is beyond its limits (E > 1024 or f > 16384).  A library
 * detail with no counterpart in the pages (the pages describe no library
 * interface). */
size_t ds4moe_workspace_size(const ds4moe_experts *ex, int T, int k);

/* Decode: out[B x d] (fp32) = the full layer output for B tokens, given the
 * routing (ids, weights) from ds4moe_route.
 *  - GEMV path, for 1 <= B <= 16 when the layer is IQ2X gate/up with Q2K
 *    down, or Q4K throughout, d and f are 256 times a power of two with
 *    d <= 8192 and f <= 8192,
 *    k <= 32, and the down kernel's staging of h fits in shared memory: per
 *    token, each selected expert's packed rows are streamed once and
 *    dequantized on the fly, gate/up fused with SwiGLU, down fused with the
 *    weighted combine and the shared expert.  Tokens run one after another,
 *    each with its own h region of the workspace; for such small batches this
 *    beats the grouped tensor-core path, whose tiles would hold one or two
 *    tokens each.  x_bf16 is read before the wait on the preceding kernel (see
 *    ds4moe_decode_gateup), so x must not be written by the kernel launched
 *    just before this call on the same stream; ds4moe_route between the two
 *    satisfies this.
 *  - Grouped path, for B > 16 and for every layer the GEMV path does not
 *    take: the permuted grouped GEMMs of ds4moe_expert_ffn_grouped (each
 *    touched expert read once), then the combine; E <= 1024, else
 *    DS4MOE_EINVAL.
 * Passage: the expert FFN with quantized routed experts and an unquantized
 * shared expert (ds4 news summary, "model weights"; upppp.jp, "asymmetric
 * 2-bit quantization"); single-token generation speed is the pages' headline
 * figure (ds4 news summary, "speed benchmarks"). */
ds4moe_status ds4moe_expert_ffn_decode(const ds4moe_experts *ex, const void *x_bf16, int B, const int32_t *ids,
                                       const float *weights, int k, float *out, void *ws, size_t ws_bytes,
                                       ds4moe_stream stream);

/* The two launches of ds4moe_expert_ffn_decode's single-token GEMV path,
 * exposed so a caller can place other work or timing events between them
 * (B = 1; same layer limits as that path; same experts, workspace and stream
 * for both).  Passage: the same expert FFN as ds4moe_expert_ffn_decode (ds4
 * news summary, "model weights"); the split into two launches is this
 * library's, with no counterpart in the pages.  ds4moe_decode_gateup streams the k selected experts' gate/up
 * rows and the shared expert's gate/up rows and leaves h_j = silu(G_j x) *
 * (U_j x) (fp32, k x f) and the shared expert's hs (fp32, f_shared) at the
 * start of the workspace; ds4moe_decode_down reads them and writes
 * out[d] = sum_j w_j D_j h_j + Ds hs (fp32).  Both are launched with
 * programmatic dependent launch: the gate/up kernel reads x and streams the
 * shared expert before it waits for the preceding kernel (normally the
 * router's top-k, which produces ids), so x must be complete before that
 * kernel starts; the down kernel reads nothing before its wait. */
ds4moe_status ds4moe_decode_gateup(const ds4moe_experts *ex, const void *x_bf16, const int32_t *ids, int k, void *ws,
                                   size_t ws_bytes, ds4moe_stream stream);
ds4moe_status ds4moe_decode_down(const ds4moe_experts *ex, const int32_t *ids, const float *weights, int k,
                                 float *out, void *ws, size_t ws_bytes, ds4moe_stream stream);

/* Single-token decode without a caller workspace, for callers that cannot
 * allocate device memory at all: an engine whose memory planner has taken all
 * of HBM and forbids further allocation, or a plugin host that exposes no
 * allocator.  The pages have no counterpart: this is a library convenience.
 * Same computation and arguments as ds4moe_expert_ffn_decode with B = 1 (and
 * the same layer limits as ds4moe_decode_gateup), but the scratch comes from
 * a 1 MiB array compiled into the library, which every GPU that loads the
 * library holds until the process exits.  Layers outside the GEMV path's
 * limits are rejected with DS4MOE_EUNSUPPORTED, and a layer whose decode
 * scratch (4 * (k*f + f_shared) bytes, each part rounded up to 256) exceeds
 * 1 MiB with DS4MOE_ENOWORKSPACE (under the present limits every supported
 * layer fits: the down kernel stages all k experts' h and the shared
 * expert's in shared memory, which bounds the scratch far below 1 MiB).  Nothing is allocated: no cudaMalloc, no
 * cudaFree.  The first call on a device looks up the array's device address
 * (once per device, with that device current) and caches it; make that
 * first call before any stream capture.  The cached address does not survive
 * cudaDeviceReset: do not use this entry point again after a reset.  All calls share the one array, which keeps the last
 * call's contents: calls whose kernels overlap on the GPU (other streams,
 * other threads) race on it, so serialize them. */
ds4moe_status ds4moe_expert_ffn_decode_noalloc(const ds4moe_experts *ex, const void *x_bf16, const int32_t *ids,
                                               const float *weights, int k, float *out, ds4moe_stream stream);

/* Prefill / many tokens.  Permutes the T*k (token, slot) pairs by expert id
 * (stable: increasing token, then slot), runs the grouped dequantize-GEMM
 * SwiGLU experts and writes
 *   y_perm  fp32 [T*k x d]: row p = w_(t,j) * y_(t,j) for the pair at
 *           permuted position p,
 *   inv_perm int32 [T*k]:   inv_perm[t*k + j] = p,
 *   y_shared fp32 [T x d]:  the shared expert's output (may be NULL iff the
 *           layer has no shared expert).
 * Follow with ds4moe_combine.  Limits: E <= 1024 (DS4MOE_EINVAL beyond),
 * f <= 16384 (DS4MOE_EUNSUPPORTED beyond).  The SwiGLU output between the
 * two expert GEMMs is kept in fp16 scaled by a power of two per 128-token
 * tile and 128-row block (1 unless the block's largest |h| exceeds 65,504),
 * and the down GEMM multiplies that block's weights back, so a large h is
 * computed exactly as a small one; DS4MOE_EDEVICE is set only for a
 * non-finite h or a scaled weight beyond the fp16 range.  Passage: the same
 * expert FFN as ds4moe_expert_ffn_decode, for prompt processing (prefill
 * speed, ds4 news summary, "speed benchmarks"); the permuted grouped form is
 * this library's design. */
ds4moe_status ds4moe_expert_ffn_grouped(const ds4moe_experts *ex, const void *x_bf16, int T, const int32_t *ids,
                                        const float *weights, int k, float *y_perm, int32_t *inv_perm,
                                        float *y_shared, void *ws, size_t ws_bytes, ds4moe_stream stream);

/* Prefill with the combine fused into the routed down GEMM: out[T x d] (fp32)
 * = the full layer output, with no y_perm, inv_perm or y_shared.  The shared
 * expert's output is stored into out first (zeros when the layer has none);
 * the routed down GEMM's epilogue then adds each weighted row w_(t,j) y_(t,j)
 * straight into out[t] with fp32 atomic adds.  The k additions to a row come
 * from different CTAs in no fixed order, so results agree with
 * ds4moe_expert_ffn_grouped + ds4moe_combine only up to fp32 rounding of the
 * summation order and may differ in the last bits from run to run.  Same
 * limits and h scaling as ds4moe_expert_ffn_grouped; out is 16-byte aligned
 * and must not overlap x or the workspace; the workspace may be smaller
 * (ds4moe_workspace_size is enough).  Passage: the weighted combine of the
 * expert outputs in the layer formula at the top of this file (ds4 news
 * summary, "model weights"); the pages fix no summation order. */
ds4moe_status ds4moe_expert_ffn_grouped_fused(const ds4moe_experts *ex, const void *x_bf16, int T,
                                              const int32_t *ids, const float *weights, int k, float *out, void *ws,
                                              size_t ws_bytes, ds4moe_stream stream);

/* out[t] = y_shared[t] + sum_{j<k} y_perm[inv_perm[t*k+j]] (j in increasing
 * order, fp32).  y_shared may be NULL.  d multiple of 4.  This is the last
 * line of the layer formula at the top of this file; the pages fix no
 * summation order, so j runs in increasing order for a deterministic result. */
ds4moe_status ds4moe_combine(const float *y_perm, const int32_t *inv_perm, const float *y_shared, int T, int d,
                             int k, float *out, ds4moe_stream stream);

/* Self-test of the device failure path (no counterpart in the pages): one
 * CTA whose thread waits, through the same bounded mbarrier wait the
 * tensor-core kernels use, on a barrier nothing arrives at.  The wait gives
 * up after 2 s and records DS4MOE_ETIMEOUT in the device error word (read it
 * with ds4moe_last_device_error); the context stays usable.  Asynchronous on
 * the stream; nothing traps or faults. */
ds4moe_status ds4moe_selftest_wait_timeout(ds4moe_stream stream);

/* Synchronizes `stream`, then reads and clears the calling device's error
 * word: *code = 0 (none), or the ds4moe_status of the first device-side
 * error since the last read (DS4MOE_EDEVICE / DS4MOE_ETIMEOUT). */
ds4moe_status ds4moe_last_device_error(ds4moe_stream stream, int32_t *code);

#ifdef __cplusplus
}
#endif
#endif /* DS4MOE_H */
