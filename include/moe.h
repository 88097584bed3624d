/*
 * moe.h — C ABI of the B200 (sm_100a) MoE FFN layer forward.
 *
 * The layer (one GPU, forward only), as the pages define it:
 *   router logits  z = x @ W_r^T                       "MoE" chapter index (llm-infra-atlas),
 *                                                      §0 data-path diagram; routing primer §三
 *   scores         s = softmax(z_t) | sigmoid(z)       "MoE 路由入门：从 Dense FFN 到 GroupedTopK" §三
 *   selection      top-K of c = s + bias (bias only    "MoE" §0 ("+bias, only for selection"), §2.2;
 *                  chooses), optionally group-limited  routing primer §六, §七, §九, §十
 *   weights        s of the chosen experts, renormal-  routing primer §四
 *                  ised, times routed_scale
 *   dispatch       P = T*K pairs bucketed by expert    routing primer §5.1
 *   expert FFN     W_down (SiLU(W_gate x) * W_up x)    routing primer §一, §5.2; MoE optimisation
 *                                                      blog ("MoE 优化的探索…") §1
 *   combine        out_t = sum_k w_tk y_tk (+ shared)  routing primer §5.3; "MoE" §0
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major, unless a
 *     function says HOST.  The library never allocates device memory: scratch comes from
 *     the caller's workspace `ws` of at least moe_workspace_size() bytes, 256-byte aligned.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream) and does no host synchronisation, except where stated.
 *   - Argument errors are returned synchronously as a moe_status_t and nothing is
 *     launched.  Errors found by a kernel (an expert id out of range, a pipeline wait that
 *     timed out) are OR-ed into a status word inside `ws`; read it with
 *     moe_get_device_status().  No kernel traps.
 *   - Base pointers of bf16 / e4m3 matrices must be 16-byte aligned (e2m1 weights:
 *     32-byte); H and I must be multiples of 128.
 *   - "FP8" below means both dtypes with e4m3 activations (MOE_DTYPE_FP8_E4M3 and
 *     MOE_DTYPE_FP8_FP4).
 *   - Weight layout is [out_features, in_features] (nn.Linear): W_r [E,H];
 *     W_gate, W_up [E,I,H]; W_down [E,H,I]; shared expert Ws_gate, Ws_up [I_shared,H],
 *     Ws_down [H,I_shared].
 *   - dtype MOE_DTYPE_BF16: x, weights, outputs bf16; fp32 accumulation.
 *     dtype MOE_DTYPE_FP8_E4M3: x is e4m3 [T,H] with fp32 power-of-two scales
 *     x_scale [T,H/128] (one per token and 128 channels); expert weights are e4m3 with
 *     fp32 scales per 128x128 block ([E,I/128,H/128] for gate/up, [E,H/128,I/128] for
 *     down); W_r stays bf16; the output is bf16.
 *     dtype MOE_DTYPE_FP8_FP4 (the FP8 x FP4 GEMM of "DeepGEMM质变…" §5.3, the Mega MoE
 *     compute unit): x as for FP8; expert weights are e2m1 (OCP MX FP4), two per byte
 *     (element 2j in the low nibble: W_gate, W_up [E,I,H/2] bytes, W_down [E,H,I/2]),
 *     base pointers 32-byte aligned, with one UE8M0 scale (2^(byte-127)) per row and 32
 *     consecutive K elements, passed as the atoms moe_prepare_fp4_scales() makes.  No
 *     shared expert, block_m 128.
 *   - Weight scale arguments (void*): fp32 block scales for MOE_DTYPE_FP8_E4M3, prepared
 *     atoms for MOE_DTYPE_FP8_FP4, ignored (may be NULL) for MOE_DTYPE_BF16.
 *   - Empty batch: T = 0 is valid.  After the parameter and workspace checks every call
 *     returns MOE_OK, and arrays with a T or T*K dimension are not touched (they may be
 *     NULL).  Outputs sized by E still describe the empty batch: moe_permute writes
 *     counts (all 0), offsets_padded and, masked, pair_of_row (all -1);
 *     moe_layer_forward zeroes counts_out when it is given.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 6

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer, small workspace */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. H not a multiple of 128)   */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, attribute, copy)        */
  MOE_ERR_TIMEOUT = 4,      /* device: a bounded pipeline wait gave up                     */
  MOE_ERR_DEVICE = 5        /* device: bad input found by a kernel (expert id out of range) */
} moe_status_t;

/* Bits of the device status word (moe_get_device_status). */
#define MOE_DEV_BAD_EXPERT_ID 0x1   /* a topk id outside [0,E): the pair was skipped      */
#define MOE_DEV_TIMEOUT 0x2         /* a GEMM pipeline wait exceeded its limit and exited */
#define MOE_DEV_CAPACITY 0x4        /* masked layout: an expert had more than masked_cap    */
                                    /* pairs; the pairs past it got no row (left out)       */
#define MOE_DEV_RANGE 0x8           /* moe_layer_forward at prefill sizes keeps the routed  */
                                    /* (and shared) expert outputs in fp16; one exceeded    */
                                    /* |y| = 65504                                          */

enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 };
enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_FP8_E4M3 = 1, MOE_DTYPE_FP8_FP4 = 2 };

typedef struct moe_params {
  int32_t T;            /* tokens                                                        */
  int32_t H;            /* hidden size (multiple of 128)                                 */
  int32_t I;            /* intermediate size of a routed expert (multiple of 128)        */
  int32_t E;            /* routed experts, 1..1024                                       */
  int32_t K;            /* experts per token, 1..min(E,32)                               */
  int32_t n_group;      /* expert groups for group-limited top-k (1 = plain top-k)       */
  int32_t topk_group;   /* groups kept                                                   */
  int32_t group_topn;   /* group score = sum of the group_topn largest selection scores  */
  int32_t score_fn;     /* MOE_SCORE_SOFTMAX or MOE_SCORE_SIGMOID                        */
  int32_t renormalize;  /* 1: divide the chosen weights by their sum                     */
  float routed_scale;   /* factor applied to the (renormalised) weights                  */
  int32_t I_shared;     /* intermediate size of the shared expert, 0 = none              */
  int32_t dtype;        /* MOE_DTYPE_BF16, MOE_DTYPE_FP8_E4M3 or MOE_DTYPE_FP8_FP4       */
  int32_t block_m;      /* row alignment of each expert's bucket: 128 (one-SM GEMM tiles), */
                        /* 256 (two-SM cta_group::2 tiles: a third less SM-side operand  */
                        /* traffic, more pad rows), 0 = default (128)                    */
  int32_t fused_combine; /* moe_layer_forward only, bf16, block_m 128: 0 = separate,     */
                        /* deterministic combine (default); 1 = the down projection adds */
                        /* w * y straight into an fp32 token accumulator with atomic     */
                        /* vector reductions (no y_perm round trip; run-to-run bits vary)*/
  int32_t masked_cap;   /* bucket layout ("MoE" chapter index §1, grouped-GEMM entry):   */
                        /* 0 = contiguous (expert e's bucket starts at offsets_padded[e],*/
                        /* a multiple of block_m, and holds exactly its pairs); > 0 =    */
                        /* masked: expert e owns the fixed rows [e*cap, (e+1)*cap), its  */
                        /* counts[e] pairs fill the first of them, the rest are unused.  */
                        /* cap is a multiple of 128, block_m must be 128.  An expert     */
                        /* with more than cap pairs keeps the first cap (in pair order)  */
                        /* and sets MOE_DEV_CAPACITY; cap >= T never drops a pair.       */
} moe_params_t;

/* ---------------------------------------------------------------------------------- */
/* Sizes                                                                               */
/* ---------------------------------------------------------------------------------- */

/* Bytes of workspace a moe_layer_forward() call needs (the per-stage calls need at most
 * this much).  0 if the parameters are invalid. */
size_t moe_workspace_size(const moe_params_t* p);

/* Bytes of workspace moe_layer_forward_host() and moe_layer_forward_host_batches() need:
 * moe_workspace_size() plus two device staging slots for the copied activations and
 * outputs.  0 if the parameters are invalid. */
size_t moe_workspace_size_host(const moe_params_t* p);

/* Bucket alignment the calls use for these parameters (128 or 256); -1 if invalid. */
int32_t moe_effective_block_m(const moe_params_t* p);

/* Row capacity that pair_of_row, x_perm and y_perm must have: the bound P + E*(block_m-1)
 * on the padded row count (contiguous layout), or E*masked_cap (masked layout).  -1 if
 * the parameters are invalid. */
int64_t moe_max_padded_rows(const moe_params_t* p);

/* ---------------------------------------------------------------------------------- */
/* Stage 1 — routing.  Routing primer §三 (router, scores), §四 (top-k, renormalise),   */
/* §六-§十 (group-limited top-k); "MoE" §0 (selection-only bias).                      */
/*   x        [T,H] bf16, or e4m3 codes with x_scale [T,H/128] (FP8 dtype)              */
/*   w_r      [E,H] bf16;  bias [E] fp32 or NULL                                        */
/*   topk_ids [T,K] int32 out: experts in descending selection score (ties: lower id)   */
/*   topk_w   [T,K] fp32 out: weights from the unbiased scores                          */
/* Uses ws for the logits (and, for FP8, a bf16 copy of x).                            */
/* ---------------------------------------------------------------------------------- */
moe_status_t moe_route(const moe_params_t* p, const void* x, const float* x_scale,
                       const void* w_r, const float* bias, int32_t* topk_ids, float* topk_w,
                       void* ws, size_t ws_bytes, void* stream);

/* GroupedTopK on given router logits [T,E] fp32 (routing primer §九, §十: the op takes
 * the logits and returns K weights and ids per token; x is not read).  Same scoring,
 * selection and weighting as moe_route; no workspace. */
moe_status_t moe_grouped_topk(const moe_params_t* p, const float* logits, const float* bias,
                              int32_t* topk_ids, float* topk_w, void* stream);

/* Auxiliary-loss-free balancing bias, one update from the per-expert loads ("MoE"
 * chapter index §2.2): bias[e] += gamma * sign(mean_e'(counts) - counts[e]).  counts [E]
 * int32 (e.g. the counts moe_permute writes), bias [E] fp32 updated in place.  The
 * bias only steers selection (moe_route); the weights never see it. */
moe_status_t moe_aux_free_bias_update(const int32_t* counts, int32_t E, float gamma,
                                      float* bias, void* stream);

/* ---------------------------------------------------------------------------------- */
/* Stage 2 — dispatch (routing primer §5.1).  Buckets the pairs p = t*K + k by expert,  */
/* stably in p, each bucket starting at a multiple of block_m.                          */
/*   topk_ids       [T,K] int32 in                                                      */
/*   counts         [E] int32 out: pairs per expert                                     */
/*   offsets_padded [E+1] int32 out: first row of each bucket; offsets_padded[E] = rows */
/*   row_of_pair    [T*K] int32 out                                                     */
/*   pair_of_row    [moe_max_padded_rows] int32 out: pair of each row, -1 on pad rows   */
/*   x_perm         [moe_max_padded_rows, H] out: x[t] copied to each pair's row, pad   */
/*                  rows zero (bf16, or e4m3 codes + x_perm_scale [rows, H/128] fp32)   */
/* An id outside [0,E) sets MOE_DEV_BAD_EXPERT_ID and that pair is left out.            */
/* Masked layout (masked_cap > 0): offsets_padded[e] = e*cap; counts[e] = rows in use,  */
/* min(pairs of e, cap); a pair past cap gets row_of_pair = -1 (MOE_DEV_CAPACITY); the  */
/* unused rows get pair_of_row = -1 but their x_perm rows are not written.              */
/* ---------------------------------------------------------------------------------- */
moe_status_t moe_permute(const moe_params_t* p, const int32_t* topk_ids, const void* x,
                         const float* x_scale, int32_t* counts, int32_t* offsets_padded,
                         int32_t* row_of_pair, int32_t* pair_of_row, void* x_perm,
                         float* x_perm_scale, void* ws, size_t ws_bytes, void* stream);

/* Allocation-free variant of moe_permute.  The pages have no counterpart: this entry
 * point exists for callers that cannot give the library device memory of its own
 * (plug-ins inside a host framework that owns all device memory and offers no scratch
 * hook; serving loops where a cudaMalloc or allocator round trip is not allowed).  It
 * takes the same inputs and outputs as moe_permute but no workspace: the per-chunk
 * expert histogram lives in a fixed 1 MiB file-scope device array that every GPU using
 * the library holds until the process exits.
 *   - Limit: ceil(T*K/256) * E <= 262144, else MOE_ERR_UNSUPPORTED (nothing launched).
 *   - device_status: optional device int32 the caller has zeroed; MOE_DEV_BAD_EXPERT_ID
 *     is OR-ed into it (NULL: not reported; bad pairs still get row_of_pair = -1).
 *   - All calls share the one array: calls that overlap on the GPU (other streams,
 *     other host threads on the same device) race.  Serialise them on one stream.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress with that device current); make that first call before
 *     any stream capture.  No call allocates or frees device memory. */
moe_status_t moe_permute_noalloc(const moe_params_t* p, const int32_t* topk_ids, const void* x,
                                 const float* x_scale, int32_t* counts, int32_t* offsets_padded,
                                 int32_t* row_of_pair, int32_t* pair_of_row, void* x_perm,
                                 float* x_perm_scale, int32_t* device_status, void* stream);

/* ---------------------------------------------------------------------------------- */
/* Stage 3 — expert FFN on the bucketed rows (routing primer §5.2; M-grouped GEMM as    */
/* in the "MoE" chapter index §1, grouped GEMM entry).                                  */
/*   y_perm[r] = W_down[e] (SiLU(W_gate[e] x_perm[r]) * W_up[e] x_perm[r])              */
/* for every row r of expert e's bucket (pad rows included; their result is unused).    */
/*   offsets_padded [E+1], counts [E] as written by moe_permute (read on the device     */
/*                  only); counts may be NULL, then pad rows are computed and stored too */
/*                  Masked layout: counts (the rows in use of each expert) is required   */
/*                  and offsets_padded may be NULL (then e*cap); 128-row tiles wholly    */
/*                  past counts[e] are skipped by every kernel                           */
/*   y_perm [moe_max_padded_rows, H] out, fp32 for MOE_DTYPE_BF16 and bf16 for FP8; rows */
/*                  past counts[e] in a bucket are not written when counts is given     */
/* The SwiGLU intermediate h (bf16, or e4m3 + scales) lives in ws.  For bf16 workloads  */
/* y_perm stays fp32 because it feeds the output directly and the final bf16 rounding   */
/* already uses most of the 2e-2 RMS error budget; the FP8 bound (6e-2) leaves room for */
/* a bf16 y_perm, which halves its HBM round trip.                                      */
/* ---------------------------------------------------------------------------------- */
moe_status_t moe_expert_ffn(const moe_params_t* p, const void* x_perm, const float* x_perm_scale,
                            const int32_t* offsets_padded, const int32_t* counts,
                            const void* w_gate, const void* w_up, const void* w_down,
                            const void* w_gate_scale, const void* w_up_scale,
                            const void* w_down_scale, void* y_perm, void* ws, size_t ws_bytes,
                            void* stream);

/* Dense SwiGLU FFN of the always-active shared expert on all T tokens ("MoE" §0, §2.1):
 *   y_shared [T,H] fp32 = Ws_down (SiLU(Ws_gate x) * Ws_up x).   bf16 dtype only. */
moe_status_t moe_shared_expert_ffn(const moe_params_t* p, const void* x, const void* ws_gate,
                                   const void* ws_up, const void* ws_down, float* y_shared,
                                   void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------- */
/* Stage 4 — combine (routing primer §5.3): out[t] = sum_k w[t,k] y_perm[row_of_pair[   */
/* t*K+k]] (+ y_shared[t]), fp32 accumulation in fixed k order, one rounding to bf16.   */
/* y_perm [rows,H] as moe_expert_ffn writes it (fp32, or bf16 for FP8); y_shared [T,H]  */
/* fp32 or NULL; out [T,H] bf16.  Pairs                                                 */
/* with row_of_pair = -1 are left out.  No atomics: bitwise reproducible.               */
/* ---------------------------------------------------------------------------------- */
moe_status_t moe_combine(const moe_params_t* p, const void* y_perm, const int32_t* row_of_pair,
                         const float* topk_w, const float* y_shared, void* out, void* stream);

/* ---------------------------------------------------------------------------------- */
/* The whole layer: route -> permute -> expert FFN -> [shared expert] -> combine, all   */
/* on `stream`, with no host synchronisation.  out [T,H] bf16.                          */
/* topk_ids_out [T,K], topk_w_out [T,K], counts_out [E] are optional copies of the      */
/* routing decision (NULL: kept in ws only).  ws_gate/ws_up/ws_down are the shared      */
/* expert's weights (required iff I_shared > 0).  For bf16 layers with T*K >= 256*E and */
/* H a multiple of 256, the routed experts' outputs pass to the combine in fp16 (2^-11  */
/* relative rounding), and so does the shared expert's output of a bf16 layer with      */
/* T >= 256 and more than 16384 pairs; an output beyond +-65504 sets MOE_DEV_RANGE in   */
/* the status word.                                                                     */
/* ---------------------------------------------------------------------------------- */
moe_status_t moe_layer_forward(const moe_params_t* p, const void* x, const float* x_scale,
                               const void* w_r, const float* bias, const void* w_gate,
                               const void* w_up, const void* w_down, const void* w_gate_scale,
                               const void* w_up_scale, const void* w_down_scale,
                               const void* ws_gate, const void* ws_up, const void* ws_down,
                               void* out, int32_t* topk_ids_out, float* topk_w_out,
                               int32_t* counts_out, void* ws, size_t ws_bytes, void* stream);

/* Same layer with HOST activations: x_host (and x_scale_host for FP8) are copied to the
 * device inside the call and the result is copied back to out_host, all enqueued on
 * `stream`.  Weights (and their FP8 scales) stay device pointers.  Host buffers should
 * be pinned; they must stay valid until the stream has passed this call
 * (cudaStreamSynchronize).  ws must hold moe_workspace_size_host() bytes. */
moe_status_t moe_layer_forward_host(const moe_params_t* p, const void* x_host,
                                    const float* x_scale_host, const void* w_r,
                                    const float* bias, const void* w_gate, const void* w_up,
                                    const void* w_down, const void* w_gate_scale,
                                    const void* w_up_scale, const void* w_down_scale,
                                    const void* ws_gate, const void* ws_up,
                                    const void* ws_down, void* out_host, void* ws,
                                    size_t ws_bytes, void* stream);

/* The same layer over n_batches independent batches of T tokens, each from and to host
 * memory: batch b's x_host[b] (and x_scale_host[b] for FP8) is copied in, the layer
 * runs, and its output is copied to out_host[b].  The copies run on two copy streams of
 * the library's own and overlap the device work of the neighbouring batches (two device
 * staging slots in ws, so batch b+1 is copied in and batch b-1 copied out while batch b
 * runs); the layer itself runs on `stream`.  The call enqueues everything and returns;
 * `stream` passes the call once every output copy has finished, and the first copy in
 * starts after the work already on `stream`.  Arrays x_host, x_scale_host (FP8 only,
 * else NULL) and out_host hold n_batches host pointers each; the same pointer may
 * repeat.  Host buffers must be pinned for the copies to overlap and must stay valid
 * until `stream` has passed the call.  ws must hold moe_workspace_size_host() bytes.
 * Calls on one device share the copy streams.  n_batches = 0 does nothing. */
moe_status_t moe_layer_forward_host_batches(const moe_params_t* p, int32_t n_batches,
                                            const void* const* x_host, const float* const* x_scale_host,
                                            const void* w_r, const float* bias, const void* w_gate,
                                            const void* w_up, const void* w_down, const void* w_gate_scale,
                                            const void* w_up_scale, const void* w_down_scale,
                                            const void* ws_gate, const void* ws_up, const void* ws_down,
                                            void* const* out_host, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------- */
/* e2m1 weight scales ("DeepGEMM质变…" §5.3 FP8 x FP4 GEMM; §一 1.3 lays the UE8M0 scale */
/* buffers out at the 128-element granularity of the tensor core's scale copy).         */
/* Converts one weight tensor's scales, once, when the weights are loaded:              */
/*   scale_words [rows, K/128] 32-bit words, byte j of word (r, kb) = UE8M0 scale of    */
/*               K elements 128 kb + 32 j ... + 31 of row r (4-byte aligned).  A row-   */
/*               major [rows, K/32] byte array of the scales is exactly this.           */
/*   atoms       out, rows * K / 32 bytes, 16-byte aligned: the 512-byte per (128 rows, */
/*               128 K) blocks that moe_expert_ffn / moe_layer_forward read.            */
/* rows (all experts of the tensor stacked: E*I for gate/up, E*H for down) and K must   */
/* be multiples of 128.  Asynchronous on `stream`; no workspace.                        */
/* ---------------------------------------------------------------------------------- */
moe_status_t moe_prepare_fp4_scales(const void* scale_words, int64_t rows, int32_t K, void* atoms,
                                    void* stream);

/* ---------------------------------------------------------------------------------- */
/* Status, tracing                                                                      */
/* ---------------------------------------------------------------------------------- */

/* Synchronises `stream`, copies the device status word of `ws` into *host_status. */
moe_status_t moe_get_device_status(const void* ws, void* stream, int32_t* host_status);
/* Clears the device status word of `ws` (asynchronous on `stream`). */
moe_status_t moe_clear_device_status(void* ws, void* stream);

/* Failure-path self-test (no counterpart on the pages).  One CTA waits on an mbarrier
 * that nothing completes, using the same bounded wait as the GEMM pipelines, with a
 * limit of limit_ms (1..2000) instead of the pipelines' 2 s.  When the limit runs out
 * the wait gives up, MOE_DEV_TIMEOUT is OR-ed into the status word of `ws` (first 256
 * bytes, 256-byte aligned), and the kernel returns: the context stays usable.
 * Asynchronous on `stream`. */
moe_status_t moe_selftest_bounded_wait(void* ws, int32_t limit_ms, void* stream);

const char* moe_status_string(moe_status_t s);
int32_t moe_abi_version(void);

/* Kernel ids for tracing.  MOE_K_PERM_GATHER also covers the layer's token-order copy and
 * MOE_K_SCALE_ATOMS the e4m3 weights' scale atoms.  Where moe_layer_forward runs the
 * shared expert as one more group of the routed two-M-tile launches (bf16, more than 16384
 * pairs, T*K >= 256*E), its work is inside MOE_K_GATEUP / MOE_K_DOWN and the two
 * MOE_K_SHARED_* ids do not occur. */
enum {
  MOE_K_ROUTER_GEMM = 0, MOE_K_TOPK = 1, MOE_K_PERM_COUNT = 2, MOE_K_PERM_SCAN = 3,
  MOE_K_PERM_RANK = 4, MOE_K_PERM_GATHER = 5, MOE_K_GATEUP = 6, MOE_K_DOWN = 7,
  MOE_K_SHARED_GATEUP = 8, MOE_K_SHARED_DOWN = 9, MOE_K_COMBINE = 10, MOE_K_DEQUANT_X = 11,
  MOE_K_SCALE_ATOMS = 12, MOE_K_COUNT = 13
};

/* Tracing: while enabled, every launch of a kernel whose bit (1u << id) is in
 * kernel_mask is bracketed by two CUDA events on its stream (at most `capacity` launches
 * are kept).  moe_trace_collect() synchronises on the recorded events, writes each
 * launch's kernel id and duration in milliseconds, returns the number written and
 * clears the record.  Process-wide, not thread-safe. */
moe_status_t moe_trace_enable(uint32_t kernel_mask, int32_t capacity);
moe_status_t moe_trace_disable(void);
int32_t moe_trace_collect(int32_t* kernel_ids, float* ms, int32_t max_out);

/* Number of kernels the library launches for one moe_layer_forward with these params. */
int32_t moe_layer_launch_count(const moe_params_t* p);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
