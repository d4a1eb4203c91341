/*
 * mxfp4_moe.h -- C ABI of the MXFP4 MoE block-verify library (B200, sm_100a).
 *
 * One speculative-decoding verify step of a mixture-of-experts target model:
 * a drafted block of K tokens per sequence (T = S*K tokens) is routed top-k,
 * grouped by expert, pushed through each expert's SwiGLU FFN whose weights
 * are OCP MXFP4, weight-combined, and the block is accepted greedily or by
 * rejection sampling.  Sources (page title, section):
 *   [P1] "mimo-v2-5-speculative-decoding-draft-scheduling"
 *   [P2] "如何评价小米6月9日发布的MiMo-V2.5-Pro-UltraSpeed模式？"
 *   [P3] "MiMo-v2.5-Pro-UltraSpeed - infra 架构解读"
 *   [P4] "mimo-tilert-1000tps-trillion-parameter-inference"
 *   [OCP] OCP Microscaling Formats (MX) v1.0 (named by [P3] and [P4]).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer argument is a DEVICE pointer owned by the caller; the
 *    library never allocates, frees or keeps a pointer after the call returns.
 *  - Work is enqueued on `stream` and runs asynchronously; no call
 *    synchronises except moe_get_device_status.
 *  - Tensors are dense, row-major (last index fastest), with the shapes given.
 *  - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *  - Return value: MOE_OK, or an error code.  Argument errors are detected on
 *    the host and returned before anything is launched.  Errors only the
 *    device can see (an expert id outside [0,E), a row with no probability
 *    mass, a bounded wait that ran out) set a sticky device status word read
 *    by moe_get_device_status; the kernel then skips the offending element
 *    and never faults.  Inputs with NaN or infinity are unsupported: results
 *    are unspecified, but no fault occurs.
 *  - Every kernel is launched with programmatic stream serialisation
 *    (programmatic dependent launch): the next kernel on the stream may
 *    become resident while the current one finishes, and waits for it
 *    (griddepcontrol.wait) before it reads the current one's output or writes
 *    anything.  A library kernel lets its successor launch only after its own
 *    wait, so when a kernel starts early everything two launches back is
 *    complete; kernels rely on that only for data the same call or the call
 *    before produced (the FFN's second GEMM reads the expert offsets before
 *    its wait).  Ordinary kernels of the caller are unaffected: without the
 *    attribute a kernel waits for full completion as usual.
 */
#ifndef MXFP4_MOE_H
#define MXFP4_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same type as cudaStream_t */

enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, k > E, ...          */
  MOE_ERR_UNSUPPORTED = 2, /* shape outside what the kernels implement    */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed         */
  MOE_ERR_WORKSPACE = 4,   /* workspace smaller than the query returned    */
  MOE_ERR_DEVICE = 5       /* device status word set (see below)           */
};

/* Device-side error details (second argument of moe_get_device_status). */
enum {
  MOE_DEV_OK = 0,
  MOE_DEV_BAD_EXPERT = 1,  /* moe_permute saw an expert id outside [0,E)   */
  MOE_DEV_NO_MASS = 2,     /* block_accept_rejection: target row all zero  */
  MOE_DEV_BAD_TOKEN = 3,   /* a draft token outside [0,V)                   */
  MOE_DEV_TIMEOUT = 4,     /* a bounded device wait ran out                */
  MOE_DEV_BAD_INDEX = 5    /* checked build (MOE_CHECKS): a pair, row or
                              offset index outside its array, replaced by 0
                              or (offsets) the call's experts left empty   */
};

/* Human-readable name of a status code (static string, never NULL). */
const char *moe_status_string(int status);

/* Library version, e.g. 1 00 00 -> 10000. */
int moe_version(void);

/*
 * moe_route_topk -- top-k expert routing of T tokens over E experts.
 *   Each token activates a few experts ([P4] "万亿参数推理为什么特别难");
 *   the router keeps high precision ([P4] "第一层：FP4 选择性量化").  Rule:
 *   expert i of a token is selected iff fewer than k experts j have
 *   logit_j > logit_i or (logit_j == logit_i and j < i); selected experts are
 *   listed by that rank (descending logit, ties to the lowest index).
 *   Weights are softmax over the k selected logits, evaluated in double
 *   precision and rounded once to float.
 *   logits   [T, E] float   (finite)
 *   topk_idx [T, k] int32   out
 *   topk_w   [T, k] float   out
 *   Limits: 1 <= k <= min(E, 32), 1 <= E <= 1024, T >= 0.
 */
int moe_route_topk(const float *logits, int T, int E, int k, int32_t *topk_idx,
                   float *topk_w, moe_stream_t stream);

/*
 * moe_permute -- stable grouping of the T*k (token, slot) pairs by expert.
 *   The pages route each token to a few experts ([P4] "万亿参数推理为什么特别难")
 *   and run the experts on the drafted block ([P3] "数据流概览"), but say
 *   nothing about how the pairs are grouped or ordered.  Reading taken here:
 *   a stable grouping, so that the order is unique and checkable --
 *   experts ascending, pairs ascending by id inside an expert.
 *   Pair id p = t*k + j.  expert_offsets[e] .. expert_offsets[e+1] is the
 *   range of sorted rows of expert e; sorted_pair lists pair ids expert by
 *   expert, ascending inside an expert; pair_row is its inverse
 *   (pair_row[sorted_pair[r]] == r).
 *   topk_idx       [T*k]  int32 in [0, E)
 *   expert_offsets [E+1]  int32 out
 *   sorted_pair    [T*k]  int32 out
 *   pair_row       [T*k]  int32 out
 *   Limits: 1 <= E <= 1024, 0 <= T*k <= 1<<24.  An id outside [0,E) sets
 *   MOE_DEV_BAD_EXPERT and that pair is left out.
 */
int moe_permute(const int32_t *topk_idx, int T, int k, int E,
                int32_t *expert_offsets, int32_t *sorted_pair,
                int32_t *pair_row, moe_stream_t stream);

/*
 * moe_route_permute -- moe_route_topk followed by moe_permute, same
 *   arguments, outputs and errors as the two calls.  For T <= 128 tokens it
 *   runs as one kernel (one CTA routes every token, then groups the pairs),
 *   saving a launch on the verify step's critical path; larger batches make
 *   the two launches.  The pages describe routing and grouping as separate
 *   steps; fusing them changes no result.
 */
int moe_route_permute(const float *logits, int T, int E, int k, int32_t *topk_idx,
                      float *topk_w, int32_t *expert_offsets, int32_t *sorted_pair,
                      int32_t *pair_row, moe_stream_t stream);

/*
 * mxfp4_moe_ffn -- SwiGLU FFN of every permuted pair over MXFP4 experts.
 *   The experts hold OCP MXFP4 weights while the rest of the model keeps
 *   higher precision ([P1] "接受率预测与动态回退机制"; [P3] "FP4 Expert 量化";
 *   [P4] "第一层：FP4 选择性量化").  Weight format [OCP]: 4-bit E2M1 codes,
 *   two per byte (element 2j in the low nibble), one E8M0 scale byte
 *   (value 2^(s-127)) per 32 consecutive elements of a row.
 *     w13_codes  [E, 2I, H/2]  uint8   rows 0..I-1 gate, I..2I-1 up
 *     w13_scales [E, 2I, H/32] uint8
 *     w2_codes   [E, H, I/2]   uint8   down projection
 *     w2_scales  [E, H, I/32]  uint8
 *   For sorted row r of expert e (token t = sorted_pair[r] / k):
 *     g = x[t] . Wg^T, u = x[t] . Wu^T   (float accumulation over the exactly
 *     dequantised weights), h = bf16(silu(g) * u), y[r] = h . Wd^T (float).
 *   x              [T, H]     bf16
 *   expert_offsets [E+1], sorted_pair [T*k]  from moe_permute
 *   y              [T*k, H]   float out, sorted-row order
 *   workspace      device scratch of at least
 *                  mxfp4_moe_ffn_workspace_bytes(T, k, H, I) bytes, 256-byte
 *                  aligned; its contents on entry do not matter.
 *   Limits: H % 128 == 0, I % 128 == 0, 1 <= E <= 1024, 1 <= k <= 32.
 *   The tensor-core variants load the code arrays by TMA: 16-byte aligned
 *   (else MOE_ERR_CUDA).  Scale arrays of any alignment; where one is
 *   16-byte aligned and its rows hold a multiple of 16 bytes (K % 512 == 0),
 *   kind::mxf8f6f4 loads it by TMA as well (same results).
 *   The kernel variant: the tensor-core one wherever its limits allow
 *   (H >= 512), else the FMA one (see mxfp4_moe_ffn_variant).
 */
size_t mxfp4_moe_ffn_workspace_bytes(int T, int k, int H, int I);

int mxfp4_moe_ffn(const uint16_t *x, int T, int H, int I, int E, int k,
                  const uint8_t *w13_codes, const uint8_t *w13_scales,
                  const uint8_t *w2_codes, const uint8_t *w2_scales,
                  const int32_t *expert_offsets, const int32_t *sorted_pair,
                  float *y, void *workspace, size_t workspace_bytes,
                  moe_stream_t stream);

/* Kernel variants of mxfp4_moe_ffn. */
enum {
  MOE_FFN_AUTO = 0,      /* tensor cores if H >= 512, else FMA                   */
  MOE_FFN_FMA = 1,       /* dequantise to registers, float FMA                   */
  MOE_FFN_TENSOR = 2,    /* tcgen05 block-scaled MMA: TENSOR_F4 while its B
                            tiles stay narrow (8*T*k <= 128 * min(T*k, E)) and
                            H, I are multiples of 256 up to 8192, else
                            TENSOR_F8; with a few tokens per expert (B tiles of
                            at most 32 columns) and I <= 4096, TENSOR_FUSED     */
  MOE_FFN_TENSOR_F8 = 3, /* kind::mxf8f6f4: padded E2M1 weights x two E4M3
                            activation terms with E8M0 block scales               */
  MOE_FFN_TENSOR_F4 = 4, /* kind::mxf4: packed E2M1 weights x eight E2M1
                            activation terms with one scale per row and term
                            (H, I multiples of 256, at most 8192)                 */
  MOE_FFN_TENSOR_FUSED = 5, /* TENSOR_F4 with both GEMMs in one persistent
                            launch (I <= 4096): the last GEMM-1 tile of each
                            expert's token block encodes its h rows and
                            publishes them by a flag, and GEMM-2 tiles wait
                            for that flag (bounded) instead of for the end
                            of a launch -- the first piece of a persistent
                            verify kernel, after the persistent engine of
                            [P4] (prior art).  Same results as TENSOR_F4.   */
  MOE_FFN_TENSOR_F8_PAIR = 6 /* TENSOR_F8 on clusters of two CTAs (H a multiple
                            of 256): each M = 256 tcgen05 MMA (cta_group::2)
                            covers two weight m-blocks, each SM of the pair
                            holding one m-block and half of the activation
                            rows, so an SM streams half the activation bytes
                            per weight byte.  Same results as TENSOR_F8.    */
};
/* Accuracy domain of the activation encodings.  FMA and TENSOR_F8 represent
 * every 32-element block of an activation row on its own scale, so they meet
 * the FFN tolerance for any finite bf16 rows and any weights whose values are
 * finite bf16 numbers.  TENSOR_F4 (which TENSOR and AUTO take for narrow
 * tiles) represents a whole row by eight terms, each element exact to about
 * 2^-16 of the row's largest magnitude; that meets the tolerance unless the
 * products of a row's 32-element blocks with their weight blocks span more
 * than about 2^16 -- small activation blocks meeting weight scales 2^16 times
 * larger than those of the row's large blocks.  Such weights (E8M0 scales
 * spread over more than 16 binades within a row, opposed to the activations)
 * need TENSOR_F8 or FMA. */

/* Same contract as mxfp4_moe_ffn with an explicit kernel variant. */
int mxfp4_moe_ffn_variant(const uint16_t *x, int T, int H, int I, int E, int k,
                          const uint8_t *w13_codes, const uint8_t *w13_scales,
                          const uint8_t *w2_codes, const uint8_t *w2_scales,
                          const int32_t *expert_offsets,
                          const int32_t *sorted_pair, float *y, void *workspace,
                          size_t workspace_bytes, int variant,
                          moe_stream_t stream);

/* The bf16 SwiGLU outputs h [T*k, I] (sorted-row order) that the last
 * mxfp4_moe_ffn call left at the start of its workspace. */
const uint16_t *mxfp4_moe_ffn_workspace_h(const void *workspace);

/*
 * mxfp4_moe_ffn_noalloc -- mxfp4_moe_ffn for callers that cannot allocate.
 *   The pages have no counterpart to this call; it exists for users of the
 *   library that are not allowed to allocate device memory: plugins hosted by
 *   an engine that reserves all device memory up front and hands its plugins
 *   no allocator, and latency-critical loops in which a cudaMalloc/cudaFree
 *   (cudaFree synchronises the device) is not acceptable.  Same contract as
 *   mxfp4_moe_ffn, except that the scratch space comes from an array of
 *   MOE_NOALLOC_SCRATCH_BYTES in the library's own device global memory,
 *   which every GPU that loads the library holds until the process exits.
 *   The caller still passes inputs and outputs.
 *   - Problems whose scratch need (mxfp4_moe_ffn_workspace_bytes) exceeds
 *     MOE_NOALLOC_SCRATCH_BYTES are rejected with MOE_ERR_WORKSPACE before
 *     anything is launched.  8 MiB covers T*k <= 64 pairs at H = 7168,
 *     I = 2048 (one 8-token block with top-8 routing).
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (the FFN writes every scratch byte it reads, so nothing needs
 *     clearing).  Calls whose executions overlap on the GPU -- on different
 *     streams, or from different host threads -- race on it; serialise them.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (8u << 20)

int mxfp4_moe_ffn_noalloc(const uint16_t *x, int T, int H, int I, int E, int k,
                          const uint8_t *w13_codes, const uint8_t *w13_scales,
                          const uint8_t *w2_codes, const uint8_t *w2_scales,
                          const int32_t *expert_offsets, const int32_t *sorted_pair,
                          float *y, moe_stream_t stream);

/*
 * moe_combine -- weighted sum of each token's k expert outputs.
 *   The pages do not state how expert outputs are merged ([P4]
 *   "万亿参数推理为什么特别难" only says each token uses a few experts).
 *   Reading taken here, the usual MoE combine with the routing weights of
 *   moe_route_topk, in a fixed order so that results are reproducible:
 *   out[t] = bf16( sum_{j<k} topk_w[t,j] * y[pair_row[t*k+j]] + residual[t] )
 *   in float, slots summed in order j = 0..k-1, residual added last.
 *   y [T*k, H] float, pair_row [T*k], topk_w [T, k] float,
 *   residual [T, H] bf16 or NULL, out [T, H] bf16 (may alias residual).
 */
int moe_combine(const float *y, const int32_t *pair_row, const float *topk_w,
                int T, int k, int H, const uint16_t *residual, uint16_t *out,
                moe_stream_t stream);

/*
 * moe_rms_norm -- parameter-free RMSNorm of bf16 rows (stacked layers).
 *   out[t] = bf16( x[t] / sqrt(mean_c x[t,c]^2 + eps) ), float arithmetic.
 *   The pages do not describe the layer stack; a pre-norm keeps stacked
 *   synthetic layers finite (each MXFP4 expert layer scales its input by
 *   ~1e8 at the configured scale range).  x, out [T, H] bf16, may alias.
 */
int moe_rms_norm(const uint16_t *x, int T, int H, float eps, uint16_t *out,
                 moe_stream_t stream);

/*
 * block_accept_greedy -- greedy prefix acceptance of S drafted blocks.
 *   Tokens the target confirms are kept; from the first wrong draft token
 *   on the target takes over ([P2] "二、投机解码").  Row i of logits checks
 *   draft[i]; accept_len = the largest a such that argmax(logits[s,i]) ==
 *   draft[s,i] for all i < a (argmax ties to the lowest token id);
 *   next_token = argmax(logits[s, a]) if a < K, else -1.
 *   logits [S, K, V] float, draft [S, K] int32,
 *   accept_len [S] int32 out, next_token [S] int32 out.  Until the call
 *   completes on the stream, the two outputs also hold its per-sequence
 *   working state (the smallest mismatch key and the rows reported); no
 *   other memory is used.  Two kernels run: a one-CTA setup, then one
 *   thread-block cluster per block row.
 *   Limits: 1 <= K <= 32, 1 <= V <= 2^26, S <= 65535 (else
 *   MOE_ERR_UNSUPPORTED).  A draft token outside [0, V) sets the device
 *   status MOE_DEV_BAD_TOKEN and counts as a mismatch.
 */
int block_accept_greedy(const float *logits, const int32_t *draft, int S, int K,
                        int V, int32_t *accept_len, int32_t *next_token,
                        moe_stream_t stream);

/*
 * block_accept_rejection -- speculative rejection sampling of S blocks.
 *   Verify by rejection sampling ([P3] "数据流概览"), lossless in the sense
 *   that the output follows the target distribution ([P2] "六、效果如何").
 *   Draft x_i is accepted iff double(u_accept[s,i]) * double(q[s,i,x_i]) <
 *   double(p[s,i,x_i]) (= u < min(1, p/q), exactly).  At the first rejected
 *   row a the token is drawn from max(0, p - q): r_v = max(0, p_v - q_v) in
 *   float, R_v = floor(r_v * 2^40) (integer), m = floor(sum(R) * U / 2^24)
 *   with U = u_resample[s] * 2^24, next_token = least v with
 *   R_0 + .. + R_v > m; if sum(R) == 0 the same draw uses floor(p_v * 2^40).
 *   All K accepted -> next_token = -1.
 *   p, q [S, K, V] float probabilities; draft [S, K] int32;
 *   u_accept [S, K], u_resample [S] float uniforms in [0,1), multiples of
 *   2^-24; accept_len [S], next_token [S] int32 out.
 *   Limits: 1 <= K <= 32, 1 <= V <= 2^24.
 */
int block_accept_rejection(const float *p, const float *q, const int32_t *draft,
                           const float *u_accept, const float *u_resample,
                           int S, int K, int V, int32_t *accept_len,
                           int32_t *next_token, moe_stream_t stream);

/*
 * block_accept_greedy_bonus -- block_accept_greedy with a bonus row.
 *   The target scores K + 1 positions per sequence: rows 0..K-1 check the K
 *   drafts as in block_accept_greedy, row K is its prediction after the
 *   whole block.  When every draft is accepted the target's own token for
 *   that next position is emitted instead of -1, so each verify step yields
 *   accept_len + 1 tokens (the target takes over after the last confirmed
 *   token, [P2] "二、投机解码"; the drafter proposes a fixed-size block,
 *   [P1] "接受率预测与动态回退机制").
 *   next_token = argmax(logits[s, accept_len]) (lowest-index ties), never -1.
 *   logits [S, K+1, V] float, draft [S, K] int32,
 *   accept_len [S], next_token [S] int32 out.
 *   Limits and errors as block_accept_greedy (K <= 32: at most 33 rows).
 */
int block_accept_greedy_bonus(const float *logits, const int32_t *draft, int S, int K,
                              int V, int32_t *accept_len, int32_t *next_token,
                              moe_stream_t stream);

/*
 * block_accept_rejection_bonus -- block_accept_rejection with a bonus row.
 *   p holds K + 1 target rows per sequence, q the K draft rows.  Rows
 *   0..K-1 are verified exactly as in block_accept_rejection (a rejection
 *   at row a draws from max(0, p - q) at row a).  When all K drafts are
 *   accepted the next token is drawn from the target row p[s, K] by the
 *   same integer rule on P_v = floor(p_v * 2^40): m = floor(sum(P) * U /
 *   2^24), U = u_resample[s] * 2^24, next_token = least v with
 *   P_0 + .. + P_v > m.  A bonus row with no mass sets MOE_DEV_NO_MASS and
 *   next_token = -1.
 *   p [S, K+1, V], q [S, K, V] float; draft [S, K]; u_accept [S, K];
 *   u_resample [S]; accept_len [S], next_token [S] int32 out.
 *   Limits as block_accept_rejection.
 */
int block_accept_rejection_bonus(const float *p, const float *q, const int32_t *draft,
                                 const float *u_accept, const float *u_resample,
                                 int S, int K, int V, int32_t *accept_len,
                                 int32_t *next_token, moe_stream_t stream);

/*
 * mxfp4_quantize -- bf16 weights to OCP MXFP4, the format the expert FFN
 *   reads ([P3] "FP4 Expert 量化"; [P4] "第一层：FP4 选择性量化"; the
 *   conversion is the one [OCP] defines).  Per 32 consecutive elements of
 *   a row: scale byte e = max(0, floor(log2 amax) - 2 + 127) (byte 0 for an
 *   all-zero block; bf16 inputs never need more than 252), and each element
 *   becomes the E2M1 code nearest to v / 2^(e-127), ties to the even code,
 *   saturating at +-6, with the sign of v (so -0 -> code 8).
 *   w      [R, K] bf16, finite, 16-byte aligned
 *   codes  [R, K/2] uint8 out (element 2j in the low nibble), 4-byte aligned
 *   scales [R, K/32] uint8 out
 *   Limits: K % 32 == 0, K >= 32, R >= 0, R * K <= 2^40.
 *   Bound by HBM: 2 bytes read and 17/32 byte written per element.
 */
int mxfp4_quantize(const uint16_t *w, int64_t R, int K, uint8_t *codes, uint8_t *scales,
                   moe_stream_t stream);

/*
 * moe_get_device_status -- synchronise `stream`, then report the sticky
 * device status word of the current device: returns MOE_OK if it is clear,
 * MOE_ERR_DEVICE if set (detail in *detail, may be NULL), MOE_ERR_CUDA on a
 * CUDA failure.  moe_clear_device_status resets it (enqueued on `stream`).
 */
int moe_get_device_status(moe_stream_t stream, int *detail);
int moe_clear_device_status(moe_stream_t stream);

/*
 * moe_set_wait_limit_ns -- time limit of the tensor-core FFN's bounded waits
 *   on the current device: 2 s by default, `ns` = 0 restores the default.
 *   (The pages have no counterpart; this is the library's failure
 *   detection.)  A wait that runs past the limit ends the kernel early: it
 *   sets MOE_DEV_TIMEOUT in the device status word, waits for the copies and
 *   tensor-core operations it has already issued (at most 2 s more), frees
 *   its tensor memory and returns, so the context stays usable and the next
 *   call runs normally.  Lowering the limit far below a kernel's run time is
 *   how that path is exercised; results of a call that timed out are
 *   unspecified.  Enqueued on `stream` (the host value is copied before the
 *   call returns).
 */
int moe_set_wait_limit_ns(uint64_t ns, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MXFP4_MOE_H */
