/*
 * ktmoe.h — C ABI of the B200 (sm_100a) DeepSeekMoE layer forward.
 *
 * One DeepSeekMoE layer computes, per token u_t (the total-output equation of
 * the "DeepSeekMoE 三改进" passage of the DeepSeek-V3 model.py notes,
 * 73biji.xyz/llm_pp_dsv3):
 *
 *     h'_t = [u_t +] sum_{shared s} FFN_s(u_t) + sum_{j<k} g_{j,t} FFN_{idx_j}(u_t)
 *
 * with FFN(v) = W2 (silu(W1 v) * W3 v) (SwiGLU; the pages only say "FFN") and
 * the routing (idx, g) of the same page's "Gate 选专家流程（model.py，五步）":
 *   1. s = sigmoid(W_g u) (or softmax over all experts), kept raw;
 *   2. keys s + b (bias b only where the layer has one, "V3 改进①"); group score
 *      = max of the group's keys (no bias) or the sum of its two largest keys
 *      (with bias);
 *   3. keep the topk_groups best groups, other experts' keys := -inf;
 *   4. global top-k over the keys;
 *   5. gather the raw s at the chosen experts, renormalise, times route_scale.
 * Ties in both top-k's go to the lower index; idx is in descending key order.
 *
 * Conventions for every entry point:
 *  - Pointers named "device" are caller-owned CUDA device memory; the library
 *    never allocates, frees or retains them. Host pointers are read only during
 *    the call.
 *  - `stream` is a cudaStream_t (0 = legacy default stream). Calls only enqueue
 *    work on it and return without synchronising, except kt_moe_check.
 *  - Layouts are row-major. Activations and expert weights share one dtype
 *    (kt_moe_config.dtype); the bias and routing weights are always fp32.
 *  - Expert weights are stacked, routed experts 0..E-1 then shared experts
 *    E..E+S-1, each in nn.Linear [out, in] order:
 *        w1, w3 : [E+S, inter, dim]   (gate and up projections)
 *        w2     : [E+S, dim, inter]   (down projection)
 *  - Return value: KT_OK (0) or a negative KT_ERR_* code. Host-side checks run
 *    before anything is enqueued; on an error return nothing was enqueued.
 *  - The library keeps no state between calls; a call's scratch lives in the
 *    caller's workspace, so concurrent calls need distinct workspaces.
 */
#ifndef KTMOE_H
#define KTMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Score function of gate step 1. */
enum { KT_SCORE_SIGMOID = 0, KT_SCORE_SOFTMAX = 1 };
/* Group score of gate step 2. AUTO = TOP2SUM when a bias is given, else AMAX. */
enum { KT_GROUP_AUTO = 0, KT_GROUP_AMAX = 1, KT_GROUP_TOP2SUM = 2 };
/* Activation / expert-weight dtype. KT_DTYPE_MXFP8: bf16 tokens, gate weights
 * and output (as KT_DTYPE_BF16); expert weights in MXFP8 (kt_moe_forward_mxfp8).
 * KT_DTYPE_MXFP4: the same with expert weights in MXFP4 (4-bit E2M1 elements;
 * also through kt_moe_forward_mxfp8 and the other MXFP8 entry points). */
enum { KT_DTYPE_F32 = 0, KT_DTYPE_BF16 = 1, KT_DTYPE_MXFP8 = 2, KT_DTYPE_MXFP4 = 3 };

enum {
  KT_OK = 0,
  KT_ERR_INVALID_CONFIG = -1, /* inconsistent config or token count               */
  KT_ERR_NULL = -2,           /* a required pointer is NULL                         */
  KT_ERR_WORKSPACE = -3,      /* workspace NULL or smaller than kt_moe_workspace_size */
  KT_ERR_ALIGN = -4,          /* a pointer is not 16-byte aligned (workspace: 256)  */
  KT_ERR_CUDA = -5,           /* a CUDA runtime call or launch failed               */
  KT_ERR_TIMEOUT = -6,        /* a bounded device-side wait gave up (kt_moe_check)  */
  KT_ERR_UNSUPPORTED = -7,    /* no sm_100 device, or a size beyond a kernel limit  */
  KT_ERR_SCRATCH_LIMIT = -8,  /* call needs more than the static scratch holds       */
  KT_ERR_BOUNDS = -9          /* checked build: an index check failed (kt_moe_check) */
};

/*
 * Layer description. The first six fields are the gate's parameters named by
 * the "Gate 选专家流程" passage (n_groups, topk_groups, topk, route_scale and
 * the sigmoid/softmax score); the rest are shapes and switches.
 *
 * Limits (KT_ERR_INVALID_CONFIG otherwise): 1 <= n_experts <= 512;
 * n_experts % n_groups == 0; 1 <= topk_groups <= n_groups <= 32;
 * 1 <= topk <= min(32, topk_groups * n_experts / n_groups); n_groups == 1
 * implies topk_groups == 1; TOP2SUM needs >= 2 experts per group;
 * 0 <= n_shared <= 8; route_scale finite and > 0; dim, inter >= 8 and
 * multiples of 8 (bf16) or 4 (fp32), so rows are 16-byte multiples; for
 * KT_DTYPE_MXFP8 and KT_DTYPE_MXFP4 multiples of 128 (one 128-element K slab).
 */
typedef struct {
  int32_t n_experts;    /* E: routed experts                                      */
  int32_t n_groups;     /* G: expert groups (1 = no group limit)                   */
  int32_t topk_groups;  /* TG: groups kept per token                              */
  int32_t topk;         /* k: routed experts per token                            */
  float route_scale;    /* multiplies the routing weights (2.5 in DeepSeek-V3)     */
  int32_t score_func;   /* KT_SCORE_SIGMOID or KT_SCORE_SOFTMAX                    */
  int32_t dim;          /* d: hidden size                                         */
  int32_t inter;        /* I: SwiGLU hidden size of one expert                     */
  int32_t n_shared;     /* S: always-on shared experts (weight 1)                  */
  int32_t norm_topk;    /* -1 auto (renormalise iff sigmoid), 0 off, 1 on          */
  int32_t group_score;  /* KT_GROUP_*                                              */
  int32_t dtype;        /* KT_DTYPE_*                                              */
  int32_t add_residual; /* 1: add u_t to the output (h'_t); 0: MoE-module output   */
  int32_t y_fp32;       /* 1: y is fp32 even for bf16 layers (the fp32 sum before   */
                        /*    its final rounding); 0: y in `dtype`                 */
} kt_moe_config;

/* Host-only validation of a config for T tokens (T >= 1, T <= 2^20). No CUDA
 * call. `has_bias` says whether a bias will be passed (it decides AUTO group
 * scoring). Returns KT_OK or KT_ERR_INVALID_CONFIG. */
int kt_moe_validate(const kt_moe_config* cfg, int64_t T, int has_bias);

/* Bytes of device workspace kt_moe_gate / kt_moe_forward need for T tokens
 * (0 if the config is invalid). No CUDA call. */
size_t kt_moe_workspace_size(const kt_moe_config* cfg, int64_t T);

/*
 * Gate only (steps 1-5 above).
 *   x        device [T, dim] (dtype)           tokens u_t
 *   w_gate   device [E, dim] (dtype)           gate weights W_g
 *   bias     device [E] fp32 or NULL           per-expert selection bias b
 *   scores_in device [T, E] fp32 or NULL       if given, used as the scores s
 *            (post score function) and x / w_gate are not read (may be NULL):
 *            the selection steps 2-5 alone, for index-exact comparisons
 *   topk_idx device [T, k] int32  (out)        chosen experts, descending key
 *   topk_w   device [T, k] fp32   (out)        routing weights g
 *   workspace device, ws_bytes >= kt_moe_workspace_size(cfg, T), 256-B aligned
 * Logits accumulate in fp32; the selection arithmetic is fp32 in the order of
 * steps 2-5 (s + b; group max or top-2 sum; sum of gathered scores in slot
 * order; division; times route_scale).
 */
int kt_moe_gate(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                const float* bias, const float* scores_in, int32_t* topk_idx,
                float* topk_w, void* workspace, size_t ws_bytes, void* stream);

/*
 * The whole layer forward.
 *   x, w_gate, bias    as for kt_moe_gate
 *   w1, w3             device [E+S, inter, dim] (dtype)
 *   w2                 device [E+S, dim, inter] (dtype)
 *   y                  device [T, dim] (out): dtype, or fp32 if cfg->y_fp32;
 *                      must not overlap x or the workspace
 *   topk_idx_out       device [T, k] int32 or NULL: the routing, if wanted
 *   topk_w_out         device [T, k] fp32 or NULL
 * The output sum runs in a fixed order per token (shared experts in index
 * order, then the k routed slots in key order, then u_t if add_residual) in
 * fp32, so repeated calls give bitwise-equal y. bf16 layers keep the SwiGLU
 * hidden vectors in bf16 (the down GEMM's tensor-core operand) and the weighted
 * expert outputs in fp32 between kernels.
 */
int kt_moe_forward(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                   const float* bias, const void* w1, const void* w3, const void* w2,
                   void* y, int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                   size_t ws_bytes, void* stream);

/* kt_moe_forward plus stage timing: `stage_events` points to KT_STAGE_EVENTS
 * cudaEvent_t handles (entries may be NULL) that are recorded on `stream` at
 * the stage boundaries, in this order: start, after the gate (logits and
 * selection), after the token permutation, after the gate/up expert GEMM,
 * after the down expert GEMM, after the combine. cudaEventElapsedTime between
 * consecutive events gives each stage's device time. Same arguments, errors
 * and results as kt_moe_forward otherwise. */
enum { KT_STAGE_EVENTS = 6 };
int kt_moe_forward_profiled(const kt_moe_config* cfg, int64_t T, const void* x,
                            const void* w_gate, const float* bias, const void* w1,
                            const void* w3, const void* w2, void* y, int32_t* topk_idx_out,
                            float* topk_w_out, void* workspace, size_t ws_bytes, void* stream,
                            void* const* stage_events);

/*
 * kt_moe_forward for callers that cannot allocate device memory. There is no
 * counterpart on the pages: this entry point exists for the calling code, not
 * for the method.
 *
 * Some callers cannot call cudaMalloc or any allocator: engines whose device
 * memory is entirely owned by their own pool (an allocation behind the pool's
 * back can fail once the pool holds the memory, or breaks its accounting),
 * latency-critical loops where cudaMalloc and cudaFree would synchronise the
 * device, and plugin hosts that hand out no workspace. They pass only inputs
 * and outputs; the scratch comes from a fixed 32 MiB device array inside this
 * library (KT_STATIC_SCRATCH_BYTES), reserved on every GPU that loads the
 * library until the process exits. A call whose scratch need
 * (kt_moe_workspace_size) exceeds that returns KT_ERR_SCRATCH_LIMIT before
 * anything is enqueued — about 78 tokens of a DeepSeek-V3-shaped layer, so
 * decode-sized batches. This entry point allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *
 * Set-up: the first call on each device, with that device current, looks up
 * the array's device address (cudaGetSymbolAddress) and does the library's
 * other one-time host set-up for that device (the expert GEMMs' shared-memory
 * limits, the tensor-map encoder); later calls only read the kept address. The
 * address is kept for the life of the process: after a cudaDeviceReset of that
 * device it is no longer valid, and this entry point must not be used again in
 * that process. Every call on a device shares the one array, which keeps the
 * previous call's contents (each call resets what must start at zero); calls
 * whose work overlaps on the GPU — concurrent streams, or host threads without
 * ordering — race on it and must be serialised by the caller.
 * Arguments, layouts, results and errors are otherwise those of
 * kt_moe_forward; kt_moe_check takes kt_moe_static_scratch() as its workspace.
 */
enum { KT_STATIC_SCRATCH_BYTES = 32 << 20 };
int kt_moe_forward_static(const kt_moe_config* cfg, int64_t T, const void* x,
                          const void* w_gate, const float* bias, const void* w1,
                          const void* w3, const void* w2, void* y, int32_t* topk_idx_out,
                          float* topk_w_out, void* stream);

/* Device address of the current device's static scratch (NULL on error); for
 * kt_moe_check and for reading its buffers after kt_moe_forward_static. */
void* kt_moe_static_scratch(void);

/*
 * Diagnostic of the device-side failure path: one kernel thread waits, through
 * the same bounded wait as the GEMM kernels, on an mbarrier that nothing
 * arrives on; after limit_ns (0 < limit_ns <= 1e9) it records the timeout in
 * the workspace error word and exits. kt_moe_check(workspace, stream) then
 * returns KT_ERR_TIMEOUT; the context stays usable (the next forward on the
 * workspace resets the word). workspace: device, 256-B aligned, at least 8 B.
 */
int kt_moe_selftest_timeout(void* workspace, int64_t limit_ns, void* stream);

/*
 * The layer forward as a replayable CUDA graph, for decode steps where the
 * launch gaps of the eight stream operations are a visible share of a step of
 * well under a millisecond. There is no counterpart on the pages (their engine
 * runs without graphs); this serves the calling code.
 *
 * kt_moe_graph_create captures one kt_moe_forward with exactly these arguments
 * (checked on the host first; same errors) on a private stream and instantiates
 * it. Every pointer is bound into the graph: each kt_moe_graph_launch runs the
 * whole forward on `stream` reading x, w_gate, bias and the weights as they are
 * then, writing y (and topk_idx_out / topk_w_out if given) and using the
 * workspace, which must stay allocated and unshared while launches are pending.
 * Results are bitwise those of kt_moe_forward on the same inputs.
 * kt_moe_graph_destroy frees the graph (NULL is ignored); the caller must not
 * destroy it while a launch is pending. The graph object and the driver's
 * graph resources are the only things allocated; kt_moe_check(workspace,
 * stream) reads the error word as for kt_moe_forward.
 */
typedef struct kt_moe_graph kt_moe_graph;
int kt_moe_graph_create(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                        const float* bias, const void* w1, const void* w3, const void* w2,
                        void* y, int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                        size_t ws_bytes, kt_moe_graph** graph_out);
/* The same for the MXFP8 form: captures one kt_moe_forward_mxfp8 with these
 * arguments (host checks and errors as for kt_moe_forward_mxfp8). */
int kt_moe_graph_create_mxfp8(const kt_moe_config* cfg, int64_t T, const void* x,
                              const void* w_gate, const float* bias, const uint8_t* w1q,
                              const uint8_t* w3q, const uint8_t* w2q, const uint8_t* sf_up,
                              const uint8_t* sf_down, void* y, int32_t* topk_idx_out,
                              float* topk_w_out, void* workspace, size_t ws_bytes,
                              kt_moe_graph** graph_out);
int kt_moe_graph_launch(kt_moe_graph* graph, void* stream);
void kt_moe_graph_destroy(kt_moe_graph* graph);

/*
 * MXFP8 expert weights: the FP8 form of the layer (cfg->dtype = KT_DTYPE_MXFP8).
 * The pages name the format family (the DeepSeek-V3 notes' FP8 mixed precision,
 * the KTransformers page's native MXFP4 routed experts) but no rule. Format:
 * E4M3 elements (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest
 * finite 448), one power-of-two scale 2^e per 32 consecutive elements along K,
 * stored as the byte e + 127. Rule: e is the smallest integer with
 * amax <= 448 * 2^e (amax = the block's largest magnitude; 0 gives e = -127),
 * each element the E4M3 round-to-nearest-even of v * 2^-e.
 *
 * kt_moe_mxfp8_quantize: row-major [rows, K] bf16 (K % 32 == 0) -> codes
 *   [rows, K] and scale bytes [rows, K/32], row-major; device pointers, 16-B
 *   aligned src and codes.
 *
 * kt_moe_mxfp8_pack: stacked bf16 expert weights (w1, w3 [E+S, inter, dim],
 *   w2 [E+S, dim, inter]) -> codes in the same layout (w1q, w3q, w2q, one byte
 *   each) and the scales packed as the grouped GEMM reads them:
 *   sf_up   (kt_moe_mxfp8_scale_bytes(cfg, 0) bytes): a 512-byte block per
 *           (group g, feature tile ft of 128, half h, K slab s of 128 along dim)
 *           at block index ((g * inter/128 + ft) * 2 + h) * dim/128 + s; in it
 *           the scale of tile row m (m < 64: W1 row 128 ft + 64 h + m; m >= 64:
 *           W3 row 128 ft + 64 h + m - 64) and K block 4 s + k1 sits at byte
 *           16 * (m % 32) + 4 * (m / 32) + k1;
 *   sf_down (kt_moe_mxfp8_scale_bytes(cfg, 1) bytes): the same for W2 with
 *           feature tiles of 256 output rows (nft = ceil(dim/256)) and K slabs
 *           along inter: block ((g * nft + ft) * 2 + h) * inter/128 + s, tile row
 *           m = W2 row 256 ft + 128 h + m (rows past dim hold 0).
 *   dim and inter must be multiples of 128.
 *
 * kt_moe_forward_mxfp8: the layer forward with packed MXFP8 weights. x, w_gate,
 *   bias, y, topk outputs, workspace (kt_moe_workspace_size with the MXFP8
 *   config) and errors as for kt_moe_forward; w3q must lie above w1q in memory
 *   (e.g. the two halves of one [2, E+S, inter, dim] buffer: the kernel reads
 *   the codes of both in one box, in address order, and the packed scales list
 *   W1 first), else KT_ERR_INVALID_CONFIG; stage_events as for
 *   kt_moe_forward_profiled (NULL for none). The gate runs in bf16 / fp32 as in
 *   the bf16 form; the tokens and the SwiGLU hidden rows are quantised to MXFP8
 *   by the rule above; the expert GEMMs accumulate in fp32 on the tensor cores
 *   (block-scaled E4M3); the output sum is the fixed-order fp32 combine.
 */
int kt_moe_mxfp8_quantize(int64_t rows, int64_t K, const void* src, uint8_t* codes,
                          uint8_t* scales, void* stream);
size_t kt_moe_mxfp8_scale_bytes(const kt_moe_config* cfg, int down);
int kt_moe_mxfp8_pack(const kt_moe_config* cfg, const void* w1, const void* w3, const void* w2,
                      uint8_t* w1q, uint8_t* w3q, uint8_t* w2q, uint8_t* sf_up, uint8_t* sf_down,
                      void* stream);
int kt_moe_forward_mxfp8(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                         const float* bias, const uint8_t* w1q, const uint8_t* w3q,
                         const uint8_t* w2q, const uint8_t* sf_up, const uint8_t* sf_down,
                         void* y, int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                         size_t ws_bytes, void* stream, void* const* stage_events);

/*
 * MXFP4 expert weights: the 4-bit form of the layer (cfg->dtype =
 * KT_DTYPE_MXFP4). The KTransformers DeepSeek page runs routed experts held
 * natively in MXFP4 ("DeepSeek V4-Flash", its training notes) and gives no
 * quantisation rule. Format: E2M1 elements (1 sign bit, 2 exponent bits with
 * bias 1, 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one
 * power-of-two scale 2^e per 32 consecutive elements along K, stored as the
 * byte e + 127. Rule (the MXFP8 rule with 6 for 448): e is the smallest integer
 * with amax <= 6 * 2^e (0 gives e = -127), each element the E2M1
 * round-to-nearest-even of v * 2^-e. Codes are packed two per byte, element 2i
 * in the low nibble of byte i, the sign in bit 3 of its nibble.
 *
 * kt_moe_mxfp4_quantize: row-major [rows, K] bf16 (K % 32 == 0) -> packed codes
 *   [rows, K/2] bytes and scale bytes [rows, K/32]; 16-B aligned src and codes.
 *
 * The MXFP8 entry points take MXFP4 configs unchanged: kt_moe_mxfp8_pack writes
 *   packed codes (w1q, w3q [E+S, inter, dim/2], w2q [E+S, dim, inter/2] bytes)
 *   and the scales in the layout above (kt_moe_mxfp8_scale_bytes, the same
 *   sizes); kt_moe_forward_mxfp8, kt_moe_graph_create_mxfp8 and the
 *   expert-parallel *_mxfp8 forms run the 4-bit layer. The code pointers must be
 *   32-byte aligned and w3q - w1q a multiple of 32 bytes (KT_ERR_ALIGN). Tokens
 *   and SwiGLU hidden rows stay MXFP8 (E4M3); the GEMMs run the block-scaled
 *   tensor-core MMA with E2M1 weights and E4M3 tokens, fp32 accumulation.
 */
int kt_moe_mxfp4_quantize(int64_t rows, int64_t K, const void* src, uint8_t* codes,
                          uint8_t* scales, void* stream);

/*
 * Expert-parallel form: the multi-card steps of "MoE 前向四步" in the DeepSeek-V3
 * model.py notes (each card loops over its own experts only, y is all-reduced
 * over the cards, the shared experts' z is added); the number of cards is the
 * expert_parallel_degree setting of the tuning section ("性能调优策略") of the
 * DeepSeek model-family article (cloud.baidu.com/article/3606489). Per rank:
 *
 * kt_moe_forward_local: the gate on all T tokens (every rank computes the same
 *   routing from the same x, w_gate, bias), then
 *     y_part[t] = [shared_begin <= t < shared_end] * sum_s FFN_s(u_t)
 *               + sum over slots j with expert_begin <= idx[t,j] < expert_end
 *                 of w[t,j] * FFN_idx[t,j](u_t)
 *   in fp32, without the residual. The shared experts' tokens are split over
 *   the ranks (the sum over ranks is the same as adding z once after the
 *   all-reduce, in one message instead of two).
 *     expert_begin, expert_end   routed experts of this rank, 0 <= b <= e <= E
 *     shared_begin, shared_end   its tokens of the shared experts, 0 <= b <= e <= T
 *     w1, w3 [ (expert_end - expert_begin) + S, inter, dim ], w2 [ ..., dim,
 *       inter ]: slot i < expert_end - expert_begin holds routed expert
 *       expert_begin + i, the last S slots the shared experts (dtype of cfg)
 *     y_part  device [T, dim] fp32 (out), 16-B aligned, not overlapping x or the
 *             workspace; every row is written (zeros for a token with no local
 *             work)
 *   x, w_gate, bias, topk outputs, workspace (kt_moe_workspace_size of the full
 *   config) and errors as for kt_moe_forward; a range outside its bounds:
 *   KT_ERR_INVALID_CONFIG; an MXFP8 config: KT_ERR_INVALID_CONFIG (use
 *   kt_moe_forward_local_mxfp8, with codes and scales from
 *   kt_moe_mxfp8_pack_local on the same local stacks, sized by
 *   kt_moe_mxfp8_scale_bytes_local: the layouts of kt_moe_mxfp8_pack with the
 *   group index g running over the local slots).
 *
 * kt_moe_forward_placed (and _mxfp8): the same with any placement of the routed
 *   experts instead of a range. expert_slot: host array of E entries, the weight
 *   slot of routed expert e on this rank or -1 if it runs elsewhere; the slots
 *   used must be exactly 0 .. n_local - 1, each once (n_local = the number of
 *   entries >= 0), else KT_ERR_INVALID_CONFIG; NULL: KT_ERR_NULL. The local
 *   stacks hold n_local routed slots, then the S shared experts; MXFP8 stacks
 *   are packed by kt_moe_mxfp8_pack_local(cfg, 0, n_local, ...). A placement by
 *   expected load (several heavy experts on different ranks) evens out the
 *   ranks' work, which a contiguous range does not under a skewed load. The
 *   table is read on the host during the call.
 *
 * kt_moe_ep_finish: after the caller's sum of y_part over the ranks into y_sum
 *   (an all-reduce; fp32 [T, dim], device), y = y_sum (+ x if add_residual) in
 *   y's type (as kt_moe_forward). y may be y_sum itself when y is fp32; any
 *   other overlap: KT_ERR_INVALID_CONFIG. x may be NULL without the residual.
 */
int kt_moe_forward_local(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                         const float* bias, int expert_begin, int expert_end,
                         int64_t shared_begin, int64_t shared_end, const void* w1, const void* w3,
                         const void* w2, float* y_part, int32_t* topk_idx_out, float* topk_w_out,
                         void* workspace, size_t ws_bytes, void* stream);
int kt_moe_forward_local_mxfp8(const kt_moe_config* cfg, int64_t T, const void* x,
                               const void* w_gate, const float* bias, int expert_begin,
                               int expert_end, int64_t shared_begin, int64_t shared_end,
                               const uint8_t* w1q, const uint8_t* w3q, const uint8_t* w2q,
                               const uint8_t* sf_up, const uint8_t* sf_down, float* y_part,
                               int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                               size_t ws_bytes, void* stream);
int kt_moe_forward_placed(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                          const float* bias, const int32_t* expert_slot, int64_t shared_begin,
                          int64_t shared_end, const void* w1, const void* w3, const void* w2,
                          float* y_part, int32_t* topk_idx_out, float* topk_w_out,
                          void* workspace, size_t ws_bytes, void* stream);
int kt_moe_forward_placed_mxfp8(const kt_moe_config* cfg, int64_t T, const void* x,
                                const void* w_gate, const float* bias, const int32_t* expert_slot,
                                int64_t shared_begin, int64_t shared_end, const uint8_t* w1q,
                                const uint8_t* w3q, const uint8_t* w2q, const uint8_t* sf_up,
                                const uint8_t* sf_down, float* y_part, int32_t* topk_idx_out,
                                float* topk_w_out, void* workspace, size_t ws_bytes,
                                void* stream);
int kt_moe_ep_finish(const kt_moe_config* cfg, int64_t T, const float* y_sum, const void* x,
                     void* y, void* stream);
size_t kt_moe_mxfp8_scale_bytes_local(const kt_moe_config* cfg, int expert_begin, int expert_end,
                                      int down);
int kt_moe_mxfp8_pack_local(const kt_moe_config* cfg, int expert_begin, int expert_end,
                            const void* w1, const void* w3, const void* w2, uint8_t* w1q,
                            uint8_t* w3q, uint8_t* w2q, uint8_t* sf_up, uint8_t* sf_down,
                            void* stream);

/*
 * Scores alone: s = the score function of the gate logits, gate step 1 of the
 * "Gate 选专家流程（model.py，五步）" passage of the DeepSeek-V3 model.py notes
 * (sigmoid, or softmax over all experts), for the balance statistics below or
 * for the caller's own use.
 *   x, w_gate   as for kt_moe_gate
 *   scores_out  device [T, E] fp32 (out)
 *   workspace   device, ws_bytes >= kt_moe_workspace_size(cfg, T), 256-B aligned
 * Computed by the same code as kt_moe_gate's selection, so kt_moe_gate with
 * scores_in = scores_out gives exactly the routing kt_moe_gate computes from x.
 */
int kt_moe_scores(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                  float* scores_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Aux-loss-free bias update ("V3 改进①：无辅助损失负载均衡" of the DeepSeek-V3
 * model.py notes: the selection bias follows each expert's load, at a speed
 * gamma). The load of expert i is the number of its picks among the T*k
 * (token, slot) pairs of topk_idx; the mean load is T*k/E. An expert above the
 * mean has its bias lowered by gamma, one below it raised by gamma, one exactly
 * at it keeps its bias (compared in integers; one fp32 addition per expert).
 *   topk_idx  device [T, k] int32: a routing (kt_moe_gate / kt_moe_forward);
 *             indices outside [0, E) are not counted
 *   bias      device [E] fp32, updated in place
 *   gamma     finite, >= 0
 *   load_out  device [E] int32 or NULL (out): the loads
 * One kernel on `stream`, no workspace. Errors: KT_ERR_INVALID_CONFIG (config,
 * T or gamma), KT_ERR_NULL, KT_ERR_ALIGN (4-B alignment), KT_ERR_CUDA.
 */
int kt_moe_bias_update(const kt_moe_config* cfg, int64_t T, const int32_t* topk_idx,
                       float* bias, float gamma, int32_t* load_out, void* stream);

/*
 * Sequence-wise balance statistics ("V3 改进②：序列级平衡损失" of the DeepSeek-V3
 * model.py notes, L_Bal = alpha * sum_i f_i * P_i) over T tokens:
 *   f_i = load_i / T                          (top-k activation frequency)
 *   P_i = (1/T) * sum_t s_{i,t} / sum_j s_{j,t} (time mean of the normalised
 *                                               affinity)
 *   scores    device [T, E] fp32: s after the score function (kt_moe_scores)
 *   topk_idx  device [T, k] int32 (indices outside [0, E) are not counted)
 *   alpha     finite
 *   f_out, P_out  device [E] fp32 (out); loss_out device [1] fp32 (out)
 *   workspace device, ws_bytes >= kt_moe_balance_workspace_size(cfg, T),
 *             256-B aligned
 * fp32 sums in a fixed order (per token, per chunk of tokens, then over the
 * chunks), so repeated calls give bitwise-equal results; the loss sums the E
 * products in double. The page gives f_i only as the activation frequency: any
 * constant factor on it (the paper's experts / top-k normalisation) is a
 * factor on alpha.
 */
size_t kt_moe_balance_workspace_size(const kt_moe_config* cfg, int64_t T);
int kt_moe_balance_stats(const kt_moe_config* cfg, int64_t T, const float* scores,
                         const int32_t* topk_idx, float alpha, float* f_out, float* P_out,
                         float* loss_out, void* workspace, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then read the device error word the last call on this
 * workspace left (a bounded wait inside a kernel that gave up sets it; in the
 * checked build, so does an index check that failed).
 * Returns KT_OK, KT_ERR_TIMEOUT, KT_ERR_BOUNDS (checked build only), or
 * KT_ERR_CUDA if the stream reports an error. */
int kt_moe_check(const void* workspace, void* stream);

/* Byte offsets of the internal buffers inside the workspace, for tests and
 * debugging (all -1 if the config is invalid). Counts: per-group row counts
 * [E+S]; offsets: exclusive prefix [E+S+1]; row_of: [T, k] row of (t, j) in the
 * expert-sorted order; tok_of: [T*k] token of each sorted row; hidden: SwiGLU
 * hidden rows [T*(k+S), inter] (dtype); expert_out: weighted expert outputs
 * [T*(k+S), dim] (fp32). Rows T*k + s*T + t belong to shared expert s.
 * meta: int32 [3] = number of GEMM chunks, gate/up tiles, down tiles; chunks:
 * int32 [n][4] = (group, first row, rows, first activation row) of chunks of at
 * most 256 rows; tiles_up / tiles_down: int32 [n][2] = (chunk, feature tile)
 * in schedule order (feature tiles of 128 / 256 rows). */
typedef struct {
  int64_t error_word;
  int64_t logits;         /* fp32 [T][E] gate logits after the call (for T <= 64 the region
                             holds logits_splits [T][E] slots of partial sums over K; the
                             first is overwritten with their sum, added in order) */
  int64_t logits_splits;
  int64_t counts;
  int64_t offsets;
  int64_t row_of;
  int64_t tok_of;
  int64_t row_weight;
  int64_t hidden;
  int64_t expert_out;
  int64_t meta;
  int64_t chunks;
  int64_t tiles_up;
  int64_t tiles_down;
  int64_t total;
  /* MXFP8 layers (else -1): xq, xs = E4M3 codes [T, dim] and scale bytes
   * [T, dim/32] of x; xperm = codes of the permuted routed rows [T*k, dim];
   * tok_sf / hid_sf = the scales of each GEMM chunk's token / hidden rows,
   * [chunk][K/128][1024 B] (two 512-byte halves of 128 rows, scale of row m and
   * K block b at 512 (m / 128) + 16 (m % 32) + 4 (m / 32 % 4) + b % 4); hidden
   * holds E4M3 codes; chunks have at most 224 rows. */
  int64_t xq;
  int64_t xs;
  int64_t xperm;
  int64_t tok_sf;
  int64_t hid_sf;
} kt_moe_ws_layout;

int kt_moe_workspace_layout(const kt_moe_config* cfg, int64_t T, kt_moe_ws_layout* out);

/* Static description of an error code. */
const char* kt_moe_strerror(int code);

/* Library version: (major << 16) | minor. */
int kt_moe_version(void);

/* 1 for the checked build (libktmoe_checked.so, compiled with -DKT_CHECKED),
 * 0 for the release build. The checked build range-checks, where it is used,
 * every index one kernel takes from another kernel's output (expert ids, the
 * row maps row_of / tok_of, the GEMM chunk and tile lists, chunk counts): a
 * failed check skips the access and records KT_ERR_BOUNDS for kt_moe_check.
 * Same entry points, same results; it is a debugging aid, not a fast path. */
int kt_moe_checked_build(void);

#ifdef __cplusplus
}
#endif

#endif /* KTMOE_H */
