/*
 * moe.h -- C ABI of the B200 (sm_100a) quantised mixture-of-experts layer.
 *
 * One MoE layer forward of the GLM-5.2 744B model as run by the colibri
 * engine: DeepSeek-V3-style sigmoid router (noaux_tc grouped top-k with a
 * correction bias, routed_scaling_factor, one shared expert) -> batch-union
 * bucketing of tokens by expert -> SwiGLU experts whose int8 / packed int4
 * weights carry per-row fp32 scales and are dequantised on use, fed by Q8_0
 * int8 activations through integer dot products -> weighted combine.
 *
 * Sources, by page title and section:
 *  [GN] GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기" -- §구현된 주요 기능
 *       (router, shared expert, quantisation kernels, integer-dot kernel with
 *       Q8_0-style int8 activations, batch-union MoE), §디스크 스트리밍 기반 MoE
 *       실행 방식 (~19 MB per int4 expert).
 *  [WP] wpnews.pro "Colibri — รัน GLM-5.2 (744B MoE) บนเครื่อง 25GB RAM ด้วย
 *       Pure C ไฟล์เดียว" -- spec table (256 experts, 8 active + 1 shared,
 *       Router: DeepSeek-V3-style sigmoid (noaux_tc)), kernel table (int8
 *       Q8_0-style; int4 packed, dequant-on-use; routing matmul in f32),
 *       "Batch-Union MoE".
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers unless the name says host; the caller owns
 *    all memory.  Arrays are dense, row-major.  Calls are asynchronous on
 *    `stream` (a cudaStream_t passed as void*; NULL = legacy default stream)
 *    unless stated otherwise.
 *  - Arguments are validated on the host before anything is launched; a bad
 *    argument returns MOE_EINVAL / MOE_EUNSUPPORTED and launches nothing.  A
 *    failed launch returns MOE_ECUDA.  No call allocates device memory on the
 *    forward path, and no call throws.
 *  - Floating point: fp32 inputs and outputs; no fast-math anywhere.
 *  - Non-finite activations or weights give undefined (but memory-safe)
 *    results; the CPU test oracle rejects them.
 *  - Concurrent calls are safe as long as each has its own workspace (the
 *    fused small-batch kernel is a cooperative grid of one CTA per SM, so two
 *    of them on different streams run one after the other).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_EINVAL = -1,       /* null / misaligned pointer, negative or inconsistent size */
    MOE_EUNSUPPORTED = -2, /* well-formed but outside what the kernels support */
    MOE_EWORKSPACE = -3,   /* workspace smaller than moe_workspace_bytes() */
    MOE_ECUDA = -4,        /* a CUDA runtime call or kernel launch failed */
    MOE_EDEVICE = -5       /* a kernel recorded a fault (see moe_get_device_error) */
} moe_status;

/* Layer hyper-parameters.  The GLM-5.2 layer is hidden 6144, inter 2048,
 * 256 experts in 8 groups, top-4 groups, top-8, 1 shared, rsf 2.5.
 * Supported: hidden and inter multiples of 32 (up to 16384); n_experts <= 1024
 * and a multiple of n_groups; 2 <= n_experts/n_groups; 1 <= topk_groups <=
 * n_groups <= 32; 1 <= top_k <= min(32, topk_groups * n_experts / n_groups);
 * n_shared 0 or 1; wbits 8, 4 or 2 (int2 runs the fused small-batch kernel
 * when hidden and inter are multiples of 64, else the multi-kernel path).
 * expert_topp: the adaptive expert top-p ([GN] §모델 다운로드와 실행, option
 * list: "--topp", an adaptive expert top-p that reads 30-40% fewer experts;
 * the pages give no rule, this library reads it as nucleus selection over the
 * top_k picks, see moe_router_select).  0, or any value >= 1, keeps every
 * pick; it must be finite and >= 0.  The field was added last so that the
 * members before it keep their offsets. */
typedef struct {
    int hidden;
    int inter;
    int n_experts;
    int n_groups;
    int topk_groups;
    int top_k;
    int n_shared;
    float routed_scaling_factor;
    int wbits;
    float expert_topp;
} moe_config;

/* Packed expert weights for n experts, laid out expert-major:
 *   w_gate, w_up : [n][inter][hidden * wbits / 8] bytes
 *   w_down       : [n][hidden][inter * wbits / 8] bytes
 *   s_gate, s_up : [n][inter] fp32 row scales;  s_down : [n][hidden]
 * Codes are two's complement; int4 packs element 2j in the low nibble and
 * 2j+1 in the high nibble of byte j, int2 packs element 4j+m in bits
 * 2m..2m+1 of byte j ([GN] quantisation-kernel bullet: int8 /
 * packed int4 / packed int2 with per-row scales; the bit layout is this
 * library's).  Weight pointers must be 16-byte aligned, scale pointers
 * 4-byte aligned. */
typedef struct {
    const uint8_t *w_gate;
    const uint8_t *w_up;
    const uint8_t *w_down;
    const float *s_gate;
    const float *s_up;
    const float *s_down;
} moe_experts;

/* Q8_0 activation quantiser ([GN] integer-dot kernel bullet; [WP] kernel table
 * "int8 (Q8_0-style)").  For each block of 32 consecutive values of each of the
 * n_rows rows of x [n_rows][cols]: d = amax/127 (fp32 IEEE divide), q =
 * round-half-away-from-zero(x * (1/d)) in [-127, 127]; a block with amax below
 * FLT_MIN stores d = 0, q = 0.  Outputs q [n_rows][cols] int8 and d
 * [n_rows][cols/32] fp32.  cols must be a multiple of 32; x 16-byte aligned. */
int moe_quantize_act_q8_0(const float *x, int64_t n_rows, int cols, int8_t *q, float *d, void *stream);

/* Per-row symmetric weight quantiser and packer (the converter's requantise
 * step; [GN] §구현된 주요 기능, offline converter bullet).  For each row of
 * w [rows][cols] fp32: s = amax / qmax (qmax 127 for int8, 7 for int4, 1 for
 * int2), code = round-half-away(w * (1/s)) clamped to [-2^(wbits-1), qmax],
 * s = 0 and codes 0 when amax < FLT_MIN.  Outputs packed
 * [rows][cols * wbits / 8] and scales [rows].  wbits is 8, 4 or 2; cols a
 * multiple of 32. */
int moe_pack_weights(const float *w, int64_t rows, int cols, int wbits, uint8_t *packed, float *scales,
                     void *stream);

/* FP8 checkpoint requantiser (the offline converter's step: [GN] §구현된 주요
 * 기능, offline converter bullet; [WP] converter list: the FP8 checkpoint is
 * dequantised with its 128 x 128 block scales and requantised into the
 * engine's per-row container).  w_fp8 [rows][cols] holds FP8 E4M3 codes (1
 * sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 subnormal;
 * S.1111.111 NaN; no infinities), block_scales [ceil(rows/block)]
 * [ceil(cols/block)] fp32 row-major; each value is code * scale of its block
 * (one fp32 multiply), and the dequantised rows are quantised and packed
 * exactly as moe_pack_weights does.  cols a multiple of 32, block a multiple
 * of 32 (128 in the checkpoint); w_fp8 and scale pointers 4-byte aligned,
 * packed 16-byte aligned.  NaN codes give unspecified codes for their row.
 * Device pointers; asynchronous on stream. */
int moe_requant_fp8(const uint8_t *w_fp8, const float *block_scales, int64_t rows, int cols, int block, int wbits,
                    uint8_t *packed, float *scales, void *stream);

/* Bytes of device workspace that moe_router_select needs for T tokens. */
size_t moe_router_workspace_bytes(const moe_config *cfg, int T);

/* Router: DeepSeek-V3-style sigmoid with noaux_tc grouped top-k ([GN]
 * §구현된 주요 기능; [WP] spec table, Router row).  For each token t of
 * x [T][hidden]:
 *   logit[e] = sum_j x[t,j] * router_w[e,j]   (fp32 inputs, fp64 sum)
 *   s[e] = sigmoid(logit[e]), c[e] = s[e] + router_bias[e]      (fp64)
 *   group score = sum of the two largest c in the group; keep the topk_groups
 *   best groups; pick the top_k largest c among their experts (ties: lower
 *   index first).  idx[t][j] (int32) lists them in descending c order and
 *   w[t][j] = s / sum(s) * routed_scaling_factor (fp32, unbiased s).
 * With 0 < expert_topp < 1 each token's picks are then ordered by their share
 *   q = s / sum(s) (fp64; larger first, ties: the earlier pick), the shortest
 *   prefix whose running sum of q (fp64, in that order) reaches expert_topp is
 *   kept (at least one pick), and the kept weights are renormalised:
 *   w[t][j] = s / sum_kept(s) * routed_scaling_factor (kept s summed in pick
 *   order).  A dropped pick keeps its position j with idx = -1 and w = 0.
 * router_w [n_experts][hidden] fp32, router_bias [n_experts] fp32.
 * workspace: >= moe_router_workspace_bytes(cfg, T) bytes, 256-byte aligned. */
int moe_router_select(const moe_config *cfg, const float *x, int T, const float *router_w,
                      const float *router_bias, int32_t *idx, float *w, void *workspace, size_t ws_bytes,
                      void *stream);

/* Batch-union bucketing ([GN] "Batch-union MoE"; [WP] "Batch-Union MoE"):
 * a stable counting sort of the T*top_k (token, slot) pairs of idx [T][top_k]
 * by expert.  counts [n_experts], offsets [n_experts+1] (exclusive prefix
 * sums, offsets[n_experts] = the number n of routed pairs, T*top_k unless
 * the top-p dropped some) and perm [T*top_k], where perm lists t*top_k + j
 * for expert 0's pairs in increasing t, then expert 1's, etc., and ends with
 * -1 for each dropped pair.  idx = -1 marks a dropped pair.  This entry
 * point has no error word, so it does not detect invalid input: an index
 * outside [-1, n_experts) is treated like a dropped pair, and a token that
 * lists the same expert twice gives colliding perm entries (moe_layer_forward
 * never produces either; its own bucketing records the index fault in its
 * workspace's error word).
 * Supports n_experts * ceil(T/32) <= 24576 (T <= 3072 at 256 experts). */
int moe_bucket_tokens(const moe_config *cfg, const int32_t *idx, int T, int32_t *counts, int32_t *offsets,
                      int32_t *perm, void *stream);

/* Bytes of device workspace that moe_layer_forward needs for up to T_max
 * tokens (0 on an invalid config). */
size_t moe_workspace_bytes(const moe_config *cfg, int T_max);

/* Initialises the part of a workspace that the fused small-batch path
 * (T <= 4) keeps from one call to the next: 1 KiB at a fixed offset holding
 * the grid-wide counters of its persistent kernel (never reset between
 * calls; each call counts from the values it finds) and a marker.  The
 * forward entry points do this themselves the first time this process passes
 * them a given workspace pointer on a given device; call it when the memory
 * behind a pointer already used with them was written by anything else since
 * (a fused forward on such a workspace records error code 3 and computes
 * nothing when the marker is gone).  Enqueued on `stream`.  workspace: >=
 * moe_workspace_bytes(cfg, T_max) bytes. */
int moe_workspace_init(const moe_config *cfg, int T_max, void *workspace, size_t ws_bytes, void *stream);

/* One MoE layer forward ([GN] §구현된 주요 기능; [WP] spec table, kernel table,
 * "Batch-Union MoE"):
 *   route (as moe_router_select), bucket (as moe_bucket_tokens), then for every
 *   selected expert e and token t routed to it, and for the shared expert on
 *   every token:
 *     g = Wg.x, u = Wu.x   with x as Q8_0 (per-block int32 dots, then
 *                          s_row * sum_b d_b * isum_b)
 *     h = silu(g) * u, quantised to Q8_0, y = Wd.h  (same integer-dot form)
 *   out[t] = sum_j w[t,j] * y_{idx[t,j]}(t) + y_shared(t)   (no residual;
 *   the sum skips the pairs the top-p dropped, whose experts are not read).
 * x [T][hidden] fp32 (16-byte aligned), out [T][hidden] fp32.  routed holds
 * n_experts experts, shared n_shared (ignored when n_shared == 0).
 * workspace: >= moe_workspace_bytes(cfg, T) bytes, 256-byte aligned; it holds
 * every intermediate of the call (see moe_workspace_view), its error word and
 * the fused path's control region (see moe_workspace_init).
 * 0 <= T; T = 0 returns MOE_OK without launching. */
int moe_layer_forward(const moe_config *cfg, const float *x, int T, const float *router_w,
                      const float *router_bias, const moe_experts *routed, const moe_experts *shared,
                      float *out, void *workspace, size_t ws_bytes, void *stream);

/* Expert-parallel share of moe_layer_forward (the pages' multi-GPU expert
 * tier, [WP] "Multi-GPU expert tier": experts spread over GPUs).  Every rank
 * routes all tokens exactly as moe_layer_forward does, then computes only the
 * picks whose expert lies in [expert_lo, expert_hi), and the shared expert
 * when with_shared is 1:
 *   out[t] = sum over those picks j of w[t,j] * y_{idx[t,j]}(t)
 *            (+ y_shared(t) when with_shared)
 * so the layer's output is the sum of the ranks' outputs when their ranges
 * cover [0, n_experts) without overlap and exactly one rank adds the shared
 * expert (each rank's sum is rounded to fp32 before that cross-rank sum).
 * Only the experts of the range (and the shared expert when with_shared) are
 * read: `routed` may point at a bank of which only those experts exist, as
 * long as expert e's data sits where it would in a full bank.  Arguments,
 * workspace (the full layer's: moe_workspace_bytes(cfg, T)) and errors as
 * for moe_layer_forward; 0 <= expert_lo <= expert_hi <= n_experts and
 * with_shared 0 or 1, else MOE_EINVAL.  The workspace view then describes
 * this call: idx / w the full routing, the buckets only the range's picks. */
int moe_layer_forward_partial(const moe_config *cfg, const float *x, int T, const float *router_w,
                              const float *router_bias, const moe_experts *routed, const moe_experts *shared,
                              int expert_lo, int expert_hi, int with_shared, float *out, void *workspace,
                              size_t ws_bytes, void *stream);

/* moe_layer_forward with HOST activations: copies x_host [T][hidden] to the
 * workspace, runs the forward, copies the result to out_host [T][hidden] and
 * synchronises `stream`.  Host buffers should be pinned (cudaHostAlloc) for
 * asynchronous copies; pageable memory works but is slower.  Weights and the
 * workspace are device memory as for moe_layer_forward. */
int moe_layer_forward_host(const moe_config *cfg, const float *x_host, int T, const float *router_w,
                           const float *router_bias, const moe_experts *routed, const moe_experts *shared,
                           float *out_host, void *workspace, size_t ws_bytes, void *stream);

/* moe_layer_forward without a caller-provided workspace.  (The pages have no
 * counterpart: this exists for callers of this library.)
 *
 * Some callers cannot allocate device memory when they want to run the layer:
 * a host framework whose allocator has already reserved the device and owns
 * every buffer, a plugin that is handed only input and output buffers, or a
 * latency-critical loop where cudaMalloc (which can synchronise the device)
 * is not allowed.  This variant allocates nothing: its scratch is a fixed
 * 8 MiB array in the library's device memory (a file-scope __device__ array),
 * which every GPU that loads the library holds until the process exits.  The
 * caller still passes x, out and the weights as for moe_layer_forward.
 *
 * Limit: the layer's workspace for T tokens must fit in 8 MiB
 * (moe_workspace_bytes(cfg, T) <= 8388608); larger T returns MOE_EWORKSPACE
 * and launches nothing.  For the GLM-5.2 layer (hidden 6144, 256 experts,
 * top-8 + 1 shared) that allows T <= 17.
 *
 * The first call on each device looks up the array's device address with that
 * device current (once per device); make that first call before any stream
 * capture.  Every call shares the one array and it keeps the last call's
 * contents; each call clears what must start at zero.  Calls whose executions
 * overlap on the GPU (different streams, or different host threads) race on
 * the array and give wrong results: serialise them.  The intermediates are not
 * reachable through moe_workspace_view; the error word is read with
 * moe_noalloc_device_error.  The looked-up address belongs to the device's
 * context as it was at that first call: do not use this entry point after
 * cudaDeviceReset (or anything else that re-creates the primary context) in
 * the same process. */
int moe_layer_forward_noalloc(const moe_config *cfg, const float *x, int T, const float *router_w,
                              const float *router_bias, const moe_experts *routed, const moe_experts *shared,
                              float *out, void *stream);

/* moe_get_device_error for the allocation-free forward: synchronises `stream`
 * and reads the error word that the last moe_layer_forward_noalloc on the
 * current device left in the library's fixed scratch (codes as for
 * moe_get_device_error; a later noalloc call on the device resets it). */
int moe_noalloc_device_error(void *stream, int32_t *code);

/* Device pointers to the intermediates a moe_layer_forward call leaves in its
 * workspace (valid after the call completes, until the next call on the same
 * workspace).  Slots: routed (token, slot) pairs occupy bucket positions
 * 0 .. n-1 (the order of perm, n = offsets[n_experts]; positions n ..
 * T*top_k-1 are unused when the top-p dropped pairs); the shared expert of
 * token t is slot T*top_k + t. */
typedef struct {
    int8_t *xq;        /* [T][hidden]   Q8_0 codes of x */
    float *xd;         /* [T][hidden/32] Q8_0 scales of x */
    int32_t *idx;      /* [T][top_k]    selected experts */
    float *w;          /* [T][top_k]    combine weights */
    int32_t *counts;   /* [n_experts] */
    int32_t *offsets;  /* [n_experts+1] */
    int32_t *perm;     /* [T*top_k] */
    int8_t *hq;        /* [slots][inter]    Q8_0 codes of h per slot */
    float *hd;         /* [slots][inter/32] Q8_0 scales of h per slot */
    float *y;          /* [slots][hidden]   expert outputs per slot (unweighted) */
    int32_t *error;    /* device error word (0 = none); error[8] and error[9] are set
                        * by a batched tensor-core forward (T >= 64) whose activations
                        * (x, resp. h) had a token with block-scale exponents more than 8
                        * apart, so that its GEMM took the fp64-epilogue form instead of
                        * the digit planes (see moe_layer_forward) */
} moe_workspace_layout;

int moe_workspace_view(const moe_config *cfg, int T, void *workspace, size_t ws_bytes,
                       moe_workspace_layout *view);

/* Per-block int32 dot products of one packed matrix with Q8_0 codes, computed
 * by the same device routine as the expert kernels ([GN] integer-dot kernel):
 * out[t][r][b] = sum_{i<32} code(W[r, 32b+i]) * q[t, 32b+i] for W packed
 * [rows][cols * wbits / 8] (wbits 8, 4 or 2) and q [n][cols] int8. */
int moe_block_dots(const uint8_t *packed, int64_t rows, int cols, int wbits, const int8_t *q, int n,
                   int32_t *out, void *stream);

/* The device routines that compute a block dot on the forward path; each
 * kernel calls exactly one of them ([GN] integer-dot kernel bullet).
 *  MOE_DOTS_MULTI_KERNEL: the multi-kernel path's k_gateup / k_down routine
 *    (int8 dp4a; int4 nibbles shifted to the top of their byte, sum >> 4;
 *    int2 fields shifted to the top over crumb-ordered codes, sum >> 6).
 *    out = the dot.
 *  MOE_DOTS_FUSED: the fused small-batch kernel's routine (int4: low nibbles
 *    in excess-8 form with the excess removed through the starting value,
 *    high nibbles as 16 * code; int2 as above without the final shift).
 *    out = the dot times 16 (int4), 64 (int2) or 1 (int8), exactly: the
 *    kernel folds that power of two into the activation scale.
 *  MOE_DOTS_TENSOR: the batched path's tensor-core routine: the packed rows
 *    widened to int8 in shared memory, one tcgen05.mma kind::i8 (K = 32, one
 *    Q8_0 block) per block into a TMEM accumulator, read back as int32.
 *    out = the dot.  Needs n <= 64 and rows of a multiple of 16 bytes
 *    (cols * wbits / 8), else MOE_EUNSUPPORTED. */
enum { MOE_DOTS_MULTI_KERNEL = 0, MOE_DOTS_FUSED = 1, MOE_DOTS_TENSOR = 2 };

/* moe_block_dots through the routine `routine` (one of MOE_DOTS_*; anything
 * else returns MOE_EUNSUPPORTED).  Same arguments and layouts as
 * moe_block_dots; every packed byte value (all 16 nibbles, all 4 int2 fields)
 * and every int8 code is accepted. */
int moe_block_dots_routine(const uint8_t *packed, int64_t rows, int cols, int wbits, const int8_t *q, int n,
                           int routine, int32_t *out, void *stream);

/* Synchronises `stream` and reads the workspace's device error word into
 * *code (0 = none).  Returns MOE_OK when it is 0, MOE_EDEVICE otherwise.
 * Codes: 1 = an index out of range reached a kernel, 2 = a device-side wait
 * ran out of time, 3 = the fused path found the workspace's control region
 * uninitialised (see moe_workspace_init).  Every wait inside a kernel is bounded by the GPU's
 * global timer: a wait for a free pipeline slot or for another CTA's
 * results gives up after 25 ms, a wait that can span one of those after
 * 100 ms; the kernel then records code 2 and returns, leaving the call's
 * outputs unspecified. */
int moe_get_device_error(void *workspace, void *stream, int32_t *code);

/* Test hook of the failure-detection tests (the pages have no counterpart).
 * With withhold_entry >= 0, every following fused small-batch forward
 * (T <= 4) issued by this process skips the publication of the h codes of
 * gate/up unit 0 of entry withhold_entry (0 = the shared expert, 1 + a = the
 * a-th selected routed expert in ascending id order), so the down projection's
 * wait for them runs out: the forward still returns MOE_OK, its error word
 * reads 2 and its output is unspecified.  wait_budget_ns > 0 replaces the
 * 25 ms bound of the producer's waits (the longer waits scale with it);
 * 0 restores it.  withhold_entry = -1 switches the fault off.  The setting is
 * process-wide; set it only while no forward is being issued from another
 * thread.  Returns MOE_EINVAL for withhold_entry < -1 or a budget outside
 * [0, 10 s]. */
int moe_debug_fault_injection(int withhold_entry, int64_t wait_budget_ns);

/* Test export of the one-token fused forward's down-row split (no GPU work,
 * no device needed): the output rows [starts[c], starts[c + 1]) that CTA c of
 * a grid of `grid` CTAs owns in the down projection and the combine, for a
 * batch of T tokens whose union holds n_entries experts (the selected ones and
 * the shared one), as every CTA of k_moe_small computes it.  starts has
 * grid + 1 entries (starts[grid] = hidden); the caller owns it.  *row_cap
 * receives the per-CTA row cap of the split (0 for an even split).  Returns
 * MOE_EINVAL for an invalid config, T outside [1, 4], n_entries outside
 * [1, 1 + min(experts, T * top_k)], grid outside [1, 4096] or null
 * pointers. */
int moe_debug_down_rows(const moe_config* cfg, int T, int n_entries, int grid, int32_t* starts, int* row_cap);

/* Device copy of the seeded input generator (SplitMix64, counter-based; see
 * the package's synth module): out[i] = sigma * z(seed, tid, offset + i) with z
 * the centred Irwin-Hall sum of twelve 16-bit uniforms.  Used to draw
 * multi-GB synthetic expert weights directly in HBM; bit-identical to the
 * host generator. */
int moe_synth_normal(uint64_t seed, uint64_t tid, int64_t offset, int64_t n, float sigma, float *out,
                     void *stream);

/* Tracing hook: CUDA events at the phase boundaries of moe_layer_forward.
 * events points to MOE_PROFILE_MAX_EVENTS cudaEvent_t handles (passed as
 * void*), or is NULL (with n_events 0) to switch tracing off; the setting
 * belongs to the calling host thread.  While it is set, every forward issued
 * from that thread records events[0] on its stream before its first launch
 * and events[i] after phase i, for i = 1 .. moe_forward_phases(cfg, T).  The
 * phases depend on the path the forward takes: the fused small-batch path
 * (T <= 4) has one phase, "fused" (both of its kernels); the other paths have
 * five: "route" (Q8_0 of x, logits, selection), "bucket" (with, at T >= 64,
 * the tensor-core path's plan and gather), "gate_up" (the gate/up kernel),
 * "down" (at T >= 64 SwiGLU and the down GEMM), "combine".  The caller keeps the events alive until they have
 * completed. */
#define MOE_PROFILE_MAX_EVENTS 8
int moe_profile_events(void *const *events, int n_events);

/* Number of traced phases of a forward with T tokens, and the name of phase
 * i (0-based; "" when out of range).  Negative status on an invalid config. */
int moe_forward_phases(const moe_config *cfg, int T);
const char *moe_forward_phase_name(const moe_config *cfg, int T, int i);

/* Number of kernel launches one moe_layer_forward with T tokens issues
 * (0 for T = 0; negative status on an invalid config). */
int moe_forward_launches(const moe_config *cfg, int T);

/* Human-readable name of a status code. */
const char *moe_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
