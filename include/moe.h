/*
 * moe.h - C ABI of the block-quantised routed mixture-of-experts FFN layer,
 * for one NVIDIA B200 (sm_100a).
 *
 * The layer is the routed MoE FFN of a Qwen3.8-Flash-Next-style model: the
 * model card "Qwen3.8-Flash-Next-Basalt" and the "llms-full.txt" FAQ describe
 * a mixture-of-experts model whose tokens each use only their selected
 * experts, and the "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model
 * card, section "What was changed", names the fast path a device-planned MoE
 * tail with grouped kernels over routed experts stored as IQ4_NL, NVFP4, Q5_1
 * or Q8_0.  Per token t the layer computes
 *
 *   l_e   = sum_h Wr[e,h] x[t,h]                    router logits (fp32 accumulate)
 *   S     = the top_k largest l_e, ties to the lower expert index
 *   g_e   = exp(l_e - max l) / sum_{j in S} exp(l_j - max l)   (softmax renormalised over S)
 *   y_e   = D_e (silu(G_e x) * (U_e x))              SwiGLU expert, fp32 accumulate
 *   out_t = sum_{e in S} g_e y_e  (+ y_shared when the pack has a shared expert)
 *
 * Memory: every pointer argument named "device" is CUDA device memory of the
 * pack's device (torch tensors qualify); "host" pointers are ordinary host
 * memory.  Device pointers must be 16-byte aligned.  The caller owns x,
 * router weights, outputs and the stream; the library owns each pack (its
 * device weight arena and a workspace sized at pack time).
 *
 * Streams and errors: argument errors return synchronously before anything is
 * enqueued.  Forward and route calls only enqueue work on `stream`; they do
 * not synchronise the host and do not allocate.  A launch failure returns
 * MOE_ERR_CUDA.  Errors raised inside kernels (a bounded wait that ran out, a
 * plan overflow) set a sticky word that moe_get_device_error() returns.  Every
 * device-side wait gives up after one to two seconds; the kernel then waits
 * (again bounded) for the copies and tensor-core operations it has already
 * issued, releases its tensor memory and returns, so the context stays usable
 * and the forward's outputs are undefined.
 * One pack runs one forward at a time: two forwards on one pack must be
 * ordered (same stream, or events); concurrent streams need separate packs.
 * The one-launch decode kernels (one token, and the device-planned tail of
 * 2-64 tokens) run one CTA per SM whose CTAs hand data to one another, so all
 * of them must be resident at once: a forward that long-running kernels of
 * another stream on the same GPU keep from some SMs waits for them, and if
 * that lasts beyond its bounded waits it records MOE_ERR_TIMEOUT (outputs
 * undefined) instead of hanging.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, top_k out of range */
    MOE_ERR_UNSUPPORTED = 2,  /* valid but not implemented (format/shape combination) */
    MOE_ERR_FMT_MISMATCH = 3, /* fmt argument disagrees with the pack */
    MOE_ERR_OOM = 4,          /* device or host allocation failed (pack only) */
    MOE_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    MOE_ERR_TIMEOUT = 6,      /* a bounded device-side wait ran out */
    MOE_ERR_DEVICE = 7,       /* a kernel detected an inconsistent plan */
    MOE_ERR_RANGE = 8         /* an intermediate left the fp16 range of the tensor-core
                                 decode path (|h| > 65504); run MOE_PATH_GROUPED instead */
} moe_status;

/* Block formats, each along the reduction (K) dimension of a weight row:
 *   Q8_0   32 weights in 34 B: fp16 d, int8 q[32]                 w = d*q
 *   Q5_1   32 weights in 24 B: fp16 d, fp16 m, u32 qh, qs[16]     w = d*q + m, q in [0,31]
 *   Q5_0   32 weights in 22 B: fp16 d, u32 qh, qs[16]             w = d*(q - 16), q in [0,31]
 *   IQ4_NL 32 weights in 18 B: fp16 d, qs[16] (4-bit indices)     w = d*T[i], T from the pack desc
 *   NVFP4  16 weights in  9 B: E4M3 scale, 8 B of E2M1 codes, and one fp32
 *          scale s per matrix                                     w = s*e4m3*e2m1
 * Byte order inside a block (little endian):
 *   Q8_0   [0,2) d  [2,34) q
 *   Q5_1   [0,2) d  [2,4) m  [4,8) qh (bit j is bit 4 of element j)  [8,24) qs
 *   Q5_0   [0,2) d  [2,6) qh  [6,22) qs (as Q5_1 without m)
 *   IQ4_NL [0,2) d  [2,18) qs
 *   for Q5_1, Q5_0 and IQ4_NL element j < 16 is the low nibble of qs[j] and element
 *   j >= 16 the high nibble of qs[j-16];
 *   NVFP4  [0] E4M3 scale  [1,9) codes: element 2i is the low, 2i+1 the high
 *   nibble of byte 1+i.
 * IQ4_NL is 4.5 bits per weight, the size the UD-IQ2_XS model card ("What was
 * changed") gives when it requantises a Q5_0 tensor (5.5 bits) to IQ4_NL.
 * A Q5_0 projection is packed as Q5_1 planes with m = -16 d (exact; 16|d| must
 * not exceed 65504, else MOE_ERR_INVALID_ARG): every kernel serves it, at two
 * more bytes per block of HBM traffic. */
typedef enum {
    MOE_FMT_FROM_PACK = 0, /* forward: accept the pack's formats */
    MOE_FMT_Q8_0 = 1,
    MOE_FMT_Q5_1 = 2,
    MOE_FMT_IQ4_NL = 3,
    MOE_FMT_NVFP4 = 4,
    MOE_FMT_Q5_0 = 5
} moe_fmt;

typedef enum { MOE_DT_F32 = 1, MOE_DT_BF16 = 2 } moe_dtype;

/* Kernel path of a forward.  AUTO picks DECODE for n_tokens <= 64 (decode and
 * speculative-verify batches) and PREFILL above when the pack can run it (both
 * projections NVFP4 - native block-scaled FP4 MMA with the activations rounded
 * to NVFP4 per token - or Q8_0 / IQ4_NL / Q5_1 in any mix - weights dequantised
 * to bf16 for bf16 MMA; hidden and inter multiples of 256, bf16 activations,
 * top_k <= 32; its buffers are sized at pack time when max_tokens > 64), else
 * GROUPED.  DECODE: one token runs the single-token streaming kernel; 2 to 64
 * tokens run the tensor-core decode (weights expanded to fp16, fp32
 * accumulation; hidden and inter multiples of 256 and every weight an fp16
 * normal number or zero, checked at pack time) as one launch, the
 * device-planned tail (TAIL, when its plan fits: top_k <= 16, the pack built
 * for at most 64 tokens), else as separate launches (DECODE_STAGED: route and
 * plan, x gather, gate/up, down, combine), else the CUDA-core grouped
 * kernels.  Packs holding an expert window always take the tail.  DENSE is the dense-batched comparison variant (pack created with
 * MOE_PACK_DENSE, n_tokens <= 64): every active expert multiplies the whole
 * batch, with a zero gate for the tokens not routed to it. */
typedef enum {
    MOE_PATH_AUTO = 0,
    MOE_PATH_DECODE = 1,   /* see above; falls back to GROUPED where its kernels do not apply */
    MOE_PATH_PREFILL = 2,
    MOE_PATH_DENSE = 3,
    MOE_PATH_GROUPED = 4,  /* decode as separate route / gate-up / down / combine launches, fp32 CUDA cores */
    MOE_PATH_DECODE_STAGED = 5, /* 2-64 tokens: the tensor-core grouped decode as separate launches (route and
                                   plan, x gather, gate/up, down, combine); MOE_ERR_UNSUPPORTED where it does
                                   not apply */
    MOE_PATH_TAIL = 6,     /* 1-64 tokens: the whole layer in one launch (routing, plan, tensor-core gate/up
                              and down over every SM, combine; hidden and inter multiples of 256, top_k <= 16,
                              fp16-representable weights); MOE_ERR_UNSUPPORTED where it does not apply */
    MOE_PATH_PREFILL_BF16 = 7 /* the prefill with every format's weights dequantised to bf16 in shared memory
                                 and bf16 MMA, NVFP4 included (its weights are exact in bf16: x is not rounded
                                 to NVFP4, h is rounded to bf16); same conditions as PREFILL */
} moe_path;

/* Description of one layer's experts, all in HOST memory; moe_pack_experts
 * copies what it needs, the caller keeps ownership.
 *   gate_up_blocks  n_experts x [2*inter rows x hidden] canonical blocks, rows
 *                   0..inter-1 are the gate projection G, inter..2*inter-1 the
 *                   up projection U, expert after expert
 *   down_blocks     n_experts x [hidden rows x inter] blocks (D)
 *   *_tensor_scale  NVFP4 only: one fp32 scale per expert, n_experts entries
 *                   (+1 for the shared expert, at index n_experts); else NULL
 *   iq4nl_table     16 int8 entries, required when a projection is IQ4_NL
 *   shared_*_blocks the always-on shared expert (gate 1), same shapes and
 *                   formats, required iff has_shared
 *   max_tokens, max_top_k  size the pack's workspace (forward refuses more)
 * Constraints: hidden and inter are multiples of 32 (all formats), hidden <=
 * 16384, inter <= 16384, 1 <= n_experts <= 1024, 1 <= max_top_k <= n_experts,
 * 1 <= max_tokens <= 65536. */
typedef struct {
    int n_experts;
    int hidden;
    int inter;
    int has_shared;
    int max_tokens;
    int max_top_k;
    moe_fmt fmt_gate_up;
    moe_fmt fmt_down;
    const void *gate_up_blocks;
    const void *down_blocks;
    const float *gate_up_tensor_scale;
    const float *down_tensor_scale;
    const int8_t *iq4nl_table;
    const void *shared_gate_up_blocks;
    const void *shared_down_blocks;
    int flags;            /* MOE_PACK_* bits, 0 for none */
    /* Expert parallelism: the pack holds only routed experts [expert_begin,
     * expert_end) of the layer's n_experts.  The block arrays (and NVFP4 scales)
     * then hold those experts, in order, followed by the shared expert when
     * has_shared.  Routing still covers all n_experts (pass the whole router);
     * a forward computes the partial layer
     *   out_t = sum_{e in S, expert_begin <= e < expert_end} g_e y_e (+ y_shared)
     * so the outputs of packs whose windows partition [0, n_experts), with the
     * shared expert in exactly one of them, sum to the layer.  0 and 0 (or 0
     * and n_experts) = every expert.  A windowed pack runs the one-launch tail
     * (1-64 tokens: AUTO, DECODE or TAIL); other paths return
     * MOE_ERR_UNSUPPORTED. */
    int expert_begin;
    int expert_end;
} moe_pack_desc;

/* moe_pack_desc.flags: size the workspace for MOE_PATH_DENSE as well (every
 * active expert times the whole batch: (n_experts + 1) * max_tokens slots). */
#define MOE_PACK_DENSE 1

typedef struct moe_pack moe_pack; /* opaque; owns device memory */

/* Sizes of a pack, for accounting (bytes are HBM bytes of the packed blocks). */
typedef struct {
    int64_t gate_up_bytes_per_expert;
    int64_t down_bytes_per_expert;
    int64_t expert_bytes;         /* gate_up + down (+ NVFP4 matrix scales) */
    int64_t arena_bytes;          /* all experts incl. shared */
    int64_t workspace_bytes;
    int device;
    /* 4-bit code lookups of the decode kernels: bit 0 set when the gate/up
     * projection's table needs the masked lookup (its entries cannot be paired
     * for the XOR-combined one), bit 1 the same for down; 0 otherwise and for
     * formats without a table */
    int code_table_masked;
} moe_pack_info;

/* Validate `desc`, repack every expert's blocks into the device layout (scales
 * split from codes, 16-byte aligned rows) and upload them to `device`; also
 * allocate the forward workspace.  Synchronous.  Rejects NVFP4 block scales
 * that are negative or NaN (MOE_ERR_INVALID_ARG).  On success *out owns the
 * device memory until moe_pack_free. */
moe_status moe_pack_experts(const moe_pack_desc *desc, int device, moe_pack **out);

/* Free a pack (synchronises its device).  NULL is accepted. */
moe_status moe_pack_free(moe_pack *pack);

moe_status moe_pack_query(const moe_pack *pack, moe_pack_info *info);

/* Workspace bytes moe_route_topk needs for n_tokens x n_experts. */
size_t moe_route_workspace_bytes(int n_tokens, int n_experts);

/* Router GEMV, softmax and top-k of n_tokens tokens.
 *   x         device, [n_tokens x hidden], fp32 or bf16 (x_dtype), row-major
 *   router_w  device, [n_experts x hidden] bf16 bits, row-major
 *   idx_out   device, [n_tokens x top_k] int32: selected experts by descending
 *             logit, ties to the lower index
 *   gate_out  device, [n_tokens x top_k] fp32 gates (sum to 1 per token)
 *   workspace device, moe_route_workspace_bytes(n_tokens, n_experts) bytes,
 *             owned by the caller; its contents need no initialisation
 * hidden % 8 == 0, 1 <= top_k <= n_experts <= 1024, n_tokens >= 0; with
 * n_tokens == 0 the call returns MOE_OK and enqueues nothing (the pointers are
 * not read and may be NULL).  More than 64 bf16 tokens
 * run the router as a tensor-core GEMM.  If one of the kernels' bounded waits
 * (the GEMM's pipeline, or the bulk copy of router rows into shared memory)
 * runs out, int32 word 1 of the workspace holds MOE_ERR_TIMEOUT afterwards. */
moe_status moe_route_topk(const void *x, moe_dtype x_dtype, const uint16_t *router_w,
                          int n_tokens, int hidden, int n_experts, int top_k, int32_t *idx_out,
                          float *gate_out, void *workspace, size_t workspace_bytes,
                          void *stream);

/* moe_route_topk without a workspace argument.  This entry point has no
 * counterpart in the pages; it exists for callers that cannot allocate device
 * memory (code running while a global-mode stream capture is open, where
 * cudaMalloc is illegal, or a host framework that forbids allocation after
 * start-up because cudaMalloc/cudaFree can synchronise the device).  Its
 * scratch is a fixed array inside the library, present on every device that
 * loads it until the process exits:
 *   n_tokens * n_experts <= 65536 (e.g. 64 x 1024), else MOE_ERR_INVALID_ARG;
 *   nothing is allocated; the ticket it needs at zero is cleared on `stream`
 *   by each call;
 *   all calls on a device share the scratch: calls that overlap on the GPU
 *   (unordered streams) race and give wrong results;
 *   the first call on a device looks up the scratch address and sets the
 *   router kernel's shared-memory limit - make it before any stream capture
 *   starts (a set-up that failed is retried by the next call);
 *   every call runs the CUDA-core router kernel, also for more than 64 bf16
 *   tokens (where moe_route_topk uses its tensor-core GEMM); its outputs are
 *   the same;
 *   a bounded wait that ran out leaves idx_out and gate_out undefined and is
 *   reported by moe_route_noalloc_status().
 * Other arguments, layouts and outputs as moe_route_topk. */
moe_status moe_route_topk_noalloc(const void *x, moe_dtype x_dtype, const uint16_t *router_w,
                                  int n_tokens, int hidden, int n_experts, int top_k,
                                  int32_t *idx_out, float *gate_out, void *stream);

/* Status of the last moe_route_topk_noalloc call on the current device:
 * MOE_OK, or MOE_ERR_TIMEOUT when one of its kernel's bounded waits ran out
 * (its outputs are then undefined).  Synchronises the device, allocates
 * nothing, and clears the recorded error. */
moe_status moe_route_noalloc_status(void);

/* Diagnostic for tests of that status: enqueues on `stream` the one-thread
 * bounded wait of moe_debug_wait_timeout with the allocation-free router's
 * error word as its target; about a second later moe_route_noalloc_status()
 * returns MOE_ERR_TIMEOUT once. */
moe_status moe_debug_noalloc_wait_timeout(void *stream);

/* The whole layer: route, plan, grouped gate/up + SwiGLU, down, combine.
 *   x        device [n_tokens x hidden] fp32 or bf16
 *   router_w device [n_experts x hidden] bf16 bits
 *   fmt      MOE_FMT_FROM_PACK, or the pack's gate/up format (checked)
 *   out      device [n_tokens x hidden] fp32
 * 0 <= n_tokens <= max_tokens, 1 <= top_k <= max_top_k.  Enqueues on `stream`
 * (a cudaStream_t; NULL is the legacy default stream).  An empty batch
 * (n_tokens == 0) returns MOE_OK after the pack, format, top_k and path checks,
 * enqueues nothing, does not read x or out (either may be NULL) and leaves the
 * routing that moe_read_routing reports as the previous forward left it. */
moe_status moe_layer_forward(const void *x, moe_dtype x_dtype, const uint16_t *router_w,
                             const moe_pack *pack, moe_fmt fmt, int n_tokens, int top_k,
                             float *out, void *stream);

/* As moe_layer_forward with an explicit kernel path (see moe_path). */
moe_status moe_layer_forward_ex(const void *x, moe_dtype x_dtype, const uint16_t *router_w,
                                const moe_pack *pack, moe_fmt fmt, int n_tokens, int top_k,
                                float *out, moe_path path, void *stream);

/* After a forward: copy its routing and plan to HOST memory (synchronises
 * `stream`).  Any pointer may be NULL.
 *   idx   [n_tokens x top_k] int32, gate [n_tokens x top_k] fp32,
 *   counts [n_experts + 1] int32 tokens per expert (last entry: shared); a
 *   windowed pack counts only its own experts (0 for the others).
 * 1 <= n_tokens <= max_tokens and 1 <= top_k <= max_top_k, else
 * MOE_ERR_INVALID_ARG; they should be the last non-empty forward's. */
moe_status moe_read_routing(const moe_pack *pack, int n_tokens, int top_k, int32_t *idx,
                            float *gate, int32_t *counts, void *stream);

/* Kernel timing of forwards, for measurement.  moe_profile_begin creates
 * CUDA events (and a small device buffer) for up to max_forwards forwards
 * (this allocates: call it before a timed region or a stream capture); each
 * later forward on the pack then
 * records an event before each of its kernels and after the last one
 * (captured as event-record nodes when the stream is capturing).
 * moe_profile_end synchronises the device, adds the elapsed times per kernel
 * over all recorded forwards into ms[32] (host memory): [0..5] route+plan,
 * gate/up, down, combine of the grouped path, the fused decode kernel, the
 * whole tensor-core prefill sequence; [6..14] the fused kernel's phases as seen
 * by its first CTA (token staging, router, barrier, plan, gate/up, barrier,
 * down, barrier, combine), from its SM clock at the device's nominal rate;
 * [15..23] from the global timer, relative to the first CTA's start: for the
 * single-token streaming kernel the last CTA start, first and last CTA to
 * publish its router rows, to issue its routed copies, to finish gate/up, to
 * end; for the router kernel of the grouped paths the last CTA start, first
 * and last CTA with x and its router rows staged, with its logits written, and
 * the top-k and plan completions ([6..14] then hold the selecting CTA's steps);
 * [24..31] the streaming kernel's first CTA's time at eight internal points.  It
 * stores the
 * forward count in *n_forwards, and frees the events.  Forwards beyond
 * max_forwards are not recorded. */
moe_status moe_profile_begin(moe_pack *pack, int max_forwards);
moe_status moe_profile_end(moe_pack *pack, double *ms, int *n_forwards);

/* Fault injection for tests of the pack's error path: after n (>= 0) more
 * device allocations by moe_pack_experts succeed, the next one fails, once:
 * moe_pack_experts then frees what it had allocated and returns MOE_ERR_OOM
 * with *out NULL.  n = -1 turns the injection off (the failing allocation
 * also turns it off); n < -1 is MOE_ERR_INVALID_ARG.  Process-wide; no device
 * is touched by this call. */
moe_status moe_debug_fail_alloc_after(int n);

/* Diagnostic for tests of the failure path: enqueues on `stream` one
 * single-thread kernel that waits on an mbarrier nothing arrives on, with the
 * bounded wait every pipeline of the library uses; after about a second it
 * gives up and records MOE_ERR_TIMEOUT in the pack's error word, which
 * moe_get_device_error then returns.  The context stays usable.  Argument and
 * launch errors as the forward. */
moe_status moe_debug_wait_timeout(const moe_pack *pack, void *stream);

/* Diagnostic for tests of the NVFP4 tensor-core prefill's activation rounding
 * (its reading of the block-scaled FP4 MMA, which needs both operands in NVFP4):
 * runs the prefill's own quantiser on `rows` plain rows and writes what it
 * produces.  bf16 x goes through the quantiser of the gate/up activations (the
 * layer input), fp32 x through the one of the down activations (h).  Per row:
 *   row_scale[r] = max_i |x[r,i]| / (6 * 448)                (fp32)
 *   scales[r,b]  = E4M3 (round to nearest even, saturating) of
 *                  max over block b of |x| / (6 * row_scale[r])
 *   codes        = E2M1 of x / (row_scale * e4m3(scale)), nearest even,
 *                  saturating; 0 for a block whose scale is 0; element 2i in
 *                  the low nibble of byte i of the row
 *   x         device [rows x cols] bf16 or fp32
 *   codes     device [rows x cols/2] bytes, scales device [rows x cols/16]
 *             E4M3 bytes (row-major), row_scale device [rows] fp32
 * 1 <= rows <= 65536, 64 <= cols <= 16384 and cols % 64 == 0.  Allocates
 * temporaries and synchronises `stream` (tests only, not for a hot path). */
moe_status moe_debug_act_quant_nvfp4(const void *x, moe_dtype x_dtype, int rows, int cols, uint8_t *codes,
                                     uint8_t *scales, float *row_scale, void *stream);

/* Diagnostic for tests of the block decoders (the formats of the Unsloth
 * dynamic-quantisation page, "Quantization types", and of the UD-IQ2_XS model
 * card, "What was changed"): decodes rows [row0, row0 + nrows) of expert slot
 * `slot` of one projection of `pack` (proj 0: gate/up, rows 0 .. 2I - 1 the
 * gate rows then the up rows; 1: down, rows 0 .. H - 1; slot e - expert_begin
 * for routed expert e, the shared expert after the routed ones) with the
 * decoders the kernels use, from the pack's own planes:
 *   kind 0  fp16 bits of the tensor-core decode's expansion (one rounding of
 *           each weight to fp16)
 *   kind 1  fp32 values of the bf16-dequantising prefill's decoder (before
 *           its rounding to bf16)
 * NVFP4 weights come out as 2 x E2M1 x E4M3: the per-expert matrix scale (and
 * the halving) stay with the kernels' epilogues.
 *   out  device [nrows x cols] (cols: H for gate/up, I for down), uint16 for
 *        kind 0, float for kind 1, 16-byte aligned
 * Enqueued on `stream`, no synchronisation.  MOE_ERR_INVALID_ARG for a bad
 * projection, slot, row range, kind or pointer. */
moe_status moe_debug_dequant_rows(const moe_pack *pack, int proj, int slot, int row0, int nrows, int kind, void *out,
                                  void *stream);

/* Diagnostic for tests of the one-launch tail's host planner; touches no
 * device.  For a launch of n_tokens tokens on a pack built for max_tokens
 * (device formats: a Q5_0 projection is planned as Q5_1) over `grid` CTAs,
 * writes out[0..7] = {1 if the tail fits else 0, raw stages, B slots, bytes of
 * a raw stage, bytes of a B slot, bytes of the rings region (the routing and
 * planning scratch overlaid on it), dynamic shared memory per CTA, tensor-memory
 * A stages}.  MOE_ERR_INVALID_ARG for a NULL out or an unknown format or dtype. */
moe_status moe_debug_tail_plan(int n_tokens, int max_tokens, int hidden, int n_experts, int inter, int top_k,
                               moe_dtype x_dtype, moe_fmt fmt_gate_up, moe_fmt fmt_down, int grid, int64_t *out);

/* Sticky device-side error of the pack (synchronises its device), then clears it. */
moe_status moe_get_device_error(const moe_pack *pack);

const char *moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
