// Internal definitions shared by the CUDA translation units of libmoe: the
// device layout of a pack, the forward workspace and the kernel argument
// blocks.  Nothing here is part of the public C ABI (include/moe.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kThreads = 256;      // threads per CTA of every kernel here
constexpr int kDecodeMaxTokens = 64;

// One projection (gate/up stacked, or down) of every expert, split into
// planes so each lane's code bytes are one aligned 16-byte load:
//   Q8_0    qs: rows x K int8 codes, stored XOR 0x80 (biased by +128)
//           sc: rows x K/32 fp16 d
//   Q5_1    qs: rows x K/2 (16 B per 32-block, canonical nibble order)
//           qh: rows x K/32 u32, sc: rows x K/32 {fp16 d, fp16 m}
//   IQ4_NL  qs: rows x K/2, sc: rows x K/32 fp16 d
//   NVFP4   qs: rows x K/2 (8 B per 16-block); sc: E4M3 block scales in the
//           tcgen05 block-scale layout (see sf_offset), shared by the decode
//           kernels and the block-scaled prefill MMA; ts: one fp32 matrix
//           scale per expert
// Expert e's plane starts at base + e * stride.
struct DevProj {
    int fmt = 0, rows = 0, cols = 0;
    const uint8_t *qs = nullptr;
    const uint8_t *sc = nullptr;
    const uint8_t *qh = nullptr;
    const float *ts = nullptr;
    int64_t qs_stride = 0, sc_stride = 0, qh_stride = 0;  // bytes per expert
    int qs_row = 0, sc_row = 0, qh_row = 0;               // bytes per row (sc_row: not NVFP4)
    int ksteps = 0;                                       // NVFP4: 64-wide K steps per row
    // scales row by row (2 bytes per 32 weights, 4 for Q5_1): the sc plane
    // itself, except for NVFP4, which keeps a second, row-major copy of its
    // E4M3 scales for the streaming decode kernel's bulk row copies
    const uint8_t *sr = nullptr;
    int64_t sr_stride = 0;
    int sr_row = 0;
    // every weight of the projection is an fp16 normal number or zero (the
    // tensor-core decode path expands blocks to fp16)
    bool f16_ok = false;
    // the same weights tile by tile for the one-launch tail: per expert slot,
    // per 128-row block, per 256-wide K chunk one contiguous block of
    // tl_block bytes (codes, then scales, then Q5_1 fifth bits) already in the
    // shared-memory layout the expanding warps read (codes in the 128-byte
    // swizzle; Q5_1 scales and fifth bits in the 32-byte swizzle), so that one
    // bulk copy moves a tile's chunk; null when the shape has no such tiles
    const uint8_t *tl = nullptr;
    int64_t tl_stride = 0;  // bytes per expert slot
    int tl_block = 0;       // bytes per (128-row block, K chunk)
};

// Sizes of one (128-row block, 256-wide K chunk) block of a tiled plane.
__host__ __device__ inline int tl_codes_bytes(int fmt) { return 128 * 128 * (fmt == MOE_FMT_Q8_0 ? 2 : 1); }
__host__ __device__ inline int tl_scales_bytes(int fmt) { return 128 * (fmt == MOE_FMT_Q5_1 ? 32 : 16); }
__host__ __device__ inline int tl_qh_bytes(int fmt) { return fmt == MOE_FMT_Q5_1 ? 128 * 32 : 0; }
__host__ __device__ inline int tl_block_bytes(int fmt) { return tl_codes_bytes(fmt) + tl_scales_bytes(fmt) + tl_qh_bytes(fmt); }

// Byte offset of E4M3 scale q (0..3) of row r in 64-wide K step s, in the
// block-scale layout of the tcgen05 block-scaled MMA: atoms of 512 bytes hold
// 128 rows x 4 scales, row r at (r % 32) * 16 + ((r / 32) % 4) * 4; atoms run
// over K steps first, then over 128-row blocks.
__host__ __device__ inline int64_t sf_offset(int r, int s, int q, int ksteps)
{
    return ((int64_t)(r >> 7) * ksteps + s) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + q;
}

// Forward workspace (device), sized at pack time for max_tokens x max_top_k.
struct Workspace {
    float *logits = nullptr;     // [T x E]
    int32_t *idx = nullptr;      // [T x k]
    float *gate = nullptr;       // [T x k]
    int32_t *cnt = nullptr;      // [E + 1]   tokens per expert (last: shared)
    int32_t *off = nullptr;      // [E + 1]   first slot of each expert
    int32_t *perm_tok = nullptr; // [T*k + T] slot -> token
    int32_t *slot_pos = nullptr; // [T x k]   (t, j) -> slot
    int4 *groups = nullptr;      // {expert, first slot, tokens, 0}
    int32_t *n_groups = nullptr;
    int32_t *ticket = nullptr;   // route kernel tickets: [0] token blocks done, [2 + b] CTAs of block b
    unsigned *bar = nullptr;     // grid barrier of the fused decode kernel {count, gen}
    int32_t *err = nullptr;      // sticky device error (moe_status)
    float *dgate = nullptr;      // dense-batched plan: per slot gate (0 when not routed)
    int32_t *n_dense_rows = nullptr;
    float *h = nullptr;          // [slots x I] (tensor-core decode: fp16 h)
    float *y = nullptr;          // [slots x H]
    uint16_t *xg = nullptr;      // [slots x H] tensor-core decode: fp16 x slot rows
    float *slot_scale = nullptr; // [slots] tensor-core decode: power-of-two scale of the slot's x
    int max_groups = 0;
    // single-token streaming kernel: {finished-CTA ticket, logits arrivals, h
    // arrivals}; all zero between launches (the last CTA to finish resets them)
    unsigned *xcnt = nullptr;
    // one-launch tail (tail_decode.cu): its counters (zero between launches)
    // and the fp32 pieces of tiles whose units span two CTAs
    unsigned *tail_ctr = nullptr;
    float *tail_part = nullptr;
};

// Tensor-core grouped decode (2 to kDecodeTcMaxN tokens): TMA maps of the
// fp16 slot rows of x and of h (workspace buffers, fixed per pack).
constexpr int kDecodeTcMaxN = 64;
struct DecodeTcMaps {
    CUtensorMap xg, h;
    CUtensorMap gu[3], dn[3];  // codes, row-major scales, fifth bits of each projection
};

struct RouteArgs {
    const void *x;
    int x_dtype;
    const uint16_t *wr;
    int T, H, E, k;
    int rt;                 // tokens staged per pass
    float *logits;
    int32_t *ticket;
    int32_t *idx;
    float *gate;
    // plan (only when do_plan)
    int do_plan, has_shared, tt;
    int32_t *cnt, *off, *perm_tok, *slot_pos, *n_groups, *err;
    int4 *groups;
    int max_groups;
    // dense-batched plan: every active expert takes the whole batch
    int dense;
    float *dgate;           // [slots] gate of (active expert, token), 0 if not routed
    int32_t *n_dense_rows;  // active experts (incl. shared) x T
    // profiling only (null otherwise): grid events folded into words 10..19 of
    // a forward's stamps, as {2^62 - first, last} global-timer pairs: 0 start,
    // 1 x and router rows staged, 2 logits written, 3 top-k done, 4 plan done; words 0..9
    // the SM clock of the selecting / planning CTA at: top-k begin, row staged,
    // selected, top-k done, plan begin, counts, scans, groups written, slot
    // order written, plan done
    long long *stamps;
};

// 16-entry code table of a 4-bit format, built on the host by build_code_table:
// entry bytes (value + bias) in t[0..3], magic = 2^23 + bias, xor_mode when the
// halves were arranged for the XOR-combined lookup (else masked select).
struct CodeTable {
    uint32_t t[4];
    float magic;
    int xor_mode;
};

struct MatvecArgs {
    DevProj w;
    const int4 *groups;
    const int32_t *n_groups;
    const int32_t *perm_tok;  // gate/up: slot -> token of x
    const void *x;            // gate/up: layer input [T x H]; down: h [slots x I] fp32
    int x_dtype;
    float *out;               // gate/up: h [slots x I]; down: y [slots x H]
    int out_stride;
    int rows_out;             // gate/up: I (row pairs); down: H
    CodeTable tab;            // 4-bit formats' code table
};

struct CombineArgs {
    const float *y;
    const int32_t *slot_pos;
    const float *gate;
    int T, k, H, has_shared;
    float *out;
};

// launchers (return cudaGetLastError of the launch)
size_t route_smem_bytes(int H, int rt, int E, int grid, int T);
void init_device_attributes();  // once per device, with that device current
int route_tokens_per_pass(int H);
cudaError_t launch_route(const RouteArgs &a, int grid, cudaStream_t s);
int route_grid(int E, int T, int rt, int num_sms);

cudaError_t launch_matvec(const MatvecArgs &a, bool gateup, int tt, int grid, cudaStream_t s);
size_t matvec_smem_bytes(const MatvecArgs &a, bool gateup, int tt);
int matvec_grid(const MatvecArgs &a, bool gateup, int tt, int num_sms);

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s);
cudaError_t launch_combine_dense(const float *y, const float *dgate, const int32_t *n_rows, int T, int H,
                                 float *out, cudaStream_t s);

// Fused decode (one cooperative launch per layer, n_tokens <= 8).
constexpr int kFusedMaxT = 8;
constexpr int kFusedMaxK = 16;

struct FusedArgs {
    const void *x;
    int x_dtype;
    const uint16_t *wr;
    int T, H, E, I, k, has_shared;
    DevProj gu, dn;
    CodeTable tab_gu, tab_dn;
    float *logits;      // [T x E]
    float *h;           // [slots x I]
    float *y;           // [slots x H] (when not rowsplit)
    float *out;         // [T x H]
    int32_t *idx_out;   // routing readback, written by CTA 0
    float *gate_out;
    int32_t *cnt_out;
    unsigned *bar;      // {arrive count, generation}
    int32_t *err;
    int rowsplit;       // down + combine by output rows in one phase
    long long *stamps;  // optional: [0..9] clock64 of CTA 0 at each phase boundary; [10..19]
                        // streaming kernel: per grid event {2^62 - first, last} global timer
    unsigned *xcnt;     // streaming kernel's hand-over counters (see Workspace)
};

// tensor-core prefill
struct PrefillWorkspace {
    float *logits = nullptr;   // [T x E]
    int32_t *idx = nullptr;    // [T x k]
    float *gate = nullptr;     // [T x k]
    int32_t *slot_pos = nullptr;
    int32_t *cnt = nullptr;    // [E + 1]
    int32_t *pad_off = nullptr, *fill = nullptr;  // [E + 1]
    int2 *tiles = nullptr;     // [max_rows / 128]  128-row M tiles
    int4 *ptiles = nullptr;    // [max_rows / 128]  pairs of M tiles of one expert (bf16 path)
    int32_t *n_tiles = nullptr, *total_rows = nullptr, *n_ptiles = nullptr;
    int32_t *perm_tok = nullptr;  // [max_rows]
    float *row_gate = nullptr, *row_scale_x = nullptr, *row_scale_h = nullptr;  // [max_rows]
    uint8_t *a_q = nullptr, *sfa = nullptr;  // gate/up activations: NVFP4 codes + scales, or bf16 rows (Q8_0)
    float *h = nullptr;                      // [max_rows x I]
    uint8_t *h_q = nullptr, *sfh = nullptr;  // NVFP4 activations of the down GEMM
    int max_rows = 0;
};

struct PrefillNvArgs {
    const void *x;  // bf16 [T x H]
    const uint16_t *wr;
    int T, H, I, E, k, has_shared;
    const DevProj *gu, *dn;
    CodeTable tab_gu, tab_dn;  // 4-bit formats (the dequantising path)
    float *out;
    int32_t *err;
    const PrefillWorkspace *ws;
    int num_sms;
};

cudaError_t prefill_set_attributes();
cudaError_t prefill_nvfp4_set_attributes();
bool prefill_nvfp4_supported(int H, int I, int E, int k);
cudaError_t prefill_nvfp4_forward(const PrefillNvArgs &a, cudaStream_t s);
// One-thread kernel that waits (bounded) on an mbarrier nothing arrives on and
// records MOE_ERR_TIMEOUT in *err: the failure-path diagnostic.
cudaError_t launch_wait_probe(int32_t *err, cudaStream_t s);
cudaError_t prefill_plan_launch(const PrefillWorkspace &w, int E, int T, int has_shared, int32_t *err, cudaStream_t s);
cudaError_t prefill_q8_set_attributes();
// Q8_0 / IQ4_NL / Q5_1 in any mix, and NVFP4 when `nvfp4` (the exact-weight variant beside the native FP4 GEMM)
bool prefill_q8_supported(int fmt_gu, int fmt_dn, int H, int I, int E, int k, bool nvfp4);
cudaError_t prefill_q8_forward(const PrefillNvArgs &a, cudaStream_t s);
cudaError_t prefill_route(const void *x_bf16, const uint16_t *wr, int T, int H, int E, int k, float *logits,
                          int32_t *idx, float *gate, int32_t *cnt, int32_t *err, cudaStream_t s);

// Streamed grouped matvec (stream_group.cu): per projection, TMA maps of the
// code / scale / fifth-bit planes (3-D: row bytes x rows x expert slots) and
// the stage layout of a 32-row block.
struct SgmProj {
    CUtensorMap map[3];
    int row_bytes[3], w[3], off[3];
    int stage_bytes, tx_bytes, fmt, ok;
};
bool sgm_prepare(const DevProj &w, int n_slots, bool gateup, SgmProj *out);
int sgm_max_groups();
int sgm_stages(const SgmProj &p, int K);
cudaError_t sgm_set_attributes();

// Tensor-core grouped decode (decode_tc.cu)
bool decode_tc_supported(const DevProj &gu, const DevProj &dn, int H, int I, int max_tokens, int max_top_k);
cudaError_t decode_tc_set_attributes();
bool decode_tc_maps(DecodeTcMaps *m, const DevProj &gu, const DevProj &dn, int n_experts, const void *xg,
                    const void *h16, int slots, int H, int I);
cudaError_t launch_decode_tc_gather(const void *x, int x_dtype, int T, int H, int k, int has_shared,
                                    const int32_t *slot_pos, void *xg, float *slot_scale, cudaStream_t s);
cudaError_t launch_decode_tc(const DecodeTcMaps &m, bool gateup, const DevProj &w, const int4 *groups,
                             const int32_t *n_groups, int H, int I, const CodeTable &tab, const float *slot_scale,
                             void *h16, float *y, int32_t *err, int max_tokens, int grid, cudaStream_t s);
cudaError_t launch_sgm(const SgmProj &p, const DevProj &w, const int4 *groups, const int32_t *n_groups,
                       const int32_t *perm_tok, const void *x, int x_dtype, float *out, int out_stride, int rows_out,
                       bool gateup, const CodeTable &tab, int32_t *err, int grid, cudaStream_t s);

// Single-token streaming decode (stream_decode.cu): same arguments as the
// fused kernel; every weight byte a CTA needs is requested by bulk copies into
// shared memory as soon as it is known.
size_t stream1_smem_bytes(const FusedArgs &a, int grid);
bool stream1_supported(const FusedArgs &a, int grid, size_t smem_limit);
int stream1_blocks_per_sm(const FusedArgs &a, size_t smem);
cudaError_t stream1_set_attributes();
cudaError_t launch_stream1(const FusedArgs &a, int grid, size_t smem, int pdl, cudaStream_t s);

// The one-launch device-planned tail of 1-64 tokens (tail_decode.cu).
struct TailPlanIn {
    int T, max_tokens, H, E, I, k, x_dtype, fmt_gu, fmt_dn, grid;
};
struct TailLaunch {
    int nr, na, nb, raw_stride, bslot, n16max, rings;
    size_t smem;
};
struct TailCall {
    const void *x;
    int x_dtype;
    const uint16_t *wr;
    int T, H, E, I, k, has_shared;
    int eb, ee;  // the pack's routed experts [eb, ee) (all: 0, E)
    const DevProj *gu, *dn;
    CodeTable tab_gu, tab_dn;
    const Workspace *ws;
    const DecodeTcMaps *maps;  // the x and h slot-row maps (16-row boxes) of the tensor-core decode
    float *out;
    long long *stamps;
};
int tail_counter_words(int E, int H, int I);
size_t tail_part_floats(int grid, int max_tokens);
bool tail_plan(const TailPlanIn &in, TailLaunch *out);  // false: the shape or the shared memory does not fit
cudaError_t tail_set_attributes();
int tail_blocks_per_sm(int fmt_gu, int fmt_dn, size_t smem);
cudaError_t launch_tail(const TailCall &t, const TailLaunch &L, int grid, int pdl, cudaStream_t s);

size_t fused_smem_bytes(const FusedArgs &a, int tt, int rowsplit);
cudaError_t fused_set_attributes();
int fused_grid(int tt, size_t smem, int num_sms);
cudaError_t launch_fused(const FusedArgs &a, int tt, int grid, size_t smem, cudaStream_t s);

}  // namespace moe
