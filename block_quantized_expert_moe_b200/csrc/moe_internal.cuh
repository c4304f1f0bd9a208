// Internal definitions shared by the CUDA translation units of libmoe: the
// device layout of a pack, the forward workspace and the kernel argument
// blocks.  Nothing here is part of the public C ABI (include/moe.h).
#pragma once

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
//   NVFP4   qs: rows x K/2 (8 B per 16-block), sc: rows x K/16 E4M3 scales,
//           ts: one fp32 matrix scale per expert
// Expert e's plane starts at base + e * stride.
struct DevProj {
    int fmt = 0, rows = 0, cols = 0;
    const uint8_t *qs = nullptr;
    const uint8_t *sc = nullptr;
    const uint8_t *qh = nullptr;
    const float *ts = nullptr;
    int64_t qs_stride = 0, sc_stride = 0, qh_stride = 0;  // bytes per expert
    int qs_row = 0, sc_row = 0, qh_row = 0;               // bytes per row
};

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
    int32_t *ticket = nullptr;   // last-CTA counter of the route kernel
    int32_t *err = nullptr;      // sticky device error (moe_status)
    float *h = nullptr;          // [slots x I]
    float *y = nullptr;          // [slots x H]
    int max_groups = 0;
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
    uint32_t tab[4];          // 16-entry code table, bytes biased by +128
    float ts_mul;             // NVFP4: folded into the block scale decode
};

struct CombineArgs {
    const float *y;
    const int32_t *slot_pos;
    const float *gate;
    int T, k, H, has_shared;
    float *out;
};

// launchers (return cudaGetLastError of the launch)
size_t route_smem_bytes(int H, int rt, int E);
void init_device_attributes();  // once per device, with that device current
int route_tokens_per_pass(int H);
cudaError_t launch_route(const RouteArgs &a, int grid, cudaStream_t s);
int route_grid(int E, int num_sms);

cudaError_t launch_matvec(const MatvecArgs &a, bool gateup, int tt, int grid, cudaStream_t s);
size_t matvec_smem_bytes(const MatvecArgs &a, bool gateup, int tt);
int matvec_grid(const MatvecArgs &a, bool gateup, int tt, int num_sms);

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s);

}  // namespace moe
