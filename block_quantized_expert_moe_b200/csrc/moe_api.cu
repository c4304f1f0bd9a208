// Host side of the C ABI in include/moe.h: argument checks, the expert pack
// (repack of canonical blocks into the device planes + upload), workspace
// management and the enqueueing of each forward's kernels.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#include "moe_internal.cuh"

namespace moe {
cudaError_t route_set_attributes();
cudaError_t matvec_set_attributes();
cudaError_t debug_act_quant(const void *x, bool bf16, int rows, int cols, uint8_t *codes, uint8_t *sf_atoms,
                            float *row_scale, int32_t *scratch, cudaStream_t s);
cudaError_t debug_dequant(const DevProj &w, const CodeTable &tab, int slot, int row0, int nrows, int kind, void *out,
                          cudaStream_t s);
}  // namespace moe

// kernel-stage slots of the profiling API (moe_profile_end's ms[])
enum { PROF_ROUTE = 0, PROF_GATE_UP = 1, PROF_DOWN = 2, PROF_COMBINE = 3, PROF_FUSED = 4, PROF_PREFILL = 5,
       PROF_STAGES = 6, PROF_PHASES = 9, PROF_GRID = 9, PROF_SUB = 8,
       PROF_OUT = PROF_STAGES + PROF_PHASES + PROF_GRID + PROF_SUB };
constexpr int kStampStride = 32;  // device stamps per recorded forward (see FusedArgs::stamps)

using namespace moe;

struct moe_pack {
    int device = 0;
    int num_sms = 0;
    int E = 0, H = 0, I = 0, has_shared = 0, max_tokens = 0, max_top_k = 0, flags = 0;
    int eb = 0, ee = 0;  // routed experts [eb, ee) are in this pack (expert parallelism)
    int n_local = 0;     // ee - eb; pack slot of expert e is e - eb, the shared expert's n_local
    int fmt_gu = 0, fmt_dn = 0;        // device formats (a Q5_0 projection runs as Q5_1)
    int fmt_gu_in = 0, fmt_dn_in = 0;  // the formats the caller packed
    DevProj gu, dn;
    CodeTable ct_gu{}, ct_dn{};
    uint8_t perm_gu[16], perm_dn[16];  // stored position of each 4-bit code
    std::vector<void *> allocations;
    Workspace ws;
    int64_t arena_bytes = 0, workspace_bytes = 0;
    int grid_cache[2][2];  // [gateup][tt==8]
    // kernel-stage timing (moe_profile_begin/end): per recorded forward, the
    // first event index and its kind (0 grouped: 5 events around route, gate/up,
    // down and combine; 1 single-kernel decode: 2 events; 2 prefill: 2 events)
    bool prof_on = false;
    std::vector<cudaEvent_t> prof_ev;
    std::vector<std::pair<int, int>> prof_fwd;
    int prof_used = 0;
    long long *prof_stamps = nullptr;  // device, kStampStride stamps per recorded forward
    int prof_nstamp = 0, prof_stamp_cap = 0;
    int fused_grid[2] = {0, 0};   // [tt==8]
    int stream1 = -1;             // single-token streaming kernel usable (-1: not yet checked)
    size_t stream1_smem = 0;
    int pdl = 1;                  // launch it as a programmatic dependent of the previous kernel
    int sgm = -1;                 // streamed grouped matvecs usable (-1: not yet checked)
    SgmProj sg_gu{}, sg_dn{};
    int dtc = -1;                 // tensor-core grouped decode usable (-1: not yet checked)
    DecodeTcMaps dtc_maps{};
    int tail_ok[kDecodeTcMaxN + 1][2];  // one-launch tail usable for T tokens, x dtype (-1: not yet checked)
    TailLaunch tail_launch[kDecodeTcMaxN + 1][2];
    bool has_prefill = false;     // tensor-core prefill workspace present
    PrefillWorkspace pws;
};

namespace {

// Code table of a 4-bit format for the decode kernels' byte-permute lookup.
// Entry bytes are value + bias; when every position pair (i, i+8) can be given
// entries whose biased bytes share their top bit, the table is laid out for the
// XOR-combined lookup (two permutes and one XOR per four nibbles) and perm[c]
// is the position code c is stored as; otherwise the masked lookup with the
// identity position.  NVFP4 entries are 2*e2m1(c) (integers -12..12), so its
// block scales carry the factor 1/2.
CodeTable build_code_table(int fmt, const int8_t *iq4, uint8_t perm[16])
{
    CodeTable ct{};
    for (int c = 0; c < 16; ++c) perm[c] = (uint8_t)c;
    if (fmt != MOE_FMT_IQ4_NL && fmt != MOE_FMT_NVFP4) return ct;
    int v[16];
    if (fmt == MOE_FMT_NVFP4) {
        const int mag[8] = {0, 1, 2, 3, 4, 6, 8, 12};
        for (int c = 0; c < 16; ++c) v[c] = (c & 8) ? -mag[c & 7] : mag[c & 7];
    } else {
        for (int c = 0; c < 16; ++c) v[c] = iq4[c];
    }
    int lo = 127, hi = -128;
    for (int c = 0; c < 16; ++c) {
        lo = std::min(lo, v[c]);
        hi = std::max(hi, v[c]);
    }
    // candidate biases keeping every byte in [0, 255]; prefer one with an even
    // split of top bits (all-equal counts as even)
    int bias = -1;
    for (int b : {192, 128, 127, 129, 126, 130}) {
        if (lo + b < 0 || hi + b > 255) continue;
        int n1 = 0;
        for (int c = 0; c < 16; ++c) n1 += (v[c] + b) >= 128;
        if (n1 % 2 == 0) {
            bias = b;
            break;
        }
    }
    uint8_t pos_code[16];
    if (bias >= 0) {
        int ones[16], zeros[16], n1 = 0, n0 = 0;
        for (int c = 0; c < 16; ++c) {
            if (v[c] + bias >= 128) ones[n1++] = c;
            else zeros[n0++] = c;
        }
        int p = 0;
        for (int i = 0; i + 1 < n1; i += 2, ++p) {
            pos_code[p] = (uint8_t)ones[i];
            pos_code[p + 8] = (uint8_t)ones[i + 1];
        }
        for (int i = 0; i + 1 < n0; i += 2, ++p) {
            pos_code[p] = (uint8_t)zeros[i];
            pos_code[p + 8] = (uint8_t)zeros[i + 1];
        }
        if (fmt == MOE_FMT_NVFP4)  // native codes stay in place (the prefill MMA reads them); bias 192
            for (int q = 0; q < 16; ++q) pos_code[q] = (uint8_t)q;  // makes every top bit equal
        for (int q = 0; q < 16; ++q) perm[pos_code[q]] = (uint8_t)q;
        uint8_t bytes[16];
        for (int i = 0; i < 8; ++i) {
            const uint8_t l = (uint8_t)(v[pos_code[i]] + bias);
            const uint8_t h = (uint8_t)(v[pos_code[i + 8]] + bias);
            bytes[i] = l;
            bytes[i + 8] = (uint8_t)(h ^ ((l & 0x80) ? 0xFF : 0x00));
        }
        for (int i = 0; i < 16; ++i) ct.t[i / 4] |= (uint32_t)bytes[i] << (8 * (i % 4));
        ct.xor_mode = 1;
    } else {
        bias = 128;
        for (int c = 0; c < 16; ++c) ct.t[c / 4] |= (uint32_t)(uint8_t)(v[c] + bias) << (8 * (c % 4));
        ct.xor_mode = 0;
    }
    ct.magic = 8388608.f + (float)bias;
    return ct;
}

std::mutex g_dev_mutex;
bool g_dev_ready[64];

moe_status init_device(int dev)
{
    std::lock_guard<std::mutex> lk(g_dev_mutex);
    if (dev < 0 || dev >= 64) return MOE_ERR_INVALID_ARG;
    if (g_dev_ready[dev]) return MOE_OK;
    if (route_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (matvec_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (fused_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (stream1_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (sgm_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (decode_tc_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (prefill_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (prefill_nvfp4_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (prefill_q8_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    if (tail_set_attributes() != cudaSuccess) return MOE_ERR_CUDA;
    g_dev_ready[dev] = true;
    return MOE_OK;
}

struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev)
    {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard()
    {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_fmt(int f) { return f >= MOE_FMT_Q8_0 && f <= MOE_FMT_Q5_0; }

// The device format of a projection: Q5_0 runs as Q5_1 with m = -16 d.
int device_fmt(int f) { return f == MOE_FMT_Q5_0 ? MOE_FMT_Q5_1 : f; }

int64_t canon_row_bytes(int fmt, int64_t cols)
{
    switch (fmt) {
    case MOE_FMT_Q8_0: return cols / 32 * 34;
    case MOE_FMT_Q5_1: return cols / 32 * 24;
    case MOE_FMT_Q5_0: return cols / 32 * 22;
    case MOE_FMT_IQ4_NL: return cols / 32 * 18;
    case MOE_FMT_NVFP4: return cols / 16 * 9;
    default: return -1;
    }
}

// Device plane sizes of one row of `cols` weights.
void plane_rows(int fmt, int cols, int &qs_row, int &sc_row, int &qh_row)
{
    qh_row = 0;
    switch (fmt) {
    case MOE_FMT_Q8_0: qs_row = cols; sc_row = cols / 32 * 2; break;
    case MOE_FMT_Q5_1:
    case MOE_FMT_Q5_0: qs_row = cols / 2; sc_row = cols / 32 * 4; qh_row = cols / 32 * 4; break;
    case MOE_FMT_IQ4_NL: qs_row = cols / 2; sc_row = cols / 32 * 2; break;
    default: qs_row = cols / 2; sc_row = 0; break;  // NVFP4: scales in the block-scale layout
    }
}

int nvfp4_ksteps(int cols) { return (cols + 63) / 64; }

// bytes of one expert's NVFP4 scale plane: 128-row blocks x K steps x 512
int64_t nvfp4_sf_bytes(int rows, int cols) { return (int64_t)((rows + 127) / 128) * nvfp4_ksteps(cols) * 512; }

int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// Repack one expert's projection (rows x cols canonical blocks) into planes.
// Returns false on an invalid NVFP4 block scale.
float half_to_float(uint16_t h)
{
    const int e = (h >> 10) & 31, m = h & 1023;
    const float mag = e == 0 ? std::ldexp((float)m, -24) : e == 31 ? INFINITY : std::ldexp((float)(1024 + m), e - 25);
    return (h & 0x8000) ? -mag : mag;
}

// fp16 bits of f, which must be exactly representable (a power-of-two multiple
// of an fp16 number within range).
uint16_t half_from_exact(float f)
{
    const uint16_t sign = std::signbit(f) ? 0x8000u : 0u;
    const float a = std::fabs(f);
    if (a == 0.f) return sign;
    int e;
    const float m = std::frexp(a, &e);  // a = m 2^e, m in [0.5, 1)
    const int E = e - 1 + 15;
    if (E >= 1) return (uint16_t)(sign | (E << 10) | (uint32_t)std::ldexp(2.f * m - 1.f, 10));
    return (uint16_t)(sign | (uint32_t)std::ldexp(a, 24));  // subnormal: a = mant 2^-24
}

bool repack_expert(int fmt, const uint8_t *src, int rows, int cols, uint8_t *qs, uint8_t *sc,
                   uint8_t *qh, uint8_t *sr, const uint8_t *perm)
{
    uint8_t pbyte[256];  // both nibbles of a code byte through the position map
    for (int b = 0; b < 256; ++b) pbyte[b] = (uint8_t)(perm[b & 15] | (perm[b >> 4] << 4));
    const int64_t rb = canon_row_bytes(fmt, cols);
    int qs_row, sc_row, qh_row;
    plane_rows(fmt, cols, qs_row, sc_row, qh_row);
    for (int r = 0; r < rows; ++r) {
        const uint8_t *row = src + (int64_t)r * rb;
        uint8_t *q = qs + (int64_t)r * qs_row;
        uint8_t *s = sc + (int64_t)r * sc_row;
        if (fmt == MOE_FMT_Q8_0) {
            for (int b = 0; b < cols / 32; ++b) {
                const uint8_t *blk = row + b * 34;
                s[2 * b] = blk[0];
                s[2 * b + 1] = blk[1];
                for (int j = 0; j < 32; ++j) q[b * 32 + j] = blk[2 + j] ^ 0x80u;  // bias by +128
            }
        } else if (fmt == MOE_FMT_Q5_1) {
            uint8_t *h = qh + (int64_t)r * qh_row;
            for (int b = 0; b < cols / 32; ++b) {
                const uint8_t *blk = row + b * 24;
                std::memcpy(s + 4 * b, blk, 4);      // d, m
                std::memcpy(h + 4 * b, blk + 4, 4);  // qh
                std::memcpy(q + 16 * b, blk + 8, 16);
            }
        } else if (fmt == MOE_FMT_Q5_0) {  // as Q5_1 planes with m = -16 d (exact)
            uint8_t *h = qh + (int64_t)r * qh_row;
            for (int b = 0; b < cols / 32; ++b) {
                const uint8_t *blk = row + b * 22;
                const float d = half_to_float((uint16_t)(blk[0] | blk[1] << 8));
                if (!(std::fabs(d) * 16.f <= 65504.f)) return false;
                const uint16_t m = half_from_exact(-16.f * d);
                s[4 * b] = blk[0];
                s[4 * b + 1] = blk[1];
                s[4 * b + 2] = (uint8_t)m;
                s[4 * b + 3] = (uint8_t)(m >> 8);
                std::memcpy(h + 4 * b, blk + 2, 4);  // qh
                std::memcpy(q + 16 * b, blk + 6, 16);
            }
        } else if (fmt == MOE_FMT_IQ4_NL) {
            for (int b = 0; b < cols / 32; ++b) {
                const uint8_t *blk = row + b * 18;
                s[2 * b] = blk[0];
                s[2 * b + 1] = blk[1];
                for (int i = 0; i < 16; ++i) q[16 * b + i] = pbyte[blk[2 + i]];
            }
        } else {
            const int ks = nvfp4_ksteps(cols);
            for (int b = 0; b < cols / 16; ++b) {
                const uint8_t *blk = row + b * 9;
                if (blk[0] >= 0x7Fu) return false;  // negative scale or NaN
                sc[sf_offset(r, b >> 2, b & 3, ks)] = blk[0];
                sr[(int64_t)r * (cols / 16) + b] = blk[0];
                std::memcpy(q + 8 * b, blk + 1, 8);
            }
        }
    }
    return true;
}

template <class F>
void parallel_for(int n, F f)
{
    unsigned hw = std::thread::hardware_concurrency();
    int nt = (int)std::min<unsigned>(hw ? hw : 1, 64u);
    nt = std::min(nt, n);
    if (nt <= 1) {
        for (int i = 0; i < n; ++i) f(i);
        return;
    }
    std::vector<std::thread> th;
    for (int t = 0; t < nt; ++t)
        th.emplace_back([&, t] {
            for (int i = t; i < n; i += nt) f(i);
        });
    for (auto &x : th) x.join();
}

void free_pack_memory(moe_pack *p)
{
    for (void *a : p->allocations) cudaFree(a);
    p->allocations.clear();
}

// Allocation-failure injection (moe_debug_fail_alloc_after): device
// allocations left before one fails; -1 = off.  The failing call turns it off.
std::atomic<int> g_fail_alloc_after{-1};

moe_status dev_alloc(moe_pack *p, size_t bytes, void **out)
{
    int left = g_fail_alloc_after.load();
    while (left >= 0 && !g_fail_alloc_after.compare_exchange_weak(left, left - 1)) {
    }
    if (left == 0) return MOE_ERR_OOM;  // the injected failure
    void *ptr = nullptr;
    if (cudaMalloc(&ptr, bytes ? bytes : 16) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_OOM;
    }
    p->allocations.push_back(ptr);
    *out = ptr;
    return MOE_OK;
}

// Whether every weight d q (Q8_0, IQ4_NL: |q| <= 128) or d q + m (Q5_1,
// q <= 31) of the scale plane `sc` is an fp16 normal number or zero: the
// tensor-core decode path expands the blocks to fp16.  NVFP4 always is (a code
// of at most 12 halves times an E4M3 scale: at most 5376, at least 2^-10).
bool f16_safe(int fmt, const std::vector<uint8_t> &sc, int64_t stride, int64_t used, int n_slots)
{
    if (fmt == MOE_FMT_NVFP4) return true;
    for (int s = 0; s < n_slots; ++s) {
        const uint8_t *p = sc.data() + (int64_t)s * stride;
        if (fmt == MOE_FMT_Q5_1) {
            for (int64_t i = 0; i + 4 <= used; i += 4) {
                const float d = half_to_float((uint16_t)(p[i] | p[i + 1] << 8));
                const float m = half_to_float((uint16_t)(p[i + 2] | p[i + 3] << 8));
                if (!(std::fabs(d) * 31.f + std::fabs(m) <= 60000.f)) return false;
            }
        } else {
            for (int64_t i = 0; i + 2 <= used; i += 2) {
                const float d = std::fabs(half_to_float((uint16_t)(p[i] | p[i + 1] << 8)));
                if (!(d == 0.f || (d >= 0x1p-14f && d * 128.f <= 60000.f))) return false;
            }
        }
    }
    return true;
}

// Build one projection's planes for all slots (routed experts + shared).
moe_status build_proj(moe_pack *p, DevProj &dp, int fmt, int rows, int cols, const uint8_t *blocks,
                      const uint8_t *shared_blocks, const float *ts, int n_slots, const uint8_t *perm)
{
    dp.fmt = device_fmt(fmt);  // fmt: the canonical blocks' format
    dp.rows = rows;
    dp.cols = cols;
    plane_rows(fmt, cols, dp.qs_row, dp.sc_row, dp.qh_row);
    dp.qs_stride = round_up((int64_t)rows * dp.qs_row, 256);
    dp.sc_stride = round_up(fmt == MOE_FMT_NVFP4 ? nvfp4_sf_bytes(rows, cols) : (int64_t)rows * dp.sc_row, 256);
    dp.ksteps = fmt == MOE_FMT_NVFP4 ? nvfp4_ksteps(cols) : 0;
    dp.qh_stride = round_up((int64_t)rows * dp.qh_row, 256);
    const bool nv = fmt == MOE_FMT_NVFP4;
    dp.sr_row = nv ? cols / 16 : dp.sc_row;
    dp.sr_stride = nv ? round_up((int64_t)rows * dp.sr_row, 256) : dp.sc_stride;
    const int64_t canon = canon_row_bytes(fmt, cols) * rows;
    std::vector<uint8_t> hq, hs, hh, hr;
    try {
        hq.assign((size_t)dp.qs_stride * n_slots, 0);
        hs.assign((size_t)dp.sc_stride * n_slots, 0);
        if (dp.qh_row) hh.assign((size_t)dp.qh_stride * n_slots, 0);
        if (nv) hr.assign((size_t)dp.sr_stride * n_slots, 0);
    } catch (const std::bad_alloc &) {
        return MOE_ERR_OOM;
    }
    std::vector<char> ok((size_t)n_slots, 1);
    parallel_for(n_slots, [&](int s) {
        const uint8_t *src = s < p->n_local ? blocks + (int64_t)s * canon : shared_blocks;
        ok[s] = repack_expert(fmt, src, rows, cols, hq.data() + (int64_t)s * dp.qs_stride,
                              hs.data() + (int64_t)s * dp.sc_stride,
                              dp.qh_row ? hh.data() + (int64_t)s * dp.qh_stride : nullptr,
                              nv ? hr.data() + (int64_t)s * dp.sr_stride : nullptr, perm);
    });
    for (char c : ok)
        if (!c) return MOE_ERR_INVALID_ARG;
    dp.f16_ok = f16_safe(dp.fmt, hs, dp.sc_stride, (int64_t)rows * dp.sc_row, n_slots);
    void *dq, *ds, *dh = nullptr, *dt = nullptr;
    moe_status st;
    if ((st = dev_alloc(p, hq.size(), &dq)) != MOE_OK) return st;
    if ((st = dev_alloc(p, hs.size(), &ds)) != MOE_OK) return st;
    if (cudaMemcpy(dq, hq.data(), hq.size(), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(ds, hs.data(), hs.size(), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    if (dp.qh_row) {
        if ((st = dev_alloc(p, hh.size(), &dh)) != MOE_OK) return st;
        if (cudaMemcpy(dh, hh.data(), hh.size(), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (fmt == MOE_FMT_NVFP4) {
        for (int s = 0; s < n_slots; ++s)
            if (!(ts[s] >= 0.f) || ts[s] > 3.0e38f) return MOE_ERR_INVALID_ARG;
        if ((st = dev_alloc(p, sizeof(float) * n_slots, &dt)) != MOE_OK) return st;
        if (cudaMemcpy(dt, ts, sizeof(float) * n_slots, cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    }
    void *dr = ds;
    if (nv) {
        if ((st = dev_alloc(p, hr.size(), &dr)) != MOE_OK) return st;
        if (cudaMemcpy(dr, hr.data(), hr.size(), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    }
    // tiled copy for the one-launch tail (shapes of whole 128-row blocks and
    // 256-wide K chunks whose weights the tensor-core decode takes)
    if (dp.f16_ok && rows % 128 == 0 && cols % 256 == 0 && p->max_tokens <= kDecodeMaxTokens) {
        const int dfmt = dp.fmt, KC = cols / 256, RB = rows / 128;
        const int cb = tl_codes_bytes(dfmt), sb = tl_scales_bytes(dfmt);
        dp.tl_block = tl_block_bytes(dfmt);
        dp.tl_stride = round_up((int64_t)RB * KC * dp.tl_block, 256);
        std::vector<uint8_t> ht;
        try {
            ht.assign((size_t)dp.tl_stride * n_slots, 0);
        } catch (const std::bad_alloc &) {
            return MOE_ERR_OOM;
        }
        const uint8_t *srm = nv ? hr.data() : hs.data();  // scales row by row
        const int64_t srm_stride = nv ? dp.sr_stride : dp.sc_stride;
        const int srm_row = nv ? dp.sr_row : dp.sc_row;
        parallel_for(n_slots, [&](int sl) {
            const uint8_t *q = hq.data() + (int64_t)sl * dp.qs_stride, *sr = srm + (int64_t)sl * srm_stride;
            const uint8_t *h = dp.qh_row ? hh.data() + (int64_t)sl * dp.qh_stride : nullptr;
            for (int rb = 0; rb < RB; ++rb)
                for (int kc = 0; kc < KC; ++kc) {
                    uint8_t *blk = ht.data() + (int64_t)sl * dp.tl_stride + ((int64_t)rb * KC + kc) * dp.tl_block;
                    for (int r = 0; r < 128; ++r) {
                        const int64_t R = (int64_t)rb * 128 + r;
                        // codes: 16-byte chunk c of a 128-byte row segment at chunk c ^ (r % 8)
                        const int nbx = dfmt == MOE_FMT_Q8_0 ? 2 : 1;
                        for (int bx = 0; bx < nbx; ++bx)
                            for (int c = 0; c < 8; ++c)
                                std::memcpy(blk + bx * 16384 + r * 128 + ((c ^ (r & 7)) << 4),
                                            q + R * dp.qs_row + (int64_t)kc * 128 * nbx + bx * 128 + c * 16, 16);
                        if (dfmt == MOE_FMT_Q5_1) {
                            // {d, m} and fifth bits: 32 bytes a row, chunk c at c ^ ((r / 4) % 2)
                            for (int c = 0; c < 2; ++c) {
                                const int o = r * 32 + ((c ^ ((r >> 2) & 1)) << 4);
                                std::memcpy(blk + cb + o, sr + R * srm_row + kc * 32 + c * 16, 16);
                                std::memcpy(blk + cb + sb + o, h + R * dp.qh_row + kc * 32 + c * 16, 16);
                            }
                        } else {
                            std::memcpy(blk + cb + r * 16, sr + R * srm_row + kc * 16, 16);
                        }
                    }
                }
        });
        void *dt2;
        if ((st = dev_alloc(p, ht.size(), &dt2)) != MOE_OK) return st;
        if (cudaMemcpy(dt2, ht.data(), ht.size(), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
        dp.tl = static_cast<const uint8_t *>(dt2);
        p->arena_bytes += (int64_t)ht.size();
    }
    dp.qs = static_cast<const uint8_t *>(dq);
    dp.sc = static_cast<const uint8_t *>(ds);
    dp.qh = static_cast<const uint8_t *>(dh);
    dp.ts = static_cast<const float *>(dt);
    dp.sr = static_cast<const uint8_t *>(dr);
    p->arena_bytes += (int64_t)(hq.size() + hs.size() + hh.size() + hr.size()) + (dt ? 4 * n_slots : 0);
    return MOE_OK;
}

moe_status build_workspace(moe_pack *p)
{
    const int64_t T = p->max_tokens, k = p->max_top_k, E = p->E;
    int64_t slots = T * (k + 1);
    if ((p->flags & MOE_PACK_DENSE) && T <= kDecodeMaxTokens) slots = std::max(slots, (E + 1) * T);
    Workspace &w = p->ws;
    w.max_groups = (int)(slots + E + 2);
    struct Item { void **dst; int64_t bytes; };
    Item items[] = {
        {(void **)&w.logits, T * E * 4}, {(void **)&w.idx, T * k * 4}, {(void **)&w.gate, T * k * 4},
        {(void **)&w.cnt, (E + 1) * 4}, {(void **)&w.off, (E + 1) * 4}, {(void **)&w.perm_tok, slots * 4},
        {(void **)&w.slot_pos, T * k * 4}, {(void **)&w.groups, (int64_t)w.max_groups * 16},
        {(void **)&w.n_groups, 4}, {(void **)&w.ticket, 64}, {(void **)&w.err, 4}, {(void **)&w.bar, 8},
        {(void **)&w.h, slots * p->I * 4}, {(void **)&w.y, slots * p->H * 4},
        {(void **)&w.dgate, slots * 4}, {(void **)&w.n_dense_rows, 4}, {(void **)&w.slot_scale, slots * 4},
        {(void **)&w.xg, slots * p->H * 2},
        {(void **)&w.xcnt, 16},
        {(void **)&w.tail_ctr, T <= kDecodeMaxTokens ? (int64_t)tail_counter_words(p->E, p->H, p->I) * 4 : 0},
        {(void **)&w.tail_part,
         T <= kDecodeMaxTokens ? (int64_t)tail_part_floats(p->num_sms, (int)T) * 4 : 0},
    };
    int64_t total = 0;
    for (auto &it : items) total += round_up(it.bytes, 256);
    void *base;
    moe_status st = dev_alloc(p, (size_t)total, &base);
    if (st != MOE_OK) return st;
    if (cudaMemset(base, 0, (size_t)total) != cudaSuccess) return MOE_ERR_CUDA;
    int64_t o = 0;
    for (auto &it : items) {
        *it.dst = static_cast<char *>(base) + o;
        o += round_up(it.bytes, 256);
    }
    p->workspace_bytes = total;
    return MOE_OK;
}

// Buffers of the tensor-core prefill (packs for more than 64 tokens whose formats it takes).
moe_status build_prefill_workspace(moe_pack *p)
{
    const int64_t T = p->max_tokens, k = p->max_top_k, E = p->E, H = p->H, I = p->I;
    const int64_t rows = round_up(T * k + T + (E + 1) * 127, 128);
    PrefillWorkspace &w = p->pws;
    w.logits = p->ws.logits;
    w.idx = p->ws.idx;
    w.gate = p->ws.gate;
    w.slot_pos = p->ws.slot_pos;
    w.cnt = p->ws.cnt;
    w.max_rows = (int)rows;
    struct Item { void **dst; int64_t bytes; };
    Item items[] = {
        {(void **)&w.pad_off, (E + 2) * 4}, {(void **)&w.fill, (E + 2) * 4}, {(void **)&w.tiles, rows / 128 * 8 + 64},
        {(void **)&w.ptiles, rows / 128 * 16 + 64}, {(void **)&w.n_ptiles, 4},
        {(void **)&w.n_tiles, 4}, {(void **)&w.total_rows, 4}, {(void **)&w.perm_tok, rows * 4},
        {(void **)&w.row_gate, rows * 4}, {(void **)&w.row_scale_x, rows * 4}, {(void **)&w.row_scale_h, rows * 4},
        {(void **)&w.a_q, rows * H * 2},  // bf16 slot rows (the NVFP4 path's codes fit in them)
        {(void **)&w.sfa, rows / 128 * (H / 64) * 512},
        {(void **)&w.h, rows * I * 4}, {(void **)&w.h_q, rows * I / 2}, {(void **)&w.sfh, rows / 128 * (I / 64) * 512},
    };
    int64_t total = 0;
    for (auto &it : items) total += round_up(it.bytes, 256);
    void *base;
    moe_status st = dev_alloc(p, (size_t)total, &base);
    if (st != MOE_OK) return st;
    if (cudaMemset(base, 0, (size_t)total) != cudaSuccess) return MOE_ERR_CUDA;
    int64_t o = 0;
    for (auto &it : items) {
        *it.dst = static_cast<char *>(base) + o;
        o += round_up(it.bytes, 256);
    }
    p->workspace_bytes += total;
    p->has_prefill = true;
    return MOE_OK;
}

moe_status check_launch(cudaError_t e)
{
    if (e == cudaSuccess) return MOE_OK;
    return MOE_ERR_CUDA;
}

// Record profiling event i of the current forward (no-op when profiling is off
// or the event budget is used up).
void prof_mark(moe_pack *p, int base, int i, cudaStream_t s)
{
    if (base < 0) return;
    cudaEvent_t ev = p->prof_ev[(size_t)base + i];
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cs);
    if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    else cudaEventRecord(ev, s);
}

}  // namespace

extern "C" {

const char *moe_status_string(moe_status s)
{
    switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_FMT_MISMATCH: return "format does not match the pack";
    case MOE_ERR_OOM: return "out of memory";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE: return "device-side plan error";
    case MOE_ERR_RANGE: return "value outside the fp16 range of the tensor-core decode path";
    default: return "unknown status";
    }
}

moe_status moe_pack_experts(const moe_pack_desc *d, int device, moe_pack **out)
{
    if (!d || !out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (d->n_experts < 1 || d->n_experts > 1024) return MOE_ERR_INVALID_ARG;
    if (d->hidden < 32 || d->hidden > 16384 || d->hidden % 32) return MOE_ERR_INVALID_ARG;
    if (d->inter < 32 || d->inter > 16384 || d->inter % 32) return MOE_ERR_INVALID_ARG;
    if (d->max_tokens < 1 || d->max_tokens > 65536) return MOE_ERR_INVALID_ARG;
    if (d->max_top_k < 1 || d->max_top_k > d->n_experts) return MOE_ERR_INVALID_ARG;
    if (!valid_fmt(d->fmt_gate_up) || !valid_fmt(d->fmt_down)) return MOE_ERR_INVALID_ARG;
    if (!d->gate_up_blocks || !d->down_blocks) return MOE_ERR_INVALID_ARG;
    if ((d->fmt_gate_up == MOE_FMT_IQ4_NL || d->fmt_down == MOE_FMT_IQ4_NL) && !d->iq4nl_table)
        return MOE_ERR_INVALID_ARG;
    if (d->fmt_gate_up == MOE_FMT_NVFP4 && !d->gate_up_tensor_scale) return MOE_ERR_INVALID_ARG;
    if (d->fmt_down == MOE_FMT_NVFP4 && !d->down_tensor_scale) return MOE_ERR_INVALID_ARG;
    if (d->has_shared && (!d->shared_gate_up_blocks || !d->shared_down_blocks)) return MOE_ERR_INVALID_ARG;
    const bool whole = (d->expert_begin == 0 && d->expert_end == 0);
    if (!whole && (d->expert_begin < 0 || d->expert_end <= d->expert_begin || d->expert_end > d->n_experts))
        return MOE_ERR_INVALID_ARG;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (device < 0 || device >= ndev) return MOE_ERR_INVALID_ARG;
    DeviceGuard g(device);
    if (!g.ok) return MOE_ERR_CUDA;
    moe_status st = init_device(device);
    if (st != MOE_OK) return st;
    moe_pack *p = new (std::nothrow) moe_pack();
    if (!p) return MOE_ERR_OOM;
    p->device = device;
    cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, device);
    p->E = d->n_experts;
    p->eb = whole ? 0 : d->expert_begin;
    p->ee = whole ? d->n_experts : d->expert_end;
    p->n_local = p->ee - p->eb;
    p->H = d->hidden;
    p->I = d->inter;
    p->has_shared = d->has_shared ? 1 : 0;
    p->max_tokens = d->max_tokens;
    p->max_top_k = d->max_top_k;
    p->flags = d->flags;
    p->fmt_gu_in = d->fmt_gate_up;
    p->fmt_dn_in = d->fmt_down;
    p->fmt_gu = device_fmt(d->fmt_gate_up);
    p->fmt_dn = device_fmt(d->fmt_down);
    p->ct_gu = build_code_table(p->fmt_gu, d->iq4nl_table, p->perm_gu);
    p->ct_dn = build_code_table(p->fmt_dn, d->iq4nl_table, p->perm_dn);
    for (auto &row : p->grid_cache) row[0] = row[1] = 0;
    for (auto &row : p->tail_ok) row[0] = row[1] = -1;
    const int n_slots = p->n_local + p->has_shared;
    std::vector<float> gts, dts;
    if (p->fmt_gu == MOE_FMT_NVFP4) gts.assign(d->gate_up_tensor_scale, d->gate_up_tensor_scale + n_slots);
    if (p->fmt_dn == MOE_FMT_NVFP4) dts.assign(d->down_tensor_scale, d->down_tensor_scale + n_slots);
    st = build_proj(p, p->gu, p->fmt_gu_in, 2 * p->I, p->H, static_cast<const uint8_t *>(d->gate_up_blocks),
                    static_cast<const uint8_t *>(d->shared_gate_up_blocks), gts.data(), n_slots, p->perm_gu);
    if (st == MOE_OK)
        st = build_proj(p, p->dn, p->fmt_dn_in, p->H, p->I, static_cast<const uint8_t *>(d->down_blocks),
                        static_cast<const uint8_t *>(d->shared_down_blocks), dts.data(), n_slots, p->perm_dn);
    if (st == MOE_OK) st = build_workspace(p);
    const bool nv = p->fmt_gu == MOE_FMT_NVFP4 && p->fmt_dn == MOE_FMT_NVFP4 &&
                    prefill_nvfp4_supported(p->H, p->I, p->E, p->max_top_k);
    // bf16-dequantising tensor-core prefill: Q8_0, IQ4_NL and Q5_1, in any mix
    const bool q8 = prefill_q8_supported(p->fmt_gu, p->fmt_dn, p->H, p->I, p->E, p->max_top_k, true);
    if (st == MOE_OK && p->max_tokens > kDecodeMaxTokens && (nv || q8)) st = build_prefill_workspace(p);
    if (st == MOE_OK && cudaDeviceSynchronize() != cudaSuccess) st = MOE_ERR_CUDA;
    if (st != MOE_OK) {
        free_pack_memory(p);
        delete p;
        return st;
    }
    *out = p;
    return MOE_OK;
}

moe_status moe_debug_fail_alloc_after(int n)
{
    if (n < -1) return MOE_ERR_INVALID_ARG;
    g_fail_alloc_after.store(n);
    return MOE_OK;
}

moe_status moe_pack_free(moe_pack *p)
{
    if (!p) return MOE_OK;
    DeviceGuard g(p->device);
    cudaDeviceSynchronize();
    free_pack_memory(p);
    delete p;
    return MOE_OK;
}

moe_status moe_pack_query(const moe_pack *p, moe_pack_info *info)
{
    if (!p || !info) return MOE_ERR_INVALID_ARG;
    // HBM bytes one expert's blocks occupy (the NVFP4 scale bytes as stored: K/16 per row)
    auto proj_bytes = [](const DevProj &d) {
        const int64_t sc = d.fmt == MOE_FMT_NVFP4 ? (int64_t)d.cols / 16 : d.sc_row;
        return (int64_t)d.rows * (d.qs_row + sc + d.qh_row);
    };
    info->gate_up_bytes_per_expert = proj_bytes(p->gu);
    info->down_bytes_per_expert = proj_bytes(p->dn);
    info->expert_bytes = info->gate_up_bytes_per_expert + info->down_bytes_per_expert +
                         (p->fmt_gu == MOE_FMT_NVFP4 ? 4 : 0) + (p->fmt_dn == MOE_FMT_NVFP4 ? 4 : 0);
    info->arena_bytes = p->arena_bytes;
    info->workspace_bytes = p->workspace_bytes;
    info->device = p->device;
    const auto masked = [](int fmt, const CodeTable &t) {
        return (fmt == MOE_FMT_IQ4_NL || fmt == MOE_FMT_NVFP4) && !t.xor_mode;
    };
    info->code_table_masked = (masked(p->fmt_gu, p->ct_gu) ? 1 : 0) | (masked(p->fmt_dn, p->ct_dn) ? 2 : 0);
    return MOE_OK;
}

size_t moe_route_workspace_bytes(int n_tokens, int n_experts)
{
    if (n_tokens < 1 || n_experts < 1) return 0;
    return 256 + (size_t)n_tokens * n_experts * sizeof(float);
}

moe_status moe_route_topk(const void *x, moe_dtype x_dtype, const uint16_t *router_w, int n_tokens,
                          int hidden, int n_experts, int top_k, int32_t *idx_out, float *gate_out,
                          void *workspace, size_t workspace_bytes, void *stream)
{
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (n_tokens < 0 || hidden < 8 || hidden % 8 || hidden > 16384) return MOE_ERR_INVALID_ARG;
    if (n_experts < 1 || n_experts > 1024 || top_k < 1 || top_k > n_experts) return MOE_ERR_INVALID_ARG;
    if (n_tokens == 0) return MOE_OK;  // an empty batch: nothing to enqueue
    if (!x || !router_w || !idx_out || !gate_out || !workspace) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(workspace)) return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < moe_route_workspace_bytes(n_tokens, n_experts)) return MOE_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status st = init_device(dev);
    if (st != MOE_OK) return st;
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    RouteArgs a{};
    a.x = x;
    a.x_dtype = x_dtype;
    a.wr = router_w;
    a.T = n_tokens;
    a.H = hidden;
    a.E = n_experts;
    a.k = top_k;
    a.rt = route_tokens_per_pass(hidden);
    a.ticket = static_cast<int32_t *>(workspace);
    a.logits = reinterpret_cast<float *>(static_cast<char *>(workspace) + 256);
    a.idx = idx_out;
    a.gate = gate_out;
    a.do_plan = 0;
    a.err = a.ticket + 1;  // word 1 of the workspace: a timed-out wait
    if (x_dtype == MOE_DT_BF16 && n_tokens > kDecodeMaxTokens) {
        // many tokens: the router as a tensor-core GEMM (word 1 of the workspace
        // records a timed-out wait), then top-k per token
        int32_t *werr = a.ticket + 1;
        if (cudaMemsetAsync(werr, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
        return check_launch(prefill_route(x, router_w, n_tokens, hidden, n_experts, top_k, a.logits, idx_out,
                                          gate_out, nullptr, werr, s));
    }
    // tickets: word 0 and words 2.. (one per 8-token block); the kernel leaves them zero
    if (cudaMemsetAsync(a.ticket, 0, 64, s) != cudaSuccess) return MOE_ERR_CUDA;
    return check_launch(launch_route(a, route_grid(n_experts, n_tokens, a.rt, sms), s));
}

moe_status moe_layer_forward_ex(const void *x, moe_dtype x_dtype, const uint16_t *router_w,
                                const moe_pack *p, moe_fmt fmt, int n_tokens, int top_k, float *out,
                                moe_path path, void *stream)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (n_tokens < 0 || n_tokens > p->max_tokens) return MOE_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > p->max_top_k) return MOE_ERR_INVALID_ARG;
    if (fmt != MOE_FMT_FROM_PACK && fmt != p->fmt_gu_in) return MOE_ERR_FMT_MISMATCH;
    const bool prefill_ok = p->has_prefill && x_dtype == MOE_DT_BF16 && top_k <= 32;
    if (path == MOE_PATH_PREFILL_BF16 &&
        (!prefill_ok || !prefill_q8_supported(p->fmt_gu, p->fmt_dn, p->H, p->I, p->E, top_k, true)))
        return MOE_ERR_UNSUPPORTED;
    if (path == MOE_PATH_AUTO)
        path = n_tokens <= kDecodeMaxTokens ? MOE_PATH_DECODE : (prefill_ok ? MOE_PATH_PREFILL : MOE_PATH_GROUPED);
    if (path == MOE_PATH_PREFILL && !prefill_ok) return MOE_ERR_UNSUPPORTED;
    if (path == MOE_PATH_DENSE && (!(p->flags & MOE_PACK_DENSE) || n_tokens > kDecodeMaxTokens))
        return MOE_ERR_UNSUPPORTED;
    if (path != MOE_PATH_DECODE && path != MOE_PATH_GROUPED && path != MOE_PATH_PREFILL && path != MOE_PATH_DENSE &&
        path != MOE_PATH_DECODE_STAGED && path != MOE_PATH_TAIL && path != MOE_PATH_PREFILL_BF16)
        return MOE_ERR_UNSUPPORTED;
    if ((path == MOE_PATH_DECODE_STAGED || path == MOE_PATH_TAIL) && n_tokens > kDecodeTcMaxN) return MOE_ERR_UNSUPPORTED;
    // a pack holding an expert window runs only the one-launch tail (its plan
    // skips the other packs' experts)
    const bool windowed = p->n_local < p->E;
    if (windowed) {
        if ((path != MOE_PATH_DECODE && path != MOE_PATH_TAIL) || n_tokens > kDecodeTcMaxN) return MOE_ERR_UNSUPPORTED;
        path = MOE_PATH_TAIL;
    }
    // an empty batch enqueues nothing and leaves the pack's routing record as it was
    if (n_tokens == 0) return MOE_OK;
    if (!x || !router_w || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    DeviceGuard g(p->device);
    if (!g.ok) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    moe_pack *pm = const_cast<moe_pack *>(p);
    const Workspace &w = p->ws;
    const int T = n_tokens, k = top_k;
    if (path == MOE_PATH_PREFILL || path == MOE_PATH_PREFILL_BF16) {
        PrefillNvArgs pa{};
        pa.x = x;
        pa.wr = router_w;
        pa.T = T;
        pa.H = p->H;
        pa.I = p->I;
        pa.E = p->E;
        pa.k = k;
        pa.has_shared = p->has_shared;
        pa.gu = &p->gu;
        pa.dn = &p->dn;
        pa.tab_gu = p->ct_gu;
        pa.tab_dn = p->ct_dn;
        pa.out = out;
        pa.err = w.err;
        pa.ws = &p->pws;
        pa.num_sms = p->num_sms;
        int pbase = -1;
        if (pm->prof_on && (size_t)pm->prof_used + 2 <= pm->prof_ev.size()) {
            pbase = pm->prof_used;
            pm->prof_used += 2;
            pm->prof_fwd.push_back({pbase, 2});
        }
        prof_mark(pm, pbase, 0, s);
        const bool native = p->fmt_gu == MOE_FMT_NVFP4 && p->fmt_dn == MOE_FMT_NVFP4 && path == MOE_PATH_PREFILL;
        moe_status st = check_launch(native ? prefill_nvfp4_forward(pa, s) : prefill_q8_forward(pa, s));
        prof_mark(pm, pbase, 1, s);
        return st;
    }
    // two or more tokens: the tensor-core grouped decode (below), else the
    // streamed grouped matvecs (rows per lane, TMA-fed) when the planes' rows
    // fit their tile loads, else the fused or plain grouped kernels
    if (pm->sgm < 0) {
        const int slots = p->n_local + (p->has_shared ? 1 : 0);
        pm->sgm = (w.max_groups <= sgm_max_groups() && p->I % 16 == 0 && p->H % 32 == 0 &&
                   sgm_prepare(p->gu, slots, true, &pm->sg_gu) && sgm_prepare(p->dn, slots, false, &pm->sg_dn) &&
                   sgm_stages(pm->sg_gu, p->H) >= 2 && sgm_stages(pm->sg_dn, p->I) >= 2)
                      ? 1
                      : 0;
    }
    if (pm->dtc < 0) {
        const int64_t slots = std::max<int64_t>((int64_t)p->max_tokens * (p->max_top_k + 1), 1);
        pm->dtc = decode_tc_supported(p->gu, p->dn, p->H, p->I, p->max_tokens, p->max_top_k) &&
                          decode_tc_maps(&pm->dtc_maps, p->gu, p->dn, p->n_local + (p->has_shared ? 1 : 0), w.xg, w.h,
                                         (int)slots, p->H, p->I)
                      ? 1
                      : 0;
    }
    // 2..64 tokens: the one-launch tail when it fits, else the tensor-core
    // grouped decode in separate launches, when the pack's weights are
    // fp16-representable (one token: the single-token streaming kernel)
    bool use_tail = false;
    if (path == MOE_PATH_TAIL || (path == MOE_PATH_DECODE && T >= 2)) {
        const int xb = x_dtype == MOE_DT_BF16 ? 1 : 0;
        int &ok = pm->tail_ok[T][xb];
        if (ok < 0) {
            TailPlanIn in{T, p->max_tokens, p->H, p->E, p->I, p->max_top_k, x_dtype, p->fmt_gu, p->fmt_dn, p->num_sms};
            TailLaunch &L = pm->tail_launch[T][xb];
            ok = pm->dtc == 1 && p->gu.tl && p->dn.tl && p->max_tokens <= kDecodeMaxTokens && tail_plan(in, &L) &&
                         tail_blocks_per_sm(p->fmt_gu, p->fmt_dn, L.smem) >= 1
                     ? 1
                     : 0;
        }
        use_tail = ok == 1;
        if (path == MOE_PATH_TAIL && !use_tail) return MOE_ERR_UNSUPPORTED;
    }
    if (use_tail) {
        TailCall tc{};
        tc.x = x;
        tc.x_dtype = x_dtype;
        tc.wr = router_w;
        tc.T = T;
        tc.H = p->H;
        tc.E = p->E;
        tc.eb = p->eb;
        tc.ee = p->ee;
        tc.I = p->I;
        tc.k = k;
        tc.has_shared = p->has_shared;
        tc.gu = &p->gu;
        tc.dn = &p->dn;
        tc.tab_gu = p->ct_gu;
        tc.tab_dn = p->ct_dn;
        tc.ws = &p->ws;
        tc.maps = &pm->dtc_maps;
        tc.out = out;
        int pbase = -1;
        if (pm->prof_on && (size_t)pm->prof_used + 2 <= pm->prof_ev.size()) {
            pbase = pm->prof_used;
            pm->prof_used += 2;
            pm->prof_fwd.push_back({pbase, 1});
            if (pm->prof_stamps && pm->prof_nstamp < pm->prof_stamp_cap)
                tc.stamps = pm->prof_stamps + kStampStride * (size_t)pm->prof_nstamp++;
        }
        prof_mark(pm, pbase, 0, s);
        moe_status st = check_launch(launch_tail(tc, pm->tail_launch[T][x_dtype == MOE_DT_BF16 ? 1 : 0], p->num_sms,
                                                 pm->pdl && pbase < 0, s));
        prof_mark(pm, pbase, 1, s);
        return st;
    }
    const bool use_dtc =
        (path == MOE_PATH_DECODE || path == MOE_PATH_DECODE_STAGED) && T >= 2 && T <= kDecodeTcMaxN && pm->dtc == 1;
    if (path == MOE_PATH_DECODE_STAGED && !use_dtc) return MOE_ERR_UNSUPPORTED;
    // one token: the single-token kernels; 2..8 tokens: the fused kernel unless
    // the streamed grouped matvecs or the tensor-core grouped decode apply
    if (path == MOE_PATH_DECODE && T <= kFusedMaxT && k <= kFusedMaxK && (T == 1 || (pm->sgm != 1 && !use_dtc))) {
        FusedArgs fa{};
        fa.x = x;
        fa.x_dtype = x_dtype;
        fa.wr = router_w;
        fa.T = T;
        fa.H = p->H;
        fa.E = p->E;
        fa.I = p->I;
        fa.k = k;
        fa.has_shared = p->has_shared;
        fa.gu = p->gu;
        fa.dn = p->dn;
        fa.tab_gu = p->ct_gu;
        fa.tab_dn = p->ct_dn;
        fa.logits = w.logits;
        fa.h = w.h;
        fa.y = w.y;
        fa.out = out;
        fa.idx_out = w.idx;
        fa.gate_out = w.gate;
        fa.cnt_out = w.cnt;
        fa.bar = w.bar;
        fa.err = w.err;
        fa.xcnt = w.xcnt;
        if (T == 1) {
            if (pm->stream1 < 0) {
                // probe with the pack's largest top-k: the layout only grows with k
                FusedArgs probe = fa;
                probe.k = p->max_top_k;
                pm->stream1 = stream1_supported(probe, p->num_sms, 226 * 1024) ? 1 : 0;
                pm->stream1_smem = pm->stream1 ? stream1_smem_bytes(probe, p->num_sms) : 0;
                // its grid hand-overs need every CTA resident at once: one CTA
                // per SM must fit (grid = SMs), checked once per pack
                if (pm->stream1 && stream1_blocks_per_sm(probe, pm->stream1_smem) < 1) pm->stream1 = 0;
            }
            if (pm->stream1 && p->max_top_k <= kFusedMaxK) {
                int pbase = -1;
                if (pm->prof_on && (size_t)pm->prof_used + 2 <= pm->prof_ev.size()) {
                    pbase = pm->prof_used;
                    pm->prof_used += 2;
                    pm->prof_fwd.push_back({pbase, 1});
                    if (pm->prof_stamps && pm->prof_nstamp < pm->prof_stamp_cap)
                        fa.stamps = pm->prof_stamps + kStampStride * (size_t)pm->prof_nstamp++;
                }
                prof_mark(pm, pbase, 0, s);
                moe_status st = check_launch(launch_stream1(fa, p->num_sms, stream1_smem_bytes(fa, p->num_sms),
                                                            pm->pdl && pbase < 0, s));
                prof_mark(pm, pbase, 1, s);
                return st;
            }
        }
        const int tt = T == 1 ? 1 : 8;
        const size_t limit = 220 * 1024;
        fa.rowsplit = fused_smem_bytes(fa, tt, 1) <= limit ? 1 : 0;
        const size_t smem = fused_smem_bytes(fa, tt, fa.rowsplit);
        if (smem <= limit) {
            int &grid = pm->fused_grid[tt == 8];
            if (!grid) grid = fused_grid(tt, 220 * 1024, p->num_sms);
            if (grid > 0) {
                int pbase = -1;
                if (pm->prof_on && (size_t)pm->prof_used + 2 <= pm->prof_ev.size()) {
                    pbase = pm->prof_used;
                    pm->prof_used += 2;
                    pm->prof_fwd.push_back({pbase, 1});
                    if (pm->prof_stamps && pm->prof_nstamp < pm->prof_stamp_cap)
                        fa.stamps = pm->prof_stamps + kStampStride * (size_t)pm->prof_nstamp++;
                }
                prof_mark(pm, pbase, 0, s);
                moe_status st = check_launch(launch_fused(fa, tt, grid, smem, s));
                prof_mark(pm, pbase, 1, s);
                return st;
            }
        }
    }
    // tokens per work group: 8 unless a single token, or 8 staged fp32 rows of
    // the longer reduction would not fit in shared memory
    const int kmax = std::max(p->H, p->I);
    const int tt = use_dtc ? kDecodeTcMaxN : (T == 1 || (size_t)8 * kmax * 4 * 33 / 32 > 200 * 1024) ? 1 : 8;
    int pbase = -1;
    if (pm->prof_on && (size_t)pm->prof_used + 5 <= pm->prof_ev.size()) {
        pbase = pm->prof_used;
        pm->prof_used += 5;
        pm->prof_fwd.push_back({pbase, 0});
    }
    prof_mark(pm, pbase, 0, s);

    RouteArgs ra{};
    ra.x = x;
    ra.x_dtype = x_dtype;
    ra.wr = router_w;
    ra.T = T;
    ra.H = p->H;
    ra.E = p->E;
    ra.k = k;
    ra.rt = route_tokens_per_pass(p->H);
    ra.logits = w.logits;
    ra.ticket = w.ticket;
    ra.idx = w.idx;
    ra.gate = w.gate;
    ra.do_plan = 1;
    ra.has_shared = p->has_shared;
    ra.tt = tt;
    ra.cnt = w.cnt;
    ra.off = w.off;
    ra.perm_tok = w.perm_tok;
    ra.slot_pos = w.slot_pos;
    ra.n_groups = w.n_groups;
    ra.err = w.err;
    ra.groups = w.groups;
    ra.max_groups = w.max_groups;
    ra.dense = path == MOE_PATH_DENSE;
    ra.dgate = w.dgate;
    ra.n_dense_rows = w.n_dense_rows;
    if (pbase >= 0 && pm->prof_stamps && pm->prof_nstamp < pm->prof_stamp_cap)
        ra.stamps = pm->prof_stamps + kStampStride * (size_t)pm->prof_nstamp++;
    moe_status st = check_launch(launch_route(ra, route_grid(p->E, T, ra.rt, p->num_sms), s));
    if (st != MOE_OK) return st;
    prof_mark(pm, pbase, 1, s);

    if (use_dtc) {
        // x into fp16 slot rows, then the two tensor-core GEMMs (y per slot);
        // the combine below sums each token's slots
        st = check_launch(launch_decode_tc_gather(x, x_dtype, T, p->H, k, p->has_shared, w.slot_pos, w.xg,
                                                  w.slot_scale, s));
        if (st != MOE_OK) return st;
        st = check_launch(launch_decode_tc(pm->dtc_maps, true, p->gu, w.groups, w.n_groups, p->H, p->I, p->ct_gu,
                                           w.slot_scale, w.h, w.y, w.err, p->max_tokens, p->num_sms, s));
        if (st != MOE_OK) return st;
        prof_mark(pm, pbase, 2, s);
        st = check_launch(launch_decode_tc(pm->dtc_maps, false, p->dn, w.groups, w.n_groups, p->H, p->I, p->ct_dn,
                                           w.slot_scale, w.h, w.y, w.err, p->max_tokens, p->num_sms, s));
        if (st != MOE_OK) return st;
        prof_mark(pm, pbase, 3, s);
    } else if (path == MOE_PATH_DECODE && T >= 2 && tt == 8 && pm->sgm == 1) {
        st = check_launch(launch_sgm(pm->sg_gu, p->gu, w.groups, w.n_groups, w.perm_tok, x, x_dtype, w.h, p->I,
                                     p->I, true, p->ct_gu, w.err, p->num_sms, s));
        if (st != MOE_OK) return st;
        prof_mark(pm, pbase, 2, s);
        st = check_launch(launch_sgm(pm->sg_dn, p->dn, w.groups, w.n_groups, w.perm_tok, w.h, MOE_DT_F32, w.y,
                                     p->H, p->H, false, p->ct_dn, w.err, p->num_sms, s));
        if (st != MOE_OK) return st;
        prof_mark(pm, pbase, 3, s);
    } else {
    MatvecArgs gu{};
    gu.w = p->gu;
    gu.groups = w.groups;
    gu.n_groups = w.n_groups;
    gu.perm_tok = w.perm_tok;
    gu.x = x;
    gu.x_dtype = x_dtype;
    gu.out = w.h;
    gu.out_stride = p->I;
    gu.rows_out = p->I;
    gu.tab = p->ct_gu;
    int &ggu = pm->grid_cache[1][tt == 8];
    if (!ggu) ggu = matvec_grid(gu, true, tt, p->num_sms);
    st = check_launch(launch_matvec(gu, true, tt, ggu, s));
    if (st != MOE_OK) return st;
    prof_mark(pm, pbase, 2, s);

    MatvecArgs dn{};
    dn.w = p->dn;
    dn.groups = w.groups;
    dn.n_groups = w.n_groups;
    dn.perm_tok = w.perm_tok;
    dn.x = w.h;
    dn.x_dtype = MOE_DT_F32;
    dn.out = w.y;
    dn.out_stride = p->H;
    dn.rows_out = p->H;
    dn.tab = p->ct_dn;
    int &gdn = pm->grid_cache[0][tt == 8];
    if (!gdn) gdn = matvec_grid(dn, false, tt, p->num_sms);
    st = check_launch(launch_matvec(dn, false, tt, gdn, s));
    if (st != MOE_OK) return st;
    prof_mark(pm, pbase, 3, s);
    }

    if (path == MOE_PATH_DENSE) {
        st = check_launch(launch_combine_dense(w.y, w.dgate, w.n_dense_rows, T, p->H, out, s));
        prof_mark(pm, pbase, 4, s);
        return st;
    }
    CombineArgs ca{};
    ca.y = w.y;
    ca.slot_pos = w.slot_pos;
    ca.gate = w.gate;
    ca.T = T;
    ca.k = k;
    ca.H = p->H;
    ca.has_shared = p->has_shared;
    ca.out = out;
    st = check_launch(launch_combine(ca, s));
    prof_mark(pm, pbase, 4, s);
    return st;
}

moe_status moe_layer_forward(const void *x, moe_dtype x_dtype, const uint16_t *router_w,
                             const moe_pack *pack, moe_fmt fmt, int n_tokens, int top_k, float *out,
                             void *stream)
{
    return moe_layer_forward_ex(x, x_dtype, router_w, pack, fmt, n_tokens, top_k, out, MOE_PATH_AUTO,
                                stream);
}

moe_status moe_read_routing(const moe_pack *p, int n_tokens, int top_k, int32_t *idx, float *gate,
                            int32_t *counts, void *stream)
{
    if (!p || n_tokens < 1 || n_tokens > p->max_tokens || top_k < 1 || top_k > p->max_top_k)
        return MOE_ERR_INVALID_ARG;
    DeviceGuard g(p->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = (size_t)n_tokens * top_k;
    if (idx && cudaMemcpyAsync(idx, p->ws.idx, n * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (gate && cudaMemcpyAsync(gate, p->ws.gate, n * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (counts && cudaMemcpyAsync(counts, p->ws.cnt, (size_t)(p->E + 1) * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_profile_begin(moe_pack *p, int max_forwards)
{
    if (!p || max_forwards < 1 || max_forwards > (1 << 20) || p->prof_on) return MOE_ERR_INVALID_ARG;
    DeviceGuard g(p->device);
    p->prof_ev.assign((size_t)max_forwards * 5, nullptr);
    for (auto &e : p->prof_ev)
        if (cudaEventCreate(&e) != cudaSuccess) {
            for (auto &f : p->prof_ev)
                if (f) cudaEventDestroy(f);
            p->prof_ev.clear();
            return MOE_ERR_CUDA;
        }
    p->prof_fwd.clear();
    p->prof_used = 0;
    p->prof_nstamp = 0;
    p->prof_stamp_cap = max_forwards;
    if (cudaMalloc(&p->prof_stamps, sizeof(long long) * kStampStride * (size_t)max_forwards) != cudaSuccess ||
        cudaMemset(p->prof_stamps, 0, sizeof(long long) * kStampStride * (size_t)max_forwards) != cudaSuccess) {
        cudaGetLastError();
        p->prof_stamps = nullptr;
        p->prof_stamp_cap = 0;
    }
    p->prof_on = true;
    return MOE_OK;
}

moe_status moe_profile_end(moe_pack *p, double *ms, int *n_forwards)
{
    if (!p || !p->prof_on) return MOE_ERR_INVALID_ARG;
    DeviceGuard g(p->device);
    moe_status st = cudaDeviceSynchronize() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    double acc[PROF_OUT] = {};
    for (const auto &f : p->prof_fwd) {
        if (st != MOE_OK) break;
        const int nint = f.second ? 1 : 4;
        for (int i = 0; i < nint; ++i) {
            float v = 0.f;
            if (cudaEventElapsedTime(&v, p->prof_ev[(size_t)f.first + i], p->prof_ev[(size_t)f.first + i + 1]) !=
                cudaSuccess) {
                st = MOE_ERR_CUDA;
                break;
            }
            acc[f.second == 1 ? PROF_FUSED : f.second == 2 ? PROF_PREFILL : i] += v;
        }
    }
    if (p->prof_stamps && p->prof_nstamp > 0 && st == MOE_OK) {
        // fused-kernel phases (CTA 0's clock): stage, router, barrier, plan,
        // gate/up, barrier, down, barrier, combine/tail
        std::vector<long long> h((size_t)kStampStride * p->prof_nstamp);
        int khz = 0;
        cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, p->device);
        if (khz > 0 && cudaMemcpy(h.data(), p->prof_stamps, h.size() * sizeof(long long), cudaMemcpyDeviceToHost) ==
                           cudaSuccess) {
            for (int f = 0; f < p->prof_nstamp; ++f) {
                const long long *c = h.data() + kStampStride * (size_t)f;
                auto span = [&](int a, int b) { return (c[a] && c[b] && c[b] > c[a]) ? (double)(c[b] - c[a]) : 0.0; };
                double ph[PROF_PHASES];
                for (int i = 0; i < 7; ++i) ph[i] = span(i, i + 1);
                ph[7] = span(7, 8);
                ph[8] = c[8] ? span(8, 9) : span(7, 9);
                for (int i = 0; i < PROF_PHASES; ++i) acc[PROF_STAGES + i] += ph[i] / khz;  // cycles / kHz = ms
                // grid-wide events (global timer, ns): first and last CTA of each,
                // relative to the first CTA's start; the first start is stored as
                // 2^62 - t so that one atomic maximum serves both
                // CTA 0 sub-steps of the streaming kernel (clock64 at [24..31]), from its start
                for (int i = 0; i < PROF_SUB; ++i)
                    if (c[24 + i] > c[0] && c[0])
                        acc[PROF_STAGES + PROF_PHASES + PROF_GRID + i] += (double)(c[24 + i] - c[0]) / khz;
                if (c[11] > 0) {
                    const long long t0 = (1ll << 62) - c[10];
                    double *gx = acc + PROF_STAGES + PROF_PHASES;
                    gx[0] += (c[11] - t0) * 1e-6;
                    for (int ev = 1; ev < 5; ++ev) {
                        if (c[11 + 2 * ev] <= 0) continue;
                        gx[2 * ev - 1] += ((1ll << 62) - c[10 + 2 * ev] - t0) * 1e-6;
                        gx[2 * ev] += (c[11 + 2 * ev] - t0) * 1e-6;
                    }
                }
            }
        }
    }
    if (p->prof_stamps) cudaFree(p->prof_stamps);
    p->prof_stamps = nullptr;
    p->prof_nstamp = p->prof_stamp_cap = 0;
    for (auto &e : p->prof_ev) cudaEventDestroy(e);
    const int n = (int)p->prof_fwd.size();
    p->prof_ev.clear();
    p->prof_fwd.clear();
    p->prof_on = false;
    p->prof_used = 0;
    if (ms)
        for (int i = 0; i < PROF_OUT; ++i) ms[i] = acc[i];
    if (n_forwards) *n_forwards = n;
    return st;
}

moe_status moe_debug_wait_timeout(const moe_pack *p, void *stream)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    DeviceGuard g(p->device);
    if (!g.ok) return MOE_ERR_CUDA;
    return check_launch(launch_wait_probe(p->ws.err, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_act_quant_nvfp4(const void *x, moe_dtype x_dtype, int rows, int cols, uint8_t *codes,
                                     uint8_t *scales, float *row_scale, void *stream)
{
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (rows < 1 || rows > 65536 || cols < 64 || cols > 16384 || cols % 64) return MOE_ERR_INVALID_ARG;
    if (!x || !codes || !scales || !row_scale || !aligned16(x) || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status st = init_device(dev);
    if (st != MOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int ks = cols / 64, blocks128 = (rows + 127) / 128;
    const size_t atom_bytes = (size_t)blocks128 * ks * 512, scratch_bytes = (size_t)(7 * rows + 8) * 4;
    void *atoms = nullptr, *scratch = nullptr;
    std::vector<uint8_t> h_atoms(atom_bytes), h_sc((size_t)rows * (cols / 16));
    st = MOE_ERR_CUDA;
    if (cudaMalloc(&atoms, atom_bytes) == cudaSuccess && cudaMalloc(&scratch, scratch_bytes) == cudaSuccess &&
        cudaMemsetAsync(atoms, 0, atom_bytes, s) == cudaSuccess &&
        cudaMemsetAsync(scratch, 0, scratch_bytes, s) == cudaSuccess &&
        debug_act_quant(x, x_dtype == MOE_DT_BF16, rows, cols, codes, static_cast<uint8_t *>(atoms), row_scale,
                        static_cast<int32_t *>(scratch), s) == cudaSuccess &&
        cudaMemcpyAsync(h_atoms.data(), atoms, atom_bytes, cudaMemcpyDeviceToHost, s) == cudaSuccess &&
        cudaStreamSynchronize(s) == cudaSuccess) {
        for (int r = 0; r < rows; ++r)
            for (int b = 0; b < cols / 16; ++b)
                h_sc[(size_t)r * (cols / 16) + b] = h_atoms[(size_t)sf_offset(r, b >> 2, b & 3, ks)];
        if (cudaMemcpy(scales, h_sc.data(), h_sc.size(), cudaMemcpyHostToDevice) == cudaSuccess) st = MOE_OK;
    }
    cudaGetLastError();
    if (atoms) cudaFree(atoms);
    if (scratch) cudaFree(scratch);
    return st;
}

moe_status moe_debug_dequant_rows(const moe_pack *p, int proj, int slot, int row0, int nrows, int kind, void *out,
                                  void *stream)
{
    if (!p || (proj != 0 && proj != 1) || (kind != 0 && kind != 1) || !out || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    const DevProj &w = proj == 0 ? p->gu : p->dn;
    if (slot < 0 || slot >= p->n_local + p->has_shared || row0 < 0 || nrows < 1 || row0 > w.rows - nrows)
        return MOE_ERR_INVALID_ARG;
    DeviceGuard g(p->device);
    return check_launch(debug_dequant(w, proj == 0 ? p->ct_gu : p->ct_dn, slot, row0, nrows, kind, out,
                                      static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_tail_plan(int n_tokens, int max_tokens, int hidden, int n_experts, int inter, int top_k,
                               moe_dtype x_dtype, moe_fmt fmt_gate_up, moe_fmt fmt_down, int grid, int64_t *out)
{
    if (!out || !valid_fmt(fmt_gate_up) || !valid_fmt(fmt_down) || (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16))
        return MOE_ERR_INVALID_ARG;
    TailPlanIn in{n_tokens, max_tokens, hidden, n_experts, inter, top_k, x_dtype, device_fmt(fmt_gate_up),
                  device_fmt(fmt_down), grid};
    TailLaunch L{};
    const bool fits = tail_plan(in, &L);
    const int64_t v[8] = {fits ? 1 : 0, L.nr, L.nb, L.raw_stride, L.bslot, L.rings, (int64_t)L.smem, L.na};
    for (int i = 0; i < 8; ++i) out[i] = fits ? v[i] : 0;
    return MOE_OK;
}

moe_status moe_get_device_error(const moe_pack *p)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    DeviceGuard g(p->device);
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    int32_t e = 0;
    if (cudaMemcpy(&e, p->ws.err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (e) cudaMemset(p->ws.err, 0, 4);
    return static_cast<moe_status>(e);
}

}  // extern "C"
