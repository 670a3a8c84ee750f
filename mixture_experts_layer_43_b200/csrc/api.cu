// api.cu -- the C ABI of libmoe_b200.so (declared in include/moe.h): argument
// checks, the plan (workspace, tensor-map encoder, tiling choices) and the
// launch sequence of each regime.  No kernel code lives here.
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <new>

#include "moe_internal.cuh"
#include "prefill.cuh"

using namespace moe;

struct moe_plan_s {
    moe_config_t cfg;
    int num_sms = 0;
    size_t smem_optin = 0;
    Workspace ws{};
    void* ws_base = nullptr;
    size_t ws_bytes = 0;
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    int route_epc = 1;
    bool coop = false;          // cooperative launches available (fused decode kernel)
    int last_launches = 0;
    // tensor maps of the weights seen by the decode regime (small cache, so a
    // caller that rotates several layers' weights does not re-encode them)
    static constexpr int kMapCache = 64;
    struct MapEntry {
        bool valid = false;
        int fs = 0;
        moe_weights_t w{};
        DecodeArgs args{};
    };
    MapEntry maps[kMapCache];
    int maps_next = 0;
    // prefill regime state (tensor maps of the last weights/x)
    PrefillState* pf = nullptr;
};

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

moe_status_t check_config(const moe_config_t* c) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->t_max < 1 || c->d_model < 128 || c->d_model % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (c->d_ff < 32 || c->d_ff % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (c->n_experts < 1 || c->n_experts > kMaxExperts) return MOE_ERR_INVALID_ARG;
    if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > kMaxTopK) return MOE_ERR_INVALID_ARG;
    if (c->n_shared < 0 || c->n_shared > kMaxShared) return MOE_ERR_INVALID_ARG;
    if (c->n_shared > 0 && (c->d_ff_shared < 32 || c->d_ff_shared % 32 != 0))
        return MOE_ERR_INVALID_ARG;
    if (c->wfmt != MOE_WFMT_BF16 && c->wfmt != MOE_WFMT_Q4_0 && c->wfmt != MOE_WFMT_Q8_0 &&
        c->wfmt != MOE_WFMT_Q5_0 && c->wfmt != MOE_WFMT_Q6_K && c->wfmt != MOE_WFMT_BF16_F16DOWN)
        return MOE_ERR_INVALID_ARG;
    // q6_K super-blocks run along the reduction dim of every matrix
    if (c->wfmt == MOE_WFMT_Q6_K &&
        (c->d_model % 256 || c->d_ff % 256 || (c->n_shared > 0 && c->d_ff_shared % 256)))
        return MOE_ERR_INVALID_ARG;
    if (c->regime < MOE_REGIME_AUTO || c->regime > MOE_REGIME_PREFILL) return MOE_ERR_INVALID_ARG;
    if (c->device < 0) return MOE_ERR_INVALID_ARG;
    // 2^31 limits of the int32 index arithmetic in the kernels
    if (static_cast<int64_t>(c->t_max) * c->top_k * c->d_model >= (1ll << 31))
        return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(c->n_experts) * c->d_ff >= (1ll << 31) ||
        static_cast<int64_t>(c->n_experts) * c->d_model >= (1ll << 31))
        return MOE_ERR_INVALID_ARG;
    if (wfmt_quantised(c->wfmt) && c->regime == MOE_REGIME_PREFILL) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

bool use_decode(const moe_plan_s* p, int T) {
    if (p->cfg.regime == MOE_REGIME_DECODE) return true;
    if (p->cfg.regime == MOE_REGIME_PREFILL) return false;
    return T <= MOE_DECODE_MAX_T || wfmt_quantised(p->cfg.wfmt);
}

moe_status_t check_matrix(const moe_matrix_t& m, bool quant) {
    if (!m.data || !aligned16(m.data)) return MOE_ERR_INVALID_ARG;
    if (quant ? (!m.scales || !aligned16(m.scales)) : (m.scales != nullptr)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// top_k and wfmt restate the plan's: a call whose k or weight format differs
// from the plan it runs on is rejected before anything is enqueued.
moe_status_t check_call(const moe_plan_s* p, const moe_weights_t* w, const void* x, int32_t T,
                        int32_t top_k, int32_t wfmt, const float* out) {
    if (!p || !w) return MOE_ERR_INVALID_ARG;
    if (top_k != p->cfg.top_k || wfmt != p->cfg.wfmt) return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > p->cfg.t_max) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !out || !aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if (!w->router_w || !aligned16(w->router_w)) return MOE_ERR_INVALID_ARG;
    if (w->router_b && (reinterpret_cast<uintptr_t>(w->router_b) & 3u)) return MOE_ERR_INVALID_ARG;
    const bool quant = wfmt_quantised(p->cfg.wfmt);     // quantised: codes + scales
    moe_status_t s;
    if ((s = check_matrix(w->gate, quant)) || (s = check_matrix(w->up, quant)) ||
        (s = check_matrix(w->down, quant)))
        return s;
    if (p->cfg.n_shared > 0 &&
        ((s = check_matrix(w->shared_gate, quant)) || (s = check_matrix(w->shared_up, quant)) ||
         (s = check_matrix(w->shared_down, quant))))
        return s;
    if (use_decode(p, T) && T > MOE_DECODE_MAX_T) return MOE_ERR_UNSUPPORTED;
    if (!use_decode(p, T) && quant) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// ------------------------------------------------------------ tensor maps
// L2 promotion no wider than the contiguous bytes one box row reads: a
// wider promotion fetches the neighbouring columns too (the next work unit's
// slice of the down matrix), which the evict-first streaming hint may evict
// again before that unit runs.
CUtensorMapL2promotion promotion_for(uint32_t row_bytes) {
    return row_bytes >= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
         : row_bytes >= 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                            : CU_TENSOR_MAP_L2_PROMOTION_L2_64B;
}

bool encode_map(moe_plan_s* p, CUtensorMap* m, CUtensorMapDataType dt, int rank,
                const void* base, const uint64_t* dims, const uint64_t* strides,
                const uint32_t* box, CUtensorMapSwizzle sw, uint32_t row_bytes) {
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult r = p->encode(m, dt, rank, const_cast<void*>(base), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, sw, promotion_for(row_bytes),
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
    return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
         : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

// bf16 stack [mats][rows][K] seen as 2D [mats*rows][K], box {box_k, box_rows}.
bool map_bf16(moe_plan_s* p, CUtensorMap* m, const void* base, int64_t mats, int64_t rows,
              int64_t K, uint32_t box_k, uint32_t box_rows) {
    uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(mats * rows)};
    uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
    uint32_t box[2] = {box_k, box_rows};
    return encode_map(p, m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                      swizzle_for(static_cast<int>(box_k) * 2), box_k * 2);
}

// Q4_0 / Q8_0 / Q5_0 / q6_K packed codes [mats][K/32][N][cb] (cb = 16 / 32 /
// 16 / 16 bytes per block row) seen as 3D {16 rows * cb, N/16, mats*K/32} in
// 32-bit words: the innermost box dimension is a whole 16-row group, one
// 256- or 512-byte line.  (Boxes of cb-byte lines move the same bytes in 16
// times as many lines, and the TMA unit's line rate then caps the stream far
// below HBM bandwidth.)  Coordinates: {0, first row / 16, block column}.
bool map_quant_codes(moe_plan_s* p, CUtensorMap* m, const void* base, int64_t mats, int64_t N,
                     int64_t K, uint32_t box_rows, uint32_t box_kb, uint32_t cb) {
    uint64_t dims[3] = {16ull * cb / 4, static_cast<uint64_t>(N / 16),
                        static_cast<uint64_t>(mats * (K / 32))};
    uint64_t strides[2] = {16ull * cb, static_cast<uint64_t>(N) * cb};
    uint32_t box[3] = {16 * cb / 4, box_rows / 16, box_kb};
    return encode_map(p, m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE, cb * box_rows);   // rows are contiguous
}

// Q4_0 / Q8_0 packed scales [mats][K/32][N] fp16 seen as 2D {N, mats*K/32}.
bool map_quant_scales(moe_plan_s* p, CUtensorMap* m, const void* base, int64_t mats, int64_t N,
                   int64_t K, uint32_t box_rows, uint32_t box_kb) {
    uint64_t dims[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(mats * (K / 32))};
    uint64_t strides[1] = {static_cast<uint64_t>(N) * 2};
    uint32_t box[2] = {box_rows, box_kb};
    return encode_map(p, m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE, 2 * box_rows);
}

// q6_K packed records [mats][K/32][N/16][160 bytes] seen as 3D {160, N/16,
// mats*K/32}; a box of box_rows rows reads box_rows/16 records.
bool map_q6_aux(moe_plan_s* p, CUtensorMap* m, const void* base, int64_t mats, int64_t N,
                int64_t K, uint32_t box_rows, uint32_t box_kb) {
    uint64_t dims[3] = {160, static_cast<uint64_t>(N / 16), static_cast<uint64_t>(mats * (K / 32))};
    uint64_t strides[2] = {160, static_cast<uint64_t>(N / 16) * 160};
    uint32_t box[3] = {160, box_rows / 16, box_kb};
    return encode_map(p, m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE, 10 * box_rows);   // records are contiguous
}

// q6_K super-block scales [mats][K/256][N] fp16 seen as 2D {N, mats*K/256};
// they follow the records in the packed scales array.
bool map_q6_d(moe_plan_s* p, CUtensorMap* m, const void* scales, int64_t mats, int64_t N, int64_t K,
              uint32_t box_rows, uint32_t box_sb) {
    const uint8_t* base = static_cast<const uint8_t*>(scales) + mats * (N / 16) * (K / 32) * 160;
    uint64_t dims[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(mats * (K / 256))};
    uint64_t strides[1] = {static_cast<uint64_t>(N) * 2};
    uint32_t box[2] = {box_rows, box_sb};
    return encode_map(p, m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE, 2 * box_rows);
}

// Q5_0 packed scales and fifth bits [mats][K/32][N/8][48 bytes] seen as 3D
// {48, N/8, mats*K/32}; a box of box_rows rows reads box_rows/8 records.
bool map_q5_aux(moe_plan_s* p, CUtensorMap* m, const void* base, int64_t mats, int64_t N,
                int64_t K, uint32_t box_rows, uint32_t box_kb) {
    uint64_t dims[3] = {48, static_cast<uint64_t>(N / 8), static_cast<uint64_t>(mats * (K / 32))};
    uint64_t strides[2] = {48, static_cast<uint64_t>(N / 8) * 48};
    uint32_t box[3] = {48, box_rows / 8, box_kb};
    return encode_map(p, m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE, 6 * box_rows);   // records are contiguous
}

bool same_weights(const moe_weights_t& a, const moe_weights_t& b) {
    return memcmp(&a, &b, sizeof(moe_weights_t)) == 0;
}

// F-slice of the decode work units: the largest of {64, 32} dividing F (and
// Fs) whose expected unit count fills the SMs in whole waves to >= 90%.
int pick_fs(const moe_plan_s* p, int T) {
    const moe_config_t& c = p->cfg;
    const double E = c.n_experts;
    const double act = E * (1.0 - pow(1.0 - static_cast<double>(c.top_k) / E, T));
    int best = 32;
    double best_eff = -1.0;
    // the row-streaming pipeline (Q4_0, Q8_0, q6_K) keeps every row group's
    // partial sums in registers, which fit for 32-row slices only
    if (c.wfmt == MOE_WFMT_Q4_0 || c.wfmt == MOE_WFMT_Q8_0 || c.wfmt == MOE_WFMT_Q6_K) return 32;
    for (int fs : {64, 32}) {
        if (c.d_ff % fs || (c.n_shared && c.d_ff_shared % fs)) continue;
        const double units = act * (c.d_ff / fs) + c.n_shared * (c.n_shared ? c.d_ff_shared / fs : 0);
        const double waves = ceil(units / p->num_sms);
        const double eff = units / (waves * p->num_sms);
        if (eff >= 0.9) return fs;
        if (eff > best_eff + 1e-9) { best_eff = eff; best = fs; }
    }
    return best;
}

DecodeArgs* build_decode_maps(moe_plan_s* p, const moe_weights_t* w, int fs) {
    for (auto& e : p->maps)
        if (e.valid && e.fs == fs && same_weights(e.w, *w)) return &e.args;
    auto& ent = p->maps[p->maps_next];
    p->maps_next = (p->maps_next + 1) % moe_plan_s::kMapCache;
    ent.valid = false;
    const moe_config_t& c = p->cfg;
    DecodeArgs& a = ent.args;
    memset(&a, 0, sizeof(a));
    const int64_t E = c.n_experts, d = c.d_model, F = c.d_ff, S = c.n_shared, Fs = c.d_ff_shared;
    bool ok = true;
    if (!wfmt_quantised(c.wfmt)) {   // bf16 (fp16 down matrices: the same 2-byte maps)
        ok &= map_bf16(p, &a.tm_gate, w->gate.data, E, F, d, 64, fs);
        ok &= map_bf16(p, &a.tm_up, w->up.data, E, F, d, 64, fs);
        ok &= map_bf16(p, &a.tm_down, w->down.data, E, d, F, fs, 128);
        if (S) {
            ok &= map_bf16(p, &a.tm_sgate, w->shared_gate.data, S, Fs, d, 64, fs);
            ok &= map_bf16(p, &a.tm_sup, w->shared_up.data, S, Fs, d, 64, fs);
            ok &= map_bf16(p, &a.tm_sdown, w->shared_down.data, S, d, Fs, fs, 128);
        }
    } else {
        // phase-A boxes: Q4_0, Q8_0 and q6_K stream 16-row groups over up to
        // 64 block columns (the row-streaming pipeline); Q5_0 streams
        // 512 / fs block columns of the whole slice
        const bool rows16 = c.wfmt == MOE_WFMT_Q4_0 || c.wfmt == MOE_WFMT_Q8_0 ||
                            c.wfmt == MOE_WFMT_Q6_K;
        const uint32_t kb = rows16 ? static_cast<uint32_t>(d / 32 < 64 ? d / 32 : 64) : 512 / fs;
        const uint32_t ar = rows16 ? 16 : fs;
        const uint32_t nb = fs / 32;
        const uint32_t cb = c.wfmt == MOE_WFMT_Q8_0 ? 32 : 16;
        a.kt = static_cast<int>(kb);
        // scales: fp16 [mats][K/32][N], or Q5_0's 48-byte records of 8 rows
        auto scales = [&](CUtensorMap* m, const void* base, int64_t mats, int64_t N, int64_t K,
                          uint32_t box_rows, uint32_t box_kb) {
            if (c.wfmt == MOE_WFMT_Q6_K) return map_q6_aux(p, m, base, mats, N, K, box_rows, box_kb);
            return c.wfmt == MOE_WFMT_Q5_0 ? map_q5_aux(p, m, base, mats, N, K, box_rows, box_kb)
                                           : map_quant_scales(p, m, base, mats, N, K, box_rows, box_kb);
        };
        if (c.wfmt == MOE_WFMT_Q6_K) {
            // super-block scales: phase A 16 rows x kb/8 super-blocks, phase B
            // 256 rows x the one super-block a slice lies in
            ok &= map_q6_d(p, &a.tm_gate_d, w->gate.scales, E, F, d, 16, kb / 8);
            ok &= map_q6_d(p, &a.tm_up_d, w->up.scales, E, F, d, 16, kb / 8);
            ok &= map_q6_d(p, &a.tm_down_d, w->down.scales, E, d, F, kQuantDownBoxRows, 1);
            if (S) {
                ok &= map_q6_d(p, &a.tm_sgate_d, w->shared_gate.scales, S, Fs, d, 16, kb / 8);
                ok &= map_q6_d(p, &a.tm_sup_d, w->shared_up.scales, S, Fs, d, 16, kb / 8);
                ok &= map_q6_d(p, &a.tm_sdown_d, w->shared_down.scales, S, d, Fs, kQuantDownBoxRows, 1);
            }
        }
        ok &= map_quant_codes(p, &a.tm_gate, w->gate.data, E, F, d, ar, kb, cb);
        ok &= map_quant_codes(p, &a.tm_up, w->up.data, E, F, d, ar, kb, cb);
        ok &= map_quant_codes(p, &a.tm_down, w->down.data, E, d, F, kQuantDownBoxRows, nb, cb);
        ok &= scales(&a.tm_gate_sc, w->gate.scales, E, F, d, ar, kb);
        ok &= scales(&a.tm_up_sc, w->up.scales, E, F, d, ar, kb);
        ok &= scales(&a.tm_down_sc, w->down.scales, E, d, F, kQuantDownBoxRows, nb);
        if (S) {
            ok &= map_quant_codes(p, &a.tm_sgate, w->shared_gate.data, S, Fs, d, ar, kb, cb);
            ok &= map_quant_codes(p, &a.tm_sup, w->shared_up.data, S, Fs, d, ar, kb, cb);
            ok &= map_quant_codes(p, &a.tm_sdown, w->shared_down.data, S, d, Fs, kQuantDownBoxRows, nb, cb);
            ok &= scales(&a.tm_sgate_sc, w->shared_gate.scales, S, Fs, d, ar, kb);
            ok &= scales(&a.tm_sup_sc, w->shared_up.scales, S, Fs, d, ar, kb);
            ok &= scales(&a.tm_sdown_sc, w->shared_down.scales, S, d, Fs, kQuantDownBoxRows, nb);
        }
    }
    if (!ok) return nullptr;
    ent.valid = true;
    ent.w = *w;
    ent.fs = fs;
    return &a;
}

moe_status_t route_decode(moe_plan_s* p, const moe_weights_t* w, const void* x, int T, float* out,
                          cudaStream_t st) {
    RouteArgs r{};
    r.x = static_cast<const uint16_t*>(x);
    r.wr = w->router_w;
    r.br = w->router_b;
    r.out = out;
    r.ws = p->ws;
    r.T = T;
    r.d = p->cfg.d_model;
    r.E = p->cfg.n_experts;
    r.k = p->cfg.top_k;
    r.S = p->cfg.n_shared;
    r.experts_per_cta = p->route_epc;
    return cuda_status(launch_decode_route(r, st));
}

// Fill the per-call fields of the decode arguments; returns the smem bytes.
moe_status_t decode_args(moe_plan_s* p, const moe_weights_t* w, const void* x, int T, float* out,
                         bool fused, DecodeArgs** out_args, int* out_fs, size_t* out_smem) {
    const moe_config_t& c = p->cfg;
    const int fs = pick_fs(p, T);
    DecodeArgs* ap = build_decode_maps(p, w, fs);
    if (!ap) return MOE_ERR_INVALID_ARG;
    DecodeArgs& a = *ap;
    a.x = static_cast<const uint16_t*>(x);
    a.out = out;
    a.items = p->ws.items;
    a.n_items = p->ws.n_items;
    a.slot_token = p->ws.slot_token;
    a.slot_w = p->ws.slot_w;
    a.err = p->ws.err;
    a.T = T;
    a.d = c.d_model;
    a.F = c.d_ff;
    a.Fs = c.n_shared ? c.d_ff_shared : 0;
    a.E = c.n_experts;
    a.S = c.n_shared;
    a.xs_stride = c.d_model * 2 + 16;
    a.wr = w->router_w;
    a.br = w->router_b;
    a.k = c.top_k;
    a.ws = p->ws;
    a.gbar = p->ws.gbar;
    const size_t extra = fused ? decode_fused_extra_smem() : 0;
    const size_t fixed = decode_smem_bytes(fs, c.wfmt, c.d_model, 0) + extra;
    const int stage = decode_stage_bytes(fs, c.wfmt);
    int ns = static_cast<int>((p->smem_optin - fixed) / (stage + 16));
    if (ns > 8) ns = 8;
    if (ns < 2) return MOE_ERR_UNSUPPORTED;
    // the fused kernel keeps its router partial sums ([experts per CTA][16][8]
    // fp32) in the ring during routing
    const size_t n_loc = (static_cast<size_t>(c.n_experts) + p->num_sms - 1) / p->num_sms;
    if (fused && static_cast<size_t>(ns) * stage < n_loc * kDecodeConsumerWarps * kDecodeTok * 4)
        return MOE_ERR_UNSUPPORTED;
    a.n_stages = ns;
    *out_args = ap;
    *out_fs = fs;
    *out_smem = decode_smem_bytes(fs, c.wfmt, c.d_model, ns) + extra;
    return MOE_OK;
}

moe_status_t experts_decode(moe_plan_s* p, const moe_weights_t* w, const void* x, int T, float* out,
                            cudaStream_t st) {
    DecodeArgs* a = nullptr;
    int fs = 0;
    size_t smem = 0;
    moe_status_t s = decode_args(p, w, x, T, out, false, &a, &fs, &smem);
    if (s) return s;
    return cuda_status(launch_decode_experts(*a, fs, p->cfg.wfmt, p->num_sms, smem, st));
}

moe_status_t forward_decode_fused(moe_plan_s* p, const moe_weights_t* w, const void* x, int T,
                                  float* out, cudaStream_t st) {
    DecodeArgs* a = nullptr;
    int fs = 0;
    size_t smem = 0;
    moe_status_t s = decode_args(p, w, x, T, out, true, &a, &fs, &smem);
    if (s) return s;
    return cuda_status(launch_decode_fused(*a, fs, p->cfg.wfmt, p->num_sms, smem, st));
}

moe_status_t copy_routing(moe_plan_s* p, int T, moe_routing_t* r, cudaStream_t st) {
    const moe_config_t& c = p->cfg;
    const size_t P = static_cast<size_t>(T) * c.top_k;
    cudaError_t e = cudaSuccess;
    if (r->ids && e == cudaSuccess)
        e = cudaMemcpyAsync(r->ids, p->ws.ids, P * 4, cudaMemcpyDeviceToDevice, st);
    if (r->weights && e == cudaSuccess)
        e = cudaMemcpyAsync(r->weights, p->ws.wts, P * 4, cudaMemcpyDeviceToDevice, st);
    if (r->counts && e == cudaSuccess)
        e = cudaMemcpyAsync(r->counts, p->ws.counts, c.n_experts * 4, cudaMemcpyDeviceToDevice, st);
    if (r->offsets && e == cudaSuccess)
        e = cudaMemcpyAsync(r->offsets, p->ws.offsets, (c.n_experts + 1) * 4,
                            cudaMemcpyDeviceToDevice, st);
    if (r->slot_pair && e == cudaSuccess)
        e = cudaMemcpyAsync(r->slot_pair, p->ws.slot_pair, P * 4, cudaMemcpyDeviceToDevice, st);
    return cuda_status(e);
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported request";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_OOM: return "out of device memory";
        case MOE_ERR_DEVICE_FLAG: return "device kernel flagged an inconsistent state";
        case MOE_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

moe_status_t moe_plan_create(const moe_config_t* cfg, moe_plan_t* out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    moe_status_t s = check_config(cfg);
    if (s) return s;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || cfg->device >= ndev) return MOE_ERR_CUDA;
    DeviceGuard dg(cfg->device);
    if (!dg.ok) return MOE_ERR_CUDA;
    int major = 0, minor = 0, sms = 0, optin = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, cfg->device) ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, cfg->device) ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, cfg->device) ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, cfg->device))
        return MOE_ERR_CUDA;
    if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED;

    moe_plan_s* p = new (std::nothrow) moe_plan_s();
    if (!p) return MOE_ERR_OOM;
    p->cfg = *cfg;
    p->num_sms = sms;
    p->smem_optin = static_cast<size_t>(optin);
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
        delete p;
        return MOE_ERR_CUDA;
    }
    p->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    int epc = 1;
    while (epc < 8 && (cfg->n_experts + epc - 1) / epc > sms) epc *= 2;
    p->route_epc = epc;
    int coop = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, cfg->device) != cudaSuccess)
        coop = 0;
    p->coop = coop != 0;

    // workspace: one allocation, carved into 256-byte aligned pieces
    const int64_t T = cfg->t_max, E = cfg->n_experts, k = cfg->top_k, d = cfg->d_model;
    const int64_t S = cfg->n_shared, Fs = cfg->d_ff_shared, F = cfg->d_ff;
    const bool prefill = !wfmt_quantised(cfg->wfmt) &&
                         (cfg->regime == MOE_REGIME_PREFILL ||
                          (cfg->regime == MOE_REGIME_AUTO && cfg->t_max > MOE_DECODE_MAX_T));
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~size_t(255); return o; };
    const size_t o_logits = take(T * E * 4), o_ids = take(T * k * 4), o_wts = take(T * k * 4);
    const size_t o_counts = take(E * 4), o_offsets = take((E + 1) * 4);
    const size_t o_sp = take(T * k * 4), o_st = take(T * k * 4), o_sw = take(T * k * 4);
    const size_t o_items = take((E + S) * sizeof(WorkItem)), o_nitems = take(16);
    const size_t o_ticket = take(16), o_err = take(16), o_gbar = take(16);
    const size_t o_tl = take(static_cast<size_t>(kDecodeTok) * E * 8);
    size_t o_xp = 0, o_hr = 0, o_hs = 0, o_tiles = 0, o_nt = 0;
    if (prefill) {
        o_xp = take(T * k * d * 2);
        o_hr = take(T * k * F * 2);
        o_hs = take(T * S * Fs * 2);
        o_tiles = take(prefill_tile_capacity(cfg) * sizeof(int32_t));
        o_nt = take(64);
    }
    p->ws_bytes = off;
    if (cudaMalloc(&p->ws_base, off) != cudaSuccess) {
        cudaGetLastError();
        delete p;
        return MOE_ERR_OOM;
    }
    uint8_t* b = static_cast<uint8_t*>(p->ws_base);
    Workspace& w = p->ws;
    w.logits = reinterpret_cast<float*>(b + o_logits);
    w.ids = reinterpret_cast<int32_t*>(b + o_ids);
    w.wts = reinterpret_cast<float*>(b + o_wts);
    w.counts = reinterpret_cast<int32_t*>(b + o_counts);
    w.offsets = reinterpret_cast<int32_t*>(b + o_offsets);
    w.slot_pair = reinterpret_cast<int32_t*>(b + o_sp);
    w.slot_token = reinterpret_cast<int32_t*>(b + o_st);
    w.slot_w = reinterpret_cast<float*>(b + o_sw);
    w.items = reinterpret_cast<WorkItem*>(b + o_items);
    w.n_items = reinterpret_cast<int32_t*>(b + o_nitems);
    w.ticket = reinterpret_cast<uint32_t*>(b + o_ticket);
    w.err = reinterpret_cast<uint32_t*>(b + o_err);
    w.gbar = reinterpret_cast<uint32_t*>(b + o_gbar);
    w.tlogits = reinterpret_cast<unsigned long long*>(b + o_tl);
    if (prefill) {
        w.x_perm = reinterpret_cast<uint16_t*>(b + o_xp);
        w.h_routed = reinterpret_cast<uint16_t*>(b + o_hr);
        w.h_shared = reinterpret_cast<uint16_t*>(b + o_hs);
        w.tiles = reinterpret_cast<int32_t*>(b + o_tiles);
        w.n_tiles = reinterpret_cast<int32_t*>(b + o_nt);
    }
    if (cudaMemset(p->ws_base, 0, off) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(p->ws_base);
        delete p;
        return MOE_ERR_CUDA;
    }
    if (prefill) {
        p->pf = prefill_state_create(p->cfg);
        if (!p->pf) {
            cudaFree(p->ws_base);
            delete p;
            return MOE_ERR_OOM;
        }
    }
    *out = p;
    return MOE_OK;
}

void moe_plan_destroy(moe_plan_t p) {
    if (!p) return;
    DeviceGuard dg(p->cfg.device);
    if (p->pf) prefill_state_destroy(p->pf);
    if (p->ws_base) cudaFree(p->ws_base);
    delete p;
}

moe_status_t moe_route(moe_plan_t p, const moe_weights_t* w, const void* x, int32_t T,
                       int32_t top_k, int32_t wfmt, float* out, void* stream) {
    moe_status_t s = check_call(p, w, x, T, top_k, wfmt, out);
    if (s) return s;
    p->last_launches = 0;
    if (T == 0) return MOE_OK;
    DeviceGuard dg(p->cfg.device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (use_decode(p, T)) {
        s = route_decode(p, w, x, T, out, st);
        if (!s) p->last_launches = 1;
        return s;
    }
    int launches = 0;
    s = prefill_route(p->pf, p->cfg, p->ws, w, static_cast<const uint16_t*>(x), T, out, st,
                      p->num_sms, &launches);
    p->last_launches = launches;
    return s;
}

moe_status_t moe_experts(moe_plan_t p, const moe_weights_t* w, const void* x, int32_t T,
                         int32_t top_k, int32_t wfmt, float* out, void* stream) {
    moe_status_t s = check_call(p, w, x, T, top_k, wfmt, out);
    if (s) return s;
    p->last_launches = 0;
    if (T == 0) return MOE_OK;
    DeviceGuard dg(p->cfg.device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (use_decode(p, T)) {
        s = experts_decode(p, w, x, T, out, st);
        if (!s) p->last_launches = 1;
        return s;
    }
    int launches = 0;
    s = prefill_experts(p->pf, p->cfg, p->ws, w, static_cast<const uint16_t*>(x), T, out, st,
                        p->num_sms, &launches);
    p->last_launches = launches;
    return s;
}

moe_status_t moe_forward(moe_plan_t p, const moe_weights_t* w, const void* x, int32_t T,
                         int32_t top_k, int32_t wfmt, float* out, moe_routing_t* routing,
                         void* stream) {
    moe_status_t s = check_call(p, w, x, T, top_k, wfmt, out);
    if (s) return s;
    p->last_launches = 0;
    if (T == 0) return MOE_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (use_decode(p, T) && p->coop) {
        DeviceGuard dg(p->cfg.device);
        s = forward_decode_fused(p, w, x, T, out, st);
        if (s == MOE_OK) {
            p->last_launches = 1;
            if (routing) s = copy_routing(p, T, routing, st);
            return s;
        }
        if (s != MOE_ERR_UNSUPPORTED) return s;
        // fall through to the two-launch path (same kernels, separate router)
    }
    s = moe_route(p, w, x, T, top_k, wfmt, out, stream);
    if (s) return s;
    const int l1 = p->last_launches;
    s = moe_experts(p, w, x, T, top_k, wfmt, out, stream);
    if (s) return s;
    p->last_launches += l1;
    if (routing) {
        DeviceGuard dg(p->cfg.device);
        s = copy_routing(p, T, routing, st);
    }
    return s;
}

moe_status_t moe_routing_get(moe_plan_t p, int32_t T, moe_routing_t* routing, void* stream) {
    if (!p || !routing || T < 0 || T > p->cfg.t_max) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    DeviceGuard dg(p->cfg.device);
    return copy_routing(p, T, routing, static_cast<cudaStream_t>(stream));
}

int32_t moe_last_launch_count(moe_plan_t p) { return p ? p->last_launches : -1; }

moe_status_t moe_get_device_status(moe_plan_t p) {
    if (!p) return MOE_ERR_INVALID_ARG;
    DeviceGuard dg(p->cfg.device);
    uint32_t v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(&v, p->ws.err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (v && cudaMemset(p->ws.err, 0, 4) != cudaSuccess) return MOE_ERR_CUDA;
    if (v & (kErrTimeout | kErrSkipped)) {
        // a launch gave up waiting (or skipped its work because of an earlier
        // timeout): leave the launch ticket count and the tagged logit words
        // clean for the next one
        if (cudaMemset(p->ws.gbar, 0, 16) != cudaSuccess ||
            cudaMemset(p->ws.tlogits, 0, static_cast<size_t>(kDecodeTok) * p->cfg.n_experts * 8) !=
                cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_ERR_TIMEOUT;
    }
    if (v) return MOE_ERR_DEVICE_FLAG;
    return MOE_OK;
}

moe_status_t moe_debug_stall_barrier(moe_plan_t p, void* stream) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!p->coop) return MOE_ERR_UNSUPPORTED;
    DeviceGuard dg(p->cfg.device);
    // a ticket count of 1 (not a multiple of the grid): the next launch's
    // CTAs draw tickets 1..G, from which the one holding ticket G derives the
    // tag 2G and the others G; its wait for logits tagged 2G (and, when it
    // publishes logits, the others' wait for logits tagged G) runs out
    cudaError_t e = cudaMemsetAsync(p->ws.gbar, 0, 16, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess)
        e = cudaMemsetAsync(p->ws.tlogits, 0, static_cast<size_t>(kDecodeTok) * p->cfg.n_experts * 8,
                            static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaMemsetAsync(p->ws.gbar, 0x01, 1, static_cast<cudaStream_t>(stream));
    return cuda_status(e);
}

moe_status_t moe_q6_k_packed_bytes(int64_t n_mats, int64_t rows, int64_t k, size_t* code_bytes,
                                   size_t* scale_bytes) {
    if (n_mats < 0 || rows < 0 || rows % 16 != 0 || k < 0 || k % 256 != 0) return MOE_ERR_INVALID_ARG;
    const int64_t blocks = n_mats * rows * (k / 32);
    if (code_bytes) *code_bytes = static_cast<size_t>(blocks) * 16;
    if (scale_bytes)
        *scale_bytes = static_cast<size_t>(blocks / 16) * 160 + static_cast<size_t>(blocks / 8) * 2;
    return MOE_OK;
}

moe_status_t moe_q6_k_pack(const void* blocks, int64_t n_mats, int64_t rows, int64_t k,
                           void* codes, void* scales, void* stream) {
    if (n_mats < 0 || rows < 0 || rows % 16 != 0 || k < 0 || k % 256 != 0) return MOE_ERR_INVALID_ARG;
    if (n_mats * rows * k == 0) return MOE_OK;
    if (!blocks || !codes || !scales || !aligned16(codes) || !aligned16(scales))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_q6_k_pack(static_cast<const uint8_t*>(blocks), n_mats, rows, k,
                                        static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                                        static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_bf16_to_f16(const void* src, int64_t n, void* dst, void* stream) {
    if (n < 0) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    if (!src || !dst || (reinterpret_cast<uintptr_t>(src) & 1u) || (reinterpret_cast<uintptr_t>(dst) & 1u))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_bf16_to_f16(static_cast<const uint16_t*>(src), n,
                                          static_cast<uint16_t*>(dst),
                                          static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_q4_0_packed_bytes(int64_t n_mats, int64_t rows, int64_t k, size_t* code_bytes,
                                   size_t* scale_bytes) {
    if (n_mats < 0 || rows < 0 || k < 0 || k % 32 != 0) return MOE_ERR_INVALID_ARG;
    const int64_t blocks = n_mats * rows * (k / 32);
    if (code_bytes) *code_bytes = static_cast<size_t>(blocks) * 16;
    if (scale_bytes) *scale_bytes = static_cast<size_t>(blocks) * 2;
    return MOE_OK;
}

moe_status_t moe_q4_0_pack(const void* blocks, int64_t n_mats, int64_t rows, int64_t k,
                           void* codes, void* scales, void* stream) {
    if (n_mats < 0 || rows < 0 || k < 0 || k % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (n_mats * rows * k == 0) return MOE_OK;
    if (!blocks || !codes || !scales || !aligned16(codes) || !aligned16(scales))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_q4_0_pack(static_cast<const uint8_t*>(blocks), n_mats, rows, k,
                                        static_cast<uint8_t*>(codes),
                                        static_cast<uint16_t*>(scales),
                                        static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_q8_0_packed_bytes(int64_t n_mats, int64_t rows, int64_t k, size_t* code_bytes,
                                   size_t* scale_bytes) {
    if (n_mats < 0 || rows < 0 || k < 0 || k % 32 != 0) return MOE_ERR_INVALID_ARG;
    const int64_t blocks = n_mats * rows * (k / 32);
    if (code_bytes) *code_bytes = static_cast<size_t>(blocks) * 32;
    if (scale_bytes) *scale_bytes = static_cast<size_t>(blocks) * 2;
    return MOE_OK;
}

moe_status_t moe_q8_0_pack(const void* blocks, int64_t n_mats, int64_t rows, int64_t k,
                           void* codes, void* scales, void* stream) {
    if (n_mats < 0 || rows < 0 || k < 0 || k % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (n_mats * rows * k == 0) return MOE_OK;
    if (!blocks || !codes || !scales || !aligned16(codes) || !aligned16(scales))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_q8_0_pack(static_cast<const uint8_t*>(blocks), n_mats, rows, k,
                                        static_cast<uint8_t*>(codes),
                                        static_cast<uint16_t*>(scales),
                                        static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_q5_0_packed_bytes(int64_t n_mats, int64_t rows, int64_t k, size_t* code_bytes,
                                   size_t* scale_bytes) {
    if (n_mats < 0 || rows < 0 || rows % 8 != 0 || k < 0 || k % 32 != 0) return MOE_ERR_INVALID_ARG;
    const int64_t blocks = n_mats * rows * (k / 32);
    if (code_bytes) *code_bytes = static_cast<size_t>(blocks) * 16;
    if (scale_bytes) *scale_bytes = static_cast<size_t>(blocks) * 6;
    return MOE_OK;
}

moe_status_t moe_q5_0_pack(const void* blocks, int64_t n_mats, int64_t rows, int64_t k,
                           void* codes, void* scales, void* stream) {
    if (n_mats < 0 || rows < 0 || rows % 8 != 0 || k < 0 || k % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (n_mats * rows * k == 0) return MOE_OK;
    if (!blocks || !codes || !scales || !aligned16(codes) || !aligned16(scales))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_q5_0_pack(static_cast<const uint8_t*>(blocks), n_mats, rows, k,
                                        static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
