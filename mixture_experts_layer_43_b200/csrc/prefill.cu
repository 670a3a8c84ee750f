// prefill.cu -- prefill regime (T > MOE_DECODE_MAX_T tokens, bf16 weights).
//
// Four launches per layer call:
//  1. prefill_router_kernel: router logits for 32 tokens per CTA with fp32
//     FMAs, top-k with renormalised weights, the CTA's per-expert histogram,
//     and the zero-fill of its rows of `out`.  The last CTA (ticket) turns
//     the histograms into per-chunk bucket bases, the per-expert counts and
//     exclusive offsets, and the tile tables of the two GEMMs.
//     ("Fused MoE Triton kernel: 5 launches instead of 24" page, fused steps
//     one and two.)
//  2. prefill_scatter_kernel: stable slot of every (token, choice) pair
//     (ascending token inside each expert) and the gather of x rows into
//     expert-contiguous X_perm.
//  3. prefill_gemm_kernel<kGateUp>: grouped GEMM H = SiLU(X_perm Wg^T) *
//     (X_perm Wu^T) over every expert's rows, plus the shared experts over
//     all tokens, on tcgen05 tensor cores (fused step three).
//  4. prefill_gemm_kernel<kDown>: grouped GEMM H Wd^T whose epilogue adds
//     w_slot * row into out[token] (fused step four, weighted aggregation);
//     the shared experts' rows are added with weight 1 ("CUDA: fuse shared
//     experts into MMVQ" page, shared experts always on).
//
// The GEMM kernel is persistent (one CTA per SM): one warp issues TMA loads
// of 128x64 A and 256x64 B tiles (128-byte swizzle) into a 4-stage ring, one
// thread issues tcgen05.mma 128x256x16 into a double-buffered fp32
// accumulator in tensor memory (2 x 256 columns), and four warps drain the
// accumulator with tcgen05.ld while the next tile's MMAs run.
#include <float.h>
#include <math.h>
#include <string.h>

#include <cudaTypedefs.h>

#include "prefill.cuh"

namespace moe {

constexpr int kChunkTok = 32;        // tokens per router / scatter CTA
constexpr int kRouterThreads = 256;
constexpr int kRouterKC = 32;        // d columns per router k-step
constexpr int kRouterEC = 64;        // experts per router pass

struct PrefillRouteArgs {
    const uint16_t* x;
    const float* wr;
    const float* br;
    float* out;
    Workspace ws;
    int32_t* hist;      // [n_chunks][E] counts, then bucket bases (in place)
    int T, d, E, k, S, F, Fs;
};

// ============================================================ router ===
__global__ void __launch_bounds__(kRouterThreads)
prefill_router_kernel(const PrefillRouteArgs a) {
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    const int E = a.E, d = a.d, k = a.k, T = a.T;
    float* s_log = reinterpret_cast<float*>(sm_raw);                   // [32][E]
    float* s_x = s_log + kChunkTok * E;                                 // [KC][32]
    float* s_w = s_x + kRouterKC * kChunkTok;                           // [KC][64]
    int* s_ids = reinterpret_cast<int*>(s_w + kRouterKC * kRouterEC);   // [32*k]
    int* s_hist = s_ids + kChunkTok * kMaxTopK;                         // [E]
    __shared__ uint32_t s_ticket;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * kChunkTok;
    const int nt = min(kChunkTok, T - t0);

    // zero-fill this chunk's rows of out
    {
        float4* o = reinterpret_cast<float4*>(a.out + static_cast<size_t>(t0) * d);
        const int n4 = nt * d / 4;
        for (int i = tid; i < n4; i += kRouterThreads) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int e = tid; e < E; e += kRouterThreads) s_hist[e] = 0;

    // logits[32 tokens][E]: thread (ty, tx) owns tokens 2ty..2ty+1, experts 4tx..4tx+3
    const int ty = tid >> 4, tx = tid & 15;
    for (int e0 = 0; e0 < E; e0 += kRouterEC) {
        const int ne = min(kRouterEC, E - e0);
        float acc[2][4] = {};
        for (int kc = 0; kc < d; kc += kRouterKC) {
            __syncthreads();
            {   // x chunk: 32 tokens x 32 columns, thread loads 4 bf16
                const int t = tid >> 3, c = (tid & 7) * 4;
                float v[4] = {0.f, 0.f, 0.f, 0.f};
                if (t < nt) {
                    const uint2 u = __ldg(reinterpret_cast<const uint2*>(
                        a.x + static_cast<size_t>(t0 + t) * d + kc + c));
                    v[0] = __uint_as_float(u.x << 16);
                    v[1] = __uint_as_float(u.x & 0xffff0000u);
                    v[2] = __uint_as_float(u.y << 16);
                    v[3] = __uint_as_float(u.y & 0xffff0000u);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) s_x[(c + q) * kChunkTok + t] = v[q];
            }
            {   // router chunk: 64 experts x 32 columns, thread loads 8 floats
                const int e = tid >> 2, c = (tid & 3) * 8;
                float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
                if (e < ne) {
                    const float* src = a.wr + static_cast<size_t>(e0 + e) * d + kc + c;
                    w0 = __ldg(reinterpret_cast<const float4*>(src));
                    w1 = __ldg(reinterpret_cast<const float4*>(src + 4));
                }
                const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int q = 0; q < 8; ++q) s_w[(c + q) * kRouterEC + e] = wv[q];
            }
            __syncthreads();
#pragma unroll 8
            for (int kk = 0; kk < kRouterKC; ++kk) {
                const float2 xv = *reinterpret_cast<const float2*>(&s_x[kk * kChunkTok + 2 * ty]);
                const float4 wv = *reinterpret_cast<const float4*>(&s_w[kk * kRouterEC + 4 * tx]);
                acc[0][0] = fmaf(xv.x, wv.x, acc[0][0]);
                acc[0][1] = fmaf(xv.x, wv.y, acc[0][1]);
                acc[0][2] = fmaf(xv.x, wv.z, acc[0][2]);
                acc[0][3] = fmaf(xv.x, wv.w, acc[0][3]);
                acc[1][0] = fmaf(xv.y, wv.x, acc[1][0]);
                acc[1][1] = fmaf(xv.y, wv.y, acc[1][1]);
                acc[1][2] = fmaf(xv.y, wv.z, acc[1][2]);
                acc[1][3] = fmaf(xv.y, wv.w, acc[1][3]);
            }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = 4 * tx + j;
                if (e < ne) {
                    float v = acc[i][j];
                    if (a.br) v += a.br[e0 + e];
                    if (isnan(v)) v = -INFINITY;
                    s_log[(2 * ty + i) * E + e0 + e] = v;
                }
            }
    }
    __syncthreads();

    // top-k per token (warp per token); taken experts are marked NaN
    for (int t = warp; t < nt; t += kRouterThreads / 32) {
        float* lg = s_log + t * E;
        float sel0 = 0.f, selv[kMaxTopK];
        int seli[kMaxTopK];
        for (int j = 0; j < k; ++j) {
            float bv = -INFINITY;
            int be = INT_MAX;
            for (int x = lane; x < E; x += 32) {
                const float v = lg[x];
                if (!isnan(v) && (v > bv || (v == bv && x < be))) { bv = v; be = x; }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oe = __shfl_xor_sync(0xffffffffu, be, off);
                if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
            }
            if (be >= E) { be = 0; if (lane == 0) atomicOr(a.ws.err, kErrBadId); }
            selv[j] = bv;
            seli[j] = be;
            __syncwarp();
            if (lane == 0) lg[be] = NAN;
            __syncwarp();
        }
        sel0 = selv[0];
        float den = 0.f;
        for (int j = 0; j < k; ++j) den += expf(selv[j] - sel0);
        if (lane < k) {
            float wj = 0.f;
            for (int j = 0; j < k; ++j) if (j == lane) wj = expf(selv[j] - sel0) / den;
            if (!(sel0 > -INFINITY)) wj = 1.f / k;
            int ij = 0;
            for (int j = 0; j < k; ++j) if (j == lane) ij = seli[j];
            const size_t p = static_cast<size_t>(t0 + t) * k + lane;
            a.ws.ids[p] = ij;
            a.ws.wts[p] = wj;
            s_ids[t * k + lane] = ij;
            atomicAdd(&s_hist[ij], 1);
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouterThreads)
        a.hist[static_cast<size_t>(blockIdx.x) * E + e] = s_hist[e];

    // ---- last CTA: bucket bases, counts, offsets, tile tables
    __threadfence();
    __syncthreads();
    if (tid == 0) s_ticket = atomicAdd(a.ws.ticket, 1u);
    __syncthreads();
    if (s_ticket != gridDim.x - 1) return;
    __threadfence();

    const int nch = gridDim.x;
    // per expert: totals and, in place, the prefix over earlier chunks
    for (int e = tid; e < E; e += kRouterThreads) {
        int run = 0;
        for (int c = 0; c < nch; ++c) {
            int* h = a.hist + static_cast<size_t>(c) * E + e;
            const int v = __ldcg(h);
            *h = run;
            run += v;
        }
        s_hist[e] = run;        // count of expert e
    }
    __syncthreads();
    // exclusive scan over experts of (count, gemm1 tiles, gemm2 tiles)
    const int nt1 = (a.F + 127) / 128, nt2 = (d + 255) / 256;
    // scratch reuse: s_ids holds 512 ints, s_x 1024, s_w 2048; E <= 256 here
    int* s_off = s_ids;
    int* s_tb1 = reinterpret_cast<int*>(s_x);
    int* s_tb2 = reinterpret_cast<int*>(s_w);
    if (tid == 0) {
        int o = 0, b1 = 0, b2 = 0;
        for (int e = 0; e < E; ++e) {
            const int c = s_hist[e];
            const int mt = (c + 127) / 128;
            s_off[e] = o; s_tb1[e] = b1; s_tb2[e] = b2;
            o += c; b1 += mt * nt1; b2 += mt * nt2;
        }
        s_off[E] = o; s_tb1[E] = b1; s_tb2[E] = b2;
    }
    __syncthreads();
    for (int e = tid; e <= E; e += kRouterThreads) {
        a.ws.offsets[e] = s_off[e];
        a.ws.tiles[e] = s_tb1[e];
        a.ws.tiles[E + 1 + e] = s_tb2[e];
        if (e < E) a.ws.counts[e] = s_hist[e];
    }
    // chunk bases += expert offset
    for (int i = tid; i < nch * E; i += kRouterThreads) a.hist[i] += s_off[i % E];
    if (tid == 0) {
        const int mts = (T + 127) / 128;
        const int nts1 = a.S * ((a.Fs + 127) / 128);
        a.ws.n_tiles[0] = s_tb1[E] + (a.S ? mts * nts1 : 0);
        a.ws.n_tiles[1] = s_tb2[E] + (a.S ? mts * nt2 : 0);
        a.ws.n_tiles[2] = s_tb1[E];
        a.ws.n_tiles[3] = s_tb2[E];
        if (s_off[E] != T * k) atomicOr(a.ws.err, kErrBadId);
        *a.ws.ticket = 0u;
    }
}

// ============================================================ scatter ===
struct ScatterArgs {
    const uint16_t* x;
    Workspace ws;
    const int32_t* hist;   // bucket bases per chunk
    int T, d, E, k;
};

__global__ void __launch_bounds__(256) prefill_scatter_kernel(const ScatterArgs a) {
    __shared__ int s_ids[kChunkTok * kMaxTopK];
    __shared__ int s_slot[kChunkTok * kMaxTopK];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * kChunkTok;
    const int nt = min(kChunkTok, a.T - t0);
    const int k = a.k, np = nt * k;
    const size_t p0 = static_cast<size_t>(t0) * k;
    for (int i = tid; i < np; i += 256) s_ids[i] = a.ws.ids[p0 + i];
    __syncthreads();
    for (int i = tid; i < np; i += 256) {
        const int e = s_ids[i];
        int rank = 0;
        for (int j = 0; j < i; ++j) rank += (s_ids[j] == e);
        const int slot = a.hist[static_cast<size_t>(blockIdx.x) * a.E + e] + rank;
        s_slot[i] = slot;
        a.ws.slot_pair[slot] = static_cast<int>(p0) + i;
        a.ws.slot_token[slot] = t0 + i / k;
        a.ws.slot_w[slot] = a.ws.wts[p0 + i];
    }
    __syncthreads();
    // gather x rows into X_perm (one warp per pair, 16 bytes per lane)
    const int cpr = a.d / 8;
    for (int i = warp; i < np; i += 8) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0 + i / k) * a.d);
        uint4* dst = reinterpret_cast<uint4*>(a.ws.x_perm + static_cast<size_t>(s_slot[i]) * a.d);
        for (int c = lane; c < cpr; c += 32) dst[c] = __ldg(src + c);
    }
}

// =============================================================== GEMM ===
constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kStageA = kBM * kBK * 2;             // 16 KB
constexpr int kStageB = kBN * kBK * 2;             // 32 KB
constexpr int kStageBytes = kStageA + kStageB;     // 48 KB
constexpr int kGemmThreads = 192;                  // producer, MMA, 4 epilogue warps
constexpr int kGateUp = 1, kDown = 2;

struct GemmArgs {
    CUtensorMap tmA_r, tmA_s;       // A: X_perm / x (gate-up), H_r / H_s (down)
    CUtensorMap tmB0_r, tmB1_r;     // gate-up: Wg, Wu; down: Wd (B1 unused)
    CUtensorMap tmB0_s, tmB1_s;     // shared counterparts
    const int32_t* offsets;
    const int32_t* counts;
    const int32_t* tile_base;       // [E+1] routed tile starts of this GEMM
    const int32_t* n_tiles;         // [0] gate-up total, [1] down total, [2],[3] routed ends
    const int32_t* slot_token;
    const float* slot_w;
    uint16_t* h_r;                  // [slots][F]
    uint16_t* h_s;                  // [T][S*Fs]
    float* out;                     // [T][d]
    uint32_t* err;
    int T, d, E, S, F, Fs;
};

struct GemmTile {
    int row0, valid;    // first A row, rows that belong to the group
    int n0;             // first output column (h column / out column)
    int brow;           // first B row in the stacked weight map (gate-up)
    int shared_s;       // shared expert of a gate-up tile (-1 routed)
    bool shared;
    int group;
    int nk;             // k blocks
};

template <int MODE>
__device__ __forceinline__ GemmTile gemm_tile(const GemmArgs& a, const int* s_tb, int routed_end,
                                              int t) {
    GemmTile g{};
    const int mode_nt = MODE == kGateUp ? (a.F + 127) / 128 : (a.d + 255) / 256;
    if (t < routed_end) {
        int lo = 0, hi = a.E;          // largest e with tile_base[e] <= t
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_tb[mid] <= t) lo = mid; else hi = mid;
        }
        const int e = lo;
        const int r = t - s_tb[e];
        const int mt = r / mode_nt, nt = r % mode_nt;
        g.group = e;
        g.shared = false;
        g.row0 = a.offsets[e] + mt * kBM;
        g.valid = min(kBM, a.counts[e] - mt * kBM);
        if (MODE == kGateUp) {
            g.n0 = nt * 128;
            g.brow = e * a.F + nt * 128;
            g.nk = a.d / kBK;
        } else {
            g.n0 = nt * kBN;
            g.brow = e * a.d + nt * kBN;
            g.nk = (a.F + kBK - 1) / kBK;
        }
        g.shared_s = -1;
    } else {
        const int r = t - routed_end;
        g.shared = true;
        g.group = a.E;
        if (MODE == kGateUp) {
            const int nts = a.S * ((a.Fs + 127) / 128);
            const int mt = r / nts, nt = r % nts;
            const int per = (a.Fs + 127) / 128;
            g.shared_s = nt / per;
            g.n0 = (nt % per) * 128;
            g.brow = g.shared_s * a.Fs + g.n0;
            g.row0 = mt * kBM;
            g.valid = min(kBM, a.T - mt * kBM);
            g.nk = a.d / kBK;
        } else {
            const int nts = (a.d + 255) / 256;
            const int mt = r / nts, nt = r % nts;
            g.shared_s = -1;
            g.n0 = nt * kBN;
            g.brow = nt * kBN;
            g.row0 = mt * kBM;
            g.valid = min(kBM, a.T - mt * kBM);
            g.nk = a.S * (a.Fs / kBK);
        }
    }
    return g;
}

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
prefill_gemm_kernel(const __grid_constant__ GemmArgs a) {
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(tempty + 2);
    int* s_abort = reinterpret_cast<int*>(s_tmem + 1);
    int* s_tb = s_abort + 1;                     // [E+1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 4); }
        *s_abort = 0;
        fence_mbar_init();
    }
    for (int e = tid; e <= a.E; e += kGemmThreads) s_tb[e] = a.tile_base[e];
    if (warp == 1) tmem_alloc(s_tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int n_tiles = a.n_tiles[MODE == kGateUp ? 0 : 1];
    const int routed_end = a.n_tiles[MODE == kGateUp ? 2 : 3];
    volatile int* abort_flag = s_abort;

    auto fail = [&]() { atomicOr(a.err, kErrTimeout); *abort_flag = 1; };

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&a.tmA_r); prefetch_tensormap(&a.tmB0_r);
            if (MODE == kGateUp) prefetch_tensormap(&a.tmB1_r);
            const uint64_t pol = l2_policy_evict_last();
            uint32_t it = 0;
            for (int t = blockIdx.x; t < n_tiles && !*abort_flag; t += gridDim.x) {
                const GemmTile g = gemm_tile<MODE>(a, s_tb, routed_end, t);
                for (int kb = 0; kb < g.nk; ++kb, ++it) {
                    const int s = it % kStages;
                    if (it >= kStages && !mbar_wait_bounded(&empty[s], ((it / kStages) - 1) & 1)) {
                        fail();
                        break;
                    }
                    if (*abort_flag) break;
                    uint8_t* A = ring + s * kStageBytes;
                    uint8_t* Bt = A + kStageA;
                    mbar_arrive_expect_tx(&full[s], kStageBytes);
                    const CUtensorMap* mA = g.shared ? &a.tmA_s : &a.tmA_r;
                    tma_load_2d(A, mA, &full[s], kb * kBK, g.row0, pol);
                    if (MODE == kGateUp) {
                        const CUtensorMap* m0 = g.shared ? &a.tmB0_s : &a.tmB0_r;
                        const CUtensorMap* m1 = g.shared ? &a.tmB1_s : &a.tmB1_r;
                        tma_load_2d(Bt, m0, &full[s], kb * kBK, g.brow, pol);
                        tma_load_2d(Bt + kStageB / 2, m1, &full[s], kb * kBK, g.brow, pol);
                    } else {
                        if (!g.shared) {
                            tma_load_2d(Bt, &a.tmB0_r, &full[s], kb * kBK, g.brow, pol);
                        } else {
                            const int per = a.Fs / kBK;
                            const int ss = kb / per, kk = kb % per;
                            tma_load_2d(Bt, &a.tmB0_s, &full[s], kk * kBK, ss * a.d + g.brow, pol);
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(kBM, kBN);
            uint32_t it = 0;
            int local = 0;
            for (int t = blockIdx.x; t < n_tiles && !*abort_flag; t += gridDim.x, ++local) {
                const GemmTile g = gemm_tile<MODE>(a, s_tb, routed_end, t);
                const int b = local & 1;
                if (local >= 2 && !mbar_wait_bounded(&tempty[b], ((local >> 1) - 1) & 1)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + b * kBN;
                for (int kb = 0; kb < g.nk; ++kb, ++it) {
                    const int s = it % kStages;
                    if (*abort_flag || !mbar_wait_bounded(&full[s], (it / kStages) & 1)) {
                        fail();
                        break;
                    }
                    tc_fence_after();
                    const uint32_t A = smem_u32(ring + s * kStageBytes);
                    const uint32_t Bt = A + kStageA;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_bf16(d_tmem, umma_desc_sw128(A + kk * 32), umma_desc_sw128(Bt + kk * 32),
                                  idesc, (kb | kk) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                umma_commit(&tfull[b]);
            }
        }
    } else {
        // ----------------------------------------------------- epilogue
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int r = q * 32 + lane;                 // tile row of this thread
        int local = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
            // every decision before the warp-collective tcgen05.ld is warp-uniform
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const GemmTile g = gemm_tile<MODE>(a, s_tb, routed_end, t);
            const int b = local & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[b], (local >> 1) & 1));
            if (!ok) {
                if (lane == 0) fail();
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * kBN;
            const bool row_ok = r < g.valid;
            if (MODE == kGateUp) {
                const int Fh = g.shared ? a.Fs : a.F;
                uint16_t* hrow = g.shared
                    ? a.h_s + static_cast<size_t>(g.row0 + r) * (a.S * a.Fs) + g.shared_s * a.Fs + g.n0
                    : a.h_r + static_cast<size_t>(g.row0 + r) * a.F + g.n0;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t gv[32], uv[32];
                    tmem_ld32(taddr + 32 * c, gv);
                    tmem_ld32(taddr + 128 + 32 * c, uv);
                    tmem_ld_wait();
                    if (row_ok && g.n0 + 32 * c < Fh) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float g0 = __uint_as_float(gv[2 * i]), g1 = __uint_as_float(gv[2 * i + 1]);
                            const float u0 = __uint_as_float(uv[2 * i]), u1 = __uint_as_float(uv[2 * i + 1]);
                            pk[i] = pack_bf16x2(g0 / (1.f + __expf(-g0)) * u0,
                                                g1 / (1.f + __expf(-g1)) * u1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(hrow + 32 * c);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            } else {
                int tok = 0;
                float w = 1.f;
                if (row_ok) {
                    if (g.shared) tok = g.row0 + r;
                    else { tok = a.slot_token[g.row0 + r]; w = a.slot_w[g.row0 + r]; }
                }
                float* orow = a.out + static_cast<size_t>(tok) * a.d + g.n0;
#pragma unroll 1
                for (int c = 0; c < kBN / 32; ++c) {
                    uint32_t yv[32];
                    tmem_ld32(taddr + 32 * c, yv);
                    tmem_ld_wait();
                    if (row_ok && g.n0 + 32 * c < a.d) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            red_add_v4_f32(orow + 32 * c + 4 * i, w * __uint_as_float(yv[4 * i]),
                                           w * __uint_as_float(yv[4 * i + 1]),
                                           w * __uint_as_float(yv[4 * i + 2]),
                                           w * __uint_as_float(yv[4 * i + 3]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

size_t gemm_smem_bytes(int E) {
    return 1024 + static_cast<size_t>(kStages) * kStageBytes + (2 * kStages + 4) * 8 + 16 +
           static_cast<size_t>(E + 2) * 4;
}

// ================================================================= host ===
struct PrefillState {
    moe_config_t cfg;
    int32_t* hist = nullptr;          // [max chunks][E]
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    // tensor-map cache (weights + x + workspace pointers)
    bool valid = false;
    moe_weights_t w{};
    const void* x = nullptr;
    int T = 0;
    GemmArgs g1{}, g2{};
};

// int32 entries of the tile tables: routed tile starts of both GEMMs.
size_t prefill_tile_capacity(const moe_config_t* cfg) {
    return 2 * (static_cast<size_t>(cfg->n_experts) + 1);
}

PrefillState* prefill_state_create(const moe_config_t& cfg) {
    PrefillState* s = new PrefillState();
    s->cfg = cfg;
    const size_t nch = (cfg.t_max + kChunkTok - 1) / kChunkTok;
    if (cudaMalloc(&s->hist, nch * cfg.n_experts * sizeof(int32_t)) != cudaSuccess) {
        cudaGetLastError();
        delete s;
        return nullptr;
    }
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
        cudaFree(s->hist);
        delete s;
        return nullptr;
    }
    s->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return s;
}

void prefill_state_destroy(PrefillState* s) {
    if (!s) return;
    if (s->hist) cudaFree(s->hist);
    delete s;
}

static bool map2d(PrefillState* st, CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                  uint64_t ld_elems, uint32_t box_cols, uint32_t box_rows) {
    uint64_t dims[2] = {cols, rows};
    uint64_t strides[1] = {ld_elems * 2};
    uint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    return st->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                      box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

moe_status_t prefill_route(PrefillState* st, const moe_config_t& c, const Workspace& ws,
                           const moe_weights_t* w, const uint16_t* x, int T, float* out,
                           cudaStream_t stream, int num_sms, int* launches) {
    (void)num_sms;
    *launches = 0;
    if (c.n_experts > 256) return MOE_ERR_UNSUPPORTED;
    PrefillRouteArgs r{};
    r.x = x; r.wr = w->router_w; r.br = w->router_b; r.out = out; r.ws = ws; r.hist = st->hist;
    r.T = T; r.d = c.d_model; r.E = c.n_experts; r.k = c.top_k; r.S = c.n_shared;
    r.F = c.d_ff; r.Fs = c.n_shared ? c.d_ff_shared : 0;
    const int nch = (T + kChunkTok - 1) / kChunkTok;
    const size_t smem = (kChunkTok * c.n_experts + kRouterKC * kChunkTok + kRouterKC * kRouterEC) * 4 +
                        (kChunkTok * kMaxTopK + c.n_experts) * 4;
    static int set_smem = 0;
    if (static_cast<int>(smem) > set_smem) {
        if (cudaFuncSetAttribute(prefill_router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        set_smem = static_cast<int>(smem);
    }
    prefill_router_kernel<<<nch, kRouterThreads, smem, stream>>>(r);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    ScatterArgs sa{};
    sa.x = x; sa.ws = ws; sa.hist = st->hist; sa.T = T; sa.d = c.d_model; sa.E = c.n_experts;
    sa.k = c.top_k;
    prefill_scatter_kernel<<<nch, 256, 0, stream>>>(sa);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    *launches = 2;
    return MOE_OK;
}

moe_status_t prefill_experts(PrefillState* st, const moe_config_t& c, const Workspace& ws,
                             const moe_weights_t* w, const uint16_t* x, int T, float* out,
                             cudaStream_t stream, int num_sms, int* launches) {
    *launches = 0;
    const int E = c.n_experts, d = c.d_model, F = c.d_ff, S = c.n_shared;
    const int Fs = S ? c.d_ff_shared : 0;
    if (F % kBK || (S && Fs % kBK)) return MOE_ERR_UNSUPPORTED;
    const uint64_t slots = static_cast<uint64_t>(c.t_max) * c.top_k;
    // x is the caller's [T][d] buffer: its map spans exactly T rows so that
    // the last tile's rows past T are zero-filled by TMA, never read
    if (!st->valid || st->x != x || st->T != T || memcmp(&st->w, w, sizeof(*w)) != 0) {
        bool ok = true;
        GemmArgs& g1 = st->g1;
        GemmArgs& g2 = st->g2;
        memset(&g1, 0, sizeof(g1));
        memset(&g2, 0, sizeof(g2));
        ok &= map2d(st, &g1.tmA_r, ws.x_perm, slots, d, d, kBK, kBM);
        ok &= map2d(st, &g1.tmA_s, x, T, d, d, kBK, kBM);
        ok &= map2d(st, &g1.tmB0_r, w->gate.data, static_cast<uint64_t>(E) * F, d, d, kBK, 128);
        ok &= map2d(st, &g1.tmB1_r, w->up.data, static_cast<uint64_t>(E) * F, d, d, kBK, 128);
        ok &= map2d(st, &g2.tmA_r, ws.h_routed, slots, F, F, kBK, kBM);
        ok &= map2d(st, &g2.tmB0_r, w->down.data, static_cast<uint64_t>(E) * d, F, F, kBK, kBN);
        if (S) {
            ok &= map2d(st, &g1.tmB0_s, w->shared_gate.data, static_cast<uint64_t>(S) * Fs, d, d, kBK, 128);
            ok &= map2d(st, &g1.tmB1_s, w->shared_up.data, static_cast<uint64_t>(S) * Fs, d, d, kBK, 128);
            ok &= map2d(st, &g2.tmA_s, ws.h_shared, c.t_max, static_cast<uint64_t>(S) * Fs,
                        static_cast<uint64_t>(S) * Fs, kBK, kBM);
            ok &= map2d(st, &g2.tmB0_s, w->shared_down.data, static_cast<uint64_t>(S) * d, Fs, Fs, kBK, kBN);
        }
        if (!ok) return MOE_ERR_INVALID_ARG;
        st->valid = true;
        st->x = x;
        st->T = T;
        st->w = *w;
    }
    for (GemmArgs* g : {&st->g1, &st->g2}) {
        g->offsets = ws.offsets;
        g->counts = ws.counts;
        g->n_tiles = ws.n_tiles;
        g->slot_token = ws.slot_token;
        g->slot_w = ws.slot_w;
        g->h_r = ws.h_routed;
        g->h_s = ws.h_shared;
        g->out = out;
        g->err = ws.err;
        g->T = T; g->d = d; g->E = E; g->S = S; g->F = F; g->Fs = Fs;
    }
    st->g1.tile_base = ws.tiles;
    st->g2.tile_base = ws.tiles + E + 1;
    const size_t smem = gemm_smem_bytes(E);
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(prefill_gemm_kernel<kGateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(gemm_smem_bytes(kMaxExperts))) != cudaSuccess ||
            cudaFuncSetAttribute(prefill_gemm_kernel<kDown>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(gemm_smem_bytes(kMaxExperts))) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr = true;
    }
    prefill_gemm_kernel<kGateUp><<<num_sms, kGemmThreads, smem, stream>>>(st->g1);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    prefill_gemm_kernel<kDown><<<num_sms, kGemmThreads, smem, stream>>>(st->g2);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    *launches = 2;
    return MOE_OK;
}

}  // namespace moe
