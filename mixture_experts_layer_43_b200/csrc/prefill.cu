// prefill.cu -- prefill regime (T > MOE_DECODE_MAX_T tokens, bf16 weights).
//
// Four launches per layer call:
//  1. prefill_router_kernel: router logits for 32 tokens per CTA on the
//     tensor cores, as accurate as fp32 FMAs (the fp32 router weights are
//     split exactly into three bf16 parts; x and router chunks stream in by
//     cp.async, two chunks in flight), top-k with renormalised weights, the
//     CTA's per-expert histogram, and the zero-fill of its rows of `out`.
//     ("Fused MoE Triton kernel: 5 launches instead of 24" page, fused steps
//     one and two.)
//  2. prefill_scatter_kernel: every CTA reduces the histograms to its chunk's
//     bucket base per expert (counts, exclusive offsets), gives each
//     (token, choice) pair its stable slot (ascending token inside each
//     expert) and gathers x rows into expert-contiguous X_perm; CTA 0 also
//     writes counts, offsets and the tile tables of the two GEMMs.
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
constexpr int kMaxDevices = 64;      // per-device launch attributes
constexpr int kRouterThreads = 256;
constexpr int kRouterKC = 64;        // d columns per router k-chunk (double-buffered)
constexpr int kRouterEC = 64;        // experts per router pass
constexpr int kRouterPitch = kRouterKC + 8;   // bf16 elements per smem row (conflict-free ldmatrix)

struct PrefillRouteArgs {
    const uint16_t* x;
    const float* wr;
    const float* br;
    float* out;
    Workspace ws;
    int32_t* hist;      // [n_chunks][E] per-chunk expert counts
    int T, d, E, k, S, F, Fs;
};

constexpr int kRouterXTile = kChunkTok * kRouterPitch;          // bf16 elements
constexpr int kRouterWTile = kRouterEC * kRouterPitch;          // bf16 elements, one part
constexpr int kRouterStages = 4;                                // raw chunks in flight
constexpr int kRouterRawW = kRouterEC * kRouterKC;             // fp32 elements of one raw w chunk

size_t router_smem_bytes(int E) {
    return static_cast<size_t>(kChunkTok) * E * 4 +                      // logits
           static_cast<size_t>(kRouterStages) * (kRouterXTile * 2 + kRouterRawW * 4) +  // raw ring
           2ull * 3 * kRouterWTile * 2 +                                  // 3 w parts, x2
           (kChunkTok * kMaxTopK + E) * 4 +                               // ids, histogram
           static_cast<size_t>(kChunkTok) * kMaxTopK * 4;                 // selected logits
}

// 16-byte asynchronous global -> shared copy (L2 only); src_bytes < 16
// zero-fills the rest of the destination (0: a row past the end).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory");
}

// ============================================================ router ===
// Logits of 32 tokens x 64 experts per pass on the tensor cores, exactly as
// accurate as fp32 arithmetic on the products: each fp32 router weight w is
// split into three bf16 parts hi + mid + lo that sum to w exactly (each part
// holds the next 8 significant bits), so every x*part product (bf16 x) is
// exact in fp32 and mma.sync accumulates the three partial logits in fp32.
// (TF32 would instead round w to 10 bits.)  64-column chunks of x and of the
// fp32 router arrive by cp.async in a ring of four (two chunks in flight
// while one is split and used); each chunk is split into the double-buffered
// bf16 tiles the mma's read.
// Warp w handles tokens 16*(w/4).. and experts 16*(w%4)..  of the pass.
__global__ void __launch_bounds__(kRouterThreads)
prefill_router_kernel(const PrefillRouteArgs a) {
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    const int E = a.E, d = a.d, k = a.k, T = a.T;
    float* s_log = reinterpret_cast<float*>(sm_raw);                   // [32][E]
    // raw ring: x chunk [32][pitch] bf16 (read by ldmatrix as is), w chunk [64][64] fp32
    __nv_bfloat16* s_xr = reinterpret_cast<__nv_bfloat16*>(s_log + kChunkTok * E);
    float* s_wr = reinterpret_cast<float*>(s_xr + kRouterStages * kRouterXTile);
    __nv_bfloat16* s_w = reinterpret_cast<__nv_bfloat16*>(s_wr + kRouterStages * kRouterRawW);  // [2][3][64][pitch]
    int* s_ids = reinterpret_cast<int*>(s_w + 2 * 3 * kRouterWTile);    // [32*k]
    int* s_hist = s_ids + kChunkTok * kMaxTopK;                         // [E]

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

    const int tg = warp >> 2, eq = warp & 3;
    const int g = lane >> 2, tig = lane & 3;
    const int nkc = d / kRouterKC;
    for (int e0 = 0; e0 < E; e0 += kRouterEC) {
        const int ne = min(kRouterEC, E - e0);
        // chunk kc -> ring stage kc % kRouterStages, by cp.async: x row tid/8,
        // 16 bytes at (tid%8)*16; w: 4 x 16 bytes, row c/16, floats (c%16)*4
        auto issue = [&](int kc) {
            const int st = kc % kRouterStages, kb = kc * kRouterKC;
            {
                const int r = tid >> 3, c8 = (tid & 7) * 8;
                const bool ok = r < nt;
                cp_async_16(smem_u32(s_xr + st * kRouterXTile + r * kRouterPitch + c8),
                            a.x + static_cast<size_t>(t0 + (ok ? r : 0)) * d + kb + c8, ok ? 16 : 0);
            }
#pragma unroll
            for (int q = 0; q < kRouterRawW / 4 / kRouterThreads; ++q) {
                const int c = q * kRouterThreads + tid, r = c >> 4, c4 = (c & 15) * 4;
                const bool ok = r < ne;
                cp_async_16(smem_u32(s_wr + st * kRouterRawW + r * kRouterKC + c4),
                            a.wr + static_cast<size_t>(e0 + (ok ? r : 0)) * d + kb + c4, ok ? 16 : 0);
            }
        };
        // exact split of a raw fp32 chunk into the hi / mid / lo bf16 tiles
        auto split = [&](int kc, int buf) {
            const float* raw = s_wr + (kc % kRouterStages) * kRouterRawW;
            __nv_bfloat16* wb = s_w + buf * 3 * kRouterWTile;
#pragma unroll
            for (int q = 0; q < kRouterRawW / 4 / kRouterThreads; ++q) {
                const int i = (q * kRouterThreads + tid) * 4, r = i / kRouterKC, c = i % kRouterKC;
                const float4 f = *reinterpret_cast<const float4*>(raw + i);
                const float p[4] = {f.x, f.y, f.z, f.w};
                uint32_t hi[2], mid[2], lo[2];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    float p0 = p[2 * h2], p1 = p[2 * h2 + 1];
                    const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                    p0 -= __low2float(h);             // exact: fp32 minus its bf16 rounding
                    p1 -= __high2float(h);
                    const __nv_bfloat162 m = __floats2bfloat162_rn(p0, p1);
                    p0 -= __low2float(m);
                    p1 -= __high2float(m);
                    const __nv_bfloat162 l = __floats2bfloat162_rn(p0, p1);   // exact: <= 8 bits left
                    hi[h2] = *reinterpret_cast<const uint32_t*>(&h);
                    mid[h2] = *reinterpret_cast<const uint32_t*>(&m);
                    lo[h2] = *reinterpret_cast<const uint32_t*>(&l);
                }
                const int o = r * kRouterPitch + c;
                *reinterpret_cast<uint2*>(wb + o) = make_uint2(hi[0], hi[1]);
                *reinterpret_cast<uint2*>(wb + kRouterWTile + o) = make_uint2(mid[0], mid[1]);
                *reinterpret_cast<uint2*>(wb + 2 * kRouterWTile + o) = make_uint2(lo[0], lo[1]);
            }
        };
        float acc[2][4] = {};
        __syncthreads();                           // previous pass done with the ring
#pragma unroll
        for (int kc = 0; kc < kRouterStages - 1; ++kc) {
            if (kc < nkc) issue(kc);
            cp_async_commit();
        }
        for (int kc = 0; kc < nkc; ++kc) {
            cp_async_wait<kRouterStages - 2>();   // this thread's copies of chunk kc landed
            __syncthreads();                       // everyone's; chunk kc-1 fully consumed
            if (kc + kRouterStages - 1 < nkc) issue(kc + kRouterStages - 1);   // into kc-1's stage
            cp_async_commit();
            const int buf = kc & 1;
            split(kc, buf);
            __syncthreads();
            const uint32_t xs = smem_u32(s_xr + (kc % kRouterStages) * kRouterXTile);
            const uint32_t ws = smem_u32(s_w + buf * 3 * kRouterWTile);
#pragma unroll
            for (int kk = 0; kk < kRouterKC / 16; ++kk) {
                uint32_t a0, a1, a2, a3;
                {
                    const int m = lane >> 3, r = lane & 7;
                    const int row = tg * 16 + ((m & 1) << 3) + r;
                    ldsm_x4(xs + (row * kRouterPitch + kk * 16 + (m >> 1) * 8) * 2, a0, a1, a2, a3);
                }
#pragma unroll
                for (int n8 = 0; n8 < 2; ++n8) {
                    const int erow = eq * 16 + n8 * 8 + (lane & 7);
                    const uint32_t boff = (erow * kRouterPitch + kk * 16 + ((lane >> 3) & 1) * 8) * 2;
#pragma unroll
                    for (int part = 0; part < 3; ++part) {
                        uint32_t b0, b1;
                        ldsm_x2(ws + part * kRouterWTile * 2 + boff, b0, b1);
                        mma_bf16_16816(acc[n8], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
        }
        cp_async_wait<0>();
        // C fragment: rows (tokens) g, g+8; columns (experts) 2tig, 2tig+1
#pragma unroll
        for (int n8 = 0; n8 < 2; ++n8)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = tg * 16 + g + (q >> 1) * 8;
                const int e = eq * 16 + n8 * 8 + 2 * tig + (q & 1);
                if (e < ne) {
                    float v = acc[n8][q];
                    if (a.br) v += a.br[e0 + e];
                    if (isnan(v)) v = -INFINITY;
                    s_log[t * E + e0 + e] = v;
                }
            }
        __syncthreads();
    }

    // top-k per token (warp per token, register-resident logits)
    for (int t = warp; t < nt; t += kRouterThreads / 32) {
        int* ids = s_ids + t * k;
        float* sel = reinterpret_cast<float*>(s_hist + E) + t * kMaxTopK;   // [32][16] scratch
        warp_topk_any(s_log + t * E, E, k, ids, sel, a.ws.err);
        __syncwarp();
        if (lane < k) {
            const float m = sel[0];
            float den = 0.f;
            for (int j = 0; j < k; ++j) den += expf(sel[j] - m);
            float wj = expf(sel[lane] - m) / den;
            if (!(m > -INFINITY)) wj = 1.f / k;
            const int ij = ids[lane];
            const size_t p = static_cast<size_t>(t0 + t) * k + lane;
            a.ws.ids[p] = ij;
            a.ws.wts[p] = wj;
            atomicAdd(&s_hist[ij], 1);
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouterThreads)
        a.hist[static_cast<size_t>(blockIdx.x) * E + e] = s_hist[e];

}

// ============================================================ scatter ===
struct ScatterArgs {
    const uint16_t* x;
    Workspace ws;
    const int32_t* hist;   // [n_chunks][E] per-chunk expert counts
    int T, d, E, k, S, F, Fs;
    int bm;                // rows of one GEMM tile (128, or 256 for a CTA pair)
};

constexpr int kScatterThreads = 256;

__global__ void __launch_bounds__(kScatterThreads) prefill_scatter_kernel(const ScatterArgs a) {
    __shared__ int s_ids[kChunkTok * kMaxTopK];
    __shared__ int s_slot[kChunkTok * kMaxTopK];
    __shared__ int s_tot[256], s_pre[256], s_off[257], s_wsum[kScatterThreads / 32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, k = a.k, c0 = blockIdx.x, nch = gridDim.x;
    const int t0 = c0 * kChunkTok;
    const int nt = min(kChunkTok, a.T - t0), np = nt * k;
    const size_t p0 = static_cast<size_t>(t0) * k;

    // per expert: total count and count in the chunks before this one;
    // nseg threads per expert split the chunk range (E <= 256)
    for (int e = tid; e < E; e += kScatterThreads) { s_tot[e] = 0; s_pre[e] = 0; }
    for (int i = tid; i < np; i += kScatterThreads) s_ids[i] = a.ws.ids[p0 + i];
    __syncthreads();
    {
        const int nseg = max(1, kScatterThreads / E);
        const int e = tid % E, seg = tid / E;
        if (seg < nseg && tid < nseg * E) {
            const int per = (nch + nseg - 1) / nseg;
            const int c_lo = seg * per, c_hi = min(nch, c_lo + per);
            int tot = 0, pre = 0;
#pragma unroll 8
            for (int c = c_lo; c < c_hi; ++c) {
                const int v = __ldg(a.hist + static_cast<size_t>(c) * E + e);
                tot += v;
                pre += (c < c0) ? v : 0;
            }
            atomicAdd(&s_tot[e], tot);
            atomicAdd(&s_pre[e], pre);
        }
    }
    __syncthreads();
    // exclusive scan of the totals over experts (one expert per thread)
    {
        const int v = tid < E ? s_tot[tid] : 0;
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += u;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; ++w) base += s_wsum[w];
        if (tid < E) s_off[tid] = base + incl - v;
        if (tid == kScatterThreads - 1) s_off[E] = base + incl;
    }
    __syncthreads();
    if (c0 == 0) {
        // counts, offsets and the GEMM tile tables (tile starts per expert)
        const int nt1 = (a.F + 127) / 128, nt2 = (a.d + 255) / 256;
        if (tid == 0) {
            int b1 = 0, b2 = 0;
            for (int e = 0; e < E; ++e) {
                const int mt = (s_tot[e] + a.bm - 1) / a.bm;
                a.ws.tiles[e] = b1;
                a.ws.tiles[E + 1 + e] = b2;
                b1 += mt * nt1;
                b2 += mt * nt2;
            }
            a.ws.tiles[E] = b1;
            a.ws.tiles[2 * E + 1] = b2;
            const int mts = (a.T + a.bm - 1) / a.bm;
            const int nts1 = a.S * ((a.Fs + 127) / 128);
            a.ws.n_tiles[0] = b1 + (a.S ? mts * nts1 : 0);
            a.ws.n_tiles[1] = b2 + (a.S ? mts * nt2 : 0);
            a.ws.n_tiles[2] = b1;
            a.ws.n_tiles[3] = b2;
            if (s_off[E] != a.T * k) atomicOr(a.ws.err, kErrBadId);
        }
        for (int e = tid; e <= E; e += kScatterThreads) {
            a.ws.offsets[e] = s_off[e];
            if (e < E) a.ws.counts[e] = s_tot[e];
        }
    }
    // stable slots: rank among the chunk's earlier pairs with the same expert
    for (int i = tid; i < np; i += kScatterThreads) {
        const int e = s_ids[i];
        int rank = 0;
        for (int j = 0; j < i; ++j) rank += (s_ids[j] == e);
        const int slot = s_off[e] + s_pre[e] + rank;
        s_slot[i] = slot;
        a.ws.slot_pair[slot] = static_cast<int>(p0) + i;
        a.ws.slot_token[slot] = t0 + i / k;
        a.ws.slot_w[slot] = a.ws.wts[p0 + i];
    }
    __syncthreads();
    // gather x rows into X_perm: a warp copies kGatherRows pairs' rows at a
    // time, 16 bytes per lane, every load of the group issued before its
    // stores (one round trip per group of rows, not per row)
    constexpr int kGatherRows = 4;
    constexpr int kWarps = kScatterThreads / 32;
    const int cpr = a.d / 8;
    for (int i0 = warp; i0 < np; i0 += kWarps * kGatherRows) {
        for (int cb = lane; cb < cpr; cb += 32 * 8) {
            uint4 v[kGatherRows][8];
#pragma unroll
            for (int p = 0; p < kGatherRows; ++p) {
                const int i = i0 + kWarps * p;
                if (i < np) {
                    const uint4* src =
                        reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0 + i / k) * a.d);
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (cb + 32 * u < cpr) v[p][u] = __ldg(src + cb + 32 * u);
                }
            }
#pragma unroll
            for (int p = 0; p < kGatherRows; ++p) {
                const int i = i0 + kWarps * p;
                if (i < np) {
                    uint4* dst = reinterpret_cast<uint4*>(a.ws.x_perm + static_cast<size_t>(s_slot[i]) * a.d);
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (cb + 32 * u < cpr) dst[cb + 32 * u] = v[p][u];
                }
            }
        }
    }
}

// =============================================================== GEMM ===
constexpr int kBM = 128, kBN = 256, kBK = 64;      // rows of A per CTA, tile columns, k-step
constexpr int kStageA = kBM * kBK * 2;             // 16 KB
constexpr int kGemmThreads = 192;                  // producer, MMA, 4 epilogue warps

// CG = 1: one CTA computes a 128 x 256 tile (A 128 rows, B 256 rows per
// stage).  CG = 2: a CTA pair computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2; each CTA holds its own 128 rows of A and half
// (128 rows) of B, so a stage is 32 KB instead of 48 KB for the same math
// per SM, and six stages fit instead of four.
template <int CG>
struct GemmCfg {
    static constexpr int BM = kBM * CG;                      // tile rows
    static constexpr int BROWS = kBN / CG;                   // B rows one CTA loads
    static constexpr int STAGE_B = BROWS * kBK * 2;
    static constexpr int STAGE = kStageA + STAGE_B;
    static constexpr int STAGES = CG == 1 ? 4 : 6;
};

// ---- CTA-pair (cluster of 2) primitives
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
                 :: "r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// TMA tile load into this CTA's shared memory whose transaction bytes
// complete on the mbarrier at `mbar` (shared::cluster address: the pair's
// first CTA).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t mbar,
                                                 int32_t c0, int32_t c1, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;"
        :: "r"(smem_u32(dst)), "l"(map), "r"(mbar), "r"(c0), "r"(c1), "l"(policy) : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n"
        " setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Arrive on `bar` (same offset) in both CTAs of the pair once every MMA this
// thread issued so far completes.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)), "h"(static_cast<uint16_t>(3)) : "memory");
}
constexpr int kGateUp = 1, kDown = 2;
constexpr int kEpiStage = 4 * 32 * 32 * 4;          // down epilogue staging, 4 KB per warp

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
    int f16;                        // h and the down matrices fp16 (else bf16)
};

struct GemmTile {
    int row0, valid;    // first A row, rows that belong to the group
    int n0;             // first output column (h column / out column)
    int brow;           // first B row in the stacked weight map (gate-up)
    int shared_s;       // shared expert of a gate-up tile (-1 routed)
    bool shared;
    int group;
    int nk;             // k blocks
    int nsw;            // > 0: a swapped tail tile with this many token columns (see below)
};

// An expert's last row tile holds `valid` < 128 rows; as a 128-row MMA tile
// the rest would be padding.  Such a tail tile (single-CTA GEMMs, routed
// experts) swaps the operands instead: the weight rows already in the stage
// become the 128-row A side and the tile's X_perm / h rows the N side,
// rounded up to 16 -- two MMAs per k step (gate and up rows, or the two
// 128-row halves of the down tile) into TMEM columns [0, N) and [128, 128 +
// N).  The loads are the same as for a normal tile.  Tails that round up to
// more than kSwapMaxN columns stay normal tiles.
constexpr int kSwapMaxN = 112;

// Tile t of the expert-major tile table (BM rows of the whole tile).
template <int MODE, int BM>
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
        g.row0 = a.offsets[e] + mt * BM;
        g.valid = min(BM, a.counts[e] - mt * BM);
        if constexpr (BM == kBM) {
            const int n16 = (g.valid + 15) & ~15;
            if (n16 <= kSwapMaxN) g.nsw = n16;
        }
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
            g.row0 = mt * BM;
            g.valid = min(BM, a.T - mt * BM);
            g.nk = a.d / kBK;
        } else {
            const int nts = (a.d + 255) / 256;
            const int mt = r / nts, nt = r % nts;
            g.shared_s = -1;
            g.n0 = nt * kBN;
            g.brow = nt * kBN;
            g.row0 = mt * BM;
            g.valid = min(BM, a.T - mt * BM);
            g.nk = a.S * (a.Fs / kBK);
        }
    }
    return g;
}

template <int MODE, int CG>
__global__ void __launch_bounds__(kGemmThreads, 1)
prefill_gemm_kernel(const __grid_constant__ GemmArgs a) {
    using C = GemmCfg<CG>;
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float* stage_out = reinterpret_cast<float*>(ring + C::STAGES * C::STAGE);   // 4 x [32][32]
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + C::STAGES * C::STAGE + kEpiStage);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(tempty + 2);
    int* s_abort = reinterpret_cast<int*>(s_tmem + 1);
    int* s_tb = s_abort + 1;                     // [E+1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CG = 2: rank 0 of the pair issues the MMAs and owns full[] and tempty[]
    const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
    const int unit = static_cast<int>(blockIdx.x) / CG, n_units = static_cast<int>(gridDim.x) / CG;
    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 4 * CG); }
        *s_abort = 0;
        fence_mbar_init();
    }
    for (int e = tid; e <= a.E; e += kGemmThreads) s_tb[e] = a.tile_base[e];
    if (warp == 1) {
        if constexpr (CG == 2) tmem_alloc_pair(s_tmem, 512);
        else tmem_alloc(s_tmem, 512);
    }
    tc_fence_before();
    if constexpr (CG == 2) cluster_sync_all();   // peer barriers initialised before any signal
    else __syncthreads();
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
            bool ok = true;
            for (int t = unit; t < n_tiles && ok && !*abort_flag; t += n_units) {
                const GemmTile g = gemm_tile<MODE, C::BM>(a, s_tb, routed_end, t);
                const int arow = g.row0 + kBM * static_cast<int>(rank);
                for (int kb = 0; kb < g.nk; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    if (it >= static_cast<uint32_t>(C::STAGES) &&
                        !mbar_wait_bounded(&empty[s], ((it / C::STAGES) - 1) & 1)) {
                        fail();
                        ok = false;
                        break;
                    }
                    if (*abort_flag) { ok = false; break; }
                    uint8_t* A = ring + s * C::STAGE;
                    uint8_t* Bt = A + kStageA;
                    const CUtensorMap* mA = g.shared ? &a.tmA_s : &a.tmA_r;
                    if constexpr (CG == 1) {
                        mbar_arrive_expect_tx(&full[s], C::STAGE);
                        tma_load_2d(A, mA, &full[s], kb * kBK, arow, pol);
                        if (MODE == kGateUp) {
                            const CUtensorMap* m0 = g.shared ? &a.tmB0_s : &a.tmB0_r;
                            const CUtensorMap* m1 = g.shared ? &a.tmB1_s : &a.tmB1_r;
                            tma_load_2d(Bt, m0, &full[s], kb * kBK, g.brow, pol);
                            tma_load_2d(Bt + C::STAGE_B / 2, m1, &full[s], kb * kBK, g.brow, pol);
                        } else if (!g.shared) {
                            tma_load_2d(Bt, &a.tmB0_r, &full[s], kb * kBK, g.brow, pol);
                        } else {
                            const int per = a.Fs / kBK;
                            const int ss = kb / per, kk = kb % per;
                            tma_load_2d(Bt, &a.tmB0_s, &full[s], kk * kBK, ss * a.d + g.brow, pol);
                        }
                    } else {
                        // both halves of the pair complete on rank 0's full[s]
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE);
                        const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
                        tma_load_2d_pair(A, mA, fb, kb * kBK, arow, pol);
                        if (MODE == kGateUp) {        // rank 0: gate rows, rank 1: up rows
                            const CUtensorMap* mb = rank == 0 ? (g.shared ? &a.tmB0_s : &a.tmB0_r)
                                                              : (g.shared ? &a.tmB1_s : &a.tmB1_r);
                            tma_load_2d_pair(Bt, mb, fb, kb * kBK, g.brow, pol);
                        } else if (!g.shared) {
                            tma_load_2d_pair(Bt, &a.tmB0_r, fb, kb * kBK, g.brow + C::BROWS * rank, pol);
                        } else {
                            const int per = a.Fs / kBK;
                            const int ss = kb / per, kk = kb % per;
                            tma_load_2d_pair(Bt, &a.tmB0_s, fb, kk * kBK,
                                             ss * a.d + g.brow + C::BROWS * rank, pol);
                        }
                    }
                }
            }
            // drain: every issued stage released by the MMAs, so no commit
            // arrives in this CTA's shared memory after it exits
            const uint32_t first = it > static_cast<uint32_t>(C::STAGES) ? it - C::STAGES : 0u;
            for (uint32_t q = first; q < it && ok; ++q)
                if (!mbar_wait_bounded(&empty[q % C::STAGES], (q / C::STAGES) & 1)) {
                    fail();
                    break;
                }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA
        if (lane == 0 && rank == 0) {
            // operand types: bf16, except fp16 h and down matrices in the down GEMM
            const uint32_t idesc = (MODE == kDown && a.f16) ? umma_idesc_f16(C::BM, kBN)
                                                            : umma_idesc_bf16(C::BM, kBN);
            uint32_t it = 0;
            int local = 0;
            for (int t = unit; t < n_tiles && !*abort_flag; t += n_units, ++local) {
                const GemmTile g = gemm_tile<MODE, C::BM>(a, s_tb, routed_end, t);
                const int b = local & 1;
                if (local >= 2 && !mbar_wait_bounded(&tempty[b], ((local >> 1) - 1) & 1)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + b * kBN;
                bool ok = true;
                for (int kb = 0; kb < g.nk; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    if (*abort_flag || !mbar_wait_bounded(&full[s], (it / C::STAGES) & 1)) {
                        fail();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t A = smem_u32(ring + s * C::STAGE);
                    const uint32_t Bt = A + kStageA;
                    if constexpr (CG == 1) {
                        if (g.nsw > 0) {
                            // swapped tail tile: weight rows x token rows
                            const uint32_t idesc_sw = (MODE == kDown && a.f16)
                                                          ? umma_idesc_f16(kBM, g.nsw)
                                                          : umma_idesc_bf16(kBM, g.nsw);
#pragma unroll
                            for (int kk = 0; kk < kBK / 16; ++kk) {
                                const uint32_t acc = (kb | kk) ? 1u : 0u;
                                umma_bf16(d_tmem, umma_desc_sw128(Bt + kk * 32),
                                          umma_desc_sw128(A + kk * 32), idesc_sw, acc);
                                umma_bf16(d_tmem + 128, umma_desc_sw128(Bt + C::STAGE_B / 2 + kk * 32),
                                          umma_desc_sw128(A + kk * 32), idesc_sw, acc);
                            }
                            umma_commit(&empty[s]);
                            continue;
                        }
                    }
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        if constexpr (CG == 2)
                            umma_bf16_pair(d_tmem, umma_desc_sw128(A + kk * 32),
                                           umma_desc_sw128(Bt + kk * 32), idesc, (kb | kk) ? 1u : 0u);
                        else
                            umma_bf16(d_tmem, umma_desc_sw128(A + kk * 32), umma_desc_sw128(Bt + kk * 32),
                                      idesc, (kb | kk) ? 1u : 0u);
                    }
                    if constexpr (CG == 2) umma_commit_pair(&empty[s]);
                    else umma_commit(&empty[s]);
                }
                if (!ok) break;
                if constexpr (CG == 2) umma_commit_pair(&tfull[b]);
                else umma_commit(&tfull[b]);
            }
        }
    } else {
        // ----------------------------------------------------- epilogue
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int r = q * 32 + lane;                 // row of this thread in its CTA's half
        int local = 0;
        for (int t = unit; t < n_tiles; t += n_units, ++local) {
            // every decision before the warp-collective tcgen05.ld is warp-uniform
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const GemmTile g = gemm_tile<MODE, C::BM>(a, s_tb, routed_end, t);
            const int b = local & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[b], (local >> 1) & 1));
            if (!ok) {
                if (lane == 0) fail();
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * kBN;
            const int row0 = g.row0 + kBM * static_cast<int>(rank);     // this CTA's rows
            const bool row_ok = r < g.valid - kBM * static_cast<int>(rank);
            if (CG == 1 && g.nsw > 0) {
                // swapped tail tile: this thread holds weight row r of the
                // tile (TMEM lane r) for every token column
#pragma unroll 1
                for (int c = 0; c < g.nsw; c += 32) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(taddr + c, v0);
                    tmem_ld32(taddr + 128 + c, v1);
                    tmem_ld_wait();
                    if (MODE == kGateUp) {
                        const int f = g.n0 + r;                      // gate row f, up row f
                        if (f < a.F) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                if (c + i < g.valid) {
                                    const float gg = __uint_as_float(v0[i]), uu = __uint_as_float(v1[i]);
                                    const float h = gg / (1.f + __expf(-gg)) * uu;
                                    a.h_r[static_cast<size_t>(row0 + c + i) * a.F + f] =
                                        a.f16 ? __half_as_ushort(__float2half_rn(h))
                                              : __bfloat16_as_ushort(__float2bfloat16_rn(h));
                                }
                            }
                        }
                    } else {
                        // rows n0 + r and n0 + 128 + r of out, one token per column
                        int tk = 0;
                        float wv = 0.f;
                        if (c + lane < g.valid) {
                            tk = a.slot_token[row0 + c + lane];
                            wv = a.slot_w[row0 + c + lane];
                        }
                        const int j0 = g.n0 + r;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int tok_i = __shfl_sync(0xffffffffu, tk, i);
                            const float w_i = __shfl_sync(0xffffffffu, wv, i);
                            if (c + i < g.valid) {
                                float* orow = a.out + static_cast<size_t>(tok_i) * a.d;
                                if (j0 < a.d) red_add_f32(orow + j0, w_i * __uint_as_float(v0[i]));
                                if (j0 + 128 < a.d) red_add_f32(orow + j0 + 128, w_i * __uint_as_float(v1[i]));
                            }
                        }
                    }
                }
            } else if (MODE == kGateUp) {
                const int Fh = g.shared ? a.Fs : a.F;
                uint16_t* hrow = g.shared
                    ? a.h_s + static_cast<size_t>(row0 + r) * (a.S * a.Fs) + g.shared_s * a.Fs + g.n0
                    : a.h_r + static_cast<size_t>(row0 + r) * a.F + g.n0;
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
                            const float h0 = g0 / (1.f + __expf(-g0)) * u0;
                            const float h1 = g1 / (1.f + __expf(-g1)) * u1;
                            pk[i] = a.f16 ? pack_f16x2(h0, h1) : pack_bf16x2(h0, h1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(hrow + 32 * c);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            } else {
                // weighted combine: each thread scales its row, a warp stages its
                // 32 rows x 32 columns (16-byte chunks XOR-swizzled by row, so
                // both the row-wise writes and the column-wise reads are free of
                // bank conflicts), then every reduction instruction adds whole
                // 128-byte row segments (4 rows per instruction)
                int tok = 0;
                float w = 0.f;
                if (row_ok) {
                    if (g.shared) { tok = row0 + r; w = 1.f; }
                    else { tok = a.slot_token[row0 + r]; w = a.slot_w[row0 + r]; }
                }
                float* stg = stage_out + (warp - 2) * (32 * 32);
                const int cc = lane & 7;
#pragma unroll 1
                for (int c = 0; c < kBN / 32; ++c) {
                    uint32_t yv[32];
                    tmem_ld32(taddr + 32 * c, yv);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<float4*>(stg + lane * 32 + ((j ^ (lane & 7)) * 4)) =
                            make_float4(w * __uint_as_float(yv[4 * j]), w * __uint_as_float(yv[4 * j + 1]),
                                        w * __uint_as_float(yv[4 * j + 2]), w * __uint_as_float(yv[4 * j + 3]));
                    __syncwarp();
                    if (g.n0 + 32 * c < a.d) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int rr = 4 * i + (lane >> 3);
                            const int tok_r = __shfl_sync(0xffffffffu, tok, rr);
                            const bool ok_r = __shfl_sync(0xffffffffu, row_ok ? 1 : 0, rr) != 0;
                            const float4 v =
                                *reinterpret_cast<const float4*>(stg + rr * 32 + ((cc ^ (rr & 7)) * 4));
                            if (ok_r)
                                red_add_v4_f32(a.out + static_cast<size_t>(tok_r) * a.d + g.n0 + 32 * c + 4 * cc,
                                               v.x, v.y, v.z, v.w);
                        }
                    }
                    __syncwarp();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&tempty[b]);
                else mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[b]), 0));
            }
        }
    }
    tc_fence_before();
    if constexpr (CG == 2) cluster_sync_all();   // no signal into a CTA that has left
    else __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        if constexpr (CG == 2) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

size_t gemm_smem_bytes(int E, int cg) {
    const size_t stages = cg == 2 ? GemmCfg<2>::STAGES : GemmCfg<1>::STAGES;
    const size_t stage = cg == 2 ? GemmCfg<2>::STAGE : GemmCfg<1>::STAGE;
    return 1024 + stages * stage + kEpiStage + (2 * stages + 4) * 8 + 16 +
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
    int cg = 0;                       // 2: CTA-pair GEMMs (cluster launch), 1: single-CTA
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

// CTA pairs (256-row tiles) only when experts average >= 1024 rows: a pair
// moves a third fewer bytes per FLOP from L2 (measured: 18% more executed
// work per clock), but each expert's last tile is then up to 255 rows of
// padding instead of 127, which on the DeepSeek-shaped layer (384 rows per
// expert on average) costs more than the pair saves (675 vs 662 us for the
// two GEMMs).  Pairs also need the device to keep one pair per two SMs
// resident; otherwise single CTAs.
static int prefill_pick_cg(PrefillState* st, int num_sms) {
    if (st->cg) return st->cg;
    int cg = 1;
    const int64_t rows_per_expert =
        static_cast<int64_t>(st->cfg.t_max) * st->cfg.top_k / st->cfg.n_experts;
    if (rows_per_expert >= 1024 && num_sms % 2 == 0 &&
        cudaFuncSetAttribute(prefill_gemm_kernel<kGateUp, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(gemm_smem_bytes(kMaxExperts, 2))) == cudaSuccess &&
        cudaFuncSetAttribute(prefill_gemm_kernel<kDown, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(gemm_smem_bytes(kMaxExperts, 2))) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(num_sms);
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = gemm_smem_bytes(kMaxExperts, 2);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2; attr[0].val.clusterDim.y = 1; attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, prefill_gemm_kernel<kGateUp, 2>, &cfg) == cudaSuccess &&
            n >= num_sms / 2)
            cg = 2;
    }
    cudaGetLastError();
    st->cg = cg;
    return cg;
}

moe_status_t prefill_route(PrefillState* st, const moe_config_t& c, const Workspace& ws,
                           const moe_weights_t* w, const uint16_t* x, int T, float* out,
                           cudaStream_t stream, int num_sms, int* launches) {
    *launches = 0;
    if (c.n_experts > 256) return MOE_ERR_UNSUPPORTED;
    PrefillRouteArgs r{};
    r.x = x; r.wr = w->router_w; r.br = w->router_b; r.out = out; r.ws = ws; r.hist = st->hist;
    r.T = T; r.d = c.d_model; r.E = c.n_experts; r.k = c.top_k; r.S = c.n_shared;
    r.F = c.d_ff; r.Fs = c.n_shared ? c.d_ff_shared : 0;
    const int nch = (T + kChunkTok - 1) / kChunkTok;
    const size_t smem = router_smem_bytes(c.n_experts);
    // the shared-memory limit is a per-device attribute: raise it once per device
    static int set_smem[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    if (static_cast<int>(smem) > set_smem[dev]) {
        if (cudaFuncSetAttribute(prefill_router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        set_smem[dev] = static_cast<int>(smem);
    }
    prefill_router_kernel<<<nch, kRouterThreads, smem, stream>>>(r);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    ScatterArgs sa{};
    sa.x = x; sa.ws = ws; sa.hist = st->hist; sa.T = T; sa.d = c.d_model; sa.E = c.n_experts;
    sa.k = c.top_k; sa.S = c.n_shared; sa.F = c.d_ff; sa.Fs = c.n_shared ? c.d_ff_shared : 0;
    sa.bm = kBM * prefill_pick_cg(st, num_sms);
    prefill_scatter_kernel<<<nch, kScatterThreads, 0, stream>>>(sa);
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
        const int cg = prefill_pick_cg(st, num_sms);
        ok &= map2d(st, &g2.tmB0_r, w->down.data, static_cast<uint64_t>(E) * d, F, F, kBK, kBN / cg);
        if (S) {
            ok &= map2d(st, &g1.tmB0_s, w->shared_gate.data, static_cast<uint64_t>(S) * Fs, d, d, kBK, 128);
            ok &= map2d(st, &g1.tmB1_s, w->shared_up.data, static_cast<uint64_t>(S) * Fs, d, d, kBK, 128);
            ok &= map2d(st, &g2.tmA_s, ws.h_shared, c.t_max, static_cast<uint64_t>(S) * Fs,
                        static_cast<uint64_t>(S) * Fs, kBK, kBM);
            ok &= map2d(st, &g2.tmB0_s, w->shared_down.data, static_cast<uint64_t>(S) * d, Fs, Fs, kBK,
                        kBN / cg);
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
        g->f16 = c.wfmt == MOE_WFMT_BF16_F16DOWN ? 1 : 0;
    }
    st->g1.tile_base = ws.tiles;
    st->g2.tile_base = ws.tiles + E + 1;
    const int cg = prefill_pick_cg(st, num_sms);
    const size_t smem = gemm_smem_bytes(E, cg);
    if (cg == 1) {
        static bool attr[kMaxDevices] = {false};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
        if (!attr[dev]) {
            if (cudaFuncSetAttribute(prefill_gemm_kernel<kGateUp, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(gemm_smem_bytes(kMaxExperts, 1))) != cudaSuccess ||
                cudaFuncSetAttribute(prefill_gemm_kernel<kDown, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(gemm_smem_bytes(kMaxExperts, 1))) != cudaSuccess)
                return MOE_ERR_CUDA;
            attr[dev] = true;
        }
        prefill_gemm_kernel<kGateUp, 1><<<num_sms, kGemmThreads, smem, stream>>>(st->g1);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
        prefill_gemm_kernel<kDown, 1><<<num_sms, kGemmThreads, smem, stream>>>(st->g2);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    } else {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(num_sms);
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2; attr[0].val.clusterDim.y = 1; attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, prefill_gemm_kernel<kGateUp, 2>, st->g1) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaLaunchKernelEx(&cfg, prefill_gemm_kernel<kDown, 2>, st->g2) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    *launches = 2;
    return MOE_OK;
}

}  // namespace moe
