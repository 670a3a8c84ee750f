// decode.cu -- decode-regime kernels (T <= MOE_DECODE_MAX_T tokens per call).
//
// moe_forward runs the whole layer as ONE cooperative launch,
// decode_fused_kernel (its phases are described above the kernel): router
// logits published with a launch tag, top-k / buckets / work list computed by
// every CTA once every logit of its tokens carries that tag, then the experts
// pipeline.  moe_route + moe_experts (and moe_forward when a
// cooperative launch cannot place one CTA per SM) use two launches instead:
//  1. decode_route_kernel: router logits (fp32 FMA), softmax + top-k with
//     renormalised weights, per-expert buckets (counts, exclusive offsets,
//     stable slot order), the expert work list, and the zero-fill of `out`.
//     ("Fused MoE Triton kernel: 5 launches instead of 24" page, fused steps
//     one and two; its launch table's routing and dispatch rows.)
//  2. decode_experts_kernel: the experts pipeline alone.
//
// The experts pipeline makes ONE pass over every active routed expert and
// every shared expert ("CUDA: fuse shared experts into MMVQ" page: shared
// experts go through the same pass as the routed ones).  Each work unit is
// (expert, slice of FS hidden rows): it streams the slice's gate/up rows,
// forms h = SiLU(gate) * up for the expert's tokens, streams the matching
// columns of the down matrix and adds w * (Wd h) into `out` (the weighted
// aggregation, fused).  Weights move HBM -> shared memory by TMA through a
// ring of stages fed by one producer warp, so every SM keeps tens of KB in
// flight ("MoE on RTX 5090 reaches 41% of bandwidth" page: small reads per
// kernel cap bandwidth; the fix it predicts is more bytes per launch).  The
// contraction over the <= 8 tokens of an expert runs on mma.sync (bf16 or
// fp16 in, fp32 accumulate); quantised codes (Q4_0, Q8_0, Q5_0, q6_K) become
// operand fragments in registers and are never written back ("MMVQ" page:
// read quantised weights once, never expand them).
#include <float.h>
#include <math.h>
#include <stddef.h>

#include "moe_internal.cuh"

namespace moe {

// ============================================================== router ===
constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;

__global__ void __launch_bounds__(kRouteThreads) decode_route_kernel(const RouteArgs a) {
    __shared__ float s_part[kRouteWarps][kDecodeTok];
    __shared__ float s_log[kDecodeTok][kMaxExperts];
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_ids[kDecodeTok * kMaxTopK];
    __shared__ float s_w[kDecodeTok * kMaxTopK];
    __shared__ float s_sel[kDecodeTok][kMaxTopK];
    __shared__ int s_wsum[kRouteWarps];
    __shared__ uint32_t s_ticket;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T, d = a.d, E = a.E, k = a.k;

    // ---- zero-fill out [T][d] (the expert kernel accumulates into it)
    {
        const int n4 = (T * d) >> 2;
        float4* o = reinterpret_cast<float4*>(a.out);
        for (int i = blockIdx.x * kRouteThreads + tid; i < n4; i += gridDim.x * kRouteThreads)
            o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // ---- logits: CTA owns experts_per_cta experts, each split over wpe warps
    const int epc = a.experts_per_cta;
    const int wpe = kRouteWarps / epc;
    const int le = warp / wpe, part = warp % wpe;
    const int e = blockIdx.x * epc + le;
    float acc[kDecodeTok];
#pragma unroll
    for (int t = 0; t < kDecodeTok; ++t) acc[t] = 0.f;
    if (e < E) {
        const int chunk = d / wpe;
        const int i_end = (part + 1) * chunk;
        const float* wrow = a.wr + static_cast<size_t>(e) * d;
        // unrolled so that several router rows' loads are in flight at once
#pragma unroll 4
        for (int i = part * chunk + lane * 4; i < i_end; i += 128) {
            const float4 wv = __ldg(reinterpret_cast<const float4*>(wrow + i));
#pragma unroll
            for (int t = 0; t < kDecodeTok; ++t) {
                if (t < T) {
                    const uint2 xv = __ldg(reinterpret_cast<const uint2*>(
                        a.x + static_cast<size_t>(t) * d + i));
                    acc[t] = fmaf(__uint_as_float(xv.x << 16), wv.x, acc[t]);
                    acc[t] = fmaf(__uint_as_float(xv.x & 0xffff0000u), wv.y, acc[t]);
                    acc[t] = fmaf(__uint_as_float(xv.y << 16), wv.z, acc[t]);
                    acc[t] = fmaf(__uint_as_float(xv.y & 0xffff0000u), wv.w, acc[t]);
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kDecodeTok; ++t) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
    }
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < kDecodeTok; ++t) s_part[warp][t] = acc[t];
    }
    __syncthreads();
    if (tid < epc * T) {
        const int le2 = tid / T, t = tid % T;
        const int e2 = blockIdx.x * epc + le2;
        if (e2 < E) {
            float s = 0.f;
            for (int p = 0; p < wpe; ++p) s += s_part[le2 * wpe + p][t];   // fixed order
            if (a.br) s += a.br[e2];
            a.ws.logits[t * E + e2] = s;
        }
    }

    // ---- the last CTA to finish does top-k, buckets and the work list
    __threadfence();
    __syncthreads();
    if (tid == 0) s_ticket = atomicAdd(a.ws.ticket, 1u);
    __syncthreads();
    if (s_ticket != gridDim.x - 1) return;
    __threadfence();

    for (int i = tid; i < T * E; i += kRouteThreads) {
        float v = __ldcg(a.ws.logits + i);
        if (isnan(v)) v = -INFINITY;               // NaN never wins a slot
        s_log[i / E][i % E] = v;
    }
    __syncthreads();

    // top-k per token: warp t (register-resident logits, see warp_topk)
    if (warp < T) {
        const int t = warp;
        warp_topk_any(s_log[t], E, k, &s_ids[t * k], s_sel[t], a.ws.err);
        __syncwarp();
        // renormalised softmax over the selected logits == softmax over all E
        // experts restricted to the top-k and renormalised
        if (lane < k) {
            const float m = s_sel[t][0];
            float den = 0.f;
            for (int j = 0; j < k; ++j) den += expf(s_sel[t][j] - m);
            float wj = expf(s_sel[t][lane] - m) / den;
            if (!(m > -INFINITY)) wj = 1.f / k;
            s_w[t * k + lane] = wj;
        }
    }
    __syncthreads();

    // buckets: counts per expert, then one block scan of (count, active) pairs
    const int P = T * k;
    for (int x = tid; x < E; x += kRouteThreads) {
        int c = 0;
        for (int p = 0; p < P; ++p) c += (s_ids[p] == x);
        s_cnt[x] = c;
    }
    __syncthreads();
    constexpr int kPer = kMaxExperts / kRouteThreads;   // experts per thread (4)
    int loc[kPer];
    int run = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int x = tid * kPer + q;
        const int c = (x < E) ? s_cnt[x] : 0;
        loc[q] = run;
        run += (c << 16) | (c > 0 ? 1 : 0);
    }
    int incl = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int base = incl - run;
    for (int w2 = 0; w2 < warp; ++w2) base += s_wsum[w2];
    int total = 0;
    for (int w2 = 0; w2 < kRouteWarps; ++w2) total += s_wsum[w2];
    const int n_routed = total & 0xffff;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int x = tid * kPer + q;
        if (x < E) {
            const int ex = base + loc[q];
            const int off = ex >> 16, act = ex & 0xffff;
            const int c = s_cnt[x];
            a.ws.counts[x] = c;
            a.ws.offsets[x] = off;
            if (c > 0) {
                if (c > kDecodeTok) atomicOr(a.ws.err, kErrTooManyTok);
                a.ws.items[act] = WorkItem{x, off, c, 0};
            }
            s_cnt[x] = off;   // reuse as offsets
        }
    }
    if (tid == 0) {
        a.ws.offsets[E] = total >> 16;
        a.ws.n_items[0] = n_routed;
        a.ws.n_items[1] = a.S;
    }
    if (tid < a.S) a.ws.items[n_routed + tid] = WorkItem{E + tid, -1, T, 0};
    __syncthreads();
    // stable slots: rank of pair p among earlier pairs with the same expert
    for (int p = tid; p < P; p += kRouteThreads) {
        const int x = s_ids[p];
        int rank = 0;
        for (int q = 0; q < p; ++q) rank += (s_ids[q] == x);
        const int slot = s_cnt[x] + rank;
        a.ws.slot_pair[slot] = p;
        a.ws.slot_token[slot] = p / k;
        a.ws.slot_w[slot] = s_w[p];
        a.ws.ids[p] = x;
        a.ws.wts[p] = s_w[p];
    }
    if (tid == 0) *a.ws.ticket = 0u;   // ready for the next call
}

cudaError_t launch_decode_route(const RouteArgs& a, cudaStream_t stream) {
    const int grid = (a.E + a.experts_per_cta - 1) / a.experts_per_cta;
    decode_route_kernel<<<grid, kRouteThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

// ============================================================ experts ===
constexpr int kConsumerWarps = kDecodeConsumerWarps;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kDecodeThreads = kConsumers + 32;   // + one producer warp

// Weight formats of the decode kernels (the values of moe_wfmt_t).
constexpr int kWfBf16 = 0, kWfQ4 = 1, kWfQ8 = 2;
constexpr int kWfQ5 = 3;
constexpr int kWfQ6 = 4;     // q6_K super-blocks (row-streaming, fp16 operands)
constexpr int kWfF16d = 5;   // bf16 gate/up, fp16 down matrices (h travels in fp16)

// The constant that turns Q5_0's bf16 operands 128 + q (q < 32, see q5_raw)
// back into its signed codes q - 16: 128 + 16.
constexpr float kQ5Offset = 144.f;

template <int FS, int WF>
struct DecodeCfg {
    static constexpr int RG = FS / 16;            // 16-row groups in a slice
    static constexpr int ROLES = 2 * RG;          // (matrix, row group) pairs of phase A
    static constexpr int KSPLIT = kConsumerWarps / ROLES;
    static_assert(KSPLIT >= 1 && ROLES * KSPLIT == kConsumerWarps, "warp roles");
    static constexpr bool QUANT = WF == kWfQ4 || WF == kWfQ8 || WF == kWfQ5 || WF == kWfQ6;
    // bf16 phase A with fp16 down matrices: h is stored as an fp16 hi + lo
    // pair and the down contraction runs on fp16 operands
    static constexpr bool HALF_DOWN = WF == kWfF16d;
    static_assert(!QUANT || FS >= 32, "quantised slices hold whole blocks");
    // fp16 tensor-core operands (see q4h_lo, q8h_lo): x staged as fp16, h as
    // an fp16 hi + lo pair, per-block corrections of the code bases
    static constexpr bool F16 = WF == kWfQ4 || WF == kWfQ6 || WF == kWfQ8;
    static constexpr bool Q8 = WF == kWfQ8;
    // q6_K: per 32-wide block and 16-row group a 160-byte record (high bits,
    // sub-block scales), per row and 256-wide super-block an fp16 scale
    static constexpr bool Q6 = WF == kWfQ6;
    static constexpr int CB = WF == kWfQ8 ? 32 : 16;   // code bytes of one block row
    // + its fp16 scale (Q5_0: + its 32-bit word of fifth bits; scale and word
    // sit in 48-byte records of 8 rows, see q5_aux)
    static constexpr int BR = CB + (WF == kWfQ5 ? 6 : 2);
    // bf16: phase A stage = gate+up [FS rows][KT cols]; phase B = down [RJ rows][FS cols]
    // Q5_0: phase A stage = gate+up [KB block cols][FS rows]; phase B =
    //       [NB block cols][RJ rows]; codes, then the 48-byte records of
    //       scales and fifth bits
    // Q4_0 / Q8_0: phase A 16 rows x 64 blocks (codes, then scales), phase B
    //       4 boxes of 256 rows (18 or 34 KB per stage)
    // q6_K: phase A 16 rows x 64 blocks (26880 B), phase B 4 boxes of 256
    // rows (4 x 7168 B)
    static constexpr int STAGE = Q6 ? 28672 : QUANT ? 2 * 512 * BR : 32768;
    static constexpr int KT = 8192 / FS;          // bf16 phase A k columns
    static constexpr int KB = 512 / FS;           // quantised phase A block columns
    static constexpr int NB = FS / 32;            // quantised block columns in a slice
    static constexpr int RJ = QUANT ? 32768 / FS : 16384 / FS;   // phase B rows per stage
    static_assert(!QUANT || RJ % kQuantDownBoxRows == 0, "whole down boxes per stage");
    static constexpr int HS = FS + 8;             // h row stride (bf16 elements)
    static constexpr int GS = FS + 4;             // gate/up result row stride (floats)
    // Row-streaming phase A (the F16 formats, experts_pipeline_rows): a stage
    // is one 16-row group of one matrix over KC <= KCMAX block columns, and
    // consumer warp w owns block columns w, w + 16, ... of every stage.
    static constexpr int KCMAX = 64;
    static constexpr int NBW = KCMAX / kConsumerWarps;   // block columns per warp
    static constexpr int GU_PARTS = F16 ? kConsumerWarps : KSPLIT;   // partial sums per output
};

struct alignas(16) DecodeSmemTail {
    int abort_flag;
    int pad[3];
};

// ((w >> s) & 0x000F000F) | 0x43004300 puts two 4-bit codes q in the low
// mantissa bits of two bf16 values 128 + q (exact): the bf16 operands of
// the Q5_0 kernels, which add the fifth bit on top (see q5_raw).
__device__ __forceinline__ uint32_t q4_raw(uint32_t w, int s) {
    return ((w >> s) & 0x000F000Fu) | 0x43004300u;
}

// The fp16 form of the same operands, one LOP3 per register (Q4_0).  In an
// fp16 value whose exponent makes the unit in the last place 1 (base 1024,
// 0x6400), a code in mantissa bits 0-3 reads as 1024 + q; with base 64
// (0x5400, ulp 1/16) a code in bits 4-7 reads as 64 + q.  Both are exact.
// So the word's codes in bits 0-3 / 16-19 (k pair 2t, 2t+1 of the first
// 16-wide half) and 4-7 / 20-23 (k pair 2t+8, 2t+9) need no shift; one
// shift by 8 brings the second half's codes to the same places.  Within a
// block, k % 16 < 8 has base 1024 and k % 16 >= 8 base 64, and the block's
// accumulator starts at -sum((base_k + 8) x_k), so that the block adds
// sum((q - 8) x) before its scale.
__device__ __forceinline__ uint32_t q4h_lo(uint32_t w) { return (w & 0x000F000Fu) | 0x64006400u; }
__device__ __forceinline__ uint32_t q4h_hi(uint32_t w) { return (w & 0x00F000F0u) | 0x54005400u; }
constexpr float kF16BaseLo = 1024.f, kF16BaseHi = 64.f;

__device__ __forceinline__ uint2 lds_u32x2(uint32_t addr) {   // addr 8-byte aligned
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

// Q8_0 on fp16 operands, one byte permute per register.  A packed byte is
// the biased code u = q + 128; with the byte 0x64 above it, it reads as the
// fp16 value 1024 + u (exact: the unit in the last place of [1024, 2048) is
// 1).  Lane tig's 32-bit word of a block half holds u of k = 2tig, 2tig+1,
// 2tig+8, 2tig+9 in its four bytes (see the Q8_0 packer), so q8h_lo gives
// the A-fragment register of the pair (2tig, 2tig+1) and q8h_hi that of
// (2tig+8, 2tig+9).  The weight is d q = d ((1024 + u) - 1152): the block's
// accumulator starts at -1152 * (sum of the block's 32 activations).
__device__ __forceinline__ uint32_t q8h_lo(uint32_t w) { return __byte_perm(w, 0x64646464u, 0x4140u); }
__device__ __forceinline__ uint32_t q8h_hi(uint32_t w) { return __byte_perm(w, 0x64646464u, 0x4342u); }
constexpr float kQ8Offset = 1024.f + 128.f;

// ---- Q5_0.  The low 4 bits of each code are packed exactly like Q4_0
// codes.  The fifth bits of a block row form one 32-bit word in which lane
// tig owns bits 4 tig + n (the code in nibble n of its code word, n = 0..3)
// and bits 16 + 4 tig + n (nibble n + 4).  q5_lane_bits moves the lane's
// eight bits to bits 4-7 and 20-23, so that (e >> n) & 0x00100010 is the
// fifth bit, worth 16, of the two codes q4_raw(w, 4n) extracts: q5_raw is
// then two bf16 values 128 + q, q in 0..31 (exact; Q5_0's weight is
// d * (q - 16), the 128 + 16 folded into kQ5Offset).
__device__ __forceinline__ uint32_t q5_lane_bits(uint32_t word, int tig) {
    return ((word >> (4 * tig)) & 0x000F000Fu) << 4;
}

__device__ __forceinline__ uint32_t q5_raw(uint32_t w, uint32_t e, int n) {
    return q4_raw(w, 4 * n) | ((e >> n) & 0x00100010u);
}

// Scale and fifth-bit word of rows r and r + 8 (r % 16 < 8) of block column
// bb in a stage region of 48-byte records [block columns][rows / 8]: a record
// holds the 8 fp16 scales of 8 consecutive rows, then their 8 words.
__device__ __forceinline__ void q5_aux(const uint8_t* aux, int bb, int nrows, int r, float& s0,
                                       float& s8, uint32_t& h0, uint32_t& h8) {
    const uint8_t* rec = aux + (bb * (nrows / 8) + (r >> 3)) * 48;
    const int i = r & 7;
    s0 = __half2float(*reinterpret_cast<const __half*>(rec + 2 * i));
    s8 = __half2float(*reinterpret_cast<const __half*>(rec + 48 + 2 * i));
    h0 = *reinterpret_cast<const uint32_t*>(rec + 16 + 4 * i);
    h8 = *reinterpret_cast<const uint32_t*>(rec + 48 + 16 + 4 * i);
}

// One Q5_0 block (32 weights along k) of rows r and r+8 of an mma A tile,
// times the B fragment of the same 32 k (b0 b1: k 0-15, b2 b3: k 16-31).
// row_r / row_r8 point at the rows' code words, e0 / e8 are q5_lane_bits of
// their fifth-bit words, c0 / c1 the accumulator starts of the lane's two
// token columns (-144 * the block's activation sums); v gets the block's
// four dot products before the block scale.  q5_block_b is the same for the
// down contraction, whose B operand is h as a bf16 pair: bh / bl hold the hi
// and lo fragments of the block's two 16-wide halves.
__device__ __forceinline__ void q5_block_a(const uint32_t* row_r, const uint32_t* row_r8,
                                           uint32_t e0, uint32_t e8, int tig, float c0, float c1,
                                           uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3,
                                           float v[4]) {
    const uint32_t w0 = row_r[tig], w8 = row_r8[tig];
    float cb0[4] = {c0, c1, c0, c1}, cb1[4] = {0.f, 0.f, 0.f, 0.f};
    mma_bf16_16816(cb0, q5_raw(w0, e0, 0), q5_raw(w8, e8, 0), q5_raw(w0, e0, 1), q5_raw(w8, e8, 1),
                   b0, b1);
    mma_bf16_16816(cb1, q5_raw(w0, e0, 2), q5_raw(w8, e8, 2), q5_raw(w0, e0, 3), q5_raw(w8, e8, 3),
                   b2, b3);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = cb0[i] + cb1[i];
}

__device__ __forceinline__ void q5_block_b(const uint32_t* row_r, const uint32_t* row_r8,
                                           uint32_t e0, uint32_t e8, int tig, float c0, float c1,
                                           const uint32_t* bh0, const uint32_t* bh1,
                                           const uint32_t* bl0, const uint32_t* bl1, float v[4]) {
    const uint32_t w0 = row_r[tig], w8 = row_r8[tig];
    const uint32_t p0 = q5_raw(w0, e0, 0), q0 = q5_raw(w8, e8, 0);
    const uint32_t p1 = q5_raw(w0, e0, 1), q1 = q5_raw(w8, e8, 1);
    const uint32_t p2 = q5_raw(w0, e0, 2), q2 = q5_raw(w8, e8, 2);
    const uint32_t p3 = q5_raw(w0, e0, 3), q3 = q5_raw(w8, e8, 3);
    float cb0[4] = {c0, c1, c0, c1}, cb1[4] = {0.f, 0.f, 0.f, 0.f};
    mma_bf16_16816(cb0, p0, q0, p1, q1, bh0[0], bh0[1]);
    mma_bf16_16816(cb1, p2, q2, p3, q3, bh1[0], bh1[1]);
    mma_bf16_16816(cb0, p0, q0, p1, q1, bl0[0], bl0[1]);
    mma_bf16_16816(cb1, p2, q2, p3, q3, bl1[0], bl1[1]);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = cb0[i] + cb1[i];
}

// Work list the experts pipeline reads: generic pointers, so the same code
// serves the two-launch path (global memory, written by the router kernel)
// and the fused kernel (shared memory, computed by every CTA itself).
struct WorkView {
    int n_routed, n_shared;
    const WorkItem* items;        // routed items (ascending expert), then shared items
    const int32_t* slot_token;    // slot -> token
    const float* slot_w;          // slot -> routing weight
};

// Shared-memory carve-up of the experts pipeline.
struct DecodeSmem {
    uint8_t* ring;
    uint8_t* xs;            // [8][xs_stride]: the T token rows of x, staged once
    float* xsum;            // [8][d/16]: block (q6_K: sub-block) accumulator starts (quantised formats)
    float* gu;              // [GU_PARTS][2][8][GS]: gate / up partial results
    __nv_bfloat16* hhi;     // [8][HS]: h = hi + lo, per slot
    __nv_bfloat16* hlo;
    float* hsum;            // [8][4]: down block (q6_K: sub-block) accumulator starts from hi + lo
    DecodeSmemTail* tail;
    uint64_t* full;
    uint64_t* empty;
};

template <int FS, int WF>
__device__ __forceinline__ DecodeSmem decode_smem(uint8_t* smem_raw, const DecodeArgs& a) {
    using C = DecodeCfg<FS, WF>;
    DecodeSmem sm;
    // align to 1 KB by pointer arithmetic on the shared array itself (a round
    // trip through an integer would hide the address space from the compiler)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    sm.ring = smem;
    sm.xs = sm.ring + static_cast<size_t>(a.n_stages) * C::STAGE;
    sm.xsum = reinterpret_cast<float*>(sm.xs + kDecodeTok * a.xs_stride);
    sm.gu = sm.xsum + kDecodeTok * (a.d / 16);
    sm.hhi = reinterpret_cast<__nv_bfloat16*>(sm.gu + C::GU_PARTS * 2 * kDecodeTok * C::GS);
    sm.hlo = sm.hhi + kDecodeTok * C::HS;
    sm.hsum = reinterpret_cast<float*>(sm.hlo + kDecodeTok * C::HS);
    sm.tail = reinterpret_cast<DecodeSmemTail*>(sm.hsum + kDecodeTok * 4);
    sm.full = reinterpret_cast<uint64_t*>(sm.tail + 1);
    sm.empty = sm.full + a.n_stages;
    return sm;
}

// Consumer threads copy the T token rows of x into shared memory once per
// launch; every work unit then addresses its tokens' rows directly.  For
// the quantised formats the same pass stores each 32-wide block's (q6_K:
// 16-wide sub-block's) accumulator start, minus the code bases times the
// block's activations (see q4h_lo, q8h_lo, q6h_regs and q5_raw).
template <int WF>
__device__ __forceinline__ void stage_x(const DecodeArgs& a, const DecodeSmem& sm, int tid) {
    const int nkb = a.d / 32;
    if constexpr (WF == kWfQ4 || WF == kWfQ6 || WF == kWfQ8) {
        // fp16 copy of x (exact for |x| >= 2^-17; below, off by at most 2^-25)
        // and each block's accumulator start: Q4_0 -sum((base_k + 8) x_k),
        // base_k 1024 for k % 16 < 8 and 64 otherwise (see q4h_lo); Q8_0
        // -1152 sum(x_k) (see q8h_lo)
        for (int idx = tid; idx < a.T * nkb; idx += kConsumers) {
            const int t = idx / nkb, kb = idx % nkb;
            const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.d + kb * 32);
            uint4* dst = reinterpret_cast<uint4*>(sm.xs + t * a.xs_stride + kb * 64);
            float s8[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 v = __ldg(src + c);
                const uint32_t q[4] = {v.x, v.y, v.z, v.w};
                uint32_t h[4];
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float lo = __uint_as_float(q[j] << 16), hi = __uint_as_float(q[j] & 0xffff0000u);
                    s += lo + hi;
                    __half2 hv = __floats2half2_rn(lo, hi);
                    h[j] = *reinterpret_cast<uint32_t*>(&hv);
                }
                dst[c] = make_uint4(h[0], h[1], h[2], h[3]);
                s8[c] = s;                                  // elements 8c .. 8c+7
            }
            if constexpr (WF == kWfQ4) {
                sm.xsum[t * nkb + kb] =
                    -((kF16BaseLo + 8.f) * (s8[0] + s8[2]) + (kF16BaseHi + 8.f) * (s8[1] + s8[3]));
            } else if constexpr (WF == kWfQ8) {
                sm.xsum[t * nkb + kb] = -kQ8Offset * ((s8[0] + s8[1]) + (s8[2] + s8[3]));
            } else {
                // q6_K: one start per 16-wide sub-block, offset 32
                sm.xsum[t * 2 * nkb + 2 * kb] = -((kF16BaseLo + 32.f) * s8[0] + (kF16BaseHi + 32.f) * s8[1]);
                sm.xsum[t * 2 * nkb + 2 * kb + 1] =
                    -((kF16BaseLo + 32.f) * s8[2] + (kF16BaseHi + 32.f) * s8[3]);
            }
        }
    } else {
    for (int idx = tid; idx < a.T * nkb; idx += kConsumers) {
        const int t = idx / nkb, kb = idx % nkb;
        const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.d + kb * 32);
        uint4* dst = reinterpret_cast<uint4*>(sm.xs + t * a.xs_stride + kb * 64);
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 v = __ldg(src + c);
            dst[c] = v;
            if constexpr (WF == kWfQ5) {
                const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    s += __uint_as_float(q[j] << 16) + __uint_as_float(q[j] & 0xffff0000u);
            }
        }
        if constexpr (WF == kWfQ5) sm.xsum[t * nkb + kb] = -kQ5Offset * s;
    }
    }
}

// The expert stage with block-column stages (bf16, bf16 with fp16 down
// matrices, Q5_0): work units are (expert, slice of FS hidden rows), shared
// experts' units first, then the routed experts' in ascending expert order
// (assignment to CTAs: see below).  The last warp (lane 0) is the TMA
// producer, the others consume.  Barriers must be initialised by the caller.
template <int FS, int WF>
__device__ __forceinline__ void experts_pipeline(const DecodeArgs& a, const DecodeSmem& sm,
                                                 const WorkView& wv) {
    using C = DecodeCfg<FS, WF>;
    const int ns = a.n_stages;
    uint8_t* ring = sm.ring;
    float* gu = sm.gu;
    __nv_bfloat16* hhi = sm.hhi;
    __nv_bfloat16* hlo = sm.hlo;
    DecodeSmemTail* tail = sm.tail;
    uint64_t* full = sm.full;
    uint64_t* empty = sm.empty;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = a.d, E = a.E;
    const int n_routed = wv.n_routed, n_shared = wv.n_shared;
    const int sl_r = a.F / FS, sl_s = a.S ? a.Fs / FS : 0;
    const int n_su = n_shared * sl_s;
    const int n_units = n_su + n_routed * sl_r;
    const int nA = C::QUANT ? (d / 32 + C::KB - 1) / C::KB : (d + C::KT - 1) / C::KT;
    const int nB = (d + C::RJ - 1) / C::RJ;
    volatile int* abort_flag = &tail->abort_flag;

    // Unit assignment: CTA b takes units b, b+G, b+2G, ...  At any moment the
    // CTAs stream neighbouring slices of the same expert, so DRAM pages and
    // L2 lines are shared by requests that arrive together.  (Every unit
    // reads its tokens' rows of x from the copy staged once per CTA, so
    // nothing is lost when consecutive units of a CTA belong to different
    // experts.)
    const int u_begin = static_cast<int>(blockIdx.x);
    const int u_end = n_units;
    const int u_step = static_cast<int>(gridDim.x);

    // unit -> (item index, slice): shared units first
    auto unit_item = [&](int u, int& ii, int& sl) {
        if (u < n_su) { ii = n_routed + u / sl_s; sl = u % sl_s; }
        else { const int v = u - n_su; ii = v / sl_r; sl = v % sl_r; }
    };
    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&a.tm_gate); prefetch_tensormap(&a.tm_up);
            prefetch_tensormap(&a.tm_down);
            if (a.S) { prefetch_tensormap(&a.tm_sgate); prefetch_tensormap(&a.tm_sup);
                       prefetch_tensormap(&a.tm_sdown); }
            if constexpr (C::QUANT) {
                prefetch_tensormap(&a.tm_gate_sc); prefetch_tensormap(&a.tm_up_sc);
                prefetch_tensormap(&a.tm_down_sc);
                if (a.S) { prefetch_tensormap(&a.tm_sgate_sc); prefetch_tensormap(&a.tm_sup_sc);
                           prefetch_tensormap(&a.tm_sdown_sc); }
            }
            const uint64_t pol = l2_policy_evict_first();
            uint32_t it = 0;
            bool ok = true;
            for (int u = u_begin; u < u_end && ok; u += u_step) {
                int ii, sl;
                unit_item(u, ii, sl);
                const WorkItem item = wv.items[ii];
                const bool shared = item.expert >= E;
                const int ex = shared ? item.expert - E : item.expert;
                const int Fh = shared ? a.Fs : a.F;
                const int f0 = sl * FS;
                const CUtensorMap* mg = shared ? &a.tm_sgate : &a.tm_gate;
                const CUtensorMap* mu = shared ? &a.tm_sup : &a.tm_up;
                const CUtensorMap* md = shared ? &a.tm_sdown : &a.tm_down;
                const CUtensorMap* mgs = shared ? &a.tm_sgate_sc : &a.tm_gate_sc;
                const CUtensorMap* mus = shared ? &a.tm_sup_sc : &a.tm_up_sc;
                const CUtensorMap* mds = shared ? &a.tm_sdown_sc : &a.tm_down_sc;
                for (int st = 0; st < nA + nB && ok; ++st, ++it) {
                    const int slot = it % ns;
                    if (it >= static_cast<uint32_t>(ns)) {
                        if (*abort_flag || !mbar_wait_bounded_sleep(&empty[slot], ((it / ns) - 1) & 1)) {
                            atomicOr(a.err, kErrTimeout); *abort_flag = 1; ok = false; break;
                        }
                    }
                    uint8_t* dst = ring + static_cast<size_t>(slot) * C::STAGE;
                    if (st < nA) {
                        if constexpr (!C::QUANT) {
                            const int k0 = st * C::KT;
                            const int nbox = min(C::KT, d - k0) / 64;
                            mbar_arrive_expect_tx(&full[slot], 2 * nbox * FS * 128);
                            const int row = ex * Fh + f0;
                            for (int b = 0; b < nbox; ++b) {
                                tma_load_2d(dst + b * FS * 128, mg, &full[slot], k0 + 64 * b, row, pol);
                                tma_load_2d(dst + FS * C::KT * 2 + b * FS * 128, mu, &full[slot],
                                            k0 + 64 * b, row, pol);
                            }
                        } else {
                            const int kb0 = st * C::KB;
                            const int c2 = ex * (d / 32) + kb0;
                            mbar_arrive_expect_tx(&full[slot], 2 * C::KB * FS * C::BR);
                            uint8_t* g = dst;
                            uint8_t* u2 = dst + C::KB * FS * C::BR;
                            // code maps address 16-row groups (one 256/512-byte line each)
                            tma_load_3d(g, mg, &full[slot], 0, f0 / 16, c2, pol);
                            tma_load_3d(u2, mu, &full[slot], 0, f0 / 16, c2, pol);
                            if constexpr (WF == kWfQ5) {
                                // 48-byte records of 8 rows: {48 bytes, rows / 8, block columns}
                                tma_load_3d(g + C::KB * FS * C::CB, mgs, &full[slot], 0, f0 / 8, c2, pol);
                                tma_load_3d(u2 + C::KB * FS * C::CB, mus, &full[slot], 0, f0 / 8, c2, pol);
                            } else {
                                tma_load_2d(g + C::KB * FS * C::CB, mgs, &full[slot], f0, c2, pol);
                                tma_load_2d(u2 + C::KB * FS * C::CB, mus, &full[slot], f0, c2, pol);
                            }
                        }
                    } else {
                        const int j0 = (st - nA) * C::RJ;
                        if constexpr (!C::QUANT) {
                            const int nbox = min(C::RJ, d - j0) / 128;
                            mbar_arrive_expect_tx(&full[slot], nbox * 128 * FS * 2);
                            for (int b = 0; b < nbox; ++b)
                                tma_load_2d(dst + b * 128 * FS * 2, md, &full[slot], f0,
                                            ex * d + j0 + 128 * b, pol);
                        } else {
                            // boxes of QB rows; rows past d (d is a multiple of 128)
                            // are out of the map and arrive as zeros
                            constexpr int QB = kQuantDownBoxRows;
                            const int nbox = (min(C::RJ, d - j0) + QB - 1) / QB;
                            const int c2 = ex * (Fh / 32) + f0 / 32;
                            mbar_arrive_expect_tx(&full[slot], nbox * C::NB * QB * C::BR);
                            for (int b = 0; b < nbox; ++b) {
                                uint8_t* bd = dst + b * (C::NB * QB * C::BR);
                                tma_load_3d(bd, md, &full[slot], 0, (j0 + QB * b) / 16, c2, pol);
                                if constexpr (WF == kWfQ5)
                                    tma_load_3d(bd + C::NB * QB * C::CB, mds, &full[slot], 0,
                                                (j0 + QB * b) / 8, c2, pol);
                                else
                                    tma_load_2d(bd + C::NB * QB * C::CB, mds, &full[slot],
                                                j0 + QB * b, c2, pol);
                            }
                        }
                    }
                }
            }
            // drain: every issued stage must land before the CTA may exit
            const uint32_t first = it > static_cast<uint32_t>(ns) ? it - ns : 0;
            for (uint32_t q = first; q < it; ++q)
                if (!mbar_wait_bounded_sleep(&full[q % ns], (q / ns) & 1)) {
                    atomicOr(a.err, kErrTimeout);
                    break;
                }
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int g = lane >> 2, tig = lane & 3;
    const int role = warp % C::ROLES, ks = warp / C::ROLES;
    const int mat = role / C::RG, rg = role % C::RG;
    const uint32_t xs_u = smem_u32(sm.xs);
    const int nkb = d / 32;
    uint32_t it = 0;

    // warp-uniform: the ldmatrix / mma.sync that follow are warp-collective;
    // fast path when the stage has landed (the abort flag matters only to a
    // wait that would otherwise run into the limit)
    auto wait_full = [&](int slot, uint32_t parity) -> bool {
        if (__all_sync(0xffffffffu, mbar_try_wait(&full[slot], parity))) return true;
        if (__any_sync(0xffffffffu, *abort_flag != 0)) return false;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded_sleep(&full[slot], parity));
        if (!ok && lane == 0) {
            atomicOr(a.err, kErrTimeout);
            *abort_flag = 1;
        }
        return ok;
    };

    for (int u = u_begin; u < u_end; u += u_step) {
        int ii, sl;
        unit_item(u, ii, sl);
        const WorkItem item = wv.items[ii];
        const bool shared = item.expert >= E;
        const int ntok = min(item.count, kDecodeTok);
        // token slot n of this item -> token row (slots past ntok reuse row 0:
        // their columns of the mma are computed and never stored)
        auto tok_of = [&](int n) -> int {
            return n < ntok ? (shared ? n : wv.slot_token[item.slot_begin + n]) : 0;
        };
        auto w_of = [&](int n) -> float {
            return n < ntok ? (shared ? 1.f : wv.slot_w[item.slot_begin + n]) : 0.f;
        };
        const uint32_t xrow = xs_u + tok_of(lane & 7) * a.xs_stride;   // B row of this lane
        const int t0 = 2 * tig, t1 = t0 + 1;
        const int tok0 = tok_of(t0), tok1 = tok_of(t1);
        const float w0 = w_of(t0), w1 = w_of(t1);
        const bool v0 = t0 < ntok, v1 = t1 < ntok;

        // ------------------------------------------- phase A: gate and up
        float cacc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int st = 0; st < nA; ++st, ++it) {
            const int slot = it % ns;
            const bool ok = wait_full(slot, (it / ns) & 1);
            const uint8_t* stage = ring + static_cast<size_t>(slot) * C::STAGE;
            if (ok) {
                if constexpr (!C::QUANT) {
                    const int k0 = st * C::KT;
                    const int kmax = min(C::KT, d - k0) / 16;
                    const uint32_t tile = smem_u32(stage) + mat * (FS * C::KT * 2);
                    const int m = lane >> 3, r = lane & 7;
                    const uint32_t arow = rg * 16 + ((m & 1) << 3) + r;
#pragma unroll 4
                    for (int kk = ks; kk < kmax; kk += C::KSPLIT) {
                        uint32_t a0, a1, a2, a3, b0, b1;
                        ldsm_x4(tile + (kk >> 2) * (FS * 128) +
                                    swz_offset(arow, (kk & 3) * 2 + (m >> 1), 128),
                                a0, a1, a2, a3);
                        ldsm_x2(xrow + (k0 + kk * 16 + ((lane >> 3) & 1) * 8) * 2, b0, b1);
                        mma_bf16_16816(cacc, a0, a1, a2, a3, b0, b1);
                    }
                } else {
                    const int kb0 = st * C::KB;
                    const int nkb_st = min(C::KB, nkb - kb0);
                    const uint8_t* mb = stage + mat * (C::KB * FS * C::BR);
                    const uint32_t* codes = reinterpret_cast<const uint32_t*>(mb);   // [KB][FS][CB]
                    const __half* scl = reinterpret_cast<const __half*>(mb + C::KB * FS * C::CB);
                    const int r0 = rg * 16 + g;
                    const float* xsum0 = sm.xsum + tok0 * nkb + kb0;
                    const float* xsum1 = sm.xsum + tok1 * nkb + kb0;
                    {
#pragma unroll 2
                    for (int bb = ks; bb < nkb_st; bb += C::KSPLIT) {
                        const uint32_t* row = codes + (bb * FS + r0) * (C::CB / 4);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(xrow + ((kb0 + bb) * 32 + (lane >> 3) * 8) * 2, b0, b1, b2, b3);
                        // Q5_0; the accumulator starts at -144 * sum(x) of the block
                        float v[4], s0, s8;
                        uint32_t h0, h8;
                        q5_aux(reinterpret_cast<const uint8_t*>(scl), bb, FS, r0, s0, s8, h0, h8);
                        q5_block_a(row, row + 8 * (C::CB / 4), q5_lane_bits(h0, tig),
                                   q5_lane_bits(h8, tig), tig, xsum0[bb], xsum1[bb], b0, b1, b2,
                                   b3, v);
                        cacc[0] = fmaf(s0, v[0], cacc[0]);
                        cacc[1] = fmaf(s0, v[1], cacc[1]);
                        cacc[2] = fmaf(s8, v[2], cacc[2]);
                        cacc[3] = fmaf(s8, v[3], cacc[3]);
                    }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        {
            // gate/up partials as [t][f]: row stride GS = FS + 4 keeps the
            // four token columns of a lane quad in distinct banks
            float* gq = gu + (ks * 2 + mat) * kDecodeTok * C::GS;
            const int r = rg * 16 + g;
            gq[t0 * C::GS + r] = cacc[0];
            gq[t1 * C::GS + r] = cacc[1];
            gq[t0 * C::GS + r + 8] = cacc[2];
            gq[t1 * C::GS + r + 8] = cacc[3];
        }
        named_bar_sync(1, kConsumers);
        // h = SiLU(gate) * up, kept as a bf16 pair hi + lo (|h - hi - lo| <= 2^-16 |h|).
        // One warp covers 32 consecutive f of one slot, i.e. one Q5_0 block of
        // the down matrix (FS * 8 is a multiple of 32: the loop is warp-uniform).
        for (int idx = tid; idx < FS * kDecodeTok; idx += kConsumers) {
            const int t = idx / FS, f = idx % FS;
            float gv = 0.f, uv = 0.f;
#pragma unroll
            for (int q = 0; q < C::KSPLIT; ++q) {
                gv += gu[((q * 2 + 0) * kDecodeTok + t) * C::GS + f];
                uv += gu[((q * 2 + 1) * kDecodeTok + t) * C::GS + f];
            }
            const float h = gv / (1.f + expf(-gv)) * uv;
            if constexpr (C::HALF_DOWN) {
                const __half hi = __float2half_rn(h);
                reinterpret_cast<__half*>(hhi)[t * C::HS + f] = hi;
                reinterpret_cast<__half*>(hlo)[t * C::HS + f] = __float2half_rn(h - __half2float(hi));
                continue;
            }
            const __nv_bfloat16 hi = __float2bfloat16_rn(h);
            const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
            hhi[t * C::HS + f] = hi;
            hlo[t * C::HS + f] = lo;
            if constexpr (C::QUANT) {
                float hs = __bfloat162float(hi) + __bfloat162float(lo);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) hs += __shfl_xor_sync(0xffffffffu, hs, off);
                if (lane == 0) sm.hsum[t * 2 + f / 32] = -kQ5Offset * hs;
            }
        }
        named_bar_sync(1, kConsumers);
        uint32_t bh[C::RG][2], bl[C::RG][2];
#pragma unroll
        for (int kk = 0; kk < C::RG; ++kk) {
            const uint32_t off = ((lane & 7) * C::HS + kk * 16 + ((lane >> 3) & 1) * 8) * 2;
            ldsm_x2(smem_u32(hhi) + off, bh[kk][0], bh[kk][1]);
            ldsm_x2(smem_u32(hlo) + off, bl[kk][0], bl[kk][1]);
        }
        float hs0[C::NB > 0 ? C::NB : 1], hs1[C::NB > 0 ? C::NB : 1];
        if constexpr (C::QUANT) {
#pragma unroll
            for (int bb = 0; bb < C::NB; ++bb) {
                hs0[bb] = sm.hsum[t0 * 2 + bb];
                hs1[bb] = sm.hsum[t1 * 2 + bb];
            }
        }

        // --------------------------------------- phase B: down + combine
        for (int st = 0; st < nB; ++st, ++it) {
            const int slot = it % ns;
            const bool ok = wait_full(slot, (it / ns) & 1);
            const uint8_t* stage = ring + static_cast<size_t>(slot) * C::STAGE;
            const int j0 = st * C::RJ;
            const int rows = min(C::RJ, d - j0);
            if (ok) {
                for (int rgb = warp; rgb < rows / 16; rgb += kConsumerWarps) {
                    float c[4] = {0.f, 0.f, 0.f, 0.f};
                    if constexpr (!C::QUANT) {
                        const uint32_t tile = smem_u32(stage);
                        const int m = lane >> 3, r = lane & 7;
                        const uint32_t arow = rgb * 16 + ((m & 1) << 3) + r;
#pragma unroll
                        for (int kk = 0; kk < C::RG; ++kk) {
                            uint32_t a0, a1, a2, a3;
                            ldsm_x4(tile + swz_offset(arow, kk * 2 + (m >> 1), FS * 2), a0, a1, a2, a3);
                            if constexpr (C::HALF_DOWN) {
                                mma_f16_16816_acc(c, a0, a1, a2, a3, bh[kk][0], bh[kk][1]);
                                mma_f16_16816_acc(c, a0, a1, a2, a3, bl[kk][0], bl[kk][1]);
                            } else {
                                mma_bf16_16816(c, a0, a1, a2, a3, bh[kk][0], bh[kk][1]);
                                mma_bf16_16816(c, a0, a1, a2, a3, bl[kk][0], bl[kk][1]);
                            }
                        }
                    } else {
                        constexpr int QB = kQuantDownBoxRows;
                        const uint8_t* bbase = stage + (rgb / (QB / 16)) * (C::NB * QB * C::BR);
                        const uint32_t* codes = reinterpret_cast<const uint32_t*>(bbase);   // [NB][128][CB]
                        const __half* scl = reinterpret_cast<const __half*>(bbase + C::NB * QB * C::CB);
                        const int rib = (rgb % (QB / 16)) * 16 + g;
                        {
#pragma unroll
                        for (int bb = 0; bb < C::NB; ++bb) {
                            const uint32_t* row = codes + (bb * QB + rib) * (C::CB / 4);
                            // Q5_0; the accumulator starts at -144 * sum(hi + lo) of the block
                            float v[4], s0, s8;
                            uint32_t h0, h8;
                            q5_aux(reinterpret_cast<const uint8_t*>(scl), bb, QB, rib, s0, s8, h0, h8);
                            q5_block_b(row, row + 8 * (C::CB / 4), q5_lane_bits(h0, tig),
                                       q5_lane_bits(h8, tig), tig, hs0[bb], hs1[bb], bh[2 * bb],
                                       bh[2 * bb + 1], bl[2 * bb], bl[2 * bb + 1], v);
                            c[0] = fmaf(s0, v[0], c[0]);
                            c[1] = fmaf(s0, v[1], c[1]);
                            c[2] = fmaf(s8, v[2], c[2]);
                            c[3] = fmaf(s8, v[3], c[3]);
                        }
                        }
                    }
                    const int j = j0 + rgb * 16 + g;
                    if (v0) {
                        red_add_f32(a.out + static_cast<size_t>(tok0) * d + j, w0 * c[0]);
                        red_add_f32(a.out + static_cast<size_t>(tok0) * d + j + 8, w0 * c[2]);
                    }
                    if (v1) {
                        red_add_f32(a.out + static_cast<size_t>(tok1) * d + j, w1 * c[1]);
                        red_add_f32(a.out + static_cast<size_t>(tok1) * d + j + 8, w1 * c[3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
    }
}


// q6_K: the four fp16 operand registers of one row's 8 codes, from its code
// word w (low 4 bits, packed like Q4_0) and its word e of high-bit pairs
// (the pair of the code in nibble n at bit {4, 8, 6, 10, 20, 24, 22, 26}[n]):
// each register is two values 1024 + q (k % 16 < 8) or 64 + q (k % 16 >= 8),
// q = low + 16 * high in 0..63, exact in fp16 (see q4h_lo).  r0, r1 feed the
// block's first 16-wide half (sub-block), r2, r3 the second.
__device__ __forceinline__ void q6h_regs(uint32_t w, uint32_t e, uint32_t& r0, uint32_t& r1,
                                         uint32_t& r2, uint32_t& r3) {
    r0 = q4h_lo(w) | (e & 0x00300030u);
    r1 = q4h_hi(w) | (e & 0x03000300u);
    const uint32_t u = w >> 8, f = e >> 2;
    r2 = q4h_lo(u) | (f & 0x00300030u);
    r3 = q4h_hi(u) | (f & 0x03000300u);
}

// The four sub-block scales d * sc of rows r and r + 8 of one q6_K block:
// sw holds the int8 sub-scales (row r: k 0-15, 16-31; row r + 8: the same).
__device__ __forceinline__ void q6_scales(uint32_t sw, float dr, float dr8, float& s00, float& s01,
                                          float& s80, float& s81) {
    s00 = dr * static_cast<float>(static_cast<int8_t>(sw & 0xffu));
    s01 = dr * static_cast<float>(static_cast<int8_t>((sw >> 8) & 0xffu));
    s80 = dr8 * static_cast<float>(static_cast<int8_t>((sw >> 16) & 0xffu));
    s81 = dr8 * static_cast<float>(static_cast<int8_t>(sw >> 24));
}

// The experts pipeline for the weight formats that feed fp16 operands to
// the tensor cores (F16: Q4_0, Q8_0, q6_K): phase A streams row groups instead of
// block columns.  A phase-A stage is 16 consecutive rows of the gate or up
// slice over the whole reduction dim (KC <= 64 block columns per stage, more
// stages per row group when d > 2048), and consumer warp w owns block
// columns w, w + 16, w + 32, w + 48 of every stage.  The x fragments and
// block corrections of those columns therefore stay in registers for the
// whole unit; each warp keeps the partial sums of every row group and both
// matrices, and one reduction over the 16 warps follows phase A.  Phase B
// (down matrix, combine) works like experts_pipeline's.
//
// The hot loops are written for the instruction count: full stages (64
// block columns, or RJ down rows) address shared memory through one 32-bit
// per-lane base plus compile-time offsets, the ring slot and phase advance
// incrementally (no division by the ring depth), and nothing branches per
// block.  Partial stages (d not a multiple of 2048, the last down rows) take
// a general path.
//
// Stage layouts.  Q4_0 / Q8_0 phase A: codes [KC][16 rows][CB = 16 / 32 B],
// scales [KC][16] fp16; phase B per 256-row box: codes [NB][256][CB],
// scales [NB][256].
// q6_K phase A: codes [KC][16][16 B], records [KC][160 B], super-block scales
// [KC/8][16] fp16; phase B per 256-row box: codes [NB][256][16 B], records
// [NB][16][160 B], super-block scales [256] fp16 (a slice of FS <= 256
// columns lies in one super-block).
template <int FS, int WF>
__device__ __forceinline__ void experts_pipeline_rows(const DecodeArgs& a, const DecodeSmem& sm,
                                                      const WorkView& wv) {
    using C = DecodeCfg<FS, WF>;
    static_assert(C::F16, "row-streaming phase A serves the fp16-operand formats");
    static_assert(FS == 32, "row-streaming slices are 32 rows");
    constexpr int QB = kQuantDownBoxRows;
    // phase-B bytes of one 256-row box
    constexpr int BOXB = C::Q6 ? C::NB * QB * 16 + C::NB * (QB / 16) * 160 + QB * 2
                               : C::NB * QB * C::BR;
    static_assert((C::RJ / QB) * BOXB <= C::STAGE, "phase-B boxes fit a stage");
    constexpr int RGW = C::RJ / 16 / kConsumerWarps;      // row groups per warp, full phase-B stage
    static_assert(RGW * kConsumerWarps * 16 == C::RJ && C::RJ % QB == 0, "phase-B split");
    constexpr int KCMAX = C::KCMAX;
    // offsets inside a full phase-A stage (KC = 64)
    constexpr uint32_t A_SCL = 16 * KCMAX * C::CB;                 // Q4_0 / Q8_0 scales
    constexpr uint32_t RGB = 16 * C::CB;                           // codes of a 16-row group
    constexpr uint32_t A_REC = 16 * KCMAX * 16;                    // q6_K records
    constexpr uint32_t A_D = KCMAX * (16 * 16 + 160);              // q6_K super-block scales
    const int ns = a.n_stages;
    uint8_t* ring = sm.ring;
    float* gu = sm.gu;
    uint64_t* full = sm.full;
    uint64_t* empty = sm.empty;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = a.d, E = a.E;
    const int nkb = d / 32;
    const int KC = a.kt;                              // block columns per phase-A stage
    const int nch = (nkb + KC - 1) / KC;              // phase-A stages per row group and matrix
    const int stage_a = C::Q6 ? KC * (16 * 16 + 160) + (KC / 8) * 32 : 16 * KC * C::BR;
    const int n_routed = wv.n_routed, n_shared = wv.n_shared;
    const int sl_r = a.F / FS, sl_s = a.S ? a.Fs / FS : 0;
    const int n_su = n_shared * sl_s;
    const int n_units = n_su + n_routed * sl_r;
    const int nA = 2 * C::RG * nch;
    const int nB = (d + C::RJ - 1) / C::RJ;
    volatile int* abort_flag = &sm.tail->abort_flag;
    const int u_begin = static_cast<int>(blockIdx.x);
    const int u_step = static_cast<int>(gridDim.x);
    auto unit_item = [&](int u, int& ii, int& sl) {
        if (u < n_su) { ii = n_routed + u / sl_s; sl = u % sl_s; }
        else { const int v = u - n_su; ii = v / sl_r; sl = v % sl_r; }
    };

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&a.tm_gate); prefetch_tensormap(&a.tm_up);
            prefetch_tensormap(&a.tm_down);
            prefetch_tensormap(&a.tm_gate_sc); prefetch_tensormap(&a.tm_up_sc);
            prefetch_tensormap(&a.tm_down_sc);
            if constexpr (C::Q6) {
                prefetch_tensormap(&a.tm_gate_d); prefetch_tensormap(&a.tm_up_d);
                prefetch_tensormap(&a.tm_down_d);
            }
            if (a.S) {
                prefetch_tensormap(&a.tm_sgate); prefetch_tensormap(&a.tm_sup);
                prefetch_tensormap(&a.tm_sdown); prefetch_tensormap(&a.tm_sgate_sc);
                prefetch_tensormap(&a.tm_sup_sc); prefetch_tensormap(&a.tm_sdown_sc);
                if constexpr (C::Q6) {
                    prefetch_tensormap(&a.tm_sgate_d); prefetch_tensormap(&a.tm_sup_d);
                    prefetch_tensormap(&a.tm_sdown_d);
                }
            }
            const uint64_t pol = l2_policy_evict_first();
            uint32_t it = 0;                  // stages issued
            int slot = 0;
            uint32_t ph = 0;                  // phase of the slot's current fill
            bool ok = true;
            for (int u = u_begin; u < n_units && ok; u += u_step) {
                int ii, sl;
                unit_item(u, ii, sl);
                const WorkItem item = wv.items[ii];
                const bool shared = item.expert >= E;
                const int ex = shared ? item.expert - E : item.expert;
                const int Fh = shared ? a.Fs : a.F;
                const int f0 = sl * FS;
                for (int st = 0; st < nA + nB && ok; ++st, ++it) {
                    if (it >= static_cast<uint32_t>(ns)) {
                        if (*abort_flag || !mbar_wait_bounded_sleep(&empty[slot], ph ^ 1u)) {
                            atomicOr(a.err, kErrTimeout); *abort_flag = 1; ok = false; break;
                        }
                    }
                    uint8_t* dst = ring + static_cast<size_t>(slot) * C::STAGE;
                    if (st < nA) {
                        // stage (row group rg, matrix mat, k chunk c)
                        const int c = st % nch, mat = (st / nch) & 1, rg = st / (2 * nch);
                        const CUtensorMap* mc = mat ? (shared ? &a.tm_sup : &a.tm_up)
                                                    : (shared ? &a.tm_sgate : &a.tm_gate);
                        const CUtensorMap* ms = mat ? (shared ? &a.tm_sup_sc : &a.tm_up_sc)
                                                    : (shared ? &a.tm_sgate_sc : &a.tm_gate_sc);
                        const int c2 = ex * nkb + c * KC;
                        const int r0 = f0 + rg * 16;
                        mbar_arrive_expect_tx(&full[slot], stage_a);
                        tma_load_3d(dst, mc, &full[slot], 0, r0 / 16, c2, pol);   // 16-row groups
                        if constexpr (C::Q6) {
                            const CUtensorMap* md = mat ? (shared ? &a.tm_sup_d : &a.tm_up_d)
                                                        : (shared ? &a.tm_sgate_d : &a.tm_gate_d);
                            tma_load_3d(dst + 16 * KC * 16, ms, &full[slot], 0, r0 / 16, c2, pol);
                            tma_load_2d(dst + KC * (16 * 16 + 160), md, &full[slot], r0,
                                        ex * (nkb / 8) + c * (KC / 8), pol);
                        } else {
                            tma_load_2d(dst + 16 * KC * C::CB, ms, &full[slot], r0, c2, pol);
                        }
                    } else {
                        const CUtensorMap* md = shared ? &a.tm_sdown : &a.tm_down;
                        const CUtensorMap* mds = shared ? &a.tm_sdown_sc : &a.tm_down_sc;
                        const int j0 = (st - nA) * C::RJ;
                        const int nbox = (min(C::RJ, d - j0) + QB - 1) / QB;
                        const int c2 = ex * (Fh / 32) + f0 / 32;
                        mbar_arrive_expect_tx(&full[slot], nbox * BOXB);
                        for (int b = 0; b < nbox; ++b) {
                            uint8_t* bd = dst + b * BOXB;
                            tma_load_3d(bd, md, &full[slot], 0, (j0 + QB * b) / 16, c2, pol);
                            if constexpr (C::Q6) {
                                const CUtensorMap* mdd = shared ? &a.tm_sdown_d : &a.tm_down_d;
                                tma_load_3d(bd + C::NB * QB * 16, mds, &full[slot], 0, (j0 + QB * b) / 16,
                                            c2, pol);
                                tma_load_2d(bd + C::NB * QB * 16 + C::NB * (QB / 16) * 160, mdd, &full[slot],
                                            j0 + QB * b, ex * (Fh / 256) + f0 / 256, pol);
                            } else {
                                tma_load_2d(bd + C::NB * QB * C::CB, mds, &full[slot], j0 + QB * b, c2,
                                            pol);
                            }
                        }
                    }
                    if (++slot == ns) { slot = 0; ph ^= 1u; }
                }
            }
            // drain: every issued stage must land before the CTA may exit
            const uint32_t first = it > static_cast<uint32_t>(ns) ? it - ns : 0;
            for (uint32_t q = first; q < it; ++q)
                if (!mbar_wait_bounded_sleep(&full[q % ns], (q / ns) & 1)) {
                    atomicOr(a.err, kErrTimeout);
                    break;
                }
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int g = lane >> 2, tig = lane & 3;
    const uint32_t xs_u = smem_u32(sm.xs);
    const uint32_t ring_u = smem_u32(ring);
    constexpr int NC = C::Q6 ? 2 : 1;                 // corrections per block (per 16-k sub-block)
    // this lane's bases inside a stage: block column (phase A) or row group
    // (phase B) `warp`, row g, code word tig
    const uint32_t lane_code = warp * RGB + g * C::CB + tig * (C::CB / 4);
    const uint32_t lane_a_scl = A_SCL + warp * 32 + g * 2;
    const uint32_t lane_a_rec = A_REC + warp * 160 + (4 * g + tig) * 4;
    const uint32_t lane_a_sub = A_REC + warp * 160 + 128 + g * 4;
    const uint32_t lane_a_d = A_D + (warp >> 3) * 32 + g * 2;
    const uint32_t lane_b_scl = C::NB * QB * C::CB + warp * 32 + g * 2;
    const uint32_t lane_b_rec = C::NB * QB * 16 + warp * 160 + (4 * g + tig) * 4;
    const uint32_t lane_b_sub = C::NB * QB * 16 + warp * 160 + 128 + g * 4;
    const uint32_t lane_b_d = C::NB * QB * 16 + C::NB * (QB / 16) * 160 + warp * 32 + g * 2;
    int slot = 0;
    uint32_t ph = 0;
    auto wait_full = [&]() -> bool {
        // fast path: the stage has landed (the abort flag matters only to a
        // wait that would otherwise run into the limit)
        if (__all_sync(0xffffffffu, mbar_try_wait(&full[slot], ph))) return true;
        if (__any_sync(0xffffffffu, *abort_flag != 0)) return false;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded_sleep(&full[slot], ph));
        if (!ok && lane == 0) {
            atomicOr(a.err, kErrTimeout);
            *abort_flag = 1;
        }
        return ok;
    };
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (++slot == ns) { slot = 0; ph ^= 1u; }
    };

    for (int u = u_begin; u < n_units; u += u_step) {
        int ii, sl;
        unit_item(u, ii, sl);
        const WorkItem item = wv.items[ii];
        const bool shared = item.expert >= E;
        const int ntok = min(item.count, kDecodeTok);
        auto tok_of = [&](int n) -> int {
            return n < ntok ? (shared ? n : wv.slot_token[item.slot_begin + n]) : 0;
        };
        auto w_of = [&](int n) -> float {
            return n < ntok ? (shared ? 1.f : wv.slot_w[item.slot_begin + n]) : 0.f;
        };
        const uint32_t xrow = xs_u + tok_of(lane & 7) * a.xs_stride;   // B row of this lane
        const int t0 = 2 * tig, t1 = t0 + 1;
        const int tok0 = tok_of(t0), tok1 = tok_of(t1);
        const float w0 = w_of(t0), w1 = w_of(t1);
        const bool v0 = t0 < ntok, v1 = t1 < ntok;

        // x fragments and corrections of this warp's block columns of chunk c
        uint32_t xf[C::NBW][4];
        float xc0[C::NBW][NC], xc1[C::NBW][NC];
        auto load_x = [&](int c) {
#pragma unroll
            for (int i = 0; i < C::NBW; ++i) {
                const int kb = c * KC + warp + kConsumerWarps * i;
                const bool in = (warp + kConsumerWarps * i) < KC && kb < nkb;
                const int kbs = in ? kb : 0;
                ldsm_x4(xrow + (kbs * 32 + (lane >> 3) * 8) * 2, xf[i][0], xf[i][1], xf[i][2], xf[i][3]);
#pragma unroll
                for (int j = 0; j < NC; ++j) {
                    xc0[i][j] = sm.xsum[(tok0 * nkb + kbs) * NC + j];
                    xc1[i][j] = sm.xsum[(tok1 * nkb + kbs) * NC + j];
                }
            }
        };
        if (nch == 1) load_x(0);

        // one 16 x 32 block: x0 / x8 code words of rows g / g+8, e its q6_K
        // high-bit word, sw the sub-scales, s0 / s8 (Q4_0) or dr / dr8 (q6_K)
        // the scales; its two 16-wide halves are independent MMAs
        // (Q4_0: the second half's MMA accumulates onto the first's, which
        // saves the adds and operand moves of a second accumulator)
        auto block_q4 = [&](int i, uint32_t x0, uint32_t x8, float s0, float s8, float (&ac)[4]) {
            const uint32_t u0 = x0 >> 8, u8 = x8 >> 8;
            float va[4];
            mma_f16_16816(va, q4h_lo(x0), q4h_lo(x8), q4h_hi(x0), q4h_hi(x8), xf[i][0], xf[i][1],
                          xc0[i][0], xc1[i][0], xc0[i][0], xc1[i][0]);
            mma_f16_16816_acc(va, q4h_lo(u0), q4h_lo(u8), q4h_hi(u0), q4h_hi(u8), xf[i][2], xf[i][3]);
            ac[0] = fmaf(s0, va[0], ac[0]);
            ac[1] = fmaf(s0, va[1], ac[1]);
            ac[2] = fmaf(s8, va[2], ac[2]);
            ac[3] = fmaf(s8, va[3], ac[3]);
        };
        // Q8_0: x0 / x8 the lane's two words (block halves) of rows g / g+8
        auto block_q8 = [&](int i, uint2 x0, uint2 x8, float s0, float s8, float (&ac)[4]) {
            float va[4];
            mma_f16_16816(va, q8h_lo(x0.x), q8h_lo(x8.x), q8h_hi(x0.x), q8h_hi(x8.x), xf[i][0], xf[i][1],
                          xc0[i][0], xc1[i][0], xc0[i][0], xc1[i][0]);
            mma_f16_16816_acc(va, q8h_lo(x0.y), q8h_lo(x8.y), q8h_hi(x0.y), q8h_hi(x8.y), xf[i][2],
                              xf[i][3]);
            ac[0] = fmaf(s0, va[0], ac[0]);
            ac[1] = fmaf(s0, va[1], ac[1]);
            ac[2] = fmaf(s8, va[2], ac[2]);
            ac[3] = fmaf(s8, va[3], ac[3]);
        };
        auto block_q6 = [&](int i, uint32_t x0, uint32_t x8, uint32_t e, uint32_t sw, float dr, float dr8,
                            float (&ac)[4]) {
            uint32_t p0, p1, p2, p3, q0, q1, q2, q3;
            q6h_regs(x0, e, p0, p1, p2, p3);
            q6h_regs(x8, __funnelshift_r(e, e, 8), q0, q1, q2, q3);
            float va[4], vb[4];
            mma_f16_16816(va, p0, q0, p1, q1, xf[i][0], xf[i][1], xc0[i][0], xc1[i][0], xc0[i][0],
                          xc1[i][0]);
            mma_f16_16816(vb, p2, q2, p3, q3, xf[i][2], xf[i][3], xc0[i][NC - 1], xc1[i][NC - 1],
                          xc0[i][NC - 1], xc1[i][NC - 1]);
            float s00, s01, s80, s81;
            q6_scales(sw, dr, dr8, s00, s01, s80, s81);
            ac[0] = fmaf(s00, va[0], fmaf(s01, vb[0], ac[0]));
            ac[1] = fmaf(s00, va[1], fmaf(s01, vb[1], ac[1]));
            ac[2] = fmaf(s80, va[2], fmaf(s81, vb[2], ac[2]));
            ac[3] = fmaf(s80, va[3], fmaf(s81, vb[3], ac[3]));
        };

        // ------------------------------------------- phase A: gate and up
        // stage group sq = (row group rg, matrix mat); one loop body for all
        // of them (not unrolled: the unit loop stays small enough for the
        // instruction cache), each group's sums stored once it is complete
        const bool fast_a = KC == KCMAX;
#pragma unroll 1
        for (int sq = 0; sq < 2 * C::RG; ++sq) {
            const int rg = sq >> 1, mat = sq & 1;
            float ac[4] = {0.f, 0.f, 0.f, 0.f};
            for (int c = 0; c < nch; ++c) {
                const bool ok = wait_full();
                if (ok) {
                    if (nch > 1) load_x(c);
                    const uint32_t st_u = ring_u + slot * C::STAGE;
                    if (__builtin_expect(fast_a && (c + 1) * KCMAX <= nkb, 1)) {
                        // all four block columns of this warp are in the stage
#pragma unroll
                        for (int i = 0; i < C::NBW; ++i) {
                            const uint32_t cb = st_u + lane_code + i * (16 * RGB);
                            if constexpr (C::Q8) {
                                const uint2 x0 = lds_u32x2(cb), x8 = lds_u32x2(cb + 8 * C::CB);
                                const float s0 = lds_f16_as_f32(st_u + lane_a_scl + i * 512);
                                const float s8 = lds_f16_as_f32(st_u + lane_a_scl + i * 512 + 16);
                                block_q8(i, x0, x8, s0, s8, ac);
                                continue;
                            }
                            const uint32_t x0 = lds_u32(cb), x8 = lds_u32(cb + 128);
                            if constexpr (C::Q6) {
                                const uint32_t e = lds_u32(st_u + lane_a_rec + i * (16 * 160));
                                const uint32_t sw = lds_u32(st_u + lane_a_sub + i * (16 * 160));
                                const float dr = lds_f16_as_f32(st_u + lane_a_d + i * 64);
                                const float dr8 = lds_f16_as_f32(st_u + lane_a_d + i * 64 + 16);
                                block_q6(i, x0, x8, e, sw, dr, dr8, ac);
                            } else {
                                const float s0 = lds_f16_as_f32(st_u + lane_a_scl + i * 512);
                                const float s8 = lds_f16_as_f32(st_u + lane_a_scl + i * 512 + 16);
                                block_q4(i, x0, x8, s0, s8, ac);
                            }
                        }
                    } else {
                        const uint8_t* stage = ring + static_cast<size_t>(slot) * C::STAGE;
                        const uint32_t* codes = reinterpret_cast<const uint32_t*>(stage);
#pragma unroll
                        for (int i = 0; i < C::NBW; ++i) {
                            const int bl = warp + kConsumerWarps * i;
                            if (bl < KC && c * KC + bl < nkb) {
                                if constexpr (C::Q8) {
                                    const uint2* row = reinterpret_cast<const uint2*>(codes) + (bl * 16 + g) * 4;
                                    const __half* scl =
                                        reinterpret_cast<const __half*>(stage + 16 * KC * C::CB);
                                    block_q8(i, row[tig], row[32 + tig], __half2float(scl[bl * 16 + g]),
                                             __half2float(scl[bl * 16 + g + 8]), ac);
                                    continue;
                                }
                                const uint32_t* row = codes + (bl * 16 + g) * 4;
                                const uint32_t x0 = row[tig], x8 = row[32 + tig];
                                if constexpr (C::Q6) {
                                    const uint32_t* rec =
                                        reinterpret_cast<const uint32_t*>(stage + 16 * KC * 16 + bl * 160);
                                    const __half* dsm =
                                        reinterpret_cast<const __half*>(stage + KC * (16 * 16 + 160));
                                    block_q6(i, x0, x8, rec[4 * g + tig], rec[32 + g],
                                             __half2float(dsm[(bl >> 3) * 16 + g]),
                                             __half2float(dsm[(bl >> 3) * 16 + g + 8]), ac);
                                } else {
                                    const __half* scl =
                                        reinterpret_cast<const __half*>(stage + 16 * KC * C::CB);
                                    block_q4(i, x0, x8, __half2float(scl[bl * 16 + g]),
                                             __half2float(scl[bl * 16 + g + 8]), ac);
                                }
                            }
                        }
                    }
                }
                release();
            }
            // this warp's partial sums of the group, [warp][mat][t][f] (row
            // stride GS)
            float* gq = gu + (warp * 2 + mat) * kDecodeTok * C::GS;
            const int r = rg * 16 + g;
            gq[t0 * C::GS + r] = ac[0];
            gq[t1 * C::GS + r] = ac[1];
            gq[t0 * C::GS + r + 8] = ac[2];
            gq[t1 * C::GS + r + 8] = ac[3];
        }
        named_bar_sync(1, kConsumers);
        // h = SiLU(gate) * up as an fp16 pair hi + lo for the token columns in
        // use (the rest are zero); one warp covers 32 consecutive f of one
        // column, i.e. one block of the down matrix.  The down block's (q6_K:
        // sub-block's) accumulator starts at -sum((base_f + offset)(hi + lo))
        // (Q8_0: -1152 sum(hi + lo)).
        for (int idx = tid; idx < FS * kDecodeTok; idx += kConsumers) {
            const int t = idx / FS, f = idx % FS;
            __half hi = __float2half_rn(0.f), lo = hi;
            float hs = 0.f;
            if (t < ntok) {
                float gv = 0.f, uv = 0.f;
#pragma unroll
                for (int q = 0; q < kConsumerWarps; ++q) {
                    gv += gu[((q * 2 + 0) * kDecodeTok + t) * C::GS + f];
                    uv += gu[((q * 2 + 1) * kDecodeTok + t) * C::GS + f];
                }
                const float h = gv / (1.f + expf(-gv)) * uv;
                hi = __float2half_rn(h);
                lo = __float2half_rn(h - __half2float(hi));
                const float base = (f & 15) < 8 ? kF16BaseLo : kF16BaseHi;
                hs = (C::Q8 ? kQ8Offset : base + (C::Q6 ? 32.f : 8.f)) *
                     (__half2float(hi) + __half2float(lo));
            }
            reinterpret_cast<__half*>(sm.hhi)[t * C::HS + f] = hi;
            reinterpret_cast<__half*>(sm.hlo)[t * C::HS + f] = lo;
            if constexpr (C::Q6) {
#pragma unroll
                for (int off = 8; off > 0; off >>= 1) hs += __shfl_xor_sync(0xffffffffu, hs, off);
                if ((lane & 15) == 0) sm.hsum[t * 4 + f / 16] = -hs;
            } else {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) hs += __shfl_xor_sync(0xffffffffu, hs, off);
                if (lane == 0) sm.hsum[t * 4 + f / 32] = -hs;
            }
        }
        named_bar_sync(1, kConsumers);
        uint32_t bh[C::RG][2], bl[C::RG][2];
#pragma unroll
        for (int kk = 0; kk < C::RG; ++kk) {
            const uint32_t off = ((lane & 7) * C::HS + kk * 16 + ((lane >> 3) & 1) * 8) * 2;
            ldsm_x2(smem_u32(sm.hhi) + off, bh[kk][0], bh[kk][1]);
            ldsm_x2(smem_u32(sm.hlo) + off, bl[kk][0], bl[kk][1]);
        }
        // corrections of the down blocks (Q4_0, Q8_0) or sub-blocks (q6_K), columns t0, t1
        constexpr int NH = C::Q6 ? 2 * C::NB : C::NB;
        float hs0[NH], hs1[NH];
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            hs0[j] = sm.hsum[t0 * 4 + j];
            hs1[j] = sm.hsum[t1 * 4 + j];
        }

        // --------------------------------------- phase B: down + combine
        // one 16-row group, given its 32-bit stage addresses: the block's
        // halves (q6_K: sub-blocks) are independent MMA chains (hi part, then
        // lo part of h)
        auto rowgroup = [&](uint32_t code_u, uint32_t scl_u, uint32_t rec_u, uint32_t sub_u,
                            uint32_t d_u, float (&c)[4]) {
            c[0] = c[1] = c[2] = c[3] = 0.f;
#pragma unroll
            for (int bb = 0; bb < C::NB; ++bb) {
                if constexpr (C::Q8) {
                    const uint2 x0 = lds_u32x2(code_u + bb * (QB * C::CB));
                    const uint2 x8 = lds_u32x2(code_u + bb * (QB * C::CB) + 8 * C::CB);
                    const uint32_t p0 = q8h_lo(x0.x), q0 = q8h_lo(x8.x);
                    const uint32_t p1 = q8h_hi(x0.x), q1 = q8h_hi(x8.x);
                    const uint32_t p2 = q8h_lo(x0.y), q2 = q8h_lo(x8.y);
                    const uint32_t p3 = q8h_hi(x0.y), q3 = q8h_hi(x8.y);
                    float va[4];
                    mma_f16_16816(va, p0, q0, p1, q1, bh[2 * bb][0], bh[2 * bb][1],
                                  hs0[bb], hs1[bb], hs0[bb], hs1[bb]);
                    mma_f16_16816_acc(va, p2, q2, p3, q3, bh[2 * bb + 1][0], bh[2 * bb + 1][1]);
                    mma_f16_16816_acc(va, p0, q0, p1, q1, bl[2 * bb][0], bl[2 * bb][1]);
                    mma_f16_16816_acc(va, p2, q2, p3, q3, bl[2 * bb + 1][0], bl[2 * bb + 1][1]);
                    const float s0 = lds_f16_as_f32(scl_u + bb * (QB * 2));
                    const float s8 = lds_f16_as_f32(scl_u + bb * (QB * 2) + 16);
                    c[0] = fmaf(s0, va[0], c[0]);
                    c[1] = fmaf(s0, va[1], c[1]);
                    c[2] = fmaf(s8, va[2], c[2]);
                    c[3] = fmaf(s8, va[3], c[3]);
                    continue;
                }
                const uint32_t x0 = lds_u32(code_u + bb * (QB * 16));
                const uint32_t x8 = lds_u32(code_u + bb * (QB * 16) + 128);
                if constexpr (C::Q6) {
                    const uint32_t e = lds_u32(rec_u + bb * (16 * 160));
                    uint32_t p0, p1, p2, p3, q0, q1, q2, q3;
                    q6h_regs(x0, e, p0, p1, p2, p3);
                    q6h_regs(x8, __funnelshift_r(e, e, 8), q0, q1, q2, q3);
                    float va[4], vb[4];
                    mma_f16_16816(va, p0, q0, p1, q1, bh[2 * bb][0], bh[2 * bb][1],
                                  hs0[2 * bb], hs1[2 * bb], hs0[2 * bb], hs1[2 * bb]);
                    mma_f16_16816(vb, p2, q2, p3, q3, bh[2 * bb + 1][0], bh[2 * bb + 1][1],
                                  hs0[2 * bb + 1], hs1[2 * bb + 1], hs0[2 * bb + 1], hs1[2 * bb + 1]);
                    mma_f16_16816_acc(va, p0, q0, p1, q1, bl[2 * bb][0], bl[2 * bb][1]);
                    mma_f16_16816_acc(vb, p2, q2, p3, q3, bl[2 * bb + 1][0], bl[2 * bb + 1][1]);
                    float s00, s01, s80, s81;
                    q6_scales(lds_u32(sub_u + bb * (16 * 160)), lds_f16_as_f32(d_u),
                              lds_f16_as_f32(d_u + 16), s00, s01, s80, s81);
                    c[0] = fmaf(s00, va[0], fmaf(s01, vb[0], c[0]));
                    c[1] = fmaf(s00, va[1], fmaf(s01, vb[1], c[1]));
                    c[2] = fmaf(s80, va[2], fmaf(s81, vb[2], c[2]));
                    c[3] = fmaf(s80, va[3], fmaf(s81, vb[3], c[3]));
                } else {
                    const uint32_t u0 = x0 >> 8, u8 = x8 >> 8;
                    const uint32_t p0 = q4h_lo(x0), q0 = q4h_lo(x8);
                    const uint32_t p1 = q4h_hi(x0), q1 = q4h_hi(x8);
                    const uint32_t p2 = q4h_lo(u0), q2 = q4h_lo(u8);
                    const uint32_t p3 = q4h_hi(u0), q3 = q4h_hi(u8);
                    // one accumulator chain: both halves of h hi, then of h lo
                    float va[4];
                    mma_f16_16816(va, p0, q0, p1, q1, bh[2 * bb][0], bh[2 * bb][1],
                                  hs0[bb], hs1[bb], hs0[bb], hs1[bb]);
                    mma_f16_16816_acc(va, p2, q2, p3, q3, bh[2 * bb + 1][0], bh[2 * bb + 1][1]);
                    mma_f16_16816_acc(va, p0, q0, p1, q1, bl[2 * bb][0], bl[2 * bb][1]);
                    mma_f16_16816_acc(va, p2, q2, p3, q3, bl[2 * bb + 1][0], bl[2 * bb + 1][1]);
                    const float s0 = lds_f16_as_f32(scl_u + bb * (QB * 2));
                    const float s8 = lds_f16_as_f32(scl_u + bb * (QB * 2) + 16);
                    c[0] = fmaf(s0, va[0], c[0]);
                    c[1] = fmaf(s0, va[1], c[1]);
                    c[2] = fmaf(s8, va[2], c[2]);
                    c[3] = fmaf(s8, va[3], c[3]);
                }
            }
        };
        float* const out0 = a.out + static_cast<size_t>(tok0) * d;   // this lane's two token rows
        float* const out1 = a.out + static_cast<size_t>(tok1) * d;
        auto combine = [&](int j, const float (&c)[4]) {      // j: first row of the group + g
            if (v0) red_add_f32_rows8(out0 + j, w0 * c[0], w0 * c[2]);
            if (v1) red_add_f32_rows8(out1 + j, w1 * c[1], w1 * c[3]);
        };
        for (int st = 0; st < nB; ++st) {
            const bool ok = wait_full();
            const int j0 = st * C::RJ;
            const int rows = min(C::RJ, d - j0);
            if (ok) {
                const uint32_t st_u = ring_u + slot * C::STAGE;
                if (__builtin_expect(rows == C::RJ, 1)) {
                    // row group warp + 16 q (q < RGW) sits in box q at group
                    // `warp` (two row groups per loop body: independent MMA
                    // chains to overlap, and still a small loop)
#pragma unroll 2
                    for (int q = 0; q < RGW; ++q) {
                        const uint32_t bq = st_u + q * BOXB;
                        float c[4];
                        rowgroup(bq + lane_code, bq + lane_b_scl, bq + lane_b_rec, bq + lane_b_sub,
                                 bq + lane_b_d, c);
                        combine(j0 + (warp + kConsumerWarps * q) * 16 + g, c);
                    }
                } else {
                    for (int rgb = warp; rgb < rows / 16; rgb += kConsumerWarps) {
                        const int grp = rgb % (QB / 16);
                        const uint32_t bq = st_u + (rgb / (QB / 16)) * BOXB;
                        const uint32_t lc = grp * RGB + g * C::CB + tig * (C::CB / 4);
                        float c[4];
                        rowgroup(bq + lc, bq + C::NB * QB * C::CB + grp * 32 + g * 2,
                                 bq + C::NB * QB * 16 + grp * 160 + (4 * g + tig) * 4,
                                 bq + C::NB * QB * 16 + grp * 160 + 128 + g * 4,
                                 bq + C::NB * QB * 16 + C::NB * (QB / 16) * 160 + grp * 32 + g * 2, c);
                        combine(j0 + rgb * 16 + g, c);
                    }
                }
            }
            release();
        }
    }
}

// The experts pipeline of the format: row-streaming for the fp16-operand
// formats, block-column stages for the others.
template <int FS, int WF>
__device__ __forceinline__ void run_experts(const DecodeArgs& a, const DecodeSmem& sm,
                                            const WorkView& wv) {
    if constexpr (DecodeCfg<FS, WF>::F16) experts_pipeline_rows<FS, WF>(a, sm, wv);
    else experts_pipeline<FS, WF>(a, sm, wv);
}

template <int FS, int WF>
__global__ void __launch_bounds__(kDecodeThreads, 1)
decode_experts_kernel(const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const DecodeSmem sm = decode_smem<FS, WF>(smem_raw, a);
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.n_stages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        sm.tail->abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < kConsumers) stage_x<WF>(a, sm, threadIdx.x);
    __syncthreads();
    const WorkView wv{a.n_items[0], a.n_items[1], a.items, a.slot_token, a.slot_w};
    run_experts<FS, WF>(a, sm, wv);
}

// ====================================================== fused decode ===
// One cooperative launch for the whole layer (T <= 8):
//   R  every CTA computes the router logits of experts b, b+G, ... (fp32 FMA,
//      each dot product split over the 16 consumer warps and summed in a
//      fixed order) and publishes them, each as one 64-bit word that also
//      holds this launch's tag; the producer warp zero-fills the CTA's share
//      of `out` meanwhile;
//   T  every CTA reads all T x E logit words, waiting (bounded) until each
//      carries this launch's tag, and computes the same top-k, renormalised
//      weights, stable slots and work list in its own shared memory; CTA 0
//      also writes the routing tables;
//   X  the experts pipeline, reading the work list from shared memory.
// There is no separate grid barrier: the tag on every logit is the only
// signal a CTA waits for (see the notes above decode_fused_kernel).
// Compared with the two-launch path this removes the launch gap between
// router and experts and the router kernel's last-CTA tail.
constexpr int kFusedMaxPairs = kDecodeTok * kMaxTopK;   // 128
constexpr int kFusedMaxItems = kFusedMaxPairs + kMaxShared;

struct alignas(16) FusedRouteSmem {
    WorkItem items[kFusedMaxItems];
    int ids[kFusedMaxPairs];
    float w[kFusedMaxPairs];
    int slot_token[kFusedMaxPairs];
    float slot_w[kFusedMaxPairs];
    uint32_t emask[kMaxExperts / 32];   // bit e: expert e was selected by some token
    int n_routed;
    int skip;                           // this launch does no work (see decode_fused_kernel)
    unsigned long long tag;             // this launch's logit tag (in the high 32 bits)
};

static_assert(kFusedMaxPairs % 4 == 0 && offsetof(FusedRouteSmem, ids) % 16 == 0,
              "pair ids read as whole int4s");
static_assert(kFusedMaxPairs <= kConsumers / 2, "pair threads and table threads are disjoint");

size_t decode_fused_extra_smem() { return sizeof(FusedRouteSmem); }

// How the CTAs of one fused launch agree that routing may start, without a
// grid barrier:
//  - Launch tag.  At its start each CTA takes a ticket: one relaxed atomic
//    increment of a 64-bit count that only grows.  The G CTAs of a launch
//    raise it from n*G to (n+1)*G, so each CTA derives the same tag
//    (n+1)*G from its own ticket, as long as every earlier launch took all
//    its tickets (after a timeout the host resets the count to 0).  The
//    ticket's latency hides behind the router loads.
//  - Logit words.  Logit (t, e) is stored as one 64-bit word, fp32 bits low
//    and the low 32 bits of the tag high (one single-copy-atomic word: a
//    reader that sees the tag sees the value).  The producer warp stores
//    them, relaxed, after a release fence that follows its zero-fill of
//    `out`.  Every launch writes all kDecodeTok token rows of its experts
//    (rows t >= T with a zero value), so before a launch writes, each word
//    holds the previous launch's tag, never the current one.
//  - `out` zero-fill.  Done by the CTAs that own experts (b < E), each of
//    which publishes logits that every CTA's warp 0 reads.
// Reader side: warp t of each CTA loads the E words of token t with relaxed
// loads until every one carries the tag (bounded by kWaitLimitNs; on
// timeout it records kErrTimeout and the CTA skips phase X) and routes on
// the values.  Its acquire fence comes after routing, at the start of phase
// X: the fence pairs with the writers' release fences, and a named barrier
// of the consumers separates it from the first add into `out`.  So every
// add follows every zero-fill, and the fence's wait overlaps the first
// weight loads instead of delaying the routing.

// Token t's routing in the fused kernel (one warp): wait until all E logit
// words of the token carry `tag`, then the top-k of the values (the caller
// issues the acquire fence later, before phase X).
// Returns false when the bounded wait ran out (the selection is then made
// from whatever the words hold; the caller aborts phase X).
template <int PER>
__device__ __forceinline__ bool fused_token_topk(const unsigned long long* row, int E, int k,
                                                 uint32_t tag, uint32_t* err, float& sel, int& id) {
    const int lane = threadIdx.x & 31;
    unsigned long long wv[PER];
    const uint64_t t0 = globaltimer_ns();
    bool ok = true;
    while (true) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int x = lane + 32 * i;
            wv[i] = ld_relaxed_u64(row + (x < E ? x : E - 1));
        }
        bool mine = true;
#pragma unroll
        for (int i = 0; i < PER; ++i) mine &= static_cast<uint32_t>(wv[i] >> 32) == tag;
        if (__all_sync(0xffffffffu, mine)) break;
        if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > kWaitLimitNs)) {
            ok = false;
            break;
        }
    }
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        v[i] = __uint_as_float(static_cast<uint32_t>(wv[i]));
        if (lane + 32 * i >= E || isnan(v[i])) v[i] = -INFINITY;
    }
    warp_topk_select<PER>(v, E, k, err, sel, id);
    return ok;
}

// The same for E > 256: the wait checks the tags only, the values are read
// again after it (64 words per lane would not fit in registers next to the
// values).
__device__ __forceinline__ bool fused_token_topk_wide(const unsigned long long* row, int E, int k,
                                                      uint32_t tag, uint32_t* err, float& sel,
                                                      int& id) {
    constexpr int PER = 32;
    const int lane = threadIdx.x & 31;
    const uint64_t t0 = globaltimer_ns();
    bool ok = true;
    while (true) {
        bool mine = true;
#pragma unroll 8
        for (int i = 0; i < PER; ++i) {
            const int x = lane + 32 * i;
            mine &= static_cast<uint32_t>(ld_relaxed_u64(row + (x < E ? x : E - 1)) >> 32) == tag;
        }
        if (__all_sync(0xffffffffu, mine)) break;
        if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > kWaitLimitNs)) {
            ok = false;
            break;
        }
    }
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int x = lane + 32 * i;
        v[i] = __uint_as_float(static_cast<uint32_t>(ld_relaxed_u64(row + (x < E ? x : E - 1))));
        if (x >= E || isnan(v[i])) v[i] = -INFINITY;
    }
    warp_topk_select<PER>(v, E, k, err, sel, id);
    return ok;
}

__device__ __forceinline__ bool fused_token_topk_any(const unsigned long long* row, int E, int k,
                                                     uint32_t tag, uint32_t* err, float& sel,
                                                     int& id) {
    if (E <= 32) return fused_token_topk<1>(row, E, k, tag, err, sel, id);
    if (E <= 64) return fused_token_topk<2>(row, E, k, tag, err, sel, id);
    if (E <= 128) return fused_token_topk<4>(row, E, k, tag, err, sel, id);
    if (E <= 256) return fused_token_topk<8>(row, E, k, tag, err, sel, id);
    return fused_token_topk_wide(row, E, k, tag, err, sel, id);
}

template <int FS, int WF>
__global__ void __launch_bounds__(kDecodeThreads, 1)
decode_fused_kernel(const __grid_constant__ DecodeArgs a) {
    using C = DecodeCfg<FS, WF>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const DecodeSmem sm = decode_smem<FS, WF>(smem_raw, a);
    FusedRouteSmem* rs = reinterpret_cast<FusedRouteSmem*>(sm.empty + a.n_stages);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T, d = a.d, E = a.E, k = a.k, S = a.S;
    const int G = gridDim.x, b = blockIdx.x;

    // The producer warp, idle until phase X, sets up the ring barriers, takes
    // the launch ticket (see the notes above), reads the sticky error word
    // and fills the CTA's share of `out`, while the consumers' router loads
    // are in flight.  A timeout of an earlier launch that the host has not
    // yet read (and cleared, resetting the ticket count and the logit words)
    // may have left the count short of a whole round, so that the CTAs of
    // this launch could derive different tags.  If a timeout is pending, the
    // whole launch skips its work, writes NaN to `out` (so a caller that
    // ignores the status cannot take the result for a valid one) and records
    // kErrSkipped.  (The flag lives in the dynamic shared memory: a static
    // __shared__ variable would add a 1 KB block, the dynamic block's
    // alignment, on top of a launch sized to the opt-in limit.)
    if (warp == kConsumerWarps) {
        int skip = 0;
        if (lane == 0) {
            const uint32_t ev = *reinterpret_cast<volatile uint32_t*>(a.err);
            const unsigned long long old = atomicAdd(reinterpret_cast<unsigned long long*>(a.gbar), 1ull);
            for (int s = 0; s < a.n_stages; ++s) {
                mbar_init(&sm.full[s], 1);
                mbar_init(&sm.empty[s], kConsumerWarps);
            }
            sm.tail->abort_flag = 0;
            fence_mbar_init();
            // fetch the tensor maps now, so the first TMA of phase X does not
            // wait for them
            prefetch_tensormap(&a.tm_gate); prefetch_tensormap(&a.tm_up); prefetch_tensormap(&a.tm_down);
            if (S) { prefetch_tensormap(&a.tm_sgate); prefetch_tensormap(&a.tm_sup);
                     prefetch_tensormap(&a.tm_sdown); }
            if constexpr (C::QUANT) {
                prefetch_tensormap(&a.tm_gate_sc); prefetch_tensormap(&a.tm_up_sc);
                prefetch_tensormap(&a.tm_down_sc);
                if (S) { prefetch_tensormap(&a.tm_sgate_sc); prefetch_tensormap(&a.tm_sup_sc);
                         prefetch_tensormap(&a.tm_sdown_sc); }
            }
            const unsigned long long gl = static_cast<unsigned long long>(G);
            rs->tag = (old - old % gl + gl) << 32;
            skip = (ev & (kErrTimeout | kErrSkipped)) != 0;
            rs->skip = skip;
        }
        skip = __shfl_sync(0xffffffffu, skip, 0);
        float4* o = reinterpret_cast<float4*>(a.out);
        const int n4 = (T * d) >> 2;
        if (skip) {
            const float qnan = __uint_as_float(0x7fc00000u);
            for (int i = b * 32 + lane; i < n4; i += G * 32) o[i] = make_float4(qnan, qnan, qnan, qnan);
        } else if (b < E) {
            const int gz = G < E ? G : E;   // the CTAs that publish logits
            for (int i = b * 32 + lane; i < n4; i += gz * 32) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            // release fence: this lane's logit words (stored after it in
            // program order) publish the zero-fill with them
            __threadfence();
        }
    }

    // ---- R: logits of this CTA's experts b, b + G, ...  Warp w sums slice w
    // of d; it takes two experts per pass, so that both weight rows and the
    // shared x slice are requested before the first use.
    float* part = reinterpret_cast<float*>(sm.ring);          // [n_loc][16 slices][8 tok]
    const int n_loc = (E - b + G - 1) / G;
    // The producer warp also publishes the logit words (after its release
    // fence); lane l takes words l and l + 32 first, whose biases it loads now.
    float bias0 = 0.f, bias1 = 0.f;
    if (warp == kConsumerWarps && a.br) {
        if (lane < n_loc * kDecodeTok) bias0 = __ldg(a.br + b + (lane / kDecodeTok) * G);
        if (lane + 32 < n_loc * kDecodeTok) bias1 = __ldg(a.br + b + ((lane + 32) / kDecodeTok) * G);
    }
    if (warp < kConsumerWarps) {
        const int chunk = d / kConsumerWarps;
        for (int loc = 0; loc < n_loc; loc += 2) {
            const bool two = loc + 1 < n_loc;
            const float* w0 = a.wr + static_cast<size_t>(b + loc * G) * d;
            const float* w1 = two ? w0 + static_cast<size_t>(G) * d : w0;
            float acc0[kDecodeTok], acc1[kDecodeTok];
#pragma unroll
            for (int t = 0; t < kDecodeTok; ++t) acc0[t] = acc1[t] = 0.f;
#pragma unroll 2
            for (int i = warp * chunk + lane * 4; i < (warp + 1) * chunk; i += 128) {
                const float4 wa = __ldg(reinterpret_cast<const float4*>(w0 + i));
                const float4 wb = __ldg(reinterpret_cast<const float4*>(w1 + i));
#pragma unroll
                for (int t = 0; t < kDecodeTok; ++t) {
                    if (t < T) {
                        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(
                            a.x + static_cast<size_t>(t) * d + i));
                        const float x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xffff0000u);
                        const float x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xffff0000u);
                        acc0[t] = fmaf(x0, wa.x, acc0[t]);
                        acc0[t] = fmaf(x1, wa.y, acc0[t]);
                        acc0[t] = fmaf(x2, wa.z, acc0[t]);
                        acc0[t] = fmaf(x3, wa.w, acc0[t]);
                        acc1[t] = fmaf(x0, wb.x, acc1[t]);
                        acc1[t] = fmaf(x1, wb.y, acc1[t]);
                        acc1[t] = fmaf(x2, wb.z, acc1[t]);
                        acc1[t] = fmaf(x3, wb.w, acc1[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < kDecodeTok; ++t) {
                if (t < T) {
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {
                        acc0[t] += __shfl_xor_sync(0xffffffffu, acc0[t], off);
                        acc1[t] += __shfl_xor_sync(0xffffffffu, acc1[t], off);
                    }
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < kDecodeTok; ++t) {
                    part[(loc * kConsumerWarps + warp) * kDecodeTok + t] = acc0[t];
                    if (two) part[((loc + 1) * kConsumerWarps + warp) * kDecodeTok + t] = acc1[t];
                }
            }
        }
    }
    __syncthreads();
    if (rs->skip) {
        if (b == 0 && tid == 0) atomicOr(a.err, kErrSkipped);
        return;
    }
    const unsigned long long tag = rs->tag;
    if (warp == kConsumerWarps) {
        // publish every token row of this CTA's experts (rows t >= T with 0):
        // relaxed stores, ordered after the zero-fill by the fence above
        for (int i = lane; i < n_loc * kDecodeTok; i += 32) {
            const int loc = i / kDecodeTok, t = i % kDecodeTok;
            const int e = b + loc * G;
            float v = 0.f;
            if (t < T) {
                for (int ch = 0; ch < kConsumerWarps; ++ch) v += part[(loc * kConsumerWarps + ch) * kDecodeTok + t];
                if (a.br) v += (i == lane) ? bias0 : (i == lane + 32) ? bias1 : a.br[e];
            }
            st_relaxed_u64(a.ws.tlogits + static_cast<size_t>(t) * E + e, tag | __float_as_uint(v));
        }
    } else {
        // x for phase X, while the logits travel
        stage_x<WF>(a, sm, tid);
        if (tid < kMaxExperts / 32) rs->emask[tid] = 0u;
        named_bar_sync(1, kConsumers);
    }

    // ---- T: routing, computed redundantly by every CTA
    const int P = T * k;
    if (warp < kConsumerWarps) {
        if (warp < T) {
            // warp t: wait for token t's logits, top-k, then the softmax over
            // the k selected logits (the same sum order as the other routing
            // paths: j = 0, 1, ...)
            const int t = warp;
            float sv;
            int sid;
            const bool ok = fused_token_topk_any(a.ws.tlogits + static_cast<size_t>(t) * E, E, k,
                                                 static_cast<uint32_t>(tag >> 32), a.err, sv, sid);
            if (!ok && lane == 0) {
                atomicOr(a.err, kErrTimeout);
                sm.tail->abort_flag = 1;
            }
            const float m = __shfl_sync(0xffffffffu, sv, 0);
            const float ej = (lane < k) ? expf(sv - m) : 0.f;
            // lanes j >= k hold 0, so the unrolled sum over kMaxTopK lanes
            // equals the sum over the k selections, in the same order
            float den = 0.f;
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) den += __shfl_sync(0xffffffffu, ej, j);
            if (lane < k) {
                float wj = ej / den;
                if (!(m > -INFINITY)) wj = 1.f / k;
                rs->ids[t * k + lane] = sid;
                rs->w[t * k + lane] = wj;
                atomicOr(&rs->emask[sid >> 5], 1u << (sid & 31));
            }
        }
        if (tid == kConsumers - 1)      // pad the pair ids to whole int4s (never below an id)
            for (int q = P; q < ((P + 3) & ~3); ++q) rs->ids[q] = 0x7fffffff;
        named_bar_sync(1, kConsumers);
        // stable slots: pairs with a smaller expert id come first, ties by pair
        // index; the first pair of each expert writes its work item, whose
        // index is the number of selected experts below it (mask popcount).
        // The routing tables in global memory (identical in every CTA) are
        // written in shares: pair p by CTA p mod G, offsets/counts of expert x
        // by CTA x mod G.
        const int4* ids4 = reinterpret_cast<const int4*>(rs->ids);
        const int nq4 = (P + 3) >> 2;
        if (tid < P) {
            const int p = tid;
            const int e = rs->ids[p];
            int lt = 0, before = 0, cnt = 0;
            for (int q4 = 0; q4 < nq4; ++q4) {
                const int4 v = ids4[q4];
                const int q = 4 * q4;
                lt += (v.x < e) + (v.y < e) + (v.z < e) + (v.w < e);
                cnt += (v.x == e) + (v.y == e) + (v.z == e) + (v.w == e);
                before += ((v.x == e) & (q < p)) + ((v.y == e) & (q + 1 < p)) +
                          ((v.z == e) & (q + 2 < p)) + ((v.w == e) & (q + 3 < p));
            }
            const int slot = lt + before;
            rs->slot_token[slot] = p / k;
            rs->slot_w[slot] = rs->w[p];
            if (before == 0) {
                int idx = __popc(rs->emask[e >> 5] & ((1u << (e & 31)) - 1u));
                const int nw = e >> 5;
#pragma unroll 8
                for (int wd = 0; wd < nw; ++wd) idx += __popc(rs->emask[wd]);
                rs->items[idx] = WorkItem{e, lt, cnt, 0};
            }
            if (p % G == b) {
                a.ws.slot_pair[slot] = p;
                a.ws.slot_token[slot] = p / k;
                a.ws.slot_w[slot] = rs->w[p];
                a.ws.ids[p] = e;
                a.ws.wts[p] = rs->w[p];
            }
        } else if (tid == kConsumers - 1) {
            int n = 0;
            const int nw = (E + 31) / 32;
#pragma unroll 8
            for (int wd = 0; wd < nw; ++wd) n += __popc(rs->emask[wd]);
            rs->n_routed = n;
            for (int s2 = 0; s2 < S; ++s2) rs->items[n + s2] = WorkItem{E + s2, -1, T, 0};
        } else if (tid >= kConsumers / 2) {
            constexpr int kTab = kConsumers / 2 - 1;    // threads kConsumers/2 .. kConsumers-2
            for (int x = b + G * (tid - kConsumers / 2); x <= E; x += G * kTab) {
                int lt = 0, cnt = 0;
                for (int q4 = 0; q4 < nq4; ++q4) {
                    const int4 v = ids4[q4];
                    lt += (v.x < x) + (v.y < x) + (v.z < x) + (v.w < x);
                    cnt += (v.x == x) + (v.y == x) + (v.z == x) + (v.w == x);
                }
                a.ws.offsets[x] = lt;
                if (x < E) a.ws.counts[x] = cnt;
            }
        }
    }
    __syncthreads();
    // acquire: the warps that read the logit words order the other CTAs'
    // zero-fill of `out` before every add of phase X (which follows a named
    // barrier of the consumers); done here, not before routing, so that it
    // overlaps the first weight loads
    if (warp < T) fence_acq_rel_gpu();
    const WorkView wv{rs->n_routed, S, rs->items, rs->slot_token, rs->slot_w};
    run_experts<FS, WF>(a, sm, wv);
}

int decode_stage_bytes(int fs, int wfmt) {
    (void)fs;
    if (wfmt == kWfQ4) return 2 * 512 * 18;
    if (wfmt == kWfQ6) return 28672;
    if (wfmt == kWfQ8) return 2 * 512 * 34;
    if (wfmt == kWfQ5) return 2 * 512 * 22;
    return 32768;
}

size_t decode_smem_bytes(int fs, int wfmt, int d, int n_stages) {
    // partial sums per gate/up output: KSPLIT, or one per warp for the
    // row-streaming formats (DecodeCfg::GU_PARTS)
    const int ksplit = (wfmt == kWfQ4 || wfmt == kWfQ6 || wfmt == kWfQ8) ? kConsumerWarps
                                                         : kConsumerWarps / (2 * (fs / 16));
    size_t b = 1024;                                            // alignment slack
    b += static_cast<size_t>(n_stages) * decode_stage_bytes(fs, wfmt);
    b += static_cast<size_t>(kDecodeTok) * (d * 2 + 16);       // staged x
    b += static_cast<size_t>(kDecodeTok) * (d / 16) * 4;       // block (sub-block) sums of x
    b += static_cast<size_t>(ksplit) * 2 * kDecodeTok * (fs + 4) * 4;  // gate/up results
    b += 2ull * kDecodeTok * (fs + 8) * 2;                      // h hi/lo
    b += static_cast<size_t>(kDecodeTok) * 4 * 4;              // block sums of h
    b += sizeof(DecodeSmemTail);
    b += 2ull * n_stages * 8;                                   // barriers
    return b;
}

template <int FS, int WF>
static cudaError_t launch_one(const DecodeArgs& a, int grid, size_t smem, cudaStream_t stream) {
    auto* k = decode_experts_kernel<FS, WF>;
    // the dynamic shared memory limit is raised once per device (and again
    // only if a later launch needs more)
    static int set_bytes[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || set_bytes[dev] < static_cast<int>(smem)) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) set_bytes[dev] = static_cast<int>(smem);
    }
    k<<<grid, kDecodeThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int FS, int WF>
static cudaError_t launch_fused_one(const DecodeArgs& a, int grid, size_t smem, cudaStream_t stream) {
    auto* k = decode_fused_kernel<FS, WF>;
    static int set_bytes[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || set_bytes[dev] < static_cast<int>(smem)) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) set_bytes[dev] = static_cast<int>(smem);
    }
    // cooperative: every CTA is resident at once, which the wait for every
    // CTA's tagged logits needs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, a);
}

cudaError_t launch_decode_fused(const DecodeArgs& a, int fs, int wfmt, int grid, size_t smem,
                                cudaStream_t stream) {
    switch (wfmt * 100 + fs) {
        case kWfBf16 * 100 + 64: return launch_fused_one<64, kWfBf16>(a, grid, smem, stream);
        case kWfBf16 * 100 + 32: return launch_fused_one<32, kWfBf16>(a, grid, smem, stream);
        case kWfF16d * 100 + 64: return launch_fused_one<64, kWfF16d>(a, grid, smem, stream);
        case kWfF16d * 100 + 32: return launch_fused_one<32, kWfF16d>(a, grid, smem, stream);
        case kWfQ4 * 100 + 32: return launch_fused_one<32, kWfQ4>(a, grid, smem, stream);
        case kWfQ6 * 100 + 32: return launch_fused_one<32, kWfQ6>(a, grid, smem, stream);
        case kWfQ8 * 100 + 32: return launch_fused_one<32, kWfQ8>(a, grid, smem, stream);
        case kWfQ5 * 100 + 64: return launch_fused_one<64, kWfQ5>(a, grid, smem, stream);
        case kWfQ5 * 100 + 32: return launch_fused_one<32, kWfQ5>(a, grid, smem, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_experts(const DecodeArgs& a, int fs, int wfmt, int grid, size_t smem,
                                  cudaStream_t stream) {
    switch (wfmt * 100 + fs) {
        case kWfBf16 * 100 + 64: return launch_one<64, kWfBf16>(a, grid, smem, stream);
        case kWfBf16 * 100 + 32: return launch_one<32, kWfBf16>(a, grid, smem, stream);
        case kWfF16d * 100 + 64: return launch_one<64, kWfF16d>(a, grid, smem, stream);
        case kWfF16d * 100 + 32: return launch_one<32, kWfF16d>(a, grid, smem, stream);
        case kWfQ4 * 100 + 32: return launch_one<32, kWfQ4>(a, grid, smem, stream);
        case kWfQ6 * 100 + 32: return launch_one<32, kWfQ6>(a, grid, smem, stream);
        case kWfQ8 * 100 + 32: return launch_one<32, kWfQ8>(a, grid, smem, stream);
        case kWfQ5 * 100 + 64: return launch_one<64, kWfQ5>(a, grid, smem, stream);
        case kWfQ5 * 100 + 32: return launch_one<32, kWfQ5>(a, grid, smem, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
