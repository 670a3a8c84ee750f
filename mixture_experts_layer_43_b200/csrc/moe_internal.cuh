// moe_internal.cuh -- internal declarations and device helpers shared by the
// kernels of libmoe_b200.so (sm_100a only).  Inline PTX for the mbarrier,
// TMA (cp.async.bulk.tensor), ldmatrix, mma.sync and reduction instructions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ----------------------------------------------------------------- limits
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 16;
constexpr int kMaxShared = 8;
constexpr int kDecodeTok = 8;        // mma N: tokens per expert pass (>= MOE_DECODE_MAX_T)
constexpr int kDecodeConsumerWarps = 16;   // consumer warps of a decode CTA (+ 1 producer)
static_assert(MOE_DECODE_MAX_T <= kDecodeTok, "decode pass holds every token");

// Device error word bits (sticky until moe_get_device_status reads them).
constexpr uint32_t kErrBadId = 1u;        // an expert id or count out of range
constexpr uint32_t kErrTimeout = 2u;      // a bounded wait ran out
constexpr uint32_t kErrTooManyTok = 4u;   // an expert got more tokens than a pass holds
// A fused decode launch found kErrTimeout (or this bit) already set when it
// started: an earlier launch may have left the launch ticket count short of a
// whole round, so the launch did no routing or expert work and wrote NaN to
// `out`.  Cleared with the timeout by moe_get_device_status, which also
// resets the ticket count and the tagged logit words.
constexpr uint32_t kErrSkipped = 8u;

// Bounded waits give up after this long (a healthy wait lasts microseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Work item of the decode regime: one expert and the tokens routed to it.
struct WorkItem {
    int32_t expert;      // 0..E-1 routed, E+s shared expert s
    int32_t slot_begin;  // first slot in the bucket order (routed) or -1 (shared: tokens 0..T-1)
    int32_t count;       // tokens in this item (<= kDecodeTok)
    int32_t pad;
};

// Plan workspace (device pointers), sized for t_max at plan creation.
struct Workspace {
    float* logits;         // [t_max][E] fp32
    int32_t* ids;          // [t_max][k]
    float* wts;            // [t_max][k]
    int32_t* counts;       // [E]
    int32_t* offsets;      // [E+1]
    int32_t* slot_pair;    // [t_max*k]
    int32_t* slot_token;   // [t_max*k]
    float* slot_w;         // [t_max*k]
    WorkItem* items;       // [E + S]
    int32_t* n_items;      // [2]: routed items, shared items
    uint32_t* ticket;      // last-CTA ticket of the decode router
    uint32_t* err;         // sticky device error word
    uint32_t* gbar;        // fused decode kernel: [0..1] 64-bit launch ticket count (8-aligned)
    unsigned long long* tlogits;  // fused decode kernel: [kDecodeTok][E] logit bits | launch tag << 32
    // prefill
    uint16_t* x_perm;      // [t_max*k][d] bf16 rows gathered per slot
    uint16_t* h_routed;    // [t_max*k][F] bf16
    uint16_t* h_shared;    // [t_max][S*Fs] bf16
    int32_t* tiles;        // prefill tile schedule
    int32_t* n_tiles;      // [4]
};

// ---------------------------------------------------------- launch args
struct RouteArgs {
    const uint16_t* x;     // [T][d] bf16
    const float* wr;       // [E][d]
    const float* br;       // [E] or nullptr
    float* out;            // [T][d] zero-filled here
    Workspace ws;
    int T, d, E, k, S;
    int experts_per_cta;   // 1, 2, 4 or 8
};

// Rows of one TMA box of a quantised down matrix in the decode kernels (the
// host builds the tensor maps with the same box).
constexpr int kQuantDownBoxRows = 256;

struct DecodeArgs {
    // bf16: 2D maps over the weight stacks.  Quantised: 3D maps over the codes.
    CUtensorMap tm_gate, tm_up, tm_down;
    CUtensorMap tm_sgate, tm_sup, tm_sdown;
    // Quantised only: Q4_0 / Q8_0 2D maps over the scales, Q5_0 3D maps over
    // the 48-byte records of scales and fifth bits.
    CUtensorMap tm_gate_sc, tm_up_sc, tm_down_sc;
    CUtensorMap tm_sgate_sc, tm_sup_sc, tm_sdown_sc;
    // q6_K only: 2D maps over the fp16 super-block scales [mats][K/256][rows]
    // (the _sc maps above cover the 160-byte records of high bits and
    // sub-block scales)
    CUtensorMap tm_gate_d, tm_up_d, tm_down_d;
    CUtensorMap tm_sgate_d, tm_sup_d, tm_sdown_d;
    const uint16_t* x;          // [T][d] bf16
    float* out;                 // [T][d] fp32, accumulated into
    const WorkItem* items;
    const int32_t* n_items;
    const int32_t* slot_token;
    const float* slot_w;
    uint32_t* err;
    int T, d, F, Fs, E, S;
    int n_stages;               // ring depth
    int xs_stride;              // bytes per token row of the staged x
    int kt;                     // phase A: k columns (bf16) / block columns (quantised) per stage
    int rj;                     // phase B: output rows per stage
    // fused single-launch path only: router inputs, routing tables, launch tickets
    const float* wr;            // [E][d]
    const float* br;            // [E] or nullptr
    int k;
    Workspace ws;
    uint32_t* gbar;             // [0..1] 64-bit launch ticket count
};

// Host launchers (decode.cu, quant_pack.cu).
cudaError_t launch_decode_route(const RouteArgs& a, cudaStream_t stream);
cudaError_t launch_decode_experts(const DecodeArgs& a, int fs, int wfmt, int grid,
                                  size_t smem, cudaStream_t stream);
size_t decode_smem_bytes(int fs, int wfmt, int d, int n_stages);
cudaError_t launch_decode_fused(const DecodeArgs& a, int fs, int wfmt, int grid, size_t smem,
                                cudaStream_t stream);
size_t decode_fused_extra_smem();
int decode_stage_bytes(int fs, int wfmt);
cudaError_t launch_q4_0_pack(const uint8_t* blocks, int64_t n_mats, int64_t rows, int64_t k,
                             uint8_t* codes, uint16_t* scales, cudaStream_t stream);
cudaError_t launch_q8_0_pack(const uint8_t* blocks, int64_t n_mats, int64_t rows, int64_t k,
                             uint8_t* codes, uint16_t* scales, cudaStream_t stream);
cudaError_t launch_q5_0_pack(const uint8_t* blocks, int64_t n_mats, int64_t rows, int64_t k,
                             uint8_t* codes, uint8_t* aux, cudaStream_t stream);
cudaError_t launch_q6_k_pack(const uint8_t* blocks, int64_t n_mats, int64_t rows, int64_t k,
                             uint8_t* codes, uint8_t* scales, cudaStream_t stream);
cudaError_t launch_bf16_to_f16(const uint16_t* src, int64_t n, uint16_t* dst, cudaStream_t stream);

// Formats whose matrices are quantised blocks (codes + scales).
inline bool wfmt_quantised(int wfmt) {
    return wfmt == MOE_WFMT_Q4_0 || wfmt == MOE_WFMT_Q8_0 || wfmt == MOE_WFMT_Q5_0 ||
           wfmt == MOE_WFMT_Q6_K;
}

// --------------------------------------------------------- device helpers
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Loads from shared memory by 32-bit shared address: the hot loops add
// compile-time offsets to one per-lane base instead of building 64-bit
// generic addresses (which also compile to generic loads).
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ float lds_f16_as_f32(uint32_t addr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed, for at most
// kWaitLimitNs.  Returns false when the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// The same wait for warps that must not take issue slots from the warps
// doing the work while they wait (the decode kernels' producer, waiting for a
// free ring slot, and consumers waiting for data): between polls the warp
// sleeps, 16 ns at first and at most 128 ns, which bounds the delay it adds
// once the phase completes.
__device__ __forceinline__ bool mbar_wait_bounded_sleep(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t ns = 16;
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
        __nanosleep(ns);
        if (ns < 128) ns <<= 1;
    }
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// TMA tiled loads (no multicast), completing on an mbarrier of this CTA.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
          "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
          "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ldmatrix: four / two 8x8 b16 matrices; row addresses from lanes 0-31 / 0-15.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                        uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r0), "=r"(r1) : "r"(addr));
}

// c += A(16x16 bf16, row-major) * B(16x8 bf16, col-major), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = A(16x16 f16, row-major) * B(16x8 f16, col-major) + c, fp32 accumulate;
// c in separate registers, so a chain can start from a precomputed value.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1,
                                              float c0, float c1, float c2, float c3) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1),
          "f"(c0), "f"(c1), "f"(c2), "f"(c3));
}

// d += A * B (f16 operands, fp32 accumulate).
__device__ __forceinline__ void mma_f16_16816_acc(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void red_add_f32(float* p, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// p[0] += a and p[8] += b (two rows of one mma fragment column), one address
// register with an immediate offset.
__device__ __forceinline__ void red_add_f32_rows8(float* p, float a, float b) {
    asm volatile("red.global.add.f32 [%0], %1;\n\tred.global.add.f32 [%0+32], %2;"
                 ::"l"(p), "f"(a), "f"(b) : "memory");
}

// Named barrier among `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile whose rows are
// `row_bytes` (128, 64 or 32) long and that TMA wrote with the swizzle mode of
// the same width: the chunk index is XORed with address bits 7.. of the row
// (128B: row % 8; 64B: (row / 2) % 4; 32B: (row / 4) % 2).  The tile base
// must be aligned to the swizzle span.
__device__ __forceinline__ uint32_t swz_offset(uint32_t row, uint32_t chunk, uint32_t row_bytes) {
    uint32_t x;
    if (row_bytes == 128) x = chunk ^ (row & 7);
    else if (row_bytes == 64) x = chunk ^ ((row >> 1) & 3);
    else x = chunk ^ ((row >> 2) & 1);
    return row * row_bytes + x * 16;
}

// ------------------------------------------------------ tcgen05 (UMMA)
// Shared-memory matrix descriptor of a K-major bf16 tile written by TMA with
// the 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart (stride
// byte offset), leading byte offset unused (1), descriptor version 1,
// layout type 2 = 128B swizzle.  `addr` is the shared address of the first
// 16-element K slice; the next UMMA_K slice starts 32 bytes later.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);   // start address
    d |= static_cast<uint64_t>(1u) << 16;                  // leading byte offset (unused)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;          // stride byte offset
    d |= static_cast<uint64_t>(1u) << 46;                  // version
    d |= static_cast<uint64_t>(2u) << 61;                  // SWIZZLE_128B
    return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D,
// both K-major, dense, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4)                                   // D format f32
         | (1u << 7)                                   // A format bf16
         | (1u << 10)                                  // B format bf16
         | (static_cast<uint32_t>(N >> 3) << 17)       // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);      // M / 16
}

// The same with fp16 A and B (format bits 0).
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
    return (1u << 4)                                   // D format f32
         | (static_cast<uint32_t>(N >> 3) << 17)       // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);      // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n"
        " setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM allocation (one full warp executes these).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (warp-wide).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void red_add_v4_f32(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// --------------------------------------------------------- warp top-k
// Order-preserving 32-bit key of a logit (NaN excluded): larger logit,
// larger key; -0 maps like +0, so that equal logits have equal keys.
__device__ __forceinline__ uint32_t logit_key(float f) {
    const uint32_t u = f == 0.f ? 0u : __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float logit_of_key(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Top-k of one token's E logits (E <= 32 * PER) by one warp, from
// registers: lane l holds the logits of experts l, l + 32, ... in v[0..PER)
// (entries past E and NaN already set to -inf).  Each value becomes its
// order-preserving key, and the lane sorts its PER keys with a bitonic
// network into selection order: descending logit, equal logits by
// ascending expert index.  Round j takes the warp maximum m of the lanes'
// first keys and the lowest expert index among the first keys equal to m
// (two integer warp reductions); the lane holding that entry drops it (its
// list moves up by one).  KMAX >= k rounds run unrolled and without
// branches (a lone warp's chain of dependent steps is what this costs, and
// a branch per round about doubled it); rounds past k change nothing that
// is returned.  Lane j < k returns selection j in (sel, id); the other
// lanes return (-inf, 0).  For PER <= 8 (E <= 256); larger E takes
// warp_topk_scan_select.
template <int PER, int KMAX>
__device__ __forceinline__ void warp_topk_sorted_select(float (&v)[PER], int E, int k,
                                                        uint32_t* err, float& sel, int& id) {
    const int lane = threadIdx.x & 31;
    uint32_t key[PER];
    int ix[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        key[i] = logit_key(v[i]);
        ix[i] = lane + 32 * i;
    }
#pragma unroll
    for (int size = 2; size <= PER; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int l = i ^ stride;
                if (l > i) {
                    // entry p goes first in this run's order
                    const int p = ((i & size) == 0) ? i : l;
                    const int q = (p == i) ? l : i;
                    const bool sw = key[q] > key[p] || (key[q] == key[p] && ix[q] < ix[p]);
                    const uint32_t tk = key[p];
                    const int ti = ix[p];
                    key[p] = sw ? key[q] : tk;
                    ix[p] = sw ? ix[q] : ti;
                    key[q] = sw ? tk : key[q];
                    ix[q] = sw ? ti : ix[q];
                }
            }
        }
    }
    uint32_t selk = 0u;
    int sid = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
        const int w = static_cast<int>(
            __reduce_min_sync(0xffffffffu, key[0] == m ? static_cast<uint32_t>(ix[0]) : 0xffffffffu));
        const bool mine = ix[0] == w;
#pragma unroll
        for (int i = 0; i + 1 < PER; ++i) {
            key[i] = mine ? key[i + 1] : key[i];
            ix[i] = mine ? ix[i + 1] : ix[i];
        }
        key[PER - 1] = mine ? 0u : key[PER - 1];     // below every logit key (-inf: 0x007fffff)
        ix[PER - 1] = mine ? 0x7fffffff : ix[PER - 1];
        selk = (lane == j) ? m : selk;
        sid = (lane == j) ? w : sid;
    }
    if (lane < k && (sid < 0 || sid >= E)) {   // cannot happen for k <= E; keep ids in range
        atomicOr(err, kErrBadId);
        sid = 0;
    }
    sel = lane < k ? logit_of_key(selk) : -INFINITY;
    id = lane < k ? sid : 0;
}

// The same selection for E up to 1024 (PER = 32), where a sorted copy would
// not fit in registers: a bitmask marks the entries already taken and round
// j scans the lane's PER keys for its best one before the same two warp
// reductions.  Same order and outputs as warp_topk_sorted_select.
template <int PER>
__device__ __forceinline__ void warp_topk_scan_select(const float (&v)[PER], int E, int k,
                                                      uint32_t* err, float& sel, int& id) {
    const int lane = threadIdx.x & 31;
    uint32_t key[PER];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        key[i] = logit_key(v[i]);
        if (lane + 32 * i >= E) taken |= 1u << i;
    }
    sel = -INFINITY;
    id = 0;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PER; ++i)   // strict '>': the lowest index wins inside a lane
            if (!((taken >> i) & 1u) && (key[i] > bk || bi == 0x7fffffff)) { bk = key[i]; bi = lane + 32 * i; }
        const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t cand = (bk == m && bi != 0x7fffffff) ? static_cast<uint32_t>(bi) : 0xffffffffu;
        int w = static_cast<int>(__reduce_min_sync(0xffffffffu, cand));
        if (w < 0 || w >= E) {
            if (lane == 0) atomicOr(err, kErrBadId);
            w = 0;
        } else if ((w & 31) == lane) {
            taken |= 1u << (w >> 5);
        }
        if (lane == j) {
            sel = logit_of_key(m);
            id = w;
        }
    }
}

template <int PER>
__device__ __forceinline__ void warp_topk_select(float (&v)[PER], int E, int k, uint32_t* err,
                                                 float& sel, int& id) {
    if constexpr (PER <= 8) {
        if (k <= 2) warp_topk_sorted_select<PER, 2>(v, E, k, err, sel, id);
        else if (k <= 4) warp_topk_sorted_select<PER, 4>(v, E, k, err, sel, id);
        else if (k <= 8) warp_topk_sorted_select<PER, 8>(v, E, k, err, sel, id);
        else warp_topk_sorted_select<PER, kMaxTopK>(v, E, k, err, sel, id);
    } else {
        warp_topk_scan_select<PER>(v, E, k, err, sel, id);
    }
}

// Top-k of a logit row in memory (shared, or global through L2 when CG: for
// logits that other CTAs of the same launch wrote).  Every load is issued
// (index clamped into the row) before the first use, so that the PER reads
// overlap; NaN reads as -inf.
template <int PER, bool CG>
__device__ __forceinline__ void warp_topk_reg(const float* row, int E, int k, uint32_t* err,
                                              float& sel, int& id) {
    const int lane = threadIdx.x & 31;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int x = lane + 32 * i;
        const int xc = x < E ? x : E - 1;
        v[i] = CG ? __ldcg(row + xc) : row[xc];
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
        if (lane + 32 * i >= E || isnan(v[i])) v[i] = -INFINITY;
    warp_topk_select<PER>(v, E, k, err, sel, id);
}

// warp_topk_reg with PER chosen from E at run time.
template <bool CG>
__device__ __forceinline__ void warp_topk_reg_any(const float* row, int E, int k, uint32_t* err,
                                                  float& sel, int& id) {
    if (E <= 32) warp_topk_reg<1, CG>(row, E, k, err, sel, id);
    else if (E <= 64) warp_topk_reg<2, CG>(row, E, k, err, sel, id);
    else if (E <= 128) warp_topk_reg<4, CG>(row, E, k, err, sel, id);
    else if (E <= 256) warp_topk_reg<8, CG>(row, E, k, err, sel, id);
    else warp_topk_reg<32, CG>(row, E, k, err, sel, id);
}

// The same selection written to shared memory: ids[j] and the selected
// logits sel[j] for j < k.
__device__ __forceinline__ void warp_topk_any(const float* row, int E, int k, int* ids, float* sel,
                                              uint32_t* err) {
    float s;
    int i;
    warp_topk_reg_any<false>(row, E, k, err, s, i);
    const int lane = threadIdx.x & 31;
    if (lane < k) {
        ids[lane] = i;
        sel[lane] = s;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
#endif  // __CUDACC__

}  // namespace moe
