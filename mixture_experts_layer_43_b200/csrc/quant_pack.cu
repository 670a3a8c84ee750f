// quant_pack.cu -- repack canonical Q4_0, Q8_0, Q5_0 blocks and q6_K
// super-blocks into the decode kernels' layout.
//
// ---- Q4_0
// Canonical block (32 weights along the reduction dim, 18 bytes): little-endian
// fp16 scale d, then 16 bytes; byte j holds code j (low nibble) and code j+16
// (high nibble); weight = d * (q - 8).  This is the Q4_0 the "MoE on RTX 5090
// reaches 41% of bandwidth" page measures (measurement-setup paragraph), with
// the block layout of the 35B-A3B Q4_0 workload.
//
// Kernel layout (same 4.5 bits per weight):
//   codes  [mat][k/32][rows][16 B]   block-column major, so an expert's slice
//                                    of rows, or a slice of block columns, is
//                                    one contiguous run for TMA
//   scales [mat][k/32][rows] fp16
// Inside a block the 32 codes are permuted so that 32-bit word `tig` (0..3)
// holds exactly the 8 codes lane tig of an mma.sync m16n8k16 A fragment needs
// for both 16-wide halves of the block:
//   bits  0- 3 code 2tig      bits 16-19 code 2tig+1
//   bits  4- 7 code 2tig+8    bits 20-23 code 2tig+9
//   bits  8-11 code 2tig+16   bits 24-27 code 2tig+17
//   bits 12-15 code 2tig+24   bits 28-31 code 2tig+25
#include "moe_internal.cuh"

namespace moe {

__global__ void q4_0_pack_kernel(const uint8_t* __restrict__ blocks, int64_t n_mats, int64_t rows,
                                 int64_t nkb, uint8_t* __restrict__ codes,
                                 uint16_t* __restrict__ scales) {
    const int64_t total = n_mats * rows * nkb;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t kb = i % nkb;
        const int64_t r = (i / nkb) % rows;
        const int64_t m = i / (nkb * rows);
        const uint8_t* src = blocks + i * 18;            // [m][r][kb] canonical
        uint8_t q[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint8_t b = src[2 + j];
            q[j] = b & 0x0f;
            q[j + 16] = b >> 4;
        }
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int e = 2 * t;
            w[t] = static_cast<uint32_t>(q[e]) | (static_cast<uint32_t>(q[e + 8]) << 4) |
                   (static_cast<uint32_t>(q[e + 16]) << 8) | (static_cast<uint32_t>(q[e + 24]) << 12) |
                   (static_cast<uint32_t>(q[e + 1]) << 16) | (static_cast<uint32_t>(q[e + 9]) << 20) |
                   (static_cast<uint32_t>(q[e + 17]) << 24) | (static_cast<uint32_t>(q[e + 25]) << 28);
        }
        const int64_t dst = (m * nkb + kb) * rows + r;   // [m][kb][r]
        *reinterpret_cast<uint4*>(codes + dst * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        scales[dst] = static_cast<uint16_t>(src[0] | (src[1] << 8));
    }
}

cudaError_t launch_q4_0_pack(const uint8_t* blocks, int64_t n_mats, int64_t rows, int64_t k,
                             uint8_t* codes, uint16_t* scales, cudaStream_t stream) {
    const int64_t total = n_mats * rows * (k / 32);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t want = (total + threads - 1) / threads;
    const int grid = static_cast<int>(want < 65536 ? want : 65536);
    q4_0_pack_kernel<<<grid, threads, 0, stream>>>(blocks, n_mats, rows, k / 32, codes, scales);
    return cudaGetLastError();
}


// ---- Q8_0
// Canonical block (32 weights, 34 bytes): little-endian fp16 scale d, then 32
// signed bytes q (element j in byte j); weight = d * q.  (The 5090 page lists
// q8_0 among the formats of the model it measures; the byte layout is the
// canonical llama.cpp one, a reading.)
//
// Kernel layout (same 8.5 bits per weight):
//   codes  [mat][k/32][rows][32 B]
//   scales [mat][k/32][rows] fp16
// Each code is stored biased, u = q + 128 (0..255), one byte per code.  A
// block row is four 8-byte lane shares; lane tig's share holds, in this
// order, the codes of elements
//   2tig, 2tig+1, 2tig+8, 2tig+9, 16+2tig, 17+2tig, 24+2tig, 25+2tig,
// i.e. its first 32-bit word covers the lane's A-fragment elements of the
// block's first 16-wide half and its second word those of the second half,
// in fragment order (pair 2tig/2tig+1, then pair 2tig+8/2tig+9).
__device__ __forceinline__ int q8_lane_elem(int t, int n) {   // n-th byte of lane t's share
    return 2 * t + (n & 1) + 8 * ((n >> 1) & 1) + 16 * (n >> 2);
}

__global__ void q8_0_pack_kernel(const uint8_t* __restrict__ blocks, int64_t n_mats, int64_t rows,
                                 int64_t nkb, uint8_t* __restrict__ codes,
                                 uint16_t* __restrict__ scales) {
    const int64_t total = n_mats * rows * nkb;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t kb = i % nkb;
        const int64_t r = (i / nkb) % rows;
        const int64_t m = i / (nkb * rows);
        const uint8_t* src = blocks + i * 34;            // [m][r][kb] canonical
        uint32_t w[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t v = 0;
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const uint32_t u = static_cast<uint32_t>(src[2 + q8_lane_elem(t, 4 * h + n)] ^ 0x80u);
                    v |= u << (8 * n);
                }
                w[2 * t + h] = v;
            }
        }
        const int64_t dst = (m * nkb + kb) * rows + r;   // [m][kb][r]
        uint4* o = reinterpret_cast<uint4*>(codes + dst * 32);
        o[0] = make_uint4(w[0], w[1], w[2], w[3]);
        o[1] = make_uint4(w[4], w[5], w[6], w[7]);
        scales[dst] = static_cast<uint16_t>(src[0] | (src[1] << 8));
    }
}

cudaError_t launch_q8_0_pack(const uint8_t* blocks, int64_t n_mats, int64_t rows, int64_t k,
                             uint8_t* codes, uint16_t* scales, cudaStream_t stream) {
    const int64_t total = n_mats * rows * (k / 32);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t want = (total + threads - 1) / threads;
    const int grid = static_cast<int>(want < 65536 ? want : 65536);
    q8_0_pack_kernel<<<grid, threads, 0, stream>>>(blocks, n_mats, rows, k / 32, codes, scales);
    return cudaGetLastError();
}



// ---- Q5_0
// Canonical block (32 weights, 22 bytes): little-endian fp16 scale d, a
// little-endian 32-bit word qh whose bit j is the fifth bit of element j,
// then 16 bytes; byte j holds the low 4 bits of element j (low nibble) and of
// element j+16 (high nibble); q = low bits + 16 * fifth bit, weight =
// d * (q - 16).  (The 5090 page lists q5_0 among the formats of the model it
// measures; the byte layout is the canonical llama.cpp one, a reading.)
//
// Kernel layout (same 5.5 bits per weight):
//   codes  [mat][k/32][rows][16 B]        the low 4 bits, packed like Q4_0
//   aux    [mat][k/32][rows/8][48 B]      per 8 consecutive rows: their 8
//                                         fp16 scales, then their 8 32-bit
//                                         words of fifth bits
// In a row's word of fifth bits, lane t (0..3) owns bits 4t+n and 16+4t+n
// (n = 0..3): the fifth bits of the codes in nibbles n and n+4 of its code
// word (elements 2t+8n and 2t+1+8n).
// lane t's 32-bit word of 4-bit values q[0..31], in the Q4_0 permutation
__device__ __forceinline__ uint32_t pack_q4_lane(const uint8_t* q, int t) {
    const int e = 2 * t;
    return static_cast<uint32_t>(q[e]) | (static_cast<uint32_t>(q[e + 8]) << 4) |
           (static_cast<uint32_t>(q[e + 16]) << 8) | (static_cast<uint32_t>(q[e + 24]) << 12) |
           (static_cast<uint32_t>(q[e + 1]) << 16) | (static_cast<uint32_t>(q[e + 9]) << 20) |
           (static_cast<uint32_t>(q[e + 17]) << 24) | (static_cast<uint32_t>(q[e + 25]) << 28);
}

__global__ void q5_0_pack_kernel(const uint8_t* __restrict__ blocks, int64_t n_mats, int64_t rows,
                                 int64_t nkb, uint8_t* __restrict__ codes, uint8_t* __restrict__ aux) {
    const int64_t total = n_mats * rows * nkb;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t kb = i % nkb;
        const int64_t r = (i / nkb) % rows;
        const int64_t m = i / (nkb * rows);
        const uint8_t* src = blocks + i * 22;            // [m][r][kb] canonical
        const uint32_t qh = static_cast<uint32_t>(src[2]) | (static_cast<uint32_t>(src[3]) << 8) |
                            (static_cast<uint32_t>(src[4]) << 16) | (static_cast<uint32_t>(src[5]) << 24);
        uint8_t lo[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            lo[j] = src[6 + j] & 0x0f;
            lo[j + 16] = src[6 + j] >> 4;
        }
        uint32_t w[4], fifth = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            w[t] = pack_q4_lane(lo, t);
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                fifth |= ((qh >> (2 * t + 8 * n)) & 1u) << (4 * t + n);
                fifth |= ((qh >> (2 * t + 1 + 8 * n)) & 1u) << (16 + 4 * t + n);
            }
        }
        const int64_t dst = (m * nkb + kb) * rows + r;   // [m][kb][r]
        *reinterpret_cast<uint4*>(codes + dst * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        uint8_t* rec = aux + ((m * nkb + kb) * (rows / 8) + r / 8) * 48;
        *reinterpret_cast<uint16_t*>(rec + 2 * (r % 8)) = static_cast<uint16_t>(src[0] | (src[1] << 8));
        *reinterpret_cast<uint32_t*>(rec + 16 + 4 * (r % 8)) = fifth;
    }
}

cudaError_t launch_q5_0_pack(const uint8_t* blocks, int64_t n_mats, int64_t rows, int64_t k,
                             uint8_t* codes, uint8_t* aux, cudaStream_t stream) {
    const int64_t total = n_mats * rows * (k / 32);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t want = (total + threads - 1) / threads;
    const int grid = static_cast<int>(want < 65536 ? want : 65536);
    q5_0_pack_kernel<<<grid, threads, 0, stream>>>(blocks, n_mats, rows, k / 32, codes, aux);
    return cudaGetLastError();
}

// ---- q6_K
// Canonical super-block (256 weights along the reduction dim, 210 bytes):
// ql[128] low 4 bits, qh[64] high 2 bits, 16 signed 8-bit sub-block scales,
// then a little-endian fp16 scale d.  Element i = 128 h + 32 c + l: low bits
// in the low (c < 2) or high (c >= 2) nibble of ql[64 h + 32 (c % 2) + l],
// high bits in bits 2c, 2c+1 of qh[32 h + l]; weight d * sc[i / 16] * (q - 32).
// (The 5090 page lists q6_K among the formats of the model it measures; the
// byte layout is the canonical llama.cpp one, a reading.)
//
// Kernel layout (same 6.5625 bits per weight):
//   codes [mat][k/32][rows][16 B]        low 4 bits, packed exactly like Q4_0
//   aux   [mat][k/32][rows/16][160 B]    per 32-wide block and 16-row group:
//           bytes 0-127: 32 words, word 4 g + t (g = 0..7, t = 0..3) the high
//             bits of lane t's 8 codes of rows g and g+8: the code in nibble n
//             of row g's code word at bits P(n) = {4, 8, 6, 10, 20, 24, 22,
//             26}[n], row g+8's at P(n) + 8 (mod 32) -- a rotation by 8 moves
//             them onto row g's places (see q6h_regs);
//           bytes 128-159: per g, the sub-block scales (int8) of row g for k
//             0-15 and 16-31 of the block, then those of row g+8;
//   d     [mat][k/256][rows] fp16        the super-block scales
// scale_bytes covers aux followed by d (d starts at the aux size, a
// multiple of 16 bytes).
__device__ __forceinline__ int q6_code(const uint8_t* sb, int i) {
    const int h = i >> 7, r = i & 127, c = r >> 5, l = r & 31;
    const int byte = sb[64 * h + 32 * (c & 1) + l];
    const int low = c >= 2 ? (byte >> 4) : (byte & 15);
    const int high = (sb[128 + 32 * h + l] >> (2 * c)) & 3;
    return low | (high << 4);
}

// one thread per (matrix, 16-row group, 32-wide block)
__global__ void q6_k_pack_kernel(const uint8_t* __restrict__ blocks, int64_t n_mats, int64_t rows,
                                 int64_t nkb, uint8_t* __restrict__ codes, uint8_t* __restrict__ aux,
                                 uint16_t* __restrict__ dsc) {
    const int64_t groups = rows / 16;
    const int64_t total = n_mats * groups * nkb;
    const int pos[8] = {4, 8, 6, 10, 20, 24, 22, 26};
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t kb = i % nkb;
        const int64_t grp = (i / nkb) % groups;
        const int64_t m = i / (nkb * groups);
        const int64_t nsb = nkb / 8;
        uint32_t hw[32];
        uint8_t subs[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) hw[q] = 0u;
        for (int rr = 0; rr < 16; ++rr) {
            const int64_t r = grp * 16 + rr;
            const uint8_t* sb = blocks + ((m * rows + r) * nsb + kb / 8) * 210;   // canonical [m][r][sb]
            const int e0 = static_cast<int>(kb % 8) * 32;                         // first element of the block
            uint8_t low[32], high[32];
            for (int j = 0; j < 32; ++j) {
                const int q = q6_code(sb, e0 + j);
                low[j] = static_cast<uint8_t>(q & 15);
                high[j] = static_cast<uint8_t>(q >> 4);
            }
            uint32_t w[4];
            for (int t = 0; t < 4; ++t) {
                const int e = 2 * t;
                w[t] = static_cast<uint32_t>(low[e]) | (static_cast<uint32_t>(low[e + 8]) << 4) |
                       (static_cast<uint32_t>(low[e + 16]) << 8) | (static_cast<uint32_t>(low[e + 24]) << 12) |
                       (static_cast<uint32_t>(low[e + 1]) << 16) | (static_cast<uint32_t>(low[e + 9]) << 20) |
                       (static_cast<uint32_t>(low[e + 17]) << 24) | (static_cast<uint32_t>(low[e + 25]) << 28);
                // nibble n of word t holds element {0, 8, 16, 24, 1, 9, 17, 25}[n] + 2t
                const int elem[8] = {e, e + 8, e + 16, e + 24, e + 1, e + 9, e + 17, e + 25};
                const int g = rr & 7, shift = rr < 8 ? 0 : 8;
                for (int n = 0; n < 8; ++n)
                    hw[4 * g + t] |= static_cast<uint32_t>(high[elem[n]]) << ((pos[n] + shift) & 31);
            }
            const int64_t dst = (m * nkb + kb) * rows + r;                        // [m][kb][r]
            *reinterpret_cast<uint4*>(codes + dst * 16) = make_uint4(w[0], w[1], w[2], w[3]);
            const int sub0 = static_cast<int>(kb % 8) * 2;
            subs[(rr & 7) * 4 + (rr < 8 ? 0 : 2) + 0] = sb[192 + sub0];
            subs[(rr & 7) * 4 + (rr < 8 ? 0 : 2) + 1] = sb[192 + sub0 + 1];
            if (kb % 8 == 0)
                dsc[(m * nsb + kb / 8) * rows + r] = static_cast<uint16_t>(sb[208] | (sb[209] << 8));
        }
        uint8_t* rec = aux + ((m * nkb + kb) * groups + grp) * 160;
        for (int q = 0; q < 32; ++q) reinterpret_cast<uint32_t*>(rec)[q] = hw[q];
        for (int q = 0; q < 32; ++q) rec[128 + q] = subs[q];
    }
}

cudaError_t launch_q6_k_pack(const uint8_t* blocks, int64_t n_mats, int64_t rows, int64_t k,
                             uint8_t* codes, uint8_t* scales, cudaStream_t stream) {
    const int64_t total = n_mats * (rows / 16) * (k / 32);
    if (total == 0) return cudaSuccess;
    const int64_t aux_bytes = total * 160;
    const int threads = 128;
    const int64_t want = (total + threads - 1) / threads;
    const int grid = static_cast<int>(want < 65536 ? want : 65536);
    q6_k_pack_kernel<<<grid, threads, 0, stream>>>(blocks, n_mats, rows, k / 32, codes, scales,
                                                   reinterpret_cast<uint16_t*>(scales + aux_bytes));
    return cudaGetLastError();
}

// ---- bf16 -> fp16 (the down matrices of MOE_WFMT_BF16_F16DOWN)
__global__ void bf16_to_f16_kernel(const uint16_t* __restrict__ src, int64_t n,
                                   uint16_t* __restrict__ dst) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float v = __uint_as_float(static_cast<uint32_t>(src[i]) << 16);
        const __half h = __float2half_rn(v);
        dst[i] = *reinterpret_cast<const uint16_t*>(&h);
    }
}

cudaError_t launch_bf16_to_f16(const uint16_t* src, int64_t n, uint16_t* dst, cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t want = (n + threads - 1) / threads;
    const int grid = static_cast<int>(want < 65536 ? want : 65536);
    bf16_to_f16_kernel<<<grid, threads, 0, stream>>>(src, n, dst);
    return cudaGetLastError();
}

}  // namespace moe
