"""Seeded synthetic inputs for the MoE SwiGLU layer forward pass.

This module is the only code shared by the CUDA path (through the bench and
the tests) and the fp64 oracle.  It generates data and nothing else: it holds
none of the layer's arithmetic (no router, no top-k, no SwiGLU, no dequant).

Workloads follow the shapes of the MoE layers the source pages discuss
("Fused MoE Triton kernel: 5 launches instead of 24" page, layer-time table:
Mixtral-8x7B and DeepSeek-MoE-16B; "MoE on RTX 5090 reaches 41% of bandwidth"
page: a 35B-A3B model with 256 experts, 8 routed + 1 shared per token, Q4_0).
No trained weights exist here, so every tensor is drawn from a seeded PCG64
stream with the distribution stated per workload.

Storage conventions (the C ABI's, see include/moe.h):
  x         bf16 bits, uint16 [T][d]
  router_w  fp32 [E][d]      (row e is expert e's router vector)
  router_b  fp32 [E] or None
  gate, up  bf16 bits [E][F][d]  (row f, reduction dim d contiguous)
  down      bf16 bits [E][d][F]  (row j, reduction dim F contiguous)
  shared_*  the same with S experts of hidden size Fs
  Q4_0      canonical 18-byte blocks along the reduction dim:
            [rows][K/32][18] = fp16 scale (little endian) + 16 code bytes,
            byte j holding element j (low nibble) and element j+16 (high).
  Q8_0      [rows][K/32][34] = fp16 scale + 32 signed code bytes.
  Q5_0      [rows][K/32][22] = fp16 scale + 32-bit little-endian word of
            fifth bits (bit j for element j) + 16 bytes of low nibbles
            packed as in Q4_0.
  q6_K      [rows][K/256][210] super-blocks of 256 weights = ql[128] (low 4
            bits) + qh[64] (high 2 bits) + 16 signed 8-bit sub-block scales
            + fp16 super-block scale; element i of a super-block takes its
            low bits from the low (quarter c = (i%128)/32 < 2) or high nibble
            of ql[64*(i//128) + 32*(c%2) + i%32] and its high bits from bits
            2c, 2c+1 of qh[32*(i//128) + i%32]; weight d*sc[i//16]*(q-32).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

WFMT_BF16 = 0
WFMT_Q4_0 = 1
WFMT_Q8_0 = 2
WFMT_Q5_0 = 3
WFMT_Q6_K = 4
WFMT_BF16_F16DOWN = 5      # gate/up bf16; down matrices rounded once to fp16
Q4_BLOCK = 32          # weights per Q4_0 block
Q4_BLOCK_BYTES = 18    # 2-byte fp16 scale + 16 bytes of 4-bit codes
Q8_BLOCK_BYTES = 34    # 2-byte fp16 scale + 32 signed 8-bit codes
Q5_BLOCK_BYTES = 22    # 2-byte fp16 scale + 4 bytes of fifth bits + 16 bytes of nibbles
Q6_SUPER = 256         # weights per q6_K super-block
Q6_SUPER_BYTES = 210   # 128 + 64 code bytes, 16 sub-block scales, 2-byte fp16 scale


@dataclasses.dataclass(frozen=True)
class MoEShape:
    """Shape of one MoE layer call."""
    name: str
    T: int            # tokens in the call
    d: int            # d_model
    E: int            # routed experts
    k: int            # top-k
    F: int            # routed expert hidden size (d_ff)
    S: int = 0        # shared experts (always on, weight 1)
    Fs: int = 0       # hidden size of each shared expert
    wfmt: int = WFMT_BF16
    zipf_bias: float = 0.0   # >0: router bias log(Zipf(s)) per expert
    w_std: float = 0.02
    wr_std: float = 0.02
    q4_scale_std: float = 0.005
    q8_scale_std: float = 0.00035
    q5_scale_std: float = 0.0025
    q6_scale_std: float = 1.5e-5     # super-block scale; sub-scales uniform on -128..127

    def replace(self, **kw) -> "MoEShape":
        return dataclasses.replace(self, **kw)


# The workloads.  Sizes are those of the layers the pages name; the names say
# what each one is.
WORKLOADS = {
    "tiny_T4_d256_E8k2_F512": MoEShape(
        "tiny_T4_d256_E8k2_F512", T=4, d=256, E=8, k=2, F=512),
    "mixtral_T8_d4096_E8k2_F14336": MoEShape(
        "mixtral_T8_d4096_E8k2_F14336", T=8, d=4096, E=8, k=2, F=14336),
    "a3b_T1_d2048_E256k8_F512_S1": MoEShape(
        "a3b_T1_d2048_E256k8_F512_S1", T=1, d=2048, E=256, k=8, F=512,
        S=1, Fs=512),
    "a3b_q4_T1_d2048_E256k8_F512_S1": MoEShape(
        "a3b_q4_T1_d2048_E256k8_F512_S1", T=1, d=2048, E=256, k=8, F=512,
        S=1, Fs=512, wfmt=WFMT_Q4_0),
    "a3b_q4_T8_d2048_E256k8_F512_S1": MoEShape(
        "a3b_q4_T8_d2048_E256k8_F512_S1", T=8, d=2048, E=256, k=8, F=512,
        S=1, Fs=512, wfmt=WFMT_Q4_0),
    # the same 35B-A3B layer with Q8_0 weights (another format of the model's mix)
    "a3b_q8_T1_d2048_E256k8_F512_S1": MoEShape(
        "a3b_q8_T1_d2048_E256k8_F512_S1", T=1, d=2048, E=256, k=8, F=512,
        S=1, Fs=512, wfmt=WFMT_Q8_0),
    "a3b_q8_T8_d2048_E256k8_F512_S1": MoEShape(
        "a3b_q8_T8_d2048_E256k8_F512_S1", T=8, d=2048, E=256, k=8, F=512,
        S=1, Fs=512, wfmt=WFMT_Q8_0),
    # ... and with Q5_0 weights (also in the model's mix)
    "a3b_q5_T1_d2048_E256k8_F512_S1": MoEShape(
        "a3b_q5_T1_d2048_E256k8_F512_S1", T=1, d=2048, E=256, k=8, F=512,
        S=1, Fs=512, wfmt=WFMT_Q5_0),
    "a3b_q5_T8_d2048_E256k8_F512_S1": MoEShape(
        "a3b_q5_T8_d2048_E256k8_F512_S1", T=8, d=2048, E=256, k=8, F=512,
        S=1, Fs=512, wfmt=WFMT_Q5_0),
    # ... and with q6_K weights (also in the model's mix; 256-weight super-blocks)
    "a3b_q6_T1_d2048_E256k8_F512_S1": MoEShape(
        "a3b_q6_T1_d2048_E256k8_F512_S1", T=1, d=2048, E=256, k=8, F=512,
        S=1, Fs=512, wfmt=WFMT_Q6_K),
    "a3b_q6_T8_d2048_E256k8_F512_S1": MoEShape(
        "a3b_q6_T8_d2048_E256k8_F512_S1", T=8, d=2048, E=256, k=8, F=512,
        S=1, Fs=512, wfmt=WFMT_Q6_K),
    # the same 35B-A3B layer in bf16 at T = 8 (about 58 distinct experts, 0.37 GB)
    "a3b_T8_d2048_E256k8_F512_S1": MoEShape(
        "a3b_T8_d2048_E256k8_F512_S1", T=8, d=2048, E=256, k=8, F=512, S=1, Fs=512),
    # A smaller case of the Mixtral-shaped decode kernel (same T, d, E, k;
    # F cut to 2048 so the whole layer is 0.4 GB) for detailed profiling.
    "mixtral_small_T8_d4096_E8k2_F2048": MoEShape(
        "mixtral_small_T8_d4096_E8k2_F2048", T=8, d=4096, E=8, k=2, F=2048),
    "deepseek_T4096_d2048_E64k6_F1408_S2": MoEShape(
        "deepseek_T4096_d2048_E64k6_F1408_S2", T=4096, d=2048, E=64, k=6,
        F=1408, S=2, Fs=1408, zipf_bias=1.1),
    # the same prefill layer with its down matrices rounded once to fp16, so
    # that h can be stored in fp16 between the two GEMMs (precision headroom)
    "deepseek_f16down_T4096_d2048_E64k6_F1408_S2": MoEShape(
        "deepseek_f16down_T4096_d2048_E64k6_F1408_S2", T=4096, d=2048, E=64, k=6,
        F=1408, S=2, Fs=1408, zipf_bias=1.1, wfmt=WFMT_BF16_F16DOWN),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f16_bits(a: np.ndarray) -> np.ndarray:
    """Round bf16 values to IEEE fp16 (nearest, ties to even; numpy's
    conversion); return the fp16 bits.  Exact for 2^-17 <= |w| <= 65504."""
    f = (np.ascontiguousarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    return f.astype(np.float16).view(np.uint16)


def _normal_bf16(rng: np.random.Generator, shape, std: float,
                 chunk: int = 1 << 24) -> np.ndarray:
    """N(0, std) samples rounded to bf16, generated in chunks to bound memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        v = rng.standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[s:e] = f32_to_bf16_bits(v)
    return out.reshape(shape)


def zipf_log_bias(E: int, s: float) -> np.ndarray:
    """Per-expert router offset log(p_e), p_e = (e+1)^-s / sum_r r^-s.

    Expert 0 is the most popular.  The normalising constant cancels in the
    softmax; it is kept so that the values are the log-probabilities.
    """
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    return np.log(p).astype(np.float32)


def q4_0_blocks(rng: np.random.Generator, rows: int, k: int,
                scale_std: float) -> np.ndarray:
    """Canonical Q4_0 blocks [rows][k/32][18] with uniform codes and
    scales |N(0, scale_std)| stored as fp16."""
    assert k % Q4_BLOCK == 0
    nb = k // Q4_BLOCK
    out = np.empty((rows, nb, Q4_BLOCK_BYTES), dtype=np.uint8)
    step = max(1, (1 << 22) // max(1, nb))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        q = rng.integers(0, 16, size=(r1 - r0, nb, Q4_BLOCK), dtype=np.uint8)
        sc = np.abs(rng.standard_normal((r1 - r0, nb), dtype=np.float32)
                    * np.float32(scale_std)).astype(np.float16)
        out[r0:r1, :, 0:2] = sc.view(np.uint8).reshape(r1 - r0, nb, 2)
        out[r0:r1, :, 2:] = q[:, :, :16] | (q[:, :, 16:] << 4)
    return out


def q8_0_blocks(rng: np.random.Generator, rows: int, k: int,
                scale_std: float) -> np.ndarray:
    """Canonical Q8_0 blocks [rows][k/32][34] with codes uniform on
    -128..127 and scales |N(0, scale_std)| stored as fp16."""
    assert k % Q4_BLOCK == 0
    nb = k // Q4_BLOCK
    out = np.empty((rows, nb, Q8_BLOCK_BYTES), dtype=np.uint8)
    step = max(1, (1 << 22) // max(1, nb))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        q = rng.integers(0, 256, size=(r1 - r0, nb, Q4_BLOCK), dtype=np.uint8)
        sc = np.abs(rng.standard_normal((r1 - r0, nb), dtype=np.float32)
                    * np.float32(scale_std)).astype(np.float16)
        out[r0:r1, :, 0:2] = sc.view(np.uint8).reshape(r1 - r0, nb, 2)
        out[r0:r1, :, 2:] = q
    return out


def q5_0_blocks(rng: np.random.Generator, rows: int, k: int,
                scale_std: float) -> np.ndarray:
    """Canonical Q5_0 blocks [rows][k/32][22] with codes uniform on 0..31
    and scales |N(0, scale_std)| stored as fp16."""
    assert k % Q4_BLOCK == 0
    nb = k // Q4_BLOCK
    out = np.empty((rows, nb, Q5_BLOCK_BYTES), dtype=np.uint8)
    step = max(1, (1 << 22) // max(1, nb))
    bit = (np.uint32(1) << np.arange(32, dtype=np.uint32)).astype(np.uint32)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        q = rng.integers(0, 32, size=(r1 - r0, nb, Q4_BLOCK), dtype=np.uint8)
        sc = np.abs(rng.standard_normal((r1 - r0, nb), dtype=np.float32)
                    * np.float32(scale_std)).astype(np.float16)
        qh = ((q >> 4).astype(np.uint32) * bit).sum(axis=2, dtype=np.uint32)
        lo = q & 15
        out[r0:r1, :, 0:2] = sc.view(np.uint8).reshape(r1 - r0, nb, 2)
        out[r0:r1, :, 2:6] = qh.astype("<u4").view(np.uint8).reshape(r1 - r0, nb, 4)
        out[r0:r1, :, 6:] = lo[:, :, :16] | (lo[:, :, 16:] << 4)
    return out


def q6_k_blocks(rng: np.random.Generator, rows: int, k: int,
                scale_std: float) -> np.ndarray:
    """Canonical q6_K super-blocks [rows][k/256][210] with codes uniform on
    0..63, sub-block scales uniform on -128..127 and super-block scales
    |N(0, scale_std)| stored as fp16."""
    assert k % Q6_SUPER == 0
    nb = k // Q6_SUPER
    out = np.empty((rows, nb, Q6_SUPER_BYTES), dtype=np.uint8)
    step = max(1, (1 << 20) // max(1, nb))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        n = r1 - r0
        q = rng.integers(0, 64, size=(n, nb, Q6_SUPER), dtype=np.uint8)
        sc = rng.integers(-128, 128, size=(n, nb, 16), dtype=np.int16).astype(np.int8)
        d = np.abs(rng.standard_normal((n, nb), dtype=np.float32)
                   * np.float32(scale_std)).astype(np.float16)
        # element i = 128 h + 32 c + l
        qq = q.reshape(n, nb, 2, 4, 32)                         # [h][c][l]
        low, high = qq & 15, qq >> 4
        ql = np.empty((n, nb, 2, 2, 32), dtype=np.uint8)        # [h][c % 2][l]
        ql[:, :, :, 0] = low[:, :, :, 0] | (low[:, :, :, 2] << 4)
        ql[:, :, :, 1] = low[:, :, :, 1] | (low[:, :, :, 3] << 4)
        qh = (high[:, :, :, 0] | (high[:, :, :, 1] << 2) | (high[:, :, :, 2] << 4)
              | (high[:, :, :, 3] << 6))                        # [h][l]
        out[r0:r1, :, 0:128] = ql.reshape(n, nb, 128)
        out[r0:r1, :, 128:192] = qh.reshape(n, nb, 64)
        out[r0:r1, :, 192:208] = sc.view(np.uint8)
        out[r0:r1, :, 208:210] = d.view(np.uint8).reshape(n, nb, 2)
    return out


@dataclasses.dataclass
class MoEInputs:
    shape: MoEShape
    x: np.ndarray                 # uint16 bf16 bits [T][d]
    router_w: np.ndarray          # float32 [E][d]
    router_b: Optional[np.ndarray]  # float32 [E] or None
    gate: np.ndarray              # bf16 bits [E][F][d] or blocks [E][F][d/32][block bytes]
    up: np.ndarray
    down: np.ndarray              # bf16 bits [E][d][F] or blocks [E][d][F/32][block bytes]
    shared_gate: Optional[np.ndarray]
    shared_up: Optional[np.ndarray]
    shared_down: Optional[np.ndarray]


def make_inputs(shape: MoEShape, seed: int = 0,
                x_only: bool = False) -> MoEInputs:
    """Generate one layer instance.  Each tensor has its own PCG64 stream
    derived from (seed, tensor index), so changing T leaves the weights
    unchanged and x's first rows are stable."""
    sh = shape

    def rng(i):
        return np.random.Generator(np.random.PCG64([seed, i]))

    x = _normal_bf16(rng(1), (sh.T, sh.d), 1.0)
    wr = (rng(2).standard_normal((sh.E, sh.d), dtype=np.float32)
          * np.float32(sh.wr_std))
    rb = zipf_log_bias(sh.E, sh.zipf_bias) if sh.zipf_bias > 0 else None
    if x_only:
        return MoEInputs(sh, x, wr, rb, None, None, None, None, None, None)
    if sh.wfmt in (WFMT_BF16, WFMT_BF16_F16DOWN):
        g = _normal_bf16(rng(3), (sh.E, sh.F, sh.d), sh.w_std)
        u = _normal_bf16(rng(4), (sh.E, sh.F, sh.d), sh.w_std)
        dn = _normal_bf16(rng(5), (sh.E, sh.d, sh.F), sh.w_std)
        if sh.S:
            sg = _normal_bf16(rng(6), (sh.S, sh.Fs, sh.d), sh.w_std)
            su = _normal_bf16(rng(7), (sh.S, sh.Fs, sh.d), sh.w_std)
            sd = _normal_bf16(rng(8), (sh.S, sh.d, sh.Fs), sh.w_std)
        else:
            sg = su = sd = None
        if sh.wfmt == WFMT_BF16_F16DOWN:     # the same bf16 draws, down rounded to fp16
            dn = bf16_bits_to_f16_bits(dn)
            sd = None if sd is None else bf16_bits_to_f16_bits(sd)
    else:
        blocks, q, nbytes, per = {
            WFMT_Q4_0: (q4_0_blocks, sh.q4_scale_std, Q4_BLOCK_BYTES, Q4_BLOCK),
            WFMT_Q8_0: (q8_0_blocks, sh.q8_scale_std, Q8_BLOCK_BYTES, Q4_BLOCK),
            WFMT_Q5_0: (q5_0_blocks, sh.q5_scale_std, Q5_BLOCK_BYTES, Q4_BLOCK),
            WFMT_Q6_K: (q6_k_blocks, sh.q6_scale_std, Q6_SUPER_BYTES, Q6_SUPER)}[sh.wfmt]

        def stack(i, mats, rows, kk):
            return blocks(rng(i), mats * rows, kk, q).reshape(mats, rows, kk // per, nbytes)
        g = stack(3, sh.E, sh.F, sh.d)
        u = stack(4, sh.E, sh.F, sh.d)
        dn = stack(5, sh.E, sh.d, sh.F)
        if sh.S:
            sg = stack(6, sh.S, sh.Fs, sh.d)
            su = stack(7, sh.S, sh.Fs, sh.d)
            sd = stack(8, sh.S, sh.d, sh.Fs)
        else:
            sg = su = sd = None
    return MoEInputs(sh, x, wr, rb, g, u, dn, sg, su, sd)


def weight_bytes_per_expert(shape: MoEShape, hidden: Optional[int] = None) -> int:
    """Bytes one expert's three matrices occupy in HBM in the kernel format."""
    F = shape.F if hidden is None else hidden
    n = 3 * F * shape.d
    if shape.wfmt in (WFMT_BF16, WFMT_BF16_F16DOWN):
        return 2 * n
    if shape.wfmt == WFMT_Q4_0:
        return n // 32 * 18   # 16 code bytes + 2 scale bytes per 32 weights
    if shape.wfmt == WFMT_Q5_0:
        return n // 32 * 22   # 16 nibble bytes + 4 fifth-bit bytes + 2 scale bytes
    if shape.wfmt == WFMT_Q6_K:
        return n // 256 * 210  # 192 code bytes + 16 sub-scales + 2 scale bytes
    return n // 32 * 34       # 32 code bytes + 2 scale bytes per 32 weights


def expert_flops(shape: MoEShape, n_tokens: int, hidden: Optional[int] = None) -> int:
    F = shape.F if hidden is None else hidden
    return 2 * 3 * F * shape.d * n_tokens


def describe(shape: MoEShape) -> str:
    fmt = {WFMT_BF16: "bf16", WFMT_Q4_0: "q4_0", WFMT_Q8_0: "q8_0",
           WFMT_Q5_0: "q5_0", WFMT_Q6_K: "q6_k", WFMT_BF16_F16DOWN: "bf16/f16-down"}[shape.wfmt]
    s = (f"T={shape.T} d={shape.d} E={shape.E} k={shape.k} F={shape.F} "
         f"S={shape.S} Fs={shape.Fs} {fmt}")
    if shape.zipf_bias:
        s += f" zipf_bias={shape.zipf_bias}"
    return s


def log2_ceil(n: int) -> int:
    return int(math.ceil(math.log2(max(1, n))))
