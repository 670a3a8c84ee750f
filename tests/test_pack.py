"""GPU test of the repacking kernels (moe_q4_0_pack, moe_q8_0_pack, moe_q5_0_pack,
moe_bf16_to_f16):
byte work, so bit-exact.  The packed arrays are decoded here with numpy by
inverting the layout include/moe.h documents, and the codes and scales must
equal those of the canonical blocks exactly."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_43_b200 import binding as B
from mixture_experts_layer_43_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


# (bit offset in the 32-bit word, element of the 32-wide block) for lane word t
def _word_slots(t):
    e = 2 * t
    return [(0, e), (4, e + 8), (8, e + 16), (12, e + 24),
            (16, e + 1), (20, e + 9), (24, e + 17), (28, e + 25)]


def _unpack_nibble_words(words):
    """[..., 4] uint32 words of one block row -> [..., 32] 4-bit values."""
    out = np.zeros(words.shape[:-1] + (32,), np.uint8)
    for t in range(4):
        for shift, idx in _word_slots(t):
            out[..., idx] = (words[..., t] >> shift) & 15
    return out


def _unpack_fifth_words(words):
    """[...] uint32 words of fifth bits of one block row -> [..., 32] bits:
    lane t's bits 4t+n and 16+4t+n belong to elements 2t+8n and 2t+1+8n."""
    out = np.zeros(words.shape + (32,), np.uint8)
    for t in range(4):
        for n in range(4):
            out[..., 2 * t + 8 * n] = (words >> (4 * t + n)) & 1
            out[..., 2 * t + 1 + 8 * n] = (words >> (16 + 4 * t + n)) & 1
    return out


def _pack_on_gpu(fn_bytes, fn_pack, canon, n_mats, rows, k):
    cb, sb = fn_bytes(n_mats, rows, k)
    src = torch.from_numpy(np.ascontiguousarray(canon).reshape(-1)).cuda()
    codes = torch.zeros(cb, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(sb // 2, dtype=torch.int16, device="cuda")
    fn_pack(src.data_ptr(), n_mats, rows, k, codes.data_ptr(), scales.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("n_mats,rows,k", [(1, 1, 32), (3, 40, 96), (2, 128, 512)])
def test_q4_0_pack_is_the_documented_permutation(n_mats, rows, k):
    rng = np.random.default_rng(n_mats * 1000 + rows)
    canon = synth.q4_0_blocks(rng, n_mats * rows, k, 0.01).reshape(n_mats, rows, k // 32, 18)
    codes, scales = _pack_on_gpu(B.moe_q4_0_packed_bytes, B.moe_q4_0_pack, canon, n_mats, rows, k)
    words = codes.view(np.uint32).reshape(n_mats, k // 32, rows, 4)
    got = _unpack_nibble_words(words).transpose(0, 2, 1, 3)          # [m][r][kb][32]
    want = np.concatenate([canon[..., 2:] & 15, canon[..., 2:] >> 4], axis=-1)
    assert np.array_equal(got, want)
    want_sc = canon[..., :2].copy().view(np.uint16)[..., 0]          # [m][r][kb]
    assert np.array_equal(scales.reshape(n_mats, k // 32, rows).transpose(0, 2, 1), want_sc)


@pytest.mark.parametrize("n_mats,rows,k", [(1, 1, 32), (3, 40, 96), (2, 128, 512)])
def test_q8_0_pack_is_the_documented_byte_order(n_mats, rows, k):
    rng = np.random.default_rng(n_mats * 1000 + rows + 7)
    canon = synth.q8_0_blocks(rng, n_mats * rows, k, 0.01).reshape(n_mats, rows, k // 32, 34)
    codes, scales = _pack_on_gpu(B.moe_q8_0_packed_bytes, B.moe_q8_0_pack, canon, n_mats, rows, k)
    packed = codes.reshape(n_mats, k // 32, rows, 32).astype(np.int32) - 128   # q = u - 128
    got = np.zeros_like(packed)
    for t in range(4):
        for n in range(8):
            got[..., 2 * t + (n & 1) + 8 * ((n >> 1) & 1) + 16 * (n >> 2)] = packed[..., 8 * t + n]
    got = got.transpose(0, 2, 1, 3)                                   # signed codes [m][r][kb][32]
    want = canon[..., 2:].copy().view(np.int8).astype(np.int32)
    assert np.array_equal(got, want)
    want_sc = canon[..., :2].copy().view(np.uint16)[..., 0]
    assert np.array_equal(scales.reshape(n_mats, k // 32, rows).transpose(0, 2, 1), want_sc)


@pytest.mark.parametrize("n_mats,rows,k", [(1, 8, 32), (3, 40, 96), (2, 128, 512)])
def test_q5_0_pack_is_the_documented_records(n_mats, rows, k):
    rng = np.random.default_rng(n_mats * 1000 + rows + 13)
    canon = synth.q5_0_blocks(rng, n_mats * rows, k, 0.01).reshape(n_mats, rows, k // 32, 22)
    codes, aux = _pack_on_gpu(B.moe_q5_0_packed_bytes, B.moe_q5_0_pack, canon, n_mats, rows, k)
    low = _unpack_nibble_words(codes.view(np.uint32).reshape(n_mats, k // 32, rows, 4))
    rec = aux.view(np.uint8).reshape(n_mats, k // 32, rows // 8, 48)
    sc = rec[..., :16].copy().view(np.uint16).reshape(n_mats, k // 32, rows)
    fifth = _unpack_fifth_words(rec[..., 16:].copy().view(np.uint32).reshape(n_mats, k // 32, rows))
    got = (low.astype(np.int32) + 16 * fifth).transpose(0, 2, 1, 3)    # [m][r][kb][32]
    qh = canon[..., 2:6].copy().view("<u4")[..., 0]
    want = np.concatenate([canon[..., 6:] & 15, canon[..., 6:] >> 4], axis=-1).astype(np.int32)
    want += 16 * ((qh[..., None] >> np.arange(32, dtype=np.uint32)) & 1).astype(np.int32)
    assert np.array_equal(got, want)
    want_sc = canon[..., :2].copy().view(np.uint16)[..., 0]
    assert np.array_equal(sc.transpose(0, 2, 1), want_sc)


def test_bf16_to_f16_every_pattern():
    """The library's bf16 -> fp16 rounding equals torch's (round to nearest
    even) bit for bit on all 65536 bf16 patterns (NaN stays NaN)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    src = torch.from_numpy(bits.view(np.int16)).cuda()
    dst = torch.zeros_like(src)
    B.moe_bf16_to_f16(src.data_ptr(), src.numel(), dst.data_ptr(),
                      torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float16)
    got = dst.cpu().view(torch.float16)
    nan = torch.isnan(want)
    assert torch.equal(torch.isnan(got), nan)
    assert torch.equal(got[~nan].view(torch.int16), want[~nan].view(torch.int16))


_Q6_POS = [4, 8, 6, 10, 20, 24, 22, 26]     # bit of the high pair of nibble n, row g


@pytest.mark.parametrize("n_mats,rows,k", [(1, 16, 256), (3, 48, 512), (2, 128, 1024)])
def test_q6_k_pack_is_the_documented_records(n_mats, rows, k):
    rng = np.random.default_rng(n_mats * 1000 + rows + 17)
    canon = synth.q6_k_blocks(rng, n_mats * rows, k, 0.01).reshape(n_mats, rows, k // 256, 210)
    codes, scales = _pack_on_gpu(B.moe_q6_k_packed_bytes, B.moe_q6_k_pack, canon, n_mats, rows, k)
    nkb = k // 32
    low = _unpack_nibble_words(codes.view(np.uint32).reshape(n_mats, nkb, rows, 4))   # [m][kb][r][32]
    sb = scales.view(np.uint8)
    aux_bytes = n_mats * nkb * (rows // 16) * 160
    rec = sb[:aux_bytes].reshape(n_mats, nkb, rows // 16, 160)
    hw = rec[..., :128].copy().view(np.uint32).reshape(n_mats, nkb, rows // 16, 8, 4)  # [g][t]
    high = np.zeros((n_mats, nkb, rows, 32), np.int32)
    for t in range(4):
        slots = _word_slots(t)                     # (bit offset, element) of nibble n = offset // 4
        for shift, idx in slots:
            n = shift // 4
            for half in (0, 1):                    # rows g and g + 8
                p = (_Q6_POS[n] + 8 * half) % 32
                v = (hw[..., t] >> p) & 3          # [m][kb][grp][g]
                rr = (np.arange(rows // 16)[:, None] * 16 + np.arange(8)[None, :] + 8 * half)
                high[:, :, rr.reshape(-1), idx] = v.reshape(n_mats, nkb, -1)
    got = (low.astype(np.int32) + 16 * high).transpose(0, 2, 1, 3).reshape(n_mats, rows, k)
    # canonical codes by the layout statement (element i = 128 h + 32 c + l)
    ql = canon[..., :128].reshape(n_mats, rows, k // 256, 2, 2, 32).astype(np.int32)
    qh = canon[..., 128:192].reshape(n_mats, rows, k // 256, 2, 32).astype(np.int32)
    want = np.zeros((n_mats, rows, k // 256, 2, 4, 32), np.int32)
    for c in range(4):
        lo = (ql[..., :, c % 2, :] >> 4) if c >= 2 else (ql[..., :, c % 2, :] & 15)
        want[..., c, :] = lo + 16 * ((qh >> (2 * c)) & 3)
    assert np.array_equal(got, want.reshape(n_mats, rows, k))
    subs = rec[..., 128:].reshape(n_mats, nkb, rows // 16, 8, 2, 2).view(np.int8)   # [g][row g/g+8][s]
    got_sc = np.zeros((n_mats, rows, nkb, 2), np.int8)
    for half in (0, 1):
        rr = (np.arange(rows // 16)[:, None] * 16 + np.arange(8)[None, :] + 8 * half).reshape(-1)
        got_sc[:, rr, :, :] = subs[:, :, :, :, half, :].reshape(n_mats, nkb, -1, 2).transpose(0, 2, 1, 3)
    want_sc = canon[..., 192:208].copy().view(np.int8).reshape(n_mats, rows, k // 256, 8, 2)
    assert np.array_equal(got_sc, want_sc.reshape(n_mats, rows, nkb, 2))
    dd = sb[aux_bytes:].copy().view(np.uint16).reshape(n_mats, k // 256, rows)
    want_d = canon[..., 208:210].copy().view(np.uint16)[..., 0]                        # [m][r][sb]
    assert np.array_equal(dd.transpose(0, 2, 1), want_d)

