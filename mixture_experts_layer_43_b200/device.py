"""Device-memory plumbing around the C ABI: upload a layer's tensors with
PyTorch (device memory and streams only), repack Q4_0 / Q8_0 / Q5_0 through
the library's own moe_q4_0_pack / moe_q8_0_pack / moe_q5_0_pack kernels, and
fill the moe_weights_t / moe_config_t structs.  No arithmetic of the layer
happens here."""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import binding as B
from . import synth


def _dev(a: np.ndarray, device) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device, non_blocking=False)


class DeviceLayer:
    """One layer instance resident in HBM, ready for moe_forward."""

    def __init__(self, inp: synth.MoEInputs, device: str = "cuda:0",
                 stream: Optional[torch.cuda.Stream] = None):
        sh = inp.shape
        self.shape = sh
        self.device = torch.device(device)
        # quantised: codes + scales (bf16, and bf16 with fp16 down matrices,
        # upload as they are)
        self.q4 = sh.wfmt in (synth.WFMT_Q4_0, synth.WFMT_Q8_0, synth.WFMT_Q5_0, synth.WFMT_Q6_K)
        packed_bytes, pack = {
            synth.WFMT_BF16: (None, None),
            synth.WFMT_BF16_F16DOWN: (None, None),
            synth.WFMT_Q6_K: (B.moe_q6_k_packed_bytes, B.moe_q6_k_pack),
            synth.WFMT_Q4_0: (B.moe_q4_0_packed_bytes, B.moe_q4_0_pack),
            synth.WFMT_Q8_0: (B.moe_q8_0_packed_bytes, B.moe_q8_0_pack),
            synth.WFMT_Q5_0: (B.moe_q5_0_packed_bytes, B.moe_q5_0_pack)}[sh.wfmt]
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.router_w = _dev(inp.router_w.astype(np.float32), self.device)
        self.router_b = None if inp.router_b is None else _dev(inp.router_b.astype(np.float32),
                                                               self.device)
        self._keep = []

        def mat(arr, n_mats, rows, k):
            if arr is None:
                return B.moe_matrix_t(None, None)
            if not self.q4:
                t = _dev(arr, self.device)
                self._keep.append(t)
                return B.moe_matrix_t(t.data_ptr(), None)
            canon = _dev(arr.reshape(-1), self.device)
            cb, sb = packed_bytes(n_mats, rows, k)
            codes = torch.empty(cb, dtype=torch.uint8, device=self.device)
            scales = torch.empty(sb // 2, dtype=torch.int16, device=self.device)
            pack(canon.data_ptr(), n_mats, rows, k, codes.data_ptr(), scales.data_ptr(),
                 st.cuda_stream)
            st.synchronize()
            del canon
            self._keep += [codes, scales]
            return B.moe_matrix_t(codes.data_ptr(), scales.data_ptr())

        E, F, d, S, Fs = sh.E, sh.F, sh.d, sh.S, sh.Fs
        w = B.moe_weights_t()
        w.router_w = self.router_w.data_ptr()
        w.router_b = self.router_b.data_ptr() if self.router_b is not None else None
        w.gate = mat(inp.gate, E, F, d)
        w.up = mat(inp.up, E, F, d)
        w.down = mat(inp.down, E, d, F)
        has_shared = S > 0 and inp.shared_gate is not None
        if has_shared:
            w.shared_gate = mat(inp.shared_gate, S, Fs, d)
            w.shared_up = mat(inp.shared_up, S, Fs, d)
            w.shared_down = mat(inp.shared_down, S, d, Fs)
        self.weights = w
        self.n_shared = S if has_shared else 0

    def clone(self) -> "DeviceLayer":
        """Same values at new device addresses (a distinct instance for
        timing with cold caches)."""
        c = DeviceLayer.__new__(DeviceLayer)
        c.shape, c.device, c.q4, c.n_shared = self.shape, self.device, self.q4, self.n_shared
        c.router_w = self.router_w.clone()
        c.router_b = None if self.router_b is None else self.router_b.clone()
        c._keep = [t.clone() for t in self._keep]
        remap = {t.data_ptr(): n.data_ptr() for t, n in zip(self._keep, c._keep)}
        w = B.moe_weights_t()
        w.router_w = c.router_w.data_ptr()
        w.router_b = c.router_b.data_ptr() if c.router_b is not None else None
        for name in ("gate", "up", "down", "shared_gate", "shared_up", "shared_down"):
            m = getattr(self.weights, name)
            setattr(w, name, B.moe_matrix_t(remap.get(m.data) if m.data else None,
                                            remap.get(m.scales) if m.scales else None))
        c.weights = w
        return c

    def config(self, t_max: int, regime: int = B.MOE_REGIME_AUTO) -> B.moe_config_t:
        sh = self.shape
        return B.moe_config_t(t_max, sh.d, sh.F, sh.E, sh.k, self.n_shared,
                              sh.Fs if self.n_shared else 0, sh.wfmt, regime,
                              self.device.index or 0)

    def weight_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self._keep)


def random_bf16_layer(shape: synth.MoEShape, seed: int, device: str = "cuda:0") -> DeviceLayer:
    """A bf16 layer whose router and x come from synth (same routing as
    make_inputs with this seed) and whose expert weights are drawn on the
    device from a seeded N(0, w_std) generator -- for timing sweeps where the
    weight values do not matter and host generation would dominate."""
    assert shape.wfmt in (synth.WFMT_BF16, synth.WFMT_BF16_F16DOWN)
    inp = synth.make_inputs(shape, seed=seed, x_only=True)
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)

    def mats(n, rows, cols, down=False):
        t = torch.randn((n, rows, cols), generator=gen, device=dev, dtype=torch.float32)
        t = (t * shape.w_std).to(torch.bfloat16).view(torch.int16)
        if down and shape.wfmt == synth.WFMT_BF16_F16DOWN:
            # the library's own rounding of the bf16 draws to fp16
            h = torch.empty_like(t)
            B.moe_bf16_to_f16(t.data_ptr(), t.numel(), h.data_ptr(),
                              torch.cuda.current_stream(dev).cuda_stream)
            return h
        return t

    L = DeviceLayer.__new__(DeviceLayer)
    L.shape, L.device, L.q4 = shape, dev, False
    L.router_w = _dev(inp.router_w.astype(np.float32), dev)
    L.router_b = None if inp.router_b is None else _dev(inp.router_b.astype(np.float32), dev)
    E, F, d, S, Fs = shape.E, shape.F, shape.d, shape.S, shape.Fs
    L._keep = [mats(E, F, d), mats(E, F, d), mats(E, d, F, down=True)]
    w = B.moe_weights_t()
    w.router_w = L.router_w.data_ptr()
    w.router_b = L.router_b.data_ptr() if L.router_b is not None else None
    w.gate = B.moe_matrix_t(L._keep[0].data_ptr(), None)
    w.up = B.moe_matrix_t(L._keep[1].data_ptr(), None)
    w.down = B.moe_matrix_t(L._keep[2].data_ptr(), None)
    L.n_shared = 0
    if S:
        L._keep += [mats(S, Fs, d), mats(S, Fs, d), mats(S, d, Fs, down=True)]
        w.shared_gate = B.moe_matrix_t(L._keep[3].data_ptr(), None)
        w.shared_up = B.moe_matrix_t(L._keep[4].data_ptr(), None)
        w.shared_down = B.moe_matrix_t(L._keep[5].data_ptr(), None)
        L.n_shared = S
    L.weights = w
    return L, inp.x


def random_layer(shape: synth.MoEShape, seed: int, device: str = "cuda:0") -> DeviceLayer:
    """A layer of any weight format whose router and x come from synth (the
    same routing as make_inputs with this seed) and whose expert weights are
    drawn on the device from a seeded generator with the workload's
    distributions -- bf16 N(0, w_std); Q4_0 / Q8_0 / Q5_0 canonical blocks
    with codes uniform on their range and scales |N(0, std)| as fp16, then
    repacked by the library's own packer.  For timing, where the weight
    values do not matter and host generation would dominate."""
    if shape.wfmt in (synth.WFMT_BF16, synth.WFMT_BF16_F16DOWN):
        return random_bf16_layer(shape, seed, device)[0]
    inp = synth.make_inputs(shape, seed=seed, x_only=True)
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    packed_bytes, pack, std = {
        synth.WFMT_Q4_0: (B.moe_q4_0_packed_bytes, B.moe_q4_0_pack, shape.q4_scale_std),
        synth.WFMT_Q8_0: (B.moe_q8_0_packed_bytes, B.moe_q8_0_pack, shape.q8_scale_std),
        synth.WFMT_Q5_0: (B.moe_q5_0_packed_bytes, B.moe_q5_0_pack, shape.q5_scale_std),
        synth.WFMT_Q6_K: (B.moe_q6_k_packed_bytes, B.moe_q6_k_pack, shape.q6_scale_std)}[shape.wfmt]
    st = torch.cuda.current_stream(dev)

    def blocks(n_rows: int, k: int) -> torch.Tensor:
        if shape.wfmt == synth.WFMT_Q6_K:
            nsb = k // 256
            q = torch.randint(0, 64, (n_rows, nsb, 2, 4, 32), generator=gen, device=dev,
                              dtype=torch.int32)                         # [h][c][l]
            low, high = q & 15, q >> 4
            ql = torch.stack([low[:, :, :, 0] | (low[:, :, :, 2] << 4),
                              low[:, :, :, 1] | (low[:, :, :, 3] << 4)], dim=3)   # [h][c%2][l]
            qh = high[:, :, :, 0] | (high[:, :, :, 1] << 2) | (high[:, :, :, 2] << 4) | \
                (high[:, :, :, 3] << 6)
            sc = torch.randint(-128, 128, (n_rows, nsb, 16), generator=gen, device=dev,
                               dtype=torch.int32).to(torch.int8).view(torch.uint8)
            dd = (torch.randn((n_rows, nsb), generator=gen, device=dev) * std).abs().half()
            return torch.cat([ql.reshape(n_rows, nsb, 128).to(torch.uint8),
                              qh.reshape(n_rows, nsb, 64).to(torch.uint8), sc,
                              dd.view(torch.uint8).reshape(n_rows, nsb, 2)], dim=2)
        nb = k // 32
        sc = (torch.randn((n_rows, nb), generator=gen, device=dev) * std).abs().half()
        sc = sc.view(torch.uint8).reshape(n_rows, nb, 2)
        if shape.wfmt == synth.WFMT_Q8_0:
            q = torch.randint(0, 256, (n_rows, nb, 32), generator=gen, device=dev,
                              dtype=torch.int32).to(torch.uint8)
            return torch.cat([sc, q], dim=2)
        if shape.wfmt == synth.WFMT_Q4_0:
            q = torch.randint(0, 16, (n_rows, nb, 32), generator=gen, device=dev,
                              dtype=torch.int32)
            qs = (q[:, :, :16] | (q[:, :, 16:] << 4)).to(torch.uint8)
            return torch.cat([sc, qs], dim=2)
        q = torch.randint(0, 32, (n_rows, nb, 32), generator=gen, device=dev, dtype=torch.int64)
        bit = torch.arange(32, device=dev, dtype=torch.int64)
        qh = ((q >> 4) << bit).sum(dim=2)                               # fifth bits, bit j
        qh = torch.stack([(qh >> (8 * i)) & 255 for i in range(4)], dim=2).to(torch.uint8)
        lo = q & 15
        qs = (lo[:, :, :16] | (lo[:, :, 16:] << 4)).to(torch.uint8)
        return torch.cat([sc, qh, qs], dim=2)

    L = DeviceLayer.__new__(DeviceLayer)
    L.shape, L.device, L.q4 = shape, dev, True
    L.router_w = _dev(inp.router_w.astype(np.float32), dev)
    L.router_b = None if inp.router_b is None else _dev(inp.router_b.astype(np.float32), dev)
    L._keep = []

    def mat(n_mats, rows, k):
        cb, sb = packed_bytes(n_mats, rows, k)
        codes = torch.empty(cb, dtype=torch.uint8, device=dev)
        scales = torch.empty(sb // 2, dtype=torch.int16, device=dev)
        step = max(1, (1 << 26) // (rows * k))                  # bound the temporaries
        if shape.wfmt == synth.WFMT_Q6_K:
            step = n_mats          # the packed scales are two arrays (aux, then d): one call
        per_c, per_s = cb // n_mats, sb // n_mats
        for m0 in range(0, n_mats, step):
            m1 = min(n_mats, m0 + step)
            canon = blocks((m1 - m0) * rows, k)
            pack(canon.data_ptr(), m1 - m0, rows, k, codes.data_ptr() + m0 * per_c,
                 scales.data_ptr() + m0 * per_s, st.cuda_stream)
            st.synchronize()
        L._keep += [codes, scales]
        return B.moe_matrix_t(codes.data_ptr(), scales.data_ptr())

    E, F, d, S, Fs = shape.E, shape.F, shape.d, shape.S, shape.Fs
    w = B.moe_weights_t()
    w.router_w = L.router_w.data_ptr()
    w.router_b = L.router_b.data_ptr() if L.router_b is not None else None
    w.gate = mat(E, F, d)
    w.up = mat(E, F, d)
    w.down = mat(E, d, F)
    L.n_shared = 0
    if S:
        w.shared_gate = mat(S, Fs, d)
        w.shared_up = mat(S, Fs, d)
        w.shared_down = mat(S, d, Fs)
        L.n_shared = S
    L.weights = w
    return L


def upload_x(x_bits: np.ndarray, device) -> torch.Tensor:
    return _dev(x_bits, torch.device(device))


class Routing:
    """Device buffers for the routing tables moe_forward can copy out."""

    def __init__(self, T: int, k: int, E: int, device):
        dev = torch.device(device)
        self.ids = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.weights = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.slot_pair = torch.empty(T * k, dtype=torch.int32, device=dev)
        self.struct = B.moe_routing_t(self.ids.data_ptr(), self.weights.data_ptr(),
                                      self.counts.data_ptr(), self.offsets.data_ptr(),
                                      self.slot_pair.data_ptr())

    def numpy(self):
        return (self.ids.cpu().numpy(), self.weights.cpu().numpy(), self.counts.cpu().numpy(),
                self.offsets.cpu().numpy(), self.slot_pair.cpu().numpy())
