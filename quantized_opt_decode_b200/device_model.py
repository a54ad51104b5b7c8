"""Device-memory plumbing: a synthetic OPT-style model and its KV caches.

torch provides the allocations; every value is produced by libflexq
(flexq_synth_* for the seeded draws, flexq_quantize_weight_q4 for the 4-bit
tiled weights).  The tensor ids and distributions follow the ``synth``
recipe, so the host-side generator reproduces any tensor for checking.
"""
from __future__ import annotations

import ctypes as C
import math

import torch

import synth
from . import flexq as fq

LINEAR = ("w_qkv", "w_o", "w_fc1", "w_fc2")


def make_config(p: dict) -> fq.flexq_config:
    return fq.flexq_config(h=p["h"], heads=p["heads"], ffn=p["ffn"], w_bits=p["w_bits"],
                           kv_bits=p["kv_bits"], ln_eps=1e-5,
                           attn_topk_permille=p.get("topk_permille", 0),
                           prefill_kv_cache=int(bool(p.get("prefill_kv_cache", False))))


def fill_normal(t: torch.Tensor, seed: int, tid: int, sigma: float = 0.02, mean: float = 0.0,
                stream=None):
    fq.flexq_synth_normal_f16(t, t.numel(), seed, tid, 0, sigma, mean, stream)


class KVCache:
    """One layer's cache: K/V codes (or fp16 values) and their (min, scale)
    metadata, laid out as include/flexq.h describes."""

    def __init__(self, cfg: fq.flexq_config, b: int, max_len: int, device="cuda"):
        d = cfg.h // cfg.heads
        slots = b * cfg.heads * max_len
        if cfg.kv_bits == 4:
            self.k = torch.zeros(slots * d // 2, dtype=torch.uint8, device=device)
            # V codes: whole 8-token blocks of 32-bit words (token-interleaved)
            l8 = (max_len + 7) // 8 * 8
            self.v = torch.zeros(b * cfg.heads * l8 * d // 2, dtype=torch.uint8, device=device)
            self.k_meta = torch.zeros(slots * (d // 64) * 2, dtype=torch.float16, device=device)
            self.v_meta = torch.zeros_like(self.k_meta)
        else:
            self.k = torch.zeros(slots * d, dtype=torch.float16, device=device)
            self.v = torch.zeros_like(self.k)
            self.k_meta = self.v_meta = None
        self.b, self.max_len, self.heads, self.d = b, max_len, cfg.heads, d
        self.struct = fq.flexq_kv(self.k.data_ptr(), self.v.data_ptr(),
                                  self.k_meta.data_ptr() if self.k_meta is not None else None,
                                  self.v_meta.data_ptr() if self.v_meta is not None else None,
                                  b, max_len)

    def nbytes(self) -> int:
        n = self.k.numel() * self.k.element_size() + self.v.numel() * self.v.element_size()
        if self.k_meta is not None:
            n += (self.k_meta.numel() + self.v_meta.numel()) * 2
        return n


class DeviceLayer:
    """One decoder layer's parameters on the device (with offload=True the four
    weight matrices end up in page-locked host memory instead)."""

    def __init__(self, cfg: fq.flexq_config, seed: int, layer: int, scratch: torch.Tensor | None,
                 device="cuda", stream=None, offload: bool = False):
        self.t = {}
        for name in synth.LAYER_TENSORS:
            shape, sigma, mean = synth.layer_tensor_spec(name, cfg.h, cfg.ffn)
            tid = synth.layer_tensor_id(layer, name)
            if name in LINEAR and cfg.w_bits == 4:
                n_out, k_in = shape
                numel = n_out * k_in
                tmp = scratch[:numel] if scratch is not None else torch.empty(
                    numel, dtype=torch.float16, device=device)
                fill_normal(tmp, seed, tid, sigma, mean, stream)
                packed = torch.empty(fq.flexq_packed_weight_bytes(n_out, k_in), dtype=torch.uint8,
                                     device=device)
                fq.flexq_quantize_weight_q4(tmp, n_out, k_in, packed, stream)
                self.t[name] = packed
            else:
                buf = torch.empty(shape, dtype=torch.float16, device=device)
                fill_normal(buf, seed, tid, sigma, mean, stream)
                self.t[name] = buf
            if offload and name in LINEAR:
                dev = self.t[name]
                host = torch.empty(dev.shape, dtype=dev.dtype, pin_memory=True)
                if stream is not None:
                    stream.synchronize()
                host.copy_(dev)
                self.t[name] = host
                del dev
        self.struct = fq.flexq_layer(*[self.t[n].data_ptr() for n in (
            "w_qkv", "w_o", "w_fc1", "w_fc2", "b_qkv", "b_o", "b_fc1", "b_fc2",
            "ln1_g", "ln1_b", "ln2_g", "ln2_b")])


class DeviceModel:
    """Synthetic model (seeded draws, 4-bit or fp16 weights) plus KV caches for
    a block of b sequences of up to max_len positions."""

    def __init__(self, preset: dict, b: int, max_len: int, layers: int | None = None,
                 device="cuda", stream=None, with_kv: bool = True, offload: bool = False):
        self.p = preset
        self.cfg = make_config(preset)
        self.seed = synth.config_seed(preset)
        self.nl = preset["layers"] if layers is None else layers
        cfg = self.cfg
        scratch = None
        if cfg.w_bits == 4:
            scratch = torch.empty(max(3 * cfg.h * cfg.h, cfg.ffn * cfg.h), dtype=torch.float16,
                                  device=device)
        self.offload = offload
        self.layers = [DeviceLayer(cfg, self.seed, i, scratch, device, stream, offload)
                       for i in range(self.nl)]
        del scratch
        self.max_pos = max_len
        self.embed_bits = preset.get("embed_bits", 16)
        self.E = torch.empty(preset["vocab"], cfg.h, dtype=torch.float16, device=device)
        self.P = torch.empty(max_len, cfg.h, dtype=torch.float16, device=device)
        self.lnf_g = torch.empty(cfg.h, dtype=torch.float16, device=device)
        self.lnf_b = torch.empty(cfg.h, dtype=torch.float16, device=device)
        fill_normal(self.E, self.seed, synth.TID_EMBED, stream=stream)
        if self.embed_bits == 4:
            # the tied embedding in the linear layers' 4-bit tiled layout
            packed = torch.empty(fq.flexq_packed_weight_bytes(preset["vocab"], cfg.h), dtype=torch.uint8,
                                 device=device)
            fq.flexq_quantize_weight_q4(self.E, preset["vocab"], cfg.h, packed, stream)
            self.E = packed
        fill_normal(self.P, self.seed, synth.TID_POS, stream=stream)
        fill_normal(self.lnf_g, self.seed, synth.TID_LNF_G, 0.02, 1.0, stream)
        fill_normal(self.lnf_b, self.seed, synth.TID_LNF_B, stream=stream)
        self.device = device
        self._layer_arr = (fq.flexq_layer * self.nl)(*[L.struct for L in self.layers])
        self.alloc_kv(b if with_kv else 0, max_len)

    def alloc_kv(self, b: int, max_len: int):
        """(Re)allocates every layer's KV cache for b sequences (none for 0)."""
        self.kv = []
        self.kv = [KVCache(self.cfg, b, max_len, self.device) for _ in range(self.nl)] if b > 0 else []
        self.b = b
        self._kv_arr = (fq.flexq_kv * max(1, len(self.kv)))(*[k.struct for k in self.kv]) \
            if self.kv else None
        self.struct = fq.flexq_model(self.cfg, self.nl, self.p["vocab"], self.max_pos, self._layer_arr,
                                     self._kv_arr, self.E.data_ptr(), self.P.data_ptr(),
                                     self.lnf_g.data_ptr(), self.lnf_b.data_ptr(), self.embed_bits)

    def weight_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for L in self.layers for t in L.t.values())


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(1, nbytes), dtype=torch.uint8, device=device)


def normal_scale(sigma: float) -> float:
    return math.sqrt(3.0) / 65536.0 * sigma


def as_void_p(t: torch.Tensor) -> C.c_void_p:
    return C.c_void_p(t.data_ptr())
