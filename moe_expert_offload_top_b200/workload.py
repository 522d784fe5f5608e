"""Runs a synthetic workload (synth.configs.MoeConfig) through the C ABI.

GpuStack owns one ft_moe handle: it fills the library's pinned pool with the
seeded expert blobs, loads shared experts and router weights to the device,
and runs steps (one batch of tokens through every layer) with ft_moe_forward.
PyTorch only provides device memory and the stream.
"""
import ctypes
import os

import numpy as np
import torch

import synth

from . import (ft_cache_reset_stats, ft_cache_resize, ft_cache_stats, ft_cache_trace,
               ft_moe_blob_bytes, ft_moe_create, ft_moe_destroy, ft_moe_forward,
               ft_moe_last_routing, ft_moe_pool_ptr, ft_moe_reserve, ft_moe_set_layers,
               ft_moe_set_mode, ft_moe_set_shared)


def _to_device_tokens(cfg, vals, bits, device):
    if cfg.x_dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(vals)).to(device)


class GpuStack:
    def __init__(self, cfg, capacity=None, device="cuda", fill_threads=None, max_tokens=None):
        self.cfg = cfg
        self.device = torch.device(device)
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        torch.cuda.set_device(self.device)
        self.C = cfg.C if capacity is None else capacity
        self.h = ft_moe_create(cfg.E, cfg.k, cfg.H, cfg.I, cfg.wdtype, self.C)
        ft_moe_set_layers(self.h, cfg.L, cfg.gating, cfg.shared)
        ft_moe_set_mode(self.h, cfg.mode == "prefill")
        self.blob = ft_moe_blob_bytes(self.h)
        assert self.blob == cfg.blob_bytes
        self.pool_base = ft_moe_pool_ptr(self.h, 0, 0)
        synth.fill_pool(cfg, self.pool_base, self.blob, fill_threads or os.cpu_count())
        self.shared_blobs = {}
        if cfg.shared:
            for l in range(cfg.L):
                b = synth.expert_blob(cfg, l, 0, shared=True)
                self.shared_blobs[l] = b
                ft_moe_set_shared(self.h, l, b)
        self.router = torch.from_numpy(
            np.stack([synth.router_weights(cfg, l) for l in range(cfg.L)])).to(self.device)
        self.xdt = torch.bfloat16 if cfg.x_dtype == "bf16" else torch.float32
        if max_tokens:
            ft_moe_reserve(self.h, max_tokens)

    # host pool, read in place (the same bytes the GPU copies into its slots)
    def pool_blob(self, layer, expert):
        addr = self.pool_base + (layer * self.cfg.E + expert) * self.blob
        return np.ctypeslib.as_array((ctypes.c_uint8 * self.blob).from_address(addr))

    def tokens(self, batch):
        vals, bits = synth.tokens(self.cfg, batch)
        return vals, _to_device_tokens(self.cfg, vals, bits, self.device)

    def forward(self, layer, x, out, stream=None):
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        ft_moe_forward(self.h, layer, x, x.shape[0], self.router[layer], out, s)

    def step(self, x, outs, stream=None):
        """x: [B, H] on device; outs: [L, B, H] on device."""
        for l in range(self.cfg.L):
            self.forward(l, x, outs[l], stream)

    def last_routing(self, T):
        ids = np.zeros((T, self.cfg.k), dtype=np.int32)
        g = np.zeros((T, self.cfg.k), dtype=np.float32)
        ft_moe_last_routing(self.h, ids, g)
        return ids, g

    def resize(self, slots):
        ft_cache_resize(self.h, slots)
        self.C = slots

    def stats(self):
        return ft_cache_stats(self.h)

    def reset_stats(self):
        ft_cache_reset_stats(self.h)

    def trace(self):
        return ft_cache_trace(self.h)

    def close(self):
        if self.h:
            torch.cuda.synchronize(self.device)
            ft_moe_destroy(self.h)
            self.h = None

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()
