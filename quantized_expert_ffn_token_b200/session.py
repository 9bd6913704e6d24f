"""Context ownership and synthetic-layer loading on top of the C ABI.

Marshalling only: weights come from the seeded generator (package ``synth``),
are generated directly on the device and handed to ``moe_load_layer``, which
repacks them in its own kernels.
"""
from __future__ import annotations

import torch

import synth
from . import capi


def config_struct(cfg: "synth.LayerConfig", max_tokens: int | None = None,
                  n_layers: int | None = None, mem_limit: int = 0, flags: int = 0) -> capi.moe_config:
    c = capi.moe_config()
    c.d_model, c.n_experts, c.d_ff, c.top_k = cfg.d, cfg.E, cfg.I, cfg.k
    c.n_shared, c.d_ff_shared = cfg.n_shared, cfg.I_s
    c.n_layers = cfg.L if n_layers is None else n_layers
    c.max_tokens = cfg.T if max_tokens is None else max_tokens
    c.fmt = capi.FORMATS[cfg.fmt]
    c.device_mem_limit = mem_limit
    c.flags = flags
    return c


def weights_struct(W: dict, keep: list) -> capi.moe_layer_weights:
    """moe_layer_weights over the tensors of ``synth.layer_weights`` (CUDA)."""
    dev = W["codes"][0].device
    rw = torch.as_tensor(W["router_w"]).to(dev).contiguous()
    rb = None if W.get("router_b") is None else torch.as_tensor(W["router_b"]).to(dev).contiguous()
    keep += [rw, rb]
    s = capi.moe_layer_weights()
    s.router_w = rw.data_ptr()
    s.router_bias = rb.data_ptr() if rb is not None else None
    for t in range(3):
        s.codes[t] = W["codes"][t].data_ptr()
        s.scales[t] = W["scales"][t].data_ptr()
        s.sh_codes[t] = W["sh_codes"][t].data_ptr() if W["sh_codes"][t].numel() else None
        s.sh_scales[t] = W["sh_scales"][t].data_ptr() if W["sh_scales"][t].numel() else None
    s.on_device = 1 if dev.type == "cuda" else 0
    return s


class Session:
    """One library context on one device."""

    def __init__(self, cfg: "synth.LayerConfig", device: int = 0, max_tokens: int | None = None,
                 n_layers: int | None = None, mem_limit: int = 0, flags: int = 0):
        self.cfg = cfg
        self.device = torch.device("cuda", device)
        self.n_layers = cfg.L if n_layers is None else n_layers
        self.ctx = capi.moe_create(config_struct(cfg, max_tokens, self.n_layers, mem_limit, flags), device)

    def load_synthetic(self, layers=None, stream=None) -> None:
        for l in (range(self.n_layers) if layers is None else layers):
            W = synth.layer_weights(self.cfg, l, device=self.device)
            keep: list = []
            capi.moe_load_layer(self.ctx, l, weights_struct(W, keep), stream)
            del W, keep

    def load(self, layer: int, W: dict, stream=None) -> None:
        keep: list = []
        capi.moe_load_layer(self.ctx, layer, weights_struct(W, keep), stream)

    def forward(self, layer: int, x: torch.Tensor, want_f32: bool = True, stream=None):
        """x: CUDA int16/bf16 [T, d].  Returns (y bf16 bits int16, y_f32, ids, w)."""
        T, d = x.shape
        dev = self.device
        y = torch.empty((T, d), dtype=torch.int16, device=dev)
        yf = torch.empty((T, d), dtype=torch.float32, device=dev) if want_f32 else None
        ids = torch.empty((T, self.cfg.k), dtype=torch.int32, device=dev)
        w = torch.empty((T, self.cfg.k), dtype=torch.float32, device=dev)
        capi.moe_forward(self.ctx, layer, x, T, y, yf, ids, w, stream)
        return y, yf, ids, w

    def close(self) -> None:
        if self.ctx is not None:
            capi.moe_destroy(self.ctx)
            self.ctx = None

    def __enter__(self) -> "Session":
        return self

    def __exit__(self, *exc) -> None:
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
