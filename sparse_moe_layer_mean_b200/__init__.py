"""Multi-Router Latent MoE layer forward for B200 (sm_100a).

The compute lives in libmrlmoe.so (CUDA, C ABI in include/mrlmoe.h); this
package is its binding.  ``MRLMoELayer`` bundles a config, device weights
and a workspace so a caller can run ``layer(x, bias)``.
"""
from __future__ import annotations

from typing import Dict, Optional

from . import _native
from ._native import (MRLMOE_BF16, MRLMOE_FP8_E4M3_BLOCK128, Config, MrlmoeError, Routing,
                      Weights, make_config, make_routing, make_weights, mrlmoe_bias_update,
                      mrlmoe_forward, mrlmoe_forward_timed, mrlmoe_get_device_status, mrlmoe_linear, mrlmoe_route,
                      mrlmoe_route_scores_static, mrlmoe_quantize_e4m3,
                      mrlmoe_workspace_size, status_string)

__all__ = ["MRLMoELayer", "Config", "Weights", "Routing", "MrlmoeError", "make_config",
           "make_weights", "make_routing", "mrlmoe_route", "mrlmoe_forward", "mrlmoe_forward_timed",
           "mrlmoe_bias_update", "mrlmoe_linear", "mrlmoe_workspace_size",
           "mrlmoe_get_device_status", "mrlmoe_route_scores_static", "mrlmoe_quantize_e4m3", "status_string", "MRLMOE_BF16",
           "MRLMOE_FP8_E4M3_BLOCK128"]


class MRLMoELayer:
    """A layer bound to device weights and a workspace sized for T tokens."""

    def __init__(self, shape, weights: Dict[str, object], T: Optional[int] = None,
                 device="cuda"):
        import torch
        self.shape = shape
        self.cfg = make_config(shape, T=T)
        self.w = weights
        self.cw = make_weights(weights)
        self.ws_bytes = mrlmoe_workspace_size(self.cfg)
        if self.ws_bytes == 0:
            raise MrlmoeError(1, "mrlmoe_workspace_size")
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)

    def routing_buffers(self, scores: bool = False):
        import torch
        c, dev = self.cfg, self.workspace.device
        Tk = c.T * c.top_k
        r = {"topk_idx": torch.empty(Tk, dtype=torch.int32, device=dev),
             "topk_w": torch.empty(Tk, dtype=torch.float32, device=dev),
             "counts": torch.empty(c.n_experts, dtype=torch.int32, device=dev),
             "offsets": torch.empty(c.n_experts + 1, dtype=torch.int32, device=dev),
             "perm": torch.empty(Tk, dtype=torch.int32, device=dev),
             "inv_perm": torch.empty(Tk, dtype=torch.int32, device=dev)}
        if scores:
            r["scores"] = torch.empty(c.T * c.n_experts, dtype=torch.float32, device=dev)
        return r

    def __call__(self, x, bias, y=None, routing: Optional[Dict[str, object]] = None, stream=None):
        import torch
        if y is None:
            y = torch.empty(self.cfg.T, self.cfg.d_model, dtype=torch.bfloat16, device=x.device)
        mrlmoe_forward(self.cfg, self.cw, bias, x, y, make_routing(routing), self.workspace,
                       self.ws_bytes, stream)
        return y

    def route(self, bias, x=None, routing: Optional[Dict[str, object]] = None,
              scores_in: bool = False, stream=None):
        routing = routing if routing is not None else self.routing_buffers()
        mrlmoe_route(self.cfg, self.cw, bias, x, scores_in, make_routing(routing), self.workspace,
                     self.ws_bytes, stream)
        return routing

    def device_status(self, stream=None) -> int:
        return mrlmoe_get_device_status(self.workspace, stream)
