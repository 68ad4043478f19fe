"""Multi-Router Latent MoE layer forward for B200 (sm_100a).

The compute lives in libmrlmoe.so (CUDA, C ABI in include/mrlmoe.h); this
package is its binding.  ``MRLMoELayer`` bundles a config, device weights
and a workspace so a caller can run ``layer(x, bias)``.

Setting the environment variable MRLMOE_CHECKS=1 (or ``checks=True``) makes
every route/forward of a layer enqueue the device check of its routing record
(mrlmoe_check_routing); a violated invariant then shows as MRLMOE_ERR_CHECK in
``device_status()`` and its bits in ``device_detail()``.
"""
from __future__ import annotations

import os
from typing import Dict, Optional

from . import _native
from ._native import (MRLMOE_BF16, MRLMOE_FP8_E4M3_BLOCK128, MRLMOE_FP4_E2M1_BLOCK128, Config, MrlmoeError, Routing,
                      Weights, make_config, make_routing, make_weights, mrlmoe_bias_update,
                      mrlmoe_forward, mrlmoe_forward_timed, mrlmoe_get_device_status, mrlmoe_linear, mrlmoe_route,
                      mrlmoe_route_scores_static, mrlmoe_quantize_e4m3, mrlmoe_check_routing,
                      mrlmoe_get_device_detail, mrlmoe_workspace_size, status_string, HOLD, CHECK_BITS)

__all__ = ["MRLMoELayer", "Config", "Weights", "Routing", "MrlmoeError", "make_config",
           "make_weights", "make_routing", "mrlmoe_route", "mrlmoe_forward", "mrlmoe_forward_timed",
           "mrlmoe_bias_update", "mrlmoe_linear", "mrlmoe_workspace_size",
           "mrlmoe_get_device_status", "mrlmoe_route_scores_static", "mrlmoe_quantize_e4m3",
           "mrlmoe_check_routing", "mrlmoe_get_device_detail", "status_string", "MRLMOE_BF16",
           "MRLMOE_FP8_E4M3_BLOCK128", "MRLMOE_FP4_E2M1_BLOCK128", "HOLD", "CHECK_BITS"]


class MRLMoELayer:
    """A layer bound to device weights and a workspace sized for T tokens."""

    def __init__(self, shape, weights: Dict[str, object], T: Optional[int] = None,
                 device="cuda", checks: Optional[bool] = None):
        import torch
        self.checks = os.environ.get("MRLMOE_CHECKS", "0") == "1" if checks is None else bool(checks)
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
        r = make_routing(routing)
        mrlmoe_forward(self.cfg, self.cw, bias, x, y, r, self.workspace, self.ws_bytes, stream)
        if self.checks:
            mrlmoe_check_routing(self.cfg, r, self.workspace, self.ws_bytes, False, stream)
        return y

    def route(self, bias, x=None, routing: Optional[Dict[str, object]] = None,
              scores_in: bool = False, stream=None):
        routing = routing if routing is not None else self.routing_buffers()
        r = make_routing(routing)
        mrlmoe_route(self.cfg, self.cw, bias, x, scores_in, r, self.workspace, self.ws_bytes, stream)
        if self.checks:
            mrlmoe_check_routing(self.cfg, r, self.workspace, self.ws_bytes, False, stream)
        return routing

    def check_routing(self, routing: Optional[Dict[str, object]] = None, clear: bool = False, stream=None):
        """Enqueue the device check of the routing record (``routing``'s
        buffers, else the workspace copy of the last route/forward)."""
        mrlmoe_check_routing(self.cfg, make_routing(routing), self.workspace, self.ws_bytes, clear, stream)

    def device_status(self, stream=None) -> int:
        return mrlmoe_get_device_status(self.workspace, stream)

    def device_detail(self, stream=None):
        """(status, check_bits) of the workspace header."""
        return mrlmoe_get_device_detail(self.workspace, stream)
