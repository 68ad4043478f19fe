"""Multi-Router Latent MoE layer for B200 (sm_100a): forward, balancing-bias
update and backward.

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
                      mrlmoe_get_device_detail, mrlmoe_workspace_size, status_string, HOLD, CHECK_BITS,
                      Grads, GRAD_FIELDS, make_grads, mrlmoe_train_workspace_size, mrlmoe_forward_train,
                      mrlmoe_backward, mrlmoe_backward_timed)

__all__ = ["MRLMoELayer", "Config", "Weights", "Routing", "MrlmoeError", "make_config",
           "make_weights", "make_routing", "mrlmoe_route", "mrlmoe_forward", "mrlmoe_forward_timed",
           "mrlmoe_bias_update", "mrlmoe_linear", "mrlmoe_workspace_size",
           "mrlmoe_get_device_status", "mrlmoe_route_scores_static", "mrlmoe_quantize_e4m3",
           "mrlmoe_check_routing", "mrlmoe_get_device_detail", "status_string", "MRLMOE_BF16",
           "MRLMOE_FP8_E4M3_BLOCK128", "MRLMOE_FP4_E2M1_BLOCK128", "HOLD", "CHECK_BITS",
           "Grads", "GRAD_FIELDS", "make_grads", "mrlmoe_train_workspace_size", "mrlmoe_forward_train",
           "mrlmoe_backward", "mrlmoe_backward_timed", "grad_buffers"]


def grad_buffers(cfg: Config, device="cuda"):
    """Device buffers for mrlmoe_backward's outputs: dx bf16, the rest fp32."""
    import torch
    T, D, L, E, F, R = cfg.T, cfg.d_model, cfg.d_lat, cfg.n_experts, cfg.d_ff, cfg.n_routers
    f32 = dict(dtype=torch.float32, device=device)
    return {"dx": torch.empty(T, D, dtype=torch.bfloat16, device=device),
            "d_w_down": torch.empty(L, D, **f32), "d_w_router": torch.empty(R, E, L, **f32),
            "d_w_gate": torch.empty(E, F, L, **f32), "d_w_up_e": torch.empty(E, F, L, **f32),
            "d_w_down_e": torch.empty(E, L, F, **f32), "d_w_sh_gate": torch.empty(F, L, **f32),
            "d_w_sh_up": torch.empty(F, L, **f32), "d_w_sh_down": torch.empty(L, F, **f32),
            "d_rms_gain": torch.empty(L, **f32), "d_w_up": torch.empty(D, L, **f32),
            "d_expert_scale": torch.empty(E, **f32)}


class MRLMoELayer:
    """A layer bound to device weights and a workspace sized for T tokens
    (``train=True``: sized for forward_train + backward as well)."""

    def __init__(self, shape, weights: Dict[str, object], T: Optional[int] = None,
                 device="cuda", checks: Optional[bool] = None, train: bool = False):
        import torch
        self.checks = os.environ.get("MRLMOE_CHECKS", "0") == "1" if checks is None else bool(checks)
        self.shape = shape
        self.cfg = make_config(shape, T=T)
        self.w = weights
        self.cw = make_weights(weights)
        self.train = bool(train)
        self.ws_bytes = (mrlmoe_train_workspace_size if train else mrlmoe_workspace_size)(self.cfg)
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

    def forward_train(self, x, bias, y=None, routing: Optional[Dict[str, object]] = None, stream=None):
        """The forward, keeping in the workspace what backward() reads."""
        import torch
        if not self.train:
            raise MrlmoeError(3, "forward_train needs a layer built with train=True")
        if y is None:
            y = torch.empty(self.cfg.T, self.cfg.d_model, dtype=torch.bfloat16, device=x.device)
        mrlmoe_forward_train(self.cfg, self.cw, bias, x, y, make_routing(routing), self.workspace, self.ws_bytes,
                             stream)
        return y

    def backward(self, x, dy, grads: Optional[Dict[str, object]] = None, accumulate: bool = False, stream=None):
        """Gradients for the last forward_train(x, ...) of this layer; with
        ``accumulate`` the weight gradients are added to ``grads``."""
        grads = grads if grads is not None else grad_buffers(self.cfg, self.workspace.device)
        mrlmoe_backward(self.cfg, self.cw, x, dy, make_grads(grads, accumulate), self.workspace, self.ws_bytes,
                        stream)
        return grads

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
