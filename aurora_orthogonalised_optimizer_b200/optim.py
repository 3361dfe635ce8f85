"""torch.optim front-ends of the library (argument marshalling only).

The Track 3 Aurora write-up steps every 2-D block matrix with
``Muon(lr=0.0375, weight_decay=0, pp_iterations=2, pp_beta=0.5)`` (Aurora +
Contra-Muon + u/w-floor) and everything else with an auxiliary fused AdamW
(betas (0.8, 0.95), eps 1e-10, weight_decay 0; embeddings lr 0.3, output
projection lr 1/320, 1-D parameters lr 0.01).  ``MuonAurora`` and
``FusedAdamW`` are those two optimizers; each ``step()`` is one call per
parameter group into libaurora_muon.so (``muon_step`` / ``adamw_step``) on
the current CUDA stream.  Optimizer state is the fp32 momentum (Muon) or the
two fp32 moments (AdamW) plus a per-group step counter, all saved by
``state_dict()``.
"""
from __future__ import annotations

from typing import Callable, Iterable, Optional, Sequence, Tuple

import torch

from . import _abi as A
from .schedules import momentum_warmup as _momentum_warmup

_GEMM = {"bf16": A.MUON_GEMM_BF16, "fp32": A.MUON_GEMM_FP32, "bf16simt": A.MUON_GEMM_BF16_SIMT}


class _Fp32State:
    """torch.optim.Optimizer.load_state_dict casts floating-point state to each
    parameter's dtype; the library's states are fp32 whatever the parameter
    dtype, so the saved fp32 tensors are put back after the base load."""

    def load_state_dict(self, state_dict):
        keep = {}
        for idx, st in state_dict["state"].items():
            keep[idx] = {k: v for k, v in st.items() if torch.is_tensor(v) and v.dtype == torch.float32}
        super().load_state_dict(state_dict)
        params = [p for g in self.param_groups for p in g["params"]]
        for idx, kv in keep.items():
            p = params[int(idx)]
            for k, v in kv.items():
                self.state[p][k] = v.to(device=p.device, dtype=torch.float32, copy=True)


class MuonAurora(_Fp32State, torch.optim.Optimizer):
    """Muon with Aurora equilibration, Contra-Muon and the u/w floor, for 2-D parameters.

    momentum_warmup: None, or (steps, start, end): mu follows a linear warm-up
      from `start` to `end` over `steps` steps (the 2024-11-10 record: 500,
      0.85, 0.95) instead of the fixed `mu`.
    lr_schedule: None, or a function of the 0-based step returning the lr
      multiplier (see schedules.wsd_multiplier).
    gemm_mode: "bf16" (tensor cores), "fp32" (fp32 FMA) or "bf16simt".
    """

    def __init__(self, params: Iterable, lr: float = 0.0375, mu: float = 0.95, nesterov: bool = True,
                 ns_steps: int = 12, ns_coefficients: Tuple[float, float, float] = (2.0, -1.5, 0.5),
                 ns_eps: float = 1e-7, aurora: bool = True, pp_iterations: int = 2, pp_beta: float = 0.5,
                 pp_eps: float = 1e-7, contra: float = 0.4, power_iters: int = 5, target_uw: float = 0.35,
                 weight_decay: float = 0.0, gemm_mode: str = "bf16",
                 momentum_warmup: Optional[Tuple[int, float, float]] = None,
                 lr_schedule: Optional[Callable[[int], float]] = None):
        if weight_decay != 0.0:
            raise ValueError("weight_decay must be 0: the u/w floor replaces it")
        defaults = dict(lr=lr, mu=mu, nesterov=nesterov, ns_steps=ns_steps, ns_coefficients=tuple(ns_coefficients),
                        ns_eps=ns_eps, aurora=aurora, pp_iterations=pp_iterations, pp_beta=pp_beta, pp_eps=pp_eps,
                        contra=contra, power_iters=power_iters, target_uw=target_uw, weight_decay=weight_decay,
                        gemm_mode=gemm_mode, momentum_warmup=momentum_warmup, step=0)
        super().__init__(params, defaults)
        for g in self.param_groups:
            for p in g["params"]:
                if p.dim() != 2:
                    raise ValueError(f"MuonAurora steps 2-D matrices only, got shape {tuple(p.shape)}")
        self.lr_schedule = lr_schedule
        self._ws = {}

    def _workspace(self, cfg: A.Config, shapes, device):
        need = A.workspace_size(cfg, shapes)
        ws = self._ws.get(device)
        if ws is None or ws.numel() < need:
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
            self._ws[device] = ws
        return ws

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for group in self.param_groups:
            k = group["step"]
            mu = group["mu"]
            if group["momentum_warmup"] is not None:
                steps, start, end = group["momentum_warmup"]
                mu = _momentum_warmup(k, steps, start, end)
            lr = group["lr"] * (self.lr_schedule(k) if self.lr_schedule is not None else 1.0)
            a, b, c = group["ns_coefficients"]
            batches = {}
            for p in group["params"]:
                if p.grad is None:
                    continue
                if not (p.is_cuda and p.is_contiguous() and p.grad.is_contiguous()):
                    raise ValueError("parameters and gradients must be contiguous CUDA tensors")
                st = self.state[p]
                if "momentum_buffer" not in st:
                    st["momentum_buffer"] = torch.zeros_like(p, dtype=torch.float32)
                key = (p.device, p.dtype, p.grad.dtype)
                batches.setdefault(key, []).append(p)
            for (device, pdt, gdt), ps in batches.items():
                cfg = A.Config(lr=lr, mu=mu, nesterov=group["nesterov"], ns_steps=group["ns_steps"], ns_a=a, ns_b=b,
                               ns_c=c, ns_eps=group["ns_eps"], aurora=group["aurora"],
                               pp_iterations=group["pp_iterations"], pp_beta=group["pp_beta"],
                               pp_eps=group["pp_eps"], contra=group["contra"], power_iters=group["power_iters"],
                               target_uw=group["target_uw"], weight_decay=0.0, gemm_mode=_GEMM[group["gemm_mode"]],
                               param_dtype=A.dtype_code(ps[0]), grad_dtype=A.dtype_code(ps[0].grad))
                ws = self._workspace(cfg, [tuple(p.shape) for p in ps], device)
                A.muon_step(cfg, ps, [p.grad for p in ps], [self.state[p]["momentum_buffer"] for p in ps],
                            None, ws)
            group["step"] = k + 1
        return loss


class FusedAdamW(_Fp32State, torch.optim.Optimizer):
    """Fused multi-tensor AdamW (torch.optim.AdamW semantics) for the auxiliary parameters.

    Defaults are the Track 3 auxiliary values: betas (0.8, 0.95), eps 1e-10,
    weight_decay 0.  Per-group lr as in the pages (embeddings 0.3, output
    projection 1/320, 1-D parameters 0.01)."""

    def __init__(self, params: Iterable, lr: float = 0.01, betas: Sequence[float] = (0.8, 0.95),
                 eps: float = 1e-10, weight_decay: float = 0.0,
                 lr_schedule: Optional[Callable[[int], float]] = None):
        defaults = dict(lr=lr, betas=tuple(betas), eps=eps, weight_decay=weight_decay, step=0)
        super().__init__(params, defaults)
        self.lr_schedule = lr_schedule

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for group in self.param_groups:
            k = group["step"]
            lr = group["lr"] * (self.lr_schedule(k) if self.lr_schedule is not None else 1.0)
            batches = {}
            for p in group["params"]:
                if p.grad is None:
                    continue
                if not (p.is_cuda and p.is_contiguous() and p.grad.is_contiguous()):
                    raise ValueError("parameters and gradients must be contiguous CUDA tensors")
                st = self.state[p]
                if "exp_avg" not in st:
                    st["exp_avg"] = torch.zeros_like(p, dtype=torch.float32)
                    st["exp_avg_sq"] = torch.zeros_like(p, dtype=torch.float32)
                batches.setdefault((p.dtype, p.grad.dtype), []).append(p)
            b1, b2 = group["betas"]
            for ps in batches.values():
                A.adamw_step(ps, [p.grad for p in ps], [self.state[p]["exp_avg"] for p in ps],
                             [self.state[p]["exp_avg_sq"] for p in ps], k + 1, lr, b1, b2, group["eps"],
                             group["weight_decay"])
            group["step"] = k + 1
        return loss
