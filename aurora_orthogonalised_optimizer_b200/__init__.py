"""Muon / Aurora optimizer step on B200 (sm_100a): C-ABI library + thin binding.

The step (momentum + Nesterov, Newton-Schulz polar, Aurora row
equilibration, Contra-Muon operator-norm subtraction with Frobenius restore,
aspect scale, u/w floor, parameter add) runs entirely in libaurora_muon.so.
"""
from . import _abi  # noqa: F401
from ._abi import (Config, MuonError, adamw_step, aurora_polar, load, make_workspace, muon_step,  # noqa: F401
                   ns_polar, opnorm_normalize, opnorm_normalize_noalloc, uw_floor_apply, workspace_size)
from . import schedules  # noqa: F401


def __getattr__(name):
    # the torch.optim front-ends import torch lazily
    if name in ("MuonAurora", "FusedAdamW"):
        from . import optim
        return getattr(optim, name)
    raise AttributeError(name)


__all__ = ["Config", "MuonError", "adamw_step", "aurora_polar", "load", "make_workspace", "muon_step", "ns_polar",
           "opnorm_normalize", "opnorm_normalize_noalloc", "uw_floor_apply", "workspace_size", "schedules",
           "MuonAurora", "FusedAdamW"]
