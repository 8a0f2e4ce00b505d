"""Moves a seeded :class:`~grouped_nf4_expert_b200.inputs.Problem` to the GPU (plumbing only)."""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import e4b


@dataclass
class DeviceProblem:
    x: "torch.Tensor"            # bf16 [T, H]
    logits: "torch.Tensor"       # float32 [T, E]
    dY: "torch.Tensor"           # bf16 [T, H]
    gate_up_nf4: "torch.Tensor"
    gate_up_absmax: "torch.Tensor"
    down_nf4: "torch.Tensor"
    down_absmax: "torch.Tensor"
    A_gu: "torch.Tensor"
    B_gu: "torch.Tensor"
    A_d: "torch.Tensor"
    B_d: "torch.Tensor"

    def base(self) -> e4b.Nf4Experts:
        return e4b.nf4_experts(self.gate_up_nf4, self.gate_up_absmax, self.down_nf4, self.down_absmax)

    def lora(self) -> e4b.Lora:
        return e4b.lora_factors(self.A_gu, self.B_gu, self.A_d, self.B_d)


def bf16_tensor(bits: np.ndarray, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def upload(prob, device="cuda") -> DeviceProblem:
    import torch

    def t(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    return DeviceProblem(
        x=bf16_tensor(prob.x, device), logits=t(prob.logits), dY=bf16_tensor(prob.dY, device),
        gate_up_nf4=t(prob.gate_up_nf4), gate_up_absmax=t(prob.gate_up_absmax),
        down_nf4=t(prob.down_nf4), down_absmax=t(prob.down_absmax),
        A_gu=bf16_tensor(prob.A_gu, device), B_gu=bf16_tensor(prob.B_gu, device),
        A_d=bf16_tensor(prob.A_d, device), B_d=bf16_tensor(prob.B_d, device))


def dims_of(cfg) -> e4b.Dims:
    return e4b.Dims(E=cfg.E, H=cfg.H, I=cfg.I, top_k=cfg.top_k, r=cfg.r, alpha=cfg.alpha)
