"""Moves seeded host workloads to a device (copies only)."""

import torch


def to_device(obj, device="cuda"):
    """Recursively copies tensors in dicts/lists to ``device``."""
    if isinstance(obj, torch.Tensor):
        return obj.to(device, non_blocking=False).contiguous()
    if isinstance(obj, dict):
        return {k: to_device(v, device) for k, v in obj.items()}
    if isinstance(obj, (list, tuple)):
        return type(obj)(to_device(v, device) for v in obj)
    return obj
