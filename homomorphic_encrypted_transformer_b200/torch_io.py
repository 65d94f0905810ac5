"""Moving uint64 residue arrays between numpy (host) and torch device tensors.

torch has no general uint64 arithmetic, so device buffers are int64 tensors
holding the same 64-bit patterns; no arithmetic is done on them here.
"""
import numpy as np
import torch


def to_device(a, device="cuda"):
    a = np.ascontiguousarray(a, dtype=np.uint64)
    return torch.from_numpy(a.view(np.int64)).to(device)


def empty_device(shape, device="cuda"):
    return torch.empty(shape, dtype=torch.int64, device=device)


def to_host(t, shape=None):
    a = t.detach().cpu().numpy().view(np.uint64)
    return a.reshape(shape) if shape is not None else a
