"""Copy a generated problem's arrays into torch tensors on a device (raw bits
reinterpreted as the storage dtypes; no conversion of values)."""

from __future__ import annotations

import numpy as np
import torch

from .gen import DT_BF16, DT_F32


def x_tensor(P, device="cuda"):
    if P.x_dtype == DT_F32:
        return torch.from_numpy(np.ascontiguousarray(P.x)).to(device)
    t = torch.from_numpy(np.ascontiguousarray(P.x).view(np.int16))
    return t.view(torch.bfloat16 if P.x_dtype == DT_BF16 else torch.float16).to(device)


def to_device(P, device="cuda"):
    def raw(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        elif a.dtype == np.uint32:
            a = a.view(np.int32)
        return torch.from_numpy(a).to(device)

    return dict(x=x_tensor(P, device), ids=raw(P.ids), packed=raw(P.packed), scales=raw(P.scales),
                aux=raw(P.aux))
