"""Shared helpers of the GPU parity tests: move seeded numpy inputs to the
device and measure relative error. No arithmetic of the method lives here."""

import numpy as np


def dev(x, dtype=None):
    import torch
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint32:
        t = torch.from_numpy(x.view(np.int32))
    elif x.dtype == np.uint16:
        t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(x)
    return t.cuda()


def host(t):
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    return t.numpy()


def rel_err(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))
