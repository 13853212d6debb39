"""Helpers shared by the GPU tests (device buffers through torch)."""
import numpy as np


def torch():
    import torch as t
    return t


def dev_bf16(a):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(t.bfloat16)


def dev_f32(a):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda")


def host(x):
    return x.float().cpu().numpy().astype(np.float64)


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)
