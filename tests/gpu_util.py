"""Helpers shared by the GPU tests: numpy (storage-precision float32) <-> torch."""
import numpy as np


def dev_tensor(x, dtype="bf16"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda().contiguous()


def dev_ids(ids):
    import torch
    return torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).cuda()


def host(t):
    import torch
    return t.detach().float().cpu().numpy() if t.dtype in (torch.bfloat16, torch.float16) else t.detach().cpu().numpy()


def workspace(nbytes):
    import torch
    return torch.empty(max(int(nbytes), 256) + 256, dtype=torch.uint8, device="cuda")


def aligned_ptr(buf):
    p = buf.data_ptr()
    return (p + 255) & ~255
