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


def import_oracle_banks(bank, banks, params, w, layer=0):
    """Load oracle HeadBanks (with from-scratch densities) into a GPU bank."""
    import torch
    from oracle import densitykv as dkv
    for hh, b in enumerate(banks):
        if b.size == 0:
            bank.import_(layer, hh, torch.zeros(0, dtype=torch.int32, device="cuda"), None, None, None, None)
            continue
        rho = dkv.densities_from_scratch(b, params)
        bank.import_(layer, hh, dev_ids(b.ids), dev_tensor(rho, "f32"), dev_tensor(b.rho0, "f32"),
                     dev_tensor(b.K, w.dtype), dev_tensor(b.V, w.dtype))
