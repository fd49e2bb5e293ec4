"""Seeded synthetic workloads (shapes and laws of the pages' settings).

Holds no arithmetic of the method: only random inputs.  Both the CUDA path
and the oracle receive the tensors made here.  Generation runs on the given
device with a torch.Generator seeded per call, so a workload is reproducible
on that device; the oracle is handed a host copy of the very same values.

Workloads (head_dim 128 unless stated):
  vectors(n, d)            i.i.d. N(0,1) fp32 rows
  unit_vectors(n, d)       normalised Gaussian rows: uniform on the sphere
  llama8b_kv               B=1, 8 KV heads, N tokens; K, V = N(0,1) * s[h,c],
                           s ~ LogNormal(0, 0.5) drawn once per (head, channel),
                           separately for K and V; bf16
  outlier_kv               B, 8 KV heads, N; N(0,1) with 3 seeded channels per
                           KV head (the same for K and V) scaled x8; bf16
  student_kv               B=1, 8 KV heads, N; 0.5 * StudentT(3) * s[h,c],
                           s ~ LogNormal(0, 1); bf16
  queries(B, Hq, d)        N(0,1) bf16, one decode query per head
The K/V tensors are returned as [B, Hkv, N, d] views of a [B, N, Hkv, d]
buffer, the layout a fused QKV projection writes.
"""

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def vectors(n: int, d: int, seed: int = 0, device="cpu") -> torch.Tensor:
    return torch.randn((n, d), generator=_gen(seed, device), device=device, dtype=torch.float32)


def unit_vectors(n: int, d: int, seed: int = 0, device="cpu") -> torch.Tensor:
    x = torch.randn((n, d), generator=_gen(seed, device), device=device, dtype=torch.float64)
    return (x / x.norm(dim=1, keepdim=True)).to(torch.float32)


def queries(B: int, Hq: int, d: int = 128, seed: int = 1, device="cpu") -> torch.Tensor:
    return torch.randn((B, Hq, d), generator=_gen(seed, device), device=device).to(torch.bfloat16)


def _bnhd(B, N, H, d, device):
    return torch.empty((B, N, H, d), dtype=torch.bfloat16, device=device)


def llama8b_kv(N: int = 32768, seed: int = 2, B: int = 1, H: int = 8, d: int = 128, device="cpu"):
    g = _gen(seed, device)
    out = []
    for _ in range(2):  # K then V
        s = torch.exp(0.5 * torch.randn((H, d), generator=g, device=device))
        buf = _bnhd(B, N, H, d, device)
        for b in range(B):
            for h in range(H):
                buf[b, :, h] = (torch.randn((N, d), generator=g, device=device) * s[h]).to(torch.bfloat16)
        out.append(buf.permute(0, 2, 1, 3))
    return out[0], out[1]


def outlier_kv(N: int = 131072, B: int = 16, seed: int = 3, H: int = 8, d: int = 128, device="cpu",
               frac: float = 0.02, factor: float = 8.0):
    g = _gen(seed, device)
    n_out = int(round(frac * d))
    scale = torch.ones((H, d), device=device)
    for h in range(H):
        ch = torch.randperm(d, generator=g, device=device)[:n_out]
        scale[h, ch] = factor
    out = []
    for _ in range(2):
        buf = _bnhd(B, N, H, d, device)
        for b in range(B):
            for h in range(H):
                buf[b, :, h] = (torch.randn((N, d), generator=g, device=device) * scale[h]).to(torch.bfloat16)
        out.append(buf.permute(0, 2, 1, 3))
    return out[0], out[1]


def _student_t3(shape, g, device):
    # t_3 = Z / sqrt(chi2_3 / 3), chi2_3 the sum of three squared normals
    z = torch.randn(shape, generator=g, device=device)
    c = torch.randn((3,) + tuple(shape), generator=g, device=device).pow(2).sum(0)
    return z / torch.sqrt(c / 3.0)


def student_kv(N: int = 1 << 20, seed: int = 5, B: int = 1, H: int = 8, d: int = 128, device="cpu"):
    g = _gen(seed, device)
    out = []
    for _ in range(2):
        s = torch.exp(torch.randn((H, d), generator=g, device=device))
        buf = _bnhd(B, N, H, d, device)
        for b in range(B):
            for h in range(H):
                for n0 in range(0, N, 1 << 18):
                    n1 = min(N, n0 + (1 << 18))
                    buf[b, n0:n1, h] = (0.5 * _student_t3((n1 - n0, d), g, device) * s[h]).to(torch.bfloat16)
        out.append(buf.permute(0, 2, 1, 3))
    return out[0], out[1]


def outlier_channels(seed: int = 3, H: int = 8, d: int = 128, frac: float = 0.02):
    """The channel sets outlier_kv scales (regenerated on the CPU)."""
    g = _gen(seed, "cpu")
    n_out = int(round(frac * d))
    return [torch.randperm(d, generator=g)[:n_out].tolist() for _ in range(H)]
