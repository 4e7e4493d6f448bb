"""Seeded synthetic inputs for low-rank compressed-KV decode attention.

This module only draws inputs: bases, keys, values, queries, lengths.  It
holds none of the method's arithmetic (no projection, no error, no
routing, no attention) and is the one module both the CUDA-path tests and
the CPU oracle tests take their inputs from.

Recipe, per (layer, kv head, K or V) independently:
  * Q = the Q factor of a QR factorisation of a 128x128 N(0,1) matrix;
  * the signal basis is Q[:, :R_sig] and the compression basis handed to
    the library is U = bf16(Q[:, :r]);
  * X = Z Q[:, :R_sig]^T + sigma N(0,1), Z[t, i] ~ N(0, i^-alpha), i = 1..R_sig;
  * exactly round(f T) seeded positions per (batch row, layer, kv head)
    become full-rank outliers: both their K and V rows are replaced by
    N(0,1) rows;
  * everything is cast to bfloat16 (round-to-nearest-even); q ~ N(0,1).
Keys carry no positional rotation.  The workloads (sizes, ranks, tau) are
the attention geometries of Llama-3.1-8B (32 q heads, 8 kv heads) and
LLaMA-7B (32 heads, MHA), head dim 128.

Random numbers come from torch generators seeded per (seed, layer, stream),
so one layer can be rebuilt without the others.  CUDA generation (Philox)
and CPU generation (Mersenne Twister) give different numbers for the same
seed; a test always feeds both sides from one draw.
"""
from dataclasses import dataclass, replace
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    layers: int
    Hq: int
    Hkv: int
    d: int
    r_k: int
    r_v: int
    T: int                 # prefill tokens per sequence (the maximum when ragged)
    R_sig: int
    alpha: float
    sigma: float
    f_out: float
    tau: float
    ragged_min: int = 0    # > 0: lengths uniform in [ragged_min, T]
    t_append: int = 0      # decode steps that each append one token

    @property
    def g(self):
        return self.Hq // self.Hkv


WORKLOADS = {
    0: Workload("tiny_gqa4_T512", B=1, layers=1, Hq=4, Hkv=1, d=128, r_k=32, r_v=32,
                T=512, R_sig=32, alpha=1.0, sigma=0.02, f_out=0.02, tau=0.3),
    1: Workload("llama31_8b_ctx8192", B=1, layers=32, Hq=32, Hkv=8, d=128, r_k=64, r_v=96,
                T=8192, R_sig=72, alpha=1.0, sigma=0.02, f_out=0.01, tau=0.25),
    2: Workload("llama31_8b_ctx32768_append64", B=1, layers=32, Hq=32, Hkv=8, d=128,
                r_k=48, r_v=80, T=32768, R_sig=72, alpha=1.0, sigma=0.02, f_out=0.01,
                tau=0.25, t_append=64),
    3: Workload("llama31_8b_b16_ragged8k_16k", B=16, layers=32, Hq=32, Hkv=8, d=128,
                r_k=64, r_v=96, T=16384, R_sig=72, alpha=1.0, sigma=0.02, f_out=0.01,
                tau=0.25, ragged_min=8192),
    4: Workload("llama7b_mha_ctx131072", B=1, layers=32, Hq=32, Hkv=32, d=128, r_k=48,
                r_v=64, T=131072, R_sig=72, alpha=1.5, sigma=0.01, f_out=0.01, tau=0.25),
}


def workload(i, **overrides):
    """Workload ``i`` with optional field overrides (smaller T, fewer layers, ...)."""
    return replace(WORKLOADS[i], **overrides)


def _gen(seed, layer, stream, device):
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(layer) * 7_919 + int(stream)) % (2 ** 63))
    return g


def seq_lengths(w, seed, device="cpu"):
    """Per-sequence prefill lengths [B] (int64): T, or uniform in [ragged_min, T]."""
    if w.ragged_min <= 0:
        return torch.full((w.B,), w.T, dtype=torch.int64)
    g = _gen(seed, 0, 99, "cpu")
    return torch.randint(w.ragged_min, w.T + 1, (w.B,), generator=g, dtype=torch.int64)


def orthonormal_bases(n, d, gen, device):
    """n independent d x d orthogonal matrices Q (float32): QR of N(0,1) draws."""
    a = torch.randn(n, d, d, generator=gen, device=device, dtype=torch.float32)
    q, _ = torch.linalg.qr(a.double())
    return q.float()


def _signal(gen, Qs, B, T, w, device):
    """[B, T, H, d] float32 rows Z Q_s^T + sigma N(0,1), column variance i^-alpha."""
    H = Qs.shape[0]
    col_sd = torch.arange(1, w.R_sig + 1, device=device, dtype=torch.float32).pow(-w.alpha / 2)
    Z = torch.randn(B, H, T, w.R_sig, generator=gen, device=device) * col_sd
    X = torch.matmul(Z, Qs[:, :, : w.R_sig].transpose(1, 2).unsqueeze(0))   # [B,H,T,d]
    X += w.sigma * torch.randn(B, H, T, w.d, generator=gen, device=device)
    return X.permute(0, 2, 1, 3)                                           # [B,T,H,d]


def make_layer(w, layer, seed, device="cpu", lengths=None):
    """Synthesise one layer: bases, prefill K/V, query, append tokens.

    Returns a dict of tensors on ``device``:
      U_k [Hkv,d,r_k] bf16, U_v [Hkv,d,r_v] bf16 (orthonormal columns, rounded),
      K, V [B,T,Hkv,d] bf16 (rows past a sequence's length are zero padding),
      lengths [B] int64, outlier_pos list of [B][Hkv] long tensors,
      q [B,Hq,d] bf16,
      K_app, V_app [B,t_append,Hkv,d] bf16 and q_app [t_append,B,Hq,d] bf16
      when the workload appends decode tokens.
    """
    device = torch.device(device)
    dev = device.type if device.type == "cpu" else device
    if lengths is None:
        lengths = seq_lengths(w, seed)
    gb = _gen(seed, layer, 1, dev)
    Qk = orthonormal_bases(w.Hkv, w.d, gb, dev)
    Qv = orthonormal_bases(w.Hkv, w.d, gb, dev)
    U_k = Qk[:, :, : w.r_k].to(torch.bfloat16).contiguous()
    U_v = Qv[:, :, : w.r_v].to(torch.bfloat16).contiguous()

    gx = _gen(seed, layer, 2, dev)
    K = _signal(gx, Qk, w.B, w.T, w, dev)
    V = _signal(gx, Qv, w.B, w.T, w, dev)
    go = _gen(seed, layer, 3, dev)
    outlier_pos = []
    for b in range(w.B):
        Tb = int(lengths[b])
        row = []
        for h in range(w.Hkv):
            n_out = int(round(w.f_out * Tb))
            pos = torch.randperm(Tb, generator=go, device=dev)[:n_out]
            pos, _ = torch.sort(pos)
            if n_out:
                K[b, pos, h] = torch.randn(n_out, w.d, generator=go, device=dev)
                V[b, pos, h] = torch.randn(n_out, w.d, generator=go, device=dev)
            row.append(pos.cpu())
        outlier_pos.append(row)
        if Tb < w.T:
            K[b, Tb:] = 0
            V[b, Tb:] = 0
    gq = _gen(seed, layer, 4, dev)
    out = dict(U_k=U_k, U_v=U_v, Qk=Qk, Qv=Qv,
               K=K.to(torch.bfloat16).contiguous(), V=V.to(torch.bfloat16).contiguous(),
               lengths=lengths.clone(), outlier_pos=outlier_pos,
               q=torch.randn(w.B, w.Hq, w.d, generator=gq, device=dev).to(torch.bfloat16))
    if w.t_append:
        Ka, Va = decode_tokens(w, Qk, Qv, w.t_append, seed, layer, device)
        out["K_app"], out["V_app"] = Ka, Va
        out["q_app"] = decode_queries(w, w.t_append, seed, layer, device)
    return out


def decode_tokens(w, Qk, Qv, n, seed, layer, device="cpu", stream=5):
    """n decode-time tokens per sequence, K and V [B,n,Hkv,d] bf16.

    Drawn like the prefill rows (same per-head signal bases Qk, Qv), with
    exactly round(f n) outlier positions per (batch row, kv head).
    """
    device = torch.device(device)
    dev = device.type if device.type == "cpu" else device
    ga = _gen(seed, layer, stream, dev)
    Ka = _signal(ga, Qk.to(dev), w.B, n, w, dev)
    Va = _signal(ga, Qv.to(dev), w.B, n, w, dev)
    n_out = int(round(w.f_out * n))
    for b in range(w.B):
        for h in range(w.Hkv):
            pos = torch.randperm(n, generator=ga, device=dev)[:n_out]
            if n_out:
                Ka[b, pos, h] = torch.randn(n_out, w.d, generator=ga, device=dev)
                Va[b, pos, h] = torch.randn(n_out, w.d, generator=ga, device=dev)
    return Ka.to(torch.bfloat16).contiguous(), Va.to(torch.bfloat16).contiguous()


def decode_queries(w, n, seed, layer, device="cpu", stream=6):
    """n decode-step queries [n,B,Hq,d] bf16, N(0,1)."""
    device = torch.device(device)
    dev = device.type if device.type == "cpu" else device
    g = _gen(seed, layer, stream, dev)
    return torch.randn(n, w.B, w.Hq, w.d, generator=g, device=dev).to(torch.bfloat16)


def pad_to(n, m):
    """n rounded up to a multiple of m."""
    return int(math.ceil(n / m) * m)
