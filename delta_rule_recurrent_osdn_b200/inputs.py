"""Seeded synthetic inputs for the OSDN forward pass.

This module is shared by the CUDA path's tests and benchmark and by the oracle side of the
tests.  It holds none of the method's arithmetic: it only draws random numbers, L2-normalises
q and k (the workloads use unit-norm queries and keys), and rounds values to the I/O dtype.

Recipe (every workload):
  * ``rng = numpy.random.default_rng(seed)`` (PCG64); draws happen in this order:
    varlen lengths (packed workloads only), q, k, v, beta logits, r logits (APF only),
    S_0 (when given), d_0 (when given);
  * q, k ~ N(0, 1) drawn in float32, L2-normalised over the key dimension per (token, head)
    in float64, cast to float32;
  * v ~ N(0, 1) in float32;
  * beta = sigmoid(N(0, 1)), r = sigmoid(N(3, 1)) per (token, head), float32 (the gates stay
    float32 in every I/O mode);
  * S_0 ~ N(0, 0.1^2) (variance 0.01) and d_0 ~ U(0.5, 1.5) where a workload passes them in;
  * bf16 workloads round q, k, v to bfloat16 (round-to-nearest-even) and keep the rounded
    values; the GPU and the oracle consume the same rounded numbers.

The workloads are shaped like the token-mixer layers of the 340M and 1.3B models in the
experiments section of the OSDN summary pages; no dataset is involved.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# name -> shape/dtype/gating of each workload (sizes as the experiments describe them)
CONFIGS = {
    "tiny_fp32": dict(B=1, T=256, H=2, Dk=64, Dv=64, chunk=64, io="f32", apf=True, eta=0.1,
                      seed=0),
    "340m": dict(B=8, T=2048, H=8, Dk=128, Dv=128, chunk=64, io="bf16", apf=False, eta=0.05,
                 seed=1),
    "1p3b_apf": dict(B=4, T=4096, H=16, Dk=128, Dv=128, chunk=64, io="bf16", apf=True, eta=0.05,
                     seed=2),
    "long_ctx": dict(B=1, T=65536, H=16, Dk=128, Dv=128, chunk=64, io="bf16", apf=True,
                     eta=0.05, seed=3, init_state=True),
    "varlen": dict(num_seqs=32, min_len=128, max_len=8192, H=16, Dk=128, Dv=128, chunk=64,
                   io="bf16", apf=True, eta=0.05, seed=4),
}


@dataclasses.dataclass
class OsdnInputs:
    """One synthetic batch.  Arrays are float32 holding values exact in the I/O dtype."""
    q: np.ndarray            # [B, T, H, Dk]
    k: np.ndarray            # [B, T, H, Dk]
    v: np.ndarray            # [B, T, H, Dv]
    beta: np.ndarray         # [B, T, H]
    r: Optional[np.ndarray]  # [B, T, H] or None (no APF: r == 1)
    eta: float
    d0: Optional[np.ndarray]  # [N, H, Dk] or None (ones)
    S0: Optional[np.ndarray]  # [N, H, Dv, Dk] or None (zeros)
    cu_seqlens: Optional[np.ndarray]  # int32 [N+1] or None (fixed length)
    io: str                  # "bf16" or "f32"
    chunk: int
    scale: float = 1.0

    @property
    def B(self):
        return self.q.shape[0]

    @property
    def T(self):
        return self.q.shape[1]

    @property
    def H(self):
        return self.q.shape[2]

    @property
    def Dk(self):
        return self.q.shape[3]

    @property
    def Dv(self):
        return self.v.shape[3]

    @property
    def N(self):
        return len(self.cu_seqlens) - 1 if self.cu_seqlens is not None else self.B

    @property
    def tokens(self):
        return self.B * self.T


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    # finite values cannot overflow uint32 here (largest is 0xFF7FFFFF + 0x8000)
    out = bits + np.uint32(0x7FFF)
    out += (bits >> np.uint32(16)) & np.uint32(1)
    out &= np.uint32(0xFFFF0000)
    out = out.view(np.float32)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.nan
    return out.reshape(x.shape)


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-z.astype(np.float64)))).astype(np.float32)


def _unit_rows(rng, shape, block=65536) -> np.ndarray:
    """N(0,1) float32 draws, L2-normalised over the last axis (norm and division in float64)."""
    x = rng.standard_normal(shape, dtype=np.float32)
    flat = x.reshape(-1, shape[-1])
    for s in range(0, flat.shape[0], block):
        blk = flat[s:s + block]
        nrm = np.sqrt(np.einsum("ij,ij->i", blk, blk, dtype=np.float64))
        nrm[nrm == 0] = 1.0
        flat[s:s + block] = (blk / nrm[:, None]).astype(np.float32)
    return x


def make_inputs(config, seed: Optional[int] = None) -> OsdnInputs:
    """Build a seeded batch from a workload name in CONFIGS or a dict of the same keys.

    Dict keys: B, T, H, Dk, Dv (or num_seqs/min_len/max_len or lengths for packed input),
    io ("bf16"|"f32"), apf (bool), eta, chunk, init_state (bool), seed.
    """
    cfg = dict(CONFIGS[config]) if isinstance(config, str) else dict(config)
    if seed is not None:
        cfg["seed"] = seed
    rng = np.random.default_rng(cfg.get("seed", 0))
    H, Dk, Dv = cfg["H"], cfg["Dk"], cfg.get("Dv", cfg["Dk"])
    cu = None
    if "lengths" in cfg or "num_seqs" in cfg:
        if "lengths" in cfg:
            lengths = np.asarray(cfg["lengths"], dtype=np.int64)
        else:
            lengths = rng.integers(cfg["min_len"], cfg["max_len"], size=cfg["num_seqs"],
                                   endpoint=True)
        cu = np.zeros(len(lengths) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(lengths)
        B, T = 1, int(cu[-1])
        N = len(lengths)
    else:
        B, T = cfg["B"], cfg["T"]
        N = B
    q = _unit_rows(rng, (B, T, H, Dk))
    k = _unit_rows(rng, (B, T, H, Dk))
    v = rng.standard_normal((B, T, H, Dv), dtype=np.float32)
    beta = _sigmoid(rng.standard_normal((B, T, H)))
    r = _sigmoid(3.0 + rng.standard_normal((B, T, H))) if cfg.get("apf", True) else None
    S0 = d0 = None
    if cfg.get("init_state", False):
        S0 = (0.1 * rng.standard_normal((N, H, Dv, Dk))).astype(np.float32)
        d0 = rng.uniform(0.5, 1.5, size=(N, H, Dk)).astype(np.float32)
    io = cfg.get("io", "bf16")
    if io == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    elif io != "f32":
        raise ValueError(f"unknown io dtype {io!r}")
    return OsdnInputs(q=q, k=k, v=v, beta=beta, r=r, eta=float(cfg.get("eta", 0.05)), d0=d0,
                      S0=S0, cu_seqlens=cu, io=io, chunk=int(cfg.get("chunk", 64)),
                      scale=float(cfg.get("scale", 1.0)))


def select(inp: OsdnInputs, seqs=None, heads=None) -> OsdnInputs:
    """Sub-batch of whole sequences and heads (for sampled checks at full size)."""
    H = inp.H
    heads = list(range(H)) if heads is None else list(heads)
    seqs = list(range(inp.N)) if seqs is None else list(seqs)

    def hsel(a):
        return None if a is None else np.ascontiguousarray(a[:, :, heads])

    if inp.cu_seqlens is None:
        def bsel(a):
            return None if a is None else np.ascontiguousarray(a[seqs])
        q, k, v, beta, r = (bsel(hsel(a)) for a in (inp.q, inp.k, inp.v, inp.beta, inp.r))
        cu = None
    else:
        cu0 = inp.cu_seqlens
        rows = np.concatenate([np.arange(cu0[n], cu0[n + 1]) for n in seqs]) if seqs else \
            np.zeros(0, dtype=np.int64)

        def tsel(a):
            return None if a is None else np.ascontiguousarray(a[:, rows])
        q, k, v, beta, r = (tsel(hsel(a)) for a in (inp.q, inp.k, inp.v, inp.beta, inp.r))
        lens = np.array([cu0[n + 1] - cu0[n] for n in seqs], dtype=np.int64)
        cu = np.zeros(len(seqs) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(lens)
    d0 = None if inp.d0 is None else np.ascontiguousarray(inp.d0[seqs][:, heads])
    S0 = None if inp.S0 is None else np.ascontiguousarray(inp.S0[seqs][:, heads])
    return dataclasses.replace(inp, q=q, k=k, v=v, beta=beta, r=r, d0=d0, S0=S0, cu_seqlens=cu)


def to_torch(inp: OsdnInputs, device="cuda"):
    """Device tensors for one batch: io tensors in the io dtype, gates/states float32,
    cu_seqlens int32.  Returns a dict keyed like the binding's arguments."""
    import torch
    dt = torch.bfloat16 if inp.io == "bf16" else torch.float32

    def io(a):
        return torch.from_numpy(a).to(device=device, dtype=dt).contiguous()

    def f32(a):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)

    out = dict(q=io(inp.q), k=io(inp.k), v=io(inp.v), beta=f32(inp.beta), r=f32(inp.r),
               d0=f32(inp.d0), S0=f32(inp.S0), eta=inp.eta, scale=inp.scale, chunk=inp.chunk)
    out["cu_seqlens"] = None if inp.cu_seqlens is None else \
        torch.from_numpy(inp.cu_seqlens.astype(np.int32)).to(device)
    return out
