"""The five SRU layer workloads and a seeded generator for their inputs.

The layer shapes stand in for the language-model and classification layers of
"When Attention Meets Fast Recurrence" (T. Lei): d = 2048 is the width used in
its Figure 2 example, d = 3072 with an unroll of 1024 is the width and training
unroll of its base models (appendix, Tables 7-8), and L = 2048 follows its test
context lengths.  No dataset is read: every input is drawn here.

Distributions (per workload, see CONFIGS):
  x ~ N(0, 1) (fp32); X = bf16(x) for the projection when it runs in bf16
  W_cat rows ~ U(-sqrt(3/d), sqrt(3/d)); v ~ U(-0.5, 0.5)
  bias = 0 or ~ N(0, 0.1) (0.1 read as the standard deviation)
  c0 = 0 or ~ N(0, 1); dh ~ N(0, 1)
  lengths l_b ~ uniform integers on [L/2, L]; positions t >= l_b are padding
  U given directly (recurrence-only workload): bf16 ~ N(0, 1)

Storage-type rounding is round-to-nearest-even from fp32 to bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest, ties to even); returns the 16-bit patterns."""
    flat = np.ascontiguousarray(a, dtype=np.float32).reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint16)
    step = 1 << 24
    for s in range(0, flat.size, step):
        u = flat[s:s + step].view(np.uint32)
        out[s:s + step] = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    return out.reshape(np.shape(a))


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def lengths_to_mask(lengths: np.ndarray, L: int) -> np.ndarray:
    """(L, B) uint8 mask, 1 where t >= lengths[b] (a padded position)."""
    t = np.arange(L)[:, None]
    return (t >= np.asarray(lengths)[None, :]).astype(np.uint8)


@dataclasses.dataclass(frozen=True)
class SRUConfig:
    name: str
    L: int
    B: int
    d: int
    n_dir: int = 1
    alpha: float = 1.0
    seed: int = 0
    proj_dtype: str = "bf16"      # "fp32", "bf16" or "none" (U supplied directly)
    bias: str = "zero"            # "zero" or "normal0.1"
    c0: str = "zero"              # "zero" or "normal"
    masked: bool = False
    v_zero: bool = False
    backward: bool = True

    @property
    def tokens(self) -> int:
        return self.L * self.B

    @property
    def N(self) -> int:
        return self.n_dir * 3 * self.d

    def replace(self, **kw) -> "SRUConfig":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, SRUConfig] = {
    # single layer, fp32 throughout, forward and backward
    "tiny_fp32": SRUConfig("tiny_fp32", L=16, B=2, d=32, seed=0, proj_dtype="fp32"),
    # single layer forward, bf16 projection, fp32 recurrence
    "lm_fwd": SRUConfig("lm_fwd", L=256, B=32, d=512, seed=1, backward=False),
    # full training step, bf16 projection
    "lm_train": SRUConfig("lm_train", L=1024, B=16, d=2048, seed=2, bias="normal0.1", c0="normal"),
    # bidirectional with padding mask
    "bidir_masked": SRUConfig("bidir_masked", L=2048, B=64, d=1024, n_dir=2, seed=3,
                              bias="normal0.1", masked=True),
    # recurrence only, U supplied directly; run with v != 0 and with v = 0
    "rec_only": SRUConfig("rec_only", L=1024, B=16, d=3072, seed=4, proj_dtype="none"),
    "rec_only_v0": SRUConfig("rec_only_v0", L=1024, B=16, d=3072, seed=4, proj_dtype="none",
                             v_zero=True),
}


def generate(cfg: SRUConfig, with_grad: Optional[bool] = None, u_direct: bool = False) -> Dict[str, np.ndarray]:
    """Draw every input of one workload, deterministically from cfg.seed.

    Returns numpy arrays (host memory):
      x (L,B,d) f32; v, bias (n_dir,2,d) f32; c0 (B,n_dir,d) f32 or None;
      mask (L,B) u8 or None; lengths (B,) or None; dh (L,B,n_dir,d) f32 (if with_grad);
      for a projected workload: X (L*B,d) and W (N,d) in the projection type
        (bf16 bit patterns as uint16, or f32), and X_f32/W_f32 (their exact fp32 values);
      for a U-given workload, or with u_direct=True: U (L,B,n_dir,3,d) ~ N(0,1) in the
        storage type (bf16 bits, or f32 for an fp32 workload) and U_f32 its exact values.
        (X W^T with these distributions has N(0,1) entries, so a drawn U has the
        distribution of a projected one.)
    """
    if with_grad is None:
        with_grad = cfg.backward
    rng = np.random.default_rng(cfg.seed)
    L, B, d, nd = cfg.L, cfg.B, cfg.d, cfg.n_dir
    out: Dict[str, Optional[np.ndarray]] = {}
    x = rng.standard_normal((L, B, d), dtype=np.float32)
    out["x"] = x
    if cfg.proj_dtype != "none" and not u_direct:
        a = math.sqrt(3.0 / d)
        W = rng.uniform(-a, a, size=(nd * 3 * d, d)).astype(np.float32)
        if cfg.proj_dtype == "bf16":
            Xb = f32_to_bf16_bits(x.reshape(L * B, d))
            Wb = f32_to_bf16_bits(W)
            out["X"], out["W"] = Xb, Wb
            out["X_f32"], out["W_f32"] = bf16_bits_to_f32(Xb), bf16_bits_to_f32(Wb)
        else:
            out["X"], out["W"] = x.reshape(L * B, d), W
            out["X_f32"], out["W_f32"] = out["X"], W
    else:
        Uf = rng.standard_normal((L, B, nd, 3, d), dtype=np.float32)
        if cfg.proj_dtype == "fp32":
            out["U"] = Uf
            out["U_f32"] = Uf
        else:
            Ub = f32_to_bf16_bits(Uf)
            del Uf
            out["U"] = Ub
            out["U_f32"] = None  # widen on demand with bf16_bits_to_f32 (saves host memory)
    v = rng.uniform(-0.5, 0.5, size=(nd, 2, d)).astype(np.float32)
    if cfg.v_zero:
        v = np.zeros_like(v)
    out["v"] = v
    if cfg.bias == "normal0.1":
        out["bias"] = (0.1 * rng.standard_normal((nd, 2, d))).astype(np.float32)
    else:
        out["bias"] = np.zeros((nd, 2, d), dtype=np.float32)
    out["c0"] = rng.standard_normal((B, nd, d), dtype=np.float32) if cfg.c0 == "normal" else None
    if cfg.masked:
        lengths = rng.integers(L // 2, L, size=B, endpoint=True)
        out["lengths"] = lengths
        out["mask"] = lengths_to_mask(lengths, L)
    else:
        out["lengths"] = None
        out["mask"] = None
    if with_grad:
        out["dh"] = rng.standard_normal((L, B, nd, d), dtype=np.float32)
    return out
