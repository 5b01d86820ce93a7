"""Helpers for the GPU tests: device copies of bf16 bit arrays and the error metrics."""
import json
import os

import numpy as np
import torch

from causal_video_diffusion_rope_b200 import dz, synth

# Tolerance of the attention output against the fp64 oracle (per call, over all
# compared elements): max |gpu - ref| <= 2e-2 and ||gpu - ref||_2 / ||ref||_2 <= 5e-3.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bits -> torch.bfloat16 CUDA tensor (same bytes)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16)


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return synth.f32_from_bf16_bits(to_bits(t)).astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    d = got - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    return max_abs, rel


def log_errors(what: str, max_abs: float, rel: float, n: int) -> None:
    """Append the measured errors to $DZ_PARITY_LOG (JSON lines) when it is set."""
    path = os.environ.get("DZ_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": what, "max_abs": max_abs, "rel_l2": rel,
                                "elements": int(n)}) + "\n")


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = "", max_abs_tol: float = MAX_ABS,
                 rel_tol: float = REL_L2):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    max_abs, rel = errors(got, ref)
    log_errors(what, max_abs, rel, got.size)
    assert max_abs <= max_abs_tol and rel <= rel_tol, \
        f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits, ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(np.ldexp(m, 8)), e - 8)


class Handle:
    """dz_attn handle for a given head count (destroyed on close)."""

    def __init__(self, heads: int, max_batch: int = 2, max_q_tokens: int = 16384,
                 max_pos_t: int = 4096, prerotate_tokens: int = 0):
        self.h = dz.dz_attn_create(dz.make_desc(num_heads=heads, max_batch=max_batch,
                                                max_q_tokens=max_q_tokens, max_pos_t=max_pos_t,
                                                prerotate_tokens=prerotate_tokens))
        self.heads = heads

    def close(self):
        if self.h:
            dz.dz_attn_destroy(self.h)
            self.h = None
