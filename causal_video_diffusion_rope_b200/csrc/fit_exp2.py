"""Fit of the cubic used by the attention kernel's FMA-pipe exp2 (csrc/dz_attn.cu, exp2_poly2).

2^x is computed as 2^n * 2^f with n = round(x) (by the 1.5 * 2^23 rounding
trick) and f = x - n in [-1/2, 1/2]; 2^f is a cubic fitted here for minimal
maximum relative error by Lawson's iteratively reweighted least squares on a
dense grid.  Run: python causal_video_diffusion_rope_b200/csrc/fit_exp2.py
"""
import numpy as np
# minimax (relative error) fit of 2^f on [-0.5, 0.5] with a cubic, by iteratively
# reweighted least squares on a dense grid (Lawson's algorithm)
f = np.linspace(-0.5, 0.5, 20001)
y = np.exp2(f)
V = np.vander(f, 4, increasing=True)
w = np.ones_like(f)
for it in range(200):
    W = w / y
    c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
    err = (V @ c - y) / y
    w = w * np.abs(err) ** 1.0
    w /= w.sum()
print("coeffs", repr(c.tolist()))
c32 = c.astype(np.float32)
# evaluate in float32 Horner as the kernel will
ff = f.astype(np.float32)
p = ((c32[3] * ff + c32[2]) * ff + c32[1]) * ff + c32[0]
print("max rel err (f32 Horner)", np.max(np.abs(p.astype(np.float64) / y - 1)))
for d in [4]:
    V = np.vander(f, d + 1, increasing=True); w = np.ones_like(f)
    for it in range(200):
        W = w / y
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        err = (V @ c - y) / y
        w = w * np.abs(err); w /= w.sum()
    print("deg", d, "max rel", np.abs(err).max(), repr(c.tolist()))
