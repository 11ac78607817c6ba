"""Temporal rotary position embedding with a capped relative index, in float64 on the CPU.

TEST INFRASTRUCTURE: see the package docstring.

The step (Long-Horizon Streaming Video Generation via Hybrid Attention with Decoupled
Distillation, §2.C "additional stabilisation", the relative RoPE constraint): a pretrained
video model has seen temporal RoPE indices only up to some maximum (21 latent frames, say);
larger indices shift the distribution. For generation of any length the temporal index is
therefore written as an offset relative to a reference frame and held below an upper bound,
in training and in inference alike.

The pages give no formula. Readings taken (each is listed with its reason in the design
notes):
  * rotary embedding in its usual form: the head dimension is read as pairs (2i, 2i + 1), and
    pair i turns by the angle p * theta_i with theta_i = base ** (-2 i / t_dims);
  * the temporal band is the first t_dims dimensions of the head (pairs i < t_dims / 2); the
    other dimensions are left as they are (a 3-D embedding turns them by spatial positions,
    which the cap does not touch);
  * p = min(f - ref_frame, cap - 1) for a token of frame f, with f >= ref_frame: the offset
    from the reference frame (for example the oldest frame the window holds), capped.
"""
from __future__ import annotations

import numpy as np


def temporal_offsets(n_tokens, tokens_per_frame, first_frame, ref_frame, cap):
    """The capped relative index p of every token (token n lies in frame first_frame +
    n // tokens_per_frame)."""
    frames = first_frame + np.arange(n_tokens) // tokens_per_frame
    off = frames - ref_frame
    if np.any(off < 0):
        raise ValueError("tokens before the reference frame")
    return np.minimum(off, cap - 1)


def rope_temporal(x, tokens_per_frame, first_frame, ref_frame, cap, t_dims, base=10000.0):
    """x: [..., n_tokens, d]. Returns x with pair i < t_dims / 2 of each token turned by
    p * base ** (-2 i / t_dims), written as the 2 x 2 rotation of (x[2i], x[2i + 1])."""
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape[-2], x.shape[-1]
    if t_dims % 2 or not 0 <= t_dims <= d:
        raise ValueError("t_dims must be even and at most d")
    p = temporal_offsets(n, tokens_per_frame, first_frame, ref_frame, cap).astype(np.float64)
    out = x.copy()
    for i in range(t_dims // 2):
        theta = base ** (-2.0 * i / t_dims)
        c, s = np.cos(p * theta), np.sin(p * theta)
        a, b = x[..., 2 * i], x[..., 2 * i + 1]
        out[..., 2 * i] = a * c - b * s
        out[..., 2 * i + 1] = a * s + b * c
    return out
