"""Seeded synthetic workloads for hybrid (softmax-window + linear-state) attention.

This module only draws numbers and names sizes. It holds none of the method's
arithmetic (no feature map, no windows, no softmax), so the fp64 oracle and the
CUDA path can both consume its tensors without sharing any computation.

The shapes stand in for the video transformers the pages evaluate on
(Wan 2.1 1.3B at 480p: 30x52 = 1560 latent tokens per frame, 21 latent frames;
Wan 2.1 14B at 720p: 45x80 = 3600 tokens per frame; Hybrid Forcing's streaming
generation at 832x480 in chunks of 3 frames with a 9-frame window; Radial
Attention's 4x-longer videos: 84 frames). The pages measure on VBench and on
trained models; neither is used here: Q, K, V are i.i.d. normal draws with those
shapes.

Random draw recipe (all configs):
  * ``numpy.random.default_rng(seed)`` (PCG64);
  * if the workload has per-head standard deviations, first ``sigma_q`` then
    ``sigma_k``, each ``uniform(0.5, 2.0, size=H)``;
  * then Q, K, V, each ``standard_normal((B, H, N, d), dtype=float32)`` in C
    order, Q and K multiplied by their per-head sigma;
  * cast to the workload dtype with round-to-nearest-even (torch ``.to``).
Streaming steps use ``default_rng([seed, step])`` and draw Q, K, V of the
current chunk, then the block mask (``random(...) < 0.5``), then force the
diagonal tiles on. A chunk's earlier denoising calls draw the same way from
``default_rng([seed, step, 1000 + call])``.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch

TILE = 128  # key/query tile edge used by the block masks


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str                  # "window" | "blockmask" | "radial" | "stream"
    B: int
    H: int
    d: int
    tokens_per_frame: int
    n_frames: int
    chunk_frames: int = 1
    halo_frames: int = 0
    window_frames: int = 0     # stream only: latest frames kept in the KV window
    n_steps: int = 0           # stream only
    dtype: str = "bf16"        # "f32" | "bf16"
    per_head_std: bool = False
    seed: int = 0
    phi: str = "elu1"          # feature map of the linear branch: "elu1" | "relu" | "exp"
    sink_frames: int = 0       # stream only: leading frames kept in the window for good
    anchor_stride: int = 0     # lvsa only: every anchor_stride-th frame is a global anchor
    rotation: int = 0          # lvsa only: shift of the anchor grid
    note: str = ""

    @property
    def N(self) -> int:
        return self.tokens_per_frame * self.n_frames

    @property
    def chunk_tokens(self) -> int:
        return self.tokens_per_frame * self.chunk_frames

    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads. Sizes follow the workload descriptions; names say what they are.
TINY_F32 = Workload(
    name="tiny_bidir_f32_T4x64", mode="window", B=1, H=2, d=64,
    tokens_per_frame=64, n_frames=4, chunk_frames=1, halo_frames=0,
    dtype="f32", note="4 frames x 8x8 tokens, window = own frame")
WAN13B_BIDIR = Workload(
    name="wan1.3b_bidir_T21x1560", mode="window", B=1, H=12, d=128,
    tokens_per_frame=1560, n_frames=21, chunk_frames=3, halo_frames=1,
    note="21 latent frames x 30x52 tokens, window = 3-frame chunk +/- 1 frame")
WAN14B_BIDIR = Workload(
    name="wan14b_720p_bidir_T21x3600", mode="window", B=1, H=40, d=128,
    tokens_per_frame=3600, n_frames=21, chunk_frames=3, halo_frames=1,
    per_head_std=True,
    note="21 latent frames x 45x80 tokens, per-head std U[0.5,2] on Q and K")
STREAM_HF = Workload(
    name="stream_T120_chunk3_win9", mode="stream", B=1, H=12, d=128,
    tokens_per_frame=1560, n_frames=120, chunk_frames=3, window_frames=9,
    n_steps=40,
    note="40 chunk steps x 3 frames, 9-frame window, Bernoulli(0.5)+diagonal tile mask")
RADIAL_84F = Workload(
    name="radial_T84x1560", mode="radial", B=1, H=12, d=128,
    tokens_per_frame=1560, n_frames=84,
    note="84 latent frames x 1560 tokens, static radial tile mask")

LVSA_126F = Workload(
    name="lvsa_T126x1560_w11_s4", mode="lvsa", B=1, H=12, d=128,
    tokens_per_frame=1560, n_frames=126, window_frames=11, anchor_stride=4,
    note="Wan-1.3B shapes at a 6x horizon (126 latent frames); structured window of 11 frames "
         "plus every 4th frame as a global anchor (about a third of the tiles kept)")

WORKLOADS = {w.name: w for w in (TINY_F32, WAN13B_BIDIR, WAN14B_BIDIR, STREAM_HF, RADIAL_84F, LVSA_126F)}


def _cast(x: np.ndarray, w: Workload) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(w.torch_dtype())


def gen_qkv(w: Workload, seed: Optional[int] = None):
    """Q, K, V of a bidirectional workload as CPU tensors in the workload dtype."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.N, w.d)
    if w.per_head_std:
        sq = rng.uniform(0.5, 2.0, size=w.H).astype(np.float32)
        sk = rng.uniform(0.5, 2.0, size=w.H).astype(np.float32)
    q = rng.standard_normal(shape, dtype=np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    if w.per_head_std:
        q *= sq[None, :, None, None]
        k *= sk[None, :, None, None]
    return _cast(q, w), _cast(k, w), _cast(v, w)


def stream_tiles_per_chunk(w: Workload) -> int:
    return -(-w.chunk_tokens // TILE)


def stream_window_chunks(w: Workload, step: int) -> int:
    """Number of chunks visible at ``step``: the sink chunks (sink_frames) that exist, then
    the rolling window of window_frames frames."""
    n_sink = w.sink_frames // w.chunk_frames
    nwc = w.window_frames // w.chunk_frames
    if step < n_sink:
        return step + 1
    return n_sink + min(step - n_sink + 1, nwc)


def gen_stream_step(w: Workload, step: int, seed: Optional[int] = None, keep_prob: float = 0.5,
                    call: Optional[int] = None):
    """Q, K, V of chunk ``step`` ([B,H,chunk_tokens,d]) and its tile mask.

    The mask is uint8 [H, tiles_per_chunk, tiles_per_chunk * n_window_chunks];
    key tiles are ordered oldest window chunk first. Tile (i, j) of the newest
    chunk's diagonal is always set; the rest is Bernoulli(keep_prob).
    ``call`` selects the inputs of an earlier (non-final) denoising call of the
    chunk, drawn from their own stream; None gives the chunk's final inputs.
    """
    base = [w.seed if seed is None else seed, step]
    rng = np.random.default_rng(base if call is None else base + [1000 + call])
    shape = (w.B, w.H, w.chunk_tokens, w.d)
    q = rng.standard_normal(shape, dtype=np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    nqt = stream_tiles_per_chunk(w)
    nwin = stream_window_chunks(w, step)
    mask = (rng.random((w.H, nqt, nqt * nwin)) < keep_prob).astype(np.uint8)
    diag = np.arange(nqt)
    mask[:, diag, nqt * (nwin - 1) + diag] = 1
    return _cast(q, w), _cast(k, w), _cast(v, w), mask


def gen_tile_mask(H: int, n_q_tiles: int, n_k_tiles: int, seed: int, keep_prob: float = 0.5):
    """A generic Bernoulli tile mask uint8 [H, nQT, nKT] for block-mask tests."""
    rng = np.random.default_rng([seed, 7919])
    return (rng.random((H, n_q_tiles, n_k_tiles)) < keep_prob).astype(np.uint8)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a CPU tensor (bf16 or f32 values) to a float64 array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
