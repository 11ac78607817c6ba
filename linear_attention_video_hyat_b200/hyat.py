"""Thin ctypes binding of libhyat (include/hyat.h).

Only argument marshalling lives here: every step of the forward pass runs in
the library's CUDA kernels. PyTorch supplies device memory (tensors and the
workspace) and the current CUDA stream. If the compiled library is missing the
import fails loudly; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhyat.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_STATE = range(6)
F32, BF16 = 0, 1
MODE_WINDOW, MODE_BLOCKMASK, MODE_RADIAL, MODE_STREAM = range(4)
FLAG_SIMT = 1
FLAG_TEST_DEVICE_TIMEOUT = 2
FLAG_SINGLE_TILE = 4
FLAG_PAIR_ONE_WARP = 8
FLAG_TEST_SOFTMAX_BRANCH = 16     # test hook: the call returns the softmax branch alone
FLAG_TEST_LINEAR_BRANCH = 32      # test hook: the call returns the linear branch alone
TILE = 128
KERNEL_KINDS = ("state", "complement", "attention", "fold", "prep")

_MODES = {"window": MODE_WINDOW, "blockmask": MODE_BLOCKMASK, "radial": MODE_RADIAL, "stream": MODE_STREAM,
          "lvsa": MODE_BLOCKMASK}   # LVSA: a block mask from lvsa_mask()

EXPORTED = (
    "hyat_workspace_bytes", "hyat_create", "hyat_fwd_bidir", "hyat_fwd_stream_step", "hyat_sync",
    "hyat_destroy", "hyat_last_error", "hyat_status_string", "hyat_plan_layout", "hyat_radial_mask",
    "hyat_stream_plan", "hyat_stream_state_bytes", "hyat_stream_get_state", "hyat_stream_set_state",
    "hyat_set_profiling", "hyat_kernel_times", "hyat_fwd_bidir_noalloc", "hyat_fwd_stream_denoise",
    "hyat_lvsa_mask", "hyat_rope_temporal", "hyat_fwd_stream_step_dev", "hyat_fwd_stream_step_graph",
    "hyat_stream_get_layout", "hyat_get_pairs",
)


class HyatError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"hyat status {status}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
        ("tokens_per_frame", ctypes.c_int32), ("n_frames", ctypes.c_int32),
        ("chunk_frames", ctypes.c_int32), ("halo_frames", ctypes.c_int32),
        ("window_frames", ctypes.c_int32), ("mode", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("phi", ctypes.c_int32), ("mask_heads", ctypes.c_int32), ("flags", ctypes.c_uint32),
        ("scale", ctypes.c_float), ("sink_frames", ctypes.c_int32),
        ("rope_t_dims", ctypes.c_int32), ("rope_cap", ctypes.c_int32), ("rope_base", ctypes.c_float),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libhyat.so not built ({LIB_PATH}); run "
                          f"`python -m linear_attention_video_hyat_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, S, I32, I64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
    CP = ctypes.POINTER(Config)
    sig = {
        "hyat_workspace_bytes": (S, [CP]),
        "hyat_create": (ctypes.c_int, [CP, P, S, P, ctypes.POINTER(P)]),
        "hyat_fwd_bidir": (ctypes.c_int, [P, P, P, P, P, P]),
        "hyat_fwd_stream_step": (ctypes.c_int, [P, P, P, P, P, P, P]),
        "hyat_fwd_stream_denoise": (ctypes.c_int, [P, P, P, P, P, P, P]),
        "hyat_fwd_stream_step_dev": (ctypes.c_int, [P, P, P, P, P, P, P]),
        "hyat_fwd_stream_step_graph": (ctypes.c_int, [P, P, P, P, P, P, P]),
        "hyat_stream_get_layout": (ctypes.c_int, [P, P, S, P, S, P, S, ctypes.POINTER(I64)]),
        "hyat_get_pairs": (ctypes.c_int, [P, P, S, ctypes.POINTER(I64)]),
        "hyat_sync": (ctypes.c_int, [P]),
        "hyat_destroy": (ctypes.c_int, [P]),
        "hyat_last_error": (ctypes.c_char_p, [P]),
        "hyat_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "hyat_plan_layout": (ctypes.c_int, [CP, P, P, S, P, S, ctypes.POINTER(I64)]),
        "hyat_radial_mask": (ctypes.c_int, [I32, I32, P, S]),
        "hyat_lvsa_mask": (ctypes.c_int, [I32, I32, I32, I32, I32, P, S]),
        "hyat_stream_plan": (ctypes.c_int, [CP, I32, P, S]),
        "hyat_stream_state_bytes": (S, [P]),
        "hyat_stream_get_state": (ctypes.c_int, [P, P, S]),
        "hyat_stream_set_state": (ctypes.c_int, [P, P, S]),
        "hyat_set_profiling": (ctypes.c_int, [P, ctypes.c_int]),
        "hyat_kernel_times": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I64), ctypes.c_int]),
        "hyat_fwd_bidir_noalloc": (ctypes.c_int, [CP, P, P, P, P, P]),
        "hyat_rope_temporal": (ctypes.c_int, [P, P, I32, I32, I32, I32, I32, I32, I32, I32, I32, ctypes.c_float, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


PHI = {"elu1": 0, "relu": 1, "exp": 2}   # hyat_phi


def make_config(mode, B, H, d, tokens_per_frame, n_frames=0, chunk_frames=1, halo_frames=0,
                window_frames=0, dtype=BF16, mask_heads=1, flags=0, scale=0.0, phi="elu1",
                sink_frames=0, rope=None) -> Config:
    """rope: None, or {"t_dims", "cap", "base"} for the capped temporal RoPE fused into a STREAM
    handle's steps (see hyat_config.rope_t_dims)."""
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    dt = {"f32": F32, "bf16": BF16}.get(dtype, dtype) if isinstance(dtype, str) else int(dtype)
    ph = PHI[phi] if isinstance(phi, str) else int(phi)
    return Config(B, H, d, tokens_per_frame, n_frames, chunk_frames, halo_frames, window_frames,
                  m, dt, ph, mask_heads, flags, float(scale), int(sink_frames),
                  int(rope["t_dims"]) if rope else 0, int(rope["cap"]) if rope else 0,
                  float(rope.get("base", 0.0)) if rope else 0.0)


def config_from_workload(w, flags=0, mask_heads=1, rope=None) -> Config:
    return make_config(w.mode, w.B, w.H, w.d, w.tokens_per_frame, w.n_frames, w.chunk_frames,
                       w.halo_frames, w.window_frames, w.dtype, mask_heads=mask_heads, flags=flags,
                       phi=getattr(w, "phi", "elu1"), sink_frames=getattr(w, "sink_frames", 0), rope=rope)


def _check(status, handle=None):
    if status != OK:
        msg = lib.hyat_last_error(handle).decode() if handle else lib.hyat_status_string(status).decode()
        raise HyatError(status, msg)


def _u8(arr) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(arr), dtype=np.uint8)


# ---------------------------------------------------------------- host hooks
def workspace_bytes(cfg: Config) -> int:
    return int(lib.hyat_workspace_bytes(ctypes.byref(cfg)))


def plan_layout(cfg: Config, mask=None):
    """Host-only layout: (work [n,8] int32, entries [m,2] int32)."""
    counts = (ctypes.c_int64 * 2)()
    m = None if mask is None else _u8(mask)
    mp = None if m is None else m.ctypes.data
    _check(lib.hyat_plan_layout(ctypes.byref(cfg), mp, None, 0, None, 0, counts))
    work = np.zeros((counts[0], 8), np.int32)
    ent = np.zeros((max(counts[1], 1), 2), np.int32)
    _check(lib.hyat_plan_layout(ctypes.byref(cfg), mp, work.ctypes.data, work.size,
                                ent.ctypes.data, ent.size, counts))
    return work, ent[:counts[1]]


def lvsa_mask(n_frames: int, tokens_per_frame: int, window_frames: int, anchor_stride: int,
              rotation: int = 0) -> np.ndarray:
    """Structured-window + rotating-anchor tile mask (see hyat_lvsa_mask) for BLOCKMASK handles."""
    nT = -(-n_frames * tokens_per_frame // TILE)
    out = np.zeros((nT, nT), np.uint8)
    _check(lib.hyat_lvsa_mask(n_frames, tokens_per_frame, window_frames, anchor_stride, rotation,
                              out.ctypes.data, out.size))
    return out


def rope_temporal(x, tokens_per_frame: int, first_frame: int, ref_frame: int, cap: int, t_dims: int,
                  base: float = 10000.0, out=None, stream=None):
    """Capped relative temporal RoPE (see hyat_rope_temporal) of a contiguous CUDA tensor
    [..., n_tokens, d] (f32 or bf16); out=x works in place."""
    dt = {torch.float32: F32, torch.bfloat16: BF16}.get(x.dtype)
    if x.device.type != "cuda" or dt is None or not x.is_contiguous() or x.dim() < 2:
        raise ValueError("need a contiguous f32 or bf16 CUDA tensor [..., n_tokens, d]")
    out = torch.empty_like(x) if out is None else out
    if out.shape != x.shape or out.dtype != x.dtype or not out.is_contiguous() or out.device != x.device:
        raise ValueError("out must match x")
    n, d = x.shape[-2], x.shape[-1]
    bh = x.numel() // max(n * d, 1) if n * d else 0
    s = torch.cuda.current_stream(x.device) if stream is None else stream
    _check(lib.hyat_rope_temporal(x.data_ptr(), out.data_ptr(), bh, n, d, dt, tokens_per_frame, first_frame,
                                  ref_frame, cap, t_dims, float(base), s.cuda_stream))
    return out


def radial_mask(n_frames: int, tokens_per_frame: int) -> np.ndarray:
    nT = -(-n_frames * tokens_per_frame // TILE)
    out = np.zeros((nT, nT), np.uint8)
    _check(lib.hyat_radial_mask(n_frames, tokens_per_frame, out.ctypes.data, out.size))
    return out


def stream_plan(cfg: Config, step: int):
    nwc = cfg.window_frames // cfg.chunk_frames + cfg.sink_frames // cfg.chunk_frames   # ring slots
    info = np.zeros(4 + nwc, np.int32)
    _check(lib.hyat_stream_plan(ctypes.byref(cfg), step, info.ctypes.data, info.size))
    return {"first_visible": int(info[0]), "n_visible": int(info[1]), "evicted": int(info[2]),
            "write_slot": int(info[3]), "slots": [int(x) for x in info[4:4 + info[1]]]}


# ---------------------------------------------------------------- device API
class Hyat:
    """A handle bound to one configuration, its workspace and (for STREAM) its state."""

    def __init__(self, cfg: Config, mask=None, device=None):
        if not torch.cuda.is_available():
            raise RuntimeError("libhyat needs a CUDA device")
        self.cfg = cfg
        self.device = torch.device(device if device is not None else "cuda")
        nbytes = workspace_bytes(cfg)
        if nbytes == 0:
            raise HyatError(ERR_INVALID_ARG, "invalid configuration")
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
            off = (-self.workspace.data_ptr()) % 256
            self._ws_ptr = self.workspace.data_ptr() + off
            self._mask = None if mask is None else _u8(mask)
            h = ctypes.c_void_p()
            st = lib.hyat_create(ctypes.byref(cfg), self._ws_ptr, nbytes,
                                 None if self._mask is None else self._mask.ctypes.data, ctypes.byref(h))
            _check(st)
        self.handle = h
        self.dtype = torch.float32 if cfg.dtype == F32 else torch.bfloat16

    def close(self):
        if getattr(self, "handle", None):
            lib.hyat_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check_t(self, t, name, rows):
        c = self.cfg
        if t.device.type != "cuda" or t.dtype != self.dtype or not t.is_contiguous():
            raise ValueError(f"{name}: need a contiguous {self.dtype} CUDA tensor")
        if tuple(t.shape) != (c.B, c.H, rows, c.d):
            raise ValueError(f"{name}: shape {tuple(t.shape)} != {(c.B, c.H, rows, c.d)}")

    def forward(self, q, k, v, out=None, stream=None):
        c = self.cfg
        n = c.tokens_per_frame * c.n_frames
        for t, nm in ((q, "q"), (k, "k"), (v, "v")):
            self._check_t(t, nm, n)
        out = torch.empty_like(q) if out is None else out
        self._check_t(out, "out", n)
        s = torch.cuda.current_stream(q.device) if stream is None else stream
        _check(lib.hyat_fwd_bidir(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  s.cuda_stream), self.handle)
        return out

    def _stream_call(self, fn, q, k, v, mask, out, stream):
        c = self.cfg
        L = c.chunk_frames * c.tokens_per_frame
        for t, nm in ((q, "q"), (k, "k"), (v, "v")):
            self._check_t(t, nm, L)
        out = torch.empty_like(q) if out is None else out
        self._check_t(out, "out", L)
        m = None if mask is None else _u8(mask)
        s = torch.cuda.current_stream(q.device) if stream is None else stream
        _check(fn(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                  None if m is None else m.ctypes.data, s.cuda_stream), self.handle)
        return out

    def stream_step(self, q, k, v, mask=None, out=None, stream=None):
        """The current chunk's final call: attend, then keep its K, V and advance."""
        return self._stream_call(lib.hyat_fwd_stream_step, q, k, v, mask, out, stream)

    def stream_step_dev(self, q, k, v, mask=None, out=None, stream=None, graph=False):
        """stream_step with the mask as a uint8 CUDA tensor (None: every tile kept); graph=True
        replays steady steps from CUDA graphs captured by the library."""
        c = self.cfg
        L = c.chunk_frames * c.tokens_per_frame
        for t, nm in ((q, "q"), (k, "k"), (v, "v")):
            self._check_t(t, nm, L)
        out = torch.empty_like(q) if out is None else out
        self._check_t(out, "out", L)
        if mask is not None and (mask.device.type != "cuda" or mask.dtype != torch.uint8 or not mask.is_contiguous()):
            raise ValueError("mask: need a contiguous uint8 CUDA tensor")
        s = torch.cuda.current_stream(q.device) if stream is None else stream
        fn = lib.hyat_fwd_stream_step_graph if graph else lib.hyat_fwd_stream_step_dev
        _check(fn(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                  None if mask is None else mask.data_ptr(), s.cuda_stream), self.handle)
        return out

    def stream_layout(self):
        """The layout the last streaming call built on the device: (work [n, 8], entries
        [n, cap, 2], plan info of that step, step)."""
        counts = (ctypes.c_int64 * 3)()
        _check(lib.hyat_stream_get_layout(self.handle, None, 0, None, 0, None, 0, counts), self.handle)
        n, ne = counts[0], counts[1]
        c = self.cfg
        slots = c.window_frames // c.chunk_frames + c.sink_frames // c.chunk_frames
        work = np.zeros((n, 8), np.int32)
        ent = np.zeros((ne, 2), np.int32)
        info = np.zeros(4 + slots, np.int32)
        _check(lib.hyat_stream_get_layout(self.handle, work.ctypes.data, work.size, ent.ctypes.data, ent.size,
                                          info.ctypes.data, info.size, counts), self.handle)
        return work, ent.reshape(n, ne // max(n, 1), 2), info, int(counts[2])

    def pairs(self):
        """The attention kernel's pair list as the last call left it: int32 [n_pairs, 4]
        {item0, item1, shared, split}; pair k runs on CTA k mod min(n_pairs, SMs)."""
        n = ctypes.c_int64()
        _check(lib.hyat_get_pairs(self.handle, None, 0, ctypes.byref(n)), self.handle)
        out = np.zeros((n.value, 4), np.int32)
        _check(lib.hyat_get_pairs(self.handle, out.ctypes.data, out.size, ctypes.byref(n)), self.handle)
        return out

    def stream_denoise(self, q, k, v, mask=None, out=None, stream=None):
        """A non-final call for the current chunk (one denoising step): attend with this
        call's K, V as the newest chunk, without advancing."""
        return self._stream_call(lib.hyat_fwd_stream_denoise, q, k, v, mask, out, stream)

    def sync(self):
        _check(lib.hyat_sync(self.handle), self.handle)

    def get_state(self) -> bytes:
        n = lib.hyat_stream_state_bytes(self.handle)
        buf = ctypes.create_string_buffer(n)
        _check(lib.hyat_stream_get_state(self.handle, ctypes.addressof(buf), n), self.handle)
        return buf.raw

    def set_state(self, blob: bytes):
        buf = ctypes.create_string_buffer(blob, len(blob))
        _check(lib.hyat_stream_set_state(self.handle, ctypes.addressof(buf), len(blob)), self.handle)

    def set_profiling(self, on: bool):
        _check(lib.hyat_set_profiling(self.handle, 1 if on else 0), self.handle)

    def kernel_times(self):
        n = len(KERNEL_KINDS)
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int64 * n)()
        _check(lib.hyat_kernel_times(self.handle, ms, cnt, n), self.handle)
        return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS)}
