"""Seeded synthetic inputs for the DSA hot path.

Holds no arithmetic of the method: it only draws bf16 tensors (see synth.c for the
counter-based generator and the token layouts).  The oracle checks, the GPU tests and the
benchmark all take their inputs from here, so both sides of every parity check see the
same values.

Workloads (the pages' long-video shapes; attention shaped like a Qwen3-30B-A3B layer):
  tiny    L=1024,  k=256,  Hq=8,  Hkv=2, D=128, HI=4,  dI=64, every tensor iid N(0,1)
  32k     L=32768, k=2048, Hq=32, Hkv=4, D=128, HI=32, dI=64, K and kI block-structured
          in 128 frames of 256 tokens
  128k    L=131072, same shapes, repeating [512 frame tokens][64 iid text tokens]
  decode  16 sequences, 131072 cached tokens (128k layout) + 256 new iid tokens each
  256k    L=262144, same shapes, 1024 x ([16 iid text tokens][240 frame tokens])
Frame tokens of K and kI are block mean N(0,1) + 0.5 * N(0,1); Q, V, qI, w are iid N(0,1).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")

LAYOUT_IID, LAYOUT_BLOCKS, LAYOUT_FRAME_TEXT, LAYOUT_TEXT_FRAME = 0, 1, 2, 3

# tensor ids inside a stream key
T_Q, T_K, T_V, T_QI, T_KI, T_W, T_KMEAN, T_KIMEAN = 1, 2, 3, 4, 5, 6, 7, 8


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", src, "-o", _SO, "-lm"])
    return _SO


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        i64, u64, ptr = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p
        lib.synth_fill_bf16.argtypes = [ptr, i64, i64, i64, u64, u64, u64, ctypes.c_int,
                                        ctypes.c_int, i64, i64, i64]
        lib.synth_fill_bf16.restype = None
        lib.synth_block_ids.argtypes = [ptr, i64, i64, ctypes.c_int, i64, i64, i64]
        lib.synth_uniform_int.argtypes = [ptr, i64, i64, u64, u64]
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Config:
    name: str
    cid: int
    L: int
    k: int
    Hq: int = 32
    Hkv: int = 4
    D: int = 128
    HI: int = 32
    dI: int = 64
    layout: int = LAYOUT_IID
    p0: int = 0
    p1: int = 0
    batch: int = 1
    steps: int = 0          # decode steps (decode workload only)
    iid_from: int = -1      # tokens at/after this position are iid text
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def total_len(self) -> int:
        """Tokens per sequence including decode steps."""
        return self.L + self.steps

    def widths(self) -> dict:
        return {"q": self.Hq * self.D, "k": self.Hkv * self.D, "v": self.Hkv * self.D,
                "qI": self.HI * self.dI, "kI": self.dI, "w": self.HI}


CONFIGS = {
    "tiny": Config("tiny", 1, 1024, 256, Hq=8, Hkv=2, HI=4),
    "32k": Config("32k", 2, 32768, 2048, layout=LAYOUT_BLOCKS, p0=256),
    "128k": Config("128k", 3, 131072, 2048, layout=LAYOUT_FRAME_TEXT, p0=512, p1=64),
    "decode": Config("decode", 4, 131072, 2048, layout=LAYOUT_FRAME_TEXT, p0=512, p1=64,
                     batch=16, steps=256, iid_from=131072),
    "256k": Config("256k", 5, 262144, 2048, layout=LAYOUT_TEXT_FRAME, p0=16, p1=240),
}

_TENSORS = {"q": (T_Q, None), "k": (T_K, T_KMEAN), "v": (T_V, None), "qI": (T_QI, None),
            "kI": (T_KI, T_KIMEAN), "w": (T_W, None)}
_HEADS = {"q": ("Hq", "D"), "k": ("Hkv", "D"), "v": ("Hkv", "D"), "qI": ("HI", "dI"),
          "kI": (None, "dI"), "w": (None, "HI")}


def stream_key(cfg: Config, seq: int, tensor_id: int) -> int:
    return (cfg.cid << 40) | (seq << 8) | tensor_id


def tensor(cfg: Config, name: str, t0: int = 0, n_tok: int | None = None, seq: int = 0,
           out: np.ndarray | None = None) -> np.ndarray:
    """bf16 bits (uint16) of tensor `name` for tokens [t0, t0+n_tok) of sequence `seq`.

    Shapes: q [n, Hq, D]; k, v [n, Hkv, D]; qI [n, HI, dI]; kI [n, dI]; w [n, HI].
    """
    lib = _load()
    if n_tok is None:
        n_tok = cfg.total_len - t0
    tid, mid = _TENSORS[name]
    C = cfg.widths()[name]
    if out is None:
        out = np.empty(n_tok * C, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.size == n_tok * C and out.flags.c_contiguous
    structured = mid is not None and cfg.layout != LAYOUT_IID
    lib.synth_fill_bf16(out.ctypes.data, t0, n_tok, C, cfg.seed, stream_key(cfg, seq, tid),
                        stream_key(cfg, seq, mid or 0), int(structured), cfg.layout, cfg.p0,
                        cfg.p1, cfg.iid_from)
    h, d = _HEADS[name]
    if h is None:
        return out.reshape(n_tok, getattr(cfg, d))
    return out.reshape(n_tok, getattr(cfg, h), getattr(cfg, d))


def inputs(cfg: Config, t0: int = 0, n_tok: int | None = None, seq: int = 0,
           names=("q", "k", "v", "qI", "kI", "w")) -> dict:
    return {n: tensor(cfg, n, t0, n_tok, seq) for n in names}


def block_ids(cfg: Config, t0: int = 0, n_tok: int | None = None) -> np.ndarray:
    lib = _load()
    if n_tok is None:
        n_tok = cfg.total_len - t0
    out = np.empty(n_tok, dtype=np.int64)
    lib.synth_block_ids(out.ctypes.data, t0, n_tok, cfg.layout, cfg.p0, cfg.p1, cfg.iid_from)
    return out


def sample_rows(n: int, hi: int, seed: int = 0, key: int = 0x5A4D) -> np.ndarray:
    """n seeded uniform integers in [0, hi)."""
    lib = _load()
    out = np.empty(n, dtype=np.int64)
    lib.synth_uniform_int(out.ctypes.data, n, hi, seed, key)
    return out


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to float64."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_torch(a: np.ndarray):
    """A torch.bfloat16 CPU tensor sharing memory with bf16 bits `a`."""
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
