"""Plain fp64 CPU oracle for RainFusion2.0 block-wise sparse attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  It shares no
code with the CUDA path (``image_dits_b200``), and neither imports the other.

The arithmetic lives in ``rf2_oracle.c`` (plain C, fp64, OpenMP); this module
only marshals numpy arrays and states the two integer readings of the paper
that the C code takes as arguments:

* ``keep_count``: how a keep ratio becomes the per-row top-n of eq. (8)
  (section 3.2 "Representative Token for Blocks").  The paper quotes only a
  sparsity ("80% sparsity", abstract and Table 1); the reading here is
  n = ceil(keep * T_b), clamped to [1, T_b], chosen before the sink is added.
* ``sink_start``: the first block of the first-frame sink (section 3.4 "First
  Frame Sink").  The first frame sits at the end of the permuted sequence, so
  every block from the one holding its first token onward touches it; the
  reading is block-level and conservative (a block with any first-frame token
  is a sink block).

bf16 tensors cross this interface as their raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

BLOCK = 64
_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rf2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (no fast-math: IEEE fp64 throughout)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.orc_permutation.argtypes = [i32] * 7 + [vp]
        lib.orc_permutation.restype = i32
        lib.orc_permute_rows.argtypes = [vp, vp, i64, i64, i64, vp]
        lib.orc_unpermute_rows.argtypes = [vp, vp, i64, i64, i64, vp]
        lib.orc_block_means.argtypes = [vp, i64, i64, i64, vp]
        lib.orc_pooled_scores.argtypes = [vp, vp, i64, i64, i64, vp]
        lib.orc_select_blocks.argtypes = [vp, i64, i64, i64, i64, vp, vp]
        lib.orc_select_cdf.argtypes = [vp, i64, i64, ctypes.c_double, i64, vp, vp, vp]
        lib.orc_masked_attention.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp, i64, vp, vp]
        lib.orc_num_threads.restype = i32
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _u16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        x = x.view(np.uint16)
    return x


def num_threads() -> int:
    return int(_load().orc_num_threads())


def num_blocks(N: int) -> int:
    """T_q = T_k = ceil(N / 64): section 3.1 (the bracket in the T_q formula
    is garbled in the source; the mask dimension ceil(N/b) fixes it)."""
    return (N + BLOCK - 1) // BLOCK


def keep_count(keep: float, Tb: int) -> int:
    n = math.ceil(keep * Tb - 1e-9)
    return max(1, min(Tb, n))


def sink_start(T: int, H: int, W: int, sink: bool, text: int = 0) -> int:
    """First sink block, or -1 when there is no full-attention region.

    With a single frame every token is a first-frame token, so every block is
    a sink block (start 0) and the mask is full.  Text tokens of a joint
    video-text attention sit after the video and join the full-attention
    region (section 3.4 groups the first frame with them): with the sink off
    the region starts at the first text token."""
    if sink:
        return ((T - 1) * H * W) // BLOCK
    if text > 0:
        return (T * H * W) // BLOCK
    return -1


def permutation(T: int, H: int, W: int, wt: int, wh: int, ww: int, sink: bool, text: int = 0) -> np.ndarray:
    """perm[p] = original index of the token at permuted position p: the
    [F,H,W] video tokens in window order, then the `text` tokens unmoved."""
    nv = T * H * W
    perm = np.empty(nv + text, dtype=np.int64)
    rc = _load().orc_permutation(T, H, W, wt, wh, ww, int(bool(sink)), _ptr(perm))
    if rc != 0:
        raise ValueError(f"orc_permutation failed ({rc})")
    perm[nv:] = np.arange(nv, nv + text)
    return perm


def permute(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """x: [..., N, d] bf16 bits -> rows reordered by perm."""
    x = _u16(x)
    N, d = x.shape[-2:]
    BH = x.size // (N * d)
    out = np.empty_like(x)
    _load().orc_permute_rows(_ptr(x), _ptr(out), BH, N, d, _ptr(np.ascontiguousarray(perm, np.int64)))
    return out


def unpermute(xp: np.ndarray, perm: np.ndarray) -> np.ndarray:
    xp = _u16(xp)
    N, d = xp.shape[-2:]
    BH = xp.size // (N * d)
    out = np.empty_like(xp)
    _load().orc_unpermute_rows(_ptr(xp), _ptr(out), BH, N, d, _ptr(np.ascontiguousarray(perm, np.int64)))
    return out


def block_means(xp: np.ndarray) -> np.ndarray:
    """[..., N, d] bf16 bits -> [..., T_b, d] float64 block means, eqs. (5)-(6)."""
    xp = _u16(xp)
    N, d = xp.shape[-2:]
    lead = xp.shape[:-2]
    BH = xp.size // (N * d)
    Tb = num_blocks(N)
    out = np.empty(lead + (Tb, d), dtype=np.float64)
    _load().orc_block_means(_ptr(xp), BH, N, d, _ptr(out))
    return out


def pooled_scores(qm: np.ndarray, km: np.ndarray) -> np.ndarray:
    """[..., T_b, d] x [..., T_b, d] -> [..., T_b, T_b] = q^ k^T / sqrt(d), eq. (7)."""
    qm = np.ascontiguousarray(qm, np.float64)
    km = np.ascontiguousarray(km, np.float64)
    Tb, d = qm.shape[-2:]
    BH = qm.size // (Tb * d)
    out = np.empty(qm.shape[:-2] + (Tb, Tb), dtype=np.float64)
    _load().orc_pooled_scores(_ptr(qm), _ptr(km), BH, Tb, d, _ptr(out))
    return out


def select_blocks(S: np.ndarray, n: int, sink_first: int):
    """Top-n per row (ties: lower j) plus the sink, eq. (8) + section 3.4.

    Returns (mask uint8 [..., T_b, T_b], thr float64 [..., T_b]) where thr is
    the n-th best score of each non-sink row (NaN on sink rows)."""
    S = np.ascontiguousarray(S, np.float64)
    Tb = S.shape[-1]
    BH = S.size // (Tb * Tb)
    if not 1 <= n <= Tb:
        raise ValueError("n out of range")
    mask = np.empty(S.shape, dtype=np.uint8)
    thr = np.empty(S.shape[:-1], dtype=np.float64)
    _load().orc_select_blocks(_ptr(S), BH, Tb, n, sink_first, _ptr(mask), _ptr(thr))
    return mask, thr


def select_cdf(S: np.ndarray, tau: float, sink_first: int):
    """CDF-threshold selection plus the sink (section 2, online adaptive
    patterns; section 3.4 for the sink).

    Per non-sink row the key blocks in the order (score desc, j asc) are kept
    until the cumulative softmax of the row's scores reaches tau.  Returns
    (mask uint8 [..., T_b, T_b], cum float64 [..., T_b, 2], bnd float64
    [..., T_b]): the cumulative probability before and after the last kept
    block, and that block's score (NaN on sink rows)."""
    S = np.ascontiguousarray(S, np.float64)
    Tb = S.shape[-1]
    BH = S.size // (Tb * Tb)
    if not 0.0 < tau <= 1.0:
        raise ValueError("tau out of range")
    mask = np.empty(S.shape, dtype=np.uint8)
    cum = np.empty(S.shape[:-1] + (2,), dtype=np.float64)
    bnd = np.empty(S.shape[:-1], dtype=np.float64)
    _load().orc_select_cdf(_ptr(S), BH, Tb, ctypes.c_double(tau), sink_first, _ptr(mask), _ptr(cum), _ptr(bnd))
    return mask, cum, bnd


def predict_mask_cdf(qp, kp, tau: float, T: int, H: int, W: int, sink: bool, text: int = 0):
    """Mask prediction with CDF-threshold selection: means, scores, CDF + sink.
    Returns (mask, cum, bnd, S)."""
    qm, km = block_means(qp), block_means(kp)
    S = pooled_scores(qm, km)
    mask, cum, bnd = select_cdf(S, tau, sink_start(T, H, W, sink, text))
    return mask, cum, bnd, S


def masked_attention(qp, kp, vp, mask: np.ndarray, items=None):
    """Softmax attention restricted to the kept blocks (section 3.1).

    qp/kp/vp: [BH, N, d] bf16 bits (permuted order); mask: [BH, T_b, T_b].
    items: optional int64 [(bh, i), ...] query blocks to evaluate (default all).
    Returns (out float64 [n_items, 64, d], lse float64 [n_items, 64]); rows
    past the end of the sequence are 0.
    """
    qp, kp, vp = _u16(qp), _u16(kp), _u16(vp)
    N, d = qp.shape[-2:]
    BH = qp.size // (N * d)
    Tb = num_blocks(N)
    mask = np.ascontiguousarray(mask, np.uint8).reshape(BH, Tb, Tb)
    if items is None:
        items = np.stack(np.meshgrid(np.arange(BH), np.arange(Tb), indexing="ij"), -1).reshape(-1, 2)
    items = np.ascontiguousarray(items, np.int64).reshape(-1, 2)
    out = np.zeros((items.shape[0], BLOCK, d), dtype=np.float64)
    lse = np.zeros((items.shape[0], BLOCK), dtype=np.float64)
    _load().orc_masked_attention(_ptr(qp), _ptr(kp), _ptr(vp), BH, N, d, _ptr(mask), _ptr(items),
                                 items.shape[0], _ptr(out), _ptr(lse))
    return out, lse


def full_attention_output(qp, kp, vp, mask):
    """All query blocks of masked_attention, reshaped to [BH, N, d]."""
    qp = _u16(qp)
    N, d = qp.shape[-2:]
    BH = qp.size // (N * d)
    out, lse = masked_attention(qp, kp, vp, mask)
    Tb = num_blocks(N)
    return (out.reshape(BH, Tb * BLOCK, d)[:, :N].copy(),
            lse.reshape(BH, Tb * BLOCK)[:, :N].copy())


def predict_mask(qp, kp, keep: float, T: int, H: int, W: int, sink: bool, text: int = 0):
    """Steps of mask prediction in the paper's order: means, scores, top-n + sink.
    Returns (mask, thr, S)."""
    qm, km = block_means(qp), block_means(kp)
    S = pooled_scores(qm, km)
    Tb = S.shape[-1]
    mask, thr = select_blocks(S, keep_count(keep, Tb), sink_start(T, H, W, sink, text))
    return mask, thr, S
