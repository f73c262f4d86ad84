"""Python binding of the C ABI in ``include/rf2.h`` (ctypes; marshalling only).

Every step of the path runs in ``librf2.so``'s CUDA kernels.  PyTorch only
provides device memory and the current stream.  There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librf2.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "librf2_checked.so")     # built with RF2_CHECKED=1

RF2_OK = 0
RF2_ERR_INVALID_ARGUMENT = 1
RF2_ERR_UNSUPPORTED = 2
RF2_ERR_INSUFFICIENT_WORKSPACE = 3
RF2_ERR_CUDA = 4
RF2_ERR_TIMEOUT = 5
RF2_ERR_RANGE = 6

# Every entry point declared in include/rf2.h.
EXPORTED = (
    "rf2_status_string", "rf2_query", "rf2_permutation_index", "rf2_permute", "rf2_unpermute",
    "rf2_predict_mask", "rf2_predict_mask_static", "rf2_permute_qk_pool", "rf2_predict_mask_pooled",
    "rf2_predict_mask_cdf", "rf2_predict_mask_cdf_pooled",
    "rf2_block_sparse_attn", "rf2_device_status", "rf2_selftest_wait_timeout",
    "rf2_attention_host_query", "rf2_attention_host", "rf2_host_events_create", "rf2_host_events_destroy",
)


class Geometry(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "heads", "head_dim", "frames", "height", "width",
        "win_t", "win_h", "win_w", "block", "first_frame_sink", "text_tokens")]


class Sizes(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int64),
        ("num_blocks", ctypes.c_int32),
        ("n_keep", ctypes.c_int32),
        ("sink_first", ctypes.c_int32),
        ("row_capacity", ctypes.c_int32),
        ("num_rows", ctypes.c_int64),
        ("col_idx_capacity", ctypes.c_int64),
        ("mask_workspace_bytes", ctypes.c_size_t),
    ]


class Rf2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_lib = None


def lib():
    """Load librf2.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


def use_library(path: str):
    """Route every call of this module through the library at `path` (for
    example CHECKED_LIB_PATH); returns the one it replaces (None if none was
    loaded yet)."""
    global _lib
    old = _lib
    _lib = load(path)
    return old


def load(path: str):
    """Load a build of the library and declare its entry points."""
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run image_dits_b200.build.build())")
    L = ctypes.CDLL(path)
    vp, i32, f64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_size_t
    G = ctypes.POINTER(Geometry)
    L.rf2_status_string.argtypes = [i32]
    L.rf2_status_string.restype = ctypes.c_char_p
    L.rf2_query.argtypes = [G, f64, ctypes.POINTER(Sizes)]
    L.rf2_permutation_index.argtypes = [G, vp]
    L.rf2_permute.argtypes = [G, vp, vp, vp]
    L.rf2_unpermute.argtypes = [G, vp, vp, vp]
    L.rf2_predict_mask.argtypes = [G, vp, vp, f64, vp, vp, vp, vp, sz, vp]
    L.rf2_predict_mask_static.argtypes = [G, vp, vp, f64, vp, vp, vp, vp]
    L.rf2_permute_qk_pool.argtypes = [G, vp, vp, vp, vp, vp, sz, vp]
    L.rf2_predict_mask_pooled.argtypes = [G, f64, vp, vp, vp, vp, sz, vp]
    L.rf2_predict_mask_cdf.argtypes = [G, vp, vp, f64, vp, vp, vp, vp, sz, vp]
    L.rf2_predict_mask_cdf_pooled.argtypes = [G, f64, vp, vp, vp, vp, sz, vp]
    L.rf2_block_sparse_attn.argtypes = [G, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.rf2_device_status.argtypes = [vp]
    L.rf2_selftest_wait_timeout.argtypes = [ctypes.c_uint32, ctypes.POINTER(ctypes.c_int32), vp]
    L.rf2_attention_host_query.argtypes = [G, f64, f64, i32, ctypes.POINTER(HostSizes)]
    L.rf2_attention_host.argtypes = [G, f64, f64, i32, vp, vp, vp, vp, vp, sz, vp, vp, vp,
                                     ctypes.POINTER(vp), i32]
    L.rf2_host_events_create.argtypes = [i32, ctypes.POINTER(vp)]
    L.rf2_host_events_destroy.argtypes = [i32, ctypes.POINTER(vp)]
    for name in EXPORTED:
        if name != "rf2_status_string":
            getattr(L, name).restype = i32
    return L


def status_string(status: int) -> str:
    return lib().rf2_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != RF2_OK:
        raise Rf2Error(status, what)


def make_geometry(batch, heads, head_dim, frames, height, width, win_t, win_h, win_w, sink, block=64,
                  text=0) -> Geometry:
    return Geometry(batch, heads, head_dim, frames, height, width, win_t, win_h, win_w, block, int(bool(sink)),
                    int(text))


def num_tokens(geom: Geometry) -> int:
    """Sequence length N: video tokens, then text tokens."""
    return geom.frames * geom.height * geom.width + geom.text_tokens


def geometry_of(wl, batch: int | None = None) -> Geometry:
    """Geometry of a ``workload.Workload``."""
    return make_geometry(wl.batch if batch is None else batch, wl.heads, wl.head_dim, wl.frames, wl.height,
                         wl.width, wl.win_t, wl.win_h, wl.win_w, wl.sink, text=wl.text_tokens)


def query(geom: Geometry, keep: float = 1.0) -> Sizes:
    out = Sizes()
    _check(lib().rf2_query(ctypes.byref(geom), float(keep), ctypes.byref(out)), "rf2_query")
    return out


def permutation_index(geom: Geometry) -> np.ndarray:
    perm = np.empty(num_tokens(geom), dtype=np.int32)
    _check(lib().rf2_permutation_index(ctypes.byref(geom), perm.ctypes.data), "rf2_permutation_index")
    return perm


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check_qkv(geom: Geometry, *ts):
    shape = (geom.batch, geom.heads, num_tokens(geom), geom.head_dim)
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and tuple(t.shape) == shape):
            raise ValueError(f"expected a contiguous CUDA bf16 tensor of shape {shape}, got "
                             f"{tuple(t.shape)} {t.dtype} {t.device}")


def permute(geom: Geometry, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _check_qkv(geom, x)
    out = torch.empty_like(x) if out is None else out
    _check_qkv(geom, out)
    _check(lib().rf2_permute(ctypes.byref(geom), x.data_ptr(), out.data_ptr(), _stream(stream)), "rf2_permute")
    return out


def unpermute(geom: Geometry, xp: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _check_qkv(geom, xp)
    out = torch.empty_like(xp) if out is None else out
    _check_qkv(geom, out)
    _check(lib().rf2_unpermute(ctypes.byref(geom), xp.data_ptr(), out.data_ptr(), _stream(stream)), "rf2_unpermute")
    return out


@dataclass
class BlockMask:
    """CSR block mask: row r = (b*heads + h)*T_b + i keeps
    col_idx[row_start[r] : row_start[r] + row_count[r]] (ascending)."""
    row_start: torch.Tensor
    row_count: torch.Tensor
    col_idx: torch.Tensor
    sizes: Sizes

    def dense(self) -> np.ndarray:
        """[B*H, T_b, T_b] uint8 on the host (for tests)."""
        Tb = self.sizes.num_blocks
        rs = self.row_start.cpu().numpy().astype(np.int64)
        rc = self.row_count.cpu().numpy().astype(np.int64)
        ci = self.col_idx.cpu().numpy()
        out = np.zeros((rs.size, Tb), np.uint8)
        for r in range(rs.size):
            out[r, ci[rs[r]:rs[r] + rc[r]]] = 1
        return out.reshape(-1, Tb, Tb)

    def kept_pairs(self) -> int:
        return int(self.row_count.sum().item())


def alloc_mask(geom: Geometry, keep: float, device) -> tuple:
    sz = query(geom, keep)
    row_start = torch.empty(sz.num_rows, dtype=torch.int32, device=device)
    row_count = torch.empty(sz.num_rows, dtype=torch.int32, device=device)
    col_idx = torch.empty(max(1, sz.col_idx_capacity), dtype=torch.int32, device=device)
    ws = torch.empty(max(16, sz.mask_workspace_bytes), dtype=torch.uint8, device=device)
    return BlockMask(row_start, row_count, col_idx, sz), ws


def predict_mask(geom: Geometry, qp: torch.Tensor, kp: torch.Tensor, keep: float, mask: BlockMask | None = None,
                 workspace: torch.Tensor | None = None, stream=None) -> BlockMask:
    _check_qkv(geom, qp, kp)
    if mask is None or workspace is None:
        m2, ws2 = alloc_mask(geom, keep, qp.device)
        mask = mask or m2
        workspace = ws2 if workspace is None else workspace
    _check(lib().rf2_predict_mask(ctypes.byref(geom), qp.data_ptr(), kp.data_ptr(), float(keep),
                                  mask.row_start.data_ptr(), mask.row_count.data_ptr(), mask.col_idx.data_ptr(),
                                  workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                  _stream(stream)), "rf2_predict_mask")
    return mask


def predict_mask_cdf(geom: Geometry, qp: torch.Tensor, kp: torch.Tensor, tau: float, mask: BlockMask | None = None,
                     workspace: torch.Tensor | None = None, stream=None) -> BlockMask:
    """CDF-threshold mask (rows sized at full capacity: alloc_mask(geom, 1.0, ...))."""
    _check_qkv(geom, qp, kp)
    if mask is None or workspace is None:
        m2, ws2 = alloc_mask(geom, 1.0, qp.device)
        mask = mask or m2
        workspace = ws2 if workspace is None else workspace
    _check(lib().rf2_predict_mask_cdf(ctypes.byref(geom), qp.data_ptr(), kp.data_ptr(), float(tau),
                                      mask.row_start.data_ptr(), mask.row_count.data_ptr(), mask.col_idx.data_ptr(),
                                      workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                      _stream(stream)), "rf2_predict_mask_cdf")
    return mask


def predict_mask_cdf_pooled(geom: Geometry, tau: float, mask: BlockMask, workspace: torch.Tensor,
                            stream=None) -> BlockMask:
    """CDF-threshold mask from the block means rf2_permute_qk_pool left in `workspace`."""
    _check(lib().rf2_predict_mask_cdf_pooled(ctypes.byref(geom), float(tau), mask.row_start.data_ptr(),
                                             mask.row_count.data_ptr(), mask.col_idx.data_ptr(),
                                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                             _stream(stream)), "rf2_predict_mask_cdf_pooled")
    return mask


def permute_qk_pool(geom: Geometry, q: torch.Tensor, k: torch.Tensor, workspace: torch.Tensor,
                    qp: torch.Tensor | None = None, kp: torch.Tensor | None = None, stream=None):
    """Permute Q and K and leave their block means in the mask workspace."""
    _check_qkv(geom, q, k)
    qp = torch.empty_like(q) if qp is None else qp
    kp = torch.empty_like(k) if kp is None else kp
    _check_qkv(geom, qp, kp)
    _check(lib().rf2_permute_qk_pool(ctypes.byref(geom), q.data_ptr(), k.data_ptr(), qp.data_ptr(), kp.data_ptr(),
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                     _stream(stream)), "rf2_permute_qk_pool")
    return qp, kp


def predict_mask_pooled(geom: Geometry, keep: float, mask: BlockMask, workspace: torch.Tensor,
                        stream=None) -> BlockMask:
    """Mask prediction from the block means rf2_permute_qk_pool left in `workspace`."""
    _check(lib().rf2_predict_mask_pooled(ctypes.byref(geom), float(keep), mask.row_start.data_ptr(),
                                         mask.row_count.data_ptr(), mask.col_idx.data_ptr(), workspace.data_ptr(),
                                         workspace.numel() * workspace.element_size(), _stream(stream)),
           "rf2_predict_mask_pooled")
    return mask


def block_sparse_attn(geom: Geometry, qp, kp, vp, mask: BlockMask, out: torch.Tensor | None = None,
                      lse: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _check_qkv(geom, qp, kp, vp)
    out = torch.empty_like(qp) if out is None else out
    _check_qkv(geom, out)
    if lse is not None:
        n = num_tokens(geom)
        if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous()
                and lse.numel() == geom.batch * geom.heads * n):
            raise ValueError("lse must be a contiguous CUDA float32 tensor of B*H*N elements")
    _check(lib().rf2_block_sparse_attn(ctypes.byref(geom), qp.data_ptr(), kp.data_ptr(), vp.data_ptr(),
                                       mask.row_start.data_ptr(), mask.row_count.data_ptr(),
                                       mask.col_idx.data_ptr(), out.data_ptr(),
                                       lse.data_ptr() if lse is not None else None, _stream(stream)),
           "rf2_block_sparse_attn")
    return out


def device_status(stream=None) -> int:
    """Synchronize and return (and clear) the device status word."""
    return int(lib().rf2_device_status(_stream(stream)))


def selftest_wait_timeout(limit_us: int = 1000, stream=None) -> int:
    """Run the library's timeout self-test (a bounded wait on a barrier that
    nothing completes, and a second wait left through the abort flag); returns
    how many of the two waits gave up.  The timeout is then in the device
    status word (``device_status()`` returns RF2_ERR_TIMEOUT once)."""
    n = ctypes.c_int32(-1)
    _check(lib().rf2_selftest_wait_timeout(ctypes.c_uint32(int(limit_us)), ctypes.byref(n), _stream(stream)),
           "rf2_selftest_wait_timeout")
    return int(n.value)


def rainfusion_attention(geom: Geometry, q, k, v, keep: float, stream=None):
    """The whole path for one attention call: permute Q/K/V (block means of Q
    and K taken on the way), predict the block mask, block-sparse attention,
    unpermute.  Returns (O, mask)."""
    mask, ws = alloc_mask(geom, keep, q.device)
    qp, kp = permute_qk_pool(geom, q, k, ws, stream=stream)
    vp = permute(geom, v, stream=stream)
    predict_mask_pooled(geom, keep, mask, ws, stream=stream)
    op = block_sparse_attn(geom, qp, kp, vp, mask, stream=stream)
    return unpermute(geom, op, stream=stream), mask


def chunk_sizes(heads: int, chunks: int, tail_split: bool = True) -> list:
    """Heads per chunk of a HostPipeline: `chunks` near-equal chunks; with
    `tail_split` the last one is further split in shrinking parts down to one
    head (the host-to-device copies set the pace, and what follows the last of
    them is the last chunk's compute and copy back)."""
    n = max(1, min(int(chunks), int(heads)))
    cuts = [round(c * heads / n) for c in range(n + 1)]
    sizes = [cuts[c + 1] - cuts[c] for c in range(n)]
    if tail_split:
        r, tail = sizes.pop(), []
        while r > 1:
            h = (r + 1) // 2
            tail.append(h)
            r -= h
        sizes += tail + ([r] if r else [])
    return sizes


class HostSizes(ctypes.Structure):
    _fields_ = [("num_chunks", ctypes.c_int32), ("max_chunk_heads", ctypes.c_int32), ("work_bytes", ctypes.c_size_t)]


def host_query(geom: Geometry, keep: float | None = None, tau: float | None = None, chunks: int = 8) -> HostSizes:
    """rf2_attention_host_query: chunk count and device scratch of rf2_attention_host."""
    out = HostSizes()
    _check(lib().rf2_attention_host_query(ctypes.byref(geom), float(keep or 0.0), float(tau or 0.0), int(chunks),
                                          ctypes.byref(out)), "rf2_attention_host_query")
    return out


class HostPipeline:
    """One attention call on host (pinned) tensors, copies overlapped with
    compute: a thin wrapper over the C call rf2_attention_host, which copies
    head chunks in on one stream, computes them on a second and copies them
    back on a third (see include/rf2.h).  Output bits equal those of the calls
    on the whole device tensors.

    Build once (the device scratch and the three streams are allocated here),
    then call `run(q, k, v, o)` with pinned host bf16 tensors [B, H, N, d].
    Selection: top-n with `keep`, or the CDF threshold with `tau`.  The B*H
    heads go in `chunks` near-equal chunks, the last of them further split in
    shrinking parts down to one head (`chunk_sizes`).
    """

    def __init__(self, geom: Geometry, keep: float | None = None, tau: float | None = None, chunks: int = 8,
                 device=None, chunk_events: bool = True):
        if (keep is None) == (tau is None):
            raise ValueError("give exactly one of keep and tau")
        self.geom, self.keep, self.tau, self.chunks = geom, keep, tau, int(chunks)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.device = dev
        sz = host_query(geom, keep, tau, self.chunks)
        self.parts = chunk_sizes(geom.batch * geom.heads, self.chunks)
        assert len(self.parts) == sz.num_chunks and max(self.parts) == sz.max_chunk_heads
        self.work = torch.empty(max(256, sz.work_bytes), dtype=torch.uint8, device=dev)
        self.shape = (geom.batch, geom.heads, num_tokens(geom), geom.head_dim)
        self.h2d, self.comp, self.d2h = (torch.cuda.Stream(device=dev) for _ in range(3))
        # chunk-by-chunk ordering of consecutive runs (chunk c waits only for chunk c of the
        # last run); without, each run waits for the whole previous one
        self.num_events = 2 * sz.num_chunks if chunk_events else 0
        self.events = (ctypes.c_void_p * self.num_events)() if chunk_events else None
        if chunk_events:
            with torch.cuda.device(dev):
                _check(lib().rf2_host_events_create(self.num_events, self.events), "rf2_host_events_create")
        self._lib = lib()

    def __del__(self):
        events = getattr(self, "events", None)
        if events is not None:
            try:
                self.d2h.synchronize()
                self._lib.rf2_host_events_destroy(self.num_events, events)
            except Exception:
                pass

    def run(self, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor, o_host: torch.Tensor):
        for t in (q_host, k_host, v_host, o_host):
            if not (t.device.type == "cpu" and t.is_pinned() and t.dtype == torch.bfloat16 and t.is_contiguous()
                    and tuple(t.shape) == self.shape):
                raise ValueError(f"expected pinned contiguous host bf16 tensors of shape {self.shape}")
        _check(lib().rf2_attention_host(ctypes.byref(self.geom), float(self.keep or 0.0), float(self.tau or 0.0),
                                        self.chunks, q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
                                        o_host.data_ptr(), self.work.data_ptr(), self.work.numel(),
                                        self.h2d.cuda_stream, self.comp.cuda_stream, self.d2h.cuda_stream,
                                        self.events, self.num_events),
               "rf2_attention_host")
        return o_host

    def synchronize(self):
        self.d2h.synchronize()
