"""Python binding of libbsa.so: frame/block-sparse video attention on B200.

Argument marshalling only.  Every computation runs in the CUDA kernels of
``libbsa.so`` (see include/bsa.h for the contract of each call); torch is
used for device memory and streams.  The library must have been built
(``python -m block_sparse_attention_lvsa_b200.build``); importing this
package raises if it is missing - there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")

BSA_OK = 0
BSA_WARN_OVER_BUDGET = 1
BSA_ERR_ARG = -1
BSA_ERR_SHAPE = -2
BSA_ERR_CUDA = -3
BSA_ERR_INDEX_RANGE = -4
BSA_ERR_TIMEOUT = -5
BSA_ERR_UNSUPPORTED = -6
BSA_ERR_WORKSPACE = -7

BSA_INDEX_LVSA_FRAMES = 1
BSA_INDEX_BLOCKS = 2
BSA_INDEX_LVSA_BLOCKS = 3
BSA_OP_BLOCKSPARSE_FWD = 1
BSA_OP_DENSE_BLOCKMASS = 2
BSA_OP_BLOCKMASS = 3

EXPORTED = ("lvsa_build_index", "lvsa_build_index_window", "attn_dense_blockmass", "attn_blockmass", "losa_select", "blocksparse_attn_fwd",
            "bsa_workspace_bytes", "bsa_get_device_status", "bsa_status_string",
            "bsa_debug_expired_wait", "bsa_version", "blocksparse_attn_fwd_noalloc")


class BsaError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {status_string(status)} ({status})")


class bsa_index(ctypes.Structure):
    """Mirror of ``struct bsa_index`` in include/bsa.h."""
    _fields_ = [
        ("kind", ctypes.c_int),
        ("T", ctypes.c_int),
        ("frames", ctypes.c_void_p),
        ("counts", ctypes.c_void_p),
        ("block", ctypes.c_int),
        ("H", ctypes.c_int),
        ("nQB", ctypes.c_int),
        ("nKB", ctypes.c_int),
        ("idx", ctypes.c_void_p),
        ("cnt", ctypes.c_void_p),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_lvsa_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, D, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float, ctypes.c_size_t
    sig = {
        "lvsa_build_index": (I, [I, I, I, I, I, P, P, P]),
        "lvsa_build_index_window": (I, [I, I, I, I, P, P, P]),
        "attn_dense_blockmass": (I, [P, P, P, I, I, I, I, F, P, P, P, P, SZ, P]),
        "attn_blockmass": (I, [P, P, P, I, I, I, F, ctypes.POINTER(bsa_index), P, P, P, P, SZ, P]),
        "losa_select": (I, [P, I, I, I, D, P, P, P]),
        "blocksparse_attn_fwd": (I, [P, P, P, I, I, I, F, ctypes.POINTER(bsa_index), P, P, P, SZ, P]),
        "bsa_workspace_bytes": (SZ, [I, I, I, I, ctypes.POINTER(bsa_index)]),
        "bsa_get_device_status": (I, [P]),
        "bsa_status_string": (ctypes.c_char_p, [I]),
        "bsa_debug_expired_wait": (I, [ctypes.c_longlong, I, P]),
        "bsa_version": (ctypes.c_char_p, []),
        "blocksparse_attn_fwd_noalloc": (I, [P, P, P, I, I, I, F, ctypes.POINTER(bsa_index), P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib():
    return _lib


def status_string(status: int) -> str:
    return _lib.bsa_status_string(int(status)).decode()


def version() -> str:
    return _lib.bsa_version().decode()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _check(call: str, rc: int, allow=(BSA_OK,)) -> int:
    if rc not in allow:
        raise BsaError(call, rc)
    return rc


def _check_qkv(q, k, v):
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors of shape [N, H, d]")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v shapes differ")


def _check_tensor(name: str, t: Optional[torch.Tensor], shape, dtype, device) -> None:
    """A caller-supplied buffer the library writes or reads by pointer: the C
    side cannot see its size, so dtype, shape, contiguity and device are
    checked here, before the call (a wrong one would mean out-of-bounds
    device accesses)."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != torch.device(device):
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _check_out(q: torch.Tensor, o: Optional[torch.Tensor], lse: Optional[torch.Tensor],
               mass: Optional[torch.Tensor] = None) -> None:
    """o like q (bf16 [N, H, d]), lse float32 [H, N], mass float32 [H, nB, nB]; same device as q."""
    N, H, _ = q.shape
    nB = math.ceil(N / 128)
    _check_tensor("o", o, q.shape, torch.bfloat16, q.device)
    _check_tensor("lse", lse, (H, N), torch.float32, q.device)
    _check_tensor("mass", mass, (H, nB, nB), torch.float32, q.device)


def _check_workspace(ws: Optional[torch.Tensor], device) -> None:
    if ws is None:
        return
    if not isinstance(ws, torch.Tensor) or not ws.is_contiguous() or ws.device != torch.device(device):
        raise ValueError(f"workspace must be a contiguous tensor on {device}")


# ----------------------------------------------------------------- calls ---
def lvsa_build_index(T: int, T_per: int, W: int, C: int, step: int,
                     frames: Optional[torch.Tensor] = None, counts: Optional[torch.Tensor] = None,
                     device=None, stream=None) -> Tuple[torch.Tensor, torch.Tensor, bool]:
    """A(t) for every frame at ``step``: (frames [T,T] int32, counts [T] int32, over_budget)."""
    dev = device if device is not None else (frames.device if frames is not None else "cuda")
    _check_tensor("frames", frames, (T, T), torch.int32, dev)
    _check_tensor("counts", counts, (T,), torch.int32, dev)
    if frames is None:
        frames = torch.empty((T, T), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty((T,), dtype=torch.int32, device=dev)
    rc = _lib.lvsa_build_index(T, T_per, W, C, step, _ptr(frames), _ptr(counts), _stream(stream))
    _check("lvsa_build_index", rc, (BSA_OK, BSA_WARN_OVER_BUDGET))
    return frames, counts, rc == BSA_WARN_OVER_BUDGET


def lvsa_build_index_window(T: int, T_per: int, W: int, step: int,
                            frames: Optional[torch.Tensor] = None, counts: Optional[torch.Tensor] = None,
                            device=None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """A(t) under the fixed-window reading (W non-anchor frames): (frames [T,T] int32, counts [T] int32)."""
    dev = device if device is not None else (frames.device if frames is not None else "cuda")
    _check_tensor("frames", frames, (T, T), torch.int32, dev)
    _check_tensor("counts", counts, (T,), torch.int32, dev)
    if frames is None:
        frames = torch.empty((T, T), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty((T,), dtype=torch.int32, device=dev)
    rc = _lib.lvsa_build_index_window(T, T_per, W, step, _ptr(frames), _ptr(counts), _stream(stream))
    _check("lvsa_build_index_window", rc)
    return frames, counts


def lvsa_index(T: int, frames: torch.Tensor, counts: torch.Tensor) -> bsa_index:
    """Index of kind BSA_INDEX_LVSA_FRAMES over device frames [T, T] and counts [T] (int32)."""
    _check_tensor("frames", frames, (T, T), torch.int32, frames.device)
    _check_tensor("counts", counts, (T,), torch.int32, frames.device)
    ix = bsa_index()
    ix.kind = BSA_INDEX_LVSA_FRAMES
    ix.T = T
    ix.frames = frames.data_ptr()
    ix.counts = counts.data_ptr()
    ix._tensors = (frames, counts)         # the struct holds raw pointers: keep the tensors alive with it
    return ix


def block_index(idx: torch.Tensor, cnt: torch.Tensor, block: int = 128) -> bsa_index:
    """Index of kind BSA_INDEX_BLOCKS over device idx [H, nQB, nKB] and cnt [H, nQB] (int32)."""
    if not isinstance(idx, torch.Tensor) or idx.dim() != 3:
        raise ValueError("idx must be an int32 tensor [H, nQB, nKB]")
    H, nQB, nKB = idx.shape
    _check_tensor("idx", idx, (H, nQB, nKB), torch.int32, idx.device)
    _check_tensor("cnt", cnt, (H, nQB), torch.int32, idx.device)
    ix = bsa_index()
    ix.kind = BSA_INDEX_BLOCKS
    ix.block, ix.H, ix.nQB, ix.nKB = block, H, nQB, nKB
    ix.idx = idx.data_ptr()
    ix.cnt = cnt.data_ptr()
    ix._tensors = (idx, cnt)               # the struct holds raw pointers: keep the tensors alive with it
    return ix


def lvsa_block_index(T: int, frames: torch.Tensor, counts: torch.Tensor, idx: torch.Tensor, cnt: torch.Tensor,
                     block: int = 128) -> bsa_index:
    """Intersection index: LVSA frame sets (frames, counts) within per-head key-block lists (idx, cnt)."""
    ix = block_index(idx, cnt, block)
    ix.kind = BSA_INDEX_LVSA_BLOCKS
    ix.T = T
    ix.frames = frames.data_ptr()
    ix.counts = counts.data_ptr()
    ix._tensors = (frames, counts, idx, cnt)
    return ix


def workspace_bytes(op: int, N: int, H: int, d: int, index: Optional[bsa_index] = None) -> int:
    n = _lib.bsa_workspace_bytes(op, N, H, d, ctypes.byref(index) if index is not None else None)
    if n == ctypes.c_size_t(-1).value:
        raise BsaError("bsa_workspace_bytes", BSA_ERR_ARG)
    return int(n)


def blocksparse_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, index: bsa_index,
                         scale: Optional[float] = None, o: Optional[torch.Tensor] = None,
                         lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                         stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Masked attention restricted to ``index``; returns (o [N,H,d] bf16, lse [H,N] f32)."""
    _check_qkv(q, k, v)
    _check_out(q, o, lse)
    _check_workspace(workspace, q.device)
    N, H, d = q.shape
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, N), dtype=torch.float32, device=q.device)
    need = workspace_bytes(BSA_OP_BLOCKSPARSE_FWD, N, H, d, index)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.blocksparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), N, H, d, float(scale), ctypes.byref(index),
                                   _ptr(o), _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream))
    _check("blocksparse_attn_fwd", rc)
    return o, lse


def blocksparse_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, index: bsa_index,
                                 o: torch.Tensor, lse: torch.Tensor, scale: Optional[float] = None,
                                 stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """blocksparse_attn_fwd without a workspace: the library's static scratch array is
    used instead, so the call allocates nothing (o and lse are the caller's)."""
    if o is None or lse is None:
        raise ValueError("blocksparse_attn_fwd_noalloc writes into the caller's o and lse")
    _check_qkv(q, k, v)
    _check_out(q, o, lse)
    N, H, d = q.shape
    if scale is None:
        scale = d ** -0.5
    rc = _lib.blocksparse_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), N, H, d, float(scale), ctypes.byref(index),
                                           _ptr(o), _ptr(lse), _stream(stream))
    _check("blocksparse_attn_fwd_noalloc", rc)
    return o, lse


def attn_dense_blockmass(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int = 128,
                         scale: Optional[float] = None, o=None, lse=None, mass=None,
                         workspace: Optional[torch.Tensor] = None, stream=None):
    """Dense attention plus LoSA block mass; returns (o, lse, mass [H, nB, nB] f32).

    ``workspace`` (uint8 CUDA tensor, 256-byte aligned) holds at least one
    head's log partial sums, nB * N * 4 bytes; more heads per pass when larger.
    When omitted, ``workspace_bytes(BSA_OP_DENSE_BLOCKMASS, ...)`` bytes are allocated.
    """
    _check_qkv(q, k, v)
    _check_out(q, o, lse, mass)
    _check_workspace(workspace, q.device)
    N, H, d = q.shape
    nB = math.ceil(N / 128)
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, N), dtype=torch.float32, device=q.device)
    if mass is None:
        mass = torch.empty((H, nB, nB), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(BSA_OP_DENSE_BLOCKMASS, N, H, d), dtype=torch.uint8,
                                device=q.device)
    rc = _lib.attn_dense_blockmass(_ptr(q), _ptr(k), _ptr(v), N, H, d, block, float(scale),
                                   _ptr(o), _ptr(lse), _ptr(mass), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check("attn_dense_blockmass", rc)
    return o, lse, mass


def attn_blockmass(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, index: bsa_index,
                   scale: Optional[float] = None, o=None, lse=None, mass=None,
                   workspace: Optional[torch.Tensor] = None, stream=None):
    """Attention restricted to ``index`` plus its LoSA block mass; returns (o, lse, mass [H, nB, nB] f32)."""
    _check_qkv(q, k, v)
    _check_out(q, o, lse, mass)
    _check_workspace(workspace, q.device)
    N, H, d = q.shape
    nB = math.ceil(N / 128)
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, N), dtype=torch.float32, device=q.device)
    if mass is None:
        mass = torch.empty((H, nB, nB), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(BSA_OP_BLOCKMASS, N, H, d, index), dtype=torch.uint8,
                                device=q.device)
    rc = _lib.attn_blockmass(_ptr(q), _ptr(k), _ptr(v), N, H, d, float(scale), ctypes.byref(index),
                             _ptr(o), _ptr(lse), _ptr(mass), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_blockmass", rc)
    return o, lse, mass


def losa_select(mass: torch.Tensor, tau: float = 0.99, idx=None, cnt=None, stream=None):
    """Minimal tau-mass key-block sets; returns (idx [H,nQB,nKB] int32 (-1 padded), cnt [H,nQB] int32)."""
    if mass.dtype != torch.float32 or not mass.is_cuda or not mass.is_contiguous() or mass.dim() != 3:
        raise ValueError("mass must be a contiguous float32 CUDA tensor [H, nQB, nKB]")
    H, nQB, nKB = mass.shape
    _check_tensor("idx", idx, (H, nQB, nKB), torch.int32, mass.device)
    _check_tensor("cnt", cnt, (H, nQB), torch.int32, mass.device)
    if idx is None:
        idx = torch.empty((H, nQB, nKB), dtype=torch.int32, device=mass.device)
    if cnt is None:
        cnt = torch.empty((H, nQB), dtype=torch.int32, device=mass.device)
    rc = _lib.losa_select(_ptr(mass), H, nQB, nKB, float(tau), _ptr(idx), _ptr(cnt), _stream(stream))
    _check("losa_select", rc)
    return idx, cnt


def get_device_status(stream=None) -> int:
    """Synchronise the stream and return + clear the device status word."""
    return int(_lib.bsa_get_device_status(_stream(stream)))


def debug_expired_wait(limit_ns: int, form: int = 0, stream=None) -> int:
    """Enqueue the expired-wait diagnostic (form 0: one thread waits, 1: the whole warp)."""
    return int(_lib.bsa_debug_expired_wait(int(limit_ns), int(form), _stream(stream)))


def lvsa_workspace_views(workspace: torch.Tensor, N: int, T: int):
    """Views of the LVSA workspace written by blocksparse_attn_fwd (layout of bsa_lib.cu).

    Returns (fbits [T, TW] int32 bit rows, tile_cnt [nB], tile_idx [nB, nB], tile_flag [nB, nB] uint8);
    row qt of tile_idx/tile_flag is valid in its first tile_cnt[qt] entries.
    """
    def up(x, a=256):
        return (x + a - 1) // a * a
    nB = math.ceil(N / 128)
    TW = (T + 31) // 32
    o_cnt = up(T * TW * 4)
    o_idx = up(o_cnt + nB * 4)
    o_flag = up(o_idx + nB * nB * 4)
    ws = workspace.view(torch.uint8)
    fbits = ws[:T * TW * 4].view(torch.int32).view(T, TW)
    cnt = ws[o_cnt:o_cnt + nB * 4].view(torch.int32)
    idx = ws[o_idx:o_idx + nB * nB * 4].view(torch.int32).view(nB, nB)
    flag = ws[o_flag:o_flag + nB * nB].view(nB, nB)
    return fbits, cnt, idx, flag
