"""DeepSeek-V4 hybrid compressed attention (CSA / HCA) on NVIDIA B200.

Thin Python binding over the C ABI of libcsa_b200.so (include/csa.h).  The functions
below only check tensor metadata and marshal pointers, sizes and the current CUDA
stream; every step of the layer runs in the library's sm_100a kernels.  If the library
is missing or cannot be loaded, every call raises: there is no other code path.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = ["csa_compress", "csa_compress_append", "csa_compress_state_bytes",
           "csa_compress_state", "csa_rope_rows", "csa_index_topk", "csa_attend", "hca_attend",
           "csa_index_topk_workspace_bytes", "csa_attend_workspace_bytes", "csa_out_proj",
           "csa_out_proj_workspace_bytes", "csa_kv_gate_proj", "library_path",
           "load_library", "launch_count", "device_status", "debug_withhold_attention_loads", "CsaError", "CSA_F32", "CSA_BF16"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libcsa_b200.so")
CSA_F32, CSA_BF16 = 0, 1
_lib = None


class CsaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__("%s returned %d: %s" % (fn, code, msg))
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libcsa_b200.so (built by __graft_entry__.build() / build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError("libcsa_b200.so is not built (%s); run `python "
                          "sparse_attention_14_b200/build.py`" % _LIB_PATH)
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    lib.csa_compress.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, ctypes.c_int, vp]
    lib.csa_compress_append.argtypes = [vp, vp, i64, i64, vp, vp, i64, i64, i64, i64, i32, i32,
                                        i32, ctypes.c_int, vp]
    lib.csa_compress_state_bytes.argtypes = [i64, i32, i32, i32, ctypes.c_int]
    lib.csa_compress_state_bytes.restype = sz
    lib.csa_rope_rows.argtypes = [vp, vp, i64, i32, i32, ctypes.c_double, i64, i64, i64, i64,
                                  ctypes.c_int, vp]
    lib.csa_index_topk.argtypes = [vp, vp, vp, i64, i64, i64, i64, i32, i32, i32, i32, vp, vp, vp,
                                   sz, ctypes.c_int, vp]
    lib.csa_index_topk_workspace_bytes.argtypes = [i64, i64, i64, i64, i32, i32, i32, i32,
                                                   ctypes.c_int]
    lib.csa_index_topk_workspace_bytes.restype = sz
    lib.csa_attend.argtypes = [vp, vp, i64, i64, vp, i64, vp, i32, vp, vp, i64, i64, i64, i32, i32,
                               i32, ctypes.c_double, i32, i32, ctypes.c_float, vp, sz,
                               ctypes.c_int, vp]
    lib.hca_attend.argtypes = [vp, vp, i64, i64, vp, i64, vp, vp, i64, i64, i64, i32, i32, i32,
                               ctypes.c_double, i32, i32, ctypes.c_float, vp, sz, ctypes.c_int, vp]
    lib.csa_attend_workspace_bytes.argtypes = [i32, i64, i64, i64, i64, i32, i32, i32,
                                               ctypes.c_int]
    lib.csa_attend_workspace_bytes.restype = sz
    for f in ("csa_compress", "csa_compress_append", "csa_rope_rows", "csa_index_topk", "csa_attend",
              "hca_attend"):
        getattr(lib, f).restype = ctypes.c_int
    lib.csa_last_error.restype = ctypes.c_char_p
    lib.csa_version.restype = ctypes.c_char_p
    lib.csa_launch_count.restype = ctypes.c_uint64
    lib.csa_device_status.restype = ctypes.c_uint32
    lib.csa_out_proj.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, vp, sz, ctypes.c_int, vp]
    lib.csa_out_proj.restype = ctypes.c_int
    lib.csa_out_proj_workspace_bytes.argtypes = [i64, i32, i32]
    lib.csa_out_proj_workspace_bytes.restype = sz
    lib.csa_kv_gate_proj.argtypes = [vp, vp, vp, vp, ctypes.c_float, vp, vp, i64, i32, i32, ctypes.c_int, vp]
    lib.csa_kv_gate_proj.restype = ctypes.c_int
    lib.csa_debug_withhold_attention_loads.argtypes = [ctypes.c_int32]
    lib.csa_debug_withhold_attention_loads.restype = ctypes.c_int
    _lib = lib
    return lib


def launch_count() -> int:
    """Kernels the library has enqueued in this process."""
    return int(load_library().csa_launch_count())


def device_status() -> int:
    """Nonzero if a kernel gave up on a bounded wait since the last call (synchronises)."""
    return int(load_library().csa_device_status())


def debug_withhold_attention_loads(on: bool) -> None:
    """Test hook: make the tensor-core attention's bounded waits run out (see csa.h)."""
    _call("csa_debug_withhold_attention_loads", int(bool(on)))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CSA_F32
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    raise TypeError("unsupported dtype %s (float32 or bfloat16)" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _call(fn: str, *args):
    lib = load_library()
    rc = getattr(lib, fn)(*args)
    if rc != 0:
        raise CsaError(fn, rc, lib.csa_last_error().decode())


def _ws(nbytes: int, device, workspace: Optional[torch.Tensor]):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def csa_compress(kv: torch.Tensor, gate: torch.Tensor, ratio: int, overlap: bool,
                 pool: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """kv, gate [B,S,D] -> pool [B, S//ratio, D] (see include/csa.h)."""
    B, S, D = kv.shape
    if gate.shape != kv.shape or gate.dtype != kv.dtype:
        raise ValueError("gate must match kv in shape and dtype")
    P = S // ratio
    if pool is None:
        pool = torch.empty((B, P, D), dtype=kv.dtype, device=kv.device)
    _call("csa_compress", _ptr(kv), _ptr(gate), _ptr(pool), B, S, D, ratio, int(bool(overlap)),
          _dtype_code(kv), _stream(stream))
    return pool


def _rows_ptr(t: torch.Tensor, D: int):
    """Pointer and sequence stride (in rows) of a [B, n, D] tensor whose rows are dense
    (a slice of a larger cache along n is fine)."""
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    B, n, d = t.shape
    if d != D or t.stride(2) != 1 or (n > 1 and t.stride(1) != D):
        raise ValueError("rows must be dense [.., D] vectors with D=%d" % D)
    if B > 1 and t.stride(0) % D != 0:
        raise ValueError("sequence stride must be a whole number of rows")
    return ctypes.c_void_p(t.data_ptr()), (t.stride(0) // D if B > 1 else n)


def csa_compress_state_bytes(B: int, D: int, ratio: int, overlap: bool,
                             dtype=torch.bfloat16) -> int:
    code = CSA_F32 if dtype == torch.float32 else CSA_BF16
    return int(load_library().csa_compress_state_bytes(B, D, ratio, int(bool(overlap)), code))


def csa_compress_state(B: int, D: int, ratio: int, overlap: bool, dtype=torch.bfloat16,
                       device="cuda") -> torch.Tensor:
    """A zeroed state [B, 2, (1+overlap)*ratio, D] for csa_compress_append."""
    L = (1 + int(bool(overlap))) * ratio
    return torch.zeros((B, 2, L, D), dtype=dtype, device=device)


def csa_compress_append(kv_new: torch.Tensor, gate_new: torch.Tensor, state: torch.Tensor,
                        pos0: int, ratio: int, overlap: bool,
                        pool: Optional[torch.Tensor] = None, stream=None) -> Optional[torch.Tensor]:
    """Append rows kv_new, gate_new [B, n, D] at positions pos0.. to the compressor state
    and write the entries that close among them into pool [B, cap, D] (see include/csa.h)."""
    B, n, D = kv_new.shape
    if gate_new.shape != kv_new.shape or gate_new.dtype != kv_new.dtype:
        raise ValueError("gate_new must match kv_new in shape and dtype")
    L = (1 + int(bool(overlap))) * ratio
    if tuple(state.shape) != (B, 2, L, D) or state.dtype != kv_new.dtype:
        raise ValueError("state must be [B, 2, %d, D] of the rows' dtype" % L)
    if pool is not None and (pool.dim() != 3 or pool.shape[0] != B or pool.shape[2] != D
                             or pool.dtype != kv_new.dtype):
        raise ValueError("pool must be [B, cap, D] of the rows' dtype")
    kp, ks = _rows_ptr(kv_new, D)
    gp, gs = _rows_ptr(gate_new, D)
    _call("csa_compress_append", kp, gp, ks, gs, _ptr(state), _ptr(pool),
          0 if pool is None else pool.shape[1], B, n, pos0, D, ratio, int(bool(overlap)),
          _dtype_code(kv_new), _stream(stream))
    return pool


def csa_rope_rows(x: torch.Tensor, pos0: int, group: int, period: int, step: int, rope_dim: int,
                  rope_base: float, out: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """Rotate the last rope_dim channels of every row of x [..., D] (rows in memory order)
    at position pos0 + ((r // group) % period) * step (see include/csa.h).  For indexer
    queries q_I [B,S_q,H_I,d_I]: group=H_I, period=S_q, step=1, pos0=q_pos0; for pooled
    index keys k_I [B,P,d_I]: group=1, period=P, step=ratio, pos0=0."""
    D = x.shape[-1]
    if out is None:
        out = torch.empty_like(x)
    if out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("out must match x in shape and dtype")
    _call("csa_rope_rows", _ptr(x), _ptr(out), x.numel() // D if D else 0, D, rope_dim,
          float(rope_base), pos0, group, period, step, _dtype_code(x), _stream(stream))
    return out


def csa_index_topk_workspace_bytes(B, S_q, q_pos0, P, H_I, d_I, ratio, topk,
                                   dtype=torch.bfloat16) -> int:
    code = CSA_F32 if dtype == torch.float32 else CSA_BF16
    return int(load_library().csa_index_topk_workspace_bytes(B, S_q, q_pos0, P, H_I, d_I, ratio,
                                                             topk, code))


def csa_index_topk(q_I: torch.Tensor, w: torch.Tensor, k_I: torch.Tensor, q_pos0: int, ratio: int,
                   topk: int, idx: Optional[torch.Tensor] = None, want_scores: bool = False,
                   workspace: Optional[torch.Tensor] = None, stream=None):
    """q_I [B,S_q,H_I,d_I], w [B,S_q,H_I], k_I [B,P,d_I] -> idx int32 [B,S_q,topk]
    (and the kept scores fp32 [B,S_q,topk] when want_scores)."""
    B, S_q, H_I, d_I = q_I.shape
    P = k_I.shape[1]
    if idx is None:
        idx = torch.empty((B, S_q, topk), dtype=torch.int32, device=q_I.device)
    scores = torch.empty((B, S_q, topk), dtype=torch.float32, device=q_I.device) if want_scores else None
    ws, wsb = _ws(csa_index_topk_workspace_bytes(B, S_q, q_pos0, P, H_I, d_I, ratio, topk,
                                                 q_I.dtype), q_I.device, workspace)
    _call("csa_index_topk", _ptr(q_I), _ptr(w), _ptr(k_I), B, S_q, q_pos0, P, H_I, d_I, ratio, topk,
          _ptr(idx), _ptr(scores), _ptr(ws), wsb, _dtype_code(q_I), _stream(stream))
    return (idx, scores) if want_scores else idx


def csa_attend_workspace_bytes(mode: int, B, S_q, S_kv, P, H, D, topk, dtype=torch.bfloat16) -> int:
    code = CSA_F32 if dtype == torch.float32 else CSA_BF16
    return int(load_library().csa_attend_workspace_bytes(mode, B, S_q, S_kv, P, H, D, topk, code))


def csa_attend(q, kv, kv_pos0: int, pool, idx, sink, q_pos0: int, rope_dim: int, rope_base: float,
               window: int, ratio: int, scale: Optional[float] = None, out=None, workspace=None,
               stream=None) -> torch.Tensor:
    """CSA attention; q [B,S_q,H,D], kv [B,S_kv,D], pool [B,P,D], idx int32 [B,S_q,k],
    sink fp32 [H] -> out [B,S_q,H,D]."""
    B, S_q, H, D = q.shape
    S_kv, P, topk = kv.shape[1], pool.shape[1], idx.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    ws, wsb = _ws(csa_attend_workspace_bytes(0, B, S_q, S_kv, P, H, D, topk, q.dtype), q.device,
                  workspace)
    _call("csa_attend", _ptr(q), _ptr(kv), S_kv, kv_pos0, _ptr(pool), P, _ptr(idx), topk, _ptr(sink),
          _ptr(out), B, S_q, q_pos0, H, D, rope_dim, rope_base, window, ratio, scale, _ptr(ws), wsb,
          _dtype_code(q), _stream(stream))
    return out


def hca_attend(q, kv, kv_pos0: int, pool, sink, q_pos0: int, rope_dim: int, rope_base: float,
               window: int, ratio: int, scale: Optional[float] = None, out=None, workspace=None,
               stream=None) -> torch.Tensor:
    """HCA attention over every visible entry (pool None or P == 0: sliding-only layer)."""
    B, S_q, H, D = q.shape
    S_kv = kv.shape[1]
    P = 0 if pool is None else pool.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    ws, wsb = _ws(csa_attend_workspace_bytes(1, B, S_q, S_kv, P, H, D, 0, q.dtype), q.device,
                  workspace)
    _call("hca_attend", _ptr(q), _ptr(kv), S_kv, kv_pos0, _ptr(pool) if P else None, P, _ptr(sink),
          _ptr(out), B, S_q, q_pos0, H, D, rope_dim, rope_base, window, ratio, scale, _ptr(ws), wsb,
          _dtype_code(q), _stream(stream))
    return out


def csa_out_proj_workspace_bytes(M: int, G: int, r: int) -> int:
    return int(load_library().csa_out_proj_workspace_bytes(M, G, r))


def csa_out_proj(o: torch.Tensor, w_a: torch.Tensor, w_b: torch.Tensor, y=None, workspace=None,
                 stream=None) -> torch.Tensor:
    """Grouped low-rank output projection: o [..., H, D] (bf16), w_a [G, r, (H/G)*D],
    w_b [hidden, G*r] -> y [..., hidden] (see include/csa.h)."""
    H, D = o.shape[-2], o.shape[-1]
    G, r, per = w_a.shape
    hidden = w_b.shape[0]
    M = o.numel() // (H * D) if H * D else 0
    if per != (H // G) * D or w_b.shape[1] != G * r:
        raise ValueError("w_a must be [G, r, (H/G)*D] and w_b [hidden, G*r]")
    if not (o.dtype == w_a.dtype == w_b.dtype):
        raise ValueError("o, w_a and w_b must share a dtype")
    if y is None:
        y = torch.empty(o.shape[:-2] + (hidden,), dtype=o.dtype, device=o.device)
    ws, wsb = _ws(csa_out_proj_workspace_bytes(M, G, r), o.device, workspace)
    _call("csa_out_proj", _ptr(o), _ptr(w_a), _ptr(w_b), _ptr(y), M, H, D, G, r, hidden, _ptr(ws),
          wsb, _dtype_code(o), _stream(stream))
    return y


def csa_kv_gate_proj(x: torch.Tensor, w_kv: torch.Tensor, w_gate: torch.Tensor,
                     kv_norm_w: torch.Tensor, eps: float = 1e-6, kv=None, gate=None, stream=None):
    """The compressor's input projections: x [..., hidden] (bf16), w_kv / w_gate [D, hidden],
    kv_norm_w [D] -> (kv, gate) [..., D] with kv RMS-normalised (see include/csa.h)."""
    hidden = x.shape[-1]
    D = w_kv.shape[0]
    M = x.numel() // hidden if hidden else 0
    if w_kv.shape != (D, hidden) or w_gate.shape != (D, hidden) or kv_norm_w.shape != (D,):
        raise ValueError("w_kv, w_gate must be [D, hidden] and kv_norm_w [D]")
    if not (x.dtype == w_kv.dtype == w_gate.dtype == kv_norm_w.dtype):
        raise ValueError("x, weights and kv_norm_w must share a dtype")
    if kv is None:
        kv = torch.empty(x.shape[:-1] + (D,), dtype=x.dtype, device=x.device)
    if gate is None:
        gate = torch.empty(x.shape[:-1] + (D,), dtype=x.dtype, device=x.device)
    _call("csa_kv_gate_proj", _ptr(x), _ptr(w_kv), _ptr(w_gate), _ptr(kv_norm_w), float(eps),
          _ptr(kv), _ptr(gate), M, hidden, D, _dtype_code(x), _stream(stream))
    return kv, gate
