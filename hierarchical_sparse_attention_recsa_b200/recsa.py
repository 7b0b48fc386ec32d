"""Python binding of the RecSA C ABI (include/recsa.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of the method: tensors are passed as raw device pointers, the
geometry as the C struct, the stream as torch's current CUDA stream unless one
is given.  A missing or unloadable library raises at import of the first call;
there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librecsa.so")

DTYPE_F32 = 0
DTYPE_BF16 = 1
MODE_RECSA = 0
MODE_ZHA = 1
MODE_GROUP = 2
KEYS_F32 = 0
KEYS_FP8 = 1
KEYS_NVFP4 = 2
KEEP_ALL = 2**31 - 1
MAX_LEVELS = 16
TRACE_MAX_K = 64
DEVERR_APPEND_FULL = 0x1
DEVERR_WAIT_TIMEOUT = 0x2

STATUS = {
    0: "RECSA_OK",
    1: "RECSA_ERR_INVALID_GEOMETRY",
    2: "RECSA_ERR_NULL",
    3: "RECSA_ERR_MISALIGNED",
    4: "RECSA_ERR_CAPACITY",
    5: "RECSA_ERR_UNSUPPORTED",
    6: "RECSA_ERR_CUDA",
    7: "RECSA_ERR_DEVICE",
}

EXPORTS = ["recsa_status_string", "recsa_validate", "recsa_num_levels", "recsa_tree_bytes",
           "recsa_build", "recsa_append", "recsa_decode", "recsa_decode_step", "recsa_prefill",
           "recsa_prefill_workspace_bytes", "recsa_prefill_static", "recsa_trace_ints",
           "recsa_tree_error", "recsa_reload_switches"]


class RecsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class CGeometry(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("leaf_block", ctypes.c_int32),
        ("branching", ctypes.c_int32),
        ("k", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("rope_enabled", ctypes.c_int32),
        ("rope_base", ctypes.c_float),
        ("batch", ctypes.c_int32),
        ("mode", ctypes.c_int32),
        ("capacity", ctypes.c_int64),
        ("top_p", ctypes.c_float),
        ("n_ref", ctypes.c_int32),
        ("key_format", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


@dataclass
class Geometry:
    """Mirror of ``recsa_geometry`` (see include/recsa.h for each field)."""

    head_dim: int
    n_q_heads: int
    n_kv_heads: int
    leaf_block: int
    branching: int
    k: int
    window: int
    batch: int
    capacity: int
    dtype: int = DTYPE_BF16
    rope_enabled: int = 1
    rope_base: float = 1e6
    mode: int = 0          # MODE_RECSA, MODE_ZHA or MODE_GROUP
    top_p: float = 0.0     # ZHA routing mass
    n_ref: int = 1         # reference queries per pooler (ZHA mode for n_ref > 1)
    key_format: int = 0    # KEYS_F32, KEYS_FP8 or KEYS_NVFP4 (ZHA mode)

    def c(self) -> CGeometry:
        return CGeometry(self.dtype, self.head_dim, self.n_q_heads, self.n_kv_heads,
                         self.leaf_block, self.branching, self.k, self.window,
                         self.rope_enabled, self.rope_base, self.batch, self.mode,
                         self.capacity, self.top_p, self.n_ref, self.key_format, 0)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == DTYPE_BF16 else torch.float32


_lib = None


def lib() -> ctypes.CDLL:
    """Load librecsa.so (built in-tree by build_lib.build())."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"RecSA CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m hierarchical_sparse_attention_recsa_b200.build_lib)")
        import torch.cuda  # noqa: F401  (loads the CUDA runtime the library links to)
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        G = ctypes.POINTER(CGeometry)
        L.recsa_status_string.restype = ctypes.c_char_p
        L.recsa_status_string.argtypes = [ctypes.c_int]
        L.recsa_validate.argtypes = [G]
        L.recsa_num_levels.argtypes = [G, i64, ctypes.POINTER(i32)]
        L.recsa_tree_bytes.argtypes = [G, ctypes.POINTER(ctypes.c_size_t)]
        L.recsa_build.argtypes = [G, vp, vp, ctypes.POINTER(i64), vp, i64, vp, vp]
        L.recsa_append.argtypes = [G, vp, vp, vp, vp, vp, vp, i64, vp, vp]
        L.recsa_decode.argtypes = [G, vp, vp, vp, vp, vp, i32, vp, vp, vp]
        L.recsa_decode_step.argtypes = [G, vp, vp, vp, vp, vp, vp, vp, i64, vp, i32, vp, vp, vp]
        L.recsa_prefill.argtypes = [G, vp, vp, vp, vp, i64, i32, vp, vp, vp, ctypes.c_size_t,
                                    vp]
        L.recsa_prefill_workspace_bytes.argtypes = [G, i32, ctypes.POINTER(ctypes.c_size_t)]
        L.recsa_prefill_static.argtypes = [G, vp, vp, vp, vp, i64, i32, vp, vp, vp]
        L.recsa_trace_ints.argtypes = [G, ctypes.POINTER(i32)]
        L.recsa_tree_error.argtypes = [G, vp, i32, ctypes.POINTER(ctypes.c_uint32), vp]
        L.recsa_reload_switches.argtypes = []
        L.recsa_reload_switches.restype = None
        for name in EXPORTS:
            if name not in ("recsa_status_string", "recsa_reload_switches"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != 0:
        raise RecsaError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the RecSA library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def recsa_validate(geom: Geometry) -> None:
    g = geom.c()
    _check(lib().recsa_validate(ctypes.byref(g)), "recsa_validate")


def recsa_num_levels(geom: Geometry, length: int) -> int:
    g = geom.c()
    out = ctypes.c_int32()
    _check(lib().recsa_num_levels(ctypes.byref(g), length, ctypes.byref(out)), "recsa_num_levels")
    return out.value


def recsa_tree_bytes(geom: Geometry) -> int:
    g = geom.c()
    out = ctypes.c_size_t()
    _check(lib().recsa_tree_bytes(ctypes.byref(g), ctypes.byref(out)), "recsa_tree_bytes")
    return out.value


def recsa_trace_ints(geom: Geometry) -> int:
    g = geom.c()
    out = ctypes.c_int32()
    _check(lib().recsa_trace_ints(ctypes.byref(g), ctypes.byref(out)), "recsa_trace_ints")
    return out.value


def recsa_build(geom: Geometry, K: torch.Tensor, V: torch.Tensor, len_host: Sequence[int],
                pooler_r: torch.Tensor, pooler_head_stride: int, tree: torch.Tensor,
                stream=None) -> None:
    """Pool the tree over the first len_host[s] tokens of each sequence (K, V
    [batch][n_kv_heads][capacity][head_dim]); pooler_r holds the pooler's
    reference vector(s), pooler_head_stride elements apart per KV head (0: one
    vector shared by every head)."""
    g = geom.c()
    lens = (ctypes.c_int64 * geom.batch)(*[int(x) for x in len_host])
    _check(lib().recsa_build(ctypes.byref(g), _ptr(K), _ptr(V), lens, _ptr(pooler_r),
                             pooler_head_stride, _ptr(tree), _stream(stream)), "recsa_build")


def recsa_append(geom: Geometry, K: torch.Tensor, V: torch.Tensor, k_new: torch.Tensor,
                 v_new: torch.Tensor, len_dev: torch.Tensor, pooler_r: torch.Tensor,
                 pooler_head_stride: int, tree: torch.Tensor, stream=None) -> None:
    """Write one token per sequence (k_new, v_new [batch][n_kv_heads][head_dim])
    at position len_dev[s], pool the nodes it completes and advance len_dev."""
    g = geom.c()
    _check(lib().recsa_append(ctypes.byref(g), _ptr(K), _ptr(V), _ptr(k_new), _ptr(v_new),
                              _ptr(len_dev), _ptr(pooler_r), pooler_head_stride, _ptr(tree),
                              _stream(stream)), "recsa_append")


def recsa_decode(geom: Geometry, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                 tree: torch.Tensor, len_dev: torch.Tensor, n_q: int, O: torch.Tensor,
                 trace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Attend n_q queries per sequence, all at position len_dev[s] - 1."""
    g = geom.c()
    _check(lib().recsa_decode(ctypes.byref(g), _ptr(Q), _ptr(K), _ptr(V), _ptr(tree),
                              _ptr(len_dev), n_q, _ptr(O), _ptr(trace), _stream(stream)),
           "recsa_decode")


def recsa_decode_step(geom: Geometry, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                      k_new: torch.Tensor, v_new: torch.Tensor, len_dev: torch.Tensor,
                      pooler_r: torch.Tensor, pooler_head_stride: int, tree: torch.Tensor,
                      n_q: int, O: torch.Tensor, trace: Optional[torch.Tensor] = None,
                      stream=None) -> None:
    """recsa_append followed by recsa_decode, in one launch."""
    g = geom.c()
    _check(lib().recsa_decode_step(ctypes.byref(g), _ptr(Q), _ptr(K), _ptr(V), _ptr(k_new),
                                   _ptr(v_new), _ptr(len_dev), _ptr(pooler_r),
                                   pooler_head_stride, _ptr(tree), n_q, _ptr(O), _ptr(trace),
                                   _stream(stream)), "recsa_decode_step")


def recsa_prefill(geom: Geometry, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                  tree: torch.Tensor, q_start: int, n_q: int, O: torch.Tensor,
                  trace: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> None:
    """Causal prefill of queries q_start .. q_start + n_q - 1 (Q and O are
    [batch][n_q][n_q_heads][head_dim]).  ``workspace``: optional device bytes,
    at least recsa_prefill_workspace_bytes(geom, n_q); with one and bf16 data
    the exact window runs on the tensor-core window kernel (RecSA and ZHA
    modes), without one the tree kernel attends it."""
    g = geom.c()
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().recsa_prefill(ctypes.byref(g), _ptr(Q), _ptr(K), _ptr(V), _ptr(tree), q_start,
                               n_q, _ptr(O), _ptr(trace), _ptr(workspace), wbytes,
                               _stream(stream)), "recsa_prefill")


def recsa_prefill_static(geom: Geometry, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                         tree: torch.Tensor, q_start: int, n_q: int, O: torch.Tensor,
                         trace: Optional[torch.Tensor] = None, stream=None) -> None:
    """recsa_prefill with the library's fixed device scratch instead of a
    caller workspace (for callers that cannot provide device memory)."""
    g = geom.c()
    _check(lib().recsa_prefill_static(ctypes.byref(g), _ptr(Q), _ptr(K), _ptr(V), _ptr(tree),
                                      q_start, n_q, _ptr(O), _ptr(trace), _stream(stream)),
           "recsa_prefill_static")


def recsa_prefill_workspace_bytes(geom: Geometry, n_q: int) -> int:
    g = geom.c()
    out = ctypes.c_size_t()
    _check(lib().recsa_prefill_workspace_bytes(ctypes.byref(g), n_q, ctypes.byref(out)),
           "recsa_prefill_workspace_bytes")
    return out.value


def recsa_tree_error(geom: Geometry, tree: torch.Tensor, clear: bool = False,
                     stream=None) -> int:
    g = geom.c()
    out = ctypes.c_uint32()
    _check(lib().recsa_tree_error(ctypes.byref(g), _ptr(tree), int(clear), ctypes.byref(out),
                                  _stream(stream)), "recsa_tree_error")
    return out.value


def recsa_reload_switches() -> None:
    """Make changes of the RECSA_* kernel-variant environment switches take
    effect (the library reads them once, at its first call)."""
    lib().recsa_reload_switches()


def recsa_status_string(status: int) -> str:
    return lib().recsa_status_string(status).decode()
