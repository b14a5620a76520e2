"""ctypes binding of libjssa.so (include/jssa.h).

Argument marshalling only: torch tensors are passed as raw device pointers together
with the current CUDA stream; every step of the decode path runs in the library's
CUDA kernels.  There is no CPU fallback: if the library is missing or the device is
not a CUDA GPU, calls fail loudly.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjssa.so")

MODE_GQA, MODE_MLA = 0, 1
OUT_F32, OUT_BF16 = 0, 1
KP_BF16, KP_FP8_E4M3 = 0, 1

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape or mode", 3: "workspace missing, misaligned or too small",
          4: "CUDA error", 5: "device-side check failed", 6: "bounded wait timed out",
          7: "beyond the built-in scratch of the allocation-free entry point"}
DEV_BAD_SEQ_LEN, DEV_BAD_INDEX, DEV_BAD_NSEL, DEV_TIMEOUT = 1, 2, 4, 8

EXPORTS = ("jssa_status_string", "jssa_version", "jssa_workspace_size", "jssa_project_keys", "jssa_score",
           "jssa_topk", "jssa_topk_noalloc", "jssa_select", "jssa_indexed_attn", "jssa_decode_step",
           "jssa_dense_decode", "jssa_gather_size", "jssa_gather_decode", "jssa_calibrate_workspace_size",
           "jssa_calibrate", "jssa_vote_select",
           "jssa_workspace_init", "jssa_read_device_status", "jssa_test_withhold_copy", "jssa_append_kv",
           "jssa_copy_mapped")


class JssaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code})")
        self.code = code


class Layout(C.Structure):
    _fields_ = [("mode", C.c_int32), ("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32),
                ("d_k", C.c_int32), ("d_v", C.c_int32), ("r", C.c_int32), ("out_dtype", C.c_int32),
                ("T_cap", C.c_int64), ("k_stride", C.c_int64 * 3), ("v_stride", C.c_int64 * 3),
                ("kp_stride", C.c_int64 * 3), ("kp_dtype", C.c_int32)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libjssa.so (once) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m token_level_sparse_jssa_b200.build` "
                           "(the CUDA path has no fallback)")
    lib = C.CDLL(path)
    vp, i32, i64, f32, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
    LP = C.POINTER(Layout)
    sig = {
        "jssa_status_string": (C.c_char_p, [C.c_int]),
        "jssa_version": (i32, []),
        "jssa_workspace_size": (C.c_int, [LP, i32, i32, C.POINTER(sz)]),
        "jssa_project_keys": (C.c_int, [LP, vp, vp, vp, vp, vp, i64, vp]),
        "jssa_score": (C.c_int, [LP, vp, vp, vp, vp, i32, vp, vp, sz, vp]),
        "jssa_topk": (C.c_int, [LP, vp, vp, i32, i32, vp, vp, vp, sz, vp]),
        "jssa_topk_noalloc": (C.c_int, [LP, vp, vp, i32, i32, vp, vp, vp]),
        "jssa_select": (C.c_int, [LP, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, sz, vp]),
        "jssa_indexed_attn": (C.c_int, [LP, vp, vp, vp, vp, i32, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "jssa_decode_step": (C.c_int, [LP, vp, vp, vp, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp, vp, vp, sz, vp]),
        "jssa_gather_size": (C.c_int, [LP, i32, i32, C.POINTER(sz)]),
        "jssa_gather_decode": (C.c_int, [LP, vp, vp, vp, vp, i32, vp, vp, i32, f32, vp, vp, vp, sz, vp, sz, vp]),
        "jssa_dense_decode": (C.c_int, [LP, vp, vp, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "jssa_calibrate_workspace_size": (C.c_int, [LP, C.POINTER(sz)]),
        "jssa_calibrate": (C.c_int, [LP, vp, vp, i64, vp, vp, vp, sz, vp]),
        "jssa_vote_select": (C.c_int, [LP, vp, vp, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp, sz, vp]),
        "jssa_workspace_init": (C.c_int, [vp, sz, vp]),
        "jssa_read_device_status": (C.c_int, [vp, sz, C.POINTER(i32), vp]),
        "jssa_test_withhold_copy": (C.c_int, [vp, sz, i32, vp]),
        "jssa_append_kv": (C.c_int, [LP, vp, vp, vp, vp, vp, vp]),
        "jssa_copy_mapped": (C.c_int, [vp, vp, C.c_size_t, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(t):
    """Device pointer of a cache tensor (strides are described by the layout)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return t
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    return t.data_ptr()


def _c(t):
    """Device pointer of a tensor the C ABI reads as densely packed (Q, O, P, idx, ...)."""
    if isinstance(t, torch.Tensor) and not t.is_contiguous():
        raise ValueError(f"contiguous tensor expected, got strides {t.stride()} for shape {tuple(t.shape)}")
    return _p(t)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _check(fn: str, code: int):
    if code != 0:
        raise JssaError(fn, code)


def _ws(ws):
    return (ws.data_ptr(), ws.numel() * ws.element_size()) if ws is not None else (None, 0)


# --------------------------------------------------------------------------- layout
def make_layout(K: torch.Tensor, V: torch.Tensor, Kp: torch.Tensor, Hq: int, r: int, mode: int = MODE_GQA,
                out_dtype: int = OUT_F32) -> Layout:
    """Layout from 4-D caches K [B, Hkv, T_cap, d_k], V [B, Hkv, T_cap, d_v] and
    Kp [B, Hkv, T_cap, r] (any strides with a contiguous last dimension).  A Kp of
    dtype bfloat16 is a bf16 cache; float8_e4m3fn or uint8 (the raw codes) an E4M3 one."""
    B, Hkv, T_cap, d_k = K.shape
    L = Layout()
    L.mode, L.B, L.Hq, L.Hkv = mode, B, Hq, Hkv
    L.d_k, L.d_v, L.r, L.out_dtype = d_k, V.shape[-1], r, out_dtype
    L.T_cap = T_cap
    if Kp.dtype == torch.bfloat16:
        L.kp_dtype = KP_BF16
    elif Kp.dtype in (torch.float8_e4m3fn, torch.uint8):
        L.kp_dtype = KP_FP8_E4M3
    else:
        raise TypeError(f"Kp must be bfloat16, float8_e4m3fn or uint8, not {Kp.dtype}")
    for i in range(3):
        L.k_stride[i] = K.stride(i)
        L.v_stride[i] = V.stride(i)
        L.kp_stride[i] = Kp.stride(i)
    return L


# --------------------------------------------------------------------------- entry points
def status_string(code: int) -> str:
    return load().jssa_status_string(code).decode()


def version() -> int:
    return load().jssa_version()


def workspace_size(L: Layout, k: int, window: int = 0) -> int:
    n = C.c_size_t(0)
    _check("jssa_workspace_size", load().jssa_workspace_size(C.byref(L), k, window, C.byref(n)))
    return n.value


def alloc_workspace(L: Layout, k: int, window: int = 0, device=None) -> torch.Tensor:
    """Caller-side allocation of the workspace (torch owns the memory), status word zeroed."""
    n = workspace_size(L, k, window)
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    workspace_init(ws)
    return ws


def append_kv(L, K_new, V_new, K, V, t_pos, stream=None):
    """Write the newest K (and V) row of every (sequence, KV head) into row t_pos[b]."""
    _check("jssa_append_kv", load().jssa_append_kv(C.byref(L), _c(K_new), _c(V_new), _p(K), _p(V), _c(t_pos),
                                                   _stream(stream)))


def copy_mapped(dst, src, nbytes=None, stream=None):
    """Copy nbytes (default: all of src) between device memory and pinned host memory with a
    kernel (jssa_copy_mapped); dst and src are contiguous tensors, either on the device or
    pinned on the host."""
    for t in (dst, src):
        if not t.is_contiguous():
            raise ValueError("contiguous tensors expected")
    n = src.numel() * src.element_size() if nbytes is None else int(nbytes)
    if n > min(src.numel() * src.element_size(), dst.numel() * dst.element_size()):
        raise ValueError("nbytes exceeds a tensor")
    _check("jssa_copy_mapped", load().jssa_copy_mapped(dst.data_ptr(), src.data_ptr(), n, _stream(stream)))


def project_keys(L, K, P, Kp, n_tokens: int, t_begin=None, seq_lens=None, stream=None):
    _check("jssa_project_keys", load().jssa_project_keys(C.byref(L), _p(K), _c(P), _p(Kp), _c(t_begin),
                                                         _c(seq_lens), n_tokens, _stream(stream)))


def score(L, Q, P, Kp, seq_lens, window: int, scores, ws, stream=None):
    w, n = _ws(ws)
    _check("jssa_score", load().jssa_score(C.byref(L), _c(Q), _c(P), _p(Kp), _c(seq_lens), window, _c(scores),
                                           w, n, _stream(stream)))


def topk(L, scores, seq_lens, k: int, window: int, idx, n_sel, ws=None, stream=None):
    w, n = _ws(ws)
    _check("jssa_topk", load().jssa_topk(C.byref(L), _c(scores), _c(seq_lens), k, window, _c(idx), _c(n_sel),
                                         w, n, _stream(stream)))


def topk_noalloc(L, scores, seq_lens, k: int, window: int, idx, n_sel, stream=None):
    """Top-k without a workspace: the library's built-in scratch (up to 256 rows) is used;
    for callers that cannot allocate device memory.  Overlapping calls race."""
    _check("jssa_topk_noalloc", load().jssa_topk_noalloc(C.byref(L), _c(scores), _c(seq_lens), k, window, _c(idx),
                                                         _c(n_sel), _stream(stream)))


def indexed_attn(L, Q, K, V, idx, k: int, n_sel, seq_lens, window: int, sm_scale: float, O, lse, ws, stream=None):
    w, n = _ws(ws)
    _check("jssa_indexed_attn", load().jssa_indexed_attn(C.byref(L), _c(Q), _p(K), _p(V), _c(idx), k, _c(n_sel),
                                                         _c(seq_lens), window, sm_scale, _c(O), _c(lse), w, n,
                                                         _stream(stream)))


def select(L, Q, K, Kp, P, seq_lens, n_new: int, k: int, window: int, idx, n_sel, ws, stream=None):
    w, n = _ws(ws)
    _check("jssa_select", load().jssa_select(C.byref(L), _c(Q), _p(K), _p(Kp), _c(P), _c(seq_lens), n_new, k,
                                             window, _c(idx), _c(n_sel), w, n, _stream(stream)))


def decode_step(L, Q, K, V, Kp, P, seq_lens, n_new: int, k: int, window: int, sm_scale: float, O, lse=None,
                idx_out=None, n_sel_out=None, ws=None, stream=None):
    w, n = _ws(ws)
    _check("jssa_decode_step", load().jssa_decode_step(C.byref(L), _c(Q), _p(K), _p(V), _p(Kp), _c(P),
                                                       _c(seq_lens), n_new, k, window, sm_scale, _c(O), _c(lse),
                                                       _c(idx_out), _c(n_sel_out), w, n, _stream(stream)))


def alloc_gather_buffer(L, k: int, window: int = 0, device="cuda"):
    """Device buffer for gather_decode (the gather-then-attend comparator)."""
    n = C.c_size_t(0)
    _check("jssa_gather_size", load().jssa_gather_size(C.byref(L), k, window, C.byref(n)))
    return torch.empty(n.value, dtype=torch.uint8, device=device)


def gather_decode(L, Q, K, V, idx, k: int, n_sel, seq_lens, window: int, sm_scale: float, O, lse, gbuf, ws,
                  stream=None):
    w, n = _ws(ws)
    _check("jssa_gather_decode", load().jssa_gather_decode(C.byref(L), _c(Q), _p(K), _p(V), _c(idx), k, _c(n_sel),
                                                           _c(seq_lens), window, sm_scale, _c(O), _c(lse), _c(gbuf),
                                                           gbuf.numel(), w, n, _stream(stream)))


def vote_select(L, Q, K, Kp, P, seq_lens, n_new: int, k: int, window: int, sm_scale: float, idx, n_sel, ws,
                stream=None):
    """Head-shared soft voting: one index set per sequence, written to every KV head's row."""
    w, n = _ws(ws)
    _check("jssa_vote_select", load().jssa_vote_select(C.byref(L), _c(Q), _p(K), _p(Kp), _c(P), _c(seq_lens), n_new,
                                                       k, window, sm_scale, _c(idx), _c(n_sel), w, n,
                                                       _stream(stream)))


def alloc_calibration_workspace(L, device="cuda"):
    """Workspace of calibrate (status word zeroed)."""
    n = C.c_size_t(0)
    _check("jssa_calibrate_workspace_size", load().jssa_calibrate_workspace_size(C.byref(L), C.byref(n)))
    ws = torch.empty(n.value, dtype=torch.uint8, device=device)
    workspace_init(ws)
    return ws


def calibrate(L, Qc, K, n_tokens: int, P, ws, eigvals=None, stream=None):
    """Spectral basis from calibration queries Qc [B, Hq, n_tokens, d_k] and cache rows [0, n_tokens)."""
    w, n = _ws(ws)
    _check("jssa_calibrate", load().jssa_calibrate(C.byref(L), _c(Qc), _p(K), n_tokens, _c(P), _c(eigvals), w, n,
                                                   _stream(stream)))


def dense_decode(L, Q, K, V, seq_lens, window: int, sm_scale: float, O, lse=None, ws=None, stream=None):
    w, n = _ws(ws)
    _check("jssa_dense_decode", load().jssa_dense_decode(C.byref(L), _c(Q), _p(K), _p(V), _c(seq_lens), window,
                                                         sm_scale, _c(O), _c(lse), w, n, _stream(stream)))


def workspace_init(ws, stream=None):
    w, n = _ws(ws)
    _check("jssa_workspace_init", load().jssa_workspace_init(w, n, _stream(stream)))


def arm_withheld_copy(ws, wait_limit_us: int, stream=None):
    """Arm the one-shot test of the bounded waits in this workspace: the next selection
    launch withholds one bulk copy in row (0, 0) and gives up waiting after wait_limit_us."""
    w, n = _ws(ws)
    _check("jssa_test_withhold_copy", load().jssa_test_withhold_copy(w, n, wait_limit_us, _stream(stream)))


def read_device_status(ws, stream=None):
    """Returns (status code, flags) and clears the device status word (synchronises)."""
    w, n = _ws(ws)
    flags = C.c_int32(0)
    code = load().jssa_read_device_status(w, n, C.byref(flags), _stream(stream))
    return code, flags.value
