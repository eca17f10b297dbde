"""Block-scaled grouped GEMM (FP8 and NVFP4) for NVIDIA B200 -- Python binding of libbsg.so.

This module only marshals arguments: every step of the computation runs in the CUDA kernels of
``lib/libbsg.so`` (sources in ``csrc/``, C ABI in ``include/bsg.h``).  PyTorch is used for device
memory and streams.  If the library is missing the import still succeeds but every call raises
``BsgError`` -- there is no CPU fallback.

Low-level calls have the C names and arguments (pointers may be ints or torch tensors)::

    bsg_fp8_grouped_gemm(A, B, a_scale, b_scale, m_indices, C, M, N, K, G, stream=None)
    bsg_nvfp4_gemm(A, B, sfa, sfb, alpha, m_indices, C, M, N, K, G, stream=None)

Convenience wrappers infer the sizes from torch tensors and allocate C when not given::

    fp8_grouped_gemm(A, B, a_scale, b_scale, m_indices, out=None)
    nvfp4_gemm(A, B, sfa, sfb, alpha, m_indices, out=None)

and the steps before the GEMM (the MoE expand permutation, then activation quantisation with a row
gather)::

    moe_permute(expert_ids, G) -> (src_rows, m_indices, dst_rows, expert_offsets)
    quantize_fp8_rows(X, src_rows=None) -> (A, a_scale)
    quantize_nvfp4_rows(X, global_scale, src_rows=None) -> (A, sfa)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libbsg.so")

BSG_OK = 0
BSG_ERR_INVALID_ARG = -1
BSG_ERR_ALIGNMENT = -2
BSG_ERR_UNSUPPORTED_SHAPE = -3
BSG_ERR_CUDA = -4
BSG_ERR_DEVICE_TIMEOUT = -5

STATUS_NAMES = {
    0: "BSG_OK", -1: "BSG_ERR_INVALID_ARG", -2: "BSG_ERR_ALIGNMENT", -3: "BSG_ERR_UNSUPPORTED_SHAPE",
    -4: "BSG_ERR_CUDA", -5: "BSG_ERR_DEVICE_TIMEOUT",
}

# Every symbol include/bsg.h declares.
EXPORTED = [
    "bsg_fp8_grouped_gemm", "bsg_nvfp4_gemm", "bsg_last_error", "bsg_get_device_status",
    "bsg_set_wait_timeout_ns", "bsg_num_tactics", "bsg_tactic_name", "bsg_choose_tactic",
    "bsg_tactic_score", "bsg_set_tactic", "bsg_set_max_ctas", "bsg_debug_set_fault", "bsg_version",
    "bsg_quantize_fp8_rows", "bsg_quantize_nvfp4_rows", "bsg_autotune_fp8", "bsg_autotune_nvfp4",
    "bsg_autotune_clear", "bsg_moe_permute_workspace_size", "bsg_moe_permute", "bsg_moe_permute_noalloc",
]


class BsgError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load(path: Optional[str] = None):
    """Load libbsg.so (once).  Raises BsgError when the library has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise BsgError(BSG_ERR_CUDA, f"{p} is missing: build it with `python -m nvfp4_grouped_gemm_indices_b200.build`")
    L = ctypes.CDLL(p)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.bsg_fp8_grouped_gemm.restype = i32
    L.bsg_fp8_grouped_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    L.bsg_nvfp4_gemm.restype = i32
    L.bsg_nvfp4_gemm.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    L.bsg_last_error.restype = ctypes.c_char_p
    L.bsg_last_error.argtypes = []
    L.bsg_get_device_status.restype = i32
    L.bsg_get_device_status.argtypes = [vp]
    L.bsg_set_wait_timeout_ns.restype = ctypes.c_uint64
    L.bsg_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    L.bsg_num_tactics.restype = i32
    L.bsg_num_tactics.argtypes = [i32]
    L.bsg_tactic_name.restype = ctypes.c_char_p
    L.bsg_tactic_name.argtypes = [i32, i32]
    L.bsg_choose_tactic.restype = i32
    L.bsg_choose_tactic.argtypes = [i32, i64, i64, i64, i64, i32]
    L.bsg_tactic_score.restype = ctypes.c_double
    L.bsg_tactic_score.argtypes = [i32, i32, i64, i64, i64, i64, i32]
    L.bsg_set_tactic.restype = i32
    L.bsg_set_tactic.argtypes = [i32, i32]
    L.bsg_set_max_ctas.restype = i32
    L.bsg_set_max_ctas.argtypes = [i32, i32]
    L.bsg_debug_set_fault.restype = i32
    L.bsg_debug_set_fault.argtypes = [i32]
    L.bsg_version.restype = ctypes.c_char_p
    L.bsg_version.argtypes = []
    L.bsg_quantize_fp8_rows.restype = i32
    L.bsg_quantize_fp8_rows.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
    L.bsg_autotune_fp8.restype = i32
    L.bsg_autotune_fp8.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, vp]
    L.bsg_autotune_nvfp4.restype = i32
    L.bsg_autotune_nvfp4.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, vp]
    L.bsg_autotune_clear.restype = None
    L.bsg_autotune_clear.argtypes = []
    L.bsg_quantize_nvfp4_rows.restype = i32
    L.bsg_quantize_nvfp4_rows.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.bsg_moe_permute_workspace_size.restype = i32
    L.bsg_moe_permute_workspace_size.argtypes = [i64, i64, i64, ctypes.POINTER(ctypes.c_size_t)]
    L.bsg_moe_permute.restype = i32
    L.bsg_moe_permute.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.bsg_moe_permute_noalloc.restype = i32
    L.bsg_moe_permute_noalloc.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp]
    if path is None:
        _lib = L
    return L


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"cannot take a device pointer of {type(x)}")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != BSG_OK:
        msg = load().bsg_last_error().decode(errors="replace")
        raise BsgError(status, msg)


# ------------------------------------------------------------------------------- C-named calls


def bsg_fp8_grouped_gemm(A, B, a_scale, b_scale, m_indices, C, M, N, K, G, stream=None):
    _check(load().bsg_fp8_grouped_gemm(_ptr(A), _ptr(B), _ptr(a_scale), _ptr(b_scale), _ptr(m_indices), _ptr(C),
                                       int(M), int(N), int(K), int(G), _stream(stream)))


def bsg_nvfp4_gemm(A, B, sfa, sfb, alpha, m_indices, C, M, N, K, G, stream=None):
    _check(load().bsg_nvfp4_gemm(_ptr(A), _ptr(B), _ptr(sfa), _ptr(sfb), _ptr(alpha), _ptr(m_indices), _ptr(C),
                                 int(M), int(N), int(K), int(G), _stream(stream)))


def bsg_quantize_fp8_rows(X, src_rows, A, a_scale, M_in, M, K, stream=None):
    _check(load().bsg_quantize_fp8_rows(_ptr(X), _ptr(src_rows), _ptr(A), _ptr(a_scale), int(M_in), int(M), int(K),
                                        _stream(stream)))


def bsg_quantize_nvfp4_rows(X, src_rows, global_scale, A, sfa, M_in, M, K, stream=None):
    _check(load().bsg_quantize_nvfp4_rows(_ptr(X), _ptr(src_rows), _ptr(global_scale), _ptr(A), _ptr(sfa),
                                          int(M_in), int(M), int(K), _stream(stream)))


def bsg_moe_permute_workspace_size(T, top_k, G) -> int:
    n = ctypes.c_size_t(0)
    _check(load().bsg_moe_permute_workspace_size(int(T), int(top_k), int(G), ctypes.byref(n)))
    return int(n.value)


def bsg_moe_permute(expert_ids, T, top_k, G, src_rows, m_indices, dst_rows, expert_offsets, workspace,
                    workspace_bytes, stream=None):
    _check(load().bsg_moe_permute(_ptr(expert_ids), int(T), int(top_k), int(G), _ptr(src_rows), _ptr(m_indices),
                                  _ptr(dst_rows), _ptr(expert_offsets), _ptr(workspace), int(workspace_bytes),
                                  _stream(stream)))


def bsg_moe_permute_noalloc(expert_ids, T, top_k, G, src_rows, m_indices, dst_rows, expert_offsets, stream=None):
    """bsg_moe_permute for callers that cannot allocate device memory: the scratch is a fixed 2 MiB
    array inside the library (see include/bsg.h for the size limit and the sharing rules)."""
    _check(load().bsg_moe_permute_noalloc(_ptr(expert_ids), int(T), int(top_k), int(G), _ptr(src_rows),
                                          _ptr(m_indices), _ptr(dst_rows), _ptr(expert_offsets), _stream(stream)))


def bsg_autotune_fp8(A, B, a_scale, b_scale, m_indices, C, M, N, K, G, reps=20, stream=None) -> int:
    r = int(load().bsg_autotune_fp8(_ptr(A), _ptr(B), _ptr(a_scale), _ptr(b_scale), _ptr(m_indices), _ptr(C),
                                    int(M), int(N), int(K), int(G), int(reps), _stream(stream)))
    _check(min(r, 0))
    return r


def bsg_autotune_nvfp4(A, B, sfa, sfb, alpha, m_indices, C, M, N, K, G, reps=20, stream=None) -> int:
    r = int(load().bsg_autotune_nvfp4(_ptr(A), _ptr(B), _ptr(sfa), _ptr(sfb), _ptr(alpha), _ptr(m_indices),
                                      _ptr(C), int(M), int(N), int(K), int(G), int(reps), _stream(stream)))
    _check(min(r, 0))
    return r


def bsg_autotune_clear():
    load().bsg_autotune_clear()


def bsg_last_error() -> str:
    return load().bsg_last_error().decode(errors="replace")


def bsg_get_device_status(stream=None):
    _check(load().bsg_get_device_status(_stream(stream)))


def bsg_set_wait_timeout_ns(ns: int) -> int:
    return int(load().bsg_set_wait_timeout_ns(int(ns)))


def bsg_num_tactics(kind: int) -> int:
    return int(load().bsg_num_tactics(int(kind)))


def bsg_tactic_name(kind: int, tactic: int) -> str:
    return load().bsg_tactic_name(int(kind), int(tactic)).decode()


def bsg_choose_tactic(kind, M, N, K, G, sm_count) -> int:
    r = int(load().bsg_choose_tactic(int(kind), int(M), int(N), int(K), int(G), int(sm_count)))
    _check(min(r, 0))
    return r


def bsg_tactic_score(kind, tactic, M, N, K, G, sm_count) -> float:
    return float(load().bsg_tactic_score(int(kind), int(tactic), int(M), int(N), int(K), int(G), int(sm_count)))


def bsg_set_tactic(kind: int, tactic: int):
    _check(load().bsg_set_tactic(int(kind), int(tactic)))


def bsg_set_max_ctas(kind: int, max_ctas: int):
    _check(load().bsg_set_max_ctas(int(kind), int(max_ctas)))


def bsg_debug_set_fault(mode: int):
    _check(load().bsg_debug_set_fault(int(mode)))


def bsg_version() -> str:
    return load().bsg_version().decode()


# ------------------------------------------------------------------------------- torch wrappers


def _need(t, dtype, name, dims=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dimensions, got {t.dim()}")


def _same_device(named, stream=None):
    """Every tensor (and the stream, if given) must be on one CUDA device; returns that device.  The
    library launches on the current device, so the wrappers make it current for the call."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device} but the other operands are on {dev}")
    if stream is not None and not isinstance(stream, int) and hasattr(stream, "device"):
        if stream.device != dev:
            raise ValueError(f"stream is on {stream.device} but the operands are on {dev}")
    return dev


def fp8_grouped_gemm(A, B, a_scale, b_scale, m_indices, out=None, stream=None):
    """A uint8/float8 [M,K], B [G,N,K], a_scale f32 [M,K/128], b_scale f32 [G,ceil(N/128),K/128],
    m_indices int32 [M] (or None when G == 1).  Returns C bf16 [M,N] (unrouted rows of a fresh C
    are zero)."""
    import torch
    A8 = A.view(torch.uint8) if A.dtype != torch.uint8 else A
    B8 = B.view(torch.uint8) if B.dtype != torch.uint8 else B
    _need(A8, torch.uint8, "A", 2)
    _need(B8, torch.uint8, "B", 3)
    M, K = A8.shape
    G, N, K2 = B8.shape
    if K2 != K:
        raise ValueError("A and B disagree on K")
    _need(a_scale, torch.float32, "a_scale")
    _need(b_scale, torch.float32, "b_scale")
    if tuple(a_scale.shape) != (M, K // 128):
        raise ValueError(f"a_scale must be [{M}, {K // 128}]")
    if tuple(b_scale.shape) != (G, (N + 127) // 128, K // 128):
        raise ValueError(f"b_scale must be [{G}, {(N + 127) // 128}, {K // 128}]")
    if m_indices is not None:
        _need(m_indices, torch.int32, "m_indices", 1)
        if m_indices.numel() != M:
            raise ValueError("m_indices must have M entries")
    if out is not None:
        _need(out, torch.bfloat16, "out", 2)
        if tuple(out.shape) != (M, N):
            raise ValueError(f"out must be [{M}, {N}]")
    dev = _same_device((("A", A8), ("B", B8), ("a_scale", a_scale), ("b_scale", b_scale),
                        ("m_indices", m_indices), ("out", out)), stream)
    with torch.cuda.device(dev):
        if out is None:
            out = torch.zeros((M, N), dtype=torch.bfloat16, device=dev)
        bsg_fp8_grouped_gemm(A8, B8, a_scale, b_scale, m_indices, out, M, N, K, G, stream)
    return out


def nvfp4_gemm(A, B, sfa, sfb, alpha, m_indices, out=None, stream=None):
    """A uint8 [M,K/2] packed E2M1, B [G,N,K/2], sfa uint8 [M,K/16], sfb uint8 [G,N,K/16],
    alpha f32 [G], m_indices int32 [M] or None (G == 1).  Returns C bf16 [M,N]."""
    import torch
    _need(A, torch.uint8, "A", 2)
    _need(B, torch.uint8, "B", 3)
    M, Kh = A.shape
    G, N, Kh2 = B.shape
    if Kh2 != Kh:
        raise ValueError("A and B disagree on K")
    K = 2 * Kh
    for t, name, shape in ((sfa, "sfa", (M, K // 16)), (sfb, "sfb", (G, N, K // 16))):
        sf8 = t.view(torch.uint8) if t.dtype != torch.uint8 else t
        _need(sf8, torch.uint8, name)
        if tuple(sf8.shape) != shape:
            raise ValueError(f"{name} must be {list(shape)}")
    _need(alpha, torch.float32, "alpha", 1)
    if alpha.numel() != G:
        raise ValueError("alpha must have G entries")
    if m_indices is not None:
        _need(m_indices, torch.int32, "m_indices", 1)
        if m_indices.numel() != M:
            raise ValueError("m_indices must have M entries")
    if out is not None:
        _need(out, torch.bfloat16, "out", 2)
        if tuple(out.shape) != (M, N):
            raise ValueError(f"out must be [{M}, {N}]")
    dev = _same_device((("A", A), ("B", B), ("sfa", sfa), ("sfb", sfb), ("alpha", alpha),
                        ("m_indices", m_indices), ("out", out)), stream)
    with torch.cuda.device(dev):
        if out is None:
            out = torch.zeros((M, N), dtype=torch.bfloat16, device=dev)
        bsg_nvfp4_gemm(A, B, sfa, sfb, alpha, m_indices, out, M, N, K, G, stream)
    return out


def moe_permute(expert_ids, G, stream=None):
    """expert_ids int32 [T, top_k] (CUDA) -> (src_rows int32 [T*top_k], m_indices int32 [T*top_k],
    dst_rows int32 [T, top_k], expert_offsets int32 [G+1]): the expert-grouped layout of the routing
    entries (see bsg_moe_permute); the scratch, when the sizes need one, is a torch allocation made
    here."""
    import torch
    _need(expert_ids, torch.int32, "expert_ids", 2)
    T, top_k = expert_ids.shape
    n = T * top_k
    dev = _same_device((("expert_ids", expert_ids),), stream)
    with torch.cuda.device(dev):
        nbytes = bsg_moe_permute_workspace_size(T, top_k, G)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None
        src = torch.empty(n, dtype=torch.int32, device=dev)
        mi = torch.empty(n, dtype=torch.int32, device=dev)
        dst = torch.empty((T, top_k), dtype=torch.int32, device=dev)
        off = torch.empty(G + 1, dtype=torch.int32, device=dev)
        bsg_moe_permute(expert_ids, T, top_k, G, src, mi, dst, off, ws, nbytes, stream)
    return src, mi, dst, off


def quantize_fp8_rows(X, src_rows=None, stream=None):
    """X bf16 [M_in, K] -> (A uint8 [M, K] E4M3 codes, a_scale f32 [M, K/128]), the FP8 GEMM's A
    operand; with src_rows (int32 [M]) output row m is input row src_rows[m]."""
    import torch
    _need(X, torch.bfloat16, "X", 2)
    M_in, K = X.shape
    M = M_in
    if src_rows is not None:
        _need(src_rows, torch.int32, "src_rows", 1)
        M = src_rows.numel()
    dev = _same_device((("X", X), ("src_rows", src_rows)), stream)
    with torch.cuda.device(dev):
        A = torch.zeros((M, K), dtype=torch.uint8, device=dev)
        s = torch.zeros((M, K // 128), dtype=torch.float32, device=dev)
        bsg_quantize_fp8_rows(X, src_rows, A, s, M_in, M, K, stream)
    return A, s


def quantize_nvfp4_rows(X, global_scale, src_rows=None, stream=None):
    """X bf16 [M_in, K], global_scale f32 [1] on the device -> (A uint8 [M, K/2] packed E2M1,
    sfa uint8 [M, K/16]), the NVFP4 GEMM's A operand."""
    import torch
    _need(X, torch.bfloat16, "X", 2)
    _need(global_scale, torch.float32, "global_scale")
    M_in, K = X.shape
    M = M_in
    if src_rows is not None:
        _need(src_rows, torch.int32, "src_rows", 1)
        M = src_rows.numel()
    dev = _same_device((("X", X), ("global_scale", global_scale), ("src_rows", src_rows)), stream)
    with torch.cuda.device(dev):
        A = torch.zeros((M, K // 2), dtype=torch.uint8, device=dev)
        sf = torch.zeros((M, K // 16), dtype=torch.uint8, device=dev)
        bsg_quantize_nvfp4_rows(X, src_rows, global_scale, A, sf, M_in, M, K, stream)
    return A, sf

