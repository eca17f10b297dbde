"""fp64 CPU oracle for the block-scaled grouped GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of ``bench.py`` may
import this package.  It shares no code with the CUDA library and never imports it.

Functions (all numpy in, numpy out):

* ``dec_e4m3(codes)``, ``dec_e2m1(nibbles)`` -- decode from the bit fields.
* ``bf16_from_f64(x)`` -- one round-to-nearest-even step from fp64 to bf16 bit patterns.
* ``fp8_grouped(...)`` -- the FP8 definition (page "FlashInfer FP8 GEMM 최적화: 윈도우 세그먼트 KG1
  프로그램으로 GPU 성능 극대화", introduction and section 1): E4M3 codes, FP32 scales per 128-element
  K block, rows routed by ``m_indices``, BF16 out.
* ``nvfp4(...)`` -- the NVFP4 definition (page "ONNX Runtime: Blackwell (SM120+)에서 NVFP4 QMoE를
  위한 네이티브 FP4xFP4 Prefill 최적화", section 1): E2M1 codes, one E4M3 scale per 16 K elements,
  per-expert FP32 ``alpha``.
* ``window_plan(m_indices, M, G)`` -- the window segmentation the pages describe (same FP8 page,
  section 2): maximal equal runs of routed rows cut at 128-row window edges.
* ``enc_e4m3``, ``enc_e2m1``, ``quant_fp8_rows``, ``quant_nvfp4_rows`` -- the step before the GEMM:
  BF16 activations (optionally gathered by a row map, the MoE expand) quantised into the GEMM's
  input formats, from the format definitions (RNE, saturating) with every step in IEEE fp32.
* ``moe_permute(expert_ids, G)`` -- the MoE expand permutation that makes each expert's rows one
  contiguous run (the expanded input rows of the ONNX Runtime page, section 1): a plain stable
  counting sort of the (token, choice) entries by expert, with the inverse map.

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` (decode tables, exact
integer grids, grouped == dense, exact rational brute force, fp64 library matmul, the printed CTA
counts of the FP8 page's benchmark table).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.bsg_oracle_dec_e4m3.restype = ctypes.c_double
        L.bsg_oracle_dec_e4m3.argtypes = [ctypes.c_uint8]
        L.bsg_oracle_dec_e2m1.restype = ctypes.c_double
        L.bsg_oracle_dec_e2m1.argtypes = [ctypes.c_uint8]
        L.bsg_oracle_bf16_from_f64.restype = ctypes.c_uint16
        L.bsg_oracle_bf16_from_f64.argtypes = [ctypes.c_double]
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.bsg_oracle_fp8_grouped.restype = ctypes.c_int
        L.bsg_oracle_fp8_grouped.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, i64, p, p]
        L.bsg_oracle_nvfp4.restype = ctypes.c_int
        L.bsg_oracle_nvfp4.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, p, i64, p, p]
        L.bsg_oracle_enc_e4m3.restype = ctypes.c_uint8
        L.bsg_oracle_enc_e4m3.argtypes = [ctypes.c_float]
        L.bsg_oracle_enc_e2m1.restype = ctypes.c_uint8
        L.bsg_oracle_enc_e2m1.argtypes = [ctypes.c_float]
        L.bsg_oracle_quant_fp8_rows.restype = ctypes.c_int
        L.bsg_oracle_quant_fp8_rows.argtypes = [p, p, i64, i64, i64, p, p]
        L.bsg_oracle_quant_nvfp4_rows.restype = ctypes.c_int
        L.bsg_oracle_quant_nvfp4_rows.argtypes = [p, p, ctypes.c_float, i64, i64, i64, p, p]
        L.bsg_oracle_moe_permute.restype = ctypes.c_int
        L.bsg_oracle_moe_permute.argtypes = [p, i64, i64, i64, p, p, p, p]
        L.bsg_oracle_max_threads.restype = ctypes.c_int
        L.bsg_oracle_set_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def dec_e4m3(codes):
    L = lib()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([L.bsg_oracle_dec_e4m3(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def dec_e2m1(nibbles):
    L = lib()
    c = np.asarray(nibbles, dtype=np.uint8)
    return np.array([L.bsg_oracle_dec_e2m1(int(x) & 0xF) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def bf16_from_f64(x):
    L = lib()
    a = np.asarray(x, dtype=np.float64)
    return np.array([L.bsg_oracle_bf16_from_f64(float(v)) for v in a.ravel()], dtype=np.uint16).reshape(a.shape)


def bf16_bits_to_f64(bits):
    """Widen bf16 bit patterns to fp64 (exact: bf16 is the top half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def _rows_arg(rows, M):
    if rows is None:
        return None, M
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, int(r.size)


def fp8_grouped(A, B, a_scale, b_scale, m_indices, M, N, K, G, rows=None, out_bf16=None,
                want_f64=False):
    """Returns (bf16 bits [n_rows,N], f64 [n_rows,N] or None).  Unrouted rows keep the initial
    contents of ``out_bf16`` (default: 0xFFFF sentinel) and NaN in the f64 output."""
    L = lib()
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    a_scale = np.ascontiguousarray(a_scale, dtype=np.float32)
    b_scale = np.ascontiguousarray(b_scale, dtype=np.float32)
    idx = None if m_indices is None else np.ascontiguousarray(m_indices, dtype=np.int32)
    r, n_rows = _rows_arg(rows, M)
    if out_bf16 is None:
        out_bf16 = np.full((n_rows, N), 0xFFFF, dtype=np.uint16)
    f64 = np.full((n_rows, N), np.nan, dtype=np.float64) if want_f64 else None
    rc = L.bsg_oracle_fp8_grouped(_ptr(A), _ptr(B), _ptr(a_scale), _ptr(b_scale), _ptr(idx), M, N, K, G,
                                  _ptr(r), n_rows, _ptr(f64), _ptr(out_bf16))
    if rc != 0:
        raise ValueError("oracle fp8_grouped: invalid sizes")
    return out_bf16, f64


def nvfp4(A, B, sfa, sfb, alpha, m_indices, M, N, K, G, rows=None, out_bf16=None, want_f64=False):
    """Returns (bf16 bits [n_rows,N], f64 [n_rows,N] or None); unrouted rows as for fp8_grouped."""
    L = lib()
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sfa = np.ascontiguousarray(sfa, dtype=np.uint8)
    sfb = np.ascontiguousarray(sfb, dtype=np.uint8)
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    idx = None if m_indices is None else np.ascontiguousarray(m_indices, dtype=np.int32)
    r, n_rows = _rows_arg(rows, M)
    if out_bf16 is None:
        out_bf16 = np.full((n_rows, N), 0xFFFF, dtype=np.uint16)
    f64 = np.full((n_rows, N), np.nan, dtype=np.float64) if want_f64 else None
    rc = L.bsg_oracle_nvfp4(_ptr(A), _ptr(B), _ptr(sfa), _ptr(sfb), _ptr(alpha), _ptr(idx), M, N, K, G,
                            _ptr(r), n_rows, _ptr(f64), _ptr(out_bf16))
    if rc != 0:
        raise ValueError("oracle nvfp4: invalid sizes")
    return out_bf16, f64


def enc_e4m3(x):
    """fp32 value(s) -> E4M3 code(s): round to nearest even, saturating at +-448."""
    L = lib()
    a = np.asarray(x, dtype=np.float32)
    return np.array([L.bsg_oracle_enc_e4m3(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def enc_e2m1(x):
    """fp32 value(s) -> E2M1 code(s) 0..15: round to nearest even, saturating at +-6."""
    L = lib()
    a = np.asarray(x, dtype=np.float32)
    return np.array([L.bsg_oracle_enc_e2m1(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def quant_fp8_rows(X_bf16_bits, M=None, src_rows=None, A=None, scale=None):
    """Activation quantisation to the FP8 GEMM's A operand: per 1 x 128 block, scale = amax/448,
    code = e4m3_rne_satfinite(x / scale), the quotient one correctly rounded fp32 division per
    element; a zero block gets zero codes.  X: uint16 bf16 bits [M_in, K]; output row m is
    input row src_rows[m] (or m).  Returns (A uint8 [M, K], scale f32 [M, K/128]); rows whose
    source is out of range keep the initial contents of A / scale (default 0xFF / NaN)."""
    L = lib()
    X = np.ascontiguousarray(X_bf16_bits, dtype=np.uint16)
    M_in, K = X.shape
    M = M_in if M is None else int(M)
    src = None if src_rows is None else np.ascontiguousarray(src_rows, dtype=np.int32)
    if A is None:
        A = np.full((M, K), 0xFF, dtype=np.uint8)
    if scale is None:
        scale = np.full((M, K // 128), np.nan, dtype=np.float32)
    rc = L.bsg_oracle_quant_fp8_rows(_ptr(X), _ptr(src), M_in, M, K, _ptr(A), _ptr(scale))
    if rc != 0:
        raise ValueError("oracle quant_fp8_rows: invalid sizes")
    return A, scale


def quant_nvfp4_rows(X_bf16_bits, gs, M=None, src_rows=None, A=None, sf=None):
    """Activation quantisation to the NVFP4 GEMM's A operand with global scale gs: per 1 x 16
    block, s = ue4m3_rne_satfinite((amax/6)/gs), code = e2m1_rne_satfinite(x / (dec(s) * gs)),
    every step one correctly rounded fp32 operation (one division per element).  Returns (A uint8 [M, K/2] packed, low nibble = lower K; sf uint8 [M, K/16])."""
    L = lib()
    X = np.ascontiguousarray(X_bf16_bits, dtype=np.uint16)
    M_in, K = X.shape
    M = M_in if M is None else int(M)
    src = None if src_rows is None else np.ascontiguousarray(src_rows, dtype=np.int32)
    if A is None:
        A = np.full((M, K // 2), 0xFF, dtype=np.uint8)
    if sf is None:
        sf = np.full((M, K // 16), 0xFF, dtype=np.uint8)
    rc = L.bsg_oracle_quant_nvfp4_rows(_ptr(X), _ptr(src), float(np.float32(gs)), M_in, M, K, _ptr(A), _ptr(sf))
    if rc != 0:
        raise ValueError("oracle quant_nvfp4_rows: invalid sizes")
    return A, sf


def moe_permute(expert_ids, G):
    """The MoE expand permutation: a stable counting sort of the (token, choice) entries of
    expert_ids [T, top_k] (token-major) by expert.  Returns (src_rows int32 [T*top_k], m_indices
    int32 [T*top_k], dst_rows int32 [T, top_k], expert_offsets int32 [G+1]); entries whose expert
    is outside [0, G) are dropped (dst_rows -1) and the unused tail positions hold -1."""
    L = lib()
    e = np.ascontiguousarray(expert_ids, dtype=np.int32)
    if e.ndim != 2:
        raise ValueError("expert_ids must be [T, top_k]")
    T, top_k = e.shape
    n = T * top_k
    src = np.empty(n, np.int32)
    mi = np.empty(n, np.int32)
    dst = np.empty((T, top_k), np.int32)
    off = np.empty(G + 1, np.int32)
    rc = L.bsg_oracle_moe_permute(_ptr(e), T, top_k, int(G), _ptr(src), _ptr(mi), _ptr(dst), _ptr(off))
    if rc != 0:
        raise ValueError("oracle moe_permute: invalid sizes")
    return src, mi, dst, off


def set_threads(n):
    lib().bsg_oracle_set_threads(int(n))


def max_threads():
    return int(lib().bsg_oracle_max_threads())


def window_plan(m_indices, M, G, window=128):
    """Window segmentation (FP8 page, section 2, program selection): cut the rows into 128-row
    windows; inside each window, every maximal stretch of consecutive rows routed to the same
    expert is one segment (window, row_lo, row_hi, g).  Rows routed nowhere (index < 0 or >= G)
    belong to no segment.  Returns the list of segments in window order."""
    segs = []
    for w in range((M + window - 1) // window):
        lo = w * window
        hi = min(M, lo + window)
        r = lo
        while r < hi:
            g = 0 if m_indices is None else int(m_indices[r])
            if g < 0 or g >= G:
                r += 1
                continue
            s = r
            while r < hi and (0 if m_indices is None else int(m_indices[r])) == g:
                r += 1
            segs.append((w, s, r, g))
    return segs


def window_grid_ctas(m_indices, M, N, G, n_tile=64, window=128):
    """CTA count of the pages' window-segment program: ceil(M/128) windows x the largest number of
    segments in any window x ceil(N/64) column tiles (FP8 page, section 2 and its benchmark table)."""
    segs = window_plan(m_indices, M, G, window)
    per_window = {}
    for (w, _, _, _) in segs:
        per_window[w] = per_window.get(w, 0) + 1
    window_runs = max(per_window.values()) if per_window else 0
    return ((M + window - 1) // window) * window_runs * ((N + n_tile - 1) // n_tile)
