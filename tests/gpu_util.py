"""Helpers for the GPU parity tests: move a workload to the device, run it through the C ABI into a
sentinel-filled output, and compare with the oracle on the same seeded inputs."""
import numpy as np
import torch

import oracle
import nvfp4_grouped_gemm_indices_b200 as bsg

# bf16 quiet-NaN bit pattern no GEMM result takes: rows the kernel must not write keep it.
SENTINEL = 0x7FC1
TOL = 8e-3  # max |gpu - ref| / (|ref| + rms(ref)) over routed rows


def to_dev(x):
    return None if x is None else torch.from_numpy(np.ascontiguousarray(x)).cuda()


def sentinel_out(M, N):
    return torch.full((M, N), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class DevWorkload:
    def __init__(self, w):
        self.w = w
        self.A = to_dev(w.A)
        self.B = to_dev(w.B)
        self.m_indices = to_dev(w.m_indices)
        if w.kind == "fp8":
            self.a_scale = to_dev(w.a_scale)
            self.b_scale = to_dev(w.b_scale)
        else:
            self.sfa = to_dev(w.sfa)
            self.sfb = to_dev(w.sfb)
            self.alpha = to_dev(w.alpha)

    def run(self, out=None, stream=None):
        w = self.w
        C = sentinel_out(w.M, w.N) if out is None else out
        if w.kind == "fp8":
            bsg.bsg_fp8_grouped_gemm(self.A, self.B, self.a_scale, self.b_scale, self.m_indices, C,
                                     w.M, w.N, w.K, w.G, stream)
        else:
            bsg.bsg_nvfp4_gemm(self.A, self.B, self.sfa, self.sfb, self.alpha, self.m_indices, C,
                               w.M, w.N, w.K, w.G, stream)
        return C


def oracle_rows(w, rows=None):
    """Oracle bf16 bits for the given rows (all rows if None), unrouted rows = SENTINEL."""
    n = w.M if rows is None else len(rows)
    out = np.full((n, w.N), SENTINEL, dtype=np.uint16)
    if w.kind == "fp8":
        oracle.fp8_grouped(w.A, w.B, w.a_scale, w.b_scale, w.m_indices, w.M, w.N, w.K, w.G, rows=rows,
                           out_bf16=out)
    else:
        oracle.nvfp4(w.A, w.B, w.sfa, w.sfb, w.alpha, w.m_indices, w.M, w.N, w.K, w.G, rows=rows, out_bf16=out)
    return out


def routed_mask(w, rows=None):
    r = np.arange(w.M) if rows is None else np.asarray(rows)
    if w.m_indices is None:
        return np.ones(len(r), dtype=bool)
    g = w.m_indices[r]
    return (g >= 0) & (g < w.G)


def compare(gpu_bits, ref_bits, routed, tol=TOL):
    """Returns (normalised error, message); asserts the routing bit-exactly."""
    unrouted = ~routed
    assert np.all(gpu_bits[unrouted] == SENTINEL), "a row that is not routed was written"
    if not routed.any():
        return 0.0, "no routed rows"
    g = oracle.bf16_bits_to_f64(gpu_bits[routed])
    r = oracle.bf16_bits_to_f64(ref_bits[routed])
    assert not np.isnan(r).any(), "oracle produced NaN"
    nan_rows = np.isnan(g).any(axis=1)
    assert not nan_rows.any(), f"{int(nan_rows.sum())} routed rows hold NaN (unwritten or bad)"
    rms = float(np.sqrt(np.mean(r * r)))
    err = np.abs(g - r) / (np.abs(r) + rms)
    worst = float(err.max())
    i, j = np.unravel_index(int(err.argmax()), err.shape)
    msg = f"max normalised error {worst:.3e} at routed row #{i} col {j}: gpu {g[i, j]} ref {r[i, j]} (rms {rms:.3e})"
    assert worst <= tol, msg
    return worst, msg


def sample_rows(w, n_random=64, seed=0, boundary_halo=2):
    """Rows within +-halo of every run boundary and of every window edge, plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    idx = w.m_indices
    if idx is not None:
        change = np.nonzero(idx[1:] != idx[:-1])[0] + 1
        for c in change.tolist():
            rows.update(range(max(0, c - boundary_halo), min(w.M, c + boundary_halo)))
    rows.update([0, w.M - 1])
    rows.update(rng.integers(0, w.M, n_random).tolist())
    return np.array(sorted(rows), dtype=np.int64)
