"""Seeded inputs on which dividing by a block scale and multiplying by its rounded reciprocal give
different quantised codes.

The activation quantisers divide each element by its block's scale (FP8: ``x / (amax/448)``; NVFP4:
``x / (dec(s) * gs)``).  The product ``x * fp32(1/scale)`` is off the correctly rounded quotient by
up to about two fp32 steps, so where the quotient lies next to a rounding boundary of the target
format (a midpoint between two neighbouring codes) the two give different codes.  These generators
search for such elements with plain numpy fp32 arithmetic (IEEE division and product) and the
library encoders of ``workloads``; nothing here comes from the oracle or the CUDA library.

* ``fp8_rows(n_blocks, seed)`` -> (bf16 bit patterns [1, 128 * n_blocks], boolean mask of the
  elements whose division and reciprocal codes differ).  Block b holds its amax at column 0, up to
  ``per_block`` adversarial elements for that amax, and small random fill below the amax.
* ``nvfp4_cases(n, seed)`` -> list of (gs, bf16 bits [1, 16 * blocks], mask): each case is one row
  quantised with its own global scale ``gs``, chosen so that one element of its first block is
  adversarial; the other blocks are random.
"""
import numpy as np

from nvfp4_grouped_gemm_indices_b200 import workloads as W


def _bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def _f32_to_bits_trunc(x):
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _e4m3_midpoints():
    vals = W.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)).astype(np.float64)
    return ((vals[:-1] + vals[1:]) / 2).astype(np.float32)


def fp8_adversarial_for(amax_bits):
    """bf16 bit patterns x (0 < x <= amax) whose E4M3 code from x / s differs from the one from
    x * fp32(1 / s), s = fp32(amax / 448)."""
    amax = _bits_to_f32(amax_bits)
    s = np.float32(amax / np.float32(448.0))
    inv = np.float32(np.float32(1.0) / s)
    mids = _e4m3_midpoints()
    centre = _f32_to_bits_trunc((mids * s).astype(np.float32)).astype(np.int64)
    cand = np.unique(np.concatenate([centre + d for d in range(-3, 4)]))
    cand = cand[(cand > 0) & (cand < 0x7F80)].astype(np.uint16)
    x = _bits_to_f32(cand)
    keep = x <= amax
    cand, x = cand[keep], x[keep]
    diff = W.e4m3_encode(x / s) != W.e4m3_encode(x * inv)
    return cand[diff]


def fp8_rows(n_blocks=64, seed=0, per_block=24):
    rng = np.random.default_rng(seed)
    row = np.zeros(128 * n_blocks, dtype=np.uint16)
    mask = np.zeros(128 * n_blocks, dtype=bool)
    b = 0
    while b < n_blocks:
        amax_bits = np.uint16(rng.integers(0x3C00, 0x4300))       # amax in [2^-7, 128)
        adv = fp8_adversarial_for(amax_bits)
        if adv.size == 0:
            continue
        adv = adv[:per_block]
        amax = _bits_to_f32(amax_bits)
        fill = (rng.uniform(-1, 1, 128) * amax * 0.9).astype(np.float32)
        blk = _f32_to_bits_trunc(fill)
        blk[0] = amax_bits
        pos = 1 + rng.permutation(127)[:adv.size]
        sign = rng.integers(0, 2, adv.size).astype(np.uint16) << 15
        blk[pos] = adv | sign
        row[128 * b:128 * (b + 1)] = blk
        mask[128 * b + pos] = True
        b += 1
    return row[None, :], mask[None, :]


_E2M1_MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)


def _nvfp4_codes(x, gs):
    """(scale code, division codes, reciprocal codes) of one 16-element block, numpy fp32."""
    amax = np.float32(np.abs(x).max())
    sc = W.e4m3_encode(np.array([amax / np.float32(6.0) / gs], np.float32))[0]
    d = np.float32(W.e4m3_decode(np.array([sc], np.uint8))[0] * gs)
    inv = np.float32(np.float32(1.0) / d)
    return sc, W.e2m1_encode(x / d), W.e2m1_encode(x * inv)


def nvfp4_cases(n=12, seed=0, blocks=4):
    """One element of block 0 is adversarial: pick x (bf16), a boundary m and a scale code sc, set
    gs so that dec(sc) * gs lands within a few fp32 steps of x / m, and keep the gs for which the
    two codes of x differ; then choose the block's amax so that the block's own scale code is sc."""
    rng = np.random.default_rng(seed)
    out = []
    tries = 0
    while len(out) < n and tries < 100000:
        tries += 1
        m = rng.choice(_E2M1_MIDS)
        sc = np.uint8(rng.integers(0x30, 0x70))
        dsc = np.float32(W.e4m3_decode(np.array([sc], np.uint8))[0])
        xb = np.uint16(rng.integers(0x3C00, 0x4400))
        x = _bits_to_f32(xb)
        g0 = np.array([np.float32((x / m) / dsc)], np.float32).view(np.uint32)[0]
        for k in range(-6, 7):
            gs = np.array([np.uint32(int(g0) + k)], np.uint32).view(np.float32)[0]
            d = np.float32(dsc * gs)
            if W.e2m1_encode(np.array([x / d], np.float32))[0] == \
                    W.e2m1_encode(np.array([x * np.float32(np.float32(1.0) / d)], np.float32))[0]:
                continue
            # an amax (bf16, >= x) whose block scale code is sc
            target = np.float32(6.0 * dsc * gs)
            for ab in _f32_to_bits_trunc(target).astype(np.int64) + np.arange(-4, 5):
                amax = _bits_to_f32(np.uint16(ab))
                if amax < x:
                    continue
                blk = _f32_to_bits_trunc((rng.uniform(-1, 1, 16) * x).astype(np.float32))
                blk[0] = np.uint16(ab)
                blk[7] = xb | (np.uint16(rng.integers(0, 2)) << 15)
                sc2, cdiv, cmul = _nvfp4_codes(_bits_to_f32(blk), gs)
                if sc2 == sc and cdiv[7] != cmul[7]:
                    row = np.concatenate([blk] + [
                        _f32_to_bits_trunc(rng.standard_normal(16).astype(np.float32) * np.float32(gs * 2000))
                        for _ in range(blocks - 1)])
                    mask = np.zeros(16 * blocks, dtype=bool)
                    mask[:16] = cdiv != cmul
                    out.append((np.float32(gs), row[None, :], mask[None, :]))
                    break
            break
    return out
