"""K-RPBH rotation of V rows (oracle side; TEST INFRASTRUCTURE ONLY).

Follows "SoloQ: Calibration-Free Quantization for Diffusion Language Models"
(method paragraph on K-RPBH): a random permutation of the coordinates, a
Hadamard transform inside each block of b coordinates, then a k x k random
orthogonal mix that combines the same in-block coordinate across the k = d/b
blocks (k = 1 is plain RPBH).  For a row vector x of length d = k*b:

    y[i]         = x[perm[i]]                              permutation
    y[r*b:(r+1)*b] <- y[r*b:(r+1)*b] @ H_b / sqrt(b)       per-block Hadamard
    w[r*b + i]   = sum_c mix[r, c] * y[c*b + i]            cross-block mix

H_b is the Sylvester Hadamard matrix (H_1 = [1], H_2n = [[H, H], [H, -H]]),
mix is orthogonal, so the whole map is orthogonal and its inverse applies
mix^T, then H_b / sqrt(b), then the inverse permutation.

Rotated-V cache (the "rotated V path" the SoloQ KV paragraph pairs with
commit-time quantization): each committed V row is rotated before its
per-token quantization; attention sums dequantized rotated rows and the
output is rotated back.  Because the codes depend on the last bit of the
rotated fp32 values, the fp32 evaluation order is part of the definition (the
pages fix none): inputs in fp32; the Hadamard as butterflies
(lo, hi) -> (lo + hi, lo - hi) over strides h = 1, 2, 4, ..., b/2; one fp32
multiply by fp32(1/sqrt(b)); the mix as a left-to-right fp32 sum over c of
fp32 products, starting from 0.  No fused multiply-add anywhere.

Pins (tests/test_oracle_pins.py): the Hadamard against scipy.linalg.hadamard,
orthogonality of the assembled matrix, the inverse, k = 1 against a scaled
Hadamard of the permuted vector, and the fp32 order against the fp64 map on
inputs where no step rounds.
"""
from __future__ import annotations

import numpy as np


def hadamard_f64(b: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order b (a power of two), fp64."""
    assert b >= 1 and b & (b - 1) == 0
    H = np.ones((1, 1))
    while H.shape[0] < b:
        H = np.block([[H, H], [H, -H]])
    return H


def check_params(perm, mix, b: int, d: int = 128):
    perm = np.asarray(perm, np.int64)
    mix = np.asarray(mix, np.float64)
    k = d // b
    assert b * k == d and b & (b - 1) == 0
    assert perm.shape == (d,) and np.array_equal(np.sort(perm), np.arange(d))
    assert mix.shape == (k, k)
    return perm, mix, k


def rotate_f64(x, perm, mix, b: int) -> np.ndarray:
    """The rotation in fp64 (exact map up to fp64 rounding), over the last axis."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    perm, mix, k = check_params(perm, mix, b, d)
    y = x[..., perm].reshape(x.shape[:-1] + (k, b))
    y = y @ (hadamard_f64(b) / np.sqrt(b))
    w = np.einsum("rc,...ci->...ri", mix, y)
    return w.reshape(x.shape)


def unrotate_f64(w, perm, mix, b: int) -> np.ndarray:
    """Inverse of rotate_f64: mix^T, per-block H_b / sqrt(b), inverse permutation."""
    w = np.asarray(w, np.float64)
    d = w.shape[-1]
    perm, mix, k = check_params(perm, mix, b, d)
    y = np.einsum("rc,...ri->...ci", mix, w.reshape(w.shape[:-1] + (k, b)))
    y = (y @ (hadamard_f64(b) / np.sqrt(b))).reshape(w.shape)
    x = np.empty_like(y)
    x[..., perm] = y
    return x


def rotation_matrix_f64(perm, mix, b: int, d: int = 128) -> np.ndarray:
    """R with rotate_f64(x) = x @ R (rows of the identity, rotated)."""
    return rotate_f64(np.eye(d), perm, mix, b)


def rotate_f32(x, perm, mix, b: int) -> np.ndarray:
    """The rotation evaluated in fp32 in the order stated in the module
    docstring (the order that decides the rotated values' last bit)."""
    x = np.asarray(x, np.float32)
    d = x.shape[-1]
    perm, mix, k = check_params(perm, mix, b, d)
    y = x[..., perm].reshape(x.shape[:-1] + (k, b)).copy()
    h = 1
    while h < b:
        # butterflies on pairs (i, i + h) with bit h of i clear
        z = y.reshape(y.shape[:-1] + (b // (2 * h), 2, h))
        lo = z[..., 0, :].copy()
        hi = z[..., 1, :].copy()
        z[..., 0, :] = lo + hi
        z[..., 1, :] = lo - hi
        y = z.reshape(y.shape)
        h *= 2
    y = y * np.float32(1.0 / np.sqrt(b))
    m32 = mix.astype(np.float32)
    w = np.zeros_like(y)
    for r in range(k):
        acc = np.zeros(y.shape[:-2] + (b,), np.float32)
        for c in range(k):
            acc = acc + m32[r, c] * y[..., c, :]
        w[..., r, :] = acc
    return w.reshape(x.shape)


def f32_to_bf16_bits(x) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (NaN kept
    as a quiet NaN).  Pinned against a brute-force nearest search."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    nan = np.isnan(np.asarray(x, np.float32))
    r = np.where(nan, (u >> np.uint64(16)) | np.uint64(0x40), r)
    return r.astype(np.uint16)

