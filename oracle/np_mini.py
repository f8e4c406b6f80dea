"""Second, independent oracle in numpy, for cross-checking the C oracle on tiny
inputs.  TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

It is written separately from kvq_oracle.c: the rotation is a numpy fp64
matrix product (FWHT mode builds the explicit permuted Hadamard matrix),
binary16 rounding is numpy's float16 cast, and decode works on logical
(unpacked) codes instead of the byte format.
"""
import numpy as np

D = 128
GS = 32


def hadamard(n):
    """Sylvester Hadamard matrix H[i][j] = (-1)^popcount(i & j)."""
    i = np.arange(n)
    bits = np.bitwise_and.outer(i, i)
    pc = np.zeros_like(bits)
    while bits.any():
        pc += bits & 1
        bits >>= 1
    return np.where(pc % 2 == 0, 1.0, -1.0)


def rotation_matrix(mode, R=None, perm=None):
    """Dense fp64 matrix M with x_rot = x @ M.  FWHT mode: y[i] = x[perm[i]],
    x_rot = y @ H / sqrt(128), so M[perm[i], :] = H[i, :] / sqrt(128)."""
    if mode == 0:
        return np.asarray(R, np.float64)
    H = hadamard(D) / np.sqrt(D)
    M = np.zeros((D, D))
    M[np.asarray(perm), :] = H
    return M


def rotate_rows_f32(x_f16, mode, R=None, perm=None):
    x = np.asarray(x_f16, np.float16).astype(np.float64).reshape(-1, D)
    return (x @ rotation_matrix(mode, R, perm)).astype(np.float32)


def quantize_rows(x):
    """Same grid as the C oracle, written with numpy float32 scalars."""
    x = np.asarray(x, np.float32).reshape(-1, D)
    n = x.shape[0]
    codes = np.zeros((n, D), np.uint8)
    s = np.zeros((n, 4), np.float16)
    z = np.zeros((n, 4), np.float16)
    three = np.float32(3.0)
    zero = np.float32(0.0)
    for r in range(n):
        for g in range(4):
            xg = x[r, g * GS:(g + 1) * GS]
            mn = np.float32(xg.min())
            mx = np.float32(xg.max())
            sh = np.float16((mx - mn) / three + zero)
            zh = np.float16(mn + zero)
            sf = np.float32(sh)
            inv = np.float32(0.0) if sf == 0 else np.float32(np.float32(1.0) / sf)
            t = (xg - np.float32(zh)).astype(np.float32) * inv
            c = np.clip(np.rint(t.astype(np.float32)), 0, 3).astype(np.uint8)
            codes[r, g * GS:(g + 1) * GS] = c
            s[r, g] = sh
            z[r, g] = zh
    return codes, s.view(np.uint16), z.view(np.uint16)


def dequant(codes, s_bits, z_bits):
    s = np.asarray(s_bits, np.uint16).view(np.float16).astype(np.float64)
    z = np.asarray(z_bits, np.uint16).view(np.float16).astype(np.float64)
    g = np.arange(D) // GS
    return codes.astype(np.float64) * s[..., g] + z[..., g]


def decode_one(q_f16, khat, vhat, mode, Rk=None, Rv=None, pk=None, pv=None):
    """q fp16 [128]; khat, vhat fp64 [L,128] in the rotated domain."""
    Mk = rotation_matrix(mode, Rk, pk)
    Mv = rotation_matrix(mode, Rv, pv)
    q = np.asarray(q_f16, np.float16).astype(np.float64) @ Mk
    s = khat @ q / np.sqrt(D)
    p = np.exp(s - s.max())
    o = (p / p.sum()) @ vhat
    return o @ Mv.T


# --- pre-RoPE grouped-head rotation ------------------------------------------------------

def group_rotation_matrix(perm):
    """x_rot = x @ M for a group row of n = len(perm) channels:
    y[i] = x[perm[i]], x_rot = y @ H_n / sqrt(n)."""
    n = len(perm)
    M = np.zeros((n, n))
    M[np.asarray(perm), :] = hadamard(n) / np.sqrt(n)
    return M


def rope_complex(x, t, base):
    """RoPE with rotate-half pairing as a complex rotation: channel c < 64
    and c + 64 are the real and imaginary parts of z_c, turned by t*theta_c,
    theta_c = base^(-2c/128)."""
    x = np.asarray(x, np.float64)
    z = x[:D // 2] + 1j * x[D // 2:]
    theta = np.power(float(base), -2.0 * np.arange(D // 2) / D)
    z = z * np.exp(1j * t * theta)
    return np.concatenate([z.real, z.imag])


def decode_prerope_one(q_f16, kgroup_hat, j, perm_group, base, vhat, pv, sink_keys=None):
    """q fp16 [128] post-RoPE; kgroup_hat fp64 [L, n] rotated group key rows
    (dequantised); j the head's slot in its group; vhat fp64 [L,128] rotated
    value rows; pv the head's value permutation; sink_keys {t: pre-RoPE key
    row} for positions kept in fp16 (their kgroup_hat rows are ignored)."""
    q = np.asarray(q_f16, np.float16).astype(np.float64)
    M = group_rotation_matrix(perm_group)
    kpre = kgroup_hat @ M.T                        # inverse of an orthogonal map
    sink_keys = sink_keys or {}
    k = np.stack([rope_complex(sink_keys[t] if t in sink_keys else kpre[t, j * D:(j + 1) * D],
                               t, base) for t in range(kpre.shape[0])])
    s = k @ q / np.sqrt(D)
    p = np.exp(s - s.max())
    o = (p / p.sum()) @ vhat
    return o @ rotation_matrix(1, perm=pv).T
