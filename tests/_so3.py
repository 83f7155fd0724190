"""Rotation tools for the equivariance tests (test-only).

Rotations are drawn uniformly on SO(3) from uniform unit quaternions (the
TransIP page samples its rotations uniformly from SO(3) for the equivariance
pairs of its training pipeline; the definition of equivariance it states,
f(phi(g) x) = rho(g) f(x), is the property these tests check).

Wigner-D matrices are fitted in FP64 by least squares from the oracle's own
spherical harmonics: D^l(R) is the matrix with Y_l(R r) = D^l(R) Y_l(r) for
every unit vector r.  Their orthogonality, determinant and group property are
checked in test_oracle_sh.py before the equivariance tests rely on them.
"""
import numpy as np

import oracle as O


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    u1, u2, u3 = rng.random(3)
    q = np.array([np.sqrt(1 - u1) * np.sin(2 * np.pi * u2), np.sqrt(1 - u1) * np.cos(2 * np.pi * u2),
                  np.sqrt(u1) * np.sin(2 * np.pi * u3), np.sqrt(u1) * np.cos(2 * np.pi * u3)])
    x, y, z, w = q
    return np.array([
        [1 - 2 * (y * y + z * z), 2 * (x * y - z * w), 2 * (x * z + y * w)],
        [2 * (x * y + z * w), 1 - 2 * (x * x + z * z), 2 * (y * z - x * w)],
        [2 * (x * z - y * w), 2 * (y * z + x * w), 1 - 2 * (x * x + y * y)],
    ])


def wigner_d(l: int, R: np.ndarray, npts: int = 64, seed: int = 7) -> np.ndarray:
    rng = np.random.default_rng(seed)
    P = rng.standard_normal((npts, 3))
    P /= np.linalg.norm(P, axis=1, keepdims=True)
    sl = slice(l * l, (l + 1) * (l + 1))
    A = O.sph_harm(l, P)[:, sl]
    B = O.sph_harm(l, P @ R.T)[:, sl]
    Dt, *_ = np.linalg.lstsq(A, B, rcond=None)
    return Dt.T


def block_rotation(irreps, R: np.ndarray, parity: int = 1) -> np.ndarray:
    """Dense representation matrix of an irreps list under R (and, with
    parity=-1, composed with inversion: each irrep picks up its parity)."""
    blocks = []
    for mul, l, p in irreps:
        D = wigner_d(l, R)
        if parity < 0 and p < 0:
            D = -D
        blocks.extend([D] * mul)
    n = sum(b.shape[0] for b in blocks)
    M = np.zeros((n, n))
    o = 0
    for b in blocks:
        k = b.shape[0]
        M[o:o + k, o:o + k] = b
        o += k
    return M
