"""Seeded synthetic inputs shaped like the systems on the Tessera pages.

This module only draws positions; it holds none of the neighbor-list
arithmetic (no wrapping, curve keys, cells or distances), so both the GPU
tests and the CPU oracle can take their inputs from it.

Workloads (stand-ins for the pages' systems; no structure file is used):

=========== ============ ======== ========================= ===== ===========================
name        atoms        box (A)  cutoff / skin (A)         cap.  structure
=========== ============ ======== ========================= ===== ===========================
uniform4k   4,096        34.47    5.75 / 1.0                256   uniform random
lattice60k  59,319       84.023   5.75 / 1.0                256   39^3 sc lattice, jitter 0.3
saltwater1m 981,975      214.256  6.0 / 1.5                 320   rigid water + 0.15 M NaCl
saltwater10m 10,291,605  468.880  5.75 / 1.0                256   as above, 151^3 sites
shell10m    10,060,000   462.949  5.75 / 1.0                320   0.12 A^-3 shell in 0.1 fill
=========== ============ ======== ========================= ===== ===========================

The per-layer cutoff 5.75 A is the four-layer, 23 A receptive field of the
Tessera abstract divided by four.  Densities: 0.1 atoms/A^3 (water-like),
0.0334 molecules/A^3 for water.  Random draws are numpy PCG64 in float64,
cast to float32 at the end; atom order is shuffled by a seeded permutation.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

AVOGADRO_PER_A3_M = 6.02214076e-4  # (mol/L) -> particles per cubic angstrom


@dataclasses.dataclass
class Workload:
    name: str
    pos: np.ndarray          # float32 [n, 4]; column 3 is zero (ignored)
    box: np.ndarray          # float32 [3]
    cutoff: float
    skin: float
    capacity: int
    sigma_step: float = 0.02     # per-step displacement (A) for skin-check loops
    steps: int = 0               # skin-check loop length for this workload
    description: str = ""

    @property
    def n(self) -> int:
        return int(self.pos.shape[0])


def _finish(xyz: np.ndarray, rng: np.random.Generator, shuffle: bool = True) -> np.ndarray:
    if shuffle:
        xyz = xyz[rng.permutation(xyz.shape[0])]
    out = np.zeros((xyz.shape[0], 4), np.float32)
    out[:, :3] = xyz.astype(np.float32)
    return out


def uniform_box(n: int, L: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return _finish(rng.random((n, 3)) * L, rng, shuffle=False)


def jittered_lattice(nside: int, spacing: float, sigma: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    g = np.arange(nside, dtype=np.float64) * spacing + 0.5 * spacing
    X, Y, Z = np.meshgrid(g, g, g, indexing="ij")
    xyz = np.stack([X.ravel(), Y.ravel(), Z.ravel()], axis=1)
    xyz += rng.normal(0.0, sigma, xyz.shape)
    return _finish(xyz, rng)


def _random_rotations(m: int, rng: np.random.Generator) -> np.ndarray:
    """Uniform random rotation matrices (Shoemake's quaternion construction)."""
    u1, u2, u3 = rng.random(m), rng.random(m), rng.random(m)
    a, b = np.sqrt(1.0 - u1), np.sqrt(u1)
    qx, qy = a * np.sin(2 * np.pi * u2), a * np.cos(2 * np.pi * u2)
    qz, qw = b * np.sin(2 * np.pi * u3), b * np.cos(2 * np.pi * u3)
    R = np.empty((m, 3, 3))
    R[:, 0, 0] = 1 - 2 * (qy * qy + qz * qz)
    R[:, 0, 1] = 2 * (qx * qy - qz * qw)
    R[:, 0, 2] = 2 * (qx * qz + qy * qw)
    R[:, 1, 0] = 2 * (qx * qy + qz * qw)
    R[:, 1, 1] = 1 - 2 * (qx * qx + qz * qz)
    R[:, 1, 2] = 2 * (qy * qz - qx * qw)
    R[:, 2, 0] = 2 * (qx * qz - qy * qw)
    R[:, 2, 1] = 2 * (qy * qz + qx * qw)
    R[:, 2, 2] = 1 - 2 * (qx * qx + qy * qy)
    return R


def salt_water(nside: int, seed: int, density: float = 0.0334, jitter: float = 0.3,
               molarity: float = 0.15, r_oh: float = 0.96, hoh_deg: float = 104.5):
    """Rigid water on a jittered simple-cubic lattice, Na+/Cl- replacing waters.

    Returns (positions float32 [n, 4], box side L).  One oxygen per lattice
    site (spacing density**(-1/3), Gaussian jitter), two hydrogens at r_oh
    with the H-O-H angle hoh_deg in a uniformly random orientation.  P =
    round(molarity * 6.022e-4 * L^3) random sites become Na+ (first P) and
    Cl- (next P), one atom at the site.
    """
    rng = np.random.default_rng(seed)
    a = density ** (-1.0 / 3.0)
    L = nside * a
    g = np.arange(nside, dtype=np.float64) * a + 0.5 * a
    X, Y, Z = np.meshgrid(g, g, g, indexing="ij")
    sites = np.stack([X.ravel(), Y.ravel(), Z.ravel()], axis=1)
    sites += rng.normal(0.0, jitter, sites.shape)
    nsite = sites.shape[0]
    P = int(round(molarity * AVOGADRO_PER_A3_M * L ** 3))
    chosen = rng.choice(nsite, size=2 * P, replace=False)
    is_ion = np.zeros(nsite, bool)
    is_ion[chosen] = True
    ions = sites[chosen]
    oxy = sites[~is_ion]
    half = math.radians(hoh_deg) / 2.0
    body = np.array([[r_oh * math.sin(half), 0.0, r_oh * math.cos(half)],
                     [-r_oh * math.sin(half), 0.0, r_oh * math.cos(half)]])
    R = _random_rotations(oxy.shape[0], rng)
    h1 = oxy + R @ body[0]
    h2 = oxy + R @ body[1]
    xyz = np.concatenate([oxy, h1, h2, ions], axis=0)
    return _finish(xyz, rng), L


def shell_in_fill(n_shell: int, n_fill: int, L: float, r_in: float, r_out: float,
                  seed: int) -> np.ndarray:
    """Uniform spherical shell (r_in <= r < r_out about the box centre) plus a
    uniform fill everywhere outside the shell, by rejection."""
    rng = np.random.default_rng(seed)
    c = np.full(3, L / 2.0)
    u = rng.random(n_shell)
    r = np.cbrt(r_in ** 3 + u * (r_out ** 3 - r_in ** 3))
    v = rng.normal(size=(n_shell, 3))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    shell = c + v * r[:, None]
    fill = np.empty((0, 3))
    while fill.shape[0] < n_fill:
        m = int((n_fill - fill.shape[0]) * 1.1) + 1024
        p = rng.random((m, 3)) * L
        d = np.linalg.norm(p - c, axis=1)
        keep = p[(d < r_in) | (d >= r_out)]
        fill = np.concatenate([fill, keep], axis=0)
    fill = fill[:n_fill]
    return _finish(np.concatenate([shell, fill], axis=0), rng)


def _cube(L: float) -> np.ndarray:
    return np.full(3, L, np.float32)


def make(name: str, seed: int | None = None) -> Workload:
    """Named workloads; default seeds 1..5 in the order of the table above."""
    if name == "uniform4k":
        L = 34.47
        pos = uniform_box(4096, L, 1 if seed is None else seed)
        return Workload(name, pos, _cube(L), 5.75, 1.0, 256, description=
                        "4,096 atoms uniform random at 0.1/A^3, cubic box 34.47 A")
    if name == "lattice60k":
        a = 0.1 ** (-1.0 / 3.0)
        pos = jittered_lattice(39, a, 0.3, 2 if seed is None else seed)
        return Workload(name, pos, _cube(39 * a), 5.75, 1.0, 256, steps=50,
                        description="59,319 atoms, 39^3 sc lattice at 0.1/A^3, jitter 0.3 A")
    if name == "saltwater1m":
        pos, L = salt_water(69, 3 if seed is None else seed)
        return Workload(name, pos, _cube(L), 6.0, 1.5, 320, description=
                        "981,975 atoms rigid water + 0.15 M NaCl, 69^3 sites")
    if name == "saltwater10m":
        pos, L = salt_water(151, 4 if seed is None else seed)
        return Workload(name, pos, _cube(L), 5.75, 1.0, 256, steps=200, description=
                        "10,291,605 atoms rigid water + 0.15 M NaCl, 151^3 sites")
    if name == "shell10m":
        vol_shell = 4.0 / 3.0 * math.pi * (150.0 ** 3 - 120.0 ** 3)
        n_shell = int(round(0.12 * vol_shell))
        n_fill = 10_060_000 - n_shell
        L = (n_fill / 0.1 + vol_shell) ** (1.0 / 3.0)
        pos = shell_in_fill(n_shell, n_fill, L, 120.0, 150.0, 5 if seed is None else seed)
        return Workload(name, pos, _cube(L), 5.75, 1.0, 320, description=
                        "10,060,000 atoms: 0.12/A^3 shell r 120-150 A in 0.1/A^3 fill")
    if name.startswith("saltwater_n"):
        nside = int(name[len("saltwater_n"):])
        pos, L = salt_water(nside, 7 if seed is None else seed)
        return Workload(name, pos, _cube(L), 5.75, 1.0, 256, description=
                        f"rigid water + 0.15 M NaCl on {nside}^3 sites")
    raise KeyError(name)


NAMES = ("uniform4k", "lattice60k", "saltwater1m", "saltwater10m", "shell10m")

# (atoms, cutoff, skin, capacity, description) of the named workloads, for
# reports that name a workload without generating it
INFO = {
    "uniform4k": (4096, 5.75, 1.0, 256, "4,096 atoms uniform random at 0.1/A^3, cubic box 34.47 A"),
    "lattice60k": (59319, 5.75, 1.0, 256, "59,319 atoms, 39^3 sc lattice at 0.1/A^3, jitter 0.3 A"),
    "saltwater1m": (981975, 6.0, 1.5, 320, "981,975 atoms rigid water + 0.15 M NaCl, 69^3 sites"),
    "saltwater10m": (10291605, 5.75, 1.0, 256,
                     "10,291,605 atoms rigid water + 0.15 M NaCl, 151^3 sites"),
    "shell10m": (10060000, 5.75, 1.0, 320,
                 "10,060,000 atoms: 0.12/A^3 shell r 120-150 A in 0.1/A^3 fill"),
}
