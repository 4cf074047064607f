"""Velocity-Verlet molecular dynamics in float64 (oracle).

Test infrastructure only (see the package docstring). Tessera page, "ten-million-atom
trajectories": the MD engine integrates the atoms locally every step and reuses the neighbor
topology while the coordinates move; it checks the run by the energy drift of a microcanonical
(NVE) simulation. FlashSchNet page, headline speed: MD throughput of batched replicas. Neither page
names the integrator; the reading here is the plain velocity-Verlet scheme (the standard symplectic
NVE integrator): per step, with a_i = F_i / m_i,

    v <- v + (dt/2) a(r);   r <- r + dt v;   v <- v + (dt/2) a(r_new).

The force routine is a parameter, so the integrator can be checked on closed-form systems.
"""
from __future__ import annotations

import numpy as np


def kinetic_energy(vel, inv_mass=None, graph_ptr=None) -> np.ndarray:
    """Per-graph kinetic energy sum_i m_i |v_i|^2 / 2 (float64 [G]); inv_mass = 1/m_i or None (1)."""
    v = np.asarray(vel, dtype=np.float64)
    m = 1.0 if inv_mass is None else 1.0 / np.asarray(inv_mass, dtype=np.float64)
    ke = 0.5 * m * np.sum(v * v, axis=1)
    gp = [0, len(v)] if graph_ptr is None else list(np.asarray(graph_ptr, dtype=np.int64))
    return np.array([ke[gp[g]:gp[g + 1]].sum() for g in range(len(gp) - 1)])


def velocity_verlet(force_fn, pos, vel, forces, dt: float, n_steps: int, inv_mass=None):
    """n_steps velocity-Verlet steps from (pos, vel) with ``forces`` = force_fn(pos)[1] on entry.

    force_fn(pos) -> (energy, forces). Returns (pos, vel, forces, energy) after the last step
    (energy None when n_steps = 0), all float64 copies; the inputs are not modified.
    """
    r = np.array(pos, dtype=np.float64)
    v = np.array(vel, dtype=np.float64)
    f = np.array(forces, dtype=np.float64)
    im = np.ones(len(r)) if inv_mass is None else np.asarray(inv_mass, dtype=np.float64)
    energy = None
    for _ in range(n_steps):
        v = v + 0.5 * dt * f * im[:, None]
        r = r + dt * v
        energy, f = force_fn(r)
        f = np.asarray(f, dtype=np.float64)
        v = v + 0.5 * dt * f * im[:, None]
    return r, v, f, energy
