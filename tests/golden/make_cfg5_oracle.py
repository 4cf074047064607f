"""Write cfg5_oracle.npz: the fp64 oracle's energy and forces of the 100,000-atom workload.

Calls only the oracle (and the seeded input generator for its inputs), never the CUDA path:
100,000 atoms uniform at 0.1 atoms/A^3 (positions default_rng(0), types default_rng(1), weights
default_rng(2)), cutoff 5 A, 3 interaction blocks, F = 128, 50 radial functions, weights rounded to
bf16 as the library holds them for the bf16 path. Stored: the energy E, the sum of |atomic
energies| (the scale of the energy tolerance), the forces as float32 [N, 3] (the float64 values
rounded once; the bf16 force bound is 1e-2 relative), and a digest of the positions and types so a
test can check that it is comparing the same system. Takes about ten minutes on eight cores.

    python tests/golden/make_cfg5_oracle.py
"""
import hashlib
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from atomistic_neighbor_list_b200 import synth  # noqa: E402


def input_digest(pos, types) -> str:
    h = hashlib.sha256()
    h.update(np.ascontiguousarray(pos, dtype=np.float32).tobytes())
    h.update(np.ascontiguousarray(types, dtype=np.int32).tobytes())
    return h.hexdigest()[:16]


def main():
    wl = synth.WORKLOADS["cfg5"]
    pos, _ = synth.positions_for(wl)
    types = synth.atom_types(len(pos), wl.n_types)
    weights = {k: synth.round_bf16(v) for k, v in synth.make_weights(wl).items()}
    model = oracle.Model.from_workload(wl, weights)
    rp, ci = oracle.neighbor_csr(pos, wl.r_c)
    E, F, e_atom = oracle.energy_forces(model, pos, types, rp, ci, return_atom_energy=True)
    np.savez_compressed(os.path.join(HERE, "cfg5_oracle.npz"), energy=E,
                        energy_scale=np.array([np.abs(e_atom).sum()]),
                        forces=F.astype(np.float32), edges=np.array([len(ci)]),
                        digest=np.array([input_digest(pos, types)]))


if __name__ == "__main__":
    main()
