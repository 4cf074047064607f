"""Plain, slow, fp64 CPU oracle for fused neighbor-list message passing.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import or call anything in this package. The product path
(``atomistic_neighbor_list_b200``) never imports it, and this package never imports the product path:
the two share nothing but the seeded input generator ``atomistic_neighbor_list_b200.synth``, which the
tests call and hand to both sides.

Every function computes a plain definition in float64 (NumPy; library primitives -- a matmul, a sort,
a sparse row sum, a k-d tree candidate search -- serve as single steps). Edges are visited in CSR
order and processed in contiguous destination-row ranges only to bound memory; every output row is
computed by the same formula whatever the chunking.

Sources (page titles, sections):

* FlashSchNet: Fast and Accurate Coarse-Grained Neural Network Molecular Dynamics -- technical summary
  section 1 (bottlenecks), 2.1 Flash Radial Basis (distance, Gaussian basis, cosine envelope),
  2.2 Flash Message Passing (cutoff mask, gather, filter multiply, reduce), 2.3 Flash Aggregation
  (destination-sorted CSR segment reduce; source-grouped reduce in the backward), 2.4 channel-wise
  16-bit quantization (fp32 positions, distances, energy accumulation and forces).
* E2Former-V2 page -- section 3.1 node-centric message passing and section 3.2 the fused kernel
  (online softmax with running maximum and normaliser, each key/value loaded once, padded
  neighbors masked); section 5.2 (verify the neighbor list).
* Tessera page -- forces as the gradient of the energy with respect to the positions.

The pages print none of the SchNet formulas; the readings used (Gaussian form and centres, cosine
envelope on the filter output, shifted softplus after the first filter layer, block and readout
layout, neighbor truncation for the capped list) are listed in the design notes and restated in each
function's docstring. Parity of those architecture choices is unpinned by the pages: they are fixed
only by the written specification that both this oracle and the CUDA path follow.
"""
from .neighbors import cutoff_sq, pair_d2, neighbor_csr, neighbor_padded  # noqa: F401
from .schnet import (  # noqa: F401
    LN2, rbf_centres, gaussian_rbf, gaussian_rbf_grad, cosine_cutoff, cosine_cutoff_grad, ssp,
    ssp_grad, filter_weights, cfconv, cfconv_pairs, undirected_pairs, Model, energies, energy_forces,
)
from .attention import (  # noqa: F401
    attention, attention_vjp, attention_equivariant, solid_harmonics, moments_to_solid,
)
from .md import kinetic_energy, velocity_verlet  # noqa: F401
