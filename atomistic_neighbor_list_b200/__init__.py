"""B200-native fused neighbor-list message passing (SchNet cfconv, neighbor attention, forces).

``atomistic_neighbor_list_b200.mp`` is the Python binding of the C-ABI library ``libmp.so``;
``atomistic_neighbor_list_b200.synth`` makes the seeded synthetic inputs.
"""
__version__ = "0.1.0"
