"""Python binding of libmp (include/mp.h): argument marshalling only.

Every computation runs in the library's CUDA kernels; this module checks tensor shapes, dtypes and
devices, passes raw device pointers and the current CUDA stream, and raises ``MpError`` on a non-zero
status. There is no fallback: if ``libmp.so`` is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_longlong, c_void_p

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmp.so")
MAX_BLOCKS = 8
FP32, BF16 = 0, 1

_STATUS = {0: "MP_OK", -1: "MP_ERR_INVALID_ARG", -2: "MP_ERR_BAD_CSR", -3: "MP_ERR_CSR_UNSORTED",
           -4: "MP_ERR_CSR_NOT_SYMMETRIC", -5: "MP_ERR_CAPACITY", -6: "MP_ERR_CUDA",
           -7: "MP_ERR_DEVICE_BOUNDS", -8: "MP_ERR_TIMEOUT", -9: "MP_ERR_UNIMPLEMENTED"}


class MpError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        self.name = _STATUS.get(status, str(status))
        super().__init__(f"{what}: {self.name} ({lib.mp_strerror(status).decode()})")


class MpConfig(ctypes.Structure):
    _fields_ = [("F", c_int), ("n_rbf", c_int), ("n_blocks", c_int), ("n_types", c_int),
                ("n_heads", c_int), ("head_dim", c_int), ("r_c", c_float), ("gamma", c_float),
                ("mu_min", c_float), ("mu_max", c_float), ("dtype", c_int), ("max_atoms", c_int),
                ("max_edges", c_longlong), ("max_graphs", c_int), ("validate", c_int)]


_FP = POINTER(c_float)


class MpWeights(ctypes.Structure):
    _fields_ = [("emb", _FP)] + [(k, _FP * MAX_BLOCKS) for k in (
        "A1", "c1", "A2", "c2", "W_in", "b_in", "W_out", "b_out")] + \
        [(k, _FP) for k in ("B1", "d1", "B2", "d2", "Wq", "Wk", "P", "p")] + [("on_device", c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built (run `python -m atomistic_neighbor_list_b200.build`);"
                          " there is no CPU or fallback path")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = c_void_p, c_int, c_longlong
    sig = {
        "mp_init": (i32, [POINTER(vp), POINTER(MpConfig), POINTER(MpWeights), vp]),
        "mp_destroy": (None, [vp]),
        "mp_strerror": (c_char_p, [i32]),
        "mp_status_sync": (i32, [vp, vp]),
        "mp_neighbor_csr": (i32, [i32, vp, vp, i32, c_float, vp, vp, i64, POINTER(i64), vp]),
        "mp_neighbor_padded": (i32, [i32, vp, vp, i32, c_float, i32, vp, vp, vp]),
        "mp_cfconv_fwd": (i32, [vp, i32, i32, i64, vp, vp, vp, vp, vp, vp]),
        "mp_attn_fwd": (i32, [vp, i32, i32, vp, vp, vp, vp, vp, vp]),
        "mp_energy_forces": (i32, [vp, i32, i64, vp, vp, vp, vp, vp, i32, vp, vp, vp]),
        "mp_profile_begin": (i32, [vp]),
        "mp_profile_end": (i32, [vp, vp]),
        "mp_profile_get": (i32, [vp, i32, POINTER(c_char_p), POINTER(c_double), POINTER(i64)]),
        "mp_launch_count": (i64, [vp]),
        "mp_set_wait_budget": (i32, [vp, i64]),
        "mp_pair_plan": (i32, [vp, i32, i64, vp, vp, vp]),
        "mp_shard_graphs": (i32, [vp, i32, i32, i32, POINTER(i32), POINTER(i32)]),
        "mp_cfconv_fwd_pairs": (i32, [vp, i32, i32, vp, vp, vp, vp]),
        "mp_set_graphs": (i32, [vp, i32]),
        "mp_md_verlet": (i32, [vp, i32, i64, vp, vp, vp, vp, c_float, i32, vp, vp, vp, vp, i32,
                               vp, vp, vp]),
        "mp_attn_bwd": (i32, [vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]),
        "mp_attn_eq_fwd": (i32, [vp, i32, i32, vp, vp, vp, vp, vp, vp]),
        "mp_spatial_order": (i32, [i32, vp, vp, i32, c_float, vp, vp]),
        "mp_md_run": (i32, [vp, i32, vp, vp, vp, vp, c_float, i32, vp, vp, i32, c_float, i32,
                            c_float, i32, vp, vp, i64, POINTER(i64), vp, vp, POINTER(i32), vp]),
        "mp_selftest_tc": (i32, [POINTER(i32)]),
        "mp_attn_fwd_noalloc": (i32, [POINTER(MpConfig), POINTER(MpWeights), i32, i32, vp, vp, vp,
                                      vp, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()

EXPORTED = ("mp_init", "mp_destroy", "mp_strerror", "mp_status_sync", "mp_neighbor_csr",
            "mp_neighbor_padded", "mp_cfconv_fwd", "mp_attn_fwd", "mp_energy_forces",
            "mp_profile_begin", "mp_profile_end", "mp_profile_get", "mp_launch_count",
            "mp_attn_fwd_noalloc", "mp_selftest_tc", "mp_set_graphs",
            "mp_md_verlet", "mp_md_run", "mp_attn_bwd", "mp_attn_eq_fwd", "mp_spatial_order",
            "mp_set_wait_budget", "mp_pair_plan", "mp_cfconv_fwd_pairs", "mp_shard_graphs")
NOALLOC_MAX_NF = 524288  # MP_NOALLOC_MAX_NF: largest N * F mp_attn_fwd_noalloc accepts


def _check(status: int, what: str):
    if status != 0:
        raise MpError(status, what)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return c_void_p(s.cuda_stream)


def _ptr(t):
    return c_void_p(t.data_ptr()) if t is not None else c_void_p(0)


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


class Context:
    """One model on one device: owns copied weights and an O(max_atoms * F) workspace."""

    def __init__(self, *, F: int, n_rbf: int, n_blocks: int, r_c: float, weights: dict,
                 max_atoms: int, max_edges: int, dtype: str = "bf16", n_types: int = 10,
                 gamma: float = 10.0, mu_min: float = 0.0, mu_max: float | None = None,
                 n_heads: int = 0, head_dim: int = 0, max_graphs: int = 1,
                 validate: bool = False):
        self.F, self.n_rbf, self.n_blocks = F, n_rbf, n_blocks
        self.dtype = dtype
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.n_heads, self.head_dim = n_heads, head_dim
        cfg = MpConfig(F=F, n_rbf=n_rbf, n_blocks=n_blocks, n_types=n_types, n_heads=n_heads,
                       head_dim=head_dim, r_c=r_c, gamma=gamma, mu_min=mu_min,
                       mu_max=r_c if mu_max is None else mu_max,
                       dtype=BF16 if dtype == "bf16" else FP32, max_atoms=max_atoms,
                       max_edges=max_edges, max_graphs=max_graphs, validate=int(validate))
        keep = []

        def arr(name):
            if name not in weights:
                return None
            a = np.ascontiguousarray(weights[name], dtype=np.float32)
            keep.append(a)
            return a.ctypes.data_as(_FP)

        w = MpWeights()
        w.emb = arr("emb")
        for b in range(min(n_blocks, MAX_BLOCKS)):
            for k in ("A1", "c1", "A2", "c2", "W_in", "b_in", "W_out", "b_out"):
                p = arr(f"{k}.{b}")
                if p is not None:
                    getattr(w, k)[b] = p
        for k in ("B1", "d1", "B2", "d2", "Wq", "Wk", "P", "p"):
            p = arr(k)
            if p is not None:
                setattr(w, k, p)
        w.on_device = 0
        self._ctx = c_void_p()
        _check(lib.mp_init(ctypes.byref(self._ctx), ctypes.byref(cfg), ctypes.byref(w),
                           _stream()), "mp_init")
        self.max_atoms, self.max_edges = max_atoms, max_edges

    @classmethod
    def from_workload(cls, wl, weights, max_atoms, max_edges, max_graphs=1, validate=False):
        return cls(F=wl.F, n_rbf=wl.n_rbf, n_blocks=wl.n_blocks, r_c=wl.r_c, weights=weights,
                   max_atoms=max_atoms, max_edges=max_edges, dtype=wl.dtype,
                   n_types=wl.n_types, gamma=wl.gamma, mu_min=wl.mu_min, mu_max=wl.mu_max,
                   n_heads=wl.n_heads if wl.kind == "attention" else 0,
                   head_dim=wl.head_dim if wl.kind == "attention" else 0,
                   max_graphs=max_graphs, validate=validate)

    def close(self):
        if getattr(self, "_ctx", None) and self._ctx.value:
            lib.mp_destroy(self._ctx)
            self._ctx = c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---------------------------------------------------------------- calls
    def cfconv_fwd(self, block, pos, row_ptr, col_idx, x, out=None, stream=None):
        N = x.shape[0]
        _need(pos, "pos", torch.float32, (N, 3))
        _need(row_ptr, "row_ptr", torch.int32, (N + 1,))
        _need(col_idx, "col_idx", torch.int32)
        _need(x, "x", self.tdtype, (N, self.F))
        if out is None:
            out = torch.empty_like(x)
        _need(out, "out", self.tdtype, (N, self.F))
        _check(lib.mp_cfconv_fwd(self._ctx, block, N, col_idx.numel(), _ptr(pos), _ptr(row_ptr),
                                 _ptr(col_idx), _ptr(x), _ptr(out), _stream(stream)),
               "mp_cfconv_fwd")
        return out

    def pair_plan(self, row_ptr, col_idx, stream=None):
        """Undirected-pair plan of a symmetric CSR for cfconv_fwd_pairs (synchronises)."""
        N = row_ptr.numel() - 1
        _need(row_ptr, "row_ptr", torch.int32, (N + 1,))
        _need(col_idx, "col_idx", torch.int32)
        _check(lib.mp_pair_plan(self._ctx, N, col_idx.numel(), _ptr(row_ptr), _ptr(col_idx),
                                _stream(stream)), "mp_pair_plan")

    def cfconv_fwd_pairs(self, block, pos, x, out=None, stream=None):
        """cfconv_fwd over the pairs of the last pair_plan: one filter per undirected pair."""
        N = x.shape[0]
        _need(pos, "pos", torch.float32, (N, 3))
        _need(x, "x", self.tdtype, (N, self.F))
        if out is None:
            out = torch.empty_like(x)
        _need(out, "out", self.tdtype, (N, self.F))
        _check(lib.mp_cfconv_fwd_pairs(self._ctx, block, N, _ptr(pos), _ptr(x), _ptr(out),
                                       _stream(stream)), "mp_cfconv_fwd_pairs")
        return out

    def attn_fwd(self, pos, nbr, mask, x, out=None, stream=None):
        N, K = nbr.shape
        _need(pos, "pos", torch.float32, (N, 3))
        _need(nbr, "nbr", torch.int32, (N, K))
        _need(mask, "mask", torch.uint8, (N, K))
        _need(x, "x", self.tdtype, (N, self.F))
        if out is None:
            out = torch.empty_like(x)
        _need(out, "out", self.tdtype, (N, self.F))
        _check(lib.mp_attn_fwd(self._ctx, N, K, _ptr(pos), _ptr(nbr), _ptr(mask), _ptr(x),
                               _ptr(out), _stream(stream)), "mp_attn_fwd")
        return out

    def attn_eq_fwd(self, pos, nbr, mask, x, out=None, stream=None):
        """mp_attn_eq_fwd: [N, 9, F] equivariant attention values (solid harmonics l <= 2)."""
        N, K = nbr.shape
        _need(pos, "pos", torch.float32, (N, 3))
        _need(nbr, "nbr", torch.int32, (N, K))
        _need(mask, "mask", torch.uint8, (N, K))
        _need(x, "x", self.tdtype, (N, self.F))
        if out is None:
            out = torch.empty((N, 9, self.F), dtype=self.tdtype, device=pos.device)
        _need(out, "out", self.tdtype, (N, 9, self.F))
        _check(lib.mp_attn_eq_fwd(self._ctx, N, K, _ptr(pos), _ptr(nbr), _ptr(mask), _ptr(x),
                                  _ptr(out), _stream(stream)), "mp_attn_eq_fwd")
        return out

    def attn_bwd(self, pos, nbr, mask, x, g_out, grad_x=None, grad_pos=None, stream=None):
        """mp_attn_bwd: (dL/dx, dL/dpos) of L = sum g_out . attn_fwd(...), both float32."""
        N, K = nbr.shape
        _need(pos, "pos", torch.float32, (N, 3))
        _need(nbr, "nbr", torch.int32, (N, K))
        _need(mask, "mask", torch.uint8, (N, K))
        _need(x, "x", self.tdtype, (N, self.F))
        _need(g_out, "g_out", torch.float32, (N, self.F))
        if grad_x is None:
            grad_x = torch.empty((N, self.F), dtype=torch.float32, device=pos.device)
        if grad_pos is None:
            grad_pos = torch.empty((N, 3), dtype=torch.float32, device=pos.device)
        _need(grad_x, "grad_x", torch.float32, (N, self.F))
        _need(grad_pos, "grad_pos", torch.float32, (N, 3))
        _check(lib.mp_attn_bwd(self._ctx, N, K, _ptr(pos), _ptr(nbr), _ptr(mask), _ptr(x),
                               _ptr(g_out), _ptr(grad_x), _ptr(grad_pos), _stream(stream)),
               "mp_attn_bwd")
        return grad_x, grad_pos

    def energy_forces(self, pos, types, row_ptr, col_idx, graph_ptr=None, energy=None,
                      forces=None, stream=None):
        N = pos.shape[0]
        _need(pos, "pos", torch.float32, (N, 3))
        _need(types, "types", torch.int32, (N,))
        _need(row_ptr, "row_ptr", torch.int32, (N + 1,))
        _need(col_idx, "col_idx", torch.int32)
        G = 1
        if graph_ptr is not None:
            _need(graph_ptr, "graph_ptr", torch.int32)
            G = graph_ptr.numel() - 1
        if energy is None:
            energy = torch.empty(G, dtype=torch.float32, device=pos.device)
        if forces is None:
            forces = torch.empty((N, 3), dtype=torch.float32, device=pos.device)
        _need(energy, "energy", torch.float32, (G,))
        _need(forces, "forces", torch.float32, (N, 3))
        _check(lib.mp_energy_forces(self._ctx, N, col_idx.numel(), _ptr(pos), _ptr(types),
                                    _ptr(row_ptr), _ptr(col_idx), _ptr(graph_ptr), G,
                                    _ptr(energy), _ptr(forces), _stream(stream)),
               "mp_energy_forces")
        return energy, forces

    def status_sync(self, stream=None):
        _check(lib.mp_status_sync(self._ctx, _stream(stream)), "device status")

    def launch_count(self) -> int:
        return int(lib.mp_launch_count(self._ctx))

    def set_wait_budget(self, ns: int):
        """mp_set_wait_budget: give up every bounded device wait after ns nanoseconds."""
        _check(lib.mp_set_wait_budget(self._ctx, int(ns)), "mp_set_wait_budget")

    def md_verlet(self, pos, vel, forces, types, row_ptr, col_idx, n_steps, dt, inv_mass=None,
                  graph_ptr=None, energy=None, kinetic=None, stream=None):
        """mp_md_verlet: n_steps velocity-Verlet steps in place on pos, vel, forces (forces must
        hold the forces at pos on entry). The CSR is kept: build it with a skin. Returns
        (energy, kinetic) of the last step; kinetic is computed when passed or requested as True."""
        N = pos.shape[0]
        _need(pos, "pos", torch.float32, (N, 3))
        _need(vel, "vel", torch.float32, (N, 3))
        _need(forces, "forces", torch.float32, (N, 3))
        _need(types, "types", torch.int32, (N,))
        _need(row_ptr, "row_ptr", torch.int32, (N + 1,))
        _need(col_idx, "col_idx", torch.int32)
        if inv_mass is not None:
            _need(inv_mass, "inv_mass", torch.float32, (N,))
        G = 1
        if graph_ptr is not None:
            _need(graph_ptr, "graph_ptr", torch.int32)
            G = graph_ptr.numel() - 1
        if energy is None:
            energy = torch.empty(G, dtype=torch.float32, device=pos.device)
        if kinetic is True:
            kinetic = torch.empty(G, dtype=torch.float32, device=pos.device)
        _need(energy, "energy", torch.float32, (G,))
        if kinetic is not None:
            _need(kinetic, "kinetic", torch.float32, (G,))
        _check(lib.mp_md_verlet(self._ctx, N, col_idx.numel(), _ptr(pos), _ptr(vel), _ptr(forces),
                                _ptr(inv_mass), float(dt), int(n_steps), _ptr(types),
                                _ptr(row_ptr), _ptr(col_idx), _ptr(graph_ptr), G, _ptr(energy),
                                _ptr(kinetic), _stream(stream)), "mp_md_verlet")
        return energy, kinetic

    def md_run(self, pos, vel, types, n_steps, dt, skin, capacity, rebuild_every=0,
               max_disp=None, check_every=1, inv_mass=None, graph_ptr=None, forces=None,
               energy=None, kinetic=None, row_ptr=None, col_idx=None, stream=None):
        """mp_md_run: n_steps velocity-Verlet steps that build and maintain their own neighbor
        list (cutoff r_c + skin; rebuilt every rebuild_every steps and whenever an atom moved more
        than max_disp, default skin / 2, since the last build). Returns a dict with energy,
        kinetic (when passed or True), forces, row_ptr, col_idx (the last list, E entries),
        n_edges and n_builds."""
        N = pos.shape[0]
        _need(pos, "pos", torch.float32, (N, 3))
        _need(vel, "vel", torch.float32, (N, 3))
        _need(types, "types", torch.int32, (N,))
        if inv_mass is not None:
            _need(inv_mass, "inv_mass", torch.float32, (N,))
        G = 1
        if graph_ptr is not None:
            _need(graph_ptr, "graph_ptr", torch.int32)
            G = graph_ptr.numel() - 1
        dev = pos.device
        forces = torch.empty((N, 3), dtype=torch.float32, device=dev) if forces is None else forces
        energy = torch.empty(G, dtype=torch.float32, device=dev) if energy is None else energy
        if kinetic is True:
            kinetic = torch.empty(G, dtype=torch.float32, device=dev)
        row_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev) if row_ptr is None else row_ptr
        if col_idx is None:
            col_idx = torch.empty(max(int(capacity), 1), dtype=torch.int32, device=dev)
        _need(forces, "forces", torch.float32, (N, 3))
        _need(energy, "energy", torch.float32, (G,))
        if kinetic is not None:
            _need(kinetic, "kinetic", torch.float32, (G,))
        _need(row_ptr, "row_ptr", torch.int32, (N + 1,))
        _need(col_idx, "col_idx", torch.int32)
        if col_idx.numel() < capacity:
            raise ValueError("col_idx: fewer entries than capacity")
        md = skin / 2 if max_disp is None else max_disp
        n_edges, n_builds = c_longlong(0), c_int(0)
        _check(lib.mp_md_run(self._ctx, N, _ptr(pos), _ptr(vel), _ptr(forces), _ptr(inv_mass),
                             float(dt), int(n_steps), _ptr(types), _ptr(graph_ptr), G, float(skin),
                             int(rebuild_every), float(md), int(check_every), _ptr(row_ptr),
                             _ptr(col_idx), int(capacity), ctypes.byref(n_edges), _ptr(energy),
                             _ptr(kinetic), ctypes.byref(n_builds), _stream(stream)), "mp_md_run")
        return {"energy": energy, "kinetic": kinetic, "forces": forces, "row_ptr": row_ptr,
                "col_idx": col_idx[: n_edges.value], "n_edges": n_edges.value,
                "n_builds": n_builds.value}

    def set_graphs(self, on: bool):
        """Record / replay energy_forces as a CUDA graph (default on; see mp_set_graphs)."""
        _check(lib.mp_set_graphs(self._ctx, 1 if on else 0), "mp_set_graphs")

    def profile_begin(self):
        _check(lib.mp_profile_begin(self._ctx), "mp_profile_begin")

    def profile_end(self, stream=None) -> dict:
        _check(lib.mp_profile_end(self._ctx, _stream(stream)), "mp_profile_end")
        out, i = {}, 0
        name, ms, n = c_char_p(), c_double(), c_longlong()
        while lib.mp_profile_get(self._ctx, i, ctypes.byref(name), ctypes.byref(ms),
                                 ctypes.byref(n)) == 0:
            out[name.value.decode()] = {"total_ms": ms.value, "launches": n.value}
            i += 1
        return out


def attn_fwd_noalloc(*, F: int, n_rbf: int, n_heads: int, head_dim: int, r_c: float,
                     weights: dict, pos, nbr, mask, x, out=None, status=None, gamma: float = 10.0,
                     mu_min: float = 0.0, mu_max: float | None = None, stream=None):
    """mp_attn_fwd_noalloc: the fp32 attention aggregation with no context and no device allocation
    inside the library. ``weights`` maps Wq, Wk, P, p, A1.0, c1.0, A2.0, c2.0 to float32 CUDA
    tensors. The caller allocates ``out`` (and the optional int32 ``status`` tensor) beforehand."""
    N, K = nbr.shape
    _need(pos, "pos", torch.float32, (N, 3))
    _need(nbr, "nbr", torch.int32, (N, K))
    _need(mask, "mask", torch.uint8, (N, K))
    _need(x, "x", torch.float32, (N, F))
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", torch.float32, (N, F))
    if status is not None:
        _need(status, "status", torch.int32, (1,))
    cfg = MpConfig(F=F, n_rbf=n_rbf, n_blocks=1, n_types=1, n_heads=n_heads, head_dim=head_dim,
                   r_c=r_c, gamma=gamma, mu_min=mu_min, mu_max=r_c if mu_max is None else mu_max,
                   dtype=FP32, max_atoms=N, max_edges=0, max_graphs=1, validate=0)
    # the C entry point reads F*F floats of Wq, Wk and A2, n_rbf*F of A1, n_rbf*n_heads of P: a
    # short or misplaced array would be read past its end, so the shapes and the device are checked
    shapes = {"Wq": (F, F), "Wk": (F, F), "P": (n_rbf, n_heads), "p": (n_heads,),
              "A1.0": (n_rbf, F), "c1.0": (F,), "A2.0": (F, F), "c2.0": (F,)}
    for key, shape in shapes.items():
        t = _need(weights[key], key, torch.float32, shape)
        if t.device != x.device:
            raise ValueError(f"{key}: must be on {x.device}, got {t.device}")
    w = MpWeights()
    for key in ("Wq", "Wk", "P", "p"):
        setattr(w, key, ctypes.cast(weights[key].data_ptr(), _FP))
    for key in ("A1", "c1", "A2", "c2"):
        getattr(w, key)[0] = ctypes.cast(weights[f"{key}.0"].data_ptr(), _FP)
    w.on_device = 1
    _check(lib.mp_attn_fwd_noalloc(ctypes.byref(cfg), ctypes.byref(w), N, K, _ptr(pos), _ptr(nbr),
                                   _ptr(mask), _ptr(x), _ptr(out), _ptr(status), _stream(stream)),
           "mp_attn_fwd_noalloc")
    return out


def selftest_tc():
    """Tensor-core layout self-check: returns the two mismatch counts (0, 0 when correct)."""
    out = (c_int * 2)()
    _check(lib.mp_selftest_tc(out), "mp_selftest_tc")
    return int(out[0]), int(out[1])


def shard_graphs(graph_ptr, rank: int, world: int):
    """mp_shard_graphs: the graphs [g0, g1) and atoms [a0, a1) of rank `rank` of `world`, for a
    host int32 graph_ptr (numpy or a CPU tensor)."""
    import numpy as np
    gp = np.ascontiguousarray(np.asarray(graph_ptr, dtype=np.int32))
    g0, g1 = c_int(0), c_int(0)
    _check(lib.mp_shard_graphs(gp.ctypes.data_as(c_void_p), len(gp) - 1, rank, world,
                               ctypes.byref(g0), ctypes.byref(g1)), "mp_shard_graphs")
    return g0.value, g1.value, int(gp[g0.value]), int(gp[g1.value])


def neighbor_csr(pos, r_c: float, graph_ptr=None, capacity: int | None = None, stream=None):
    """Destination-sorted CSR neighbor list on the device: (row_ptr int32 [N+1], col_idx int32 [E])."""
    N = pos.shape[0]
    _need(pos, "pos", torch.float32, (N, 3))
    G = 1
    if graph_ptr is not None:
        _need(graph_ptr, "graph_ptr", torch.int32)
        G = graph_ptr.numel() - 1
    row_ptr = torch.empty(N + 1, dtype=torch.int32, device=pos.device)
    if capacity is None:
        # a first pass counts the edges; the second writes them into an exactly sized array
        n = c_longlong(0)
        st = lib.mp_neighbor_csr(N, _ptr(pos), _ptr(graph_ptr), G, r_c, _ptr(row_ptr),
                                 c_void_p(0), 0, ctypes.byref(n), _stream(stream))
        if st not in (0, -5):
            _check(st, "mp_neighbor_csr")
        capacity = max(int(n.value), 1)
    col_idx = torch.empty(capacity, dtype=torch.int32, device=pos.device)
    n = c_longlong(0)
    _check(lib.mp_neighbor_csr(N, _ptr(pos), _ptr(graph_ptr), G, r_c, _ptr(row_ptr), _ptr(col_idx),
                               capacity, ctypes.byref(n), _stream(stream)), "mp_neighbor_csr")
    return row_ptr, col_idx[: n.value]


def spatial_order(pos, cell: float, graph_ptr=None, stream=None):
    """mp_spatial_order: int32 [N] permutation grouping the atoms of each graph by grid cell."""
    N = pos.shape[0]
    _need(pos, "pos", torch.float32, (N, 3))
    G = 1
    if graph_ptr is not None:
        _need(graph_ptr, "graph_ptr", torch.int32)
        G = graph_ptr.numel() - 1
    perm = torch.empty(N, dtype=torch.int32, device=pos.device)
    _check(lib.mp_spatial_order(N, _ptr(pos), _ptr(graph_ptr), G, float(cell), _ptr(perm),
                                _stream(stream)), "mp_spatial_order")
    return perm


def neighbor_padded(pos, r_c: float, K: int, graph_ptr=None, stream=None):
    """Capped, padded neighbor list on the device: (nbr int32 [N,K], mask uint8 [N,K])."""
    N = pos.shape[0]
    _need(pos, "pos", torch.float32, (N, 3))
    G = 1
    if graph_ptr is not None:
        _need(graph_ptr, "graph_ptr", torch.int32)
        G = graph_ptr.numel() - 1
    nbr = torch.empty((N, K), dtype=torch.int32, device=pos.device)
    mask = torch.empty((N, K), dtype=torch.uint8, device=pos.device)
    _check(lib.mp_neighbor_padded(N, _ptr(pos), _ptr(graph_ptr), G, r_c, K, _ptr(nbr), _ptr(mask),
                                  _stream(stream)), "mp_neighbor_padded")
    return nbr, mask
