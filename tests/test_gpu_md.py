"""Velocity-Verlet MD through mp_md_verlet vs the fp64 oracle integrator driven by the oracle's
forces: a few steps agree within the energy/forces tolerances, the fp32 path conserves the total
energy to second order in dt, a CUDA-graph replay gives the same bits as plain launches, and the
per-replica kinetic energies follow the graph partition."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from atomistic_neighbor_list_b200 import synth
from helpers import TOL_BF16_FEAT, TOL_BF16_FORCE, oracle_csr, oracle_weights, rel_rms

pytestmark = pytest.mark.gpu
DEV = "cuda"
SKIN = 0.5


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as m
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def md_inputs(wl, seed=0):
    """Positions, graph_ptr, types, 1/m (m = 1 + type) and small random velocities."""
    pos, gp = synth.positions_for(wl, seed)
    n = len(pos)
    types = synth.atom_types(n, wl.n_types)
    im = (1.0 / (1.0 + types.astype(np.float64))).astype(np.float32)
    v0 = (np.random.default_rng(seed + 7).normal(size=(n, 3)) * np.sqrt(im)[:, None] * 0.05)
    return pos, gp, types, im, v0.astype(np.float32)


class MdRun:
    """One system on both sides: the CUDA context and the oracle model, with the CSR built at
    r_c + skin (checked bit for bit between the two) and kept for the whole run."""

    def __init__(self, mp, wl, seed=0):
        self.wl = wl
        self.pos, self.gp, self.types, self.im, self.v0 = md_inputs(wl, seed)
        n = len(self.pos)
        self.G = len(self.gp) - 1
        self.gp_d = dev(self.gp) if self.G > 1 else None
        self.rp, self.ci = mp.neighbor_csr(dev(self.pos), wl.r_c + SKIN, graph_ptr=self.gp_d)
        self.orp, self.oci = oracle_csr(self.pos, wl.r_c + SKIN, self.rp, self.ci,
                                        self.gp if self.G > 1 else None)
        self.ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=n,
                                            max_edges=max(self.ci.numel(), 1), max_graphs=self.G)
        self.model = oracle.Model.from_workload(wl, oracle_weights(synth.make_weights(wl),
                                                                   wl.dtype))

    def device_state(self):
        pos, vel = dev(self.pos), dev(self.v0)
        types = dev(self.types)
        e, f = self.ctx.energy_forces(pos, types, self.rp, self.ci, self.gp_d)
        return pos, vel, f, types, e

    def oracle_force(self, r):
        return oracle.energy_forces(self.model, r, self.types, self.orp, self.oci,
                                    self.gp if self.G > 1 else None)


@pytest.mark.parametrize("dtype,n", [("fp32", 600), ("bf16", 600)])
def test_md_verlet_matches_oracle(mp, dtype, n):
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], n), dtype=dtype)
    run = MdRun(mp, wl)
    pos, vel, f, types, _ = run.device_state()
    dt, steps = 0.01, 3
    e, ke = run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, steps, dt, inv_mass=dev(run.im),
                              kinetic=True)
    torch.cuda.synchronize()
    run.ctx.status_sync()
    _, f0, e_atom = oracle.energy_forces(run.model, run.pos, run.types, run.orp, run.oci,
                                         return_atom_energy=True)
    r, v, fr, er = oracle.velocity_verlet(run.oracle_force, run.pos, run.v0, f0, dt, steps, run.im)
    got_r, got_v, got_f = (t.cpu().numpy().astype(np.float64) for t in (pos, vel, f))
    assert np.abs(r - run.pos).max() < SKIN / 2
    # forces and velocities at the force bounds; positions: coordinates up to ~20 A are stored in
    # fp32 (ulp 2e-6 A), so 2e-5 A is ten ulps (fp32) and 2e-4 A leaves room for the bf16 forces
    ftol = 1e-5 if dtype == "fp32" else TOL_BF16_FORCE
    assert np.abs(got_r - r).max() <= (2e-5 if dtype == "fp32" else 2e-4)
    assert rel_rms(got_v, v) <= ftol
    assert rel_rms(got_f, fr) <= ftol
    ke_ref = oracle.kinetic_energy(v, run.im)
    assert abs(float(ke[0]) - ke_ref[0]) <= (1e-5 if dtype == "fp32" else TOL_BF16_FEAT) * ke_ref[0]
    # energy: relative to the sum of |atomic energies| (at the start) as in the energy/forces tests
    tol = 1e-5 if dtype == "fp32" else TOL_BF16_FEAT
    assert abs(float(e[0]) - er[0]) <= tol * np.abs(e_atom).sum()


def test_md_fp32_energy_error_second_order(mp):
    """NVE: the worst total-energy error along the same trajectory falls ~4x when dt halves."""
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], 400), dtype="fp32")
    run = MdRun(mp, wl, seed=1)
    im_d = dev(run.im)
    worst = []
    for dt, steps in ((0.02, 12), (0.01, 24)):
        pos, vel, f, types, e = run.device_state()
        ke0 = run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, 0, dt, inv_mass=im_d,
                                kinetic=True)[1]
        etot0 = float(e[0]) + float(ke0[0])
        w = 0.0
        for _ in range(steps):
            e, ke = run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, 1, dt, inv_mass=im_d,
                                      kinetic=True)
            w = max(w, abs(float(e[0]) + float(ke[0]) - etot0))
        assert float((pos.cpu() - torch.from_numpy(run.pos)).abs().max()) < SKIN / 2
        worst.append(w)
    run.ctx.status_sync()
    assert worst[0] > 1e-4 and 3.2 < worst[0] / worst[1] < 5.0, worst


def test_md_bf16_energy_bounded(mp):
    """bf16 features make the forces a rounded gradient, so the bf16 run has no dt^2 law; its
    total energy stays within the bf16 energy tolerance (relative to the sum of |atomic energies|)
    over 40 steps."""
    wl = synth.scaled(synth.WORKLOADS["cfg2"], 600)
    run = MdRun(mp, wl, seed=2)
    pos, vel, f, types, e = run.device_state()
    im_d = dev(run.im)
    ke0 = run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, 0, 0.01, inv_mass=im_d,
                            kinetic=True)[1]
    etot0 = float(e[0]) + float(ke0[0])
    w = 0.0
    for _ in range(8):
        e, ke = run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, 5, 0.01, inv_mass=im_d,
                                  kinetic=True)
        w = max(w, abs(float(e[0]) + float(ke[0]) - etot0))
    run.ctx.status_sync()
    _, _, e_atom = oracle.energy_forces(run.model, run.pos, run.types, run.orp, run.oci,
                                        return_atom_energy=True)
    assert np.isfinite(w) and w <= TOL_BF16_FEAT * np.abs(e_atom).sum(), (w, float(ke0[0]))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_md_graph_replay_matches_plain_launches(mp, dtype):
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], 2000), dtype=dtype)
    run_g = MdRun(mp, wl, seed=3)
    run_p = MdRun(mp, wl, seed=3)
    run_p.ctx.set_graphs(False)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        sg = run_g.device_state()
        sp = run_p.device_state()
        l0 = run_g.ctx.launch_count()
        eg, kg = run_g.ctx.md_verlet(*sg[:4], run_g.rp, run_g.ci, 6, 0.01,
                                     inv_mass=dev(run_g.im), kinetic=True)
        lg = run_g.ctx.launch_count() - l0
        l1 = run_p.ctx.launch_count()
        ep, kp = run_p.ctx.md_verlet(*sp[:4], run_p.rp, run_p.ci, 6, 0.01,
                                     inv_mass=dev(run_p.im), kinetic=True)
        lp = run_p.ctx.launch_count() - l1
    side.synchronize()
    assert lg == lp and lg > 6
    for a, b in zip(sg[:3], sp[:3]):
        assert torch.equal(a, b)
    assert torch.equal(eg, ep) and torch.equal(kg, kp)
    run_g.ctx.status_sync()
    run_p.ctx.status_sync()


def test_md_replicas_per_graph_energies(mp):
    wl = dataclasses.replace(synth.WORKLOADS["cfg3"], n_atoms=4 * 250, replicas=4)
    run = MdRun(mp, wl, seed=4)
    pos, vel, f, types, _ = run.device_state()
    e, ke = run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, 3, 0.01, inv_mass=dev(run.im),
                              graph_ptr=run.gp_d, kinetic=True)
    torch.cuda.synchronize()
    run.ctx.status_sync()
    e0, f0 = run.oracle_force(run.pos)
    r, v, fr, er = oracle.velocity_verlet(run.oracle_force, run.pos, run.v0, f0, 0.01, 3, run.im)
    assert e.shape == (4,) and ke.shape == (4,)
    ke_ref = oracle.kinetic_energy(v, run.im, run.gp)
    assert np.allclose(ke.cpu().numpy(), ke_ref, rtol=TOL_BF16_FEAT, atol=0)
    scale = np.abs(er).max() + 1.0
    assert np.max(np.abs(e.cpu().numpy() - er)) <= TOL_BF16_FEAT * scale
    assert rel_rms(f.cpu().numpy(), fr) <= TOL_BF16_FORCE


def test_md_zero_steps_and_argument_errors(mp):
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], 300), dtype="fp32")
    run = MdRun(mp, wl)
    pos, vel, f, types, _ = run.device_state()
    p0 = pos.clone()
    _, ke = run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, 0, 0.01, kinetic=True)
    torch.cuda.synchronize()
    assert torch.equal(pos, p0)
    assert abs(float(ke[0]) - oracle.kinetic_energy(run.v0)[0]) <= 1e-5 * float(ke[0])
    for bad in (float("nan"), float("inf")):
        with pytest.raises(mp.MpError) as err:
            run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, 1, bad)
        assert err.value.name == "MP_ERR_INVALID_ARG"
    with pytest.raises(mp.MpError) as err:
        run.ctx.md_verlet(pos, vel, f, types, run.rp, run.ci, -1, 0.01)
    assert err.value.name == "MP_ERR_INVALID_ARG"
    assert torch.equal(pos, p0)


def test_md_no_atoms(mp):
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], 8), dtype="fp32")
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=8, max_edges=1,
                                   max_graphs=2)
    z3 = torch.empty((0, 3), device=DEV)
    rp = torch.zeros(1, dtype=torch.int32, device=DEV)
    ci = torch.empty(0, dtype=torch.int32, device=DEV)
    gp = torch.zeros(3, dtype=torch.int32, device=DEV)
    e = torch.full((2,), 7.0, device=DEV)
    k = torch.full((2,), 7.0, device=DEV)
    ctx.md_verlet(z3, z3.clone(), z3.clone(), torch.empty(0, dtype=torch.int32, device=DEV), rp, ci,
                  4, 0.01, graph_ptr=gp, energy=e, kinetic=k)
    torch.cuda.synchronize()
    ctx.status_sync()
    assert torch.equal(e.cpu(), torch.zeros(2)) and torch.equal(k.cpu(), torch.zeros(2))


# ----------------------------------------------------------------------------- list maintenance
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_md_verlet_skin_list_costs_only_the_cut(mp, dtype):
    """Each step cuts the list to the pairs within r_c before the force kernels: a list built at
    r_c + 1 A and the exact r_c list give the same trajectory (the pairs between r_c and r_c + 1 A
    have f_c = f_c' = 0; the two runs differ only where a pair crossed r_c during the steps, by
    the rounding of a different tile partition). 3,000 atoms: many tiles on every CTA."""
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], 3000), dtype=dtype)
    pos, _, types, im, v0 = md_inputs(wl, seed=3)
    p0 = dev(pos)
    rp_s, ci_s = mp.neighbor_csr(p0, wl.r_c + 1.0)
    rp_x, ci_x = mp.neighbor_csr(p0, wl.r_c)
    assert ci_s.numel() > 1.5 * ci_x.numel()
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=len(pos),
                                  max_edges=ci_s.numel())
    runs = []
    for rp, ci in ((rp_s, ci_s), (rp_x, ci_x)):
        p, v, t = dev(pos), dev(v0), dev(types)
        _, f = ctx.energy_forces(p, t, rp_x, ci_x)
        f = f.clone()
        e, _ = ctx.md_verlet(p, v, f, t, rp, ci, 4, 0.002, inv_mass=dev(im))
        torch.cuda.synchronize()
        ctx.status_sync()
        runs.append((p.cpu().numpy(), f.cpu().numpy(), float(e[0])))
    (ps, fs, es), (px, fx, ex) = runs
    ftol, etol = (1e-5, 1e-6) if dtype == "fp32" else (5e-3, 1e-4)
    assert np.abs(ps - px).max() <= 1e-5
    assert rel_rms(fs, fx) <= ftol
    assert abs(es - ex) <= etol * abs(ex)


def fast_system(n=300, seed=5, vscale=1.5):
    """fp32, one interaction block; velocities large enough that atoms cross the rebuild limit."""
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], n), dtype="fp32", n_blocks=1)
    pos, _, types, im, _ = md_inputs(wl, seed)
    v0 = (np.random.default_rng(seed + 20).normal(size=(n, 3)) * np.sqrt(im)[:, None] * vscale)
    return wl, pos, types, im, v0.astype(np.float32)


def test_md_run_matches_fresh_exact_lists(mp):
    """mp_md_run keeps an r_c + skin list and rebuilds it when an atom has moved skin / 2; the
    oracle's forces come from an exact r_c list built afresh at every evaluation. The two
    trajectories agree, so no pair was ever missing from the kept list."""
    wl, pos, types, im, v0 = fast_system()
    skin, dt, steps = 0.5, 0.01, 40
    cap = 2 * len(oracle.neighbor_csr(pos, wl.r_c + skin)[1]) + 1024
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=len(pos), max_edges=cap)
    p, v = dev(pos), dev(v0)
    side = torch.cuda.Stream()  # a stream of its own: the steps are replayed from graphs
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        out = ctx.md_run(p, v, dev(types), steps, dt, skin, cap, inv_mass=dev(im), kinetic=True)
    side.synchronize()
    ctx.status_sync()
    model = oracle.Model.from_workload(wl, synth.make_weights(wl))

    def fresh(r):
        rp, ci = oracle.neighbor_csr(r, wl.r_c)
        return oracle.energy_forces(model, r, types, rp, ci)

    e0, f0 = fresh(pos.astype(np.float64))
    r, vr, fr, er = oracle.velocity_verlet(fresh, pos, v0, f0, dt, steps, im)
    got = p.cpu().numpy().astype(np.float64)
    assert np.abs(r - pos).max() > 2 * skin  # far enough that the list had to be rebuilt
    assert out["n_builds"] >= 3
    # 40 fp32 steps at high velocity: the fp32 rounding of each step grows along the trajectory
    # (and the two sides cut their lists at different moments), so 1e-3 instead of the one-step
    # bounds
    assert np.abs(got - r).max() <= 1e-3
    assert rel_rms(v.cpu().numpy(), vr) <= 1e-3
    assert rel_rms(out["forces"].cpu().numpy(), fr) <= 1e-3
    # the list kept at the end holds every pair within r_c at the final positions
    orp, oci = oracle.neighbor_csr(got.astype(np.float32), wl.r_c)
    rp, ci = out["row_ptr"].cpu().numpy(), out["col_idx"].cpu().numpy()
    kept = {(i, j) for i in range(len(got)) for j in ci[rp[i]:rp[i + 1]]}
    need = {(i, j) for i in range(len(got)) for j in oci[orp[i]:orp[i + 1]]}
    assert need <= kept


def test_md_run_schedule_and_capacity(mp):
    wl, pos, types, im, _ = fast_system(seed=6, vscale=0.0)
    v0 = np.zeros_like(pos)
    cap = 2 * len(oracle.neighbor_csr(pos, wl.r_c + 0.5)[1]) + 1024
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=len(pos), max_edges=cap)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        out = ctx.md_run(dev(pos), dev(v0), dev(types), 25, 0.001, 0.5, cap, rebuild_every=10,
                         max_disp=0.0)
        assert out["n_builds"] == 3  # at the start, after 10 and after 20 steps
        out = ctx.md_run(dev(pos), dev(v0), dev(types), 25, 0.001, 0.5, cap)
        assert out["n_builds"] == 1  # atoms at rest never reach the displacement limit
        with pytest.raises(mp.MpError) as err:
            ctx.md_run(dev(pos), dev(v0), dev(types), 5, 0.001, 0.5, 10)
        assert err.value.name == "MP_ERR_CAPACITY"
        with pytest.raises(mp.MpError) as err:
            ctx.md_run(dev(pos), dev(v0), dev(types), 5, 0.001, -0.5, cap)
        assert err.value.name == "MP_ERR_INVALID_ARG"
    side.synchronize()
    ctx.status_sync()
