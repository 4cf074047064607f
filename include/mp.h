/*
 * mp.h -- C ABI of libmp: fused neighbor-list message passing on NVIDIA B200 (sm_100a).
 *
 * The library computes, for SchNet-style atomistic force fields, the continuous-filter convolution
 * over a destination-sorted CSR neighbor list (distance, Gaussian radial basis, cosine envelope,
 * filter MLP, neighbor gather, filter product and segment sum fused in one pass, no atomics and no
 * edge-by-feature tensor in memory), a neighbor attention aggregation with an online softmax over a
 * padded neighbor list, and the energy with forces F = -dE/dr from a fused backward pass.
 *
 * Sources (page titles and sections):
 *   [FS]  FlashSchNet: Fast and Accurate Coarse-Grained Neural Network Molecular Dynamics --
 *         technical summary s.1 (bottlenecks), s.2.1 Flash Radial Basis, s.2.2 Flash Message Passing,
 *         s.2.3 Flash Aggregation (CSR segment reduce by destination, by source in the backward),
 *         s.2.4 channel-wise 16-bit quantization (positions, distances, energy accumulation and
 *         forces stay fp32).
 *   [E2]  E2Former-V2 page -- s.3.1 node-centric message passing, s.3.2 fused kernel (online softmax
 *         with running maximum and normaliser, each key/value loaded once, padded neighbors masked,
 *         parallel over destination atoms), s.5.2 (verify the neighbor list).
 *   [TS]  Tessera page -- neighbor search and reuse, forces as the energy gradient.
 *
 * Conventions for every call:
 *   - Array arguments are DEVICE pointers on the current CUDA device unless stated otherwise; the
 *     caller owns them. Layouts are dense row-major. Positions are float32 [N][3] (Angstrom).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and is complete
 *     only once that stream is synchronised. Calls do not synchronise, except where stated.
 *   - Every call returns an mp_status. On any error no output is specified. Host-side argument
 *     checks run before any launch. With mp_config.validate != 0 the CSR is also checked on the
 *     device first (one stream synchronisation); a bad list returns MP_ERR_BAD_CSR /
 *     MP_ERR_CSR_UNSORTED / MP_ERR_CSR_NOT_SYMMETRIC and nothing else runs. Compute kernels clamp
 *     every index they read to the array bounds and raise MP_ERR_DEVICE_BOUNDS (reported by the
 *     next mp_status_sync) instead of reading out of bounds.
 *   - The CSR neighbor list: row_ptr int32 [N+1] with row_ptr[0] = 0 and row_ptr[N] = E,
 *     col_idx int32 [E]; row i lists the sources j of edges j -> i, strictly ascending, j != i,
 *     and no edge crosses a graph (replica). [FS s.2.3]
 */
#ifndef MP_H_
#define MP_H_

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MP_OK = 0,
  MP_ERR_INVALID_ARG = -1,        /* null pointer, size out of range, unsupported configuration */
  MP_ERR_BAD_CSR = -2,            /* row_ptr not monotone, wrong ends, or a column out of range */
  MP_ERR_CSR_UNSORTED = -3,       /* a row not strictly ascending, or a self edge */
  MP_ERR_CSR_NOT_SYMMETRIC = -4,  /* energy/forces need j in N(i) <=> i in N(j) */
  MP_ERR_CAPACITY = -5,           /* N, E or a row exceeds what the context / output can hold */
  MP_ERR_CUDA = -6,               /* a CUDA runtime call or launch failed */
  MP_ERR_DEVICE_BOUNDS = -7,      /* a kernel met an index outside its arrays and skipped it */
  MP_ERR_TIMEOUT = -8,            /* a bounded device wait ran out */
  MP_ERR_UNIMPLEMENTED = -9
} mp_status;

typedef enum { MP_FP32 = 0, MP_BF16 = 1 } mp_dtype;

#define MP_MAX_BLOCKS 8

/* Model and capacity. Radial basis: e_k(d) = exp(-gamma (d - mu_k)^2), k = 0..n_rbf-1, with
 * mu_k = mu_min + k (mu_max - mu_min)/(n_rbf - 1); envelope f_c(d) = (cos(pi d/r_c) + 1)/2 for
 * d < r_c, else 0 [FS s.2.1]. Filter W(d) = f_c(d) (ssp(e(d) A1 + c1) A2 + c2) with
 * ssp(x) = ln(e^x/2 + 1/2). Interaction block: h = x W_in + b_in; m = cfconv(h);
 * x <- x + m W_out + b_out. Readout e_i = ssp(x_i B1 + d1) B2 + d2 (F -> F/2 -> 1).        */
typedef struct {
  int F;               /* channels: 64 or 128 */
  int n_rbf;           /* radial functions, 2..64 */
  int n_blocks;        /* interaction blocks, 1..MP_MAX_BLOCKS */
  int n_types;         /* embedding rows (atom / bead types), >= 1 */
  int n_heads;         /* attention heads; n_heads * head_dim == F */
  int head_dim;
  float r_c;           /* cutoff radius (Angstrom), > 0 */
  float gamma;         /* Gaussian width parameter (1/Angstrom^2), > 0 */
  float mu_min, mu_max;/* first and last radial centre */
  mp_dtype dtype;      /* MP_FP32: fp32 features and math; MP_BF16: bf16 features and weights,
                          fp32 accumulation; positions, distances, energy and forces fp32 [FS s.2.4] */
  int max_atoms;       /* capacity of the internal workspace */
  long long max_edges;
  int max_graphs;      /* replicas per energy call */
  int validate;        /* != 0: check the CSR on the device before each call */
} mp_config;

/* Weights: float32 row-major [in][out] arrays, host pointers (on_device = 0) or device pointers
 * (on_device = 1). mp_init copies them (rounding to bf16, ties to even, under MP_BF16); the caller
 * may free them after mp_init returns. Entries a call does not need may be NULL: energy/forces need
 * emb, the first n_blocks entries of every per-block array and B1, d1, B2, d2; the cfconv needs
 * A1, c1, A2, c2 of its block; the attention needs Wq, Wk, P, p and block 0's filter.       */
typedef struct {
  const float* emb;                       /* [n_types][F] */
  const float* A1[MP_MAX_BLOCKS];         /* [n_rbf][F] */
  const float* c1[MP_MAX_BLOCKS];         /* [F] */
  const float* A2[MP_MAX_BLOCKS];         /* [F][F] */
  const float* c2[MP_MAX_BLOCKS];         /* [F] */
  const float* W_in[MP_MAX_BLOCKS];       /* [F][F] */
  const float* b_in[MP_MAX_BLOCKS];       /* [F] */
  const float* W_out[MP_MAX_BLOCKS];      /* [F][F] */
  const float* b_out[MP_MAX_BLOCKS];      /* [F] */
  const float* B1;                        /* [F][F/2] */
  const float* d1;                        /* [F/2] */
  const float* B2;                        /* [F/2][1] */
  const float* d2;                        /* [1] */
  const float* Wq;                        /* [F][F] attention query projection (no bias) */
  const float* Wk;                        /* [F][F] attention key projection (no bias) */
  const float* P;                         /* [n_rbf][n_heads] radial-basis logit bias */
  const float* p;                         /* [n_heads] */
  int on_device;
} mp_weights;

typedef struct mp_ctx mp_ctx;             /* opaque; one per device and model */

/* Create a context on the current device: validates cfg, copies the weights, allocates the
 * workspace (O(max_atoms * F * n_blocks) bytes, never O(E * F)). Synchronises `stream`.
 * Errors: MP_ERR_INVALID_ARG, MP_ERR_CUDA.                                                  */
int mp_init(mp_ctx** ctx, const mp_config* cfg, const mp_weights* w, void* stream);

/* Release everything the context owns (synchronises the device first). NULL is ignored.     */
void mp_destroy(mp_ctx* ctx);

/* A static English description of a status code.                                           */
const char* mp_strerror(int status);

/* Synchronise `stream` and return (then clear) the device status word of the context:
 * MP_OK, MP_ERR_DEVICE_BOUNDS or MP_ERR_CAPACITY raised by a kernel since the last call.    */
int mp_status_sync(mp_ctx* ctx, void* stream);

/* Neighbor list by the exact rule [FS s.2.3; E2 s.5.2; TS neighbor search]: j is a neighbor of
 * i iff i != j, both in the same graph, and d2 < r_c*r_c, where d2 = (dx*dx + dy*dy) + dz*dz
 * with (dx,dy,dz) = r_j - r_i, every step one correctly rounded float64 operation on the
 * float32 positions (no fused multiply-add), r_c the float32 cutoff widened to float64.
 * graph_ptr: int32 [n_graphs+1] contiguous atom ranges (device), or NULL for one graph.
 * Output: row_ptr [N+1], col_idx [capacity] (device), rows sorted by source index.
 * *n_edges (HOST pointer) receives E. Synchronises `stream` (to read E).
 * Scratch: the cell grid and the sorted positions, O(N) bytes, stream-ordered from a memory pool
 * the library keeps per device; the pool keeps what was freed for the next call (it holds at
 * most the largest scratch live at once) instead of returning it at each synchronisation.
 * Errors: MP_ERR_INVALID_ARG, MP_ERR_CAPACITY (E > capacity; row_ptr is valid, col_idx not). */
int mp_neighbor_csr(int N, const float* pos, const int* graph_ptr, int n_graphs, float r_c,
                    int* row_ptr, int* col_idx, long long capacity, long long* n_edges,
                    void* stream);

/* Fixed-width neighbor list for the attention aggregation [E2 s.3.2: padded neighbors are
 * skipped by a mask]. Same rule as mp_neighbor_csr; a row with more than K neighbors keeps the
 * K nearest by (d2, j); kept neighbors are stored by ascending j, then nbr = -1, mask = 0.
 * nbr int32 [N][K], mask uint8 [N][K] (device). A row with more than 1024 candidates raises
 * MP_ERR_CAPACITY (reported by the return value; synchronises `stream`). Scratch as
 * mp_neighbor_csr.                                                                            */
int mp_neighbor_padded(int N, const float* pos, const int* graph_ptr, int n_graphs, float r_c,
                       int K, int* nbr, unsigned char* mask, void* stream);

/* A spatial order of the atoms for locality of the row gathers [TS: atoms organised along a
 * space-filling curve]: perm[k] = index of the atom placed at position k. Within each graph the
 * atoms are grouped by cell of the grid mp_neighbor_csr uses (cells at least `cell` wide over the
 * graph's bounding box, visited x fastest, then y, then z), atoms of a cell in ascending index
 * order; graphs keep their ranges, so graph_ptr stays valid for the permuted system. A caller
 * that applies the permutation to its per-atom arrays (positions, types, velocities, features)
 * gets the same physics with neighbors close in memory (the energy and forces are those of the
 * relabelled system). perm: int32 [N] (device). Synchronises `stream`. Scratch as
 * mp_neighbor_csr.
 * Errors: MP_ERR_INVALID_ARG, MP_ERR_CAPACITY, MP_ERR_CUDA.                                    */
int mp_spatial_order(int N, const float* pos, const int* graph_ptr, int n_graphs, float cell,
                     int* perm, void* stream);

/* Replica sharding over `world` ranks [FS: replicas are independent systems, simulated in one
 * batch through graph_ptr]: rank `rank` takes the contiguous graphs [*g0, *g1), boundary k placed
 * at the graph start nearest to the atom target graph_ptr[0] + total k / world (the later start
 * on a tie), so every graph goes to exactly one rank, in order, and each rank's atom count is
 * within one largest graph of total / world. A rank simulates its graphs with no communication (its own neighbor list,
 * energy_forces on its atoms); an empty range ([g, g)) is possible when world > n_graphs.
 * graph_ptr: HOST int32 [n_graphs + 1], nondecreasing. No device work.
 * Errors: MP_ERR_INVALID_ARG.                                                                    */
int mp_shard_graphs(const int* graph_ptr, int n_graphs, int rank, int world, int* g0, int* g1);

/* One continuous-filter convolution [FS s.2.1-2.3] with block `block`'s filter weights:
 *   out_i = sum_{j in row i} x_j (.) W(|r_i - r_j|),   rows with no edges give 0.
 * x, out: [N][F] of the context dtype (float or bf16), 16-byte aligned (rows are read and
 * written as 16-byte vectors); out must not alias x. No atomics: each output row is written once.
 * Errors: MP_ERR_INVALID_ARG (also for a misaligned x or out), MP_ERR_CAPACITY, CSR errors
 * (validate).                                                                                   */
int mp_cfconv_fwd(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                  const int* row_ptr, const int* col_idx, const void* x, void* out, void* stream);

/* Undirected-pair plan of a symmetric neighbor list [FS s.2.3: the symmetric list; s.2.4: the
 * filter MLP], kept in the context for mp_cfconv_fwd_pairs: the pairs {i, j} (i < j) once each,
 * grouped by blocks of 128 atoms into tiles of 128 pairs of one block pair, and the order in
 * which the pair kernel's partial rows are summed. Built on the device from the CSR (which must
 * be symmetric, as any cutoff list is: with validate set this is checked first); the plan does
 * not hold the positions, so it stays valid for every configuration the same list serves.
 * Workspace: O(E) ints plus one 64 KiB fp32 partial block per run of tiles, allocated here
 * (grown when a larger list comes) and freed by mp_destroy. Synchronises `stream`.
 * Errors: MP_ERR_INVALID_ARG, MP_ERR_CAPACITY (more than 32768 upper pairs of one 128-atom
 * block, more than 1024 block pairs of one block, or N > 8388608), MP_ERR_DEVICE_BOUNDS (a
 * column index outside [0, N)), MP_ERR_CUDA, CSR errors (validate).                            */
int mp_pair_plan(mp_ctx* ctx, int N, long long E, const int* row_ptr, const int* col_idx,
                 void* stream);
/* mp_energy_forces (bf16 tensor-core configuration) runs its forward cfconv passes over the pairs
 * of this plan when it is called with the same N, E, row_ptr and col_idx buffers the plan was
 * built from: the plan stands for the list those buffers held at mp_pair_plan time, so a caller
 * that rewrites the list in place must call mp_pair_plan again (or build the plan of another list)
 * before the next mp_energy_forces. Calls on other buffers use the directed kernels.           */

/* mp_cfconv_fwd over the pairs of the current plan: the filter W(d_ij) = W(d_ji) evaluated once
 * per pair and both messages taken from it, x_j (.) W to row i and x_i (.) W to row j, on the
 * tensor cores; each row written once by a fixed-order sum of per-run fp32 partials (no
 * atomics, results bitwise repeatable). Same out as mp_cfconv_fwd on the plan's list. Needs the
 * bf16 tensor-core configuration (F = 128) and a plan of the same N (the list of the last
 * mp_pair_plan call). x, out: [N][F] bf16, 16-byte aligned, out must not alias x.
 * Errors: MP_ERR_INVALID_ARG (no plan, another N, misaligned x or out), MP_ERR_UNIMPLEMENTED
 * (fp32 or another F), MP_ERR_CUDA.                                                           */
int mp_cfconv_fwd_pairs(mp_ctx* ctx, int block, int N, const float* pos, const void* x,
                        void* out, void* stream);

/* Neighbor attention aggregation with an online softmax [E2 s.3.1-3.2]. With q = x Wq,
 * k = x Wk split into n_heads heads of head_dim channels, for each valid slot j of row i
 * (mask != 0 and 0 <= nbr < N):
 *   l_ijh = q_ih . k_jh / sqrt(head_dim) + sum_k e_k(d_ij) P_kh + p_h,
 *   out_i[h] = sum_j softmax_j(l_ijh) (x_j (.) W(d_ij))[h]   (block 0's filter),
 * a row with no valid slot gives 0. nbr int32 [N][K], mask uint8 [N][K], x/out [N][F] of the
 * context dtype. Errors: MP_ERR_INVALID_ARG, MP_ERR_CAPACITY.                                */
int mp_attn_fwd(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                const unsigned char* mask, const void* x, void* out, void* stream);

/* Neighbor attention with an equivariant value path [E2 s.3.1: direction enters only through
 * the values]: the softmax weights of mp_attn_fwd, with each value coupled to the regular solid
 * harmonics of the edge vector up to l = 2,
 *   out_i[lm][c] = sum_j alpha_ij,h(c) (x_j (.) W(d_ij))[c] S_lm(r_j - r_i),
 * S_lm(r) = |r|^l Y_lm(r / |r|) with Y the real spherical harmonics orthonormal on the sphere, in
 * the order (l,m) = (0,0), (1,-1), (1,0), (1,1), (2,-2), (2,-1), (2,0), (2,1), (2,2); so
 * out_i[0] = mp_attn_fwd(...)_i / (2 sqrt(pi)) and out_i[1..3] rotate as (y, z, x).
 * out: [N][9][F] of the context dtype (device). The harmonics are evaluated per edge on chip
 * (the page's node-centric factorisation through source and destination positions gives the same
 * sum but loses digits to cancellation in fp32). Fp32 math on the CUDA cores. Same arguments,
 * conventions and errors as mp_attn_fwd.                                                      */
int mp_attn_eq_fwd(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                   const unsigned char* mask, const void* x, void* out, void* stream);

/* Backward of mp_attn_fwd [E2 s.3.2; TS forces are position gradients]: for L = sum_i g_out_i .
 * out_i, returns grad_x = dL/dx (float32 [N][F]) and grad_pos = dL/dr (float32 [N][3]; the
 * forces are -grad_pos when L is an energy), through q, k, the radial logit bias, the filter
 * W(d) and its envelope. Same nbr / mask / x conventions as mp_attn_fwd; g_out float32 [N][F].
 * Two passes without atomics: per destination row (softmax statistics, dL/dq, the row-side
 * position terms), then per source atom over the transposed list (dL/dk, the value path, the
 * source-side position terms); deterministic. Needs n_heads * head_dim = F, n_heads <= 32,
 * head_dim dividing 32, and 16 K n_heads + 16 K bytes of per-row slot data on chip beside the
 * filter weights (K <= 256 at F = 128, n_rbf = 50, 16 heads), else MP_ERR_CAPACITY; N K < 2^31.
 * Allocates and frees O(N K) bytes of stream-ordered scratch (the transposed list) from the
 * library's per-device pool (as mp_neighbor_csr).
 * Errors: MP_ERR_INVALID_ARG, MP_ERR_CAPACITY, MP_ERR_CUDA.                                    */
int mp_attn_bwd(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                const unsigned char* mask, const void* x, const float* g_out, float* grad_x,
                float* grad_pos, void* stream);

/* Allocation-free attention aggregation (no counterpart in the paper; added for callers that
 * cannot allocate device memory). Some hosts own every byte of device memory through their own
 * pool or budget and hand a library only pre-allocated buffers -- an MD engine's plugin
 * interface, a serving process under a fixed memory plan -- and a stray cudaMalloc (which can
 * also synchronise the device) is not allowed there. mp_init allocates a workspace, so such
 * callers use this entry point instead: it needs no context and calls no cudaMalloc, cudaFree or
 * other allocating routine. It computes exactly what mp_attn_fwd computes on the fp32 path.
 *   cfg: F, n_rbf, n_heads, head_dim, r_c, gamma, mu_min, mu_max are used; dtype must be MP_FP32.
 *   w:   DEVICE pointers (on_device = 1) to fp32 Wq, Wk, P, p and A1[0], c1[0], A2[0], c2[0],
 *        used as given (no copy, no rounding).
 *   x, out: float32 [N][F] (device); status: optional device int that receives the kernel status
 *        bits of this call (0 = fine; non-zero = an out-of-range neighbor index was skipped).
 * Scratch: the query and key rows live in one static device array compiled into the library,
 * 256 B + 8 * MP_NOALLOC_MAX_NF bytes (about 4 MiB) on every device that loads it, held until the
 * process exits; N * F above MP_NOALLOC_MAX_NF returns MP_ERR_CAPACITY (N <= 4096 at F = 128).
 * The first call on a device looks up the array's device address (once per device, with that
 * device current); make that first call before any stream capture. Every call shares the array
 * and it keeps the last call's contents: calls that overlap on the GPU (on different streams, or
 * from different threads) race on it and must be serialised by the caller.
 * Errors: MP_ERR_INVALID_ARG, MP_ERR_CAPACITY, MP_ERR_CUDA.                                    */
#define MP_NOALLOC_MAX_NF 524288
int mp_attn_fwd_noalloc(const mp_config* cfg, const mp_weights* w, int N, int K,
                        const float* pos, const int* nbr, const unsigned char* mask,
                        const float* x, float* out, int* status, void* stream);

/* Energy and forces [FS s.1, s.2.3 backward by source; TS forces = -dE/dr]: embedding, n_blocks
 * interaction blocks, readout; energy[g] = sum of atomic energies of graph g (fp32);
 * forces [N][3] = -dE/dr (fp32) from the fused backward over the same CSR, which must be
 * symmetric (true for any cutoff graph). types int32 [N] in [0, n_types); graph_ptr int32
 * [n_graphs+1] (device) or NULL with n_graphs = 1. Errors: MP_ERR_INVALID_ARG,
 * MP_ERR_CAPACITY, CSR errors (validate).                                                   */
int mp_energy_forces(mp_ctx* ctx, int N, long long E, const float* pos, const int* types,
                     const int* row_ptr, const int* col_idx, const int* graph_ptr, int n_graphs,
                     float* energy, float* forces, void* stream);

/* CUDA graphs for mp_energy_forces (on by default; a library addition, no counterpart on the
 * pages). On a stream other than the legacy default stream, with profiling and validate off and
 * no capture already in progress on it, a call records its kernels as a graph; a later call with
 * the same N, E, n_graphs, array pointers and stream replays that graph (one launch), reading
 * whatever the arrays hold then (new positions in the same buffer, for an MD step). A call with
 * other arguments records a new graph in place of the old one. If recording fails, the call runs
 * its kernels one by one and graphs stay off for the context. on = 0 turns graphs off and drops
 * the recorded graph. Errors: MP_ERR_INVALID_ARG.                                            */
int mp_set_graphs(mp_ctx* ctx, int on);

/* n_steps of velocity-Verlet molecular dynamics driven by mp_energy_forces [TS: the MD engine
 * integrates the atoms locally each step and keeps the neighbor topology while coordinates move;
 * CUDA graphs replay the fixed-shape step. FS: MD of batched replicas, throughput in
 * timestep x molecule per second]. One step, for every atom i:
 *   v_i += (dt/2) F_i / m_i;  r_i += dt v_i;  (energy, F) = mp_energy_forces(r);
 *   v_i += (dt/2) F_i / m_i.
 *   pos, vel, forces: float32 [N][3] (device), updated in place. On entry `forces` must hold the
 *     forces at `pos` (from mp_energy_forces, or a previous call); on return pos, vel, forces and
 *     energy belong to the last step.
 *   inv_mass: float32 [N] 1/m_i (device), or NULL for unit masses. dt: time step (any finite value;
 *     units are the caller's, consistent with the energy unit and masses).
 *   The CSR (row_ptr, col_idx, graph_ptr) is NOT rebuilt: it must stay a superset of the pairs
 *     within r_c for all n_steps, e.g. built with cutoff r_c + skin and rebuilt by the caller
 *     before any atom has moved skin / 2 (pairs beyond r_c contribute exactly 0). Each step first
 *     cuts it to the pairs with d^2 < r_c^2 at that step's positions (fp32, each product and sum
 *     rounded on its own, so the cut list stays symmetric) in scratch from the library's pool
 *     (4 (N + 1) + 4 E bytes for the call), and runs the force kernels on the cut list: a skin
 *     costs the cut, not force work on the pairs beyond r_c.
 *   kinetic: float32 [n_graphs] (device), or NULL: per-graph kinetic energy sum m_i |v_i|^2 / 2
 *     after the last step (fixed-order reduction).
 *   On a non-default stream with graphs on, the step is recorded once as a CUDA graph and
 *   replayed n_steps times; otherwise its kernels are launched step by step. n_steps = 0 only
 *   computes kinetic. Errors: MP_ERR_INVALID_ARG (also for a non-finite dt), MP_ERR_CAPACITY,
 *   MP_ERR_CUDA, CSR errors (validate, checked once per call).                              */
int mp_md_verlet(mp_ctx* ctx, int N, long long E, float* pos, float* vel, float* forces,
                 const float* inv_mass, float dt, int n_steps, const int* types,
                 const int* row_ptr, const int* col_idx, const int* graph_ptr, int n_graphs,
                 float* energy, float* kinetic, void* stream);

/* Velocity-Verlet MD that maintains its own neighbor list [TS: the neighbor topology is reused
 * while the coordinates move; it is rebuilt at a fixed step interval, or early, after a global
 * check, once an atom has moved more than a displacement limit]. The call builds the list with
 * cutoff r_c + skin at the current positions (mp_neighbor_csr into row_ptr / col_idx, capacity
 * entries), evaluates energy and forces with it (`forces` need not hold anything on entry), then
 * runs n_steps steps of mp_md_verlet's scheme. It rebuilds the list after every rebuild_every
 * steps (0: never on a schedule) and after any check that finds an atom more than max_disp from
 * where it was at the last build (checked every check_every >= 1 steps; max_disp <= 0 disables
 * it). At a rebuild the energy and forces of the current positions are evaluated again with the
 * new list only if some atom has moved more than skin / 2 since the previous build (otherwise
 * the old list already held every pair within r_c and they are unchanged).
 * The forces equal those of an exact r_c list at every step as long as no atom gets further than
 * skin / 2 from its position at the last build between two checks; max_disp <= skin / 2 with
 * check_every = 1 guarantees it.
 *   row_ptr int32 [N+1], col_idx int32 [capacity] (device): the list, owned by the caller;
 *   *n_edges (HOST) receives the edge count of the last build, *n_builds (HOST, or NULL) the
 *   number of builds. Other arguments as mp_md_verlet (the force kernels run on the list cut to
 *   r_c at each step's positions, as there). Each check and each build synchronises
 *   `stream`; steps between checks are replayed from one recorded CUDA graph per build.
 * Errors: MP_ERR_INVALID_ARG (non-finite dt, skin or max_disp, skin < 0, check_every < 1,
 * rebuild_every < 0), MP_ERR_CAPACITY (a list larger than capacity or the context's max_edges:
 * the call stops there, with pos / vel of the last completed step), MP_ERR_CUDA.             */
int mp_md_run(mp_ctx* ctx, int N, float* pos, float* vel, float* forces, const float* inv_mass,
              float dt, int n_steps, const int* types, const int* graph_ptr, int n_graphs,
              float skin, int rebuild_every, float max_disp, int check_every, int* row_ptr,
              int* col_idx, long long capacity, long long* n_edges, float* energy,
              float* kinetic, int* n_builds, void* stream);

/* Kernel timing for measurement. mp_profile_begin makes later calls record a CUDA event pair
 * around every kernel they launch (on the caller's stream); mp_profile_end synchronises the
 * stream and folds the pairs into per-kernel totals, readable by index with mp_profile_get
 * (name: static string; returns MP_ERR_INVALID_ARG past the last kernel).                   */
int mp_profile_begin(mp_ctx* ctx);
int mp_profile_end(mp_ctx* ctx, void* stream);
int mp_profile_get(mp_ctx* ctx, int index, const char** name, double* total_ms,
                   long long* launches);

/* Number of kernels this context has launched since mp_init.                               */
long long mp_launch_count(mp_ctx* ctx);

/* Budget of the bounded device waits (a library addition, no counterpart on the pages). The
 * warp-specialised tensor-core kernels hand tiles between their warp roles through shared-memory
 * barriers; every such wait gives up after `ns` nanoseconds of GPU global time (default
 * 2,000,000,000), after which the kernel stops its roles in order (each MMA-issuing thread still
 * waits, with the default budget, for everything it issued), frees its tensor memory, returns
 * normally and raises MP_ERR_TIMEOUT, read by the next mp_status_sync; outputs are then
 * unspecified. A small budget makes waits run out on purpose (a test of that path); 0 gives up
 * unless the awaited phase is already complete. Later calls of the context use the new budget
 * (a recorded energy/forces graph is dropped, since it holds the old one). Applies to the cfconv
 * forward and backward kernels of the bf16 path.
 * Errors: MP_ERR_INVALID_ARG (ns < 0).                                                       */
int mp_set_wait_budget(mp_ctx* ctx, long long ns);

/* Diagnostic: run the tensor-core layout self-check on the current device (one CTA; exact small-
 * integer products through the shared-memory operand layouts the kernels use). mismatches (HOST,
 * int[2]) receives the number of wrong outputs of the two checks (0 = pass; negative = an MMA did
 * not complete within its bounded wait). Synchronises the device. Errors: MP_ERR_CUDA.       */
int mp_selftest_tc(int* mismatches);

#ifdef __cplusplus
}
#endif
#endif /* MP_H_ */
