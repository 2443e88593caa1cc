/*
 * reann.h -- C ABI of libreann.so, a B200 (sm_100a) implementation of the
 * energy+force evaluation of the REANN message-passing neural-network
 * potential and of velocity-Verlet MD driven by it.
 *
 * The operations follow "Efficient Parallelization of Message Passing
 * Neural Network Potentials for Large-Scale Molecular Dynamics" (Xia and
 * Jiang):
 *   - embedded atom density, section "REANN Architecture", Eq. 1;
 *   - message (orbital-coefficient) update by per-element atomic networks,
 *     Eq. 2; atomic energies from the last layer's density (Eq. 3 input);
 *   - forces by the chain rule through every layer, Eqs. 3-5, evaluated as
 *     vector-Jacobian products (section "Parallelization Algorithm");
 *   - one neighbour list built once and reused by all T layers (same
 *     section, Fig. 2), with a Verlet skin (section "Introduction");
 *   - the local/ghost-atom spatial decomposition with a per-layer ghost
 *     refresh (Fig. 3a, Fig. 4), as a single-GPU checking mode.
 *
 * Conventions shared by every entry point:
 *   units     A, eV, fs, amu; forces eV/A; velocities A/fs.
 *   box       orthorhombic, fully periodic, edges box[3] (A), each at least
 *             2 (r_cut + skin).
 *   arrays    per-atom vectors are row-major [n][3] in the caller's atom
 *             order.  Any array pointer may point to device memory or to
 *             host memory (pinned or pageable); the library detects which
 *             with cudaPointerGetAttributes and copies host arrays through
 *             its own device buffers on the given stream (the thermostat's
 *             random numbers are the one host-only array).  The caller owns
 *             every array it passes; the library owns the context and all
 *             workspaces.
 *   streams   work is enqueued on the caller's stream; calls that return a
 *             host value (energy, statistics, counters) synchronise it.
 *   errors    every call returns a reann_status; reann_last_error() gives a
 *             message.  Conditions found on the device (neighbour capacity,
 *             skin violation, non-finite values) are recorded in a status
 *             word that the next synchronising call reads.  No call aborts
 *             or traps the device.
 *   threads   a context is not thread-safe; use one context per thread.
 */
#ifndef REANN_H
#define REANN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct reann_ctx reann_ctx; /* opaque */
typedef void *reann_stream;         /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    REANN_OK = 0,
    REANN_ERR_ARG = 1,       /* invalid argument or configuration */
    REANN_ERR_BOX = 2,       /* box edge <= 0 or < 2 (r_cut + skin) */
    REANN_ERR_CAPACITY = 3,  /* a fixed-size buffer would overflow */
    REANN_ERR_NONFINITE = 4, /* NaN/Inf in positions, energy or forces */
    REANN_ERR_SKIN = 5,      /* an atom moved more than skin/2 since the list was built */
    REANN_ERR_STATE = 6,     /* call out of order, e.g. forces before a neighbour list */
    REANN_ERR_CUDA = 7,      /* a CUDA runtime call failed */
    REANN_ERR_TIMEOUT = 8,   /* a bounded device wait gave up */
    REANN_ERR_UNSUPPORTED = 9,
    REANN_ERR_INDEX = 10     /* checked builds: an internal index was outside its array */
} reann_status;

/*
 * Model hyperparameters (section "REANN Architecture").  D = n_radial *
 * (l_max + 1) features per atom: feature (n, l) sits at index
 * l * n_radial + n.  Radial primitive n has centre mu_n = r_cut n /
 * (n_radial - 1) and width alpha; the cutoff function is
 * (cos(pi r / r_cut) + 1) / 2 for r < r_cut.
 */
typedef struct {
    int32_t n_elements;    /* 1..8 */
    int32_t T;             /* message-passing layers, 1..8 */
    int32_t n_radial;      /* N_phi: 8 or 10 */
    int32_t l_max;         /* L: 2 */
    int32_t hidden[2];     /* atomic-network hidden widths: 64 or 128 each */
    double r_cut;          /* A */
    double skin;           /* A; the list radius is r_cut + skin */
    double alpha;          /* A^-2 */
    int32_t mlp_precision; /* 0 = fp32-accurate networks: on the tensor cores as three tf32 passes
                                  (operands split hi + lo) for hidden widths [64, 64] with Eq. 1's
                                  densities, on the CUDA cores otherwise;
                              1 = bf16 tensor-core GEMMs (16-bit split activations), fp32 accumulate;
                              2 = fp32 networks on the CUDA cores for every shape (a reference
                                  for measuring the tensor-core paths) */
    int32_t dd_grid[3];    /* {0,0,0} = monolithic; else subdomains per axis (checking mode) */
    int32_t dd_stale_ghosts; /* checking mode only: 1 = skip the per-layer ghost refresh (negative control) */
    int32_t density_form;    /* 0 = Eq. 1: rho_(n,l) = sum_tau w_tau A_{n,tau}^2, D_rho = N_phi (L+1) features;
                                1 = pair products rho_(n,m,l) = sum_tau w_tau A_{n,tau} A_{m,tau} for n <= m,
                                    D_rho = N_phi (N_phi+1)(L+1)/2 features (the density dimension stated in
                                    section "REANN Architecture"); N_phi = 8, L = 2 and equal hidden
                                    widths only (REANN_ERR_UNSUPPORTED otherwise).  The messages c keep
                                    one value per (n, l) in both forms. */
} reann_config;

/*
 * Weight blob (float32, read once by reann_create):
 *   C0[n_elements][D]                      initial coefficients c^0 per element
 *   for t = 0..T-2, for e = 0..n_elements-1: coefficient network M^t_e (rho^t -> c^{t+1}), n_out = D
 *   for e = 0..n_elements-1:                 energy network N_e (rho^{T-1} -> E_i), n_out = 1
 * and each network is
 *   shift[Dr], scale[Dr], W1[H1][Dr], b1[H1], W2[H2][H1], b2[H2], W3[n_out][H2], b3[n_out]
 * evaluating y = W3 tanh(W2 tanh(W1 ((x - shift) / scale) + b1) + b2) + b3, with
 * D = N_phi (L+1) coefficients per atom and Dr density features per atom
 * (Dr = D, or N_phi (N_phi+1)(L+1)/2 for density_form = 1).
 */

typedef struct {
    double e_pot;       /* potential energy after the last step, eV */
    double e_kin;       /* kinetic energy after the last step, eV */
    double e_pot0;      /* potential energy at entry, eV */
    double e_kin0;      /* kinetic energy at entry, eV */
    int64_t rebuilds;   /* neighbour-list rebuilds during the call */
    int64_t steps;      /* steps completed */
    double e_thermostat; /* energy the thermostat added during the call, eV (0 for reann_md_step) */
} reann_md_stats;

typedef struct {
    int64_t n_atoms;
    int64_t nnz;                 /* neighbour-list entries (ordered pairs within r_cut + skin) */
    int64_t capacity;            /* allocated neighbour-list entries */
    int64_t max_row;             /* longest neighbour row */
    int64_t active_pairs;        /* ordered pairs within r_cut at the last evaluation */
    int64_t builds;              /* neighbour-list builds since creation */
    int64_t evaluations;         /* energy+force evaluations since creation */
    int64_t ghost_slots;         /* domain-decomposed mode: ghost atoms over all subdomains;
                                    halo plan: this process's ghost atoms */
    int64_t ghost_bytes_fwd;     /* domain-decomposed mode: bytes gathered per layer, forward;
                                    halo plan: coefficient bytes this process sends per layer */
    int64_t ghost_bytes_bwd;     /* domain-decomposed mode: bytes reduced per layer, backward;
                                    halo plan: gradient-partial bytes this process sends per layer */
    int64_t kernel_launches;     /* kernels this context has launched since creation */
    int32_t cells[3];            /* cell grid of the neighbour search */
    int32_t reserved;
} reann_counters;

/* Kernel groups timed by reann_profile / reann_profile_read. */
typedef enum {
    REANN_K_ACTIVE = 0,      /* compaction of the pairs within r_cut */
    REANN_K_DENSITY = 1,     /* orbital + density forward, one launch per layer (Eq. 1) */
    REANN_K_MLP_FWD = 2,     /* coefficient networks, forward (Eq. 2) */
    REANN_K_MLP_ENERGY = 3,  /* energy network, forward + input gradient */
    REANN_K_EDGE_BWD = 4,    /* edge VJP + force gather, one launch per layer (Eqs. 3-4) */
    REANN_K_MLP_BWD = 5,     /* coefficient networks, input gradient (Eq. 5) */
    REANN_K_ENERGY_SUM = 6,  /* energy reduction */
    REANN_K_INTEGRATE = 7,   /* velocity-Verlet kicks and drift */
    REANN_K_NEIGHBORS = 8,   /* binning + neighbour list build (all kernels of one build) */
    REANN_K_OTHER = 9,       /* gathers, scatters, checks */
    REANN_K_GHOST = 10,      /* domain-decomposed mode: ghost planning and per-layer ghost refresh */
    REANN_K_COUNT = 11
} reann_kernel_group;

/*
 * Creates a context on CUDA device `device` and uploads the weights.
 * weights: host float32 blob of nbytes bytes laid out as above (nbytes
 * must match the configuration exactly).  On success *out receives the
 * context.  Errors: REANN_ERR_ARG (bad configuration or blob size),
 * REANN_ERR_UNSUPPORTED (a hyperparameter outside the compiled set),
 * REANN_ERR_CUDA.
 */
reann_status reann_create(const reann_config *cfg, const void *weights, size_t nbytes, int device, reann_ctx **out);

/* Frees the context and every workspace.  NULL is accepted. */
reann_status reann_destroy(reann_ctx *ctx);

/*
 * Builds the neighbour list (section "Parallelization Algorithm": built once,
 * reused by every layer) for n atoms.
 * pos: float32 [n][3] positions (A), any image; types: int32 [n] element
 * indices in [0, n_elements); box: host double[3].
 * Atoms are binned into cells at least r_cut + skin wide by a counting sort
 * on (element, cell), and the list holds every ordered pair (i, j), i != j,
 * whose minimum-image distance satisfies (dx*dx + dy*dy) + dz*dz <
 * (r_cut + skin)^2, evaluated in fp64 without fused multiply-add.  Rows
 * are sorted.  Allocates workspaces for n atoms (the only call besides
 * reann_create that allocates).  Synchronises the stream once to size the
 * list.  Errors: REANN_ERR_ARG, REANN_ERR_BOX, REANN_ERR_NONFINITE,
 * REANN_ERR_CAPACITY (more than 2^31-1 entries), REANN_ERR_CUDA.
 */
reann_status reann_build_neighbors(reann_ctx *ctx, int64_t n, const float *pos, const int32_t *types,
                                   const double box[3], reann_stream stream);

/*
 * One energy+force evaluation (Eqs. 1-5) at positions pos (float32 [n][3],
 * same atoms and types as the last reann_build_neighbors).
 * energy: host double*, receives E = sum_i E_i (eV), may be NULL.
 * forces: float32 [n][3] (eV/A), may be NULL.
 * atom_energy: float32 [n] (eV), may be NULL.
 * Does not allocate.  Synchronises the stream (to return the energy and
 * the device status).  Errors: REANN_ERR_STATE (no list), REANN_ERR_SKIN
 * (an atom moved more than skin/2 since the list was built: rebuild and
 * call again; outputs are then not valid), REANN_ERR_NONFINITE,
 * REANN_ERR_CUDA.
 */
reann_status reann_energy_forces(reann_ctx *ctx, const float *pos, double *energy, float *forces,
                                 float *atom_energy, reann_stream stream);

/*
 * nsteps of velocity Verlet with time step dt_fs:
 *   v += F/m dt/2;  x += v dt;  wrap x into [0, L);  rebuild the list when
 *   an atom has moved more than skin/2 since the last build;  F = -dE/dx;
 *   v += F/m dt/2.
 * The acceleration unit is 1 eV/(A amu) = 1/103.6426965 A/fs^2.
 * x: double [n][3] (A) and v: double [n][3] (A/fs), updated in place.
 * mass_amu: host double[n_elements].  stats (host, may be NULL) receives
 * energies and counts.  Forces are evaluated once per step on the float32
 * rounding of x, plus once at entry -- unless the call continues the
 * previous one (x and v bitwise equal to what the previous reann_md_step
 * on this context returned, same dt and masses, no other call in between),
 * in which case the resident state, list and forces are reused and the
 * trajectory is identical to one longer call.  Whether a call continues is
 * decided while it runs: when the previous call left a valid state with the
 * same dt and masses, the steps start from that state at once, and x and v
 * are moved in and compared with it on a library stream meanwhile; if they
 * differ, that run is discarded and the call starts again from the x and v
 * it read in (x and v are written only after the comparison, or, for the
 * discarded run's x, overwritten by the result of the restart).  Requires a prior
 * reann_build_neighbors for the same atoms and types (positions may have
 * moved; the list is rebuilt at entry).  Allocates only if the neighbour
 * list outgrows its capacity.  The steps between list rebuilds, but the last
 * one, run as one device-side graph loop (a WHILE node that stops at a
 * rebuild or an error), so the stream is synchronised once per such stretch,
 * once per rebuild, and at the end; with the loop unavailable (eager launches
 * for profiling, or a runtime without conditional graph nodes) once per step.
 * The final x is copied out on a
 * library stream during the last step's force evaluation; every return,
 * error returns included, waits for that copy, so x and v are not written
 * after the call returns.  Errors: as reann_energy_forces.
 */
reann_status reann_md_step(reann_ctx *ctx, int32_t nsteps, double dt_fs, double *x, double *v,
                           const double *mass_amu, reann_md_stats *stats, reann_stream stream);

/*
 * nsteps of canonical (NVT) MD, the ensemble of the capsid production run on
 * the Tessera page (abstract): the reann_md_step update, and after each
 * step's closing half kick stochastic velocity rescaling (Bussi, Donadio and
 * Parrinello, J. Chem. Phys. 126, 014101 (2007)).  With K the kinetic energy,
 * Nf = 3n - 3, Kt = Nf kB T / 2 and c = exp(-dt / tau), every velocity is
 * scaled by sqrt(K' / K),
 *   K' = K + (1 - c) (Kt (R1^2 + S) / Nf - K) + 2 R1 sqrt(c (1 - c) K Kt / Nf),
 * computed on the device from the device-side K (no synchronisation).
 * temperature_K > 0; tau_fs >= 0 (0: K drawn afresh each step; +inf: NVE).
 * noise: HOST double [nsteps][2], the step's (R1, S): R1 a standard normal
 * number and S >= 0 a sum of Nf - 1 squared standard normals, drawn by the
 * caller, so that the run is reproducible and comparable with any other
 * implementation given the same numbers.  stats->e_thermostat receives the
 * summed K' - K (the conserved quantity is E_pot + E_kin - e_thermostat).
 * Continuations, allocation, synchronisation and errors as reann_md_step;
 * also REANN_ERR_ARG for fewer than two atoms, a device noise pointer or a
 * non-finite (or negative S) noise entry.  Three kernel launches per step
 * beyond reann_md_step's.
 */
reann_status reann_md_step_nvt(reann_ctx *ctx, int32_t nsteps, double dt_fs, double temperature_K, double tau_fs,
                               const double *noise, double *x, double *v, const double *mass_amu,
                               reann_md_stats *stats, reann_stream stream);

/* Copies the counters of the context into *out (host).  Synchronises nothing. */
reann_status reann_get_counters(const reann_ctx *ctx, reann_counters *out);

/*
 * One process's share of a spatial decomposition over several processes or
 * GPUs: the per-layer halo exchange of section "Parallelization Algorithm"
 * (Figs. 3-4, Eqs. 3-5).  The caller owns the decomposition and the transport;
 * the library evaluates its own atoms and moves rows to and from two
 * library-owned device buffers at the points where the method exchanges data.
 *
 * Atoms are in the caller's order: n_local own atoms, then n_ghost ghosts
 * (other processes' atoms within r_cut + skin of this process's own atoms,
 * e.g. of its region, grouped by the process that owns them).  send_index
 * (host, [n_send]) lists the own atoms, by caller index, that are ghosts of
 * other processes, in the order the exchange function sends them (grouped by
 * destination); an own atom may appear several times.
 *
 * reann_halo_plan sets this up (allocates the exchange buffers); then
 * reann_build_neighbors takes n = n_local + n_ghost atoms and builds rows for
 * own atoms (all neighbours) and for ghosts (own neighbours only).  The plan
 * stays until the next reann_halo_plan; reann_energy_forces and the MD calls
 * refuse a context with a plan (REANN_ERR_STATE).  Errors: REANN_ERR_ARG
 * (sizes, an entry outside [0, n_local)), REANN_ERR_STATE (domain-decomposed
 * checking mode), REANN_ERR_CUDA.
 */
reann_status reann_halo_plan(reann_ctx *ctx, int64_t n_local, int64_t n_ghost, const int32_t *send_index,
                             int64_t n_send);

/*
 * The exchange function the caller provides.  kind:
 *   REANN_EXCHANGE_COEF (after coefficient network t-1, layer = t = 1..T-1):
 *     send = own atoms' c^t rows in send_index order [send_rows = n_send][width = D];
 *     recv must receive the ghosts' c^t rows in ghost order [recv_rows = n_ghost][D].
 *   REANN_EXCHANGE_COEF_GRAD (after layer t's edge pass, layer = t = T-1..1):
 *     send = the ghosts' partial dE/dc^t from this process's energies [n_ghost][D];
 *     recv must receive the partials other processes computed for this
 *     process's sent rows, in send_index order [n_send][D]; they are added.
 *   REANN_EXCHANGE_FORCE (once, layer = 0): the same with partial forces [.][3].
 * send and recv are library-owned device buffers (float32, row-major); the
 * send rows are complete in `stream` order when the function is called, and
 * the received rows must be in place, in `stream` order, before work the
 * library enqueues on `stream` after it returns (enqueue the transfer on
 * `stream`, or synchronise it and copy).  Return 0, or nonzero to abort the
 * evaluation with REANN_ERR_CUDA.
 */
enum { REANN_EXCHANGE_COEF = 0, REANN_EXCHANGE_COEF_GRAD = 1, REANN_EXCHANGE_FORCE = 2 };
typedef int32_t (*reann_exchange_fn)(void *user, int32_t kind, int32_t layer, const float *send, int64_t send_rows,
                                     float *recv, int64_t recv_rows, int32_t width, reann_stream stream);

/*
 * Energy and forces of this process's own atoms under a halo plan.  pos: all
 * n_local + n_ghost positions (float32 [n][3], caller order; the caller moves
 * the ghosts' positions); *energy (host): the sum of the own atoms' energies;
 * forces [n_local][3] and atom_energy [n_local] (nullable): own atoms, forces
 * including the partials received from the other processes.  Host or device
 * arrays as in reann_energy_forces.  Calls `exchange` 2 (T - 1) + 1 times, in
 * the same order on every process.  Synchronises the stream at the end.
 * Errors: REANN_ERR_STATE (no plan or no list), REANN_ERR_ARG,
 * REANN_ERR_SKIN, REANN_ERR_NONFINITE, REANN_ERR_CUDA, REANN_ERR_TIMEOUT.
 */
reann_status reann_energy_forces_halo(reann_ctx *ctx, const float *pos, double *energy, float *forces,
                                      float *atom_energy, reann_exchange_fn exchange, void *user,
                                      reann_stream stream);

/* Message of the last error on this context (or of the last failed create when ctx is NULL). */
const char *reann_last_error(const reann_ctx *ctx);

/*
 * Diagnostics (parity tests).  Copies the current neighbour list in the
 * caller's atom order: row[n+1] (int64) and col[nnz] (int32), rows sorted
 * by caller index.  Host or device pointers; cap is col's length.
 * Synchronises the stream.  Errors: REANN_ERR_STATE, REANN_ERR_CAPACITY.
 */
reann_status reann_get_neighbors(reann_ctx *ctx, int64_t *row, int32_t *col, int64_t cap, reann_stream stream);

/*
 * Diagnostics (parity tests).  After reann_energy_forces, copies layer t's
 * per-atom embedded density rho^t (float32 [n][Dr], Dr as in the weight blob)
 * and coefficients c^t (float32 [n][D]) in the caller's atom order.  Either
 * pointer may be NULL.
 * Synchronises the stream.  Errors: REANN_ERR_STATE, REANN_ERR_ARG.
 */
reann_status reann_get_features(reann_ctx *ctx, int32_t t, float *rho, float *coef, reann_stream stream);

/*
 * Diagnostics (measurement).  enable != 0 starts timing every kernel launch
 * of this context with a CUDA event pair recorded on the launching stream,
 * and clears the accumulated times; enable == 0 stops it.  Timing adds two
 * event records per launch and never synchronises by itself; the times are
 * collected at the synchronisations the other calls already make.
 */
reann_status reann_profile(reann_ctx *ctx, int32_t enable);

/*
 * Accumulated device time (ms) and launch count of one kernel group since
 * the last reann_profile(ctx, 1).  Errors: REANN_ERR_ARG.
 */
reann_status reann_profile_read(const reann_ctx *ctx, int32_t group, double *ms, int64_t *launches);

/*
 * Allocation-free pair list (the paper has no counterpart: this serves
 * callers, not the method).  Some callers cannot allocate device memory:
 * programs that own the whole device through their own pool or a fixed
 * memory budget (an MD engine's force plug-in, for example, receives its
 * buffers and may not grow the footprint), and latency-critical loops that
 * avoid cudaMalloc/cudaFree because those can synchronise the whole device.
 * This call needs no context and allocates nothing: the caller passes inputs
 * and outputs, and the scratch
 * (cell bins, sorted cell lists, row counts) lives in one fixed file-scope
 * device array of about 2.5 MB that every GPU loading the library holds until
 * the process exits.
 *
 * Computes the list reann_build_neighbors builds, in the caller's order: row
 * [n+1] (device int32) receives the offsets, col [cap] (device int32) every j
 * with (i, j), i != j, within r_cut + skin under the same fp64 no-FMA test,
 * rows sorted by j.  pos: device float32 [n][3] (A); box: host double[3];
 * nnz: host, receives the list length.  At most 131,072 atoms: larger n is
 * rejected with REANN_ERR_CAPACITY before any GPU work; if the list outgrows
 * cap, or has more than 2^31-1 entries (the int32 offsets' range),
 * REANN_ERR_CAPACITY is returned with *nnz set and col not written (row is
 * meaningful only when the list fits the int32 range).  Other errors:
 * REANN_ERR_ARG, REANN_ERR_BOX, REANN_ERR_NONFINITE, REANN_ERR_CUDA;
 * reann_last_error(NULL) gives the message.
 *
 * All calls share the scratch array and it keeps the last call's contents;
 * each call clears what must start at zero.  Calls whose GPU work overlaps
 * (two streams, or two host threads on one device) race on the array:
 * serialise them.  The first call on a device looks up the array's device
 * address with that device current (cudaGetSymbolAddress); make that first
 * call before any stream capture.  The address is kept for the rest of the
 * process: after cudaDeviceReset on a device the array may move, so the call
 * must not be used on that device again.  Synchronises the stream twice.
 */
reann_status reann_pair_list_noalloc(int64_t n, const float *pos, const double box[3], double r_cut, double skin,
                                     int32_t *row, int32_t *col, int64_t cap, int64_t *nnz, reann_stream stream);

/*
 * Checked builds.  libreann_checked.so is this library compiled with
 * REANN_CHECKED: every index that a kernel reads from a neighbour list, a
 * permutation, a ghost map or a halo list (and every row end of a list) is
 * tested against the length of the array it indexes before use.  One out of
 * range is replaced by 0, so the access stays inside the array; the call
 * that ran the kernel then returns REANN_ERR_INDEX, its outputs not valid.
 * No device trap is used.  Valid inputs give the same results as the
 * unchecked build.  Returns 1 in a checked build, 0 otherwise.
 */
int32_t reann_checked(void);

/*
 * Fault injection for the checked build, on the host side (nothing is made
 * to fault on the device): writes j into entry k (0 <= k < nnz, the list's
 * internal order) of the neighbour list the next energy+force call reads, as
 * a damaged list would hold it.  With j outside [0, n) that call returns
 * REANN_ERR_INDEX; reann_build_neighbors rebuilds the list.  Synchronises the
 * device.  Errors: REANN_ERR_UNSUPPORTED (unchecked build), REANN_ERR_STATE
 * (no list), REANN_ERR_ARG (k outside the list), REANN_ERR_CUDA.
 */
reann_status reann_debug_set_neighbor(reann_ctx *ctx, int64_t k, int32_t j);

#ifdef __cplusplus
}
#endif
#endif /* REANN_H */
