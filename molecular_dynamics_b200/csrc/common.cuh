// Internal declarations shared by the translation units of libreann.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <string>
#include <vector>

#include "../../include/reann.h"

namespace reann {

constexpr int NT = 10;          // Cartesian tuples for L = 2
constexpr int MAX_ELEMENTS = 8;
constexpr int MAX_T = 8;

// device status bits (or-ed into ctx->d_status)
enum : int {
    ST_NONFINITE = 1,
    ST_CAPACITY = 2,
    ST_SKIN = 4,
    ST_BADTYPE = 8,
    ST_TIMEOUT = 16,
    ST_INDEX = 32,      // checked builds: an index outside its array
};

// Checked builds (compiled with REANN_CHECKED): every index read from a
// neighbour list, permutation, ghost map or halo list is tested against the
// length of the array it indexes before use.  One out of range or-s ST_INDEX
// into the status word and is replaced by 0, so the access stays inside the
// array; the results of that call are then wrong and the call reports
// REANN_ERR_INDEX.  Other builds: no test, the index is used as read.
#ifdef REANN_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif
__device__ __forceinline__ int64_t checked(int64_t j, int64_t n, int *status) {
    if constexpr (kChecked) {
        if (j < 0 || j >= n) {
            atomicOr(status, ST_INDEX);
            return 0;
        }
    }
    return j;
}
// a row's end offset, tested against the list's length the same way
__device__ __forceinline__ int checked_end(int q1, int64_t len, int *status) {
    if constexpr (kChecked) {
        if (q1 < 0 || q1 > len) {
            atomicOr(status, ST_INDEX);
            return 0;
        }
    }
    return q1;
}

// geometry and model constants passed by value to the edge kernels
struct EdgeParams {
    double box[3];
    double inv_box[3];
    float L_hi[3], L_lo[3], inv_L[3];   // box edge as an fp32 pair L_hi + L_lo, and 1/L
    float r_cut, r_cut2;
    // theta = pi r / (2 r_c) as r th_hi + r th_lo, and the Gaussian centres
    // mu_n = r_c n / (N_phi - 1) as mu_hi[n] + mu_lo[n]: fp32 pairs of the fp64
    // constants, so that no constant carries a rounding error that every
    // atom would share (a systematic shift of the centres or of the cutoff
    // argument biases a large system's energy)
    float th_hi, th_lo;
    float alpha;
    float neg_alpha_log2e;   // -alpha log2(e): exp(-alpha t^2) = 2^(t^2 neg_alpha_log2e)
    float mu_hi[16], mu_lo[16];
    int64_t n_rows;   // rows (atoms and ghost slots) a neighbour index may name
    int64_t n_list;   // entries of the neighbour list (its capacity)
    int *status;      // device status word (checked builds)
};

// offsets (in floats) of one atomic network inside the device weight blob
struct NetOffsets {
    int64_t shift, scale, W1, b1, W2, b2, W3, b3;
    int n_out;
};

// Lane decomposition of the edge kernels: a slot of LPE = N_phi / 2 lanes
// works on one edge, lane `sub` of the slot owning radial indices 2 sub and
// 2 sub + 1.  dE/dA rows (G) are stored lane-interleaved so that a slot's
// loads of one neighbour's row are contiguous: the 20 values of lane `sub`
// sit at
//   p = (idx / 4) * 4 LPE + 4 sub + idx % 4,
// with idx = 2 tau + m for radial index 2 sub + m in the pair order, where
// each float4 holds two tuples' (m = 0, m = 1) pairs for packed fp32
// arithmetic, and idx = 10 m + tau in the radial-major order.  The backward
// pass of layer t takes the pair order except for N_phi = 8 at t >= 1 (see
// the edge kernels), and the networks write each layer's rows in its order.
__host__ __device__ constexpr bool g_pairs(int NP, int layer) { return !(NP == 8 && layer >= 1); }
__host__ __device__ constexpr int g_lane_index(int m, int tau, bool pairs) {
    return pairs ? 2 * tau + m : m * NT + tau;
}
__host__ __device__ constexpr int g_slot_index(int n, int tau, int NP, bool pairs) {
    return (g_lane_index(n % 2, tau, pairs) / 4) * 4 * (NP / 2) + 4 * (n / 2) + g_lane_index(n % 2, tau, pairs) % 4;
}
// inverse: the (radial index, tuple) stored at position p, as n * 10 + tau
__host__ __device__ constexpr int g_slot_source(int p, int NP, bool pairs) {
    return (2 * ((p % (4 * (NP / 2))) / 4) +
            (pairs ? ((p / (4 * (NP / 2))) * 4 + p % 4) % 2 : ((p / (4 * (NP / 2))) * 4 + p % 4) / NT)) * NT +
           (pairs ? ((p / (4 * (NP / 2))) * 4 + p % 4) / 2 : ((p / (4 * (NP / 2))) * 4 + p % 4) % NT);
}
constexpr bool g_slot_roundtrip(int NP, bool pairs) {
    for (int n = 0; n < NP; ++n)
        for (int t = 0; t < NT; ++t)
            if (g_slot_source(g_slot_index(n, t, NP, pairs), NP, pairs) != n * NT + t) return false;
    return true;
}
static_assert(g_slot_roundtrip(8, true) && g_slot_roundtrip(10, true) && g_slot_roundtrip(8, false) &&
                  g_slot_roundtrip(10, false),
              "dE/dA lane orders are permutations");

struct Ctx;

// --- host orchestration helpers (defined across the .cu files) -------------
cudaError_t scan_exclusive(const int *in, int *out, int64_t n, int64_t *d_total, void *tmp, cudaStream_t s);
// message returned by reann_last_error(NULL) on this host thread
void set_context_free_error(const std::string &msg);
size_t scan_tmp_bytes(int64_t n);

}  // namespace reann

// The context.  All device pointers are owned by the context.
struct reann_ctx {
    reann_config cfg;
    int device = 0;
    int sm_count = 0;
    int NP = 0, D = 0, NA = 0, T = 0, ne = 0, H1 = 0, H2 = 0;
    int DR = 0;   // density features per atom (network input width): D, or N_phi (N_phi+1)(L+1)/2 in the pair form

    // weights.  The networks' input shifts live apart from the blob: the
    // density kernels subtract them in fp64 before rounding to fp32 (d_rho
    // holds rho - shift), so a feature close to its shift keeps its relative
    // precision; the device blob's shift entries are zero.
    float *d_w = nullptr;
    float *d_shift = nullptr;          // [T][ne][DR]: layer t feeds M^t (t < T-1) or the energy network
    std::vector<float> h_shift;
    int64_t n_w = 0;
    std::vector<reann::NetOffsets> coef_nets;  // [(T-1) * ne]
    std::vector<reann::NetOffsets> energy_nets;  // [ne]

    // atoms
    int64_t n = 0;          // atoms the workspaces are sized for
    int64_t n_alloc = 0;
    bool have_list = false;
    bool have_eval = false;
    double box[3] = {0, 0, 0};
    int m[3] = {0, 0, 0};   // cells per axis
    int ncell = 0;
    int nbins = 0;          // ne * ncell
    int64_t nbins_alloc = 0;
    std::vector<int> elem_start;  // [ne + 1], host copy of the element segments
    int *h_seg = nullptr;         // pinned [MAX_ELEMENTS + 1]
    std::vector<float> h_C0;      // element coefficient table c^0

    // neighbour search
    int *d_bin_count = nullptr, *d_bin_start = nullptr, *d_bin_fill = nullptr;
    int *d_key = nullptr;          // caller order
    int *d_perm = nullptr;         // internal -> caller
    int *d_perm_tmp = nullptr;
    int *d_inv = nullptr;          // caller -> internal
    int *d_types_caller = nullptr; // caller order
    float4 *d_pos = nullptr;       // [n_slots] internal order: x, y, z, type bits
    float4 *d_pos_build = nullptr; // positions at the last build
    int *d_row = nullptr;          // [n + 1]
    int *d_cnt = nullptr;          // [n]
    int *d_col = nullptr;          // [cap]
    int *d_act_cnt = nullptr;      // [n]
    int *d_act_col = nullptr;      // [cap]
    float4 *d_act_geo = nullptr;   // [cap] displacement and distance of each active entry
    float *d_act_dr = nullptr;     // [cap] fp32-accurate paths: r - fp32(r) of each active entry, from the
                                   // exact displacement (the densities are stiff in r: Gaussian slopes 2 alpha t)
    int64_t nnz = 0, cap = 0, max_row = 0;
    void *d_scan_tmp = nullptr;
    size_t scan_tmp_size = 0;
    int64_t *d_i64 = nullptr;      // small scratch of int64 scalars
    int64_t *h_i64 = nullptr;      // pinned mirror

    // multi-process spatial decomposition (reann_halo_plan): caller atoms
    // [0, n_local) are this process's own, [n_local, n) ghosts from other
    // processes; internal order keeps the own atoms in [0, n_local)
    bool halo = false;
    int64_t n_local = 0;           // atoms whose densities, networks and energies this process evaluates
    int64_t n_ghost_plan = 0;
    int64_t n_send = 0;            // rows this process sends (its own atoms that are ghosts elsewhere)
    int *d_send_caller = nullptr;  // [n_send] caller index of each sent row
    int64_t n_send_atoms = 0;      // distinct own atoms among them
    int *d_send_atom = nullptr;    // [n_send_atoms] their caller indices, ascending
    int *d_send_off = nullptr;     // [n_send_atoms + 1] offsets into d_send_order
    int *d_send_order = nullptr;   // [n_send] sent-row positions grouped by atom, ascending
    float *d_xsend = nullptr, *d_xrecv = nullptr;   // exchange buffers
    int64_t xbuf_alloc = 0;        // floats in each
    int64_t halo_bytes_fwd = 0, halo_bytes_bwd = 0; // per layer, this process's send side

    // domain-decomposed checking mode: slots [0, n) local atoms, [n, n_slots) ghosts
    bool dd = false;
    int64_t n_slots = 0, slots_alloc = 0;
    int64_t dd_ghosts = 0;
    int *d_dd_sub = nullptr;       // [n] subdomain of each internal atom
    unsigned *d_dd_bits = nullptr; // [P][ceil(n/32)] ghost membership
    int *d_dd_prefix = nullptr, *d_dd_cnt = nullptr;
    int64_t dd_words_alloc = 0;
    int *d_dd_owner = nullptr;     // [n_ghost] internal index of each ghost's owner
    int64_t dd_owner_alloc = 0;
    int *d_col_dd = nullptr;       // [cap] list columns as slots
    int64_t col_dd_alloc = 0;

    // per-layer activations
    float *d_A = nullptr;      // [T][n][NA]
    float *d_rho = nullptr;    // [T][n][D]
    float *d_coef = nullptr;   // [T][n_slots][D]  (layer 0 unused: c^0 comes from C0)
    float *d_G = nullptr;      // [n_slots][NA]  dE/dA^t
    float *d_dc = nullptr;     // [n][D]   dE/dc^t
    float *d_tanhd = nullptr;  // [T-1][n][2 H] tanh' of both hidden layers (three-pass tf32 networks)
    float *d_Ei = nullptr;     // [n]
    float *d_F = nullptr;      // [n][3] internal order
    double *d_Epart = nullptr; // block partial sums of E
    double *d_E = nullptr;     // [4] energies (pot, kin, ...)
    int n_part = 0;

    // MLP tile tables: per tile (element, first row, rows); 32-row tiles for
    // the CUDA-core networks, 128-row tiles for the tensor-core networks
    int4 *d_tiles = nullptr;
    int n_tiles = 0, n_tiles_alloc = 0;
    int4 *d_tiles128 = nullptr;
    int n_tiles128 = 0, n_tiles128_alloc = 0;
    int n_tc_ranges = 0;   // tensor-core network blocks; their ranges follow the 128-row tiles

    // staging for host arrays and caller-order scratch
    float *d_stage_f = nullptr;    // [n][3] floats
    int *d_stage_i = nullptr;      // [n]
    double *d_stage_x = nullptr;   // [n][3]
    double *d_stage_v = nullptr;   // [n][3]
    float *d_stage_e = nullptr;    // [n]
    float *d_diag = nullptr;       // [n][max(D, NA)] diagnostics scratch
    // MD state in internal order
    double *d_x = nullptr, *d_v = nullptr;  // [n][3]
    // state returned by the last MD call (caller order), for continuation checks,
    // and the buffer pair the next call writes (swapped per continuing call, so a
    // call's comparison reads the previous result while its own steps run)
    double *d_last_x = nullptr, *d_last_v = nullptr;
    double *d_last_x_alt = nullptr, *d_last_v_alt = nullptr;
    // a continuing call's copy of the caller's x and v, moved in and compared on
    // i_stream while the steps run (i_ev: start, caller's x read, comparison done)
    double *d_in_x = nullptr, *d_in_v = nullptr;
    cudaStream_t i_stream = nullptr;
    cudaEvent_t i_ev[3] = {nullptr, nullptr, nullptr};
    bool md_valid = false;
    double md_dt = 0.0;
    double md_mass[reann::MAX_ELEMENTS] = {};
    // one MD step's energy+force evaluation and closing half kick as a CUDA
    // graph, captured on a library stream once per neighbour list (and per
    // dt / masses) and replayed for the following steps
    cudaStream_t g_stream = nullptr;
    cudaEvent_t g_ev[2] = {nullptr, nullptr};
    cudaGraphExec_t g_exec = nullptr;
    bool g_valid = false;
    // what a captured graph bakes in -- buffer addresses, sizes, the box --
    // changes only when layout_gen does (a caller's list build, a grown
    // buffer, new network tiles, the checking mode's ghost maps); an MD
    // rebuild that reuses every buffer keeps the graphs
    int64_t layout_gen = 0;
    int64_t g_gen = -1, l_gen = -1;
    double g_dt = 0.0;
    double g_inv_mass[reann::MAX_ELEMENTS] = {};
    int64_t g_launches = 0;   // kernels one replay runs
    // the final positions of an MD call are copied out on this stream while
    // the last step's forces are evaluated
    cudaStream_t o_stream = nullptr;
    cudaEvent_t o_ev[2] = {nullptr, nullptr};
    bool g_disabled = false;  // REANN_GRAPHS=0 in the environment
    // MD calls of two or more steps replay whole stretches between neighbour
    // rebuilds as one graph: a WHILE node whose body is one step (kick-drift,
    // a gate kernel, then under an IF node energy+forces, the closing kick and
    // the thermostat); the host synchronises once per launch, not per step
    cudaGraphExec_t l_exec = nullptr;
    bool l_valid = false;
    bool l_disabled = false;  // REANN_LOOP=0, or the loop graph could not be built
    double l_dt = 0.0;
    double l_inv_mass[reann::MAX_ELEMENTS] = {};
    double l_thermo[3] = {-1.0, 0.0, 0.0};   // thermostat c, Kt, Nf of the captured loop (c < 0: none)
    int64_t l_step_launches = 0;              // kernels one loop iteration runs
    int *d_loop = nullptr;    // [4]: steps admitted, steps requested, end reason, first step index
    int *h_loop = nullptr;    // pinned mirror
    double *d_noise = nullptr;    // NVT: the call's two numbers per step
    int64_t noise_alloc = 0;

    // status
    int *d_status = nullptr;
    int *h_status = nullptr;   // pinned
    double *h_E = nullptr;     // pinned

    reann_counters counters{};
    std::string last_error;

    // per-launch CUDA-event timing (reann_profile)
    bool prof = false;
    struct ProfRec {
        int group;
        cudaEvent_t a, b;
    };
    std::vector<ProfRec> prof_pending;
    std::vector<cudaEvent_t> prof_pool;
    double prof_ms[REANN_K_COUNT] = {};
    int64_t prof_n[REANN_K_COUNT] = {};
};

namespace reann {
// Brackets one kernel launch: counts it and, when profiling, records an event
// pair on the launching stream.
struct LaunchScope {
    reann_ctx *c;
    int group;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    LaunchScope(reann_ctx *c_, int g, cudaStream_t s_, int kernels = 1);
    ~LaunchScope();
};
void prof_harvest(reann_ctx *c);  // after a synchronisation of the stream
}  // namespace reann
#define REANN_CAT2(a, b) a##b
#define REANN_CAT(a, b) REANN_CAT2(a, b)
#define REANN_TIMED(...) ::reann::LaunchScope REANN_CAT(_reann_scope_, __LINE__)(__VA_ARGS__)
