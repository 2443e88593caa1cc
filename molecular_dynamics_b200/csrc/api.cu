// C ABI entry points of libreann.so (declared in include/reann.h).
//
// Orchestration of one energy+force evaluation, following "Efficient
// Parallelization of Message Passing Neural Network Potentials for
// Large-Scale Molecular Dynamics":
//   forward  (section "REANN Architecture", Eqs. 1-2)
//     t = 0 .. T-1:  A^t, rho^t from c^t (c^0 = element table)   [edge.cu]
//                    c^{t+1} = M^t(rho^t) for t < T-1            [mlp*.cu]
//     E_i = N(rho^{T-1}) and G^{T-1} = dE/dA^{T-1}                [mlp*.cu]
//   backward (section "Parallelization Algorithm", Eqs. 3-5)
//     t = T-1 .. 0:  F += edge VJP, dE/dc^t                      [edge.cu]
//                    G^{t-1} from M^{t-1}'s VJP (Eq. 5)          [mlp*.cu]
//   E = sum_i E_i (deterministic fp64 tree)                      [md.cu]
// The networks run on the tensor cores: bf16 operands (mlp_tc.cu; mlp_tc_pair.cu
// for the pair-product densities) or fp32-accurate three-pass tf32 for hidden
// widths [64, 64] (mlp_tc32.cu); the other fp32 shapes, and mlp_precision 2,
// use the CUDA cores (mlp.cu).
// reann_md_step replays each step's evaluation and closing half kick as a
// CUDA graph captured once per neighbour list (ef_and_kick).
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"

using namespace reann;

namespace {

thread_local std::string g_create_error;

struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

reann_status fail(reann_ctx *c, reann_status st, const std::string &msg) {
    if (c) c->last_error = msg;
    else g_create_error = msg;
    return st;
}

reann_status cuda_fail(reann_ctx *c, cudaError_t e, const char *where) {
    cudaGetLastError();
    return fail(c, REANN_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

#define CK(call)                                              \
    do {                                                      \
        cudaError_t _e = (call);                              \
        if (_e != cudaSuccess) return cuda_fail(c, _e, #call); \
    } while (0)

bool is_device_ptr(const void *p) {
    if (!p) return false;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

template <class T>
cudaError_t dalloc(T **p, size_t count) {
    if (*p) {
        cudaFree(*p);
        *p = nullptr;
    }
    if (count == 0) count = 1;
    return cudaMalloc((void **)p, sizeof(T) * count);
}

template <class T>
void dfree(T *&p) {
    if (p) cudaFree(p);
    p = nullptr;
}

int64_t net_size(const reann_ctx *c, int n_out) {
    return 2LL * c->DR + (int64_t)c->H1 * c->DR + c->H1 + (int64_t)c->H2 * c->H1 + c->H2 + (int64_t)n_out * c->H2 +
           n_out;
}

NetOffsets bind_net(const reann_ctx *c, int64_t &off, int n_out) {
    NetOffsets o;
    o.n_out = n_out;
    o.shift = off; off += c->DR;
    o.scale = off; off += c->DR;
    o.W1 = off; off += (int64_t)c->H1 * c->DR;
    o.b1 = off; off += c->H1;
    o.W2 = off; off += (int64_t)c->H2 * c->H1;
    o.b2 = off; off += c->H2;
    o.W3 = off; off += (int64_t)n_out * c->H2;
    o.b3 = off; off += n_out;
    return o;
}

void free_atoms(reann_ctx *c) {
    dfree(c->d_key); dfree(c->d_perm); dfree(c->d_perm_tmp); dfree(c->d_inv); dfree(c->d_types_caller);
    dfree(c->d_pos); dfree(c->d_pos_build); dfree(c->d_row); dfree(c->d_cnt); dfree(c->d_act_cnt);
    dfree(c->d_A); dfree(c->d_rho); dfree(c->d_coef); dfree(c->d_G); dfree(c->d_dc); dfree(c->d_Ei);
    dfree(c->d_F); dfree(c->d_Epart); dfree(c->d_stage_f); dfree(c->d_stage_i); dfree(c->d_stage_x);
    dfree(c->d_stage_v); dfree(c->d_stage_e); dfree(c->d_x); dfree(c->d_v); dfree(c->d_diag);
    dfree(c->d_last_x); dfree(c->d_last_v); dfree(c->d_dd_sub); dfree(c->d_tanhd);
    dfree(c->d_last_x_alt); dfree(c->d_last_v_alt); dfree(c->d_in_x); dfree(c->d_in_v);
    c->md_valid = false;
    c->slots_alloc = 0;
    c->n_alloc = 0;
}

reann_status ensure_atoms(reann_ctx *c, int64_t n) {
    if (n <= c->n_alloc && c->d_row) return REANN_OK;
    free_atoms(c);
    size_t N = (size_t)n;
    CK(dalloc(&c->d_key, N));
    CK(dalloc(&c->d_perm, N));
    CK(dalloc(&c->d_perm_tmp, N));
    CK(dalloc(&c->d_inv, N));
    CK(dalloc(&c->d_types_caller, N));
    CK(dalloc(&c->d_pos, N));
    CK(dalloc(&c->d_pos_build, N));
    CK(dalloc(&c->d_row, N + 1));
    CK(dalloc(&c->d_cnt, N));
    CK(dalloc(&c->d_act_cnt, N));
    CK(dalloc(&c->d_A, (size_t)c->T * N * c->NA));
    CK(dalloc(&c->d_rho, (size_t)c->T * N * c->DR));
    CK(dalloc(&c->d_coef, (size_t)c->T * N * c->D));
    CK(dalloc(&c->d_G, N * c->NA));
    CK(dalloc(&c->d_dc, N * c->D));
    CK(dalloc(&c->d_Ei, N));
    CK(dalloc(&c->d_F, 3 * N));
    CK(dalloc(&c->d_Epart, N / 256 + 2));
    CK(dalloc(&c->d_stage_f, 3 * N));
    CK(dalloc(&c->d_stage_i, N));
    CK(dalloc(&c->d_stage_x, 3 * N));
    CK(dalloc(&c->d_stage_v, 3 * N));
    CK(dalloc(&c->d_stage_e, N));
    CK(dalloc(&c->d_x, 3 * N));
    CK(dalloc(&c->d_v, 3 * N));
    CK(dalloc(&c->d_diag, N * (size_t)std::max(c->DR, c->NA)));
    CK(dalloc(&c->d_last_x, 3 * N));
    CK(dalloc(&c->d_last_v, 3 * N));
    CK(dalloc(&c->d_last_x_alt, 3 * N));
    CK(dalloc(&c->d_last_v_alt, 3 * N));
    CK(dalloc(&c->d_in_x, 3 * N));
    CK(dalloc(&c->d_in_v, 3 * N));
    if (c->dd) CK(dalloc(&c->d_dd_sub, N));
    if (c->cfg.mlp_precision == 0 && tc32_supported(c))
        CK(dalloc(&c->d_tanhd, (size_t)std::max(c->T - 1, 1) * N * (size_t)(c->H1 + c->H2)));
    c->slots_alloc = n;
    c->n_alloc = n;
    return REANN_OK;
}

// slot-sized arrays (positions, coefficients, dE/dA) for n_slots >= n slots;
// the first n positions are kept
reann_status ensure_slots(reann_ctx *c, int64_t n_slots, cudaStream_t s) {
    if (n_slots != c->n_slots) ++c->layout_gen;
    c->n_slots = n_slots;
    if (n_slots <= c->slots_alloc) return REANN_OK;
    float4 *pos = nullptr;
    CK(cudaMalloc(&pos, sizeof(float4) * (size_t)n_slots));
    if (c->n > 0) CK(cudaMemcpyAsync(pos, c->d_pos, sizeof(float4) * (size_t)c->n, cudaMemcpyDeviceToDevice, s));
    CK(cudaStreamSynchronize(s));
    dfree(c->d_pos);
    c->d_pos = pos;
    CK(dalloc(&c->d_coef, (size_t)c->T * n_slots * c->D));
    CK(dalloc(&c->d_G, (size_t)n_slots * c->NA));
    c->slots_alloc = n_slots;
    return REANN_OK;
}

reann_status ensure_scan_tmp(reann_ctx *c, int64_t n) {
    size_t need = scan_tmp_bytes(n);
    if (need <= c->scan_tmp_size) return REANN_OK;
    if (c->d_scan_tmp) cudaFree(c->d_scan_tmp);
    c->d_scan_tmp = nullptr;
    CK(cudaMalloc(&c->d_scan_tmp, need));
    c->scan_tmp_size = need;
    return REANN_OK;
}

reann_status ensure_bins(reann_ctx *c) {
    if (c->nbins <= c->nbins_alloc) return REANN_OK;
    CK(dalloc(&c->d_bin_count, (size_t)c->nbins + 1));
    CK(dalloc(&c->d_bin_start, (size_t)c->nbins + 1));
    CK(dalloc(&c->d_bin_fill, (size_t)c->nbins + 1));
    c->nbins_alloc = c->nbins;
    return REANN_OK;
}

reann_status ensure_capacity(reann_ctx *c, int64_t nnz) {
    if (nnz <= c->cap && c->d_col) return REANN_OK;
    ++c->layout_gen;
    int64_t cap = nnz + nnz / 5 + 1024;
    if (cap > INT32_MAX) cap = INT32_MAX;
    CK(dalloc(&c->d_col, (size_t)cap));
    CK(dalloc(&c->d_act_col, (size_t)cap));
    CK(dalloc(&c->d_act_geo, (size_t)cap));
    if (c->cfg.mlp_precision != 1) CK(dalloc(&c->d_act_dr, (size_t)cap));
    c->cap = cap;
    return REANN_OK;
}

cudaError_t sync_stream(reann_ctx *c, cudaStream_t s) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) prof_harvest(c);
    return e;
}

// status word -> API status
reann_status check_status(reann_ctx *c, int st) {
    if (st & ST_INDEX) return fail(c, REANN_ERR_INDEX, "an internal index was outside its array (checked build)");
    if (st & ST_BADTYPE) return fail(c, REANN_ERR_ARG, "atom type outside [0, n_elements)");
    if (st & ST_NONFINITE) return fail(c, REANN_ERR_NONFINITE, "non-finite position, energy or force");
    if (st & ST_CAPACITY) return fail(c, REANN_ERR_CAPACITY, "neighbour capacity exceeded");
    if (st & ST_TIMEOUT) return fail(c, REANN_ERR_TIMEOUT, "a bounded device wait gave up");
    if (st & ST_SKIN) return fail(c, REANN_ERR_SKIN, "an atom moved more than skin/2 since the neighbour list was built");
    return REANN_OK;
}

// Binning + CSR for the caller-order float positions/types already on the
// device.  Reads nnz back (one synchronisation) and grows the list if needed.
reann_status build_internal(reann_ctx *c, const float *d_pos_caller, const int *d_types_caller, cudaStream_t s) {
    if (c->dd) ++c->layout_gen;   // the checking mode's ghost maps and slot count change with the list
    CK(cudaMemsetAsync(c->d_status, 0, sizeof(int), s));
    CK(launch_build(c, d_pos_caller, d_types_caller, s));
    CK(cudaMemcpyAsync(c->h_i64, c->d_i64, sizeof(int64_t) * 3, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_status, c->d_status, sizeof(int), cudaMemcpyDeviceToHost, s));
    // element segment starts: bin_start[e * ncell]
    for (int e = 0; e <= c->ne; ++e)
        CK(cudaMemcpyAsync(c->h_seg + e, c->d_bin_start + (int64_t)e * c->ncell, sizeof(int), cudaMemcpyDeviceToHost, s));
    CK(sync_stream(c, s));
    reann_status st = check_status(c, *c->h_status & ~ST_SKIN);
    if (st) return st;
    int64_t nnz = c->h_i64[1];
    if (nnz > INT32_MAX) return fail(c, REANN_ERR_CAPACITY, "neighbour list exceeds 2^31-1 entries");
    if ((st = ensure_capacity(c, nnz))) return st;
    CK(launch_fill(c, s));
    c->nnz = nnz;
    c->max_row = c->h_i64[2];
    // tile tables of the atomic networks: element segments cut into 32-row
    // (CUDA cores) and 128-row (tensor cores) tiles; segments only change when
    // the atoms' element counts do
    bool same = c->elem_start.size() == (size_t)c->ne + 1 &&
                std::equal(c->elem_start.begin(), c->elem_start.end(), c->h_seg);
    if (!same) {
        ++c->layout_gen;
        std::vector<int4> tiles, tiles128;
        for (int e = 0; e < c->ne; ++e) {
            for (int r = c->h_seg[e]; r < c->h_seg[e + 1]; r += 32)
                tiles.push_back(make_int4(e, r, std::min(32, c->h_seg[e + 1] - r), 0));
            for (int r = c->h_seg[e]; r < c->h_seg[e + 1]; r += 128)
                tiles128.push_back(make_int4(e, r, std::min(128, c->h_seg[e + 1] - r), 0));
        }
        if ((int)tiles.size() > c->n_tiles_alloc) {
            CK(dalloc(&c->d_tiles, tiles.size()));
            c->n_tiles_alloc = (int)tiles.size();
        }
        // block ranges of the tensor-core networks, stored after the 128-row
        // tiles: each block takes a contiguous run of one element's tiles (its
        // weights are loaded once), at most one block per SM
        const int n128 = (int)tiles128.size();
        std::vector<int4> table(tiles128);
        if (n128) {
            const int blocks = std::max(1, c->sm_count - c->ne);
            const int per = (n128 + blocks - 1) / blocks;
            for (int t = 0; t < n128;) {
                int u = t;
                while (u < n128 && tiles128[u].x == tiles128[t].x) ++u;
                const int k = (u - t + per - 1) / per;
                for (int b = 0; b < k; ++b)
                    table.push_back(make_int4(t + (int)((int64_t)(u - t) * b / k),
                                              t + (int)((int64_t)(u - t) * (b + 1) / k), tiles128[t].x, 0));
                t = u;
            }
        }
        if ((int)table.size() > c->n_tiles128_alloc) {
            CK(dalloc(&c->d_tiles128, table.size()));
            c->n_tiles128_alloc = (int)table.size();
        }
        if (!tiles.empty())
            CK(cudaMemcpyAsync(c->d_tiles, tiles.data(), sizeof(int4) * tiles.size(), cudaMemcpyHostToDevice, s));
        if (!table.empty())
            CK(cudaMemcpyAsync(c->d_tiles128, table.data(), sizeof(int4) * table.size(), cudaMemcpyHostToDevice, s));
        CK(sync_stream(c, s));
        c->n_tiles = (int)tiles.size();
        c->n_tiles128 = n128;
        c->n_tc_ranges = (int)table.size() - n128;
        c->elem_start.assign(c->h_seg, c->h_seg + c->ne + 1);
    }
    c->n_slots = c->n;
    if (c->dd) {
        int64_t ng = 0;
        CK(dd_plan(c, s, &ng));
        if (ng > INT32_MAX - c->n) return fail(c, REANN_ERR_CAPACITY, "too many ghost slots");
        if (ng > c->dd_owner_alloc) {
            CK(dalloc(&c->d_dd_owner, (size_t)ng));
            c->dd_owner_alloc = ng;
        }
        if (c->cap > c->col_dd_alloc) {
            CK(dalloc(&c->d_col_dd, (size_t)c->cap));
            c->col_dd_alloc = c->cap;
        }
        reann_status st2 = ensure_slots(c, c->n + ng, s);
        if (st2) return st2;
        c->dd_ghosts = ng;
        CK(dd_finish(c, s));
        c->counters.ghost_slots = ng;
        c->counters.ghost_bytes_fwd = ng * c->D * (int64_t)sizeof(float);
        c->counters.ghost_bytes_bwd = ng * c->NA * (int64_t)sizeof(float);
    }
    c->have_list = true;
    c->counters.builds++;
    return REANN_OK;
}

// One energy+force evaluation on the internal positions d_pos.
reann_status run_ef(reann_ctx *c, cudaStream_t s) {
    const bool tc = c->cfg.mlp_precision == 1, pair = c->cfg.density_form == 1;
    const bool tc32 = c->cfg.mlp_precision == 0 && tc32_supported(c);
    const int64_t cstride = c->n_slots * c->D;
    // domain-decomposed mode: ghost positions follow their owners
    if (c->dd) CK(dd_gather_rows(c, reinterpret_cast<float *>(c->d_pos), 4, s));
    CK(launch_active(c, s));
    for (int t = 0; t < c->T; ++t) {
        CK(launch_density_fwd(c, t, s));
        if (t + 1 < c->T) {
            CK(tc ? (pair ? launch_mlp_tc_pair_coef_fwd(c, t, s) : launch_mlp_tc_coef_fwd(c, t, s))
                  : (tc32 ? launch_mlp_tc32_coef_fwd(c, t, s) : launch_mlp_coef_fwd(c, t, s)));
            // the per-layer message sync: ghost c^{t+1} from the owners (or, as
            // a negative control, the ghosts keep c^0)
            if (c->dd) {
                float *coef = c->d_coef + (t + 1) * cstride;
                CK(c->cfg.dd_stale_ghosts ? dd_stale_coef(c, coef, s) : dd_gather_rows(c, coef, c->D, s));
            }
        }
    }
    CK(tc ? (pair ? launch_mlp_tc_pair_energy(c, s) : launch_mlp_tc_energy(c, s))
          : (tc32 ? launch_mlp_tc32_energy(c, s) : launch_mlp_energy(c, s)));
    if (c->dd) CK(dd_gather_rows(c, c->d_G, c->NA, s));
    for (int t = c->T - 1; t >= 0; --t) {
        CK(launch_edge_bwd(c, t, t != c->T - 1, s));
        if (t >= 1) {
            CK(tc ? (pair ? launch_mlp_tc_pair_coef_bwd(c, t, s) : launch_mlp_tc_coef_bwd(c, t, s))
                  : (tc32 ? launch_mlp_tc32_coef_bwd(c, t, s) : launch_mlp_coef_bwd(c, t, s)));
            if (c->dd) CK(dd_gather_rows(c, c->d_G, c->NA, s));
        }
    }
    CK(launch_energy_sum(c, s));
    c->counters.evaluations++;
    c->have_eval = true;
    return REANN_OK;
}

// The part of an MD step after the skin check: energy+forces and the second
// half kick.  Eager launches on `s` while profiling (per-launch events) or with
// REANN_GRAPHS=0; otherwise one CUDA graph replay, captured on the library's
// stream the first time a neighbour list (with this dt and these masses) is
// used and ordered against `s` with events.
reann_status ef_and_kick(reann_ctx *c, double dt_fs, const double *inv_mass, cudaStream_t s) {
    reann_status st;
    if (c->prof || c->g_disabled || c->n == 0) {
        if ((st = run_ef(c, s))) return st;
        CK(launch_md_kick(c, dt_fs, inv_mass, s));
        return REANN_OK;
    }
    if (!c->g_stream) {
        CK(cudaStreamCreateWithFlags(&c->g_stream, cudaStreamNonBlocking));
        for (auto &ev : c->g_ev) CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    }
    const bool same = c->g_valid && c->g_gen == c->layout_gen && c->g_dt == dt_fs &&
                      std::equal(inv_mass, inv_mass + c->ne, c->g_inv_mass);
    CK(cudaEventRecord(c->g_ev[0], s));
    CK(cudaStreamWaitEvent(c->g_stream, c->g_ev[0], 0));
    if (!same) {
        if (c->g_exec) {
            cudaGraphExecDestroy(c->g_exec);
            c->g_exec = nullptr;
        }
        const int64_t k0 = c->counters.kernel_launches, e0 = c->counters.evaluations;
        CK(cudaStreamBeginCapture(c->g_stream, cudaStreamCaptureModeThreadLocal));
        st = run_ef(c, c->g_stream);
        cudaError_t ek = st ? cudaSuccess : launch_md_kick(c, dt_fs, inv_mass, c->g_stream);
        cudaGraph_t g = nullptr;
        cudaError_t ee = cudaStreamEndCapture(c->g_stream, &g);
        c->g_launches = c->counters.kernel_launches - k0;
        c->counters.kernel_launches = k0;
        c->counters.evaluations = e0;
        if (st || ek || ee) {
            if (g) cudaGraphDestroy(g);
            if (st) return st;
            CK(ek ? ek : ee);
        }
        cudaError_t ei = cudaGraphInstantiate(&c->g_exec, g, 0);
        cudaGraphDestroy(g);
        CK(ei);
        c->g_valid = true;
        c->g_gen = c->layout_gen;
        c->g_dt = dt_fs;
        std::copy(inv_mass, inv_mass + c->ne, c->g_inv_mass);
    }
    CK(cudaGraphLaunch(c->g_exec, c->g_stream));
    CK(cudaEventRecord(c->g_ev[1], c->g_stream));
    CK(cudaStreamWaitEvent(s, c->g_ev[1], 0));
    c->counters.kernel_launches += c->g_launches;
    c->counters.evaluations++;
    c->have_eval = true;
    return REANN_OK;
}

// Builds the device-side step loop (see reann_ctx::l_exec) for the current
// list, dt, masses and thermostat: a WHILE node whose body is kick-drift and
// the gate, followed by an IF node holding energy+forces, the closing kick and
// (NVT) the thermostat with its numbers read from d_noise.  Bodies are filled
// by stream capture on the library stream.
cudaError_t capture_loop(reann_ctx *c, double dt_fs, const double *inv_mass, const double *mass,
                         const BussiParams *B) {
    if (c->l_exec) {
        cudaGraphExecDestroy(c->l_exec);
        c->l_exec = nullptr;
    }
    c->l_valid = false;
    const int64_t k0 = c->counters.kernel_launches, e0 = c->counters.evaluations;
    cudaGraph_t lg = nullptr;
    cudaError_t e = cudaGraphCreate(&lg, 0);
    if (e) return e;
    struct Cleanup {
        cudaGraph_t g;
        reann_ctx *c;
        int64_t k0, e0;
        ~Cleanup() {
            if (g) cudaGraphDestroy(g);
            c->counters.kernel_launches = k0;
            c->counters.evaluations = e0;
        }
    } cleanup{lg, c, k0, e0};
    cudaGraphConditionalHandle h_while, h_step;
    if ((e = cudaGraphConditionalHandleCreate(&h_while, lg, 1, cudaGraphCondAssignDefault))) return e;
    cudaGraphNodeParams wp = {};
    wp.type = cudaGraphNodeTypeConditional;
    wp.conditional.handle = h_while;
    wp.conditional.type = cudaGraphCondTypeWhile;
    wp.conditional.size = 1;
    cudaGraphNode_t wnode;
    if ((e = cudaGraphAddNode(&wnode, lg, nullptr, 0, &wp))) return e;
    cudaGraph_t body = wp.conditional.phGraph_out[0];
    if ((e = cudaGraphConditionalHandleCreate(&h_step, body, 0, cudaGraphCondAssignDefault))) return e;
    // body: kick-drift, then the gate
    cudaGraph_t got = nullptr;
    if ((e = cudaStreamBeginCaptureToGraph(c->g_stream, body, nullptr, nullptr, 0, cudaStreamCaptureModeThreadLocal)))
        return e;
    cudaError_t e1 = launch_md_kick_drift(c, dt_fs, inv_mass, c->d_status + 1, c->g_stream);
    cudaError_t e2 = e1 ? e1 : launch_loop_gate(c, h_while, h_step, c->g_stream);
    e = cudaStreamEndCapture(c->g_stream, &got);
    if (e2) return e2;
    if (e) return e;
    // the gate is the body's one node without dependents
    size_t nn = 0;
    if ((e = cudaGraphGetNodes(body, nullptr, &nn))) return e;
    std::vector<cudaGraphNode_t> nodes(nn);
    if ((e = cudaGraphGetNodes(body, nodes.data(), &nn))) return e;
    cudaGraphNode_t leaf = nullptr;
    for (auto nd : nodes) {
        size_t nd_out = 0;
        if ((e = cudaGraphNodeGetDependentNodes(nd, nullptr, &nd_out))) return e;
        if (nd_out == 0) leaf = nd;
    }
    if (!leaf) return cudaErrorInvalidValue;
    cudaGraphNodeParams ip = {};
    ip.type = cudaGraphNodeTypeConditional;
    ip.conditional.handle = h_step;
    ip.conditional.type = cudaGraphCondTypeIf;
    ip.conditional.size = 1;
    cudaGraphNode_t inode;
    if ((e = cudaGraphAddNode(&inode, body, &leaf, 1, &ip))) return e;
    cudaGraph_t step_body = ip.conditional.phGraph_out[0];
    // the admitted step: energy+forces, closing kick, thermostat
    const int64_t k1 = c->counters.kernel_launches;
    if ((e = cudaStreamBeginCaptureToGraph(c->g_stream, step_body, nullptr, nullptr, 0,
                                           cudaStreamCaptureModeThreadLocal)))
        return e;
    reann_status st = run_ef(c, c->g_stream);
    e1 = st ? cudaSuccess : launch_md_kick(c, dt_fs, inv_mass, c->g_stream);
    if (!st && !e1 && B) e1 = launch_thermostat(c, mass, *B, c->d_E + 2, c->g_stream, c->d_noise, c->d_loop);
    e = cudaStreamEndCapture(c->g_stream, &got);
    if (st) return cudaErrorInvalidValue;
    if (e1) return e1;
    if (e) return e;
    c->l_step_launches = c->counters.kernel_launches - k0;
    (void)k1;
    if ((e = cudaGraphInstantiate(&c->l_exec, lg, 0))) {
        c->l_exec = nullptr;
        return e;
    }
    c->l_valid = true;
    c->l_gen = c->layout_gen;
    c->l_dt = dt_fs;
    std::copy(inv_mass, inv_mass + c->ne, c->l_inv_mass);
    c->l_thermo[0] = B ? B->c : -1.0;
    c->l_thermo[1] = B ? B->kt : 0.0;
    c->l_thermo[2] = B ? B->nf : 0.0;
    return cudaSuccess;
}

void fill_counters(reann_ctx *c) {
    c->counters.n_atoms = c->n;
    c->counters.nnz = c->nnz;
    c->counters.capacity = c->cap;
    c->counters.max_row = c->max_row;
    for (int a = 0; a < 3; ++a) c->counters.cells[a] = c->m[a];
}

}  // namespace

namespace reann {

void set_context_free_error(const std::string &msg) { g_create_error = msg; }

LaunchScope::LaunchScope(reann_ctx *c_, int g, cudaStream_t s_, int kernels) : c(c_), group(g), s(s_) {
    c->counters.kernel_launches += kernels;
    if (!c->prof) return;
    for (cudaEvent_t *ev : {&a, &b}) {
        if (!c->prof_pool.empty()) {
            *ev = c->prof_pool.back();
            c->prof_pool.pop_back();
        } else if (cudaEventCreate(ev) != cudaSuccess) {
            cudaGetLastError();
            *ev = nullptr;
        }
    }
    if (a && b) cudaEventRecord(a, s);
}

LaunchScope::~LaunchScope() {
    if (!a || !b) {
        if (a) c->prof_pool.push_back(a);
        if (b) c->prof_pool.push_back(b);
        return;
    }
    cudaEventRecord(b, s);
    c->prof_pending.push_back({group, a, b});
}

void prof_harvest(reann_ctx *c) {
    for (auto &r : c->prof_pending) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
            c->prof_ms[r.group] += ms;
            c->prof_n[r.group] += 1;
        } else {
            cudaGetLastError();
        }
        c->prof_pool.push_back(r.a);
        c->prof_pool.push_back(r.b);
    }
    c->prof_pending.clear();
}

}  // namespace reann

// ---------------------------------------------------------------------------

extern "C" reann_status reann_create(const reann_config *cfg, const void *weights, size_t nbytes, int device,
                                     reann_ctx **out) {
    if (!cfg || !weights || !out) return fail(nullptr, REANN_ERR_ARG, "null argument");
    *out = nullptr;
    if (cfg->n_elements < 1 || cfg->n_elements > MAX_ELEMENTS || cfg->T < 1 || cfg->T > MAX_T ||
        !(cfg->r_cut > 0) || !(cfg->skin >= 0) || !(cfg->alpha > 0) || !std::isfinite(cfg->r_cut) ||
        !std::isfinite(cfg->skin) || cfg->mlp_precision < 0 || cfg->mlp_precision > 2)
        return fail(nullptr, REANN_ERR_ARG, "invalid configuration");
    if (cfg->mlp_precision == 1 && (cfg->hidden[0] != 128 || cfg->hidden[1] != 128))
        return fail(nullptr, REANN_ERR_UNSUPPORTED, "bf16 tensor-core networks need hidden widths [128, 128]");
    if (cfg->l_max != 2 || (cfg->n_radial != 8 && cfg->n_radial != 10) ||
        (cfg->hidden[0] != 64 && cfg->hidden[0] != 128) || (cfg->hidden[1] != 64 && cfg->hidden[1] != 128))
        return fail(nullptr, REANN_ERR_UNSUPPORTED, "supported: l_max 2, n_radial 8 or 10, hidden widths 64 or 128");
    {
        const bool any = cfg->dd_grid[0] || cfg->dd_grid[1] || cfg->dd_grid[2];
        for (int a = 0; a < 3; ++a)
            if (any && (cfg->dd_grid[a] < 1 || cfg->dd_grid[a] > 64))
                return fail(nullptr, REANN_ERR_ARG, "dd_grid: all zero, or 1..64 subdomains per axis");
        if (cfg->dd_stale_ghosts < 0 || cfg->dd_stale_ghosts > 1) return fail(nullptr, REANN_ERR_ARG, "dd_stale_ghosts");
    }
    if (cfg->density_form < 0 || cfg->density_form > 1) return fail(nullptr, REANN_ERR_ARG, "density_form is 0 or 1");
    if (cfg->density_form == 1 && (cfg->n_radial != 8 || cfg->l_max != 2 || cfg->hidden[0] != cfg->hidden[1]))
        return fail(nullptr, REANN_ERR_UNSUPPORTED,
                    "the pair-product density form is built for N_phi = 8, L = 2 and equal hidden widths");
    reann_ctx *c = new reann_ctx();
    c->cfg = *cfg;
    c->device = device;
    {
        const char *gv = std::getenv("REANN_GRAPHS");
        c->g_disabled = gv && std::strcmp(gv, "0") == 0;
        const char *lv = std::getenv("REANN_LOOP");
        c->l_disabled = lv && std::strcmp(lv, "0") == 0;
    }
    c->NP = cfg->n_radial;
    c->D = c->NP * (cfg->l_max + 1);
    c->DR = cfg->density_form == 1 ? c->NP * (c->NP + 1) / 2 * (cfg->l_max + 1) : c->D;
    c->NA = c->NP * NT;
    c->T = cfg->T;
    c->ne = cfg->n_elements;
    c->H1 = cfg->hidden[0];
    c->H2 = cfg->hidden[1];
    c->dd = cfg->dd_grid[0] > 0;
    int64_t expect = (int64_t)c->ne * c->D + (int64_t)(c->T - 1) * c->ne * net_size(c, c->D) + (int64_t)c->ne * net_size(c, 1);
    if ((int64_t)nbytes != expect * (int64_t)sizeof(float)) {
        delete c;
        return fail(nullptr, REANN_ERR_ARG, "weight blob size does not match the configuration (expected " +
                                                std::to_string(expect * sizeof(float)) + " bytes)");
    }
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
        cudaGetLastError();
        delete c;
        return fail(nullptr, REANN_ERR_CUDA, "no such CUDA device");
    }
    DeviceGuard guard(device);
    int64_t off = (int64_t)c->ne * c->D;
    for (int t = 0; t + 1 < c->T; ++t)
        for (int e = 0; e < c->ne; ++e) c->coef_nets.push_back(bind_net(c, off, c->D));
    for (int e = 0; e < c->ne; ++e) c->energy_nets.push_back(bind_net(c, off, 1));
    c->n_w = expect;
    c->h_C0.assign((const float *)weights, (const float *)weights + (size_t)c->ne * c->D);
    // shifts out of the blob (see reann_ctx::d_shift)
    std::vector<float> blob((const float *)weights, (const float *)weights + expect);
    c->h_shift.assign((size_t)c->T * c->ne * c->DR, 0.f);
    for (int t = 0; t < c->T; ++t)
        for (int e = 0; e < c->ne; ++e) {
            const NetOffsets &o = t + 1 < c->T ? c->coef_nets[t * c->ne + e] : c->energy_nets[e];
            for (int f = 0; f < c->DR; ++f) {
                c->h_shift[((size_t)t * c->ne + e) * c->DR + f] = blob[o.shift + f];
                blob[o.shift + f] = 0.f;
            }
        }
    cudaError_t e;
    cudaDeviceProp prop;
    if ((e = cudaGetDeviceProperties(&prop, device)) ||
        (e = cudaMalloc(&c->d_w, nbytes)) ||
        (e = cudaMemcpy(c->d_w, blob.data(), nbytes, cudaMemcpyHostToDevice)) ||
        (e = cudaMalloc(&c->d_shift, sizeof(float) * c->h_shift.size())) ||
        (e = cudaMemcpy(c->d_shift, c->h_shift.data(), sizeof(float) * c->h_shift.size(), cudaMemcpyHostToDevice)) ||
        (e = cudaMalloc(&c->d_status, sizeof(int) * 4)) ||
        (e = cudaMemset(c->d_status, 0, sizeof(int) * 4)) ||
        (e = cudaMalloc(&c->d_i64, sizeof(int64_t) * 8)) ||
        (e = cudaMemset(c->d_i64, 0, sizeof(int64_t) * 8)) ||
        (e = cudaMalloc(&c->d_E, sizeof(double) * 4)) ||
        (e = cudaMallocHost(&c->h_status, sizeof(int) * 4)) ||
        (e = cudaMallocHost(&c->h_i64, sizeof(int64_t) * 8)) ||
        (e = cudaMallocHost(&c->h_E, sizeof(double) * 6)) ||
        (e = cudaMallocHost(&c->h_seg, sizeof(int) * (MAX_ELEMENTS + 1)))) {
        std::string msg = std::string("CUDA initialisation failed: ") + cudaGetErrorString(e);
        cudaGetLastError();
        reann_destroy(c);
        return fail(nullptr, REANN_ERR_CUDA, msg);
    }
    c->sm_count = prop.multiProcessorCount;
    *out = c;
    return REANN_OK;
}

extern "C" reann_status reann_destroy(reann_ctx *c) {
    if (!c) return REANN_OK;
    DeviceGuard guard(c->device);
    free_atoms(c);
    dfree(c->d_w); dfree(c->d_shift); dfree(c->d_bin_count); dfree(c->d_bin_start); dfree(c->d_bin_fill); dfree(c->d_col);
    dfree(c->d_dd_bits); dfree(c->d_dd_prefix); dfree(c->d_dd_cnt); dfree(c->d_dd_owner); dfree(c->d_col_dd);
    dfree(c->d_act_col); dfree(c->d_act_geo); dfree(c->d_act_dr); dfree(c->d_tiles); dfree(c->d_tiles128); dfree(c->d_status); dfree(c->d_i64); dfree(c->d_E);
    if (c->d_scan_tmp) cudaFree(c->d_scan_tmp);
    if (c->h_status) cudaFreeHost(c->h_status);
    if (c->h_i64) cudaFreeHost(c->h_i64);
    if (c->h_E) cudaFreeHost(c->h_E);
    if (c->h_seg) cudaFreeHost(c->h_seg);
    for (auto &r : c->prof_pending) {
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    for (auto ev : c->prof_pool) cudaEventDestroy(ev);
    dfree(c->d_send_caller); dfree(c->d_send_atom); dfree(c->d_send_off); dfree(c->d_send_order);
    dfree(c->d_xsend); dfree(c->d_xrecv);
    if (c->g_exec) cudaGraphExecDestroy(c->g_exec);
    if (c->l_exec) cudaGraphExecDestroy(c->l_exec);
    if (c->d_loop) cudaFree(c->d_loop);
    if (c->h_loop) cudaFreeHost(c->h_loop);
    if (c->d_noise) cudaFree(c->d_noise);
    for (auto ev : c->g_ev)
        if (ev) cudaEventDestroy(ev);
    if (c->g_stream) cudaStreamDestroy(c->g_stream);
    for (auto ev : c->o_ev)
        if (ev) cudaEventDestroy(ev);
    if (c->o_stream) cudaStreamDestroy(c->o_stream);
    for (auto ev : c->i_ev)
        if (ev) cudaEventDestroy(ev);
    if (c->i_stream) cudaStreamDestroy(c->i_stream);
    delete c;
    return REANN_OK;
}

extern "C" reann_status reann_build_neighbors(reann_ctx *c, int64_t n, const float *pos, const int32_t *types,
                                              const double box[3], reann_stream stream) {
    if (!c) return REANN_ERR_ARG;
    if (n < 0 || (n > 0 && (!pos || !types)) || !box) return fail(c, REANN_ERR_ARG, "invalid arguments");
    if (n >= INT32_MAX) return fail(c, REANN_ERR_CAPACITY, "too many atoms");
    DeviceGuard guard(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    double rl = c->cfg.r_cut + c->cfg.skin;
    for (int a = 0; a < 3; ++a)
        if (!(box[a] > 0) || !std::isfinite(box[a]) || box[a] < 2.0 * rl)
            return fail(c, REANN_ERR_BOX, "box edge must be finite and at least 2 (r_cut + skin)");
    if (c->halo && n != c->n_local + c->n_ghost_plan)
        return fail(c, REANN_ERR_ARG, "with a halo plan, n must be the plan's own plus ghost atoms");
    reann_status st;
    if ((st = ensure_atoms(c, n))) return st;
    ++c->layout_gen;   // a caller's build may change n, the box or any buffer
    c->n = n;
    c->have_list = c->have_eval = false;
    c->md_valid = false;
    int ncell = 1;
    for (int a = 0; a < 3; ++a) {
        c->box[a] = box[a];
        c->m[a] = std::max(1, (int)std::floor(box[a] / rl));
        ncell *= c->m[a];
    }
    c->ncell = ncell;
    c->nbins = ncell * c->ne * (c->halo ? 2 : 1);   // a halo plan's ghosts bin in classes of their own
    if ((st = ensure_bins(c))) return st;
    if ((st = ensure_scan_tmp(c, std::max<int64_t>(n, c->nbins)))) return st;
    const float *d_pos = pos;
    if (n > 0 && !is_device_ptr(pos)) {
        CK(cudaMemcpyAsync(c->d_stage_f, pos, sizeof(float) * 3 * n, cudaMemcpyHostToDevice, s));
        d_pos = c->d_stage_f;
    }
    if (n > 0) CK(cudaMemcpyAsync(c->d_types_caller, types, sizeof(int) * n, cudaMemcpyDefault, s));
    if ((st = build_internal(c, d_pos, c->d_types_caller, s))) return st;
    CK(sync_stream(c, s));
    fill_counters(c);
    return REANN_OK;
}

extern "C" reann_status reann_energy_forces(reann_ctx *c, const float *pos, double *energy, float *forces,
                                            float *atom_energy, reann_stream stream) {
    if (!c) return REANN_ERR_ARG;
    if (!c->have_list) return fail(c, REANN_ERR_STATE, "reann_build_neighbors must come first");
    if (c->halo) return fail(c, REANN_ERR_STATE, "a halo plan needs reann_energy_forces_halo");
    if (c->n > 0 && !pos) return fail(c, REANN_ERR_ARG, "null positions");
    DeviceGuard guard(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t n = c->n;
    c->md_valid = false;
    CK(cudaMemsetAsync(c->d_status, 0, sizeof(int), s));
    if (n > 0) {
        const float *d_pos = pos;
        if (!is_device_ptr(pos)) {
            CK(cudaMemcpyAsync(c->d_stage_f, pos, sizeof(float) * 3 * n, cudaMemcpyHostToDevice, s));
            d_pos = c->d_stage_f;
        }
        CK(launch_pos_from_caller(c, d_pos, s));
        CK(launch_skin_check(c, c->d_status, s));
    }
    reann_status st = run_ef(c, s);
    if (st) return st;
    bool f_dev = forces && is_device_ptr(forces), e_dev = atom_energy && is_device_ptr(atom_energy);
    float *fo = forces ? (f_dev ? forces : c->d_stage_f) : nullptr;
    float *eo = atom_energy ? (e_dev ? atom_energy : c->d_stage_e) : nullptr;
    CK(launch_scatter_outputs(c, fo, eo, s));
    if (forces && !f_dev && n > 0)
        CK(cudaMemcpyAsync(forces, c->d_stage_f, sizeof(float) * 3 * n, cudaMemcpyDeviceToHost, s));
    if (atom_energy && !e_dev && n > 0)
        CK(cudaMemcpyAsync(atom_energy, c->d_stage_e, sizeof(float) * n, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_E, c->d_E, sizeof(double), cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_status, c->d_status, sizeof(int), cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_i64 + 3, c->d_i64 + 3, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
    CK(sync_stream(c, s));
    c->counters.active_pairs = c->h_i64[3];
    fill_counters(c);
    if (energy) *energy = c->h_E[0];
    return check_status(c, *c->h_status);
}

constexpr double KB_EV = 8.617333262e-5;   // Boltzmann constant, eV/K (CODATA 2018)

// Canonical sampling by stochastic velocity rescaling: target temperature,
// coupling time and the caller's two random numbers per step (host).
struct NvtArgs {
    double temperature, tau;
    const double *noise;
};

// The steps of one MD call (velocity Verlet, with the thermostat applied after
// each step's closing half kick when nvt is given), from the resident state
// (resume) or from the caller-order state in d_stage_x / d_stage_v; results to
// the caller's x, v.  spec: the caller's x and v are being read in and
// compared on i_stream (a continuing call); writes to them wait for that.
// The d_E slots: [0] energy, [1] kinetic energy, [2] the step's rescaling
// factor, [3] thermostat work of this call.
static reann_status md_steps(reann_ctx *c, int32_t nsteps, double dt_fs, double *x, double *v, bool x_dev, bool v_dev,
                             const double *mass, const double *inv_mass, reann_md_stats *stats, cudaStream_t s,
                             const NvtArgs *nvt, BussiParams B, bool resume, bool spec) {
    const int64_t n = c->n;
    const size_t bytes3 = sizeof(double) * 3 * (size_t)n;
    reann_status st;
    int64_t rebuilds = 0;
    int32_t done = 0;
    c->md_valid = false;
    CK(cudaMemsetAsync(c->d_status, 0, sizeof(int) * 2, s));
    if (!resume) {
        if (n > 0) {
            // caller-order state (wrapped into the box) -> list -> internal order
            CK(launch_wrap_state(c, c->d_stage_x, c->d_stage_f, s));
            if ((st = build_internal(c, c->d_stage_f, c->d_types_caller, s))) return st;
            CK(launch_md_gather(c, c->d_stage_x, c->d_stage_v, s));
        }
        CK(cudaMemsetAsync(c->d_status, 0, sizeof(int) * 2, s));
        if ((st = run_ef(c, s))) return st;
    }
    CK(launch_kinetic(c, mass, c->d_E + 1, s));
    CK(cudaMemcpyAsync(c->h_E + 2, c->d_E, sizeof(double) * 2, cudaMemcpyDeviceToHost, s));
    CK(cudaMemsetAsync(c->d_E + 3, 0, sizeof(double), s));
    // the positions are final after the last step's drift (and list check):
    // they go out on the copy stream while that step's forces are evaluated.
    // Every return after that waits for the copy (the caller's buffer must
    // not be written after the call returns).
    struct CopyWait {
        cudaStream_t s = nullptr;
        ~CopyWait() {
            if (s) cudaStreamSynchronize(s);
        }
    } x_wait;
    if (nsteps > 0 && n > 0 && !c->o_stream) {
        CK(cudaStreamCreateWithFlags(&c->o_stream, cudaStreamNonBlocking));
        for (auto &ev : c->o_ev) CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    }
    int32_t step = 0;
    // all steps but the last between rebuilds on the device (one host
    // synchronisation per stretch); the last step keeps the overlapped copy-out
    const bool loop = !c->prof && !c->g_disabled && !c->l_disabled && n > 0 && nsteps >= 2;
    if (loop && nvt) {
        if (2 * (int64_t)nsteps > c->noise_alloc) {
            if (c->d_noise) cudaFree(c->d_noise);
            c->d_noise = nullptr;
            c->noise_alloc = 0;
            c->l_valid = false;   // the loop graph reads the noise through this pointer
            CK(cudaMalloc(&c->d_noise, sizeof(double) * 2 * (size_t)nsteps));
            c->noise_alloc = 2 * (int64_t)nsteps;
        }
        CK(cudaMemcpyAsync(c->d_noise, nvt->noise, sizeof(double) * 2 * (size_t)nsteps, cudaMemcpyHostToDevice, s));
    }
    while (loop && !c->l_disabled && step < nsteps - 1) {
        if (!c->g_stream) {
            CK(cudaStreamCreateWithFlags(&c->g_stream, cudaStreamNonBlocking));
            for (auto &ev : c->g_ev) CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
        }
        if (!c->d_loop) {
            CK(cudaMalloc(&c->d_loop, sizeof(int) * 4));
            CK(cudaMallocHost(&c->h_loop, sizeof(int) * 4));
        }
        const bool same = c->l_valid && c->l_gen == c->layout_gen && c->l_dt == dt_fs &&
                          std::equal(inv_mass, inv_mass + c->ne, c->l_inv_mass) &&
                          (nvt ? (c->l_thermo[0] == B.c && c->l_thermo[1] == B.kt && c->l_thermo[2] == B.nf)
                               : c->l_thermo[0] < 0);
        if (!same) {
            CK(cudaStreamSynchronize(s));
            cudaError_t el = capture_loop(c, dt_fs, inv_mass, mass, nvt ? &B : nullptr);
            if (el) {
                // this runtime or driver cannot build the loop graph: per-step graphs from here on
                cudaGetLastError();
                c->l_disabled = true;
                break;
            }
        }
        c->h_loop[0] = 0;
        c->h_loop[1] = nsteps - 1 - step;
        c->h_loop[2] = 0;
        c->h_loop[3] = step;
        CK(cudaMemcpyAsync(c->d_loop, c->h_loop, sizeof(int) * 4, cudaMemcpyHostToDevice, s));
        CK(cudaEventRecord(c->g_ev[0], s));
        CK(cudaStreamWaitEvent(c->g_stream, c->g_ev[0], 0));
        CK(cudaGraphLaunch(c->l_exec, c->g_stream));
        CK(cudaEventRecord(c->g_ev[1], c->g_stream));
        CK(cudaStreamWaitEvent(s, c->g_ev[1], 0));
        CK(cudaMemcpyAsync(c->h_loop, c->d_loop, sizeof(int) * 4, cudaMemcpyDeviceToHost, s));
        CK(cudaMemcpyAsync(c->h_status, c->d_status, sizeof(int) * 2, cudaMemcpyDeviceToHost, s));
        CK(sync_stream(c, s));
        const int admitted = c->h_loop[0];
        c->counters.kernel_launches += (int64_t)admitted * c->l_step_launches + (c->h_loop[2] == 3 ? 0 : 2);
        c->counters.evaluations += admitted;
        c->have_eval = c->have_eval || admitted > 0;
        step += admitted;
        done += admitted;
        if (c->h_loop[2] == 2 || (st = check_status(c, c->h_status[0] & ~ST_SKIN))) {
            if (!st) st = check_status(c, c->h_status[0]);
            return st ? st : fail(c, REANN_ERR_CUDA, "device step loop stopped on an error");
        }
        if (c->h_loop[2] == 1) {
            // step `step` has drifted and tripped the skin check: rebuild, then finish it here
            CK(launch_md_scatter(c, c->d_stage_x, c->d_stage_v, c->d_stage_f, s));
            if ((st = build_internal(c, c->d_stage_f, c->d_types_caller, s))) return st;
            CK(launch_md_gather(c, c->d_stage_x, c->d_stage_v, s));
            CK(cudaMemsetAsync(c->d_status, 0, sizeof(int) * 2, s));
            ++rebuilds;
            if ((st = ef_and_kick(c, dt_fs, inv_mass, s))) return st;
            if (nvt) {
                B.r1 = nvt->noise[2 * step];
                B.s = nvt->noise[2 * step + 1];
                CK(launch_thermostat(c, mass, B, c->d_E + 2, s));
            }
            ++step;
            ++done;
        }
    }
    for (; step < nsteps; ++step) {
        CK(launch_md_kick_drift(c, dt_fs, inv_mass, c->d_status + 1, s));
        CK(cudaMemcpyAsync(c->h_status, c->d_status, sizeof(int) * 2, cudaMemcpyDeviceToHost, s));
        CK(sync_stream(c, s));
        if ((st = check_status(c, c->h_status[0]))) return st;
        if (c->h_status[1]) {
            CK(launch_md_scatter(c, c->d_stage_x, c->d_stage_v, c->d_stage_f, s));
            if ((st = build_internal(c, c->d_stage_f, c->d_types_caller, s))) return st;
            CK(launch_md_gather(c, c->d_stage_x, c->d_stage_v, s));
            CK(cudaMemsetAsync(c->d_status, 0, sizeof(int) * 2, s));
            ++rebuilds;
        }
        if (step == nsteps - 1 && n > 0) {
            CK(launch_md_scatter(c, c->d_last_x, nullptr, nullptr, s));
            CK(cudaEventRecord(c->o_ev[0], s));
            CK(cudaStreamWaitEvent(c->o_stream, c->o_ev[0], 0));
            // a continuing call: the caller's x must have been read in before it is written
            if (spec) CK(cudaStreamWaitEvent(c->o_stream, c->i_ev[1], 0));
            x_wait.s = c->o_stream;
            CK(cudaMemcpyAsync(x, c->d_last_x, bytes3, x_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                               c->o_stream));
            CK(cudaEventRecord(c->o_ev[1], c->o_stream));
        }
        if ((st = ef_and_kick(c, dt_fs, inv_mass, s))) return st;
        if (nvt) {
            B.r1 = nvt->noise[2 * step];
            B.s = nvt->noise[2 * step + 1];
            CK(launch_thermostat(c, mass, B, c->d_E + 2, s));
        }
        ++done;
    }
    CK(launch_kinetic(c, mass, c->d_E + 1, s));
    CK(cudaMemcpyAsync(c->h_E, c->d_E, sizeof(double) * 2, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_E + 4, c->d_E + 3, sizeof(double), cudaMemcpyDeviceToHost, s));
    if (spec) {
        // a continuing call: the caller's x and v are read in and compared before they are written
        CK(cudaStreamWaitEvent(s, c->i_ev[2], 0));
        CK(cudaMemcpyAsync(c->h_status + 2, c->d_status + 2, sizeof(int), cudaMemcpyDeviceToHost, s));
    }
    if (n > 0) {
        // final state in caller order: kept for continuation checks, then copied out
        const bool x_out = x_wait.s != nullptr;
        CK(launch_md_scatter(c, x_out ? nullptr : c->d_last_x, c->d_last_v, nullptr, s));
        if (!x_out)
            CK(cudaMemcpyAsync(x, c->d_last_x, bytes3, x_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                               s));
        CK(cudaMemcpyAsync(v, c->d_last_v, bytes3, v_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost, s));
        if (x_out) CK(cudaStreamWaitEvent(s, c->o_ev[1], 0));
    }
    CK(cudaMemcpyAsync(c->h_status, c->d_status, sizeof(int), cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_i64 + 3, c->d_i64 + 3, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
    CK(sync_stream(c, s));
    c->counters.active_pairs = c->h_i64[3];
    c->md_valid = (c->h_status[0] & ~ST_SKIN) == 0;
    c->md_dt = dt_fs;
    std::copy(mass, mass + c->ne, c->md_mass);
    fill_counters(c);
    if (stats) {
        stats->e_pot = c->h_E[0];
        stats->e_kin = c->h_E[1];
        stats->e_pot0 = c->h_E[2];
        stats->e_kin0 = c->h_E[3];
        stats->rebuilds = rebuilds;
        stats->steps = done;
        stats->e_thermostat = c->h_E[4];
    }
    return check_status(c, c->h_status[0] & ~ST_SKIN);
}

// One MD call: argument checks, the continuation decision and the caller's
// state moved in (overlapped with the steps when the call continues), then
// md_steps.
static reann_status md_run(reann_ctx *c, int32_t nsteps, double dt_fs, double *x, double *v, const double *mass_amu,
                           reann_md_stats *stats, reann_stream stream, const NvtArgs *nvt) {
    if (!c) return REANN_ERR_ARG;
    if (!c->have_list) return fail(c, REANN_ERR_STATE, "reann_build_neighbors must come first");
    if (c->halo) return fail(c, REANN_ERR_STATE, "MD steps over a halo plan are not provided (energy+forces only)");
    if (nsteps < 0 || !std::isfinite(dt_fs) || !mass_amu || (c->n > 0 && (!x || !v)))
        return fail(c, REANN_ERR_ARG, "invalid arguments");
    BussiParams B{};
    if (nvt) {
        if (!(nvt->temperature > 0) || !std::isfinite(nvt->temperature) || !(nvt->tau >= 0))
            return fail(c, REANN_ERR_ARG, "temperature must be positive and finite, tau non-negative");
        if (c->n < 2) return fail(c, REANN_ERR_ARG, "the thermostat needs at least two atoms");
        if (nsteps > 0 && (!nvt->noise || is_device_ptr(nvt->noise)))
            return fail(c, REANN_ERR_ARG, "noise must be a host array of two numbers per step");
        for (int64_t k = 0; k < 2 * (int64_t)nsteps; ++k)
            if (!std::isfinite(nvt->noise[k]) || (k % 2 == 1 && nvt->noise[k] < 0))
                return fail(c, REANN_ERR_ARG, "noise must be finite, with S >= 0");
        B.nf = (double)(3 * c->n - 3);
        B.kt = 0.5 * B.nf * KB_EV * nvt->temperature;
        B.c = nvt->tau > 0 ? std::exp(-dt_fs / nvt->tau) : 0.0;
    }
    double inv_mass[MAX_ELEMENTS], mass[MAX_ELEMENTS];
    for (int e = 0; e < c->ne; ++e) {
        if (!(mass_amu[e] > 0) || !std::isfinite(mass_amu[e])) return fail(c, REANN_ERR_ARG, "masses must be positive");
        mass[e] = mass_amu[e];
        inv_mass[e] = 1.0 / mass_amu[e];
    }
    DeviceGuard guard(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t n = c->n;
    const size_t bytes3 = sizeof(double) * 3 * (size_t)n;
    const bool x_dev = is_device_ptr(x), v_dev = is_device_ptr(v);
    // A continuation -- the caller passes back exactly the state the last call
    // returned, with the same time step and masses -- starts from the resident
    // state and forces at once; the caller's x and v are moved in and compared
    // with that state on a second stream meanwhile, and the call starts again
    // from them if they differ.
    const bool spec = n > 0 && c->md_valid && c->md_dt == dt_fs && std::equal(mass, mass + c->ne, c->md_mass);
    struct StreamWait {
        cudaStream_t s = nullptr;
        ~StreamWait() {
            if (s) cudaStreamSynchronize(s);
        }
    } in_wait;
    if (spec) {
        if (!c->i_stream) {
            CK(cudaStreamCreateWithFlags(&c->i_stream, cudaStreamNonBlocking));
            for (auto &ev : c->i_ev) CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
        }
        CK(cudaMemsetAsync(c->d_status + 2, 0, sizeof(int), s));
        CK(cudaEventRecord(c->i_ev[0], s));
        CK(cudaStreamWaitEvent(c->i_stream, c->i_ev[0], 0));
        in_wait.s = c->i_stream;
        CK(cudaMemcpyAsync(c->d_in_x, x, bytes3, x_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice,
                           c->i_stream));
        CK(cudaEventRecord(c->i_ev[1], c->i_stream));
        CK(cudaMemcpyAsync(c->d_in_v, v, bytes3, v_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice,
                           c->i_stream));
        CK(launch_md_compare(c, c->d_in_x, c->d_in_v, c->d_last_x, c->d_last_v, c->d_status + 2, c->i_stream));
        CK(cudaEventRecord(c->i_ev[2], c->i_stream));
        // this call's result goes to the other buffer pair; the comparison reads the last one
        std::swap(c->d_last_x, c->d_last_x_alt);
        std::swap(c->d_last_v, c->d_last_v_alt);
    } else if (n > 0) {
        CK(cudaMemcpyAsync(c->d_stage_x, x, bytes3, x_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, s));
        CK(cudaMemcpyAsync(c->d_stage_v, v, bytes3, v_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, s));
    }
    const reann_counters counters0 = c->counters;
    reann_status st = md_steps(c, nsteps, dt_fs, x, v, x_dev, v_dev, mass, inv_mass, stats, s, nvt, B, spec, spec);
    if (!spec) return st;
    CK(cudaStreamSynchronize(c->i_stream));
    in_wait.s = nullptr;
    if (st == REANN_OK && c->h_status[2] == 0) return st;
    if (st != REANN_OK) {
        // the steps stopped early: was the resident state the caller's?
        CK(cudaMemcpyAsync(c->h_status + 2, c->d_status + 2, sizeof(int), cudaMemcpyDeviceToHost, c->i_stream));
        CK(cudaStreamSynchronize(c->i_stream));
        if (c->h_status[2] == 0) return st;
    }
    // the caller's state differs from the resident one: start again from the copy read in
    // (the caller's x may already hold the discarded run's positions)
    c->counters = counters0;
    c->md_valid = false;
    CK(cudaMemcpyAsync(c->d_stage_x, c->d_in_x, bytes3, cudaMemcpyDeviceToDevice, s));
    CK(cudaMemcpyAsync(c->d_stage_v, c->d_in_v, bytes3, cudaMemcpyDeviceToDevice, s));
    return md_steps(c, nsteps, dt_fs, x, v, x_dev, v_dev, mass, inv_mass, stats, s, nvt, B, false, false);
}

extern "C" reann_status reann_md_step(reann_ctx *c, int32_t nsteps, double dt_fs, double *x, double *v,
                                      const double *mass_amu, reann_md_stats *stats, reann_stream stream) {
    return md_run(c, nsteps, dt_fs, x, v, mass_amu, stats, stream, nullptr);
}

extern "C" reann_status reann_md_step_nvt(reann_ctx *c, int32_t nsteps, double dt_fs, double temperature_K,
                                          double tau_fs, const double *noise, double *x, double *v,
                                          const double *mass_amu, reann_md_stats *stats, reann_stream stream) {
    const NvtArgs nvt{temperature_K, tau_fs, noise};
    return md_run(c, nsteps, dt_fs, x, v, mass_amu, stats, stream, &nvt);
}

// ---------------------------------------------------------------------------
// One process's share of a spatial decomposition (halo.cu has the row moves).

extern "C" reann_status reann_halo_plan(reann_ctx *c, int64_t n_local, int64_t n_ghost, const int32_t *send_index,
                                        int64_t n_send) {
    if (!c) return REANN_ERR_ARG;
    if (n_local < 0 || n_ghost < 0 || n_send < 0 || (n_send > 0 && !send_index) || n_local + n_ghost >= INT32_MAX)
        return fail(c, REANN_ERR_ARG, "invalid halo plan sizes");
    if (c->dd) return fail(c, REANN_ERR_STATE, "a halo plan and the domain-decomposed checking mode exclude each other");
    std::vector<int32_t> idx(send_index, send_index + n_send);
    for (int32_t a : idx)
        if (a < 0 || a >= n_local) return fail(c, REANN_ERR_ARG, "send_index entries must be own atoms, 0 <= i < n_local");
    // sent rows grouped by own atom (ascending), positions ascending within an atom
    std::vector<int32_t> order(n_send);
    for (int64_t k = 0; k < n_send; ++k) order[k] = (int32_t)k;
    std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) { return idx[x] < idx[y]; });
    std::vector<int32_t> atoms, off;
    for (int64_t k = 0; k < n_send; ++k) {
        if (k == 0 || idx[order[k]] != idx[order[k - 1]]) {
            atoms.push_back(idx[order[k]]);
            off.push_back((int32_t)k);
        }
    }
    off.push_back((int32_t)n_send);
    DeviceGuard guard(c->device);
    dfree(c->d_send_caller); dfree(c->d_send_atom); dfree(c->d_send_off); dfree(c->d_send_order);
    const int width = std::max(c->D, 3);
    const int64_t rows = std::max<int64_t>(std::max(n_send, n_ghost), 1);
    if (rows * width > c->xbuf_alloc) {
        dfree(c->d_xsend); dfree(c->d_xrecv);
        c->xbuf_alloc = 0;
        CK(dalloc(&c->d_xsend, (size_t)(rows * width)));
        CK(dalloc(&c->d_xrecv, (size_t)(rows * width)));
        c->xbuf_alloc = rows * width;
    }
    CK(dalloc(&c->d_send_caller, (size_t)std::max<int64_t>(n_send, 1)));
    CK(dalloc(&c->d_send_order, (size_t)std::max<int64_t>(n_send, 1)));
    CK(dalloc(&c->d_send_atom, std::max<size_t>(atoms.size(), 1)));
    CK(dalloc(&c->d_send_off, off.size()));
    if (n_send > 0) {
        CK(cudaMemcpy(c->d_send_caller, idx.data(), sizeof(int32_t) * n_send, cudaMemcpyHostToDevice));
        CK(cudaMemcpy(c->d_send_order, order.data(), sizeof(int32_t) * n_send, cudaMemcpyHostToDevice));
        CK(cudaMemcpy(c->d_send_atom, atoms.data(), sizeof(int32_t) * atoms.size(), cudaMemcpyHostToDevice));
    }
    CK(cudaMemcpy(c->d_send_off, off.data(), sizeof(int32_t) * off.size(), cudaMemcpyHostToDevice));
    c->halo = true;
    c->n_local = n_local;
    c->n_ghost_plan = n_ghost;
    c->n_send = n_send;
    c->n_send_atoms = (int64_t)atoms.size();
    c->halo_bytes_fwd = n_send * c->D * (int64_t)sizeof(float);
    c->halo_bytes_bwd = n_ghost * c->D * (int64_t)sizeof(float);
    c->have_list = c->have_eval = false;   // the list must be rebuilt for the plan's atoms
    c->md_valid = false;
    return REANN_OK;
}

extern "C" reann_status reann_energy_forces_halo(reann_ctx *c, const float *pos, double *energy, float *forces,
                                                 float *atom_energy, reann_exchange_fn exchange, void *user,
                                                 reann_stream stream) {
    if (!c) return REANN_ERR_ARG;
    if (!c->halo) return fail(c, REANN_ERR_STATE, "reann_halo_plan must come first");
    if (!c->have_list) return fail(c, REANN_ERR_STATE, "reann_build_neighbors must come first");
    if ((c->n > 0 && !pos) || !exchange) return fail(c, REANN_ERR_ARG, "null positions or exchange function");
    DeviceGuard guard(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t n = c->n, nl = c->n_local, ng = c->n - c->n_local;
    c->md_valid = false;
    CK(cudaMemsetAsync(c->d_status, 0, sizeof(int), s));
    if (n > 0) {
        const float *d_pos = pos;
        if (!is_device_ptr(pos)) {
            CK(cudaMemcpyAsync(c->d_stage_f, pos, sizeof(float) * 3 * n, cudaMemcpyHostToDevice, s));
            d_pos = c->d_stage_f;
        }
        CK(launch_pos_from_caller(c, d_pos, s));
        CK(launch_skin_check(c, c->d_status, s));
    }
    auto call = [&](int kind, int layer, int width, int64_t send_rows, int64_t recv_rows) -> reann_status {
        const int32_t rc = exchange(user, kind, layer, c->d_xsend, send_rows, c->d_xrecv, recv_rows, width, stream);
        if (rc != 0) return fail(c, REANN_ERR_CUDA, "the exchange function failed (" + std::to_string(rc) + ")");
        return REANN_OK;
    };
    reann_status st;
    const bool tc = c->cfg.mlp_precision == 1, pair = c->cfg.density_form == 1;
    const bool tc32 = c->cfg.mlp_precision == 0 && tc32_supported(c);
    const int64_t cstride = c->n_slots * c->D;
    // ghost rows of dE/dA are zero throughout: a ghost's energy is its owner's
    if (ng > 0) CK(cudaMemsetAsync(c->d_G + nl * c->NA, 0, sizeof(float) * (size_t)(ng * c->NA), s));
    CK(launch_active(c, s));
    for (int t = 0; t < c->T; ++t) {
        CK(launch_density_fwd(c, t, s));
        if (t + 1 < c->T) {
            float *coef = c->d_coef + (t + 1) * cstride;
            CK(tc ? (pair ? launch_mlp_tc_pair_coef_fwd(c, t, s) : launch_mlp_tc_coef_fwd(c, t, s))
                  : (tc32 ? launch_mlp_tc32_coef_fwd(c, t, s) : launch_mlp_coef_fwd(c, t, s)));
            // forward exchange: own c^{t+1} rows out, ghost rows in
            CK(launch_halo_pack_own(c, coef, c->D, s));
            if ((st = call(REANN_EXCHANGE_COEF, t + 1, c->D, c->n_send, ng))) return st;
            CK(launch_halo_unpack_ghosts(c, coef, c->D, s));
        }
    }
    CK(tc ? (pair ? launch_mlp_tc_pair_energy(c, s) : launch_mlp_tc_energy(c, s))
          : (tc32 ? launch_mlp_tc32_energy(c, s) : launch_mlp_energy(c, s)));
    for (int t = c->T - 1; t >= 0; --t) {
        CK(launch_edge_bwd(c, t, t != c->T - 1, s));
        if (t >= 1) {
            // reverse exchange: ghost partials of dE/dc^t back to their owners
            CK(launch_halo_pack_ghosts(c, c->d_dc, c->D, s));
            if ((st = call(REANN_EXCHANGE_COEF_GRAD, t, c->D, ng, c->n_send))) return st;
            CK(launch_halo_add_partials(c, c->d_dc, c->D, s));
            CK(tc ? (pair ? launch_mlp_tc_pair_coef_bwd(c, t, s) : launch_mlp_tc_coef_bwd(c, t, s))
                  : (tc32 ? launch_mlp_tc32_coef_bwd(c, t, s) : launch_mlp_coef_bwd(c, t, s)));
        }
    }
    // ghost force partials back to their owners
    CK(launch_halo_pack_ghosts(c, c->d_F, 3, s));
    if ((st = call(REANN_EXCHANGE_FORCE, 0, 3, ng, c->n_send))) return st;
    CK(launch_halo_add_partials(c, c->d_F, 3, s));
    CK(launch_energy_sum(c, s));
    c->counters.evaluations++;
    c->have_eval = true;
    bool f_dev = forces && is_device_ptr(forces), e_dev = atom_energy && is_device_ptr(atom_energy);
    float *fo = forces ? (f_dev ? forces : c->d_stage_f) : nullptr;
    float *eo = atom_energy ? (e_dev ? atom_energy : c->d_stage_e) : nullptr;
    CK(launch_scatter_outputs(c, fo, eo, s));
    if (forces && !f_dev && nl > 0)
        CK(cudaMemcpyAsync(forces, c->d_stage_f, sizeof(float) * 3 * nl, cudaMemcpyDeviceToHost, s));
    if (atom_energy && !e_dev && nl > 0)
        CK(cudaMemcpyAsync(atom_energy, c->d_stage_e, sizeof(float) * nl, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_E, c->d_E, sizeof(double), cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_status, c->d_status, sizeof(int), cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(c->h_i64 + 3, c->d_i64 + 3, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
    CK(sync_stream(c, s));
    c->counters.active_pairs = c->h_i64[3];
    c->counters.ghost_slots = ng;
    c->counters.ghost_bytes_fwd = c->halo_bytes_fwd;
    c->counters.ghost_bytes_bwd = c->halo_bytes_bwd;
    fill_counters(c);
    if (energy) *energy = c->h_E[0];
    return check_status(c, *c->h_status);
}

extern "C" reann_status reann_get_counters(const reann_ctx *c, reann_counters *out) {
    if (!c || !out) return REANN_ERR_ARG;
    *out = c->counters;
    return REANN_OK;
}

extern "C" const char *reann_last_error(const reann_ctx *c) {
    return c ? c->last_error.c_str() : g_create_error.c_str();
}

extern "C" reann_status reann_get_neighbors(reann_ctx *c, int64_t *row, int32_t *col, int64_t cap,
                                            reann_stream stream) {
    if (!c || !row || (!col && cap > 0)) return REANN_ERR_ARG;
    if (!c->have_list) return fail(c, REANN_ERR_STATE, "no neighbour list");
    if (cap < c->nnz) return fail(c, REANN_ERR_CAPACITY, "col is shorter than the list (" + std::to_string(c->nnz) + ")");
    DeviceGuard guard(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t n = c->n;
    std::vector<int> hrow(n + 1), hcol(c->nnz > 0 ? c->nnz : 1), hperm(n > 0 ? n : 1);
    CK(cudaMemcpyAsync(hrow.data(), c->d_row, sizeof(int) * (n + 1), cudaMemcpyDeviceToHost, s));
    if (c->nnz > 0) CK(cudaMemcpyAsync(hcol.data(), c->d_col, sizeof(int) * c->nnz, cudaMemcpyDeviceToHost, s));
    if (n > 0) CK(cudaMemcpyAsync(hperm.data(), c->d_perm, sizeof(int) * n, cudaMemcpyDeviceToHost, s));
    CK(sync_stream(c, s));
    std::vector<int64_t> orow(n + 1, 0);
    for (int64_t i = 0; i < n; ++i) orow[hperm[i] + 1] = hrow[i + 1] - hrow[i];
    for (int64_t a = 0; a < n; ++a) orow[a + 1] += orow[a];
    std::vector<int32_t> ocol(c->nnz > 0 ? c->nnz : 1);
    for (int64_t i = 0; i < n; ++i) {
        int64_t a = hperm[i], o = orow[a];
        for (int q = hrow[i]; q < hrow[i + 1]; ++q) ocol[o++] = hperm[hcol[q]];
        std::sort(ocol.begin() + orow[a], ocol.begin() + o);
    }
    CK(cudaMemcpy(row, orow.data(), sizeof(int64_t) * (n + 1), cudaMemcpyDefault));
    if (c->nnz > 0) CK(cudaMemcpy(col, ocol.data(), sizeof(int32_t) * c->nnz, cudaMemcpyDefault));
    return REANN_OK;
}

extern "C" int32_t reann_checked(void) { return kChecked ? 1 : 0; }

extern "C" reann_status reann_debug_set_neighbor(reann_ctx *c, int64_t k, int32_t j) {
    if (!c) return REANN_ERR_ARG;
    if (!kChecked) return fail(c, REANN_ERR_UNSUPPORTED, "fault injection needs the checked build");
    if (!c->have_list) return fail(c, REANN_ERR_STATE, "no neighbour list");
    if (k < 0 || k >= c->nnz) return fail(c, REANN_ERR_ARG, "entry outside the neighbour list");
    DeviceGuard guard(c->device);
    CK(cudaDeviceSynchronize());
    int *col = c->dd ? c->d_col_dd : c->d_col;
    CK(cudaMemcpy(col + k, &j, sizeof(int32_t), cudaMemcpyHostToDevice));
    return REANN_OK;
}

extern "C" reann_status reann_get_features(reann_ctx *c, int32_t t, float *rho, float *coef, reann_stream stream) {
    if (!c) return REANN_ERR_ARG;
    if (t < 0 || t >= c->T) return fail(c, REANN_ERR_ARG, "layer out of range");
    if (!c->have_eval) return fail(c, REANN_ERR_STATE, "no evaluation yet");
    DeviceGuard guard(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t n = c->n, nD = n * c->D, nR = n * c->DR;
    if (n == 0) return REANN_OK;
    if (rho) {
        // stored as rho - shift of the atom's element: the shift is added back here
        CK(launch_to_caller_rows(c, c->d_rho + t * nR, c->DR, c->d_diag, s));
        std::vector<float> h((size_t)nR);
        std::vector<int> types(n);
        CK(cudaMemcpyAsync(h.data(), c->d_diag, sizeof(float) * nR, cudaMemcpyDeviceToHost, s));
        CK(cudaMemcpyAsync(types.data(), c->d_types_caller, sizeof(int) * n, cudaMemcpyDeviceToHost, s));
        CK(sync_stream(c, s));
        for (int64_t a = 0; a < n; ++a)
            for (int f = 0; f < c->DR; ++f)
                h[a * c->DR + f] += c->h_shift[((size_t)t * c->ne + types[a]) * c->DR + f];
        CK(cudaMemcpy(rho, h.data(), sizeof(float) * nR, cudaMemcpyDefault));
    }
    if (coef) {
        if (t == 0) {
            std::vector<int> types(n);
            CK(cudaMemcpy(types.data(), c->d_types_caller, sizeof(int) * n, cudaMemcpyDeviceToHost));
            std::vector<float> h((size_t)nD);
            for (int64_t a = 0; a < n; ++a)
                std::memcpy(&h[a * c->D], &c->h_C0[(size_t)types[a] * c->D], sizeof(float) * c->D);
            CK(cudaMemcpy(coef, h.data(), sizeof(float) * nD, cudaMemcpyDefault));
        } else {
            CK(launch_to_caller_rows(c, c->d_coef + t * c->n_slots * c->D, c->D, c->d_diag, s));
            CK(cudaMemcpyAsync(coef, c->d_diag, sizeof(float) * nD, cudaMemcpyDefault, s));
            CK(sync_stream(c, s));
        }
    }
    return REANN_OK;
}

extern "C" reann_status reann_profile(reann_ctx *c, int32_t enable) {
    if (!c) return REANN_ERR_ARG;
    DeviceGuard guard(c->device);
    c->prof = enable != 0;
    if (c->prof) {
        for (auto &r : c->prof_pending) {
            c->prof_pool.push_back(r.a);
            c->prof_pool.push_back(r.b);
        }
        c->prof_pending.clear();
        for (int g = 0; g < REANN_K_COUNT; ++g) {
            c->prof_ms[g] = 0.0;
            c->prof_n[g] = 0;
        }
    }
    return REANN_OK;
}

extern "C" reann_status reann_profile_read(const reann_ctx *c, int32_t group, double *ms, int64_t *launches) {
    if (!c || group < 0 || group >= REANN_K_COUNT) return REANN_ERR_ARG;
    if (ms) *ms = c->prof_ms[group];
    if (launches) *launches = c->prof_n[group];
    return REANN_OK;
}
