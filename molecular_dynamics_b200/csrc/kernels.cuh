// Launch wrappers shared between translation units.
#pragma once

#include "common.cuh"

namespace reann {

struct BinParams {
    double box[3];
    double inv_box[3];
    int m[3];
    int ncell;
    int ne;
    // bin classes: the ne elements, and with a halo plan (multi-process
    // decomposition) ne more for the ghost atoms, caller indices >= n_local;
    // ghost rows list only the process's own atoms
    int nclass;
    int64_t n_local;
    double thr;  // (r_cut + skin)^2
};

BinParams make_bin_params(const reann_ctx *c);
EdgeParams make_edge_params(const reann_ctx *c);

// neighbour search (nbr.cu)
cudaError_t launch_build(reann_ctx *c, const float *d_pos_caller, const int *d_types_caller, cudaStream_t s);
cudaError_t launch_fill(reann_ctx *c, cudaStream_t s);
cudaError_t launch_skin_check(reann_ctx *c, int *flag, cudaStream_t s);

// edge kernels (edge.cu)
cudaError_t launch_active(reann_ctx *c, cudaStream_t s);
cudaError_t launch_density_fwd(reann_ctx *c, int t, cudaStream_t s);
cudaError_t launch_edge_bwd(reann_ctx *c, int t, bool accumulate, cudaStream_t s);

// atomic networks (mlp.cu)
cudaError_t launch_mlp_coef_fwd(reann_ctx *c, int t, cudaStream_t s);   // rho^t -> c^{t+1}
cudaError_t launch_mlp_energy(reann_ctx *c, cudaStream_t s);            // rho^{T-1} -> E_i, G^{T-1}
cudaError_t launch_mlp_coef_bwd(reann_ctx *c, int t, cudaStream_t s);   // (rho^{t-1}, dE/dc^t) -> G^{t-1}

// domain-decomposed checking mode (dd.cu)
cudaError_t dd_plan(reann_ctx *c, cudaStream_t s, int64_t *n_ghost);
cudaError_t dd_finish(reann_ctx *c, cudaStream_t s);
cudaError_t dd_gather_rows(reann_ctx *c, float *base, int width, cudaStream_t s);
cudaError_t dd_stale_coef(reann_ctx *c, float *coef, cudaStream_t s);

// atomic networks on tcgen05 tensor cores, bf16 operands (mlp_tc.cu)
cudaError_t launch_mlp_tc_coef_fwd(reann_ctx *c, int t, cudaStream_t s);
cudaError_t launch_mlp_tc_energy(reann_ctx *c, cudaStream_t s);
cudaError_t launch_mlp_tc_coef_bwd(reann_ctx *c, int t, cudaStream_t s);
// fp32-accurate networks on tcgen05 tensor cores, three tf32 passes (mlp_tc32.cu)
bool tc32_supported(const reann_ctx *c);
cudaError_t launch_mlp_tc32_coef_fwd(reann_ctx *c, int t, cudaStream_t s);
cudaError_t launch_mlp_tc32_energy(reann_ctx *c, cudaStream_t s);
cudaError_t launch_mlp_tc32_coef_bwd(reann_ctx *c, int t, cudaStream_t s);
// tensor-core networks for the pair-product density form (mlp_tc_pair.cu)
cudaError_t launch_mlp_tc_pair_coef_fwd(reann_ctx *c, int t, cudaStream_t s);
cudaError_t launch_mlp_tc_pair_energy(reann_ctx *c, cudaStream_t s);
cudaError_t launch_mlp_tc_pair_coef_bwd(reann_ctx *c, int t, cudaStream_t s);

// a process's share of a multi-process decomposition (halo.cu): rows between
// internal order and the exchange buffers
cudaError_t launch_halo_pack_own(reann_ctx *c, const float *src, int width, cudaStream_t s);
cudaError_t launch_halo_pack_ghosts(reann_ctx *c, const float *src, int width, cudaStream_t s);
cudaError_t launch_halo_unpack_ghosts(reann_ctx *c, float *dst, int width, cudaStream_t s);
cudaError_t launch_halo_add_partials(reann_ctx *c, float *dst, int width, cudaStream_t s);

// atoms whose densities, networks and energies this context evaluates: all,
// or a halo plan's own atoms (the ghosts follow them in internal order)
inline int64_t centres(const reann_ctx *c) { return c->halo ? c->n_local : c->n; }

// reductions, gathers and the integrator (md.cu)
cudaError_t launch_pos_from_caller(reann_ctx *c, const float *d_pos_caller, cudaStream_t s);
cudaError_t launch_energy_sum(reann_ctx *c, cudaStream_t s);            // -> d_E[0], status on non-finite
cudaError_t launch_scatter_outputs(reann_ctx *c, float *d_forces, float *d_atom_energy, cudaStream_t s);
cudaError_t launch_md_gather(reann_ctx *c, const double *d_x_caller, const double *d_v_caller, cudaStream_t s);
cudaError_t launch_md_scatter(reann_ctx *c, double *d_x_caller, double *d_v_caller, float *d_pos_caller,
                              cudaStream_t s);
cudaError_t launch_md_kick_drift(reann_ctx *c, double dt, const double *inv_mass, int *flag, cudaStream_t s);
cudaError_t launch_md_kick(reann_ctx *c, double dt, const double *inv_mass, cudaStream_t s);
cudaError_t launch_kinetic(reann_ctx *c, const double *mass, double *d_out, cudaStream_t s);
// One step of stochastic velocity rescaling: d_state[0] <- the factor, d_state[1] += K' - K.
struct BussiParams {
    double c, kt, nf, r1, s;   // exp(-dt/tau), Kt (eV), Nf, the step's normal and chi-square numbers
};
// d_noise / d_loop (both or neither): the step's numbers come from the device
// noise array at the device-side loop's current step instead of from B
cudaError_t launch_thermostat(reann_ctx *c, const double *mass, const BussiParams &B, double *d_state,
                              cudaStream_t s, const double *d_noise = nullptr, const int *d_loop = nullptr);
// the device-side step loop's gate (md.cu)
cudaError_t launch_loop_gate(reann_ctx *c, cudaGraphConditionalHandle h_while, cudaGraphConditionalHandle h_step,
                             cudaStream_t s);
cudaError_t launch_md_compare(reann_ctx *c, const double *x, const double *v, const double *lx, const double *lv,
                              int *flag, cudaStream_t s);
cudaError_t launch_wrap_state(reann_ctx *c, double *d_x_caller, float *d_pos_caller, cudaStream_t s);
cudaError_t launch_to_caller_rows(reann_ctx *c, const float *d_internal, int width, float *d_caller, cudaStream_t s);

}  // namespace reann
