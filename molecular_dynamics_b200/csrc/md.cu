// Reductions, order changes between the caller's atom order and the internal
// (element, cell) order, and the velocity-Verlet integrator.
//
// The integrator is the plain velocity-Verlet update that drives the NVE runs
// of "Efficient Parallelization of Message Passing Neural Network Potentials
// for Large-Scale Molecular Dynamics" (section "Strong Scaling", NVE energy
// conservation): v += F/m dt/2; x += v dt; F(x); v += F/m dt/2.  State x, v is
// fp64; the force evaluation reads the fp32 rounding of x.
#include "common.cuh"
#include "kernels.cuh"

namespace reann {

constexpr double ACC_UNIT = 1.0 / 103.6426965;   // eV/(A amu) -> A/fs^2
constexpr double KE_UNIT = 103.6426965;          // amu A^2/fs^2 -> eV
constexpr int RED_THREADS = 256;

static inline unsigned blocks(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

__global__ void k_pos_from_caller(int64_t n, const float *__restrict__ pos, const int *__restrict__ perm,
                                  const int *__restrict__ types, float4 *__restrict__ pos4, int *__restrict__ status) {
    int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n) return;
    int64_t a = checked(perm[s], n, status);
    float x = pos[3 * a], y = pos[3 * a + 1], z = pos[3 * a + 2];
    if (!isfinite(x) || !isfinite(y) || !isfinite(z)) atomicOr(status, ST_NONFINITE);
    pos4[s] = make_float4(x, y, z, __int_as_float(types[a]));
}

cudaError_t launch_pos_from_caller(reann_ctx *c, const float *d_pos_caller, cudaStream_t s) {
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (c->n > 0)
        k_pos_from_caller<<<blocks(c->n, 256), 256, 0, s>>>(c->n, d_pos_caller, c->d_perm, c->d_types_caller,
                                                            c->d_pos, c->d_status);
    return cudaGetLastError();
}

// Deterministic fp64 sum: fixed per-block tree, then one block over the partials.
__device__ __forceinline__ double block_sum(double v) {
    __shared__ double sh[RED_THREADS];
    sh[threadIdx.x] = v;
    __syncthreads();
    for (int w = RED_THREADS / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
        __syncthreads();
    }
    double r = sh[0];
    __syncthreads();
    return r;
}

__global__ void k_energy_partial(int64_t n, const float *__restrict__ Ei, const float *__restrict__ F,
                                 double *__restrict__ part, int *__restrict__ status) {
    int64_t i = (int64_t)blockIdx.x * RED_THREADS + threadIdx.x;
    double v = 0.0;
    bool bad = false;
    if (i < n) {
        float e = Ei[i];
        v = (double)e;
        bad = !isfinite(e) || !isfinite(F[3 * i]) || !isfinite(F[3 * i + 1]) || !isfinite(F[3 * i + 2]);
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, ST_NONFINITE);
    double s = block_sum(v);
    if (threadIdx.x == 0) part[blockIdx.x] = s;
}

__global__ void k_sum_partials(int np, const double *__restrict__ part, double *__restrict__ out) {
    double v = 0.0;
    for (int k = threadIdx.x; k < np; k += RED_THREADS) v += part[k];
    double s = block_sum(v);
    if (threadIdx.x == 0) *out = s;
}

cudaError_t launch_energy_sum(reann_ctx *c, cudaStream_t s) {
    const int64_t nc = centres(c);
    int np = (int)blocks(nc, RED_THREADS);
    REANN_TIMED(c, REANN_K_ENERGY_SUM, s, 2);
    if (nc > 0) k_energy_partial<<<np, RED_THREADS, 0, s>>>(nc, c->d_Ei, c->d_F, c->d_Epart, c->d_status);
    k_sum_partials<<<1, RED_THREADS, 0, s>>>(nc > 0 ? np : 0, c->d_Epart, c->d_E);
    return cudaGetLastError();
}

__global__ void k_scatter_outputs(int64_t n, const int *__restrict__ perm, const float *__restrict__ F,
                                  const float *__restrict__ Ei, float *__restrict__ Fo, float *__restrict__ Eo,
                                  int *__restrict__ status) {
    int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n) return;
    int64_t a = checked(perm[s], n, status);
    if (Fo) {
        Fo[3 * a] = F[3 * s];
        Fo[3 * a + 1] = F[3 * s + 1];
        Fo[3 * a + 2] = F[3 * s + 2];
    }
    if (Eo) Eo[a] = Ei[s];
}

cudaError_t launch_scatter_outputs(reann_ctx *c, float *d_forces, float *d_atom_energy, cudaStream_t s) {
    const int64_t nc = centres(c);   // own atoms sit at internal [0, nc) and caller [0, nc)
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (nc > 0 && (d_forces || d_atom_energy))
        k_scatter_outputs<<<blocks(nc, 256), 256, 0, s>>>(nc, c->d_perm, c->d_F, c->d_Ei, d_forces, d_atom_energy,
                                                          c->d_status);
    return cudaGetLastError();
}

// internal rows of `width` floats -> caller order
__global__ void k_rows_to_caller(int64_t n, int width, const int *__restrict__ perm, const float *__restrict__ in,
                                 float *__restrict__ out, int *__restrict__ status) {
    int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n * width) return;
    int64_t s = k / width, f = k % width;
    out[checked(perm[s], n, status) * width + f] = in[k];
}

cudaError_t launch_to_caller_rows(reann_ctx *c, const float *d_internal, int width, float *d_caller, cudaStream_t s) {
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (c->n > 0) k_rows_to_caller<<<blocks(c->n * width, 256), 256, 0, s>>>(c->n, width, c->d_perm, d_internal, d_caller,
                                                                            c->d_status);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// MD state

__global__ void k_md_gather(int64_t n, const int *__restrict__ perm, const double *__restrict__ xc,
                            const double *__restrict__ vc, double *__restrict__ x, double *__restrict__ v,
                            int *__restrict__ status) {
    int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n) return;
    int64_t a = checked(perm[s], n, status);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        x[3 * s + k] = xc[3 * a + k];
        v[3 * s + k] = vc[3 * a + k];
    }
}

cudaError_t launch_md_gather(reann_ctx *c, const double *d_x_caller, const double *d_v_caller, cudaStream_t s) {
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (c->n > 0) k_md_gather<<<blocks(c->n, 256), 256, 0, s>>>(c->n, c->d_perm, d_x_caller, d_v_caller, c->d_x, c->d_v,
                                                                 c->d_status);
    return cudaGetLastError();
}

__global__ void k_md_scatter(int64_t n, const int *__restrict__ perm, const double *__restrict__ x,
                             const double *__restrict__ v, double *__restrict__ xc, double *__restrict__ vc,
                             float *__restrict__ pc, int *__restrict__ status) {
    int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n) return;
    int64_t a = checked(perm[s], n, status);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        double xv = x[3 * s + k];
        if (xc) xc[3 * a + k] = xv;
        if (vc) vc[3 * a + k] = v[3 * s + k];
        if (pc) pc[3 * a + k] = (float)xv;
    }
}

cudaError_t launch_md_scatter(reann_ctx *c, double *d_x_caller, double *d_v_caller, float *d_pos_caller,
                              cudaStream_t s) {
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (c->n > 0)
        k_md_scatter<<<blocks(c->n, 256), 256, 0, s>>>(c->n, c->d_perm, c->d_x, c->d_v, d_x_caller, d_v_caller,
                                                       d_pos_caller, c->d_status);
    return cudaGetLastError();
}

// flag = 1 when the caller-order state (x, v) differs bitwise from the state
// the previous MD call returned
__global__ void k_md_compare(int64_t m, const unsigned long long *__restrict__ x, const unsigned long long *__restrict__ v,
                             const unsigned long long *__restrict__ lx, const unsigned long long *__restrict__ lv,
                             int *__restrict__ flag) {
    int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    bool diff = k < m && (x[k] != lx[k] || v[k] != lv[k]);
    if (__any_sync(0xffffffffu, diff) && (threadIdx.x & 31) == 0) atomicOr(flag, 1);
}

cudaError_t launch_md_compare(reann_ctx *c, const double *x, const double *v, const double *lx, const double *lv,
                              int *flag, cudaStream_t s) {
    int64_t m = 3 * c->n;
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (m > 0)
        k_md_compare<<<blocks(m, 256), 256, 0, s>>>(m, (const unsigned long long *)x, (const unsigned long long *)v,
                                                    (const unsigned long long *)lx, (const unsigned long long *)lv,
                                                    flag);
    return cudaGetLastError();
}

// caller-order fp64 positions wrapped into [0, L) in place, plus their fp32 copy
__global__ void k_wrap_state(int64_t n, double bx, double by, double bz, double *__restrict__ x,
                             float *__restrict__ p) {
    int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= 3 * n) return;
    double L = (k % 3 == 0) ? bx : ((k % 3 == 1) ? by : bz);
    double v = x[k];
    v -= L * floor(v / L);
    if (v >= L) v -= L;
    x[k] = v;
    p[k] = (float)v;
}

cudaError_t launch_wrap_state(reann_ctx *c, double *d_x_caller, float *d_pos_caller, cudaStream_t s) {
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (c->n > 0)
        k_wrap_state<<<blocks(3 * c->n, 256), 256, 0, s>>>(c->n, c->box[0], c->box[1], c->box[2], d_x_caller,
                                                           d_pos_caller);
    return cudaGetLastError();
}

struct MdParams {
    double inv_mass[MAX_ELEMENTS];
    double half_dt_acc;   // dt/2 * ACC_UNIT
    double dt;
    double box[3];
    double half_skin2;
};

// v += F/m dt/2; x += v dt; wrap into [0, L); fp32 copy; flag a rebuild when
// the fp32 position moved more than skin/2 from the build position.
__global__ void k_md_kick_drift(int64_t n, double *__restrict__ x, double *__restrict__ v, const float *__restrict__ F,
                                float4 *__restrict__ pos4, const float4 *__restrict__ pos_build, MdParams M,
                                int *__restrict__ flag) {
    int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    bool moved = false;
    if (s < n) {
        float4 p = pos4[s];
        int e = __float_as_int(p.w);
        double k = M.half_dt_acc * M.inv_mass[e];
        float q[3];
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            double vv = v[3 * s + a] + k * (double)F[3 * s + a];
            double xx = x[3 * s + a] + M.dt * vv;
            xx -= M.box[a] * floor(xx / M.box[a]);
            if (xx >= M.box[a]) xx -= M.box[a];
            v[3 * s + a] = vv;
            x[3 * s + a] = xx;
            q[a] = (float)xx;
        }
        pos4[s] = make_float4(q[0], q[1], q[2], p.w);
        float4 b = pos_build[s];
        double d[3] = {(double)q[0] - (double)b.x, (double)q[1] - (double)b.y, (double)q[2] - (double)b.z};
#pragma unroll
        for (int a = 0; a < 3; ++a) d[a] -= M.box[a] * rint(d[a] / M.box[a]);
        double r2 = d[0] * d[0] + d[1] * d[1] + d[2] * d[2];
        moved = !(r2 <= M.half_skin2);
    }
    if (__any_sync(0xffffffffu, moved) && (threadIdx.x & 31) == 0) atomicOr(flag, 1);
}

static MdParams md_params(const reann_ctx *c, double dt, const double *inv_mass) {
    MdParams M;
    for (int e = 0; e < MAX_ELEMENTS; ++e) M.inv_mass[e] = e < c->ne ? inv_mass[e] : 0.0;
    M.half_dt_acc = 0.5 * dt * ACC_UNIT;
    M.dt = dt;
    for (int a = 0; a < 3; ++a) M.box[a] = c->box[a];
    double h = 0.5 * c->cfg.skin;
    M.half_skin2 = h * h;
    return M;
}

cudaError_t launch_md_kick_drift(reann_ctx *c, double dt, const double *inv_mass, int *flag, cudaStream_t s) {
    MdParams M = md_params(c, dt, inv_mass);
    REANN_TIMED(c, REANN_K_INTEGRATE, s, 1);
    if (c->n > 0)
        k_md_kick_drift<<<blocks(c->n, 256), 256, 0, s>>>(c->n, c->d_x, c->d_v, c->d_F, c->d_pos, c->d_pos_build, M,
                                                          flag);
    return cudaGetLastError();
}

__global__ void k_md_kick(int64_t n, double *__restrict__ v, const float *__restrict__ F,
                          const float4 *__restrict__ pos4, MdParams M) {
    int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n) return;
    int e = __float_as_int(pos4[s].w);
    double k = M.half_dt_acc * M.inv_mass[e];
#pragma unroll
    for (int a = 0; a < 3; ++a) v[3 * s + a] += k * (double)F[3 * s + a];
}

cudaError_t launch_md_kick(reann_ctx *c, double dt, const double *inv_mass, cudaStream_t s) {
    MdParams M = md_params(c, dt, inv_mass);
    REANN_TIMED(c, REANN_K_INTEGRATE, s, 1);
    if (c->n > 0) k_md_kick<<<blocks(c->n, 256), 256, 0, s>>>(c->n, c->d_v, c->d_F, c->d_pos, M);
    return cudaGetLastError();
}

__global__ void k_kinetic_partial(int64_t n, const double *__restrict__ v, const float4 *__restrict__ pos4,
                                  MdParams M, double *__restrict__ part) {
    int64_t s = (int64_t)blockIdx.x * RED_THREADS + threadIdx.x;
    double k = 0.0;
    if (s < n) {
        int e = __float_as_int(pos4[s].w);
        double m = M.inv_mass[e];   // holds the mass here
        k = 0.5 * m * (v[3 * s] * v[3 * s] + v[3 * s + 1] * v[3 * s + 1] + v[3 * s + 2] * v[3 * s + 2]) * KE_UNIT;
    }
    double t = block_sum(k);
    if (threadIdx.x == 0) part[blockIdx.x] = t;
}

cudaError_t launch_kinetic(reann_ctx *c, const double *mass, double *d_out, cudaStream_t s) {
    MdParams M = md_params(c, 0.0, mass);
    int np = (int)blocks(c->n, RED_THREADS);
    REANN_TIMED(c, REANN_K_OTHER, s, 2);
    if (c->n > 0) k_kinetic_partial<<<np, RED_THREADS, 0, s>>>(c->n, c->d_v, c->d_pos, M, c->d_Epart);
    k_sum_partials<<<1, RED_THREADS, 0, s>>>(c->n > 0 ? np : 0, c->d_Epart, d_out);
    return cudaGetLastError();
}

// Stochastic velocity rescaling (Bussi, Donadio and Parrinello, J. Chem. Phys.
// 126, 014101 (2007)), the thermostat of the NVT runs named on the Tessera
// page (abstract): K' = K + (1 - c)(Kt (R1^2 + S)/Nf - K) + 2 R1 sqrt(c (1 - c)
// K Kt / Nf), every velocity scaled by sqrt(K' / K).  One block sums the
// kinetic-energy partials in the fixed tree order of k_sum_partials, takes the
// factor and adds K' - K to the work accumulator; the next kernel scales.
// K' is a sum of squares in exact arithmetic; a rounding below zero is
// clamped to it.
// With `noise` given (the device-side step loop), the step's two numbers are
// read at index loop[3] + loop[0] - 1: the first step of the launch plus the
// steps the loop gate has admitted so far, minus the current one.
__global__ void k_bussi_factor(int np, const double *__restrict__ part, BussiParams B, const double *__restrict__ noise,
                               const int *__restrict__ loop, double *__restrict__ state) {
    double v = 0.0;
    for (int k = threadIdx.x; k < np; k += RED_THREADS) v += part[k];
    double K = block_sum(v);
    if (threadIdx.x == 0) {
        if (noise) {
            const int64_t step = (int64_t)loop[3] + loop[0] - 1;
            B.r1 = noise[2 * step];
            B.s = noise[2 * step + 1];
        }
        double alpha = 1.0, Kn = K;
        if (K > 0.0) {
            Kn = K + (1.0 - B.c) * (B.kt * (B.r1 * B.r1 + B.s) / B.nf - K) +
                 2.0 * B.r1 * sqrt(B.c * (1.0 - B.c) * K * B.kt / B.nf);
            Kn = fmax(Kn, 0.0);
            alpha = sqrt(Kn / K);
        }
        state[0] = alpha;
        state[1] += Kn - K;
    }
}

__global__ void k_scale_velocities(int64_t m, double *__restrict__ v, const double *__restrict__ alpha) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < m) v[i] *= *alpha;
}

cudaError_t launch_thermostat(reann_ctx *c, const double *mass, const BussiParams &B, double *d_state,
                              cudaStream_t s, const double *d_noise, const int *d_loop) {
    MdParams M = md_params(c, 0.0, mass);
    int np = (int)blocks(c->n, RED_THREADS);
    if (c->n == 0) return cudaSuccess;
    REANN_TIMED(c, REANN_K_INTEGRATE, s, 3);
    k_kinetic_partial<<<np, RED_THREADS, 0, s>>>(c->n, c->d_v, c->d_pos, M, c->d_Epart);
    k_bussi_factor<<<1, RED_THREADS, 0, s>>>(np, c->d_Epart, B, d_noise, d_loop, d_state);
    k_scale_velocities<<<blocks(3 * c->n, 256), 256, 0, s>>>(3 * c->n, c->d_v, d_state);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Device-side step loop.  After each kick-drift the gate decides on the GPU
// whether the step may go on without the host: not when an earlier kernel
// flagged an error (status[0]) or the skin check tripped (status[1]), which
// need the host (error return, neighbour-list rebuild).  loop[0] counts the
// steps admitted in this launch, loop[1] is the number requested, loop[2] the
// reason the loop ended (1 rebuild, 2 error, 3 all steps done).  The gate sets
// the IF handle that runs the step's energy+forces and closing kick, and the
// WHILE handle that runs the next step.
__global__ void k_loop_gate(const int *__restrict__ status, int *__restrict__ loop, cudaGraphConditionalHandle h_while,
                            cudaGraphConditionalHandle h_step) {
    if (threadIdx.x != 0) return;
    const int err = status[0] & ~ST_SKIN, trip = status[1];
    if (err || trip) {
        loop[2] = err ? 2 : 1;
        cudaGraphSetConditional(h_step, 0);
        cudaGraphSetConditional(h_while, 0);
        return;
    }
    const int d = loop[0] + 1;
    loop[0] = d;
    cudaGraphSetConditional(h_step, 1);
    const bool more = d < loop[1];
    if (!more) loop[2] = 3;
    cudaGraphSetConditional(h_while, more ? 1u : 0u);
}

cudaError_t launch_loop_gate(reann_ctx *c, cudaGraphConditionalHandle h_while, cudaGraphConditionalHandle h_step,
                             cudaStream_t s) {
    REANN_TIMED(c, REANN_K_INTEGRATE, s, 1);
    k_loop_gate<<<1, 32, 0, s>>>(c->d_status, c->d_loop, h_while, h_step);
    return cudaGetLastError();
}

}  // namespace reann
