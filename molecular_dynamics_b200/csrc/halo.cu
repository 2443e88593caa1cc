// One process's share of a spatial decomposition over several processes
// (GPUs): the per-layer halo exchange of "Efficient Parallelization of Message
// Passing Neural Network Potentials for Large-Scale Molecular Dynamics",
// section "Parallelization Algorithm" (Figs. 3-4, Eqs. 3-5).
//
// A process evaluates the densities, networks and atomic energies of its own
// atoms.  Its list also holds ghost atoms -- other processes' atoms within the
// list radius of its region -- whose coefficients c^t it receives from their
// owners after every coefficient network (forward exchange).  Differentiating
// its own energies touches the ghosts too: the edges from own atoms to ghosts
// give partial gradients dE/dc^t and partial forces for ghost atoms, which go
// back to the owners and are added to theirs (reverse exchange: dE/dc^t after
// every layer's edge pass, so the owners' coefficient-network backward sees
// the complete gradient; forces once at the end).  Ghost rows of dE/dA stay
// zero: a ghost's own energy belongs to its owner.
//
// This file holds the row movement between the library's internal order and
// the exchange buffers.  Rows sent are own atoms in the caller's send-list
// order; ghost rows are in the caller's ghost order (caller indices n_local,
// n_local + 1, ...).  Partials received for the send list are added to the own
// atoms in a fixed order (an atom sent to several processes gets several), so
// results do not depend on arrival order.  The transfer itself is the
// caller's exchange function (an NCCL all-to-all, host-staged messages, ...).
#include "common.cuh"
#include "kernels.cuh"

namespace reann {
namespace {

inline unsigned nblocks(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

// dst[k] = src[inv[caller[k]]] (rows of `width` floats); caller == nullptr:
// ghost rows, caller index n_local + k.  n: rows of src (own atoms and ghosts)
__global__ void k_halo_pack(int64_t rows, int width, const int *__restrict__ caller, int64_t n_local,
                            const int *__restrict__ inv, const float *__restrict__ src, float *__restrict__ dst,
                            int64_t n, int *__restrict__ status) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= rows * width) return;
    const int64_t r = k / width, f = k - r * width;
    const int64_t a = caller ? checked(caller[r], n_local, status) : n_local + r;
    dst[k] = src[checked(inv[a], n, status) * width + f];
}

// ghost rows of dst (internal order) = recv rows in ghost order
__global__ void k_halo_unpack_ghosts(int64_t rows, int width, int64_t n_local, const int *__restrict__ inv,
                                     const float *__restrict__ recv, float *__restrict__ dst, int64_t n,
                                     int *__restrict__ status) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= rows * width) return;
    const int64_t r = k / width, f = k - r * width;
    dst[checked(inv[n_local + r], n, status) * width + f] = recv[k];
}

// own rows of dst += the partials received for their send-list entries, summed
// in ascending send-list position
__global__ void k_halo_add_partials(int64_t atoms, int width, const int *__restrict__ atom_caller,
                                    const int *__restrict__ off, const int *__restrict__ order,
                                    const int *__restrict__ inv, const float *__restrict__ recv,
                                    float *__restrict__ dst, int64_t n_local, int64_t n_send, int64_t n,
                                    int *__restrict__ status) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= atoms * width) return;
    const int64_t u = k / width, f = k - u * width;
    float s = 0.f;
    const int p1 = checked_end(off[u + 1], n_send, status);
    for (int p = off[u]; p < p1; ++p) s += recv[checked(order[p], n_send, status) * width + f];
    float *d = dst + checked(inv[checked(atom_caller[u], n_local, status)], n, status) * width + f;
    *d += s;
}

}  // namespace

cudaError_t launch_halo_pack_own(reann_ctx *c, const float *src, int width, cudaStream_t s) {
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (c->n_send > 0)
        k_halo_pack<<<nblocks(c->n_send * width, 256), 256, 0, s>>>(c->n_send, width, c->d_send_caller, c->n_local,
                                                                    c->d_inv, src, c->d_xsend, c->n, c->d_status);
    return cudaGetLastError();
}

cudaError_t launch_halo_pack_ghosts(reann_ctx *c, const float *src, int width, cudaStream_t s) {
    const int64_t ng = c->n - c->n_local;
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (ng > 0)
        k_halo_pack<<<nblocks(ng * width, 256), 256, 0, s>>>(ng, width, nullptr, c->n_local, c->d_inv, src,
                                                             c->d_xsend, c->n, c->d_status);
    return cudaGetLastError();
}

cudaError_t launch_halo_unpack_ghosts(reann_ctx *c, float *dst, int width, cudaStream_t s) {
    const int64_t ng = c->n - c->n_local;
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (ng > 0)
        k_halo_unpack_ghosts<<<nblocks(ng * width, 256), 256, 0, s>>>(ng, width, c->n_local, c->d_inv, c->d_xrecv,
                                                                      dst, c->n, c->d_status);
    return cudaGetLastError();
}

cudaError_t launch_halo_add_partials(reann_ctx *c, float *dst, int width, cudaStream_t s) {
    REANN_TIMED(c, REANN_K_OTHER, s, 1);
    if (c->n_send_atoms > 0)
        k_halo_add_partials<<<nblocks(c->n_send_atoms * width, 256), 256, 0, s>>>(
            c->n_send_atoms, width, c->d_send_atom, c->d_send_off, c->d_send_order, c->d_inv, c->d_xrecv, dst,
            c->n_local, c->n_send, c->n, c->d_status);
    return cudaGetLastError();
}

}  // namespace reann
