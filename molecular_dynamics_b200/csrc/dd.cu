// Single-GPU domain-decomposed (DD) checking mode.
//
// "Efficient Parallelization of Message Passing Neural Network Potentials for
// Large-Scale Molecular Dynamics", section "Parallelization Algorithm": each
// process owns the local atoms (LAs) of its subdomain and keeps copies of the
// ghost atoms (GAs) within the cutoff of its LAs (Fig. 3a); in every
// message-passing layer the GAs' messages (orbital coefficients c^t) are
// synchronised from the processes that own them (Fig. 4a), and the backward
// pass exchanges the gradient pieces that belong to neighbouring processes
// (Fig. 4b, Eqs. 3-5).  Here the subdomains are emulated inside one GPU:
//
//   slots   [0, N)            local atoms, in the monolithic internal order
//           [N, N + n_ghost)  ghost copies, grouped by subdomain, each with
//                             the internal index of its owner
//   list    the monolithic CSR with each column j of a row of atom i replaced
//           by the ghost slot of j in i's subdomain when j belongs to another
//           subdomain (row offsets and entry order unchanged)
//   layer t forward: ghost c^t <- owner c^t (in-HBM gather, counted bytes);
//           backward: ghost dE/dA^t <- owner dE/dA^t (the gather form of the
//           backward needs the neighbours' dE/dA rows, so the gradient pieces
//           of the ghosts travel the same way as the messages)
//
// Every local atom sees exactly the values and the summation order of the
// monolithic run, so the two must agree bit for bit.  With the per-layer
// refresh switched off (negative control) the ghosts keep their initial
// coefficients c^0: T = 1 still agrees (only c^0 is used), T >= 2 must not
// (Fig. 3c: ghost features from incomplete information are wrong).
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace reann {

static inline unsigned blocks(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

__device__ __forceinline__ int dd_axis(float xf, double L, int p) {
    const double x = (double)xf;
    const double u = x - L * floor(x / L);
    const int s = (int)(u * (double)p / L);
    return s < 0 ? 0 : (s >= p ? p - 1 : s);
}

struct DDGrid {
    double box[3];
    int p[3];
};

__global__ void k_dd_subdomain(int n, const float4 *__restrict__ pos, DDGrid g, int *__restrict__ sub) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float4 x = pos[i];
    sub[i] = (dd_axis(x.x, g.box[0], g.p[0]) * g.p[1] + dd_axis(x.y, g.box[1], g.p[1])) * g.p[2] +
             dd_axis(x.z, g.box[2], g.p[2]);
}

// bit (s, j) set when atom j of another subdomain is a list neighbour of a local atom of s
__global__ void k_dd_mark(int n, const int *__restrict__ row, const int *__restrict__ col, const int *__restrict__ sub,
                          int64_t words, unsigned *__restrict__ bits, int64_t n_list, int *__restrict__ status) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int s = sub[i];
    const int q1 = checked_end(row[i + 1], n_list, status);
    for (int q = row[i]; q < q1; ++q) {
        const int j = (int)checked(col[q], n, status);
        if (sub[j] != s) atomicOr(&bits[(int64_t)s * words + (j >> 5)], 1u << (j & 31));
    }
}

__global__ void k_dd_popc(int64_t total_words, const unsigned *__restrict__ bits, int *__restrict__ cnt) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k < total_words) cnt[k] = __popc(bits[k]);
}

// ghost slots in (subdomain, owner index) order
__global__ void k_dd_owners(int64_t total_words, int64_t words, int n, const unsigned *__restrict__ bits,
                            const int *__restrict__ prefix, int *__restrict__ owner) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= total_words) return;
    unsigned w = bits[k];
    int o = prefix[k];
    const int j0 = (int)(k % words) * 32;
    while (w) {
        const int b = __ffs(w) - 1;
        owner[o++] = j0 + b;
        w &= w - 1;
    }
}

__device__ __forceinline__ int dd_ghost_slot(int s, int j, int64_t words, int n, const unsigned *__restrict__ bits,
                                             const int *__restrict__ prefix) {
    const int64_t k = (int64_t)s * words + (j >> 5);
    const unsigned below = bits[k] & ((1u << (j & 31)) - 1u);
    return n + prefix[k] + __popc(below);
}

__global__ void k_dd_remap(int n, const int *__restrict__ row, const int *__restrict__ col,
                           const int *__restrict__ sub, int64_t words, const unsigned *__restrict__ bits,
                           const int *__restrict__ prefix, int *__restrict__ dd_col, int64_t n_list,
                           int *__restrict__ status) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int s = sub[i];
    const int q1 = checked_end(row[i + 1], n_list, status);
    for (int q = row[i]; q < q1; ++q) {
        const int j = (int)checked(col[q], n, status);
        dd_col[q] = sub[j] == s ? j : dd_ghost_slot(s, j, words, n, bits, prefix);
    }
}

// rows of `width` floats: dst[n + g] = src[owner[g]]
__global__ void k_dd_gather(int64_t n_ghost, int width, int n, const int *__restrict__ owner, float *__restrict__ base,
                            int *__restrict__ status) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n_ghost * width) return;
    const int64_t g = k / width, f = k % width;
    base[((int64_t)n + g) * width + f] = base[checked(owner[g], n, status) * width + f];
}

// negative control: ghost coefficient rows keep the element's initial c^0
__global__ void k_dd_stale(int64_t n_ghost, int D, int n, const int *__restrict__ owner,
                           const float4 *__restrict__ pos, const float *__restrict__ C0, float *__restrict__ coef,
                           int *__restrict__ status) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n_ghost * D) return;
    const int64_t g = k / D, f = k % D;
    const int e = __float_as_int(pos[checked(owner[g], n, status)].w);
    coef[((int64_t)n + g) * D + f] = C0[e * D + f];
}

cudaError_t dd_gather_rows(reann_ctx *c, float *base, int width, cudaStream_t s) {
    if (c->dd_ghosts == 0) return cudaSuccess;
    REANN_TIMED(c, REANN_K_GHOST, s);
    k_dd_gather<<<blocks(c->dd_ghosts * width, 256), 256, 0, s>>>(c->dd_ghosts, width, (int)c->n, c->d_dd_owner, base,
                                                                  c->d_status);
    return cudaGetLastError();
}

cudaError_t dd_stale_coef(reann_ctx *c, float *coef, cudaStream_t s) {
    if (c->dd_ghosts == 0) return cudaSuccess;
    REANN_TIMED(c, REANN_K_GHOST, s);
    k_dd_stale<<<blocks(c->dd_ghosts * c->D, 256), 256, 0, s>>>(c->dd_ghosts, c->D, (int)c->n, c->d_dd_owner,
                                                                  c->d_pos, c->d_w, coef, c->d_status);
    return cudaGetLastError();
}

// Builds the ghost sets, the ghost owner list and the remapped list for the
// current internal order.  Returns the number of ghost slots in *n_ghost
// (one synchronisation).  The caller sizes the slot arrays and then calls
// dd_finish to write the remapped columns.
cudaError_t dd_plan(reann_ctx *c, cudaStream_t s, int64_t *n_ghost) {
    const int64_t n = c->n;
    const int P = c->cfg.dd_grid[0] * c->cfg.dd_grid[1] * c->cfg.dd_grid[2];
    const int64_t words = (n + 31) / 32;
    const int64_t total_words = (int64_t)P * words;
    cudaError_t e;
    DDGrid g;
    for (int a = 0; a < 3; ++a) {
        g.box[a] = c->box[a];
        g.p[a] = c->cfg.dd_grid[a];
    }
    if (total_words > c->dd_words_alloc) {
        if (c->d_dd_bits) cudaFree(c->d_dd_bits);
        if (c->d_dd_prefix) cudaFree(c->d_dd_prefix);
        if (c->d_dd_cnt) cudaFree(c->d_dd_cnt);
        c->d_dd_bits = nullptr;
        c->d_dd_prefix = c->d_dd_cnt = nullptr;
        if ((e = cudaMalloc(&c->d_dd_bits, sizeof(unsigned) * (size_t)(total_words + 1)))) return e;
        if ((e = cudaMalloc(&c->d_dd_prefix, sizeof(int) * (size_t)(total_words + 1)))) return e;
        if ((e = cudaMalloc(&c->d_dd_cnt, sizeof(int) * (size_t)(total_words + 1)))) return e;
        c->dd_words_alloc = total_words;
        if (c->d_scan_tmp) cudaFree(c->d_scan_tmp);
        c->scan_tmp_size = scan_tmp_bytes(std::max<int64_t>(total_words, std::max<int64_t>(n, c->nbins)));
        if ((e = cudaMalloc(&c->d_scan_tmp, c->scan_tmp_size))) return e;
    }
    if (n == 0) {
        *n_ghost = 0;
        return cudaSuccess;
    }
    {
        REANN_TIMED(c, REANN_K_GHOST, s, 7);
        k_dd_subdomain<<<blocks(n, 256), 256, 0, s>>>((int)n, c->d_pos, g, c->d_dd_sub);
        if ((e = cudaMemsetAsync(c->d_dd_bits, 0, sizeof(unsigned) * (size_t)total_words, s))) return e;
        k_dd_mark<<<blocks(n, 128), 128, 0, s>>>((int)n, c->d_row, c->d_col, c->d_dd_sub, words, c->d_dd_bits,
                                                 c->cap, c->d_status);
        k_dd_popc<<<blocks(total_words, 256), 256, 0, s>>>(total_words, c->d_dd_bits, c->d_dd_cnt);
        if ((e = scan_exclusive(c->d_dd_cnt, c->d_dd_prefix, total_words, c->d_i64 + 5, c->d_scan_tmp, s))) return e;
    }
    if ((e = cudaMemcpyAsync(c->h_i64 + 5, c->d_i64 + 5, sizeof(int64_t), cudaMemcpyDeviceToHost, s))) return e;
    if ((e = cudaStreamSynchronize(s))) return e;
    prof_harvest(c);
    *n_ghost = c->h_i64[5];
    return cudaGetLastError();
}

cudaError_t dd_finish(reann_ctx *c, cudaStream_t s) {
    const int64_t n = c->n;
    const int P = c->cfg.dd_grid[0] * c->cfg.dd_grid[1] * c->cfg.dd_grid[2];
    const int64_t words = (n + 31) / 32;
    const int64_t total_words = (int64_t)P * words;
    if (n == 0) return cudaSuccess;
    REANN_TIMED(c, REANN_K_GHOST, s, 3);
    k_dd_owners<<<blocks(total_words, 256), 256, 0, s>>>(total_words, words, (int)n, c->d_dd_bits, c->d_dd_prefix,
                                                         c->d_dd_owner);
    k_dd_remap<<<blocks(n, 128), 128, 0, s>>>((int)n, c->d_row, c->d_col, c->d_dd_sub, words, c->d_dd_bits,
                                              c->d_dd_prefix, c->d_col_dd, c->cap, c->d_status);
    // ghost positions and types for the current build
    k_dd_gather<<<blocks(c->dd_ghosts * 4, 256), 256, 0, s>>>(c->dd_ghosts, 4, (int)n, c->d_dd_owner,
                                                              reinterpret_cast<float *>(c->d_pos), c->d_status);
    return cudaGetLastError();
}

}  // namespace reann
