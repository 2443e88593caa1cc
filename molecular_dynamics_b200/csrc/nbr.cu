// Neighbour search: counting sort of atoms into (element, cell) bins and a
// CSR full neighbour list with a Verlet skin.
//
// "Efficient Parallelization of Message Passing Neural Network Potentials for
// Large-Scale Molecular Dynamics", section "Parallelization Algorithm": the
// neighbour list is computed once and reused by every message-passing layer
// (Fig. 2); each atom keeps a full list (Fig. 3a).  The skin follows the
// "Introduction" (an additional skin distance lowers the rebuild frequency).
//
// Internal atom order is (element, cell, caller index).  Each element's atoms
// form one contiguous segment (the atomic networks run on contiguous rows),
// and inside a segment atoms are in cell order (neighbour gathers stay local).
// With a halo plan (a process's share of a spatial decomposition) the ghost
// atoms copied from other processes follow all own atoms, in segments of
// their own, and their rows list own atoms only: the edges a process must
// differentiate for the partial gradients it returns to the ghosts' owners
// (section "Parallelization Algorithm", Fig. 4).
#include "common.cuh"
#include "kernels.cuh"

namespace reann {

// ---------------------------------------------------------------------------
// exclusive scan of int32 counts (three passes: block sums, scan of the block
// sums in one block, block-local scan with offsets).  The total is written as
// int64 so that overflow of the int32 offsets can be detected by the caller.

constexpr int SCAN_THREADS = 256;
constexpr int SCAN_ITEMS = 8;
constexpr int SCAN_CHUNK = SCAN_THREADS * SCAN_ITEMS;

size_t scan_tmp_bytes(int64_t n) {
    int64_t nb = (n + SCAN_CHUNK - 1) / SCAN_CHUNK;
    return sizeof(int64_t) * (size_t)(nb + 1);
}

__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t *total) {
    __shared__ int64_t warp_sums[SCAN_THREADS / 32];
    int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int64_t w = lane < SCAN_THREADS / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int64_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < SCAN_THREADS / 32) warp_sums[lane] = w;
    }
    __syncthreads();
    int64_t base = warp > 0 ? warp_sums[warp - 1] : 0;
    if (total) *total = warp_sums[SCAN_THREADS / 32 - 1];
    __syncthreads();
    return base + x - v;
}

__global__ void k_scan_block_sums(const int *__restrict__ in, int64_t n, int64_t *__restrict__ bsum) {
    int64_t base = (int64_t)blockIdx.x * SCAN_CHUNK;
    int64_t s = 0;
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        int64_t i = base + (int64_t)k * SCAN_THREADS + threadIdx.x;
        if (i < n) s += in[i];
    }
    int64_t tot;
    block_exclusive_scan(s, &tot);
    if (threadIdx.x == 0) bsum[blockIdx.x] = tot;
}

__global__ void k_scan_block_offsets(int64_t *__restrict__ bsum, int64_t nb, int64_t *__restrict__ d_total) {
    int64_t carry = 0;
    for (int64_t base = 0; base < nb; base += SCAN_THREADS) {
        int64_t i = base + threadIdx.x;
        int64_t v = i < nb ? bsum[i] : 0;
        int64_t tot;
        int64_t ex = block_exclusive_scan(v, &tot);
        if (i < nb) bsum[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0 && d_total) *d_total = carry;
}

__global__ void k_scan_apply(const int *__restrict__ in, int *__restrict__ out, int64_t n,
                             const int64_t *__restrict__ bsum, const int64_t *__restrict__ d_total) {
    int64_t base = (int64_t)blockIdx.x * SCAN_CHUNK + (int64_t)threadIdx.x * SCAN_ITEMS;
    int v[SCAN_ITEMS];
    int64_t s = 0;
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        int64_t i = base + k;
        v[k] = i < n ? in[i] : 0;
        s += v[k];
    }
    int64_t ex = block_exclusive_scan(s, nullptr) + bsum[blockIdx.x];
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        int64_t i = base + k;
        if (i < n) out[i] = (int)ex;
        ex += v[k];
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) out[n] = (int)*d_total;
}

// out[0..n] = exclusive scan of in[0..n-1], out[n] = total (int32); *d_total = total (int64).
cudaError_t scan_exclusive(const int *in, int *out, int64_t n, int64_t *d_total, void *tmp, cudaStream_t s) {
    int64_t nb = (n + SCAN_CHUNK - 1) / SCAN_CHUNK;
    if (nb < 1) nb = 1;
    int64_t *bsum = (int64_t *)tmp;
    k_scan_block_sums<<<(unsigned)nb, SCAN_THREADS, 0, s>>>(in, n, bsum);
    k_scan_block_offsets<<<1, SCAN_THREADS, 0, s>>>(bsum, nb, d_total);
    k_scan_apply<<<(unsigned)nb, SCAN_THREADS, 0, s>>>(in, out, n, bsum, d_total);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// binning

__device__ __forceinline__ int cell_axis(float xf, double L, int m) {
    double x = (double)xf;
    double u = x - L * floor(x / L);
    int c = (int)(u * (double)m / L);
    return c < 0 ? 0 : (c >= m ? m - 1 : c);
}

__global__ void k_bin_count(int64_t n, const float *__restrict__ pos, const int *__restrict__ types, BinParams B,
                            int *__restrict__ key, int *__restrict__ bin_count, int *__restrict__ status) {
    int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (a >= n) return;
    float x = pos[3 * a], y = pos[3 * a + 1], z = pos[3 * a + 2];
    int e = types[a];
    int bad = 0;
    if (!isfinite(x) || !isfinite(y) || !isfinite(z)) { bad |= ST_NONFINITE; x = y = z = 0.f; }
    if (e < 0 || e >= B.ne) { bad |= ST_BADTYPE; e = 0; }
    if (bad) atomicOr(status, bad);
    int cx = cell_axis(x, B.box[0], B.m[0]);
    int cy = cell_axis(y, B.box[1], B.m[1]);
    int cz = cell_axis(z, B.box[2], B.m[2]);
    const int cls = a >= B.n_local ? B.ne + e : e;   // ghosts after every own atom
    int k = cls * B.ncell + (cx * B.m[1] + cy) * B.m[2] + cz;
    key[a] = k;
    atomicAdd(&bin_count[k], 1);
}

__global__ void k_bin_scatter(int64_t n, const int *__restrict__ key, const int *__restrict__ bin_start,
                              int *__restrict__ bin_fill, int *__restrict__ perm_tmp) {
    int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (a >= n) return;
    int k = key[a];
    int slot = bin_start[k] + atomicAdd(&bin_fill[k], 1);
    perm_tmp[slot] = (int)a;
}

// One warp per bin: order the bin's atoms by caller index (ranks are unique),
// which makes the internal order independent of atomic arrival order.
__global__ void k_bin_sort(int nbins, const int *__restrict__ bin_start, const int *__restrict__ perm_tmp,
                           int *__restrict__ perm) {
    int b = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    int lane = threadIdx.x & 31;
    if (b >= nbins) return;
    int s0 = bin_start[b], s1 = bin_start[b + 1];
    for (int p = s0 + lane; p < s1; p += 32) {
        int v = perm_tmp[p];
        int rank = 0;
        for (int q = s0; q < s1; ++q) rank += perm_tmp[q] < v;
        perm[s0 + rank] = v;
    }
}

__global__ void k_gather_pos(int64_t n, const float *__restrict__ pos, const int *__restrict__ types,
                             const int *__restrict__ perm, float4 *__restrict__ pos4, float4 *__restrict__ pos_build,
                             int *__restrict__ inv, int *__restrict__ status) {
    int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n) return;
    int a = (int)checked(perm[s], n, status);
    float4 p = make_float4(pos[3 * (int64_t)a], pos[3 * (int64_t)a + 1], pos[3 * (int64_t)a + 2], __int_as_float(types[a]));
    pos4[s] = p;
    pos_build[s] = p;
    inv[a] = (int)s;
}

// ---------------------------------------------------------------------------
// CSR neighbour list

// Minimum-image squared distance in fp64 with every operation rounded
// separately (no contraction), exactly as the list definition states:
// d = x_j - x_i; d -= L k with k = rint(d / L); r2 = (dx dx + dy dy) + dz dz.
// k is taken as rint(d (1/L)): the product can differ from the quotient only
// in the last bit, which changes k only when d / L is within an ulp of a
// half-integer -- a pair half a box apart, never closer than r_cut + skin
// (the box is at least twice that) -- so every listed pair gets the same k,
// the same d and the same r2 as with the division.
__device__ __forceinline__ double list_r2(float4 pi, float4 pj, const BinParams &B) {
    double d[3] = {__dsub_rn((double)pj.x, (double)pi.x), __dsub_rn((double)pj.y, (double)pi.y),
                   __dsub_rn((double)pj.z, (double)pi.z)};
#pragma unroll
    for (int a = 0; a < 3; ++a) d[a] = __dsub_rn(d[a], __dmul_rn(B.box[a], rint(d[a] * B.inv_box[a])));
    return __dadd_rn(__dadd_rn(__dmul_rn(d[0], d[0]), __dmul_rn(d[1], d[1])), __dmul_rn(d[2], d[2]));
}

// the distinct cells within one step of c along an axis of m cells, ascending
__device__ __forceinline__ int axis_stencil(int c, int m, int out[3]) {
    if (m < 3) {
        for (int s = 0; s < m; ++s) out[s] = s;
        return m;
    }
    int a = c == 0 ? m - 1 : c - 1, b = c, d = c == m - 1 ? 0 : c + 1;
    // sort three distinct values
    int lo = min(a, min(b, d)), hi = max(a, max(b, d));
    out[0] = lo;
    out[1] = a + b + d - lo - hi;
    out[2] = hi;
    return 3;
}

// Rows of the list, one thread per atom walking the stencil cells (e, x, y, z
// ascending) and, inside a cell, ascending j.  Small systems, whose atoms
// alone leave most of the GPU idle, take a group of GL lanes per atom instead:
// the group tests GL candidates of a cell at once (a cell's atoms are
// contiguous in internal order), and a ballot counts the hits and, in the fill
// pass, places them in candidate order -- the same columns in the same order.
// (Measured per build: 3,000 water molecules' atoms 0.63 -> 0.12 ms with 32
// lanes; on the 108k-1M-atom systems one thread per atom is fastest.)
template <bool FILL, int GL>
__global__ void __launch_bounds__(128) k_nbr(int n, const float4 *__restrict__ pos, const int *__restrict__ bin_start,
                                             BinParams B, const int *__restrict__ row, int *__restrict__ cnt,
                                             int *__restrict__ col) {
    static_assert(GL >= 1 && GL <= 32 && (32 % GL) == 0, "lane groups tile a warp");
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int i = t / GL, sub = t % GL;
    // a group's lanes share i, so a group is either entirely in range or entirely out
    if (i >= n) return;
    const int gbase = (threadIdx.x & 31) & ~(GL - 1);
    const unsigned gmask = GL == 32 ? 0xffffffffu : (((1u << GL) - 1u) << gbase);
    float4 pi = pos[i];
    int sx[3], sy[3], sz[3];
    int nx = axis_stencil(cell_axis(pi.x, B.box[0], B.m[0]), B.m[0], sx);
    int ny = axis_stencil(cell_axis(pi.y, B.box[1], B.m[1]), B.m[1], sy);
    int nz = axis_stencil(cell_axis(pi.z, B.box[2], B.m[2]), B.m[2], sz);
    int c = 0;
    int o = FILL ? row[i] : 0;
    // own atoms come first in internal order; a ghost's row lists own atoms only
    const int ncls = i >= B.n_local ? B.ne : B.nclass;
    for (int e = 0; e < ncls; ++e) {
        for (int a = 0; a < nx; ++a)
            for (int b = 0; b < ny; ++b)
                for (int d = 0; d < nz; ++d) {
                    int k = e * B.ncell + (sx[a] * B.m[1] + sy[b]) * B.m[2] + sz[d];
                    const int j1 = bin_start[k + 1];
                    if (GL == 1) {
                        for (int j = bin_start[k]; j < j1; ++j) {
                            if (j == i) continue;
                            if (list_r2(pi, pos[j], B) < B.thr) {
                                if (FILL) col[o + c] = j;
                                ++c;
                            }
                        }
                        continue;
                    }
                    for (int base = bin_start[k]; base < j1; base += GL) {
                        const int j = base + sub;
                        const bool hit = j < j1 && j != i && list_r2(pi, pos[j], B) < B.thr;
                        const unsigned gb = GL == 32 ? __ballot_sync(gmask, hit)
                                                     : (__ballot_sync(gmask, hit) >> gbase) & ((1u << GL) - 1u);
                        if (FILL && hit) col[o + c + __popc(gb & ((1u << sub) - 1u))] = j;
                        c += __popc(gb);
                    }
                }
    }
    if (!FILL && sub == 0) cnt[i] = c;
}


__global__ void k_row_max(int n, const int *__restrict__ cnt, int64_t *__restrict__ out) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    int v = i < n ? cnt[i] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0 && v > 0) atomicMax((unsigned long long *)out, (unsigned long long)v);
}

// Sets ST_SKIN when any atom has moved more than skin/2 (minimum image) since
// the list was built.
__global__ void k_max_disp(int n, const float4 *__restrict__ pos, const float4 *__restrict__ pos_build, BinParams B,
                           double half_skin2, int *__restrict__ flag) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    bool moved = false;
    if (i < n) {
        float4 a = pos[i], b = pos_build[i];
        double d[3] = {(double)a.x - (double)b.x, (double)a.y - (double)b.y, (double)a.z - (double)b.z};
#pragma unroll
        for (int k = 0; k < 3; ++k) d[k] -= B.box[k] * rint(d[k] / B.box[k]);
        double r2 = d[0] * d[0] + d[1] * d[1] + d[2] * d[2];
        moved = !(r2 <= half_skin2);
    }
    if (__any_sync(0xffffffffu, moved) && (threadIdx.x & 31) == 0) atomicOr(flag, ST_SKIN);
}

// ---------------------------------------------------------------------------
// host side

static inline unsigned blocks(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

// lanes per atom of the list kernels: enough threads for about 512 per SM
static int nbr_lanes(const reann_ctx *c, int64_t n) {
    int gl = 1;
    while (gl < 32 && n * gl < (int64_t)c->sm_count * 512) gl *= 2;
    return gl;
}

template <bool FILL>
static void launch_nbr(const reann_ctx *c, int64_t n, const BinParams &B, const int *row, int *cnt, int *col,
                       cudaStream_t s) {
    const int gl = nbr_lanes(c, n);
#define REANN_NBR(GLV) \
    k_nbr<FILL, GLV><<<blocks(n * GLV, 128), 128, 0, s>>>((int)n, c->d_pos, c->d_bin_start, B, row, cnt, col)
    switch (gl) {
        case 1: REANN_NBR(1); break;
        case 2: REANN_NBR(2); break;
        case 4: REANN_NBR(4); break;
        case 8: REANN_NBR(8); break;
        case 16: REANN_NBR(16); break;
        default: REANN_NBR(32); break;
    }
#undef REANN_NBR
}

cudaError_t launch_build(reann_ctx *c, const float *d_pos_caller, const int *d_types_caller, cudaStream_t s) {
    BinParams B = make_bin_params(c);
    int64_t n = c->n;
    cudaError_t e;
    REANN_TIMED(c, REANN_K_NEIGHBORS, s, 12);
    if ((e = cudaMemsetAsync(c->d_bin_count, 0, sizeof(int) * (size_t)(c->nbins + 1), s))) return e;
    if ((e = cudaMemsetAsync(c->d_bin_fill, 0, sizeof(int) * (size_t)(c->nbins + 1), s))) return e;
    if (n > 0) {
        k_bin_count<<<blocks(n, 256), 256, 0, s>>>(n, d_pos_caller, d_types_caller, B, c->d_key, c->d_bin_count,
                                                   c->d_status);
    }
    if ((e = scan_exclusive(c->d_bin_count, c->d_bin_start, c->nbins, c->d_i64 + 0, c->d_scan_tmp, s))) return e;
    if (n > 0) {
        k_bin_scatter<<<blocks(n, 256), 256, 0, s>>>(n, c->d_key, c->d_bin_start, c->d_bin_fill, c->d_perm_tmp);
        k_bin_sort<<<blocks((int64_t)c->nbins * 32, 256), 256, 0, s>>>(c->nbins, c->d_bin_start, c->d_perm_tmp,
                                                                       c->d_perm);
        k_gather_pos<<<blocks(n, 256), 256, 0, s>>>(n, d_pos_caller, d_types_caller, c->d_perm, c->d_pos,
                                                    c->d_pos_build, c->d_inv, c->d_status);
        launch_nbr<false>(c, n, B, nullptr, c->d_cnt, nullptr, s);
    }
    if ((e = scan_exclusive(c->d_cnt, c->d_row, n, c->d_i64 + 1, c->d_scan_tmp, s))) return e;
    if ((e = cudaMemsetAsync(c->d_i64 + 2, 0, sizeof(int64_t), s))) return e;
    if (n > 0) k_row_max<<<blocks(n, 256), 256, 0, s>>>((int)n, c->d_cnt, c->d_i64 + 2);
    return cudaGetLastError();
}

cudaError_t launch_fill(reann_ctx *c, cudaStream_t s) {
    BinParams B = make_bin_params(c);
    REANN_TIMED(c, REANN_K_NEIGHBORS, s);
    if (c->n > 0)
        launch_nbr<true>(c, c->n, B, c->d_row, nullptr, c->d_col, s);
    return cudaGetLastError();
}

cudaError_t launch_skin_check(reann_ctx *c, int *flag, cudaStream_t s) {
    BinParams B = make_bin_params(c);
    double h = 0.5 * c->cfg.skin;
    REANN_TIMED(c, REANN_K_OTHER, s);
    if (c->n > 0)
        k_max_disp<<<blocks(c->n, 256), 256, 0, s>>>((int)c->n, c->d_pos, c->d_pos_build, B, h * h, flag);
    return cudaGetLastError();
}

BinParams make_bin_params(const reann_ctx *c) {
    BinParams B;
    for (int a = 0; a < 3; ++a) {
        B.box[a] = c->box[a];
        B.inv_box[a] = 1.0 / c->box[a];
        B.m[a] = c->m[a];
    }
    B.ncell = c->ncell;
    B.ne = c->ne;
    B.nclass = c->halo ? 2 * c->ne : c->ne;
    B.n_local = c->halo ? c->n_local : c->n;
    double rl = c->cfg.r_cut + c->cfg.skin;
    B.thr = rl * rl;
    return B;
}

}  // namespace reann
