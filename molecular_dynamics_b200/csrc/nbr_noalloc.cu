// Allocation-free pair list: the same neighbour list reann_build_neighbors
// builds, for callers that must not allocate device memory.
//
// Who cannot allocate, and why: host programs that hand the whole device to
// their own memory pool or run under a fixed memory budget (an MD engine's
// force-evaluation plug-in, for example, receives its buffers and may not
// grow the footprint), and latency-critical loops that must not call
// cudaMalloc or cudaFree because those calls can synchronise the whole device
// and stall other streams.  Such a caller passes its own input and output
// buffers; all scratch this call needs lives in one file-scope __device__
// array of fixed size, present on every GPU that loads the library until the
// process exits.
//
// The result is bit-identical to reann_get_neighbors after
// reann_build_neighbors: every ordered pair (i, j), i != j, whose
// minimum-image distance satisfies (dx*dx + dy*dy) + dz*dz < (r_cut + skin)^2
// in fp64 with each operation rounded separately, rows in the caller's atom
// order and sorted by j.
//
// Sharing rules: every call uses the same array and leaves its contents
// behind; each call clears what must start at zero.  Two calls whose GPU work
// overlaps (different streams, or different host threads on one device) race
// on the array and corrupt each other's result: serialise them.  The first
// call on a device looks up the array's device address (cudaGetSymbolAddress)
// with that device current; make that first call before any stream capture.
// The address is kept for the life of the process: after cudaDeviceReset on
// a device the array may move, and this call must not be used on that device
// again in the same process.
#include <mutex>

#include "common.cuh"

namespace reann {
namespace {

constexpr int NA_MAX_ATOMS = 131072;
constexpr int NA_MAX_CELLS = 32768;
constexpr int NA_SCAN_THREADS = 1024;

struct NoAllocScratch {
    int cell_count[NA_MAX_CELLS + 1];
    int cell_start[NA_MAX_CELLS + 1];
    int cell_fill[NA_MAX_CELLS + 1];
    int cell_of[NA_MAX_ATOMS];
    int unsorted[NA_MAX_ATOMS];
    int sorted[NA_MAX_ATOMS];
    int row_count[NA_MAX_ATOMS];
    long long total;
    int status;
};

// About 2.5 MB of device memory on every GPU that loads the library.
static __device__ __align__(256) NoAllocScratch g_noalloc_scratch;

struct Grid {
    double box[3];
    int m[3];
    int ncell;
    double thr;
};

__device__ __forceinline__ int na_cell_axis(float xf, double L, int m) {
    const double x = (double)xf;
    const double u = x - L * floor(x / L);
    const int c = (int)(u * (double)m / L);
    return c < 0 ? 0 : (c >= m ? m - 1 : c);
}

// the list's distance test: fp64, every operation rounded on its own
__device__ __forceinline__ double na_r2(const float *pi, const float *pj, const Grid &g) {
    double d[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        double v = __dsub_rn((double)pj[a], (double)pi[a]);
        d[a] = __dsub_rn(v, __dmul_rn(g.box[a], rint(__ddiv_rn(v, g.box[a]))));
    }
    return __dadd_rn(__dadd_rn(__dmul_rn(d[0], d[0]), __dmul_rn(d[1], d[1])), __dmul_rn(d[2], d[2]));
}

__device__ __forceinline__ int na_stencil(int c, int m, int out[3]) {
    if (m < 3) {
        for (int s = 0; s < m; ++s) out[s] = s;
        return m;
    }
    const int a = c == 0 ? m - 1 : c - 1, b = c, d = c == m - 1 ? 0 : c + 1;
    const int lo = min(a, min(b, d)), hi = max(a, max(b, d));
    out[0] = lo;
    out[1] = a + b + d - lo - hi;
    out[2] = hi;
    return 3;
}

__global__ void k_na_clear(NoAllocScratch *S, int ncell) {
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k <= ncell; k += gridDim.x * blockDim.x) {
        S->cell_count[k] = 0;
        S->cell_fill[k] = 0;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        S->total = 0;
        S->status = 0;
    }
}

__global__ void k_na_bin(NoAllocScratch *S, int n, const float *__restrict__ pos, Grid g) {
    const int a = blockIdx.x * blockDim.x + threadIdx.x;
    if (a >= n) return;
    float x = pos[3 * a], y = pos[3 * a + 1], z = pos[3 * a + 2];
    if (!isfinite(x) || !isfinite(y) || !isfinite(z)) {
        atomicOr(&S->status, ST_NONFINITE);
        x = y = z = 0.f;
    }
    const int c = (na_cell_axis(x, g.box[0], g.m[0]) * g.m[1] + na_cell_axis(y, g.box[1], g.m[1])) * g.m[2] +
                  na_cell_axis(z, g.box[2], g.m[2]);
    S->cell_of[a] = c;
    atomicAdd(&S->cell_count[c], 1);
}

// single-block exclusive scan of in[0..len) into out[0..len], out[len] = total
__device__ void na_block_scan(const int *in, int *out, int len, long long *total) {
    __shared__ long long warp_sums[NA_SCAN_THREADS / 32];
    __shared__ long long carry;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < len; base += NA_SCAN_THREADS) {
        const int k = base + threadIdx.x;
        const long long v = k < len ? in[k] : 0;
        long long x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            long long w = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sums[lane] = w;
        }
        __syncthreads();
        const long long ex = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
        if (k < len) out[k] = (int)ex;
        __syncthreads();
        if (threadIdx.x == 0) carry += warp_sums[NA_SCAN_THREADS / 32 - 1];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        out[len] = (int)carry;
        if (total) *total = carry;
    }
}

__global__ void __launch_bounds__(NA_SCAN_THREADS) k_na_scan_cells(NoAllocScratch *S, int ncell) {
    na_block_scan(S->cell_count, S->cell_start, ncell, nullptr);
}

__global__ void k_na_scatter(NoAllocScratch *S, int n) {
    const int a = blockIdx.x * blockDim.x + threadIdx.x;
    if (a >= n) return;
    const int c = S->cell_of[a];
    S->unsorted[S->cell_start[c] + atomicAdd(&S->cell_fill[c], 1)] = a;
}

// one warp per cell: order the cell's atoms by index (ranks are unique)
__global__ void k_na_sort_cells(NoAllocScratch *S, int ncell) {
    const int c = (int)(((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (c >= ncell) return;
    const int s0 = S->cell_start[c], s1 = S->cell_start[c + 1];
    for (int p = s0 + lane; p < s1; p += 32) {
        const int v = S->unsorted[p];
        int rank = 0;
        for (int q = s0; q < s1; ++q) rank += S->unsorted[q] < v;
        S->sorted[s0 + rank] = v;
    }
}

// count (FILL = false) or write (FILL = true) each atom's row; a written row
// is then sorted by neighbour index (rows are short)
template <bool FILL>
__global__ void k_na_rows(NoAllocScratch *S, int n, const float *__restrict__ pos, Grid g,
                          const int *__restrict__ row, int *__restrict__ col) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float *pi = pos + 3 * (int64_t)i;
    int sx[3], sy[3], sz[3];
    const int nx = na_stencil(na_cell_axis(pi[0], g.box[0], g.m[0]), g.m[0], sx);
    const int ny = na_stencil(na_cell_axis(pi[1], g.box[1], g.m[1]), g.m[1], sy);
    const int nz = na_stencil(na_cell_axis(pi[2], g.box[2], g.m[2]), g.m[2], sz);
    const int o = FILL ? row[i] : 0;
    int cnt = 0;
    for (int a = 0; a < nx; ++a)
        for (int b = 0; b < ny; ++b)
            for (int d = 0; d < nz; ++d) {
                const int c = (sx[a] * g.m[1] + sy[b]) * g.m[2] + sz[d];
                for (int q = S->cell_start[c]; q < S->cell_start[c + 1]; ++q) {
                    const int j = S->sorted[q];
                    if (j == i) continue;
                    if (na_r2(pi, pos + 3 * (int64_t)j, g) < g.thr) {
                        if (FILL) col[o + cnt] = j;
                        ++cnt;
                    }
                }
            }
    if (!FILL) {
        S->row_count[i] = cnt;
    } else {
        int *r = col + o;
        for (int p = 1; p < cnt; ++p) {
            const int v = r[p];
            int k = p - 1;
            while (k >= 0 && r[k] > v) {
                r[k + 1] = r[k];
                --k;
            }
            r[k + 1] = v;
        }
    }
}

__global__ void __launch_bounds__(NA_SCAN_THREADS) k_na_scan_rows(NoAllocScratch *S, int n, int *__restrict__ row) {
    na_block_scan(S->row_count, row, n, &S->total);
}

std::mutex g_addr_mutex;
NoAllocScratch *g_addr[64] = {};

reann_status na_fail(reann_status st, const std::string &msg) {
    set_context_free_error(msg);   // read back with reann_last_error(NULL)
    return st;
}

}  // namespace
}  // namespace reann

using namespace reann;

extern "C" reann_status reann_pair_list_noalloc(int64_t n, const float *pos, const double box[3], double r_cut,
                                                double skin, int32_t *row, int32_t *col, int64_t cap, int64_t *nnz,
                                                reann_stream stream) {
    if (n < 0 || !box || !row || !nnz || (n > 0 && !pos) || cap < 0 || (cap > 0 && !col) || !(r_cut > 0) ||
        !(skin >= 0))
        return na_fail(REANN_ERR_ARG, "invalid arguments");
    if (n > NA_MAX_ATOMS)
        return na_fail(REANN_ERR_CAPACITY, "reann_pair_list_noalloc handles at most " + std::to_string(NA_MAX_ATOMS) +
                                               " atoms (" + std::to_string(n) + " given)");
    const double rl = r_cut + skin;
    Grid g;
    int ncell = 1;
    for (int a = 0; a < 3; ++a) {
        if (!(box[a] > 0) || !std::isfinite(box[a]) || box[a] < 2.0 * rl)
            return na_fail(REANN_ERR_BOX, "box edge must be finite and at least 2 (r_cut + skin)");
        g.box[a] = box[a];
        g.m[a] = std::max(1, (int)std::floor(box[a] / rl));
        ncell *= g.m[a];
    }
    // coarser cells (still at least r_cut + skin wide) when the grid exceeds the scratch
    while (ncell > NA_MAX_CELLS) {
        int a = 0;
        for (int b = 1; b < 3; ++b)
            if (g.m[b] > g.m[a]) a = b;
        g.m[a] = std::max(1, g.m[a] / 2);
        ncell = g.m[0] * g.m[1] * g.m[2];
    }
    g.ncell = ncell;
    g.thr = rl * rl;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return na_fail(REANN_ERR_CUDA, "no current CUDA device");
    }
    NoAllocScratch *S = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_addr_mutex);
        if (!g_addr[dev]) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess || !p) {
                cudaGetLastError();
                return na_fail(REANN_ERR_CUDA, std::string("cudaGetSymbolAddress failed: ") + cudaGetErrorString(e));
            }
            g_addr[dev] = static_cast<NoAllocScratch *>(p);
        }
        S = g_addr[dev];
    }
    cudaStream_t s = (cudaStream_t)stream;
    const int N = (int)n;
    const unsigned nb = (unsigned)((n + 255) / 256);
    k_na_clear<<<(ncell + 256) / 256, 256, 0, s>>>(S, ncell);
    if (N > 0) k_na_bin<<<nb, 256, 0, s>>>(S, N, pos, g);
    k_na_scan_cells<<<1, NA_SCAN_THREADS, 0, s>>>(S, ncell);
    if (N > 0) {
        k_na_scatter<<<nb, 256, 0, s>>>(S, N);
        k_na_sort_cells<<<(unsigned)(((int64_t)ncell * 32 + 255) / 256), 256, 0, s>>>(S, ncell);
        k_na_rows<false><<<nb, 256, 0, s>>>(S, N, pos, g, nullptr, nullptr);
    }
    k_na_scan_rows<<<1, NA_SCAN_THREADS, 0, s>>>(S, N, row);
    if ((e = cudaGetLastError()) != cudaSuccess) {
        cudaStreamSynchronize(s);
        cudaGetLastError();
        return na_fail(REANN_ERR_CUDA, std::string("CUDA error: ") + cudaGetErrorString(e));
    }
    long long total = 0;
    int status = 0;
    if ((e = cudaMemcpyAsync(&total, &S->total, sizeof(long long), cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(&status, &S->status, sizeof(int), cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess) {
        cudaGetLastError();
        return na_fail(REANN_ERR_CUDA, std::string("CUDA error: ") + cudaGetErrorString(e));
    }
    *nnz = total;
    if (status & ST_NONFINITE) return na_fail(REANN_ERR_NONFINITE, "non-finite position");
    // row offsets are int32: a longer list is rejected before anything is written to col
    if (total > INT32_MAX) return na_fail(REANN_ERR_CAPACITY, "neighbour list exceeds 2^31-1 entries");
    if (total > cap)
        return na_fail(REANN_ERR_CAPACITY, "col holds " + std::to_string(cap) + " entries, the list has " +
                                               std::to_string(total));
    if (N > 0) k_na_rows<true><<<nb, 256, 0, s>>>(S, N, pos, g, row, col);
    if ((e = cudaGetLastError()) != cudaSuccess || (e = cudaStreamSynchronize(s)) != cudaSuccess) {
        cudaGetLastError();
        return na_fail(REANN_ERR_CUDA, std::string("CUDA error: ") + cudaGetErrorString(e));
    }
    return REANN_OK;
}
