// Per-element atomic networks, fp32 on the CUDA cores.
//
// "Efficient Parallelization of Message Passing Neural Network Potentials for
// Large-Scale Molecular Dynamics", section "REANN Architecture": the
// coefficient update c^t_i = M^{t-1}_i(rho^{t-1}_i) (Eq. 2) and the atomic
// energy E_i from the last layer's density; section "Parallelization
// Algorithm", Eqs. 3 and 5: their vector-Jacobian products.  Each network is
// y = W3 tanh(W2 tanh(W1 ((x - shift) / scale) + b1) + b2) + b3, one per layer
// and element of the centre atom.
//
// Atoms of one element are contiguous rows (internal order), so a tile of TM
// rows uses one network.  A persistent block keeps its element's weights in
// shared memory across tiles.  The backward kernels finish with
//   G[i][n,tau] = dE/dA^t_{i,n,tau} = 2 w_tau A^t_{i,n,tau} dE/drho^t_{i,(n,l)},
// the derivative of the squared sum of Eq. 1 (in the pair-product form
// G[i][n,tau] = l!/tau! sum_m (1 + [m = n]) A^t_{i,m,tau} dE/drho^t_{i,(n,m,l)}),
// so the edge pass can read G (stored in the edge kernels' lane-interleaved
// order, see g_slot_index).
#include "common.cuh"
#include "kernels.cuh"

namespace reann {

constexpr int MLP_TM = 32;
constexpr int MLP_THREADS = 256;

struct MlpNets {
    NetOffsets net[MAX_ELEMENTS];
    int g_pairs;   // lane order of the dE/dA rows written (g_pairs of their layer)
};

enum { MODE_FWD = 0, MODE_ENERGY = 1, MODE_BWD = 2 };

// C[r][c] = sum_k X[r*LDX + k] * W(c, k) for r < TM, c < N, handed to epi(r, c, v).
// TRANS = false: W(c, k) = W[c*LDW + k]; TRANS = true: W(c, k) = W[k*LDW + c].
template <int TM, int N, int K, int LDX, int LDW, bool TRANS, class Epi>
__device__ __forceinline__ void gemm_tile(const float *X, const float *W, Epi epi) {
    constexpr int RM = 4;
    constexpr int RN = (N % 4 == 0) ? 4 : ((N % 3 == 0) ? 3 : ((N % 2 == 0) ? 2 : 1));
    constexpr int RG = TM / RM, CG = N / RN, TASKS = RG * CG;
    for (int task = threadIdx.x; task < TASKS; task += blockDim.x) {
        int rg = task % RG, cg = task / RG;
        float acc[RM][RN];
#pragma unroll
        for (int i = 0; i < RM; ++i)
#pragma unroll
            for (int j = 0; j < RN; ++j) acc[i][j] = 0.f;
#pragma unroll 4
        for (int k = 0; k < K; ++k) {
            float a[RM], b[RN];
#pragma unroll
            for (int i = 0; i < RM; ++i) a[i] = X[(rg + i * RG) * LDX + k];
#pragma unroll
            for (int j = 0; j < RN; ++j) b[j] = TRANS ? W[k * LDW + cg * RN + j] : W[(cg * RN + j) * LDW + k];
#pragma unroll
            for (int i = 0; i < RM; ++i)
#pragma unroll
                for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < RM; ++i)
#pragma unroll
            for (int j = 0; j < RN; ++j) epi(rg + i * RG, cg * RN + j, acc[i][j]);
    }
}

// DIN: density features per atom (network input width): D = 3 N_phi, or
// 3 N_phi (N_phi+1)/2 for the pair-product form
template <int NP, int H1, int H2, int MODE, int DIN>
struct MlpLayout {
    static constexpr int D = 3 * NP;
    static constexpr int NA = NP * NT;
    static constexpr int DOUT = MODE == MODE_ENERGY ? 1 : D;
    static constexpr int LDX = DIN + 1, LD1 = H1 + 1, LD2 = H2 + 1, LDY = D + 1;
    static constexpr int oW1 = 0;
    static constexpr int oW2 = oW1 + H1 * LDX;
    static constexpr int oW3 = oW2 + H2 * LD1;
    static constexpr int ob1 = oW3 + DOUT * LD2;
    static constexpr int ob2 = ob1 + H1;
    static constexpr int ob3 = ob2 + H2;
    static constexpr int oshift = ob3 + DOUT;
    static constexpr int oscale = oshift + DIN;
    static constexpr int oX = oscale + DIN;
    static constexpr int oA1 = oX + MLP_TM * LDX;
    static constexpr int oA2 = oA1 + MLP_TM * LD1;
    static constexpr int oB1 = oA2 + MLP_TM * LD2;
    static constexpr int oB2 = oB1 + (MODE == MODE_FWD ? 0 : MLP_TM * LD1);
    static constexpr int oY = oB2 + (MODE == MODE_FWD ? 0 : MLP_TM * LD2);
    static constexpr int total = oY + (MODE == MODE_BWD ? MLP_TM * LDY : 0);
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int NP, int H1, int H2, int MODE, int DIN>
__global__ void __launch_bounds__(MLP_THREADS) k_mlp(const int4 *__restrict__ tiles, int n_tiles,
                                                     const float *__restrict__ w, MlpNets nets,
                                                     const float *__restrict__ X, float *__restrict__ Y,
                                                     const float *__restrict__ dY, float *__restrict__ Ei,
                                                     const float *__restrict__ A, float *__restrict__ Gout) {
    using Lay = MlpLayout<NP, H1, H2, MODE, DIN>;
    constexpr int D = Lay::D, NA = Lay::NA, DOUT = Lay::DOUT;
    constexpr bool PAIR = DIN != D;
    constexpr int LDX = Lay::LDX, LD1 = Lay::LD1, LD2 = Lay::LD2, LDY = Lay::LDY;
    extern __shared__ float sm[];
    float *sW1 = sm + Lay::oW1, *sW2 = sm + Lay::oW2, *sW3 = sm + Lay::oW3;
    float *sb1 = sm + Lay::ob1, *sb2 = sm + Lay::ob2, *sb3 = sm + Lay::ob3;
    float *sshift = sm + Lay::oshift, *sscale = sm + Lay::oscale;
    float *sX = sm + Lay::oX, *sA1 = sm + Lay::oA1, *sA2 = sm + Lay::oA2;
    float *sB1 = sm + Lay::oB1, *sB2 = sm + Lay::oB2, *sY = sm + Lay::oY;
    const int tid = threadIdx.x;
    int cur = -1;

    for (int ti = blockIdx.x; ti < n_tiles; ti += gridDim.x) {
        int4 tile = tiles[ti];
        const int e = tile.x, r0 = tile.y, rows = tile.z;
        if (e != cur) {
            __syncthreads();
            const NetOffsets &o = nets.net[e];
            for (int k = tid; k < H1 * DIN; k += MLP_THREADS) sW1[(k / DIN) * LDX + k % DIN] = w[o.W1 + k];
            for (int k = tid; k < H2 * H1; k += MLP_THREADS) sW2[(k / H1) * LD1 + k % H1] = w[o.W2 + k];
            for (int k = tid; k < DOUT * H2; k += MLP_THREADS) sW3[(k / H2) * LD2 + k % H2] = w[o.W3 + k];
            for (int k = tid; k < H1; k += MLP_THREADS) sb1[k] = w[o.b1 + k];
            for (int k = tid; k < H2; k += MLP_THREADS) sb2[k] = w[o.b2 + k];
            for (int k = tid; k < DOUT; k += MLP_THREADS) sb3[k] = w[o.b3 + k];
            for (int k = tid; k < DIN; k += MLP_THREADS) {
                sshift[k] = w[o.shift + k];
                sscale[k] = w[o.scale + k];
            }
            cur = e;
        }
        __syncthreads();
        for (int k = tid; k < MLP_TM * DIN; k += MLP_THREADS) {
            int r = k / DIN, f = k % DIN;
            float v = r < rows ? X[(int64_t)(r0 + r) * DIN + f] : 0.f;
            sX[r * LDX + f] = (v - sshift[f]) / sscale[f];
        }
        if (MODE == MODE_BWD)
            for (int k = tid; k < MLP_TM * D; k += MLP_THREADS) {
                int r = k / D, f = k % D;
                sY[r * LDY + f] = r < rows ? dY[(int64_t)(r0 + r) * D + f] : 0.f;
            }
        __syncthreads();
        gemm_tile<MLP_TM, H1, DIN, LDX, LDX, false>(sX, sW1, [&](int r, int c, float v) {
            sA1[r * LD1 + c] = tanhf(v + sb1[c]);
        });
        __syncthreads();
        gemm_tile<MLP_TM, H2, H1, LD1, LD1, false>(sA1, sW2, [&](int r, int c, float v) {
            sA2[r * LD2 + c] = tanhf(v + sb2[c]);
        });
        __syncthreads();
        if (MODE == MODE_FWD) {
            gemm_tile<MLP_TM, DOUT, H2, LD2, LD2, false>(sA2, sW3, [&](int r, int c, float v) {
                if (r < rows) Y[(int64_t)(r0 + r) * D + c] = v + sb3[c];
            });
        } else {
            if (MODE == MODE_ENERGY) {
                gemm_tile<MLP_TM, 1, H2, LD2, LD2, false>(sA2, sW3, [&](int r, int c, float v) {
                    if (r < rows) Ei[r0 + r] = v + sb3[0];
                });
                // dE_i/da2 = W3[0][k]
                for (int k = tid; k < MLP_TM * H2; k += MLP_THREADS) {
                    int r = k / H2, h = k % H2;
                    float a = sA2[r * LD2 + h];
                    sB2[r * LD2 + h] = sW3[h] * (1.f - a * a);
                }
            } else {
                gemm_tile<MLP_TM, H2, D, LDY, LD2, true>(sY, sW3, [&](int r, int c, float v) {
                    float a = sA2[r * LD2 + c];
                    sB2[r * LD2 + c] = v * (1.f - a * a);
                });
            }
            __syncthreads();
            gemm_tile<MLP_TM, H1, H2, LD2, LD1, true>(sB2, sW2, [&](int r, int c, float v) {
                float a = sA1[r * LD1 + c];
                sB1[r * LD1 + c] = v * (1.f - a * a);
            });
            __syncthreads();
            // dE/drho = (W1^T g1) / scale, stored over sX
            gemm_tile<MLP_TM, DIN, H1, LD1, LDX, true>(sB1, sW1, [&](int r, int c, float v) {
                sX[r * LDX + c] = v / sscale[c];
            });
            __syncthreads();
            // G rows are stored in the edge kernels' lane-interleaved order
            for (int k = tid; k < rows * NA; k += MLP_THREADS) {
                const int r = k / NA, q = k % NA;
                const int src = g_slot_source(q, NP, nets.g_pairs);
                const int nn = src / NT, u = src % NT;
                const int l = u == 0 ? 0 : (u < 4 ? 1 : 2);
                const int64_t rb = (int64_t)(r0 + r) * NA;
                if (PAIR) {
                    // dE/dA_{n,tau} = l!/tau! sum_m (1 + [m = n]) A_{m,tau} dE/drho_(min(n,m), max(n,m), l)
                    constexpr int PP = NP * (NP + 1) / 2;
                    const float *g = sX + r * LDX + l * PP;
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < NP; ++m) {
                        const int lo = m < nn ? m : nn, hi = m < nn ? nn : m;
                        const float f = (m == nn ? 2.f : 1.f) * g[lo * NP - lo * (lo - 1) / 2 + (hi - lo)];
                        acc = fmaf(f, A[rb + m * NT + u], acc);
                    }
                    Gout[rb + q] = (u >= 7 ? 2.f : 1.f) * acc;
                } else {
                    const float wt = u >= 7 ? 4.f : 2.f;  // 2 * l!/(lx! ly! lz!)
                    Gout[rb + q] = wt * A[rb + src] * sX[r * LDX + l * NP + nn];
                }
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// host side

template <int NP, int H1, int H2, int MODE, int DIN>
static cudaError_t run_mlp(reann_ctx *c, const MlpNets &nets, const float *X, float *Y, const float *dY, float *Ei,
                           const float *A, float *G, cudaStream_t s) {
    using Lay = MlpLayout<NP, H1, H2, MODE, DIN>;
    static_assert(Lay::bytes <= 227 * 1024, "one block must fit an SM's shared memory");
    static bool configured[64] = {};
    auto kern = k_mlp<NP, H1, H2, MODE, DIN>;
    if (c->device < 0 || c->device >= 64) return cudaErrorInvalidDevice;
    if (!configured[c->device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::bytes);
        if (e) return e;
        configured[c->device] = true;
    }
    if (c->n_tiles == 0) return cudaSuccess;
    int per_sm = (int)((227 * 1024) / (Lay::bytes + 1024));
    if (per_sm < 1) per_sm = 1;
    int grid = c->sm_count * per_sm;
    if (grid > c->n_tiles) grid = c->n_tiles;
    REANN_TIMED(c, MODE == MODE_FWD ? REANN_K_MLP_FWD : (MODE == MODE_ENERGY ? REANN_K_MLP_ENERGY : REANN_K_MLP_BWD), s);
    kern<<<grid, MLP_THREADS, Lay::bytes, s>>>(c->d_tiles, c->n_tiles, c->d_w, nets, X, Y, dY, Ei, A, G);
    return cudaGetLastError();
}

template <int MODE>
static cudaError_t dispatch(reann_ctx *c, const MlpNets &nets, const float *X, float *Y, const float *dY, float *Ei,
                            const float *A, float *G, cudaStream_t s) {
    if (c->DR != c->D) {
        // pair-product densities: N_phi = 8, L = 2
        if (c->NP == 8 && c->H1 == 64 && c->H2 == 64) return run_mlp<8, 64, 64, MODE, 108>(c, nets, X, Y, dY, Ei, A, G, s);
        if (c->NP == 8 && c->H1 == 128 && c->H2 == 128)
            return run_mlp<8, 128, 128, MODE, 108>(c, nets, X, Y, dY, Ei, A, G, s);
        return cudaErrorInvalidValue;
    }
#define REANN_MLP_CASE(NPV, A1, A2)                                                          \
    if (c->NP == NPV && c->H1 == A1 && c->H2 == A2)                                           \
        return run_mlp<NPV, A1, A2, MODE, 3 * NPV>(c, nets, X, Y, dY, Ei, A, G, s);
    REANN_MLP_CASE(8, 64, 64)
    REANN_MLP_CASE(8, 128, 128)
    REANN_MLP_CASE(8, 64, 128)
    REANN_MLP_CASE(8, 128, 64)
    REANN_MLP_CASE(10, 64, 64)
    REANN_MLP_CASE(10, 128, 128)
    REANN_MLP_CASE(10, 64, 128)
    REANN_MLP_CASE(10, 128, 64)
#undef REANN_MLP_CASE
    return cudaErrorInvalidValue;
}

static MlpNets nets_of(const std::vector<NetOffsets> &v, int first, int ne, int NP, int layer) {
    MlpNets m;
    m.g_pairs = g_pairs(NP, layer);
    for (int e = 0; e < ne; ++e) m.net[e] = v[first + e];
    return m;
}

cudaError_t launch_mlp_coef_fwd(reann_ctx *c, int t, cudaStream_t s) {
    const int64_t nR = c->n * c->DR;
    return dispatch<MODE_FWD>(c, nets_of(c->coef_nets, t * c->ne, c->ne, c->NP, 0), c->d_rho + t * nR,
                              c->d_coef + (t + 1) * c->n_slots * c->D, nullptr, nullptr, nullptr, nullptr, s);
}

cudaError_t launch_mlp_energy(reann_ctx *c, cudaStream_t s) {
    const int64_t nR = c->n * c->DR, nA = c->n * c->NA;
    const int t = c->T - 1;
    return dispatch<MODE_ENERGY>(c, nets_of(c->energy_nets, 0, c->ne, c->NP, c->T - 1), c->d_rho + t * nR, nullptr,
                                 nullptr, c->d_Ei, c->d_A + t * nA, c->d_G, s);
}

cudaError_t launch_mlp_coef_bwd(reann_ctx *c, int t, cudaStream_t s) {
    // network M^{t-1}: input rho^{t-1}, upstream gradient dE/dc^t, output G^{t-1}
    const int64_t nR = c->n * c->DR, nA = c->n * c->NA;
    return dispatch<MODE_BWD>(c, nets_of(c->coef_nets, (t - 1) * c->ne, c->ne, c->NP, t - 1), c->d_rho + (t - 1) * nR,
                              nullptr, c->d_dc, nullptr, c->d_A + (t - 1) * nA, c->d_G, s);
}

}  // namespace reann
