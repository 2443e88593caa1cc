// Edge kernels: orbital + embedded-density forward and the reverse-mode edge
// pass that produces forces and the gradient with respect to the neighbours'
// coefficients.
//
// "Efficient Parallelization of Message Passing Neural Network Potentials for
// Large-Scale Molecular Dynamics", section "REANN Architecture", Eq. 1:
//   A^t_{i,n,tau} = sum_j c^t_{j,(n,l)} phi_n(r_ij) Y_tau(d_ij),
//   rho^t_{i,(n,l)} = sum_{|tau|=l} l!/(lx! ly! lz!) (A^t_{i,n,tau})^2,
// with phi_n(r) = exp(-alpha (r - mu_n)^2) (cos(pi r / r_c) + 1) / 2 and the
// Cartesian monomials Y_tau(d) = dx^lx dy^ly dz^lz of the displacement
// d_ij = x_j - x_i.  Section "Parallelization Algorithm", Eqs. 3-5 give the
// forces through the chain rule; here they are evaluated as vector-Jacobian
// products and gathered per atom, with no atomics:
//   F_k = sum_j sum_{n,tau} H_{n,tau} (phi_n'(r) Y_tau d / r + phi_n grad Y_tau),
//   H_{n,tau} = G_k[n,tau] c_j[n,l] + (-1)^l G_j[n,tau] c_k[n,l],
//   dE/dc_k[n,l] = (-1)^l sum_j phi_n(r) sum_{|tau|=l} G_j[n,tau] Y_tau(d),
// where d = x_j - x_k and G = dE/dA.  Both directed edges k->j and j->k are
// folded into the row of k because the list is symmetric; the parity (-1)^l
// comes from Y_tau(-d) = (-1)^l Y_tau(d).
//
// The backward pass uses the special-function unit (__sincosf, __fdividef, and
// the exponential as __expf or as ex2.approx of t^2 (-alpha log2 e)): the
// arguments are bounded (sine/cosine argument in [0, pi), exponent <= 0) and
// only forces depend on them.  The forward pass keeps an accurate expf and
// evaluates the cutoff as a polynomial accurate to fp32 rounding: the densities
// feed standardised network inputs, where the intrinsics' ~1e-7 errors showed
// up as 1e-5-level per-atom energy errors.
//
// Tuple order inside one radial index n: (000); (100)(010)(001);
// (200)(020)(002)(110)(101)(011).  Feature (n, l) sits at index l*N_phi + n.
// With pair-product densities (density_form = 1) the density pass writes A
// only and k_rho_pair forms rho_(n,m,l) = sum_tau l!/tau! A_{n,tau} A_{m,tau};
// the backward pass is the same in both forms (it consumes G = dE/dA).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace reann {

EdgeParams make_edge_params(const reann_ctx *c) {
    EdgeParams P;
    for (int a = 0; a < 3; ++a) {
        P.box[a] = c->box[a];
        P.inv_box[a] = 1.0 / c->box[a];
        P.L_hi[a] = (float)c->box[a];
        P.L_lo[a] = (float)(c->box[a] - (double)P.L_hi[a]);
        P.inv_L[a] = (float)(1.0 / c->box[a]);
    }
    P.r_cut = (float)c->cfg.r_cut;
    P.r_cut2 = (float)(c->cfg.r_cut * c->cfg.r_cut);
    const double th = 0.5 * 3.14159265358979323846 / c->cfg.r_cut;
    P.th_hi = (float)th;
    P.th_lo = (float)(th - (double)P.th_hi);
    P.alpha = (float)c->cfg.alpha;
    P.neg_alpha_log2e = (float)(-c->cfg.alpha * 1.44269504088896340736);
    for (int k = 0; k < 16; ++k) {
        const double mu = k < c->cfg.n_radial ? c->cfg.r_cut * k / (double)(c->cfg.n_radial - 1) : 0.0;
        P.mu_hi[k] = (float)mu;
        P.mu_lo[k] = (float)(mu - (double)P.mu_hi[k]);
    }
    P.n_rows = c->n_slots;
    P.n_list = c->cap;
    P.status = c->d_status;
    return P;
}

// Minimum-image displacement x_j - x_i in fp32 without losing the fp32
// precision of the result: TwoSum gives s + t = x_j - x_i exactly; the image
// shift k L is removed from s exactly (for k != 0, s and k L_hi are within a
// factor of two, so the difference is exact) and the small terms t - k L_lo
// added last.  The result is the correctly rounded displacement up to the
// L_lo rounding (~1e-13 A).
__device__ __forceinline__ float min_image(float xi, float xj, float L_hi, float L_lo, float inv_L) {
    const float s = xj - xi;
    const float bb = s - xj;
    const float t = (xj - (s - bb)) + (-xi - bb);
    const float k = rintf(s * inv_L);
    return (s - k * L_hi) + (t - k * L_lo);
}

__device__ __forceinline__ float3 displacement(float4 pi, float4 pj, const EdgeParams &P) {
    return make_float3(min_image(pi.x, pj.x, P.L_hi[0], P.L_lo[0], P.inv_L[0]),
                       min_image(pi.y, pj.y, P.L_hi[1], P.L_lo[1], P.inv_L[1]),
                       min_image(pi.z, pj.z, P.L_hi[2], P.L_lo[2], P.inv_L[2]));
}

// ---------------------------------------------------------------------------
// active pairs: the entries of each row closer than r_cut, compacted to the
// front of the row's slot (same offsets as the full list), each with its
// displacement and distance (dx, dy, dz, r), which every edge pass of the
// evaluation then reads instead of recomputing.
template <bool DR, int LPR, int B>   // DR: also the distance rounding residuals (fp32-accurate paths)
__global__ void __launch_bounds__(128, 8) k_active(int n, const float4 *__restrict__ pos, const int *__restrict__ row,
                                                 const int *__restrict__ col, int *__restrict__ act_cnt,
                                                 int *__restrict__ act_col, float4 *__restrict__ act_geo,
                                                 float *__restrict__ act_dr, EdgeParams P,
                                                 unsigned long long *__restrict__ total) {
    // LPR lanes per row (32 / LPR rows per warp): the lanes of a row test
    // consecutive entries, B per lane with their loads issued together, and a
    // ballot over the row's lanes compacts the active ones in row order, so the
    // writes stay contiguous.  Warps stride over the rows (the next row's
    // position and bounds are loaded while the current one is tested) and add
    // their count of active pairs to the total once.
    static_assert(LPR == 8 || LPR == 16 || LPR == 32, "rows of 8, 16 or 32 lanes");
    constexpr int RPW = 32 / LPR;
    const int lane = threadIdx.x & 31, sl = lane % LPR;
    const unsigned rmask = LPR == 32 ? 0xffffffffu : ((1u << LPR) - 1u) << (lane - sl);
    unsigned long long tot = 0;
    int i = (blockIdx.x * 4 + (threadIdx.x >> 5)) * RPW + lane / LPR;
    const int stride = gridDim.x * 4 * RPW;
    float4 pi_n = i < n ? pos[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    int q0_n = i < n ? row[i] : 0, q1_n = i < n ? row[i + 1] : 0;
    for (; i < n; i += stride) {
        const float4 pi = pi_n;
        const int q0 = q0_n, q1 = checked_end(q1_n, P.n_list, P.status);
        if (i + stride < n) {
            pi_n = pos[i + stride];
            q0_n = row[i + stride];
            q1_n = row[i + stride + 1];
        }
        int k = 0;
        for (int base = q0; base < q1; base += LPR * B) {
            int j[B];
            float4 pj[B];
#pragma unroll
            for (int b = 0; b < B; ++b) {
                const int q = base + LPR * b + sl;
                j[b] = q < q1 ? (int)checked(col[q], P.n_rows, P.status) : -1;
            }
#pragma unroll
            for (int b = 0; b < B; ++b) pj[b] = j[b] >= 0 ? pos[j[b]] : pi;
#pragma unroll
            for (int b = 0; b < B; ++b) {
                if (base + LPR * b >= q1) break;
                const float3 d = displacement(pi, pj[b], P);
                const float r2 = d.x * d.x + d.y * d.y + d.z * d.z;
                const bool act = j[b] >= 0 && r2 < P.r_cut2;
                const unsigned mask = __ballot_sync(rmask, act) & rmask;
                if (act) {
                    const int o = q0 + k + __popc(mask & ((1u << lane) - 1u));
                    act_col[o] = j[b];
                    float r = sqrtf(r2);
                    if (DR) {
                        // the fp32-accurate paths: r from the exact displacement of the
                        // fp32 positions, correctly rounded, and its rounding residual
                        double e[3] = {(double)pj[b].x - (double)pi.x, (double)pj[b].y - (double)pi.y,
                                       (double)pj[b].z - (double)pi.z};
#pragma unroll
                        for (int a = 0; a < 3; ++a) e[a] -= P.box[a] * rint(e[a] * P.inv_box[a]);
                        const double r64 = sqrt(e[0] * e[0] + e[1] * e[1] + e[2] * e[2]);
                        r = (float)r64;
                        act_dr[o] = (float)(r64 - (double)r);
                    }
                    act_geo[o] = make_float4(d.x, d.y, d.z, r);
                }
                k += __popc(mask);
            }
        }
        if (sl == 0) act_cnt[i] = k;
        tot += (unsigned long long)k;
    }
    if (sl == 0 && tot) atomicAdd(total, tot);
}

cudaError_t launch_active(reann_ctx *c, cudaStream_t s) {
    if (c->n == 0) return cudaSuccess;
    EdgeParams P = make_edge_params(c);
    cudaError_t e = cudaMemsetAsync(c->d_i64 + 3, 0, sizeof(int64_t), s);
    if (e) return e;
    REANN_TIMED(c, REANN_K_ACTIVE, s);
    // two rows per warp, 16 lanes x 4 entries each (a whole warp per row left most
    // lanes idle on rows of ~80 entries and kept half as many gathers in flight)
    constexpr int LPR = 16, B = 4, RPB = 4 * (32 / LPR);   // rows per block and pass
    // one resident wave (8 blocks of 128 threads per SM at <= 64 registers)
    const unsigned grid = (unsigned)std::min<int64_t>((c->n + RPB - 1) / RPB, (int64_t)c->sm_count * 8);
    const int *col = c->dd ? c->d_col_dd : c->d_col;
    unsigned long long *total = (unsigned long long *)(c->d_i64 + 3);
    if (c->d_act_dr)
        k_active<true, LPR, B><<<grid, 128, 0, s>>>((int)c->n, c->d_pos, c->d_row, col, c->d_act_cnt, c->d_act_col,
                                                    c->d_act_geo, c->d_act_dr, P, total);
    else
        k_active<false, LPR, B><<<grid, 128, 0, s>>>((int)c->n, c->d_pos, c->d_row, col, c->d_act_cnt,
                                                     c->d_act_col, c->d_act_geo, nullptr, P, total);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Lane decomposition shared by both edge passes: a slot of LPE = N_phi / 2
// lanes owns one centre atom and walks its active neighbours in row order;
// lane `sub` owns radial indices 2 sub and 2 sub + 1.  A warp holds
// CPW = 32 / LPE slots (8 centres for N_phi = 8).  The slot's lanes read one
// neighbour's coefficients and dE/dA row as contiguous runs, and each lane
// keeps only its own radial indices' accumulators, so the forward needs no
// cross-lane reduction and the backward only a sum of the force over the slot.
// f_c(r) = (cos(pi r / r_c) + 1) / 2 = cos^2(theta), theta = pi r / (2 r_c) in
// [0, pi/2): the Taylor series of cos to theta^14 in Horner form (truncation
// below theta^16 / 16! < 7e-11), squared.
__device__ __forceinline__ float cutoff_cos2(float theta) {
    const float z = theta * theta;
    float c = -1.0f / 87178291200.0f;
    c = fmaf(c, z, 1.0f / 479001600.0f);
    c = fmaf(c, z, -1.0f / 3628800.0f);
    c = fmaf(c, z, 1.0f / 40320.0f);
    c = fmaf(c, z, -1.0f / 720.0f);
    c = fmaf(c, z, 1.0f / 24.0f);
    c = fmaf(c, z, -0.5f);
    c = fmaf(c, z, 1.0f);
    return c * c;
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): one instruction applies the
// same operation to a lane's two radial indices.
__device__ __forceinline__ float2 bc2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
// 2^x per component on the SFU (x <= 0 here)
__device__ __forceinline__ float2 exp2_sfu(float2 x) {
    float2 y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y.x) : "f"(x.x));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y.y) : "f"(x.y));
    return y;
}

// Row splitting for small systems (SPLIT): a centre's row is walked by S
// adjacent slots of one warp (part p takes entries p, p + S, ...), whose
// partial sums are then added in a fixed butterfly over the slots' lanes, so a
// system with too few atoms to fill the GPU still does.  S is a power of two
// with S * LPE <= 32 (N_phi = 8 only); S = 1 is the plain one-slot walk.
template <class T>
__device__ __forceinline__ T parts_sum(T v, int lpe, int S) {
    for (int off = lpe; off < lpe * S; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <int NP>
struct Lanes {
    static constexpr int LPE = NP / 2;
    static constexpr int CPW = 32 / LPE;        // centres per warp
    static constexpr int USED = CPW * LPE;
    static constexpr int CPB = 4 * CPW;         // centres per 128-thread block
};

// ACC64: the fp32-accurate paths form the orbital products c phi Y and
// accumulate A in fp64 (phi itself stays fp32), form rho - shift in fp64, and
// take the Gaussian centres and the cutoff factor as fp32 pairs with r's
// rounding residual: on the stiff gas workload the fp32 rounding of these
// products and sums left a force error of 1.1e-4 eV/A against the oracle, 8e-5
// with them, at 1.4-1.5x the kernel time.  The bf16-network path, whose force
// tolerance is 5e-3 eV/A, keeps the plain fp32 forms.
template <bool ACC64>
using acc_t = typename std::conditional<ACC64, double, float>::type;

template <int NP, bool ACC64, bool SPLIT>
__global__ void __launch_bounds__(128) k_density_fwd(int n, const int *__restrict__ row,
                                                     const int *__restrict__ act_cnt, const int *__restrict__ act_col,
                                                     const float4 *__restrict__ act_geo, const float4 *__restrict__ pos,
                                                     const float *__restrict__ coef, const float *__restrict__ C0,
                                                     int ne, float *__restrict__ A_out, float *__restrict__ rho_out,
                                                     const float *__restrict__ shift, const float *__restrict__ act_dr,
                                                     EdgeParams P, int S) {
    using Ln = Lanes<NP>;
    constexpr int D = 3 * NP, NA = NP * NT, LPE = Ln::LPE;
    __shared__ __align__(16) float sC0[MAX_ELEMENTS * D];
    for (int k = threadIdx.x; k < ne * D; k += blockDim.x) sC0[k] = C0[k];
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = lane / LPE, sub = lane % LPE;
    const int gs = blockIdx.x * Ln::CPB + warp * Ln::CPW + slot;
    const int i = SPLIT ? gs / S : gs, part = SPLIT ? gs - i * S : 0, stride = SPLIT ? S : 1;
    const bool live = lane < Ln::USED && i < n;
    if (!SPLIT && !live) return;   // split rows: every lane takes part in the parts' sum
    const int n0 = 2 * sub;

    using R = acc_t<ACC64>;
    R acc[2][NT];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int u = 0; u < NT; ++u) acc[m][u] = R(0);
    const float mh[2] = {P.mu_hi[n0], P.mu_hi[n0 + 1]};
    const int q0 = live ? row[i] + part : 0, q1 = live ? checked_end(row[i] + act_cnt[i], P.n_list, P.status) : 0;
    int j_next = q0 < q1 ? (int)checked(act_col[q0], P.n_rows, P.status) : 0;
    float4 g_next = q0 < q1 ? act_geo[q0] : make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (!ACC64) {
        // fp32 sums: the lane's two radial indices as packed pairs (m = 0, m = 1)
        float2 acc2[NT];
#pragma unroll
        for (int u = 0; u < NT; ++u) acc2[u] = bc2(0.f);
        const float2 NMU = make_float2(-mh[0], -mh[1]);
        for (int q = q0; q < q1; q += stride) {
            const int j = j_next;
            const float4 g = g_next;
            if (q + stride < q1) {
                j_next = (int)checked(act_col[q + stride], P.n_rows, P.status);
                g_next = act_geo[q + stride];
            }
            const float r = g.w;
            const float fc = cutoff_cos2(r * P.th_hi);
            const float *cj = coef ? coef + (int64_t)j * D : sC0 + (ne > 1 ? __float_as_int(pos[j].w) * D : 0);
            float2 C[3];
#pragma unroll
            for (int l = 0; l < 3; ++l) C[l] = *reinterpret_cast<const float2 *>(cj + l * NP + n0);
            const float2 t = add2(bc2(r), NMU);
            const float2 e = mul2(mul2(t, t), bc2(-P.alpha));
            const float2 phi = mul2(make_float2(expf(e.x), expf(e.y)), bc2(fc));
            const float2 a0 = mul2(C[0], phi), a1 = mul2(C[1], phi), a2 = mul2(C[2], phi);
            const float2 DX = bc2(g.x), DY = bc2(g.y), DZ = bc2(g.z);
            acc2[0] = add2(acc2[0], a0);
            acc2[1] = fma2(a1, DX, acc2[1]);
            acc2[2] = fma2(a1, DY, acc2[2]);
            acc2[3] = fma2(a1, DZ, acc2[3]);
            acc2[4] = fma2(a2, mul2(DX, DX), acc2[4]);
            acc2[5] = fma2(a2, mul2(DY, DY), acc2[5]);
            acc2[6] = fma2(a2, mul2(DZ, DZ), acc2[6]);
            acc2[7] = fma2(a2, mul2(DX, DY), acc2[7]);
            acc2[8] = fma2(a2, mul2(DX, DZ), acc2[8]);
            acc2[9] = fma2(a2, mul2(DY, DZ), acc2[9]);
        }
#pragma unroll
        for (int u = 0; u < NT; ++u) {
            acc[0][u] = acc2[u].x;
            acc[1][u] = acc2[u].y;
        }
    } else {
        const float ml[2] = {P.mu_lo[n0], P.mu_lo[n0 + 1]};
        float dr_next = act_dr && q0 < q1 ? act_dr[q0] : 0.f;
        for (int q = q0; q < q1; q += stride) {
            // the next edge's index and geometry are in flight while this one computes
            const int j = j_next;
            const float4 g = g_next;         // dx, dy, dz, r
            const float dr = dr_next;        // r - fp32(r)
            if (q + stride < q1) {
                j_next = (int)checked(act_col[q + stride], P.n_rows, P.status);
                g_next = act_geo[q + stride];
                if (act_dr) dr_next = act_dr[q + stride];
            }
            const float r = g.w;
            const float fc = cutoff_cos2(fmaf(r, P.th_hi, r * P.th_lo));
            // first layer: c^0 by element (no lookup with a single element)
            const float *cj = coef ? coef + (int64_t)j * D : sC0 + (ne > 1 ? __float_as_int(pos[j].w) * D : 0);
            float c[3][2];
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                const float2 v = *reinterpret_cast<const float2 *>(cj + l * NP + n0);
                c[l][0] = v.x;
                c[l][1] = v.y;
            }
            const R gx = g.x, gy = g.y, gz = g.z;
            const R Y[NT] = {R(1), gx, gy, gz, gx * gx, gy * gy, gz * gz, gx * gy, gx * gz, gy * gz};
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                // the Gaussians' slope 2 alpha t makes them the part of the density most
                // sensitive to r: t takes the centres' second fp32 halves and r's
                // rounding residual
                const float t = ((r - mh[m]) - ml[m]) + dr;
                const float phi = expf(-P.alpha * t * t) * fc;
                const R a0 = R(c[0][m]) * phi, a1 = R(c[1][m]) * phi, a2 = R(c[2][m]) * phi;
                acc[m][0] += a0;
#pragma unroll
                for (int u = 1; u < 4; ++u) acc[m][u] = fma(a1, Y[u], acc[m][u]);
#pragma unroll
                for (int u = 4; u < NT; ++u) acc[m][u] = fma(a2, Y[u], acc[m][u]);
            }
        }
    }
    if (SPLIT) {
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int u = 0; u < NT; ++u) acc[m][u] = parts_sum(acc[m][u], LPE, S);
        if (!live || part != 0) return;
    }
    float *Ao = A_out + (int64_t)i * NA;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int nn = n0 + m;
        const R *v = acc[m];
#pragma unroll
        for (int u = 0; u < NT; u += 2)
            *reinterpret_cast<float2 *>(Ao + nn * NT + u) = make_float2((float)v[u], (float)v[u + 1]);
        if (!rho_out) continue;   // pair form: rho from A in k_rho_pair
        // rho - shift in fp64 (the networks see (rho - shift) / scale, which the
        // fp32 rounding of rho itself would blur when rho is close to its shift)
        // (on the bf16-network path in fp32)
        float *ro = rho_out + (int64_t)i * D;
        const float *sh = shift + (ne > 1 ? __float_as_int(pos[i].w) : 0) * D;
        R x[NT];
#pragma unroll
        for (int u = 0; u < NT; ++u) x[u] = ACC64 ? v[u] : R((float)v[u]);
        ro[nn] = (float)(x[0] * x[0] - (R)sh[nn]);
        ro[NP + nn] = (float)(x[1] * x[1] + x[2] * x[2] + x[3] * x[3] - (R)sh[NP + nn]);
        ro[2 * NP + nn] = (float)(x[4] * x[4] + x[5] * x[5] + x[6] * x[6] + R(2) * (x[7] * x[7] + x[8] * x[8] + x[9] * x[9]) -
                                  (R)sh[2 * NP + nn]);
    }
}

// backward: same slots and lanes.  Lane `sub` keeps G_k and c_k of its two
// radial indices in registers and reads the neighbour's 20 interleaved dE/dA
// values (radial-major lane order) as five float4 (the slot's four lanes read
// 64 contiguous bytes per load).  dE/dc_k of the lane's radial indices needs no reduction; the force
// is summed over the slot's lanes in a fixed order.
template <int NP, bool HAS_DC, bool SPLIT>
__global__ void __launch_bounds__(128, 6) k_edge_bwd(int n, const int *__restrict__ row,
                                                  const int *__restrict__ act_cnt, const int *__restrict__ act_col,
                                                  const float4 *__restrict__ act_geo, const float4 *__restrict__ pos,
                                                  const float *__restrict__ coef, const float *__restrict__ C0, int ne,
                                                  const float *__restrict__ G, float *__restrict__ F,
                                                  float *__restrict__ dc, bool accumulate, EdgeParams P, int S) {
    static_assert(!g_pairs(NP, HAS_DC ? 1 : 0), "scalar backward reads the radial-major lane order");
    using Ln = Lanes<NP>;
    constexpr int D = 3 * NP, NA = NP * NT, LPE = Ln::LPE;
    __shared__ __align__(16) float sC0[MAX_ELEMENTS * D];
    for (int k = threadIdx.x; k < ne * D; k += blockDim.x) sC0[k] = C0[k];
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = lane / LPE, sub = lane % LPE;
    const int gs = blockIdx.x * Ln::CPB + warp * Ln::CPW + slot;
    const int i = SPLIT ? gs / S : gs, part = SPLIT ? gs - i * S : 0, stride = SPLIT ? S : 1;
    const bool live = lane < Ln::USED && i < n;
    const int n0 = 2 * sub;

    float fx = 0.f, fy = 0.f, fz = 0.f;
    float dck[2][3] = {{0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}};
    if (live) {
        float gk[2 * NT], ck[3][2];
        {
            const float4 *g4 = reinterpret_cast<const float4 *>(G + (int64_t)i * NA);
#pragma unroll
            for (int q = 0; q < 5; ++q) {
                const float4 v = g4[q * LPE + sub];
                gk[4 * q] = v.x; gk[4 * q + 1] = v.y; gk[4 * q + 2] = v.z; gk[4 * q + 3] = v.w;
            }
            const float *cp = coef ? coef + (int64_t)i * D : sC0 + __float_as_int(pos[i].w) * D;
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                const float2 v = *reinterpret_cast<const float2 *>(cp + l * NP + n0);
                ck[l][0] = v.x;
                ck[l][1] = v.y;
            }
        }
        // the backward takes the constants' fp32 values: its rounding shifts forces by
        // ~1e-6 eV/A, and the fp32 pairs cost 8 % of its time
        const float mh[2] = {P.mu_hi[n0], P.mu_hi[n0 + 1]};
        const int q0 = row[i] + part, q1 = checked_end(row[i] + act_cnt[i], P.n_list, P.status);
        // the edge list takes ordinary cached loads: its 16-byte entries share
        // 32-byte sectors with the next edge's, and evict-first loads made the
        // second read of a sector go back to DRAM (1.6x the traffic, no faster)
        int j_next = q0 < q1 ? (int)checked(__ldg(act_col + q0), P.n_rows, P.status) : 0;
        float4 geo_next = q0 < q1 ? __ldg(act_geo + q0) : make_float4(0.f, 0.f, 0.f, 1.f);
        for (int q = q0; q < q1; q += stride) {
            // the next edge's index and geometry are in flight while this one computes
            const int j = j_next;
            const float4 geo = geo_next;
            if (q + stride < q1) {
                j_next = (int)checked(__ldg(act_col + q + stride), P.n_rows, P.status);
                geo_next = __ldg(act_geo + q + stride);
            }
            const float3 d = make_float3(geo.x, geo.y, geo.z);
            const float r = geo.w;
            const float inv_r = __fdividef(1.0f, r);
            float sn, cs;
            __sincosf(r * (2.f * P.th_hi), &sn, &cs);   // 2 theta in [0, pi)
            const float fc = 0.5f * (cs + 1.0f);
            const float dfc = -P.th_hi * sn;
            float gj[2 * NT], cj[3][2];
            {
                const float4 *g4 = reinterpret_cast<const float4 *>(G + (int64_t)j * NA);
#pragma unroll
                for (int q2 = 0; q2 < 5; ++q2) {
                    const float4 v = __ldg(g4 + q2 * LPE + sub);
                    gj[4 * q2] = v.x; gj[4 * q2 + 1] = v.y; gj[4 * q2 + 2] = v.z; gj[4 * q2 + 3] = v.w;
                }
                if (!HAS_DC && ne == 1) {
                    // first layer, one element: every atom carries the same c^0
#pragma unroll
                    for (int l = 0; l < 3; ++l) {
                        cj[l][0] = ck[l][0];
                        cj[l][1] = ck[l][1];
                    }
                } else {
                    const float *cp = coef ? coef + (int64_t)j * D : sC0 + __float_as_int(pos[j].w) * D;
#pragma unroll
                    for (int l = 0; l < 3; ++l) {
                        const float2 v = *reinterpret_cast<const float2 *>(cp + l * NP + n0);
                        cj[l][0] = v.x;
                        cj[l][1] = v.y;
                    }
                }
            }
            const float xx = d.x * d.x, yy = d.y * d.y, zz = d.z * d.z;
            const float xy = d.x * d.y, xz = d.x * d.z, yz = d.y * d.z;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const float t = r - mh[m];
                const float g = __expf(-P.alpha * t * t);
                const float phi = g * fc;
                const float dphi = g * (-2.0f * P.alpha * t * fc + dfc);
                const float *a = &gk[m * NT];
                const float *b = &gj[m * NT];
                const float c0j = cj[0][m], c1j = cj[1][m], c2j = cj[2][m];
                const float c0k = ck[0][m], c1k = ck[1][m], c2k = ck[2][m];
                // l = 0 (parity +), l = 1 (parity -), l = 2 (parity +)
                const float H0 = a[0] * c0j + b[0] * c0k;
                const float Hx = a[1] * c1j - b[1] * c1k;
                const float Hy = a[2] * c1j - b[2] * c1k;
                const float Hz = a[3] * c1j - b[3] * c1k;
                const float Hxx = a[4] * c2j + b[4] * c2k;
                const float Hyy = a[5] * c2j + b[5] * c2k;
                const float Hzz = a[6] * c2j + b[6] * c2k;
                const float Hxy = a[7] * c2j + b[7] * c2k;
                const float Hxz = a[8] * c2j + b[8] * c2k;
                const float Hyz = a[9] * c2j + b[9] * c2k;
                const float Pv = H0 + Hx * d.x + Hy * d.y + Hz * d.z + Hxx * xx + Hyy * yy + Hzz * zz + Hxy * xy +
                                 Hxz * xz + Hyz * yz;
                const float Qx = Hx + 2.f * Hxx * d.x + Hxy * d.y + Hxz * d.z;
                const float Qy = Hy + 2.f * Hyy * d.y + Hxy * d.x + Hyz * d.z;
                const float Qz = Hz + 2.f * Hzz * d.z + Hxz * d.x + Hyz * d.y;
                const float s = dphi * Pv * inv_r;
                fx += s * d.x + phi * Qx;
                fy += s * d.y + phi * Qy;
                fz += s * d.z + phi * Qz;
                if (HAS_DC) {
                    const float S1 = b[1] * d.x + b[2] * d.y + b[3] * d.z;
                    const float S2 = b[4] * xx + b[5] * yy + b[6] * zz + b[7] * xy + b[8] * xz + b[9] * yz;
                    dck[m][0] += phi * b[0];
                    dck[m][1] -= phi * S1;
                    dck[m][2] += phi * S2;
                }
            }
        }
    }
    if (SPLIT) {
        fx = parts_sum(fx, LPE, S);
        fy = parts_sum(fy, LPE, S);
        fz = parts_sum(fz, LPE, S);
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int l = 0; l < 3; ++l) dck[m][l] = parts_sum(dck[m][l], LPE, S);
    }
    // force: sum over the slot's lanes (sub 0 .. LPE-1) in a fixed order
    const int base = (lane / LPE) * LPE;
    float sx = 0.f, sy = 0.f, sz = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < LPE; ++s2) {
        const int src = base + s2 < 32 ? base + s2 : lane;
        sx += __shfl_sync(0xffffffffu, fx, src);
        sy += __shfl_sync(0xffffffffu, fy, src);
        sz += __shfl_sync(0xffffffffu, fz, src);
    }
    if (!live || part != 0) return;
    if (sub == 0) {
        float *Fo = F + 3 * (int64_t)i;
        if (accumulate) {
            sx += Fo[0];
            sy += Fo[1];
            sz += Fo[2];
        }
        Fo[0] = sx;
        Fo[1] = sy;
        Fo[2] = sz;
    }
    if (HAS_DC) {
        float *o = dc + (int64_t)i * D;
#pragma unroll
        for (int l = 0; l < 3; ++l) *reinterpret_cast<float2 *>(o + l * NP + n0) = make_float2(dck[0][l], dck[1][l]);
    }
}

// Packed form of the backward pass for rows in the pair lane order: each
// float4 of a dE/dA row holds two tuples' (m = 0, m = 1) pairs, and the
// per-edge arithmetic runs on those pairs with packed fp32 instructions
// (sm_100 f32x2), half the instructions of the scalar form.  With the
// coefficient gradient at N_phi = 8 the pairs' extra live registers spill at
// the 80 registers that six blocks per SM allow and the scalar form above is
// faster (1M-atom Ag: first layer 1.96 -> 1.66 ms packed, later layers 2.16
// -> 2.41 ms, 2.71 ms at five blocks per SM without spills); for N_phi = 10 the
// packed form is faster in every layer (108k atoms: 0.49 -> 0.45 ms, and 0.40
// ms at five blocks per SM, where its 96 registers do not spill; first layer
// 0.33 -> 0.29 ms at six).
template <int NP, bool HAS_DC, bool SPLIT>
__global__ void __launch_bounds__(128, (NP == 10 && HAS_DC) ? 5 : 6)
    k_edge_bwd_pk(int n, const int *__restrict__ row, const int *__restrict__ act_cnt, const int *__restrict__ act_col,
                  const float4 *__restrict__ act_geo, const float4 *__restrict__ pos, const float *__restrict__ coef,
                  const float *__restrict__ C0, int ne, const float *__restrict__ G, float *__restrict__ F,
                  float *__restrict__ dc, bool accumulate, EdgeParams P, int S) {
    static_assert(g_pairs(NP, HAS_DC ? 1 : 0), "packed backward reads the pair lane order");
    using Ln = Lanes<NP>;
    constexpr int D = 3 * NP, NA = NP * NT, LPE = Ln::LPE;
    __shared__ __align__(16) float sC0[MAX_ELEMENTS * D];
    for (int k = threadIdx.x; k < ne * D; k += blockDim.x) sC0[k] = C0[k];
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = lane / LPE, sub = lane % LPE;
    const int gs = blockIdx.x * Ln::CPB + warp * Ln::CPW + slot;
    const int i = SPLIT ? gs / S : gs, part = SPLIT ? gs - i * S : 0, stride = SPLIT ? S : 1;
    const bool live = lane < Ln::USED && i < n;
    const int n0 = 2 * sub;

    // force and dE/dc_k partials as (m = 0, m = 1) pairs
    float2 fx = bc2(0.f), fy = bc2(0.f), fz = bc2(0.f);
    // dE/dc_k: sum phi G_j Y per l (l = 1 without its sign)
    float2 dck[3] = {bc2(0.f), bc2(0.f), bc2(0.f)};
    if (live) {
        // gk[2 tau + m]: dE/dA of the centre for radial index n0 + m;
        // ck[l]: its coefficients (n0, n0 + 1), l = 1 held with its parity sign
        float gk[2 * NT];
        float2 ck[3];
        {
            const float4 *g4 = reinterpret_cast<const float4 *>(G + (int64_t)i * NA);
#pragma unroll
            for (int q = 0; q < 5; ++q) {
                const float4 v = g4[q * LPE + sub];
                gk[4 * q] = v.x; gk[4 * q + 1] = v.y; gk[4 * q + 2] = v.z; gk[4 * q + 3] = v.w;
            }
            const float *cp = coef ? coef + (int64_t)i * D : sC0 + __float_as_int(pos[i].w) * D;
#pragma unroll
            for (int l = 0; l < 3; ++l) ck[l] = *reinterpret_cast<const float2 *>(cp + l * NP + n0);
            ck[1] = make_float2(-ck[1].x, -ck[1].y);
        }
        // the backward takes the constants' fp32 values: its rounding shifts forces by
        // ~1e-6 eV/A, and the fp32 pairs cost 8 % of its time
        const float2 nmu = make_float2(-P.mu_hi[n0], -P.mu_hi[n0 + 1]);
        const int q0 = row[i] + part, q1 = checked_end(row[i] + act_cnt[i], P.n_list, P.status);
        // the edge list takes ordinary cached loads: its 16-byte entries share
        // 32-byte sectors with the next edge's, and evict-first loads made the
        // second read of a sector go back to DRAM (1.6x the traffic, no faster)
        int j_next = q0 < q1 ? (int)checked(__ldg(act_col + q0), P.n_rows, P.status) : 0;
        float4 geo_next = q0 < q1 ? __ldg(act_geo + q0) : make_float4(0.f, 0.f, 0.f, 1.f);
        for (int q = q0; q < q1; q += stride) {
            // the next edge's index and geometry are in flight while this one computes
            const int j = j_next;
            const float4 geo = geo_next;
            if (q + stride < q1) {
                j_next = (int)checked(__ldg(act_col + q + stride), P.n_rows, P.status);
                geo_next = __ldg(act_geo + q + stride);
            }
            const float r = geo.w;
            const float inv_r = __fdividef(1.0f, r);
            float sn, cs;
            __sincosf(r * (2.f * P.th_hi), &sn, &cs);   // 2 theta in [0, pi)
            const float fc = 0.5f * (cs + 1.0f);
            const float dfc = -P.th_hi * sn;
            float gj[2 * NT];
            float2 cj[3];
            {
                const float4 *g4 = reinterpret_cast<const float4 *>(G + (int64_t)j * NA);
#pragma unroll
                for (int q2 = 0; q2 < 5; ++q2) {
                    const float4 v = __ldg(g4 + q2 * LPE + sub);
                    gj[4 * q2] = v.x; gj[4 * q2 + 1] = v.y; gj[4 * q2 + 2] = v.z; gj[4 * q2 + 3] = v.w;
                }
                if (!HAS_DC && ne == 1) {
                    // first layer, one element: every atom carries the same c^0
                    cj[0] = ck[0];
                    cj[1] = make_float2(-ck[1].x, -ck[1].y);
                    cj[2] = ck[2];
                } else {
                    const float *cp = coef ? coef + (int64_t)j * D : sC0 + __float_as_int(pos[j].w) * D;
#pragma unroll
                    for (int l = 0; l < 3; ++l) cj[l] = *reinterpret_cast<const float2 *>(cp + l * NP + n0);
                }
            }
            // phi_n = g_n fc and phi_n' / r = g_n (-2 alpha t_n fc + fc') / r, t_n = r - mu_n;
            // H_tau = G_k c_j + (-1)^l G_j c_k, folded tuple by tuple into
            //   Pv = sum_tau H_tau Y_tau and Q = sum_tau H_tau grad Y_tau,
            // and (layers >= 1) S_l = sum_{|tau|=l} G_j Y_tau
#define GK2(u) make_float2(gk[2 * (u)], gk[2 * (u) + 1])
#define GJ2(u) make_float2(gj[2 * (u)], gj[2 * (u) + 1])
            const float2 DX = bc2(geo.x), DY = bc2(geo.y), DZ = bc2(geo.z);
            const float2 t = add2(bc2(r), nmu);
            const float2 g = exp2_sfu(mul2(mul2(t, t), bc2(P.neg_alpha_log2e)));
            const float2 phi = mul2(g, bc2(fc));
            const float2 dphir = mul2(g, fma2(t, bc2(-2.0f * P.alpha * fc * inv_r), bc2(dfc * inv_r)));
            float2 Pv, Qx, Qy, Qz, S1, S2, Y2, H;
            Pv = fma2(GK2(0), cj[0], mul2(GJ2(0), ck[0]));
            Qx = fma2(GK2(1), cj[1], mul2(GJ2(1), ck[1]));
            Pv = fma2(Qx, DX, Pv);
            Qy = fma2(GK2(2), cj[1], mul2(GJ2(2), ck[1]));
            Pv = fma2(Qy, DY, Pv);
            Qz = fma2(GK2(3), cj[1], mul2(GJ2(3), ck[1]));
            Pv = fma2(Qz, DZ, Pv);
            if (HAS_DC) S1 = fma2(GJ2(3), DZ, fma2(GJ2(2), DY, mul2(GJ2(1), DX)));
            Y2 = mul2(DX, DX);
            H = fma2(GK2(4), cj[2], mul2(GJ2(4), ck[2]));
            Pv = fma2(H, Y2, Pv);
            Qx = fma2(H, add2(DX, DX), Qx);
            if (HAS_DC) S2 = mul2(GJ2(4), Y2);
            Y2 = mul2(DY, DY);
            H = fma2(GK2(5), cj[2], mul2(GJ2(5), ck[2]));
            Pv = fma2(H, Y2, Pv);
            Qy = fma2(H, add2(DY, DY), Qy);
            if (HAS_DC) S2 = fma2(GJ2(5), Y2, S2);
            Y2 = mul2(DZ, DZ);
            H = fma2(GK2(6), cj[2], mul2(GJ2(6), ck[2]));
            Pv = fma2(H, Y2, Pv);
            Qz = fma2(H, add2(DZ, DZ), Qz);
            if (HAS_DC) S2 = fma2(GJ2(6), Y2, S2);
            Y2 = mul2(DX, DY);
            H = fma2(GK2(7), cj[2], mul2(GJ2(7), ck[2]));
            Pv = fma2(H, Y2, Pv);
            Qx = fma2(H, DY, Qx);
            Qy = fma2(H, DX, Qy);
            if (HAS_DC) S2 = fma2(GJ2(7), Y2, S2);
            Y2 = mul2(DX, DZ);
            H = fma2(GK2(8), cj[2], mul2(GJ2(8), ck[2]));
            Pv = fma2(H, Y2, Pv);
            Qx = fma2(H, DZ, Qx);
            Qz = fma2(H, DX, Qz);
            if (HAS_DC) S2 = fma2(GJ2(8), Y2, S2);
            Y2 = mul2(DY, DZ);
            H = fma2(GK2(9), cj[2], mul2(GJ2(9), ck[2]));
            Pv = fma2(H, Y2, Pv);
            Qy = fma2(H, DZ, Qy);
            Qz = fma2(H, DY, Qz);
            if (HAS_DC) S2 = fma2(GJ2(9), Y2, S2);
            const float2 sv = mul2(dphir, Pv);
            fx = fma2(sv, DX, fma2(phi, Qx, fx));
            fy = fma2(sv, DY, fma2(phi, Qy, fy));
            fz = fma2(sv, DZ, fma2(phi, Qz, fz));
            if (HAS_DC) {
                dck[0] = fma2(phi, GJ2(0), dck[0]);
                dck[1] = fma2(phi, S1, dck[1]);
                dck[2] = fma2(phi, S2, dck[2]);
            }
#undef GK2
#undef GJ2
        }
    }
    // force: the lane's pair, then (split rows) the parts, then the slot's lanes
    // (sub 0 .. LPE-1), in a fixed order
    float lx = fx.x + fx.y, ly = fy.x + fy.y, lz = fz.x + fz.y;
    if (SPLIT) {
        lx = parts_sum(lx, LPE, S);
        ly = parts_sum(ly, LPE, S);
        lz = parts_sum(lz, LPE, S);
#pragma unroll
        for (int l = 0; l < 3; ++l) dck[l] = make_float2(parts_sum(dck[l].x, LPE, S), parts_sum(dck[l].y, LPE, S));
    }
    const int base = (lane / LPE) * LPE;
    float sx = 0.f, sy = 0.f, sz = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < LPE; ++s2) {
        const int src = base + s2 < 32 ? base + s2 : lane;
        sx += __shfl_sync(0xffffffffu, lx, src);
        sy += __shfl_sync(0xffffffffu, ly, src);
        sz += __shfl_sync(0xffffffffu, lz, src);
    }
    if (!live || part != 0) return;
    if (sub == 0) {
        float *Fo = F + 3 * (int64_t)i;
        if (accumulate) {
            sx += Fo[0];
            sy += Fo[1];
            sz += Fo[2];
        }
        Fo[0] = sx;
        Fo[1] = sy;
        Fo[2] = sz;
    }
    if (HAS_DC) {
        float *o = dc + (int64_t)i * D;
        *reinterpret_cast<float2 *>(o + n0) = dck[0];
        *reinterpret_cast<float2 *>(o + NP + n0) = make_float2(-dck[1].x, -dck[1].y);
        *reinterpret_cast<float2 *>(o + 2 * NP + n0) = dck[2];
    }
}

// ---------------------------------------------------------------------------
// Pair-product densities (density_form = 1): rho_(n,m,l) = sum_{|tau|=l}
// l!/tau! A_{n,tau} A_{m,tau} for n <= m, at index l P + pair(n, m) with
// P = N_phi (N_phi+1)/2 and pair(n, m) = n N_phi - n (n-1)/2 + (m - n); the
// density dimension N_phi (N_phi+1)(L+1)/2 of section "REANN Architecture".
// One thread per (atom, pair); the atom's A row is read from L1.
template <int NP>
__global__ void __launch_bounds__(256) k_rho_pair(int n, const float *__restrict__ A, float *__restrict__ rho,
                                                  const float4 *__restrict__ pos, const float *__restrict__ shift,
                                                  int ne) {
    constexpr int P = NP * (NP + 1) / 2, NA = NP * NT, DR = 3 * P;
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= (int64_t)n * P) return;
    const int64_t i = k / P;
    const int p = (int)(k - i * P);
    int a = 0, first = 0;
    while (first + (NP - a) <= p) {   // row a of the upper triangle holds pairs (a, a..NP-1)
        first += NP - a;
        ++a;
    }
    const int b = a + (p - first);
    const float *x = A + i * NA + a * NT, *y = A + i * NA + b * NT;
    float *ro = rho + i * DR;
    const float *sh = shift + (ne > 1 ? __float_as_int(pos[i].w) : 0) * DR;
    double q[NT];
#pragma unroll
    for (int u = 0; u < NT; ++u) q[u] = (double)x[u] * (double)y[u];
    // rho - shift in fp64, as in the square form
    ro[p] = (float)(q[0] - (double)sh[p]);
    ro[P + p] = (float)(q[1] + q[2] + q[3] - (double)sh[P + p]);
    ro[2 * P + p] = (float)(q[4] + q[5] + q[6] + 2.0 * (q[7] + q[8] + q[9]) - (double)sh[2 * P + p]);
}

// ---------------------------------------------------------------------------
// host wrappers

// parts per centre row (row splitting): 1 unless the centres alone would give
// fewer than four 128-thread blocks per SM (N_phi = 8 only)
static int edge_parts(const reann_ctx *c, int64_t centres) {
    if (c->NP != 8) return 1;
    int S = 1;
    while (S < 8 && (centres * S + Lanes<8>::CPB - 1) / Lanes<8>::CPB < 4 * (int64_t)c->sm_count) S *= 2;
    return S;
}

cudaError_t launch_density_fwd(reann_ctx *c, int t, cudaStream_t s) {
    const int64_t nc = centres(c);
    if (nc == 0) return cudaSuccess;
    EdgeParams P = make_edge_params(c);
    const float *coef = t == 0 ? nullptr : c->d_coef + (int64_t)t * c->n_slots * c->D;
    float *A = c->d_A + (int64_t)t * c->n * c->NA;
    const bool pair = c->cfg.density_form == 1;
    float *rho = pair ? nullptr : c->d_rho + (int64_t)t * c->n * c->D;
    const float *shift = c->d_shift + (int64_t)t * c->ne * c->DR;
    const bool acc64 = c->cfg.mlp_precision != 1;   // the fp32-accurate paths
    const int S = edge_parts(c, nc);
    REANN_TIMED(c, REANN_K_DENSITY, s, pair ? 2 : 1);
    if (pair && c->NP != 8) return cudaErrorInvalidValue;
#define REANN_DENSITY(NPV, ACC, SPL, RHO)                                                                        \
    k_density_fwd<NPV, ACC, SPL><<<(unsigned)((nc * S + Lanes<NPV>::CPB - 1) / Lanes<NPV>::CPB), 128, 0, s>>>(     \
        (int)nc, c->d_row, c->d_act_cnt, c->d_act_col, c->d_act_geo, c->d_pos, coef, c->d_w, c->ne, A, RHO, shift,    \
        c->d_act_dr, P, S)
    if (c->NP == 8) {
        if (S > 1) {
            if (acc64) REANN_DENSITY(8, true, true, rho); else REANN_DENSITY(8, false, true, rho);
        } else {
            if (acc64) REANN_DENSITY(8, true, false, rho); else REANN_DENSITY(8, false, false, rho);
        }
    } else if (c->NP == 10) {
        if (acc64) REANN_DENSITY(10, true, false, rho); else REANN_DENSITY(10, false, false, rho);
    } else {
        return cudaErrorInvalidValue;
    }
#undef REANN_DENSITY
    if (pair) {
        // rho from A in k_rho_pair (the density pass wrote A only)
        const int64_t threads = nc * (8 * 9 / 2);
        k_rho_pair<8><<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
            (int)nc, A, c->d_rho + (int64_t)t * c->n * c->DR, c->d_pos, shift, c->ne);
    }
    return cudaGetLastError();
}

cudaError_t launch_edge_bwd(reann_ctx *c, int t, bool accumulate, cudaStream_t s) {
    if (c->n == 0) return cudaSuccess;
    EdgeParams P = make_edge_params(c);
    const float *coef = t == 0 ? nullptr : c->d_coef + (int64_t)t * c->n_slots * c->D;
    const bool has_dc = t >= 1;
    const int S = edge_parts(c, c->n);
    REANN_TIMED(c, REANN_K_EDGE_BWD, s);
#define REANN_EDGE_BWD(K, NPV, DC, SPL)                                                                          \
    K<NPV, DC, SPL><<<(unsigned)((c->n * S + Lanes<NPV>::CPB - 1) / Lanes<NPV>::CPB), 128, 0, s>>>(                 \
        (int)c->n, c->d_row, c->d_act_cnt, c->d_act_col, c->d_act_geo, c->d_pos, coef, c->d_w, c->ne, c->d_G, c->d_F, \
        c->d_dc, accumulate, P, S)
    // the kernel reads the lane order the networks wrote for this layer (g_pairs)
    if (c->NP == 8) {
        if (S > 1) {
            if (has_dc) REANN_EDGE_BWD(k_edge_bwd, 8, true, true); else REANN_EDGE_BWD(k_edge_bwd_pk, 8, false, true);
        } else {
            if (has_dc) REANN_EDGE_BWD(k_edge_bwd, 8, true, false); else REANN_EDGE_BWD(k_edge_bwd_pk, 8, false, false);
        }
    } else if (c->NP == 10) {
        if (has_dc) REANN_EDGE_BWD(k_edge_bwd_pk, 10, true, false);
        else REANN_EDGE_BWD(k_edge_bwd_pk, 10, false, false);
    } else {
        return cudaErrorInvalidValue;
    }
#undef REANN_EDGE_BWD
    return cudaGetLastError();
}

}  // namespace reann
