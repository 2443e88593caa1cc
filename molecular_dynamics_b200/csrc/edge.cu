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
// comes from Y_tau(-d) = (-1)^l Y_tau(d).  The per-atom active-pair counts
// of the last evaluation choose the lanes per centre of the backward pass.
//
// Tuple order inside one radial index n: (000); (100)(010)(001);
// (200)(020)(002)(110)(101)(011).  Feature (n, l) sits at index l*N_phi + n.
#include "common.cuh"
#include "kernels.cuh"

namespace reann {

EdgeParams make_edge_params(const reann_ctx *c) {
    EdgeParams P;
    for (int a = 0; a < 3; ++a) {
        P.box[a] = c->box[a];
        P.inv_box[a] = 1.0 / c->box[a];
    }
    P.r_cut = (float)c->cfg.r_cut;
    P.r_cut2 = (float)(c->cfg.r_cut * c->cfg.r_cut);
    P.pi_over_rc = (float)(3.14159265358979323846 / c->cfg.r_cut);
    P.alpha = (float)c->cfg.alpha;
    P.mu_step = (float)(c->cfg.r_cut / (c->cfg.n_radial - 1));
    return P;
}

// Minimum-image displacement x_j - x_i: difference and image shift in fp64
// (so that boundary-crossing pairs keep full precision), rounded to fp32.
__device__ __forceinline__ float3 displacement(float4 pi, float4 pj, const EdgeParams &P) {
    double dx = (double)pj.x - (double)pi.x;
    double dy = (double)pj.y - (double)pi.y;
    double dz = (double)pj.z - (double)pi.z;
    dx -= P.box[0] * rint(dx * P.inv_box[0]);
    dy -= P.box[1] * rint(dy * P.inv_box[1]);
    dz -= P.box[2] * rint(dz * P.inv_box[2]);
    return make_float3((float)dx, (float)dy, (float)dz);
}

// ---------------------------------------------------------------------------
// active pairs: the entries of each row closer than r_cut, compacted to the
// front of the row's slot (same offsets as the full list).
__global__ void __launch_bounds__(128) k_active(int n, const float4 *__restrict__ pos, const int *__restrict__ row,
                                                const int *__restrict__ col, int *__restrict__ act_cnt,
                                                int *__restrict__ act_col, EdgeParams P,
                                                unsigned long long *__restrict__ total) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    int k = 0;
    if (i < n) {
        float4 pi = pos[i];
        int q0 = row[i], q1 = row[i + 1];
        for (int q = q0; q < q1; ++q) {
            int j = col[q];
            float3 d = displacement(pi, pos[j], P);
            float r2 = d.x * d.x + d.y * d.y + d.z * d.z;
            if (r2 < P.r_cut2) act_col[q0 + k++] = j;
        }
        act_cnt[i] = k;
    }
    unsigned long long v = (unsigned long long)k;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0 && v) atomicAdd(total, v);
}

cudaError_t launch_active(reann_ctx *c, cudaStream_t s) {
    if (c->n == 0) return cudaSuccess;
    EdgeParams P = make_edge_params(c);
    cudaError_t e = cudaMemsetAsync(c->d_i64 + 3, 0, sizeof(int64_t), s);
    if (e) return e;
    REANN_TIMED(c, REANN_K_ACTIVE, s);
    k_active<<<(unsigned)((c->n + 127) / 128), 128, 0, s>>>((int)c->n, c->d_pos, c->d_row, c->d_col, c->d_act_cnt,
                                                            c->d_act_col, P, (unsigned long long *)(c->d_i64 + 3));
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// loads of one atom's D coefficients (layer 0: the element table in shared
// memory; later layers: the message vector written by the coefficient network)

template <int D>
__device__ __forceinline__ void load_coef(float (&c)[D], const float *__restrict__ coef, const float *sC0, int j,
                                          int type_j) {
    if (coef) {
        const float *p = coef + (int64_t)j * D;
        if (D % 4 == 0) {
#pragma unroll
            for (int k = 0; k < D / 4; ++k) {
                float4 v = __ldg(reinterpret_cast<const float4 *>(p) + k);
                c[4 * k] = v.x; c[4 * k + 1] = v.y; c[4 * k + 2] = v.z; c[4 * k + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < D / 2; ++k) {
                float2 v = __ldg(reinterpret_cast<const float2 *>(p) + k);
                c[2 * k] = v.x; c[2 * k + 1] = v.y;
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < D; ++k) c[k] = sC0[type_j * D + k];
    }
}

// ---------------------------------------------------------------------------
// forward: one thread per centre atom, A^t accumulated in registers over the
// centre's active neighbours in row order (deterministic), then rho^t.
template <int NP>
__global__ void __launch_bounds__(128) k_density_fwd(int n, const float4 *__restrict__ pos, const int *__restrict__ row,
                                                     const int *__restrict__ act_cnt, const int *__restrict__ act_col,
                                                     const float *__restrict__ coef, const float *__restrict__ C0,
                                                     int ne, float *__restrict__ A_out, float *__restrict__ rho_out,
                                                     EdgeParams P) {
    constexpr int D = 3 * NP, NA = NP * NT;
    __shared__ float sC0[MAX_ELEMENTS * D];
    for (int k = threadIdx.x; k < ne * D; k += blockDim.x) sC0[k] = C0[k];
    __syncthreads();
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;

    float acc[NA];
#pragma unroll
    for (int k = 0; k < NA; ++k) acc[k] = 0.f;
    float4 pi = pos[i];
    int q0 = row[i], cnt = act_cnt[i];
    for (int q = q0; q < q0 + cnt; ++q) {
        int j = act_col[q];
        float4 pj = pos[j];
        float3 d = displacement(pi, pj, P);
        float r = sqrtf(d.x * d.x + d.y * d.y + d.z * d.z);
        float fc = 0.5f * (cospif(r * (1.0f / P.r_cut) ) + 1.0f);
        float c[D];
        load_coef<D>(c, coef, sC0, j, __float_as_int(pj.w));
        const float Y[NT] = {1.f, d.x, d.y, d.z, d.x * d.x, d.y * d.y, d.z * d.z, d.x * d.y, d.x * d.z, d.y * d.z};
#pragma unroll
        for (int nn = 0; nn < NP; ++nn) {
            float t = r - (float)nn * P.mu_step;
            float phi = expf(-P.alpha * t * t) * fc;
            float a0 = c[nn] * phi, a1 = c[NP + nn] * phi, a2 = c[2 * NP + nn] * phi;
            acc[nn * NT + 0] += a0;
#pragma unroll
            for (int u = 1; u < 4; ++u) acc[nn * NT + u] += a1 * Y[u];
#pragma unroll
            for (int u = 4; u < NT; ++u) acc[nn * NT + u] += a2 * Y[u];
        }
    }
    float *Ao = A_out + (int64_t)i * NA;
#pragma unroll
    for (int k = 0; k < NA / 4; ++k)
        reinterpret_cast<float4 *>(Ao)[k] = make_float4(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
    float rho[D];
#pragma unroll
    for (int nn = 0; nn < NP; ++nn) {
        const float *a = &acc[nn * NT];
        rho[nn] = a[0] * a[0];
        rho[NP + nn] = a[1] * a[1] + a[2] * a[2] + a[3] * a[3];
        rho[2 * NP + nn] = a[4] * a[4] + a[5] * a[5] + a[6] * a[6] + 2.f * (a[7] * a[7] + a[8] * a[8] + a[9] * a[9]);
    }
    float *ro = rho_out + (int64_t)i * D;
#pragma unroll
    for (int k = 0; k < D / 2; ++k) reinterpret_cast<float2 *>(ro)[k] = make_float2(rho[2 * k], rho[2 * k + 1]);
}

// ---------------------------------------------------------------------------
// backward: a group of W lanes per centre atom k.  G_k and c_k sit in shared
// memory (read as broadcasts); lane g of the group takes the centre's active
// neighbours g, g + W, ...; the per-lane force and dE/dc_k partials are summed
// by a fixed shuffle tree, so the result is deterministic.
template <int NP, bool HAS_DC, int W>
__global__ void __launch_bounds__(128) k_edge_bwd(int n, const float4 *__restrict__ pos, const int *__restrict__ row,
                                                  const int *__restrict__ act_cnt, const int *__restrict__ act_col,
                                                  const float *__restrict__ coef, const float *__restrict__ C0, int ne,
                                                  const float *__restrict__ G, float *__restrict__ F,
                                                  float *__restrict__ dc, bool accumulate, EdgeParams P) {
    constexpr int D = 3 * NP, NA = NP * NT, GROUPS = 128 / W;
    __shared__ float sC0[MAX_ELEMENTS * D];
    __shared__ float sG[GROUPS][NA];
    __shared__ float sc[GROUPS][D];
    for (int k = threadIdx.x; k < ne * D; k += blockDim.x) sC0[k] = C0[k];
    const int grp = threadIdx.x / W, gl = threadIdx.x % W;
    const int i = blockIdx.x * GROUPS + grp;
    const bool live = i < n;
    float4 pi = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live) {
        pi = pos[i];
        for (int k = gl; k < NA; k += W) sG[grp][k] = G[(int64_t)i * NA + k];
    }
    __syncthreads();
    if (live) {
        if (coef) {
            for (int k = gl; k < D; k += W) sc[grp][k] = coef[(int64_t)i * D + k];
        } else {
            const int ti = __float_as_int(pi.w);
            for (int k = gl; k < D; k += W) sc[grp][k] = sC0[ti * D + k];
        }
    }
    __syncthreads();
    const float *Gk = sG[grp];
    const float *ck = sc[grp];

    float fx = 0.f, fy = 0.f, fz = 0.f;
    float dck[HAS_DC ? D : 1];
#pragma unroll
    for (int k = 0; k < (HAS_DC ? D : 1); ++k) dck[k] = 0.f;

    const int q0 = live ? row[i] : 0, cnt = live ? act_cnt[i] : 0;
    for (int q = q0 + gl; q < q0 + cnt; q += W) {
        const int j = act_col[q];
        const float4 pj = pos[j];
        const float3 d = displacement(pi, pj, P);
        const float r = sqrtf(d.x * d.x + d.y * d.y + d.z * d.z);
        const float inv_r = 1.0f / r;
        float sn, cs;
        sincospif(r * (1.0f / P.r_cut), &sn, &cs);
        const float fc = 0.5f * (cs + 1.0f);
        const float dfc = -0.5f * P.pi_over_rc * sn;
        const float *cjp = coef ? coef + (int64_t)j * D : sC0 + __float_as_int(pj.w) * D;
        const float xx = d.x * d.x, yy = d.y * d.y, zz = d.z * d.z;
        const float xy = d.x * d.y, xz = d.x * d.z, yz = d.y * d.z;
        const float *Gj = G + (int64_t)j * NA;
#pragma unroll
        for (int nn = 0; nn < NP; ++nn) {
            const float t = r - (float)nn * P.mu_step;
            const float g = expf(-P.alpha * t * t);
            const float phi = g * fc;
            const float dphi = g * (-2.0f * P.alpha * t * fc + dfc);
            float gj[NT];
#pragma unroll
            for (int u = 0; u < NT / 2; ++u) {
                const float2 v = __ldg(reinterpret_cast<const float2 *>(Gj + nn * NT) + u);
                gj[2 * u] = v.x;
                gj[2 * u + 1] = v.y;
            }
            const float *gk = &Gk[nn * NT];
            const float c0j = cjp[nn], c1j = cjp[NP + nn], c2j = cjp[2 * NP + nn];
            const float c0k = ck[nn], c1k = ck[NP + nn], c2k = ck[2 * NP + nn];
            // l = 0 (parity +), l = 1 (parity -), l = 2 (parity +)
            const float H0 = gk[0] * c0j + gj[0] * c0k;
            const float Hx = gk[1] * c1j - gj[1] * c1k;
            const float Hy = gk[2] * c1j - gj[2] * c1k;
            const float Hz = gk[3] * c1j - gj[3] * c1k;
            const float Hxx = gk[4] * c2j + gj[4] * c2k;
            const float Hyy = gk[5] * c2j + gj[5] * c2k;
            const float Hzz = gk[6] * c2j + gj[6] * c2k;
            const float Hxy = gk[7] * c2j + gj[7] * c2k;
            const float Hxz = gk[8] * c2j + gj[8] * c2k;
            const float Hyz = gk[9] * c2j + gj[9] * c2k;
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
                const float S0 = gj[0];
                const float S1 = gj[1] * d.x + gj[2] * d.y + gj[3] * d.z;
                const float S2 = gj[4] * xx + gj[5] * yy + gj[6] * zz + gj[7] * xy + gj[8] * xz + gj[9] * yz;
                dck[nn] += phi * S0;
                dck[NP + nn] -= phi * S1;
                dck[2 * NP + nn] += phi * S2;
            }
        }
    }
    // sum over the group's lanes (groups are aligned W-lane segments of a warp)
#pragma unroll
    for (int o = W / 2; o > 0; o >>= 1) {
        fx += __shfl_xor_sync(0xffffffffu, fx, o);
        fy += __shfl_xor_sync(0xffffffffu, fy, o);
        fz += __shfl_xor_sync(0xffffffffu, fz, o);
        if (HAS_DC) {
#pragma unroll
            for (int k = 0; k < D; ++k) dck[k] += __shfl_xor_sync(0xffffffffu, dck[k], o);
        }
    }
    if (live && gl == 0) {
        float *Fo = F + 3 * (int64_t)i;
        if (accumulate) {
            fx += Fo[0];
            fy += Fo[1];
            fz += Fo[2];
        }
        Fo[0] = fx;
        Fo[1] = fy;
        Fo[2] = fz;
        if (HAS_DC) {
            float *o = dc + (int64_t)i * D;
#pragma unroll
            for (int k = 0; k < D / 2; ++k) reinterpret_cast<float2 *>(o)[k] = make_float2(dck[2 * k], dck[2 * k + 1]);
        }
    }
}

// ---------------------------------------------------------------------------
// host wrappers

cudaError_t launch_density_fwd(reann_ctx *c, int t, cudaStream_t s) {
    if (c->n == 0) return cudaSuccess;
    EdgeParams P = make_edge_params(c);
    const float *coef = t == 0 ? nullptr : c->d_coef + (int64_t)t * c->n * c->D;
    float *A = c->d_A + (int64_t)t * c->n * c->NA;
    float *rho = c->d_rho + (int64_t)t * c->n * c->D;
    unsigned g = (unsigned)((c->n + 127) / 128);
    REANN_TIMED(c, REANN_K_DENSITY, s);
    if (c->NP == 8)
        k_density_fwd<8><<<g, 128, 0, s>>>((int)c->n, c->d_pos, c->d_row, c->d_act_cnt, c->d_act_col, coef, c->d_w,
                                           c->ne, A, rho, P);
    else if (c->NP == 10)
        k_density_fwd<10><<<g, 128, 0, s>>>((int)c->n, c->d_pos, c->d_row, c->d_act_cnt, c->d_act_col, coef, c->d_w,
                                            c->ne, A, rho, P);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

// lanes per centre: about a third of the mean active degree, 4..16
static int group_width(const reann_ctx *c) {
    double deg = c->n > 0 ? (double)c->counters.active_pairs / (double)c->n : 0.0;
    if (deg <= 0.0) deg = c->n > 0 ? 0.6 * (double)c->nnz / (double)c->n : 0.0;
    return deg >= 36.0 ? 16 : (deg >= 18.0 ? 8 : 4);
}

template <int NP, bool DC, int W>
static void edge_bwd_launch(reann_ctx *c, const float *coef, bool accumulate, const EdgeParams &P, cudaStream_t s) {
    constexpr int GROUPS = 128 / W;
    unsigned g = (unsigned)((c->n + GROUPS - 1) / GROUPS);
    k_edge_bwd<NP, DC, W><<<g, 128, 0, s>>>((int)c->n, c->d_pos, c->d_row, c->d_act_cnt, c->d_act_col, coef, c->d_w,
                                            c->ne, c->d_G, c->d_F, c->d_dc, accumulate, P);
}

template <int NP, bool DC>
static void edge_bwd_width(reann_ctx *c, const float *coef, bool accumulate, const EdgeParams &P, cudaStream_t s) {
    switch (group_width(c)) {
        case 16: edge_bwd_launch<NP, DC, 16>(c, coef, accumulate, P, s); break;
        case 8: edge_bwd_launch<NP, DC, 8>(c, coef, accumulate, P, s); break;
        default: edge_bwd_launch<NP, DC, 4>(c, coef, accumulate, P, s); break;
    }
}

cudaError_t launch_edge_bwd(reann_ctx *c, int t, bool accumulate, cudaStream_t s) {
    if (c->n == 0) return cudaSuccess;
    EdgeParams P = make_edge_params(c);
    const float *coef = t == 0 ? nullptr : c->d_coef + (int64_t)t * c->n * c->D;
    const bool has_dc = t >= 1;
    REANN_TIMED(c, REANN_K_EDGE_BWD, s);
    if (c->NP == 8) {
        if (has_dc) edge_bwd_width<8, true>(c, coef, accumulate, P, s);
        else edge_bwd_width<8, false>(c, coef, accumulate, P, s);
    } else if (c->NP == 10) {
        if (has_dc) edge_bwd_width<10, true>(c, coef, accumulate, P, s);
        else edge_bwd_width<10, false>(c, coef, accumulate, P, s);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace reann
