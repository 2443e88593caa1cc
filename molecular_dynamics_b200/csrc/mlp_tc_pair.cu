// Tensor-core atomic networks for the pair-product density form
// (density_form = 1, N_phi = 8, L = 2: 108 density features per atom, the
// dimension N_phi (N_phi+1)(L+1)/2 stated in section "REANN Architecture" of
// "Efficient Parallelization of Message Passing Neural Network Potentials for
// Large-Scale Molecular Dynamics").  Same networks, split-bf16 operands and
// fp32 TMEM accumulators as mlp_tc.cu; what differs is the width of the first
// layer (K = 112, the 108 features padded) and of the input-gradient product
// (N = 112), which no longer fit two tiles in flight per SM.  So one 512-thread
// block per SM works on one 128-atom tile at a time: warp w reads TMEM lanes
// 32 (w % 4) .. + 31, and warp group w / 4 takes one 32-column chunk of every
// 128-wide accumulator.
//
// Inputs: the next tile's 108-wide rho rows (432-byte rows, whole 16-byte
// units) are copied into the input operand buffer by one bulk copy, issued by
// thread 0 as soon as the current tile's first product has read that buffer,
// so the copy runs behind the rest of the tile; each thread then converts 8
// features of a row at a time, standardised and split into bf16 hi + lo, in
// place.  Outputs leave through the activation tile once the last product has
// read it: the coefficient rows, or the 108-wide dE/drho rows.
// dE/dA (Eq. 4 for the pair form):
//   G_{n,tau} = l!/tau! sum_m (1 + [m = n]) A_{m,tau} dE/drho_(min(n,m), max(n,m), l),
// four threads per atom, each owning two radial indices and writing its 20
// values as five float4 in the edge kernels' lane-interleaved order.
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace reann {
namespace {

constexpr int PT = 512;       // threads per block
constexpr int PNP = 8;        // N_phi
constexpr int PP = PNP * (PNP + 1) / 2;   // radial pairs
constexpr int DIN = 3 * PP;   // 108 density features
constexpr int KIN = 112;      // padded to a multiple of 16
constexpr int PD = 3 * PNP;   // 24 coefficients
constexpr int PNA = PNP * NT; // 80 A values per atom
constexpr int GXS = DIN + 1;  // padded fp32 row stride of dE/drho rows
constexpr int YS = PD + 1;    // padded fp32 row stride of output rows

template <int MODE>
struct PairLayout {
    static constexpr int W1 = 0;                                  // [128][KIN]
    static constexpr int W2 = W1 + 128 * KIN * 2;                 // [128][128]
    static constexpr int W3 = W2 + 128 * 128 * 2;                 // [KPAD][128]
    static constexpr int X = W3 + KPAD * 128 * 2;                 // [TM][KIN] x 2
    static constexpr int DY = X + 2 * TM * KIN * 2;               // [TM][KPAD] x 2 (BWD)
    static constexpr int ACT = DY + (MODE == TC_BWD ? 2 * TM * KPAD * 2 : 0);  // [TM][128] x 2
    static constexpr int F32 = ACT + 2 * TM * 128 * 2;
    static constexpr int nf32 = 128 + 128 + KPAD + 2 * KIN + 128 + 4 * TM;   // b1, b2, b3, shift, 1/scale, w3, e parts
    static constexpr int BAR = F32 + nf32 * 4;   // MMA-completion mbarrier; input-copy mbarrier at BAR + 8
    static constexpr int bytes = BAR + 32;
    static constexpr int C_Z1 = 0, C_Z2 = 128, C_P = 256, C_OUT = 384;
    static_assert(TM * GXS * 4 <= 2 * TM * 128 * 2, "dE/drho rows fit the activation tile");
    static_assert(TM * YS * 4 <= 2 * TM * 128 * 2, "output rows fit the activation tile");
    static_assert(TM * DIN * 4 <= 2 * TM * KIN * 2 && (DIN * 4) % 16 == 0, "raw rows fit the input tile, 16-byte rows");
    static_assert(BAR % 16 == 0, "aligned barriers");
    static_assert(X % 16 == 0 && DY % 16 == 0 && ACT % 16 == 0 && F32 % 16 == 0, "16-byte aligned tiles");
};

// one value as a bf16 pair (hi = bf16(v), lo = bf16(v - hi)) at (r, k) of two K-major tiles
__device__ __forceinline__ void st_elem2(unsigned char *hi, unsigned char *lo, int R, int r, int k, float v) {
    const uint32_t a = __float_as_uint(v) + 0x8000u;
    const float l = v - __uint_as_float(a & 0xFFFF0000u);
    const uint32_t off = kmaj(r, k, R);
    *reinterpret_cast<unsigned short *>(hi + off) = (unsigned short)(a >> 16);
    *reinterpret_cast<unsigned short *>(lo + off) = (unsigned short)((__float_as_uint(l) + 0x8000u) >> 16);
}

template <int MODE>
__global__ void __launch_bounds__(PT, 1)
    k_mlp_tc_pair(const int4 *__restrict__ tiles, int n_tiles, const float *__restrict__ w, TcNets nets,
                  const float *__restrict__ X, float *__restrict__ Y, const float *__restrict__ dY,
                  float *__restrict__ Ei, const float *__restrict__ A, float *__restrict__ Gout,
                  int *__restrict__ status) {
    using L = PairLayout<MODE>;
    constexpr int DOUT = MODE == TC_ENERGY ? 1 : PD;
    extern __shared__ __align__(1024) unsigned char sm[];
    float *f32 = reinterpret_cast<float *>(sm + L::F32);
    float *sb1 = f32, *sb2 = sb1 + 128, *sb3 = sb2 + 128, *sshift = sb3 + KPAD, *sinv = sshift + KIN,
          *sw3 = sinv + KIN, *se = sw3 + 128;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *cbar = reinterpret_cast<uint64_t *>(sm + L::BAR + 8);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::BAR + 16);
    unsigned char *x_hi = sm + L::X, *x_lo = x_hi + TM * KIN * 2;
    unsigned char *dy_hi = sm + L::DY, *dy_lo = dy_hi + TM * KPAD * 2;
    unsigned char *act_hi = sm + L::ACT, *act_lo = act_hi + TM * 128 * 2;
    float *ystage = reinterpret_cast<float *>(act_hi);   // output rows (forward), after the last product
    float *gxs = reinterpret_cast<float *>(act_hi);      // dE/drho rows, after the last product

    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & (TM - 1);
    const int qc = tid / TM;
    const int c = 32 * qc;
    const uint32_t base = smem_u32(sm);
    auto sa = [&](const unsigned char *p) { return base + (uint32_t)(p - sm); };

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(cbar)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the upstream-gradient operand starts at zero: its padding columns
    // (24..31) are never written again (the input operand's padding, features
    // 108..111, is rewritten with every tile)
    if (MODE == TC_BWD)
        for (int k = tid; k < (2 * TM * KPAD * 2) / 16; k += PT)
            reinterpret_cast<uint4 *>(dy_hi)[k] = make_uint4(0u, 0u, 0u, 0u);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint32_t phase = 0;
    bool failed = false;
    int cur = -1;

    auto wait_mma = [&]() -> bool {
        bool ok = bar_wait(bar, phase);
        phase ^= 1u;
        fence_after();
        return !__syncthreads_or(!ok);
    };
    auto handoff = [&]() {
        fence_smem_to_async();
        fence_before();
        __syncthreads();
    };

    // raw rows: the next tile's (contiguous) rows are prefetched into L2 while
    // the current tile computes; each tile then loads its own rows from L2 in
    // element order (coalesced), so no registers stay live across a tile
    constexpr int NCH = KIN / 8;                      // 14 eight-feature chunks per row
    constexpr int NXC = (TM * NCH + PT - 1) / PT;    // 4 chunks per thread
    constexpr int NDR = (TM * PD + PT - 1) / PT;     // 6
    int4 tl = blockIdx.x < n_tiles ? tiles[blockIdx.x] : make_int4(0, 0, 0, 0);
    // a tile's raw rho rows -> the input operand buffer by one bulk copy
    // (thread 0), completion on cbar
    uint32_t cphase = 0;
    bool copy_pending = false;
    auto copy_rows = [&](int rr0, int rrows) {
        if (tid == 0) {
            const uint32_t nb = (uint32_t)(rrows * DIN * 4);
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(cbar)), "r"(nb)
                         : "memory");
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                         ::"r"(sa(x_hi)), "l"(X + (int64_t)rr0 * DIN), "r"(nb), "r"(smem_u32(cbar))
                         : "memory");
        }
        copy_pending = true;
    };
    if (tl.z > 0) copy_rows(tl.y, tl.z);
    for (int ti = blockIdx.x; ti < n_tiles && !failed; ti += gridDim.x) {
        const int4 tile = tl;
        const int e = tile.x, r0 = tile.y, rows = tile.z;
        tl = ti + (int)gridDim.x < n_tiles ? tiles[ti + gridDim.x] : make_int4(0, 0, 0, 0);
        if (e != cur) {
            const NetOffsets &o = nets.net[e];
            for (int k = tid; k < 128 * KIN; k += PT) {
                const int n = k / KIN, f = k % KIN;
                st_elem(sm + L::W1, 128, n, f, f < DIN ? w[o.W1 + (int64_t)n * DIN + f] : 0.f);
            }
            for (int k = tid; k < 128 * 128; k += PT) st_elem(sm + L::W2, 128, k / 128, k % 128, w[o.W2 + k]);
            for (int k = tid; k < KPAD * 128; k += PT) {
                const int n = k / 128, h = k % 128;
                st_elem(sm + L::W3, KPAD, n, h, n < DOUT ? w[o.W3 + (int64_t)n * 128 + h] : 0.f);
            }
            for (int k = tid; k < 128; k += PT) {
                sb1[k] = w[o.b1 + k];
                sb2[k] = w[o.b2 + k];
                sw3[k] = MODE == TC_ENERGY ? w[o.W3 + k] : 0.f;
            }
            for (int k = tid; k < KPAD; k += PT) sb3[k] = k < DOUT ? w[o.b3 + k] : 0.f;
            for (int k = tid; k < KIN; k += PT) {
                sshift[k] = k < DIN ? w[o.shift + k] : 0.f;
                sinv[k] = k < DIN ? 1.0f / w[o.scale + k] : 0.f;
            }
            cur = e;
            __syncthreads();
        }
        if (tid == 0) {
            if (MODE != TC_FWD) prefetch_l2(A + (int64_t)r0 * PNA, (uint32_t)(rows * PNA * 4));
            if (MODE == TC_BWD && tl.z > 0) prefetch_l2(dY + (int64_t)tl.y * PD, (uint32_t)(tl.z * PD * 4));
        }
        // the tile's raw rows have arrived in the input buffer: each thread reads
        // 8-feature chunks (chunk k / TM of row k % TM: a warp takes one chunk of
        // 32 consecutive rows, so neither the 432-byte-strided reads nor the
        // K-major operand stores meet a bank twice), then, once every thread has
        // read its chunks, writes them standardised and split bf16 in place
        // (features past 108 and rows past the tile's end as zeros)
        {
            const bool landed = bar_wait(cbar, cphase);
            cphase ^= 1u;
            copy_pending = !landed;
            if (__syncthreads_or(!landed)) { failed = true; break; }
            const float *xs = reinterpret_cast<const float *>(x_hi);
            float xr[NXC][8];
#pragma unroll
            for (int u = 0; u < NXC; ++u) {
                const int k = tid + u * PT, rk = k % TM, f0 = 8 * (k / TM);
#pragma unroll
                for (int h4 = 0; h4 < 8; h4 += 4) {
                    const bool ok = k < TM * NCH && rk < rows && f0 + h4 < DIN;
                    const float4 t = ok ? *reinterpret_cast<const float4 *>(xs + rk * DIN + f0 + h4)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    xr[u][h4] = t.x, xr[u][h4 + 1] = t.y, xr[u][h4 + 2] = t.z, xr[u][h4 + 3] = t.w;
                }
            }
            __syncthreads();
#pragma unroll
            for (int u = 0; u < NXC; ++u) {
                const int k = tid + u * PT, rk = k % TM, f0 = 8 * (k / TM);
                if (k < TM * NCH) {
#pragma unroll
                    for (int e2 = 0; e2 < 8; ++e2)
                        xr[u][e2] = rk < rows ? (xr[u][e2] - sshift[f0 + e2]) * sinv[f0 + e2] : 0.f;
                    st_chunk2(x_hi, x_lo, TM, rk, f0, xr[u]);
                }
            }
        }
        if (MODE == TC_BWD) {
            const float *dg = dY + (int64_t)r0 * PD;
            float dr[NDR];
#pragma unroll
            for (int u = 0; u < NDR; ++u) {
                const int k = tid + u * PT;
                dr[u] = k < rows * PD ? dg[k] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < NDR; ++u) {
                const int k = tid + u * PT;
                if (k < rows * PD) {
                    const int rk = k / PD, f = k - rk * PD;
                    st_elem2(dy_hi, dy_lo, TM, rk, f, dr[u]);
                }
            }
        }
        handoff();

        if (tid == 0) {
            fence_after();
            gemm2<128, KIN, false, 0>(tmem + L::C_Z1, sa(x_hi), sa(x_lo), base + L::W1);
            if (MODE == TC_BWD) gemm2<128, KPAD, true, KPAD>(tmem + L::C_P, sa(dy_hi), sa(dy_lo), base + L::W3);
            mma_commit(bar);
        }
        if (!wait_mma()) { failed = true; break; }
        // the first product has read the input buffer: the next tile's raw rows may land there
        if (tl.z > 0) copy_rows(tl.y, tl.z);
        {
            float v[32];
            tmem_ld32(lane_base + L::C_Z1 + c, v);
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = tanh_fast(v[u] + sb1[c + u]);
#pragma unroll
            for (int u = 0; u < 32; u += 8) st_chunk2(act_hi, act_lo, TM, row, c + u, &v[u]);
        }
        handoff();
        if (tid == 0) {
            fence_after();
            gemm2<128, 128, false, 0>(tmem + L::C_Z2, sa(act_hi), sa(act_lo), base + L::W2);
            mma_commit(bar);
        }
        if (!wait_mma()) { failed = true; break; }

        if (MODE == TC_FWD) {
            {
                float v[32];
                tmem_ld32(lane_base + L::C_Z2 + c, v);
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] = tanh_fast(v[u] + sb2[c + u]);
#pragma unroll
                for (int u = 0; u < 32; u += 8) st_chunk2(act_hi, act_lo, TM, row, c + u, &v[u]);
            }
            handoff();
            if (tid == 0) {
                fence_after();
                gemm2<KPAD, 128, false, 0>(tmem + L::C_OUT, sa(act_hi), sa(act_lo), base + L::W3);
                mma_commit(bar);
            }
            if (!wait_mma()) { failed = true; break; }
            {
                float v[8];
                tmem_ld8(lane_base + L::C_OUT + 8 * qc, v);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int f = 8 * qc + u;
                    if (f < PD) ystage[row * YS + f] = v[u] + sb3[f];
                }
            }
            __syncthreads();
            float *yo = Y + (int64_t)r0 * PD;
            for (int k = tid; k < rows * PD; k += PT) {
                const int rk = k / PD;
                yo[k] = ystage[rk * YS + (k - rk * PD)];
            }
        } else {
            {
                float z[32], up[32];
                tmem_ld32(lane_base + L::C_Z2 + c, z);
                if (MODE == TC_BWD) tmem_ld32(lane_base + L::C_P + c, up);
                float e_row = 0.f;
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const float a = tanh_fast(z[u] + sb2[c + u]);
                    const float g = MODE == TC_ENERGY ? sw3[c + u] : up[u];
                    if (MODE == TC_ENERGY) e_row = fmaf(sw3[c + u], a, e_row);
                    z[u] = g * (1.f - a * a);
                }
#pragma unroll
                for (int u = 0; u < 32; u += 8) st_chunk2(act_hi, act_lo, TM, row, c + u, &z[u]);
                if (MODE == TC_ENERGY) se[qc * TM + row] = e_row;
            }
            handoff();
            if (MODE == TC_ENERGY && qc == 0 && row < rows)
                Ei[r0 + row] = ((se[row] + se[TM + row]) + (se[2 * TM + row] + se[3 * TM + row])) + sb3[0];
            if (tid == 0) {
                fence_after();
                gemm2<128, 128, true, 128>(tmem + L::C_P, sa(act_hi), sa(act_lo), base + L::W2);
                mma_commit(bar);
            }
            if (!wait_mma()) { failed = true; break; }
            {
                float p[32], z[32];
                tmem_ld32(lane_base + L::C_P + c, p);
                tmem_ld32(lane_base + L::C_Z1 + c, z);
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const float a = tanh_fast(z[u] + sb1[c + u]);
                    p[u] *= 1.f - a * a;
                }
#pragma unroll
                for (int u = 0; u < 32; u += 8) st_chunk2(act_hi, act_lo, TM, row, c + u, &p[u]);
            }
            handoff();
            // dE/dx = g1 W1 (MN-major view of W1): the 112 padded input columns
            if (tid == 0) {
                fence_after();
                gemm2<KIN, 128, true, 128>(tmem + L::C_OUT, sa(act_hi), sa(act_lo), base + L::W1);
                mma_commit(bar);
            }
            if (!wait_mma()) { failed = true; break; }
            // dE/drho rows through the activation tile (consumed by the last product)
            {
                float v[32];
                tmem_ld32(lane_base + L::C_OUT + c, v);
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int f = c + u;
                    if (f < DIN) gxs[row * GXS + f] = v[u] * sinv[f];
                }
            }
            __syncthreads();
            // G = dE/dA: thread (atom rk, part) takes radial indices n = 2 part, 2 part + 1.  It
            // loads its quarter of the atom's A row (A_{m,tau} for m = 2 part, 2 part + 1: five
            // float4) and receives the other quarters from the atom's three other lanes by warp
            // shuffles.  Per l it forms the coupling rows M_{n,m} = (1 + [m = n])
            // dE/drho_(min, max of n m, l) once and streams A_{m,tau}; its 20 results are the
            // lane-interleaved positions 16 q + 4 part + e (q < 5, e < 4), i.e. five float4 stores.
            {
                const int rk = tid >> 2, part = tid & 3, lead = tid & 28;
                const bool live = rk < rows;
                const float *g = gxs + rk * GXS;
                float aq[2 * NT];   // A_{2 part + s, tau} at 10 s + tau
                {
                    const float4 *a4 =
                        reinterpret_cast<const float4 *>(A + (int64_t)(r0 + (live ? rk : 0)) * PNA) + 5 * part;
#pragma unroll
                    for (int q = 0; q < 5; ++q) {
                        const float4 v = live ? __ldg(a4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
                        aq[4 * q] = v.x, aq[4 * q + 1] = v.y, aq[4 * q + 2] = v.z, aq[4 * q + 3] = v.w;
                    }
                }
                float acc[2][NT];
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
                    for (int u = 0; u < NT; ++u) acc[s2][u] = 0.f;
#pragma unroll
                for (int l = 0; l < 3; ++l) {
                    float M[2][PNP];
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2) {
                        const int n = 2 * part + s2;
#pragma unroll
                        for (int m = 0; m < PNP; ++m) {
                            const int lo = m < n ? m : n, hi = m < n ? n : m;
                            M[s2][m] = (m == n ? 2.f : 1.f) * g[l * PP + lo * PNP - lo * (lo - 1) / 2 + (hi - lo)];
                        }
                    }
#pragma unroll
                    for (int u = 0; u < NT; ++u) {
                        // the tuples of order l: u in [0, 1), [1, 4), [4, 10)
                        if (u < (l == 0 ? 0 : (l == 1 ? 1 : 4)) || u >= (l == 0 ? 1 : (l == 1 ? 4 : 10))) continue;
#pragma unroll
                        for (int m = 0; m < PNP; ++m) {
                            const float a = __shfl_sync(0xffffffffu, aq[(m & 1) * NT + u], lead + (m >> 1));
                            acc[0][u] = fmaf(M[0][m], a, acc[0][u]);
                            acc[1][u] = fmaf(M[1][m], a, acc[1][u]);
                        }
                    }
                }
                if (live) {
                    float4 *go4 = reinterpret_cast<float4 *>(Gout + (int64_t)(r0 + rk) * PNA);
                    // l!/tau! times the sums, in the layer's lane order (pairs: idx = 2 tau + s,
                    // radial-major: idx = 10 s + tau)
                    auto put = [&](auto pairs) {
#pragma unroll
                        for (int q = 0; q < 5; ++q) {
                            float v[4];
#pragma unroll
                            for (int e2 = 0; e2 < 4; ++e2) {
                                const int idx = 4 * q + e2;
                                const int s2 = pairs ? idx % 2 : idx / NT, u = pairs ? idx / 2 : idx % NT;
                                v[e2] = (u >= 7 ? 2.f : 1.f) * acc[s2][u];
                            }
                            go4[4 * q + part] = make_float4(v[0], v[1], v[2], v[3]);
                        }
                    };
                    if (nets.g_pairs) put(std::true_type{});
                    else put(std::false_type{});
                }
            }
        }
        fence_before();
        __syncthreads();
    }

    // a copy still in flight (the block left early) lands before the block exits
    if (copy_pending) bar_wait(cbar, cphase & 1u);
    if (failed && tid == 0) atomicOr(status, ST_TIMEOUT);
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

template <int MODE>
cudaError_t run_pair(reann_ctx *c, const TcNets &nets, const float *X, float *Y, const float *dY, float *Ei,
                     const float *A, float *G, cudaStream_t s) {
    using L = PairLayout<MODE>;
    static_assert(L::bytes > 116 * 1024 && L::bytes <= 227 * 1024, "one block per SM keeps TMEM allocation safe");
    static bool configured[64] = {};
    auto kern = k_mlp_tc_pair<MODE>;
    if (c->device < 0 || c->device >= 64) return cudaErrorInvalidDevice;
    if (!configured[c->device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::bytes);
        if (e) return e;
        configured[c->device] = true;
    }
    if (c->n_tiles128 == 0) return cudaSuccess;
    const int grid = c->sm_count < c->n_tiles128 ? c->sm_count : c->n_tiles128;
    REANN_TIMED(c, MODE == TC_FWD ? REANN_K_MLP_FWD : (MODE == TC_ENERGY ? REANN_K_MLP_ENERGY : REANN_K_MLP_BWD), s);
    kern<<<grid, PT, L::bytes, s>>>(c->d_tiles128, c->n_tiles128, c->d_w, nets, X, Y, dY, Ei, A, G, c->d_status);
    return cudaGetLastError();
}

TcNets pair_nets(const std::vector<NetOffsets> &v, int first, int ne, int NP, int layer) {
    TcNets m;
    m.g_pairs = g_pairs(NP, layer);
    for (int e = 0; e < ne; ++e) m.net[e] = v[first + e];
    return m;
}

}  // namespace

cudaError_t launch_mlp_tc_pair_coef_fwd(reann_ctx *c, int t, cudaStream_t s) {
    const int64_t nR = c->n * c->DR;
    return run_pair<TC_FWD>(c, pair_nets(c->coef_nets, t * c->ne, c->ne, c->NP, 0), c->d_rho + t * nR,
                            c->d_coef + (t + 1) * c->n_slots * c->D, nullptr, nullptr, nullptr, nullptr, s);
}

cudaError_t launch_mlp_tc_pair_energy(reann_ctx *c, cudaStream_t s) {
    const int64_t nR = c->n * c->DR, nA = c->n * c->NA;
    const int t = c->T - 1;
    return run_pair<TC_ENERGY>(c, pair_nets(c->energy_nets, 0, c->ne, c->NP, c->T - 1), c->d_rho + t * nR, nullptr,
                               nullptr, c->d_Ei, c->d_A + t * nA, c->d_G, s);
}

cudaError_t launch_mlp_tc_pair_coef_bwd(reann_ctx *c, int t, cudaStream_t s) {
    const int64_t nR = c->n * c->DR, nA = c->n * c->NA;
    return run_pair<TC_BWD>(c, pair_nets(c->coef_nets, (t - 1) * c->ne, c->ne, c->NP, t - 1), c->d_rho + (t - 1) * nR,
                            nullptr, c->d_dc, nullptr, c->d_A + (t - 1) * nA, c->d_G, s);
}

}  // namespace reann
