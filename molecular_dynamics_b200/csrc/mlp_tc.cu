// Per-element atomic networks on the 5th-generation tensor cores (tcgen05),
// bf16 operands with fp32 accumulation in tensor memory.  Weights are bf16
// values; activations and gradients enter each GEMM as a pair of bf16 terms
// (hi = bf16(v), lo = bf16(v - hi)), two MMA passes into one accumulator, so
// an operand keeps 16 significant bits.
//
// Same networks as mlp.cu ("Efficient Parallelization of Message Passing
// Neural Network Potentials for Large-Scale Molecular Dynamics", section "REANN
// Architecture", Eq. 2 and the atomic energy; section "Parallelization
// Algorithm", Eqs. 3 and 5 for the vector-Jacobian products):
//   y = W3 tanh(W2 tanh(W1 ((x - shift) / scale) + b1) + b2) + b3.
// A tile is 128 atoms of one element.  Each layer is one 128 x N x K GEMM
// (tcgen05.mma, M = 128, K = 16 per instruction) whose accumulator sits in
// TMEM; TMEM lane i holds atom i, so the epilogue (bias, tanh, tanh', the
// energy dot product) is per atom with no cross-lane reduction.  The epilogue
// writes the next layer's bf16 operand straight into shared memory in the
// canonical K-major layout (one activation buffer, reused by every layer once
// the product that read it has completed), and one thread issues the next MMA.
//
// Block: 512 threads, one per SM (shared memory > half an SM), working through
// a contiguous range of one element's tiles (the element's weights are loaded
// once).  The block runs two independent groups of 256 threads, each on every
// other tile of the range with its own 256 TMEM columns, operand buffers,
// MMA-completion mbarrier and named barrier, so one group's epilogue overlaps
// the other's products.  In a group, warp w reads TMEM lanes 32 (w % 4) .. + 31
// and half (w / 4) % 2 takes 64 columns of every 128-wide accumulator.  The
// epilogues keep the special-function unit (tanh) and the issue slots busy
// while they run: bf16 rounding of the split operands is done with integer
// instructions so that the special-function pipe only evaluates tanh.  The coefficient backward recomputes the first layer's
// pre-activation (one small product) instead of keeping it, to fit 256 columns.
//
// Global traffic: the forward and energy networks' raw input rows arrive by
// one bulk copy per tile (issued by thread 0 into the group's X buffer as soon
// as the previous tile's first product has read it), or, for rows that are not
// whole 16-byte units, are loaded in element order and transposed to rows
// through the idle activation buffer; the coefficient backward loads each
// row's rho and upstream gradient per thread; forward outputs leave through
// the activation buffer as contiguous stores; for the energy network and the
// coefficient backward the tile's A rows are prefetched into L2 at the start of
// the tile and loaded into registers while the tile's last product runs, and
// dE/dA = 2 w_tau A dE/drho is written one warp per row in the edge kernels'
// lane-interleaved order.  Tile descriptors are read one tile ahead.  All
// MMA-completion waits are bounded: a wait that gives up is recorded, the group
// learns of it at its next barrier (a barrier with an OR over its threads, so
// all leave together), sets ST_TIMEOUT, frees its tensor memory and returns.
// The shared-memory operand layout is described in tc_common.cuh.
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace reann {
namespace {

constexpr int TC_THREADS = 512;    // two independent groups of 256 threads
constexpr int TC_GROUP = 256;

// named barrier of one thread group (ids 1 and 2; 0 is __syncthreads), and
// the same barrier with an OR over the group's predicates
__device__ __forceinline__ void group_sync(int g) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(TC_GROUP) : "memory");
}
__device__ __forceinline__ bool group_or(int g, bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, o;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred o, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, o;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(1 + g), "r"(TC_GROUP)
        : "memory");
    return r != 0;
}

template <int NP, int H1, int H2, int MODE>
struct TcLayout {
    static constexpr int D = 3 * NP;
    static constexpr int NA = NP * NT;
    static constexpr int RS = D + 1;          // padded fp32 row stride of staged rows (odd: no bank conflicts)
    static constexpr int GXS = KPAD + 1;      // padded row stride of dE/drho rows
    // shared by both groups: bf16 weight tiles, K-major, one copy each (the
    // backward products read them through the MN-major view), fp32 vectors
    static constexpr int W1 = 0;                                 // [H1][KPAD]
    static constexpr int W2 = W1 + H1 * KPAD * 2;                // [H2][H1]
    static constexpr int W3 = W2 + H2 * H1 * 2;                  // [KPAD][H2] (rows >= n_out are zero)
    static constexpr int F32 = W3 + KPAD * H2 * 2;
    static constexpr int nf32 = H1 + H2 + KPAD + 2 * KPAD + H2;  // b1, b2, b3, shift, 1/scale, w3
    static constexpr int GRP = (F32 + nf32 * 4 + 15) / 16 * 16;
    // per group (offsets inside the group's region):
    //   ACT  [TM][128] bf16 hi + lo: the operand of layers 2 and 3 (and of the
    //        VJP products), reused by every layer once the product that read it
    //        has completed; between products it also holds the raw input rows
    //        of the forward and energy networks (fp32 [TM][RS]), the dY
    //        operand of the backward (hi + lo at ACT_DY),
    //        the output rows and the dE/drho rows
    //   X    [TM][KPAD] bf16 hi + lo, kept for the whole tile (the backward
    //        recomputes layer 1 from it)
    static constexpr int ACT = 0;
    static constexpr int ACT_DY = 48 * 1024;
    static constexpr int X = ACT + 2 * TM * 128 * 2;
    static constexpr int SE = X + 2 * TM * KPAD * 2;             // energy partials [2][TM] fp32
    static constexpr int BAR = SE + 2 * TM * 4;                  // MMA-completion mbarrier
    static constexpr int CBAR = BAR + 8;                         // input-copy mbarrier
    static constexpr int GROUP_BYTES = BAR + 16;
    // forward and energy: the next tile's raw rows are copied into X (a bulk
    // copy, 16-byte units) once the current tile's first product has read X
    static constexpr bool BULK = MODE != TC_BWD && (D * 4) % 16 == 0;
    static_assert(TM * D * 4 <= 2 * TM * KPAD * 2, "raw input rows fit the X operand buffer");
    static constexpr int SLOT = GRP + 2 * GROUP_BYTES;           // TMEM base address
    static constexpr int bytes = SLOT + 16;
    static_assert(TM * RS * 4 <= ACT_DY && ACT_DY + 2 * TM * KPAD * 2 <= X, "input staging fits the ACT buffer");
    static_assert(TM * GXS * 4 <= X && TM * RS * 4 <= X, "output staging fits the ACT buffer");
    static_assert(GRP % 16 == 0 && GROUP_BYTES % 16 == 0, "16-byte aligned operand tiles");
    // TMEM columns of a group (its base is 256 g): two 128-column accumulators
    static constexpr int C_A = 0, C_B = 128;
};

// Two independent groups of 256 threads (8 warps) per block, each working on
// its own tiles of the block's tile range with its own TMEM columns, operand
// buffers, MMA-completion barrier and named barrier, so that one group's
// epilogue (tanh on the special-function pipe, shared-memory stores) overlaps
// the other's tensor-core products.  Inside a group, warp w reads TMEM lanes
// 32 (w % 4) .. + 31 and thread half h = (w / 4) % 2 takes columns 64 h .. 64 h + 63
// of every 128-wide accumulator.
template <int NP, int H1, int H2, int MODE>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_mlp_tc(const int4 *__restrict__ tiles, const int4 *__restrict__ ranges, const float *__restrict__ w,
             TcNets nets, const float *__restrict__ X, float *__restrict__ Y, const float *__restrict__ dY,
             float *__restrict__ Ei, const float *__restrict__ A, float *__restrict__ Gout, int *__restrict__ status) {
    static_assert(H1 == 128 && H2 == 128, "two 32-column chunks per thread and layer");
    using L = TcLayout<NP, H1, H2, MODE>;
    constexpr int D = L::D, NA = L::NA, RS = L::RS;
    constexpr int DOUT = MODE == TC_ENERGY ? 1 : D;
    extern __shared__ __align__(1024) unsigned char sm[];
    float *f32 = reinterpret_cast<float *>(sm + L::F32);
    float *sb1 = f32, *sb2 = sb1 + H1, *sb3 = sb2 + H2, *sshift = sb3 + KPAD, *sinv = sshift + KPAD,
          *sw3 = sinv + KPAD;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int g = tid / TC_GROUP, gt = tid - g * TC_GROUP, gw = gt >> 5;
    const int row = gt & (TM - 1);             // this thread's atom within the tile (TMEM lane)
    const int h = gt / TM;                     // column half
    unsigned char *gs = sm + L::GRP + g * L::GROUP_BYTES;
    unsigned char *act_hi = gs + L::ACT, *act_lo = act_hi + TM * 128 * 2;
    unsigned char *dy_hi = gs + L::ACT_DY, *dy_lo = dy_hi + TM * KPAD * 2;
    unsigned char *x_hi = gs + L::X, *x_lo = x_hi + TM * KPAD * 2;
    float *stage = reinterpret_cast<float *>(gs + L::ACT);
    float *se = reinterpret_cast<float *>(gs + L::SE);
    uint64_t *bar = reinterpret_cast<uint64_t *>(gs + L::BAR);
    uint64_t *cbar = reinterpret_cast<uint64_t *>(gs + L::CBAR);
    const uint32_t base = smem_u32(sm);
    auto sa = [&](const unsigned char *p) { return base + (uint32_t)(p - sm); };

    const int4 rg = ranges[blockIdx.x];        // (first tile, end tile, element, -)
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (gt == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(cbar)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    {
        // the block's element: weights -> bf16 tiles and fp32 vectors
        const NetOffsets &o = nets.net[rg.z];
        for (int k = tid; k < H1 * KPAD; k += TC_THREADS) {
            int n = k / KPAD, f = k % KPAD;
            st_elem(sm + L::W1, H1, n, f, f < D ? w[o.W1 + (int64_t)n * D + f] : 0.f);
        }
        for (int k = tid; k < H2 * H1; k += TC_THREADS) st_elem(sm + L::W2, H2, k / H1, k % H1, w[o.W2 + k]);
        for (int k = tid; k < KPAD * H2; k += TC_THREADS) {
            int n = k / H2, hh = k % H2;
            st_elem(sm + L::W3, KPAD, n, hh, n < DOUT ? w[o.W3 + (int64_t)n * H2 + hh] : 0.f);
        }
        for (int k = tid; k < H1; k += TC_THREADS) sb1[k] = w[o.b1 + k];
        for (int k = tid; k < H2; k += TC_THREADS) {
            sb2[k] = w[o.b2 + k];
            sw3[k] = MODE == TC_ENERGY ? w[o.W3 + k] : 0.f;
        }
        for (int k = tid; k < KPAD; k += TC_THREADS) {
            sb3[k] = k < DOUT ? w[o.b3 + k] : 0.f;
            sshift[k] = k < D ? w[o.shift + k] : 0.f;
            sinv[k] = k < D ? 1.0f / w[o.scale + k] : 0.f;
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot + (uint32_t)(256 * g);
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint32_t phase = 0;
    bool failed = false, bad = false;

    // completion of the MMA group the group's thread 0 committed; a wait that
    // gave up is recorded and acted on at the group's next barrier (the TMEM
    // values read meanwhile are discarded)
    auto wait_mma = [&]() {
        bad |= !bar_wait(bar, phase);
        phase ^= 1u;
        fence_after();
    };
    // operand stores (generic proxy) and TMEM reads done -> next MMA may
    // start; true if a wait of the group gave up
    auto handoff = [&]() -> bool {
        fence_smem_to_async();
        fence_before();
        return group_or(g, bad);
    };

    // dE/dA positions of this lane (element pk = lane + 32 j of a row, in the
    // edge kernels' lane-interleaved order), packed: source A index (bits 0-7),
    // dE/drho index (bits 8-15), mixed second-order tuple (bit 16: 2 w_tau = 4)
    constexpr int NJ = (NA + 31) / 32;
    int posj[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int pk = (tid & 31) + 32 * j;
        const int src = g_slot_source(pk < NA ? pk : 0, NP, nets.g_pairs), nn = src / NT, u = src - nn * NT;
        const int gi = (u == 0 ? 0 : (u < 4 ? 1 : 2)) * NP + nn;
        posj[j] = src | (gi << 8) | ((u >= 7 ? 1 : 0) << 16);
    }

    // tile descriptors are loaded one tile ahead, off the tile's critical path
    int next_r0 = 0, next_rows = 0;
    if (rg.x + g < rg.y) next_r0 = tiles[rg.x + g].y, next_rows = tiles[rg.x + g].z;
    // raw rows of a tile -> X by one bulk copy (thread 0), completion on cbar
    uint32_t cphase = 0;
    bool copy_pending = false;
    auto copy_rows = [&](int rr0, int rrows) {
        if (gt == 0) {
            const uint32_t nb = (uint32_t)(rrows * D * 4);
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(cbar)), "r"(nb)
                         : "memory");
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                         ::"r"(sa(x_hi)), "l"(X + (int64_t)rr0 * D), "r"(nb), "r"(smem_u32(cbar))
                         : "memory");
        }
        copy_pending = true;
    };
    if (L::BULK && rg.x + g < rg.y) copy_rows(next_r0, next_rows);
    for (int ti = rg.x + g; ti < rg.y && !failed; ti += 2) {
        const int r0 = next_r0, rows = next_rows;
        if (ti + 2 < rg.y) next_r0 = tiles[ti + 2].y, next_rows = tiles[ti + 2].z;
        // energy and backward: the tile's A rows are read at the end; start
        // moving them into L2 now
        if (MODE != TC_FWD && gt == 0) prefetch_l2(A + (int64_t)r0 * NA, (uint32_t)(rows * NA * 4));
        // input tile, standardised rho (and the upstream gradient) split into
        // bf16 hi/lo.  Coefficient backward: each thread loads its own row's 16
        // features of both (columns 16 h .. 16 h + 15, zero past D) as float2
        // pairs straight into registers.  Forward and energy with 16-byte rows:
        // the raw rows were copied into X while the previous tile computed.
        // Otherwise: contiguous raw rows -> padded fp32 rows in ACT.  Where the
        // rows are loaded here, the group's next tile's rows are moved into L2
        // meanwhile.
        const bool live = row < rows;
        if (MODE == TC_BWD) {
            const int64_t atom = r0 + (live ? row : 0);
            const float *xr = X + atom * D, *dr = dY + atom * D;
            float v[16], gv[16];
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
                const int f = 16 * h + u;
                const bool ok = live && f < D;
                const float2 t = ok ? *reinterpret_cast<const float2 *>(xr + f) : make_float2(0.f, 0.f);
                const float2 q = ok ? *reinterpret_cast<const float2 *>(dr + f) : make_float2(0.f, 0.f);
                v[u] = t.x, v[u + 1] = t.y, gv[u] = q.x, gv[u + 1] = q.y;
            }
            if (gt == 0 && ti + 2 < rg.y) {
                prefetch_l2_span(X + (int64_t)next_r0 * D, (size_t)next_rows * D * 4);
                prefetch_l2_span(dY + (int64_t)next_r0 * D, (size_t)next_rows * D * 4);
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int f = 16 * h + u;
                v[u] = live ? (v[u] - sshift[f]) * sinv[f] : 0.f;
            }
            st_chunk2(x_hi, x_lo, TM, row, 16 * h, v);
            st_chunk2(x_hi, x_lo, TM, row, 16 * h + 8, v + 8);
            st_chunk2(dy_hi, dy_lo, TM, row, 16 * h, gv);
            st_chunk2(dy_hi, dy_lo, TM, row, 16 * h + 8, gv + 8);
        } else if (L::BULK) {
            // this tile's raw rows arrived in X by the bulk copy; each thread
            // takes its row's 16 features (16-byte loads), then, once the group
            // has read them all, overwrites X with the bf16 operand
            const bool landed = bar_wait(cbar, cphase);
            bad |= !landed;
            cphase ^= 1u;
            copy_pending = !landed;
            const float *xs = reinterpret_cast<const float *>(x_hi) + row * D;
            float v[16];
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
                const int f = 16 * h + u;
                const float4 t = live && f < D ? *reinterpret_cast<const float4 *>(xs + f) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[u] = t.x, v[u + 1] = t.y, v[u + 2] = t.z, v[u + 3] = t.w;
            }
            group_sync(g);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int f = 16 * h + u;
                v[u] = live && f < D ? (v[u] - sshift[f]) * sinv[f] : 0.f;
            }
            st_chunk2(x_hi, x_lo, TM, row, 16 * h, v);
            st_chunk2(x_hi, x_lo, TM, row, 16 * h + 8, v + 8);
        } else {
            if (gt == 0 && ti + 2 < rg.y) prefetch_l2_span(X + (int64_t)next_r0 * D, (size_t)next_rows * D * 4);
            float *xs = stage;
            const float *xg = X + (int64_t)r0 * D;
            for (int k = gt; k < rows * D; k += TC_GROUP) {
                const int rk = k / D, f = k - rk * D;
                xs[rk * RS + f] = xg[k];
            }
            group_sync(g);
#pragma unroll
            for (int c8 = 0; c8 < 16; c8 += 8) {
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int f = 16 * h + c8 + u;
                    v[u] = live && f < D ? (xs[row * RS + f] - sshift[f]) * sinv[f] : 0.f;
                }
                st_chunk2(x_hi, x_lo, TM, row, 16 * h + c8, v);
            }
        }
        if (handoff()) { failed = true; break; }

        // layer 1 (and, for the coefficient backward, dE/da2 = dY W3 via the MN-major view of W3)
        if (gt == 0) {
            fence_after();
            gemm2<H1, KPAD, false, 0>(tmem + L::C_A, sa(x_hi), sa(x_lo), base + L::W1);
            if (MODE == TC_BWD) gemm2<H2, KPAD, true, KPAD>(tmem + L::C_B, sa(dy_hi), sa(dy_lo), base + L::W3);
            mma_commit(bar);
        }
        wait_mma();
        // X has been read by the product: the group's next tile's raw rows may land there
        if (L::BULK && ti + 2 < rg.y) copy_rows(next_r0, next_rows);
        // a1 = tanh(z1 + b1)
#pragma unroll 1
        for (int c = 64 * h; c < 64 * h + 64; c += 32) {
            float v[32];
            tmem_ld32(lane_base + L::C_A + c, v);
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = tanh_fast(v[u] + sb1[c + u]);
#pragma unroll
            for (int u = 0; u < 32; u += 8) st_chunk2(act_hi, act_lo, TM, row, c + u, &v[u]);
        }
        if (handoff()) { failed = true; break; }
        // z2 = a1 W2^T: into B (forward, energy) or over z1 in A (backward, whose B holds dY W3)
        constexpr int C_Z2 = MODE == TC_BWD ? L::C_A : L::C_B;
        if (gt == 0) {
            fence_after();
            gemm2<H2, H1, false, 0>(tmem + C_Z2, sa(act_hi), sa(act_lo), base + L::W2);
            mma_commit(bar);
        }
        wait_mma();

        if (MODE == TC_FWD) {
            // a2 = tanh(z2 + b2), then y = a2 W3^T + b3 (into A)
#pragma unroll 1
            for (int c = 64 * h; c < 64 * h + 64; c += 32) {
                float v[32];
                tmem_ld32(lane_base + C_Z2 + c, v);
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] = tanh_fast(v[u] + sb2[c + u]);
#pragma unroll
                for (int u = 0; u < 32; u += 8) st_chunk2(act_hi, act_lo, TM, row, c + u, &v[u]);
            }
            if (handoff()) { failed = true; break; }
            if (gt == 0) {
                fence_after();
                gemm2<KPAD, H2, false, 0>(tmem + L::C_A, sa(act_hi), sa(act_lo), base + L::W3);
                mma_commit(bar);
            }
            wait_mma();
            // y rows through ACT (the last product has consumed it), then contiguous stores
#pragma unroll
            for (int c8 = 0; c8 < 16; c8 += 8) {
                float v[8];
                tmem_ld8(lane_base + L::C_A + 16 * h + c8, v);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int f = 16 * h + c8 + u;
                    if (f < D) stage[row * RS + f] = v[u] + sb3[f];
                }
            }
            group_sync(g);
            float *yo = Y + (int64_t)r0 * D;
            for (int k = gt; k < rows * D; k += TC_GROUP) {
                const int rk = k / D;
                yo[k] = stage[rk * RS + (k - rk * D)];
            }
        } else {
            // g2 = dE/dz2 = (energy: w3, backward: dY W3) * (1 - a2^2); energy E_i = w3 . a2 + b3
            float e_row = 0.f;
#pragma unroll 1
            for (int c = 64 * h; c < 64 * h + 64; c += 32) {
                float z[32], up[32];
                tmem_ld32(lane_base + C_Z2 + c, z);
                if (MODE == TC_BWD) tmem_ld32(lane_base + L::C_B + c, up);
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const float a = tanh_fast(z[u] + sb2[c + u]);
                    const float gg = MODE == TC_ENERGY ? sw3[c + u] : up[u];
                    if (MODE == TC_ENERGY) e_row = fmaf(sw3[c + u], a, e_row);
                    z[u] = gg * (1.f - a * a);
                }
#pragma unroll
                for (int u = 0; u < 32; u += 8) st_chunk2(act_hi, act_lo, TM, row, c + u, &z[u]);
            }
            if (MODE == TC_ENERGY) se[h * TM + row] = e_row;
            if (handoff()) { failed = true; break; }
            if (MODE == TC_ENERGY && h == 0 && row < rows) Ei[r0 + row] = (se[row] + se[TM + row]) + sb3[0];
            // p1 = g2 W2 (MN-major view of W2) into B; the backward recomputes z1
            // = x W1^T into A (its first copy was overwritten by z2)
            if (gt == 0) {
                fence_after();
                gemm2<H1, H2, true, H2>(tmem + L::C_B, sa(act_hi), sa(act_lo), base + L::W2);
                if (MODE == TC_BWD) gemm2<H1, KPAD, false, 0>(tmem + L::C_A, sa(x_hi), sa(x_lo), base + L::W1);
                mma_commit(bar);
            }
            wait_mma();
            // g1 = p1 (1 - tanh^2(z1 + b1)), tanh' from the fp32 pre-activation in TMEM
#pragma unroll 1
            for (int c = 64 * h; c < 64 * h + 64; c += 32) {
                float p[32], z[32];
                tmem_ld32(lane_base + L::C_B + c, p);
                tmem_ld32(lane_base + L::C_A + c, z);
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const float a = tanh_fast(z[u] + sb1[c + u]);
                    p[u] *= 1.f - a * a;
                }
#pragma unroll
                for (int u = 0; u < 32; u += 8) st_chunk2(act_hi, act_lo, TM, row, c + u, &p[u]);
            }
            if (handoff()) { failed = true; break; }
            // dE/dx = g1 W1 (MN-major view of W1), into A
            if (gt == 0) {
                fence_after();
                gemm2<KPAD, H1, true, H1>(tmem + L::C_A, sa(act_hi), sa(act_lo), base + L::W1);
                mma_commit(bar);
            }
            // while the product runs: this warp's A rows for G = dE/dA = 2 w_tau A
            // dE/drho (warp per row, lanes along the row in the edge kernels'
            // lane-interleaved order, contiguous stores), RQ rows per pass
            constexpr int WARPS = TC_GROUP / 32, RQ = 8;
            const float *ag = A + (int64_t)r0 * NA;
            float *go = Gout + (int64_t)r0 * NA;
            float av[RQ][NJ];
            auto load_rows = [&](int rb) {
#pragma unroll
                for (int q = 0; q < RQ; ++q) {
                    const int rk = rb + q * WARPS;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int pk = (tid & 31) + 32 * j;
                        av[q][j] = (rk < rows && pk < NA) ? ag[(int64_t)rk * NA + (posj[j] & 255)] : 0.f;
                    }
                }
            };
            load_rows(gw);
            wait_mma();
            // dE/drho = (g1 W1) / scale, rows through ACT (consumed by the last product)
            float *gxs = stage;
#pragma unroll
            for (int c8 = 0; c8 < 16; c8 += 8) {
                float v[8];
                tmem_ld8(lane_base + L::C_A + 16 * h + c8, v);
#pragma unroll
                for (int u = 0; u < 8; ++u) gxs[row * L::GXS + 16 * h + c8 + u] = v[u] * sinv[16 * h + c8 + u];
            }
            group_sync(g);
            for (int rb = gw; rb < rows; rb += RQ * WARPS) {
                if (rb != gw) load_rows(rb);
#pragma unroll
                for (int q = 0; q < RQ; ++q) {
                    const int rk = rb + q * WARPS;
                    if (rk >= rows) break;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int pk = (tid & 31) + 32 * j;
                        const int c = posj[j];
                        if (pk < NA)
                            go[(int64_t)rk * NA + pk] =
                                ((c >> 16) ? 4.f : 2.f) * av[q][j] * gxs[rk * L::GXS + ((c >> 8) & 255)];
                    }
                }
            }
        }
        // the next tile's input staging overwrites ACT: all of this tile's reads are done
        fence_before();
        if (group_or(g, bad)) { failed = true; break; }
    }

    // a copy still in flight (a group that left early) lands before the block exits
    if (copy_pending) bar_wait(cbar, cphase & 1u);
    if (failed && gt == 0) atomicOr(status, ST_TIMEOUT);
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*tmem_slot),
                                "r"(TMEM_COLS));
}

template <int NP, int H1, int H2, int MODE>
cudaError_t run_tc(reann_ctx *c, const TcNets &nets, const float *X, float *Y, const float *dY, float *Ei,
                   const float *A, float *G, cudaStream_t s) {
    using L = TcLayout<NP, H1, H2, MODE>;
    static_assert(L::bytes > 116 * 1024 && L::bytes <= 227 * 1024, "one block per SM keeps TMEM allocation safe");
    static_assert((NA_BYTES<NP>() % 16) == 0, "A rows must be whole 16-byte units for the L2 prefetch");
    static bool configured[64] = {};
    auto kern = k_mlp_tc<NP, H1, H2, MODE>;
    if (c->device < 0 || c->device >= 64) return cudaErrorInvalidDevice;
    if (!configured[c->device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::bytes);
        if (e) return e;
        configured[c->device] = true;
    }
    if (c->n_tc_ranges == 0) return cudaSuccess;
    REANN_TIMED(c, MODE == TC_FWD ? REANN_K_MLP_FWD : (MODE == TC_ENERGY ? REANN_K_MLP_ENERGY : REANN_K_MLP_BWD), s);
    kern<<<c->n_tc_ranges, TC_THREADS, L::bytes, s>>>(c->d_tiles128, c->d_tiles128 + c->n_tiles128, c->d_w, nets, X,
                                                      Y, dY, Ei, A, G, c->d_status);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t dispatch_tc(reann_ctx *c, const TcNets &nets, const float *X, float *Y, const float *dY, float *Ei,
                        const float *A, float *G, cudaStream_t s) {
    if (c->NP == 8 && c->H1 == 128 && c->H2 == 128) return run_tc<8, 128, 128, MODE>(c, nets, X, Y, dY, Ei, A, G, s);
    if (c->NP == 10 && c->H1 == 128 && c->H2 == 128) return run_tc<10, 128, 128, MODE>(c, nets, X, Y, dY, Ei, A, G, s);
    return cudaErrorInvalidValue;
}

TcNets tc_nets(const std::vector<NetOffsets> &v, int first, int ne, int NP, int layer) {
    TcNets m;
    m.g_pairs = g_pairs(NP, layer);
    for (int e = 0; e < ne; ++e) m.net[e] = v[first + e];
    return m;
}

}  // namespace

cudaError_t launch_mlp_tc_coef_fwd(reann_ctx *c, int t, cudaStream_t s) {
    const int64_t nD = c->n * c->D;
    return dispatch_tc<TC_FWD>(c, tc_nets(c->coef_nets, t * c->ne, c->ne, c->NP, 0), c->d_rho + t * nD,
                               c->d_coef + (t + 1) * c->n_slots * c->D, nullptr, nullptr, nullptr, nullptr, s);
}

cudaError_t launch_mlp_tc_energy(reann_ctx *c, cudaStream_t s) {
    const int64_t nD = c->n * c->D, nA = c->n * c->NA;
    const int t = c->T - 1;
    return dispatch_tc<TC_ENERGY>(c, tc_nets(c->energy_nets, 0, c->ne, c->NP, c->T - 1), c->d_rho + t * nD, nullptr,
                                  nullptr, c->d_Ei, c->d_A + t * nA, c->d_G, s);
}

cudaError_t launch_mlp_tc_coef_bwd(reann_ctx *c, int t, cudaStream_t s) {
    const int64_t nD = c->n * c->D, nA = c->n * c->NA;
    return dispatch_tc<TC_BWD>(c, tc_nets(c->coef_nets, (t - 1) * c->ne, c->ne, c->NP, t - 1), c->d_rho + (t - 1) * nD,
                               nullptr, c->d_dc, nullptr, c->d_A + (t - 1) * nA, c->d_G, s);
}

}  // namespace reann
