// Per-element atomic networks at fp32 accuracy on the 5th-generation tensor
// cores (tcgen05, kind::tf32): hidden widths [64, 64], square-form densities.
//
// Same networks as mlp.cu and mlp_tc.cu ("Efficient Parallelization of Message
// Passing Neural Network Potentials for Large-Scale Molecular Dynamics",
// section "REANN Architecture", Eq. 2 and the atomic energy; section
// "Parallelization Algorithm", Eqs. 3 and 5 for the vector-Jacobian products):
//   y = W3 tanh(W2 tanh(W1 ((x - shift) / scale) + b1) + b2) + b3.
// Every operand -- fp32 weights and fp32 activations alike -- enters a product
// as a pair of tf32 values (hi + lo, 22 significant bits), and each product is
// three tf32 passes into one fp32 accumulator in tensor memory (tc_common.cuh),
// which agrees with fp32 arithmetic to its rounding level -- what the fp32
// path's 1e-4 eV/A force tolerance needs (16-bit operands, as in the bf16
// path, do not meet it).  tanh is evaluated to fp32 accuracy from the
// exponential (tanh.approx, accurate to about 11 bits, is not used here).
//
// Three launches per layer, as on the other network paths:
//   forward (coefficient networks): x -> c^{t+1}; the derivatives
//     tanh'(z1), tanh'(z2) of every atom are written out for the backward
//     (one column-major block per tile, so a warp's accesses are contiguous);
//   energy: E_i and dE/dA of the last layer (forward and VJP in one pass);
//   backward (coefficient networks): dE/dc^{t+1} -> dE/dA^t from the stored
//     derivative rows -- three products, no recomputed forward.
// The VJP products read transposed copies of the weight tiles (K-major, as
// every operand here); each launch loads only the orientations it uses.
//
// A tile is 128 atoms of one element; TMEM lane i holds atom i.  Block: 512
// threads, one per SM, on a contiguous range of one element's tiles (weights
// loaded once), split into two independent groups of 256 threads that take
// every other tile with their own 256 TMEM columns, operand planes,
// MMA-completion mbarrier and named barrier, so one group's epilogue overlaps
// the other's products.  In a group, warp w reads TMEM lanes 32 (w % 4) .. + 31
// and half h = (w / 4) % 2 takes columns 32 h .. 32 h + 31 of every 64-wide
// accumulator.  MMA-completion waits are bounded: a wait that gives up sets
// ST_TIMEOUT and the block frees its tensor memory and returns.
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace reann {
namespace {

constexpr int T32_THREADS = 512;   // two independent groups of 256 threads
constexpr int T32_GROUP = 256;
constexpr int H = 64;              // hidden width of both layers

__device__ __forceinline__ void grp_sync(int g) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(T32_GROUP) : "memory");
}
__device__ __forceinline__ bool grp_or(int g, bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, o;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred o, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, o;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(1 + g), "r"(T32_GROUP)
        : "memory");
    return r != 0;
}

// Shared memory of one launch: the weight tiles its products read (K-major,
// fp32 tf32 values, hi plane then lo plane each), the fp32 vectors, then the
// two groups.  Tiles (rows x K):
//   W1  [H][KPAD]  W1[h][f]        z1 = x W1^T           (forward, energy)
//   W2  [H][H]     W2[h2][h1]      z2 = a1 W2^T          (forward, energy)
//   W3  [KPAD][H]  W3[o][h]        y  = a2 W3^T          (forward)
//   W3T [H][KPAD]  W3[o][h] at (h, o)   u  = dY W3       (backward)
//   W2T [H][H]     W2[h2][h1] at (h1, h2) p1 = g2 W2     (energy, backward)
//   W1T [KPAD][H]  W1[h][f] at (f, h)   dx = g1 W1       (energy, backward)
template <int MODE>
struct T32Layout {
    static constexpr int SQ = H * KPAD * 4;             // one plane of an [H][KPAD] or [KPAD][H] tile
    static constexpr int HH = H * H * 4;                // one plane of an [H][H] tile
    static constexpr bool FWD = MODE == TC_FWD, EN = MODE == TC_ENERGY, BW = MODE == TC_BWD;
    static constexpr int W1 = 0;
    static constexpr int W2 = W1 + (FWD || EN ? 2 * SQ : 0);
    static constexpr int W3 = W2 + (FWD || EN ? 2 * HH : 0);
    static constexpr int W3T = W3 + (FWD ? 2 * SQ : 0);
    static constexpr int W2T = W3T + (BW ? 2 * SQ : 0);
    static constexpr int W1T = W2T + (EN || BW ? 2 * HH : 0);
    static constexpr int F32 = W1T + (EN || BW ? 2 * SQ : 0);
    static constexpr int nf32 = H + H + KPAD + KPAD + KPAD + H;   // b1, b2, b3, shift, scale, w3
    static constexpr int GRP = (F32 + nf32 * 4 + 127) / 128 * 128;
    // per group: ACT holds the operand of the product in flight, hi plane then
    // lo plane: first the [TM][KPAD] input (x, or dY in the backward), then
    // the [TM][H] activations and gradients; once a tile's last product has
    // completed it stages the output rows
    static constexpr int ACT = 0;
    static constexpr int X_PLANE = TM * KPAD * 4;       // 16 KB
    static constexpr int ACT_PLANE = TM * H * 4;        // 32 KB
    static constexpr int SE = ACT + 2 * ACT_PLANE;      // energy partials of the upper column half [TM]
    static constexpr int BAR = SE + TM * 4;
    static constexpr int GROUP_BYTES = BAR + 16;
    static constexpr int SLOT = GRP + 2 * GROUP_BYTES;
    static constexpr int bytes = SLOT + 16;
    static constexpr int RS = KPAD + 1;                 // stride of staged output rows (odd)
    static_assert(TM * RS * 4 <= SE, "output rows fit the activation planes");
    static_assert(2 * X_PLANE + TM * RS * 4 <= SE, "raw input rows fit beside the input planes");
    static_assert(GROUP_BYTES % 16 == 0 && GRP % 16 == 0, "16-byte aligned operand planes");
    // TMEM columns of a group (base 256 g)
    static constexpr int C_A = 0, C_B = 64, C_C = 128;
};

// this thread's 32 derivative values of one layer (its row, columns 32 h ..
// + 31), stored column-major inside the tile: column c of the tile's rows at
// c * rows, so a warp's 32 rows of one column are 32 consecutive floats
__device__ __forceinline__ void store_cols(float *dst, int stride, const float (&v)[32]) {
#pragma unroll
    for (int u = 0; u < 32; ++u) dst[(int64_t)u * stride] = v[u];
}
__device__ __forceinline__ void load_cols(const float *src, int stride, float (&v)[32]) {
#pragma unroll
    for (int u = 0; u < 32; ++u) v[u] = __ldg(src + (int64_t)u * stride);
}

template <int NP, int MODE>
__global__ void __launch_bounds__(T32_THREADS, 1)
    k_mlp_tc32(const int4 *__restrict__ tiles, const int4 *__restrict__ ranges, const float *__restrict__ w,
               TcNets nets, const float *__restrict__ X, float *__restrict__ Y, const float *__restrict__ dY,
               float *__restrict__ Ei, const float *__restrict__ A, float *__restrict__ Gout,
               float *__restrict__ Dt, int *__restrict__ status) {
    using L = T32Layout<MODE>;
    constexpr int D = 3 * NP, NA = NP * NT;
    constexpr int DOUT = MODE == TC_ENERGY ? 1 : D;
    static_assert(D <= KPAD, "features fit the padded width");
    extern __shared__ __align__(1024) unsigned char sm[];
    float *f32 = reinterpret_cast<float *>(sm + L::F32);
    float *sb1 = f32, *sb2 = sb1 + H, *sb3 = sb2 + H, *sshift = sb3 + KPAD, *sscale = sshift + KPAD,
          *sw3 = sscale + KPAD;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int g = tid / T32_GROUP, gt = tid - g * T32_GROUP, gw = gt >> 5;
    const int row = gt & (TM - 1);    // this thread's atom in the tile (TMEM lane)
    const int h = gt / TM;            // column half
    unsigned char *gs = sm + L::GRP + g * L::GROUP_BYTES;
    unsigned char *x_hi = gs + L::ACT, *x_lo = x_hi + L::X_PLANE;
    unsigned char *act_hi = gs + L::ACT, *act_lo = act_hi + L::ACT_PLANE;
    float *stage = reinterpret_cast<float *>(gs + L::ACT);
    float *se = reinterpret_cast<float *>(gs + L::SE);
    uint64_t *bar = reinterpret_cast<uint64_t *>(gs + L::BAR);
    const uint32_t base = smem_u32(sm);
    auto sa = [&](const unsigned char *p) { return base + (uint32_t)(p - sm); };
    auto hi_of = [&](int off) { return base + (uint32_t)off; };

    const int4 rg = ranges[blockIdx.x];   // (first tile, end tile, element, -)
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (gt == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    {
        // the block's element: the weight tiles this launch reads, split tf32 hi/lo
        const NetOffsets &o = nets.net[rg.z];
        for (int k = tid; k < H * KPAD; k += T32_THREADS) {
            const int a = k / KPAD, f = k % KPAD;   // hidden index, feature index
            const float w1 = f < D ? w[o.W1 + (int64_t)a * D + f] : 0.f;
            const float w3 = f < DOUT ? w[o.W3 + (int64_t)f * H + a] : 0.f;
            if (L::FWD || L::EN) st_elem_tf32(sm + L::W1, sm + L::W1 + L::SQ, H, a, f, w1);
            if (L::FWD) st_elem_tf32(sm + L::W3, sm + L::W3 + L::SQ, KPAD, f, a, w3);
            if (L::BW) st_elem_tf32(sm + L::W3T, sm + L::W3T + L::SQ, H, a, f, w3);
            if (L::EN || L::BW) st_elem_tf32(sm + L::W1T, sm + L::W1T + L::SQ, KPAD, f, a, w1);
        }
        for (int k = tid; k < H * H; k += T32_THREADS) {
            const int r = k / H, c = k % H;
            const float v = w[o.W2 + k];   // W2[r][c]
            if (L::FWD || L::EN) st_elem_tf32(sm + L::W2, sm + L::W2 + L::HH, H, r, c, v);
            if (L::EN || L::BW) st_elem_tf32(sm + L::W2T, sm + L::W2T + L::HH, H, c, r, v);
        }
        for (int k = tid; k < H; k += T32_THREADS) {
            sb1[k] = w[o.b1 + k];
            sb2[k] = w[o.b2 + k];
            sw3[k] = MODE == TC_ENERGY ? w[o.W3 + k] : 0.f;
        }
        for (int k = tid; k < KPAD; k += T32_THREADS) {
            sb3[k] = k < DOUT ? w[o.b3 + k] : 0.f;
            sshift[k] = k < D ? w[o.shift + k] : 0.f;
            sscale[k] = k < D ? w[o.scale + k] : 1.f;
        }
    }
    fence_smem_to_async();
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot + (uint32_t)(256 * g);
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint32_t phase = 0;
    bool failed = false;

    auto wait_mma = [&]() -> bool {
        const bool ok = bar_wait(bar, phase);
        phase ^= 1u;
        fence_after();
        return !grp_or(g, !ok);
    };
    auto handoff = [&]() {
        fence_smem_to_async();
        fence_before();
        grp_sync(g);
    };
    // one product into TMEM columns `col`, issued by the group's thread 0
    auto product = [&](int col, auto gemm) -> bool {
        if (gt == 0) {
            fence_after();
            gemm(tmem + (uint32_t)col);
            mma_commit(bar);
        }
        return wait_mma();
    };

    // dE/dA positions of this lane in the edge kernels' lane-interleaved row
    // order: source A index (bits 0-7), dE/drho index (bits 8-15), mixed
    // second-order tuple (bit 16: 2 w_tau = 4)
    constexpr int NJ = (NA + 31) / 32;
    int posj[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int pk = (tid & 31) + 32 * j;
        const int src = g_slot_source(pk < NA ? pk : 0, NP, nets.g_pairs), nn = src / NT, u = src - nn * NT;
        const int gi = (u == 0 ? 0 : (u < 4 ? 1 : 2)) * NP + nn;
        posj[j] = src | (gi << 8) | ((u >= 7 ? 1 : 0) << 16);
    }

    for (int ti = rg.x + g; ti < rg.y && !failed; ti += 2) {
        const int4 tile = tiles[ti];
        const int r0 = tile.y, rows = tile.z;
        const bool live = row < rows;
        // the tile's derivative block [2H][rows] at Dt + r0 2H: tanh'(z1) in columns
        // [0, H), tanh'(z2) in [H, 2H); this thread's first column 32 h
        float *dt_col = Dt + (int64_t)r0 * (2 * H) + (int64_t)(32 * h) * rows + row;
        if (MODE != TC_FWD && gt == 0) prefetch_l2(A + (int64_t)r0 * NA, (uint32_t)(rows * NA * 4));
        // input: the tile's contiguous raw rows (x, or dY in the backward) in
        // element order into padded rows in the free half of the activation
        // planes, then this thread's 16 features (x standardised), split tf32
        {
            float *xs = reinterpret_cast<float *>(gs + L::ACT + 2 * L::X_PLANE);
            const float *src = (MODE == TC_BWD ? dY : X) + (int64_t)r0 * D;
            for (int k = gt; k < rows * D; k += T32_GROUP) {
                const int rk = k / D, f = k - rk * D;
                xs[rk * L::RS + f] = src[k];
            }
            grp_sync(g);
#pragma unroll
            for (int c4 = 0; c4 < 16; c4 += 4) {
                float v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int f = 16 * h + c4 + u;
                    const bool ok = live && f < D;
                    const float x = ok ? xs[row * L::RS + f] : 0.f;
                    v[u] = !ok ? 0.f : (MODE == TC_BWD ? x : (x - sshift[f]) / sscale[f]);
                }
                st_chunk4_tf32(x_hi, x_lo, TM, row, 16 * h + c4, v);
            }
        }
        handoff();

        float d1[32];   // tanh'(z1) of this thread's columns (energy and backward)
        if (MODE == TC_BWD) {
            // u = dY W3 into A, then g2 = u tanh'(z2) (stored by the forward)
            float d2[32];
            if (live) load_cols(dt_col + H * rows, rows, d2);
            if (live) load_cols(dt_col, rows, d1);
            if (!product(L::C_A, [&](uint32_t d) { gemm3_tf32<H, KPAD>(d, sa(x_hi), sa(x_lo), hi_of(L::W3T),
                                                                         hi_of(L::W3T + L::SQ)); })) {
                failed = true;
                break;
            }
            float v[32];
            tmem_ld32(lane_base + L::C_A + 32 * h, v);
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = live ? v[u] * d2[u] : 0.f;
#pragma unroll
            for (int u = 0; u < 32; u += 4) st_chunk4_tf32(act_hi, act_lo, TM, row, 32 * h + u, &v[u]);
        } else {
            // layer 1: z1 = x W1^T into A; a1 = tanh(z1 + b1)
            if (!product(L::C_A, [&](uint32_t d) { gemm3_tf32<H, KPAD>(d, sa(x_hi), sa(x_lo), hi_of(L::W1),
                                                                         hi_of(L::W1 + L::SQ)); })) {
                failed = true;
                break;
            }
            float v[32];
            tmem_ld32(lane_base + L::C_A + 32 * h, v);
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                v[u] = tanh_f32(v[u] + sb1[32 * h + u]);
                d1[u] = 1.f - v[u] * v[u];
            }
            if (MODE == TC_FWD && live) store_cols(dt_col, rows, d1);
#pragma unroll
            for (int u = 0; u < 32; u += 4) st_chunk4_tf32(act_hi, act_lo, TM, row, 32 * h + u, &v[u]);
            handoff();
            // layer 2: z2 = a1 W2^T into B
            if (!product(L::C_B, [&](uint32_t d) { gemm3_tf32<H, H>(d, sa(act_hi), sa(act_lo), hi_of(L::W2),
                                                                      hi_of(L::W2 + L::HH)); })) {
                failed = true;
                break;
            }
            tmem_ld32(lane_base + L::C_B + 32 * h, v);
            float e_row = 0.f;
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const float a = tanh_f32(v[u] + sb2[32 * h + u]);
                if (MODE == TC_FWD) {
                    v[u] = a;
                } else {
                    // g2 = dE/dz2 = w3 (1 - a2^2); E_i = w3 . a2 + b3
                    e_row = fmaf(sw3[32 * h + u], a, e_row);
                    v[u] = sw3[32 * h + u] * (1.f - a * a);
                }
            }
            if (MODE == TC_FWD && live) {
                float d2[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) d2[u] = 1.f - v[u] * v[u];
                store_cols(dt_col + H * rows, rows, d2);
            }
#pragma unroll
            for (int u = 0; u < 32; u += 4) st_chunk4_tf32(act_hi, act_lo, TM, row, 32 * h + u, &v[u]);
            if (MODE == TC_ENERGY && h == 1) se[row] = e_row;
            handoff();
            if (MODE == TC_ENERGY && h == 0 && live) Ei[r0 + row] = (e_row + se[row]) + sb3[0];
        }

        if (MODE == TC_FWD) {
            // y = a2 W3^T + b3 (into C), rows through the free activation planes
            if (!product(L::C_C, [&](uint32_t d) { gemm3_tf32<KPAD, H>(d, sa(act_hi), sa(act_lo), hi_of(L::W3),
                                                                         hi_of(L::W3 + L::SQ)); })) {
                failed = true;
                break;
            }
#pragma unroll
            for (int c8 = 0; c8 < 16; c8 += 8) {
                float v[8];
                tmem_ld8(lane_base + L::C_C + 16 * h + c8, v);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int f = 16 * h + c8 + u;
                    if (f < D) stage[row * L::RS + f] = v[u] + sb3[f];
                }
            }
            grp_sync(g);
            float *yo = Y + (int64_t)r0 * D;
            for (int k = gt; k < rows * D; k += T32_GROUP) {
                const int rk = k / D;
                yo[k] = stage[rk * L::RS + (k - rk * D)];
            }
        } else {
            if (MODE == TC_BWD) handoff();
            // p1 = g2 W2 (into B), g1 = p1 tanh'(z1)
            if (!product(L::C_B, [&](uint32_t d) { gemm3_tf32<H, H>(d, sa(act_hi), sa(act_lo), hi_of(L::W2T),
                                                                      hi_of(L::W2T + L::HH)); })) {
                failed = true;
                break;
            }
            {
                float p[32];
                tmem_ld32(lane_base + L::C_B + 32 * h, p);
#pragma unroll
                for (int u = 0; u < 32; ++u) p[u] = live ? p[u] * d1[u] : 0.f;
#pragma unroll
                for (int u = 0; u < 32; u += 4) st_chunk4_tf32(act_hi, act_lo, TM, row, 32 * h + u, &p[u]);
            }
            handoff();
            // dE/dx = g1 W1 (into C); dE/drho = (g1 W1) / scale, rows through the free planes
            if (!product(L::C_C, [&](uint32_t d) { gemm3_tf32<KPAD, H>(d, sa(act_hi), sa(act_lo), hi_of(L::W1T),
                                                                         hi_of(L::W1T + L::SQ)); })) {
                failed = true;
                break;
            }
            float *gxs = stage;
#pragma unroll
            for (int c8 = 0; c8 < 16; c8 += 8) {
                float v[8];
                tmem_ld8(lane_base + L::C_C + 16 * h + c8, v);
#pragma unroll
                for (int u = 0; u < 8; ++u) gxs[row * L::RS + 16 * h + c8 + u] = v[u] / sscale[16 * h + c8 + u];
            }
            grp_sync(g);
            // G = dE/dA = 2 w_tau A dE/drho, warp per row in the edge kernels'
            // lane-interleaved order; four rows' A values loaded before any is used
            const float *ag = A + (int64_t)r0 * NA;
            float *go = Gout + (int64_t)r0 * NA;
            for (int rb = gw; rb < rows; rb += 4 * (T32_GROUP / 32)) {
                float av[4][NJ];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int rk = rb + q * (T32_GROUP / 32);
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int pk = (tid & 31) + 32 * j;
                        av[q][j] = (rk < rows && pk < NA) ? ag[(int64_t)rk * NA + (posj[j] & 255)] : 0.f;
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int rk = rb + q * (T32_GROUP / 32);
                    if (rk >= rows) break;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int pk = (tid & 31) + 32 * j;
                        const int c = posj[j];
                        if (pk < NA)
                            go[(int64_t)rk * NA + pk] =
                                ((c >> 16) ? 4.f : 2.f) * av[q][j] * gxs[rk * L::RS + ((c >> 8) & 255)];
                    }
                }
            }
        }
        // the next tile's operands overwrite the planes: this tile's reads are done
        fence_before();
        grp_sync(g);
    }

    if (failed && gt == 0) atomicOr(status, ST_TIMEOUT);
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*tmem_slot),
                                "r"(TMEM_COLS));
}

template <int NP, int MODE>
cudaError_t run_tc32(reann_ctx *c, const TcNets &nets, const float *X, float *Y, const float *dY, float *Ei,
                     const float *A, float *G, float *Dt, cudaStream_t s) {
    using L = T32Layout<MODE>;
    static_assert(L::bytes > 116 * 1024 && L::bytes <= 227 * 1024, "one block per SM keeps TMEM allocation safe");
    static_assert((NA_BYTES<NP>() % 16) == 0, "A rows must be whole 16-byte units for the L2 prefetch");
    static bool configured[64] = {};
    auto kern = k_mlp_tc32<NP, MODE>;
    if (c->device < 0 || c->device >= 64) return cudaErrorInvalidDevice;
    if (!configured[c->device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::bytes);
        if (e) return e;
        configured[c->device] = true;
    }
    if (c->n_tc_ranges == 0) return cudaSuccess;
    REANN_TIMED(c, MODE == TC_FWD ? REANN_K_MLP_FWD : (MODE == TC_ENERGY ? REANN_K_MLP_ENERGY : REANN_K_MLP_BWD), s);
    kern<<<c->n_tc_ranges, T32_THREADS, L::bytes, s>>>(c->d_tiles128, c->d_tiles128 + c->n_tiles128, c->d_w, nets, X,
                                                        Y, dY, Ei, A, G, Dt, c->d_status);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t dispatch_tc32(reann_ctx *c, const TcNets &nets, const float *X, float *Y, const float *dY, float *Ei,
                          const float *A, float *G, float *Dt, cudaStream_t s) {
    if (c->H1 != H || c->H2 != H || !c->d_tanhd) return cudaErrorInvalidValue;
    if (c->NP == 8) return run_tc32<8, MODE>(c, nets, X, Y, dY, Ei, A, G, Dt, s);
    if (c->NP == 10) return run_tc32<10, MODE>(c, nets, X, Y, dY, Ei, A, G, Dt, s);
    return cudaErrorInvalidValue;
}

TcNets nets_of(const std::vector<NetOffsets> &v, int first, int ne, int NP, int layer) {
    TcNets m;
    m.g_pairs = g_pairs(NP, layer);
    for (int e = 0; e < ne; ++e) m.net[e] = v[first + e];
    return m;
}

}  // namespace

bool tc32_supported(const reann_ctx *c) {
    return c->H1 == H && c->H2 == H && (c->NP == 8 || c->NP == 10) && c->DR == c->D;
}

// tanh' of coefficient network t: n 2H values at d_tanhd + t n 2H, one
// column-major [2H][rows] block per 128-row tile at the tile's first row x 2H
static float *tanhd_rows(reann_ctx *c, int t) { return c->d_tanhd + (int64_t)t * c->n * (2 * H); }

cudaError_t launch_mlp_tc32_coef_fwd(reann_ctx *c, int t, cudaStream_t s) {
    const int64_t nD = c->n * c->D;
    return dispatch_tc32<TC_FWD>(c, nets_of(c->coef_nets, t * c->ne, c->ne, c->NP, 0), c->d_rho + t * nD,
                                 c->d_coef + (t + 1) * c->n_slots * c->D, nullptr, nullptr, nullptr, nullptr,
                                 tanhd_rows(c, t), s);
}

cudaError_t launch_mlp_tc32_energy(reann_ctx *c, cudaStream_t s) {
    const int64_t nD = c->n * c->D, nA = c->n * c->NA;
    const int t = c->T - 1;
    return dispatch_tc32<TC_ENERGY>(c, nets_of(c->energy_nets, 0, c->ne, c->NP, c->T - 1), c->d_rho + t * nD, nullptr,
                                    nullptr, c->d_Ei, c->d_A + t * nA, c->d_G, c->d_tanhd, s);
}

cudaError_t launch_mlp_tc32_coef_bwd(reann_ctx *c, int t, cudaStream_t s) {
    const int64_t nA = c->n * c->NA;
    return dispatch_tc32<TC_BWD>(c, nets_of(c->coef_nets, (t - 1) * c->ne, c->ne, c->NP, t - 1), nullptr, nullptr,
                                 c->d_dc, nullptr, c->d_A + (t - 1) * nA, c->d_G, tanhd_rows(c, t - 1), s);
}

}  // namespace reann
