// tcgen05 building blocks shared by the tensor-core network kernels
// (mlp_tc.cu, mlp_tc_pair.cu, mlp_tc32.cu): shared-memory and instruction
// descriptors, the split-bf16 and three-pass tf32 GEMMs issued by one thread,
// MMA completion on an mbarrier with a bounded wait, TMEM loads, the L2
// prefetch of global ranges, and the hi/lo operand stores.
//
// Shared-memory operand layout (K-major, no swizzle): an R x K bf16 tile keeps
// element (r, k) at byte (k/8) R 16 + (r/8) 128 + (r%8) 16 + (k%8) 2, i.e.
// 8-row x 16-byte core matrices, 128 B between 8-row groups (SBO) and R*16 B
// between 16-byte K chunks (LBO).
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"

namespace reann {
namespace {

constexpr int TM = 128;            // atoms per tile (MMA M)
constexpr int KPAD = 32;           // feature dimension padded to a multiple of 16
constexpr int TMEM_COLS = 512;

enum { TC_FWD = 0, TC_ENERGY = 1, TC_BWD = 2 };

template <int NP>
__host__ __device__ constexpr int NA_BYTES() { return NP * NT * 4; }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t kmaj(int r, int k, int R) {
    return (uint32_t)((k >> 3) * (R * 16) + (r >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
}

// shared-memory matrix descriptor: start, LBO, SBO (bytes), version 1, no swizzle
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, M = 128
__host__ __device__ constexpr uint32_t idesc_bf16(int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// D[128 x N] (+)= (A_hi + A_lo)[128 x K] B^T over two passes (split bf16
// activations, exact bf16 weights).  B is either a canonical K-major N x K tile
// (BT = false) or, BT = true, the MN-major view of a stored K-major tile with
// R_B = K rows and N columns: the same bytes, read transposed.  For that view
// the 16-byte chunks run along N (stride R_B*16 between chunk groups, the SBO)
// and 8-row groups run along K (stride 128, the LBO).
template <int N, int K, bool BT, int RB>
__device__ __forceinline__ void gemm2(uint32_t d_tmem, uint32_t a_hi, uint32_t a_lo, uint32_t b_smem) {
    constexpr uint32_t idesc = idesc_bf16(N) | (BT ? (1u << 16) : 0u);
    uint32_t acc = 0;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        const uint32_t a_smem = pass == 0 ? a_hi : a_lo;
#pragma unroll
        for (int s = 0; s < K / 16; ++s) {
            uint64_t a = sdesc(a_smem + (uint32_t)(2 * s * TM * 16), TM * 16, 128);
            uint64_t b = BT ? sdesc(b_smem + (uint32_t)(256 * s), 128, RB * 16)
                            : sdesc(b_smem + (uint32_t)(2 * s * N * 16), N * 16, 128);
            mma_bf16(d_tmem, a, b, idesc, acc);
            acc = 1;
        }
    }
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// bounded wait for the barrier phase with the given parity
__device__ __forceinline__ bool bar_wait(uint64_t *bar, uint32_t parity) {
    uint32_t a = smem_u32(bar);
    for (int it = 0; it < (1 << 20); ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(a), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}

// 32 consecutive fp32 TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    // the wait names the loaded registers, so no use of them is scheduled before it
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
}

__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 8 values (columns c..c+7 of row r) as a bf16 pair, hi = bf16(v) and
// lo = bf16(v - hi) (16 significant bits), into one 16-byte chunk of each
// K-major tile.  Rounding to bf16 is done on the bit pattern (add half a bf16
// ulp, keep the upper 16 bits: round to nearest, ties away from zero), which
// runs on the integer pipe; v - hi is exact in fp32.
__device__ __forceinline__ void st_chunk2(unsigned char *hi, unsigned char *lo, int R, int r, int c, const float *v) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int u = 0; u < 8; u += 2) {
        const uint32_t a = __float_as_uint(v[u]) + 0x8000u, b = __float_as_uint(v[u + 1]) + 0x8000u;
        const float la = v[u] - __uint_as_float(a & 0xFFFF0000u);
        const float lb = v[u + 1] - __uint_as_float(b & 0xFFFF0000u);
        h[u / 2] = __byte_perm(a, b, 0x7632);
        l[u / 2] = __byte_perm(__float_as_uint(la) + 0x8000u, __float_as_uint(lb) + 0x8000u, 0x7632);
    }
    const uint32_t off = kmaj(r, c, R);
    *reinterpret_cast<uint4 *>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4 *>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

// one bf16 element of a K-major tile (weight preparation)
__device__ __forceinline__ void st_elem(unsigned char *tile, int R, int r, int k, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(tile + kmaj(r, k, R)) = __float2bfloat16_rn(x);
}

struct TcNets {
    NetOffsets net[MAX_ELEMENTS];
    int g_pairs;   // lane order of the dE/dA rows written (g_pairs of their layer)
};

// 8 consecutive fp32 TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = __uint_as_float(r[k]);
}

// L2 prefetch of a contiguous global range (bulk, no shared-memory destination);
// address 16-byte aligned, size a multiple of 16
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// L2 prefetch of the whole 16-byte units inside [p, p + bytes) (the bulk
// prefetch takes 16-byte aligned spans)
__device__ __forceinline__ void prefetch_l2_span(const void *p, size_t bytes) {
    const uintptr_t a = ((uintptr_t)p + 15) & ~(uintptr_t)15, e = ((uintptr_t)p + bytes) & ~(uintptr_t)15;
    if (e > a) prefetch_l2(reinterpret_cast<const void *>(a), (uint32_t)(e - a));
}

}  // namespace
}  // namespace reann

// ---------------------------------------------------------------------------
// fp32-accurate products on the tf32 tensor-core path (kind::tf32).  Operands
// are fp32 containers in shared memory whose low 13 mantissa bits are zero:
// every value v is stored as hi = tf32(v) and lo = tf32(v - hi), both rounded
// to nearest, so hi + lo carries 22 significant bits.  A product is three
// passes into one fp32 accumulator, A_hi B_hi + A_lo B_hi + A_hi B_lo (the
// dropped A_lo B_lo is below 2^-24 of the product).  Tile layout as above with
// 4-byte elements: an R x K tile keeps (r, k) at byte
// (k/4) R 16 + (r/8) 128 + (r%8) 16 + (k%4) 4, and one K = 8 instruction step
// covers two 16-byte chunks, exactly as one K = 16 step of bf16 does.
namespace reann {
namespace {

// instruction descriptor, kind::tf32: D fp32, A and B tf32, M = 128
__host__ __device__ constexpr uint32_t idesc_tf32(int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ uint32_t kmaj32(int r, int k, int R) {
    return (uint32_t)((k >> 2) * (R * 16) + (r >> 3) * 128 + (r & 7) * 16 + (k & 3) * 4);
}

// D[128 x N] = A B^T, A = A_hi + A_lo and B = B_hi + B_lo, both K-major
// (B an N x K tile), in three passes.  The two small passes run first: the
// accumulator then receives the large products last, which measured 3x
// closer to an fp32 FMA chain (rms error 1.6e-7 vs 4.8e-7 of the result's
// scale) than the reverse order.  (The MN-major descriptor view of a tf32
// tile, which would let one tile serve both orientations, produced zeros on
// this part; the vector-Jacobian products use transposed copies instead.)
template <int N, int K>
__device__ __forceinline__ void gemm3_tf32(uint32_t d_tmem, uint32_t a_hi, uint32_t a_lo, uint32_t b_hi,
                                           uint32_t b_lo) {
    constexpr uint32_t idesc = idesc_tf32(N);
    uint32_t acc = 0;
#pragma unroll
    for (int pass = 0; pass < 3; ++pass) {
        const uint32_t a_smem = pass == 0 ? a_lo : a_hi;
        const uint32_t b_smem = pass == 1 ? b_lo : b_hi;
#pragma unroll
        for (int s = 0; s < K / 8; ++s) {
            uint64_t a = sdesc(a_smem + (uint32_t)(2 * s * TM * 16), TM * 16, 128);
            uint64_t b = sdesc(b_smem + (uint32_t)(2 * s * N * 16), N * 16, 128);
            mma_tf32(d_tmem, a, b, idesc, acc);
            acc = 1;
        }
    }
}

// tf32 value nearest to v (ties away from zero), as fp32 bits
__device__ __forceinline__ uint32_t tf32_rn(float v) { return (__float_as_uint(v) + 0x1000u) & 0xFFFFE000u; }

// 4 values (columns c..c+3 of row r) as hi = tf32(v), lo = tf32(v - hi) into one
// 16-byte chunk of each plane; integer instructions except the exact subtraction
__device__ __forceinline__ void st_chunk4_tf32(unsigned char *hi, unsigned char *lo, int R, int r, int c,
                                               const float *v) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        h[u] = tf32_rn(v[u]);
        l[u] = tf32_rn(v[u] - __uint_as_float(h[u]));
    }
    const uint32_t off = kmaj32(r, c, R);
    *reinterpret_cast<uint4 *>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4 *>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

// one weight element split into the hi and lo planes of a K-major tile
__device__ __forceinline__ void st_elem_tf32(unsigned char *hi, unsigned char *lo, int R, int r, int k, float x) {
    const uint32_t off = kmaj32(r, k, R), h = tf32_rn(x);
    *reinterpret_cast<uint32_t *>(hi + off) = h;
    *reinterpret_cast<uint32_t *>(lo + off) = tf32_rn(x - __uint_as_float(h));
}

// tanh to fp32 accuracy in absolute terms, 1 - 2 / (exp(2|x|) + 1) with the
// sign of x: the exponential and the reciprocal on the special-function unit;
// the absolute error stays at the fp32 rounding level of the result (what the
// next product sees), and large |x| saturates to +-1 without overflow trouble
__device__ __forceinline__ float tanh_f32(float x) {
    const float e = __expf(2.f * fabsf(x));
    return copysignf(1.f - __fdividef(2.f, e + 1.f), x);
}

}  // namespace
}  // namespace reann
