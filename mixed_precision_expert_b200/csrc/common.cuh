// Device-side building blocks shared by the mpe kernels (sm_100a).
//
// Packed format (the library's own definition of PagedWeight's "pages of
// varying bit-widths"): a matrix [R x K] is cut into chunks of 16 rows x 128
// codes; chunk (tau, j) holds the 16 blocks of rows 16 tau .. 16 tau + 15 at
// block column j, 16 b bytes per block, rows in order. A block is four
// quarters of 32 codes (4 b bytes each). Inside a quarter the 32 offset-binary
// codes c'_0..c'_31 are b little-endian words:
//   b = 8: word w holds c'_{4w+i} at bit 16(i&1) + 8(i>>1), i < 4
//   b = 4: word w holds c'_{8w+i} at bit 16(i&1) + 4(i>>1), i < 8
//   b = 3: word v holds c'_{10v+i} at bit 16(i&1) + 3(i>>1), i < 10; bit n of
//          c'_30 / c'_31 is bit 15 / 31 of word n (n < 3)
// so each pair (c'_{2m}, c'_{2m+1}) sits in matching positions of the two
// 16-bit halves of a word and unpacks to one bf16x2 register.
// An expert stream is the chunks of W1 (gate [F x H]) and W3 (up [F x H])
// interleaved -- chunk 2c is W1's chunk c, 2c+1 is W3's -- then those of W2
// (down [H x F]) with each pair of row tiles interleaved -- tile 2v's chunk j at
// 2 (v nj + j), tile 2v+1's at 2 (v nj + j) + 1 (nj = F / 128). A tile's gate
// and up chunks, or a tile pair's down chunks, for consecutive block columns
// are therefore one contiguous run. Chunk c of an expert lives in page
// pidx[first + c / cpp] at byte (c % cpp) * 256 b, cpp = page_bytes / (256 b).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "mpe.h"

namespace mpe {

constexpr int kRowsPerChunk = 16;
constexpr int kCodesPerBlock = 128;

__host__ __device__ constexpr int chunk_bytes(int b) { return 256 * b; }
__host__ __device__ constexpr int block_bytes(int b) { return 16 * b; }
__host__ __device__ inline int chunks_per_page(int b, uint32_t page_bytes) {
    return (int)(page_bytes / (uint32_t)(256 * b));
}
__host__ __device__ constexpr int q_levels(int b) { return (1 << (b - 1)) - 1; }

// Device copy of one page-table entry (same layout as mpe_pte).
struct Pte {
    uint8_t bits;
    uint8_t pad[3];
    float scale;
    uint32_t first;
    uint32_t n_pages;
};
static_assert(sizeof(Pte) == sizeof(mpe_pte), "pte layout");

// What every kernel needs to reach an expert's pages.
struct PagedExperts {
    uint8_t* pool;
    const Pte* pte;
    const uint32_t* pidx;
    uint32_t page_bytes;
    int E, H, F;
};

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bit) {
    atomicOr(status, bit);
}

// chunks of one [F x H] matrix: the stream holds 2 of these interleaved (W1, W3),
// then W2's chunks (tile pairs interleaved) from index 2 * chunks_w1
__host__ __device__ inline int chunks_w1(int H, int F) { return (F / 16) * (H / 128); }

// Address of chunk c of an expert.
__device__ __forceinline__ const uint8_t* chunk_addr(const PagedExperts& P, const Pte& pte,
                                                     int b, int c) {
    const int cpp = chunks_per_page(b, P.page_bytes);
    const uint32_t page = P.pidx[pte.first + (uint32_t)(c / cpp)];
    return P.pool + (size_t)page * P.page_bytes + (size_t)(c % cpp) * chunk_bytes(b);
}

// ---------------------------------------------------------------------------
// the quantizer's rounding: k = round-half-even(w / s), exactly
// ---------------------------------------------------------------------------
// Rare path: r = w (1/s) lies within 2^-14 of a half-integer, so the exact
// quotient w / s decides. The sign of the single-rounded fma (k -+ 1/2) s - w is
// exact: ties go to the even integer.
static __device__ __noinline__ float tie_fix(float w, float s, float kf) {
    const float lo = __fmaf_rn(__fsub_rn(kf, 0.5f), s, -w);  // (k - 1/2) s - w
    const float hi = __fmaf_rn(__fadd_rn(kf, 0.5f), s, -w);  // (k + 1/2) s - w
    const bool odd = (((int)kf) & 1) != 0;
    if (lo > 0.0f) return __fsub_rn(kf, 1.0f);
    if (hi < 0.0f) return __fadd_rn(kf, 1.0f);
    if (lo == 0.0f && odd) return __fsub_rn(kf, 1.0f);
    if (hi == 0.0f && odd) return __fadd_rn(kf, 1.0f);
    return kf;
}

// Window of the exact repair. For |w / s| <= 127.00003 (|w| <= max|w|, s =
// RN(max|w| / q)) and inv_s = RN(1 / s), r = RN(w inv_s) has a relative error
// below 2^-23, so |r - w/s| < 127.00003 * 2^-23 < 2^-16. When |r - k| <= 1/2 -
// 2^-14 for the integer k nearest r, the exact quotient is within 1/2 - 2^-14 +
// 2^-16 < 1/2 of k, so k is its rounding; only codes closer than 2^-14 to a
// half-integer go to tie_fix (the window keeps a factor 4 over the bound).
constexpr float kNearTie = 0.49993896484375f;  // 1/2 - 2^-14

// k as a float for |w / s| < 2^8, s > 0, inv_s = RN(1 / s): adding 1.5 * 2^23
// rounds r = w inv_s to an integer (ties to even), which agrees with rounding
// the exact quotient unless r lies within 2^-14 of a half-integer, where
// tie_fix decides.
__device__ __forceinline__ float exact_code(float w, float s, float inv_s) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    const float r = __fmul_rn(w, inv_s);
    const float kf = __fsub_rn(__fadd_rn(r, kRound), kRound);
    return fabsf(__fsub_rn(r, kf)) > kNearTie ? tie_fix(w, s, kf) : kf;
}

// ---------------------------------------------------------------------------
// timers and bounded waits
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Upper bound on any single device-side wait: far above a healthy wait (a few
// microseconds), far below anything that looks like a hang.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// 1-D bulk copy global -> shared (no multicast), completing on an mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// One potentially-blocking test of an mbarrier phase: the hardware suspends
// the thread until the phase completes or the suspend hint (ns) runs out, so
// waiting warps do not spin on the issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}

// Plain arrive (no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bring a global line into L1 ahead of use.
__device__ __forceinline__ void prefetch_l1(const void* p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Bring a global line into L2 ahead of use.
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Programmatic dependent launch. griddep_wait blocks until the preceding
// kernel in the stream has completed and its memory is visible (a no-op when
// the launch was not programmatic); griddep_launch_dependents lets the next
// kernel's CTAs start once every CTA of this grid has issued it or exited.
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Wait for phase `parity` of an mbarrier, giving up after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
}

// Latency-critical wait (an MMA issuer): a non-blocking test first, which costs
// far less than the potentially suspending try_wait when the phase is already
// complete; then the bounded wait.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;
    return mbar_wait_bounded(bar, parity);
}

// ---------------------------------------------------------------------------
// tensor-core fragment (legacy warp-level mma, bf16 inputs, fp32 accumulate)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// bf16x2 helpers for the unpack: OR-ing a small unsigned field into the
// mantissa of bf16 128.0 (0x4300) gives the exact value 128 + field; one
// bf16x2 subtract / fma then yields the signed code k, exactly.
// ---------------------------------------------------------------------------
constexpr uint32_t kMagic = 0x43004300u;  // bf16x2 (128, 128)

// d = (a & mask) | magic, one lop3 (truth table 0xEA = (A & B) | C)
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t mask, uint32_t magic) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
    return d;
}

// d = (~a & mask) | magic, one lop3 (truth table 0xAE = (~A & B) | C)
__device__ __forceinline__ uint32_t andnot_or(uint32_t a, uint32_t mask, uint32_t magic) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xAE;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
    return d;
}

__device__ __forceinline__ uint32_t shr(uint32_t a, uint32_t n) {
    uint32_t d;
    asm("shr.b32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(n));
    return d;
}

__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t m, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(m), "r"(c));
    return d;
}

// bf16 bit patterns used by the unpack
constexpr uint32_t kBf2_132 = 0x43044304u;  // 128 + 4  (3-bit offset)
constexpr uint32_t kBf2_136 = 0x43084308u;  // 128 + 8  (4-bit offset)
constexpr uint32_t kBf2_eighth = 0x3E003E00u;  // 0.125
constexpr uint32_t kBf2_m20 = 0xC1A0C1A0u;  // -20 = -(128/8 + 4)

// Signed codes of pair m (0..15) of one quarter as bf16x2, from the quarter's
// raw words w[] (b words for b = 3, 4; for b = 8 the thread holds the two
// 16-byte halves of a 32-code range, see decode.cu).
template <int B>
__device__ __forceinline__ uint32_t unpack_pair(const uint32_t* w, int m);

template <>
__device__ __forceinline__ uint32_t unpack_pair<4>(const uint32_t* w, int m) {
    const uint32_t v = (m & 3) ? shr(w[m >> 2], 4 * (m & 3)) : w[m >> 2];
    return bf2_sub(and_or(v, 0x000F000Fu, kMagic), kBf2_136);
}

template <>
__device__ __forceinline__ uint32_t unpack_pair<8>(const uint32_t* w, int m) {
    const uint32_t v = (m & 1) ? shr(w[m >> 1], 8) : w[m >> 1];
    const uint32_t lo = and_or(v, 0x007F007Fu, kMagic);   // 128 + (u & 127)
    const uint32_t hi = andnot_or(v, 0x00800080u, kMagic);  // 256 - 128 * bit7(u)
    return bf2_sub(lo, hi);                                // u - 128 = k
}

template <>
__device__ __forceinline__ uint32_t unpack_pair<3>(const uint32_t* w, int m) {
    if (m == 15) {
        uint32_t t = and_or(shr(w[0], 15), 0x00010001u, kMagic);
        t = and_or(shr(w[1], 14), 0x00020002u, t);
        t = and_or(shr(w[2], 13), 0x00040004u, t);
        return bf2_sub(t, kBf2_132);
    }
    const int v = m / 5, f = m % 5;
    const int sh = f < 2 ? 0 : (f < 4 ? 6 : 12);
    const uint32_t x = sh ? shr(w[v], sh) : w[v];
    if (f == 1 || f == 3) {
        return bf2_fma(and_or(x, 0x00380038u, kMagic), kBf2_eighth, kBf2_m20);  // (128+8u)/8 - 20
    }
    return bf2_sub(and_or(x, 0x00070007u, kMagic), kBf2_132);  // 128 + u - 132
}

// Offset form of the unpack for b = 3, 4: the same single lop3 per field without
// the subtraction, i.e. the exact bf16 integer k + off instead of k, with
//   b = 4: off = 136 (128 + 8) for every code;
//   b = 3: off = 132 (128 + 4) for the fields at bits 0-2 / 6-8 / 12-14 and the
//          assembled 16th pair, and off = 20 (16 + 4) for the fields at bits 3-5 /
//          9-11, which OR into bf16 16.0 (mantissa unit 1/8, so 16 + u exactly).
// An MMA over these values gives K x + off . x; the decode kernels subtract the
// off . x term, computed by one more MMA whose A operand is the constant offset
// pattern, in fp32.
constexpr uint32_t kMagic16 = 0x41804180u;  // bf16x2 (16, 16)

template <int B>
__device__ __forceinline__ uint32_t unpack_pair_off(const uint32_t* w, int m);

template <>
__device__ __forceinline__ uint32_t unpack_pair_off<4>(const uint32_t* w, int m) {
    const uint32_t v = (m & 3) ? shr(w[m >> 2], 4 * (m & 3)) : w[m >> 2];
    return and_or(v, 0x000F000Fu, kMagic);
}

template <>
__device__ __forceinline__ uint32_t unpack_pair_off<3>(const uint32_t* w, int m) {
    if (m == 15) {
        uint32_t t = and_or(shr(w[0], 15), 0x00010001u, kMagic);
        t = and_or(shr(w[1], 14), 0x00020002u, t);
        return and_or(shr(w[2], 13), 0x00040004u, t);
    }
    const int v = m / 5, f = m % 5;
    const int sh = f < 2 ? 0 : (f < 4 ? 6 : 12);
    const uint32_t x = sh ? shr(w[v], sh) : w[v];
    if (f == 1 || f == 3) return and_or(x, 0x00380038u, kMagic16);  // 16 + u
    return and_or(x, 0x00070007u, kMagic);                            // 128 + u
}

// bf16x2 offset of pair m (both halves) in the offset form above.
template <int B>
__host__ __device__ constexpr uint32_t pair_offset(int m) {
    return B == 4 ? 0x43084308u                                             // 136
                  : ((m < 15 && (m % 5 == 1 || m % 5 == 3)) ? 0x41A041A0u   // 20
                                                            : 0x43044304u);  // 132
}

}  // namespace mpe
