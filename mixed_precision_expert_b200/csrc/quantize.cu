// Per-expert absmax quantizer and packer.
//
// PagedWeight, "Implementation Details", quantization scheme:
//   Q(w) = round(w / s) * s,  s = max|w| / (2^(b-1) - 1),  one s per expert.
// Here: m_e = max |w| over the expert's fp16 master (exact integer max of the
// magnitude bits), s_e = RN_f32(m_e / q_b), k = round-half-even of the exact
// quotient w / s_e (it lies in [-q_b, q_b], so the clamp is a no-op; see
// round_bits), stored offset-binary in the packed chunk format (common.cuh)
// inside the expert's pages.
#include <algorithm>

#include "internal.h"

namespace mpe {
namespace {

constexpr int kAbsmaxThreads = 256;
constexpr int kAbsmaxUnroll = 4;
constexpr int64_t kAbsmaxSegVec = 8192;  // 16-byte vectors (65536 weights) per CTA

// Integer max of (h & 0x7FFF) over a segment of one expert. The magnitude bits
// of an fp16 order exactly like |w|, so the max is exact and order-free; a
// value >= 0x7C00 means the master holds an Inf or a NaN.
__global__ void __launch_bounds__(kAbsmaxThreads)
k_absmax(const void* const* masters, const int32_t* list, int64_t n_vec, uint32_t* absmax) {
    const int e = list[blockIdx.y];
    const uint4* src = reinterpret_cast<const uint4*>(masters[e]);
    const int64_t beg = (int64_t)blockIdx.x * kAbsmaxSegVec;
    const int64_t end = min(beg + kAbsmaxSegVec, n_vec);
    uint32_t m = 0;
    for (int64_t i = beg + threadIdx.x; i < end; i += kAbsmaxThreads * kAbsmaxUnroll) {
        uint4 v[kAbsmaxUnroll];
#pragma unroll
        for (int u = 0; u < kAbsmaxUnroll; ++u) {
            const int64_t idx = i + (int64_t)u * kAbsmaxThreads;
            v[u] = idx < end ? __ldcs(src + idx) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kAbsmaxUnroll; ++u) {
            m = __vmaxu2(m, v[u].x & 0x7FFF7FFFu);
            m = __vmaxu2(m, v[u].y & 0x7FFF7FFFu);
            m = __vmaxu2(m, v[u].z & 0x7FFF7FFFu);
            m = __vmaxu2(m, v[u].w & 0x7FFF7FFFu);
        }
    }
    m = max(m & 0xFFFFu, m >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ uint32_t red[kAbsmaxThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = red[0];
        for (int w = 1; w < kAbsmaxThreads / 32; ++w) r = max(r, red[w]);
        atomicMax(absmax + e, r);
    }
}

// s_e = RN_f32(m_e / q_b); a non-finite master gets a NaN scale and a status bit.
__global__ void k_scales(Pte* pte, const uint32_t* absmax, int E, uint32_t* status) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const int b = pte[e].bits;
    if (b != 3 && b != 4 && b != 8) return;
    const uint32_t m = absmax[e];
    if (m >= 0x7C00u) {
        pte[e].scale = __int_as_float(0x7FC00000);
        set_status(status, MPE_STATUS_NONFINITE);
        return;
    }
    const float mf = __half2float(__ushort_as_half((unsigned short)m));
    pte[e].scale = (m == 0) ? 0.0f : __fdiv_rn(mf, (float)q_levels(b));
}

// Rounding of one weight. r = w * (1/s) is within ~2^-16 of the exact
// quotient (|w/s| < 2^8). Adding 1.5 * 2^23 rounds r to an integer, ties to
// even, and leaves that integer k in the low mantissa bits: the returned bit
// pattern is 0x4B400000 + k, which the packing below turns into k + 2^(b-1)
// without extracting k first. Rounding r agrees with rounding the exact
// quotient unless r lies within 2^-14 of a half-integer; then tie_fix settles
// the exact code and the pattern moves by its difference from k.
//
// No clamp is needed: |w| <= max|w| = m and s = RN(m / q) give
// |r| <= q (1 + 3 * 2^-24) < q + 1/2, so k lies in [-q, q] (the exact tie
// repair never leaves that range either). This holds because the master is
// immutable after quantize_experts (its absmax is cached).
__device__ __forceinline__ uint32_t round_bits(float w, float s, float inv_s) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23, bits 0x4B400000
    const float r = __fmul_rn(w, inv_s);
    const float rf = __fadd_rn(r, kRound);
    const float kf = __fsub_rn(rf, kRound);
    uint32_t bits = __float_as_uint(rf);
    if (fabsf(__fsub_rn(r, kf)) > kNearTie)
        bits += (uint32_t)((int)tie_fix(w, s, kf) - (int)kf);
    return bits;
}

// Weights 2i, 2i+1 of a quarter's raw fp16 data (four 16-byte vectors).
__device__ __forceinline__ float2 raw_pair(const uint4 (&raw)[4], int i) {
    const uint4 v = raw[i >> 2];
    const uint32_t x = (i & 3) == 0 ? v.x : (i & 3) == 1 ? v.y : (i & 3) == 2 ? v.z : v.w;
    return __half22float2(*reinterpret_cast<const __half2*>(&x));
}

__device__ __forceinline__ float raw_weight(const uint4 (&raw)[4], int c) {
    const float2 f = raw_pair(raw, c >> 1);
    return (c & 1) ? f.y : f.x;
}

// Bit position of code c'_i of a quarter inside its word (widths 4 and 8;
// width 3 below): fields pair up in the two 16-bit halves.
template <int B>
__host__ __device__ constexpr int field_shift(int i) {
    return B == 8 ? 16 * (i & 1) + 8 * ((i & 3) >> 1) : 16 * (i & 1) + 4 * ((i & 7) >> 1);
}

// One packed word: codes c0 .. c0+n-1 of the quarter at bit positions sh(i),
// as sum_i (k_i + 2^(b-1)) << sh(i) = const + sum_i bits_i << sh(i) (mod 2^32),
// bits_i = 0x4B400000 + k_i the pattern of r_i + 1.5 * 2^23: one multiply-add a
// code. If any code of the word lies within 2^-14 of a half-integer, the word
// is recomputed with the exact rounding (round_bits): one branch a word.
template <int B, int N, typename Shift>
__device__ __forceinline__ uint32_t encode_word(const uint4 (&raw)[4], int c0, float s,
                                                float inv_s, Shift sh) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23, bits 0x4B400000
    constexpr uint32_t bias = (1u << (B - 1)) - 0x4B400000u;  // mod 2^32
    uint32_t x = 0;
#pragma unroll
    for (int i = 0; i < N; ++i) x += bias << sh(i);
    const uint32_t x0 = x;
    bool near = false;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const float r = __fmul_rn(raw_weight(raw, c0 + i), inv_s);
        const float rf = __fadd_rn(r, kRound);
        near |= fabsf(__fsub_rn(r, __fsub_rn(rf, kRound))) > kNearTie;
        x += __float_as_uint(rf) << sh(i);
    }
    if (near) {
        x = x0;
#pragma unroll
        for (int i = 0; i < N; ++i) x += round_bits(raw_weight(raw, c0 + i), s, inv_s) << sh(i);
    }
    return x;
}

// Encode one quarter (32 consecutive weights of a row, raw fp16 in registers)
// and store its b words.
template <int B>
__device__ __forceinline__ void encode_quarter(const uint4 (&raw)[4], float s, float inv_s,
                                               uint8_t* dst) {
    if constexpr (B == 8 || B == 4) {
        constexpr int PER = 32 / B;  // codes per word
        uint32_t wv[B];
#pragma unroll
        for (int w = 0; w < B; ++w)
            wv[w] = encode_word<B, PER>(raw, PER * w, s, inv_s,
                                        [](int i) { return field_shift<B>(i); });
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        if constexpr (B == 8)
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
    } else {
        // word v holds c'_{10v+i} at bit 16(i&1) + 3(i>>1) (i < 10); bit v of
        // c'_30 / c'_31 is bit 15 / 31 of word v
        constexpr uint32_t bias = 4u - 0x4B400000u;
        const uint32_t u30 = round_bits(raw_weight(raw, 30), s, inv_s) + bias;  // k_30 + 4
        const uint32_t u31 = round_bits(raw_weight(raw, 31), s, inv_s) + bias;
        uint32_t* d32 = reinterpret_cast<uint32_t*>(dst);
#pragma unroll
        for (int v = 0; v < 3; ++v) {
            uint32_t x = encode_word<3, 10>(raw, 10 * v, s, inv_s,
                                            [](int i) { return 16 * (i & 1) + 3 * (i >> 1); });
            x += ((u30 >> v) & 1u) << 15;
            x += ((u31 >> v) & 1u) << 31;
            d32[v] = x;
        }
    }
}

// One warp per chunk (16 rows x 128 codes): item i of the launch is (expert
// list[i / nc], stream chunk i % nc). Lane l encodes quarter (l & 3) of rows
// (l >> 2) and (l >> 2) + 8; its quarters are the chunk's l and l + 32, so the
// lanes' stores cover the chunk contiguously. 4 CTAs per SM (64 registers):
// more resident warps hide the loads better than a persistent grid whose
// warps prefetch their next chunk (measured: 0.98 against 0.77 of the HBM
// copy rate on a 5.6 GB master).
struct EncItem {
    const uint4* r0;  // this lane's first quarter (row rho); the second is 8 rows on
    const uint4* r8;
    uint8_t* dst;     // the chunk in its page
    float s, inv_s;
    int b;            // 0: skip (non-finite master: left unencoded, status already set)
};

__device__ __forceinline__ EncItem enc_item(const PagedExperts& P, const void* const* masters,
                                            const int32_t* list, int nc, long long item,
                                            int lane) {
    const int li = (int)(item / nc);
    const int c = (int)(item - (long long)li * nc);
    const int e = list[li];
    const Pte pte = P.pte[e];
    EncItem it;
    it.b = pte.bits;
    it.s = pte.scale;
    if (!(it.s >= 0.0f)) it.b = 0;
    it.inv_s = it.s > 0.0f ? __frcp_rn(it.s) : 0.0f;
    const int H = P.H, F = P.F;
    const int nc1 = chunks_w1(H, F);
    // stream chunk c: W1 / W3 chunks alternate (2 cc + m); W2's tiles 2v and
    // 2v+1 alternate by block column (2 (v nj + j) + i)
    int K, tau, j;
    size_t moff;
    if (c < 2 * nc1) {
        K = H;
        const int cc = c >> 1, nj = K / kCodesPerBlock;
        moff = (c & 1) ? (size_t)F * H : 0;
        tau = cc / nj;
        j = cc - tau * nj;
    } else {
        K = F;
        const int cc = c - 2 * nc1, nj = K / kCodesPerBlock;
        moff = 2 * (size_t)F * H;
        const int pr = cc >> 1, v = pr / nj;
        j = pr - v * nj;
        tau = 2 * v + (cc & 1);
    }
    const int rho = lane >> 2, q = lane & 3;
    const __half* base = reinterpret_cast<const __half*>(masters[e]) + moff;
    const __half* r0 = base + (size_t)(tau * 16 + rho) * K + 128 * j + 32 * q;
    it.r0 = reinterpret_cast<const uint4*>(r0);
    it.r8 = reinterpret_cast<const uint4*>(r0 + (size_t)8 * K);
    it.dst = it.b ? const_cast<uint8_t*>(chunk_addr(P, pte, it.b, c)) : nullptr;
    return it;
}

__device__ __forceinline__ void enc_load(const EncItem& it, uint4 (&q0)[4], uint4 (&q8)[4]) {
    if (!it.b) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        q0[i] = __ldcs(it.r0 + i);
        q8[i] = __ldcs(it.r8 + i);
    }
}

__device__ __forceinline__ void enc_store(const EncItem& it, const uint4 (&q0)[4],
                                          const uint4 (&q8)[4], int lane) {
    switch (it.b) {
        case 3:
            encode_quarter<3>(q0, it.s, it.inv_s, it.dst + 12 * lane);
            encode_quarter<3>(q8, it.s, it.inv_s, it.dst + 12 * (lane + 32));
            break;
        case 4:
            encode_quarter<4>(q0, it.s, it.inv_s, it.dst + 16 * lane);
            encode_quarter<4>(q8, it.s, it.inv_s, it.dst + 16 * (lane + 32));
            break;
        case 8:
            encode_quarter<8>(q0, it.s, it.inv_s, it.dst + 32 * lane);
            encode_quarter<8>(q8, it.s, it.inv_s, it.dst + 32 * (lane + 32));
            break;
        default:
            break;
    }
}

constexpr int kEncThreads = 256;
constexpr int kEncWarps = kEncThreads / 32;

__global__ void __launch_bounds__(kEncThreads, 4)
k_encode(PagedExperts P, const void* const* masters, const int32_t* list) {
    const int nc = 3 * chunks_w1(P.H, P.F);
    const int lane = threadIdx.x & 31;
    const int c = blockIdx.x * kEncWarps + (threadIdx.x >> 5);
    if (c >= nc) return;
    const EncItem it = enc_item(P, masters, list, nc, (long long)blockIdx.y * nc + c, lane);
    // both quarters' weights in flight before any arithmetic
    uint4 q0[4], q8[4];
    enc_load(it, q0, q8);
    enc_store(it, q0, q8, lane);
}

// Measured quantization error of every expert at every width (PagedWeight,
// "Quality-Aware Quantization": the mean squared error is the page's example
// loss, and experts differ in sensitivity). For width b the expert's own
// s_b = RN_f32(m / q_b) and codes k = round-half-even(w / s_b) give the error
// w - k s_b, which is exact in float32: |w - k s_b| <= s_b / 2, and when k != 0
// |w| >= s_b / 2 puts w's last bit at or above s_b's, so the error is a
// multiple of s_b's last bit below 2^24 of them (k = 0 leaves w itself). Each
// error, scaled to an integer in units of Q_b = 2^min(e_b - 23, -24) (e_b the
// exponent of s_b), is squared and summed exactly in integers: the sum does
// not depend on the order, so the result is reproducible bit for bit.
//
// Fast form (s_3 < 1, every width's Q_b = 2^(e_b - 23)): scaled errors are
// below 2^23, squares below 2^46; a thread sums at most 2^7 of them per width
// in 64 bits and a block's sum stays below 2^62. Wide form (s_3 >= 1): scaled
// errors up to 2^39, squares and sums in 128 bits. Either form ends in a
// 128-bit total per (expert, width) kept as two 64-bit words, added with
// atomics and an explicit carry.
constexpr int kMseThreads = 256;
constexpr int64_t kMseSegVec = 4096;  // 16-byte vectors (32768 weights) per CTA
static_assert(kMseSegVec * 8 / kMseThreads <= 128, "fast-form per-thread bound");

struct MseWidth {
    float s, inv_s, sc;  // scale, its reciprocal, 1 / Q_b
};

__device__ __forceinline__ MseWidth mse_width(float mf, int q) {
    MseWidth w;
    w.s = __fdiv_rn(mf, (float)q);
    w.inv_s = __frcp_rn(w.s);
    const int eb = (int)((__float_as_uint(w.s) >> 23) & 0xFF) - 127;  // s is normal
    const int shift = max(23 - eb, 24);                                // -log2 Q_b
    w.sc = __uint_as_float((uint32_t)(127 + shift) << 23);
    return w;
}

// k = round-half-even(w / s) exactly (same rounding as the encoder), then the
// scaled error (w - k s) / Q as an exactly integer-valued float.
__device__ __forceinline__ float mse_scaled_error(float w, const MseWidth& m) {
    const float kf = exact_code(w, m.s, m.inv_s);
    return __fmul_rn(__fmaf_rn(-kf, m.s, w), m.sc);  // exact error, exact scaling
}

__device__ __forceinline__ void add128(unsigned long long& lo, unsigned long long& hi,
                                       unsigned long long alo, unsigned long long ahi) {
    const unsigned long long t = lo + alo;
    hi += ahi + (t < lo ? 1ull : 0ull);
    lo = t;
}

template <bool WIDE>
__device__ __forceinline__ void mse_accumulate(float w, const MseWidth (&mw)[3],
                                               unsigned long long (&lo)[3],
                                               unsigned long long (&hi)[3]) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const float v = mse_scaled_error(w, mw[i]);
        if constexpr (WIDE) {
            const unsigned long long a = (unsigned long long)llabs(__float2ll_rn(v));
            add128(lo[i], hi[i], a * a, __umul64hi(a, a));
        } else {
            const int a = __float2int_rn(v);
            lo[i] += (unsigned long long)((long long)a * a);
        }
    }
}

// acc: [E][3][2] (low word, high word), zeroed by the caller.
__global__ void __launch_bounds__(kMseThreads)
k_mse_sum(const void* const* masters, int64_t n_vec, const uint32_t* absmax,
          unsigned long long* acc) {
    const int e = blockIdx.y;
    const uint32_t m = absmax[e];
    if (m == 0 || m >= 0x7C00u) return;  // zero expert: no error; non-finite: reported by the finisher
    const float mf = __half2float(__ushort_as_half((unsigned short)m));
    MseWidth mw[3];
    mw[0] = mse_width(mf, 3);
    mw[1] = mse_width(mf, 7);
    mw[2] = mse_width(mf, 127);
    const bool wide = mw[0].s >= 1.0f;  // s_3 is the largest scale
    const uint4* src = reinterpret_cast<const uint4*>(masters[e]);
    const int64_t beg = (int64_t)blockIdx.x * kMseSegVec;
    const int64_t end = min(beg + kMseSegVec, n_vec);
    unsigned long long lo[3] = {0, 0, 0}, hi[3] = {0, 0, 0};
    constexpr int kUnroll = 4;  // 16-byte loads in flight per thread
    for (int64_t i0 = beg + threadIdx.x; i0 < end; i0 += kMseThreads * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + (int64_t)u * kMseThreads;
            v[u] = i < end ? __ldcs(src + i) : make_uint4(0, 0, 0, 0);  // zeros add no error
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[h]));
                if (wide) {
                    mse_accumulate<true>(f.x, mw, lo, hi);
                    mse_accumulate<true>(f.y, mw, lo, hi);
                } else {
                    mse_accumulate<false>(f.x, mw, lo, hi);
                    mse_accumulate<false>(f.y, mw, lo, hi);
                }
            }
        }
    }
    __shared__ unsigned long long red_lo[kMseThreads / 32][3], red_hi[kMseThreads / 32][3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            add128(lo[i], hi[i], __shfl_xor_sync(0xffffffffu, lo[i], o),
                   __shfl_xor_sync(0xffffffffu, hi[i], o));
    }
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            red_lo[warp][i] = lo[i];
            red_hi[warp][i] = hi[i];
        }
    }
    __syncthreads();
    if (threadIdx.x < 3) {
        const int i = threadIdx.x;
        unsigned long long l = 0, h = 0;
        for (int w = 0; w < kMseThreads / 32; ++w) add128(l, h, red_lo[w][i], red_hi[w][i]);
        unsigned long long* a = acc + ((size_t)e * 3 + i) * 2;
        const unsigned long long old = atomicAdd(a, l);
        const unsigned long long carry = (old + l < old) ? 1ull : 0ull;
        if (h + carry) atomicAdd(a + 1, h + carry);
    }
}

// Round a 128-bit integer to the nearest float64 (ties to even): the top 64
// bits with the rest folded into their last bit (a sticky bit far below the
// rounding position), converted once, then scaled by a power of two.
__device__ __forceinline__ double u128_to_double(unsigned long long lo, unsigned long long hi) {
    if (hi == 0) return __ull2double_rn(lo);
    const int lz = __clzll((long long)hi);
    const int sh = 64 - lz;  // 1 .. 64
    const unsigned long long top = lz == 0 ? hi : (hi << lz) | (lo >> sh);
    const unsigned long long rest = lz == 0 ? lo : (lo << lz);
    return ldexp(__ull2double_rn(top | (rest != 0 ? 1ull : 0ull)), sh);
}

// mse[e][i] = RN(RN(sum of squared errors) / n): the 128-bit total rounded to
// float64 and scaled by Q_b^2 (exact), then one float64 division by n.
__global__ void k_mse_finish(const unsigned long long* acc, const uint32_t* absmax, int E,
                             double n, double* mse) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= 3 * E) return;
    const int e = t / 3, i = t - 3 * e;
    const uint32_t m = absmax[e];
    if (m >= 0x7C00u) {
        mse[t] = __longlong_as_double(0x7FF8000000000000ll);
        return;
    }
    if (m == 0) {
        mse[t] = 0.0;
        return;
    }
    const float mf = __half2float(__ushort_as_half((unsigned short)m));
    const MseWidth mw = mse_width(mf, i == 0 ? 3 : (i == 1 ? 7 : 127));
    const int shift = (int)((__float_as_uint(mw.sc) >> 23) & 0xFF) - 127;
    const double sum_sq = ldexp(u128_to_double(acc[2 * t], acc[2 * t + 1]), -2 * shift);
    mse[t] = __ddiv_rn(sum_sq, n);
}

// Copy expert e's chunk stream out of its pages, in stream order.
__global__ void k_gather_stream(PagedExperts P, int e, uint8_t* dst) {
    const Pte pte = P.pte[e];
    const int b = pte.bits;
    if (b != 3 && b != 4 && b != 8) return;
    const int nc = 3 * chunks_w1(P.H, P.F);
    const int cb = chunk_bytes(b);
    for (int c = blockIdx.x; c < nc; c += gridDim.x) {
        const uint4* src = reinterpret_cast<const uint4*>(chunk_addr(P, pte, b, c));
        uint4* d = reinterpret_cast<uint4*>(dst + (size_t)c * cb);
        for (int i = threadIdx.x; i < cb / 16; i += blockDim.x) d[i] = src[i];
    }
}

}  // namespace

PagedExperts paged(const mpe_ctx* c) {
    PagedExperts P;
    P.pool = c->pool;
    P.pte = c->d_pte;
    P.pidx = c->d_pidx;
    P.page_bytes = c->page_bytes;
    P.E = c->E;
    P.H = c->H;
    P.F = c->F;
    return P;
}

void launch_absmax(mpe_ctx* c, const int32_t* d_list, int n_list) {
    const int64_t n_vec = (int64_t)3 * c->H * c->F / 8;
    dim3 grid((unsigned)((n_vec + kAbsmaxSegVec - 1) / kAbsmaxSegVec), (unsigned)n_list);
    k_absmax<<<grid, kAbsmaxThreads, 0, c->stream>>>(c->d_masters, d_list, n_vec, c->d_absmax);
    c->launches++;
}

void launch_scales_on(mpe_ctx* c, Pte* pte, cudaStream_t st) {
    k_scales<<<(c->E + 127) / 128, 128, 0, st>>>(pte, c->d_absmax, c->E, c->d_status);
    c->launches++;
}

void launch_scales(mpe_ctx* c) { launch_scales_on(c, c->d_pte, c->stream); }

void launch_encode_on(mpe_ctx* c, const PagedExperts& P, const int32_t* d_list, int n_list,
                      cudaStream_t st) {
    const int nc = 3 * chunks_w1(c->H, c->F);
    dim3 grid((unsigned)((nc + kEncWarps - 1) / kEncWarps), (unsigned)n_list);
    k_encode<<<grid, kEncThreads, 0, st>>>(P, c->d_masters, d_list);
    c->launches++;
}

void launch_encode(mpe_ctx* c, const int32_t* d_list, int n_list) {
    launch_encode_on(c, paged(c), d_list, n_list, c->stream);
}

void launch_measure_mse(mpe_ctx* c, unsigned long long* d_acc, double* d_mse) {
    const int64_t n_vec = (int64_t)3 * c->H * c->F / 8;
    cudaMemsetAsync(d_acc, 0, sizeof(unsigned long long) * 6 * c->E, c->stream);
    dim3 grid((unsigned)((n_vec + kMseSegVec - 1) / kMseSegVec), (unsigned)c->E);
    k_mse_sum<<<grid, kMseThreads, 0, c->stream>>>(c->d_masters, n_vec, c->d_absmax, d_acc);
    k_mse_finish<<<(3 * c->E + 127) / 128, 128, 0, c->stream>>>(
        d_acc, c->d_absmax, c->E, (double)(n_vec * 8), d_mse);
    c->launches += 2;
}

void launch_gather_stream(mpe_ctx* c, int e, uint8_t* dst) {
    k_gather_stream<<<148, 128, 0, c->stream>>>(paged(c), e, dst);
    c->launches++;
}

}  // namespace mpe
