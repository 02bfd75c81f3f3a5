// Budgeted per-expert precision, solved exactly on the device.
//
// PagedWeight, "Quality-Aware Quantization": minimise sum_e p_e L(b_e) subject
// to sum_e b_e W_e <= B with b_e in {3, 4, 8} (the widths of the page's
// "Code Illustration"). L(b) = 1 / (2^(b-1) - 1)^2, the mean squared error of
// a uniform symmetric quantizer up to a common factor.
//
// Dynamic program in units of g = gcd(W_e): R = floor((B - 3 sum W) / g) units
// may be spent; raising expert e from 3 to 4 bits costs W_e / g units, from 3
// to 8 bits 5 W_e / g. D_e[r] = least objective over experts 0..e spending
// exactly r units. Widths are tried in the order 3, 4, 8 and replace only on
// a strictly smaller value; the final budget is the smallest r reaching the
// minimum; a backtrack recovers the widths. Every product and sum is one
// correctly rounded float64 operation (no fused multiply-add), so the result
// is reproducible bit for bit.
//
// With a loss table (float64[E][3], widths 3, 4, 8) the cost of expert e at
// width b is p_e * loss[e][b] instead of p_e * L(b), e.g. the measured mean
// squared error of each expert's own quantization; the all-8 shortcut for a
// budget of 8 sum W or more is then not taken (the program itself decides).
#include "internal.h"

namespace mpe {
namespace {

__device__ __forceinline__ double dinf() { return __longlong_as_double(0x7FF0000000000000ll); }

constexpr int kThreads = 1024;
// Dynamic shared memory for the two DP rows and the choice table (see below).
constexpr size_t kAllocSmemMax = 200 * 1024;

// Budget states r = 0 .. R. Thread t evaluates states t, t + 1024, ...: the 32
// lanes of a warp hold 32 consecutive states, so each expert step is one
// pass (one state per thread up to 1,024 states) and one barrier. A choice is
// a 2-bit code (0: 3 bits, 1: 4 bits, 2: 8 bits); a warp's 32 codes are two
// ballot words (low and high code bits), word w of an expert row covering
// states 32 w .. 32 w + 31. ON_CHIP: both DP rows and the table live in
// shared memory; otherwise in the global buffers D and choice. The host
// supplies sum W and g = gcd(W) (no serial 64-bit arithmetic on the device).
__host__ __device__ constexpr uint32_t choice_words(uint64_t R) { return (uint32_t)(R / 32 + 1); }

// One cell of the program: the least objective over experts 0..e spending
// exactly q units, from row Dp of experts 0..e-1; code = the width taken (0:
// 3 bits, 1: 4, 2: 8). Widths are tried 3, 4, 8 and replace only on a strictly
// smaller value; an unreachable predecessor is +inf and stays +inf.
__device__ __forceinline__ double dp_cell(const double* Dp, uint32_t q, uint32_t u4, uint32_t u8,
                                          double c3, double c4, double c8, uint32_t& code) {
    const double x3 = __dadd_rn(Dp[q], c3);
    const double x4 = q >= u4 ? __dadd_rn(Dp[q - u4], c4) : dinf();
    const double x8 = q >= u8 ? __dadd_rn(Dp[q - u8], c8) : dinf();
    double best = dinf();
    code = 0;
    if (x3 < best) best = x3;
    if (x4 < best) { best = x4; code = 1; }
    if (x8 < best) { best = x8; code = 2; }
    return best;
}

template <bool ON_CHIP>
__global__ void __launch_bounds__(kThreads)
k_allocate(const double* p, const double* loss, const uint64_t* W, int E, uint64_t B,
           uint64_t sum_w, uint64_t g, uint8_t* bits, int32_t* status, uint32_t* choice,
           double* D, int state_cap) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ uint32_t s_up4[MPE_MAX_EXPERTS];
    __shared__ uint32_t s_up8[MPE_MAX_EXPERTS];
    __shared__ double s_p[MPE_MAX_EXPERTS];
    __shared__ double s_rv[kThreads / 32];
    __shared__ uint32_t s_ri[kThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31;
    int mode;  // 0 = solve, 1 = infeasible, 2 = all 8, 3 = state cap
    uint64_t R64 = 0;
    if (B < 3 * sum_w) {
        mode = 1;
    } else if (B >= 8 * sum_w && !loss) {
        mode = 2;
    } else {
        R64 = (B - 3 * sum_w) / g;
        const uint64_t rmax = 5 * (sum_w / g);
        if (R64 > rmax) R64 = rmax;
        mode = (R64 + 1 > (uint64_t)state_cap) ? 3 : 0;
    }
    if (tid == 0) *status = mode;
    if (mode == 2) {
        for (int e = tid; e < E; e += kThreads) bits[e] = 8;
        return;
    }
    if (mode != 0) return;
    const uint32_t R = (uint32_t)R64;
    const uint32_t nw = choice_words(R);  // ballot-word pairs per expert row
    for (int e = tid; e < E; e += kThreads) {
        const uint64_t u4 = W[e] / g, u8 = 5 * (W[e] / g);
        s_up4[e] = (uint32_t)min(u4, (uint64_t)R + 1);
        s_up8[e] = (uint32_t)min(u8, (uint64_t)R + 1);
        s_p[e] = p[e];
    }
    double* Dcur = ON_CHIP ? reinterpret_cast<double*>(dyn) : D;
    double* Dnext = Dcur + (R + 1);
    uint32_t* chw = ON_CHIP ? reinterpret_cast<uint32_t*>(dyn + 16 * (size_t)(R + 1)) : choice;
    const double L3 = __ddiv_rn(1.0, 9.0);
    const double L4 = __ddiv_rn(1.0, 49.0);
    const double L8 = __ddiv_rn(1.0, 16129.0);
    for (uint32_t r = tid; r <= R; r += kThreads) Dcur[r] = (r == 0) ? 0.0 : dinf();
    __syncthreads();
    // Two experts per barrier: the thread that owns state r of expert e + 1
    // also evaluates expert e at r, r - u4' and r - u8' (u' of expert e + 1)
    // from the row of expert e - 1 -- the same operations in the same order as
    // the owners of those states, so every value is the one a one-expert step
    // would store -- and then expert e + 1 at r. An odd last expert takes a
    // step of its own.
    auto costs = [&](int e, double& c3, double& c4, double& c8) {
        const double pe = s_p[e];
        c3 = __dmul_rn(pe, loss ? loss[3 * e] : L3);
        c4 = __dmul_rn(pe, loss ? loss[3 * e + 1] : L4);
        c8 = __dmul_rn(pe, loss ? loss[3 * e + 2] : L8);
    };
    auto store_codes = [&](int e, uint32_t r0, uint32_t code) {
        const uint32_t lo = __ballot_sync(0xffffffffu, code & 1u);
        const uint32_t hi = __ballot_sync(0xffffffffu, code >> 1);
        if (lane == 0) {
            uint32_t* ch = chw + (size_t)e * 2 * nw + 2 * (r0 / 32);
            ch[0] = lo;
            ch[1] = hi;
        }
    };
    int e = 0;
    for (; e + 1 < E; e += 2) {
        double a3, a4, a8, b3, b4, b8;
        costs(e, a3, a4, a8);
        costs(e + 1, b3, b4, b8);
        const uint32_t ua4 = s_up4[e], ua8 = s_up8[e];
        const uint32_t ub4 = s_up4[e + 1], ub8 = s_up8[e + 1];
        // warp-uniform trip count: every lane takes part in the ballots
        for (uint32_t r0 = tid - lane; r0 <= R; r0 += kThreads) {
            const uint32_t r = r0 + lane;
            uint32_t ca = 0, cb = 0;
            if (r <= R) {
                uint32_t unused;
                const double d0 = dp_cell(Dcur, r, ua4, ua8, a3, a4, a8, ca);
                const double d4 = r >= ub4 ? dp_cell(Dcur, r - ub4, ua4, ua8, a3, a4, a8, unused)
                                           : dinf();
                const double d8 = r >= ub8 ? dp_cell(Dcur, r - ub8, ua4, ua8, a3, a4, a8, unused)
                                           : dinf();
                const double x3 = __dadd_rn(d0, b3);
                const double x4 = r >= ub4 ? __dadd_rn(d4, b4) : dinf();
                const double x8 = r >= ub8 ? __dadd_rn(d8, b8) : dinf();
                double best = dinf();
                if (x3 < best) best = x3;
                if (x4 < best) { best = x4; cb = 1; }
                if (x8 < best) { best = x8; cb = 2; }
                Dnext[r] = best;
            }
            store_codes(e, r0, ca);
            store_codes(e + 1, r0, cb);
        }
        __syncthreads();
        double* t = Dcur;
        Dcur = Dnext;
        Dnext = t;
    }
    if (e < E) {
        double c3, c4, c8;
        costs(e, c3, c4, c8);
        const uint32_t u4 = s_up4[e], u8 = s_up8[e];
        for (uint32_t r0 = tid - lane; r0 <= R; r0 += kThreads) {
            const uint32_t r = r0 + lane;
            uint32_t code = 0;
            if (r <= R) Dnext[r] = dp_cell(Dcur, r, u4, u8, c3, c4, c8, code);
            store_codes(e, r0, code);
        }
        __syncthreads();
        double* t = Dcur;
        Dcur = Dnext;
        Dnext = t;
    }
    // argmin over the budget states, ties to the smallest state
    double bv = dinf();
    uint32_t bi = 0xFFFFFFFFu;
    for (uint32_t r = tid; r <= R; r += kThreads)
        if (Dcur[r] < bv) { bv = Dcur[r]; bi = r; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const uint32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov < bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) {
        s_rv[tid >> 5] = bv;
        s_ri[tid >> 5] = bi;
    }
    __syncthreads();
    if (tid == 0) {
        bv = s_rv[0];
        bi = s_ri[0];
        for (int w = 1; w < kThreads / 32; ++w)
            if (s_rv[w] < bv || (s_rv[w] == bv && s_ri[w] < bi)) { bv = s_rv[w]; bi = s_ri[w]; }
        uint32_t r = bi;
        for (int e = E - 1; e >= 0; --e) {
            const uint32_t* ch = chw + (size_t)e * 2 * nw + 2 * (r / 32);
            const uint32_t code = ((ch[0] >> (r % 32)) & 1u) | (((ch[1] >> (r % 32)) & 1u) << 1);
            bits[e] = code == 0 ? 3 : (code == 1 ? 4 : 8);
            r -= code == 0 ? 0u : (code == 1 ? s_up4[e] : s_up8[e]);
        }
    }
}

// The page's simplified allocator ("Code Illustration",
// compute_budgeted_precision) with a budget repair, one CTA: each expert's
// budget share B p_e / sum p in bits per weight, rounded up to 3 / 4 / 8 (3 if
// at most 3, 4 if at most 4, else 8); then, in ascending (p_e, e), each expert
// is downgraded one width at a time until sum b_e W_e <= B. The sum of p runs
// in ascending e (one thread) and every operation is one correctly rounded
// float64 step, so the widths are reproducible bit for bit. status: 0 solved,
// 1 infeasible (B < 3 sum W).
constexpr int kPropThreads = 256;
constexpr int kPropSort = MPE_MAX_EXPERTS;  // sort capacity (a power of two)

__global__ void __launch_bounds__(kPropThreads)
k_allocate_proportional(const double* p, const uint64_t* W, int E, uint64_t B, uint64_t sum_w,
                        uint8_t* bits_out, int32_t* status) {
    __shared__ double s_key[kPropSort];
    __shared__ int32_t s_idx[kPropSort];
    __shared__ uint8_t s_bits[MPE_MAX_EXPERTS];
    __shared__ double s_total;
    const int tid = threadIdx.x;
    if (B < 3 * sum_w) {
        if (tid == 0) *status = 1;
        return;
    }
    if (tid == 0) {
        double t = 0.0;
        for (int e = 0; e < E; ++e) t = __dadd_rn(t, p[e]);
        s_total = t;
        *status = 0;
    }
    __syncthreads();
    const double total = s_total;
    const double Bd = __ull2double_rn(B);
    for (int e = tid; e < E; e += kPropThreads) {
        const double pe = p[e];
        const double share = total > 0.0 ? __ddiv_rn(__dmul_rn(Bd, pe), total) : 0.0;
        const double pw = __ddiv_rn(share, __ull2double_rn(W[e]));
        s_bits[e] = pw <= 3.0 ? 3 : (pw <= 4.0 ? 4 : 8);
    }
    // bitonic sort of (p_e, e) ascending; padding sorts last
    int n = 1;
    while (n < E) n <<= 1;
    for (int i = tid; i < n; i += kPropThreads) {
        s_key[i] = i < E ? p[i] : __longlong_as_double(0x7FF0000000000000ll);
        s_idx[i] = i < E ? i : 0x7FFFFFFF;
    }
    __syncthreads();
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < n; i += kPropThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const bool up = (i & k) == 0;
                    const bool gt = s_key[i] > s_key[l] || (s_key[i] == s_key[l] && s_idx[i] > s_idx[l]);
                    if (gt == up) {
                        const double tk = s_key[i];
                        s_key[i] = s_key[l];
                        s_key[l] = tk;
                        const int ti = s_idx[i];
                        s_idx[i] = s_idx[l];
                        s_idx[l] = ti;
                    }
                }
            }
            __syncthreads();
        }
    }
    if (tid == 0) {
        uint64_t used = 0;
        for (int e = 0; e < E; ++e) used += (uint64_t)s_bits[e] * W[e];
        for (int r = 0; r < E && used > B; ++r) {
            const int e = s_idx[r];
            if (s_bits[e] == 8) {
                s_bits[e] = 4;
                used -= 4 * W[e];
            }
            if (used <= B) break;
            if (s_bits[e] == 4) {
                s_bits[e] = 3;
                used -= W[e];
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPropThreads) bits_out[e] = s_bits[e];
}

}  // namespace

size_t allocate_choice_bytes(int E, uint64_t R) {
    return (size_t)E * 2 * choice_words(R) * sizeof(uint32_t);
}

void launch_allocate(cudaStream_t st, const double* p, const double* loss, const uint64_t* W,
                     int E, uint64_t B, uint64_t sum_w, uint64_t g, uint8_t* bits_out,
                     int32_t* status, uint8_t* choice, double* D, int state_cap, uint64_t R) {
    uint32_t* chw = reinterpret_cast<uint32_t*>(choice);
    // R is the host's count of budget units (same formula as the kernel's);
    // it only sizes the on-chip buffers
    const size_t smem = 16 * (size_t)(R + 1) + allocate_choice_bytes(E, R);
    if (smem <= kAllocSmemMax) {
        // the attribute is per device: set it on every launch that needs it
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(k_allocate<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        k_allocate<true><<<1, kThreads, smem, st>>>(p, loss, W, E, B, sum_w, g, bits_out, status,
                                                    chw, D, state_cap);
    } else {
        k_allocate<false><<<1, kThreads, 0, st>>>(p, loss, W, E, B, sum_w, g, bits_out, status,
                                                  chw, D, state_cap);
    }
}

void launch_allocate_proportional(cudaStream_t st, const double* p, const uint64_t* W, int E,
                                  uint64_t B, uint64_t sum_w, uint8_t* bits_out, int32_t* status) {
    k_allocate_proportional<<<1, kPropThreads, 0, st>>>(p, W, E, B, sum_w, bits_out, status);
}

}  // namespace mpe
