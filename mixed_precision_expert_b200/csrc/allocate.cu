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
#include "internal.h"

namespace mpe {
namespace {

__device__ __forceinline__ double dinf() { return __longlong_as_double(0x7FF0000000000000ll); }

__device__ uint64_t gcd_u64(uint64_t a, uint64_t b) {
    while (b) {
        const uint64_t t = a % b;
        a = b;
        b = t;
    }
    return a;
}

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads)
k_allocate(const double* p, const uint64_t* W, int E, uint64_t B, uint8_t* bits,
           int32_t* status, uint8_t* choice, double* D, int state_cap) {
    __shared__ int s_mode;      // 0 = solve, 1 = infeasible, 2 = all 8, 3 = state cap
    __shared__ uint32_t s_R;
    __shared__ uint64_t s_g;
    __shared__ uint32_t s_up4[MPE_MAX_EXPERTS];
    __shared__ uint32_t s_up8[MPE_MAX_EXPERTS];
    const int tid = threadIdx.x;
    if (tid == 0) {
        uint64_t sum_w = 0, g = 0;
        for (int e = 0; e < E; ++e) {
            sum_w += W[e];
            g = gcd_u64(g, W[e]);
        }
        s_g = g;
        if (B < 3 * sum_w) {
            s_mode = 1;
        } else if (B >= 8 * sum_w) {
            s_mode = 2;
        } else {
            uint64_t R = (B - 3 * sum_w) / g;
            const uint64_t rmax = 5 * (sum_w / g);
            if (R > rmax) R = rmax;
            if (R + 1 > (uint64_t)state_cap) {
                s_mode = 3;
            } else {
                s_mode = 0;
                s_R = (uint32_t)R;
            }
        }
        *status = s_mode;
    }
    __syncthreads();
    const int mode = s_mode;
    if (mode == 2) {
        for (int e = tid; e < E; e += kThreads) bits[e] = 8;
        return;
    }
    if (mode != 0) return;
    const uint32_t R = s_R;
    const uint64_t g = s_g;
    for (int e = tid; e < E; e += kThreads) {
        const uint64_t u4 = W[e] / g, u8 = 5 * (W[e] / g);
        s_up4[e] = (uint32_t)min(u4, (uint64_t)R + 1);
        s_up8[e] = (uint32_t)min(u8, (uint64_t)R + 1);
    }
    const double L3 = __ddiv_rn(1.0, 9.0);
    const double L4 = __ddiv_rn(1.0, 49.0);
    const double L8 = __ddiv_rn(1.0, 16129.0);
    double* Dcur = D;
    double* Dnext = D + (R + 1);
    for (uint32_t r = tid; r <= R; r += kThreads) Dcur[r] = (r == 0) ? 0.0 : dinf();
    __syncthreads();
    for (int e = 0; e < E; ++e) {
        const double pe = p[e];
        const double c3 = __dmul_rn(pe, L3);
        const double c4 = __dmul_rn(pe, L4);
        const double c8 = __dmul_rn(pe, L8);
        const uint32_t u4 = s_up4[e], u8 = s_up8[e];
        uint8_t* ch = choice + (size_t)e * (R + 1);
        for (uint32_t r = tid; r <= R; r += kThreads) {
            double best = dinf();
            uint8_t bb = 0;
            double prev = Dcur[r];
            if (prev != dinf()) {
                const double cand = __dadd_rn(prev, c3);
                if (cand < best) { best = cand; bb = 3; }
            }
            if (r >= u4) {
                prev = Dcur[r - u4];
                if (prev != dinf()) {
                    const double cand = __dadd_rn(prev, c4);
                    if (cand < best) { best = cand; bb = 4; }
                }
            }
            if (r >= u8) {
                prev = Dcur[r - u8];
                if (prev != dinf()) {
                    const double cand = __dadd_rn(prev, c8);
                    if (cand < best) { best = cand; bb = 8; }
                }
            }
            Dnext[r] = best;
            ch[r] = bb;
        }
        __syncthreads();
        double* t = Dcur;
        Dcur = Dnext;
        Dnext = t;
    }
    if (tid == 0) {
        uint32_t rb = 0;
        for (uint32_t r = 1; r <= R; ++r)
            if (Dcur[r] < Dcur[rb]) rb = r;
        uint32_t r = rb;
        for (int e = E - 1; e >= 0; --e) {
            const uint8_t b = choice[(size_t)e * (R + 1) + r];
            bits[e] = b;
            r -= (b == 3) ? 0u : (b == 4 ? s_up4[e] : s_up8[e]);
        }
    }
}

}  // namespace

void launch_allocate(cudaStream_t st, const double* p, const uint64_t* W, int E, uint64_t B,
                     uint8_t* bits_out, int32_t* status, uint8_t* choice, double* D,
                     int state_cap) {
    k_allocate<<<1, kThreads, 0, st>>>(p, W, E, B, bits_out, status, choice, D, state_cap);
}

}  // namespace mpe
