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
// Dynamic shared memory for the two DP rows and the choice table (see below).
constexpr size_t kAllocSmemMax = 200 * 1024;

// Choices are 2-bit codes (0: 3 bits, 1: 4 bits, 2: 8 bits), four budget
// states per byte; each thread evaluates one state per pass and the first
// lane of every four writes their byte. When both DP rows and the table fit in shared memory
// (R <= smem_R; -1 = no on-chip buffers) the whole solve stays on chip -- every expert step is a
// shared-memory pass plus one barrier, and the serial backtrack reads shared
// memory -- else rows and table live in the global buffers D and choice.
__global__ void __launch_bounds__(kThreads)
k_allocate(const double* p, const uint64_t* W, int E, uint64_t B, uint8_t* bits,
           int32_t* status, uint8_t* choice, double* D, int state_cap, int64_t smem_R) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ int s_mode;      // 0 = solve, 1 = infeasible, 2 = all 8, 3 = state cap
    __shared__ uint32_t s_R;
    __shared__ uint64_t s_g;
    __shared__ uint32_t s_up4[MPE_MAX_EXPERTS];
    __shared__ uint32_t s_up8[MPE_MAX_EXPERTS];
    __shared__ double s_p[MPE_MAX_EXPERTS];
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
    const uint32_t nq = (R + 4) / 4;  // choice bytes per expert
    for (int e = tid; e < E; e += kThreads) {
        const uint64_t u4 = W[e] / g, u8 = 5 * (W[e] / g);
        s_up4[e] = (uint32_t)min(u4, (uint64_t)R + 1);
        s_up8[e] = (uint32_t)min(u8, (uint64_t)R + 1);
        s_p[e] = p[e];
    }
    const bool on_chip = (int64_t)R <= smem_R;
    double* Dcur = on_chip ? reinterpret_cast<double*>(dyn) : D;
    double* Dnext = Dcur + (R + 1);
    uint8_t* chb = on_chip ? dyn + 16 * (size_t)(R + 1) : choice;
    const double L3 = __ddiv_rn(1.0, 9.0);
    const double L4 = __ddiv_rn(1.0, 49.0);
    const double L8 = __ddiv_rn(1.0, 16129.0);
    for (uint32_t r = tid; r <= R; r += kThreads) Dcur[r] = (r == 0) ? 0.0 : dinf();
    __syncthreads();
    for (int e = 0; e < E; ++e) {
        const double pe = s_p[e];
        const double c3 = __dmul_rn(pe, L3);
        const double c4 = __dmul_rn(pe, L4);
        const double c8 = __dmul_rn(pe, L8);
        const uint32_t u4 = s_up4[e], u8 = s_up8[e];
        uint8_t* ch = chb + (size_t)e * nq;
        // one state a thread; the loop bound is the same for every thread (the
        // code packing below shuffles across the warp)
        for (uint32_t base = 0; base <= R; base += kThreads) {
            const uint32_t r = base + tid;
            uint32_t code = 0;
            if (r <= R) {
                // an unreachable predecessor is +inf and its candidate stays +inf
                const double x3 = __dadd_rn(Dcur[r], c3);
                const double x4 = r >= u4 ? __dadd_rn(Dcur[r - u4], c4) : dinf();
                const double x8 = r >= u8 ? __dadd_rn(Dcur[r - u8], c8) : dinf();
                double best = dinf();
                if (x3 < best) best = x3;
                if (x4 < best) { best = x4; code = 1; }
                if (x8 < best) { best = x8; code = 2; }
                Dnext[r] = best;
            }
            // lanes 4m .. 4m+3 hold states 4m' .. 4m'+3: one byte of codes
            const uint32_t k1 = __shfl_down_sync(0xffffffffu, code, 1);
            const uint32_t k2 = __shfl_down_sync(0xffffffffu, code, 2);
            const uint32_t k3 = __shfl_down_sync(0xffffffffu, code, 3);
            if ((tid & 3) == 0 && r <= R) ch[r >> 2] = (uint8_t)(code | k1 << 2 | k2 << 4 | k3 << 6);
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
            const uint32_t code = (chb[(size_t)e * nq + r / 4] >> (2 * (r % 4))) & 3u;
            bits[e] = code == 0 ? 3 : (code == 1 ? 4 : 8);
            r -= code == 0 ? 0u : (code == 1 ? s_up4[e] : s_up8[e]);
        }
    }
}

}  // namespace

size_t allocate_choice_bytes(int E, uint64_t R) { return (size_t)E * (size_t)((R + 4) / 4); }

void launch_allocate(cudaStream_t st, const double* p, const uint64_t* W, int E, uint64_t B,
                     uint8_t* bits_out, int32_t* status, uint8_t* choice, double* D,
                     int state_cap, uint64_t R) {
    // R is the host's count of budget units (same formula as the kernel's);
    // it only sizes the on-chip buffers
    const size_t smem = 16 * (size_t)(R + 1) + allocate_choice_bytes(E, R);
    const bool on_chip = smem <= kAllocSmemMax;
    // the attribute is per device: set it on every launch that needs it
    if (on_chip && smem > 48 * 1024)
        cudaFuncSetAttribute(k_allocate, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_allocate<<<1, kThreads, on_chip ? smem : 0, st>>>(p, W, E, B, bits_out, status, choice, D,
                                                        state_cap, on_chip ? (int64_t)R : -1);
}

}  // namespace mpe
