// Top-k weighted combine: out[t] = bf16( sum_j w[t, j] sum_p y[p][pos_j] ) with
// pos_j = inv[t*k + j] the route position of token t's j-th slot, summed in
// fp32 with slots j = 0..k-1 outermost and K parts p = 0..P-1 inside (the down
// kernels already applied the scale); slots with an id outside [0, E)
// contribute nothing. Deterministic: no atomics.
//
// SwiGLU reduce (gate/up split over K): h[pos][f] = bf16( silu(g) v ) with
// g = sum_p gv[p][pos][0][f], v = sum_p gv[p][pos][1][f] (already scaled).
#include <algorithm>

#include "internal.h"

namespace mpe {
namespace {

__global__ void __launch_bounds__(256)
k_swiglu_reduce(const float* gv, const int32_t* offsets, int E, int F, int parts,
                size_t part_stride, __nv_bfloat16* h) {
    // the down kernel after this one reads only route outputs before its own wait
    griddep_launch_dependents();
    griddep_wait();
    const int n_pos = offsets[E];
    const size_t total = (size_t)n_pos * F;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t pos = i / F, f = i - pos * F;
        float g = 0.0f, v = 0.0f;
        for (int p = 0; p < parts; ++p) {
            const float* src = gv + (size_t)p * part_stride + pos * 2 * F + f;
            g += src[0];
            v += src[F];
        }
        h[pos * F + f] = __float2bfloat16_rn(g / (1.0f + __expf(-g)) * v);
    }
}

// out[t] = bf16( sum_j w[t, j] * sum_p y[p][inv[t k + j]] ): y is stored by
// route position in P K-part slices (fp32), or as one bf16 slice on the
// tensor-core path; slots in
// order, parts summed first in part order; dropped slots (inv < 0) add
// nothing. One thread per 4 columns of one token; a CTA covers 512 columns of
// one token row (grid: tokens x column blocks). The token's positions and
// weights are read once into shared memory, so every thread can issue all its
// slots' loads before the first sum.
constexpr int kCombineSlots = 8;  // slots whose loads are in flight together

template <bool SINGLE>  // one part (no K split): fewer registers, more CTAs
__global__ void __launch_bounds__(128)
k_combine_by_position(const float* y, const int32_t* inv, const float* w, int T, int k, int H,
                      int parts, size_t part_stride, __nv_bfloat16* out) {
    __shared__ int s_pos[32];
    __shared__ float s_w[32];
    griddep_wait();
    griddep_launch_dependents();
    const int t = blockIdx.x;
    if (threadIdx.x < k) {
        s_pos[threadIdx.x] = inv[t * k + threadIdx.x];
        s_w[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    const int i = blockIdx.y * blockDim.x + threadIdx.x;  // float4 column index
    if (i >= H / 4) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (SINGLE) {
        for (int j0 = 0; j0 < k; j0 += kCombineSlots) {
            float4 v[kCombineSlots];
#pragma unroll
            for (int r = 0; r < kCombineSlots; ++r) {
                const int pos = j0 + r < k ? s_pos[j0 + r] : -1;
                v[r] = pos >= 0 ? reinterpret_cast<const float4*>(y + (size_t)pos * H)[i]
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int r = 0; r < kCombineSlots; ++r) {
                if (j0 + r >= k || s_pos[j0 + r] < 0) continue;
                const float wj = s_w[j0 + r];
                acc.x = fmaf(wj, v[r].x, acc.x);
                acc.y = fmaf(wj, v[r].y, acc.y);
                acc.z = fmaf(wj, v[r].z, acc.z);
                acc.w = fmaf(wj, v[r].w, acc.w);
            }
        }
    } else {
        for (int j = 0; j < k; ++j) {
            const int pos = s_pos[j];
            if (pos < 0) continue;
            const float wj = s_w[j];
            const float4* src = reinterpret_cast<const float4*>(y + (size_t)pos * H) + i;
            const size_t stride = part_stride / 4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            // parts summed in order; up to 16 independent loads in flight
            for (int p0 = 0; p0 < parts; p0 += 16) {
                float4 u[16];
#pragma unroll
                for (int r = 0; r < 16; ++r)
                    if (p0 + r < parts) u[r] = src[(size_t)(p0 + r) * stride];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    if (p0 + r < parts) {
                        v.x += u[r].x;
                        v.y += u[r].y;
                        v.z += u[r].z;
                        v.w += u[r].w;
                    }
                }
            }
            acc.x = fmaf(wj, v.x, acc.x);
            acc.y = fmaf(wj, v.y, acc.y);
            acc.z = fmaf(wj, v.z, acc.z);
            acc.w = fmaf(wj, v.w, acc.w);
        }
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(out + (size_t)t * H)[i] = pk;
}

// The tensor-core path's combine: y holds bf16(s acc) by route position (one
// part). One CTA per token, a thread 8 columns (one 16-byte load a slot, the
// token's slots all in flight), the same slot-order fp32 sum.
constexpr int kCombBf16Threads = 256;

__global__ void __launch_bounds__(kCombBf16Threads)
k_combine_bf16y(const __nv_bfloat16* y, const int32_t* inv, const float* w, int k, int H,
                __nv_bfloat16* out) {
    __shared__ int s_pos[32];
    __shared__ float s_w[32];
    griddep_wait();
    griddep_launch_dependents();
    const int t = blockIdx.x;
    if (threadIdx.x < k) {
        s_pos[threadIdx.x] = inv[t * k + threadIdx.x];
        s_w[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < H / 8; i += kCombBf16Threads) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < k; j0 += kCombineSlots) {
            uint4 v[kCombineSlots];
#pragma unroll
            for (int r = 0; r < kCombineSlots; ++r) {
                const int pos = j0 + r < k ? s_pos[j0 + r] : -1;
                v[r] = pos >= 0 ? reinterpret_cast<const uint4*>(y + (size_t)pos * H)[i]
                                : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int r = 0; r < kCombineSlots; ++r) {
                if (j0 + r >= k || s_pos[j0 + r] < 0) continue;
                const float wj = s_w[j0 + r];
                const uint32_t u[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[2 * q] = fmaf(wj, __uint_as_float(u[q] << 16), acc[2 * q]);
                    acc[2 * q + 1] = fmaf(wj, __uint_as_float(u[q] & 0xFFFF0000u), acc[2 * q + 1]);
                }
            }
        }
        uint4 pk;
        uint32_t* pw = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
            pw[q] = *reinterpret_cast<uint32_t*>(&b2);
        }
        reinterpret_cast<uint4*>(out + (size_t)t * H)[i] = pk;
    }
}

}  // namespace

void launch_swiglu_reduce(mpe_ctx* c, size_t Tk, int parts) {
    const size_t total = Tk * c->F;
    const int grid = (int)std::min<size_t>((total + 255) / 256, 148 * 8);
    launch_pdl(k_swiglu_reduce, dim3(grid), dim3(256), 0, c->stream, (const float*)c->s.part,
               (const int32_t*)c->s.offsets, c->E, c->F, parts, (size_t)2 * Tk * c->F, c->s.h);
    c->launches++;
}

void launch_combine_by_position(mpe_ctx* c, const float* w, int T, int k, int parts,
                                __nv_bfloat16* out, bool y_bf16) {
    const int n4 = c->H / 4;
    dim3 grid((unsigned)T, (unsigned)((n4 + 127) / 128));
    if (y_bf16)
        launch_pdl(k_combine_bf16y, dim3((unsigned)T), dim3(kCombBf16Threads), 0, c->stream,
                   (const __nv_bfloat16*)c->s.y, (const int32_t*)c->s.inv, w, k, c->H, out);
    else if (parts == 1)
        launch_pdl(k_combine_by_position<true>, grid, dim3(128), 0, c->stream,
                   (const float*)c->s.y, (const int32_t*)c->s.inv, w, T, k, c->H, parts,
                   (size_t)T * k * c->H, out);
    else
        launch_pdl(k_combine_by_position<false>, grid, dim3(128), 0, c->stream,
                   (const float*)c->s.y, (const int32_t*)c->s.inv, w, T, k, c->H, parts,
                   (size_t)T * k * c->H, out);
    c->launches++;
}

}  // namespace mpe
