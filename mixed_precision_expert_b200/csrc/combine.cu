// Top-k weighted combine: out[t] = bf16( sum_j y[t*k + j] ), the slots summed in
// order j = 0..k-1 in fp32 (the down kernel already applied w[t, j]); slots with
// an id outside [0, E) contribute nothing. Deterministic: no atomics.
#include "internal.h"

namespace mpe {
namespace {

__global__ void __launch_bounds__(256)
k_combine(const float* y, const int32_t* ids, int T, int k, int H, int E, __nv_bfloat16* out) {
    const int t = blockIdx.x;
    const int n4 = H / 4;
    for (int i = blockIdx.y * blockDim.x + threadIdx.x; i < n4; i += gridDim.y * blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int e = ids[t * k + j];
            if (e < 0 || e >= E) continue;
            const float4 v = reinterpret_cast<const float4*>(y + (size_t)(t * k + j) * H)[i];
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>(out + (size_t)t * H)[i] = pk;
    }
}

}  // namespace

void launch_combine(mpe_ctx* c, const int32_t* ids, int T, int k, __nv_bfloat16* out) {
    const int n4 = c->H / 4;
    dim3 grid((unsigned)T, (unsigned)((n4 + 255) / 256));
    k_combine<<<grid, 256, 0, c->stream>>>(c->s.y, ids, T, k, c->H, c->E, out);
    c->launches++;
}

}  // namespace mpe
