// Dynamic error compensation of salient input channels (streaming path).
//
// DecDEC summary, 3.1-3.2: a quantized linear W^ x becomes (W^ + R (.) M) x
// with R = W - W^ the residual and M a binary mask of whole input channels,
// those whose activations have the largest magnitudes (salient channels);
// Figure 4: compensating channels in that order lowers the error fastest.
// Per input row -- a token's x for the gate and up projections, a routed
// position's h for the down projection -- the n channels of largest |x|
// (ties to the lower index) are kept:
//   k_select_channels  the row's kept channels, ascending, by a two-pass radix
//                      select on the bf16 magnitude bits (an exact order on
//                      the stored values, so no rounding can change it);
//   k_comp_gateup,     sum over kept c of R[:, c] x_c for W1 and W3 (one more
//   k_comp_down        K-part slice beside the gate/up partials), or for W2
//                      (one more slice beside the down partials): the SwiGLU
//                      reduce and the combine add the slices in part order.
// R is not stored. The context keeps each expert's fp16 master transposed (the
// residual store: an input channel's weight column is contiguous), and
// R[:, c] = w - s k with the expert's current scale s and code
// k = round-half-even(w / s) is recomputed exactly (|w - s k| <= s / 2 is exact
// in fp32), so a kept channel's compensated weights are exactly the fp16
// master values. The store lives in device memory or, like the paper's
// CPU-side residuals, in mapped pinned host memory that the kernels read over
// the bus.
#include <cuda_fp16.h>

#include <algorithm>

#include "internal.h"

namespace mpe {
namespace {

constexpr int kHistCopies = 8;     // histogram copies, one per group of warps
constexpr int kCompThreads = 256;

// Exclusive prefix sum of one int per thread over a CTA of TH threads; *total
// gets the sum. Ends with a barrier, so the scratch can be reused at once.
template <int TH>
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    int before = 0, all = 0;
    for (int w = 0; w < TH / 32; ++w) {
        const int t = s_warp[w];
        if (w < warp) before += t;
        all += t;
    }
    *total = all;
    __syncthreads();
    return before + inc - v;
}

// Kept channels of row r: out[r][0 .. min(n, n_cols)), ascending. Rows at or
// beyond *n_rows_dev (when given) are skipped. One CTA of TH threads a row
// (1024 for long rows: short per-thread loops; 256 for short ones).
template <int TH>
__global__ void __launch_bounds__(TH)
k_select_channels(const __nv_bfloat16* rows, size_t ld, int n_cols, const int32_t* n_rows_dev,
                  int n, int32_t* out) {
    const int row = blockIdx.x;
    if (n_rows_dev && row >= *n_rows_dev) return;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(rows) + (size_t)row * ld;
    int32_t* o = out + (size_t)row * n;
    const int tid = threadIdx.x;
    if (n >= n_cols) {
        for (int c = tid; c < n_cols; c += TH) o[c] = c;
        return;
    }
    // the row's magnitude keys, read once (all loads in flight) into shared memory
    extern __shared__ uint16_t r[];
#pragma unroll 8
    for (int c = tid; c < n_cols; c += TH) r[c] = src[c] & 0x7FFF;
    __syncthreads();
    // per-warp histograms; lanes that hit the same bin add once (match_any), so
    // the common case -- most magnitudes in a few exponent bins -- costs a few
    // shared atomics per warp instruction instead of 32 on one address
    __shared__ int hist[kHistCopies][256];
    __shared__ int s_warp[TH / 32];
    __shared__ int s_b1, s_above, s_thr, s_take;
    const int lane = tid & 31, warp = tid >> 5;
    auto count = [&](int bin, bool valid) {
        const unsigned active = __ballot_sync(0xffffffffu, valid);
        if (!valid) return;
        const unsigned peers = __match_any_sync(active, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[warp % kHistCopies][bin], __popc(peers));
    };
    auto zero = [&]() {
        for (int i = tid; i < kHistCopies * 256; i += TH) (&hist[0][0])[i] = 0;
    };
    auto merged = [&](int bin) {
        int t = 0;
#pragma unroll
        for (int w = 0; w < kHistCopies; ++w) t += hist[w][bin];
        return t;
    };
    const int n_iter = (n_cols + TH - 1) / TH;  // whole warps iterate together
    // pass 1: the high byte of the 15 magnitude bits
    zero();
    __syncthreads();
    for (int it = 0; it < n_iter; ++it) {
        const int c = it * TH + tid;
        const bool v = c < n_cols;
        count(v ? r[c] >> 8 : 0, v);
    }
    __syncthreads();
    // the bin where the count from the top first reaches n: thread t < 256
    // holds bin 255 - t (the others 0), so an exclusive scan gives the keys in
    // the bins above it
    static_assert(TH >= 256, "one thread per bin");
    {
        int all;
        const int h = tid < 256 ? merged(255 - tid) : 0;
        const int above = block_exclusive_scan<TH>(h, s_warp, &all);
        if (tid < 256 && above < n && above + h >= n) {
            s_b1 = 255 - tid;
            s_above = above;  // keys whose high byte exceeds the bin
        }
    }
    __syncthreads();
    const int b1 = s_b1;
    // pass 2: the low byte among keys with that high byte
    zero();
    __syncthreads();
    for (int it = 0; it < n_iter; ++it) {
        const int c = it * TH + tid;
        const int key = c < n_cols ? r[c] : -1;
        const bool v = key >= 0 && (key >> 8) == b1;
        count(v ? key & 255 : 0, v);
    }
    __syncthreads();
    {
        int all;
        const int h = tid < 256 ? merged(255 - tid) : 0;
        const int above = s_above + block_exclusive_scan<TH>(h, s_warp, &all);
        if (tid < 256 && above < n && above + h >= n) {
            s_thr = (b1 << 8) | (255 - tid);  // the n-th largest key
            s_take = n - above;               // keys equal to it that are kept (lowest indices)
        }
    }
    __syncthreads();
    const int thr = s_thr, take = s_take;
    // pass 3: in index order, every key above the threshold and the first
    // `take` keys equal to it. Thread t walks its own contiguous segment, so
    // index order is thread order: one scan places each thread's equal keys,
    // a second its kept ones.
    const int seg = (n_cols + TH - 1) / TH;
    const int c_lo = min(n_cols, tid * seg), c_hi = min(n_cols, c_lo + seg);
    int n_gt = 0, n_eq = 0;
    for (int c = c_lo; c < c_hi; ++c) {
        const int key = r[c];
        n_gt += key > thr;
        n_eq += key == thr;
    }
    int total;
    const int eq_before = block_exclusive_scan<TH>(n_eq, s_warp, &total);
    const int eq_keep = max(0, min(n_eq, take - eq_before));
    int at = block_exclusive_scan<TH>(n_gt + eq_keep, s_warp, &total);
    int eq_seen = 0;
    for (int c = c_lo; c < c_hi; ++c) {
        const int key = r[c];
        bool keep = key > thr;
        if (key == thr) keep = eq_seen++ < eq_keep;
        if (keep && at < n) o[at++] = c;  // exactly n are kept; the bound is a safety net
    }
}

// Codes k = round(w / s) of a batch of weights by the quantizer's fast rule
// (w (1/s) rounded by the 1.5 * 2^23 add); if any lies within 2^-14 of a
// half-integer the batch is redone with the exact rule, so the codes are the
// encoder's. s = 0 (an all-zero expert: inv_s = 0) gives k = 0, and a
// non-finite master's NaN scale gives NaN, which propagates.
template <int NW>
__device__ __forceinline__ void batch_codes(const float (&w)[NW], float s, float inv_s,
                                            float (&kf)[NW]) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    bool near = false;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        const float r = __fmul_rn(w[i], inv_s);
        kf[i] = __fsub_rn(__fadd_rn(r, kRound), kRound);
        near |= fabsf(__fsub_rn(r, kf[i])) > kNearTie;
    }
    if (near) {
#pragma unroll
        for (int i = 0; i < NW; ++i) kf[i] = exact_code(w[i], s, inv_s);
    }
}

// One CTA per (route position, 512 output columns): the position's kept
// channels and their activations in shared memory, then per column pair the
// sum over kept channels of R[col][c] x_c, reading the store's contiguous
// column c. GATEUP: x is the token's row, the store holds W1^T and W3^T
// ([H][F] each) and the result goes to out[pos][0 .. F) (gate) and
// out[pos][F .. 2F) (up); down: x is h[pos], the store's W2^T is [F][H] and
// the result goes to out[pos][0 .. H).
template <bool GATEUP>
__global__ void __launch_bounds__(kCompThreads)
k_comp(const Pte* pte, const int32_t* perm, const int32_t* offsets, int E, int k,
       const __nv_bfloat16* x, const int32_t* sel, int n, int cnt, const __half* store, int H,
       int F, float* out) {
    __shared__ int s_c[MPE_MAX_COMP_CHANNELS];
    __shared__ float s_x[MPE_MAX_COMP_CHANNELS];
    __shared__ int s_off[MPE_MAX_EXPERTS + 1];
    // the prologue is a chain of dependent loads, so it is kept short: the
    // bucket offsets come in all at once and are searched in shared memory
    const int pos = blockIdx.x;
    const int a_pos = GATEUP ? __ldg(perm + pos) : 0;  // issued early, used below
    for (int i = threadIdx.x; i <= E; i += kCompThreads) s_off[i] = __ldg(offsets + i);
    __syncthreads();
    if (pos >= s_off[E]) return;
    int e = 0;
    {
        int hi = E - 1;
        while (e < hi) {  // the expert with s_off[e] <= pos < s_off[e + 1]
            const int mid = (e + hi + 1) >> 1;
            if (s_off[mid] <= pos) e = mid;
            else hi = mid - 1;
        }
    }
    const float s = __ldg(&pte[e].scale);
    const float inv_s = s > 0.0f ? __frcp_rn(s) : 0.0f;
    const int K = GATEUP ? H : F;   // input channels
    const int N = GATEUP ? F : H;   // output columns of one matrix
    const int row = GATEUP ? a_pos / k : pos;
    for (int i = threadIdx.x; i < cnt; i += kCompThreads) {
        const int c = __ldg(sel + (size_t)row * n + i);
        s_c[i] = c;
        s_x[i] = __bfloat162float(x[(size_t)row * K + c]);
    }
    __syncthreads();
    const int col = 2 * (blockIdx.y * kCompThreads + threadIdx.x);
    if (col >= N) return;
    const size_t mat = (size_t)H * F;
    const __half* base = store + (size_t)e * 3 * mat + (GATEUP ? 0 : 2 * mat);
    constexpr int NM = GATEUP ? 2 : 1;  // matrices: W1 and W3, or W2
    constexpr int NW = 8 * NM;          // weights of one batch of four channels
    // Batches of four kept channels (past the end: the last channel again,
    // weighted 0). The next batch's packed weights are loaded before the
    // current batch's codes and residuals R = w - s k (exact in fp32) are
    // computed and accumulated against the activations.
    auto fetch = [&](int i0, uint32_t (&pk)[4 * NM]) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const size_t at = (size_t)s_c[min(i0 + q, cnt - 1)] * N + col;
#pragma unroll
            for (int m = 0; m < NM; ++m)
                pk[q * NM + m] = __ldg(reinterpret_cast<const unsigned int*>(base + m * mat + at));
        }
    };
    float acc[2 * NM] = {};
    uint32_t cur[4 * NM];
    fetch(0, cur);
    for (int i = 0; i < cnt; i += 4) {
        uint32_t nxt[4 * NM];
        fetch(i + 4 < cnt ? i + 4 : i, nxt);
        float w[NW];
#pragma unroll
        for (int v = 0; v < 4 * NM; ++v) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&cur[v]));
            w[2 * v] = f.x;
            w[2 * v + 1] = f.y;
        }
        float kf[NW];
        batch_codes<NW>(w, s, inv_s, kf);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float xc = i + q < cnt ? s_x[i + q] : 0.0f;
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int wi = (q * NM + m) * 2 + h;
                    acc[2 * m + h] = __fmaf_rn(__fmaf_rn(-kf[wi], s, w[wi]), xc, acc[2 * m + h]);
                }
        }
#pragma unroll
        for (int v = 0; v < 4 * NM; ++v) cur[v] = nxt[v];
    }
    if constexpr (GATEUP) {
        float* dst = out + (size_t)pos * 2 * F + col;
        dst[0] = acc[0];
        dst[1] = acc[1];
        dst[F] = acc[2];
        dst[F + 1] = acc[3];
    } else {
        float* dst = out + (size_t)pos * H + col;
        dst[0] = acc[0];
        dst[1] = acc[1];
    }
}

// The residual store of one expert matrix: in [R][C] (row-major fp16) ->
// out [C][R], 32 x 32 tiles through shared memory. down == false: W1 and W3
// ([F][H]; grid z = 2 e + m), down == true: W2 ([H][F]; grid z = e).
__global__ void __launch_bounds__(256)
k_transpose_masters(const void* const* masters, int H, int F, bool down, __half* store) {
    __shared__ __half tile[32][34];
    const int e = down ? blockIdx.z : blockIdx.z >> 1;
    const int m = down ? 2 : (blockIdx.z & 1);
    const int R = down ? H : F, C = down ? F : H;
    const size_t mat = (size_t)H * F;
    const __half* in = reinterpret_cast<const __half*>(masters[e]) + m * mat;
    __half* out = store + (size_t)e * 3 * mat + m * mat;
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
#pragma unroll
    for (int i = 0; i < 32; i += 8)
        tile[ty + i][tx] = in[(size_t)(r0 + ty + i) * C + c0 + tx];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 32; i += 8)
        out[(size_t)(c0 + ty + i) * R + r0 + tx] = tile[tx][ty + i];
}

}  // namespace

void launch_transpose_masters(mpe_ctx* c, __half* store) {
    k_transpose_masters<<<dim3((unsigned)(c->H / 32), (unsigned)(c->F / 32), (unsigned)(2 * c->E)),
                          256, 0, c->stream>>>(c->d_masters, c->H, c->F, false, store);
    k_transpose_masters<<<dim3((unsigned)(c->F / 32), (unsigned)(c->H / 32), (unsigned)c->E), 256,
                          0, c->stream>>>(c->d_masters, c->H, c->F, true, store);
    c->launches += 2;
}

void launch_select_channels(mpe_ctx* c, const __nv_bfloat16* rows, size_t ld, int n_rows,
                            int n_cols, const int32_t* n_rows_dev, int n, int32_t* out,
                            cudaStream_t st) {
    if (n_rows <= 0) return;
    // the staged row: 2 bytes a column (rows longer than ~110K columns would
    // exceed a CTA's shared memory; the widths of this path are far below)
    const size_t smem = (size_t)n_cols * sizeof(uint16_t);
    auto launch = [&](auto kernel, int th) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kernel<<<(unsigned)n_rows, th, smem, st>>>(rows, ld, n_cols, n_rows_dev, n, out);
    };
    if (n_cols >= 8192)
        launch(k_select_channels<1024>, 1024);
    else
        launch(k_select_channels<256>, 256);
    if (c) c->launches++;
}

void launch_comp_gateup(mpe_ctx* c, const __nv_bfloat16* x, int k, size_t Tk, const int32_t* sel,
                        int n, const __half* store, float* out) {
    const int cnt = std::min(n, c->H);
    dim3 grid((unsigned)Tk, (unsigned)((c->F / 2 + kCompThreads - 1) / kCompThreads));
    k_comp<true><<<grid, kCompThreads, 0, c->stream>>>(c->d_pte, c->s.perm, c->s.offsets, c->E,
                                                       k, x, sel, n, cnt, store, c->H, c->F, out);
    c->launches++;
}

void launch_comp_down(mpe_ctx* c, size_t Tk, const int32_t* sel, int n, const __half* store,
                      float* out) {
    const int cnt = std::min(n, c->F);
    dim3 grid((unsigned)Tk, (unsigned)((c->H / 2 + kCompThreads - 1) / kCompThreads));
    k_comp<false><<<grid, kCompThreads, 0, c->stream>>>(c->d_pte, c->s.perm, c->s.offsets,
                                                        c->E, 1, c->s.h, sel, n, cnt, store,
                                                        c->H, c->F, out);
    c->launches++;
}

}  // namespace mpe
