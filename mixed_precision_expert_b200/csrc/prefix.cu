// Prefix-compatible variant: a nested quantization grid stored in layers, so a
// width change drops or adds layers instead of re-encoding the expert.
//
// The bitplane idea (store a high-precision code so that every lower precision
// is a prefix of it) applied to PagedWeight's paged experts ("Dynamic Paging";
// "Implementation Details": precision follows KV-cache occupancy). The main
// format's symmetric grid is not nested across widths, so this variant uses
// 2^b uniform bins over [-m, m] (m = max |w|), the bin centre as value:
//   u8 = clamp(floor(128 w / m) + 128, 0, 255),  u_b = u8 >> (8 - b),
//   w^_b = (m / 2^b) (2 u_b + 1 - 2^b).
// Layers: A = u8 >> 5 (3 bits), B = bit 4, C = u8 & 15; a b-bit expert holds
// A (b = 3), A B (b = 4) or A B C (b = 8), each layer in its own pages, rows
// of W1 | W3 | W2 in order, 32-code groups of 3 / 1 / 4 words (code i at bits
// bits*i of the group's little-endian string). Lowering a width frees the
// dropped layers' pages and encodes nothing; raising it encodes only the
// added layers (one read of the master).
//
// The forward pass is a plain CUDA-core grouped GEMV (bucket the routed
// positions by expert; per expert and 16-row tile, every layer group is
// unpacked once and multiplied with up to 8 of the expert's tokens at a time;
// SwiGLU; down; combine in slot order). It is the reference implementation
// of the variant, not tuned like the main format's kernels.
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "internal.h"

namespace mpe {
int report_global_error(int code, const char* msg);
}

struct mpe_prefix {
    int device = 0;
    int E = 0, H = 0, F = 0;
    uint32_t page_bytes = MPE_DEFAULT_PAGE_BYTES;
    uint32_t pool_pages = 0;
    cudaStream_t stream = nullptr;
    std::string err;
    uint8_t* pool = nullptr;
    // host bookkeeping: free bitmap, pages[e][layer], widths, master pointers
    std::vector<uint8_t> free;
    std::vector<std::vector<uint32_t>> pages;  // [e * 3 + layer]
    std::vector<uint8_t> bits;
    std::vector<const void*> masters;
    bool quantized = false;
    // device state
    void* d_table = nullptr;        // PxExpert[E]
    uint32_t* d_pidx = nullptr;     // page-index array
    uint32_t* d_absmax = nullptr;   // fp16 bits of m_e
    const void** d_masters = nullptr;
    int32_t* d_jobs = nullptr;      // (expert, layer) pairs to encode
    size_t jobs_cap = 0;
    // forward scratch
    int32_t* d_count = nullptr;     // [E + 1] offsets
    int32_t* d_list = nullptr;      // assignments grouped by expert
    __nv_bfloat16* d_h = nullptr;   // [T k][F]
    float* d_y = nullptr;           // [T k][H]
    size_t cap_assign = 0;
    uint8_t* d_gather = nullptr;
    size_t gather_cap = 0;
};

namespace mpe {
namespace {

constexpr int kLayers = 3;
constexpr int kGroupCodes = 32;
__host__ __device__ constexpr int layer_bits(int L) { return L == 0 ? 3 : (L == 1 ? 1 : 4); }
__host__ __device__ constexpr int group_words(int L) { return L == 0 ? 3 : (L == 1 ? 1 : 4); }
__host__ __device__ constexpr int layer_count(int b) { return b == 3 ? 1 : (b == 4 ? 2 : 3); }

struct PxExpert {
    uint32_t first[kLayers];  // a layer's first entry in the page-index array
    float m;                  // max |w| (0: all-zero expert)
    int bits;
};

struct PxPaged {
    const uint8_t* pool;
    const PxExpert* ex;
    const uint32_t* pidx;
    uint32_t page_bytes;
    int H, F;
};

__host__ __device__ inline uint32_t groups_per_page(int L, uint32_t page_bytes) {
    return page_bytes / (4u * group_words(L));
}

// Address of group g (in stream order) of layer L of an expert.
__device__ __forceinline__ const uint32_t* group_addr(const PxPaged& P, const PxExpert& x, int L,
                                                      uint32_t g) {
    const uint32_t gpp = groups_per_page(L, P.page_bytes);
    const uint32_t page = P.pidx[x.first[L] + g / gpp];
    return reinterpret_cast<const uint32_t*>(P.pool + (size_t)page * P.page_bytes +
                                             (size_t)(g % gpp) * 4 * group_words(L));
}

// u8 = clamp(floor(128 w / m) + 128, 0, 255) exactly: the rounded quotient's
// floor is off by at most one, and the sign of the single-rounded fma
// 128 w - k m is the sign of the exact difference.
__device__ __forceinline__ int prefix_code(float w, float m, float inv_m) {
    if (!(m > 0.0f)) return 128;
    const float w128 = 128.0f * w;  // exact
    float k = floorf(__fmul_rn(w128, inv_m));  // within one of the exact floor
    if (__fmaf_rn(-k, m, w128) < 0.0f) k -= 1.0f;
    else if (__fmaf_rn(-(k + 1.0f), m, w128) >= 0.0f) k += 1.0f;
    return min(255, max(0, (int)k + 128));
}

__global__ void __launch_bounds__(256)
k_px_absmax(const void* const* masters, int64_t n_vec, uint32_t* absmax) {
    const int e = blockIdx.y;
    const uint4* src = reinterpret_cast<const uint4*>(masters[e]);
    uint32_t mx = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = __ldcs(src + i);
        mx = __vmaxu2(mx, v.x & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.y & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.z & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.w & 0x7FFF7FFFu);
    }
    mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) atomicMax(absmax + e, mx);
}

// m of each expert into its table entry (a non-finite master gets NaN and a
// status bit; its layers are left unencoded).
__global__ void k_px_scales(PxExpert* ex, const uint32_t* absmax, int E, uint32_t* status) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const uint32_t m = absmax[e];
    if (m >= 0x7C00u) {
        ex[e].m = __int_as_float(0x7FC00000);
        if (status) set_status(status, MPE_STATUS_NONFINITE);
        return;
    }
    ex[e].m = __half2float(__ushort_as_half((unsigned short)m));
}

// One thread per 32-code group of one expert's job: the group's 32 master
// weights -> u8 (once) -> the bits of every layer in the job's mask -> each
// layer's words in its page. jobs: (expert, layer mask) pairs.
__global__ void __launch_bounds__(256)
k_px_encode(PxPaged P, uint8_t* pool, const void* const* masters, const int32_t* jobs,
            uint32_t n_groups) {
    const int e = jobs[2 * blockIdx.y], mask = jobs[2 * blockIdx.y + 1];
    const uint32_t g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n_groups) return;
    const PxExpert x = P.ex[e];
    if (!(x.m >= 0.0f)) return;  // non-finite master
    const float inv_m = x.m > 0.0f ? __frcp_rn(x.m) : 0.0f;
    const uint4* src = reinterpret_cast<const uint4*>(masters[e]) + (size_t)g * 4;
    uint32_t wa[3] = {0, 0, 0}, wb = 0, wc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const uint4 q = __ldcs(src + v);
        const uint32_t h2[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2[j]));
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                const int i = 8 * v + 2 * j + hlf;  // code index in the group
                const uint32_t u8 = (uint32_t)prefix_code(hlf ? f.y : f.x, x.m, inv_m);
                const int pos = 3 * i, wi = pos >> 5, sh = pos & 31;  // layer A
                wa[wi] |= (u8 >> 5) << sh;
                if (sh > 29) wa[wi + 1] |= (u8 >> 5) >> (32 - sh);
                wb |= ((u8 >> 4) & 1u) << i;                          // layer B
                wc[i >> 3] |= (u8 & 15u) << (4 * (i & 7));            // layer C
            }
        }
    }
#pragma unroll
    for (int L = 0; L < kLayers; ++L) {
        if (!((mask >> L) & 1)) continue;
        const uint32_t gpp = groups_per_page(L, P.page_bytes);
        const uint32_t page = P.pidx[x.first[L] + g / gpp];
        uint32_t* dst = reinterpret_cast<uint32_t*>(pool + (size_t)page * P.page_bytes +
                                                    (size_t)(g % gpp) * 4 * group_words(L));
        if (L == 0) { dst[0] = wa[0]; dst[1] = wa[1]; dst[2] = wa[2]; }
        else if (L == 1) { dst[0] = wb; }
        else { dst[0] = wc[0]; dst[1] = wc[1]; dst[2] = wc[2]; dst[3] = wc[3]; }
    }
}

// Layer L of expert e in stream order (introspection).
__global__ void k_px_gather(PxPaged P, int e, int L, uint32_t n_groups, uint32_t* dst) {
    const PxExpert x = P.ex[e];
    for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < n_groups;
         g += gridDim.x * blockDim.x) {
        const uint32_t* s = group_addr(P, x, L, g);
        for (int w = 0; w < group_words(L); ++w) dst[(size_t)g * group_words(L) + w] = s[w];
    }
}

// Bucket the assignments by expert (one CTA): off[e] .. off[e+1] of list
// hold expert e's assignment indices (any order: each assignment's result is
// computed on its own, and the combine sums slots in order). Invalid ids are
// left out and flagged.
constexpr int kBucketThreads = 1024;
__global__ void __launch_bounds__(kBucketThreads)
k_px_bucket(const int32_t* ids, int Tk, int E, int32_t* off, int32_t* list, uint32_t* status) {
    __shared__ int cnt[MPE_MAX_EXPERTS + 1];
    __shared__ int s_warp[kBucketThreads / 32];
    for (int e = threadIdx.x; e <= E; e += kBucketThreads) cnt[e] = 0;
    __syncthreads();
    for (int a = threadIdx.x; a < Tk; a += kBucketThreads) {
        const int e = ids[a];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else if (status) set_status(status, MPE_STATUS_BAD_EXPERT_ID);
    }
    __syncthreads();
    // exclusive scan of cnt[0 .. E) (E <= 1024: one entry a thread)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int v = threadIdx.x < E ? cnt[threadIdx.x] : 0;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += s_warp[w];
    const int excl = before + inc - v;
    __syncthreads();
    if (threadIdx.x < E) {
        off[threadIdx.x] = excl;
        cnt[threadIdx.x] = excl;  // now a cursor
    }
    if (threadIdx.x == kBucketThreads - 1) off[E] = before + inc;
    __syncthreads();
    for (int a = threadIdx.x; a < Tk; a += kBucketThreads) {
        const int e = ids[a];
        if (e >= 0 && e < E) list[atomicAdd(&cnt[e], 1)] = a;
    }
}

constexpr int kPxWarps = 8;   // a CTA: 8 warps x 2 rows = one 16-row tile
constexpr int kPxTok = 8;     // tokens multiplied per pass over the tile

// The stored words of group g of an expert (layers A, B, C as its width has).
struct GroupWords {
    uint32_t a0, a1, a2, b, c[4];
};

__device__ __forceinline__ GroupWords group_words_of(const PxPaged& P, const PxExpert& x,
                                                     uint32_t g) {
    GroupWords w{};
    const uint32_t* a = group_addr(P, x, 0, g);
    w.a0 = a[0];
    w.a1 = a[1];
    w.a2 = a[2];
    if (x.bits >= 4) w.b = *group_addr(P, x, 1, g);
    if (x.bits == 8) {
        const uint32_t* cc = group_addr(P, x, 2, g);
        w.c[0] = cc[0]; w.c[1] = cc[1]; w.c[2] = cc[2]; w.c[3] = cc[3];
    }
    return w;
}

// Code i of the group as c = 2 u_b + 1 - 2^b (an odd integer); i is a
// compile-time constant after unrolling.
__device__ __forceinline__ float code_at(const GroupWords& w, int i, int b) {
    const int pos = 3 * i;
    uint32_t u = pos < 32 ? (w.a0 >> pos) : (pos < 64 ? (w.a1 >> (pos - 32)) : (w.a2 >> (pos - 64)));
    if (pos < 32 && pos + 3 > 32) u |= w.a1 << (32 - pos);
    if (pos >= 32 && pos < 64 && pos + 3 > 64) u |= w.a2 << (64 - pos);
    u &= 7u;
    if (b >= 4) u = (u << 1) | ((w.b >> i) & 1u);
    if (b == 8) u = (u << 4) | ((w.c[i >> 3] >> (4 * (i & 7))) & 15u);
    return (float)(2 * (int)u + 1 - (1 << b));
}

// GATEUP: CTA (e, tile) computes h[a][r] = silu(s g) (s v) for the tile's 16
// features r and every assignment a of expert e (g, v from rows r of W1, W3);
// down: y[a][o] = s (W2 row o) . h[a] for the tile's 16 outputs o.
template <bool GATEUP>
__global__ void __launch_bounds__(kPxWarps * 32, 2)
k_px_gemv(PxPaged P, const int32_t* off, const int32_t* list, int k, const __nv_bfloat16* act,
          __nv_bfloat16* h_out, float* y_out) {
    extern __shared__ __align__(16) __nv_bfloat16 s_act[];  // [kPxTok][K]
    const int e = blockIdx.x;
    const int a0 = off[e], n = off[e + 1] - a0;
    if (n == 0) return;
    const PxExpert x = P.ex[e];
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float s = x.m / (float)(1 << x.bits);  // exact: m over a power of two
    const int r0 = blockIdx.y * 16 + 2 * warp;   // this warp's two rows (features / outputs)
    const int ng = K / kGroupCodes;
    for (int t0 = 0; t0 < n; t0 += kPxTok) {
        const int nt = min(kPxTok, n - t0);
        __syncthreads();  // the previous pass is done with s_act
        // staged code-position major, [i][t][g] for element k = 32 g + i of
        // token t, so the lanes (one group each) read consecutive words
        // a thread takes one (token, group): 64 contiguous bytes in, 32 stores
        // whose addresses run along g across the warp (no bank conflicts)
        for (int idx = threadIdx.x; idx < nt * ng; idx += blockDim.x) {
            const int t = idx / ng, g = idx - t * ng;
            const int a = list[a0 + t0 + t];
            const __nv_bfloat16* src =
                (GATEUP ? act + (size_t)(a / k) * H : act + (size_t)a * F) + g * kGroupCodes;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 v = reinterpret_cast<const uint4*>(src)[q];
                const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = 8 * q + 2 * j;  // elements i and i + 1
                    s_act[((size_t)i * kPxTok + t) * ng + g] =
                        __ushort_as_bfloat16((unsigned short)(wd[j] & 0xFFFFu));
                    s_act[((size_t)(i + 1) * kPxTok + t) * ng + g] =
                        __ushort_as_bfloat16((unsigned short)(wd[j] >> 16));
                }
            }
        }
        __syncthreads();
        // GATEUP: the two features r0, r0 + 1, each a W1 and a W3 row
        // (accumulators [feature][matrix][token]); down: two W2 rows. Lane l
        // takes groups l, l + 32, ...: a group's words are read once and its
        // codes, eight at a time, multiplied with every token of the pass.
        constexpr int NM = GATEUP ? 2 : 1;
        float acc[2][NM][kPxTok];
#pragma unroll
        for (int f = 0; f < 2; ++f)
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int t = 0; t < kPxTok; ++t) acc[f][m][t] = 0.0f;
        for (int g = lane; g < ng; g += 32) {
#pragma unroll
            for (int f = 0; f < 2; ++f)
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    // group index in the expert's stream: W1 rows, then W3 rows
                    // (H / 32 groups each), then W2 rows (F / 32 groups each)
                    const uint32_t gi =
                        GATEUP ? (uint32_t)(m * F + r0 + f) * (uint32_t)ng + g
                               : (uint32_t)(2 * F) * (uint32_t)(H / kGroupCodes) +
                                     (uint32_t)(r0 + f) * (uint32_t)ng + g;
                    const GroupWords gw = group_words_of(P, x, gi);
#pragma unroll
                    for (int i0 = 0; i0 < kGroupCodes; i0 += 8) {
                        float c[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) c[i] = code_at(gw, i0 + i, x.bits);
#pragma unroll
                        for (int t = 0; t < kPxTok; ++t) {
                            if (t >= nt) break;
                            const __nv_bfloat16* xg = s_act + (size_t)t * ng + g;
                            float sum = acc[f][m][t];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                sum = fmaf(c[i], __bfloat162float(xg[(size_t)(i0 + i) * kPxTok * ng]), sum);
                            acc[f][m][t] = sum;
                        }
                    }
                }
        }
#pragma unroll
        for (int f = 0; f < 2; ++f)
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int t = 0; t < kPxTok; ++t)
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        acc[f][m][t] += __shfl_xor_sync(0xffffffffu, acc[f][m][t], o);
        if (lane == 0) {
            for (int t = 0; t < nt; ++t) {
                const int a = list[a0 + t0 + t];
#pragma unroll
                for (int f = 0; f < 2; ++f) {
                    if constexpr (GATEUP) {
                        const float gv = s * acc[f][0][t], uv = s * acc[f][NM - 1][t];
                        h_out[(size_t)a * F + r0 + f] =
                            __float2bfloat16_rn(gv / (1.0f + __expf(-gv)) * uv);
                    } else {
                        y_out[(size_t)a * H + r0 + f] = s * acc[f][0][t];
                    }
                }
            }
        }
    }
}

// out[t] = bf16(sum_j w[t, j] y[t k + j]) over the valid slots, in slot order.
__global__ void k_px_combine(const float* y, const int32_t* ids, const float* w, int T, int k,
                             int E, int H, __nv_bfloat16* out) {
    const int t = blockIdx.x;
    for (int o = threadIdx.x; o < H; o += blockDim.x) {
        float acc = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int e = ids[t * k + j];
            if (e < 0 || e >= E) continue;
            acc = fmaf(w[t * k + j], y[(size_t)(t * k + j) * H + o], acc);
        }
        out[(size_t)t * H + o] = __float2bfloat16_rn(acc);
    }
}

int px_fail(mpe_prefix* p, int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    if (p) p->err = buf;
    return report_global_error(code, buf);
}

#define PCK(call)                                                                          \
    do {                                                                                   \
        cudaError_t e_ = (call);                                                           \
        if (e_ != cudaSuccess)                                                             \
            return px_fail(p, MPE_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

uint32_t layer_pages(int L, const mpe_prefix* p) {
    const uint64_t groups = (uint64_t)3 * p->H * p->F / kGroupCodes;
    const uint32_t gpp = groups_per_page(L, p->page_bytes);
    return (uint32_t)((groups + gpp - 1) / gpp);
}

struct PxDevice {
    explicit PxDevice(int dev) { cudaGetDevice(&old); cudaSetDevice(dev); }
    ~PxDevice() { cudaSetDevice(old); }
    int old = 0;
};

PxPaged paged_of(const mpe_prefix* p) {
    PxPaged P;
    P.pool = p->pool;
    P.ex = reinterpret_cast<const PxExpert*>(p->d_table);
    P.pidx = p->d_pidx;
    P.page_bytes = p->page_bytes;
    P.H = p->H;
    P.F = p->F;
    return P;
}

// Take n lowest free pages from `free` (a copy); false if too few.
bool take_pages(std::vector<uint8_t>& free, uint32_t n, std::vector<uint32_t>& out) {
    out.clear();
    for (uint32_t i = 0; i < free.size() && out.size() < n; ++i)
        if (free[i]) out.push_back(i);
    if (out.size() < n) return false;
    for (uint32_t i : out) free[i] = 0;
    return true;
}

// Upload the expert table and page-index array (layers A, B, C in order).
int upload_table(mpe_prefix* p) {
    std::vector<PxExpert> ex(p->E);
    std::vector<uint32_t> idx;
    for (int e = 0; e < p->E; ++e) {
        for (int L = 0; L < kLayers; ++L) {
            ex[e].first[L] = (uint32_t)idx.size();
            const auto& pg = p->pages[(size_t)e * kLayers + L];
            idx.insert(idx.end(), pg.begin(), pg.end());
        }
        ex[e].bits = p->bits[e];
        ex[e].m = 0.0f;  // filled on the device from the absmax
    }
    // keep m: the table's m entries are rewritten by k_px_scales after the copy
    PCK(cudaMemcpyAsync(p->d_table, ex.data(), sizeof(PxExpert) * p->E, cudaMemcpyHostToDevice,
                        p->stream));
    if (!idx.empty())
        PCK(cudaMemcpyAsync(p->d_pidx, idx.data(), sizeof(uint32_t) * idx.size(),
                            cudaMemcpyHostToDevice, p->stream));
    k_px_scales<<<(p->E + 127) / 128, 128, 0, p->stream>>>(
        reinterpret_cast<PxExpert*>(p->d_table), p->d_absmax, p->E, nullptr);
    // the host vectors die at return: wait for the copies
    PCK(cudaStreamSynchronize(p->stream));
    return MPE_OK;
}

int encode_jobs(mpe_prefix* p, const std::vector<int32_t>& jobs) {
    const int n = (int)jobs.size() / 2;
    if (n == 0) return MPE_OK;
    if ((size_t)jobs.size() > p->jobs_cap) {
        cudaFree(p->d_jobs);
        p->d_jobs = nullptr;
        p->jobs_cap = 0;
        PCK(cudaMalloc(&p->d_jobs, sizeof(int32_t) * jobs.size()));
        p->jobs_cap = jobs.size();
    }
    PCK(cudaMemcpyAsync(p->d_jobs, jobs.data(), sizeof(int32_t) * jobs.size(),
                        cudaMemcpyHostToDevice, p->stream));
    const uint32_t n_groups = (uint32_t)((uint64_t)3 * p->H * p->F / kGroupCodes);
    dim3 grid((n_groups + 255) / 256, (unsigned)n);
    k_px_encode<<<grid, 256, 0, p->stream>>>(paged_of(p), p->pool, p->d_masters, p->d_jobs,
                                            n_groups);
    PCK(cudaGetLastError());
    PCK(cudaStreamSynchronize(p->stream));  // the job list is host memory
    return MPE_OK;
}

}  // namespace
}  // namespace mpe

using namespace mpe;

extern "C" {

int mpe_prefix_create(mpe_prefix** out, const mpe_config* cfg) {
    if (!out || !cfg) return report_global_error(MPE_ERR_INVALID, "null argument");
    *out = nullptr;
    if (cfg->E < 1 || cfg->E > MPE_MAX_EXPERTS || cfg->H < 128 || cfg->F < 128 ||
        cfg->H % 128 || cfg->F % 128)
        return report_global_error(MPE_ERR_INVALID, "bad E, H or F");
    const uint32_t P = cfg->page_bytes ? cfg->page_bytes : MPE_DEFAULT_PAGE_BYTES;
    if (P < 4096 || P % 4096) return report_global_error(MPE_ERR_INVALID, "bad page_bytes");
    auto* p = new mpe_prefix();
    int dev = cfg->device;
    if (dev < 0) cudaGetDevice(&dev);
    p->device = dev;
    p->E = cfg->E;
    p->H = cfg->H;
    p->F = cfg->F;
    p->page_bytes = P;
    p->stream = reinterpret_cast<cudaStream_t>(cfg->stream);
    uint32_t all8 = 0;
    for (int L = 0; L < kLayers; ++L) all8 += layer_pages(L, p);
    p->pool_pages = cfg->pool_pages ? cfg->pool_pages : all8 * (uint32_t)p->E;
    PxDevice guard(dev);
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    if (!ok(cudaMalloc(&p->pool, (size_t)p->pool_pages * P)) ||
        !ok(cudaMalloc(&p->d_table, sizeof(PxExpert) * p->E)) ||
        !ok(cudaMalloc(&p->d_pidx, sizeof(uint32_t) * p->pool_pages)) ||
        !ok(cudaMalloc(&p->d_absmax, sizeof(uint32_t) * p->E)) ||
        !ok(cudaMalloc(&p->d_masters, sizeof(void*) * p->E))) {
        cudaGetLastError();
        mpe_prefix_destroy(p);
        return report_global_error(MPE_ERR_CUDA, "prefix store: device allocation failed");
    }
    p->free.assign(p->pool_pages, 1);
    p->pages.assign((size_t)p->E * kLayers, {});
    p->bits.assign(p->E, 0);
    *out = p;
    return MPE_OK;
}

void mpe_prefix_destroy(mpe_prefix* p) {
    if (!p) return;
    {
        PxDevice guard(p->device);
        cudaStreamSynchronize(p->stream);
        cudaFree(p->pool); cudaFree(p->d_table); cudaFree(p->d_pidx); cudaFree(p->d_absmax);
        cudaFree(p->d_masters); cudaFree(p->d_jobs); cudaFree(p->d_count); cudaFree(p->d_list);
        cudaFree(p->d_h); cudaFree(p->d_y); cudaFree(p->d_gather);
    }
    delete p;
}

const char* mpe_prefix_last_error(mpe_prefix* p) { return p ? p->err.c_str() : ""; }

int mpe_prefix_quantize(mpe_prefix* p, const void* const* master_f16, const uint8_t* bits) {
    if (!p) return report_global_error(MPE_ERR_INVALID, "null store");
    if (!master_f16 || !bits) return px_fail(p, MPE_ERR_INVALID, "null argument");
    for (int e = 0; e < p->E; ++e) {
        if (bits[e] != 3 && bits[e] != 4 && bits[e] != 8)
            return px_fail(p, MPE_ERR_INVALID, "bits[%d]=%d not 3/4/8", e, bits[e]);
        if (!master_f16[e] || (reinterpret_cast<uintptr_t>(master_f16[e]) & 15))
            return px_fail(p, MPE_ERR_INVALID, "master[%d] null or not 16-byte aligned", e);
    }
    PxDevice guard(p->device);
    // placement: lowest free pages, experts ascending, layers A, B, C
    std::vector<uint8_t> free(p->pool_pages, 1);
    std::vector<std::vector<uint32_t>> pages((size_t)p->E * kLayers);
    std::vector<int32_t> jobs;  // (expert, mask of the layers to encode)
    for (int e = 0; e < p->E; ++e) {
        for (int L = 0; L < layer_count(bits[e]); ++L)
            if (!take_pages(free, layer_pages(L, p), pages[(size_t)e * kLayers + L]))
                return px_fail(p, MPE_ERR_POOL, "page pool exhausted");
        jobs.push_back(e);
        jobs.push_back((1 << layer_count(bits[e])) - 1);
    }
    p->free = std::move(free);
    p->pages = std::move(pages);
    p->bits.assign(bits, bits + p->E);
    p->masters.assign(master_f16, master_f16 + p->E);
    PCK(cudaMemcpyAsync(p->d_masters, p->masters.data(), sizeof(void*) * p->E,
                        cudaMemcpyHostToDevice, p->stream));
    PCK(cudaMemsetAsync(p->d_absmax, 0, sizeof(uint32_t) * p->E, p->stream));
    const int64_t n_vec = (int64_t)3 * p->H * p->F / 8;
    k_px_absmax<<<dim3(64, (unsigned)p->E), 256, 0, p->stream>>>(p->d_masters, n_vec,
                                                                 p->d_absmax);
    PCK(cudaGetLastError());
    int r;
    if ((r = upload_table(p))) return r;
    if ((r = encode_jobs(p, jobs))) return r;
    p->quantized = true;
    return MPE_OK;
}

int mpe_prefix_repage(mpe_prefix* p, const uint8_t* new_bits, uint64_t* bytes_moved_out) {
    if (!p) return report_global_error(MPE_ERR_INVALID, "null store");
    if (!new_bits) return px_fail(p, MPE_ERR_INVALID, "null argument");
    if (!p->quantized) return px_fail(p, MPE_ERR_ORDER, "repage before quantize");
    for (int e = 0; e < p->E; ++e)
        if (new_bits[e] != 3 && new_bits[e] != 4 && new_bits[e] != 8)
            return px_fail(p, MPE_ERR_INVALID, "bits[%d]=%d not 3/4/8", e, new_bits[e]);
    PxDevice guard(p->device);
    std::vector<uint8_t> free = p->free;
    std::vector<std::vector<uint32_t>> pages = p->pages;
    std::vector<int> changed;
    for (int e = 0; e < p->E; ++e)
        if (new_bits[e] != p->bits[e]) changed.push_back(e);
    for (int e : changed)  // dropped layers first, ascending e
        for (int L = layer_count(new_bits[e]); L < kLayers; ++L) {
            for (uint32_t pg : pages[(size_t)e * kLayers + L]) free[pg] = 1;
            pages[(size_t)e * kLayers + L].clear();
        }
    std::vector<int32_t> jobs;
    uint64_t moved = 0;
    const uint64_t W = (uint64_t)3 * p->H * p->F;
    for (int e : changed) {  // then the added layers, ascending e
        int mask = 0;
        for (int L = layer_count(p->bits[e]); L < layer_count(new_bits[e]); ++L) {
            if (!take_pages(free, layer_pages(L, p), pages[(size_t)e * kLayers + L]))
                return px_fail(p, MPE_ERR_POOL, "page pool exhausted");  // nothing changed
            moved += W * layer_bits(L) / 8;
            mask |= 1 << L;
        }
        if (mask) {
            jobs.push_back(e);
            jobs.push_back(mask);
            moved += 2 * W;  // the master is read once
        }
    }
    // the forward passes launched so far may still read the dropped pages
    PCK(cudaStreamSynchronize(p->stream));
    p->free = std::move(free);
    p->pages = std::move(pages);
    p->bits.assign(new_bits, new_bits + p->E);
    int r;
    if ((r = upload_table(p))) return r;
    if ((r = encode_jobs(p, jobs))) return r;
    if (bytes_moved_out) *bytes_moved_out = moved;
    return MPE_OK;
}

int mpe_prefix_read_layer(mpe_prefix* p, int32_t e, int32_t layer, void* host_dst, size_t bytes) {
    if (!p) return report_global_error(MPE_ERR_INVALID, "null store");
    if (!p->quantized) return px_fail(p, MPE_ERR_ORDER, "read before quantize");
    if (e < 0 || e >= p->E || layer < 0 || layer >= kLayers || !host_dst)
        return px_fail(p, MPE_ERR_INVALID, "bad expert, layer or buffer");
    if (layer >= layer_count(p->bits[e])) return px_fail(p, MPE_ERR_INVALID, "layer not stored");
    const uint32_t n_groups = (uint32_t)((uint64_t)3 * p->H * p->F / kGroupCodes);
    const size_t need = (size_t)n_groups * 4 * group_words(layer);
    if (bytes < need) return px_fail(p, MPE_ERR_INVALID, "buffer %zu < %zu bytes", bytes, need);
    PxDevice guard(p->device);
    if (need > p->gather_cap) {
        cudaFree(p->d_gather);
        p->d_gather = nullptr;
        p->gather_cap = 0;
        PCK(cudaMalloc(&p->d_gather, need));
        p->gather_cap = need;
    }
    k_px_gather<<<148, 256, 0, p->stream>>>(paged_of(p), e, layer, n_groups,
                                            reinterpret_cast<uint32_t*>(p->d_gather));
    PCK(cudaGetLastError());
    PCK(cudaMemcpyAsync(host_dst, p->d_gather, need, cudaMemcpyDeviceToHost, p->stream));
    PCK(cudaStreamSynchronize(p->stream));
    return MPE_OK;
}

int mpe_prefix_get_absmax(mpe_prefix* p, float* m_host) {
    if (!p) return report_global_error(MPE_ERR_INVALID, "null store");
    if (!p->quantized || !m_host) return px_fail(p, MPE_ERR_INVALID, "not quantized or null");
    PxDevice guard(p->device);
    std::vector<PxExpert> ex(p->E);
    PCK(cudaMemcpyAsync(ex.data(), p->d_table, sizeof(PxExpert) * p->E, cudaMemcpyDeviceToHost,
                        p->stream));
    PCK(cudaStreamSynchronize(p->stream));
    for (int e = 0; e < p->E; ++e) m_host[e] = ex[e].m;
    return MPE_OK;
}

int mpe_prefix_moe_ffn(mpe_prefix* p, const void* x, int32_t T, const int32_t* ids,
                       const float* w, int32_t k, void* out) {
    if (!p) return report_global_error(MPE_ERR_INVALID, "null store");
    if (T < 0 || k < 1 || k > 32) return px_fail(p, MPE_ERR_INVALID, "bad T or k");
    if (T == 0) return MPE_OK;
    if (!x || !ids || !w || !out) return px_fail(p, MPE_ERR_INVALID, "null argument");
    if (reinterpret_cast<uintptr_t>(x) & 15) return px_fail(p, MPE_ERR_INVALID, "x not 16-byte aligned");
    if (!p->quantized) return px_fail(p, MPE_ERR_ORDER, "moe_ffn before quantize");
    PxDevice guard(p->device);
    const size_t Tk = (size_t)T * k;
    if (Tk > p->cap_assign) {
        PCK(cudaStreamSynchronize(p->stream));
        cudaFree(p->d_count); cudaFree(p->d_list); cudaFree(p->d_h); cudaFree(p->d_y);
        p->d_count = p->d_list = nullptr;
        p->d_h = nullptr;
        p->d_y = nullptr;
        p->cap_assign = 0;
        PCK(cudaMalloc(&p->d_count, sizeof(int32_t) * (p->E + 1)));
        PCK(cudaMalloc(&p->d_list, sizeof(int32_t) * Tk));
        PCK(cudaMalloc(&p->d_h, sizeof(__nv_bfloat16) * Tk * p->F));
        PCK(cudaMalloc(&p->d_y, sizeof(float) * Tk * p->H));
        p->cap_assign = Tk;
    }
    k_px_bucket<<<1, kBucketThreads, 0, p->stream>>>(ids, (int)Tk, p->E, p->d_count, p->d_list,
                                                     nullptr);
    const PxPaged P = paged_of(p);
    const size_t smem_gu = (size_t)kPxTok * p->H * sizeof(__nv_bfloat16);
    const size_t smem_dn = (size_t)kPxTok * p->F * sizeof(__nv_bfloat16);
    if (smem_gu > 227 * 1024 || smem_dn > 227 * 1024)
        return px_fail(p, MPE_ERR_INVALID, "H or F too large for the prefix forward pass");
    cudaFuncSetAttribute(k_px_gemv<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_gu);
    cudaFuncSetAttribute(k_px_gemv<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dn);
    k_px_gemv<true><<<dim3((unsigned)p->E, (unsigned)(p->F / 16)), kPxWarps * 32, smem_gu,
                      p->stream>>>(P, p->d_count, p->d_list, k,
                                   reinterpret_cast<const __nv_bfloat16*>(x), p->d_h, nullptr);
    k_px_gemv<false><<<dim3((unsigned)p->E, (unsigned)(p->H / 16)), kPxWarps * 32, smem_dn,
                       p->stream>>>(P, p->d_count, p->d_list, k, p->d_h, nullptr, p->d_y);
    k_px_combine<<<(unsigned)T, 256, 0, p->stream>>>(p->d_y, ids, w, T, k, p->E, p->H,
                                                    reinterpret_cast<__nv_bfloat16*>(out));
    PCK(cudaGetLastError());
    return MPE_OK;
}

}  // extern "C"
