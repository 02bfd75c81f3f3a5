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
// A (b = 3), A B (b = 4) or A B C (b = 8), each layer in its own pages. A
// layer is a chunk stream in the main format's layout at the layer's width
// (A: the 3-bit quarter layout, B: a 1-bit quarter with code pair m at bits
// m and 16 + m, C: the 4-bit one; chunks of 16 rows x 128 codes in the expert
// stream's order), so chunk n of every layer covers the same weights.
// Lowering a width frees the dropped layers' pages and encodes nothing;
// raising it encodes only the added layers (one read of the master).
//
// The forward pass runs the streaming kernels of the main format (decode.cu)
// through a context view over this store's pool: their copy warp fetches a
// share's run of every stored layer, their consumers merge the layers' bits
// in registers into the mma operands (the per-width scale and offset folded
// into the page-table mirror and the offset sums).
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
    uint8_t* d_gather = nullptr;
    size_t gather_cap = 0;
    // forward pass: a context view over the pool, with a page-table mirror
    // (width, layer A's first entry, the width's scale) and the first
    // entries of layers B and C
    mpe_ctx* view = nullptr;
    mpe::Pte* d_vpte = nullptr;
    uint32_t* d_lfirst = nullptr;
};

namespace mpe {
namespace {

constexpr int kLayers = 3;
__host__ __device__ constexpr int layer_bits(int L) { return L == 0 ? 3 : (L == 1 ? 1 : 4); }
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

// chunks of a layer in one page (whole chunks, 256 * layer bits bytes each)
__host__ __device__ inline uint32_t layer_cpp(int L, uint32_t page_bytes) {
    return page_bytes / (256u * layer_bits(L));
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

// One thread per (chunk, row, quarter) of one expert's job: the quarter's 32
// master weights -> u8 (once) -> the quarter's words of every layer in the
// job's mask, each into its layer's chunk. jobs: (expert, layer mask) pairs.
__global__ void __launch_bounds__(256)
k_px_encode(PxPaged P, uint8_t* pool, const void* const* masters, const int32_t* jobs,
            uint32_t n_chunks) {
    const int e = jobs[2 * blockIdx.y], mask = jobs[2 * blockIdx.y + 1];
    const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t c = tid >> 6;  // chunk in the expert stream's order
    if (c >= n_chunks) return;
    const int rho = (tid >> 2) & 15, q = tid & 3;
    const PxExpert x = P.ex[e];
    if (!(x.m >= 0.0f)) return;  // non-finite master
    const int H = P.H, F = P.F;
    const uint32_t nc1 = (uint32_t)(F / 16) * (H / 128);
    size_t src;  // the quarter's first weight in the master (W1 | W3 | W2)
    if (c < 2 * nc1) {  // W1 / W3 chunks alternate
        const uint32_t u = c >> 1, nj = H / 128;
        src = (size_t)(c & 1) * F * H + (size_t)(16 * (u / nj) + rho) * H + 128 * (u % nj) + 32 * q;
    } else {  // W2: tile pairs alternate by block column
        const uint32_t c2 = c - 2 * nc1, u = c2 >> 1, nj = F / 128;
        const uint32_t tau = 2 * (u / nj) + (c2 & 1);
        src = (size_t)2 * F * H + (size_t)(16 * tau + rho) * F + 128 * (u % nj) + 32 * q;
    }
    const float inv_m = x.m > 0.0f ? __frcp_rn(x.m) : 0.0f;
    const uint4* s4 =
        reinterpret_cast<const uint4*>(reinterpret_cast<const __half*>(masters[e]) + src);
    uint32_t wa[3] = {0, 0, 0}, wb = 0, wc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const uint4 q4 = __ldcs(s4 + v);
        const uint32_t h2[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int jw = 0; jw < 4; ++jw) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2[jw]));
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                const int i = 8 * v + 2 * jw + hlf;  // code of the quarter
                const uint32_t u8 = (uint32_t)prefix_code(hlf ? f.y : f.x, x.m, inv_m);
                const uint32_t A = u8 >> 5;
                if (i < 30) {  // 3-bit quarter: c'_{10v'+i'} at 16 (i'&1) + 3 (i'>>1)
                    const int ii = i % 10;
                    wa[i / 10] |= A << (16 * (ii & 1) + 3 * (ii >> 1));
                } else {       // bit n of c'_30 / c'_31 at bit 15 / 31 of word n
                    const int top = i == 30 ? 15 : 31;
#pragma unroll
                    for (int n = 0; n < 3; ++n) wa[n] |= ((A >> n) & 1u) << top;
                }
                wb |= ((u8 >> 4) & 1u) << (16 * (i & 1) + (i >> 1));            // 1-bit
                wc[i >> 3] |= (u8 & 15u) << (16 * (i & 1) + 4 * ((i & 7) >> 1));  // 4-bit
            }
        }
    }
#pragma unroll
    for (int L = 0; L < kLayers; ++L) {
        if (!((mask >> L) & 1)) continue;
        const uint32_t cpp = layer_cpp(L, P.page_bytes);
        const uint32_t page = P.pidx[x.first[L] + c / cpp];
        const int lb = layer_bits(L);
        uint32_t* dst = reinterpret_cast<uint32_t*>(
            pool + (size_t)page * P.page_bytes + (size_t)(c % cpp) * 256 * lb + rho * 16 * lb +
            q * 4 * lb);
        if (L == 0) { dst[0] = wa[0]; dst[1] = wa[1]; dst[2] = wa[2]; }
        else if (L == 1) { dst[0] = wb; }
        else { *reinterpret_cast<uint4*>(dst) = make_uint4(wc[0], wc[1], wc[2], wc[3]); }
    }
}

// Layer L of expert e in stream order (introspection).
__global__ void k_px_gather(PxPaged P, int e, int L, uint32_t n_words, uint32_t* dst) {
    const PxExpert x = P.ex[e];
    const uint32_t cw = 64u * layer_bits(L);  // words a chunk
    const uint32_t cpp = layer_cpp(L, P.page_bytes);
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n_words;
         i += gridDim.x * blockDim.x) {
        const uint32_t c = i / cw;
        const uint32_t page = P.pidx[x.first[L] + c / cpp];
        dst[i] = reinterpret_cast<const uint32_t*>(P.pool + (size_t)page * P.page_bytes +
                                                   (size_t)(c % cpp) * 4 * cw)[i % cw];
    }
}

// The forward pass's view of the table: per expert its width, layer A's first
// page-index entry and the width's scale (w^ = s (unpacked - offset) with
// s = m / 4, m / 8, m / 128 for 3, 4, 8 bits: powers of two, exact), and the
// first entries of layers B and C.
__global__ void k_px_view_table(const PxExpert* ex, Pte* vpte, uint32_t* lfirst, int E,
                                uint32_t pages_a) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const PxExpert x = ex[e];
    Pte t{};
    t.bits = (uint8_t)x.bits;
    t.scale = x.m * (x.bits == 3 ? 0.25f : (x.bits == 4 ? 0.125f : 0.0078125f));
    t.first = x.first[0];
    t.n_pages = pages_a;
    vpte[e] = t;
    lfirst[2 * e] = x.first[1];
    lfirst[2 * e + 1] = x.first[2];
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

uint32_t n_chunks_of(const mpe_prefix* p) { return (uint32_t)(3 * (p->F / 16) * (p->H / 128)); }

uint32_t layer_pages(int L, const mpe_prefix* p) {
    const uint32_t cpp = layer_cpp(L, p->page_bytes);
    return (n_chunks_of(p) + cpp - 1) / cpp;
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
    k_px_view_table<<<(p->E + 127) / 128, 128, 0, p->stream>>>(
        reinterpret_cast<const PxExpert*>(p->d_table), p->d_vpte, p->d_lfirst, p->E,
        layer_pages(0, p));
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
    const uint32_t nch = n_chunks_of(p);
    dim3 grid((nch * 64 + 255) / 256, (unsigned)n);  // a thread per chunk row quarter
    k_px_encode<<<grid, 256, 0, p->stream>>>(paged_of(p), p->pool, p->d_masters, p->d_jobs, nch);
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
        !ok(cudaMalloc(&p->d_masters, sizeof(void*) * p->E)) ||
        !ok(cudaMalloc(&p->d_vpte, sizeof(Pte) * p->E)) ||
        !ok(cudaMalloc(&p->d_lfirst, sizeof(uint32_t) * 2 * p->E)) ||
        !ok(cudaMemset(p->d_vpte, 0, sizeof(Pte) * p->E))) {
        cudaGetLastError();
        mpe_prefix_destroy(p);
        return report_global_error(MPE_ERR_CUDA, "prefix store: device allocation failed");
    }
    if (create_view(&p->view, dev, p->E, p->H, p->F, P, p->stream, p->pool, p->d_vpte, p->d_pidx,
                    p->pool_pages, p->d_lfirst) != MPE_OK) {
        mpe_prefix_destroy(p);
        return report_global_error(MPE_ERR_CUDA, "prefix store: forward view setup failed");
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
        mpe_destroy(p->view);
        cudaFree(p->pool); cudaFree(p->d_table); cudaFree(p->d_pidx); cudaFree(p->d_absmax);
        cudaFree(p->d_masters); cudaFree(p->d_jobs); cudaFree(p->d_gather);
        cudaFree(p->d_vpte); cudaFree(p->d_lfirst);
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
    const uint32_t n_words = n_chunks_of(p) * 64u * layer_bits(layer);
    const size_t need = (size_t)n_words * 4;
    if (bytes < need) return px_fail(p, MPE_ERR_INVALID, "buffer %zu < %zu bytes", bytes, need);
    PxDevice guard(p->device);
    if (need > p->gather_cap) {
        cudaFree(p->d_gather);
        p->d_gather = nullptr;
        p->gather_cap = 0;
        PCK(cudaMalloc(&p->d_gather, need));
        p->gather_cap = need;
    }
    k_px_gather<<<148, 256, 0, p->stream>>>(paged_of(p), e, layer, n_words,
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
    if (!p->quantized) return px_fail(p, MPE_ERR_ORDER, "moe_ffn before quantize");
    PxDevice guard(p->device);
    // the streaming path of the main format, reading this store's layers
    const int r = mpe_moe_ffn(p->view, x, T, ids, w, k, out);
    if (r != MPE_OK) return px_fail(p, r, "%s", mpe_last_error(p->view));
    return MPE_OK;
}

}  // extern "C"
