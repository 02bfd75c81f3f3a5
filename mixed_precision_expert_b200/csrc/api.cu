// C ABI of libmpe: context, page allocator, page table and the call sequence
// of each entry point (see include/mpe.h for the contract of every call).
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <numeric>

#include "internal.h"

namespace mpe {
// selftest.cu: a bounded wait that runs out (status MPE_STATUS_WAIT_TIMEOUT)
void launch_wait_selftest(mpe_ctx* c, uint64_t limit_ns);
void route_set_smem_limits();
void decode_set_smem_limits();
}  // namespace mpe

using namespace mpe;

namespace {

thread_local std::string g_err;

int fail_global(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int fail(mpe_ctx* c, int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    if (c) c->err = buf;
    g_err = buf;
    return code;
}

#define CK(call)                                                                           \
    do {                                                                                   \
        cudaError_t e_ = (call);                                                           \
        if (e_ != cudaSuccess)                                                             \
            return fail(c, MPE_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

#define CKLAUNCH()                                                                         \
    do {                                                                                   \
        cudaError_t e_ = cudaGetLastError();                                               \
        if (e_ != cudaSuccess)                                                             \
            return fail(c, MPE_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e_)); \
    } while (0)

// Make the context's device current for the duration of a call.
struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        cudaGetDevice(&prev);
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur = -1;
        cudaGetDevice(&cur);
        if (prev >= 0 && cur != prev) cudaSetDevice(prev);
    }
};

int pages_needed(int b, int H, int F, uint32_t page_bytes) {
    const int nc = 3 * chunks_w1(H, F);
    const int cpp = chunks_per_page(b, page_bytes);
    return (nc + cpp - 1) / cpp;
}

bool valid_bits(int b) { return b == 3 || b == 4 || b == 8; }

// Lowest-index-first page moves for the experts whose width changes: their
// pages are released (ascending e), then allocated (ascending e) from the
// lowest free pages. Transactional: the plan is built beside the allocator
// (a copy of the free bitmap and new page lists for the changed experts only)
// and applied by commit_pages; on shortage it returns false and nothing changes.
struct PagePlan {
    std::vector<uint8_t> free;
    std::vector<std::pair<int, std::vector<uint32_t>>> moved;
};

// The lowest free page at or after `from` (pool_pages if none): memchr scans
// the byte map many pages at a time.
uint32_t next_free(const std::vector<uint8_t>& free, uint32_t from, uint32_t pool_pages) {
    if (from >= pool_pages) return pool_pages;
    const void* hit = std::memchr(free.data() + from, 1, pool_pages - from);
    return hit ? (uint32_t)(static_cast<const uint8_t*>(hit) - free.data()) : pool_pages;
}

// `need` lowest free pages from `cursor` on, taken in runs (freed pages come
// back as long runs): marks them used, writes them to `out` and advances the
// cursor; false if the pool runs out (the map is a plan's copy: nothing is
// committed then).
bool take_lowest(std::vector<uint8_t>& free, uint32_t& cursor, uint32_t pool_pages, int need,
                 std::vector<uint32_t>& out) {
    out.resize((size_t)need);
    uint8_t* f = free.data();
    int got = 0;
    while (got < need) {
        cursor = next_free(free, cursor, pool_pages);
        if (cursor >= pool_pages) return false;
        while (got < need && cursor < pool_pages && f[cursor]) {
            f[cursor] = 0;
            out[(size_t)got++] = cursor++;
        }
    }
    return true;
}

bool plan_pages(const mpe_ctx* c, const std::vector<uint8_t>& new_bits, PagePlan& plan,
                std::vector<int>& changed) {
    changed.clear();
    for (int e = 0; e < c->E; ++e)
        if (new_bits[e] != c->bits[e]) changed.push_back(e);
    plan.free = c->alloc.free;
    plan.moved.clear();
    for (int e : changed)
        for (uint32_t p : c->alloc.pages[e]) plan.free[p] = 1;
    uint32_t cursor = 0;
    for (int e : changed) {
        const int need = pages_needed(new_bits[e], c->H, c->F, c->page_bytes);
        std::vector<uint32_t> pg;
        if (!take_lowest(plan.free, cursor, c->pool_pages, need, pg)) return false;
        plan.moved.emplace_back(e, std::move(pg));
    }
    return true;
}

void commit_pages(mpe_ctx* c, PagePlan& plan, const std::vector<uint8_t>& new_bits) {
    c->alloc.free.swap(plan.free);
    for (auto& m : plan.moved) c->alloc.pages[m.first] = std::move(m.second);
    c->bits = new_bits;
}

// Overlapped repage plan: the changed experts' old pages stay allocated (work
// on the current page table still reads them), their new pages come from the
// pages free now (lowest first, ascending e); `release` lists the old pages,
// returned to the pool at the commit. Transactional like plan_pages.
bool plan_pages_overlapped(const mpe_ctx* c, const std::vector<uint8_t>& new_bits,
                           PagePlan& plan, std::vector<int>& changed,
                           std::vector<uint32_t>& release) {
    changed.clear();
    release.clear();
    for (int e = 0; e < c->E; ++e)
        if (new_bits[e] != c->bits[e]) changed.push_back(e);
    plan.free = c->alloc.free;
    plan.moved.clear();
    uint32_t cursor = 0;
    for (int e : changed) {
        const int need = pages_needed(new_bits[e], c->H, c->F, c->page_bytes);
        std::vector<uint32_t> pg;
        if (!take_lowest(plan.free, cursor, c->pool_pages, need, pg)) return false;
        release.insert(release.end(), c->alloc.pages[e].begin(), c->alloc.pages[e].end());
        plan.moved.emplace_back(e, std::move(pg));
    }
    return true;
}

// Side stream, events and the second page table, made on the first
// overlapped repage.
int ensure_side(mpe_ctx* c) {
    if (c->side) return MPE_OK;
    // the lowest priority: when the forward calls run on a stream of higher
    // priority, the block scheduler starts their CTAs before the encode's
    int least = 0, greatest = 0;
    CK(cudaDeviceGetStreamPriorityRange(&least, &greatest));
    CK(cudaStreamCreateWithPriority(&c->side, cudaStreamNonBlocking, least));
    CK(cudaEventCreateWithFlags(&c->side_done, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&c->old_table_free, cudaEventDisableTiming));
    CK(cudaEventRecord(c->old_table_free, c->stream));
    CK(cudaMalloc(&c->d_pte_next, sizeof(Pte) * c->E));
    CK(cudaMalloc(&c->d_pidx_next, sizeof(uint32_t) * c->pool_pages));
    CK(cudaMalloc(&c->d_list_next, sizeof(int32_t) * c->E));
    CK(cudaMallocHost(&c->h_pte_next_pinned, sizeof(Pte) * c->E));
    CK(cudaMallocHost(&c->h_pidx_next_pinned, sizeof(uint32_t) * c->pool_pages));
    CK(cudaMallocHost(&c->h_list_next_pinned, sizeof(int32_t) * c->E));
    return MPE_OK;
}

// Switch to the prepared page table: later work on the context stream waits
// for the side stream's encode; the old pages return to the pool, and the
// next overlapped repage will not write them before the work launched so far
// (which may read them) has finished.
int commit_pending(mpe_ctx* c) {
    if (!c->pending) return MPE_OK;
    CK(cudaStreamWaitEvent(c->stream, c->side_done, 0));
    c->epoch++;  // the table pointers swap
    std::swap(c->d_pte, c->d_pte_next);
    std::swap(c->d_pidx, c->d_pidx_next);
    c->pidx_count = c->pidx_count_next;
    for (uint32_t pg : c->pending_release) c->alloc.free[pg] = 1;
    c->pending_release.clear();
    CK(cudaEventRecord(c->old_table_free, c->stream));
    c->pending = false;
    return MPE_OK;
}

// Rebuild the page table (compact page-index array, experts in order) in the
// pinned staging and upload it (async; the staging is reused only after the
// previous upload finished).
// The page table of the allocator's current state into host staging.
uint32_t fill_table(mpe_ctx* c, Pte* h_pte, uint32_t* h_pidx) {
    uint32_t n = 0;
    for (int e = 0; e < c->E; ++e) {
        Pte& p = c->pte[e];
        const std::vector<uint32_t>& pg = c->alloc.pages[e];
        p.bits = c->bits[e];
        p.first = n;
        p.n_pages = (uint32_t)pg.size();
        if (!pg.empty()) std::memcpy(h_pidx + n, pg.data(), sizeof(uint32_t) * pg.size());
        n += (uint32_t)pg.size();
    }
    std::memcpy(h_pte, c->pte.data(), sizeof(Pte) * c->E);
    return n;
}

int upload_table(mpe_ctx* c) {
    CK(cudaEventSynchronize(c->upload_done));
    const uint32_t n = fill_table(c, c->h_pte_pinned, c->h_pidx_pinned);
    c->pidx_count = n;
    CK(cudaMemcpyAsync(c->d_pte, c->h_pte_pinned, sizeof(Pte) * c->E, cudaMemcpyHostToDevice,
                       c->stream));
    if (n)
        CK(cudaMemcpyAsync(c->d_pidx, c->h_pidx_pinned, sizeof(uint32_t) * n,
                           cudaMemcpyHostToDevice, c->stream));
    CK(cudaEventRecord(c->upload_done, c->stream));
    return MPE_OK;
}

int upload_list(mpe_ctx* c, const std::vector<int>& list) {
    // the list staging is shared with the previous call: wait for its upload
    CK(cudaEventSynchronize(c->list_done));
    for (size_t i = 0; i < list.size(); ++i) c->h_list_pinned[i] = list[i];
    CK(cudaMemcpyAsync(c->d_list, c->h_list_pinned, sizeof(int32_t) * list.size(),
                       cudaMemcpyHostToDevice, c->stream));
    CK(cudaEventRecord(c->list_done, c->stream));
    return MPE_OK;
}

template <typename T>
int dev_alloc(mpe_ctx* c, T** p, size_t n) {
    *p = nullptr;
    if (n == 0) n = 1;
    CK(cudaMalloc(reinterpret_cast<void**>(p), n * sizeof(T)));
    c->epoch++;  // a captured forward may hold the old pointer
    return MPE_OK;
}

void free_scratch(Scratch& s) {
    cudaFree(s.perm); cudaFree(s.inv); cudaFree(s.offsets); cudaFree(s.wg); cudaFree(s.n_wg);
    cudaFree(s.hist); cudaFree(s.h); cudaFree(s.y); cudaFree(s.part); cudaFree(s.task_ctr);
    cudaFree(s.xp);
    for (int i = 0; i < 2; ++i) {
        cudaFree(s.x_stage[i]); cudaFree(s.ids_stage[i]); cudaFree(s.w_stage[i]);
        cudaFree(s.out_stage[i]);
    }
    s = Scratch{};
}

int wg_capacity(int E, size_t Tk, int group) {
    return (int)(std::min<size_t>((size_t)E, Tk) + Tk / group + 1);
}

int ensure_scratch(mpe_ctx* c, size_t Tk) {
    Scratch& s = c->s;
    if (Tk <= s.cap_assign && s.perm) return MPE_OK;
    CK(cudaStreamSynchronize(c->stream));
    // the host staging survives (it is sized by ensure_stage)
    Scratch keep;
    keep.stage_tokens = s.stage_tokens;
    for (int i = 0; i < 2; ++i) {
        keep.x_stage[i] = s.x_stage[i]; keep.ids_stage[i] = s.ids_stage[i];
        keep.w_stage[i] = s.w_stage[i]; keep.out_stage[i] = s.out_stage[i];
        s.x_stage[i] = nullptr; s.ids_stage[i] = nullptr; s.w_stage[i] = nullptr;
        s.out_stage[i] = nullptr;
    }
    free_scratch(s);
    s.stage_tokens = keep.stage_tokens;
    for (int i = 0; i < 2; ++i) {
        s.x_stage[i] = keep.x_stage[i]; s.ids_stage[i] = keep.ids_stage[i];
        s.w_stage[i] = keep.w_stage[i]; s.out_stage[i] = keep.out_stage[i];
    }
    size_t cap = 1024;
    while (cap < Tk) cap *= 2;
    const int E = c->E;
    int r;
    if ((r = dev_alloc(c, &s.perm, cap))) return r;
    if ((r = dev_alloc(c, &s.inv, cap))) return r;
    if ((r = dev_alloc(c, &s.offsets, E + 1))) return r;
    if ((r = dev_alloc(c, &s.wg, 3 * (size_t)wg_capacity(E, cap, 1)))) return r;
    if ((r = dev_alloc(c, &s.n_wg, 4))) return r;
    s.hist_cap = ((cap + 1023) / 1024) * E;
    if ((r = dev_alloc(c, &s.hist, s.hist_cap))) return r;
    if ((r = dev_alloc(c, &s.h, cap * c->F))) return r;
    s.y_cap = cap * c->H;
    if ((r = dev_alloc(c, &s.y, s.y_cap))) return r;
    s.cap_assign = cap;
    if ((r = dev_alloc(c, &s.task_ctr, 6))) return r;
    CK(cudaMemset(s.task_ctr, 0, 6 * sizeof(int32_t)));
    return MPE_OK;
}

int ensure_stage(mpe_ctx* c, int T, int k) {
    Scratch& s = c->s;
    if ((size_t)T <= s.stage_tokens && s.x_stage[0] && (size_t)T * k <= s.cap_assign) return MPE_OK;
    // host-buffer calls still in flight use the staging
    if (c->host_stream) CK(cudaStreamSynchronize(c->host_stream));
    if (c->in_stream) CK(cudaStreamSynchronize(c->in_stream));
    if (c->out_stream) CK(cudaStreamSynchronize(c->out_stream));
    CK(cudaStreamSynchronize(c->stream));
    size_t cap = 64;
    while (cap < (size_t)T) cap *= 2;
    int r;
    for (int i = 0; i < 2; ++i) {
        cudaFree(s.x_stage[i]); cudaFree(s.ids_stage[i]); cudaFree(s.w_stage[i]);
        cudaFree(s.out_stage[i]);
        s.x_stage[i] = s.out_stage[i] = nullptr;
        s.ids_stage[i] = nullptr;
        s.w_stage[i] = nullptr;
    }
    s.stage_tokens = 0;
    for (int i = 0; i < 2; ++i) {
        if ((r = dev_alloc(c, reinterpret_cast<__nv_bfloat16**>(&s.x_stage[i]), cap * c->H))) return r;
        if ((r = dev_alloc(c, reinterpret_cast<__nv_bfloat16**>(&s.out_stage[i]), cap * c->H)))
            return r;
        if ((r = dev_alloc(c, &s.ids_stage[i], cap * 32))) return r;
        if ((r = dev_alloc(c, &s.w_stage[i], cap * 32))) return r;
    }
    s.stage_tokens = cap;
    return MPE_OK;
}

// Run the allocator kernel on the context's stream and fetch the widths
// (pinned staging; the expert sizes are uploaded once).
int run_allocate(mpe_ctx* c, const double* p, uint64_t B, std::vector<uint8_t>& out,
                 cudaStream_t st) {
    const int E = c->E;
    for (int e = 0; e < E; ++e)
        if (!(p[e] >= 0.0) || !std::isfinite(p[e]))
            return fail(c, MPE_ERR_INVALID, "importance p[%d] must be finite and >= 0", e);
    const uint64_t w_e = (uint64_t)3 * c->H * c->F;
    const uint64_t sum_w = w_e * E;
    if (B < 3 * sum_w) return fail(c, MPE_ERR_INFEASIBLE, "budget %llu < 3 * sum W = %llu",
                                   (unsigned long long)B, (unsigned long long)(3 * sum_w));
    const uint64_t g = w_e;
    const bool measured = c->allocator == MPE_ALLOCATOR_MEASURED;
    const bool exact = c->allocator == MPE_ALLOCATOR_EXACT || measured;
    if (measured && !c->loss_valid) {
        // the master never changes while the context lives: measure once
        if (!c->absmax_valid) return fail(c, MPE_ERR_ORDER, "measured loss before quantize_experts");
        launch_measure_mse(c, c->d_mse_acc, c->d_loss);
        CKLAUNCH();
        if (st != c->stream) CK(cudaStreamSynchronize(c->stream));  // once per context
        c->loss_valid = true;
    }
    if (c->memo_valid && c->memo_allocator == c->allocator && c->memo_B == B &&
        std::memcmp(c->memo_p.data(), p, sizeof(double) * E) == 0) {
        out = c->memo_bits;
        return MPE_OK;
    }
    uint64_t R = (B >= 8 * sum_w && !measured) ? 0 : (B - 3 * sum_w) / g;
    R = std::min<uint64_t>(R, 5 * (sum_w / g));
    if (exact && R + 1 > MPE_ALLOC_STATE_CAP) return fail(c, MPE_ERR_STATE_CAP, "too many states");
    const size_t need = exact ? allocate_choice_bytes(E, R) : 0;
    if (need > c->choice_cap) {
        cudaFree(c->d_choice);
        CK(cudaMalloc(&c->d_choice, need));
        c->choice_cap = need;
    }
    if (!c->w_uploaded) {
        for (int e = 0; e < E; ++e) c->h_w_pinned[e] = w_e;
        CK(cudaMemcpyAsync(c->d_W, c->h_w_pinned, sizeof(uint64_t) * E, cudaMemcpyHostToDevice,
                           st));
        c->w_uploaded = true;
    }
    // the staging is free: the previous call ended with a synchronize
    std::memcpy(c->h_p_pinned, p, sizeof(double) * E);
    CK(cudaMemcpyAsync(c->d_p, c->h_p_pinned, sizeof(double) * E, cudaMemcpyHostToDevice,
                       st));
    if (exact)
        launch_allocate(st, c->d_p, measured ? c->d_loss : nullptr, c->d_W, E, B, sum_w, g,
                        c->d_bits_out, c->d_alloc_status, c->d_choice, c->d_D,
                        MPE_ALLOC_STATE_CAP, R);
    else
        launch_allocate_proportional(st, c->d_p, c->d_W, E, B, sum_w, c->d_bits_out,
                                     c->d_alloc_status);
    c->launches++;
    CKLAUNCH();
    CK(cudaMemcpyAsync(c->h_alloc_pinned, c->d_alloc_status, sizeof(int32_t),
                       cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(c->h_alloc_pinned + 1, c->d_bits_out, E, cudaMemcpyDeviceToHost,
                       st));
    CK(cudaStreamSynchronize(st));
    const int32_t status = c->h_alloc_pinned[0];
    if (status == 1) return fail(c, MPE_ERR_INFEASIBLE, "budget below 3 bits per weight");
    if (status == 3) return fail(c, MPE_ERR_STATE_CAP, "too many allocation states");
    const uint8_t* bits = reinterpret_cast<const uint8_t*>(c->h_alloc_pinned + 1);
    out.assign(bits, bits + E);
    c->memo_p.assign(p, p + E);
    c->memo_B = B;
    c->memo_allocator = c->allocator;
    c->memo_bits = out;
    c->memo_valid = true;
    return MPE_OK;
}

}  // namespace

namespace mpe {
// Records a message for mpe_last_error_global (context-free calls in other files).
int report_global_error(int code, const char* msg) { return fail_global(code, "%s", msg); }

int create_view(mpe_ctx** out, int device, int E, int H, int F, uint32_t page_bytes,
                cudaStream_t stream, uint8_t* pool, Pte* d_pte, uint32_t* d_pidx,
                uint32_t pool_pages, const uint32_t* lfirst) {
    *out = nullptr;
    auto* c = new mpe_ctx();
    c->view = true;
    c->device = device;
    DeviceGuard guard(device);
    c->E = E;
    c->H = H;
    c->F = F;
    c->page_bytes = page_bytes;
    c->path = MPE_PATH_DECODE;
    c->stream = stream;
    c->pool_pages = pool_pages;
    c->pool = pool;
    c->d_pte = d_pte;
    c->d_pidx = d_pidx;
    c->px_lfirst = lfirst;
    c->absmax_valid = true;  // the viewed store checks its own state
    if (cudaMalloc(&c->d_status, sizeof(uint32_t)) != cudaSuccess ||
        cudaMemset(c->d_status, 0, sizeof(uint32_t)) != cudaSuccess) {
        cudaGetLastError();
        mpe_destroy(c);
        return fail_global(MPE_ERR_CUDA, "view: device allocation failed");
    }
    route_set_smem_limits();
    decode_set_smem_limits();
    *out = c;
    return MPE_OK;
}
}  // namespace mpe

extern "C" {

int32_t mpe_version(void) { return 100; }

const char* mpe_last_error_global(void) { return g_err.c_str(); }

const char* mpe_last_error(mpe_ctx* c) { return c ? c->err.c_str() : g_err.c_str(); }

uint64_t mpe_kernel_launches(mpe_ctx* c) { return c ? c->launches : 0; }

int mpe_create(mpe_ctx** out, const mpe_config* cfg) {
    if (!out || !cfg) return fail_global(MPE_ERR_INVALID, "null argument");
    *out = nullptr;
    if (cfg->E < 1 || cfg->E > MPE_MAX_EXPERTS)
        return fail_global(MPE_ERR_INVALID, "E=%d out of range", cfg->E);
    if (cfg->H <= 0 || cfg->F <= 0 || cfg->H % 128 || cfg->F % 128)
        return fail_global(MPE_ERR_INVALID, "H and F must be positive multiples of 128");
    const uint32_t pb = cfg->page_bytes ? cfg->page_bytes : MPE_DEFAULT_PAGE_BYTES;
    if (pb < 4096 || pb % 4096)
        return fail_global(MPE_ERR_INVALID, "page_bytes must be a multiple of 4096");
    if (cfg->path < MPE_PATH_AUTO || cfg->path > MPE_PATH_PREFILL)
        return fail_global(MPE_ERR_INVALID, "bad path");
    int dev = cfg->device;
    if (dev < 0 && cudaGetDevice(&dev) != cudaSuccess)
        return fail_global(MPE_ERR_CUDA, "no CUDA device");
    auto* c = new mpe_ctx();
    c->device = dev;
    DeviceGuard guard(dev);
    c->E = cfg->E;
    c->H = cfg->H;
    c->F = cfg->F;
    c->page_bytes = pb;
    c->path = cfg->path;
    c->stream = reinterpret_cast<cudaStream_t>(cfg->stream);
    c->pool_pages = cfg->pool_pages ? cfg->pool_pages
                                    : (uint32_t)(c->E * pages_needed(8, c->H, c->F, pb));
    auto bail = [&](int r) {
        mpe_destroy(c);
        return r;
    };
    int r;
    const size_t pool_bytes = (size_t)c->pool_pages * pb;
    if (cudaMalloc(&c->pool, pool_bytes) != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return fail_global(MPE_ERR_CUDA, "pool allocation of %zu bytes failed", pool_bytes);
    }
    if ((r = dev_alloc(c, &c->d_pte, c->E))) return bail(r);
    if ((r = dev_alloc(c, &c->d_pidx, c->pool_pages))) return bail(r);
    if ((r = dev_alloc(c, &c->d_absmax, c->E))) return bail(r);
    if ((r = dev_alloc(c, &c->d_status, 1))) return bail(r);
    if ((r = dev_alloc(c, &c->d_masters, c->E))) return bail(r);
    if ((r = dev_alloc(c, &c->d_list, c->E))) return bail(r);
    if ((r = dev_alloc(c, &c->d_p, c->E))) return bail(r);
    if ((r = dev_alloc(c, &c->d_W, c->E))) return bail(r);
    if ((r = dev_alloc(c, &c->d_bits_out, c->E))) return bail(r);
    if ((r = dev_alloc(c, &c->d_alloc_status, 1))) return bail(r);
    if ((r = dev_alloc(c, &c->d_D, 2 * (size_t)MPE_ALLOC_STATE_CAP))) return bail(r);
    if ((r = dev_alloc(c, &c->d_loss, 3 * (size_t)c->E))) return bail(r);
    if ((r = dev_alloc(c, &c->d_mse_acc, 6 * (size_t)c->E))) return bail(r);
    if (cudaMallocHost(&c->h_pte_pinned, sizeof(Pte) * c->E) != cudaSuccess ||
        cudaMallocHost(&c->h_pidx_pinned, sizeof(uint32_t) * c->pool_pages) != cudaSuccess ||
        cudaMallocHost(&c->h_list_pinned, sizeof(int32_t) * c->E) != cudaSuccess ||
        cudaMallocHost(&c->h_masters_pinned, sizeof(void*) * c->E) != cudaSuccess ||
        cudaMallocHost(&c->h_p_pinned, sizeof(double) * c->E) != cudaSuccess ||
        cudaMallocHost(&c->h_w_pinned, sizeof(uint64_t) * c->E) != cudaSuccess ||
        cudaMallocHost(&c->h_alloc_pinned, sizeof(int32_t) * (1 + (c->E + 3) / 4)) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->upload_done, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->list_done, cudaEventDisableTiming) != cudaSuccess)
        return bail(fail_global(MPE_ERR_CUDA, "host staging allocation failed"));
    if (cudaMemset(c->d_pte, 0, sizeof(Pte) * c->E) != cudaSuccess ||
        cudaMemset(c->d_status, 0, sizeof(uint32_t)) != cudaSuccess ||
        cudaEventRecord(c->upload_done, c->stream) != cudaSuccess ||
        cudaEventRecord(c->list_done, c->stream) != cudaSuccess)
        return bail(fail_global(MPE_ERR_CUDA, "initialisation failed"));
    c->bits.assign(c->E, 0);
    c->pte.assign(c->E, Pte{});
    c->masters.assign(c->E, nullptr);
    c->alloc.free.assign(c->pool_pages, 1);
    c->alloc.pages.assign(c->E, {});
    route_set_smem_limits();
    decode_set_smem_limits();
    prefill_set_smem_limits();
    if (cudaGetLastError() != cudaSuccess)
        return bail(fail_global(MPE_ERR_CUDA, "kernel attribute setup failed"));
    *out = c;
    return MPE_OK;
}

void mpe_destroy(mpe_ctx* c) {
    if (!c) return;
    {
        DeviceGuard guard(c->device);
        cudaStreamSynchronize(c->stream);
        // host-buffer calls still queued read and write the staging
        for (cudaStream_t st : {c->host_stream, c->in_stream, c->out_stream})
            if (st) cudaStreamSynchronize(st);
        if (c->side) {
            cudaStreamSynchronize(c->side);
            cudaStreamDestroy(c->side);
            cudaEventDestroy(c->side_done);
            cudaEventDestroy(c->old_table_free);
            cudaFree(c->d_pte_next); cudaFree(c->d_pidx_next); cudaFree(c->d_list_next);
            cudaFreeHost(c->h_pte_next_pinned); cudaFreeHost(c->h_pidx_next_pinned);
            cudaFreeHost(c->h_list_next_pinned);
        }
        free_scratch(c->s);
        if (c->view) {  // the viewed store owns these
            c->pool = nullptr;
            c->d_pte = nullptr;
            c->d_pidx = nullptr;
        }
        cudaFree(c->pool); cudaFree(c->d_pte); cudaFree(c->d_pidx); cudaFree(c->d_absmax);
        cudaFree(c->d_status); cudaFree(c->d_masters); cudaFree(c->d_list); cudaFree(c->d_p);
        cudaFree(c->d_W); cudaFree(c->d_bits_out); cudaFree(c->d_alloc_status);
        cudaFree(c->d_choice); cudaFree(c->d_D); cudaFree(c->d_gather);
        cudaFree(c->d_loss); cudaFree(c->d_mse_acc);
        cudaFree(c->comp_dev); cudaFree(c->sel_x); cudaFree(c->sel_h);
        for (int i = 0; i < 2; ++i)
            if (c->fwd_exec[i]) cudaGraphExecDestroy(c->fwd_exec[i]);
        if (c->host_stream) {
            cudaStreamSynchronize(c->host_stream);
            cudaStreamDestroy(c->host_stream);
        }
        for (cudaStream_t st : {c->in_stream, c->out_stream, c->alloc_stream})
            if (st) {
                cudaStreamSynchronize(st);
                cudaStreamDestroy(st);
            }
        if (c->host_ready) cudaEventDestroy(c->host_ready);
        for (int i = 0; i < 2; ++i) {
            if (c->in_done[i]) cudaEventDestroy(c->in_done[i]);
            if (c->fwd_done[i]) cudaEventDestroy(c->fwd_done[i]);
            if (c->out_done[i]) cudaEventDestroy(c->out_done[i]);
        }
        if (c->comp_host) cudaFreeHost(c->comp_host);
        cudaFreeHost(c->h_pte_pinned); cudaFreeHost(c->h_pidx_pinned);
        cudaFreeHost(c->h_list_pinned); cudaFreeHost(c->h_masters_pinned);
        cudaFreeHost(c->h_p_pinned); cudaFreeHost(c->h_w_pinned); cudaFreeHost(c->h_alloc_pinned);
        if (c->upload_done) cudaEventDestroy(c->upload_done);
        if (c->list_done) cudaEventDestroy(c->list_done);
        for (const ProfileRecord& r : c->prof) {
            cudaEventDestroy(r.start);
            cudaEventDestroy(r.stop);
        }
        for (cudaEvent_t e : c->event_pool) cudaEventDestroy(e);
        cudaGetLastError();
    }
    delete c;
}

int mpe_set_stream(mpe_ctx* c, void* stream) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    c->stream = reinterpret_cast<cudaStream_t>(stream);
    c->epoch++;
    return MPE_OK;
}

int mpe_set_path(mpe_ctx* c, int32_t path) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (path < MPE_PATH_AUTO || path > MPE_PATH_PREFILL) return fail(c, MPE_ERR_INVALID, "bad path");
    c->path = path;
    c->epoch++;
    return MPE_OK;
}

namespace {

// The exact program on a temporary device copy of its inputs; loss (host
// float64[E][3]) may be null for the fixed L(b).
int allocate_exact(const double* p, const double* loss, const uint64_t* W, int32_t E,
                   uint64_t B_bits, uint8_t* bits_out) {
    if (!p || !W || !bits_out) return fail_global(MPE_ERR_INVALID, "null argument");
    if (E < 1 || E > MPE_MAX_EXPERTS) return fail_global(MPE_ERR_INVALID, "E out of range");
    uint64_t sum_w = 0, g = 0;
    for (int e = 0; e < E; ++e) {
        if (W[e] == 0) return fail_global(MPE_ERR_INVALID, "W[%d] = 0", e);
        if (!(p[e] >= 0.0) || !std::isfinite(p[e]))
            return fail_global(MPE_ERR_INVALID, "p[%d] must be finite and >= 0", e);
        if (loss)
            for (int i = 0; i < 3; ++i)
                if (!(loss[3 * e + i] >= 0.0) || !std::isfinite(loss[3 * e + i]))
                    return fail_global(MPE_ERR_INVALID, "loss[%d][%d] must be finite and >= 0", e, i);
        sum_w += W[e];
        g = std::gcd(g, W[e]);
    }
    if (B_bits < 3 * sum_w) return fail_global(MPE_ERR_INFEASIBLE, "budget below 3 bits per weight");
    uint64_t R = (B_bits >= 8 * sum_w && !loss) ? 0 : (B_bits - 3 * sum_w) / g;
    R = std::min<uint64_t>(R, 5 * (sum_w / g));
    if (R + 1 > MPE_ALLOC_STATE_CAP) return fail_global(MPE_ERR_STATE_CAP, "too many states");
    double* dp = nullptr; uint64_t* dW = nullptr; uint8_t* db = nullptr; int32_t* ds = nullptr;
    uint8_t* dch = nullptr; double* dD = nullptr; double* dl = nullptr;
    int rc = MPE_OK;
    int32_t st = -1;
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    if (!ok(cudaMalloc(&dp, sizeof(double) * E)) || !ok(cudaMalloc(&dW, sizeof(uint64_t) * E)) ||
        !ok(cudaMalloc(&db, E)) || !ok(cudaMalloc(&ds, sizeof(int32_t))) ||
        !ok(cudaMalloc(&dch, allocate_choice_bytes(E, R))) ||
        !ok(cudaMalloc(&dD, 2 * sizeof(double) * (R + 1))) ||
        (loss && !ok(cudaMalloc(&dl, 3 * sizeof(double) * E))) ||
        !ok(cudaMemcpy(dp, p, sizeof(double) * E, cudaMemcpyHostToDevice)) ||
        (loss && !ok(cudaMemcpy(dl, loss, 3 * sizeof(double) * E, cudaMemcpyHostToDevice))) ||
        !ok(cudaMemcpy(dW, W, sizeof(uint64_t) * E, cudaMemcpyHostToDevice))) {
        rc = fail_global(MPE_ERR_CUDA, "allocate_bits: %s", cudaGetErrorString(cudaGetLastError()));
    } else {
        launch_allocate(nullptr, dp, dl, dW, E, B_bits, sum_w, g, db, ds, dch, dD,
                        MPE_ALLOC_STATE_CAP, R);
        if (!ok(cudaGetLastError()) || !ok(cudaMemcpy(&st, ds, sizeof(int32_t), cudaMemcpyDeviceToHost)) ||
            !ok(cudaMemcpy(bits_out, db, E, cudaMemcpyDeviceToHost)))
            rc = fail_global(MPE_ERR_CUDA, "allocate_bits kernel: %s",
                             cudaGetErrorString(cudaGetLastError()));
        else if (st == 1)
            rc = fail_global(MPE_ERR_INFEASIBLE, "budget below 3 bits per weight");
        else if (st == 3)
            rc = fail_global(MPE_ERR_STATE_CAP, "too many allocation states");
    }
    cudaFree(dp); cudaFree(dW); cudaFree(db); cudaFree(ds); cudaFree(dch); cudaFree(dD);
    cudaFree(dl);
    return rc;
}

}  // namespace

int mpe_allocate_bits(const double* p, const uint64_t* W, int32_t E, uint64_t B_bits,
                      uint8_t* bits_out) {
    return allocate_exact(p, nullptr, W, E, B_bits, bits_out);
}

int mpe_allocate_bits_table(const double* p, const double* loss, const uint64_t* W, int32_t E,
                            uint64_t B_bits, uint8_t* bits_out) {
    if (!loss) return fail_global(MPE_ERR_INVALID, "null argument");
    return allocate_exact(p, loss, W, E, B_bits, bits_out);
}

int mpe_measure_loss(mpe_ctx* c, double* loss_host) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (!loss_host) return fail(c, MPE_ERR_INVALID, "null argument");
    if (!c->absmax_valid) return fail(c, MPE_ERR_ORDER, "measure_loss before quantize_experts");
    if (!c->loss_valid) {
        launch_measure_mse(c, c->d_mse_acc, c->d_loss);
        CKLAUNCH();
        c->loss_valid = true;
    }
    CK(cudaMemcpyAsync(loss_host, c->d_loss, 3 * sizeof(double) * c->E, cudaMemcpyDeviceToHost,
                       c->stream));
    CK(cudaStreamSynchronize(c->stream));
    return MPE_OK;
}

int mpe_allocate_bits_proportional(const double* p, const uint64_t* W, int32_t E,
                                   uint64_t B_bits, uint8_t* bits_out) {
    if (!p || !W || !bits_out) return fail_global(MPE_ERR_INVALID, "null argument");
    if (E < 1 || E > MPE_MAX_EXPERTS) return fail_global(MPE_ERR_INVALID, "E out of range");
    uint64_t sum_w = 0;
    for (int e = 0; e < E; ++e) {
        if (W[e] == 0) return fail_global(MPE_ERR_INVALID, "W[%d] = 0", e);
        if (!(p[e] >= 0.0) || !std::isfinite(p[e]))
            return fail_global(MPE_ERR_INVALID, "p[%d] must be finite and >= 0", e);
        sum_w += W[e];
    }
    if (B_bits < 3 * sum_w) return fail_global(MPE_ERR_INFEASIBLE, "budget below 3 bits per weight");
    double* dp = nullptr; uint64_t* dW = nullptr; uint8_t* db = nullptr; int32_t* ds = nullptr;
    int rc = MPE_OK;
    int32_t st = -1;
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    if (!ok(cudaMalloc(&dp, sizeof(double) * E)) || !ok(cudaMalloc(&dW, sizeof(uint64_t) * E)) ||
        !ok(cudaMalloc(&db, E)) || !ok(cudaMalloc(&ds, sizeof(int32_t))) ||
        !ok(cudaMemcpy(dp, p, sizeof(double) * E, cudaMemcpyHostToDevice)) ||
        !ok(cudaMemcpy(dW, W, sizeof(uint64_t) * E, cudaMemcpyHostToDevice))) {
        rc = fail_global(MPE_ERR_CUDA, "allocate_bits_proportional: %s",
                         cudaGetErrorString(cudaGetLastError()));
    } else {
        launch_allocate_proportional(nullptr, dp, dW, E, B_bits, sum_w, db, ds);
        if (!ok(cudaGetLastError()) || !ok(cudaMemcpy(&st, ds, sizeof(int32_t), cudaMemcpyDeviceToHost)) ||
            !ok(cudaMemcpy(bits_out, db, E, cudaMemcpyDeviceToHost)))
            rc = fail_global(MPE_ERR_CUDA, "allocate_bits_proportional kernel: %s",
                             cudaGetErrorString(cudaGetLastError()));
        else if (st == 1)
            rc = fail_global(MPE_ERR_INFEASIBLE, "budget below 3 bits per weight");
    }
    cudaFree(dp); cudaFree(dW); cudaFree(db); cudaFree(ds);
    return rc;
}

int mpe_set_compensation(mpe_ctx* c, int32_t n_channels, int32_t store) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (n_channels < 0 || n_channels > MPE_MAX_COMP_CHANNELS)
        return fail(c, MPE_ERR_INVALID, "n_channels %d outside 0 .. %d", n_channels,
                    MPE_MAX_COMP_CHANNELS);
    if (store != MPE_STORE_DEVICE && store != MPE_STORE_HOST)
        return fail(c, MPE_ERR_INVALID, "bad store %d", store);
    DeviceGuard guard(c->device);
    CK(cudaStreamSynchronize(c->stream));
    const bool keep = n_channels > 0 && c->comp_store && c->comp_store_kind == store;
    if (!keep) {
        cudaFree(c->comp_dev);
        if (c->comp_host) cudaFreeHost(c->comp_host);
        c->comp_dev = nullptr;
        c->comp_host = nullptr;
        c->comp_store = nullptr;
        c->comp_n = 0;
    }
    c->epoch++;
    if (n_channels == 0) return MPE_OK;
    if (!c->absmax_valid) return fail(c, MPE_ERR_ORDER, "compensation before quantize_experts");
    if (!keep) {
        const size_t bytes = (size_t)3 * c->H * c->F * c->E * sizeof(__half);
        if (store == MPE_STORE_DEVICE) {
            if (cudaMalloc(&c->comp_dev, bytes) != cudaSuccess) {
                cudaGetLastError();
                return fail(c, MPE_ERR_CUDA, "residual store: %zu bytes of device memory", bytes);
            }
            c->comp_store = c->comp_dev;
        } else {
            void* dev = nullptr;
            if (cudaHostAlloc(&c->comp_host, bytes, cudaHostAllocMapped | cudaHostAllocPortable) !=
                    cudaSuccess ||
                cudaHostGetDevicePointer(&dev, c->comp_host, 0) != cudaSuccess) {
                cudaGetLastError();
                if (c->comp_host) cudaFreeHost(c->comp_host);
                c->comp_host = nullptr;
                return fail(c, MPE_ERR_CUDA, "residual store: %zu bytes of mapped host memory",
                            bytes);
            }
            c->comp_store = reinterpret_cast<const __half*>(dev);
        }
        c->comp_store_kind = store;
        launch_transpose_masters(c, const_cast<__half*>(c->comp_store));
        CKLAUNCH();
        CK(cudaStreamSynchronize(c->stream));
    }
    c->comp_n = n_channels;
    c->epoch++;
    return MPE_OK;
}

int mpe_get_kept_channels(mpe_ctx* c, int32_t which, int32_t* idx_host, size_t cap) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (!idx_host || (which != 0 && which != 1)) return fail(c, MPE_ERR_INVALID, "bad argument");
    if (c->comp_n == 0 || c->last_T == 0) return fail(c, MPE_ERR_ORDER, "no compensated forward yet");
    const size_t rows = which == 0 ? (size_t)c->last_T : (size_t)c->last_T * c->last_k;
    const size_t need = rows * (size_t)c->comp_n;
    if (cap < need) return fail(c, MPE_ERR_INVALID, "cap %zu < %zu entries", cap, need);
    DeviceGuard guard(c->device);
    CK(cudaMemcpyAsync(idx_host, which == 0 ? c->sel_x : c->sel_h, need * sizeof(int32_t),
                       cudaMemcpyDeviceToHost, c->stream));
    CK(cudaStreamSynchronize(c->stream));
    return MPE_OK;
}

int mpe_selftest_wait(mpe_ctx* c, uint64_t limit_ns) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (limit_ns == 0 || limit_ns > 1000000000ull)
        return fail(c, MPE_ERR_INVALID, "limit_ns must be in 1 .. 1e9");
    DeviceGuard guard(c->device);
    launch_wait_selftest(c, limit_ns);
    CKLAUNCH();
    CK(cudaStreamSynchronize(c->stream));
    return MPE_OK;
}

int mpe_select_salient(const void* rows_bf16, int32_t n_rows, int32_t n_cols, int32_t n,
                       int32_t* idx_out, void* stream) {
    if (n_rows < 0 || n_cols < 1 || n < 1 || n > MPE_MAX_COMP_CHANNELS)
        return fail_global(MPE_ERR_INVALID, "bad n_rows %d, n_cols %d or n %d", n_rows, n_cols, n);
    if (n_rows == 0) return MPE_OK;
    if (!rows_bf16 || !idx_out) return fail_global(MPE_ERR_INVALID, "null argument");
    launch_select_channels(nullptr, reinterpret_cast<const __nv_bfloat16*>(rows_bf16),
                           (size_t)n_cols, n_rows, n_cols, nullptr, n, idx_out,
                           reinterpret_cast<cudaStream_t>(stream));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_global(MPE_ERR_CUDA, "select_salient: %s", cudaGetErrorString(e));
    return MPE_OK;
}

int mpe_set_allocator(mpe_ctx* c, int32_t allocator) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (allocator != MPE_ALLOCATOR_EXACT && allocator != MPE_ALLOCATOR_PROPORTIONAL &&
        allocator != MPE_ALLOCATOR_MEASURED)
        return fail(c, MPE_ERR_INVALID, "bad allocator %d", allocator);
    c->allocator = allocator;
    return MPE_OK;
}

int mpe_quantize_experts(mpe_ctx* c, const void* const* master_f16, const uint8_t* bits) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (!master_f16 || !bits) return fail(c, MPE_ERR_INVALID, "null argument");
    for (int e = 0; e < c->E; ++e) {
        if (!valid_bits(bits[e])) return fail(c, MPE_ERR_INVALID, "bits[%d]=%d not 3/4/8", e, bits[e]);
        if (!master_f16[e] || (reinterpret_cast<uintptr_t>(master_f16[e]) & 15))
            return fail(c, MPE_ERR_INVALID, "master[%d] null or not 16-byte aligned", e);
    }
    DeviceGuard guard(c->device);
    int r0;
    if ((r0 = commit_pending(c))) return r0;
    std::vector<uint8_t> nb(bits, bits + c->E);
    PagePlan plan;
    std::vector<int> changed;
    if (!plan_pages(c, nb, plan, changed)) return fail(c, MPE_ERR_POOL, "page pool exhausted");
    commit_pages(c, plan, nb);
    int r;
    if ((r = upload_table(c))) return r;
    // master pointers and the all-experts list
    CK(cudaEventSynchronize(c->upload_done));
    for (int e = 0; e < c->E; ++e) {
        c->masters[e] = master_f16[e];
        c->h_masters_pinned[e] = master_f16[e];
    }
    CK(cudaMemcpyAsync(c->d_masters, c->h_masters_pinned, sizeof(void*) * c->E,
                       cudaMemcpyHostToDevice, c->stream));
    std::vector<int> all(c->E);
    std::iota(all.begin(), all.end(), 0);
    if ((r = upload_list(c, all))) return r;
    CK(cudaMemsetAsync(c->d_absmax, 0, sizeof(uint32_t) * c->E, c->stream));
    launch_absmax(c, c->d_list, c->E);
    launch_scales(c);
    launch_encode(c, c->d_list, c->E);
    if (c->comp_n > 0) launch_transpose_masters(c, const_cast<__half*>(c->comp_store));
    CKLAUNCH();
    c->absmax_valid = true;
    c->loss_valid = false;
    c->memo_valid = false;  // a measured-loss allocation depends on the master
    return MPE_OK;
}

int mpe_repage(mpe_ctx* c, uint64_t B_bits, const double* p, int32_t* n_changed_out) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (!p) return fail(c, MPE_ERR_INVALID, "null importances");
    if (!c->absmax_valid) return fail(c, MPE_ERR_ORDER, "repage before quantize_experts");
    DeviceGuard guard(c->device);
    std::vector<uint8_t> nb;
    int r;
    if ((r = commit_pending(c))) return r;
    if (!c->alloc_stream) {
        int least = 0, greatest = 0;
        CK(cudaDeviceGetStreamPriorityRange(&least, &greatest));
        CK(cudaStreamCreateWithPriority(&c->alloc_stream, cudaStreamNonBlocking, greatest));
    }
    // the widths: solved beside the work already queued on the context stream
    // (the solve reads only the importances and sizes), so the host plans the
    // page moves while that work runs; the moves and the encode are queued on
    // the context stream behind it
    if ((r = run_allocate(c, p, B_bits, nb, c->alloc_stream))) return r;
    if (nb == c->bits) {  // no width changes: the pages, table and scales stand
        if (n_changed_out) *n_changed_out = 0;
        return MPE_OK;
    }
    PagePlan plan;
    std::vector<int> changed;
    if (!plan_pages(c, nb, plan, changed)) return fail(c, MPE_ERR_POOL, "page pool exhausted");
    commit_pages(c, plan, nb);
    if ((r = upload_table(c))) return r;
    launch_scales(c);
    if (!changed.empty()) {
        if ((r = upload_list(c, changed))) return r;
        launch_encode(c, c->d_list, (int)changed.size());
    }
    CKLAUNCH();
    if (n_changed_out) *n_changed_out = (int32_t)changed.size();
    return MPE_OK;
}

int mpe_repage_async(mpe_ctx* c, uint64_t B_bits, const double* p, int32_t* n_changed_out) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (!p) return fail(c, MPE_ERR_INVALID, "null importances");
    if (!c->absmax_valid) return fail(c, MPE_ERR_ORDER, "repage before quantize_experts");
    if (c->pending) return fail(c, MPE_ERR_ORDER, "an overlapped repage is pending: commit it");
    DeviceGuard guard(c->device);
    int r;
    if ((r = ensure_side(c))) return r;
    std::vector<uint8_t> nb;
    if ((r = run_allocate(c, p, B_bits, nb, c->side))) return r;
    PagePlan plan;
    std::vector<int> changed;
    std::vector<uint32_t> release;
    if (!plan_pages_overlapped(c, nb, plan, changed, release))
        return fail(c, MPE_ERR_POOL, "page pool exhausted (an overlapped repage needs free "
                                     "pages for the changed experts' new pages)");
    commit_pages(c, plan, nb);
    // the next table (run_allocate synchronised the side stream, so its
    // staging is free)
    c->pidx_count_next = fill_table(c, c->h_pte_next_pinned, c->h_pidx_next_pinned);
    CK(cudaMemcpyAsync(c->d_pte_next, c->h_pte_next_pinned, sizeof(Pte) * c->E,
                       cudaMemcpyHostToDevice, c->side));
    if (c->pidx_count_next)
        CK(cudaMemcpyAsync(c->d_pidx_next, c->h_pidx_next_pinned,
                           sizeof(uint32_t) * c->pidx_count_next, cudaMemcpyHostToDevice,
                           c->side));
    // pages freed by the last commit may still be read by work launched before it
    CK(cudaStreamWaitEvent(c->side, c->old_table_free, 0));
    launch_scales_on(c, c->d_pte_next, c->side);
    if (!changed.empty()) {
        for (size_t i = 0; i < changed.size(); ++i) c->h_list_next_pinned[i] = changed[i];
        CK(cudaMemcpyAsync(c->d_list_next, c->h_list_next_pinned, sizeof(int32_t) * changed.size(),
                           cudaMemcpyHostToDevice, c->side));
        PagedExperts P = paged(c);
        P.pte = c->d_pte_next;
        P.pidx = c->d_pidx_next;
        launch_encode_on(c, P, c->d_list_next, (int)changed.size(), c->side);
    }
    CKLAUNCH();
    CK(cudaEventRecord(c->side_done, c->side));
    c->pending_release = std::move(release);
    c->pending = true;
    if (n_changed_out) *n_changed_out = (int32_t)changed.size();
    return MPE_OK;
}

int mpe_repage_commit(mpe_ctx* c, int32_t wait, int32_t* committed) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    DeviceGuard guard(c->device);
    if (c->pending && !wait) {
        const cudaError_t q = cudaEventQuery(c->side_done);
        if (q == cudaErrorNotReady) {
            if (committed) *committed = 0;
            return MPE_OK;
        }
        if (q != cudaSuccess) return fail(c, MPE_ERR_CUDA, "%s", cudaGetErrorString(q));
    }
    int r;
    if ((r = commit_pending(c))) return r;
    if (committed) *committed = 1;
    return MPE_OK;
}

static cudaEvent_t take_event(mpe_ctx* c) {
    if (!c->event_pool.empty()) {
        cudaEvent_t e = c->event_pool.back();
        c->event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Brackets one kernel launch with an event pair when tracing is on.
struct KernelSpan {
    mpe_ctx* c;
    ProfileRecord r{};
    KernelSpan(mpe_ctx* ctx, int slot) : c(ctx) {
        if (!c->profiling) return;
        r.slot = slot;
        r.start = take_event(c);
        r.stop = take_event(c);
        cudaEventRecord(r.start, c->stream);
    }
    ~KernelSpan() {
        if (!c->profiling || !r.start) return;
        cudaEventRecord(r.stop, c->stream);
        c->prof.push_back(r);
    }
};

// Average assignments per expert from which MPE_PATH_AUTO takes the tensor-core
// (prefill) path: below it most experts see fewer tokens than half an MMA tile
// and the streaming decode kernels move fewer bytes per token.
constexpr size_t kPrefillMinAvg = 32;

static bool use_prefill(const mpe_ctx* c, size_t Tk) {
    if (c->comp_n > 0) return false;  // compensation runs on the streaming path
    if (c->path == MPE_PATH_PREFILL) return true;
    if (c->path == MPE_PATH_DECODE) return false;
    return Tk >= kPrefillMinAvg * (size_t)c->E;
}

static int grow_y(mpe_ctx* c, size_t need_y) {
    if (need_y <= c->s.y_cap) return MPE_OK;
    CK(cudaStreamSynchronize(c->stream));
    cudaFree(c->s.y);
    c->s.y = nullptr;
    c->s.y_cap = 0;
    int r;
    if ((r = dev_alloc(c, &c->s.y, need_y))) return r;
    c->s.y_cap = need_y;
    return MPE_OK;
}

static int grow_xp(mpe_ctx* c, size_t need) {
    if (need <= c->s.xp_cap) return MPE_OK;
    CK(cudaStreamSynchronize(c->stream));
    cudaFree(c->s.xp);
    c->s.xp = nullptr;
    c->s.xp_cap = 0;
    int r;
    if ((r = dev_alloc(c, &c->s.xp, need))) return r;
    c->s.xp_cap = need;
    return MPE_OK;
}

// kept-channel lists for Tk rows (x uses the first T of them)
static int grow_sel(mpe_ctx* c, size_t Tk) {
    const size_t need = Tk * (size_t)c->comp_n;
    if (need <= c->sel_cap) return MPE_OK;
    CK(cudaStreamSynchronize(c->stream));
    cudaFree(c->sel_x);
    cudaFree(c->sel_h);
    c->sel_x = c->sel_h = nullptr;
    c->sel_cap = 0;
    int r;
    if ((r = dev_alloc(c, &c->sel_x, need))) return r;
    if ((r = dev_alloc(c, &c->sel_h, need))) return r;
    c->sel_cap = need;
    return MPE_OK;
}

static int moe_ffn_device(mpe_ctx* c, const void* x, int32_t T, const int32_t* ids,
                          const float* w, int32_t k, void* out) {
    const size_t Tk = (size_t)T * k;
    int r;
    if ((r = ensure_scratch(c, Tk))) return r;
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (use_prefill(c, Tk)) {
        if ((r = grow_y(c, (Tk * c->H + 1) / 2))) return r;  // bf16 y (capacity in floats)
        if ((r = grow_xp(c, Tk * c->H))) return r;
        {
            KernelSpan sp(c, 0);
            launch_route(c, ids, (int)Tk, k, c->s.perm, c->s.offsets, c->s.inv, kPrefillGroup);
        }
        {
            KernelSpan sp(c, 7);
            launch_permute_tokens(c, xb, k);
        }
        {
            KernelSpan sp(c, 5);
            if ((r = launch_prefill_gateup(c, Tk))) return r;
        }
        {
            KernelSpan sp(c, 6);
            if ((r = launch_prefill_down(c, Tk))) return r;
        }
        {
            KernelSpan sp(c, 4);
            launch_combine_by_position(c, w, T, k, 1, reinterpret_cast<__nv_bfloat16*>(out), true);
        }
        CKLAUNCH();
        return MPE_OK;
    }
    {
        KernelSpan sp(c, 0);
        launch_route(c, ids, (int)Tk, k, c->s.perm, c->s.offsets, c->s.inv, kDecodeGroup);
    }
    DecodePlan pl;
    decode_plan(c, Tk, pl);
    // compensation adds one slice after the gate/up partials and one after the
    // down partials, so the gate/up kernel always writes partials then
    const int ec = c->comp_n > 0 ? 1 : 0;
    const int p_gu = pl.p_gu + ec, p_dn = pl.p_dn + ec;
    const size_t need_part = p_gu > 1 ? (size_t)p_gu * 2 * Tk * c->F : 0;
    if (need_part > c->s.part_cap) {
        CK(cudaStreamSynchronize(c->stream));
        cudaFree(c->s.part);
        c->s.part = nullptr;
        c->s.part_cap = 0;
        if ((r = dev_alloc(c, &c->s.part, need_part))) return r;
        c->s.part_cap = need_part;
    }
    if ((r = grow_y(c, (size_t)p_dn * Tk * c->H))) return r;
    if (ec) {
        if ((r = grow_sel(c, Tk))) return r;
        c->last_T = T;
        c->last_k = k;
        KernelSpan sp(c, 8);
        launch_select_channels(c, xb, c->H, T, c->H, nullptr, c->comp_n, c->sel_x, c->stream);
    }
    {
        KernelSpan sp(c, 1);
        launch_decode_gateup(c, xb, k, Tk, pl.p_gu, pl.kb_gu, pl.claim, ec != 0);
    }
    if (ec) {
        KernelSpan sp(c, 9);
        launch_comp_gateup(c, xb, k, Tk, c->sel_x, c->comp_n, c->comp_store,
                           c->s.part + (size_t)pl.p_gu * 2 * Tk * c->F);
    }
    if (p_gu > 1) {
        KernelSpan sp(c, 2);
        launch_swiglu_reduce(c, Tk, p_gu);
    }
    if (ec) {
        KernelSpan sp(c, 8);
        launch_select_channels(c, c->s.h, c->F, (int)Tk, c->F, c->s.offsets + c->E, c->comp_n,
                               c->sel_h, c->stream);
    }
    {
        KernelSpan sp(c, 3);
        launch_decode_down(c, Tk, pl.p_dn, pl.kb_dn, pl.claim);
    }
    if (ec) {
        KernelSpan sp(c, 9);
        launch_comp_down(c, Tk, c->sel_h, c->comp_n, c->comp_store,
                         c->s.y + (size_t)pl.p_dn * Tk * c->H);
    }
    {
        KernelSpan sp(c, 4);
        launch_combine_by_position(c, w, T, k, p_dn, reinterpret_cast<__nv_bfloat16*>(out), false);
    }
    CKLAUNCH();
    return MPE_OK;
}

int mpe_moe_ffn(mpe_ctx* c, const void* x, int32_t T, const int32_t* ids, const float* w,
                int32_t k, void* out) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (T < 0 || k < 1 || k > 32) return fail(c, MPE_ERR_INVALID, "bad T=%d or k=%d", T, k);
    if (T == 0) return MPE_OK;
    if ((long long)T * k > MPE_MAX_ASSIGNMENTS)
        return fail(c, MPE_ERR_INVALID, "T*k = %lld exceeds %d", (long long)T * k,
                    MPE_MAX_ASSIGNMENTS);
    if (!x || !ids || !w || !out) return fail(c, MPE_ERR_INVALID, "null argument");
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15)
        return fail(c, MPE_ERR_INVALID, "x and out must be 16-byte aligned");
    if (!c->absmax_valid) return fail(c, MPE_ERR_ORDER, "moe_ffn before quantize_experts");
    if (c->comp_n > 0 && c->path == MPE_PATH_PREFILL)
        return fail(c, MPE_ERR_INVALID, "compensation runs on the streaming path only");
    DeviceGuard guard(c->device);
    return moe_ffn_device(c, x, T, ids, w, k, out);
}

// The forward's kernels of a host-buffer call on c->stream (the internal
// stream), reading staging slot `slot`. They run as a CUDA graph (one per
// slot) once the same (T, k) comes again with nothing reallocated or switched
// in between (the first call of a shape sizes every buffer, the next call of
// each slot captures, later ones replay): one launch instead of one per kernel.
static int host_kernels(mpe_ctx* c, int slot, int32_t T, int32_t k) {
    Scratch& s = c->s;
    const bool same = c->fwd_T == T && c->fwd_k == k && c->fwd_epoch == c->epoch;
    int r = MPE_OK;
    auto plain = [&]() {
        return moe_ffn_device(c, s.x_stage[slot], T, s.ids_stage[slot], s.w_stage[slot], k,
                              s.out_stage[slot]);
    };
    if (same && c->fwd_exec[slot] && !c->profiling) {
        CK(cudaGraphLaunch(c->fwd_exec[slot], c->stream));
        c->launches += c->fwd_launches;
    } else if (same && !c->profiling) {
        cudaGraph_t g = nullptr;
        CK(cudaStreamBeginCapture(c->stream, cudaStreamCaptureModeThreadLocal));
        const uint64_t l0 = c->launches;
        r = plain();
        const cudaError_t ce = cudaStreamEndCapture(c->stream, &g);
        if (r == MPE_OK && ce == cudaSuccess && c->epoch == c->fwd_epoch) {
            cudaGraphExec_t exec = nullptr;
            const cudaError_t ie = cudaGraphInstantiate(&exec, g, 0);
            cudaGraphDestroy(g);
            if (ie != cudaSuccess) return fail(c, MPE_ERR_CUDA, "graph instantiate: %s", cudaGetErrorString(ie));
            c->fwd_exec[slot] = exec;
            c->fwd_launches = c->launches - l0;
            CK(cudaGraphLaunch(c->fwd_exec[slot], c->stream));
        } else {
            if (g) cudaGraphDestroy(g);
            cudaGetLastError();
            if (r) return r;
            if (ce != cudaSuccess) return fail(c, MPE_ERR_CUDA, "graph capture: %s", cudaGetErrorString(ce));
            // something was reallocated while capturing: run it plainly
            if ((r = plain())) return r;
        }
    } else {
        if (c->fwd_exec[0] || c->fwd_exec[1]) {
            // a queued call may still be running one of them
            CK(cudaStreamSynchronize(c->host_stream));
            for (int i = 0; i < 2; ++i)
                if (c->fwd_exec[i]) {
                    cudaGraphExecDestroy(c->fwd_exec[i]);
                    c->fwd_exec[i] = nullptr;
                }
        }
        if ((r = plain())) return r;
        c->fwd_T = T;
        c->fwd_k = k;
        c->fwd_epoch = c->epoch;
    }
    return MPE_OK;
}

// Queue one host-buffer call: inputs in on in_stream, the forward on the
// internal stream, the output out on out_stream; returns its ticket. Three
// streams, so that a call's inputs land while the previous call computes and
// its output leaves while the next one does. Ordering, per staging slot: the
// inputs land after the slot's previous forward has read them, the forward
// waits for its inputs, for the slot's previous output copy and for the work
// already queued on the context stream, the output copy waits for the
// forward, and the context stream's later work waits for the forward.
static int host_submit(mpe_ctx* c, const void* x_host, int32_t T, const int32_t* ids_host,
                       const float* w_host, int32_t k, void* out_host, uint64_t* ticket) {
    Scratch& s = c->s;
    const int slot = (int)(c->host_seq & 1u);
    const size_t xb = (size_t)T * c->H * 2;
    CK(cudaStreamWaitEvent(c->in_stream, c->fwd_done[slot], 0));
    CK(cudaMemcpyAsync(s.x_stage[slot], x_host, xb, cudaMemcpyHostToDevice, c->in_stream));
    CK(cudaMemcpyAsync(s.ids_stage[slot], ids_host, (size_t)T * k * 4, cudaMemcpyHostToDevice,
                       c->in_stream));
    CK(cudaMemcpyAsync(s.w_stage[slot], w_host, (size_t)T * k * 4, cudaMemcpyHostToDevice,
                       c->in_stream));
    CK(cudaEventRecord(c->in_done[slot], c->in_stream));
    CK(cudaEventRecord(c->host_ready, c->stream));
    CK(cudaStreamWaitEvent(c->host_stream, c->host_ready, 0));
    CK(cudaStreamWaitEvent(c->host_stream, c->in_done[slot], 0));
    CK(cudaStreamWaitEvent(c->host_stream, c->out_done[slot], 0));
    const cudaStream_t user = c->stream;
    c->stream = c->host_stream;
    const int r = host_kernels(c, slot, T, k);
    c->stream = user;
    if (r) return r;
    CK(cudaEventRecord(c->fwd_done[slot], c->host_stream));
    CK(cudaStreamWaitEvent(c->stream, c->fwd_done[slot], 0));
    CK(cudaStreamWaitEvent(c->out_stream, c->fwd_done[slot], 0));
    CK(cudaMemcpyAsync(out_host, s.out_stage[slot], xb, cudaMemcpyDeviceToHost, c->out_stream));
    CK(cudaEventRecord(c->out_done[slot], c->out_stream));
    *ticket = c->host_seq++;
    return MPE_OK;
}

static int host_call_checks(mpe_ctx* c, int32_t T, int32_t k, const void* x_host,
                            const int32_t* ids_host, const float* w_host, void* out_host) {
    if (T < 0 || k < 1 || k > 32) return fail(c, MPE_ERR_INVALID, "bad T=%d or k=%d", T, k);
    if ((long long)T * k > MPE_MAX_ASSIGNMENTS)
        return fail(c, MPE_ERR_INVALID, "T*k = %lld exceeds %d", (long long)T * k,
                    MPE_MAX_ASSIGNMENTS);
    if (T > 0 && (!x_host || !ids_host || !w_host || !out_host))
        return fail(c, MPE_ERR_INVALID, "null argument");
    if (!c->absmax_valid) return fail(c, MPE_ERR_ORDER, "moe_ffn before quantize_experts");
    if (c->comp_n > 0 && c->path == MPE_PATH_PREFILL)
        return fail(c, MPE_ERR_INVALID, "compensation runs on the streaming path only");
    return MPE_OK;
}

static int host_setup(mpe_ctx* c, int32_t T, int32_t k) {
    int r;
    if ((r = ensure_scratch(c, (size_t)T * k))) return r;
    if ((r = ensure_stage(c, T, k))) return r;
    if (!c->host_stream) {
        CK(cudaStreamCreateWithFlags(&c->host_stream, cudaStreamNonBlocking));
        CK(cudaStreamCreateWithFlags(&c->in_stream, cudaStreamNonBlocking));
        CK(cudaStreamCreateWithFlags(&c->out_stream, cudaStreamNonBlocking));
        CK(cudaEventCreateWithFlags(&c->host_ready, cudaEventDisableTiming));
        for (int i = 0; i < 2; ++i) {
            CK(cudaEventCreateWithFlags(&c->in_done[i], cudaEventDisableTiming));
            CK(cudaEventCreateWithFlags(&c->fwd_done[i], cudaEventDisableTiming));
            CK(cudaEventCreateWithFlags(&c->out_done[i], cudaEventDisableTiming));
        }
    }
    return MPE_OK;
}

static int host_wait(mpe_ctx* c, uint64_t ticket) {
    if (ticket >= c->host_seq) return fail(c, MPE_ERR_INVALID, "ticket %llu not issued",
                                           (unsigned long long)ticket);
    // the slot's latest output copy is this call's or a later one's (the
    // output stream runs them in order)
    CK(cudaEventSynchronize(c->out_done[ticket & 1u]));
    return MPE_OK;
}

int mpe_moe_ffn_host(mpe_ctx* c, const void* x_host, int32_t T, const int32_t* ids_host,
                     const float* w_host, int32_t k, void* out_host) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    int r;
    if ((r = host_call_checks(c, T, k, x_host, ids_host, w_host, out_host))) return r;
    if (T == 0) return MPE_OK;
    DeviceGuard guard(c->device);
    if ((r = host_setup(c, T, k))) return r;
    // the call is synchronous: queued like an asynchronous one, then waited for
    uint64_t t = 0;
    if ((r = host_submit(c, x_host, T, ids_host, w_host, k, out_host, &t))) return r;
    return host_wait(c, t);
}

int mpe_moe_ffn_host_async(mpe_ctx* c, const void* x_host, int32_t T, const int32_t* ids_host,
                           const float* w_host, int32_t k, void* out_host, uint64_t* ticket) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (!ticket) return fail(c, MPE_ERR_INVALID, "null ticket");
    int r;
    if ((r = host_call_checks(c, T, k, x_host, ids_host, w_host, out_host))) return r;
    DeviceGuard guard(c->device);
    if (T == 0) {  // nothing to queue, nothing to wait for
        *ticket = UINT64_MAX;
        return MPE_OK;
    }
    if ((r = host_setup(c, T, k))) return r;
    return host_submit(c, x_host, T, ids_host, w_host, k, out_host, ticket);
}

int mpe_host_wait(mpe_ctx* c, uint64_t ticket) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (ticket == UINT64_MAX) return MPE_OK;
    DeviceGuard guard(c->device);
    return host_wait(c, ticket);
}

int mpe_route(mpe_ctx* c, const int32_t* ids, int32_t T, int32_t k, int32_t* perm,
              int32_t* offsets, int32_t* inv) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (T < 0 || k < 1 || k > 32) return fail(c, MPE_ERR_INVALID, "bad T or k");
    if ((long long)T * k > MPE_MAX_ASSIGNMENTS)
        return fail(c, MPE_ERR_INVALID, "T*k = %lld exceeds %d", (long long)T * k,
                    MPE_MAX_ASSIGNMENTS);
    if (!ids || !perm || !offsets || !inv) return fail(c, MPE_ERR_INVALID, "null argument");
    DeviceGuard guard(c->device);
    const size_t Tk = (size_t)T * k;
    int r;
    if ((r = ensure_scratch(c, Tk))) return r;
    if (Tk == 0) {
        CK(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (c->E + 1), c->stream));
        return MPE_OK;
    }
    launch_route(c, ids, (int)Tk, k, perm, offsets, inv, kDecodeGroup);
    CKLAUNCH();
    return MPE_OK;
}

int mpe_get_page_table(mpe_ctx* c, mpe_pte* pte_host, uint32_t* page_idx_host, size_t cap) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    DeviceGuard guard(c->device);
    int rc;
    if ((rc = commit_pending(c))) return rc;
    CK(cudaStreamSynchronize(c->stream));
    if (pte_host) CK(cudaMemcpy(pte_host, c->d_pte, sizeof(Pte) * c->E, cudaMemcpyDeviceToHost));
    if (page_idx_host) {
        if (cap < c->pidx_count)
            return fail(c, MPE_ERR_INVALID, "cap %zu < %u", cap, (unsigned)c->pidx_count);
        if (c->pidx_count)
            CK(cudaMemcpy(page_idx_host, c->d_pidx, sizeof(uint32_t) * c->pidx_count,
                          cudaMemcpyDeviceToHost));
    }
    return MPE_OK;
}

size_t mpe_expert_stream_bytes(mpe_ctx* c, int32_t e) {
    if (!c || e < 0 || e >= c->E || !valid_bits(c->bits[e])) return 0;
    return (size_t)3 * chunks_w1(c->H, c->F) * chunk_bytes(c->bits[e]);
}

int mpe_read_expert_packed(mpe_ctx* c, int32_t e, void* host_dst, size_t bytes) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (e < 0 || e >= c->E || !host_dst) return fail(c, MPE_ERR_INVALID, "bad expert or buffer");
    const size_t n = mpe_expert_stream_bytes(c, e);
    if (n == 0) return fail(c, MPE_ERR_ORDER, "expert %d not quantized", e);
    if (bytes < n) return fail(c, MPE_ERR_INVALID, "buffer %zu < stream %zu", bytes, n);
    DeviceGuard guard(c->device);
    {
        const int rc = commit_pending(c);
        if (rc) return rc;
    }
    if (n > c->gather_cap) {
        CK(cudaStreamSynchronize(c->stream));
        cudaFree(c->d_gather);
        c->d_gather = nullptr;
        CK(cudaMalloc(&c->d_gather, n));
        c->gather_cap = n;
    }
    launch_gather_stream(c, e, c->d_gather);
    CKLAUNCH();
    CK(cudaMemcpyAsync(host_dst, c->d_gather, n, cudaMemcpyDeviceToHost, c->stream));
    CK(cudaStreamSynchronize(c->stream));
    return MPE_OK;
}

int mpe_get_scales(mpe_ctx* c, float* scale_host, float* absmax_host) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    DeviceGuard guard(c->device);
    {
        const int rc = commit_pending(c);
        if (rc) return rc;
    }
    CK(cudaStreamSynchronize(c->stream));
    if (scale_host) {
        std::vector<Pte> p(c->E);
        CK(cudaMemcpy(p.data(), c->d_pte, sizeof(Pte) * c->E, cudaMemcpyDeviceToHost));
        for (int e = 0; e < c->E; ++e) scale_host[e] = p[e].scale;
    }
    if (absmax_host) {
        std::vector<uint32_t> m(c->E);
        CK(cudaMemcpy(m.data(), c->d_absmax, sizeof(uint32_t) * c->E, cudaMemcpyDeviceToHost));
        for (int e = 0; e < c->E; ++e) {
            const __half h = __ushort_as_half((unsigned short)(m[e] & 0xFFFF));
            absmax_host[e] = __half2float(h);
        }
    }
    return MPE_OK;
}

int mpe_get_bits(mpe_ctx* c, uint8_t* bits_host) {
    if (!c || !bits_host) return fail_global(MPE_ERR_INVALID, "null argument");
    std::memcpy(bits_host, c->bits.data(), c->E);
    return MPE_OK;
}

int mpe_profile_enable(mpe_ctx* c, int32_t enable) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    c->profiling = enable != 0;
    return MPE_OK;
}

int mpe_profile_read(mpe_ctx* c, double* ms_host, int64_t* launches_host, int32_t n_slots,
                     int32_t reset) {
    if (!c) return fail_global(MPE_ERR_INVALID, "null context");
    if (n_slots < 0) return fail(c, MPE_ERR_INVALID, "n_slots < 0");
    DeviceGuard guard(c->device);
    CK(cudaStreamSynchronize(c->stream));
    std::vector<double> ms(kProfileSlots, 0.0);
    std::vector<int64_t> cnt(kProfileSlots, 0);
    for (const ProfileRecord& r : c->prof) {
        float t = 0.0f;
        CK(cudaEventElapsedTime(&t, r.start, r.stop));
        ms[r.slot] += t;
        cnt[r.slot] += 1;
    }
    for (int i = 0; i < n_slots; ++i) {
        if (ms_host) ms_host[i] = i < kProfileSlots ? ms[i] : 0.0;
        if (launches_host) launches_host[i] = i < kProfileSlots ? cnt[i] : 0;
    }
    if (reset) {
        for (const ProfileRecord& r : c->prof) {
            c->event_pool.push_back(r.start);
            c->event_pool.push_back(r.stop);
        }
        c->prof.clear();
    }
    return MPE_OK;
}

int mpe_get_status(mpe_ctx* c, uint32_t* status_out, int32_t clear) {
    if (!c || !status_out) return fail_global(MPE_ERR_INVALID, "null argument");
    DeviceGuard guard(c->device);
    CK(cudaStreamSynchronize(c->stream));
    CK(cudaMemcpy(status_out, c->d_status, sizeof(uint32_t), cudaMemcpyDeviceToHost));
    if (clear) CK(cudaMemset(c->d_status, 0, sizeof(uint32_t)));
    return MPE_OK;
}

}  // extern "C"
