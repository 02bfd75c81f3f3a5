// Host-side context of libmpe and the launch wrappers each kernel file exports.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <string>
#include <utility>
#include <vector>

#include "common.cuh"
#include "mpe.h"

namespace mpe {

// Tokens per work group of the decode kernels (up to two 8-token mma n-tiles,
// which share every unpacked weight fragment, so a heavily routed expert's
// pages are unpacked once per 16 tokens): an expert with more tokens is
// served by several groups, which read its pages close together in time
// (mostly from L2).
constexpr int kDecodeGroup = 16;

struct Scratch {
    size_t cap_assign = 0;   // T*k capacity
    int32_t* perm = nullptr;
    int32_t* inv = nullptr;
    int32_t* offsets = nullptr;  // E+1
    int32_t* wg = nullptr;       // work groups: 3 ints each
    int32_t* n_wg = nullptr;     // {total, 8-bit, 4-bit, 3-bit} work groups
    int32_t* hist = nullptr;     // per-chunk histograms (large-T route)
    size_t hist_cap = 0;
    __nv_bfloat16* h = nullptr;  // [cap_assign x F]
    float* y = nullptr;          // [P][T*k][H] down outputs (P K-part slices)
    float* part = nullptr;       // gate/up split-K partials [P][T*k][2][F]
    size_t part_cap = 0;         // floats
    size_t y_cap = 0;            // floats in y (P slices of T*k x H)
    int32_t* task_ctr = nullptr; // 6 task counters (3 classes x 2 kernels), zeroed by route
    __nv_bfloat16* xp = nullptr; // routed tokens in route-position order [xp_cap x H] (tensor-core path)
    size_t xp_cap = 0;           // elements
    // staging for the host-buffer entry points: two slots, so that one
    // call's copies overlap the neighbouring call's forward pass
    size_t stage_tokens = 0;
    void* x_stage[2] = {nullptr, nullptr};
    int32_t* ids_stage[2] = {nullptr, nullptr};
    float* w_stage[2] = {nullptr, nullptr};
    void* out_stage[2] = {nullptr, nullptr};
};

// CUDA-event records around the forward-pass kernels (optional tracing).
// route, gate/up, swiglu reduce, down, combine, tensor-core gate/up, tensor-core
// down, token permute (tensor-core path), salient-channel selection,
// compensation
constexpr int kProfileSlots = 10;
struct ProfileRecord {
    int slot;
    cudaEvent_t start, stop;
};

struct HostAllocator {
    std::vector<uint8_t> free;             // 1 = free page
    std::vector<std::vector<uint32_t>> pages;
};

}  // namespace mpe

#include "context.h"

namespace mpe {

PagedExperts paged(const mpe_ctx* c);

// api.cu: a context over another store's pages and page table, for the
// forward pass only (streaming path); the store keeps ownership of pool,
// d_pte and d_pidx. lfirst: per expert the first page-index entries of the
// layered store's layers B and C.
int create_view(mpe_ctx** out, int device, int E, int H, int F, uint32_t page_bytes,
                cudaStream_t stream, uint8_t* pool, Pte* d_pte, uint32_t* d_pidx,
                uint32_t pool_pages, const uint32_t* lfirst);

// Launch with programmatic stream serialization: the kernel may start while
// the preceding kernel in the stream drains; it must call griddep_wait before
// it reads anything that kernel writes.
template <typename... KArgs, typename... Actual>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Actual&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Actual>(args)...);
}

// quantize.cu
void launch_absmax(mpe_ctx* c, const int32_t* d_list, int n_list);
void launch_scales(mpe_ctx* c);
void launch_encode(mpe_ctx* c, const int32_t* d_list, int n_list);
// the same on an explicit page table / stream (overlapped repage)
void launch_scales_on(mpe_ctx* c, Pte* pte, cudaStream_t st);
void launch_encode_on(mpe_ctx* c, const PagedExperts& P, const int32_t* d_list, int n_list,
                      cudaStream_t st);
void launch_gather_stream(mpe_ctx* c, int e, uint8_t* dst);
// mse[e][0..2] = measured quantization MSE of expert e at 3 / 4 / 8 bits (uses
// the cached absmax); acc: [E][3][2] 64-bit words of scratch
void launch_measure_mse(mpe_ctx* c, unsigned long long* d_acc, double* d_mse);

// allocate.cu
// sum_w = sum of W, g = gcd(W) (host-computed); R = budget units (sizes the
// on-chip buffers); loss = float64[E][3] per-expert losses or null for L(b)
void launch_allocate(cudaStream_t st, const double* p, const double* loss, const uint64_t* W,
                     int E, uint64_t B, uint64_t sum_w, uint64_t g, uint8_t* bits_out,
                     int32_t* status, uint8_t* choice, double* D, int state_cap, uint64_t R);
// bytes of the global choice table for E experts and R budget units
size_t allocate_choice_bytes(int E, uint64_t R);
// the page's proportional rule with a budget repair (status 1: infeasible)
void launch_allocate_proportional(cudaStream_t st, const double* p, const uint64_t* W, int E,
                                  uint64_t B, uint64_t sum_w, uint8_t* bits_out, int32_t* status);

// compensate.cu (salient-channel error compensation, streaming path)
// the residual store: every expert's master transposed per matrix
void launch_transpose_masters(mpe_ctx* c, __half* store);
// kept channels of rows [n_rows][ld] (first n_cols used), out [n_rows][n];
// rows at or beyond *n_rows_dev skipped when it is given; c may be null
void launch_select_channels(mpe_ctx* c, const __nv_bfloat16* rows, size_t ld, int n_rows,
                            int n_cols, const int32_t* n_rows_dev, int n, int32_t* out,
                            cudaStream_t st);
// compensation slices: gate/up out [Tk][2F], down out [Tk][H]
void launch_comp_gateup(mpe_ctx* c, const __nv_bfloat16* x, int k, size_t Tk, const int32_t* sel,
                        int n, const __half* store, float* out);
void launch_comp_down(mpe_ctx* c, size_t Tk, const int32_t* sel, int n, const __half* store,
                      float* out);

// route.cu
void launch_route(mpe_ctx* c, const int32_t* ids, int Tk, int k, int32_t* perm,
                  int32_t* offsets, int32_t* inv, int group);
// zero-on-route counters: the route kernel clears task_ctr[0..1]

// decode.cu
struct DecodePlan {
    int p_gu = 1, kb_gu = 1, p_dn = 1, kb_dn = 1, claim = 1;
};
void decode_plan(mpe_ctx* c, size_t Tk, DecodePlan& pl);
// partials: write the gate/up partial slice even when parts == 1 (a later
// pass adds more slices before the SwiGLU)
void launch_decode_gateup(mpe_ctx* c, const __nv_bfloat16* x, int k, size_t Tk, int parts,
                          int kb, int claim, bool partials);
void launch_decode_down(mpe_ctx* c, size_t Tk, int parts, int kb, int claim);

// prefill.cu (tcgen05 grouped GEMM; work groups of up to kPrefillGroup positions)
constexpr int kPrefillGroup = 192;
void prefill_set_smem_limits();
// xp[pos] = x[perm[pos] / k] for the routed positions
void launch_permute_tokens(mpe_ctx* c, const __nv_bfloat16* x, int k);
int launch_prefill_gateup(mpe_ctx* c, size_t Tk);
int launch_prefill_down(mpe_ctx* c, size_t Tk);

// combine.cu
void launch_swiglu_reduce(mpe_ctx* c, size_t Tk, int parts);
// y stored by route position in `parts` K-part slices; the top-k weights are
// applied here
void launch_combine_by_position(mpe_ctx* c, const float* w, int T, int k, int parts,
                                __nv_bfloat16* out, bool y_bf16);

}  // namespace mpe
