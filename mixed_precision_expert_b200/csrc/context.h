// The context behind the C ABI's opaque mpe_ctx: host state, device buffers
// and streams of one MoE layer's paged experts. Host-side only (no kernel
// reads it); included by internal.h after the helper types it uses.
#pragma once

struct mpe_ctx {
    int device = 0;
    int E = 0, H = 0, F = 0;
    uint32_t page_bytes = MPE_DEFAULT_PAGE_BYTES;
    uint32_t pool_pages = 0;
    int path = MPE_PATH_AUTO;
    int allocator = MPE_ALLOCATOR_EXACT;   // the width rule repage uses
    cudaStream_t stream = nullptr;
    std::string err;
    uint64_t launches = 0;

    // device state
    uint8_t* pool = nullptr;
    mpe::Pte* d_pte = nullptr;
    uint32_t* d_pidx = nullptr;
    uint32_t* d_absmax = nullptr;     // fp16 bits of max|w| per expert
    uint32_t* d_status = nullptr;
    const void** d_masters = nullptr; // E device pointers
    int32_t* d_list = nullptr;        // expert list for encode
    double* d_p = nullptr;            // allocator inputs
    uint64_t* d_W = nullptr;
    uint8_t* d_bits_out = nullptr;
    int32_t* d_alloc_status = nullptr;
    uint8_t* d_choice = nullptr;
    size_t choice_cap = 0;
    double* d_D = nullptr;            // two DP rows
    double* d_loss = nullptr;         // measured MSE per expert and width [E][3]
    // salient-channel compensation: channels kept per row (0: off), the
    // residual store (device or mapped host memory) and the kept-channel lists
    int comp_n = 0;
    int comp_store_kind = MPE_STORE_DEVICE;
    const __half* comp_store = nullptr;  // device-visible address of the store
    __half* comp_dev = nullptr;          // the store when in device memory
    void* comp_host = nullptr;           // the store when in mapped host memory
    int32_t* sel_x = nullptr;            // [T][comp_n] kept channels of x
    int32_t* sel_h = nullptr;            // [T k][comp_n] kept channels of h
    size_t sel_cap = 0;                  // entries of each
    int last_T = 0, last_k = 0;          // shape of the last compensated forward
    unsigned long long* d_mse_acc = nullptr;  // its exact sums [E][3][2]
    bool loss_valid = false;          // d_loss holds the current master's values
    // the last allocation's inputs and widths: the same (B, p, width rule,
    // losses) give the same widths, so a repeat skips the allocator kernel
    bool memo_valid = false;
    int memo_allocator = -1;
    uint64_t memo_B = 0;
    std::vector<double> memo_p;
    std::vector<uint8_t> memo_bits;
    uint8_t* d_gather = nullptr;      // expert stream gather buffer
    size_t gather_cap = 0;

    // host mirrors
    std::vector<const void*> masters;
    std::vector<uint8_t> bits;
    std::vector<mpe::Pte> pte;
    uint32_t pidx_count = 0;                // entries of the page-index array in use
    mpe::Pte* h_pte_pinned = nullptr;       // upload staging (pinned)
    uint32_t* h_pidx_pinned = nullptr;
    int32_t* h_list_pinned = nullptr;
    const void** h_masters_pinned = nullptr;
    double* h_p_pinned = nullptr;           // allocator staging: importances in,
    uint64_t* h_w_pinned = nullptr;         // expert sizes (uploaded once),
    int32_t* h_alloc_pinned = nullptr;      // status word + widths out
    bool w_uploaded = false;
    cudaEvent_t upload_done = nullptr;      // page-table staging free again
    cudaEvent_t list_done = nullptr;        // expert-list staging free again
    bool absmax_valid = false;
    mpe::HostAllocator alloc;
    mpe::Scratch s;

    // the width rule of a synchronous repage runs here, at the highest
    // priority, beside the work already queued on `stream` (it reads only the
    // importances and sizes); the page moves and the encode stay on `stream`
    cudaStream_t alloc_stream = nullptr;

    // overlapped repage (mpe_repage_async / mpe_repage_commit): the next page
    // table is prepared and the changed experts encoded on `side` while work
    // on `stream` keeps reading the current table
    cudaStream_t side = nullptr;
    mpe::Pte* d_pte_next = nullptr;
    uint32_t* d_pidx_next = nullptr;
    int32_t* d_list_next = nullptr;
    mpe::Pte* h_pte_next_pinned = nullptr;
    uint32_t* h_pidx_next_pinned = nullptr;
    int32_t* h_list_next_pinned = nullptr;
    uint32_t pidx_count_next = 0;
    cudaEvent_t side_done = nullptr;        // the pending repage's device work finished
    cudaEvent_t old_table_free = nullptr;   // work launched before the last commit finished
    bool pending = false;
    std::vector<uint32_t> pending_release;  // old pages of the changed experts

    // the host-buffer forward replays a CUDA graph of its kernels (one per
    // staging slot) on an internal stream once the same (T, k) repeats;
    // `epoch` counts changes that invalidate a captured graph (any device
    // reallocation, a table swap, a new path or compensation setting). The
    // copies in run on in_stream, the copies out on out_stream; per slot,
    // in_done / fwd_done / out_done mark the last call's inputs landed,
    // forward finished and output copied; host_seq counts the calls
    // submitted (tickets).
    uint64_t epoch = 0;
    cudaStream_t host_stream = nullptr;
    cudaStream_t in_stream = nullptr;
    cudaStream_t out_stream = nullptr;
    cudaEvent_t host_ready = nullptr;
    cudaEvent_t in_done[2] = {nullptr, nullptr};
    cudaEvent_t fwd_done[2] = {nullptr, nullptr};
    cudaEvent_t out_done[2] = {nullptr, nullptr};
    uint64_t host_seq = 0;
    cudaGraphExec_t fwd_exec[2] = {nullptr, nullptr};
    int fwd_T = 0, fwd_k = 0;
    uint64_t fwd_epoch = ~0ull;
    uint64_t fwd_launches = 0;

    // a view over another store's pages (the prefix-compatible layered store
    // runs its forward pass through one): pool, page table and page-index
    // array belong to that store; px_lfirst holds, per expert, the first
    // page-index entries of its layers B and C
    bool view = false;
    const uint32_t* px_lfirst = nullptr;

    // tracing
    bool profiling = false;
    std::vector<mpe::ProfileRecord> prof;
    std::vector<cudaEvent_t> event_pool;
};
