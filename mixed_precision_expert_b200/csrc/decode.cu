// Decode-sized expert FFN: grouped GEMV / skinny GEMM straight from the pages.
//
// PagedWeight, "Dynamic Paging": the pass fetches the active experts' pages
// and dequantizes them on the fly; nothing is materialised in full precision
// (decode is memory-bound -- DecDEC summary, 2.1 -- so the packed bytes are
// the cost). Per expert e with scale s_e and codes K1, K3, K2:
//   gate/up:  g = s_e (K1 x), v = s_e (K3 x), h = silu(g) v   (h stored bf16)
//   down:     y_a = w_a s_e (K2 h_a)                          (y stored fp32)
//
// Work is cut into tasks (work group of <= 16 tokens of one expert, 16-row
// output tile, K part); a persistent grid of warps claims tasks from a global
// counter. Every warp streams its tasks' chunks (16 rows x 128 codes each)
// through its own 3-stage shared-memory ring, filled by 1-D bulk copies
// (cp.async.bulk, no multicast) that complete on mbarriers, and keeps the
// ring full across task boundaries. Lanes unpack codes to exact bf16 integers
// in registers (common.cuh) and feed mma.sync m16n8k16: weights are the
// 16-row A operand, up to two 8-token n-tiles of activations are B, and the
// per-expert scale multiplies the fp32 accumulator at the end. A task whose K
// range is split in P parts writes fp32 partials; the last part to finish
// (arrival counter per tile) sums the P partials in part order -- the result
// does not depend on arrival order -- and applies the epilogue.
//
// k-permutation: inside a 128-code block, thread t (= lane & 3) owns 16 code
// pairs; mma step c (0..7) uses its pairs 2c and 2c+1 as the logical k-pairs
// t and t+4. Pair m of thread t covers codes
//   b = 3, 4: 32 t + 2m                      (quarter t)
//   b = 8:    16 t + 2m (m < 8), 64 + 16 t + 2(m - 8) (m >= 8)
// and the activation registers are loaded with the same permutation.
#include <cstdlib>

#include "internal.h"

namespace mpe {
namespace {

constexpr int kWarps = 4;
constexpr int kStages = 3;
constexpr int kStageBytes = 2048;  // per matrix per stage
constexpr int kMaxTiles = kDecodeGroup / 8;

template <int B>
struct Geo {
    static constexpr int CB = 256 * B;                           // chunk bytes
    static constexpr int J = (2048 / CB) > 0 ? (2048 / CB) : 1;  // chunks per stage
    static constexpr int WORDS = (B == 8) ? 8 : B;               // raw words per row
};

__host__ __device__ inline int stage_chunks(int b) { return b == 8 ? 1 : 2; }

struct StageDesc {
    int task;  // -1: no more work
    int j0;
    int nch;
    int pad;
};

struct Args {
    PagedExperts P;
    const int32_t* wg;          // work groups sorted by width class: 8-bit, 4-bit, 3-bit
    const int32_t* n_wg_class;  // groups per class (3)
    const int32_t* perm;
    int k;
    const __nv_bfloat16* act;  // gate/up: x [T x H]; down: h [Tk x F] in perm order
    __nv_bfloat16* h_out;      // gate/up: h [Tk x F]
    float* y_out;              // down: y [P][Tk][H], row a = assignment
    const float* topk_w;       // down: [Tk]
    float* part;               // gate/up split-K partials [P][Tk][2][F]
    size_t part_stride;        // floats per part slice (gate/up partials or down y)
    int32_t* task_ctr;         // claimed-task counters (one per class), zero at launch
    int parts;                 // P
    int kb;                    // blocks per part
    int claim;                 // tasks claimed per atomic
    uint32_t* status;
};

__host__ __device__ constexpr size_t ring_bytes(int nm) { return (size_t)kWarps * kStages * nm * kStageBytes; }
__host__ __device__ constexpr size_t smem_bytes(int nm);

struct Task {
    int gi, tau, p, e, pos0, ntok, bits, j_lo, j_hi;
    float scale;
};

struct ProducerState {
    int task, tau, j, j_hi, claim_left, done;
    Pte pte;
};

__host__ __device__ constexpr size_t smem_bytes(int nm) {
    return ring_bytes(nm) + kWarps * kStages * (sizeof(uint64_t) + sizeof(StageDesc)) +
           kWarps * sizeof(ProducerState);
}

// Task order: tile fastest, then K part, then work group, so tasks claimed
// close together read the same activation K-range (L1 hits) and sweep one
// expert's pages.
__device__ __forceinline__ void split_task(int task, int n_tiles, int parts, int& gi, int& tau,
                                           int& p) {
    tau = task % n_tiles;
    const int u = task / n_tiles;
    p = u % parts;
    gi = u / parts;
}

// Raw words of this thread's share of one row's block (chunk row `r`).
template <int B>
__device__ __forceinline__ void load_row_words(const uint8_t* chunk, int r, int t, int g,
                                               uint32_t (&w)[Geo<B>::WORDS]) {
    const uint8_t* blk = chunk + r * block_bytes(B);
    if constexpr (B == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(blk + 16 * t);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (B == 3) {
        const uint32_t* p = reinterpret_cast<const uint32_t*>(blk + 12 * t);
        w[0] = p[0]; w[1] = p[1]; w[2] = p[2];
    } else {
        // odd rows read their two 16-byte pieces in the other order so that
        // the 8 lanes of a shared-memory phase hit 8 distinct 16-byte banks
        const int odd = g & 1;
        const uint4 v0 = *reinterpret_cast<const uint4*>(blk + 64 * odd + 16 * t);
        const uint4 v1 = *reinterpret_cast<const uint4*>(blk + 64 * (1 - odd) + 16 * t);
        const uint4 lo = odd ? v1 : v0;
        const uint4 hi = odd ? v0 : v1;
        w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
        w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
    }
}

// Activation pairs of half h (mma steps 4h .. 4h+3) of block j for one token
// row: 8 registers = pairs 8h .. 8h+7 of this thread (k permutation above).
__device__ __forceinline__ void load_act_half(const __nv_bfloat16* row, int j, int t, int b8,
                                              int h, uint32_t (&xb)[8]) {
    if (row == nullptr) {
#pragma unroll
        for (int i = 0; i < 8; ++i) xb[i] = 0u;
        return;
    }
    const int off = b8 ? (64 * h + 16 * t) : (32 * t + 16 * h);
    const uint4* p = reinterpret_cast<const uint4*>(row + 128 * j + off);
    const uint4 v0 = __ldg(p), v1 = __ldg(p + 1);
    xb[0] = v0.x; xb[1] = v0.y; xb[2] = v0.z; xb[3] = v0.w;
    xb[4] = v1.x; xb[5] = v1.y; xb[6] = v1.z; xb[7] = v1.w;
}

// One stage: nch blocks (j0 ..) of NM matrices for the current task, with NT
// 8-token n-tiles (compile-time, so no per-mma guards). Each block is done in
// two halves (mma steps 0-3, then 4-7) to bound the live registers: the
// second half's activations load while the first computes.
template <int B, int NM, int NT>
__device__ __forceinline__ void consume(const uint8_t* stage, int j0, int nch,
                                        const __nv_bfloat16* const (&arow)[kMaxTiles], int g,
                                        int t, float (&acc)[kMaxTiles][NM][4]) {
    using G = Geo<B>;
    for (int jj = 0; jj < nch; ++jj) {
        const int j = j0 + jj;
        uint32_t xa[NT][8], xz[NT][8];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) load_act_half(arow[nt], j, t, B == 8, 0, xa[nt]);
        uint32_t wr[NM][2][G::WORDS];
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            const uint8_t* chunk = stage + (size_t)m * kStageBytes + jj * G::CB;
            load_row_words<B>(chunk, g, t, g, wr[m][0]);
            load_row_words<B>(chunk, g + 8, t, g, wr[m][1]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) load_act_half(arow[nt], j, t, B == 8, 1, xz[nt]);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const uint32_t a0 = unpack_pair<B>(wr[m][0], 2 * c);
                const uint32_t a1 = unpack_pair<B>(wr[m][1], 2 * c);
                const uint32_t a2 = unpack_pair<B>(wr[m][0], 2 * c + 1);
                const uint32_t a3 = unpack_pair<B>(wr[m][1], 2 * c + 1);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint32_t b0 = c < 4 ? xa[nt][2 * c] : xz[nt][2 * c - 8];
                    const uint32_t b1 = c < 4 ? xa[nt][2 * c + 1] : xz[nt][2 * c - 7];
                    mma_bf16_16816(acc[nt][m], a0, a1, a2, a3, b0, b1);
                }
            }
        }
    }
}

// Finish a task. One K part (P = 1): gate/up applies SwiGLU and stores h
// (bf16); down stores y_a = w_a s_e acc (fp32). Several parts: the task's
// scaled partial goes to its own slice of the partial buffer -- gate/up
// gv[p][pos][m][row] = s_e acc, down y[p][a][row] = w_a s_e acc -- and a later
// pass sums the slices in part order (deterministic, no atomics).
template <bool GATEUP>
__device__ __forceinline__ void finish(const Args& a, const Task& T,
                                       float (&acc)[kMaxTiles][GATEUP ? 2 : 1][4], int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int F = a.P.F, H = a.P.H;
#pragma unroll
    for (int nt = 0; nt < kMaxTiles; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int n = nt * 8 + 2 * t + (q & 1);
            if (n >= T.ntok) continue;
            const int row = T.tau * 16 + g + 8 * (q >> 1);
            const int pos = T.pos0 + n;
            if (GATEUP) {
                const float gv = T.scale * acc[nt][0][q];
                const float uv = T.scale * acc[nt][GATEUP ? 1 : 0][q];
                if (a.parts == 1) {
                    const float hv = gv / (1.0f + __expf(-gv)) * uv;
                    a.h_out[(size_t)pos * F + row] = __float2bfloat16_rn(hv);
                } else {
                    float* dst = a.part + (size_t)T.p * a.part_stride + ((size_t)pos * 2) * F + row;
                    dst[0] = gv;
                    dst[F] = uv;
                }
            } else {
                const int asg = a.perm[pos];
                a.y_out[(size_t)T.p * a.part_stride + (size_t)asg * H + row] =
                    a.topk_w[asg] * (T.scale * acc[nt][0][q]);
            }
        }
}

// Per-warp shared-memory layout: ring, mbarriers, stage descriptors, producer state.
struct WarpSmem {
    uint8_t* ring;
    uint64_t* bars;
    StageDesc* descs;
    ProducerState* ps;
};

// All tasks of one width class, as a persistent per-warp pipeline. `seq`
// counts the stages this warp has used so far (it sets the mbarrier phases)
// and carries over from one class to the next.
template <int B, bool GATEUP>
__device__ __forceinline__ bool run_class(const Args& a, const WarpSmem& w, int group0,
                                          int n_groups, int32_t* ctr, int& seq) {
    using G = Geo<B>;
    constexpr int NM = GATEUP ? 2 : 1;
    const PagedExperts& P = a.P;
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int R = GATEUP ? F : H;
    const int nj = K / kCodesPerBlock, n_tiles = R / 16;
    const int nc1 = chunks_w1(H, F);
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n_tasks = n_groups * n_tiles * a.parts;
    if (n_tasks == 0) return true;

    // ---- producer (lane 0) ----
    auto issue = [&](int s) {
        ProducerState& ps = *w.ps;
        if (ps.done) return;
        if (ps.task < 0 || ps.j >= ps.j_hi) {
            // next task: the rest of the claimed batch, else claim a new batch
            int nt;
            if (ps.claim_left > 0) {
                nt = ps.task + 1;
                --ps.claim_left;
            } else {
                nt = atomicAdd(ctr, a.claim);
                ps.claim_left = a.claim - 1;
            }
            if (nt >= n_tasks) {
                w.descs[s] = StageDesc{-1, 0, 0, 0};
                mbar_arrive(&w.bars[s]);
                ps.done = 1;
                return;
            }
            int gi, p;
            split_task(nt, n_tiles, a.parts, gi, ps.tau, p);
            ps.task = nt;
            ps.pte = P.pte[a.wg[3 * (group0 + gi)]];
            ps.j = p * a.kb;
            ps.j_hi = min(nj, ps.j + a.kb);
        }
        const int nch = min(G::J, ps.j_hi - ps.j);
        w.descs[s] = StageDesc{ps.task, ps.j, nch, 0};
        mbar_arrive_expect_tx(&w.bars[s], (uint32_t)(nch * G::CB * NM));
        const int cpp = chunks_per_page(B, P.page_bytes);
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            const int cbase = (GATEUP ? m * nc1 : 2 * nc1) + ps.tau * nj;
            uint8_t* dst = w.ring + (size_t)(s * NM + m) * kStageBytes;
            int done = 0;
            while (done < nch) {
                const int c = cbase + ps.j + done;
                const int n = min(nch - done, cpp - c % cpp);
                bulk_g2s(dst + done * G::CB, chunk_addr(P, ps.pte, B, c), (uint32_t)(n * G::CB),
                         &w.bars[s]);
                done += n;
            }
        }
        ps.j += nch;
    };

    // prime the ring: stages seq .. seq + kStages - 1
    if (lane == 0) {
        *w.ps = ProducerState{-1, 0, 0, 0, 0, 0, Pte{}};
        fence_proxy_async_smem();
        for (int r = 0; r < kStages; ++r) issue((seq + r) % kStages);
    }
    __syncwarp();

    // ---- consumer (all lanes) ----
    int cur = -1;
    Task T{};
    const __nv_bfloat16* arow[kMaxTiles] = {nullptr, nullptr};
    int ntiles = 0;
    float acc[kMaxTiles][NM][4];
    for (;; ++seq) {
        const int s = seq % kStages;
        if (!mbar_wait_bounded(&w.bars[s], (uint32_t)((seq / kStages) & 1))) {
            if (lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
            // let copies already issued land before shared memory goes away
            for (int r = seq + 1; r < seq + kStages; ++r)
                mbar_wait_bounded(&w.bars[r % kStages], (uint32_t)((r / kStages) & 1));
            return false;
        }
        const StageDesc d = w.descs[s];
        if (d.task < 0) {  // terminator: no more tasks of this class for this warp
            if (cur >= 0) finish<GATEUP>(a, T, acc, lane);
            ++seq;          // the terminator used this stage
            break;
        }
        if (d.task != cur) {
            if (cur >= 0) finish<GATEUP>(a, T, acc, lane);
            cur = d.task;
            split_task(cur, n_tiles, a.parts, T.gi, T.tau, T.p);
            T.gi += group0;
            T.e = a.wg[3 * T.gi];
            T.pos0 = a.wg[3 * T.gi + 1];
            T.ntok = a.wg[3 * T.gi + 2];
            T.bits = B;
            T.scale = P.pte[T.e].scale;
            T.j_lo = T.p * a.kb;
            T.j_hi = min(nj, T.j_lo + a.kb);
            ntiles = (T.ntok + 7) / 8;
#pragma unroll
            for (int nt = 0; nt < kMaxTiles; ++nt) {
                const int n = nt * 8 + g;
                arow[nt] = nullptr;
                if (n < T.ntok) {
                    const int pos = T.pos0 + n;
                    const int row = GATEUP ? (a.perm[pos] / a.k) : pos;
                    arow[nt] = a.act + (size_t)row * K;
                }
#pragma unroll
                for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[nt][m][q] = 0.0f;
            }
        }
        const uint8_t* stage = w.ring + (size_t)s * NM * kStageBytes;
        if (ntiles == 1)
            consume<B, NM, 1>(stage, d.j0, d.nch, arow, g, t, acc);
        else
            consume<B, NM, kMaxTiles>(stage, d.j0, d.nch, arow, g, t, acc);
        __syncwarp();
        if (lane == 0) {
            fence_proxy_async_smem();
            issue(s);
        }
    }
    return true;
}

template <bool GATEUP>
__global__ void __launch_bounds__(kWarps * 32, 4) k_decode(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int NM = GATEUP ? 2 : 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpSmem w;
    w.ring = smem + (size_t)warp * kStages * NM * kStageBytes;
    w.bars = reinterpret_cast<uint64_t*>(smem + ring_bytes(NM)) + warp * kStages;
    w.descs =
        reinterpret_cast<StageDesc*>(smem + ring_bytes(NM) + kWarps * kStages * sizeof(uint64_t)) +
        warp * kStages;
    w.ps = reinterpret_cast<ProducerState*>(smem + ring_bytes(NM) +
                                            kWarps * kStages * (sizeof(uint64_t) + sizeof(StageDesc))) +
           warp;
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&w.bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const int n8 = a.n_wg_class[0], n4 = a.n_wg_class[1], n3 = a.n_wg_class[2];
    int seq = 0;
    if (!run_class<8, GATEUP>(a, w, 0, n8, a.task_ctr + 0, seq)) return;
    if (!run_class<4, GATEUP>(a, w, n8, n4, a.task_ctr + 1, seq)) return;
    run_class<3, GATEUP>(a, w, n8 + n4, n3, a.task_ctr + 2, seq);
}

int g_num_sms = 0;

}  // namespace

void decode_set_smem_limits() {
    cudaFuncSetAttribute(k_decode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes(2));
    cudaFuncSetAttribute(k_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes(1));
}

// K parts per task: enough tasks that every warp of the persistent grid gets
// about `per_warp` of them, at least 4 blocks per part.
int decode_parts(int est_groups, int n_tiles, int nj, int total_warps, int per_warp) {
    const long target = (long)per_warp * total_warps;
    int P = 1;
    const int pmax = max(1, nj / 4);
    while (P < pmax && (long)est_groups * n_tiles * P < target) ++P;
    return P;
}

static int env_int(const char* name, int dflt) {
    const char* v = getenv(name);
    return v ? atoi(v) : dflt;
}

void decode_plan(mpe_ctx* c, size_t Tk, DecodePlan& pl) {
    if (!g_num_sms) cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, c->device);
    const int warps = g_num_sms * 4 * kWarps;
    const int groups = (int)std::min<size_t>((size_t)c->E, Tk);
    const int per_warp = env_int("MPE_DECODE_TASKS_PER_WARP", 4);
    pl.claim = std::max(1, env_int("MPE_DECODE_CLAIM", 1));
    const int nj_gu = c->H / kCodesPerBlock, nj_dn = c->F / kCodesPerBlock;
    int p = decode_parts(groups, c->F / 16, nj_gu, warps, per_warp);
    pl.kb_gu = (nj_gu + p - 1) / p;
    pl.p_gu = (nj_gu + pl.kb_gu - 1) / pl.kb_gu;
    p = decode_parts(groups, c->H / 16, nj_dn, warps, per_warp);
    pl.kb_dn = (nj_dn + p - 1) / p;
    pl.p_dn = (nj_dn + pl.kb_dn - 1) / pl.kb_dn;
}

static int persistent_grid(mpe_ctx* c, const void* fn, size_t smem) {
    if (!g_num_sms) cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, c->device);
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kWarps * 32, smem);
    return g_num_sms * std::max(1, per_sm);
}

void launch_decode_gateup(mpe_ctx* c, const __nv_bfloat16* x, int k, size_t Tk, int parts,
                          int kb, int claim) {
    Args a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg_class = c->s.n_wg + 1;
    a.perm = c->s.perm;
    a.k = k;
    a.act = x;
    a.h_out = c->s.h;
    a.part = c->s.part;
    a.part_stride = (size_t)2 * Tk * c->F;
    a.claim = claim;
    a.task_ctr = c->s.task_ctr;
    a.parts = parts;
    a.kb = kb;
    a.status = c->d_status;
    const int grid = persistent_grid(c, (const void*)k_decode<true>, smem_bytes(2));
    k_decode<true><<<grid, kWarps * 32, smem_bytes(2), c->stream>>>(a);
    c->launches++;
}

void launch_decode_down(mpe_ctx* c, const float* topk_w, size_t Tk, int parts, int kb,
                        int claim) {
    Args a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg_class = c->s.n_wg + 1;
    a.perm = c->s.perm;
    a.k = 1;
    a.act = c->s.h;
    a.y_out = c->s.y;
    a.topk_w = topk_w;
    a.part = c->s.part;
    a.part_stride = (size_t)Tk * c->H;
    a.claim = claim;
    a.task_ctr = c->s.task_ctr + 3;
    a.parts = parts;
    a.kb = kb;
    a.status = c->d_status;
    const int grid = persistent_grid(c, (const void*)k_decode<false>, smem_bytes(1));
    k_decode<false><<<grid, kWarps * 32, smem_bytes(1), c->stream>>>(a);
    c->launches++;
}

}  // namespace mpe
