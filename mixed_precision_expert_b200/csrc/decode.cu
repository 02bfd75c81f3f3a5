// Decode-sized expert FFN: grouped GEMV / skinny GEMM straight from the pages.
//
// PagedWeight, "Dynamic Paging": the pass fetches the active experts' pages
// and dequantizes them on the fly; nothing is materialised in full precision
// (decode is memory-bound -- DecDEC summary, 2.1 -- so the packed bytes are
// the cost). Per expert e with scale s_e and codes K1, K3, K2:
//   gate/up:  g = s_e (K1 x), v = s_e (K3 x), h = silu(g) v   (h stored bf16)
//   down:     y_a = w_a s_e (K2 h_a)                          (y stored fp32)
//
// Warp-specialised persistent kernel. A CTA has 8 consumer warps and 1
// producer warp and works on one task at a time: a work group (<= 16 tokens of
// one expert) x 8 consecutive 16-row output tiles (one per consumer warp) x a
// K part. The producer warp claims tasks from a per-width-class counter and,
// for each block column j of the task, fills one slot of the CTA's
// shared-memory ring with the 8 tiles' chunks (one 1-D bulk copy per tile and
// matrix, issued by 8-16 producer lanes in parallel, no multicast; a full
// mbarrier counts the bytes) and prefetches the block's activation lines into
// L1. Consumer warps wait on the slot's full barrier, copy their chunk's words
// to registers, release the slot on its empty barrier (8 arrivals) and only
// then unpack (common.cuh) and multiply with mma.sync m16n8k16 -- weights are
// the 16-row A operand, one or two 8-token n-tiles of activations are B, fp32
// accumulate, the per-expert scale applied once at the end. A task whose K
// range is split in P parts writes a scaled partial to its own slice; a later
// pass sums the slices in part order (deterministic, no atomics).
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

constexpr int kConsumers = 8;                    // consumer warps per CTA (one tile each)
constexpr int kThreads = (kConsumers + 1) * 32;  // + the producer warp
constexpr int kRingBytes = 96 * 1024;            // shared-memory ring per CTA
constexpr int kMaxSlots = 16;
constexpr int kMaxTiles = kDecodeGroup / 8;

// A slot holds J consecutive block columns of 8 tiles. The bulk-copy engine
// takes ~80 cycles per copy whatever its size up to a few KB, so a tile's
// chunks for the slot -- gate and up interleaved, consecutive block columns,
// one contiguous run of its page -- go in one copy, as many columns as keep a
// slot within 32 KB (three slots per 96 KB ring): gate/up 2 (3, 4 bits) or 1
// (8 bits), down 5 / 4 / 2.
template <int B, int NM>
struct Geo {
    static constexpr int CB = 256 * B;                   // chunk bytes
    static constexpr int J = 32768 / (kConsumers * NM * CB);  // block columns per slot
    static constexpr int TILE = NM * J * CB;             // one warp's share of a slot
    static constexpr int SLOT = kConsumers * TILE;       // J block columns of 8 tiles
    static constexpr int S = (kRingBytes / SLOT) < kMaxSlots ? (kRingBytes / SLOT) : kMaxSlots;
    static constexpr int WORDS = (B == 8) ? 8 : B;       // raw words per row
    static_assert(S >= 3 && J >= 1, "ring geometry");
};

struct SlotDesc {
    int task;  // -1: no more tasks of this class
    int j;     // first block column held by the slot
    int nc;    // block columns held (1 .. J)
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
    uint32_t* status;
};

__host__ __device__ constexpr size_t smem_bytes() {
    return (size_t)kRingBytes + kMaxSlots * (2 * sizeof(uint64_t) + sizeof(SlotDesc));
}

// CTA task order: tile group fastest, then K part, then work group, so tasks
// claimed close together read the same activation K-range and sweep one
// expert's pages.
__device__ __forceinline__ void split_task(int task, int n_tq, int parts, int& gi, int& tq,
                                           int& p) {
    tq = task % n_tq;
    const int u = task / n_tq;
    p = u % parts;
    gi = u / parts;
}

// Raw words of this thread's share of one row's block (chunk row `r`).
template <int B>
__device__ __forceinline__ void load_row_words(const uint8_t* chunk, int r, int t, int g,
                                               uint32_t (&w)[Geo<B, 1>::WORDS]) {
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

// Unpack and multiply one block (128 codes of 16 rows, NM matrices) with NT
// 8-token n-tiles of activations. Widths 3 and 4 unpack to the offset form
// (k + off, see common.cuh) and accumulate off . x once per n-tile in accc,
// which the caller subtracts before finishing the task; width 8 unpacks to k.
template <int B, int NM, int NT>
__device__ __forceinline__ void block_mma(const uint32_t (&wr)[NM][2][Geo<B, 1>::WORDS],
                                          const uint32_t (&xa)[kMaxTiles][8],
                                          const uint32_t (&xz)[kMaxTiles][8],
                                          float (&acc)[kMaxTiles][NM][4],
                                          float (&accc)[kMaxTiles][4]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            uint32_t a0, a1, a2, a3;
            if constexpr (B == 8) {
                a0 = unpack_pair<B>(wr[m][0], 2 * c);
                a1 = unpack_pair<B>(wr[m][1], 2 * c);
                a2 = unpack_pair<B>(wr[m][0], 2 * c + 1);
                a3 = unpack_pair<B>(wr[m][1], 2 * c + 1);
            } else {
                a0 = unpack_pair_off<B>(wr[m][0], 2 * c);
                a1 = unpack_pair_off<B>(wr[m][1], 2 * c);
                a2 = unpack_pair_off<B>(wr[m][0], 2 * c + 1);
                a3 = unpack_pair_off<B>(wr[m][1], 2 * c + 1);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint32_t b0 = c < 4 ? xa[nt][2 * c] : xz[nt][2 * c - 8];
                const uint32_t b1 = c < 4 ? xa[nt][2 * c + 1] : xz[nt][2 * c - 7];
                mma_bf16_16816(acc[nt][m], a0, a1, a2, a3, b0, b1);
            }
        }
        if constexpr (B != 8) {
            // rows of the offset matrix are all alike: rows g and g+8 share a value
            const uint32_t o0 = pair_offset<B>(2 * c), o1 = pair_offset<B>(2 * c + 1);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint32_t b0 = c < 4 ? xa[nt][2 * c] : xz[nt][2 * c - 8];
                const uint32_t b1 = c < 4 ? xa[nt][2 * c + 1] : xz[nt][2 * c - 7];
                mma_bf16_16816(accc[nt], o0, o0, o1, o1, b0, b1);
            }
        }
    }
}

struct Task {
    int gi, tau, p, pos0, ntok, j_hi;
    float scale;
    bool valid;  // this warp's tile exists
};

// Finish a task. One K part (P = 1): gate/up applies SwiGLU and stores h
// (bf16); down stores y_a = w_a s_e acc (fp32). Several parts: the task's
// scaled partial goes to its own slice of the partial buffer -- gate/up
// gv[p][pos][m][row] = s_e acc, down y[p][a][row] = w_a s_e acc -- and a later
// pass sums the slices in part order (deterministic, no atomics).
template <bool GATEUP>
__device__ __forceinline__ void finish(const Args& a, const Task& T,
                                       float (&acc)[kMaxTiles][GATEUP ? 2 : 1][4], int lane) {
    if (!T.valid) return;
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

struct CtaSmem {
    uint8_t* ring;
    uint64_t* full;   // per slot: 1 producer arrival + transaction bytes
    uint64_t* empty;  // per slot: one arrival per consumer warp
    SlotDesc* descs;
};

// Producer warp: all tasks of one width class. Lane l < 8 owns the copy stream
// of tile l (a page cursor in registers): per slot one run of NM x jc chunks
// (gate/up: W1 and W3 alternate). Lane 0 claims tasks, arms the full barriers
// and writes the slot descriptors; every lane prefetches one activation line. `ep`/`used` track the empty barriers'
// phases per slot across classes.
template <int B, bool GATEUP>
__device__ __forceinline__ bool produce_class(const Args& a, const CtaSmem& sm, int group0,
                                              int n_groups, int32_t* ctr, uint32_t& ep,
                                              uint32_t& used) {
    constexpr int NM = GATEUP ? 2 : 1;
    using G = Geo<B, NM>;
    constexpr int S = G::S;
    const PagedExperts& P = a.P;
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int R = GATEUP ? F : H;
    const int nj = K / kCodesPerBlock, n_tiles = R / 16;
    const int n_tq = (n_tiles + kConsumers - 1) / kConsumers;
    const int nc1 = chunks_w1(H, F);
    const int lane = threadIdx.x & 31;
    const int n_tasks = n_groups * n_tq * a.parts;
    if (n_tasks == 0) return true;
    const int cpp = chunks_per_page(B, P.page_bytes);
    const int my_w = lane;
    const bool copier = lane < kConsumers;

    int s = 0;
    int task = -1, j = 0, j_hi = 0;
    uint32_t first = 0;
    int pslot = 0, poff = 0;           // this lane's page cursor
    bool my_tile = false;
    const __nv_bfloat16* pre_row = nullptr;  // this lane's activation row to prefetch
    int pre_half = 0;
    int active = 0;                    // tiles present in the current task
    for (;;) {
        // slot s must have been released by all consumers since its last fill
        if ((used >> s) & 1u) {
            if (!mbar_wait_bounded(&sm.empty[s], (ep >> s) & 1u)) {
                if (lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
                return false;
            }
            ep ^= 1u << s;
        }
        used |= 1u << s;
        if (task < 0 || j >= j_hi) {
            int nt = 0;
            if (lane == 0) nt = atomicAdd(ctr, 1);
            nt = __shfl_sync(0xffffffffu, nt, 0);
            if (nt >= n_tasks) {
                if (lane == 0) {
                    sm.descs[s] = SlotDesc{-1, 0};
                    mbar_arrive(&sm.full[s]);
                }
                __syncwarp();
                return true;
            }
            int gi, tq, p;
            split_task(nt, n_tq, a.parts, gi, tq, p);
            task = nt;
            gi += group0;
            const int e = a.wg[3 * gi];
            const int pos0 = a.wg[3 * gi + 1], ntok = a.wg[3 * gi + 2];
            first = P.pte[e].first;
            j = p * a.kb;
            j_hi = min(nj, j + a.kb);
            active = min(kConsumers, n_tiles - tq * kConsumers);
            const int tau = tq * kConsumers + my_w;
            my_tile = copier && my_w < active;
            if (my_tile) {
                const int c = GATEUP ? 2 * (tau * nj + j) : 2 * nc1 + tau * nj + j;
                pslot = c / cpp;
                poff = c - pslot * cpp;
            }
            pre_row = nullptr;
            pre_half = lane & 1;
            if ((lane >> 1) < ntok) {
                const int pos = pos0 + (lane >> 1);
                pre_row = a.act + (size_t)(GATEUP ? (a.perm[pos] / a.k) : pos) * K;
            }
        }
        const int jc = min(G::J, j_hi - j);  // block columns in this slot
        if (lane == 0) {
            sm.descs[s] = SlotDesc{task, j, jc};
            mbar_arrive_expect_tx(&sm.full[s], (uint32_t)(active * NM * jc * G::CB));
        }
        __syncwarp();
        if (my_tile) {
            // NM x jc consecutive chunks of this tile; a page boundary splits the
            // copy in two
            uint8_t* dst = sm.ring + (size_t)s * G::SLOT + (size_t)lane * G::TILE;
            const int total = NM * jc;
            const int n1 = min(total, cpp - poff);
            bulk_g2s(dst, P.pool + (size_t)P.pidx[first + pslot] * P.page_bytes +
                              (size_t)poff * G::CB,
                     (uint32_t)(n1 * G::CB), &sm.full[s]);
            poff += n1;
            if (poff == cpp) {
                ++pslot;
                poff = 0;
            }
            if (n1 < total) {
                bulk_g2s(dst + n1 * G::CB, P.pool + (size_t)P.pidx[first + pslot] * P.page_bytes,
                         (uint32_t)((total - n1) * G::CB), &sm.full[s]);
                poff = total - n1;
            }
        }
        if (pre_row) {
#pragma unroll
            for (int jj = 0; jj < G::J; ++jj)
                if (jj < jc) prefetch_l1(pre_row + 128 * (j + jj) + 64 * pre_half);
        }
        j += jc;
        s = (s + 1 == S) ? 0 : s + 1;
    }
}

// Consumer warp w: all tasks of one width class, tile w of each task.
template <int B, bool GATEUP>
__device__ __forceinline__ bool consume_class(const Args& a, const CtaSmem& sm, int group0,
                                              int n_groups, uint32_t& fp, int w) {
    constexpr int NM = GATEUP ? 2 : 1;
    using G = Geo<B, NM>;
    constexpr int S = G::S;
    const PagedExperts& P = a.P;
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int R = GATEUP ? F : H;
    const int nj = K / kCodesPerBlock, n_tiles = R / 16;
    const int n_tq = (n_tiles + kConsumers - 1) / kConsumers;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    if (n_groups * n_tq * a.parts == 0) return true;

    int cur = -1;
    Task T{};
    const __nv_bfloat16* arow[kMaxTiles] = {nullptr, nullptr};
    int ntiles = 0;
    float acc[kMaxTiles][NM][4];
    float accc[kMaxTiles][4];  // offset term (widths 3, 4), subtracted at the task's end
    uint32_t xa[kMaxTiles][8], xz[kMaxTiles][8];
    // acc <- acc - off . x for every matrix (a no-op for width 8)
    auto settle = [&]() {
        if constexpr (B != 8) {
#pragma unroll
            for (int nt = 0; nt < kMaxTiles; ++nt)
#pragma unroll
                for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[nt][m][q] -= accc[nt][q];
        }
    };
    for (int s = 0;; s = (s + 1 == S) ? 0 : s + 1) {
        const uint32_t par = (fp >> s) & 1u;
        fp ^= 1u << s;
        if (!mbar_wait_bounded(&sm.full[s], par)) {
            if (lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
            return false;
        }
        const SlotDesc d = sm.descs[s];
        if (d.task < 0) {  // terminator
            settle();
            finish<GATEUP>(a, T, acc, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
            return true;
        }
        if (d.task != cur) {
            if (cur >= 0) {
                settle();
                finish<GATEUP>(a, T, acc, lane);
            }
            cur = d.task;
            int tq;
            split_task(cur, n_tq, a.parts, T.gi, tq, T.p);
            T.gi += group0;
            T.tau = tq * kConsumers + w;
            T.valid = T.tau < n_tiles;
            const int e = a.wg[3 * T.gi];
            T.pos0 = a.wg[3 * T.gi + 1];
            T.ntok = a.wg[3 * T.gi + 2];
            T.scale = P.pte[e].scale;
            T.j_hi = min(nj, T.p * a.kb + a.kb);
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
#pragma unroll
                for (int q = 0; q < 4; ++q) accc[nt][q] = 0.0f;
            }
        }
        if (!T.valid) {  // this warp has no tile in the task: release at once
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
            continue;
        }
        const uint8_t* tile = sm.ring + (size_t)s * G::SLOT + (size_t)w * G::TILE;
#pragma unroll
        for (int jj = 0; jj < G::J; ++jj) {
            if (jj >= d.nc) break;
            uint32_t wr[NM][2][G::WORDS];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const uint8_t* chunk = tile + (jj * NM + m) * G::CB;
                load_row_words<B>(chunk, g, t, g, wr[m][0]);
                load_row_words<B>(chunk, g + 8, t, g, wr[m][1]);
            }
            if (jj + 1 == d.nc) {  // the slot's last words are in registers: release it
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);
            }
            const int j = d.j + jj;
            load_act_half(arow[0], j, t, B == 8, 0, xa[0]);
            load_act_half(arow[0], j, t, B == 8, 1, xz[0]);
            if (ntiles > 1) {
                load_act_half(arow[1], j, t, B == 8, 0, xa[1]);
                load_act_half(arow[1], j, t, B == 8, 1, xz[1]);
                block_mma<B, NM, kMaxTiles>(wr, xa, xz, acc, accc);
            } else {
                block_mma<B, NM, 1>(wr, xa, xz, acc, accc);
            }
        }
    }
}

template <bool GATEUP>
__global__ void __launch_bounds__(kThreads, 2) k_decode(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    CtaSmem sm;
    sm.ring = smem;
    sm.full = reinterpret_cast<uint64_t*>(smem + kRingBytes);
    sm.empty = sm.full + kMaxSlots;
    sm.descs = reinterpret_cast<SlotDesc*>(sm.empty + kMaxSlots);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxSlots; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kConsumers);
        }
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();
    const int n8 = a.n_wg_class[0], n4 = a.n_wg_class[1], n3 = a.n_wg_class[2];
    if (warp == kConsumers) {
        uint32_t ep = 0, used = 0;
        (void)lane;
        if (!produce_class<8, GATEUP>(a, sm, 0, n8, a.task_ctr + 0, ep, used)) return;
        if (!produce_class<4, GATEUP>(a, sm, n8, n4, a.task_ctr + 1, ep, used)) return;
        produce_class<3, GATEUP>(a, sm, n8 + n4, n3, a.task_ctr + 2, ep, used);
    } else {
        uint32_t fp = 0;
        if (!consume_class<8, GATEUP>(a, sm, 0, n8, fp, warp)) return;
        if (!consume_class<4, GATEUP>(a, sm, n8, n4, fp, warp)) return;
        consume_class<3, GATEUP>(a, sm, n8 + n4, n3, fp, warp);
    }
}

int g_num_sms = 0;

}  // namespace

void decode_set_smem_limits() {
    cudaFuncSetAttribute(k_decode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes());
    cudaFuncSetAttribute(k_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes());
}

// K parts per task: enough CTA tasks that every CTA of the persistent grid gets
// about `per_cta` of them, at least 4 blocks per part.
int decode_parts(int est_groups, int n_tq, int nj, int total_ctas, int per_cta) {
    const long target = (long)per_cta * total_ctas;
    int P = 1;
    const int pmax = max(1, nj / 4);
    while (P < pmax && (long)est_groups * n_tq * P < target) ++P;
    return P;
}

static int env_int(const char* name, int dflt) {
    const char* v = getenv(name);
    return v ? atoi(v) : dflt;
}

void decode_plan(mpe_ctx* c, size_t Tk, DecodePlan& pl) {
    if (!g_num_sms) cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, c->device);
    const int ctas = g_num_sms * 2;
    const int groups = (int)std::min<size_t>((size_t)c->E, Tk);
    const int per_cta = env_int("MPE_DECODE_TASKS_PER_CTA", 8);
    pl.claim = 1;
    const int nj_gu = c->H / kCodesPerBlock, nj_dn = c->F / kCodesPerBlock;
    int p = decode_parts(groups, (c->F / 16 + kConsumers - 1) / kConsumers, nj_gu, ctas, per_cta);
    pl.kb_gu = (nj_gu + p - 1) / p;
    pl.p_gu = (nj_gu + pl.kb_gu - 1) / pl.kb_gu;
    p = decode_parts(groups, (c->H / 16 + kConsumers - 1) / kConsumers, nj_dn, ctas, per_cta);
    pl.kb_dn = (nj_dn + p - 1) / p;
    pl.p_dn = (nj_dn + pl.kb_dn - 1) / pl.kb_dn;
}

static int persistent_grid(mpe_ctx* c, const void* fn, size_t smem) {
    if (!g_num_sms) cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, c->device);
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
    return g_num_sms * std::max(1, per_sm);
}

void launch_decode_gateup(mpe_ctx* c, const __nv_bfloat16* x, int k, size_t Tk, int parts,
                          int kb, int claim) {
    (void)claim;
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
    a.task_ctr = c->s.task_ctr;
    a.parts = parts;
    a.kb = kb;
    a.status = c->d_status;
    const int grid = persistent_grid(c, (const void*)k_decode<true>, smem_bytes());
    k_decode<true><<<grid, kThreads, smem_bytes(), c->stream>>>(a);
    c->launches++;
}

void launch_decode_down(mpe_ctx* c, const float* topk_w, size_t Tk, int parts, int kb,
                        int claim) {
    (void)claim;
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
    a.task_ctr = c->s.task_ctr + 3;
    a.parts = parts;
    a.kb = kb;
    a.status = c->d_status;
    const int grid = persistent_grid(c, (const void*)k_decode<false>, smem_bytes());
    k_decode<false><<<grid, kThreads, smem_bytes(), c->stream>>>(a);
    c->launches++;
}

}  // namespace mpe
