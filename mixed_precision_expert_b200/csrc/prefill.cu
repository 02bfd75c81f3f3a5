// Prefill-sized expert FFN on the 5th-generation tensor cores (tcgen05).
//
// PagedWeight, "Dynamic Paging": the active experts' pages are dequantized on
// the fly and multiplied with the tokens; at prefill sizes (hundreds of tokens
// per expert) this is a dense grouped GEMM per expert, computed transposed so
// that the dequantized weights never touch shared memory:
//   gate/up: G^T = K1 X^T and V^T = K3 X^T for the same 128 features in two
//            accumulators, h = silu(s G) (s V) -> bf16
//   down:    Y^T = K2 h^T, y[pos][o] = bf16(s Y[pos][o]) (by route position; the
//            combine applies the top-k weights and sums each token's slots in
//            fp32)
// The MMA's A operand (128 weight rows x K) lives in TENSOR MEMORY, written by
// the producer warps straight from the registers they unpacked it into; the B
// operand (the tile's tokens, K-major, SWIZZLE_128B) arrives in shared memory
// by one TMA tile copy per stage: the routed tokens are first written in route
// position order (a tile's tokens are then consecutive rows), because gathering
// scattered 128-byte rows reaches only a fraction of the L2 bandwidth that
// contiguous boxes do; fp32 accumulators live in tensor memory.
//
// Two facts set the shape (measured on B200): the thread that issues a
// tcgen05.mma of M = 128, K = 16 is held ~300 cycles whatever N is (up to 256),
// while MMAs issued by two threads into two accumulators overlap (~150 cycles
// each); and the token tiles stream from L2 into an SM at ~37 bytes a cycle,
// so a 128-row weight tile fed by its own token stage is bound by that ingress.
// A task is therefore a PAIR of weight tiles over one work group of up to
// kNT = 192 tokens: both tiles read each token stage (half the ingress per
// FLOP), each tile has its own accumulator (192 columns) and its own issuing
// thread, and each its own 2-stage ring of A operands of K = 64: 2 x 192 +
// 4 x 32 = 512 tensor-memory columns. The accumulators are single-buffered:
// the epilogue of a pair runs while the next pair's A stages and token stages
// fill, and the next MMAs wait for it.
//
// Persistent warp-specialised kernel, one CTA per SM, 19 warps:
//   warps 0-7   dequant producers: warp w owns tile w / 4 of the pair and
//               tensor-memory lanes 32 (w % 4) .. of it; each thread owns one
//               A row and per K-step unpacks 32 bf16 pairs (half a 128-code
//               block) into two tcgen05.st; the next K-step's packed words are
//               loaded a step ahead, an L2 prefetch cursor runs 4 blocks ahead.
//   warps 8-15  epilogue: gate/up, each half of them takes half the tokens
//               and reads a feature's gate and up values from the same lane of
//               the two accumulators (the pair is the gate rows and the up rows
//               of 128 features); down, each half takes one tile. The results
//               are staged token-major in shared memory and leave as 256-byte
//               row runs of h or y in 16-byte stores.
//   warp 16     token loader (one thread): per K-step (64 K of the group's
//               rows) it arms the stage's barrier with the byte count and
//               issues one TMA tile copy of kNT rows, completing on it.
//   warps 17-18 MMA issuers, one thread each, one tile each:
//               tcgen05.mma.cta_group::1.kind::f16, A from tensor memory, B
//               (the shared token stage) from shared memory, M = 128, four
//               MMAs per K-step; a token stage is released when both commit.
// Work: tasks (route work group of <= kNT positions of one expert) x (pair of
// tiles of 64 features (gate/up) or 128 outputs (down)); CTA b takes tasks
// b, b + grid, ...
// Every wait is bounded.
#include <cuda.h>

#include <cstdio>
#include <mutex>

#include "internal.h"

namespace mpe {
namespace {

constexpr int kNT = kPrefillGroup;            // tokens per tile (MMA N at most)
constexpr int kACol0 = 2 * kNT;               // A rings after the two accumulators
constexpr int kAStageCols = 32;               // K = 64 per stage: 32 bf16x2 columns
constexpr int kAStages = 2;                   // A stages per tile of a pair
constexpr int kTStages = 5;                   // shared-memory token ring (K = 64 each)
constexpr int kTStageBytes = kNT * 128;
static_assert(kACol0 + 2 * kAStages * kAStageCols <= 512, "tensor memory plan");
static_assert(kNT % 16 == 0 && kNT <= 256, "MMA N");
static_assert(kTStageBytes % 1024 == 0, "swizzle atoms");

// tensor-memory column of A stage s of tile x (0, 1) of the pair
__host__ __device__ constexpr uint32_t a_col(int x, int s) {
    return (uint32_t)(kACol0 + (x * kAStages + s) * kAStageCols);
}

// producers: warp w works on tile w / 4 of the pair, every K-step, and
// tensor-memory lanes 32 (w % 4) .. (more producer warps measured no faster,
// and the register budget of a larger CTA starves the epilogue)
constexpr int kProdWarps = 8;
constexpr int kEpiWarp0 = 8;   // warps 8-15: tile (w - 8) / 4, TMEM lane quarter w % 4
constexpr int kLoadWarp = 16;
constexpr int kMmaWarp = 17;   // issues tile 0's MMAs (accumulator 0)
constexpr int kMmaWarp2 = 18;  // issues tile 1's MMAs (accumulator 1)
static_assert(kEpiWarp0 % 4 == 0 && kEpiWarp0 + 8 == kLoadWarp, "epilogue warps");
constexpr int kPThreads = 32 * (kMmaWarp2 + 1);

// The epilogue stages a tile's outputs, token-major (kNT rows of up to 128
// bf16: 64 features of h, or 128 outputs of y), and writes them as whole row
// runs with 16-byte stores (a lane writing its own output column would store
// 2 bytes at a time). One staging tile per weight tile of the pair.
constexpr int kOStageCols = 128;
// 16-column tensor-memory loads the epilogue keeps in flight per wait; the
// accumulator has kNT = 192 columns, a multiple of 16 * kEpiBatch, so a batch
// never reads past the accumulator (columns past the group are read, unused)
constexpr int kEpiBatch = 4;
static_assert(kNT % (16 * kEpiBatch) == 0, "epilogue batches within the accumulator");
constexpr size_t kOStageBytes = (size_t)kNT * kOStageCols * 2;
constexpr size_t kSmem = 1024 + (size_t)kTStages * kTStageBytes + 2 * kOStageBytes + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");

// silu(g) v with the sigmoid as 1/2 + tanh(g / 2) / 2: one MUFU instruction
// (tanh.approx, absolute error about 2^-11) instead of an exponential and a
// reciprocal. The epilogue is bound by the latency of its instruction chain
// (measured: 481 -> 424 us for the gate/up launch of the 8192-token layer);
// the approximation stays below the bf16 rounding of h (2^-9 relative).
__device__ __forceinline__ float silu_mul(float g, float v) {
    float th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(0.5f * g));
    return g * fmaf(0.5f, th, 0.5f) * v;
}

struct PArgs {
    PagedExperts P;
    const int32_t* wg;     // work groups (expert, first position, count), <= kNT positions
    const int32_t* n_wg;   // total groups
    __nv_bfloat16* h_out;      // gate/up: h [Tk x F] by position
    __nv_bfloat16* y_out;      // down: s y [Tk x H] in bf16, by route position
    uint32_t* status;
};

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
    // K-major, SWIZZLE_128B: 8-row groups 1024 bytes apart; LBO unused
    uint64_t d = (uint64_t)((saddr & 0x3FFFF) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;  // sm100 descriptor version
    d |= (uint64_t)2 << 61;  // SWIZZLE_128B
    return d;
}

// kind::f16 instruction descriptor: D f32, A and B bf16, both K-major.
__device__ __forceinline__ uint32_t umma_idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem]^T
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// A box of kNT rows x 64 bf16 columns at (column x, row y) of the tensor map's
// matrix into shared memory, SWIZZLE_128B; rows past the matrix read as zero.
// Completes on bar.
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, int x, int y,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// A task: one work group (<= kNT positions of one expert) x one pair of
// weight tiles, tiles 2 np and 2 np + 1 (64 features each for gate/up, 128
// outputs for down); the second exists when 2 np + 1 < n_nt.
struct Tile {
    int e, pos0, ntok, np, bits;
    uint32_t first;
    float scale;
};

__device__ __forceinline__ Tile load_tile(const PArgs& a, int task, int n_np) {
    Tile T;
    const int gi = task / n_np;
    T.np = task - gi * n_np;
    T.e = a.wg[3 * gi];
    T.pos0 = a.wg[3 * gi + 1];
    T.ntok = a.wg[3 * gi + 2];
    const Pte pte = a.P.pte[T.e];
    T.bits = pte.bits;
    T.first = pte.first;
    T.scale = pte.scale;
    return T;
}

// Position in a ring of mbarrier-guarded slots, carried across tiles.
struct Ring {
    int s = 0;
    uint32_t phase = 0;  // parity of each slot's next completion to wait for
    uint32_t used = 0;   // slots filled at least once
    template <int N>
    __device__ __forceinline__ void advance() { s = (s + 1 == N) ? 0 : s + 1; }
};

// ---------------------------------------------------------------------------
// dequant producers
// ---------------------------------------------------------------------------
// Packed words of half a 128-code block of one row: 2 quarters of B words
// (b = 3: 24 bytes at 8-byte alignment; b = 4, 8: 32 / 64 bytes, 16-aligned).
template <int B>
__device__ __forceinline__ void load_half(const uint8_t* src, uint32_t (&w)[2 * B]) {
    if constexpr (B == 3) {
        const uint2* p = reinterpret_cast<const uint2*>(src);
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const uint2 v = __ldg(p + i);
            w[2 * i] = v.x;
            w[2 * i + 1] = v.y;
        }
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
        for (int i = 0; i < B / 2; ++i) {
            const uint4 v = __ldg(p + i);
            w[4 * i] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
    }
}

// One producer warp, tile x of a pair: its 32 rows (lane quarter lq) of the A
// operand for every K-step kk of the task, i.e. half kk & 1 of block column
// kk >> 1. `g0` is the task's first global K-step, which fixes the A stage
// (g % kAStages of tile x's ring) and its reuse parity. An absent second tile
// (2 np + 1 == n_nt) writes nothing but keeps the barrier protocol.
template <int B, bool GATEUP>
__device__ __forceinline__ bool produce_tile(const PArgs& a, const Tile& T, int x, bool present,
                                             int lq, int lane, uint32_t tbase, uint64_t* full,
                                             uint64_t* a_empty, uint32_t g0) {
    const PagedExperts& P = a.P;
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int nj = K / kCodesPerBlock;
    const int nk = 2 * nj;
    const int nc1 = chunks_w1(H, F);
    const int cpp = chunks_per_page(B, P.page_bytes);
    const int nt = 2 * T.np + x;
    uint64_t* aempty = a_empty + x * kAStages;
    if (!present) {
        for (int kk = 0; kk < nk; ++kk) {
            const uint32_t g = g0 + kk;
            const uint32_t m = g / kAStages;
            if (m > 0 && !mbar_wait_bounded(&aempty[g - m * kAStages], (m - 1) & 1u)) return false;
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[g % kTStages]);
        }
        return true;
    }
    // this thread's A row: gate/up feature np*128 + 32 lq + lane of W1 (tile 0)
    // or W3 (tile 1); down: output nt*128 + 32 lq + lane of W2. Its chunk for
    // block column j is c + 2 j: the stream interleaves W1 and W3 chunks, and
    // W2's tile pairs.
    constexpr int cs = 2;
    int c, rr;
    if (GATEUP) {
        const int f = T.np * 128 + lq * 32 + lane;
        c = 2 * ((f >> 4) * nj) + x;
        rr = f & 15;
    } else {
        const int o = nt * 128 + lq * 32 + lane;
        c = 2 * nc1 + 2 * ((o >> 5) * nj) + ((o >> 4) & 1);
        rr = o & 15;
    }
    const int rowoff = rr * block_bytes(B);
    // the words of K-step kk: half kk & 1 of the row's block in chunk c + 2 (kk >> 1)
    auto src = [&](int kk) {
        const int ci = c + cs * (kk >> 1);
        const int sl = ci / cpp;
        return P.pool + (size_t)P.pidx[T.first + sl] * P.page_bytes +
               (size_t)(ci - sl * cpp) * chunk_bytes(B) + rowoff + (kk & 1) * 8 * B;
    };
    // a cursor kPrefetch block columns ahead pulls this row's packed words into
    // L2 (no registers held), so the register loads one K-step ahead hit L2
    constexpr int kPrefetch = 4;
    for (int i = 1; i < kPrefetch && i < nj; ++i) prefetch_l2(src(2 * i));
    uint32_t ring[2][2 * B];
    load_half<B>(src(0), ring[0]);
    const uint32_t lane_base = (uint32_t)(lq * 32) << 16;
    for (int k0 = 0; k0 < nk; k0 += 2) {
#pragma unroll
        for (int ui = 0; ui < 2; ++ui) {
            const int kk = k0 + ui;  // nk is even: kk < nk
            if (kk + 1 < nk) load_half<B>(src(kk + 1), ring[ui ^ 1]);
            if (ui == 0 && (kk >> 1) + kPrefetch < nj) prefetch_l2(src(kk + 2 * kPrefetch));
            const uint32_t g = g0 + kk;
            const uint32_t m = g / kAStages;
            const int s = (int)(g - m * kAStages);
            if (m > 0) {
                if (!mbar_wait_bounded(&aempty[s], (m - 1) & 1u)) return false;
                tc_fence_after();
            }
            const uint32_t dst = tbase + lane_base + a_col(x, s);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t v[16];
#pragma unroll
                for (int p = 0; p < 16; ++p) v[p] = unpack_pair<B>(&ring[ui][q * B], p);
                tmem_st16(dst + 16 * q, v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[g % kTStages]);
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// token loader (one thread): stage j of a tile holds columns 64 j .. 64 j + 63 of
// rows pos0 .. pos0 + kNT - 1 of the position-ordered activations. Rows past
// the group belong to other groups (or read as zero past the matrix): the MMA
// columns they feed are never stored.
// ---------------------------------------------------------------------------
template <bool GATEUP>
__device__ __forceinline__ bool load_tile_tokens(const PArgs& a, const CUtensorMap* map,
                                                 const Tile& T, uint8_t* tring, uint64_t* full,
                                                 uint64_t* t_empty, Ring& tr) {
    const int nts = (GATEUP ? a.P.H : a.P.F) / 64;
    for (int j = 0; j < nts; ++j) {
        const int s = tr.s;
        if ((tr.used >> s) & 1u) {
            if (!mbar_wait_bounded(&t_empty[s], (tr.phase >> s) & 1u)) return false;
            tr.phase ^= 1u << s;
        }
        tr.used |= 1u << s;
        mbar_arrive_expect_tx(&full[s], (uint32_t)kTStageBytes);
        tma_tile(smem_u32(tring + (size_t)s * kTStageBytes), map, 64 * j, T.pos0, &full[s]);
        tr.advance<kTStages>();
    }
    return true;
}

// xp[pos] = x[perm[pos] / k] for pos < offsets[E]: one warp per row, 16-byte
// chunks (H a multiple of 128); a lane issues all its loads of up to 4 KB of
// the row before its stores.
__global__ void __launch_bounds__(256)
k_permute_rows(const __nv_bfloat16* x, const int32_t* perm, const int32_t* n_valid, int k,
               int H, __nv_bfloat16* xp) {
    constexpr int kU = 8;  // 16-byte chunks in flight per lane
    const int n = *n_valid;
    const int lane = threadIdx.x & 31;
    const int chunks = H / 8;
    for (int pos = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; pos < n;
         pos += (gridDim.x * blockDim.x) >> 5) {
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(perm[pos] / k) * H);
        uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)pos * H);
        for (int base = 0; base < chunks; base += 32 * kU) {
            uint4 v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = base + lane + 32 * u;
                v[u] = i < chunks ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = base + lane + 32 * u;
                if (i < chunks) dst[i] = v[u];
            }
        }
    }
}

template <bool GATEUP>
__global__ void __launch_bounds__(kPThreads, 1)
k_prefill(const __grid_constant__ CUtensorMap tmap, PArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tring = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    // full[g % kTStages]: K-step g is ready -- both tiles' A stages written (eight
    // producer warps) and its token stage landed (the loader's arrive + the
    // copy's bytes)
    __nv_bfloat16* ostage =
        reinterpret_cast<__nv_bfloat16*>(tring + (size_t)kTStages * kTStageBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(tring + (size_t)kTStages * kTStageBytes +
                                                 2 * kOStageBytes);
    uint64_t* a_empty = full + kTStages;          // [tile][kAStages]: that tile's MMAs done
    uint64_t* t_empty = a_empty + 2 * kAStages;   // both tiles' MMAs done with the token stage
    uint64_t* d_full = t_empty + kTStages;        // [tile]: accumulator complete
    uint64_t* d_empty = d_full + 2;               // [tile]: the epilogue has read it
    uint64_t* drain = d_empty + 2;
    uint64_t* epi_bar = drain + 1;                // [tile]: its four epilogue warps meet
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_bar + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.P.H, F = a.P.F;
    // gate/up: pair np = the gate rows (tile 0) and the up rows (tile 1) of
    // features np*128 ..; down: pair np = outputs np*256 .. in two tiles of 128
    const int n_nt = GATEUP ? F / 64 : H / 128;
    const int n_np = (n_nt + 1) / 2;       // tile pairs
    const int nk = (GATEUP ? H : F) / 64;  // K-steps (A stages, token stages) per task, even
    const int n_tasks = (*a.n_wg) * n_np;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 32) {
        for (int i = 0; i < kTStages; ++i) {
            mbar_init(&full[i], kProdWarps + 1);  // the producer warps of both tiles + the loader
            mbar_init(&t_empty[i], 2);            // the commits of both MMA issuers
        }
        for (int i = 0; i < 2 * kAStages; ++i) mbar_init(&a_empty[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&d_full[i], 1);   // issuer i's commit
            mbar_init(&d_empty[i], GATEUP ? 8 : 4);  // the epilogue warps that read it
        }
        mbar_init(drain, 2);
        mbar_init(&epi_bar[0], 4);
        mbar_init(&epi_bar[1], 4);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    bool ok = true;

    if (warp < kProdWarps) {
        // ---------------- dequant producers ----------------
        const int x = warp >> 2, lq = warp & 3;
        uint32_t g0 = 0;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x, g0 += nk) {
            const Tile T = load_tile(a, task, n_np);
            const bool present = 2 * T.np + x < n_nt;
            switch (T.bits) {
                case 3: ok = produce_tile<3, GATEUP>(a, T, x, present, lq, lane, tbase, full, a_empty, g0); break;
                case 4: ok = produce_tile<4, GATEUP>(a, T, x, present, lq, lane, tbase, full, a_empty, g0); break;
                default: ok = produce_tile<8, GATEUP>(a, T, x, present, lq, lane, tbase, full, a_empty, g0); break;
            }
        }
    } else if (warp == kLoadWarp) {
        // ---------------- token loader ----------------
        Ring tr;
        if (lane == 0)
            for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
                const Tile T = load_tile(a, task, n_np);
                ok = load_tile_tokens<GATEUP>(a, &tmap, T, tring, full, t_empty, tr);
            }
        // on a failed wait, give copies still in flight time to land before the
        // CTA releases its shared memory (every copy was consumed otherwise)
        if (!ok) {
            const uint64_t t0 = global_ns();
            while (global_ns() - t0 < 1000000ull) {
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp || warp == kMmaWarp2) {
        // ---------------- MMA issuers (one thread each) ----------------
        // issuer x multiplies tile x's A stages into accumulator x; both read
        // the shared token stage. An absent tile still commits every stage.
        const int x = warp - kMmaWarp;
        if (lane == 0) {
            // The issuing thread is on the critical path: each tcgen05.mma holds it
            // for hundreds of cycles, so the bookkeeping between MMAs is kept to a
            // few instructions (ring slots and phase bits as counters and bit masks).
            int ts = 0, as = 0;        // token slot (g % kTStages), A slot (g % kAStages)
            uint32_t fph = 0;          // phase parity to wait for, per full[] slot
            uint32_t dph = 0;          // parity of the next d_empty[x] completion
            bool first = true;
            const uint64_t desc0 = umma_desc(smem_u32(tring));
            const uint32_t dcol = tbase + (uint32_t)(x * kNT);
            uint64_t* aempty = a_empty + x * kAStages;
            int task = blockIdx.x;
            int ntok = task < n_tasks ? load_tile(a, task, n_np).ntok : 0;
            int np = task < n_tasks ? task % n_np : 0;
            for (; task < n_tasks && ok; task += gridDim.x) {
                // the next task's token count and pair, fetched while this one runs
                const int nxt = task + (int)gridDim.x;
                const int ntok_next = nxt < n_tasks ? a.wg[3 * (nxt / n_np) + 2] : 0;
                const int np_next = nxt < n_tasks ? nxt % n_np : 0;
                // the single accumulator: the epilogue of the previous task has read it
                if (!first) {
                    if (!mbar_wait_bounded(&d_empty[x], dph)) { ok = false; break; }
                    dph ^= 1u;
                }
                first = false;
                const bool present = 2 * np + x < n_nt;
                const uint32_t idesc = umma_idesc(128, (ntok + 15) & ~15);
                for (int kk = 0; kk < nk; ++kk) {
                    if (!mbar_wait_spin(&full[ts], (fph >> ts) & 1u)) { ok = false; break; }
                    fph ^= 1u << ts;
                    tc_fence_after();
                    if (present) {
                        const uint64_t bd = desc0 + (uint64_t)(ts * (kTStageBytes >> 4));
                        const uint32_t acol = tbase + a_col(x, as);
                        umma_ts(dcol, acol, bd, idesc, kk ? 1u : 0u);
                        umma_ts(dcol, acol + 8, bd + 2, idesc, 1u);
                        umma_ts(dcol, acol + 16, bd + 4, idesc, 1u);
                        umma_ts(dcol, acol + 24, bd + 6, idesc, 1u);
                    }
                    umma_commit(&aempty[as]);
                    umma_commit(&t_empty[ts]);
                    ts = (ts + 1 == kTStages) ? 0 : ts + 1;
                    as = (as + 1 == kAStages) ? 0 : as + 1;
                }
                if (!ok) break;
                umma_commit(&d_full[x]);
                ntok = ntok_next;
                np = np_next;
            }
            // every MMA issued by this thread has finished before TMEM is freed
            umma_commit(drain);
            if (!mbar_wait_bounded(drain, 0)) ok = false;
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 8-15, TMEM lanes 32 (w % 4) ..) ----------------
        // gate/up: warps (w - 8) / 4 = hx take tokens [96 hx, 96 hx + 96) of both
        // accumulators: a thread reads its feature's gate and up values (the
        // same lane of the two tiles) and forms h = silu(s g) (s v). Down:
        // warps (w - 8) / 4 = x take tile x. Results are staged token-major in
        // shared memory, the accumulators released, then the staged rows leave
        // as 16-byte stores (256-byte runs: 128 features of h, 128 outputs of y).
        const int hx = (warp - kEpiWarp0) >> 2, lq = warp & 3;
        const int et = threadIdx.x - 32 * (kEpiWarp0 + 4 * hx);  // 0 .. 127
        __nv_bfloat16* st = ostage + (size_t)(GATEUP ? 0 : hx) * (kOStageBytes / 2);
        // a barrier of the group's four epilogue warps on an mbarrier (a bounded
        // wait: a warp that gave up elsewhere makes the others give up too)
        uint32_t eph = 0;
        auto epi_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&epi_bar[hx]);
            const bool got = mbar_wait_bounded(&epi_bar[hx], eph);
            eph ^= 1u;
            return got;
        };
        // rows [r0, r1) of the staging tile (128 columns) -> dst + row * ld
        auto copy_out = [&](__nv_bfloat16* dst, size_t ld, int r0, int r1) {
            const int col = (et & 15) * 8;
            for (int r = r0 + (et >> 4); r < r1; r += 8)
                *reinterpret_cast<uint4*>(dst + (size_t)r * ld + col) =
                    *reinterpret_cast<const uint4*>(st + r * kOStageCols + col);
        };
        const uint32_t lanes = (uint32_t)(lq * 32) << 16;
        uint32_t ph = 0;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
            const Tile T = load_tile(a, task, n_np);
            // the previous task's rows have left the staging tile
            if (!epi_sync()) { ok = false; break; }
            if (GATEUP) {
                if (!mbar_wait_bounded(&d_full[0], ph) || !mbar_wait_bounded(&d_full[1], ph)) {
                    ok = false;
                    break;
                }
                ph ^= 1u;
                tc_fence_after();
                const int r0 = hx * (kNT / 2), r1 = min(T.ntok, r0 + kNT / 2);
                const int fl = lq * 32 + lane;  // feature within the pair
#pragma unroll 1
                for (int c0 = r0; c0 < r1; c0 += 32) {
                    uint32_t g[2][16], v[2][16];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        tmem_ld16(tbase + lanes + (uint32_t)(c0 + 16 * u), g[u]);
                        tmem_ld16(tbase + lanes + (uint32_t)(kNT + c0 + 16 * u), v[u]);
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int t = c0 + 16 * u + i;
                            const float gg = T.scale * __uint_as_float(g[u][i]);
                            const float vv = T.scale * __uint_as_float(v[u][i]);
                            if (t < r1) st[t * kOStageCols + fl] = __float2bfloat16_rn(silu_mul(gg, vv));
                        }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&d_empty[0]);
                    mbar_arrive(&d_empty[1]);
                }
                if (r0 < r1) {
                    if (!epi_sync()) { ok = false; break; }
                    copy_out(a.h_out + (size_t)T.pos0 * F + T.np * 128, (size_t)F, r0, r1);
                } else if (!epi_sync()) {
                    ok = false;
                    break;
                }
            } else {
                const int x = hx;
                const int nt = 2 * T.np + x;
                if (!mbar_wait_bounded(&d_full[x], ph)) { ok = false; break; }
                ph ^= 1u;
                tc_fence_after();
                const bool present = nt < n_nt;
                if (present) {
                    const int ol = lq * 32 + lane;  // output within the tile
#pragma unroll 1
                    for (int c0 = 0; c0 < T.ntok; c0 += 16 * kEpiBatch) {
                        uint32_t y[kEpiBatch][16];
#pragma unroll
                        for (int u = 0; u < kEpiBatch; ++u)
                            tmem_ld16(tbase + lanes + (uint32_t)(x * kNT + c0 + 16 * u), y[u]);
                        tmem_wait_ld();
#pragma unroll
                        for (int u = 0; u < kEpiBatch; ++u)
#pragma unroll
                            for (int i = 0; i < 16; i += 2) {
                                // two tokens' values in one packed conversion
                                const int t = c0 + 16 * u + i;
                                const __nv_bfloat162 two = __floats2bfloat162_rn(
                                    T.scale * __uint_as_float(y[u][i]),
                                    T.scale * __uint_as_float(y[u][i + 1]));
                                if (t < T.ntok) st[t * kOStageCols + ol] = __low2bfloat16(two);
                                if (t + 1 < T.ntok)
                                    st[(t + 1) * kOStageCols + ol] = __high2bfloat16(two);
                            }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&d_empty[x]);
                if (!epi_sync()) { ok = false; break; }
                if (present)
                    copy_out(a.y_out + (size_t)T.pos0 * H + nt * 128, (size_t)H, 0, T.ntok);
            }
        }
    }
    if (!ok && lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(512));
    }
}

// one persistent CTA per SM (the tensor-memory plan admits no second)
int sm_count(int device) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device);
    return n > 0 ? n : 1;
}

typedef CUresult (*TensorMapEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                         const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                         const cuuint32_t*, CUtensorMapInterleave,
                                         CUtensorMapSwizzle, CUtensorMapL2promotion,
                                         CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime.
TensorMapEncodeTiled encoder() {
    static TensorMapEncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TensorMapEncodeTiled>(p);
    });
    return fn;
}

int encode_fail(mpe_ctx* c, const char* what, int code) {
    char buf[128];
    snprintf(buf, sizeof(buf), "%s (%d)", what, code);
    c->err = buf;
    return MPE_ERR_CUDA;
}

// Row-major bf16 [rows x cols] in global memory, read as boxes of kNT rows x 64
// columns (128-byte row pieces) with the 128-byte swizzle the MMA's B descriptor
// expects. base 16-byte aligned, cols a multiple of 64.
int encode_rows(mpe_ctx* c, CUtensorMap* map, const void* base, size_t rows, int cols) {
    TensorMapEncodeTiled enc = encoder();
    if (!enc) return encode_fail(c, "cuTensorMapEncodeTiled is not available", 0);
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kNT};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return encode_fail(c, "tensor map encode failed", (int)r);
    return MPE_OK;
}

}  // namespace

void prefill_set_smem_limits() {
    cudaFuncSetAttribute(k_prefill<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    cudaFuncSetAttribute(k_prefill<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
}

void launch_permute_tokens(mpe_ctx* c, const __nv_bfloat16* x, int k) {
    k_permute_rows<<<sm_count(c->device) * 8, 256, 0, c->stream>>>(
        x, c->s.perm, c->s.offsets + c->E, k, c->H, c->s.xp);
    c->launches++;
}

int launch_prefill_gateup(mpe_ctx* c, size_t Tk) {
    alignas(64) CUtensorMap map;
    int r;
    if ((r = encode_rows(c, &map, c->s.xp, Tk, c->H))) return r;
    PArgs a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg = c->s.n_wg;
    a.h_out = c->s.h;
    a.status = c->d_status;
    k_prefill<true><<<sm_count(c->device), kPThreads, kSmem, c->stream>>>(map, a);
    c->launches++;
    return MPE_OK;
}

int launch_prefill_down(mpe_ctx* c, size_t Tk) {
    alignas(64) CUtensorMap map;
    int r;
    if ((r = encode_rows(c, &map, c->s.h, Tk, c->F))) return r;
    PArgs a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg = c->s.n_wg;
    a.y_out = reinterpret_cast<__nv_bfloat16*>(c->s.y);
    a.status = c->d_status;
    k_prefill<false><<<sm_count(c->device), kPThreads, kSmem, c->stream>>>(map, a);
    c->launches++;
    return MPE_OK;
}

}  // namespace mpe
