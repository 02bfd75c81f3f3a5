// Prefill-sized expert FFN on the 5th-generation tensor cores (tcgen05).
//
// PagedWeight, "Dynamic Paging": the active experts' pages are dequantized on
// the fly and multiplied with the tokens; at prefill sizes (hundreds of tokens
// per expert) this is a dense grouped GEMM per expert, computed transposed so
// that the dequantized weights never touch shared memory:
//   gate/up: [G; V]^T = [K1; K3] X^T with the rows of K1 and K3 interleaved
//            (feature f's gate row, then its up row), h = silu(s G) (s V) -> bf16
//   down:    Y^T = K2 h^T, y[pos][o] = s Y[pos][o] (fp32, by route position; the
//            combine applies the top-k weights and sums each token's slots)
// The MMA's A operand (128 weight rows x K) lives in TENSOR MEMORY, written by
// the producer warps straight from the registers they unpacked it into; the B
// operand (the tile's tokens, K-major, SWIZZLE_128B) arrives in shared memory
// by one TMA tile copy per stage: the routed tokens are first written in route
// position order (a tile's tokens are then consecutive rows), because gathering
// scattered 128-byte rows reaches only a fraction of the L2 bandwidth that
// contiguous boxes do; fp32 accumulators live in tensor memory.
//
// A tcgen05.mma of M = 128, K = 16 costs a fixed ~118 cycles up to N ~ 208 and
// about N / 1.85 cycles beyond, so a tile carries up to kNT = 208 tokens (N
// rounds the group up to 16): two accumulator buffers of 208 columns (the
// epilogue of one tile overlaps the MMAs of the next) and a 3-stage ring of A
// operands of K = 64 fill the 512 tensor-memory columns.
//
// Persistent warp-specialised kernel, one CTA per SM, 14 warps:
//   warps 0-7   dequant producers: warp w owns tensor-memory lanes 32 (w % 4) ..
//               and half w / 4 of every 128-code block (one A stage); each
//               thread owns one A row and per stage unpacks 32 bf16 pairs into
//               two tcgen05.st. The packed words of the next block are loaded a
//               whole block ahead into statically named registers.
//   warps 8-11  epilogue: tcgen05.ld of their 32 accumulator lanes; gate/up
//               pairs lanes 2i (gate) and 2i+1 (up) with one shuffle per two
//               tokens and stores h; down scales and stores y rows.
//   warp 12     token loader (one thread): per stage (64 K of the tile's rows)
//               it arms the stage's barrier with the byte count and issues one
//               TMA tile copy of kNT rows, which completes on the barrier.
//   warp 13     MMA issuer (one thread): tcgen05.mma.cta_group::1.kind::f16,
//               A from tensor memory, B from shared memory, M = 128, four MMAs
//               per stage.
// Work: tiles of <= kNT positions of one expert (route work groups) x 64
// features (gate/up) or 128 outputs (down); CTA b takes tiles b, b + grid, ...
// Every wait is bounded.
#include <cuda.h>

#include <cstdio>
#include <mutex>

#include "internal.h"

namespace mpe {
namespace {

constexpr int kNT = kPrefillGroup;            // tokens per tile (MMA N at most)
constexpr int kACol0 = 2 * kNT;               // A ring after the two accumulators
constexpr int kAStageCols = 32;               // K = 64 per stage: 32 bf16x2 columns
constexpr int kAStages = (512 - kACol0) / kAStageCols;
constexpr int kTStages = 7;                   // shared-memory token ring (K = 64 each)
constexpr int kTStageBytes = kNT * 128;
static_assert(kAStages >= 3 && kACol0 + kAStages * kAStageCols <= 512, "tensor memory plan");
static_assert(kNT % 16 == 0 && kNT <= 256, "MMA N");
static_assert(kTStageBytes % 1024 == 0, "swizzle atoms");

constexpr int kProdWarps = 8;
constexpr int kEpiWarp0 = 8;  // warps 8-11: warp % 4 covers all four TMEM lane quarters
constexpr int kLoadWarp = 12;
constexpr int kMmaWarp = 13;
static_assert(kEpiWarp0 % 4 == 0 && kEpiWarp0 + 4 == kLoadWarp, "epilogue warps");
constexpr int kPThreads = 32 * (kMmaWarp + 1);

constexpr size_t kSmem = 1024 + (size_t)kTStages * kTStageBytes + 1024;

struct PArgs {
    PagedExperts P;
    const int32_t* wg;     // work groups (expert, first position, count), <= kNT positions
    const int32_t* n_wg;   // total groups
    __nv_bfloat16* h_out;      // gate/up: h [Tk x F] by position
    float* y_out;              // down: y [Tk x H] by route position
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

struct Tile {
    int e, pos0, ntok, nt, bits;
    uint32_t first;
    float scale;
};

__device__ __forceinline__ Tile load_tile(const PArgs& a, int task, int n_nt) {
    Tile T;
    const int gi = task / n_nt;
    T.nt = task - gi * n_nt;
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

// One producer warp, one tile: half `hp` of every block column j, i.e. the
// A stage of K = 64 that is the tile's K-step 2 j + hp; `g0` is the tile's first
// global K-step (even), which fixes the A stage and its reuse parity.
template <int B, bool GATEUP>
__device__ __forceinline__ bool produce_tile(const PArgs& a, const Tile& T, int hp, int lq,
                                             int lane, uint32_t tbase, uint64_t* full,
                                             uint64_t* a_empty, uint32_t g0) {
    const PagedExperts& P = a.P;
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int nj = K / kCodesPerBlock;
    const int nc1 = chunks_w1(H, F);
    const int cpp = chunks_per_page(B, P.page_bytes);
    // this thread's A row: gate/up feature nt*64 + 16 lq + lane/2 of W1 (even
    // lanes) or W3 (odd lanes); down: output nt*128 + 32 lq + lane of W2. Its
    // chunk for block column j is c + 2 j: the stream interleaves W1 and W3
    // chunks, and W2's tile pairs.
    constexpr int cs = 2;
    int c, rr;
    if (GATEUP) {
        const int f = T.nt * 64 + lq * 16 + (lane >> 1);
        c = 2 * ((f >> 4) * nj) + (lane & 1);
        rr = f & 15;
    } else {
        const int o = T.nt * 128 + lq * 32 + lane;
        c = 2 * nc1 + 2 * ((o >> 5) * nj) + ((o >> 4) & 1);
        rr = o & 15;
    }
    int pslot = c / cpp;
    int poff = c - pslot * cpp;
    const int off = rr * block_bytes(B) + hp * 8 * B;
    auto src = [&]() {
        return P.pool + (size_t)P.pidx[T.first + pslot] * P.page_bytes +
               (size_t)poff * chunk_bytes(B) + off;
    };
    // a second cursor kPrefetch block columns ahead pulls this row's packed words
    // into L2 (no registers held), so the register loads one block ahead hit L2
    constexpr int kPrefetch = 4;
    int fslot = (c + kPrefetch * cs) / cpp;
    int foff = (c + kPrefetch * cs) - fslot * cpp;
    const int fmax = c + nj * cs;  // the row's chunks end here
    int fchunk = c + kPrefetch * cs;
    for (int i = 1; i < kPrefetch && i < nj; ++i) {
        const int ci = c + i * cs;
        const int si = ci / cpp;
        prefetch_l2(P.pool + (size_t)P.pidx[T.first + si] * P.page_bytes +
                    (size_t)(ci - si * cpp) * chunk_bytes(B) + off);
    }
    uint32_t ring[2][2 * B];
    load_half<B>(src(), ring[0]);
    const uint32_t lane_base = (uint32_t)(lq * 32) << 16;
    for (int j0 = 0; j0 < nj; j0 += 2) {
#pragma unroll
        for (int ui = 0; ui < 2; ++ui) {
            const int j = j0 + ui;
            if (j >= nj) break;
            if (j + 1 < nj) {
                poff += cs;
                if (poff >= cpp) {
                    poff -= cpp;
                    ++pslot;
                }
                load_half<B>(src(), ring[ui ^ 1]);
            }
            if (fchunk < fmax) {
                prefetch_l2(P.pool + (size_t)P.pidx[T.first + fslot] * P.page_bytes +
                            (size_t)foff * chunk_bytes(B) + off);
                fchunk += cs;
                foff += cs;
                if (foff >= cpp) {
                    foff -= cpp;
                    ++fslot;
                }
            }
            const uint32_t g = g0 + 2 * j + hp;
            const uint32_t m = g / kAStages;
            const int s = (int)(g - m * kAStages);
            if (m > 0) {
                if (!mbar_wait_bounded(&a_empty[s], (m - 1) & 1u)) return false;
                tc_fence_after();
            }
            const uint32_t dst = tbase + lane_base + (uint32_t)(kACol0 + s * kAStageCols);
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
            if (lane == 0) {
                const uint32_t fm = g / kTStages;
                mbar_arrive(&full[g - fm * kTStages]);
            }
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
// chunks (H a multiple of 128).
__global__ void __launch_bounds__(256)
k_permute_rows(const __nv_bfloat16* x, const int32_t* perm, const int32_t* n_valid, int k,
               int H, __nv_bfloat16* xp) {
    const int n = *n_valid;
    const int lane = threadIdx.x & 31;
    const int chunks = H / 8;
    for (int pos = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; pos < n;
         pos += (gridDim.x * blockDim.x) >> 5) {
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(perm[pos] / k) * H);
        uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)pos * H);
        for (int i = lane; i < chunks; i += 32) dst[i] = __ldg(src + i);
    }
}

template <bool GATEUP>
__global__ void __launch_bounds__(kPThreads, 1)
k_prefill(const __grid_constant__ CUtensorMap tmap, PArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tring = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    // full[g % kTStages]: K-step g is ready -- its A stage written (four producer
    // warps) and its token stage landed (the loader's arrive + the copy's bytes)
    uint64_t* full = reinterpret_cast<uint64_t*>(tring + (size_t)kTStages * kTStageBytes);
    uint64_t* a_empty = full + kTStages;
    uint64_t* t_empty = a_empty + kAStages;
    uint64_t* d_full = t_empty + kTStages;
    uint64_t* d_empty = d_full + 2;
    uint64_t* drain = d_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.P.H, F = a.P.F;
    const int n_nt = GATEUP ? F / 64 : H / 128;
    const int nk = (GATEUP ? H : F) / 64;  // K-steps (A stages, token stages) per tile, even
    const int n_tasks = (*a.n_wg) * n_nt;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 32) {
        for (int i = 0; i < kTStages; ++i) {
            mbar_init(&full[i], 5);  // four producer warps of the step's half + the loader
            mbar_init(&t_empty[i], 1);
        }
        for (int i = 0; i < kAStages; ++i) mbar_init(&a_empty[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&d_full[i], 1);
            mbar_init(&d_empty[i], 4);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    bool ok = true;

    if (warp < kProdWarps) {
        // ---------------- dequant producers ----------------
        const int hp = warp >> 2, lq = warp & 3;
        uint32_t g0 = 0;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x, g0 += nk) {
            const Tile T = load_tile(a, task, n_nt);
            switch (T.bits) {
                case 3: ok = produce_tile<3, GATEUP>(a, T, hp, lq, lane, tbase, full, a_empty, g0); break;
                case 4: ok = produce_tile<4, GATEUP>(a, T, hp, lq, lane, tbase, full, a_empty, g0); break;
                default: ok = produce_tile<8, GATEUP>(a, T, hp, lq, lane, tbase, full, a_empty, g0); break;
            }
        }
    } else if (warp == kLoadWarp) {
        // ---------------- token loader ----------------
        Ring tr;
        if (lane == 0)
            for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
                const Tile T = load_tile(a, task, n_nt);
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
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            // The issuing thread is on the critical path: a tcgen05.mma of this shape
            // holds it ~120 cycles and only about one more MMA queues behind the
            // one executing, so the bookkeeping between MMAs is kept to a few
            // instructions (ring slots and phase bits as counters and bit masks).
            int ts = 0, as = 0;              // full/token slot (g % kTStages), A slot (g % kAStages)
            uint32_t fph = 0;                // phase parity to wait for, per full[] slot
            int db = 0;                      // accumulator buffer
            uint32_t dph = 0, dused = 0;
            const uint64_t desc0 = umma_desc(smem_u32(tring));
            const uint32_t acol0 = tbase + (uint32_t)kACol0;
            int task = blockIdx.x;
            int ntok = task < n_tasks ? load_tile(a, task, n_nt).ntok : 0;
            for (; task < n_tasks && ok; task += gridDim.x) {
                // the next tile's token count, fetched while this one runs
                const int nxt = task + (int)gridDim.x;
                const int ntok_next = nxt < n_tasks ? a.wg[3 * (nxt / n_nt) + 2] : 0;
                if ((dused >> db) & 1u) {
                    if (!mbar_wait_bounded(&d_empty[db], (dph >> db) & 1u)) { ok = false; break; }
                    dph ^= 1u << db;
                }
                dused |= 1u << db;
                const uint32_t idesc = umma_idesc(128, (ntok + 15) & ~15);
                const uint32_t dcol = tbase + (uint32_t)(db * kNT);
                for (int kk = 0; kk < nk; ++kk) {
                    if (!mbar_wait_spin(&full[ts], (fph >> ts) & 1u)) { ok = false; break; }
                    fph ^= 1u << ts;
                    tc_fence_after();
                    const uint64_t bd = desc0 + (uint64_t)(ts * (kTStageBytes >> 4));
                    const uint32_t acol = acol0 + (uint32_t)(as * kAStageCols);
                    umma_ts(dcol, acol, bd, idesc, kk ? 1u : 0u);
                    umma_ts(dcol, acol + 8, bd + 2, idesc, 1u);
                    umma_ts(dcol, acol + 16, bd + 4, idesc, 1u);
                    umma_ts(dcol, acol + 24, bd + 6, idesc, 1u);
                    umma_commit(&a_empty[as]);
                    umma_commit(&t_empty[ts]);
                    ts = (ts + 1 == kTStages) ? 0 : ts + 1;
                    as = (as + 1 == kAStages) ? 0 : as + 1;
                }
                if (!ok) break;
                umma_commit(&d_full[db]);
                db ^= 1;
                ntok = ntok_next;
            }
            // every MMA issued by this thread has finished before TMEM is freed
            umma_commit(drain);
            if (!mbar_wait_bounded(drain, 0)) ok = false;
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 8-11: TMEM lanes 32 (warp % 4) ..) ----------------
        const int lq = warp & 3;
        const bool odd = lane & 1;
        Ring dr;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
            const Tile T = load_tile(a, task, n_nt);
            const int b = dr.s;
            if (!mbar_wait_bounded(&d_full[b], (dr.phase >> b) & 1u)) { ok = false; break; }
            dr.phase ^= 1u << b;
            tc_fence_after();
            const uint32_t tl = tbase + ((uint32_t)(lq * 32) << 16) + (uint32_t)(b * kNT);
            if (GATEUP) {
                // even lane: gate of feature f, odd lane: up of f; per 16 tokens the
                // even lane finishes tokens 0-7 and the odd lane tokens 8-15
                const int f = T.nt * 64 + lq * 16 + (lane >> 1);
#pragma unroll 1
                for (int c0 = 0; c0 < T.ntok; c0 += 16) {
                    uint32_t d[16];
                    tmem_ld16(tl + c0, d);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t recv = __shfl_xor_sync(0xffffffffu, odd ? d[i] : d[8 + i], 1);
                        const float gg = T.scale * __uint_as_float(odd ? recv : d[i]);
                        const float vv = T.scale * __uint_as_float(odd ? d[8 + i] : recv);
                        const int t = c0 + i + (odd ? 8 : 0);
                        if (t < T.ntok)
                            a.h_out[(size_t)(T.pos0 + t) * F + f] =
                                __float2bfloat16_rn(__fdividef(gg, 1.0f + __expf(-gg)) * vv);
                    }
                }
            } else {
                const int o = T.nt * 128 + lq * 32 + lane;  // output feature
                float* dst = a.y_out + (size_t)T.pos0 * H + o;
#pragma unroll 1
                for (int c0 = 0; c0 < T.ntok; c0 += 16) {
                    uint32_t y[16];
                    tmem_ld16(tl + c0, y);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < T.ntok) dst[(size_t)(c0 + i) * H] = T.scale * __uint_as_float(y[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[b]);
            dr.advance<2>();
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
    a.y_out = c->s.y;
    a.status = c->d_status;
    k_prefill<false><<<sm_count(c->device), kPThreads, kSmem, c->stream>>>(map, a);
    c->launches++;
    return MPE_OK;
}

}  // namespace mpe
