// Prefill-sized expert FFN on the 5th-generation tensor cores (tcgen05).
//
// PagedWeight, "Dynamic Paging": the active experts' pages are dequantized on
// the fly and multiplied with the tokens; at prefill sizes (hundreds of tokens
// per expert) this is a dense grouped GEMM per expert, computed transposed so
// that the dequantized weights never touch shared memory:
//   gate/up: G^T = K1 X^T, V^T = K3 X^T (features x tokens),
//            h = silu(s G) (s V) -> bf16, h[pos][f]
//   down:    Y^T = K2 h^T, y[a][o] = w_a s Y[a][o] (fp32, summed by the combine)
// The MMA's A operand (128 weight rows x K) lives in TENSOR MEMORY, written by
// the producer warps straight from the registers they unpacked it into; the B
// operand (the tile's tokens, K-major, SWIZZLE_128B) is gathered into shared
// memory; fp32 accumulators live in tensor memory.
//
// Persistent warp-specialised kernel, one CTA per SM, 15 warps:
//   warps 0-7   dequant producers: warp w owns weight matrix w / 4 of the tile
//               (gate/up: W1, W3 rows of 128 features; down: two 128-row tiles
//               of W2) and tensor-memory lanes 32 (w % 4) ..; each thread owns
//               one weight row. Per K-step of 32 codes (one quarter block) it
//               unpacks 16 bf16 pairs and stores them with one tcgen05.st. The
//               packed words come from a register ring filled one load unit
//               (4 K-steps; 2 for 8-bit) ahead, statically named so no load is
//               waited on before its K-step.
//   warps 8-11  epilogue: tcgen05.ld of their 32 accumulator lanes, expert scale
//               and SwiGLU (gate/up) or top-k weight (down), global stores.
//   warps 12-13 token loaders: cp.async gather of the tile's token rows (128
//               bytes = 64 K per stage) into a 6-stage swizzled ring.
//   warp 14     MMA issuer (one thread): tcgen05.mma.cta_group::1.kind::f16,
//               A from tensor memory, B from shared memory, M = 128,
//               N = the tile's tokens rounded up to 16 (<= 96), K = 16.
// Tensor memory (512 columns): two accumulator buffers of 2 x 96 columns (the
// epilogue of one tile overlaps the MMAs of the next) and a 4-stage ring of A
// operands (2 matrices x 16 columns per K-step). Work: tiles of <= 96 positions
// of one expert (route work groups) x 128 output features (gate/up) or
// 256 (down); CTA b takes tiles b, b + grid, ... Every wait is bounded.
#include "internal.h"

namespace mpe {
namespace {

constexpr int kNT = kPrefillGroup;  // tokens per tile (MMA N at most)
constexpr int kNM = 2;              // A matrices per tile
constexpr int kAStages = 4;         // tensor-memory A ring (K = 32 each)
constexpr int kTStages = 6;         // shared-memory token ring (K = 64 each)
constexpr int kTLag = 3;            // cp.async groups in flight per loader thread
constexpr int kTStageBytes = kNT * 128;
constexpr int kDCols = kNM * kNT;             // one accumulator buffer
constexpr int kACol0 = 2 * kDCols;            // A ring after the two buffers
constexpr int kAStageCols = kNM * 16;         // 16 bf16x2 columns per matrix
static_assert(kACol0 + kAStages * kAStageCols == 512, "tensor memory plan");
static_assert(kNT % 16 == 0 && kNT <= 256, "MMA N");
static_assert(kTStageBytes % 1024 == 0, "swizzle atoms");
static_assert(kTStages > kTLag, "token ring");

constexpr int kProdWarps = 8;
constexpr int kLoadWarp0 = 12;
constexpr int kLoadWarps = 2;
constexpr int kMmaWarp = 14;
constexpr int kPThreads = 32 * (kMmaWarp + 1);
constexpr int kLoadThreads = 32 * kLoadWarps;
constexpr int kRowsPerLoader = kNT * 8 / kLoadThreads;  // 16-byte chunks per thread per stage
static_assert(kNT * 8 % kLoadThreads == 0 && kLoadThreads % 8 == 0, "loader split");

constexpr size_t kSmem = 1024 + (size_t)kTStages * kTStageBytes + 1024;

struct PArgs {
    PagedExperts P;
    const int32_t* wg;     // work groups (expert, first position, count), <= kNT positions
    const int32_t* n_wg;   // total groups
    const int32_t* perm;
    int k;
    const __nv_bfloat16* act;  // gate/up: x [T x H] by token; down: h [Tk x F] by position
    __nv_bfloat16* h_out;      // gate/up: h [Tk x F] by position
    float* y_out;              // down: y [Tk x H] by assignment
    const float* topk_w;       // down: [Tk]
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

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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
// Load unit: U K-steps of 32 codes of one row (b = 3, 4: a whole 128-code
// block, 48 / 64 bytes; b = 8: half a block, 64 bytes); kRing units in flight.
template <int B>
struct Unit {
    static constexpr int U = (B == 8) ? 2 : 4;
    static constexpr int W = U * B;  // 32-bit words
};
constexpr int kRing = 2;

template <int B>
__device__ __forceinline__ void load_unit(const uint8_t* src, uint32_t (&w)[Unit<B>::W]) {
    const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int i = 0; i < Unit<B>::W / 4; ++i) {
        const uint4 v = __ldg(p + i);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
    }
}

// One producer warp: all K-steps of one tile for its matrix.
template <int B, bool GATEUP>
__device__ __forceinline__ bool produce_tile(const PArgs& a, const Tile& T, int m, int lq,
                                             int lane, uint32_t tbase, uint64_t* a_full,
                                             uint64_t* a_empty, Ring& ar) {
    using UT = Unit<B>;
    constexpr int kUnitsPerChunk = 4 / UT::U;
    const PagedExperts& P = a.P;
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int nunits = K / 32 / UT::U;
    const int nj = K / kCodesPerBlock;
    const int nc1 = chunks_w1(H, F);
    const int cpp = chunks_per_page(B, P.page_bytes);
    // this warp's matrix: gate/up W1 (m = 0) or W3 (m = 1) rows nt*128 ..;
    // down: W2 rows (2 nt + m) * 128 .. (inactive past H)
    const int mt = GATEUP ? T.nt : 2 * T.nt + m;
    const bool active = GATEUP || mt * 128 < H;
    const int row = mt * 128 + lq * 32 + lane;  // weight row within its matrix
    int pslot = 0, poff = 0;
    if (active) {
        const int c = (GATEUP ? m * nc1 : 2 * nc1) + (row >> 4) * nj;
        pslot = c / cpp;
        poff = c - pslot * cpp;
    }
    const int rho_off = (row & 15) * block_bytes(B);
    int lu = 0;  // next unit to load
    auto load_next = [&](uint32_t (&w)[UT::W]) {
        if (lu < nunits && active) {
            if (lu > 0 && (lu % kUnitsPerChunk) == 0) {  // next block column: next chunk
                if (++poff == cpp) {
                    ++pslot;
                    poff = 0;
                }
            }
            load_unit<B>(P.pool + (size_t)P.pidx[T.first + pslot] * P.page_bytes +
                             (size_t)poff * chunk_bytes(B) + rho_off +
                             (lu % kUnitsPerChunk) * UT::W * 4,
                         w);
        }
        ++lu;
    };
    uint32_t ring[kRing][UT::W];
#pragma unroll
    for (int i = 0; i < kRing - 1; ++i) load_next(ring[i]);
    const uint32_t lane_base = (uint32_t)(lq * 32) << 16;
    for (int u0 = 0; u0 < nunits; u0 += kRing) {
#pragma unroll
        for (int ui = 0; ui < kRing; ++ui) {
            if (u0 + ui >= nunits) break;
            load_next(ring[(ui + kRing - 1) % kRing]);
#pragma unroll
            for (int q = 0; q < UT::U; ++q) {
                const int s = ar.s;
                if ((ar.used >> s) & 1u) {
                    if (!mbar_wait_bounded(&a_empty[s], (ar.phase >> s) & 1u)) return false;
                    ar.phase ^= 1u << s;
                    tc_fence_after();
                }
                ar.used |= 1u << s;
                if (active) {
                    uint32_t v[16];
#pragma unroll
                    for (int p = 0; p < 16; ++p) v[p] = unpack_pair<B>(&ring[ui][q * B], p);
                    tmem_st16(tbase + lane_base + (uint32_t)(kACol0 + s * kAStageCols + m * 16), v);
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[s]);
                ar.advance<kAStages>();
            }
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// token loaders: thread lt copies 16-byte chunk (lt & 7) of rows (lt >> 3) + 8 i
// ---------------------------------------------------------------------------
struct LoadState {
    Ring r;
    int pub = 0;    // oldest issued stage not yet published
    int npend = 0;  // issued stages not yet published
};

template <bool GATEUP>
__device__ __forceinline__ bool load_tile_tokens(const PArgs& a, const Tile& T, int lt,
                                                 uint8_t* tring, uint64_t* t_full,
                                                 uint64_t* t_empty, LoadState& ls) {
    const int K = GATEUP ? a.P.H : a.P.F;
    const int nts = K / 64;
    const int c = lt & 7;
    const int r0 = lt >> 3;
    // rows past the group are not loaded: the MMA columns they feed are never stored
    int src_row[kRowsPerLoader];  // activation row of each of this thread's tile rows, or -1
#pragma unroll
    for (int i = 0; i < kRowsPerLoader; ++i) {
        const int r = r0 + (kLoadThreads / 8) * i;
        src_row[i] = -1;
        if (r < T.ntok) {
            const int pos = T.pos0 + r;
            src_row[i] = GATEUP ? (a.perm[pos] / a.k) : pos;
        }
    }
    const __nv_bfloat16* act = a.act + 8 * c;
    const int lane = lt & 31;
    for (int j = 0; j < nts; ++j) {
        const int s = ls.r.s;
        if ((ls.r.used >> s) & 1u) {
            if (!mbar_wait_bounded(&t_empty[s], (ls.r.phase >> s) & 1u)) return false;
            ls.r.phase ^= 1u << s;
        }
        ls.r.used |= 1u << s;
        uint8_t* st = tring + (size_t)s * kTStageBytes;
#pragma unroll
        for (int i = 0; i < kRowsPerLoader; ++i) {
            const int r = r0 + (kLoadThreads / 8) * i;
            if (src_row[i] >= 0)
                cp_async16(st + r * 128 + ((c ^ (r & 7)) << 4), act + (size_t)src_row[i] * K + 64 * j);
        }
        cp_async_commit();
        ls.r.advance<kTStages>();
        if (++ls.npend > kTLag) {
            cp_async_wait<kTLag>();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&t_full[ls.pub]);
            ls.pub = (ls.pub + 1 == kTStages) ? 0 : ls.pub + 1;
            --ls.npend;
        }
    }
    return true;
}

template <bool GATEUP>
__global__ void __launch_bounds__(kPThreads, 1) k_prefill(PArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tring = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* a_full = reinterpret_cast<uint64_t*>(tring + (size_t)kTStages * kTStageBytes);
    uint64_t* a_empty = a_full + kAStages;
    uint64_t* t_full = a_empty + kAStages;
    uint64_t* t_empty = t_full + kTStages;
    uint64_t* d_full = t_empty + kTStages;
    uint64_t* d_empty = d_full + 2;
    uint64_t* drain = d_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.P.H, F = a.P.F;
    const int n_nt = GATEUP ? F / 128 : (H / 128 + 1) / 2;
    const int nk = (GATEUP ? H : F) / 32;
    const int n_tasks = (*a.n_wg) * n_nt;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 32) {
        for (int i = 0; i < kAStages; ++i) {
            mbar_init(&a_full[i], kProdWarps);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < kTStages; ++i) {
            mbar_init(&t_full[i], kLoadWarps);
            mbar_init(&t_empty[i], 1);
        }
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
        const int m = warp >> 2, lq = warp & 3;
        Ring ar;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
            const Tile T = load_tile(a, task, n_nt);
            switch (T.bits) {
                case 3: ok = produce_tile<3, GATEUP>(a, T, m, lq, lane, tbase, a_full, a_empty, ar); break;
                case 4: ok = produce_tile<4, GATEUP>(a, T, m, lq, lane, tbase, a_full, a_empty, ar); break;
                default: ok = produce_tile<8, GATEUP>(a, T, m, lq, lane, tbase, a_full, a_empty, ar); break;
            }
        }
    } else if (warp >= kLoadWarp0 && warp < kLoadWarp0 + kLoadWarps) {
        // ---------------- token loaders ----------------
        const int lt = threadIdx.x - 32 * kLoadWarp0;
        LoadState ls;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
            const Tile T = load_tile(a, task, n_nt);
            ok = load_tile_tokens<GATEUP>(a, T, lt, tring, t_full, t_empty, ls);
        }
        cp_async_wait<0>();
        if (ok) {
            fence_proxy_async_smem();
            __syncwarp();
            for (; ls.npend > 0; --ls.npend) {
                if (lane == 0) mbar_arrive(&t_full[ls.pub]);
                ls.pub = (ls.pub + 1 == kTStages) ? 0 : ls.pub + 1;
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            Ring ar, tr, dr;
            uint32_t a_ph = 0, t_ph = 0;
            for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
                const Tile T = load_tile(a, task, n_nt);
                const int b = dr.s;
                if ((dr.used >> b) & 1u) {
                    if (!mbar_wait_bounded(&d_empty[b], (dr.phase >> b) & 1u)) { ok = false; break; }
                    dr.phase ^= 1u << b;
                }
                dr.used |= 1u << b;
                tc_fence_after();
                const int nmma = (T.ntok + 15) & ~15;
                const uint32_t idesc = umma_idesc(128, nmma);
                const bool act1 = GATEUP || (2 * T.nt + 1) * 128 < H;
                const uint32_t dcol = tbase + (uint32_t)(b * kDCols);
                for (int kk = 0; kk < nk; ++kk) {
                    const int ts = tr.s;
                    if ((kk & 1) == 0) {
                        if (!mbar_wait_bounded(&t_full[ts], (t_ph >> ts) & 1u)) { ok = false; break; }
                        t_ph ^= 1u << ts;
                    }
                    const int as = ar.s;
                    if (!mbar_wait_bounded(&a_full[as], (a_ph >> as) & 1u)) { ok = false; break; }
                    a_ph ^= 1u << as;
                    tc_fence_after();
                    const uint32_t tsm = smem_u32(tring + (size_t)ts * kTStageBytes) + (kk & 1) * 64;
#pragma unroll
                    for (int mm = 0; mm < kNM; ++mm) {
                        if (mm == 1 && !act1) break;
#pragma unroll
                        for (int k16 = 0; k16 < 2; ++k16)
                            umma_ts(dcol + mm * kNT,
                                    tbase + (uint32_t)(kACol0 + as * kAStageCols + mm * 16 + k16 * 8),
                                    umma_desc(tsm + k16 * 32), idesc, (kk | k16) ? 1u : 0u);
                    }
                    umma_commit(&a_empty[as]);
                    ar.advance<kAStages>();
                    if (kk & 1) {
                        umma_commit(&t_empty[ts]);
                        tr.advance<kTStages>();
                    }
                }
                if (!ok) break;
                umma_commit(&d_full[b]);
                dr.advance<2>();
            }
            // every MMA issued by this thread has finished before TMEM is freed
            umma_commit(drain);
            if (!mbar_wait_bounded(drain, 0)) ok = false;
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 8-11: TMEM lanes 32 (warp % 4) ..) ----------------
        const int lq = warp & 3;
        Ring dr;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
            const Tile T = load_tile(a, task, n_nt);
            const int b = dr.s;
            if (!mbar_wait_bounded(&d_full[b], (dr.phase >> b) & 1u)) { ok = false; break; }
            dr.phase ^= 1u << b;
            tc_fence_after();
            const uint32_t tl = tbase + ((uint32_t)(lq * 32) << 16) + (uint32_t)(b * kDCols);
            if (GATEUP) {
                const int f = T.nt * 128 + lq * 32 + lane;  // this lane's feature
                const bool odd = lane & 1;
#pragma unroll 1
                for (int c0 = 0; c0 < T.ntok; c0 += 16) {
                    uint32_t g[16], v[16];
                    tmem_ld16(tl + c0, g);
                    tmem_ld16(tl + kNT + c0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        uint32_t hb[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const float gg = T.scale * __uint_as_float(g[2 * i + u]);
                            const float vv = T.scale * __uint_as_float(v[2 * i + u]);
                            hb[u] = __bfloat16_as_ushort(
                                __float2bfloat16_rn(__fdividef(gg, 1.0f + __expf(-gg)) * vv));
                        }
                        // lanes 2l, 2l+1 swap halves so each stores a (f even, f odd)
                        // pair: the even lane for token t, the odd lane for t + 1
                        const uint32_t recv = __shfl_xor_sync(0xffffffffu, odd ? hb[0] : hb[1], 1);
                        const int t = c0 + 2 * i + (odd ? 1 : 0);
                        const uint32_t lo = odd ? recv : hb[0];
                        const uint32_t hi = odd ? hb[1] : recv;
                        if (t < T.ntok)
                            *reinterpret_cast<uint32_t*>(a.h_out + (size_t)(T.pos0 + t) * F + (f & ~1)) =
                                lo | (hi << 16);
                    }
                }
            } else {
#pragma unroll 1
                for (int mm = 0; mm < kNM; ++mm) {
                    if ((2 * T.nt + mm) * 128 >= H) break;
                    const int o = (2 * T.nt + mm) * 128 + lq * 32 + lane;  // output feature
#pragma unroll 1
                    for (int c0 = 0; c0 < T.ntok; c0 += 16) {
                        uint32_t y[16];
                        tmem_ld16(tl + mm * kNT + c0, y);
                        // assignment and weight of tokens c0 .. c0 + 15 (lanes 0..15)
                        int asg = 0;
                        float wt = 0.0f;
                        if (lane < 16 && c0 + lane < T.ntok) {
                            asg = a.perm[T.pos0 + c0 + lane];
                            wt = a.topk_w[asg];
                        }
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int ai = __shfl_sync(0xffffffffu, asg, i);
                            const float wi = __shfl_sync(0xffffffffu, wt, i);
                            if (c0 + i < T.ntok)
                                a.y_out[(size_t)ai * H + o] = wi * (T.scale * __uint_as_float(y[i]));
                        }
                    }
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

}  // namespace

void prefill_set_smem_limits() {
    cudaFuncSetAttribute(k_prefill<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    cudaFuncSetAttribute(k_prefill<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
}

void launch_prefill_gateup(mpe_ctx* c, const __nv_bfloat16* x, int k) {
    PArgs a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg = c->s.n_wg;
    a.perm = c->s.perm;
    a.k = k;
    a.act = x;
    a.h_out = c->s.h;
    a.status = c->d_status;
    k_prefill<true><<<sm_count(c->device), kPThreads, kSmem, c->stream>>>(a);
    c->launches++;
}

void launch_prefill_down(mpe_ctx* c, const float* topk_w) {
    PArgs a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg = c->s.n_wg;
    a.perm = c->s.perm;
    a.k = 1;
    a.act = c->s.h;
    a.y_out = c->s.y;
    a.topk_w = topk_w;
    a.status = c->d_status;
    k_prefill<false><<<sm_count(c->device), kPThreads, kSmem, c->stream>>>(a);
    c->launches++;
}

}  // namespace mpe
