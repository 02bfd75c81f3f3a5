// Prefill-sized expert FFN on the 5th-generation tensor cores (tcgen05).
//
// PagedWeight, "Dynamic Paging": the active experts' pages are dequantized on
// the fly and multiplied with the tokens; at prefill sizes (hundreds of
// tokens per expert) this is a dense grouped GEMM per expert:
//   gate/up: G = X W1^T, V = X W3^T (tokens x F), h = silu(s G) (s V) -> bf16
//   down:    Y = h W2^T (tokens x H), y_a = w_a s Y_a -> bf16 per assignment
//
// Persistent warp-specialised kernel, one CTA per SM, 9 warps:
//   warps 0-3  producers: thread i owns tile row i. Per K-step of 64 it
//              gathers its token row's 128 bytes with cp.async (zero fill
//              past the group) and dequantizes its weight row's 64 codes
//              (one half block of the packed chunk format) to exact bf16
//              integers in registers, writing both into SWIZZLE_128B
//              K-major shared-memory tiles (16-byte chunk c of row r at
//              c ^ (r & 7)); the packed words of the next K-step are loaded
//              while the current one is unpacked.
//   warp 8     MMA issuer (one thread): tcgen05.mma.cta_group::1.kind::f16,
//              M = 128 tokens, N = 128 features, K = 16, fp32 accumulators in
//              tensor memory; tcgen05.commit releases each stage and signals
//              a finished accumulator.
//   warps 4-7  epilogue: tcgen05.ld of their 32 accumulator lanes, apply the
//              per-expert scale and SwiGLU (gate/up) or the top-k weight
//              (down), store bf16.
// Tensor memory holds two (gate/up: G and V) or four (down) accumulators so
// the epilogue of one tile overlaps the MMAs of the next. Work: tiles of <= 128
// positions of one expert (route work groups) x 128 output features; CTA b
// takes tiles b, b + grid, ... Every wait is bounded.
#include "internal.h"

namespace mpe {
namespace {

constexpr int kPM = 128;            // tokens per tile (MMA M)
constexpr int kPN = 128;            // features per tile (MMA N)
constexpr int kPK = 64;             // K per stage: one 128-byte swizzled row
constexpr int kTile = 128 * 128;    // bytes of one 128 x 64 bf16 operand tile
constexpr int kPThreads = 288;      // 4 producer + 4 epilogue + 1 MMA warps
constexpr int kMmaWarp = 8;

struct PArgs {
    PagedExperts P;
    const int32_t* wg;     // work groups (expert, first position, count), <= 128 positions
    const int32_t* n_wg;   // total groups
    const int32_t* perm;
    int k;
    const __nv_bfloat16* act;  // gate/up: x [T x H] by token; down: h [Tk x F] by position
    __nv_bfloat16* h_out;      // gate/up: h [Tk x F] by position
    float* y_out;              // down: y [Tk x H] by assignment, w * s * (h . K2 row)
    const float* topk_w;       // down: [Tk]
    uint32_t* status;
};

template <bool GATEUP>
struct PGeo {
    static constexpr int NM = GATEUP ? 2 : 1;       // weight matrices per tile
    static constexpr int STAGE = (1 + NM) * kTile;  // A tile + NM B tiles
    static constexpr int S = GATEUP ? 4 : 6;        // stages
    static constexpr int NB = GATEUP ? 2 : 4;       // accumulator buffers
    static constexpr int ACC_COLS = NM * kPN;       // TMEM columns per buffer
    static constexpr size_t SMEM = 1024 + (size_t)S * STAGE + 512;
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
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                     uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
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

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
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

// The packed words of one half block (64 codes = 2 quarters) of one row.
template <int B>
struct HalfRow {
    static constexpr int W = 2 * B;  // words: 3-bit 6, 4-bit 8, 8-bit 16
    uint32_t w[W];
};

template <int B>
__device__ __forceinline__ void load_half(const uint8_t* src, HalfRow<B>& h) {
    if constexpr (B == 3) {
        const uint2* p = reinterpret_cast<const uint2*>(src);
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const uint2 v = __ldg(p + i);
            h.w[2 * i] = v.x;
            h.w[2 * i + 1] = v.y;
        }
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
        for (int i = 0; i < B / 2; ++i) {
            const uint4 v = __ldg(p + i);
            h.w[4 * i] = v.x;
            h.w[4 * i + 1] = v.y;
            h.w[4 * i + 2] = v.z;
            h.w[4 * i + 3] = v.w;
        }
    }
}

// Unpack 64 codes (natural k order) to bf16 and store one swizzled 128-byte row.
template <int B>
__device__ __forceinline__ void store_half(const HalfRow<B>& h, uint8_t* tile, int row) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint32_t* qw = h.w + q * B;  // the quarter's B words
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {   // 16-byte chunk = 4 pairs
            uint4 v;
            v.x = unpack_pair<B>(qw, 4 * c4 + 0);
            v.y = unpack_pair<B>(qw, 4 * c4 + 1);
            v.z = unpack_pair<B>(qw, 4 * c4 + 2);
            v.w = unpack_pair<B>(qw, 4 * c4 + 3);
            const int c = q * 4 + c4;  // chunk of the 128-byte row
            *reinterpret_cast<uint4*>(tile + row * 128 + ((c ^ (row & 7)) << 4)) = v;
        }
    }
}

// Pipeline position of one producer thread, carried across tiles.
struct ProdState {
    int s = 0;        // next stage to fill
    int pub = 0;      // oldest filled stage not yet published
    int npend = 0;    // filled stages not yet published
    uint32_t ep = 0;  // parity of each stage's empty barrier
    uint32_t used = 0;
};

// cp.async groups a producer keeps in flight before publishing a stage.
constexpr int kLag = 2;
static_assert(PGeo<true>::S > kLag && PGeo<false>::S > kLag, "stages must exceed the publish lag");

// Producer thread `row`: all K-steps of one tile of width class B. The packed
// words are loaded two K-steps ahead of their unpack; a stage is published
// (full barrier) once the cp.async group kLag stages later has been issued.
template <int B, bool GATEUP>
__device__ __forceinline__ bool produce_tile(const PArgs& a, const Tile& T, int row,
                                             uint8_t* stages, uint64_t* full, uint64_t* empty,
                                             ProdState& ps) {
    using PG = PGeo<GATEUP>;
    constexpr int NM = PG::NM;
    const PagedExperts& P = a.P;
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int nk = K / kPK;
    const int nj = K / kCodesPerBlock;
    const int nc1 = chunks_w1(H, F);
    const int cpp = chunks_per_page(B, P.page_bytes);
    // token (A) row
    const __nv_bfloat16* arow = nullptr;
    if (row < T.ntok) {
        const int pos = T.pos0 + row;
        arow = a.act + (size_t)(GATEUP ? (a.perm[pos] / a.k) : pos) * K;
    }
    // weight (B) row: output feature f of each matrix, with a page cursor per
    // matrix pointing at the chunk of the next K-step to load
    const int f = T.nt * kPN + row;
    int pslot[NM], poff[NM];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
        const int c = (GATEUP ? m * nc1 : 2 * nc1) + (f >> 4) * nj;
        pslot[m] = c / cpp;
        poff[m] = c - pslot[m] * cpp;
    }
    const int rho_off = (f & 15) * block_bytes(B);
    int kl = 0;  // next K-step to load
    auto load_step = [&](HalfRow<B> (&w)[NM]) {
        if (kl > 0 && (kl & 1) == 0) {
#pragma unroll
            for (int m = 0; m < NM; ++m)
                if (++poff[m] == cpp) {
                    ++pslot[m];
                    poff[m] = 0;
                }
        }
#pragma unroll
        for (int m = 0; m < NM; ++m)
            load_half<B>(P.pool + (size_t)P.pidx[T.first + pslot[m]] * P.page_bytes +
                             (size_t)poff[m] * chunk_bytes(B) + rho_off + (kl & 1) * 8 * B,
                         w[m]);
        ++kl;
    };
    HalfRow<B> w0[NM], w1[NM];
    load_step(w0);
    if (nk > 1) load_step(w1);
    for (int kk = 0; kk < nk; ++kk) {
        const int s = ps.s;
        // the slot must have been released by the MMAs that read it last
        if ((ps.used >> s) & 1u) {
            if (!mbar_wait_bounded(&empty[s], (ps.ep >> s) & 1u)) return false;
            ps.ep ^= 1u << s;
        }
        ps.used |= 1u << s;
        uint8_t* st = stages + (size_t)s * PG::STAGE;
        // A: 8 x 16 bytes of the token row (zero fill past the group)
        const __nv_bfloat16* src = arow ? arow + kk * kPK : a.act;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            cp_async16(st + row * 128 + ((c ^ (row & 7)) << 4), src + 8 * c, arow ? 16u : 0u);
        cp_async_commit();
        HalfRow<B> w2[NM];
        if (kk + 2 < nk) load_step(w2);
        // B: dequantize this K-step's half blocks into the swizzled tiles
#pragma unroll
        for (int m = 0; m < NM; ++m) store_half<B>(w0[m], st + (1 + m) * kTile, row);
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            w0[m] = w1[m];
            w1[m] = w2[m];
        }
        ps.s = (s + 1 == PG::S) ? 0 : s + 1;
        if (++ps.npend > kLag) {
            cp_async_wait<kLag>();
            fence_proxy_async_smem();
            mbar_arrive(&full[ps.pub]);
            ps.pub = (ps.pub + 1 == PG::S) ? 0 : ps.pub + 1;
            --ps.npend;
        }
    }
    return true;
}

template <bool GATEUP>
__global__ void __launch_bounds__(kPThreads, 1) k_prefill(PArgs a) {
    using PG = PGeo<GATEUP>;
    constexpr int NM = PG::NM;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + (size_t)PG::S * PG::STAGE);
    uint64_t* empty = full + PG::S;
    uint64_t* accfull = empty + PG::S;
    uint64_t* accempty = accfull + PG::NB;
    uint64_t* drain = accempty + PG::NB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.P.H, F = a.P.F;
    const int R = GATEUP ? F : H;
    const int K = GATEUP ? H : F;
    const int n_nt = R / kPN;
    const int nk = K / kPK;
    const int n_tasks = (*a.n_wg) * n_nt;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 32) {
        for (int i = 0; i < PG::S; ++i) {
            mbar_init(&full[i], 128);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < PG::NB; ++i) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], 128);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    bool ok = true;

    if (warp < 4) {
        // ---------------- producers ----------------
        const int row = threadIdx.x;
        ProdState ps;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
            const Tile T = load_tile(a, task, n_nt);
            switch (T.bits) {
                case 3: ok = produce_tile<3, GATEUP>(a, T, row, stages, full, empty, ps); break;
                case 4: ok = produce_tile<4, GATEUP>(a, T, row, stages, full, empty, ps); break;
                default: ok = produce_tile<8, GATEUP>(a, T, row, stages, full, empty, ps); break;
            }
        }
        cp_async_wait<0>();
        if (ok) {
            fence_proxy_async_smem();
            for (; ps.npend > 0; --ps.npend) {
                mbar_arrive(&full[ps.pub]);
                ps.pub = (ps.pub + 1 == PG::S) ? 0 : ps.pub + 1;
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = umma_idesc(kPM, kPN);
            int s = 0, b = 0;
            uint32_t fp = 0, aep = 0, aused = 0;
            for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
                if ((aused >> b) & 1u) {
                    if (!mbar_wait_bounded(&accempty[b], (aep >> b) & 1u)) { ok = false; break; }
                    aep ^= 1u << b;
                }
                aused |= 1u << b;
                tc_fence_after();
                const uint32_t dcol = tbase + (uint32_t)(b * PG::ACC_COLS);
                for (int kk = 0; kk < nk; ++kk) {
                    if (!mbar_wait_bounded(&full[s], (fp >> s) & 1u)) { ok = false; break; }
                    fp ^= 1u << s;
                    tc_fence_after();
                    const uint32_t st = smem_u32(stages + (size_t)s * PG::STAGE);
#pragma unroll
                    for (int k16 = 0; k16 < kPK / 16; ++k16) {
                        const uint64_t ad = umma_desc(st + k16 * 32);
#pragma unroll
                        for (int m = 0; m < NM; ++m) {
                            const uint64_t bd = umma_desc(st + (1 + m) * kTile + k16 * 32);
                            umma(dcol + m * kPN, ad, bd, idesc, (kk | k16) ? 1u : 0u);
                        }
                    }
                    umma_commit(&empty[s]);  // frees the stage when these MMAs finish
                    s = (s + 1 == PG::S) ? 0 : s + 1;
                }
                if (!ok) break;
                umma_commit(&accfull[b]);
                b = (b + 1 == PG::NB) ? 0 : b + 1;
            }
            // every MMA issued by this thread has finished before TMEM is freed
            umma_commit(drain);
            if (!mbar_wait_bounded(drain, 0)) ok = false;
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 4-7: TMEM lanes 32 (warp % 4) ..) ----------------
        const int lane_grp = warp & 3;
        const int row = lane_grp * 32 + lane;
        int b = 0;
        uint32_t afp = 0;
        for (int task = blockIdx.x; task < n_tasks && ok; task += gridDim.x) {
            const Tile T = load_tile(a, task, n_nt);
            if (!mbar_wait_bounded(&accfull[b], (afp >> b) & 1u)) { ok = false; break; }
            afp ^= 1u << b;
            tc_fence_after();
            const uint32_t tl = tbase + ((uint32_t)(lane_grp * 32) << 16) + (uint32_t)(b * PG::ACC_COLS);
            const bool valid = row < T.ntok;
            const int pos = T.pos0 + row;
            if (GATEUP) {
                __nv_bfloat16* dst = a.h_out + (size_t)pos * F + T.nt * kPN;
#pragma unroll 1
                for (int c0 = 0; c0 < kPN; c0 += 16) {
                    uint32_t g[16], v[16];
                    tmem_ld16(tl + c0, g);
                    tmem_ld16(tl + kPN + c0, v);
                    tmem_wait_ld();
                    uint32_t hv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float h2[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const float gg = T.scale * __uint_as_float(g[2 * i + u]);
                            const float vv = T.scale * __uint_as_float(v[2 * i + u]);
                            h2[u] = gg / (1.0f + __expf(-gg)) * vv;
                        }
                        __nv_bfloat162 p = __floats2bfloat162_rn(h2[0], h2[1]);
                        hv[i] = *reinterpret_cast<uint32_t*>(&p);
                    }
                    if (valid) {
                        reinterpret_cast<uint4*>(dst + c0)[0] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                        reinterpret_cast<uint4*>(dst + c0)[1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
                    }
                }
            } else {
                int asg = 0;
                float wt = 0.0f;
                if (valid) {
                    asg = a.perm[pos];
                    wt = a.topk_w[asg];
                }
                float* dst = a.y_out + (size_t)asg * H + T.nt * kPN;
#pragma unroll 1
                for (int c0 = 0; c0 < kPN; c0 += 16) {
                    uint32_t y[16];
                    tmem_ld16(tl + c0, y);
                    tmem_wait_ld();
                    float yv[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) yv[i] = wt * (T.scale * __uint_as_float(y[i]));
                    if (valid) {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            reinterpret_cast<float4*>(dst + c0)[i] =
                                make_float4(yv[4 * i], yv[4 * i + 1], yv[4 * i + 2], yv[4 * i + 3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&accempty[b]);
            b = (b + 1 == PG::NB) ? 0 : b + 1;
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

}  // namespace

void prefill_set_smem_limits() {
    cudaFuncSetAttribute(k_prefill<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)PGeo<true>::SMEM);
    cudaFuncSetAttribute(k_prefill<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)PGeo<false>::SMEM);
}

// one persistent CTA per SM (the shared-memory footprint admits no second)
static int sms(mpe_ctx* c) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, c->device);
    return n > 0 ? n : 1;
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
    k_prefill<true><<<sms(c), kPThreads, PGeo<true>::SMEM, c->stream>>>(a);
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
    k_prefill<false><<<sms(c), kPThreads, PGeo<false>::SMEM, c->stream>>>(a);
    c->launches++;
}

}  // namespace mpe
