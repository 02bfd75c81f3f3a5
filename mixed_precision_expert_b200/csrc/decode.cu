// Decode-sized expert FFN: grouped GEMV / skinny GEMM straight from the pages.
//
// PagedWeight, "Dynamic Paging": the pass fetches the active experts' pages
// and dequantizes them on the fly; nothing is materialised in full precision
// (the DecDEC summary, 2.1, notes decode is memory-bound, so the packed bytes
// are the cost). Per expert e with scale s_e and codes K1, K3, K2:
//   gate/up:  g = s_e (K1 x), v = s_e (K3 x), h = silu(g) v   (h stored bf16)
//   down:     y_a = w_a s_e (K2 h_a)                          (y stored fp32)
//
// One CTA = one work group (<= 16 tokens of one expert) x one 16-row tile of
// the output; its 4 warps split K. Each warp streams its chunks (16 rows x 128
// codes) of the matrix tile through a 3-stage shared-memory ring filled by
// 1-D bulk copies (cp.async.bulk, no multicast) that complete on mbarriers;
// lane 0 issues, all lanes wait (bounded). Lanes unpack codes to exact bf16
// integers in registers (common.cuh) and feed mma.sync m16n8k16 with the
// weights as the 16-row A operand and up to two 8-token n-tiles of
// activations as B; the per-expert scale multiplies the fp32 accumulator in
// the epilogue.
//
// k-permutation: inside a 128-code block, thread t (= lane & 3) owns 16 code
// pairs; mma step c (0..7) uses its pairs 2c and 2c+1 as the logical k-pairs
// t and t+4. Pair m of thread t covers codes
//   b = 3, 4: 32 t + 2m                      (quarter t)
//   b = 8:    16 t + 2m (m < 8), 64 + 16 t + 2(m - 8) (m >= 8)
// and the activation registers are loaded with the same permutation.
#include "internal.h"

namespace mpe {
namespace {

constexpr int kWarps = 4;
constexpr int kStages = 3;
constexpr int kStageBytes = 2048;  // per matrix per stage
constexpr int kMaxTiles = kDecodeGroup / 8;

template <int B>
struct Geo {
    static constexpr int CB = 256 * B;                              // chunk bytes
    static constexpr int J = (2048 / CB) > 0 ? (2048 / CB) : 1;     // chunks per stage
    static constexpr int WORDS = (B == 8) ? 8 : B;                  // raw words per row
};

struct Args {
    PagedExperts P;
    const int32_t* wg;
    const int32_t* n_wg;
    const int32_t* perm;
    int k;
    const __nv_bfloat16* act;  // gate/up: x [T x H]; down: h [Tk x F] in perm order
    __nv_bfloat16* h_out;      // gate/up: h [Tk x F]
    float* y_out;              // down: y [Tk x H], row a = assignment
    const float* topk_w;       // down: [Tk]
    uint32_t* status;
};

constexpr size_t smem_bytes(int nm) {
    return (size_t)kWarps * kStages * nm * kStageBytes + kWarps * kStages * sizeof(uint64_t);
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

// This thread's 16 activation pairs of block j for one token row (same k
// permutation as the weights).
template <int B>
__device__ __forceinline__ void load_act(const __nv_bfloat16* row, int j, int t,
                                         uint32_t (&xb)[16]) {
    if (row == nullptr) {
#pragma unroll
        for (int i = 0; i < 16; ++i) xb[i] = 0u;
        return;
    }
    const __nv_bfloat16* base = row + 128 * j;
    uint4 v[4];
    if constexpr (B == 8) {
        const uint4* p0 = reinterpret_cast<const uint4*>(base + 16 * t);
        const uint4* p1 = reinterpret_cast<const uint4*>(base + 64 + 16 * t);
        v[0] = __ldg(p0);
        v[1] = __ldg(p0 + 1);
        v[2] = __ldg(p1);
        v[3] = __ldg(p1 + 1);
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(base + 32 * t);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __ldg(p + i);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xb[4 * i + 0] = v[i].x;
        xb[4 * i + 1] = v[i].y;
        xb[4 * i + 2] = v[i].z;
        xb[4 * i + 3] = v[i].w;
    }
}

template <int B, bool GATEUP>
__device__ __forceinline__ void run(const Args& a, uint8_t* smem, int e, int pos0, int ntok,
                                    const Pte& pte) {
    using G = Geo<B>;
    constexpr int NM = GATEUP ? 2 : 1;
    const PagedExperts& P = a.P;
    const int H = P.H, F = P.F;
    const int K = GATEUP ? H : F;
    const int nj = K / kCodesPerBlock;
    const int tau = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nc1 = chunks_w1(H, F);
    const int j_lo = (warp * nj) / kWarps, j_hi = ((warp + 1) * nj) / kWarps;
    const int nst = (j_hi - j_lo + G::J - 1) / G::J;

    uint8_t* wsm = smem + (size_t)warp * kStages * NM * kStageBytes;
    uint64_t* bars =
        reinterpret_cast<uint64_t*>(smem + (size_t)kWarps * kStages * NM * kStageBytes) +
        warp * kStages;

    // activation rows of this thread's tokens (n-tile nt, token nt*8 + g)
    const __nv_bfloat16* arow[kMaxTiles];
#pragma unroll
    for (int nt = 0; nt < kMaxTiles; ++nt) {
        const int n = nt * 8 + g;
        arow[nt] = nullptr;
        if (n < ntok) {
            const int pos = pos0 + n;
            const int row = GATEUP ? (a.perm[pos] / a.k) : pos;
            arow[nt] = a.act + (size_t)row * K;
        }
    }
    const int ntiles = (ntok + 7) / 8;

    auto chunk_of = [&](int m, int j) -> int {
        if (GATEUP) return m * nc1 + tau * nj + j;
        return 2 * nc1 + tau * nj + j;
    };
    auto issue = [&](int i) {
        const int s = i % kStages;
        const int j0 = j_lo + i * G::J;
        const int nch = min(G::J, j_hi - j0);
        mbar_arrive_expect_tx(&bars[s], (uint32_t)(nch * G::CB * NM));
        const int cpp = chunks_per_page(B, P.page_bytes);
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            uint8_t* dst = wsm + (size_t)(s * NM + m) * kStageBytes;
            int done = 0;
            while (done < nch) {
                const int c = chunk_of(m, j0 + done);
                const int n = min(nch - done, cpp - c % cpp);
                bulk_g2s(dst + done * G::CB, chunk_addr(P, pte, B, c), (uint32_t)(n * G::CB),
                         &bars[s]);
                done += n;
            }
        }
    };

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        fence_proxy_async_smem();
        for (int i = 0; i < min(kStages, nst); ++i) issue(i);
    }
    __syncwarp();

    float acc[kMaxTiles][NM][4];
#pragma unroll
    for (int nt = 0; nt < kMaxTiles; ++nt)
#pragma unroll
        for (int m = 0; m < NM; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][m][i] = 0.0f;

    bool ok = true;
    int i = 0;
    for (; i < nst; ++i) {
        const int s = i % kStages;
        if (!mbar_wait_bounded(&bars[s], (uint32_t)((i / kStages) & 1))) {
            ok = false;
            break;
        }
        const int j0 = j_lo + i * G::J;
        const int nch = min(G::J, j_hi - j0);
        for (int jj = 0; jj < nch; ++jj) {
            const int j = j0 + jj;
            uint32_t wr[NM][2][G::WORDS];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const uint8_t* chunk = wsm + (size_t)(s * NM + m) * kStageBytes + jj * G::CB;
                load_row_words<B>(chunk, g, t, g, wr[m][0]);
                load_row_words<B>(chunk, g + 8, t, g, wr[m][1]);
            }
            uint32_t xb[kMaxTiles][16];
#pragma unroll
            for (int nt = 0; nt < kMaxTiles; ++nt) {
                if (nt < ntiles) load_act<B>(arow[nt], j, t, xb[nt]);
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) {
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    const uint32_t a0 = unpack_pair<B>(wr[m][0], 2 * c);
                    const uint32_t a1 = unpack_pair<B>(wr[m][1], 2 * c);
                    const uint32_t a2 = unpack_pair<B>(wr[m][0], 2 * c + 1);
                    const uint32_t a3 = unpack_pair<B>(wr[m][1], 2 * c + 1);
#pragma unroll
                    for (int nt = 0; nt < kMaxTiles; ++nt) {
                        if (nt < ntiles)
                            mma_bf16_16816(acc[nt][m], a0, a1, a2, a3, xb[nt][2 * c],
                                           xb[nt][2 * c + 1]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0 && i + kStages < nst) {
            fence_proxy_async_smem();
            issue(i + kStages);
        }
    }
    if (!ok) {
        if (lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
        // let every copy already issued land before the CTA's smem goes away
        for (int r = i; r < min(nst, i + kStages); ++r)
            mbar_wait_bounded(&bars[r % kStages], (uint32_t)((r / kStages) & 1));
    }

    // cross-warp reduction over the K split, through shared memory
    __syncthreads();
    float* red = reinterpret_cast<float*>(smem);
    constexpr int PER = kMaxTiles * NM * 4;
#pragma unroll
    for (int nt = 0; nt < kMaxTiles; ++nt)
#pragma unroll
        for (int m = 0; m < NM; ++m)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                red[((warp * PER) + (nt * NM + m) * 4 + q) * 32 + lane] = acc[nt][m][q];
    __syncthreads();
    if (warp != 0) return;
    const float s = pte.scale;
#pragma unroll
    for (int nt = 0; nt < kMaxTiles; ++nt) {
        if (nt >= ntiles) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float sum[NM];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                float v = 0.0f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) v += red[((w * PER) + (nt * NM + m) * 4 + q) * 32 + lane];
                sum[m] = v;
            }
            const int row = tau * 16 + g + 8 * (q >> 1);
            const int n = nt * 8 + 2 * t + (q & 1);
            if (n >= ntok) continue;
            const int pos = pos0 + n;
            if (GATEUP) {
                const float gv = s * sum[0];
                const float uv = s * sum[NM - 1];
                const float hv = gv / (1.0f + __expf(-gv)) * uv;
                a.h_out[(size_t)pos * F + row] = __float2bfloat16_rn(hv);
            } else {
                const int asg = a.perm[pos];
                a.y_out[(size_t)asg * H + row] = a.topk_w[asg] * (s * sum[0]);
            }
        }
    }
}

template <bool GATEUP>
__global__ void __launch_bounds__(kWarps * 32) k_decode(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int gi = blockIdx.x;
    if (gi >= *a.n_wg) return;
    const int e = a.wg[3 * gi], pos0 = a.wg[3 * gi + 1], ntok = a.wg[3 * gi + 2];
    const Pte pte = a.P.pte[e];
    switch (pte.bits) {
        case 3: run<3, GATEUP>(a, smem, e, pos0, ntok, pte); break;
        case 4: run<4, GATEUP>(a, smem, e, pos0, ntok, pte); break;
        case 8: run<8, GATEUP>(a, smem, e, pos0, ntok, pte); break;
        default: break;
    }
}

}  // namespace

void decode_set_smem_limits() {
    cudaFuncSetAttribute(k_decode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes(2));
    cudaFuncSetAttribute(k_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes(1));
}

void launch_decode_gateup(mpe_ctx* c, const __nv_bfloat16* x, int k, int wg_bound) {
    Args a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg = c->s.n_wg;
    a.perm = c->s.perm;
    a.k = k;
    a.act = x;
    a.h_out = c->s.h;
    a.status = c->d_status;
    dim3 grid((unsigned)wg_bound, (unsigned)(c->F / 16));
    k_decode<true><<<grid, kWarps * 32, smem_bytes(2), c->stream>>>(a);
    c->launches++;
}

void launch_decode_down(mpe_ctx* c, const float* topk_w, int wg_bound) {
    Args a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg = c->s.n_wg;
    a.perm = c->s.perm;
    a.k = 1;
    a.act = c->s.h;
    a.y_out = c->s.y;
    a.topk_w = topk_w;
    a.status = c->d_status;
    dim3 grid((unsigned)wg_bound, (unsigned)(c->H / 16));
    k_decode<false><<<grid, kWarps * 32, smem_bytes(1), c->stream>>>(a);
    c->launches++;
}

}  // namespace mpe
