// Decode-sized expert FFN: grouped GEMV / skinny GEMM straight from the pages.
//
// PagedWeight, "Dynamic Paging": the pass fetches the active experts' pages
// and dequantizes them on the fly; nothing is materialised in full precision
// (decode is memory-bound -- DecDEC summary, 2.1 -- so the packed bytes are
// the cost). Per expert e with scale s_e and codes K1, K3, K2:
//   gate/up:  g = s_e (K1 x), v = s_e (K3 x), h = silu(g) v   (h stored bf16)
//   down:     y_pos = s_e (K2 h_pos)                         (y stored fp32 by
//             route position; the combine applies the top-k weights)
//
// Warp-specialised persistent kernel. A CTA (one per SM) has 14 consumer
// warps, 1 copy warp and 1 task warp and works on one task at a time: a work
// group (<= 16 tokens of one expert) x 14 (gate/up: one per consumer warp) or
// 28 (down: two per warp) consecutive 16-row output tiles x a K part.
//   task warp:  claims tasks from a per-width-class counter and resolves them
//               (expert, tokens, activation rows, scale, first page entry)
//               into a 4-entry task queue in shared memory, ahead of use, so
//               no other warp waits on a chain of dependent global loads;
//   copy warp:  for each queued task and each group of J block columns, fills
//               one slot of the CTA's shared-memory ring with the task's
//               chunks (one 1-D bulk copy per consumer share, issued by 14
//               lanes in parallel, no multicast; a full mbarrier counts the
//               bytes) and prefetches the block's activation lines into L1;
//   consumers:  wait on the slot's full barrier, copy their chunk's words to
//               registers, release the slot on its empty barrier and only then
//               unpack (common.cuh) and multiply with mma.sync m16n8k16 --
//               weights are the 16-row A operand, one or two 8-token
//               n-tiles of activations are B (they share every unpacked
//               weight fragment; a down warp's two tiles interleave step
//               by step), fp32 accumulate,
//               the per-expert scale applied once at the end.
// A task whose K range is split in P parts writes a scaled partial to its own
// slice; a later pass sums the slices in part order (deterministic, no
// atomics). The forward-pass kernels chain with programmatic dependent launch:
// a kernel starts while its predecessor drains and waits (griddepcontrol) only
// where it reads what the predecessor wrote.
//
// k-permutation: inside a 128-code block, thread t (= lane & 3) owns 16 code
// pairs; mma step c (0..7) uses its pairs 2c and 2c+1 as the logical k-pairs
// t and t+4. Pair m of thread t covers codes
//   b = 3, 4: 32 t + 2m                      (quarter t)
//   b = 8:    16 t + 2m (m < 8), 64 + 16 t + 2(m - 8) (m >= 8)
// and the activation registers are loaded with the same permutation.
//
// The same kernels serve the prefix-compatible layered store (template flag
// PX, prefix.cu): its layers A, B, C are chunk streams in this format's
// layout, so the copy warp fetches one run per stored layer for each share
// (from that layer's pages) and the consumers merge the layers' words in
// registers (UnpackRegs<3>, UnpackPx4, UnpackPx8 below; quarter permutation
// at every width); the per-width scale and offsets come in through the page
// table mirror and the offset sums.
#include <cstdlib>

#include "internal.h"

namespace mpe {
namespace {

// 16 warps per SM in all: ptxas rounds a CTA's warps up to a multiple of 4
// when it sets the register budget, and 16 warps leave 128 registers a thread
// (17-20 warps would leave 96, too few for the gate/up consumer).
constexpr int kConsumers = 14;                   // consumer warps per CTA
constexpr int kCopyWarp = kConsumers;            // fills the ring
constexpr int kTaskWarp = kConsumers + 1;        // claims and resolves tasks
constexpr int kThreads = (kConsumers + 2) * 32;  // one CTA per SM
constexpr int kRingBytes = 192 * 1024;           // shared-memory ring per CTA
constexpr int kSlotBudget = 56 * 1024;           // at least three slots per ring
constexpr int kMaxSlots = 16;
constexpr int kTaskQ = 4;                        // resolved tasks queued ahead
constexpr int kMaxTiles = kDecodeGroup / 8;

// Tiles per consumer warp: the down kernel gives each warp two 16-row tiles
// that share one activation fragment (its rows stream 1 weight byte per 2
// activation bytes through L1 otherwise); gate/up already multiplies two
// matrices per fragment.
__host__ __device__ constexpr int tiles_per_warp(bool gateup) { return gateup ? 1 : 2; }
__host__ __device__ constexpr int tiles_per_task(bool gateup) {
    return kConsumers * tiles_per_warp(gateup);
}

// A slot holds J consecutive block columns of every tile of a task, one share
// per consumer warp. The bulk-copy engine takes ~80 cycles per copy whatever
// its size up to a few KB, so a share's chunks for the slot -- gate and up of
// its tile interleaved, or its two down tiles interleaved, for consecutive
// block columns: one contiguous run of the page -- go in one copy, as many
// columns as keep a slot within 56 KB (at least three slots per 192 KB ring):
// gate/up 2 (3, 4 bits) or 1 (8 bits), down (two tiles a warp) 2 / 2 / 1.
template <int B, int NM, int TPW>
struct Geo {
    static constexpr int CB = 256 * B;                   // chunk bytes
    static constexpr int J = kSlotBudget / (kConsumers * TPW * NM * CB);  // columns per slot
    static constexpr int TILEB = NM * J * CB;            // one tile's share of a slot
    static constexpr int SLOT = kConsumers * TPW * TILEB;
    static constexpr int S = (kRingBytes / SLOT) < kMaxSlots ? (kRingBytes / SLOT) : kMaxSlots;
    static constexpr int WORDS = (B == 8) ? 8 : B;       // raw words per row
    static_assert(S >= 3 && J >= 1, "ring geometry");
};
template <int B>
using GeoGU = Geo<B, 2, tiles_per_warp(true)>;
template <int B>
using GeoDN = Geo<B, 1, tiles_per_warp(false)>;
// Each width class starts its ring at slot 0; a new class's slot i must lie
// within the previous class's slots 0..i, so slot sizes may not grow from one
// class to the next (the classes run 8, 4, 3 bits).
static_assert(GeoGU<8>::SLOT >= GeoGU<4>::SLOT && GeoGU<4>::SLOT >= GeoGU<3>::SLOT &&
                  GeoDN<8>::SLOT >= GeoDN<4>::SLOT && GeoDN<4>::SLOT >= GeoDN<3>::SLOT,
              "slot sizes per class");
static_assert(tiles_per_task(true) <= 32 && tiles_per_task(false) <= 32, "one copy lane a tile");

constexpr int kFirstSlot = 1;  // the slot opens its task
constexpr int kLastSlot = 2;   // the slot closes its task

struct SlotDesc {
    int q;      // task-queue entry of the slot's task; -1: no more tasks of this class
    int j;      // first block column held by the slot (end of class: the queue entry)
    int nc;     // block columns held (1 .. J)
    int flags;  // kFirstSlot | kLastSlot
};

// One resolved task, written by the task warp, read by the copy warp and the
// consumers when the task starts.
struct TaskMeta {
    int valid;   // 0: no more tasks of this width class
    int tq;      // tile group: tiles n tq .. n tq + n - 1, n = tiles_per_task
    int p;       // K part
    int pos0;    // first route position of the work group
    int ntok;    // tokens in the group (1 .. kDecodeGroup)
    int j0, j_hi;  // block columns [j0, j_hi)
    float scale;   // s_e
    uint32_t first;  // the expert's first entry in the page-index array
    uint32_t lfirst[2];  // layered store: first entries of layers B and C
    int rows[kDecodeGroup];  // activation row of each token (x row, or h row = position)
    // widths 3 and 4: off . x of each token over the task's K range, the term
    // the offset-form unpack adds to every row (written after the rest, see
    // tq_sum)
    float offsum[kDecodeGroup];
};

struct Args {
    PagedExperts P;
    const int32_t* wg;          // work groups sorted by width class: 8-bit, 4-bit, 3-bit
    const int32_t* n_wg_class;  // groups per class (3)
    const int32_t* perm;
    int k;
    const __nv_bfloat16* act;  // gate/up: x [T x H]; down: h [Tk x F] in perm order
    __nv_bfloat16* h_out;      // gate/up: h [Tk x F]
    float* y_out;              // down: y [P][Tk][H], row = route position
    float* part;               // gate/up split-K partials [P][Tk][2][F]
    size_t part_stride;        // floats per part slice (gate/up partials or down y)
    int32_t* task_ctr;         // claimed-task counters (one per class), zero at launch
    int parts;                 // P
    int direct_h;              // gate/up with P = 1: write h itself (else the partial)
    int kb;                    // blocks per part
    uint32_t* status;
    // layered (prefix-compatible) store: per expert the first page-index
    // entries of layers B and C (layer A's is the page table's `first`);
    // null for the main format
    const uint32_t* lfirst;
};

constexpr size_t kBarOff = kRingBytes;
constexpr size_t kDescOff = kBarOff + (2 * kMaxSlots + 3 * kTaskQ) * sizeof(uint64_t);
constexpr size_t kTaskOff = kDescOff + kMaxSlots * sizeof(SlotDesc);

__host__ __device__ constexpr size_t smem_bytes() {
    return kTaskOff + kTaskQ * sizeof(TaskMeta);
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
                                               uint32_t (&w)[Geo<B, 1, 1>::WORDS]) {
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

// The unpack's masks and magic numbers, held in registers. Each is produced by
// an opaque move once per consumer class, so the compiler keeps it in a
// register for the LOP3s instead of materialising the constant beside every
// use (the register budget allows it).
__device__ __forceinline__ uint32_t reg_const(uint32_t v) {
    uint32_t d;
    asm volatile("mov.b32 %0, %1;" : "=r"(d) : "r"(v));
    return d;
}

template <int N>
__device__ __forceinline__ uint32_t shr_imm(uint32_t a) {
    uint32_t d;
    asm("shr.b32 %0, %1, %2;" : "=r"(d) : "r"(a), "n"(N));
    return d;
}

template <int B>
struct UnpackRegs;

template <>
struct UnpackRegs<4> {
    uint32_t mask, magic;
    __device__ __forceinline__ UnpackRegs() : mask(reg_const(0x000F000Fu)), magic(reg_const(kMagic)) {}
    // pair m (0..15) of a quarter's 4 words, offset form: k + 136
    __device__ __forceinline__ uint32_t pair(const uint32_t* w, int m) const {
        const uint32_t x = w[m >> 2];
        const uint32_t v = (m & 3) == 0 ? x
                           : (m & 3) == 1 ? shr_imm<4>(x)
                           : (m & 3) == 2 ? shr_imm<8>(x)
                                          : shr_imm<12>(x);
        return and_or(v, mask, magic);
    }
};

template <>
struct UnpackRegs<3> {
    uint32_t m7, m38, b1, b2, b4, magic, magic16;
    __device__ __forceinline__ UnpackRegs()
        : m7(reg_const(0x00070007u)), m38(reg_const(0x00380038u)), b1(reg_const(0x00010001u)),
          b2(reg_const(0x00020002u)), b4(reg_const(0x00040004u)), magic(reg_const(kMagic)),
          magic16(reg_const(kMagic16)) {}
    // pair m (0..15) of a quarter's 3 words, offset form (see unpack_pair_off)
    __device__ __forceinline__ uint32_t pair(const uint32_t* w, int m) const {
        if (m == 15) {
            uint32_t t = and_or(shr_imm<15>(w[0]), b1, magic);
            t = and_or(shr_imm<14>(w[1]), b2, t);
            return and_or(shr_imm<13>(w[2]), b4, t);
        }
        const int v = m / 5, f = m % 5;
        const uint32_t x = f < 2 ? w[v] : (f < 4 ? shr_imm<6>(w[v]) : shr_imm<12>(w[v]));
        if (f == 1 || f == 3) return and_or(x, m38, magic16);  // 16 + u
        return and_or(x, m7, magic);                            // 128 + u
    }
};

template <>
struct UnpackRegs<8> {
    uint32_t m7f, m80, magic;
    __device__ __forceinline__ UnpackRegs()
        : m7f(reg_const(0x007F007Fu)), m80(reg_const(0x00800080u)), magic(reg_const(kMagic)) {}
    // pair m (0..15) of the thread's two 16-byte pieces: the signed code k
    __device__ __forceinline__ uint32_t pair(const uint32_t* w, int m) const {
        const uint32_t v = (m & 1) ? shr_imm<8>(w[m >> 1]) : w[m >> 1];
        const uint32_t lo = and_or(v, m7f, magic);     // 128 + (u & 127)
        const uint32_t hi = andnot_or(v, m80, magic);  // 256 - 128 * bit7(u)
        return bf2_sub(lo, hi);                        // u - 128 = k
    }
};

// Layered (prefix-compatible) store. Its layers are chunk streams in the
// main format's layout: A (u8 >> 5) in the 3-bit quarter layout, B (bit 4 of
// u8) in the 1-bit one (code pair m at bits m and 16 + m of the quarter's
// word), C (u8 & 15) in the 4-bit one; a b-bit expert keeps A (b = 3), A B
// (b = 4) or A B C (b = 8). The consumer's words of one row: A in w[0..2],
// B in w[3], C in w[4..7]. A 3-bit expert is the main 3-bit format with
// u = A (UnpackRegs<3>).
// a >> s for s > 0, a << -s for s < 0 (s is a constant once the block loop
// is unrolled)
__device__ __forceinline__ uint32_t shift_by(uint32_t a, int s) {
    return s > 0 ? (a >> s) : (s < 0 ? (a << (-s)) : a);
}

// 4 bits, u4 = 2 A + B, with half the work on the FMA pipe: A through the
// main 3-bit unpack (128 + A, or 16 + A for fields 1 and 3), B from the
// shifted B word at bit p = m & 3 (one shift serves four pairs) under the
// negative magic -2^(7-p) with the bit inverted: -(2^(7-p) + 1) + B. Then
// 2 (A value) + (B value) = const + u4 in one bf16x2 fma, exact: every const
// + u4 here is an integer of at most 8 significant bits (127 .. 254 for the
// 128 + A pairs, -97 .. 30 for the 16 + A ones).
struct UnpackPx4 {
    UnpackRegs<3> a;
    uint32_t two, n128, n64, n32, n16;
    __device__ __forceinline__ UnpackPx4()
        : two(reg_const(0x40004000u)), n128(reg_const(0xC300C300u)), n64(reg_const(0xC280C280u)),
          n32(reg_const(0xC200C200u)), n16(reg_const(0xC180C180u)) {}
    __device__ __forceinline__ uint32_t pair(const uint32_t* w, int m) const {
        const uint32_t va = a.pair(w, m);
        const int p = m & 3;
        const uint32_t bw = shift_by(w[3], 4 * (m >> 2));
        const uint32_t nm = p == 0 ? n128 : (p == 1 ? n64 : (p == 2 ? n32 : n16));
        return bf2_fma(va, two, andnot_or(bw, 0x00010001u << p, nm));
    }
};

// 8 bits, as two mma operands into one accumulator: hi = 16 (const + u4) from
// layers A and B (the 4-bit form above with every magic scaled by 16, so A
// gives 2048 + 16 A or 256 + 16 A, B gives -(2^(11-p) + 16) + 16 B, and one
// bf16x2 fma 2 hi_A + hi_B, exact), lo = 128 + C (the main 4-bit unpack of
// layer C). Their products summed in the accumulator are (16 const + 128 +
// u8) x, u8 = 16 u4 + C.
struct UnpackPx8 {
    uint32_t m2048, m256, two, n2048, n1024, n512, n256, magic;
    __device__ __forceinline__ UnpackPx8()
        : m2048(reg_const(0x45004500u)), m256(reg_const(0x43804380u)), two(reg_const(0x40004000u)),
          n2048(reg_const(0xC500C500u)), n1024(reg_const(0xC480C480u)),
          n512(reg_const(0xC400C400u)), n256(reg_const(0xC380C380u)), magic(reg_const(kMagic)) {}
    __device__ __forceinline__ uint32_t hi(const uint32_t* w, int m) const {
        uint32_t va;
        if (m == 15) {
            va = and_or(shr_imm<15>(w[0]), 0x00010001u, m2048);
            va = and_or(shr_imm<14>(w[1]), 0x00020002u, va);
            va = and_or(shr_imm<13>(w[2]), 0x00040004u, va);
        } else {
            const int v = m / 5, f = m % 5;
            const uint32_t x = f < 2 ? w[v] : (f < 4 ? shr_imm<6>(w[v]) : shr_imm<12>(w[v]));
            va = (f == 1 || f == 3) ? and_or(x, 0x00380038u, m256) : and_or(x, 0x00070007u, m2048);
        }
        const int p = m & 3;
        const uint32_t nm = p == 0 ? n2048 : (p == 1 ? n1024 : (p == 2 ? n512 : n256));
        const uint32_t vb = andnot_or(shift_by(w[3], 4 * (m >> 2)), 0x00010001u << p, nm);
        return bf2_fma(va, two, vb);
    }
    __device__ __forceinline__ uint32_t lo(const uint32_t* w, int m) const {
        return and_or(shift_by(w[4 + (m >> 2)], 4 * (m & 3)), 0x000F000Fu, magic);
    }
};

// The unpacker of a width class.
template <int B, bool PX>
struct Unpacker : UnpackRegs<B> {};
template <>
struct Unpacker<4, true> : UnpackPx4 {};
template <>
struct Unpacker<8, true> : UnpackPx8 {};

// Offset the unpack adds to code position c (0..31) of a quarter, which the
// task warp's offset sums remove: main format 136 (b = 4) or 132 / 20 by pair
// (b = 3); layered store, where a weight is (m / 2^b)(2 u + 1 - 2^b) =
// s (unpacked - offset) with s = m / 4, m / 8, m / 128: 131.5 / 19.5 by pair
// (b = 3), const + 7.5 (b = 4; const = 2 c_A - 2^(7-p) - 1 with c_A = 128 or
// 16 and p = pair & 3, as UnpackPx4 builds it), 16 const + 255.5 (b = 8,
// the same const, as UnpackPx8's two operands add up).
template <int B, bool PX>
__device__ __forceinline__ float code_offset(int c) {
    const int m = c >> 1;
    const bool mid = m < 15 && (m % 5 == 1 || m % 5 == 3);
    if constexpr (!PX) {
        if constexpr (B == 4) return 136.0f;
        return mid ? 20.0f : 132.0f;
    } else {
        const float cst = 2.0f * (mid ? 16.0f : 128.0f) - (float)(128 >> (m & 3)) - 1.0f;
        if constexpr (B == 8) return 16.0f * cst + 255.5f;
        if constexpr (B == 4) return cst + 7.5f;
        return mid ? 19.5f : 131.5f;
    }
}

// Layered store: a row's words of one chunk of a consumer share. The share
// holds each layer's chunks as one run (A, then B, then C), each run sized
// for the slot's J block columns; `ci` is the chunk's index in its run.
template <int B, int RUN>  // RUN: chunks per layer run of a share
__device__ __forceinline__ void load_row_words_px(const uint8_t* share, int ci, int r, int t,
                                                  uint32_t (&w)[Geo<B, 1, 1>::WORDS]) {
    const uint32_t* a = reinterpret_cast<const uint32_t*>(share + ci * 768 + r * 48 + 12 * t);
    w[0] = a[0];
    w[1] = a[1];
    w[2] = a[2];
    if constexpr (B >= 4)
        w[3] = *reinterpret_cast<const uint32_t*>(share + RUN * 768 + ci * 256 + r * 16 + 4 * t);
    if constexpr (B == 8) {
        const uint4 c =
            *reinterpret_cast<const uint4*>(share + RUN * 1024 + ci * 1024 + r * 64 + 16 * t);
        w[4] = c.x; w[5] = c.y; w[6] = c.z; w[7] = c.w;
    }
}

// Unpack and multiply one block (128 codes of 16 rows, NM matrices, NTILE
// tiles) with NT 8-token n-tiles of activations: every unpacked weight
// fragment serves all n-tiles. Widths 3 and 4 unpack to the offset form
// (k + off, see common.cuh), whose off . x term the task's offset sums remove;
// width 8 unpacks to k. One n-tile loads the block's activations up front;
// two load them half a block at a time (the same 16 registers).
template <int B, bool PX, int NM, int NT, int NTILE, int TPW>
__device__ __forceinline__ void block_mma(const Unpacker<B, PX>& U,
                                          const uint32_t (&wr)[TPW][NM][2][Geo<B, 1, 1>::WORDS],
                                          const __nv_bfloat16* const (&arow)[kMaxTiles], int j,
                                          int t, float (&acc)[TPW][kMaxTiles][NM][4]) {
    constexpr bool b8 = B == 8 && !PX;  // the main 8-bit k permutation
    constexpr int HALVES = NT == 1 ? 1 : 2;  // activation loads per block
    constexpr int CH = 8 / HALVES;           // mma steps per load
#pragma unroll
    for (int h = 0; h < HALVES; ++h) {
        uint32_t x[NT][16 / HALVES];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            if constexpr (HALVES == 1) {
                uint32_t xa[8], xz[8];
                load_act_half(arow[nt], j, t, b8, 0, xa);
                load_act_half(arow[nt], j, t, b8, 1, xz);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    x[nt][i] = xa[i];
                    x[nt][8 + i] = xz[i];
                }
            } else {
                uint32_t xh[8];
                load_act_half(arow[nt], j, t, b8, h, xh);
#pragma unroll
                for (int i = 0; i < 8; ++i) x[nt][i] = xh[i];
            }
        }
#pragma unroll
        for (int cc = 0; cc < CH; ++cc) {
            const int c = h * CH + cc;
#pragma unroll
            for (int i = 0; i < NTILE; ++i)
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    if constexpr (PX && B == 8) {  // two operands, one accumulator
                        const uint32_t a0 = U.hi(wr[i][m][0], 2 * c);
                        const uint32_t a1 = U.hi(wr[i][m][1], 2 * c);
                        const uint32_t a2 = U.hi(wr[i][m][0], 2 * c + 1);
                        const uint32_t a3 = U.hi(wr[i][m][1], 2 * c + 1);
                        const uint32_t c0 = U.lo(wr[i][m][0], 2 * c);
                        const uint32_t c1 = U.lo(wr[i][m][1], 2 * c);
                        const uint32_t c2 = U.lo(wr[i][m][0], 2 * c + 1);
                        const uint32_t c3 = U.lo(wr[i][m][1], 2 * c + 1);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            mma_bf16_16816(acc[i][nt][m], a0, a1, a2, a3, x[nt][2 * cc],
                                           x[nt][2 * cc + 1]);
                            mma_bf16_16816(acc[i][nt][m], c0, c1, c2, c3, x[nt][2 * cc],
                                           x[nt][2 * cc + 1]);
                        }
                    } else {
                        const uint32_t a0 = U.pair(wr[i][m][0], 2 * c);
                        const uint32_t a1 = U.pair(wr[i][m][1], 2 * c);
                        const uint32_t a2 = U.pair(wr[i][m][0], 2 * c + 1);
                        const uint32_t a3 = U.pair(wr[i][m][1], 2 * c + 1);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_bf16_16816(acc[i][nt][m], a0, a1, a2, a3, x[nt][2 * cc],
                                           x[nt][2 * cc + 1]);
                    }
                }
        }
    }
}

struct Task {
    int tau, p, pos0, ntok, j_hi;  // tau: the warp's first tile
    float scale;
    bool valid;   // the warp's tiles exist
};

// Finish a task. One K part (P = 1): gate/up applies SwiGLU and stores h
// (bf16); down stores y_pos = s_e acc (fp32). Several parts: the task's
// scaled partial goes to its own slice of the partial buffer -- gate/up
// gv[p][pos][m][row] = s_e acc, down y[p][pos][row] = s_e acc -- and a later
// pass sums the slices in part order (deterministic, no atomics).
template <bool GATEUP>
__device__ __forceinline__ void finish(const Args& a, const Task& T, int tau,
                                       const float (&acc)[kMaxTiles][GATEUP ? 2 : 1][4],
                                       int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int F = a.P.F, H = a.P.H;
#pragma unroll
    for (int nt = 0; nt < kMaxTiles; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int n = nt * 8 + 2 * t + (q & 1);
            if (n >= T.ntok) continue;
            const int row = tau * 16 + g + 8 * (q >> 1);
            const int pos = T.pos0 + n;
            if (GATEUP) {
                const float gv = T.scale * acc[nt][0][q];
                const float uv = T.scale * acc[nt][GATEUP ? 1 : 0][q];
                if (a.direct_h) {
                    const float hv = gv / (1.0f + __expf(-gv)) * uv;
                    a.h_out[(size_t)pos * F + row] = __float2bfloat16_rn(hv);
                } else {
                    float* dst = a.part + (size_t)T.p * a.part_stride + ((size_t)pos * 2) * F + row;
                    dst[0] = gv;
                    dst[F] = uv;
                }
            } else {
                a.y_out[(size_t)T.p * a.part_stride + (size_t)pos * H + row] =
                    T.scale * acc[nt][0][q];
            }
        }
}

struct CtaSmem {
    uint8_t* ring;
    uint64_t* full;      // per slot: 1 producer arrival + transaction bytes
    uint64_t* empty;     // per slot: one arrival per consumer warp
    uint64_t* tq_full;   // per queue entry: the task warp's arrival (task resolved)
    uint64_t* tq_sum;    // per queue entry: the task warp's arrival (offset sums written)
    uint64_t* tq_empty;  // per queue entry: the copy warp + every consumer warp
    SlotDesc* descs;
    TaskMeta* taskq;
};

__device__ __forceinline__ uint32_t next_q(uint32_t q) { return q + 1 == kTaskQ ? 0u : q + 1; }

// Task warp: claims the tasks of one width class in counter order and writes
// each, resolved, into the next free queue entry; then one end-of-class entry.
// For widths 3 and 4 (every width of the layered store) it then adds up, per
// token, off(k) x[k] over the task's K range in fp32 (the offset-form unpack
// adds off(k) to every code; the consumers subtract this sum once per task)
// and signals tq_sum. In the down
// kernel the activations come from the preceding kernel, so the first sum
// waits for it (`need_wait`). `q` and the phase bits `ph` / `used` of the
// queue's empty barriers carry over between classes.
template <int B, bool GATEUP, bool PX>
__device__ __forceinline__ bool resolve_class(const Args& a, const CtaSmem& sm, int group0,
                                              int n_groups, int32_t* ctr, uint32_t& q,
                                              uint32_t& ph, uint32_t& used, bool& need_wait) {
    const PagedExperts& P = a.P;
    const int K = GATEUP ? P.H : P.F;
    const int R = GATEUP ? P.F : P.H;
    const int nj = K / kCodesPerBlock;
    constexpr int TT = tiles_per_task(GATEUP);
    const int n_tq = (R / 16 + TT - 1) / TT;
    const int n_tasks = n_groups * n_tq * a.parts;
    const int lane = threadIdx.x & 31;
    for (;;) {
        if ((used >> q) & 1u) {
            if (!mbar_wait_bounded(&sm.tq_empty[q], (ph >> q) & 1u)) {
                if (lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
                return false;
            }
            ph ^= 1u << q;
        }
        used |= 1u << q;
        int t = 0;
        if (lane == 0 && n_tasks > 0) t = atomicAdd(ctr, 1);
        t = __shfl_sync(0xffffffffu, t, 0);
        TaskMeta* m = sm.taskq + q;
        const bool more = t < n_tasks;
        if (more) {
            int gi, tq, p;
            split_task(t, n_tq, a.parts, gi, tq, p);
            gi += group0;
            // route outputs are read through L2 (written by the preceding kernel)
            const int e = __ldcg(a.wg + 3 * gi);
            const int pos0 = __ldcg(a.wg + 3 * gi + 1);
            const int ntok = __ldcg(a.wg + 3 * gi + 2);
            if (lane < ntok)
                m->rows[lane] = GATEUP ? __ldcg(a.perm + pos0 + lane) / a.k : pos0 + lane;
            if (lane == 0) {
                m->valid = 1;
                m->tq = tq;
                m->p = p;
                m->pos0 = pos0;
                m->ntok = ntok;
                m->j0 = p * a.kb;
                m->j_hi = min(nj, p * a.kb + a.kb);
                m->scale = __ldcg(&P.pte[e].scale);
                m->first = __ldcg(&P.pte[e].first);
                if constexpr (PX) {
                    m->lfirst[0] = __ldg(a.lfirst + 2 * e);
                    m->lfirst[1] = __ldg(a.lfirst + 2 * e + 1);
                }
            }
        } else if (lane == 0) {
            m->valid = 0;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tq_full[q]);
        if (more) {
            if constexpr (B != 8 || PX) {
                if (need_wait) {
                    griddep_wait();
                    need_wait = false;
                }
                // lane l adds 8 consecutive codes per 256: positions 8 (l % 4) .. + 7
                // of a quarter. All tokens at once (loads of 8 rows in flight per
                // step), then one transposing reduction of the 16 sums.
                static_assert(kDecodeGroup == 16, "the reduction below folds 16 sums");
                float off[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) off[e] = code_offset<B, PX>(8 * (lane & 3) + e);
                const int k_lo = 128 * m->j0, k_hi = 128 * m->j_hi, ntok = m->ntok;
                float sum[kDecodeGroup];
#pragma unroll
                for (int i = 0; i < kDecodeGroup; ++i) sum[i] = 0.0f;
                for (int k = k_lo + 8 * lane; k < k_hi; k += 256) {
#pragma unroll
                    for (int h8 = 0; h8 < kDecodeGroup; h8 += 8) {
                        if (h8 >= ntok) break;
                        uint4 v[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            v[i] = h8 + i < ntok
                                       ? __ldg(reinterpret_cast<const uint4*>(
                                             a.act + (size_t)m->rows[h8 + i] * K + k))
                                       : make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint32_t wv[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float lo = __uint_as_float(wv[e] << 16);
                                const float hi = __uint_as_float(wv[e] & 0xFFFF0000u);
                                sum[h8 + i] = fmaf(off[2 * e], lo, sum[h8 + i]);
                                sum[h8 + i] = fmaf(off[2 * e + 1], hi, sum[h8 + i]);
                            }
                        }
                    }
                }
                // fold: at offset 16 a lane keeps the half of the sums its lane bit
                // 4 selects and adds its partner's copy of that half; then 8, 4, 2
                // (halving again), and 1. Lane l ends with token (l >> 1) & 15.
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const bool up = (lane & 16) != 0;
                    const float send = up ? sum[i] : sum[i + 8];
                    const float keep = up ? sum[i + 8] : sum[i];
                    sum[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool up = (lane & 8) != 0;
                    const float send = up ? sum[i] : sum[i + 4];
                    const float keep = up ? sum[i + 4] : sum[i];
                    sum[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const bool up = (lane & 4) != 0;
                    const float send = up ? sum[i] : sum[i + 2];
                    const float keep = up ? sum[i + 2] : sum[i];
                    sum[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                }
                {
                    const bool up = (lane & 2) != 0;
                    const float send = up ? sum[0] : sum[1];
                    const float keep = up ? sum[1] : sum[0];
                    sum[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                }
                sum[0] += __shfl_xor_sync(0xffffffffu, sum[0], 1);
                const int tok = (lane >> 1) & 15;
                if ((lane & 1) == 0 && tok < ntok) m->offsum[tok] = sum[0];
                __syncwarp();
            }
            if (lane == 0) mbar_arrive(&sm.tq_sum[q]);
        }
        q = next_q(q);
        if (!more) return true;
    }
}

// Copy warp: every task of one width class, from the queue. Lane w owns the
// copy stream of consumer w's share of the task (a page cursor in registers,
// the next page's index loaded ahead): per slot one run of NM x TPW x jc
// chunks (gate/up: W1 and W3 of the tile alternate; down: the share's two
// tiles alternate). Lane 0 arms the full barriers and writes the slot descriptors;
// every lane prefetches one activation line. `ep` / `used` track the slots'
// empty-barrier phases across classes, `fph` the queue's full-barrier phases.
// In the down kernel the activations (h) come from the preceding kernel, so
// the warp waits for it (`need_wait`) before its first prefetch. The layered
// store copies each layer's run of the share from that layer's pages (the
// runs sit one after another in the share: A, B, C).
template <int B, bool GATEUP, bool PX>
__device__ __forceinline__ bool produce_class(const Args& a, const CtaSmem& sm, uint32_t& q,
                                              uint32_t& fph, uint32_t& ep, uint32_t& used,
                                              bool& need_wait) {
    constexpr int NM = GATEUP ? 2 : 1;
    constexpr int TT = tiles_per_task(GATEUP);
    using G = Geo<B, NM, tiles_per_warp(GATEUP)>;
    constexpr int S = G::S;
    const PagedExperts& P = a.P;
    const int K = GATEUP ? P.H : P.F;
    const int R = GATEUP ? P.F : P.H;
    const int nj = K / kCodesPerBlock, n_tiles = R / 16;
    const int nc1 = chunks_w1(P.H, P.F);
    constexpr int TPW = tiles_per_warp(GATEUP);
    // layers of the class (one for the main format) and their geometry
    constexpr int NL = PX ? (B == 3 ? 1 : (B == 4 ? 2 : 3)) : 1;
    int lcb[NL], lcpp[NL], lnp[NL], lrun[NL];
#pragma unroll
    for (int L = 0; L < NL; ++L) {
        const int lb = PX ? (L == 0 ? 3 : (L == 1 ? 1 : 4)) : B;
        lcb[L] = 256 * lb;
        lcpp[L] = chunks_per_page(lb, P.page_bytes);
        lnp[L] = (3 * nc1 + lcpp[L] - 1) / lcpp[L];
        // the run's offset in a share: the runs before it, J columns each
        lrun[L] = L == 0 ? 0 : (L == 1 ? TPW * NM * G::J * 768 : TPW * NM * G::J * 1024);
    }
    const int lane = threadIdx.x & 31;
    const bool copier = lane < kConsumers;  // lane w copies consumer w's share

    auto acquire = [&](int s) -> bool {
        if ((used >> s) & 1u) {
            if (!mbar_wait_bounded(&sm.empty[s], (ep >> s) & 1u)) {
                if (lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
                return false;
            }
            ep ^= 1u << s;
        }
        used |= 1u << s;
        return true;
    };

    int s = 0;
    for (;;) {
        if (!mbar_wait_bounded(&sm.tq_full[q], (fph >> q) & 1u)) {
            if (lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
            return false;
        }
        fph ^= 1u << q;
        const TaskMeta* m = sm.taskq + q;
        const int valid = m->valid;
        int tq = 0, j = 0, j_hi = 0;
        uint32_t first[NL];
        const __nv_bfloat16* pre_row = nullptr;  // this lane's activation row to prefetch
        if (valid) {
            tq = m->tq;
            j = m->j0;
            j_hi = m->j_hi;
            first[0] = m->first;
#pragma unroll
            for (int L = 1; L < NL; ++L) first[L] = m->lfirst[L - 1];
            if ((lane >> 1) < m->ntok) pre_row = a.act + (size_t)m->rows[lane >> 1] * K;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tq_empty[q]);
        const uint32_t mq = q;
        q = next_q(q);
        if (!valid) {  // end of the class: a terminator slot names the queue entry
            if (!acquire(s)) return false;
            if (lane == 0) {
                sm.descs[s] = SlotDesc{-1, (int)mq, 0, 0};
                mbar_arrive(&sm.full[s]);
            }
            __syncwarp();
            return true;
        }
        const int active = min(TT, n_tiles - tq * TT);  // tiles (a multiple of TPW)
        const bool my_tile = copier && lane * TPW < active;
        int pslot[NL], poff[NL];
        uint32_t page[NL], page_next[NL];
#pragma unroll
        for (int L = 0; L < NL; ++L) {
            pslot[L] = poff[L] = 0;
            page[L] = page_next[L] = 0;
        }
        if (my_tile) {
            // the share's first chunk: gate/up interleaves W1 and W3 of a tile,
            // down the two tiles (2v, 2v+1) of the share: two chunks a column
            // (the same index in every layer)
            const int tau = tq * TT + lane * TPW;
            const int c = GATEUP ? 2 * (tau * nj + j) : 2 * nc1 + 2 * ((tau >> 1) * nj + j);
#pragma unroll
            for (int L = 0; L < NL; ++L) {
                pslot[L] = c / lcpp[L];
                poff[L] = c - pslot[L] * lcpp[L];
                page[L] = __ldcg(P.pidx + first[L] + pslot[L]);
                if (pslot[L] + 1 < lnp[L]) page_next[L] = __ldcg(P.pidx + first[L] + pslot[L] + 1);
            }
        }
        const int jstart = j;
        const int pre_half = lane & 1;
        while (j < j_hi) {
            if (!acquire(s)) return false;
            const int jc = min(G::J, j_hi - j);  // block columns in this slot
            if (lane == 0) {
                sm.descs[s] = SlotDesc{(int)mq, j, jc,
                                       (j == jstart ? kFirstSlot : 0) |
                                           (j + jc >= j_hi ? kLastSlot : 0)};
                mbar_arrive_expect_tx(&sm.full[s], (uint32_t)(active * NM * jc * G::CB));
            }
            __syncwarp();
            if (my_tile) {
                // the share's NM x TPW x jc consecutive chunks (two a block
                // column) of each layer; a page boundary splits a copy in two
                uint8_t* share = sm.ring + (size_t)s * G::SLOT + (size_t)lane * TPW * G::TILEB;
                const int total = NM * TPW * jc;
#pragma unroll
                for (int L = 0; L < NL; ++L) {
                    uint8_t* dst = share + lrun[L];
                    const int n1 = min(total, lcpp[L] - poff[L]);
                    bulk_g2s(dst, P.pool + (size_t)page[L] * P.page_bytes + (size_t)poff[L] * lcb[L],
                             (uint32_t)(n1 * lcb[L]), &sm.full[s]);
                    poff[L] += n1;
                    if (poff[L] == lcpp[L]) {
                        ++pslot[L];
                        poff[L] = 0;
                        page[L] = page_next[L];
                        if (pslot[L] + 1 < lnp[L])
                            page_next[L] = __ldcg(P.pidx + first[L] + pslot[L] + 1);
                    }
                    if (n1 < total) {
                        bulk_g2s(dst + n1 * lcb[L], P.pool + (size_t)page[L] * P.page_bytes,
                                 (uint32_t)((total - n1) * lcb[L]), &sm.full[s]);
                        poff[L] = total - n1;
                    }
                }
            }
            if (need_wait) {
                griddep_wait();
                need_wait = false;
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
}

// Consumer warp w: all tasks of one width class, tiles w * TPW .. of each
// task. `fp` tracks the slots' full-barrier phases across classes, `sph` the
// queue's offset-sum barrier phases. A warp holds its task's queue entry until
// the task's last slot, where it reads the offset sums.
template <int B, bool GATEUP, bool PX>
__device__ __forceinline__ bool consume_class(const Args& a, const CtaSmem& sm, uint32_t& fp,
                                              uint32_t& sph, int w) {
    constexpr int NM = GATEUP ? 2 : 1;
    constexpr int TPW = tiles_per_warp(GATEUP);
    using G = Geo<B, NM, TPW>;
    constexpr int S = G::S;
    const PagedExperts& P = a.P;
    const int K = GATEUP ? P.H : P.F;
    const int R = GATEUP ? P.F : P.H;
    const int n_tiles = R / 16;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;

    Task T{};
    const __nv_bfloat16* arow[kMaxTiles] = {};
    int ntiles = 0;
    float acc[TPW][kMaxTiles][NM][4];
    const Unpacker<B, PX> U;
    // widths 3, 4: acc <- acc - off . x for every tile and matrix, with the
    // task warp's per-token sums (accumulator column n = token n)
    auto settle = [&](const TaskMeta* m) {
        if constexpr (B != 8 || PX) {
            const int t = lane & 3;
#pragma unroll
            for (int nt = 0; nt < kMaxTiles; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = nt * 8 + 2 * t + h;
                    const float o = n < T.ntok ? m->offsum[n] : 0.0f;
#pragma unroll
                    for (int i = 0; i < TPW; ++i)
#pragma unroll
                        for (int mm = 0; mm < NM; ++mm) {
                            acc[i][nt][mm][h] -= o;
                            acc[i][nt][mm][h + 2] -= o;
                        }
                }
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
        if (d.q < 0) {  // end of the class
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.tq_empty[d.j]);
                mbar_arrive(&sm.empty[s]);
            }
            return true;
        }
        // the task's last slot: offset sums, finish, release the queue entry
        auto close_task = [&]() -> bool {
            const uint32_t sp = (sph >> d.q) & 1u;
            sph ^= 1u << d.q;
            const TaskMeta* m = sm.taskq + d.q;
            if (T.valid) {
                if constexpr (B != 8 || PX) {
                    if (!mbar_wait_bounded(&sm.tq_sum[d.q], sp)) {
                        if (lane == 0) set_status(a.status, MPE_STATUS_WAIT_TIMEOUT);
                        return false;
                    }
                    settle(m);
                }
                finish<GATEUP>(a, T, T.tau, acc[0], lane);
                if constexpr (TPW > 1) finish<GATEUP>(a, T, T.tau + 1, acc[1], lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tq_empty[d.q]);
            return true;
        };
        if (d.flags & kFirstSlot) {
            const TaskMeta* m = sm.taskq + d.q;
            T.tau = m->tq * tiles_per_task(GATEUP) + w * TPW;
            // a task's tile count is even (H and F are multiples of 128), so a
            // down warp with a first tile also has its second
            T.valid = T.tau < n_tiles;
            T.p = m->p;
            T.pos0 = m->pos0;
            T.ntok = m->ntok;
            T.j_hi = m->j_hi;
            T.scale = m->scale;
            ntiles = (T.ntok + 7) / 8;
#pragma unroll
            for (int nt = 0; nt < kMaxTiles; ++nt) {
                const int n = nt * 8 + g;
                arow[nt] = n < T.ntok ? a.act + (size_t)m->rows[n] * K : nullptr;
#pragma unroll
                for (int i = 0; i < TPW; ++i)
#pragma unroll
                    for (int mm = 0; mm < NM; ++mm)
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[i][nt][mm][q] = 0.0f;
            }
        }
        if (!T.valid) {  // this warp has no tile in the task: release at once
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
            if ((d.flags & kLastSlot) && !close_task()) return false;
            continue;
        }
        const int t = lane & 3;
        const uint8_t* tiles = sm.ring + (size_t)s * G::SLOT + (size_t)w * TPW * G::TILEB;
        // the block columns of a slot stay a loop: each block is a large
        // unrolled body, and the code for one width class has to stay in the
        // instruction cache (with this loop unrolled, 16-token groups cost the
        // Mixtral-shaped layer 5 %; rolled, they cost nothing)
#pragma unroll 1
        for (int jj = 0; jj < G::J; ++jj) {
            if (jj >= d.nc) break;
            uint32_t wr[TPW][NM][2][G::WORDS];
#pragma unroll
            for (int i = 0; i < TPW; ++i) {
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    const int ci = (jj * TPW + i) * NM + m;  // chunk of the share
                    if constexpr (PX) {
                        constexpr int RUN = TPW * NM * G::J;
                        load_row_words_px<B, RUN>(tiles, ci, g, t, wr[i][m][0]);
                        load_row_words_px<B, RUN>(tiles, ci, g + 8, t, wr[i][m][1]);
                    } else {
                        const uint8_t* chunk = tiles + ci * G::CB;
                        load_row_words<B>(chunk, g, t, g, wr[i][m][0]);
                        load_row_words<B>(chunk, g + 8, t, g, wr[i][m][1]);
                    }
                }
            }
            if (jj + 1 == d.nc) {  // the slot's last words are in registers: release it
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);
            }
            const int j = d.j + jj;
            // one instantiation per n-tile count that can occur: the unrolled
            // block is large, and duplicates cost instruction fetch
            if constexpr (kMaxTiles > 1) {
                if (ntiles > 1) {
                    block_mma<B, PX, NM, kMaxTiles, TPW, TPW>(U, wr, arow, j, t, acc);
                    continue;
                }
            }
            block_mma<B, PX, NM, 1, TPW, TPW>(U, wr, arow, j, t, acc);
        }
        if ((d.flags & kLastSlot) && !close_task()) return false;
    }
}

template <bool GATEUP, bool PX>
__global__ void __launch_bounds__(kThreads, 1) k_decode(Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    CtaSmem sm;
    sm.ring = smem;
    sm.full = reinterpret_cast<uint64_t*>(smem + kBarOff);
    sm.empty = sm.full + kMaxSlots;
    sm.tq_full = sm.empty + kMaxSlots;
    sm.tq_sum = sm.tq_full + kTaskQ;
    sm.tq_empty = sm.tq_sum + kTaskQ;
    sm.descs = reinterpret_cast<SlotDesc*>(smem + kDescOff);
    sm.taskq = reinterpret_cast<TaskMeta*>(smem + kTaskOff);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxSlots; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kConsumers);
        }
        for (int q = 0; q < kTaskQ; ++q) {
            mbar_init(&sm.tq_full[q], 1);
            mbar_init(&sm.tq_sum[q], 1);
            mbar_init(&sm.tq_empty[q], kConsumers + 1);
        }
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();
    if (warp == kTaskWarp) {
        // gate/up: the work groups and task counters come from the route kernel
        // just before; down: that kernel finished before the one that precedes
        // this launch let it start (the offset sums over h wait for it)
        if (GATEUP) griddep_wait();
        if (lane == 0) griddep_launch_dependents();
        const int n8 = __ldcg(a.n_wg_class), n4 = __ldcg(a.n_wg_class + 1),
                  n3 = __ldcg(a.n_wg_class + 2);
        uint32_t q = 0, ph = 0, used = 0;
        bool need_wait = !GATEUP;
        if (!resolve_class<8, GATEUP, PX>(a, sm, 0, n8, a.task_ctr + 0, q, ph, used, need_wait)) return;
        if (!resolve_class<4, GATEUP, PX>(a, sm, n8, n4, a.task_ctr + 1, q, ph, used, need_wait)) return;
        resolve_class<3, GATEUP, PX>(a, sm, n8 + n4, n3, a.task_ctr + 2, q, ph, used, need_wait);
    } else if (warp == kCopyWarp) {
        uint32_t q = 0, fph = 0, ep = 0, used = 0;
        bool need_wait = !GATEUP;
        if (!produce_class<8, GATEUP, PX>(a, sm, q, fph, ep, used, need_wait)) return;
        if (!produce_class<4, GATEUP, PX>(a, sm, q, fph, ep, used, need_wait)) return;
        produce_class<3, GATEUP, PX>(a, sm, q, fph, ep, used, need_wait);
    } else {
        // down: h is written by the preceding kernel
        if (!GATEUP) griddep_wait();
        uint32_t fp = 0, sph = 0;
        if (!consume_class<8, GATEUP, PX>(a, sm, fp, sph, warp)) return;
        if (!consume_class<4, GATEUP, PX>(a, sm, fp, sph, warp)) return;
        consume_class<3, GATEUP, PX>(a, sm, fp, sph, warp);
    }
}

int g_num_sms = 0;

}  // namespace

void decode_set_smem_limits() {
    cudaFuncSetAttribute(k_decode<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes());
    cudaFuncSetAttribute(k_decode<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes());
    cudaFuncSetAttribute(k_decode<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes());
    cudaFuncSetAttribute(k_decode<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes());
}

// K parts per task: enough CTA tasks that every CTA of the persistent grid gets
// about `per_cta` of them, at least 4 blocks per part.
int decode_parts(int est_groups, int n_tq, int nj, int total_ctas, int per_cta, int min_kb) {
    const long target = (long)per_cta * total_ctas;
    int P = 1;
    const int pmax = max(1, nj / min_kb);
    while (P < pmax && (long)est_groups * n_tq * P < target) ++P;
    return P;
}

static int env_int(const char* name, int dflt) {
    const char* v = getenv(name);
    return v ? atoi(v) : dflt;
}

void decode_plan(mpe_ctx* c, size_t Tk, DecodePlan& pl) {
    if (!g_num_sms) cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, c->device);
    const int ctas = g_num_sms;
    const int groups = (int)std::min<size_t>((size_t)c->E, Tk);
    // tasks per CTA (measured best: gate/up 6, down 8); tuning overrides
    const int pc_env = env_int("MPE_DECODE_TASKS_PER_CTA", 0);
    const int pc_gu_env = env_int("MPE_DECODE_TASKS_PER_CTA_GATEUP", 0);
    const int pc_dn_env = env_int("MPE_DECODE_TASKS_PER_CTA_DOWN", 0);
    const int pc_gu = pc_gu_env > 0 ? pc_gu_env : (pc_env > 0 ? pc_env : 6);
    const int pc_dn = pc_dn_env > 0 ? pc_dn_env : (pc_env > 0 ? pc_env : 8);
    // at least this many block columns per K part (a part's fixed costs)
    const int min_kb_gu = std::max(1, env_int("MPE_DECODE_MIN_KB_GATEUP", 4));
    const int min_kb_dn = std::max(1, env_int("MPE_DECODE_MIN_KB_DOWN", 4));
    pl.claim = 1;
    const int nj_gu = c->H / kCodesPerBlock, nj_dn = c->F / kCodesPerBlock;
    const int tt_gu = tiles_per_task(true), tt_dn = tiles_per_task(false);
    int p = decode_parts(groups, (c->F / 16 + tt_gu - 1) / tt_gu, nj_gu, ctas, pc_gu, min_kb_gu);
    pl.kb_gu = (nj_gu + p - 1) / p;
    pl.p_gu = (nj_gu + pl.kb_gu - 1) / pl.kb_gu;
    p = decode_parts(groups, (c->H / 16 + tt_dn - 1) / tt_dn, nj_dn, ctas, pc_dn, min_kb_dn);
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
                          int kb, int claim, bool partials) {
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
    a.direct_h = (parts == 1 && !partials) ? 1 : 0;
    a.kb = kb;
    a.status = c->d_status;
    a.lfirst = c->px_lfirst;
    auto* fn = c->px_lfirst ? k_decode<true, true> : k_decode<true, false>;
    const int grid = persistent_grid(c, (const void*)fn, smem_bytes());
    launch_pdl(fn, dim3(grid), dim3(kThreads), smem_bytes(), c->stream, a);
    c->launches++;
}

void launch_decode_down(mpe_ctx* c, size_t Tk, int parts, int kb, int claim) {
    (void)claim;
    Args a{};
    a.P = paged(c);
    a.wg = c->s.wg;
    a.n_wg_class = c->s.n_wg + 1;
    a.perm = c->s.perm;
    a.k = 1;
    a.act = c->s.h;
    a.y_out = c->s.y;
    a.part = c->s.part;
    a.part_stride = (size_t)Tk * c->H;
    a.task_ctr = c->s.task_ctr + 3;
    a.parts = parts;
    a.kb = kb;
    a.status = c->d_status;
    a.lfirst = c->px_lfirst;
    auto* fn = c->px_lfirst ? k_decode<false, true> : k_decode<false, false>;
    const int grid = persistent_grid(c, (const void*)fn, smem_bytes());
    launch_pdl(fn, dim3(grid), dim3(kThreads), smem_bytes(), c->stream, a);
    c->launches++;
}

}  // namespace mpe
