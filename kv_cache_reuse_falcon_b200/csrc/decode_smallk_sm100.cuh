// Rank decode for small candidate counts (k <= 64 per request), sm_100a.
//
// The rank decode of [review] §2.4 / [notes] §6: the k candidates of request r
// attend to pool rows 0..n_r-1 of slot s_r (layer l, head h) and to
// themselves.  With few candidates a request is a stream of cached K/V rows
// read once against a handful of queries, so the pass is bound by HBM, not by
// the tensor cores.  This kernel therefore puts the KEYS on the MMA's M
// dimension, so no tensor-core row and no softmax thread is spent on padding
// candidates:
//
//   S^T = K Q^T   M = 128 keys, N = k padded to 16/32/64, K = D
//   O  += P V     M = 64 candidate rows for N <= 32, else 128 (rows past the
//                 padded count are discarded), N = D, K = 128 keys; P (bf16) is
//                 staged through shared memory in the 128-byte-swizzled K-major
//                 layout of a query tile, V is read MN-major as the prefill
//                 reads it.  An M = 64 product reads half the P operand; its
//                 row r sits in TMEM lane 32 (r / 16) + r % 16
//
// Softmax thread t owns key t of a tile (TMEM lane t): it loads that key's N
// scores, and the per-candidate statistics are reductions over threads.  The
// reference maximum of each candidate moves only when some score would
// exceed it by more than 2^8 (one vote per tile among the four softmax warps;
// the exact column maxima are computed only then), so the common tile costs
// N scalings, N exponentials, N two-byte stores of P and one warp
// reduce-scatter of the column sums.  O accumulates in TMEM with one lane per
// candidate row, so the epilogue thread of candidate c reads its own row.
//
// Work: the 128-key tiles of all (request, key/value head) pairs, pair-major
// (tpp tiles per pair, from the pool's capacity), are cut into one contiguous
// range per block, so every block gets the same number of tiles (handing out
// more, smaller ranges from a counter measured slower: each extra piece costs
// an epilogue).  A block's range falls into one or more pieces (pair, tile
// run); each piece is an item.
// A pair covered by one piece writes its output directly; otherwise each piece
// leaves an unnormalised partial (O, m, l) per candidate in the caller's
// workspace, and the last piece of the pair to finish - found with a per-pair
// arrival counter - merges the partials with the candidate's own key (self
// term) and writes the output.
//
// Warp roles (256 threads; two blocks per SM where shared memory and TMEM
// allow):
//   warps 0-1  epilogue: the own scores, the final O rows (from the TMEM
//              lanes of the candidate rows), partials, arrival counter and merge
//   warp 2     TMA producer: walks the block's items, loads Q (N candidate rows), and
//              drives two streams into the ring - K tiles (a slot refills as
//              soon as its S MMA is done) and V tiles (once its P.V is done)
//   warp 3     MMA issuer (one elected thread), owns TMEM: issues S^T as K
//              lands (up to four S buffers ahead of the softmax) and P.V as P
//              is written, each as its inputs arrive
//   warps 4-7  softmax (thread t: key t of a tile, TMEM lane t); the four
//              warps vote with one named-barrier reduction per tile
// O has two TMEM buffers and the softmax hands each item's statistics (m, l)
// to the epilogue through a two-entry buffer, so the key stream of the next
// item runs while the epilogue of the last one waits on its stores and its
// arrival counter: the ring does not stall at item boundaries.
// Over an E4M3 pool (kE4M3) TMA brings each tile's codes into a staging ring
// instead, and the producer and the two epilogue warps each expand a third of
// every K and V tile into the ring's bfloat16 layout (see sk_expand_e4m3); the
// epilogue warps expand while they wait.
// Every mbarrier wait is bounded (see sm100_ptx.cuh); a block that gives up
// reports UNIPIN_ERR_DEVICE_TIMEOUT and exits cleanly.  The softmax warps
// leave their loop only together, on a named-barrier reduction, so none is
// left waiting at such a barrier.
#pragma once

#include "kvpool_sm100.cuh"
#include "sm100_ptx.cuh"
#include "tmem_wide.cuh"
#include "unipin.h"

namespace unipin {

constexpr int kSkKeys = 128;        // keys per tile (the MMA's M)
constexpr int kSkThreads = 256;
constexpr int kSkEpiWarps = 2;      // warps 0-1
constexpr int kSkProducerWarp = 2;
constexpr int kSkMmaWarp = 3;
constexpr int kSkSoftmaxWarp0 = 4;  // warps 4-7
constexpr int kSkItemSlots = 4;
constexpr int kSkConsumers = 7;     // the MMA warp, the four softmax and the two epilogue warps pop every item
constexpr int kSkMaxSplit = 16;     // key splits per (request, head) at most
constexpr float kSkRescaleLog2 = 8.0f;

// Candidate columns the kernel is compiled for, given the largest k.
__host__ __device__ constexpr int sk_pad_n(int k) { return k <= 16 ? 16 : k <= 32 ? 32 : 64; }
__host__ __device__ constexpr int sk_tmem_cols(int c) { return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512; }

// kE4M3: the pool holds E4M3 codes; TMA brings each key tile's K and V codes
// into a staging ring and the producer warp expands them into the bfloat16
// ring stages the MMAs read (the same layout TMA writes for a bfloat16 pool).
template <int D, int N, bool kE4M3 = false>
struct SkCfg {
    static_assert(D == 64 || D == 128, "small-k decode: head dim 64 or 128");
    static_assert(N == 16 || N == 32 || N == 64, "small-k decode: padded candidate count");
    static_assert(N <= kSkEpiWarps * 32, "small-k decode: one epilogue thread per candidate column");
    static constexpr int kChunks = D / 64;                 // 64-element boxes across D
    static constexpr int kAtom = kSkKeys * 128;            // 128 rows of 128 bytes (one swizzle block column)
    static constexpr int kTileKV = kChunks * kAtom;        // one K or V tile
    static constexpr int kStageBytes = 2 * kTileKV;        // V tile, then K tile
    static constexpr int kAtomQ = N * 128;                 // N candidate rows of one 64-element box
    static constexpr int kQBytes = kChunks * kAtomQ;
    // P: N candidate rows x 128 keys bf16, two 64-key boxes of N rows x 128 bytes.
    // The P.V MMA reads 128 rows from each box base; rows N..127 fall on
    // whatever follows in shared memory and give discarded output rows.
    static constexpr int kPBox = N * 128;
    static constexpr int kPBytes = 2 * kPBox;
    static constexpr bool kPv64 = N <= 32;                 // P.V with M = 64 (rows 0..63 of P)
    static constexpr int kPvRows = kPv64 ? 64 : 128;
    // TMEM columns: kSBufs S^T buffers of N columns from 0 (four where they fit
    // beside two O buffers in the block's share, so that S runs well ahead of
    // the softmax), then two O buffers of D columns.
    static constexpr int kSBufs = (D == 64 ? sk_tmem_cols(4 * N + 2 * D) <= 256 : sk_tmem_cols(4 * N + 2 * D) <= 512) ? 4 : 2;
    static constexpr int kColO = kSBufs * N;
    static constexpr int kTmemCols = sk_tmem_cols(kSBufs * N + 2 * D);
    static_assert(kTmemCols <= 512, "small-k decode: TMEM columns");
    // Scratch floats: softmax red[4][N], mref[N], corr[N]; hand-off hand_m[2][N],
    // hand_l[2][N]; epilogue coef_b[N], wts[kSkMaxSplit][N], last[4].
    static constexpr int kScratchFloats = 4 * N + 2 * N + 4 * N + N + kSkMaxSplit * N + 4;
    static constexpr int kScratchBytes = (kScratchFloats * 4 + 1023) / 1024 * 1024;
    static constexpr int kBarBytes = 1024;
    static constexpr int kTile8 = kSkKeys * D;             // E4M3 codes of one K or V tile (rows of D bytes)
    static constexpr int kStage8 = 2 * kTile8;             // K codes, then V codes
    // two blocks per SM: 2 x (113 KB + the 1 KB the runtime keeps per block) = 228 KB
    static constexpr int budget_for(int ctas) { return ctas == 2 ? 113 * 1024 : 226 * 1024; }
    // Q is double-buffered (the next item's Q loads during this item); P is
    // double-buffered (the softmax writes P_{i+1} while P.V of tile i runs)
    // unless a single buffer buys one more ring stage, since the ring depth sets
    // the bytes in flight.
    static constexpr int fixed_bytes(int pbufs, int stages8)
    {
        return 2 * kQBytes + pbufs * kPBytes + kScratchBytes + kBarBytes + stages8 * kStage8;
    }
    static constexpr int stages_for(int ctas, int pbufs, int stages8)
    {
        return (budget_for(ctas) - fixed_bytes(pbufs, stages8)) / kStageBytes;
    }
    // E4M3 staging: two stages where two bfloat16 stages still fit, else one
    static constexpr int stages8_for(int ctas) { return !kE4M3 ? 0 : (stages_for(ctas, 1, 2) >= 2 ? 2 : 1); }
    static constexpr int kCtasPerSm =
        (D == 64 && kTmemCols <= 256 && stages_for(2, 1, stages8_for(2)) >= 2) ? 2 : 1;
    static constexpr int kBudget = budget_for(kCtasPerSm);
    static constexpr int kStages8 = stages8_for(kCtasPerSm);
    static constexpr int kQBufs = 2;
    static constexpr int kPBufs = stages_for(kCtasPerSm, 1, kStages8) > stages_for(kCtasPerSm, 2, kStages8) ? 1 : 2;
    static constexpr int kStagesFit = stages_for(kCtasPerSm, kPBufs, kStages8);
    static constexpr int kStages = kStagesFit > 6 ? 6 : kStagesFit;
    static_assert(kStages >= 2, "small-k decode: ring depth");
    static_assert(kPBufs <= 2, "small-k decode: the barrier layout holds two P buffers");
    static constexpr int kOffP = 0;                                  // first: the 128-row reads overhang
    static constexpr int kOffRing = kPBufs * kPBytes;                // into the ring that follows
    static constexpr int kOffQ = kOffRing + kStages * kStageBytes;
    static constexpr int kOffStage8 = kOffQ + kQBufs * kQBytes;     // E4M3 staging ring
    static constexpr int kOffScratch = kOffStage8 + kStages8 * kStage8;
    static constexpr int kOffBar = kOffScratch + kScratchBytes;
    static constexpr int kSmemBytes = kOffBar + kBarBytes;
    static_assert(kSmemBytes <= kBudget, "small-k decode: shared memory budget");
    static_assert(kSkMaxSplit * N * 4 <= kPBytes, "merge weights fit a P buffer");
    static_assert((kPBufs - 1) * kPBytes + kPBox + kPvRows * 128 <= kSmemBytes, "P box reads stay in shared memory");
};

struct SkE4M3Mul {
    uint32_t c1, c2;   // bfloat16x2 factors: the first product, then the second (c2 = 0: none)
};

struct SkParams {
    const __nv_bfloat16* q;        // [T, H, D] candidate queries
    const __nv_bfloat16* k_self;   // [T, H, D] candidate keys (self term)
    const __nv_bfloat16* v_self;   // [T, H, D] candidate values (self term)
    void* out;                     // [T, H, D] fp32 or bf16
    float* part_o;                 // [nsplit, T, H, D] unnormalised partial O (nsplit > 1)
    float* part_ml;                // [nsplit, T, H, 2] (m in log2 units, l)
    unsigned* pair_cnt;            // [R * H] arrival counters, zeroed before the launch (nsplit > 1)
    const int* cu;                 // [R + 1]
    const int* past;               // [R]
    const int* slots;              // [R]
    int R, H;                      // requests, query heads
    int G;                         // query heads per key/value head
    int total_rows;                // T
    int out_fp32;
    int layer, S, n_cap;
    int nsplit;                    // partial slots per pair: the most pieces any pair has
    int tpp;                       // key tiles per pair
    long long total_tiles;         // pairs * tpp
    int nranges;                   // contiguous tile ranges, one per block
    float sl2;                     // scale * log2(e)
    int* status;
    unsigned long long wait_limit_ns;
    unsigned poll_ns;              // back-off of the polling producer and MMA warps when nothing is ready
    float k_scale, v_scale;        // E4M3 pool: code c stands for value(c) * scale
    SkE4M3Mul k_mul, v_mul;        // the same scales as bfloat16 factors (see SkE4M3Mul)
};

// What every role derives identically from an item index.  An item is a
// (request, key/value head, run of key tiles); its candidate columns are the
// pairs (candidate c, query head g of the group) in the order n = c * G + g.
struct SkWork {
    bool rows_ok;   // the request's candidate rows are addressable (cu in range, k * G <= N)
    bool valid;     // rows_ok and slot / history length in range
    int r, h, split, pair;   // h: the key/value head; split: the piece's index among its pair's
    int npieces;             // pieces that cover the pair
    int tok0, kc, npast, slot;
    int ncol;                // valid candidate columns, kc * G
    int nt_all;     // key tiles covering [0, npast)
    int t_begin, nt;
};

// Range b is tiles [b T / B, (b + 1) T / B) (B ranges); the range holding tile x.
__device__ __forceinline__ long long sk_range_start(const SkParams& p, long long b)
{
    return b * p.total_tiles / p.nranges;
}
__device__ __forceinline__ long long sk_block_of(const SkParams& p, long long x)
{
    return ((x + 1) * p.nranges - 1) / p.total_tiles;
}

// Item g = (range g >> 20, its piece g & 0xFFFFF).  Whether the piece exists.
__device__ __forceinline__ bool sk_piece_exists(const SkParams& p, long long g)
{
    const long long b = g >> 20;
    const long long pair = sk_range_start(p, b) / p.tpp + (g & 0xFFFFF);
    return pair * p.tpp < sk_range_start(p, b + 1);
}

template <int N>
__device__ __forceinline__ SkWork sk_make_work(const SkParams& p, long long g)
{
    SkWork w;
    const long long b = g >> 20;
    const long long s0 = sk_range_start(p, b), s1 = sk_range_start(p, b + 1);
    const long long pair = s0 / p.tpp + (g & 0xFFFFF);
    const long long p0 = pair * p.tpp;
    const long long lo = s0 > p0 ? s0 : p0;
    const long long hi = s1 < p0 + p.tpp ? s1 : p0 + p.tpp;
    const long long first = sk_block_of(p, p0), last = sk_block_of(p, p0 + p.tpp - 1);
    w.pair = (int)pair;
    w.split = (int)(b - first);
    w.npieces = (int)(last - first + 1);
    const int hkv = p.H / p.G;
    w.r = w.pair / hkv;
    w.h = w.pair - w.r * hkv;
    w.tok0 = p.cu[w.r];
    w.kc = p.cu[w.r + 1] - w.tok0;
    w.npast = p.past[w.r];
    w.slot = p.slots[w.r];
    w.ncol = w.kc * p.G;
    w.rows_ok = w.tok0 >= 0 && w.kc >= 0 && w.ncol <= N && (long long)w.tok0 + w.kc <= (long long)p.total_rows;
    w.valid = w.rows_ok && w.slot >= 0 && w.slot < p.S && w.npast >= 0 && w.npast <= p.n_cap;
    w.nt_all = w.valid ? (w.npast + kSkKeys - 1) / kSkKeys : 0;
    const int t0 = (int)(lo - p0), t1 = (int)(hi - p0);
    w.t_begin = min(t0, w.nt_all);
    const int t_end = min(t1, w.nt_all);
    w.nt = (w.valid && w.kc > 0) ? max(t_end - w.t_begin, 0) : 0;
    return w;
}

// Key tile t covers keys [lo, min(lo + 128, npast)); the last tile of a
// ragged history is loaded right-aligned so that no row at or beyond npast is
// read (rows before 0 come back as zeros); keys below lo are masked.
__device__ __forceinline__ int sk_tile_start(int t, int nt_all, int npast)
{
    const int lo = t * kSkKeys;
    return (t == nt_all - 1 && (npast % kSkKeys) != 0) ? npast - kSkKeys : lo;
}

// Warp reduce-scatter over the 32 lanes of N per-lane values (max or sum).
// Afterwards v[e], e < max(N/32, 1), holds the reduction of column
// sk_owned_col<N>(lane, e): lane*(N/32) + e for N >= 32, lane/2 for N = 16.
template <int n, int o, bool kMax>
__device__ __forceinline__ void sk_rs_step(float* v, int lane)
{
    if constexpr (o >= 1) {
        if constexpr (n > 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int e = 0; e < n / 2; ++e) {
                const float keep = upper ? v[e + n / 2] : v[e];
                const float give = upper ? v[e] : v[e + n / 2];
                const float got = __shfl_xor_sync(0xffffffffu, give, o);
                v[e] = kMax ? fmaxf(keep, got) : keep + got;
            }
            sk_rs_step<n / 2, o / 2, kMax>(v, lane);
        } else {
            const float got = __shfl_xor_sync(0xffffffffu, v[0], o);
            v[0] = kMax ? fmaxf(v[0], got) : v[0] + got;
            sk_rs_step<1, o / 2, kMax>(v, lane);
        }
    }
}

template <int N>
__device__ __forceinline__ int sk_owned_col(int lane, int e)
{
    return N >= 32 ? lane * (N / 32) + e : (lane >> 1);
}

template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&r)[N])
{
    if constexpr (N == 16) tmem_ld16(taddr, r);
    else if constexpr (N == 32) tmem_ld32(taddr, r);
    else if constexpr (N == 64) tmem_ld64(taddr, r);
    else tmem_ld128(taddr, r);
}

// q . k of one head row (D bf16 each), all loads issued before the sums.
template <int D>
__device__ __forceinline__ float sk_dot_bf16(const __nv_bfloat16* a, const __nv_bfloat16* b)
{
    const uint4* a4 = reinterpret_cast<const uint4*>(a);
    const uint4* b4 = reinterpret_cast<const uint4*>(b);
    uint4 qa[D / 8], ka[D / 8];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        qa[c] = __ldg(a4 + c);
        ka[c] = __ldg(b4 + c);
    }
    float d0 = 0.f, d1 = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const __nv_bfloat162* qh = reinterpret_cast<const __nv_bfloat162*>(&qa[c]);
        const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&ka[c]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 qf = __bfloat1622float2(qh[e]);
            const float2 kf = __bfloat1622float2(kh[e]);
            d0 = fmaf(qf.x, kf.x, d0);
            d1 = fmaf(qf.y, kf.y, d1);
        }
    }
    return d0 + d1;
}

// Four consecutive outputs (fp32 or bf16) from 16-byte-aligned storage.
__device__ __forceinline__ void sk_store4(void* out, int out_fp32, size_t idx, float4 v)
{
    if (out_fp32)
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + idx) = v;
    else
        *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + idx) =
            make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

// Expanding E4M3 codes in shared memory.
//
// E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits) and bfloat16
// (sign, 8 exponent bits with bias 127, 7 mantissa bits) differ, for the bits
// they share, only in the exponent bias.  A code's sign moved to bit 15 and its
// seven exponent/mantissa bits to bits 4..10 is therefore a bfloat16 of value
// value(code) * 2^-120 - for subnormal codes too, which land on bfloat16
// subnormals with the same factor - except the two NaN codes (0x7F, 0xFF).
// One bfloat16 product by scale * 2^120 (or by 2^120, exact, then by scale)
// rounds value(code) * scale once to nearest even.  Where scale is itself a
// bfloat16 value and 2^-117 <= scale <= 2^118, that product is exact in
// float32, so this equals bfloat16(value(code) * scale) computed with a float32
// product, the pool's reading rule.  The host takes this kernel for an E4M3
// pool only then.  NaN codes are detected per tile; a tile holding one is
// expanded again by the conversion instructions, which give NaN.

// Codes in bytes b_lo, b_hi of w -> bfloat16x2 of value * 2^-120 (lo half from b_lo)
template <uint32_t kSel>
__device__ __forceinline__ uint32_t sk_e4m3x2_raw(uint32_t w)
{
    const uint32_t x = __byte_perm(w, 0u, kSel);   // b_lo in byte 1, b_hi in byte 3, zero bytes between
    return (x & 0x80008000u) | ((x >> 4) & 0x07F007F0u);
}

__device__ __forceinline__ uint32_t sk_bf16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Three warps (the producer and the two epilogue warps, on three different SM
// sub-partitions: the expansion is bound by the integer pipes) expand each key
// tile of E4M3 codes (128 rows of D bytes, as TMA lands them without swizzle)
// into the bfloat16 tile the MMAs read: 64-element boxes of 128 rows x 128
// bytes whose 16-byte units are swizzled by the row (unit j of row r at
// j ^ (r & 7)), the layout a 128-byte-swizzled TMA load writes.  A lane step
// turns 8 codes (one 8-byte read; 16 lanes read 128 contiguous bytes) into 8
// values (one 16-byte write; 8 lanes fill one 128-byte row); expander e of the
// three takes steps [kSteps e / 3, kSteps (e + 1) / 3) of every lane.
constexpr int kSkExpanders = 3;

template <int D>
struct SkExpandSteps {
    static constexpr int kSteps = kSkKeys * D / 8 / 32;   // 8-code steps per lane and tile
    static constexpr int kPerRow = D / 8;
    __device__ static int begin(int e) { return kSteps * e / kSkExpanders; }
};

// Step s of this lane: its codes' byte offset in the staged tile and its values'
// byte offset in the bfloat16 tile.
template <int D>
__device__ __forceinline__ uint32_t sk_expand_dst(int lane, int s)
{
    const int u = lane + s * 32;
    const int r = u / SkExpandSteps<D>::kPerRow;
    const int j = u % SkExpandSteps<D>::kPerRow;   // elements 8j .. 8j+7 of row r
    return (j >> 3) * (kSkKeys * 128) + r * 128 + (((j & 7) ^ (r & 7)) << 4);
}

// Steps [s0, s1): the codes of up to kBatch steps are read into registers
// before any value is written (their reads are in flight together).  Returns
// (warp-uniform) whether those codes hold a NaN code.
template <int D, bool kTwo>
__device__ __forceinline__ bool sk_expand_e4m3_fast(uint32_t dst, uint32_t src, SkE4M3Mul m, int lane, int s0,
                                                    int s1)
{
    constexpr int kBatch = 4;
    const uint32_t src_l = src + lane * 8;
    uint32_t nan_bits = 0;
#pragma unroll 1
    for (int b = s0; b < s1; b += kBatch) {
        uint32_t cx[kBatch], cy[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            cx[i] = 0u;
            cy[i] = 0u;
            if (b + i < s1)
                asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(cx[i]), "=r"(cy[i]) : "r"(src_l + (b + i) * 256));
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            if (b + i < s1) {
                // bit 7 of a byte of (code & 0x7F) + 1 is set exactly for the NaN codes
                nan_bits |= ((cx[i] & 0x7F7F7F7Fu) + 0x01010101u) | ((cy[i] & 0x7F7F7F7Fu) + 0x01010101u);
                uint32_t o0 = sk_bf16x2_mul(sk_e4m3x2_raw<0x1404u>(cx[i]), m.c1);
                uint32_t o1 = sk_bf16x2_mul(sk_e4m3x2_raw<0x3424u>(cx[i]), m.c1);
                uint32_t o2 = sk_bf16x2_mul(sk_e4m3x2_raw<0x1404u>(cy[i]), m.c1);
                uint32_t o3 = sk_bf16x2_mul(sk_e4m3x2_raw<0x3424u>(cy[i]), m.c1);
                if constexpr (kTwo) {
                    o0 = sk_bf16x2_mul(o0, m.c2);
                    o1 = sk_bf16x2_mul(o1, m.c2);
                    o2 = sk_bf16x2_mul(o2, m.c2);
                    o3 = sk_bf16x2_mul(o3, m.c2);
                }
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + sk_expand_dst<D>(lane, b + i)),
                             "r"(o0), "r"(o1), "r"(o2), "r"(o3)
                             : "memory");
            }
        }
    }
    return __any_sync(0xffffffffu, (nan_bits & 0x80808080u) != 0);
}

// The same steps by the conversion instructions (exact for every code, NaN included).
template <int D>
__device__ __forceinline__ void sk_expand_e4m3_cvt(uint8_t* dst, const uint8_t* src, float scale, int lane, int s0,
                                                   int s1)
{
    for (int s = s0; s < s1; ++s) {
        const uint4 vals = bf16x8_from_e4m3(*reinterpret_cast<const uint2*>(src + (lane + s * 32) * 8), scale);
        *reinterpret_cast<uint4*>(dst + sk_expand_dst<D>(lane, s)) = vals;
    }
}

// Expander e's share of one tile.  Not inlined: the three expanding warps and
// both tiles (K, V) run one copy of the code, which stays in the instruction cache.
template <int D>
__device__ __noinline__ void sk_expand_e4m3(uint8_t* dst, const uint8_t* src, SkE4M3Mul m, float scale, int lane,
                                            int e)
{
    const int s0 = SkExpandSteps<D>::begin(e), s1 = SkExpandSteps<D>::begin(e + 1);
    const bool has_nan = m.c2 != 0u ? sk_expand_e4m3_fast<D, true>(smem_u32(dst), smem_u32(src), m, lane, s0, s1)
                                    : sk_expand_e4m3_fast<D, false>(smem_u32(dst), smem_u32(src), m, lane, s0, s1);
    if (has_nan) {
        __syncwarp();
        sk_expand_e4m3_cvt<D>(dst, src, scale, lane, s0, s1);
    }
}

template <int D, int N, bool kE4M3>
__global__ void __launch_bounds__(kSkThreads, SkCfg<D, N, kE4M3>::kCtasPerSm)
    decode_smallk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const SkParams p)
{
    using C = SkCfg<D, N, kE4M3>;
    constexpr int NS = C::kStages;
    constexpr int NP = C::kPBufs;
    constexpr int NQ = C::kQBufs;
    constexpr int NS8 = C::kStages8;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == (int)UNIPIN_ERR_DEVICE_TIMEOUT) return;
    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0) report(p.status, (int)UNIPIN_ERR_CUDA);
        return;
    }
    uint8_t* ring = smem + C::kOffRing;
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sP = smem + C::kOffP;
    float* red = reinterpret_cast<float*>(smem + C::kOffScratch);   // [4][N] softmax
    float* mref = red + 4 * N;                                      // [N] reference max (log2 units)
    float* corr = mref + N;                                         // [N]
    float* hand_m = corr + N;                                       // [2][N] item statistics, softmax -> epilogue
    float* hand_l = hand_m + 2 * N;                                 // [2][N]
    float* coef_b = hand_l + 2 * N;                                 // [N] epilogue: weight of the own value
    float* wts = coef_b + N;                                        // [kSkMaxSplit][N] epilogue: split weights
    volatile int* last_flag = reinterpret_cast<volatile int*>(wts + kSkMaxSplit * N);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_q = bars + 0;            // [2] Q buffer landed
    uint64_t* q_empty = bars + 2;          // [2] the last S MMA of the item using Q buffer b finished
    uint64_t* pv_done = bars + 4;          // [2] O += P V of P buffer b finished
    uint64_t* p_full = bars + 6;           // [2] P buffer written (4 softmax warps)
    uint64_t* o_full = bars + 8;           // [2] the last P.V of the item in O buffer b finished
    uint64_t* o_free = bars + 10;          // [2] O buffer b read out (2 epilogue warps)
    uint64_t* h_full = bars + 12;          // [2] hand-off entry written (4 softmax warps)
    uint64_t* h_free = bars + 14;          // [2] hand-off entry read (2 epilogue warps)
    uint64_t* egrp = bars + 16;            // epilogue-group barrier (2 warps)
    uint64_t* bar_drain = bars + 17;
    uint64_t* s_full = bars + 18;          // [kSBufs] S^T buffer computed
    uint64_t* s_free = s_full + C::kSBufs; // [kSBufs] S^T buffer read out (4 softmax warps)
    uint64_t* k_full = s_free + C::kSBufs; // [NS] K tile landed
    uint64_t* k_empty = k_full + NS;       // [NS] its S MMA finished
    uint64_t* v_full = k_empty + NS;       // [NS] V tile landed
    uint64_t* v_empty = v_full + NS;       // [NS] its P.V finished
    uint64_t* k8_full = v_empty + NS;      // [NS8] E4M3 pool: K codes landed in staging
    uint64_t* v8_full = k8_full + NS8;     // [NS8] V codes landed
    uint64_t* k8_empty = v8_full + NS8;    // [NS8] K codes read by the three expanders
    uint64_t* v8_empty = k8_empty + NS8;   // [NS8] V codes read
    uint64_t* item_full = v8_empty + NS8;  // [kSkItemSlots]
    uint64_t* item_empty = item_full + kSkItemSlots;
    volatile long long* item_ring = reinterpret_cast<volatile long long*>(item_empty + kSkItemSlots);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_empty + 2 * kSkItemSlots);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_q + b, 1);
            mbar_init(q_empty + b, 1);
            mbar_init(pv_done + b, 1);
            mbar_init(p_full + b, 4);
            mbar_init(o_full + b, 1);
            mbar_init(o_free + b, kSkEpiWarps);
            mbar_init(h_full + b, 4);
            mbar_init(h_free + b, kSkEpiWarps);
        }
        for (int b = 0; b < C::kSBufs; ++b) {
            mbar_init(s_full + b, 1);
            mbar_init(s_free + b, 4);
        }
        mbar_init(egrp, kSkEpiWarps);
        mbar_init(bar_drain, 1);
        for (int s = 0; s < NS; ++s) {
            // an E4M3 pool's tiles are written by the three expanders, a bfloat16 pool's by one TMA load
            mbar_init(k_full + s, kE4M3 ? kSkExpanders : 1);
            mbar_init(k_empty + s, 1);
            mbar_init(v_full + s, kE4M3 ? kSkExpanders : 1);
            mbar_init(v_empty + s, 1);
        }
        for (int s = 0; s < NS8; ++s) {
            mbar_init(k8_full + s, 1);
            mbar_init(v8_full + s, 1);
            mbar_init(k8_empty + s, kSkExpanders);
            mbar_init(v8_empty + s, kSkExpanders);
        }
        for (int s = 0; s < kSkItemSlots; ++s) {
            mbar_init(item_full + s, 1);
            mbar_init(item_empty + s, kSkConsumers);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (threadIdx.x < N) mref[threadIdx.x] = -INFINITY;
    if (warp == kSkMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns, (int)UNIPIN_ERR_DEVICE_TIMEOUT};
    int n_items = 0;
    // Consumers: the next item (warp-uniform), waiting with `wait`
    auto pop_item_w = [&](bool& ok, long long& g, auto&& wait) -> bool {
        const int si = n_items % kSkItemSlots;
        ok = wait(item_full + si, (uint32_t)((n_items / kSkItemSlots) & 1));
        if (!ok) return false;
        g = item_ring[si];
        __syncwarp();
        if (lane == 0) mbar_arrive(item_empty + si);
        ++n_items;
        return g >= 0;
    };
    auto pop_item = [&](bool& ok, long long& g) -> bool {
        return pop_item_w(ok, g, [&](uint64_t* bar, uint32_t ph) {
            return __all_sync(0xffffffffu, mbar_wait(bar, ph, ctl));
        });
    };
    const bool leader = lane == 0;
    // E4M3 pool: expander e's share of the next K tile and of the next V tile
    // whose codes have landed and whose bfloat16 ring slot is free (warp-uniform;
    // kx / vx count the tiles this warp has expanded).  True if it did any.
    auto expand_step = [&](int e, int& kx, int& vx) -> bool {
        bool prog = false;
        if constexpr (kE4M3) {
            uint8_t* stage8 = smem + C::kOffStage8;
            const int ks8 = kx % NS8, kst = kx % NS;
            if (__all_sync(0xffffffffu, mbar_test_wait(k8_full + ks8, (kx / NS8) & 1) &&
                                            (kx < NS || mbar_test_wait(k_empty + kst, ((kx / NS) - 1) & 1)))) {
                sk_expand_e4m3<D>(ring + kst * C::kStageBytes + C::kTileKV, stage8 + ks8 * C::kStage8, p.k_mul,
                                  p.k_scale, lane, e);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(k_full + kst);
                    mbar_arrive(k8_empty + ks8);
                }
                ++kx;
                prog = true;
            }
            const int vs8 = vx % NS8, vst = vx % NS;
            if (__all_sync(0xffffffffu, mbar_test_wait(v8_full + vs8, (vx / NS8) & 1) &&
                                            (vx < NS || mbar_test_wait(v_empty + vst, ((vx / NS) - 1) & 1)))) {
                sk_expand_e4m3<D>(ring + vst * C::kStageBytes, stage8 + vs8 * C::kStage8 + C::kTile8, p.v_mul,
                                  p.v_scale, lane, e);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(v_full + vst);
                    mbar_arrive(v8_empty + vs8);
                }
                ++vx;
                prog = true;
            }
        }
        return prog;
    };

    if (warp == kSkProducerWarp) {
        // ------------------------------------------------------------ producer
        // Two streams into the ring: K tiles (freed when their S MMA finishes)
        // and V tiles (freed when their P.V finishes).  A K slot thus refills
        // while the softmax still works on that tile, and V, needed only after
        // the softmax, is requested as soon as its slot frees.  One polling loop
        // drives both (warp-uniform; the leader lane issues the copies).
        if (leader) {
            tma_prefetch_map(&tm_q);
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
        }
        struct PItem {
            int plane, t_begin, nt, nt_all, npast;
        };
        PItem items[4];          // items with tiles whose V stream has not finished, by sequence % 4
        int uk = 0, uv = 0;      // K / V tiles issued (global tile index)
        int nk = 0, nv = 0;      // items with tiles started by the K stream / finished by the V stream
        int ik = 0, iv = 0;      // tile within the current K / V item
        int nq = 0;
        int kc8 = 0, vc8 = 0;    // E4M3 pool: K / V tiles this warp has expanded its share of
        uint8_t* stage8 = smem + C::kOffStage8;
        bool k_has = false, q_done = false, claim_done = false, ok = true;
        int q_h = 0, q_tok = 0;
        long long g_next = (long long)blockIdx.x << 20;   // the block's pieces, in order
        uint64_t t_prog = global_timer_ns();
        for (uint32_t spin = 1;; ++spin) {
            bool prog = false;
            // 1. publish the next item once the K stream has finished its current one
            if (!k_has && !claim_done && nk - nv < 3) {
                const int si = n_items % kSkItemSlots;
                if (n_items < kSkItemSlots ||
                    __all_sync(0xffffffffu, mbar_test_wait(item_empty + si, ((n_items / kSkItemSlots) - 1) & 1))) {
                    const long long g = g_next;
                    const bool found = sk_piece_exists(p, g);
                    ++g_next;
                    if (leader) {
                        item_ring[si] = found ? g : -1;
                        mbar_arrive(item_full + si);   // release: the consumers see the ring entry
                    }
                    ++n_items;
                    prog = true;
                    if (!found) {
                        claim_done = true;
                    } else {
                        const SkWork w = sk_make_work<N>(p, g);
                        if (w.nt > 0) {
                            items[nk % 4] = PItem{(p.layer * p.S + w.slot) * (p.H / p.G) + w.h, w.t_begin, w.nt,
                                                  w.nt_all, w.npast};
                            q_h = w.h;
                            q_tok = w.tok0;
                            ++nk;
                            k_has = true;
                            ik = 0;
                            q_done = false;
                        }
                    }
                }
            }
            // 2. K stream: the item's Q, then its K tiles
            if (k_has) {
                if (!q_done) {
                    const int qb = nq % NQ;
                    if (nq < NQ || __all_sync(0xffffffffu, mbar_test_wait(q_empty + qb, ((nq / NQ) - 1) & 1))) {
                        if (leader) {
                            mbar_arrive_expect_tx(bar_q + qb, C::kQBytes);
                            for (int c = 0; c < C::kChunks; ++c)
                                // N / G candidate tokens x the G query heads of key/value head q_h
                                tma_load_3d(sQ + qb * C::kQBytes + c * C::kAtomQ, &tm_q, bar_q + qb, c * 64, q_h * p.G,
                                            q_tok);
                        }
                        ++nq;
                        q_done = true;
                        prog = true;
                    }
                }
                const int st = uk % NS;
                bool k_go;
                if constexpr (kE4M3)   // the staging slot's last codes were read by all expanders
                    k_go = q_done && (uk < NS8 || __all_sync(0xffffffffu, mbar_test_wait(k8_empty + uk % NS8,
                                                                                         ((uk / NS8) - 1) & 1)));
                else
                    k_go = q_done &&
                           (uk < NS || __all_sync(0xffffffffu, mbar_test_wait(k_empty + st, ((uk / NS) - 1) & 1)));
                if (k_go) {
                    const PItem& it = items[(nk - 1) % 4];
                    const int start = sk_tile_start(it.t_begin + ik, it.nt_all, it.npast);
                    if (leader) {
                        if constexpr (kE4M3) {
                            const int s8 = uk % NS8;
                            mbar_arrive_expect_tx(k8_full + s8, C::kTile8);
                            tma_load_3d(stage8 + s8 * C::kStage8, &tm_k, k8_full + s8, 0, start, it.plane);
                        } else {
                            uint8_t* dst = ring + st * C::kStageBytes + C::kTileKV;
                            mbar_arrive_expect_tx(k_full + st, C::kTileKV);
                            for (int c = 0; c < C::kChunks; ++c)
                                tma_load_3d(dst + c * C::kAtom, &tm_k, k_full + st, c * 64, start, it.plane);
                        }
                    }
                    ++uk;
                    prog = true;
                    if (++ik == it.nt) k_has = false;
                }
            }
            // 3. V stream: V_u once K_u has been issued
            if (uv < uk) {
                const int st = uv % NS;
                bool v_go;
                if constexpr (kE4M3)
                    v_go = uv < NS8 ||
                           __all_sync(0xffffffffu, mbar_test_wait(v8_empty + uv % NS8, ((uv / NS8) - 1) & 1));
                else
                    v_go = uv < NS || __all_sync(0xffffffffu, mbar_test_wait(v_empty + st, ((uv / NS) - 1) & 1));
                if (v_go) {
                    const PItem& it = items[nv % 4];
                    const int start = sk_tile_start(it.t_begin + iv, it.nt_all, it.npast);
                    if (leader) {
                        if constexpr (kE4M3) {
                            const int s8 = uv % NS8;
                            mbar_arrive_expect_tx(v8_full + s8, C::kTile8);
                            tma_load_3d(stage8 + s8 * C::kStage8 + C::kTile8, &tm_v, v8_full + s8, 0, start,
                                        it.plane);
                        } else {
                            uint8_t* dst = ring + st * C::kStageBytes;
                            mbar_arrive_expect_tx(v_full + st, C::kTileKV);
                            for (int c = 0; c < C::kChunks; ++c)
                                tma_load_3d(dst + c * C::kAtom, &tm_v, v_full + st, c * 64, start, it.plane);
                        }
                    }
                    ++uv;
                    prog = true;
                    if (++iv == it.nt) {
                        iv = 0;
                        ++nv;
                    }
                }
            }
            // 4. this warp's share of the code expansion (expander 0)
            if constexpr (kE4M3)
                if ((kc8 < uk || vc8 < uv) && expand_step(0, kc8, vc8)) prog = true;
            // every copy issued (and, for codes, expanded)
            if (claim_done && !k_has && uv == uk && (!kE4M3 || (kc8 == uk && vc8 == uv))) break;
            if (prog) {
                t_prog = global_timer_ns();
            } else {
                __nanosleep(p.poll_ns);
                if ((spin & 15) == 0) {
                    // warp-uniform: give up when the block aborted or nothing moved for too long
                    const bool aborted = *abort_flag != 0;
                    const bool stop = __any_sync(0xffffffffu, aborted || global_timer_ns() - t_prog > p.wait_limit_ns);
                    if (stop) {
                        if (leader && !aborted) {
                            *abort_flag = 1;
                            report(p.status, (int)UNIPIN_ERR_DEVICE_TIMEOUT);
                        }
                        ok = false;
                        break;
                    }
                }
            }
        }
        if (!ok && !claim_done && leader) {
            const int si = n_items % kSkItemSlots;
            if (n_items < kSkItemSlots ||
                mbar_wait_drain(item_empty + si, ((n_items / kSkItemSlots) - 1) & 1, p.wait_limit_ns)) {
                item_ring[si] = -1;
                mbar_arrive(item_full + si);
                ++n_items;
            }
        }
        if (leader) {
            // Let every copy this warp started land before the block exits.
            if constexpr (kE4M3) {
                for (int v = (uk > NS8 ? uk - NS8 : 0); v < uk; ++v)
                    mbar_wait_drain(k8_full + v % NS8, (v / NS8) & 1, p.wait_limit_ns);
                for (int v = (uv > NS8 ? uv - NS8 : 0); v < uv; ++v)
                    mbar_wait_drain(v8_full + v % NS8, (v / NS8) & 1, p.wait_limit_ns);
            } else {
                for (int v = (uk > NS ? uk - NS : 0); v < uk; ++v)
                    mbar_wait_drain(k_full + v % NS, (v / NS) & 1, p.wait_limit_ns);
                for (int v = (uv > NS ? uv - NS : 0); v < uv; ++v)
                    mbar_wait_drain(v_full + v % NS, (v / NS) & 1, p.wait_limit_ns);
            }
            for (int v = (nq > NQ ? nq - NQ : 0); v < nq; ++v)
                mbar_wait_drain(bar_q + v % NQ, (v / NQ) & 1, p.wait_limit_ns);
            for (int v = (n_items > kSkItemSlots ? n_items - kSkItemSlots : 0); v < n_items; ++v)
                mbar_wait_drain(item_empty + v % kSkItemSlots, (v / kSkItemSlots) & 1, p.wait_limit_ns);
        }
    } else if (warp == kSkMmaWarp) {
        // --------------------------------------------------------- MMA issuer
        // Two streams, issued as their inputs arrive (one polling loop):
        //   S^T_i = K_i Q^T  once K_i has landed and an S buffer is free; up to
        //                    kSBufs tiles ahead of the softmax, across items;
        //   O += P_i V_i     once the softmax has written P_i and V_i has landed
        //                    (the first of an item also needs its O buffer back
        //                    from the epilogue).  Item j accumulates in O buffer j % 2.
        constexpr int NSB = C::kSBufs;
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kSkKeys, N, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(C::kPvRows, D, true, false);
        const uint32_t ring_a = smem_u32(ring);
        // K (A of S^T): K-major, 128-byte rows, 8-row groups 1024 bytes apart.
        const uint64_t dk0 = smem_desc(ring_a + C::kTileKV, 16, 1024, kLayoutSw128);
        const uint64_t dq0 = smem_desc(smem_u32(sQ), 16, 1024, kLayoutSw128);
        // V (B of O += P V, MN-major): 64-element head-dim blocks 16 KB apart, 8-key groups 1024 bytes apart.
        const uint64_t dv0 = smem_desc(ring_a, C::kAtom, 1024, kLayoutSw128);
        // P (A of O += P V): K-major rows of 64 keys per box, 8-row groups 1024 bytes apart.
        const uint64_t dp0 = smem_desc(smem_u32(sP), 16, 1024, kLayoutSw128);
        int pv_nt[8];                 // tile counts of the items with tiles whose P.V are not all issued
        int nqueued = 0, npv_item = 0;
        int gs = 0;                   // S tiles issued (= global tile index of the next S)
        int gp = 0;                   // P.V products issued
        int is = 0, s_nt = 0, nq = 0, ip = 0;
        bool s_has = false, s_done = false, q_ok = false, ok = true;
        uint64_t t_prog = global_timer_ns();
        for (uint32_t spin = 1;; ++spin) {
            bool prog = false;
            // ---- S stream: take the next item with tiles
            if (!s_has && !s_done && nqueued - npv_item < 7) {
                const int si = n_items % kSkItemSlots;
                if (__all_sync(0xffffffffu, mbar_test_wait(item_full + si, (n_items / kSkItemSlots) & 1))) {
                    const long long g = item_ring[si];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(item_empty + si);
                    ++n_items;
                    prog = true;
                    if (g < 0) {
                        s_done = true;
                    } else {
                        const SkWork w = sk_make_work<N>(p, g);
                        if (w.nt > 0) {
                            pv_nt[nqueued % 8] = w.nt;
                            ++nqueued;
                            s_has = true;
                            s_nt = w.nt;
                            is = 0;
                            q_ok = false;
                        }
                    }
                }
            }
            if (s_has) {
                const int qb = nq % NQ;
                if (!q_ok && __all_sync(0xffffffffu, mbar_test_wait(bar_q + qb, (nq / NQ) & 1))) q_ok = true;
                const int st = gs % NS;
                const int sb = gs % NSB;
                if (q_ok && __all_sync(0xffffffffu, mbar_test_wait(k_full + st, (gs / NS) & 1) &&
                                                        (gs < NSB || mbar_test_wait(s_free + sb, ((gs / NSB) - 1) & 1)))) {
                    tc_fence_after_sync();
                    if (leader) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const int box = kk / 4;
                            const int in_row = (kk % 4) * 32;
                            const uint64_t a = dk0 + (uint64_t)((st * C::kStageBytes + box * C::kAtom + in_row) >> 4);
                            const uint64_t b = dq0 + (uint64_t)((qb * C::kQBytes + box * C::kAtomQ + in_row) >> 4);
                            umma_bf16_ss(tmem + sb * N, a, b, idesc_qk, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(s_full + sb);
                        umma_commit(k_empty + st);
                        if (is == s_nt - 1) umma_commit(q_empty + qb);
                    }
                    ++gs;
                    prog = true;
                    if (++is == s_nt) {
                        s_has = false;
                        ++nq;
                    }
                }
            }
            // ---- P.V stream: tiles whose S was issued
            if (gp < gs) {
                const int nt = pv_nt[npv_item % 8];
                const int ob = npv_item & 1;
                const int pb = gp % NP;
                const int st = gp % NS;
                if (__all_sync(0xffffffffu, mbar_test_wait(p_full + pb, (gp / NP) & 1) &&
                                                mbar_test_wait(v_full + st, (gp / NS) & 1) &&
                                                (ip > 0 || npv_item < 2 ||
                                                 mbar_test_wait(o_free + ob, ((npv_item >> 1) - 1) & 1)))) {
                    tc_fence_after_sync();
                    if (leader) {
                        // K-steps of 16 keys: 32 bytes within a P row (then the second box), 16 V rows
#pragma unroll
                        for (int kk = 0; kk < kSkKeys / 16; ++kk) {
                            const uint64_t a =
                                dp0 + (uint64_t)((pb * C::kPBytes + (kk / 4) * C::kPBox + (kk % 4) * 32) >> 4);
                            const uint64_t b = dv0 + (uint64_t)((st * C::kStageBytes + kk * 2048) >> 4);
                            umma_bf16_ss(tmem + C::kColO + ob * D, a, b, idesc_pv, (ip > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(pv_done + pb);
                        umma_commit(v_empty + st);
                        if (ip == nt - 1) umma_commit(o_full + ob);
                    }
                    ++gp;
                    prog = true;
                    if (++ip == nt) {
                        ip = 0;
                        ++npv_item;
                    }
                }
            }
            if (s_done && !s_has && gp == gs) break;
            if (prog) {
                t_prog = global_timer_ns();
            } else {
                __nanosleep(p.poll_ns);
                if ((spin & 15) == 0) {
                    // warp-uniform: give up when the block aborted or nothing moved for too long
                    const bool aborted = *abort_flag != 0;
                    const bool stop = __any_sync(0xffffffffu, aborted || global_timer_ns() - t_prog > p.wait_limit_ns);
                    if (stop) {
                        if (leader && !aborted) {
                            *abort_flag = 1;
                            report(p.status, (int)UNIPIN_ERR_DEVICE_TIMEOUT);
                        }
                        ok = false;
                        break;
                    }
                }
            }
        }
        (void)ok;
        if (leader) {
            umma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.wait_limit_ns);
        }
    } else if (warp >= kSkSoftmaxWarp0) {
        // ------------------------------------------------------------ softmax
        // The four warps move in step: each named-barrier reduction below is
        // reached by all 128 threads, and they leave the item loop only
        // together, on such a reduction (bounded waits only flag a failure).
        const int wq = warp - kSkSoftmaxWarp0;                   // TMEM lane quarter
        const int t = wq * 32 + lane;                            // key of a tile; O row t (candidate t)
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        constexpr int kBar = 1;                                  // named barrier of the group
        constexpr int kGroup = 128;
        constexpr int NSB = C::kSBufs;
        const float sl2 = p.sl2;
        int gs = 0, gp = 0, nb = 0, nh = 0;
        bool pending_fail = false;                               // a wait after the last reduction failed
        int pv_seen[2] = {0, 0};
        long long g;
        // Wait until the P.V product with global index gidx has finished
        // (completions of each P buffer are consumed in order); warp-uniform.
        auto wait_pv = [&](int gidx) {
            if (gidx < 0) return true;
            const int pb = gidx % NP;
            const int n = gidx / NP;
            bool r = true;
            while (r && pv_seen[pb] <= n) {
                r = __all_sync(0xffffffffu, mbar_wait(pv_done + pb, pv_seen[pb] & 1, ctl));
                ++pv_seen[pb];
            }
            tc_fence_after_sync();
            return r;
        };
        for (;;) {
            bool okp;
            const bool got = pop_item(okp, g);
            if (bar_red_or(kBar, kGroup, !okp || pending_fail || *abort_flag != 0)) break;
            if (!got) break;   // the end marker: the same ring entry for every warp
            const SkWork w = sk_make_work<N>(p, g);
            if (!w.rows_ok && t == 0) report(p.status, (int)UNIPIN_ERR_OUT_OF_RANGE);
            if (w.rows_ok && !w.valid && t == 0 && w.split == 0) report(p.status, (int)UNIPIN_ERR_OUT_OF_RANGE);
            const int ob = nb & 1;
            const uint32_t tO = lane_base + C::kColO + ob * D;
            // per-thread partial column sums of P (owned columns), relative to mref
            constexpr int kOwn = N >= 32 ? N / 32 : 1;
            float lown[kOwn];
#pragma unroll
            for (int e = 0; e < kOwn; ++e) lown[e] = 0.f;
            bool quit = false;
            for (int i = 0; i < w.nt; ++i) {
                const int tile = w.t_begin + i;
                const int lo = tile * kSkKeys;
                const int start = sk_tile_start(tile, w.nt_all, w.npast);
                const int key = start + t;
                const bool key_ok = key >= lo && key < w.npast;
                const int sb = gs % NSB;
                const bool ok_s = __all_sync(0xffffffffu, mbar_wait(s_full + sb, (gs / NSB) & 1, ctl));
                float x[N];
                bool need = false;
                if (ok_s) {
                    tc_fence_after_sync();
                    uint32_t sraw[N];
                    tmem_ld_n<N>(lane_base + sb * N, sraw);
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_free + sb);
#pragma unroll
                    for (int c = 0; c < N; ++c)
                        x[c] = (key_ok && c < w.ncol) ? __uint_as_float(sraw[c]) * sl2 : -INFINITY;
                    // vote: does any score exceed its candidate's reference max by > 2^8?
#pragma unroll
                    for (int c = 0; c < N; c += 4) {
                        const float4 m4 = *reinterpret_cast<const float4*>(mref + c);
                        need |= x[c] > m4.x + kSkRescaleLog2;
                        need |= x[c + 1] > m4.y + kSkRescaleLog2;
                        need |= x[c + 2] > m4.z + kSkRescaleLog2;
                        need |= x[c + 3] > m4.w + kSkRescaleLog2;
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < N; ++c) x[c] = -INFINITY;
                }
                ++gs;
                const bool fail_s = !ok_s || pending_fail || *abort_flag != 0;
                bool ok_w = true;
                if (bar_red_or(kBar, kGroup, need || fail_s)) {
                    if (bar_red_or(kBar, kGroup, fail_s)) {
                        quit = true;
                        break;
                    }
                    // exact column maxima of this tile (16 columns at a time: lane pair l/2
                    // owns column c0 + l/2); move every reference max to it
#pragma unroll
                    for (int c0 = 0; c0 < N; c0 += 16) {
                        float cm[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c) cm[c] = x[c0 + c];
                        sk_rs_step<16, 16, true>(cm, lane);
                        if ((lane & 1) == 0) red[wq * N + c0 + (lane >> 1)] = cm[0];
                    }
                    bar_group_sync(kBar, kGroup);
                    if (t < N) {
                        const float mt = fmaxf(fmaxf(red[t], red[N + t]), fmaxf(red[2 * N + t], red[3 * N + t]));
                        const float mo = mref[t];
                        const float mn = fmaxf(mo, mt);
                        corr[t] = (mo == -INFINITY) ? 0.f : ex2_approx(mo - mn);
                        mref[t] = mn;
                    }
                    bar_group_sync(kBar, kGroup);
#pragma unroll
                    for (int e = 0; e < kOwn; ++e) lown[e] *= corr[sk_owned_col<N>(lane, e)];
                    if (i > 0) {
                        // rescale the O rows accumulated so far (after the last P.V): row c is candidate c
                        ok_w = wait_pv(gp - 1);
                        // O row r: TMEM lane r (M = 128), or lane 32 (r / 16) + r % 16 (M = 64)
                        if (ok_w && wq * (C::kPv64 ? 16 : 32) < N) {
                            const int orow = C::kPv64 ? (lane < 16 ? wq * 16 + lane : 0) : t;
                            const float cf = corr[orow < N ? orow : 0];
#pragma unroll
                            for (int c0 = 0; c0 < D; c0 += 16) {
                                uint32_t o[16];
                                tmem_ld16(tO + c0, o);
#pragma unroll
                                for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * cf);
                                tmem_st16(tO + c0, o);
                            }
                        }
                    }
                }
                // P = 2^(x - m)
#pragma unroll
                for (int c = 0; c < N; c += 4) {
                    const float4 m4 = *reinterpret_cast<const float4*>(mref + c);
                    const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float mu = mm[e] == -INFINITY ? 0.f : mm[e];
                        x[c + e] = ex2_approx(x[c + e] - mu);
                    }
                }
                // the P buffer is free once the P.V that last read it has finished
                const int pb = gp % NP;
                const bool ok_p = ok_w && wait_pv(gp - NP);
                if (ok_p) {
                    // column t of P: key t of the tile is element t % 64 of a 128-byte row of box t / 64
                    uint8_t* pbox = sP + pb * C::kPBytes + (t / 64) * C::kPBox;
                    const int kx = t % 64;
#pragma unroll
                    for (int c = 0; c < N; ++c)
                        *reinterpret_cast<__nv_bfloat16*>(pbox + c * 128 + ((((kx >> 3) ^ (c & 7))) << 4) +
                                                          (kx & 7) * 2) = __float2bfloat16_rn(x[c]);
                    fence_proxy_async_smem();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(p_full + pb);
                } else {
                    pending_fail = true;   // decided together at the next reduction
                }
                ++gp;
                sk_rs_step<N, 16, false>(x, lane);
#pragma unroll
                for (int e = 0; e < kOwn; ++e) lown[e] += x[e];
            }
            if (quit) break;
            // hand the item's statistics to the epilogue (every item, so both sides count alike)
            const int hb = nh & 1;
            if (w.nt > 0) {
#pragma unroll
                for (int e = 0; e < kOwn; ++e)
                    if (N >= 32 || (lane & 1) == 0) red[wq * N + sk_owned_col<N>(lane, e)] = lown[e];
            }
            const bool ok_h = nh < 2 || __all_sync(0xffffffffu, mbar_wait(h_free + hb, ((nh >> 1) - 1) & 1, ctl));
            if (bar_red_or(kBar, kGroup, !ok_h || pending_fail || *abort_flag != 0)) break;
            if (t < N) {
                hand_l[hb * N + t] = w.nt > 0 ? red[t] + red[N + t] + red[2 * N + t] + red[3 * N + t] : 0.f;
                hand_m[hb * N + t] = w.nt > 0 ? mref[t] : -INFINITY;
                mref[t] = -INFINITY;   // ready for the next item
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(h_full + hb);
            ++nh;
            if (w.nt > 0) ++nb;
            // red and mref are reused by the next item
            bar_group_sync(kBar, kGroup);
        }
    } else {
        // ----------------------------------------------------------- epilogue
        // candidate column t: O row t is TMEM lane t (M = 128 P.V) or lane 32 (t / 16) + t % 16
        // (M = 64: lanes 16-31 of each warp hold no row and take no column)
        const int t = C::kPv64 ? (lane < 16 ? warp * 16 + lane : kSkEpiWarps * 32) : (int)threadIdx.x;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const int hkv = p.H / p.G;
        int nb = 0, nh = 0;
        uint32_t negrp = 0;
        bool ok = true;
        long long g;
        // Over an E4M3 pool these two warps are expanders 1 and 2: every wait whose end
        // may need their share of the expansion keeps expanding meanwhile.
        int ekx = 0, evx = 0;
        auto epi_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            if constexpr (!kE4M3) {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, ctl));
            } else {
                uint64_t t0 = global_timer_ns();
                for (uint32_t it = 1;; ++it) {
                    if (__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) return true;
                    if (expand_step(1 + warp, ekx, evx)) {
                        t0 = global_timer_ns();
                        continue;
                    }
                    __nanosleep(p.poll_ns);
                    if ((it & 15) == 0) {
                        const bool aborted = *abort_flag != 0;
                        if (__any_sync(0xffffffffu, aborted || global_timer_ns() - t0 > p.wait_limit_ns)) {
                            if (lane == 0 && !aborted) {
                                *abort_flag = 1;
                                report(p.status, (int)UNIPIN_ERR_DEVICE_TIMEOUT);
                            }
                            return false;
                        }
                    }
                }
            }
        };
        while (pop_item_w(ok, g, epi_wait)) {
            const SkWork w = sk_make_work<N>(p, g);
            // Column t = (candidate t / G, query head w.h * G + t % G): its output row, its own
            // key/value row, and its own score (log2 units), taken while the item's keys stream.
            const size_t qrow = (size_t)(w.tok0 + t / p.G) * p.H + w.h * p.G + t % p.G;
            const size_t kvrow = (size_t)(w.tok0 + t / p.G) * hkv + w.h;
            const bool mine = w.valid && t < w.ncol;
            const float ss_own = mine ? p.sl2 * sk_dot_bf16<D>(p.q + qrow * D, p.k_self + kvrow * D) : -INFINITY;
            // the item's statistics
            const int hb = nh & 1;
            if (!(ok = epi_wait(h_full + hb, (nh >> 1) & 1))) break;
            const float l_c = t < N ? hand_l[hb * N + t] : 0.f;
            const float m_c = t < N ? hand_m[hb * N + t] : -INFINITY;
            __syncwarp();
            if (lane == 0) mbar_arrive(h_free + hb);
            ++nh;
            if (!w.rows_ok) continue;
            // O row t, 32 columns at a time (warp-collective loads where the warp holds candidate rows)
            const int ob = nb & 1;
            const bool have_o = w.nt > 0 && warp * (C::kPv64 ? 16 : 32) < N;
            if (w.nt > 0) {
                if (!(ok = epi_wait(o_full + ob, (nb >> 1) & 1))) break;
                tc_fence_after_sync();
            }
            // final coefficients (one split): out = (a O + b v_self) / (a l + b)
            float ca = 0.f, cb = 0.f;
            if (w.npieces == 1 && mine) {
                const float mf = fmaxf(m_c, ss_own);
                const float a = (m_c == -INFINITY) ? 0.f : ex2_approx(m_c - mf);
                const float b = ex2_approx(ss_own - mf);
                const float inv = 1.f / (l_c * a + b);
                ca = a * inv;
                cb = b * inv;
            }
            float* po = p.part_o + ((size_t)w.split * p.total_rows * p.H + qrow) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                if (have_o) {
                    tmem_ld32(lane_base + C::kColO + ob * D + c0, o);
                } else {
#pragma unroll
                    for (int d = 0; d < 32; ++d) o[d] = 0u;
                }
                if (w.npieces == 1) {
                    // a rejected request (ca = cb = 0) gets zero rows
                    if (t < w.ncol) {
                        const uint4* v4 = reinterpret_cast<const uint4*>(p.v_self + kvrow * D + c0);
#pragma unroll
                        for (int d8 = 0; d8 < 4; ++d8) {
                            const uint4 vb = mine ? __ldg(v4 + d8) : make_uint4(0u, 0u, 0u, 0u);
                            const __nv_bfloat162* vh = reinterpret_cast<const __nv_bfloat162*>(&vb);
                            float r[8];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 vf = __bfloat1622float2(vh[e]);
                                r[2 * e] = __uint_as_float(o[d8 * 8 + 2 * e]) * ca + cb * vf.x;
                                r[2 * e + 1] = __uint_as_float(o[d8 * 8 + 2 * e + 1]) * ca + cb * vf.y;
                            }
                            sk_store4(p.out, p.out_fp32, qrow * D + c0 + d8 * 8, make_float4(r[0], r[1], r[2], r[3]));
                            sk_store4(p.out, p.out_fp32, qrow * D + c0 + d8 * 8 + 4, make_float4(r[4], r[5], r[6], r[7]));
                        }
                    }
                } else if (t < w.ncol) {
#pragma unroll
                    for (int d = 0; d < 32; d += 4)
                        *reinterpret_cast<float4*>(po + c0 + d) =
                            make_float4(__uint_as_float(o[d]), __uint_as_float(o[d + 1]), __uint_as_float(o[d + 2]),
                                        __uint_as_float(o[d + 3]));
                }
            }
            if (w.nt > 0) {
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_free + ob);
                ++nb;
            }
            if (w.npieces == 1) continue;
            // publish the partial; the last split of this (request, head) to arrive merges
            if (t < w.ncol) {
                float* ml = p.part_ml + ((size_t)w.split * p.total_rows * p.H + qrow) * 2;
                ml[0] = w.valid ? m_c : -INFINITY;
                ml[1] = w.valid ? l_c : 0.f;
            }
            __threadfence();
            if (!(ok = warp_group_sync(egrp, negrp, ctl, lane))) break;
            if (t == 0) {
                const unsigned prev = atomicAdd(p.pair_cnt + w.pair, 1u);
                *last_flag = prev == (unsigned)(w.npieces - 1);
            }
            if (!(ok = warp_group_sync(egrp, negrp, ctl, lane))) break;
            if (*last_flag) {
                __threadfence();
                if (t < w.ncol) {
                    // weights of the splits and of the own key: LSE merge in log2 units
                    float ms[kSkMaxSplit], ls[kSkMaxSplit];
#pragma unroll
                    for (int s = 0; s < kSkMaxSplit; ++s) {
                        float2 ml = make_float2(-INFINITY, 0.f);
                        if (s < w.npieces)
                            ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + ((size_t)s * p.total_rows * p.H + qrow) * 2));
                        ms[s] = ml.x;
                        ls[s] = ml.y;
                    }
                    float mf = ss_own;
#pragma unroll
                    for (int s = 0; s < kSkMaxSplit; ++s) mf = fmaxf(mf, ms[s]);
                    const float b = ex2_approx(ss_own - mf);
                    float den = b;
#pragma unroll
                    for (int s = 0; s < kSkMaxSplit; ++s) {
                        const float a = (ms[s] == -INFINITY || !(ls[s] > 0.f)) ? 0.f : ex2_approx(ms[s] - mf);
                        den = fmaf(a, ls[s], den);
                        if (s < w.npieces) wts[s * N + t] = a;
                    }
                    // a rejected request (no own score: every term -inf) gets zero weights
                    const float inv = w.valid ? 1.f / den : 0.f;
                    for (int s = 0; s < w.npieces; ++s) wts[s * N + t] *= inv;
                    coef_b[t] = w.valid ? b * inv : 0.f;
                }
                if (!(ok = warp_group_sync(egrp, negrp, ctl, lane))) break;
                // out = b v_self + sum_s w_s O_s, four head-dim elements per thread and step;
                // four steps' loads are issued before their sums
                constexpr int kQ = D / 4;
                constexpr int kEt = kSkEpiWarps * 32;
                const int total = w.ncol * kQ;
                const size_t split_stride = (size_t)p.total_rows * p.H * D;
                for (int base = 0; base < total; base += 4 * kEt) {
                    float4 acc[4];
                    size_t idx[4];
                    int cc[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int q = base + u * kEt + (int)threadIdx.x;
                        const bool act = q < total;
                        cc[u] = act ? q / kQ : -1;
                        const int c = act ? cc[u] : 0;
                        // column c: candidate c / G, query head w.h * G + c % G
                        idx[u] = ((size_t)(w.tok0 + c / p.G) * p.H + w.h * p.G + c % p.G) * D + (q % kQ) * 4;
                        const size_t vidx = ((size_t)(w.tok0 + c / p.G) * hkv + w.h) * D + (q % kQ) * 4;
                        acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (act) {
                            const uint2 vb = __ldg(reinterpret_cast<const uint2*>(p.v_self + vidx));
                            const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vb.x));
                            const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vb.y));
                            const float cbv = coef_b[c];
                            acc[u] = make_float4(cbv * v01.x, cbv * v01.y, cbv * v23.x, cbv * v23.y);
                        }
                    }
#pragma unroll
                    for (int s = 0; s < kSkMaxSplit; ++s) {
                        if (s < w.npieces) {
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                if (cc[u] >= 0) {
                                    const float4 pv =
                                        __ldcg(reinterpret_cast<const float4*>(p.part_o + s * split_stride + idx[u]));
                                    const float wv = wts[s * N + cc[u]];
                                    acc[u].x = fmaf(wv, pv.x, acc[u].x);
                                    acc[u].y = fmaf(wv, pv.y, acc[u].y);
                                    acc[u].z = fmaf(wv, pv.z, acc[u].z);
                                    acc[u].w = fmaf(wv, pv.w, acc[u].w);
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (cc[u] >= 0) sk_store4(p.out, p.out_fp32, idx[u], acc[u]);
                }
            }
            // last_flag, coef_b and wts are reused by the next item
            if (!(ok = warp_group_sync(egrp, negrp, ctl, lane))) break;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kSkMmaWarp) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace unipin
