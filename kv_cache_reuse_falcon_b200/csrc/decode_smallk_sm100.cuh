// Rank decode for small candidate counts (k <= 128 per request), sm_100a.
//
// The rank decode of [review] §2.4 / [notes] §6: the k candidates of request r
// attend to pool rows 0..n_r-1 of slot s_r (layer l, head h) and to
// themselves.  With few candidates a request is a stream of cached K/V rows
// read once against a handful of queries, so the pass is bound by HBM, not by
// the tensor cores.  This kernel therefore puts the KEYS on the MMA's M
// dimension, so no tensor-core row and no softmax thread is spent on padding
// candidates:
//
//   S^T = K Q^T   M = 128 keys, N = k padded to 16/32/64/128, K = D
//   O  += P V     M = 128 candidate rows (rows past the padded count are
//                 discarded), N = D, K = 128 keys; P (bf16) is staged through
//                 shared memory in the 128-byte-swizzled K-major layout of a
//                 query tile, V is read MN-major as the prefill reads it
//
// Softmax thread t owns key t of a tile (TMEM lane t): it loads that key's N
// scores, and the per-candidate statistics are reductions over threads.  The
// reference maximum of each candidate moves only when some score would
// exceed it by more than 2^8 (one vote per tile among the four softmax warps;
// the exact column maxima are computed only then), so the common tile costs
// N scalings, N exponentials, N two-byte stores of P and one warp
// reduce-scatter of the column sums.  O accumulates in TMEM with lane =
// candidate, so the epilogue thread of candidate c reads its own row.
//
// Work item = (request, head, key split).  The key range of a request is cut
// into `nsplit` runs of whole 128-key tiles so that every SM has several
// items; each item leaves an unnormalised partial (O, m, l) per candidate in
// the caller's workspace, and the last item of a (request, head) to finish -
// found with a per-pair arrival counter - merges the partials with the
// candidate's own key (self term) and writes the output.  With one split the
// item writes the output directly.
//
// Warp roles (192 threads, two blocks per SM where shared memory and TMEM
// allow, so one block's per-item latencies hide behind the other's stream):
//   warps 0-3  softmax and epilogue (thread t: key t of a tile; candidate t's
//              output row in the epilogue)
//   warp 4     TMA producer: claims items, loads Q (N candidate rows) and the
//              V and K tiles of each key tile into a ring of stages
//   warp 5     MMA issuer (one elected thread), owns TMEM
// Every wait is bounded (see sm100_ptx.cuh); a block that gives up reports
// UNIPIN_ERR_DEVICE_TIMEOUT and exits cleanly.
#pragma once

#include "sm100_ptx.cuh"
#include "tmem_wide.cuh"
#include "unipin.h"

namespace unipin {

constexpr int kSkKeys = 128;        // keys per tile (the MMA's M)
constexpr int kSkThreads = 192;
constexpr int kSkItemSlots = 4;
constexpr int kSkConsumers = 5;     // the MMA warp and the four softmax warps pop every item
constexpr int kSkMaxSplit = 16;     // key splits per (request, head) at most
constexpr float kSkRescaleLog2 = 8.0f;

// Candidate columns the kernel is compiled for, given the largest k.
__host__ __device__ constexpr int sk_pad_n(int k) { return k <= 16 ? 16 : k <= 32 ? 32 : k <= 64 ? 64 : 128; }
__host__ __device__ constexpr int sk_tmem_cols(int c) { return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512; }

template <int D, int N>
struct SkCfg {
    static_assert(D == 64 || D == 128, "small-k decode: head dim 64 or 128");
    static_assert(N == 16 || N == 32 || N == 64 || N == 128, "small-k decode: padded candidate count");
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
    // TMEM columns: S^T buffers at 0 and N, O (D columns) at 2N.
    static constexpr int kColO = 2 * N;
    static constexpr int kTmemCols = sk_tmem_cols(2 * N + D);
    static constexpr int kCtasPerSm = (D == 64 && kTmemCols <= 256) ? 2 : 1;
    // Scratch floats: red[4][N], mref[N], corr[N], coef_b[N], flags[2][4],
    // selfs[kSkItemSlots][N]; merge weights reuse a P buffer.
    static constexpr int kScratchBytes = ((4 * N + 3 * N + 8 + kSkItemSlots * N) * 4 + 1023) / 1024 * 1024;
    static constexpr int kBarBytes = 1024;
    static constexpr int kBudget = kCtasPerSm == 2 ? 112 * 1024 : 226 * 1024;
    // Double-buffer Q (the next item's Q loads during this item) and P^T (the
    // softmax writes P_{i+1} while P.V of tile i runs) where a two-stage ring
    // still fits; single buffers otherwise.
    static constexpr int fixed_bytes(int qbufs, int pbufs)
    {
        return qbufs * kQBytes + pbufs * kPBytes + kScratchBytes + kBarBytes;
    }
    static constexpr bool fits(int qbufs, int pbufs) { return kBudget - fixed_bytes(qbufs, pbufs) >= 2 * kStageBytes; }
    static constexpr int kQBufs = fits(2, 1) ? 2 : 1;
    static constexpr int kPBufs = fits(kQBufs, 2) ? 2 : 1;
    static constexpr int kStagesFit = (kBudget - fixed_bytes(kQBufs, kPBufs)) / kStageBytes;
    static constexpr int kStages = kStagesFit > 6 ? 6 : kStagesFit;
    static_assert(kStages >= 2, "small-k decode: ring depth");
    static constexpr int kOffP = 0;                                  // first: the 128-row reads overhang
    static constexpr int kOffRing = kPBufs * kPBytes;                // into the ring that follows
    static constexpr int kOffQ = kOffRing + kStages * kStageBytes;
    static constexpr int kOffScratch = kOffQ + kQBufs * kQBytes;
    static constexpr int kOffBar = kOffScratch + kScratchBytes;
    static constexpr int kSmemBytes = kOffBar + kBarBytes;
    static_assert(kSmemBytes <= kBudget, "small-k decode: shared memory budget");
    static_assert(kSkMaxSplit * N * 4 <= kPBytes, "merge weights fit a P buffer");
    static_assert((kPBufs - 1) * kPBytes + kPBox + kSkKeys * 128 <= kSmemBytes, "P box reads stay in shared memory");
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
    int nsplit, tiles_per_split;
    float sl2;                     // scale * log2(e)
    int* status;
    unsigned long long wait_limit_ns;
    unsigned long long* sched;     // zeroed item counter or null (static striding)
};

// What every role derives identically from an item index.  An item is a
// (request, key/value head, run of key tiles); its candidate columns are the
// pairs (candidate c, query head g of the group) in the order n = c * G + g.
struct SkWork {
    bool rows_ok;   // the request's candidate rows are addressable (cu in range, k * G <= N)
    bool valid;     // rows_ok and slot / history length in range
    int r, h, split, pair;   // h: the key/value head
    int tok0, kc, npast, slot;
    int ncol;                // valid candidate columns, kc * G
    int nt_all;     // key tiles covering [0, npast)
    int t_begin, nt;
};

template <int N>
__device__ __forceinline__ SkWork sk_make_work(const SkParams& p, long long g)
{
    SkWork w;
    w.pair = (int)(g / p.nsplit);
    w.split = (int)(g - (long long)w.pair * p.nsplit);
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
    w.t_begin = min(w.split * p.tiles_per_split, w.nt_all);
    const int t_end = min(w.t_begin + p.tiles_per_split, w.nt_all);
    w.nt = (w.valid && w.kc > 0) ? t_end - w.t_begin : 0;
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

template <int D, int N>
__global__ void __launch_bounds__(kSkThreads, SkCfg<D, N>::kCtasPerSm)
    decode_smallk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const SkParams p)
{
    using C = SkCfg<D, N>;
    constexpr int NS = C::kStages;
    constexpr int NP = C::kPBufs;
    constexpr int NQ = C::kQBufs;
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
    float* red = reinterpret_cast<float*>(smem + C::kOffScratch);   // [4][N]
    float* mref = red + 4 * N;                                      // [N] reference max (log2 units)
    float* corr = mref + N;                                         // [N]
    float* coef_b = corr + N;                                       // [N] merge: weight of the own value
    volatile int* flags = reinterpret_cast<volatile int*>(coef_b + N);   // [2][4]
    float* selfs = coef_b + N + 8;                                  // [kSkItemSlots][N] own scores, per item slot
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_q = bars + 0;            // [2] Q buffer landed
    uint64_t* q_empty = bars + 2;          // [2] the last S MMA of the item using Q buffer b finished
    uint64_t* s_full = bars + 4;           // [2] S^T buffer computed
    uint64_t* s_free = bars + 6;           // [2] S^T buffer read out (4 softmax warps)
    uint64_t* p_full = bars + 8;           // [2] P^T buffer written (4 softmax warps)
    uint64_t* pv_done = bars + 10;         // [2] O^T += V^T P^T of P buffer b finished
    uint64_t* grp = bars + 12;             // softmax-group barrier (4 warps)
    uint64_t* bar_drain = bars + 13;
    uint64_t* kv_full = bars + 14;         // [NS]
    uint64_t* kv_empty = kv_full + NS;     // [NS]
    uint64_t* item_full = kv_empty + NS;   // [kSkItemSlots]
    uint64_t* item_empty = item_full + kSkItemSlots;
    volatile long long* item_ring = reinterpret_cast<volatile long long*>(item_empty + kSkItemSlots);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_empty + 2 * kSkItemSlots);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_q + b, 1);
            mbar_init(q_empty + b, 1);
            mbar_init(s_full + b, 1);
            mbar_init(s_free + b, 4);
            mbar_init(p_full + b, 4);
            mbar_init(pv_done + b, 1);
        }
        mbar_init(grp, 4);
        mbar_init(bar_drain, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(kv_full + s, 1);
            mbar_init(kv_empty + s, 1);
        }
        for (int s = 0; s < kSkItemSlots; ++s) {
            mbar_init(item_full + s, 1);
            mbar_init(item_empty + s, kSkConsumers);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (threadIdx.x < N) mref[threadIdx.x] = -INFINITY;
    if (warp == 5) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns, (int)UNIPIN_ERR_DEVICE_TIMEOUT};
    const long long total_items = (long long)p.R * (p.H / p.G) * p.nsplit;
    int n_items = 0;
    // Consumers: the next item (warp-uniform); `own` receives selfs[slot][own_col] read
    // before the slot is released (the producer may refill it right after).
    auto pop_item = [&](bool& ok, long long& g, int own_col, float& own) -> bool {
        const int si = n_items % kSkItemSlots;
        ok = __all_sync(0xffffffffu, mbar_wait(item_full + si, (n_items / kSkItemSlots) & 1, ctl));
        if (!ok) return false;
        g = item_ring[si];
        own = (own_col >= 0 && own_col < N) ? selfs[si * N + own_col] : -INFINITY;
        __syncwarp();
        if (lane == 0) mbar_arrive(item_empty + si);
        ++n_items;
        return g >= 0;
    };
    const bool leader = lane == 0;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (leader) {
            tma_prefetch_map(&tm_q);
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
        }
        int u = 0, nq = 0;
        bool ok = true;
        long long g_static = blockIdx.x;
        while (ok) {
            const int si = n_items % kSkItemSlots;
            if (n_items >= kSkItemSlots) {
                ok = __all_sync(0xffffffffu, mbar_wait(item_empty + si, ((n_items / kSkItemSlots) - 1) & 1, ctl));
                if (!ok) break;
            }
            long long g = 0;
            if (p.sched) {
                if (leader) g = (long long)atomicAdd(p.sched, 1ull);
                g = __shfl_sync(0xffffffffu, g, 0);
            } else {
                g = g_static;
                g_static += gridDim.x;
            }
            const bool found = g < total_items;
            SkWork w;
            if (found) {
                // the own score of every candidate column (log2 units), off the softmax warps' path
                w = sk_make_work<N>(p, g);
                if (w.valid) {
                    const int hkv = p.H / p.G;
                    for (int n = lane; n < w.ncol; n += 32) {
                        const size_t qrow = (size_t)(w.tok0 + n / p.G) * p.H + w.h * p.G + n % p.G;
                        const size_t kvrow = (size_t)(w.tok0 + n / p.G) * hkv + w.h;
                        selfs[si * N + n] = p.sl2 * sk_dot_bf16<D>(p.q + qrow * D, p.k_self + kvrow * D);
                    }
                }
                __syncwarp();
            }
            if (leader) {
                item_ring[si] = found ? g : -1;
                mbar_arrive(item_full + si);   // release: the consumers see selfs[si] with the item
            }
            ++n_items;
            if (!found) break;
            if (w.nt == 0) continue;
            const int qb = nq % NQ;
            if (nq >= NQ) {
                ok = __all_sync(0xffffffffu, mbar_wait(q_empty + qb, ((nq / NQ) - 1) & 1, ctl));
                if (!ok) break;
            }
            if (leader) {
                mbar_arrive_expect_tx(bar_q + qb, C::kQBytes);
                for (int c = 0; c < C::kChunks; ++c)
                    // N / G candidate tokens x the G query heads of key/value head w.h
                    tma_load_3d(sQ + qb * C::kQBytes + c * C::kAtomQ, &tm_q, bar_q + qb, c * 64, w.h * p.G, w.tok0);
            }
            ++nq;
            const int plane = (p.layer * p.S + w.slot) * (p.H / p.G) + w.h;
            for (int i = 0; ok && i < w.nt; ++i) {
                const int start = sk_tile_start(w.t_begin + i, w.nt_all, w.npast);
                const int st = u % NS;
                if (u >= NS) {
                    ok = __all_sync(0xffffffffu, mbar_wait(kv_empty + st, ((u / NS) - 1) & 1, ctl));
                    if (!ok) break;
                }
                if (leader) {
                    uint8_t* dst = ring + st * C::kStageBytes;
                    mbar_arrive_expect_tx(kv_full + st, C::kStageBytes);
                    for (int c = 0; c < C::kChunks; ++c) {
                        tma_load_3d(dst + c * C::kAtom, &tm_v, kv_full + st, c * 64, start, plane);
                        tma_load_3d(dst + C::kTileKV + c * C::kAtom, &tm_k, kv_full + st, c * 64, start, plane);
                    }
                }
                ++u;
            }
        }
        if (!ok && leader) {
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
            for (int v = (u > NS ? u - NS : 0); v < u; ++v)
                mbar_wait_drain(kv_full + v % NS, (v / NS) & 1, p.wait_limit_ns);
            for (int v = (nq > NQ ? nq - NQ : 0); v < nq; ++v)
                mbar_wait_drain(bar_q + v % NQ, (v / NQ) & 1, p.wait_limit_ns);
            for (int v = (n_items > kSkItemSlots ? n_items - kSkItemSlots : 0); v < n_items; ++v)
                mbar_wait_drain(item_empty + v % kSkItemSlots, (v / kSkItemSlots) & 1, p.wait_limit_ns);
        }
    } else if (warp == 5) {
        // --------------------------------------------------------- MMA issuer
        // Per key tile i: S^T_i = K_i Q^T, then O^T += V_{i-1}^T P^T_{i-1} once
        // the softmax has written P_{i-1}; so S_{i+1} is computed while the
        // softmax works on S_i.
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kSkKeys, N, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true, false);
        const uint32_t ring_a = smem_u32(ring);
        // K (A of S^T): K-major, 128-byte rows, 8-row groups 1024 bytes apart.
        const uint64_t dk0 = smem_desc(ring_a + C::kTileKV, 16, 1024, kLayoutSw128);
        // V (B of O += P V, MN-major): 64-element head-dim blocks 16 KB apart,
        // 8-key groups 1024 bytes apart.
        const uint64_t dv0 = smem_desc(ring_a, C::kAtom, 1024, kLayoutSw128);
        const uint64_t dq0 = smem_desc(smem_u32(sQ), 16, 1024, kLayoutSw128);
        // P (A of O += P V): K-major rows of 64 keys per box, 8-row groups 1024 bytes apart.
        const uint64_t dp0 = smem_desc(smem_u32(sP), 16, 1024, kLayoutSw128);
        const uint32_t tO = tmem + C::kColO;
        int u = 0, nq = 0;
        int gs = 0;            // S tiles issued
        int gp = 0;            // P.V products issued
        int pfull_seen[2] = {0, 0};
        bool ok = true;
        long long g;
        auto issue_pv = [&](int st, int pb, bool acc) {
            // K-steps of 16 keys: 32 bytes within a P row (then the second box), 16 V rows
#pragma unroll
            for (int kk = 0; kk < kSkKeys / 16; ++kk) {
                const uint64_t a = dp0 + (uint64_t)((pb * C::kPBytes + (kk / 4) * C::kPBox + (kk % 4) * 32) >> 4);
                const uint64_t b = dv0 + (uint64_t)((st * C::kStageBytes + kk * 2048) >> 4);
                umma_bf16_ss(tO, a, b, idesc_pv, (acc || kk > 0) ? 1u : 0u);
            }
            umma_commit(pv_done + pb);
            umma_commit(kv_empty + st);
        };
        auto wait_p = [&](int gidx) {
            const int pb = gidx % NP;
            const int n = gidx / NP;
            bool r = true;
            while (r && pfull_seen[pb] <= n) {
                r = __all_sync(0xffffffffu, mbar_wait(p_full + pb, pfull_seen[pb] & 1, ctl));
                ++pfull_seen[pb];
            }
            tc_fence_after_sync();
            return r;
        };
        float unused_own;
        while (pop_item(ok, g, -1, unused_own)) {
            const SkWork w = sk_make_work<N>(p, g);
            if (w.nt == 0) continue;
            const int qb = nq % NQ;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_q + qb, (nq / NQ) & 1, ctl));
            if (!ok) break;
            ++nq;
            for (int i = 0; ok && i < w.nt; ++i) {
                // S_i needs K_i landed and an S buffer the softmax has read out; P.V of
                // tile i-1 needs P_{i-1}.  Issue each as soon as its inputs are there: a
                // P.V queued behind the next tile's data would hold its ring stage, and
                // the ring would then have a single load in flight.
                const int st = (u + i) % NS;
                const int sb = gs & 1;
                bool need_qk = true;
                bool need_pv = i >= 1;
                const uint64_t t0 = global_timer_ns();
                for (uint32_t spin = 1; need_qk || need_pv; ++spin) {
                    if (need_pv) {
                        const int pb = gp % NP;
                        if (__all_sync(0xffffffffu, mbar_test_wait(p_full + pb, pfull_seen[pb] & 1))) {
                            ++pfull_seen[pb];
                            tc_fence_after_sync();
                            if (leader) issue_pv((u + i - 1) % NS, pb, i - 1 > 0);
                            ++gp;
                            need_pv = false;
                        }
                    }
                    if (need_qk && __all_sync(0xffffffffu, mbar_test_wait(kv_full + st, ((u + i) / NS) & 1) &&
                                                              (gs < 2 || mbar_test_wait(s_free + sb, ((gs >> 1) - 1) & 1)))) {
                        tc_fence_after_sync();
                        if (leader) {
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const int box = kk / 4;
                                const int in_row = (kk % 4) * 32;
                                const uint64_t a =
                                    dk0 + (uint64_t)((st * C::kStageBytes + box * C::kAtom + in_row) >> 4);
                                const uint64_t b = dq0 + (uint64_t)((qb * C::kQBytes + box * C::kAtomQ + in_row) >> 4);
                                umma_bf16_ss(tmem + sb * N, a, b, idesc_qk, kk > 0 ? 1u : 0u);
                            }
                            umma_commit(s_full + sb);
                            if (i == w.nt - 1) umma_commit(q_empty + qb);
                        }
                        ++gs;
                        need_qk = false;
                    }
                    if ((spin & 31) == 0) {
                        // warp-uniform: every lane leaves the loop together
                        const bool aborted = *abort_flag != 0;
                        const bool stop = __any_sync(0xffffffffu, aborted || global_timer_ns() - t0 > p.wait_limit_ns);
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
            if (!ok) break;
            if (!(ok = wait_p(gp))) break;
            if (leader) issue_pv((u + w.nt - 1) % NS, gp % NP, w.nt > 1);
            ++gp;
            u += w.nt;
        }
        if (leader) {
            umma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.wait_limit_ns);
        }
    } else {
        // ------------------------------------------------- softmax + epilogue
        const int t = threadIdx.x;                               // key of a tile / candidate row of O
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sl2 = p.sl2;
        int gs = 0, gp = 0;
        int pv_seen[2] = {0, 0};
        uint32_t ngrp = 0;
        bool ok = true;
        long long g;
        // Wait until the P.V product with global index gidx has finished
        // (completions of each P buffer are consumed in order).
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
        float own_popped;
        while (pop_item(ok, g, threadIdx.x, own_popped)) {
            const SkWork w = sk_make_work<N>(p, g);
            if (!w.rows_ok) {
                if (t == 0) report(p.status, (int)UNIPIN_ERR_OUT_OF_RANGE);
                continue;
            }
            if (!w.valid && t == 0 && w.split == 0) report(p.status, (int)UNIPIN_ERR_OUT_OF_RANGE);
            // Column t = (candidate t / G, query head w.h * G + t % G): its output row, its own
            // key/value row, and its own score (log2 units), taken while the first tile is in flight.
            const int hkv = p.H / p.G;
            const size_t qrow = (size_t)(w.tok0 + t / p.G) * p.H + w.h * p.G + t % p.G;
            const size_t kvrow = (size_t)(w.tok0 + t / p.G) * hkv + w.h;
            const float ss_own = (t < w.ncol && w.valid) ? own_popped : -INFINITY;
            // per-thread partial column sums of P (owned columns), relative to mref
            constexpr int kOwn = N >= 32 ? N / 32 : 1;
            float lown[kOwn];
#pragma unroll
            for (int e = 0; e < kOwn; ++e) lown[e] = 0.f;
            for (int i = 0; i < w.nt; ++i) {
                const int tile = w.t_begin + i;
                const int lo = tile * kSkKeys;
                const int start = sk_tile_start(tile, w.nt_all, w.npast);
                const int key = start + t;
                const bool key_ok = key >= lo && key < w.npast;
                const int sb = gs & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(s_full + sb, (gs >> 1) & 1, ctl));
                if (!ok) break;
                tc_fence_after_sync();
                uint32_t sraw[N];
                tmem_ld_n<N>(lane_base + sb * N, sraw);
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_free + sb);
                ++gs;
                float x[N];
#pragma unroll
                for (int c = 0; c < N; ++c)
                    x[c] = (key_ok && c < w.ncol) ? __uint_as_float(sraw[c]) * sl2 : -INFINITY;
                // vote: does any score exceed its candidate's reference max by > 2^8?
                bool need = false;
#pragma unroll
                for (int c = 0; c < N; c += 4) {
                    const float4 m4 = *reinterpret_cast<const float4*>(mref + c);
                    need |= x[c] > m4.x + kSkRescaleLog2;
                    need |= x[c + 1] > m4.y + kSkRescaleLog2;
                    need |= x[c + 2] > m4.z + kSkRescaleLog2;
                    need |= x[c + 3] > m4.w + kSkRescaleLog2;
                }
                const int fb = ngrp & 1;
                const int warp_need = __any_sync(0xffffffffu, need) ? 1 : 0;
                if (lane == 0) flags[fb * 4 + warp] = warp_need;
                if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
                const bool any_need = (flags[fb * 4 + 0] | flags[fb * 4 + 1] | flags[fb * 4 + 2] | flags[fb * 4 + 3]) != 0;
                if (any_need) {
                    // exact column maxima of this tile; move every reference max to it
                    float cm[N];
#pragma unroll
                    for (int c = 0; c < N; ++c) cm[c] = x[c];
                    sk_rs_step<N, 16, true>(cm, lane);
#pragma unroll
                    for (int e = 0; e < kOwn; ++e)
                        if (N >= 32 || (lane & 1) == 0) red[warp * N + sk_owned_col<N>(lane, e)] = cm[e];
                    if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
                    if (t < N) {
                        const float mt = fmaxf(fmaxf(red[t], red[N + t]), fmaxf(red[2 * N + t], red[3 * N + t]));
                        const float mo = mref[t];
                        const float mn = fmaxf(mo, mt);
                        corr[t] = (mo == -INFINITY) ? 0.f : ex2_approx(mo - mn);
                        mref[t] = mn;
                    }
                    if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
#pragma unroll
                    for (int e = 0; e < kOwn; ++e) lown[e] *= corr[sk_owned_col<N>(lane, e)];
                    if (i > 0) {
                        // rescale the O rows accumulated so far (after the last P.V): row c is candidate c
                        if (!(ok = wait_pv(gp - 1))) break;
                        if (warp * 32 < N) {
                            const float cf = corr[t < N ? t : 0];
#pragma unroll
                            for (int c0 = 0; c0 < D; c0 += 16) {
                                uint32_t o[16];
                                tmem_ld16(lane_base + C::kColO + c0, o);
#pragma unroll
                                for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * cf);
                                tmem_st16(lane_base + C::kColO + c0, o);
                            }
                        }
                    }
                }
                // P = 2^(x - m)
                float ps[N];
#pragma unroll
                for (int c = 0; c < N; c += 4) {
                    const float4 m4 = *reinterpret_cast<const float4*>(mref + c);
                    const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float mu = mm[e] == -INFINITY ? 0.f : mm[e];
                        ps[c + e] = ex2_approx(x[c + e] - mu);
                    }
                }
                // the P buffer is free once the P.V that last read it has finished
                const int pb = gp % NP;
                if (!(ok = wait_pv(gp - NP))) break;
                // column t of P: key t of the tile is element t % 64 of a 128-byte row of box t / 64
                {
                    uint8_t* pbox = sP + pb * C::kPBytes + (t / 64) * C::kPBox;
                    const int kx = t % 64;
#pragma unroll
                    for (int c = 0; c < N; ++c)
                        *reinterpret_cast<__nv_bfloat16*>(pbox + c * 128 + ((((kx >> 3) ^ (c & 7))) << 4) +
                                                          (kx & 7) * 2) = __float2bfloat16_rn(ps[c]);
                }
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full + pb);
                ++gp;
                sk_rs_step<N, 16, false>(ps, lane);
#pragma unroll
                for (int e = 0; e < kOwn; ++e) lown[e] += ps[e];
            }
            if (!ok) break;
            // ------------------------------------------------------ epilogue
            // the own value row is fetched before the last wait, so its latency overlaps it
            // (where registers allow: the widest variant keeps it in the store loop)
            constexpr bool kPrefetchV = N <= 32;
            uint4 vrow[kPrefetchV ? D / 8 : 1];
            if (kPrefetchV && p.nsplit == 1 && t < w.ncol) {
                const uint4* v4 = reinterpret_cast<const uint4*>(p.v_self + kvrow * D);
#pragma unroll
                for (int d8 = 0; d8 < D / 8; ++d8) vrow[d8] = __ldg(v4 + d8);
            }
            if (w.nt > 0 && !(ok = wait_pv(gp - 1))) break;
#pragma unroll
            for (int e = 0; e < kOwn; ++e)
                if (N >= 32 || (lane & 1) == 0) red[warp * N + sk_owned_col<N>(lane, e)] = lown[e];
            if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
            // thread t < N: candidate t's sum, max and output coefficients
            float m_c = -INFINITY, l_c = 0.f, ca = 0.f, cb = 0.f;
            if (t < N) {
                l_c = red[t] + red[N + t] + red[2 * N + t] + red[3 * N + t];
                m_c = w.nt > 0 ? mref[t] : -INFINITY;
                mref[t] = -INFINITY;   // ready for the next item
                if (p.nsplit == 1 && t < w.ncol && w.valid) {
                    // final: (a O + b v_self) / (a l + b)
                    const float mf = fmaxf(m_c, ss_own);
                    const float a = (m_c == -INFINITY) ? 0.f : ex2_approx(m_c - mf);
                    const float b = ex2_approx(ss_own - mf);
                    const float inv = 1.f / (l_c * a + b);
                    ca = a * inv;
                    cb = b * inv;
                }
            }
            // O row t = candidate t (warp-collective load where the warp holds candidate rows)
            uint32_t o[D];
            if (w.nt > 0 && warp * 32 < N) {
                if constexpr (D == 64) tmem_ld64(lane_base + C::kColO, o);
                else tmem_ld128(lane_base + C::kColO, o);
            } else {
#pragma unroll
                for (int d = 0; d < D; ++d) o[d] = 0u;
            }
            tc_fence_before_sync();
            if (t < w.ncol) {
                const size_t row = qrow;
                if (p.nsplit == 1) {
#pragma unroll
                    for (int d8 = 0; d8 < D / 8; ++d8) {
                        uint4 vb;
                        if constexpr (kPrefetchV) vb = vrow[d8];
                        else vb = __ldg(reinterpret_cast<const uint4*>(p.v_self + kvrow * D) + d8);
                        const __nv_bfloat162* vh = reinterpret_cast<const __nv_bfloat162*>(&vb);
                        float r[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 vf = __bfloat1622float2(vh[e]);
                            r[2 * e] = __uint_as_float(o[d8 * 8 + 2 * e]) * ca + cb * vf.x;
                            r[2 * e + 1] = __uint_as_float(o[d8 * 8 + 2 * e + 1]) * ca + cb * vf.y;
                        }
                        sk_store4(p.out, p.out_fp32, row * D + d8 * 8, make_float4(r[0], r[1], r[2], r[3]));
                        sk_store4(p.out, p.out_fp32, row * D + d8 * 8 + 4, make_float4(r[4], r[5], r[6], r[7]));
                    }
                } else {
                    float* po = p.part_o + ((size_t)w.split * p.total_rows * p.H + row) * D;
#pragma unroll
                    for (int d = 0; d < D; d += 4)
                        *reinterpret_cast<float4*>(po + d) =
                            make_float4(__uint_as_float(o[d]), __uint_as_float(o[d + 1]), __uint_as_float(o[d + 2]),
                                        __uint_as_float(o[d + 3]));
                    float* ml = p.part_ml + ((size_t)w.split * p.total_rows * p.H + row) * 2;
                    ml[0] = w.valid ? m_c : -INFINITY;
                    ml[1] = w.valid ? l_c : 0.f;
                }
            }
            if (p.nsplit > 1) {
                // publish the partial; the last split of this (request, head) to arrive merges
                __threadfence();
                if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
                if (t == 0) {
                    const unsigned prev = atomicAdd(p.pair_cnt + w.pair, 1u);
                    *last_flag = prev == (unsigned)(p.nsplit - 1);
                }
                if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
                if (*last_flag) {
                    __threadfence();
                    float* wts = reinterpret_cast<float*>(sP + (gp % NP) * C::kPBytes);   // [kSkMaxSplit][N]
                    if (t < w.ncol) {
                        // weights of the splits and of the own key: LSE merge in log2 units
                        const size_t row = qrow;
                        float ms[kSkMaxSplit], ls[kSkMaxSplit];
#pragma unroll
                        for (int s = 0; s < kSkMaxSplit; ++s) {
                            float2 ml = make_float2(-INFINITY, 0.f);
                            if (s < p.nsplit)
                                ml = __ldcg(reinterpret_cast<const float2*>(
                                    p.part_ml + ((size_t)s * p.total_rows * p.H + row) * 2));
                            ms[s] = ml.x;
                            ls[s] = ml.y;
                        }
                        float mf = ss_own;
#pragma unroll
                        for (int s = 0; s < kSkMaxSplit; ++s) mf = fmaxf(mf, ms[s]);
                        const float b = ex2_approx(ss_own - mf);
                        float den = b;
                        float a[kSkMaxSplit];
#pragma unroll
                        for (int s = 0; s < kSkMaxSplit; ++s) {
                            a[s] = (ms[s] == -INFINITY || !(ls[s] > 0.f)) ? 0.f : ex2_approx(ms[s] - mf);
                            den = fmaf(a[s], ls[s], den);
                        }
                        // a rejected request (no own score: every term -inf) gets zero weights
                        const float inv = w.valid ? 1.f / den : 0.f;
#pragma unroll
                        for (int s = 0; s < kSkMaxSplit; ++s)
                            if (s < p.nsplit) wts[s * N + t] = w.valid ? a[s] * inv : 0.f;
                        coef_b[t] = w.valid ? b * inv : 0.f;
                    }
                    if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
                    // out = b v_self + sum_s w_s O_s, four head-dim elements per thread and step;
                    // four steps' loads are issued before their sums
                    constexpr int kQ = D / 4;
                    const int total = w.ncol * kQ;
                    const size_t split_stride = (size_t)p.total_rows * p.H * D;
                    for (int base = 0; base < total; base += 4 * 128) {
                        float4 acc[4];
                        size_t idx[4];
                        int cc[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int q = base + u * 128 + t;
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
                            if (s < p.nsplit) {
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
            }
            // scratch (red, weights) is reused by the next item
            if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace unipin
