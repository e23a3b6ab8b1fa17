// M-FALCON masked attention engine for sm_100a.
//
// Work item = (segment, head, pair of 128-row query tiles A and B[, key split]).
// The two tiles share every K/V tile; each has its own softmax warpgroup and
// its own MMA-issuing warp, and the next key tile's S = Q K^T of a tile is
// computed while its softmax works on the current one.  Blocks are
// persistent (one per SM) and take items from the producer warp; the next
// item's Q and first K/V tiles load, and its first S MMAs run, while the
// softmax warpgroups finish the previous item's epilogue.
//
// The same engine runs the prefill and the rank decode.  In both, the part
// of a row's key set that is a contiguous run of keys 0..kmax-1 goes through
// the tensor cores with the causal predicate j <= i, and a candidate's own
// key (the diagonal of the candidate block) is merged in afterwards as a
// per-row fp32 dot product:
//   prefill ([notes] §3 "attention mask"):  past row i sees j <= i < n_b;
//       candidate row i >= n_b sees all j < n_b plus itself (self term).
//   rank decode ([review] §2.4, [notes] §6):  keys are pool rows 0..n_r-1 of
//       the request's slot; every candidate sees all of them plus itself.
// Key tiles past kmax are never visited; key tiles entirely below the
// diagonal and below kmax skip the per-element predicate.
//
// Warp roles (384 threads):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread r owns
//              query row r = TMEM lane r, so the row max and row sum stay in
//              one thread's registers; S is read from TMEM with one wide load,
//              P (bf16) is written to its own TMEM columns and consumed from
//              there by the P.V MMA.  The O accumulator is rescaled in TMEM
//              only when a row max grows by more than 2^8 (stale maxima keep
//              P <= 2^8, exact after the final division).
//              Because P does not overwrite S, the next key tile's S = Q K^T
//              is computed while this tile's softmax runs: the tensor cores
//              never wait for a softmax to finish before starting on the next S.
//   warp 8     TMA producer: claims work items (from a counter in the caller's
//              workspace, or by a fixed stride) and hands them to the other
//              warps through a small shared-memory ring; per item it loads the
//              Q tiles, then K_i and V_i of key tile i together into one slot
//              of a ring of shared-memory slots (the ring runs across items).
//   warps 9, 10 the UMMA issuers of tile A and tile B (one elected thread each);
//              warp 9 also allocates TMEM.  Per key tile each waits only for
//              "S read out" (which also says the next slot has landed) and
//              "P stored": a wait issued right behind MMAs stalls the issuing
//              warp until they drain, so the fewer the better.
//   warp 11    pool writer (prefill with a pool): each segment's last query-tile
//              pair loads every past K/V tile of its head exactly once, and this
//              warp copies those tiles from the ring into the segment's pool
//              slot; it releases every ring use as the third arrival of the
//              slot's empty barrier.
// Every warp maps a global item index to its segment with the same
// warp-cooperative walker (ItemWalker).
//
// Key tiles are kN = 64 keys wide at D = 128 and 128 keys otherwise, so that
// each query tile's S (kN columns), P (kN/2 columns of bf16 pairs) and O (D
// columns) fit its half of the 512 TMEM columns:
//   tile X: S at 256X, P at 256X + kN, O at 256X + 256 - D.
#pragma once

#include "sm100_ptx.cuh"
#include "tmem_wide.cuh"
#include "unipin.h"

namespace unipin {

constexpr int kBlockM = 128;     // query rows per tile = TMEM lanes
constexpr int kPairRows = 2 * kBlockM;
constexpr int kThreads = 384;
// Register split: the block launches with kLaunchRegs per thread (the most
// 384 threads can have); the producer/MMA warpgroup gives registers back and
// the two softmax warpgroups take them (per head dim, in AttnCfg).
constexpr int kLaunchRegs = 168;
constexpr int kItemSlots = 4;        // items handed from the producer warp to the others
constexpr int kItemConsumers = 11;   // the two MMA warps, the eight softmax warps, the pool writer
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;   // rescale O only when a row max grows by > 2^8

// Key tile width (keys per S tile).  The prefill takes 64 keys at every head
// dim: a shorter softmax loop per tile (less code for the instruction cache,
// finer pipelining); the rank decode through this engine (many candidates)
// takes 128 keys at D <= 64, which halves its per-tile synchronisation.
__host__ __device__ constexpr int key_tile_width(int D, bool decode) { return (D == 128 || !decode) ? 64 : 128; }

template <int D, bool kDecode>
struct AttnCfg {
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    static constexpr int kN = key_tile_width(D, kDecode);       // keys per K/V tile
    static constexpr int kBoxD = D >= 64 ? 64 : D;              // elements per TMA box row
    static constexpr int kChunks = D / kBoxD;                   // boxes across D
    static constexpr int kRowBytes = kBoxD * 2;                 // 128 (SW128) or 64 (SW64)
    static constexpr uint32_t kLayout = kRowBytes == 128 ? kLayoutSw128 : kLayoutSw64;
    static constexpr int kAtomQ = kBlockM * kRowBytes;          // one box of 128 query rows
    static constexpr int kAtomKV = kN * kRowBytes;              // one box of kN key rows
    static constexpr int kTileQ = kBlockM * D * 2;              // one Q tile
    static constexpr int kTileKV = kN * D * 2;                  // one K or V tile
    static constexpr int kSlotBytes = 2 * kTileKV;              // a ring slot: K and V of one key tile
    static constexpr int kStages = (128 * 1024) / kSlotBytes;   // ring slots
    // Pairs in every four of P's exponentials taken by the FMA-pipe polynomial (the rest
    // by the MUFU ex2).  One in four at every D: two or three in four measured slower at
    // D = 64 (the D = 64 prefill is not bound by the MUFU) and at D = 128.
    static constexpr int kPolyOf4 = 1;
    static constexpr int kOffQ = 0;                             // Q_A, Q_B
    static constexpr int kOffRing = 2 * kTileQ;
    static constexpr int kOffBar = kOffRing + kStages * kSlotBytes;
    static constexpr int kSmemBytes = kOffBar + 512;
    // TMEM columns of tile X's S, P and O, relative to 256 X (O aligned to D)
    static constexpr int kColS = 0;
    static constexpr int kColP = kN;
    static constexpr int kColO = 256 - D;
    static_assert(kColP + kN / 2 <= kColO, "TMEM budget per query tile");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    // Registers per thread of the producer/MMA warpgroup and of the softmax
    // warpgroups: a softmax thread holds a row of kN scores; 128 + 2*128
    // threads share the launch's 384 * 168.
    static constexpr int kRegsOther = kN == 64 ? 152 : 136;
    static constexpr int kRegsSoftmax = kN == 64 ? 176 : 184;
    static_assert(128 * kRegsOther + 256 * kRegsSoftmax <= kThreads * kLaunchRegs, "register split");
};

struct AttnParams {
    const __nv_bfloat16* q;       // [T, H, D] query-side tokens
    const __nv_bfloat16* k_self;  // [T, H, D] key of each query token (self term)
    const __nv_bfloat16* v_self;  // [T, H, D] value of each query token (self term)
    void* out;                    // [T, H, D] fp32 or bf16
    float* part_o;                // split-n partials [nsplit, T, H, D] (decode, nsplit > 1)
    float* part_ml;               // split-n row stats [nsplit, T, H, 2] = (m in log2 units, l)
    const int* cu;                // [nseg + 1]
    const int* past;              // [nseg]
    const int* slots;             // [nseg] (decode)
    int nseg;
    int H;                        // query heads
    int G;                        // query heads per key/value head (H = G * key/value heads)
    int max_rows;                 // host bound on rows per segment
    int total_rows;               // T
    int out_fp32;
    int layer, S, n_cap;          // pool geometry (decode)
    int nsplit;                   // decode: key-range splits per query-tile pair
    float sl2;                    // scale * log2(e)
    int* status;
    unsigned long long wait_limit_ns;
    unsigned long long* sched;    // zeroed item counter (dynamic scheduling) or null (static striding)
    float* lse;                   // [T, H] row statistic log2(sum_j 2^(s_ij * sl2)) or null (prefill)
    int store_pool;               // prefill: also write the past K/V into slots[seg] of the pool
    void* pool_k;                 // [L, S, H, n_cap, D] (prefill pool write)
    void* pool_v;
};

// Key tile t of nt covering keys [0, kmax): tiles are kN wide from key 0;
// a ragged last tile is loaded right-aligned (start = kmax - kN, possibly
// negative: the TMA fills rows before 0 with zeros) so that it never reads
// rows at or beyond kmax; keys below `lo` were already covered and are masked.
template <int kN>
__device__ __forceinline__ void key_tile(int t, int nt, int kmax, int& start, int& lo)
{
    lo = t * kN;
    start = (t == nt - 1 && (kmax % kN) != 0) ? kmax - kN : lo;
}

// Warp-cooperative map from a global item index g (segment-major: the items
// of segment 0, then of segment 1, ...) to its segment.  Every lane of the
// calling warp must call locate() together; all lanes get the same answer.
struct ItemWalker {
    const int* cu;
    int nseg, max_rows, mult;     // mult = items per query-tile pair
    int c0;                       // first segment of the loaded chunk of 32
    long long base;               // items before segment c0
    int cnt, pre;                 // this lane's segment: item count, exclusive prefix in chunk
    int chunk_total;
    int* status;

    __device__ void load_chunk(int lane)
    {
        const int s = c0 + lane;
        int items = 0;
        if (s < nseg) {
            const int len = cu[s + 1] - cu[s];
            if (len < 0 || len > max_rows) {
                report(status, (int)UNIPIN_ERR_OUT_OF_RANGE);   // such a segment yields no item
            } else {
                items = ((len + kPairRows - 1) / kPairRows) * mult;
            }
        }
        int incl = items;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        cnt = items;
        pre = incl - items;
        chunk_total = __shfl_sync(0xffffffffu, incl, 31);
    }

    __device__ void init(const AttnParams& p, int lane)
    {
        cu = p.cu;
        nseg = p.nseg;
        max_rows = p.max_rows;
        mult = p.H * p.nsplit;
        status = p.status;
        c0 = 0;
        base = 0;
        load_chunk(lane);
    }

    // Segment and index within the segment of global item g; g must not
    // decrease between calls.  Returns false when g is past the last item.
    __device__ bool locate(int lane, long long g, int& seg, int& local)
    {
        while (g >= base + chunk_total) {
            if (c0 + 32 >= nseg) return false;
            base += chunk_total;
            c0 += 32;
            load_chunk(lane);
        }
        const long long rel = g - base;
        const unsigned hit = __ballot_sync(0xffffffffu, cnt > 0 && rel >= pre && rel < pre + cnt);
        const int L = __ffs(hit) - 1;
        seg = c0 + L;
        local = (int)(rel - __shfl_sync(0xffffffffu, pre, L));
        return true;
    }
};

// Everything about one item that every role derives identically.
struct Work {
    bool valid;
    bool store;                 // prefill: this item writes the segment's past K/V tiles to the pool
    bool rows_ok;               // the segment's rows lie inside the token tensors
    int seg, h, split;
    int tok0, npast, slot;
    int qrow0;                  // first row of tile A within the segment
    int nrows_a, nrows_b;       // rows of tile A / B (B may have none)
    bool has_b;
    int pos0;                   // mask position of row 0 of tile A
    int kmax_a, kmax_b, kmax;   // key ranges; tile geometry follows kmax
    int nt_all, t_begin;
    int nt_a, nt_b, nt;         // key tiles swept for A, B, and loaded
};

template <bool kDecode, int kN>
__device__ __forceinline__ Work make_work(const AttnParams& p, int seg, int local)
{
    Work w;
    w.seg = seg;
    const int per_pair = p.H * p.nsplit;
    const int pair_rank = local / per_pair;
    const int rest = local - pair_rank * per_pair;
    w.h = rest / p.nsplit;
    w.split = rest - w.h * p.nsplit;
    w.tok0 = p.cu[seg];
    const int nrows_seg = p.cu[seg + 1] - w.tok0;
    w.npast = p.past[seg];
    w.slot = (kDecode || p.store_pool) ? p.slots[seg] : 0;
    w.rows_ok = w.tok0 >= 0 && nrows_seg >= 0 && (long long)w.tok0 + nrows_seg <= (long long)p.total_rows;
    bool bad = !w.rows_ok || w.npast < 0;
    if (kDecode)
        bad = bad || w.slot < 0 || w.slot >= p.S || w.npast > p.n_cap;
    else
        bad = bad || w.npast > nrows_seg;
    w.valid = !bad;
    const int npairs = (nrows_seg + kPairRows - 1) / kPairRows;
    // Prefill: the costliest pair of a segment (the last) comes first.
    const int qp = kDecode ? pair_rank : (npairs - 1 - pair_rank);
    w.qrow0 = qp * kPairRows;
    w.nrows_a = min(kBlockM, nrows_seg - w.qrow0);
    w.nrows_b = min(kBlockM, nrows_seg - w.qrow0 - kBlockM);
    w.has_b = w.nrows_b > 0;
    w.pos0 = kDecode ? w.npast + w.qrow0 : w.qrow0;
    w.kmax_a = kDecode ? w.npast : min(w.qrow0 + w.nrows_a, w.npast);
    w.kmax_b = !w.has_b ? 0 : (kDecode ? w.npast : min(w.qrow0 + kBlockM + w.nrows_b, w.npast));
    // Tile A's range is a prefix of B's with identical tiles (kmax_a < kmax_b
    // only when kmax_a is a multiple of 128, hence of kN).
    w.kmax = w.has_b ? w.kmax_b : w.kmax_a;
    w.nt_all = (w.kmax + kN - 1) / kN;
    w.t_begin = 0;
    int t_end_a = (w.kmax_a + kN - 1) / kN;
    int t_end_b = (w.kmax_b + kN - 1) / kN;
    if (kDecode && p.nsplit > 1) {
        const int per = (w.nt_all + p.nsplit - 1) / p.nsplit;
        w.t_begin = min(w.split * per, w.nt_all);
        t_end_a = min(w.t_begin + per, t_end_a);
        t_end_b = min(w.t_begin + per, t_end_b);
    }
    w.nt_a = max(t_end_a - w.t_begin, 0);
    w.nt_b = w.has_b ? max(t_end_b - w.t_begin, 0) : 0;
    w.nt = w.valid ? max(w.nt_a, w.nt_b) : 0;
    if (!w.valid) w.nt_a = w.nt_b = 0;
    // The segment's last pair sees every past key (kmax = npast) and is its first item.
    w.store = !kDecode && p.store_pool && w.valid && pair_rank == 0 && (w.h % p.G) == 0 && w.slot >= 0 &&
              w.slot < p.S && w.npast <= p.n_cap;
    return w;
}

template <int D, bool kDecode>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_pk,
                    const __grid_constant__ CUtensorMap tm_pv, const AttnParams p)
{
    using C = AttnCfg<D, kDecode>;
    constexpr int NS = C::kStages;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    // A timeout recorded earlier means a block of this or a previous launch
    // gave up; later blocks skip their work instead of waiting again.
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == (int)UNIPIN_ERR_DEVICE_TIMEOUT) return;
    if ((smem_u32(smem) & 1023u) != 0) {   // the layout needs 1024-byte aligned tiles
        if (threadIdx.x == 0) report(p.status, (int)UNIPIN_ERR_CUDA);
        return;
    }
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* ring = smem + C::kOffRing;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_q = bars + 0;           // Q tiles of the current item landed
    uint64_t* q_empty = bars + 1;         // every S MMA of an item finished with Q
    uint64_t* s_full = bars + 2;          // [2] S_X computed
    uint64_t* p_full = bars + 4;          // [2] P_X stored
    uint64_t* pv_done = bars + 6;         // [2] O_X += P_X V finished (P_X free, O_X stable)
    uint64_t* bar_drain = bars + 8;       // [2] (bars + 8, bars + 9)
    uint64_t* s_free = bars + 10;         // [2] S_X read into registers
    uint64_t* kv_full = bars + 12;        // [NS]
    uint64_t* kv_empty = bars + 12 + NS;  // [NS]
    uint64_t* item_full = bars + 12 + 2 * NS;      // [kItemSlots]
    uint64_t* item_empty = item_full + kItemSlots;  // [kItemSlots]
    volatile long long* item_ring = reinterpret_cast<volatile long long*>(item_empty + kItemSlots);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_empty + 2 * kItemSlots);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(q_empty, 2);            // one arrival from each MMA warp
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full + x, 1);
            mbar_init(s_free + x, 4);     // one arrival per softmax warp
            mbar_init(p_full + x, 4);
            mbar_init(pv_done + x, 1);
        }
        mbar_init(bar_drain + 0, 1);
        mbar_init(bar_drain + 1, 1);
        for (int s = 0; s < kItemSlots; ++s) {
            mbar_init(item_full + s, 1);
            mbar_init(item_empty + s, kItemConsumers);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(kv_full + s, 1);
            mbar_init(kv_empty + s, 3);   // each MMA warp and the pool writer
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns, (int)UNIPIN_ERR_DEVICE_TIMEOUT};
    ItemWalker walk;
    walk.init(p, lane);
    int seg, local;
    int n_items = 0;     // items taken from the ring by this warp
    // Consumers: next item from the producer's ring (warp-uniform); false at the end.
    auto pop_item = [&](bool& ok_flag) -> bool {
        const int slot_i = n_items % kItemSlots;
        ok_flag = __all_sync(0xffffffffu, mbar_wait(item_full + slot_i, (n_items / kItemSlots) & 1, ctl));
        if (!ok_flag) return false;
        const long long g = item_ring[slot_i];
        __syncwarp();
        if (lane == 0) mbar_arrive(item_empty + slot_i);
        ++n_items;
        if (g < 0) return false;
        return walk.locate(lane, g, seg, local);
    };

    // The producer and MMA warps run their loops with all 32 lanes (the item
    // walker is warp-collective); waits are taken by every lane and made
    // warp-uniform, and only lane 0 issues copies, MMAs and commits.
    const bool leader = lane == 0;
    if (warp >= 8) {
      setmaxnreg_dec<C::kRegsOther>();   // all four warps of the third warpgroup
      if (warp == 8) {
        // ------------------------------------------------------- producer
        if (leader) {
            tma_prefetch_map(&tm_q);
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
        }
        int u = 0;          // ring uses issued so far (use u lives in slot u % NS)
        int nq = 0;         // Q loads issued so far
        bool ok = true;
        long long g_static = blockIdx.x;
        while (ok) {
            // claim the next item and hand it to the other warps
            const int slot_i = n_items % kItemSlots;
            if (n_items >= kItemSlots) {
                ok = __all_sync(0xffffffffu, mbar_wait(item_empty + slot_i, ((n_items / kItemSlots) - 1) & 1, ctl));
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
            const bool found = walk.locate(lane, g, seg, local);
            if (leader) {
                item_ring[slot_i] = found ? g : -1;
                mbar_arrive(item_full + slot_i);   // release semantics publish the ring entry
            }
            ++n_items;
            if (!found) break;
            const Work w = make_work<kDecode, C::kN>(p, seg, local);
            if (!w.valid) {
                if (leader) report(p.status, (int)UNIPIN_ERR_OUT_OF_RANGE);
                continue;
            }
            if (w.nt == 0) continue;
            // Q of this item may overwrite Q of the previous one once its S MMAs are done.
            if (nq > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(q_empty, (nq - 1) & 1, ctl));
                if (!ok) break;
            }
            if (leader) {
                mbar_arrive_expect_tx(bar_q, (w.has_b ? 2 : 1) * C::kTileQ);
                for (int x = 0; x < (w.has_b ? 2 : 1); ++x)
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(sQ + x * C::kTileQ + c * C::kAtomQ, &tm_q, bar_q, c * C::kBoxD, w.h,
                                    w.tok0 + w.qrow0 + x * kBlockM);
            }
            ++nq;
            const int hkv = w.h / p.G;   // the key/value head query head w.h reads
            const int pool_plane = (p.layer * p.S + w.slot) * (p.H / p.G) + hkv;
            for (int i = 0; ok && i < w.nt; ++i) {      // K_i and V_i into one slot
                int start, lo;
                key_tile<C::kN>(w.t_begin + i, w.nt_all, w.kmax, start, lo);
                const int st = u % NS;
                if (u >= NS) {
                    ok = __all_sync(0xffffffffu, mbar_wait(kv_empty + st, ((u / NS) - 1) & 1, ctl));
                    if (!ok) break;
                }
                if (leader) {
                    mbar_arrive_expect_tx(kv_full + st, C::kSlotBytes);
                    for (int kv = 0; kv < 2; ++kv) {
                        const CUtensorMap* map = kv == 0 ? &tm_k : &tm_v;
                        uint8_t* dst = ring + st * C::kSlotBytes + kv * C::kTileKV;
                        for (int c = 0; c < C::kChunks; ++c) {
                            if (kDecode)
                                tma_load_3d(dst + c * C::kAtomKV, map, kv_full + st, c * C::kBoxD, start,
                                            pool_plane);
                            else
                                tma_load_3d(dst + c * C::kAtomKV, map, kv_full + st, c * C::kBoxD, hkv,
                                            w.tok0 + start);
                        }
                    }
                }
                ++u;
            }
        }
        if (!ok && leader) {
            // stop the consumers: an end marker in the next ring slot
            const int slot_i = n_items % kItemSlots;
            if (n_items < kItemSlots ||
                mbar_wait_drain(item_empty + slot_i, ((n_items / kItemSlots) - 1) & 1, p.wait_limit_ns)) {
                item_ring[slot_i] = -1;
                mbar_arrive(item_full + slot_i);
                ++n_items;
            }
        }
        if (leader) {
            // Consume the last arrival of every barrier the other warps signal to
            // this warp, so nothing lands in shared memory after the block exits.
            for (int v = (n_items > kItemSlots ? n_items - kItemSlots : 0); v < n_items; ++v)
                mbar_wait_drain(item_empty + v % kItemSlots, (v / kItemSlots) & 1, p.wait_limit_ns);
            if (nq > 0) mbar_wait_drain(q_empty, (nq - 1) & 1, p.wait_limit_ns);
            for (int v = (u > NS ? u - NS : 0); v < u; ++v)
                mbar_wait_drain(kv_empty + v % NS, (v / NS) & 1, p.wait_limit_ns);
        }
    } else if (warp == 11) {
        // ----------------------------------------------------- pool writer
        if (p.store_pool && leader) {
            tma_prefetch_map(&tm_pk);
            tma_prefetch_map(&tm_pv);
        }
        int u = 0;
        bool ok = true;
        while (pop_item(ok)) {
            const Work w = make_work<kDecode, C::kN>(p, seg, local);
            if (!kDecode && p.store_pool && w.valid && (local / p.H) == 0 && (w.h % p.G) == 0 && !w.store &&
                leader)
                report(p.status, (int)UNIPIN_ERR_OUT_OF_RANGE);   // slot id or history length beyond the pool
            const int plane = (p.layer * p.S + w.slot) * (p.H / p.G) + w.h / p.G;
            for (int i = 0; i < w.nt; ++i, ++u) {
                const int st = u % NS;
                ok = __all_sync(0xffffffffu, mbar_wait(kv_full + st, (u / NS) & 1, ctl));
                if (!ok) break;
                if (w.store) {
                    int start, lo;
                    key_tile<C::kN>(w.t_begin + i, w.nt_all, w.kmax, start, lo);
                    const uint8_t* src[2] = {ring + st * C::kSlotBytes, ring + st * C::kSlotBytes + C::kTileKV};
                    if (start >= 0) {
                        // the whole tile is rows start .. start+kN-1 of the slot (all below npast)
                        if (leader) {
                            for (int c = 0; c < C::kChunks; ++c) {
                                tma_store_3d(&tm_pk, src[0] + c * C::kAtomKV, c * C::kBoxD, start, plane);
                                tma_store_3d(&tm_pv, src[1] + c * C::kAtomKV, c * C::kBoxD, start, plane);
                            }
                            bulk_commit_group();
                            bulk_wait_read_all();
                        }
                    } else {
                        // a history shorter than one tile: rows 0 .. kmax-1 sit at tile rows
                        // -start .. kN-1; un-swizzle them with plain 16-byte copies
                        constexpr int kVecs = C::kRowBytes / 16;
                        const int units = w.kmax * C::kChunks * kVecs;
                        for (int x = lane; x < units; x += 32) {
                            const int j = x % kVecs;
                            const int c = (x / kVecs) % C::kChunks;
                            const int rr = x / (kVecs * C::kChunks);
                            const int sr = rr - start;
                            const int sw = C::kRowBytes == 128 ? (sr & 7) : ((sr >> 1) & 3);
                            const size_t dst = (((size_t)plane * p.n_cap + rr) * (D * 2)) + c * C::kRowBytes + j * 16;
                            const int so = c * C::kAtomKV + sr * C::kRowBytes + ((j ^ sw) << 4);
                            *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.pool_k) + dst) =
                                *reinterpret_cast<const uint4*>(src[0] + so);
                            *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.pool_v) + dst) =
                                *reinterpret_cast<const uint4*>(src[1] + so);
                        }
                    }
                }
                __syncwarp();
                if (leader) mbar_arrive(kv_empty + st);
            }
            if (!ok) break;
        }
        if (leader) bulk_wait_all();   // every pool store has landed before the block exits
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------- UMMA issuers
        // Warp 9 issues the MMAs of tile A, warp 10 those of tile B.  Per key
        // tile i of its query tile a warp issues
        //   S_{i+1} = Q K_{i+1}^T  as soon as the softmax has read S_i out,
        //   O += P_i V_i           as soon as the softmax has stored P_i,
        // so S_{i+1} is being computed while the softmax works on S_i.  Both
        // warps release every K/V ring use and every Q load (arrival count 2);
        // a use a warp does not need is still released, after its fill, so
        // the two warps' arrivals stay in phase.
        const int x = warp - 9;
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, C::kN, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
        // Descriptors are built once; a K-step moves only the start-address
        // field (low 14 bits, in 16-byte units), by compile-time offsets.
        const uint64_t dq0 = smem_desc(smem_u32(sQ) + x * C::kTileQ, 16, 8 * C::kRowBytes, C::kLayout);
        const uint64_t dk0 = smem_desc(smem_u32(ring), 16, 8 * C::kRowBytes, C::kLayout);
        const uint64_t dv0 = smem_desc(smem_u32(ring) + C::kTileKV, C::kAtomKV, 8 * C::kRowBytes, C::kLayout);
        const uint32_t tS = tmem + x * 256 + C::kColS;
        const uint32_t tP = tmem + x * 256 + C::kColP;
        const uint32_t tO = tmem + x * 256 + C::kColO;
        // S_x = Q_x K^T: both operands K-major in shared memory; K-steps of 16
        // elements (32 bytes within a swizzle row, then the next box of D).
        auto issue_qk = [&](int st) {
            const uint64_t b0 = dk0 + (uint64_t)((st * C::kSlotBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                constexpr int kStep = 32;
                const uint32_t in_row = (kk * kStep) % C::kRowBytes;
                const uint32_t box = kk * kStep / C::kRowBytes;
                umma_bf16_ss(tS, dq0 + ((box * C::kAtomQ + in_row) >> 4), b0 + ((box * C::kAtomKV + in_row) >> 4),
                             idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(s_full + x);
        };
        // O_x += P_x V: P from TMEM (8 columns of bf16 pairs per 16 keys), V
        // read MN-major (D contiguous); K-steps of 16 keys.
        auto issue_pv = [&](int st, bool acc) {
            const uint64_t b0 = dv0 + (uint64_t)((st * C::kSlotBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < C::kN / 16; ++kk) {
                const uint32_t off = (kk * 16 * C::kRowBytes) >> 4;
                umma_bf16_ts(tO, tP + kk * 8, b0 + off, idesc_pv, (acc || kk > 0) ? 1u : 0u);
            }
            umma_commit(pv_done + x);
        };
        auto wait_fill = [&](int u) {
            return __all_sync(0xffffffffu, mbar_wait(kv_full + u % NS, (u / NS) & 1, ctl));
        };
        int u = 0;                 // ring uses consumed
        int nq = 0;                // items with MMAs
        int np = 0;                // p_full completions consumed
        int nsq = 0;               // S tiles issued (each is read out once: one s_free completion)
        bool ok = true;
        // S_x may be overwritten once the softmax has read out the previous S_x.
        auto wait_s_free = [&]() {
            if (nsq == 0) return true;
            const bool r = __all_sync(0xffffffffu, mbar_wait(s_free + x, (nsq - 1) & 1, ctl));
            tc_fence_after_sync();
            return r;
        };
        while (pop_item(ok)) {
            const Work w = make_work<kDecode, C::kN>(p, seg, local);
            if (w.nt == 0) continue;
            const int ntx = x == 0 ? w.nt_a : w.nt_b;
            // Q landed: this also means both warps released the previous Q.
            ok = __all_sync(0xffffffffu, mbar_wait(bar_q, nq & 1, ctl)) && wait_fill(u);
            if (!ok) break;
            tc_fence_after_sync();
            if (ntx > 0) {
                if (!(ok = wait_s_free())) break;
                if (leader) {
                    issue_qk(u % NS);
                    if (ntx == 1) umma_commit(q_empty);            // no S MMA of this tile after this
                }
                ++nsq;
            } else if (leader) {
                mbar_arrive(q_empty);
            }
            for (int i = 0; ok && i < w.nt; ++i) {
                // Slot u holds K_i and V_i; slot u + 1 holds K_{i+1}.
                if (i < ntx) {
                    if (i + 1 < ntx) {
                        // s_free also says that slot u + 1 has landed: the softmax
                        // checks it before it signals, off this warp's critical path
                        // (a wait issued behind MMAs costs this warp until they drain).
                        if (!(ok = wait_s_free())) break;
                        if (leader) {
                            issue_qk((u + 1) % NS);
                            if (i + 2 == ntx) umma_commit(q_empty);   // that was this tile's last S MMA
                        }
                        ++nsq;
                    }
                    ok = __all_sync(0xffffffffu, mbar_wait(p_full + x, np & 1, ctl));
                    if (!ok) break;
                    ++np;
                    tc_fence_after_sync();
                    if (leader) {
                        issue_pv(u % NS, i > 0);
                        umma_commit(kv_empty + u % NS);
                    }
                } else {
                    // K_i/V_i are only for the other tile: release the slot once it has landed
                    if (!(ok = wait_fill(u))) break;
                    if (leader) mbar_arrive(kv_empty + u % NS);
                }
                ++u;
            }
            ++nq;
        }
        if (leader) {
            // Every MMA issued above completes before TMEM is released.
            umma_commit(bar_drain + x);
            mbar_wait_drain(bar_drain + x, 0, p.wait_limit_ns);
        }
    }
    } else {
        setmaxnreg_inc<C::kRegsSoftmax>();
        // ------------------------------------------------ softmax + epilogue
        const int x = warp / 4;                            // 0: tile A, 1: tile B
        const int r = threadIdx.x - x * kBlockM;           // query row in the tile
        const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
        const uint32_t tS = tmem + x * 256 + C::kColS + lane_off;
        const uint32_t tP = tmem + x * 256 + C::kColP + lane_off;
        const uint32_t tO = tmem + x * 256 + C::kColO + lane_off;
        const float sl2 = p.sl2;
        const bool split_mode = kDecode && p.nsplit > 1;
        constexpr int kN = C::kN;
        int ns = 0;          // s_full completions consumed
        int npv = 0;         // pv_done completions consumed
        int u_sm = 0;        // ring slot uses (key tiles loaded) before the current item
        auto wait_pv = [&]() {
            const bool r = __all_sync(0xffffffffu, mbar_wait(pv_done + x, npv & 1, ctl));
            ++npv;
            tc_fence_after_sync();
            return r;
        };
        bool ok = true;
        while (pop_item(ok)) {
            const Work w = make_work<kDecode, C::kN>(p, seg, local);
            const int u_item = u_sm;
            u_sm += w.nt;
            if (!w.valid) {
                // A segment whose history length or slot id is out of range: its rows get
                // zeros (a split partial marked invalid, l = -1, which the merge turns into
                // zeros), so no row is left holding another call's values.
                const int nrows_x = x == 0 ? w.nrows_a : w.nrows_b;
                if (w.rows_ok && r < nrows_x) {
                    const size_t tok = (size_t)w.tok0 + w.qrow0 + x * kBlockM + r;
                    if (split_mode) {
                        float* ml = p.part_ml + (((size_t)w.split * p.total_rows + tok) * p.H + w.h) * 2;
                        ml[0] = -INFINITY;
                        ml[1] = -1.f;
                    } else if (p.out_fp32) {
                        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (tok * p.H + w.h) * D);
#pragma unroll
                        for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + (tok * p.H + w.h) * D);
#pragma unroll
                        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                continue;
            }
            const int ntx = x == 0 ? w.nt_a : w.nt_b;
            const int nrows_x = x == 0 ? w.nrows_a : w.nrows_b;
            if (nrows_x <= 0) continue;
            const int kmax_x = x == 0 ? w.kmax_a : w.kmax_b;
            const int posx0 = w.pos0 + x * kBlockM;       // mask position of row 0 of this tile
            const int irow = posx0 + r;
            const bool row_valid = r < nrows_x;
            const long long tok = (long long)w.tok0 + w.qrow0 + x * kBlockM + r;
            const size_t base = ((size_t)tok * p.H + w.h) * D;
            const size_t base_kv = ((size_t)tok * (p.H / p.G) + w.h / p.G) * D;   // the row's own key/value
            // self term: a candidate row's own key (prefill rows i >= n_b; every decode row)
            const bool self = row_valid && !split_mode && (kDecode || irow >= w.npast);
            float ss = -INFINITY;
            if (self) {
                // issued before the first S wait so its latency overlaps the MMAs
                const uint4* q4 = reinterpret_cast<const uint4*>(p.q + base);
                const uint4* k4 = reinterpret_cast<const uint4*>(p.k_self + base_kv);
                float dot0 = 0.f, dot1 = 0.f;
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const uint4 qa = __ldg(q4 + c), ka = __ldg(k4 + c);
                    const __nv_bfloat162* qh = reinterpret_cast<const __nv_bfloat162*>(&qa);
                    const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&ka);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 qf = __bfloat1622float2(qh[e]);
                        const float2 kf = __bfloat1622float2(kh[e]);
                        dot0 = fmaf(qf.x, kf.x, dot0);
                        dot1 = fmaf(qf.y, kf.y, dot1);
                    }
                }
                ss = (dot0 + dot1) * sl2;
            }
            float m = -INFINITY;     // reference max (log2 units) the P values and O are relative to
            float l = 0.f;           // row sum relative to m
            for (int i = 0; i < ntx; ++i) {
                int start, lo;
                key_tile<C::kN>(w.t_begin + i, w.nt_all, w.kmax, start, lo);
                const bool full_tile = (start == lo) && (start + kN <= kmax_x) && (start + kN - 1 <= posx0);
                // warp-uniform: the TMEM accesses below are warp-collective
                ok = __all_sync(0xffffffffu, mbar_wait(s_full + x, ns & 1, ctl));
                if (!ok) break;
                ++ns;
                tc_fence_after_sync();
                uint32_t s[kN];
                if constexpr (kN == 128)
                    tmem_ld128(tS, s);
                else
                    tmem_ld64(tS, s);
                // S is in registers: the next S may be written over it.  The next S
                // also needs K_{i+1}; the first warp of the group signals only once
                // its ring slot has landed, so the MMA warp waits on s_free alone.
                if (i + 1 < ntx && (warp % 4) == 0) {
                    const int un = u_item + i + 1;
                    ok = __all_sync(0xffffffffu, mbar_wait(kv_full + un % NS, (un / NS) & 1, ctl));
                    if (!ok) break;
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_free + x);
                // P_x and O_x belong to the previous tile's P.V until it finishes
                // (at tile 0 the previous item's last P.V was waited for before its epilogue).
                bool pv_waited = i == 0;
                if (!full_tile) {
#pragma unroll
                    for (int e = 0; e < kN; ++e) {
                        const int j = start + e;
                        if (!(j >= lo && j < kmax_x && j <= irow)) s[e] = 0xff800000u;   // -inf
                    }
                }
                float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
                for (int e = 0; e < kN; e += 8) {
                    mx0 = max3f(mx0, __uint_as_float(s[e]), __uint_as_float(s[e + 1]));
                    mx1 = max3f(mx1, __uint_as_float(s[e + 2]), __uint_as_float(s[e + 3]));
                    mx2 = max3f(mx2, __uint_as_float(s[e + 4]), __uint_as_float(s[e + 5]));
                    mx3 = max3f(mx3, __uint_as_float(s[e + 6]), __uint_as_float(s[e + 7]));
                }
                const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
                // Lazy rescale: move the reference max only when some row of the
                // warp would otherwise see P > 2^8; then every row moves to its own max.
                const bool need = m_tile > m + kRescaleLog2;
                if (__any_sync(0xffffffffu, need)) {
                    const float m_new = fmaxf(m, m_tile);
                    const float corr = (m == -INFINITY) ? 0.f : ex2_approx(m - m_new);
                    if (i > 0) {
                        if (!(ok = wait_pv())) break;
                        pv_waited = true;
                        // in 8-column pieces: the scores of the tile stay live meanwhile
#pragma unroll
                        for (int c = 0; c < D / 8; ++c) {
                            uint32_t o[8];
                            tmem_ld8(tO + c * 8, o);
#pragma unroll
                            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
                            tmem_st8(tO + c * 8, o);
                        }
                    }
                    l *= corr;
                    m = m_new;
                }
                const float m_use = (m == -INFINITY) ? 0.f : m;
                // P = 2^(s * scale * log2e - m): packed fp32 pairs; kPolyOf4 pairs in
                // four take the polynomial exp2 on the FMA pipe, the rest the MUFU ex2,
                // so the two pipes share the load.  P is written in pieces of 64 keys
                // (32 columns of bf16 pairs).
                const uint64_t sc2 = f2_pack(sl2, sl2);
                const uint64_t nm2 = f2_pack(-m_use, -m_use);
                uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int half = 0; half < kN / 64; ++half) {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int e = half * 64 + 2 * c;
                        const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), sc2, nm2);
                        float p0, p1;
                        if ((c & 3) >= 4 - C::kPolyOf4) {
                            exp2_poly2(x2, p0, p1);
                        } else {
                            float x0, x1;
                            f2_unpack(x2, x0, x1);
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                        }
                        acc[c & 3] = f2_add(acc[c & 3], f2_pack(p0, p1));
                        pk[c] = pack_bf16x2(p0, p1);
                    }
                    if (half == 0 && !pv_waited) {
                        if (!(ok = wait_pv())) break;
                    }
                    if (half + 1 < kN / 64)
                        tmem_st32_nowait(tP + half * 32, pk);   // its latency overlaps the next piece
                    else
                        tmem_st32(tP + half * 32, pk);          // waits for every piece
                }
                if (!ok) break;
                {
                    const uint64_t a01 = f2_add(acc[0], acc[1]);
                    const uint64_t a23 = f2_add(acc[2], acc[3]);
                    float lo, hi;
                    f2_unpack(f2_add(a01, a23), lo, hi);
                    l += lo + hi;
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full + x);
            }
            if (!ok) break;
            // ---- epilogue: the own value (self term) is fetched before waiting for O
            uint4 vr[D / 8];
            {
                const uint4* v4 = reinterpret_cast<const uint4*>(p.v_self + base_kv);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) vr[c] = self ? __ldg(v4 + c) : make_uint4(0u, 0u, 0u, 0u);
            }
            if (ntx > 0 && !(ok = wait_pv())) break;   // the last P.V: O_x is final
            float a = 1.f, b = 0.f, inv = 0.f;
            if (row_valid && !split_mode) {
                const float m_fin = fmaxf(m, ss);
                a = (m == -INFINITY) ? 0.f : ex2_approx(m - m_fin);
                b = self ? ex2_approx(ss - m_fin) : 0.f;
                const float denom = l * a + b;
                inv = denom > 0.f ? 1.f / denom : 0.f;
                if (!kDecode && p.lse) p.lse[(size_t)tok * p.H + w.h] = m_fin + log2f(denom);
            }
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (ntx > 0) {
                    tmem_ld32(tO + c * 32, o);   // warp-collective: every lane loads
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0u;
                }
                if (row_valid && split_mode) {
                    float* dst = p.part_o + ((size_t)w.split * p.total_rows * p.H) * D + base + c * 32;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(dst + e) =
                            make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                                        __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
                }
                if (row_valid && !split_mode) {
                    float res[32];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 va = vr[c * 4 + q];
                        const __nv_bfloat162* vh = reinterpret_cast<const __nv_bfloat162*>(&va);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 vf = __bfloat1622float2(vh[e]);
                            res[q * 8 + 2 * e] = (__uint_as_float(o[q * 8 + 2 * e]) * a + b * vf.x) * inv;
                            res[q * 8 + 2 * e + 1] = (__uint_as_float(o[q * 8 + 2 * e + 1]) * a + b * vf.y) * inv;
                        }
                    }
                    if (p.out_fp32) {
                        float* dst = reinterpret_cast<float*>(p.out) + base + c * 32;
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(dst + e) =
                                make_float4(res[e], res[e + 1], res[e + 2], res[e + 3]);
                    } else {
                        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + base + c * 32;
#pragma unroll
                        for (int e = 0; e < 32; e += 8)
                            *reinterpret_cast<uint4*>(dst + e) =
                                make_uint4(pack_bf16x2(res[e], res[e + 1]), pack_bf16x2(res[e + 2], res[e + 3]),
                                           pack_bf16x2(res[e + 4], res[e + 5]), pack_bf16x2(res[e + 6], res[e + 7]));
                    }
                }
            }
            if (split_mode && row_valid) {
                float* ml = p.part_ml + (((size_t)w.split * p.total_rows + tok) * p.H + w.h) * 2;
                ml[0] = m;
                ml[1] = l;
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Evaluates the FMA-pipe exp2 used by the softmax on n inputs (for tests).
__global__ void exp2_poly_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int n)
{
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float a = x[i];
    const float b = (i + 1 < n) ? x[i + 1] : 0.f;
    float r0, r1;
    exp2_poly2(f2_pack(a, b), r0, r1);
    y[i] = r0;
    if (i + 1 < n) y[i + 1] = r1;
}

// Split-n merge for the rank decode: each (candidate, head) row combines the
// nsplit partial (O, m, l) of its pool sweep with its own key (self term).
// One warp per row; the self dot product is reduced with warp shuffles.
template <int D>
__global__ void __launch_bounds__(256)
    decode_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                        const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_self,
                        const __nv_bfloat16* __restrict__ v_self, void* out, int out_fp32, int total_rows, int H,
                        int G, int nsplit, float sl2)
{
    constexpr int E = D / 32;   // elements per lane
    const int lane = threadIdx.x % 32;
    const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;   // tok * H + h
    if (row >= (long long)total_rows * H) return;
    const size_t base = (size_t)row * D + lane * E;
    // the row's own key/value: token row / H, key/value head (row % H) / G
    const size_t base_kv = ((size_t)(row / H) * (H / G) + (row % H) / G) * D + lane * E;
    float dot = 0.f;
    float vv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        dot = fmaf(__bfloat162float(q[base + e]), __bfloat162float(k_self[base_kv + e]), dot);
        vv[e] = __bfloat162float(v_self[base_kv + e]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float ss = dot * sl2;
    float m_fin = ss;
    bool invalid = false;   // the request was rejected on the device: its rows are zeros
    for (int s = 0; s < nsplit; ++s) {
        const float ms = part_ml[((size_t)s * total_rows * H + row) * 2];
        invalid |= part_ml[((size_t)s * total_rows * H + row) * 2 + 1] < 0.f;
        m_fin = fmaxf(m_fin, ms);
    }
    float acc[E];
    const float bself = ex2_approx(ss - m_fin);
    float den = bself;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = bself * vv[e];
    for (int s = 0; s < nsplit; ++s) {
        const float ms = part_ml[((size_t)s * total_rows * H + row) * 2];
        const float ls = part_ml[((size_t)s * total_rows * H + row) * 2 + 1];
        if (ms == -INFINITY || !(ls > 0.f)) continue;
        const float w = ex2_approx(ms - m_fin);
        den += w * ls;
        const float* po = part_o + (size_t)s * total_rows * H * D + base;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(w, po[e], acc[e]);
    }
    const float inv = invalid ? 0.f : 1.f / den;
    if (invalid) {
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
    }
    if (out_fp32) {
        float* dst = reinterpret_cast<float*>(out) + base;
#pragma unroll
        for (int e = 0; e < E; ++e) dst[e] = acc[e] * inv;
    } else {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out) + base;
#pragma unroll
        for (int e = 0; e < E; ++e) dst[e] = __float2bfloat16_rn(acc[e] * inv);
    }
}

}  // namespace unipin
