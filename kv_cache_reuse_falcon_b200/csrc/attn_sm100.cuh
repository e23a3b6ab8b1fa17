// M-FALCON masked attention engine for sm_100a: one thread block per
// (segment, head, 128-row query tile), tcgen05 UMMA with TMEM accumulators,
// TMA-staged K/V tiles, fp32 online softmax with one TMEM lane (one thread)
// per query row.
//
// The same engine runs the prefill and the rank decode.  In both, the part
// of a row's key set that is a contiguous run of keys 0..kmax-1 goes through
// the tensor cores with the causal predicate j <= i, and a candidate's own
// key (the diagonal of the candidate block) is merged in afterwards as a
// per-row fp32 dot product:
//   prefill ([notes] §3 "attention mask"):  kmax = min(rows in the tile's reach, n_b);
//       past row i sees j <= i < n_b; candidate row i >= n_b sees all j < n_b,
//       plus itself through the self term.
//   rank decode ([review] §2.4, [notes] §6):  keys are pool rows 0..n_r-1 of
//       the request's slot; every candidate sees all of them, plus itself.
// Fully masked key tiles are never visited (the tile loop stops at kmax), and
// key tiles entirely below the diagonal and below kmax skip the per-element
// predicate.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r; row max and
//              row sum stay in that thread's registers, so no shuffles are
//              needed for the row statistics; corrects O in TMEM when the
//              row max grows; writes P (bf16) to shared memory; epilogue.
//   warp 4     TMA producer (Q once, then K/V tiles through a 2-stage ring).
//   warp 5     TMEM allocator and the single UMMA-issuing thread.
#pragma once

#include "sm100_ptx.cuh"
#include "unipin.h"

namespace unipin {

constexpr int kBlockM = 128;   // query rows per tile = TMEM lanes
constexpr int kBlockN = 128;   // keys per tile
constexpr int kThreads = 192;
constexpr int kTmemCols = 256; // S: 128 columns, O: D <= 128 columns
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct AttnCfg {
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    static constexpr int kBoxD = D >= 64 ? 64 : D;              // elements per TMA box row
    static constexpr int kChunks = D / kBoxD;                   // boxes across D
    static constexpr int kRowBytes = kBoxD * 2;                 // 128 (SW128) or 64 (SW64)
    static constexpr uint32_t kLayout = kRowBytes == 128 ? kLayoutSw128 : kLayoutSw64;
    static constexpr int kAtomBytes = kBlockM * kRowBytes;      // one box of 128 rows
    static constexpr int kTileBytes = kBlockM * D * 2;          // Q, K or V tile
    static constexpr int kStages = 2;
    static constexpr int kPBytes = kBlockM * kBlockN * 2;       // P tile, bf16, SW128 K-major
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffP = kOffV + kStages * kTileBytes;
    static constexpr int kOffBar = kOffP + kPBytes;
    static constexpr int kSmemBytes = kOffBar + 128;
    static constexpr int kMinBlocks = D <= 64 ? 2 : 1;
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
    int H;
    int max_rows;                 // host bound on rows per segment (grid size)
    int total_rows;               // T
    int out_fp32;
    int layer, S, n_cap;          // pool geometry (decode)
    int nsplit;                   // decode: key-range splits per query tile
    float sl2;                    // scale * log2(e)
    int* status;
    unsigned long long wait_limit_ns;
};

// Key tile t of nt covering keys [0, kmax): tiles are 128 wide from key 0;
// a ragged last tile is loaded right-aligned (start = kmax - 128, possibly
// negative: the TMA fills rows before 0 with zeros) so that it never reads
// rows at or beyond kmax; keys below `lo` were already covered and are masked.
__device__ __forceinline__ void key_tile(int t, int nt, int kmax, int& start, int& lo)
{
    lo = t * kBlockN;
    start = (t == nt - 1 && (kmax % kBlockN) != 0) ? kmax - kBlockN : lo;
}

template <int D, bool kDecode>
__global__ void __launch_bounds__(kThreads, AttnCfg<D>::kMinBlocks)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p)
{
    using C = AttnCfg<D>;
    constexpr int NS = C::kStages;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int seg = blockIdx.z;
    const int h = blockIdx.y;

    // ------------------------------------------------------------ work unit
    // A timeout recorded earlier means a block of this or a previous launch
    // gave up; later blocks skip their work instead of waiting again.
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == (int)UNIPIN_ERR_DEVICE_TIMEOUT) return;
    const int tok0 = p.cu[seg];
    const int nrows_seg = p.cu[seg + 1] - tok0;
    const int npast = p.past[seg];
    int slot = 0;
    bool bad = tok0 < 0 || nrows_seg < 0 || nrows_seg > p.max_rows || npast < 0 ||
               (long long)tok0 + nrows_seg > (long long)p.total_rows;
    if (kDecode) {
        slot = p.slots[seg];
        bad = bad || slot < 0 || slot >= p.S || npast > p.n_cap;
    } else {
        bad = bad || npast > nrows_seg;
    }
    if (bad) {
        if (threadIdx.x == 0 && p.status) atomicCAS(p.status, 0, (int)UNIPIN_ERR_OUT_OF_RANGE);
        return;
    }
    const int ntiles_q = (nrows_seg + kBlockM - 1) / kBlockM;
    const int split = kDecode ? (int)(blockIdx.x % p.nsplit) : 0;
    const int qidx = kDecode ? (int)(blockIdx.x / p.nsplit) : (int)blockIdx.x;
    if (qidx >= ntiles_q) return;
    // Prefill: the costliest query tile of a segment (the last) launches first.
    const int qt = kDecode ? qidx : (ntiles_q - 1 - qidx);
    const int qrow0 = qt * kBlockM;
    const int nrows = min(kBlockM, nrows_seg - qrow0);
    const int causal0 = kDecode ? npast + qrow0 : qrow0;   // mask position of row 0
    const int kmax = kDecode ? npast : min(qrow0 + nrows, npast);
    const int nt_all = (kmax + kBlockN - 1) / kBlockN;
    int t_begin = 0, t_end = nt_all;
    if (kDecode && p.nsplit > 1) {
        const int per = (nt_all + p.nsplit - 1) / p.nsplit;
        t_begin = min(split * per, nt_all);
        t_end = min(t_begin + per, nt_all);
    }
    const int nt = t_end - t_begin;   // key tiles this block sweeps

    if ((smem_u32(smem) & 1023u) != 0) {   // layout needs 1024-byte aligned tiles
        if (threadIdx.x == 0 && p.status) atomicCAS(p.status, 0, (int)UNIPIN_ERR_CUDA);
        return;
    }
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sP = smem + C::kOffP;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_q = bars + 0;
    uint64_t* bar_s = bars + 1;
    uint64_t* bar_p = bars + 2;
    uint64_t* bar_o = bars + 3;
    uint64_t* bar_drain = bars + 4;
    uint64_t* full = bars + 5;          // [NS]
    uint64_t* empty = bars + 5 + NS;    // [NS]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5 + 2 * NS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_p, kBlockM);
        mbar_init(bar_o, 1);
        mbar_init(bar_drain, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem;          // 128 fp32 columns
    const uint32_t tO = tmem + 128;    // D fp32 columns

    WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns, (int)UNIPIN_ERR_DEVICE_TIMEOUT};

    if (warp == 4) {
        // ------------------------------------------------------- producer
        if (lane == 0 && nt > 0) {
            tma_prefetch_map(&tm_q);
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
            int last_use[NS];
            for (int s = 0; s < NS; ++s) last_use[s] = -1;
            mbar_arrive_expect_tx(bar_q, C::kTileBytes);
            for (int c = 0; c < C::kChunks; ++c)
                tma_load_3d(sQ + c * C::kAtomBytes, &tm_q, bar_q, c * C::kBoxD, h, tok0 + qrow0);
            const int pool_row = ((p.layer * p.S + slot) * p.H + h);
            for (int i = 0; i < nt; ++i) {
                const int t = t_begin + i;
                const int st = i % NS;
                if (i >= NS && !mbar_wait(empty + st, ((i / NS) - 1) & 1, ctl)) break;
                int start, lo;
                key_tile(t, nt_all, kmax, start, lo);
                mbar_arrive_expect_tx(full + st, 2 * C::kTileBytes);
                uint8_t* dk = sK + st * C::kTileBytes;
                uint8_t* dv = sV + st * C::kTileBytes;
                for (int c = 0; c < C::kChunks; ++c) {
                    if (kDecode) {
                        tma_load_3d(dk + c * C::kAtomBytes, &tm_k, full + st, c * C::kBoxD, start, pool_row);
                        tma_load_3d(dv + c * C::kAtomBytes, &tm_v, full + st, c * C::kBoxD, start, pool_row);
                    } else {
                        tma_load_3d(dk + c * C::kAtomBytes, &tm_k, full + st, c * C::kBoxD, h, tok0 + start);
                        tma_load_3d(dv + c * C::kAtomBytes, &tm_v, full + st, c * C::kBoxD, h, tok0 + start);
                    }
                }
                last_use[st] = i / NS;
            }
            // Let every issued copy land before shared memory is released.
            mbar_wait_drain(bar_q, 0, p.wait_limit_ns);
            for (int s = 0; s < NS; ++s)
                if (last_use[s] >= 0) mbar_wait_drain(full + s, last_use[s] & 1, p.wait_limit_ns);
        }
    } else if (warp == 5) {
        // ------------------------------------------------------ UMMA issuer
        if (lane == 0 && nt > 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
            // S = Q K^T: A = Q (K-major), B = K tile (K-major); K-steps of 16 elements (32 bytes).
            auto issue_qk = [&](int st) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk * 32 / C::kRowBytes) * C::kAtomBytes + (kk * 32) % C::kRowBytes;
                    const uint64_t a = smem_desc(aQ + off, 16, 8 * C::kRowBytes, C::kLayout);
                    const uint64_t b = smem_desc(aK + st * C::kTileBytes + off, 16, 8 * C::kRowBytes, C::kLayout);
                    umma_bf16_ss(tS, a, b, idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O += P V: A = P (K-major over keys, 128-byte swizzle, two 64-key atoms),
            // B = V tile read MN-major (D contiguous); K-steps of 16 keys.
            auto issue_pv = [&](int st, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    const uint32_t offp = (kk / 4) * (kBlockM * 128) + (kk % 4) * 32;
                    const uint64_t a = smem_desc(aP + offp, 16, 1024, kLayoutSw128);
                    const uint32_t offv = kk * 16 * C::kRowBytes;
                    const uint64_t b = smem_desc(aV + st * C::kTileBytes + offv, C::kAtomBytes,
                                                 8 * C::kRowBytes, C::kLayout);
                    umma_bf16_ss(tO, a, b, idesc_pv, (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(bar_q, 0, ctl);
            for (int i = 0; ok && i < nt; ++i) {
                if (i > 0) {
                    if (!(ok = mbar_wait(bar_p, (i - 1) & 1, ctl))) break;
                    tc_fence_after_sync();
                    issue_pv((i - 1) % NS, i - 1 > 0);
                    umma_commit(bar_o);
                    if (i - 1 + NS < nt) umma_commit(empty + (i - 1) % NS);
                }
                if (!(ok = mbar_wait(full + i % NS, (i / NS) & 1, ctl))) break;
                tc_fence_after_sync();
                issue_qk(i % NS);
                umma_commit(bar_s);
            }
            if (ok && mbar_wait(bar_p, (nt - 1) & 1, ctl)) {
                tc_fence_after_sync();
                issue_pv((nt - 1) % NS, nt - 1 > 0);
                umma_commit(bar_o);
            }
            // Every MMA issued above completes before TMEM is released.
            umma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.wait_limit_ns);
        }
    } else {
        // ------------------------------------------------ softmax + epilogue
        const int r = threadIdx.x;                       // query row in the tile
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const int irow = causal0 + r;                    // mask position of this row
        const float sl2 = p.sl2;
        float m = -INFINITY;                             // running max, log2 units
        float l = 0.f;                                   // running sum
        bool ok = true;
        for (int i = 0; i < nt; ++i) {
            const int t = t_begin + i;
            int start, lo;
            key_tile(t, nt_all, kmax, start, lo);
            const bool full_tile = (start == lo) && (start + kBlockN <= kmax) && (start + kBlockN - 1 <= causal0);
            // Waits are made warp-uniform: the TMEM loads below are warp-collective.
            ok = __all_sync(0xffffffffu, mbar_wait(bar_s, i & 1, ctl));
            if (!ok) break;
            tc_fence_after_sync();
            // pass 1: row max of the allowed scores
            float mx = -INFINITY;
#pragma unroll
            for (int c4 = 0; c4 < kBlockN / 32; ++c4) {
                uint32_t v[32];
                tmem_ld32(tS + lane_off + c4 * 32, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int j = start + c4 * 32 + e;
                    const bool allow = full_tile || (j >= lo && j < kmax && j <= irow);
                    if (allow) mx = fmaxf(mx, __uint_as_float(v[e]));
                }
            }
            const float m_new = fmaxf(m, mx * sl2);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            if (i > 0) {
                // P buffer and O are only touched after the previous P.V finished.
                ok = __all_sync(0xffffffffu, mbar_wait(bar_o, (i - 1) & 1, ctl));
                if (!ok) break;
                tc_fence_after_sync();
                // The TMEM load/store below are warp-collective, so the branch is
                // taken by the whole warp when any row's max grew; rows whose
                // max did not grow scale by 1.
                if (__any_sync(0xffffffffu, m_new > m)) {
                    const float corr = (m_new > m) ? ex2_approx(m - m_use) : 1.f;
                    l *= corr;
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + lane_off + c * 32, o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
                        tmem_st32(tO + lane_off + c * 32, o);
                    }
                }
            }
            // pass 2: P = 2^(s*scale*log2e - m), rounded to bf16; row sum of the rounded values
            float ls = 0.f;
            uint8_t* prow = sP + r * 128;
#pragma unroll
            for (int c4 = 0; c4 < kBlockN / 32; ++c4) {
                uint32_t v[32];
                tmem_ld32(tS + lane_off + c4 * 32, v);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int j = start + c4 * 32 + e;
                    const bool a0 = full_tile || (j >= lo && j < kmax && j <= irow);
                    const bool a1 = full_tile || (j + 1 >= lo && j + 1 < kmax && j + 1 <= irow);
                    const float p0 = a0 ? ex2_approx(fmaf(__uint_as_float(v[e]), sl2, -m_use)) : 0.f;
                    const float p1 = a1 ? ex2_approx(fmaf(__uint_as_float(v[e + 1]), sl2, -m_use)) : 0.f;
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                    ls += __low2float(b2) + __high2float(b2);
                    pk[e / 2] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                // keys c4*32 .. c4*32+31 live in 64-key atom (c4/2), 16-byte chunks (c4%2)*4 .. +3
                uint8_t* atom = prow + (c4 / 2) * (kBlockM * 128);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int chunk = ((c4 % 2) * 4 + q) ^ (r & 7);
                    *reinterpret_cast<uint4*>(atom + chunk * 16) =
                        make_uint4(pk[4 * q + 0], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
            l += ls;
            m = m_new;
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(bar_p);
        }
        if (ok && nt > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_o, (nt - 1) & 1, ctl));
            tc_fence_after_sync();
        }
        if (ok) {
            const bool row_valid = r < nrows;
            const long long tok = (long long)tok0 + qrow0 + r;
            const size_t base = ((size_t)tok * p.H + h) * D;
            const bool split_mode = kDecode && p.nsplit > 1;
            // self term: a candidate row's own key (prefill rows i >= n_b; every decode row)
            const bool self = !split_mode && (kDecode || irow >= npast);
            float a = 1.f, b = 0.f, inv = 0.f;
            if (row_valid && !split_mode) {
                float ss = -INFINITY;
                if (self) {
                    const uint4* q4 = reinterpret_cast<const uint4*>(p.q + base);
                    const uint4* k4 = reinterpret_cast<const uint4*>(p.k_self + base);
                    float dot = 0.f;
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) {
                        const uint4 qa = q4[c], ka = k4[c];
                        const __nv_bfloat162* qh = reinterpret_cast<const __nv_bfloat162*>(&qa);
                        const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&ka);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 qf = __bfloat1622float2(qh[e]);
                            const float2 kf = __bfloat1622float2(kh[e]);
                            dot = fmaf(qf.x, kf.x, dot);
                            dot = fmaf(qf.y, kf.y, dot);
                        }
                    }
                    ss = dot * sl2;
                }
                const float m_fin = fmaxf(m, ss);
                a = (m == -INFINITY) ? 0.f : ex2_approx(m - m_fin);
                b = self ? ex2_approx(ss - m_fin) : 0.f;
                const float denom = l * a + b;
                inv = denom > 0.f ? 1.f / denom : 0.f;
            }
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (nt > 0) {
                    tmem_ld32(tO + lane_off + c * 32, o);   // warp-collective: every lane loads
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0u;
                }
                if (!row_valid) continue;
                if (split_mode) {
                    float* dst = p.part_o + ((size_t)split * p.total_rows * p.H) * D + base + c * 32;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(dst + e) =
                            make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                                        __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
                    continue;
                }
                float res[32];
                if (self) {
                    const uint4* v4 = reinterpret_cast<const uint4*>(p.v_self + base + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 va = v4[q];
                        const __nv_bfloat162* vh = reinterpret_cast<const __nv_bfloat162*>(&va);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 vf = __bfloat1622float2(vh[e]);
                            res[q * 8 + 2 * e] = (__uint_as_float(o[q * 8 + 2 * e]) * a + b * vf.x) * inv;
                            res[q * 8 + 2 * e + 1] = (__uint_as_float(o[q * 8 + 2 * e + 1]) * a + b * vf.y) * inv;
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) res[e] = __uint_as_float(o[e]) * a * inv;
                }
                if (p.out_fp32) {
                    float* dst = reinterpret_cast<float*>(p.out) + base + c * 32;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(dst + e) = make_float4(res[e], res[e + 1], res[e + 2], res[e + 3]);
                } else {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + base + c * 32;
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        __nv_bfloat162 b0 = __floats2bfloat162_rn(res[e], res[e + 1]);
                        __nv_bfloat162 b1 = __floats2bfloat162_rn(res[e + 2], res[e + 3]);
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(res[e + 4], res[e + 5]);
                        __nv_bfloat162 b3 = __floats2bfloat162_rn(res[e + 6], res[e + 7]);
                        w.x = *reinterpret_cast<uint32_t*>(&b0);
                        w.y = *reinterpret_cast<uint32_t*>(&b1);
                        w.z = *reinterpret_cast<uint32_t*>(&b2);
                        w.w = *reinterpret_cast<uint32_t*>(&b3);
                        *reinterpret_cast<uint4*>(dst + e) = w;
                    }
                }
            }
            if (split_mode && row_valid) {
                float* ml = p.part_ml + (((size_t)split * p.total_rows + tok) * p.H + h) * 2;
                ml[0] = m;
                ml[1] = l;
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Split-n merge for the rank decode: each (candidate, head) row combines the
// nsplit partial (O, m, l) of its pool sweep with its own key (self term).
// One warp per row; the self dot product is reduced with warp shuffles.
template <int D>
__global__ void __launch_bounds__(256)
    decode_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                        const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_self,
                        const __nv_bfloat16* __restrict__ v_self, void* out, int out_fp32, int total_rows, int H,
                        int nsplit, float sl2)
{
    constexpr int E = D / 32;   // elements per lane
    const int lane = threadIdx.x % 32;
    const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;   // tok * H + h
    if (row >= (long long)total_rows * H) return;
    const size_t base = (size_t)row * D + lane * E;
    float dot = 0.f;
    float vv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        dot = fmaf(__bfloat162float(q[base + e]), __bfloat162float(k_self[base + e]), dot);
        vv[e] = __bfloat162float(v_self[base + e]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float ss = dot * sl2;
    float m_fin = ss;
    for (int s = 0; s < nsplit; ++s) {
        const float ms = part_ml[((size_t)s * total_rows * H + row) * 2];
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
    const float inv = 1.f / den;
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
