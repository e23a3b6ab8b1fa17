// Gradients of the M-FALCON masked attention on sm_100a.
//
// [review] §2.2 trains the whole sequence [past || candidates] in one pass
// under the mask (the joint objective).  With P_ij = 2^(s_ij * sl2 - lse_i)
// (sl2 = scale * log2 e, lse_i the forward's row statistic in the same
// units), O_i = sum_j P_ij v_j and the upstream gradient dO:
//   Dvec_i = dO_i . O_i
//   dP_ij  = dO_i . v_j,   dS_ij = P_ij (dP_ij - Dvec_i)
//   dV_j   = sum_i P_ij dO_i
//   dK_j   = scale * sum_i dS_ij q_i
//   dQ_i   = scale * sum_j dS_ij k_j
// over the allowed pairs.  Two kernels:
//   bwd_prep_kernel  one warp per (token, key/value head): Dvec_i of each of
//       its G query heads, and for a candidate row its own key (the diagonal
//       of the candidate block) entirely - it is the only row that sees that
//       key, so dK and dV of a candidate come from here alone, summed over
//       the group - plus that term's share of dQ; a past row's dQ starts at
//       zero.
//   bwd_kv_kernel    one block per (segment, key/value head, tile of 128 past
//       keys), sweeping the query tiles of each of the G query heads in turn
//       (dK and dV of the tile accumulate over all of them):
//       K and V of the tile stay in shared memory while the block sweeps the
//       128-row query tiles that see them (from the tile's own rows to the
//       segment end; past rows causally, every candidate row fully), with
//       the keys on the MMA's M dimension:
//         S^T  = K Q^T,  dP^T = V dO^T                (TMEM, lane = key)
//         P^T, dS^T from S^T, dP^T, lse and Dvec      (softmax warps, bf16
//                                                      back into TMEM and
//                                                      dS^T into smem)
//         dV  += P^T dO,  dK += dS^T Q                (A from TMEM)
//         dQ_tile = dS K                              (A = dS from smem)
//       and adds dQ_tile into the fp32 dQ with vector reductions; at the end
//       it writes the tile's dK, dV rows.
// Warp roles of bwd_kv_kernel (192 threads): warps 0-3 softmax and the dQ /
// dK / dV epilogues (thread t: key t of the tile, query row t of a dQ tile),
// warp 4 TMA producer, warp 5 MMA issuer (owns TMEM).  Every wait is bounded.
#pragma once

#include "sm100_ptx.cuh"
#include "tmem_wide.cuh"
#include "unipin.h"

namespace unipin {

constexpr int kBwThreads = 192;
constexpr int kBwRows = 128;   // keys per key tile and queries per query tile

template <int D>
struct BwCfg {
    static_assert(D == 32 || D == 64 || D == 128, "backward: head dim 32, 64 or 128");
    static constexpr int kBoxElems = D >= 64 ? 64 : D;              // elements of a row in one TMA box
    static constexpr int kBoxes = D / kBoxElems;                    // boxes across D (2 at D = 128)
    static constexpr int kRowBytes = kBoxElems * 2;
    static constexpr uint32_t kLayout = D >= 64 ? kLayoutSw128 : kLayoutSw64;
    static constexpr int kBox = kBwRows * kRowBytes;                // 128 rows of one box
    static constexpr int kTile = kBoxes * kBox;                     // 128 rows of K, V, Q or dO
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kTile;
    static constexpr int kOffQ = 2 * kTile;                         // [2] query-tile buffers
    static constexpr int kOffDO = 4 * kTile;                        // [2]
    static constexpr int kOffDS = 6 * kTile;                        // dS^T: 128 keys x 128 queries bf16 (2 x 16 KB)
    static constexpr int kOffStat = kOffDS + 32768;                 // lse[2][128], dvec[2][128]
    static constexpr int kOffBar = kOffStat + 4 * kBwRows * 4;
    static constexpr int kSmemBytes = kOffBar + 256;
    // TMEM columns (512 allocated)
    static constexpr int kColS = 0;        // S^T (128), then P^T as bf16 pairs (64)
    static constexpr int kColDP = 128;     // dP^T (128), then dS^T as bf16 pairs (64)
    static constexpr int kColDV = 256;
    static constexpr int kColDK = 256 + D;
    // dQ of a query tile: its own D columns where they fit; at D = 128 two halves of
    // 64 columns in the score columns that P^T and dS^T leave free (64-127, 192-255),
    // so the next tile's S^T and dP^T wait until the softmax has read them out.
    static constexpr bool kSplitDQ = 256 + 3 * D > 512;
    static constexpr int kDQHalf = kSplitDQ ? D / 2 : D;
    static constexpr int dq_col(int half) { return kSplitDQ ? (half == 0 ? 64 : 192) : 256 + 2 * D; }
    static_assert(kSplitDQ ? (kColDK + D <= 512 && kDQHalf <= 64) : (256 + 3 * D <= 512), "TMEM budget");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct BwParams {
    const __nv_bfloat16* q;     // [T, H, D]
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const __nv_bfloat16* o;     // forward output
    const __nv_bfloat16* dout;  // upstream gradient
    const float* lse;           // [T, H] forward row statistic, log2 units
    float* dq;                  // [T, H, D]
    float* dk;
    float* dv;
    float* dvec;                // [T, H] workspace
    const int* cu;
    const int* past;
    int B, H, total_rows, max_rows;   // H: query heads
    int G;                            // query heads per key/value head
    float scale, sl2;
    int* status;
    unsigned long long wait_limit_ns;
};

// A segment's rows are addressable and its past length is in range.
__device__ __forceinline__ bool bw_segment_ok(const BwParams& p, int b, int& tok0, int& len, int& npast)
{
    tok0 = p.cu[b];
    len = p.cu[b + 1] - tok0;
    npast = p.past[b];
    return tok0 >= 0 && len >= 0 && len <= p.max_rows && (long long)tok0 + len <= (long long)p.total_rows &&
           npast >= 0 && npast <= len;
}

// One warp per (token, key/value head): Dvec, the candidate self term, dQ initialisation.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwParams p)
{
    constexpr int E = D / 32;
    const int lane = threadIdx.x % 32;
    const int hkv = p.H / p.G;
    const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;   // token * hkv + kv head
    if (row >= (long long)p.total_rows * hkv) return;
    const long long t = row / hkv;
    const int hk = (int)(row - t * hkv);
    // segment of token t: the last b with cu[b] <= t
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (p.cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    int tok0, len, npast;
    const bool ok = bw_segment_ok(p, lo, tok0, len, npast) && t >= tok0 && t < (long long)tok0 + len;
    const bool cand = ok && (t - tok0) >= npast;
    const size_t kbase = (size_t)row * D + lane * E;
    float kv[E], vv[E], dk[E], dv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        kv[e] = __bfloat162float(p.k[kbase + e]);
        vv[e] = __bfloat162float(p.v[kbase + e]);
        dk[e] = 0.f;
        dv[e] = 0.f;
    }
    for (int g = 0; g < p.G; ++g) {
        const long long qr = t * p.H + (long long)hk * p.G + g;   // query row (token, query head)
        const size_t base = (size_t)qr * D + lane * E;
        float o[E], gd[E], qv[E];
        float dvec = 0.f, qk = 0.f, gv = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            o[e] = __bfloat162float(p.o[base + e]);
            gd[e] = __bfloat162float(p.dout[base + e]);
            qv[e] = __bfloat162float(p.q[base + e]);
            dvec = fmaf(gd[e], o[e], dvec);
            qk = fmaf(qv[e], kv[e], qk);
            gv = fmaf(gd[e], vv[e], gv);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            dvec += __shfl_xor_sync(0xffffffffu, dvec, off);
            qk += __shfl_xor_sync(0xffffffffu, qk, off);
            gv += __shfl_xor_sync(0xffffffffu, gv, off);
        }
        if (lane == 0) p.dvec[qr] = dvec;
        float pq = 0.f, ds = 0.f;
        if (cand) {
            pq = ex2_approx(qk * p.sl2 - p.lse[qr]);   // the row's weight on its own key
            ds = pq * (gv - dvec);
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
            p.dq[base + e] = cand ? p.scale * ds * kv[e] : 0.f;
            dk[e] = fmaf(p.scale * ds, qv[e], dk[e]);
            dv[e] = fmaf(pq, gd[e], dv[e]);
        }
    }
    if (cand || !ok) {                            // past keys of a valid segment: bwd_kv_kernel
#pragma unroll
        for (int e = 0; e < E; ++e) {
            p.dk[kbase + e] = dk[e];
            p.dv[kbase + e] = dv[e];
        }
    }
    if (!ok && lane == 0) report(p.status, (int)UNIPIN_ERR_OUT_OF_RANGE);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

template <int D>
__global__ void __launch_bounds__(kBwThreads, 1)
    bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwParams p)
{
    using C = BwCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    // item: key tile kt of (segment b, key/value head h); key-tile-major so the longest sweeps start first
    const int hkv = p.H / p.G;
    const int bh_count = p.B * hkv;
    const int kt = blockIdx.x / bh_count;
    const int bh = blockIdx.x - kt * bh_count;
    const int b = bh / hkv, h = bh - (bh / hkv) * hkv;
    int tok0, len, npast;
    if (!bw_segment_ok(p, b, tok0, len, npast)) return;   // bwd_prep_kernel zeroed and reported it
    const int j0 = kt * kBwRows;
    if (j0 >= npast) return;
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == (int)UNIPIN_ERR_DEVICE_TIMEOUT) return;
    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0) report(p.status, (int)UNIPIN_ERR_CUDA);
        return;
    }
    const int nqt = (len - j0 + kBwRows - 1) / kBwRows;   // query tiles kt .. kt + nqt - 1 of one query head
    const int nq = nqt * p.G;                             // swept for each of the G query heads in turn

    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sDO = smem + C::kOffDO;
    uint8_t* sDS = smem + C::kOffDS;
    float* s_lse = reinterpret_cast<float*>(smem + C::kOffStat);   // [2][128]
    float* s_dvec = s_lse + 2 * kBwRows;                            // [2][128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_kv = bars + 0;
    uint64_t* bar_qdo = bars + 1;      // [2]
    uint64_t* qdo_empty = bars + 3;    // [2]
    uint64_t* s_ready = bars + 5;
    uint64_t* p_ready = bars + 6;
    uint64_t* mma2_done = bars + 7;
    uint64_t* grp = bars + 8;
    uint64_t* bar_drain = bars + 9;
    uint64_t* dq_free = bars + 10;     // dQ read out of TMEM (4 softmax warps; split dQ only)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar_qdo + x, 1);
            mbar_init(qdo_empty + x, 1);
        }
        mbar_init(s_ready, 1);
        mbar_init(p_ready, 4);
        mbar_init(mma2_done, 1);
        mbar_init(grp, 4);
        mbar_init(bar_drain, 1);
        mbar_init(dq_free, 4);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns, (int)UNIPIN_ERR_DEVICE_TIMEOUT};
    const bool leader = lane == 0;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (leader) {
            tma_prefetch_map(&tm_q);
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
            tma_prefetch_map(&tm_do);
            mbar_arrive_expect_tx(bar_kv, 2 * C::kTile);
            for (int c = 0; c < C::kBoxes; ++c) {
                tma_load_3d(sK + c * C::kBox, &tm_k, bar_kv, c * C::kBoxElems, h, tok0 + j0);
                tma_load_3d(sV + c * C::kBox, &tm_v, bar_kv, c * C::kBoxElems, h, tok0 + j0);
            }
        }
        bool ok = true;
        for (int qi = 0; ok && qi < nq; ++qi) {
            const int qb = qi & 1;
            if (qi >= 2) {
                ok = __all_sync(0xffffffffu, mbar_wait(qdo_empty + qb, ((qi >> 1) - 1) & 1, ctl));
                if (!ok) break;
            }
            if (leader) {
                const int row0 = tok0 + j0 + (qi % nqt) * kBwRows;
                const int hq = h * p.G + qi / nqt;
                mbar_arrive_expect_tx(bar_qdo + qb, 2 * C::kTile);
                for (int c = 0; c < C::kBoxes; ++c) {
                    tma_load_3d(sQ + qb * C::kTile + c * C::kBox, &tm_q, bar_qdo + qb, c * C::kBoxElems, hq, row0);
                    tma_load_3d(sDO + qb * C::kTile + c * C::kBox, &tm_do, bar_qdo + qb, c * C::kBoxElems, hq, row0);
                }
            }
        }
        if (leader) {
            // every copy lands before the block exits
            mbar_wait_drain(bar_kv, 0, p.wait_limit_ns);
            for (int v = (nq > 2 ? nq - 2 : 0); v < nq; ++v)
                mbar_wait_drain(bar_qdo + (v & 1), (v >> 1) & 1, p.wait_limit_ns);
        }
    } else if (warp == 5) {
        // --------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_s = idesc_bf16_f32(kBwRows, kBwRows, false, false);
        constexpr uint32_t idesc_g = idesc_bf16_f32(kBwRows, D, true, false);    // A from TMEM, B MN-major
        constexpr uint32_t idesc_q = idesc_bf16_f32(kBwRows, C::kDQHalf, true, true);   // A (dS) and B (K) MN-major
        const uint64_t dK_kmaj = smem_desc(smem_u32(sK), 16, 8 * C::kRowBytes, C::kLayout);
        const uint64_t dV_kmaj = smem_desc(smem_u32(sV), 16, 8 * C::kRowBytes, C::kLayout);
        const uint64_t dQ_kmaj = smem_desc(smem_u32(sQ), 16, 8 * C::kRowBytes, C::kLayout);
        const uint64_t dDO_kmaj = smem_desc(smem_u32(sDO), 16, 8 * C::kRowBytes, C::kLayout);
        // MN-major operands span D in boxes kBox bytes apart
        const uint64_t dQ_mn = smem_desc(smem_u32(sQ), C::kBox, 8 * C::kRowBytes, C::kLayout);
        const uint64_t dDO_mn = smem_desc(smem_u32(sDO), C::kBox, 8 * C::kRowBytes, C::kLayout);
        const uint64_t dK_mn = smem_desc(smem_u32(sK), C::kBox, 8 * C::kRowBytes, C::kLayout);
        const uint64_t dDS_mn = smem_desc(smem_u32(sDS), 16384, 1024, kLayoutSw128);
        bool ok = __all_sync(0xffffffffu, mbar_wait(bar_kv, 0, ctl));
        for (int qi = 0; ok && qi < nq; ++qi) {
            const int qb = qi & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_qdo + qb, (qi >> 1) & 1, ctl));
            if (!ok) break;
            // split dQ: the last tile's dQ halves sit in the score columns until read out
            if (C::kSplitDQ && qi > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(dq_free, (qi - 1) & 1, ctl));
                if (!ok) break;
            }
            tc_fence_after_sync();
            const uint64_t qoff = (uint64_t)((qb * C::kTile) >> 4);
            if (leader) {
                // S^T = K Q^T and dP^T = V dO^T: K-steps of 16 elements (32 bytes of a box row)
                constexpr int kStepsPerBox = C::kBoxElems / 16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)(((kk / kStepsPerBox) * C::kBox + (kk % kStepsPerBox) * 32) >> 4);
                    umma_bf16_ss(tmem + C::kColS, dK_kmaj + off, dQ_kmaj + qoff + off, idesc_s, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)(((kk / kStepsPerBox) * C::kBox + (kk % kStepsPerBox) * 32) >> 4);
                    umma_bf16_ss(tmem + C::kColDP, dV_kmaj + off, dDO_kmaj + qoff + off, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(s_ready);
            }
            ok = __all_sync(0xffffffffu, mbar_wait(p_ready, qi & 1, ctl));
            if (!ok) break;
            tc_fence_after_sync();
            if (leader) {
                // K-steps of 16 queries: 8 TMEM columns of bf16 pairs, 16 rows of Q / dO
#pragma unroll
                for (int kk = 0; kk < kBwRows / 16; ++kk) {
                    const uint64_t off = qoff + (uint64_t)((kk * 16 * C::kRowBytes) >> 4);
                    const uint32_t acc = (qi > 0 || kk > 0) ? 1u : 0u;
                    umma_bf16_ts(tmem + C::kColDV, tmem + C::kColS + kk * 8, dDO_mn + off, idesc_g, acc);
                    umma_bf16_ts(tmem + C::kColDK, tmem + C::kColDP + kk * 8, dQ_mn + off, idesc_g, acc);
                }
                // dQ_tile = dS K: K-steps of 16 keys (2 KB of dS^T, 16 rows of K); at D = 128 in two
                // halves of 64 head-dim columns (one K box each)
#pragma unroll
                for (int half = 0; half < D / C::kDQHalf; ++half)
#pragma unroll
                    for (int kk = 0; kk < kBwRows / 16; ++kk)
                        umma_bf16_ss(tmem + C::dq_col(half), dDS_mn + (uint64_t)((kk * 2048) >> 4),
                                     dK_mn + (uint64_t)((half * C::kBox + kk * 16 * C::kRowBytes) >> 4), idesc_q,
                                     kk > 0 ? 1u : 0u);
                umma_commit(mma2_done);
                umma_commit(qdo_empty + qb);
            }
        }
        if (leader) {
            umma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.wait_limit_ns);
        }
    } else {
        // ------------------------------------------------- softmax + epilogues
        const int t = threadIdx.x;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const int key = j0 + t;                 // key row of this thread within the segment
        const bool key_ok = key < npast;
        uint32_t ngrp = 0;
        bool ok = true;
        for (int qi = 0; qi < nq; ++qi) {
            const int sb = qi & 1;
            const int qrow0 = j0 + (qi % nqt) * kBwRows;   // first query row of the tile (segment position)
            const int hq = h * p.G + qi / nqt;              // its query head
            {
                const int r = qrow0 + t;
                const size_t idx = (size_t)(tok0 + r) * p.H + hq;
                s_lse[sb * kBwRows + t] = r < len ? p.lse[idx] : 0.f;
                s_dvec[sb * kBwRows + t] = r < len ? p.dvec[idx] : 0.f;
            }
            if (!(ok = warp_group_sync(grp, ngrp, ctl, lane))) break;
            ok = __all_sync(0xffffffffu, mbar_wait(s_ready, qi & 1, ctl));
            if (!ok) break;
            tc_fence_after_sync();
            const float* lse_t = s_lse + sb * kBwRows;
            const float* dvec_t = s_dvec + sb * kBwRows;
            // a full tile needs no mask: every key is past, every row in the segment and after the keys
            const bool full = (qrow0 >= j0 + kBwRows) && (qrow0 + kBwRows <= len) && (j0 + kBwRows <= npast);
#pragma unroll 1
            for (int c0 = 0; c0 < kBwRows; c0 += 32) {
                uint32_t sraw[32], draw[32];
                tmem_ld32(lane_base + C::kColS + c0, sraw);
                tmem_ld32(lane_base + C::kColDP + c0, draw);
                uint32_t pk[16], dk2[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float pp[2], dd[2];
#pragma unroll
                    for (int f = 0; f < 2; ++f) {
                        const int c = c0 + e + f;
                        const int row = qrow0 + c;
                        const bool allowed = full || (key_ok && row < len && (row >= npast || key <= row));
                        const float pv = allowed ? ex2_approx(__uint_as_float(sraw[e + f]) * p.sl2 - lse_t[c]) : 0.f;
                        pp[f] = pv;
                        dd[f] = pv * (__uint_as_float(draw[e + f]) - dvec_t[c]);
                    }
                    pk[e / 2] = pack_bf16x2(pp[0], pp[1]);
                    dk2[e / 2] = pack_bf16x2(dd[0], dd[1]);
                }
                // P^T and dS^T over columns already read (chunk c0 writes columns c0/2 .. c0/2 + 15)
                tmem_st16(lane_base + C::kColS + c0 / 2, pk);
                tmem_st16(lane_base + C::kColDP + c0 / 2, dk2);
                // dS^T row t into the 128-byte-swizzled, query-major layout the dQ MMA reads
                uint8_t* rowp = sDS + (c0 / 64) * 16384 + t * 128;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int chunk = ((c0 % 64) / 8 + j) ^ (t % 8);
                    *reinterpret_cast<uint4*>(rowp + (chunk << 4)) =
                        make_uint4(dk2[4 * j], dk2[4 * j + 1], dk2[4 * j + 2], dk2[4 * j + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_ready);
            // dQ of this query tile: row t of the TMEM tile, added into the fp32 gradient
            ok = __all_sync(0xffffffffu, mbar_wait(mma2_done, qi & 1, ctl));
            if (!ok) break;
            tc_fence_after_sync();
            const int row = qrow0 + t;
#pragma unroll
            for (int half = 0; half < D / C::kDQHalf; ++half) {
                uint32_t dqr[C::kDQHalf];
                if constexpr (C::kDQHalf == 64) tmem_ld64(lane_base + C::dq_col(half), dqr);
                else tmem_ld32(lane_base + C::dq_col(half), dqr);
                if (row < len) {
                    float* dst = p.dq + ((size_t)(tok0 + row) * p.H + hq) * D + half * C::kDQHalf;
#pragma unroll
                    for (int e = 0; e < C::kDQHalf; e += 4)
                        red_add_v4(dst + e, p.scale * __uint_as_float(dqr[e]), p.scale * __uint_as_float(dqr[e + 1]),
                                   p.scale * __uint_as_float(dqr[e + 2]), p.scale * __uint_as_float(dqr[e + 3]));
                }
            }
            tc_fence_before_sync();
            if (C::kSplitDQ) {
                __syncwarp();
                if (lane == 0) mbar_arrive(dq_free);
            }
        }
        if (ok) {
            // the tile's dK (scaled) and dV rows; all of this block's MMAs have finished.  The
            // TMEM loads are warp-collective: every lane loads, keys past the history store nothing.
            constexpr int kChunk = D >= 64 ? 64 : D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += kChunk) {
                uint32_t g[kChunk];
                if constexpr (kChunk == 64) tmem_ld64(lane_base + C::kColDK + c0, g);
                else tmem_ld32(lane_base + C::kColDK + c0, g);
                if (key_ok) {
                    float* dkd = p.dk + ((size_t)(tok0 + key) * hkv + h) * D + c0;
#pragma unroll
                    for (int e = 0; e < kChunk; e += 4)
                        *reinterpret_cast<float4*>(dkd + e) =
                            make_float4(p.scale * __uint_as_float(g[e]), p.scale * __uint_as_float(g[e + 1]),
                                        p.scale * __uint_as_float(g[e + 2]), p.scale * __uint_as_float(g[e + 3]));
                }
                if constexpr (kChunk == 64) tmem_ld64(lane_base + C::kColDV + c0, g);
                else tmem_ld32(lane_base + C::kColDV + c0, g);
                if (key_ok) {
                    float* dvd = p.dv + ((size_t)(tok0 + key) * hkv + h) * D + c0;
#pragma unroll
                    for (int e = 0; e < kChunk; e += 4)
                        *reinterpret_cast<float4*>(dvd + e) =
                            make_float4(__uint_as_float(g[e]), __uint_as_float(g[e + 1]), __uint_as_float(g[e + 2]),
                                        __uint_as_float(g[e + 3]));
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace unipin
