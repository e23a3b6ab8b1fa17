// Host side of the C ABI declared in include/unipin.h: argument checks,
// TMA tensor-map construction, grid sizing and kernel launches.  Everything
// here is asynchronous on the caller's stream; nothing allocates.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "unipin.h"
#include "sm100_ptx.cuh"
#include "attn_sm100.cuh"
#include "bwd_sm100.cuh"
#include "decode_smallk_sm100.cuh"
#include "kvpool_sm100.cuh"

using namespace unipin;

namespace {

constexpr int kNumSmsHint = 148;   // B200
constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_init_mutex;
bool g_device_ready[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

unsigned long long wait_limit_ns()
{
    static unsigned long long v = [] {
        const char* s = std::getenv("UNIPIN_WAIT_LIMIT_MS");
        long long ms = s ? std::atoll(s) : 0;
        if (ms <= 0) ms = 2000;
        return (unsigned long long)ms * 1000000ull;
    }();
    return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SM count of the current device (queried once per device; the B200 count if
// the query fails, e.g. on a machine without a device).
int current_sms()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return kNumSmsHint;
    if (g_num_sms[dev] > 0) return g_num_sms[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return kNumSmsHint;
    g_num_sms[dev] = n;
    return n;
}

// Persistent grid: `per_sm` blocks per SM, fewer if there cannot be that many items.
unsigned persistent_blocks(long long item_bound, int per_sm = 1)
{
    const long long sms = (long long)current_sms() * per_sm;
    long long n = item_bound < sms ? item_bound : sms;
    return (unsigned)(n < 1 ? 1 : n);
}

template <typename K>
int set_attn_attr(K kernel, int smem_bytes)
{
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
        return UNIPIN_ERR_CUDA;
    // The kernel moves registers between warpgroups; that is only safe when it
    // launches with exactly the per-thread count the split was computed for.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return UNIPIN_ERR_CUDA;
    if (fa.numRegs != kLaunchRegs) return UNIPIN_ERR_UNSUPPORTED;
    return UNIPIN_OK;
}

template <int D>
int set_attn_attrs()
{
    int rc = set_attn_attr(attn_fwd_kernel<D, false>, AttnCfg<D, false>::kSmemBytes);
    if (rc != UNIPIN_OK) return rc;
    return set_attn_attr(attn_fwd_kernel<D, true>, AttnCfg<D, true>::kSmemBytes);
}

template <int D, int N, bool kE4M3>
int set_sk_attr()
{
    if (cudaFuncSetAttribute(decode_smallk_kernel<D, N, kE4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SkCfg<D, N, kE4M3>::kSmemBytes) != cudaSuccess)
        return UNIPIN_ERR_CUDA;
    // All of the SM's on-chip memory as shared memory, so that two blocks fit where they are meant to.
    if (cudaFuncSetAttribute(decode_smallk_kernel<D, N, kE4M3>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return UNIPIN_ERR_CUDA;
    return UNIPIN_OK;
}

template <int D, bool kE4M3>
int set_sk_attrs()
{
    int rc = set_sk_attr<D, 16, kE4M3>();
    if (rc == UNIPIN_OK) rc = set_sk_attr<D, 32, kE4M3>();
    if constexpr (!(kE4M3 && D == 64))   // that pool is decoded from a dequantized copy (sk_takes_pool)
        if (rc == UNIPIN_OK) rc = set_sk_attr<D, 64, kE4M3>();
    return rc;
}

// Once per device: check it is an sm_100 part, resolve the tensor-map
// encoder from the driver and raise the kernels' shared-memory limit.
int ensure_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return UNIPIN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return UNIPIN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_init_mutex);
    if (g_device_ready[dev]) return UNIPIN_OK;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return UNIPIN_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return UNIPIN_ERR_CUDA;
    if (major != 10 || minor != 0) return UNIPIN_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        g_num_sms[dev] < 1)
        return UNIPIN_ERR_CUDA;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return UNIPIN_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    int rc = set_attn_attrs<32>();
    if (rc == UNIPIN_OK) rc = set_attn_attrs<64>();
    if (rc == UNIPIN_OK) rc = set_attn_attrs<128>();
    if (rc == UNIPIN_OK) rc = set_sk_attrs<64, false>();
    if (rc == UNIPIN_OK) rc = set_sk_attrs<128, false>();
    if (rc == UNIPIN_OK) rc = set_sk_attrs<64, true>();
    if (rc == UNIPIN_OK) rc = set_sk_attrs<128, true>();
    if (rc == UNIPIN_OK &&
        (cudaFuncSetAttribute(bwd_kv_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              BwCfg<32>::kSmemBytes) != cudaSuccess ||
         cudaFuncSetAttribute(bwd_kv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              BwCfg<64>::kSmemBytes) != cudaSuccess ||
         cudaFuncSetAttribute(bwd_kv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              BwCfg<128>::kSmemBytes) != cudaSuccess))
        rc = UNIPIN_ERR_CUDA;
    if (rc != UNIPIN_OK) return rc;
    g_device_ready[dev] = true;
    return UNIPIN_OK;
}

// bf16 3-D tensor map, dims innermost first, strides in bytes for dims 1 and 2.
int make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t st1, uint64_t st2,
             uint32_t b0, uint32_t b1, uint32_t b2, int D)
{
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {st1, st2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t elem[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = D >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, elem,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

// Packed token tensor [T, H, D]: boxes of `rows` tokens x `heads` heads x (D or
// 64) elements (128 query rows, one key tile, or the candidates of a request
// for a group of query heads).
int make_token_map(CUtensorMap* m, const void* base, int T, int H, int D, int rows, int heads = 1)
{
    const uint32_t box_d = D >= 64 ? 64u : (uint32_t)D;
    return make_map(m, base, (uint64_t)D, (uint64_t)H, (uint64_t)T, (uint64_t)D * 2, (uint64_t)H * D * 2, box_d,
                    (uint32_t)heads, (uint32_t)rows, D);
}

// E4M3 pool [L, S, H, n_cap, D] of one-byte codes viewed as (D, n_cap, L*S*H):
// boxes of `rows` whole rows (D bytes each) of one plane, unswizzled.
int make_pool_map_e4m3(CUtensorMap* m, const void* base, const unipin_kvpool* pool, int rows)
{
    const int D = pool->D;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)pool->n_cap, (cuuint64_t)pool->L * pool->S * pool->H};
    cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)pool->n_cap * D};
    cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)rows, 1};
    cuuint32_t elem[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, elem,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

// Pool [L, S, H, n_cap, D] viewed as (D, n_cap, L*S*H): boxes of `rows` history rows of one plane.
int make_pool_map(CUtensorMap* m, const void* base, const unipin_kvpool* pool, int rows)
{
    const int D = pool->D;
    const uint32_t box_d = D >= 64 ? 64u : (uint32_t)D;
    const uint64_t planes = (uint64_t)pool->L * pool->S * pool->H;
    return make_map(m, base, (uint64_t)D, (uint64_t)pool->n_cap, planes, (uint64_t)D * 2,
                    (uint64_t)pool->n_cap * D * 2, box_d, (uint32_t)rows, 1, D);
}

// The pool's heads are key/value heads: H (query heads) must be a multiple of them.
int check_pool(const unipin_kvpool* pool, int H, int D, int layer)
{
    if (!pool || !pool->k || !pool->v) return UNIPIN_ERR_INVALID_ARG;
    if (pool->L < 1 || pool->S < 1 || pool->n_cap < 1 || pool->H < 1 || H % pool->H != 0 || pool->D != D)
        return UNIPIN_ERR_INVALID_ARG;
    if (pool->dtype != UNIPIN_POOL_BF16 && pool->dtype != UNIPIN_POOL_E4M3) return UNIPIN_ERR_INVALID_ARG;
    if (pool->dtype == UNIPIN_POOL_E4M3 &&
        (!(pool->k_scale > 0.f) || !std::isfinite(pool->k_scale) || !(pool->v_scale > 0.f) ||
         !std::isfinite(pool->v_scale) || !std::isfinite(1.f / pool->k_scale) || !std::isfinite(1.f / pool->v_scale)))
        return UNIPIN_ERR_INVALID_ARG;
    if (!aligned16(pool->k) || !aligned16(pool->v)) return UNIPIN_ERR_MISALIGNED;
    if (layer < 0 || layer >= pool->L) return UNIPIN_ERR_OUT_OF_RANGE;
    if ((uint64_t)pool->L * pool->S * pool->H >= (1ull << 31)) return UNIPIN_ERR_INVALID_ARG;
    return UNIPIN_OK;
}

bool supported_d(int D) { return D == 32 || D == 64 || D == 128; }

// tpk, tpv: the pool as the prefill's fused pool write stores into it (unused otherwise).
template <bool kDecode>
int launch_attn(int D, dim3 grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const CUtensorMap& tpk, const CUtensorMap& tpv, const AttnParams& p, cudaStream_t s)
{
    switch (D) {
    case 32:
        attn_fwd_kernel<32, kDecode><<<grid, kThreads, AttnCfg<32, kDecode>::kSmemBytes, s>>>(tq, tk, tv, tpk, tpv, p);
        break;
    case 64:
        attn_fwd_kernel<64, kDecode><<<grid, kThreads, AttnCfg<64, kDecode>::kSmemBytes, s>>>(tq, tk, tv, tpk, tpv, p);
        break;
    case 128:
        attn_fwd_kernel<128, kDecode><<<grid, kThreads, AttnCfg<128, kDecode>::kSmemBytes, s>>>(tq, tk, tv, tpk, tpv,
                                                                                               p);
        break;
    default:
        return UNIPIN_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

int launch_pool_write(const unipin_kvpool* pool, int layer, const void* k, const void* v, const int* cu,
                      const int* past, const int* slots, int B, int H, int D, int max_past, int total_tokens,
                      int* status, cudaStream_t s)
{
    if (B == 0 || max_past == 0) return UNIPIN_OK;
    const long long vecs = (long long)max_past * (D / 8);
    const long long blocks = (vecs + 255) / 256;
    dim3 grid((unsigned)(blocks < 65535 ? blocks : 65535), (unsigned)H, (unsigned)B);
    if (pool->dtype == UNIPIN_POOL_E4M3) {
        PoolWriteE4M3Params q;
        q.k = static_cast<const uint4*>(k);
        q.v = static_cast<const uint4*>(v);
        q.pool_k = static_cast<uint2*>(pool->k);
        q.pool_v = static_cast<uint2*>(pool->v);
        q.cu = cu;
        q.past = past;
        q.slots = slots;
        q.H = H;
        q.D = D;
        q.S = pool->S;
        q.n_cap = pool->n_cap;
        q.layer = layer;
        q.total_tokens = total_tokens;
        q.inv_k = 1.f / pool->k_scale;
        q.inv_v = 1.f / pool->v_scale;
        q.status = status;
        kvpool_write_e4m3_kernel<<<grid, 256, 0, s>>>(q);
        return cudaGetLastError() == cudaSuccess ? UNIPIN_OK : UNIPIN_ERR_CUDA;
    }
    PoolWriteParams p;
    p.k = static_cast<const uint4*>(k);
    p.v = static_cast<const uint4*>(v);
    p.pool_k = static_cast<uint4*>(pool->k);
    p.pool_v = static_cast<uint4*>(pool->v);
    p.cu = cu;
    p.past = past;
    p.slots = slots;
    p.H = H;
    p.D = D;
    p.S = pool->S;
    p.n_cap = pool->n_cap;
    p.layer = layer;
    p.total_tokens = total_tokens;
    p.status = status;
    kvpool_write_kernel<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

int decode_nsplit(int R, int H, int D, int max_k, int n_cap, int sms)
{
    if (R < 1 || H < 1 || max_k < 1 || n_cap < 1) return 1;
    const long long units = (long long)R * H * ((max_k + kPairRows - 1) / kPairRows);
    const long long slots = (long long)sms;   // one block per SM (all of TMEM)
    const long long target = 4 * slots;
    if (units >= 2 * slots) return 1;   // two or more waves already: no split
    const int key_tiles = (n_cap + key_tile_width(D, true) - 1) / key_tile_width(D, true);
    long long ns = (target + units - 1) / units;
    const long long cap = key_tiles / 2 > 1 ? key_tiles / 2 : 1;   // at least two key tiles per split
    if (ns > cap) ns = cap;
    if (ns > 32) ns = 32;
    return (int)(ns < 1 ? 1 : ns);
}

constexpr size_t kSchedBytes = 256;   // work counter at the start of every workspace

size_t decode_workspace_bytes(int nsplit, int total_cand, int H, int D)
{
    if (nsplit <= 1) return kSchedBytes;
    const size_t rows = (size_t)nsplit * (size_t)total_cand * (size_t)H;
    return kSchedBytes + rows * (size_t)D * sizeof(float) + rows * 2 * sizeof(float);
}

// ---- small-k rank decode (keys as the MMA's M; decode_smallk_sm100.cuh)

// Requests with at most this many candidate columns (candidates x query heads per
// key/value head) take the small-k kernel (D 64 or 128); beyond 64 columns the
// many-candidate engine measured faster.
constexpr int kSmallKMax = 64;

bool use_small_k(int D, int max_k, int G)
{
    return (D == 64 || D == 128) && max_k >= 1 && (long long)max_k * G <= kSmallKMax && kSmallKMax % G == 0;
}

// An E4M3 scale as the bfloat16x2 factors of the small-k kernel's code
// expansion (see SkE4M3Mul); false where the scale is not a bfloat16 value in
// [2^-117, 2^118], the range in which the expansion equals the pool's reading rule.
bool sk_e4m3_mul(float scale, SkE4M3Mul* m)
{
    uint32_t bits;
    std::memcpy(&bits, &scale, sizeof bits);
    if ((bits & 0xFFFFu) != 0 || !(scale >= std::ldexp(1.f, -117) && scale <= std::ldexp(1.f, 118))) return false;
    auto bf16x2 = [](float x) {
        uint32_t b;
        std::memcpy(&b, &x, sizeof b);
        return (b >> 16) | (b & 0xFFFF0000u);
    };
    if (scale < 128.f) {   // scale * 2^120 stays below 2^127
        m->c1 = bf16x2(std::ldexp(scale, 120));
        m->c2 = 0;
    } else {
        m->c1 = bf16x2(std::ldexp(1.f, 120));
        m->c2 = bf16x2(scale);
    }
    return true;
}

// Whether the small-k kernel decodes this pool in place: a bfloat16 pool, or an
// E4M3 pool whose two scales the kernel's expansion takes, except at D = 64 with
// 64 candidate columns, where the code staging leaves room for one block per SM
// only and decoding a dequantized copy measured faster.
bool sk_takes_pool(const unipin_kvpool* pool, int D, int max_k, int G)
{
    if (!use_small_k(D, max_k, G)) return false;
    if (pool->dtype != UNIPIN_POOL_E4M3) return true;
    if (D == 64 && sk_pad_n(max_k * G) == 64) return false;
    SkE4M3Mul m;
    return sk_e4m3_mul(pool->k_scale, &m) && sk_e4m3_mul(pool->v_scale, &m);
}

template <bool kE4M3>
int sk_ctas_per_sm_t(int D, int N)
{
    if (D == 64) {
        switch (N) {
        case 16: return SkCfg<64, 16, kE4M3>::kCtasPerSm;
        case 32: return SkCfg<64, 32, kE4M3>::kCtasPerSm;
        default: return SkCfg<64, 64, kE4M3>::kCtasPerSm;
        }
    }
    switch (N) {
    case 16: return SkCfg<128, 16, kE4M3>::kCtasPerSm;
    case 32: return SkCfg<128, 32, kE4M3>::kCtasPerSm;
    default: return SkCfg<128, 64, kE4M3>::kCtasPerSm;
    }
}

int sk_ctas_per_sm(int D, int N, bool e4m3)
{
    return e4m3 ? sk_ctas_per_sm_t<true>(D, N) : sk_ctas_per_sm_t<false>(D, N);
}

// Tile ranges (blocks) per resident block slot (1: one wave of blocks);
// UNIPIN_DECODE_ITEMS_PER_BLOCK overrides it.
int sk_items_per_block()
{
    static int v = [] {
        const char* s = std::getenv("UNIPIN_DECODE_ITEMS_PER_BLOCK");
        int n = s ? std::atoi(s) : 0;
        return n > 0 ? n : 1;
    }();
    return v;
}

// Back-off (ns) of the small-k kernel's polling warps; UNIPIN_DECODE_POLL_NS overrides it.
unsigned sk_poll_ns()
{
    static unsigned v = [] {
        const char* s = std::getenv("UNIPIN_DECODE_POLL_NS");
        int n = s ? std::atoi(s) : -1;
        return (unsigned)(n >= 0 ? (n > 10000 ? 10000 : n) : 64);
    }();
    return v;
}

struct SkPlan {
    int N, blocks_per_sm;
    int tpp;                // key tiles per (request, key/value head) pair
    long long total_tiles;  // pairs * tpp
    int nranges;            // contiguous tile ranges, one per block
    int nsplit;             // the most pieces (ranges) any pair is cut into
};

// The tiles of all pairs, pair-major, cut into `nranges` equal contiguous
// ranges: about sk_items_per_block() ranges per resident block, fewer when a
// pair would be cut into more than kSkMaxSplit pieces (a range then spans at
// least tpp / (kSkMaxSplit - 1) tiles).  With split = false one range per
// pair (no partials).  The candidate columns of a pair are (candidate, query
// head of the group): max_k * G of them.
SkPlan sk_plan(int R, int H_kv, int G, int D, int max_k, int n_cap, int sms, bool e4m3, bool split = true)
{
    SkPlan pl;
    pl.N = sk_pad_n(max_k * G);
    pl.blocks_per_sm = sk_ctas_per_sm(D, pl.N, e4m3);
    pl.tpp = (n_cap + kSkKeys - 1) / kSkKeys;
    const long long pairs = (long long)R * H_kv;
    pl.total_tiles = pairs * pl.tpp;
    long long B = pairs;
    if (split) {
        B = (long long)sk_items_per_block() * sms * pl.blocks_per_sm;
        const long long min_tiles = (pl.tpp + kSkMaxSplit - 2) / (kSkMaxSplit - 1);
        if (B > pl.total_tiles / min_tiles) B = pl.total_tiles / min_tiles;
        if (B < 1) B = 1;
    }
    pl.nranges = (int)B;
    // the most pieces of a pair: blocks holding its first and last tile
    int most = 1;
    for (long long q = 0; q < pairs; ++q) {
        const long long x0 = q * pl.tpp, x1 = x0 + pl.tpp - 1;
        const long long b0 = ((x0 + 1) * B - 1) / pl.total_tiles, b1 = ((x1 + 1) * B - 1) / pl.total_tiles;
        if (b1 - b0 + 1 > most) most = (int)(b1 - b0 + 1);
    }
    pl.nsplit = most;
    return pl;
}

// Workspace of the small-k decode: work counter, per-(request, head) arrival
// counters, then the split partials O [nsplit, T, H, D] and (m, l) [nsplit, T, H, 2].
size_t sk_counter_bytes(int R, int H) { return ((size_t)R * H * sizeof(unsigned) + 255) / 256 * 256; }

size_t sk_workspace_bytes(const SkPlan& pl, int R, int H, int D, int total_cand)
{
    if (pl.nsplit <= 1) return kSchedBytes;
    const size_t rows = (size_t)pl.nsplit * (size_t)total_cand * (size_t)H;
    return kSchedBytes + sk_counter_bytes(R, H) + rows * (size_t)D * sizeof(float) + rows * 2 * sizeof(float);
}

template <int D, int N, bool kE4M3>
int launch_sk_kernel(unsigned grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const SkParams& p, cudaStream_t s)
{
    decode_smallk_kernel<D, N, kE4M3><<<grid, kSkThreads, SkCfg<D, N, kE4M3>::kSmemBytes, s>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

template <int D, bool kE4M3>
int launch_sk_d(int N, unsigned grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const SkParams& p, cudaStream_t s)
{
    switch (N) {
    case 16: return launch_sk_kernel<D, 16, kE4M3>(grid, tq, tk, tv, p, s);
    case 32: return launch_sk_kernel<D, 32, kE4M3>(grid, tq, tk, tv, p, s);
    default:
        if constexpr (kE4M3 && D == 64)
            return UNIPIN_ERR_UNSUPPORTED;   // not routed here (sk_takes_pool)
        else
            return launch_sk_kernel<D, 64, kE4M3>(grid, tq, tk, tv, p, s);
    }
}

int rank_decode_small_k(const void* q_c, const void* k_c, const void* v_c, void* out, int out_fp32,
                        const int* cu_seqlens_c, const int* slot_ids, const int* past_lens, int R, int H, int D,
                        int max_k, int total_cand, float scale, const unipin_kvpool* pool, int layer,
                        void* workspace, size_t workspace_bytes, int* dev_status, cudaStream_t s)
{
    const int G = H / pool->H;
    const bool e4m3 = pool->dtype == UNIPIN_POOL_E4M3;
    SkPlan pl = sk_plan(R, pool->H, G, D, max_k, pool->n_cap, current_sms(), e4m3);
    if (pl.nsplit > 1 && (!workspace || workspace_bytes < sk_workspace_bytes(pl, R, H, D, total_cand)))
        pl = sk_plan(R, pool->H, G, D, max_k, pool->n_cap, current_sms(), e4m3, false);
    if (pl.nsplit > 1 && cudaMemsetAsync(workspace, 0, kSchedBytes + sk_counter_bytes(R, H), s) != cudaSuccess)
        return UNIPIN_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    int rc;
    // the N candidate columns: N / G tokens x the G query heads of one key/value head
    if ((rc = make_token_map(&tq, q_c, total_cand, H, D, pl.N / G, G)) != UNIPIN_OK) return rc;
    if (e4m3) {
        if ((rc = make_pool_map_e4m3(&tk, pool->k, pool, kSkKeys)) != UNIPIN_OK) return rc;
        if ((rc = make_pool_map_e4m3(&tv, pool->v, pool, kSkKeys)) != UNIPIN_OK) return rc;
    } else {
        if ((rc = make_pool_map(&tk, pool->k, pool, kSkKeys)) != UNIPIN_OK) return rc;
        if ((rc = make_pool_map(&tv, pool->v, pool, kSkKeys)) != UNIPIN_OK) return rc;
    }

    SkParams p = {};
    p.q = static_cast<const __nv_bfloat16*>(q_c);
    p.k_self = static_cast<const __nv_bfloat16*>(k_c);
    p.v_self = static_cast<const __nv_bfloat16*>(v_c);
    p.out = out;
    p.cu = cu_seqlens_c;
    p.past = past_lens;
    p.slots = slot_ids;
    p.R = R;
    p.H = H;
    p.G = G;
    p.total_rows = total_cand;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.layer = layer;
    p.S = pool->S;
    p.n_cap = pool->n_cap;
    p.nsplit = pl.nsplit;
    p.tpp = pl.tpp;
    p.total_tiles = pl.total_tiles;
    p.nranges = pl.nranges;
    p.sl2 = scale * kLog2e;
    p.status = dev_status;
    p.wait_limit_ns = wait_limit_ns();
    p.poll_ns = sk_poll_ns();
    p.k_scale = pool->k_scale;
    p.v_scale = pool->v_scale;
    if (e4m3 && (!sk_e4m3_mul(pool->k_scale, &p.k_mul) || !sk_e4m3_mul(pool->v_scale, &p.v_mul)))
        return UNIPIN_ERR_INVALID_ARG;
    if (pl.nsplit > 1) {
        char* ws = static_cast<char*>(workspace);
        p.pair_cnt = reinterpret_cast<unsigned*>(ws + kSchedBytes);
        p.part_o = reinterpret_cast<float*>(ws + kSchedBytes + sk_counter_bytes(R, H));
        p.part_ml = p.part_o + (size_t)pl.nsplit * total_cand * H * D;
    }
    const unsigned grid = (unsigned)pl.nranges;
    if (e4m3)
        return D == 64 ? launch_sk_d<64, true>(pl.N, grid, tq, tk, tv, p, s)
                       : launch_sk_d<128, true>(pl.N, grid, tq, tk, tv, p, s);
    return D == 64 ? launch_sk_d<64, false>(pl.N, grid, tq, tk, tv, p, s)
                   : launch_sk_d<128, false>(pl.N, grid, tq, tk, tv, p, s);
}

__global__ void bounded_wait_selftest_kernel(int* status, unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    WaitCtl ctl{&abort_flag, status, limit_ns, (int)UNIPIN_ERR_DEVICE_TIMEOUT};
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, ctl);   // nothing ever arrives
    __syncthreads();
}

// Scratch for unipin_rank_decode_attn_noalloc: device memory the library
// owns from the moment the module loads on a device until the process exits,
// so callers of that entry point never allocate.  Host code only sees a
// stand-in for this symbol; its device address comes from
// cudaGetSymbolAddress, looked up once per device.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_addr[kMaxDevices] = {};

int noalloc_scratch_address(void** addr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return UNIPIN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return UNIPIN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_init_mutex);
    if (!g_noalloc_addr[dev]) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_noalloc_scratch) != cudaSuccess || a == nullptr) return UNIPIN_ERR_CUDA;
        g_noalloc_addr[dev] = a;
    }
    *addr = g_noalloc_addr[dev];
    return UNIPIN_OK;
}

// An E4M3 pool is decoded from bfloat16 rows expanded into the workspace: the
// remapped slot ids [R] (256-byte block), then K and V of a pool [1, R, H, n_cap, D].
size_t dequant_slab_bytes(const unipin_kvpool* pool, int R)
{
    const size_t rows = (size_t)R * pool->H * pool->n_cap * pool->D;
    return ((size_t)R * sizeof(int) + 255) / 256 * 256 + 2 * ((rows * 2 + 255) / 256 * 256);
}

int rank_decode_e4m3(const void* q_c, const void* k_c, const void* v_c, void* out, int out_fp32,
                     const int* cu_seqlens_c, const int* slot_ids, const int* past_lens, int R, int H, int D,
                     int max_k, int total_cand, float scale, const unipin_kvpool* pool, int layer, void* workspace,
                     size_t workspace_bytes, int* dev_status, cudaStream_t s)
{
    const size_t slab = dequant_slab_bytes(pool, R);
    if (!workspace || workspace_bytes < slab) return UNIPIN_ERR_INVALID_ARG;
    if (R > 65535 || pool->H > 65535) return UNIPIN_ERR_INVALID_ARG;
    char* ws = static_cast<char*>(workspace);
    const size_t slots_bytes = ((size_t)R * sizeof(int) + 255) / 256 * 256;
    const size_t plane = (((size_t)R * pool->H * pool->n_cap * pool->D) * 2 + 255) / 256 * 256;
    unipin_kvpool bf = *pool;
    bf.k = ws + slots_bytes;
    bf.v = ws + slots_bytes + plane;
    bf.L = 1;
    bf.S = R;
    bf.dtype = UNIPIN_POOL_BF16;
    PoolDequantParams p;
    p.pool_k = static_cast<const uint2*>(pool->k);
    p.pool_v = static_cast<const uint2*>(pool->v);
    p.out_k = static_cast<uint4*>(bf.k);
    p.out_v = static_cast<uint4*>(bf.v);
    p.out_slots = reinterpret_cast<int*>(ws);
    p.past = past_lens;
    p.slots = slot_ids;
    p.H = pool->H;
    p.D = D;
    p.S = pool->S;
    p.n_cap = pool->n_cap;
    p.layer = layer;
    p.k_scale = pool->k_scale;
    p.v_scale = pool->v_scale;
    const long long vecs = (long long)pool->n_cap * (D / 8);
    const long long blocks = (vecs + 255) / 256;
    dim3 grid((unsigned)(blocks < 65535 ? blocks : 65535), (unsigned)pool->H, (unsigned)R);
    kvpool_dequant_kernel<<<grid, 256, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return UNIPIN_ERR_CUDA;
    return unipin_rank_decode_attn(q_c, k_c, v_c, out, out_fp32, cu_seqlens_c, p.out_slots, past_lens, R, H, D, max_k,
                                   total_cand, scale, &bf, 0, ws + slab, workspace_bytes - slab, dev_status, s);
}

}  // namespace

extern "C" {

const char* unipin_status_string(int status)
{
    switch (status) {
    case UNIPIN_OK: return "UNIPIN_OK";
    case UNIPIN_ERR_INVALID_ARG: return "UNIPIN_ERR_INVALID_ARG";
    case UNIPIN_ERR_UNSUPPORTED: return "UNIPIN_ERR_UNSUPPORTED";
    case UNIPIN_ERR_MISALIGNED: return "UNIPIN_ERR_MISALIGNED";
    case UNIPIN_ERR_OUT_OF_RANGE: return "UNIPIN_ERR_OUT_OF_RANGE";
    case UNIPIN_ERR_CUDA: return "UNIPIN_ERR_CUDA";
    case UNIPIN_ERR_DEVICE_TIMEOUT: return "UNIPIN_ERR_DEVICE_TIMEOUT";
    default: return "UNIPIN_ERR_UNKNOWN";
    }
}

size_t unipin_masked_prefill_workspace_size(void) { return kSchedBytes; }

int unipin_masked_prefill_attn(const void* q, const void* k, const void* v, void* out, int out_fp32, float* lse,
                               const int* cu_seqlens, const int* past_lens, int B, int H, int H_kv, int D,
                               int max_seqlen, int total_tokens, float scale, const unipin_kvpool* pool,
                               const int* slot_ids, int layer, void* workspace, size_t workspace_bytes,
                               int* dev_status, void* stream)
{
    if (B < 0 || H < 1 || H_kv < 1 || H % H_kv != 0 || max_seqlen < 0 || total_tokens < 0)
        return UNIPIN_ERR_INVALID_ARG;
    if (!supported_d(D)) return UNIPIN_ERR_UNSUPPORTED;
    if (!(scale > 0.f) || !std::isfinite(scale)) return UNIPIN_ERR_INVALID_ARG;
    if (pool) {
        int rc = check_pool(pool, H, D, layer);
        if (rc != UNIPIN_OK) return rc;
        if (pool->H != H_kv || !slot_ids) return UNIPIN_ERR_INVALID_ARG;
    }
    if (B == 0 || total_tokens == 0 || max_seqlen == 0) return UNIPIN_OK;
    if (!q || !k || !v || !out || !cu_seqlens || !past_lens) return UNIPIN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return UNIPIN_ERR_MISALIGNED;
    if (workspace && !aligned16(workspace)) return UNIPIN_ERR_MISALIGNED;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return UNIPIN_ERR_MISALIGNED;
    int rc = ensure_device();
    if (rc != UNIPIN_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned long long* sched = nullptr;
    if (workspace && workspace_bytes >= kSchedBytes) {
        sched = static_cast<unsigned long long*>(workspace);
        if (cudaMemsetAsync(sched, 0, sizeof(unsigned long long), s) != cudaSuccess) return UNIPIN_ERR_CUDA;
    }

    CUtensorMap tq, tk, tv, tpk, tpv;
    if ((rc = make_token_map(&tq, q, total_tokens, H, D, kBlockM)) != UNIPIN_OK) return rc;
    if ((rc = make_token_map(&tk, k, total_tokens, H_kv, D, key_tile_width(D, false))) != UNIPIN_OK) return rc;
    if ((rc = make_token_map(&tv, v, total_tokens, H_kv, D, key_tile_width(D, false))) != UNIPIN_OK) return rc;
    // A bfloat16 pool takes the past K/V tiles the kernel loads anyway (no second
    // pass); an E4M3 pool is written by the quantizing pool-write kernel after it.
    const bool fuse_pool = pool && pool->dtype == UNIPIN_POOL_BF16;
    if (fuse_pool) {
        if ((rc = make_pool_map(&tpk, pool->k, pool, key_tile_width(D, false))) != UNIPIN_OK) return rc;
        if ((rc = make_pool_map(&tpv, pool->v, pool, key_tile_width(D, false))) != UNIPIN_OK) return rc;
    } else {
        tpk = tk;
        tpv = tv;
    }

    AttnParams p = {};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k_self = static_cast<const __nv_bfloat16*>(k);
    p.v_self = static_cast<const __nv_bfloat16*>(v);
    p.out = out;
    p.cu = cu_seqlens;
    p.past = past_lens;
    p.slots = nullptr;
    p.nseg = B;
    p.H = H;
    p.G = H / H_kv;
    p.max_rows = max_seqlen;
    p.total_rows = total_tokens;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.nsplit = 1;
    p.sl2 = scale * kLog2e;
    p.status = dev_status;
    p.wait_limit_ns = wait_limit_ns();
    p.sched = sched;
    p.lse = lse;
    if (fuse_pool) {
        p.store_pool = 1;
        p.pool_k = pool->k;
        p.pool_v = pool->v;
        p.slots = slot_ids;
        p.layer = layer;
        p.S = pool->S;
        p.n_cap = pool->n_cap;
    }
    const long long bound = (long long)B * H * ((max_seqlen + kPairRows - 1) / kPairRows);
    dim3 grid(persistent_blocks(bound), 1, 1);
    rc = launch_attn<false>(D, grid, tq, tk, tv, tpk, tpv, p, s);
    if (rc != UNIPIN_OK || !pool || fuse_pool) return rc;
    if (B > 65535 || pool->H > 65535) return UNIPIN_ERR_INVALID_ARG;
    return launch_pool_write(pool, layer, k, v, cu_seqlens, past_lens, slot_ids, B, pool->H, D, max_seqlen,
                             total_tokens, dev_status, s);
}

int unipin_kvpool_write(const unipin_kvpool* pool, int layer, const void* k, const void* v, const int* cu_seqlens,
                        const int* past_lens, const int* slot_ids, int B, int max_past, int total_tokens,
                        int* dev_status, void* stream)
{
    if (!pool) return UNIPIN_ERR_INVALID_ARG;
    if (B < 0 || max_past < 0 || total_tokens < 0) return UNIPIN_ERR_INVALID_ARG;
    if (!supported_d(pool->D)) return UNIPIN_ERR_UNSUPPORTED;
    int rc = check_pool(pool, pool->H, pool->D, layer);
    if (rc != UNIPIN_OK) return rc;
    if (max_past > pool->n_cap) return UNIPIN_ERR_OUT_OF_RANGE;
    if (B == 0 || max_past == 0 || total_tokens == 0) return UNIPIN_OK;
    if (!k || !v || !cu_seqlens || !past_lens || !slot_ids) return UNIPIN_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v)) return UNIPIN_ERR_MISALIGNED;
    if (B > 65535 || pool->H > 65535) return UNIPIN_ERR_INVALID_ARG;
    rc = ensure_device();
    if (rc != UNIPIN_OK) return rc;
    return launch_pool_write(pool, layer, k, v, cu_seqlens, past_lens, slot_ids, B, pool->H, pool->D, max_past,
                             total_tokens, dev_status, static_cast<cudaStream_t>(stream));
}

size_t unipin_rank_decode_workspace_size(int R, int H, int H_kv, int D, int max_k, int total_cand, int n_cap)
{
    if (R < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || !supported_d(D) || max_k < 1 || total_cand < 1 || n_cap < 1)
        return 0;
    // The split grows with the SM count: size for the larger of this device's and a B200's.
    const int sms = current_sms() > kNumSmsHint ? current_sms() : kNumSmsHint;
    const int G = H / H_kv;
    if (use_small_k(D, max_k, G))
        return sk_workspace_bytes(sk_plan(R, H_kv, G, D, max_k, n_cap, sms, false), R, H, D, total_cand);
    return decode_workspace_bytes(decode_nsplit(R, H, D, max_k, n_cap, sms), total_cand, H, D);
}

size_t unipin_rank_decode_pool_workspace_size(const unipin_kvpool* pool, int R, int H, int max_k, int total_cand)
{
    if (!pool || pool->H < 1 || H < 1 || H % pool->H != 0) return 0;
    const size_t base = unipin_rank_decode_workspace_size(R, H, pool->H, pool->D, max_k, total_cand, pool->n_cap);
    if (base == 0 || pool->dtype != UNIPIN_POOL_E4M3) return base;
    const int G = H / pool->H;
    if (sk_takes_pool(pool, pool->D, max_k, G)) {
        // the small-k kernel reads the codes itself: only its partials
        const int sms = current_sms() > kNumSmsHint ? current_sms() : kNumSmsHint;
        const size_t e = sk_workspace_bytes(sk_plan(R, pool->H, G, pool->D, max_k, pool->n_cap, sms, true), R, H,
                                            pool->D, total_cand);
        return e > base ? e : base;
    }
    return dequant_slab_bytes(pool, R) + base;
}

int unipin_rank_decode_attn(const void* q_c, const void* k_c, const void* v_c, void* out, int out_fp32,
                            const int* cu_seqlens_c, const int* slot_ids, const int* past_lens, int R, int H, int D,
                            int max_k, int total_cand, float scale, const unipin_kvpool* pool, int layer,
                            void* workspace, size_t workspace_bytes, int* dev_status, void* stream)
{
    if (R < 0 || H < 1 || max_k < 0 || total_cand < 0) return UNIPIN_ERR_INVALID_ARG;
    if (!supported_d(D)) return UNIPIN_ERR_UNSUPPORTED;
    if (!(scale > 0.f) || !std::isfinite(scale)) return UNIPIN_ERR_INVALID_ARG;
    int rc = check_pool(pool, H, D, layer);
    if (rc != UNIPIN_OK) return rc;
    if (R == 0 || total_cand == 0 || max_k == 0) return UNIPIN_OK;
    if (!q_c || !k_c || !v_c || !out || !cu_seqlens_c || !slot_ids || !past_lens) return UNIPIN_ERR_INVALID_ARG;
    if (!aligned16(q_c) || !aligned16(k_c) || !aligned16(v_c) || !aligned16(out)) return UNIPIN_ERR_MISALIGNED;
    if (workspace && !aligned16(workspace)) return UNIPIN_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != UNIPIN_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pool->dtype == UNIPIN_POOL_E4M3 && !sk_takes_pool(pool, D, max_k, H / pool->H))
        return rank_decode_e4m3(q_c, k_c, v_c, out, out_fp32, cu_seqlens_c, slot_ids, past_lens, R, H, D, max_k,
                                total_cand, scale, pool, layer, workspace, workspace_bytes, dev_status, s);
    if (use_small_k(D, max_k, H / pool->H))
        return rank_decode_small_k(q_c, k_c, v_c, out, out_fp32, cu_seqlens_c, slot_ids, past_lens, R, H, D, max_k,
                                   total_cand, scale, pool, layer, workspace, workspace_bytes, dev_status, s);

    int nsplit = decode_nsplit(R, H, D, max_k, pool->n_cap, current_sms());
    if (nsplit > 1 && (!workspace || workspace_bytes < decode_workspace_bytes(nsplit, total_cand, H, D))) nsplit = 1;
    unsigned long long* sched = nullptr;
    if (workspace && workspace_bytes >= kSchedBytes) {
        sched = static_cast<unsigned long long*>(workspace);
        if (cudaMemsetAsync(sched, 0, sizeof(unsigned long long), s) != cudaSuccess) return UNIPIN_ERR_CUDA;
    }

    CUtensorMap tq, tk, tv;
    if ((rc = make_token_map(&tq, q_c, total_cand, H, D, kBlockM)) != UNIPIN_OK) return rc;
    if ((rc = make_pool_map(&tk, pool->k, pool, key_tile_width(D, true))) != UNIPIN_OK) return rc;
    if ((rc = make_pool_map(&tv, pool->v, pool, key_tile_width(D, true))) != UNIPIN_OK) return rc;

    AttnParams p = {};
    p.q = static_cast<const __nv_bfloat16*>(q_c);
    p.k_self = static_cast<const __nv_bfloat16*>(k_c);
    p.v_self = static_cast<const __nv_bfloat16*>(v_c);
    p.out = out;
    p.cu = cu_seqlens_c;
    p.past = past_lens;
    p.slots = slot_ids;
    p.nseg = R;
    p.H = H;
    p.G = H / pool->H;
    p.max_rows = max_k;
    p.total_rows = total_cand;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.layer = layer;
    p.S = pool->S;
    p.n_cap = pool->n_cap;
    p.nsplit = nsplit;
    p.sl2 = scale * kLog2e;
    p.status = dev_status;
    p.wait_limit_ns = wait_limit_ns();
    p.sched = sched;
    if (nsplit > 1) {
        p.part_o = reinterpret_cast<float*>(static_cast<char*>(workspace) + kSchedBytes);
        p.part_ml = p.part_o + (size_t)nsplit * total_cand * H * D;
    }
    const long long bound = (long long)R * H * nsplit * ((max_k + kPairRows - 1) / kPairRows);
    dim3 grid(persistent_blocks(bound), 1, 1);
    rc = launch_attn<true>(D, grid, tq, tk, tv, tk, tv, p, s);
    if (rc != UNIPIN_OK || nsplit == 1) return rc;

    const long long rows = (long long)total_cand * H;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    switch (D) {
    case 32:
        decode_merge_kernel<32><<<blocks, 256, 0, s>>>(p.part_o, p.part_ml, p.q, p.k_self, p.v_self, out,
                                                       p.out_fp32, total_cand, H, p.G, nsplit, p.sl2);
        break;
    case 64:
        decode_merge_kernel<64><<<blocks, 256, 0, s>>>(p.part_o, p.part_ml, p.q, p.k_self, p.v_self, out,
                                                       p.out_fp32, total_cand, H, p.G, nsplit, p.sl2);
        break;
    default:
        decode_merge_kernel<128><<<blocks, 256, 0, s>>>(p.part_o, p.part_ml, p.q, p.k_self, p.v_self, out,
                                                        p.out_fp32, total_cand, H, p.G, nsplit, p.sl2);
        break;
    }
    return cudaGetLastError() == cudaSuccess ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

int unipin_rank_decode_attn_noalloc(const void* q_c, const void* k_c, const void* v_c, void* out, int out_fp32,
                                    const int* cu_seqlens_c, const int* slot_ids, const int* past_lens, int R,
                                    int H, int D, int max_k, int total_cand, float scale,
                                    const unipin_kvpool* pool, int layer, int* dev_status, void* stream)
{
    if (!pool) return UNIPIN_ERR_INVALID_ARG;
    if (R < 0 || H < 1 || max_k < 0 || total_cand < 0) return UNIPIN_ERR_INVALID_ARG;
    if (!supported_d(D)) return UNIPIN_ERR_UNSUPPORTED;
    if (R == 0 || total_cand == 0 || max_k == 0) return UNIPIN_OK;
    if (pool->H < 1 || H % pool->H != 0) return UNIPIN_ERR_INVALID_ARG;
    // an E4M3 pool needs a dequantised copy unless the small-k kernel reads its codes
    if (pool->dtype == UNIPIN_POOL_E4M3 && !sk_takes_pool(pool, D, max_k, H / pool->H))
        return UNIPIN_ERR_UNSUPPORTED;
    // A shape whose split-n partials would not fit the array runs unsplit (the
    // regular call's fallback for a small workspace): slower, same result.
    void* scratch = nullptr;
    const int rc = noalloc_scratch_address(&scratch);
    if (rc != UNIPIN_OK) return rc;
    return unipin_rank_decode_attn(q_c, k_c, v_c, out, out_fp32, cu_seqlens_c, slot_ids, past_lens, R, H, D, max_k,
                                   total_cand, scale, pool, layer, scratch, kNoAllocScratchBytes, dev_status, stream);
}

size_t unipin_rank_decode_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

size_t unipin_masked_prefill_bwd_workspace_size(int total_tokens, int H)
{
    if (total_tokens < 0 || H < 1) return 0;
    return ((size_t)total_tokens * H * sizeof(float) + 15) / 16 * 16;
}

int unipin_masked_prefill_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                              const float* lse, float* dq, float* dk, float* dv, const int* cu_seqlens,
                              const int* past_lens, int B, int H, int H_kv, int D, int max_seqlen,
                              int total_tokens, float scale, void* workspace, size_t workspace_bytes,
                              int* dev_status, void* stream)
{
    if (B < 0 || H < 1 || H_kv < 1 || H % H_kv != 0 || max_seqlen < 0 || total_tokens < 0)
        return UNIPIN_ERR_INVALID_ARG;
    if (!supported_d(D)) return UNIPIN_ERR_UNSUPPORTED;
    if (!(scale > 0.f) || !std::isfinite(scale)) return UNIPIN_ERR_INVALID_ARG;
    if (B == 0 || total_tokens == 0 || max_seqlen == 0) return UNIPIN_OK;
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !cu_seqlens || !past_lens || !workspace)
        return UNIPIN_ERR_INVALID_ARG;
    if (workspace_bytes < unipin_masked_prefill_bwd_workspace_size(total_tokens, H)) return UNIPIN_ERR_INVALID_ARG;
    for (const void* ptr : {q, k, v, out, dout, (const void*)lse, (const void*)dq, (const void*)dk, (const void*)dv,
                            (const void*)workspace})
        if (!aligned16(ptr)) return UNIPIN_ERR_MISALIGNED;
    const long long items = (long long)B * H_kv * ((max_seqlen + kBwRows - 1) / kBwRows);
    if (items >= (1ll << 31)) return UNIPIN_ERR_INVALID_ARG;
    int rc = ensure_device();
    if (rc != UNIPIN_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    BwParams p = {};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.o = static_cast<const __nv_bfloat16*>(out);
    p.dout = static_cast<const __nv_bfloat16*>(dout);
    p.lse = lse;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dvec = static_cast<float*>(workspace);
    p.cu = cu_seqlens;
    p.past = past_lens;
    p.B = B;
    p.H = H;
    p.G = H / H_kv;
    p.total_rows = total_tokens;
    p.max_rows = max_seqlen;
    p.scale = scale;
    p.sl2 = scale * kLog2e;
    p.status = dev_status;
    p.wait_limit_ns = wait_limit_ns();

    const long long rows = (long long)total_tokens * H_kv;   // one warp per (token, key/value head)
    const unsigned prep_blocks = (unsigned)((rows + 7) / 8);
    if (D == 32)
        bwd_prep_kernel<32><<<prep_blocks, 256, 0, s>>>(p);
    else if (D == 64)
        bwd_prep_kernel<64><<<prep_blocks, 256, 0, s>>>(p);
    else
        bwd_prep_kernel<128><<<prep_blocks, 256, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return UNIPIN_ERR_CUDA;

    CUtensorMap tq, tk, tv, tdo;
    if ((rc = make_token_map(&tq, q, total_tokens, H, D, kBwRows)) != UNIPIN_OK) return rc;
    if ((rc = make_token_map(&tk, k, total_tokens, H_kv, D, kBwRows)) != UNIPIN_OK) return rc;
    if ((rc = make_token_map(&tv, v, total_tokens, H_kv, D, kBwRows)) != UNIPIN_OK) return rc;
    if ((rc = make_token_map(&tdo, dout, total_tokens, H, D, kBwRows)) != UNIPIN_OK) return rc;
    if (D == 32)
        bwd_kv_kernel<32><<<(unsigned)items, kBwThreads, BwCfg<32>::kSmemBytes, s>>>(tq, tk, tv, tdo, p);
    else if (D == 64)
        bwd_kv_kernel<64><<<(unsigned)items, kBwThreads, BwCfg<64>::kSmemBytes, s>>>(tq, tk, tv, tdo, p);
    else
        bwd_kv_kernel<128><<<(unsigned)items, kBwThreads, BwCfg<128>::kSmemBytes, s>>>(tq, tk, tv, tdo, p);
    return cudaGetLastError() == cudaSuccess ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}



int unipin_selftest_exp2(const float* x, float* y, int n, void* stream)
{
    if (n < 0 || (n > 0 && (!x || !y))) return UNIPIN_ERR_INVALID_ARG;
    if (n == 0) return UNIPIN_OK;
    const int threads = 256;
    const int blocks = (n / 2 + threads) / threads;
    exp2_poly_selftest_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

int unipin_selftest_bounded_wait(int* dev_status, unsigned int limit_us, void* stream)
{
    if (!dev_status || limit_us == 0) return UNIPIN_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return UNIPIN_ERR_CUDA;
    bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        dev_status, (unsigned long long)limit_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

}  // extern "C"
