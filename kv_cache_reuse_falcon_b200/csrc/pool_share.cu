// Serving-side pieces around the KV pool ([notes] UniPinRec reproduction
// notes, §6 "serving: cross-process KV sharing"; [review] UniPinRec paper
// review, §2.4 co-serving): the retrieval process owns the pool and hands its
// memory to the ranking process through CUDA IPC handles, and it gives every
// request a pool slot in round-robin order, reusing a slot once the ranking
// side is done with it.  Host code only; no kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "unipin.h"

namespace {

typedef CUresult (*PFN_getAddressRange)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange through the runtime's driver entry point (the library
// does not link libcuda).
PFN_getAddressRange address_range_fn()
{
    static std::once_flag once;
    static PFN_getAddressRange fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_getAddressRange>(p);
    });
    return fn;
}

bool pool_shape_ok(int L, int S, int H, int n_cap, int D, int dtype)
{
    return L >= 1 && S >= 1 && H >= 1 && n_cap >= 1 && (D == 32 || D == 64 || D == 128) &&
           (dtype == UNIPIN_POOL_BF16 || dtype == UNIPIN_POOL_E4M3);
}

size_t pool_bytes(int L, int S, int H, int n_cap, int D, int dtype)
{
    return (size_t)L * S * H * n_cap * D * (dtype == UNIPIN_POOL_E4M3 ? 1 : 2);
}

// Handle and byte offset of the allocation that holds [ptr, ptr + bytes).
int export_one(const void* ptr, size_t bytes, unsigned char (&handle)[64], unsigned long long& offset)
{
    PFN_getAddressRange range = address_range_fn();
    if (!range) return UNIPIN_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return UNIPIN_ERR_INVALID_ARG;
    const unsigned long long off = reinterpret_cast<CUdeviceptr>(ptr) - base;
    if (off + bytes > size) return UNIPIN_ERR_OUT_OF_RANGE;   // the pool runs past its allocation
    cudaIpcMemHandle_t h;
    static_assert(sizeof(h) == 64, "CUDA IPC handle size");
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
        cudaGetLastError();
        return UNIPIN_ERR_CUDA;
    }
    std::memcpy(handle, &h, sizeof(h));
    offset = off;
    return UNIPIN_OK;
}

}  // namespace

struct unipin_slot_ring {
    std::mutex mu;
    std::vector<unsigned char> in_use;   // per slot: handed out and not yet released
    int next = 0;                        // where the round-robin scan starts
    int n_free = 0;
};

extern "C" {

int unipin_kvpool_share_export(const unipin_kvpool* pool, unipin_kvpool_share* out)
{
    if (!pool || !out || !pool->k || !pool->v) return UNIPIN_ERR_INVALID_ARG;
    if (!pool_shape_ok(pool->L, pool->S, pool->H, pool->n_cap, pool->D, pool->dtype)) return UNIPIN_ERR_INVALID_ARG;
    unipin_kvpool_share s;
    std::memset(&s, 0, sizeof(s));
    const size_t bytes = pool_bytes(pool->L, pool->S, pool->H, pool->n_cap, pool->D, pool->dtype);
    int rc = export_one(pool->k, bytes, s.k_handle, s.k_offset);
    if (rc == UNIPIN_OK) rc = export_one(pool->v, bytes, s.v_handle, s.v_offset);
    if (rc != UNIPIN_OK) return rc;
    s.L = pool->L;
    s.S = pool->S;
    s.H = pool->H;
    s.n_cap = pool->n_cap;
    s.D = pool->D;
    s.dtype = pool->dtype;
    s.k_scale = pool->k_scale;
    s.v_scale = pool->v_scale;
    *out = s;
    return UNIPIN_OK;
}

int unipin_kvpool_share_open(const unipin_kvpool_share* in, unipin_kvpool* out)
{
    if (!in || !out) return UNIPIN_ERR_INVALID_ARG;
    if (!pool_shape_ok(in->L, in->S, in->H, in->n_cap, in->D, in->dtype)) return UNIPIN_ERR_INVALID_ARG;
    cudaIpcMemHandle_t hk, hv;
    std::memcpy(&hk, in->k_handle, sizeof(hk));
    std::memcpy(&hv, in->v_handle, sizeof(hv));
    void* bk = nullptr;
    void* bv = nullptr;
    if (cudaIpcOpenMemHandle(&bk, hk, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        return UNIPIN_ERR_CUDA;
    }
    if (cudaIpcOpenMemHandle(&bv, hv, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        cudaIpcCloseMemHandle(bk);
        return UNIPIN_ERR_CUDA;
    }
    out->k = static_cast<char*>(bk) + in->k_offset;
    out->v = static_cast<char*>(bv) + in->v_offset;
    out->L = in->L;
    out->S = in->S;
    out->H = in->H;
    out->n_cap = in->n_cap;
    out->D = in->D;
    out->dtype = in->dtype;
    out->k_scale = in->k_scale;
    out->v_scale = in->v_scale;
    return UNIPIN_OK;
}

int unipin_kvpool_share_close(const unipin_kvpool_share* in, unipin_kvpool* opened)
{
    if (!in || !opened || !opened->k || !opened->v) return UNIPIN_ERR_INVALID_ARG;
    void* bk = static_cast<char*>(opened->k) - in->k_offset;
    void* bv = static_cast<char*>(opened->v) - in->v_offset;
    const bool ok = cudaIpcCloseMemHandle(bk) == cudaSuccess && cudaIpcCloseMemHandle(bv) == cudaSuccess;
    if (!ok) cudaGetLastError();
    opened->k = opened->v = nullptr;
    return ok ? UNIPIN_OK : UNIPIN_ERR_CUDA;
}

int unipin_slot_ring_create(int S, unipin_slot_ring** out)
{
    if (!out || S < 1) return UNIPIN_ERR_INVALID_ARG;
    unipin_slot_ring* r = new (std::nothrow) unipin_slot_ring;
    if (!r) return UNIPIN_ERR_INVALID_ARG;
    r->in_use.assign((size_t)S, 0);
    r->n_free = S;
    *out = r;
    return UNIPIN_OK;
}

int unipin_slot_ring_acquire(unipin_slot_ring* ring, int n, int* slot_ids)
{
    if (!ring || n < 0 || (n > 0 && !slot_ids)) return UNIPIN_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(ring->mu);
    if (n > ring->n_free) return UNIPIN_ERR_OUT_OF_RANGE;
    const int S = (int)ring->in_use.size();
    int got = 0;
    for (int step = 0; step < S && got < n; ++step) {
        const int s = (ring->next + step) % S;
        if (!ring->in_use[s]) {
            ring->in_use[s] = 1;
            slot_ids[got++] = s;
            if (got == n) ring->next = (s + 1) % S;
        }
    }
    ring->n_free -= n;
    return UNIPIN_OK;
}

int unipin_slot_ring_release(unipin_slot_ring* ring, int n, const int* slot_ids)
{
    if (!ring || n < 0 || (n > 0 && !slot_ids)) return UNIPIN_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(ring->mu);
    const int S = (int)ring->in_use.size();
    // all or nothing: every id must be in use and appear once
    std::vector<unsigned char> seen((size_t)S, 0);
    for (int i = 0; i < n; ++i) {
        const int s = slot_ids[i];
        if (s < 0 || s >= S || !ring->in_use[s] || seen[s]) return UNIPIN_ERR_INVALID_ARG;
        seen[s] = 1;
    }
    for (int i = 0; i < n; ++i) ring->in_use[slot_ids[i]] = 0;
    ring->n_free += n;
    return UNIPIN_OK;
}

int unipin_slot_ring_free_count(unipin_slot_ring* ring)
{
    if (!ring) return UNIPIN_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(ring->mu);
    return ring->n_free;
}

void unipin_slot_ring_destroy(unipin_slot_ring* ring)
{
    delete ring;
}

}  // extern "C"
