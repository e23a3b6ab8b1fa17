// Pool write: copies the past K/V rows of each segment from the packed
// token-major layout [T, H, D] into the head-major pool [L, S, H, n_cap, D]
// at the segment's slot ([review] §2.4: retrieval writes the history K/V into
// the shared pool; [notes] §6: pool shape [L, S, H, n, D]).
//
// Memory-bound byte copy.  Each thread moves 16-byte vectors; consecutive
// threads walk one pool row after another, so the pool side (the write) is
// fully contiguous and each token-major source row is read as whole 32-byte
// sectors.
#pragma once

#include <cstdint>

#include "unipin.h"

namespace unipin {

struct PoolWriteParams {
    const uint4* k;        // [T, H, D] bf16 viewed as 16-byte vectors
    const uint4* v;
    uint4* pool_k;         // [L, S, H, n_cap, D]
    uint4* pool_v;
    const int* cu;
    const int* past;
    const int* slots;
    int H, D, S, n_cap, layer;
    int total_tokens;      // T
    int* status;
};

__global__ void __launch_bounds__(256) kvpool_write_kernel(const PoolWriteParams p)
{
    const int b = blockIdx.z;
    const int h = blockIdx.y;
    const int n = p.past[b];
    const int slot = p.slots[b];
    const int start = p.cu[b];
    const int len = p.cu[b + 1] - start;
    if (n < 0 || n > p.n_cap || n > len || slot < 0 || slot >= p.S || start < 0 ||
        (long long)start + n > (long long)p.total_tokens) {
        if (threadIdx.x == 0 && blockIdx.x == 0 && p.status) atomicCAS(p.status, 0, (int)UNIPIN_ERR_OUT_OF_RANGE);
        return;
    }
    const int vpr = p.D / 8;   // 16-byte vectors per row
    const long long total = (long long)n * vpr;
    const long long src_row0 = (long long)start * p.H + h;                                  // in rows of D
    const long long dst_row0 = (((long long)p.layer * p.S + slot) * p.H + h) * (long long)p.n_cap;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long j = idx / vpr;
        const int c = (int)(idx - j * vpr);
        const long long src = (src_row0 + j * p.H) * vpr + c;
        const long long dst = (dst_row0 + j) * vpr + c;
        const uint4 kv = __ldg(p.k + src);
        const uint4 vv = __ldg(p.v + src);
        p.pool_k[dst] = kv;
        p.pool_v[dst] = vv;
    }
}

}  // namespace unipin
