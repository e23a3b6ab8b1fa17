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
#include <cuda_bf16.h>
#include <cuda_fp16.h>

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

// E4M3 pools.  Writing stores E4M3(x * inv_scale): the bfloat16 input widened,
// one float32 product, then the hardware's nearest-even conversion that
// saturates to the largest finite code (448).  Reading expands code c to
// bfloat16(value(c) * scale): E4M3 -> f16 is exact, the product is one
// float32 rounding, the bfloat16 rounding is to nearest even.

// two floats -> two E4M3 codes (lo in the low byte)
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// eight bfloat16 (16 bytes) -> eight E4M3 codes (8 bytes), x * inv each
__device__ __forceinline__ uint2 e4m3x8_from_bf16(uint4 x, float inv)
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __fmul_rn(__uint_as_float(w[i] << 16), inv);
        const float hi = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv);
        c[i] = e4m3x2_from_f32(lo, hi);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// eight E4M3 codes -> eight bfloat16, value * scale each
__device__ __forceinline__ uint4 bf16x8_from_e4m3(uint2 codes, float scale)
{
    const uint32_t w[2] = {codes.x, codes.y};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint16_t pair = (uint16_t)(w[i >> 1] >> ((i & 1) * 16));
        uint32_t h2;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
        const float lo = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))), scale);
        const float hi = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h2 >> 16))), scale);
        const uint32_t blo = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
        const uint32_t bhi = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
        o[i] = blo | (bhi << 16);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

struct PoolWriteE4M3Params {
    const uint4* k;        // [T, H, D] bf16 viewed as 16-byte vectors
    const uint4* v;
    uint2* pool_k;         // [L, S, H, n_cap, D] E4M3 codes viewed as 8-byte vectors
    uint2* pool_v;
    const int* cu;
    const int* past;
    const int* slots;
    int H, D, S, n_cap, layer;
    int total_tokens;
    float inv_k, inv_v;    // float32 reciprocals of the pool's scales
    int* status;
};

// The rows and grid of kvpool_write_kernel; each thread turns 8 elements into 8 codes.
__global__ void __launch_bounds__(256) kvpool_write_e4m3_kernel(const PoolWriteE4M3Params p)
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
    const int vpr = p.D / 8;
    const long long total = (long long)n * vpr;
    const long long src_row0 = (long long)start * p.H + h;
    const long long dst_row0 = (((long long)p.layer * p.S + slot) * p.H + h) * (long long)p.n_cap;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long j = idx / vpr;
        const int c = (int)(idx - j * vpr);
        const long long src = (src_row0 + j * p.H) * vpr + c;
        const long long dst = (dst_row0 + j) * vpr + c;
        p.pool_k[dst] = e4m3x8_from_bf16(__ldg(p.k + src), p.inv_k);
        p.pool_v[dst] = e4m3x8_from_bf16(__ldg(p.v + src), p.inv_v);
    }
}

struct PoolDequantParams {
    const uint2* pool_k;   // [L, S, H, n_cap, D] E4M3 codes viewed as 8-byte vectors
    const uint2* pool_v;
    uint4* out_k;          // [R, H, n_cap, D] bfloat16 viewed as 16-byte vectors: a pool with L = 1, S = R
    uint4* out_v;
    int* out_slots;        // [R]: r, or -1 where request r's slot or length is out of range
    const int* past;
    const int* slots;
    int H, D, S, n_cap, layer;
    float k_scale, v_scale;
};

// Rows 0..n_r-1 of request r's slot (layer `layer`, every head) expanded into
// slot r of a bfloat16 pool; the rank decode then reads that pool.  Grid:
// (row-vector chunks, H, R).
__global__ void __launch_bounds__(256) kvpool_dequant_kernel(const PoolDequantParams p)
{
    const int r = blockIdx.z;
    const int h = blockIdx.y;
    const int n = p.past[r];
    const int slot = p.slots[r];
    const bool ok = slot >= 0 && slot < p.S && n >= 0 && n <= p.n_cap;
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) p.out_slots[r] = ok ? r : -1;
    if (!ok) return;   // the decode rejects the request (zero rows, status)
    const int vpr = p.D / 8;
    const long long total = (long long)n * vpr;
    const long long src_row0 = (((long long)p.layer * p.S + slot) * p.H + h) * (long long)p.n_cap;
    const long long dst_row0 = ((long long)r * p.H + h) * (long long)p.n_cap;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long j = idx / vpr;
        const int c = (int)(idx - j * vpr);
        const long long src = (src_row0 + j) * vpr + c;
        const long long dst = (dst_row0 + j) * vpr + c;
        p.out_k[dst] = bf16x8_from_e4m3(__ldg(p.pool_k + src), p.k_scale);
        p.out_v[dst] = bf16x8_from_e4m3(__ldg(p.pool_v + src), p.v_scale);
    }
}

}  // namespace unipin
