// zha_device.cuh -- warp/block primitives shared by the ZHA kernels (sm_100a).
//
// Determinism rule used by every kernel: each elementary reduction has one
// fixed evaluation order.  A per-lane dot product is a fmaf chain over the
// lane's slice in element order, and a cross-lane sum is the xor butterfly
// 16, 8, 4, 2, 1.  The reduce-scatter below gives bit-identical sums to that
// butterfly (fp addition is commutative), so the build kernel and the append
// kernel, which run the same device functions, store identical summaries.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace zha {

constexpr unsigned FULL = 0xffffffffu;

// ---- element loads -------------------------------------------------------

// Load VEC consecutive elements of a row as fp32.  T is float or uint16_t
// (bf16 bits); VEC*sizeof(T) is 4, 8 or 16 bytes and the address is aligned
// to that size.
template <typename T, int VEC>
struct Vec;

template <>
struct Vec<float, 2> {
    static __device__ __forceinline__ void load(const float *p, float (&o)[2]) {
        float2 v = *reinterpret_cast<const float2 *>(p);
        o[0] = v.x; o[1] = v.y;
    }
};
template <>
struct Vec<float, 4> {
    static __device__ __forceinline__ void load(const float *p, float (&o)[4]) {
        float4 v = *reinterpret_cast<const float4 *>(p);
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
};
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
template <>
struct Vec<uint16_t, 2> {
    static __device__ __forceinline__ void load(const uint16_t *p, float (&o)[2]) {
        uint32_t w = *reinterpret_cast<const uint32_t *>(p);
        o[0] = bf_lo(w); o[1] = bf_hi(w);
    }
};
template <>
struct Vec<uint16_t, 4> {
    static __device__ __forceinline__ void load(const uint16_t *p, float (&o)[4]) {
        uint2 w = *reinterpret_cast<const uint2 *>(p);
        o[0] = bf_lo(w.x); o[1] = bf_hi(w.x); o[2] = bf_lo(w.y); o[3] = bf_hi(w.y);
    }
};
template <>
struct Vec<uint16_t, 8> {
    static __device__ __forceinline__ void load(const uint16_t *p, float (&o)[8]) {
        uint4 w = *reinterpret_cast<const uint4 *>(p);
        o[0] = bf_lo(w.x); o[1] = bf_hi(w.x); o[2] = bf_lo(w.y); o[3] = bf_hi(w.y);
        o[4] = bf_lo(w.z); o[5] = bf_hi(w.z); o[6] = bf_lo(w.w); o[7] = bf_hi(w.w);
    }
};

// Streaming (evict-first) variants for data read exactly once per call.
template <typename T, int VEC>
struct VecStream;
template <>
struct VecStream<float, 4> {
    static __device__ __forceinline__ void load(const float *p, float (&o)[4]) {
        float4 v = __ldcs(reinterpret_cast<const float4 *>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
};
template <>
struct VecStream<uint16_t, 8> {
    static __device__ __forceinline__ void load(const uint16_t *p, float (&o)[8]) {
        uint4 w = __ldcs(reinterpret_cast<const uint4 *>(p));
        o[0] = bf_lo(w.x); o[1] = bf_hi(w.x); o[2] = bf_lo(w.y); o[3] = bf_hi(w.y);
        o[4] = bf_lo(w.z); o[5] = bf_hi(w.z); o[6] = bf_lo(w.w); o[7] = bf_hi(w.w);
    }
};

// ---- fixed-order arithmetic ---------------------------------------------

// Per-lane partial dot product: fmaf chain in element order.
template <int VEC>
__device__ __forceinline__ float lane_dot(const float (&a)[VEC], const float (&b)[VEC]) {
    float acc = a[0] * b[0];
#pragma unroll
    for (int v = 1; v < VEC; ++v) acc = fmaf(a[v], b[v], acc);
    return acc;
}

// Xor-butterfly sum over all 32 lanes (every lane gets the sum).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(FULL, v, off);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, off));
    return v;
}

// Reduce-scatter of V values over the LANES lowest lane bits (LANES a power of
// two, V a multiple of LANES).  Afterwards v[0 .. V/LANES) of lane l hold the
// sums of the original indices [(l % LANES) * V/LANES, ... + V/LANES).  Each
// sum equals the xor-butterfly sum over those lanes, bit for bit.
template <int V, int LANES = 32>
__device__ __forceinline__ void reduce_scatter(float (&v)[V], int lane) {
    static_assert(V % LANES == 0, "V must be a multiple of LANES");
#pragma unroll
    for (int off = LANES / 2, n = V; off >= 1; off >>= 1, n >>= 1) {
        const int half = n / 2;
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = upper ? v[k] : v[k + half];
            const float keep = upper ? v[k + half] : v[k];
            const float recv = __shfl_xor_sync(FULL, send, off);
            v[k] = keep + recv;
        }
    }
}

// ---- ordering keys and fixed-point masses --------------------------------

// Map a float to a uint32 that sorts DESCENDING in the float: larger float
// -> smaller key.  NaN is not expected (scores are finite or -inf).
__device__ __forceinline__ uint32_t desc_key(float f) {
    uint32_t u = __float_as_uint(f);
    uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ~asc;
}
__device__ __forceinline__ float desc_key_to_float(uint32_t k) {
    uint32_t asc = ~k;
    uint32_t u = (asc & 0x80000000u) ? (asc & 0x7fffffffu) : ~asc;
    return __uint_as_float(u);
}

// Probability mass in 2^-40 fixed point: integer sums are exact and order
// independent, so every top-p decision is deterministic.
constexpr int MASS_FRAC_BITS = 40;
__device__ __forceinline__ unsigned long long mass_fx(float w) {
    return __float2ull_rn(w * 1099511627776.0f);  // 2^40
}

// ---- block helpers --------------------------------------------------------

// Inclusive scan of one uint32 per thread over the block; returns the
// inclusive prefix and writes the block total to *total.  `sh` holds
// blockDim/32 uint32.
__device__ __forceinline__ uint32_t block_scan_u32(uint32_t x, uint32_t *sh, uint32_t *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t v = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        uint32_t y = __shfl_up_sync(FULL, v, off);
        if (lane >= off) v += y;
    }
    if (lane == 31) sh[wid] = v;
    __syncthreads();
    if (wid == 0) {
        uint32_t s = lane < nw ? sh[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            uint32_t y = __shfl_up_sync(FULL, s, off);
            if (lane >= off) s += y;
        }
        if (lane < nw) sh[lane] = s;
    }
    __syncthreads();
    uint32_t base = wid > 0 ? sh[wid - 1] : 0;
    uint32_t tot = sh[nw - 1];
    __syncthreads();
    *total = tot;
    return base + v;
}

__device__ __forceinline__ unsigned long long block_scan_u64(unsigned long long x,
                                                             unsigned long long *sh,
                                                             unsigned long long *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    unsigned long long v = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        unsigned long long y = __shfl_up_sync(FULL, v, off);
        if (lane >= off) v += y;
    }
    if (lane == 31) sh[wid] = v;
    __syncthreads();
    if (wid == 0) {
        unsigned long long s = lane < nw ? sh[lane] : 0ull;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            unsigned long long y = __shfl_up_sync(FULL, s, off);
            if (lane >= off) s += y;
        }
        if (lane < nw) sh[lane] = s;
    }
    __syncthreads();
    unsigned long long base = wid > 0 ? sh[wid - 1] : 0ull;
    unsigned long long tot = sh[nw - 1];
    __syncthreads();
    *total = tot;
    return base + v;
}

__device__ __forceinline__ float block_max(float x, float *sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    x = warp_max(x);
    if (lane == 0) sh[wid] = x;
    __syncthreads();
    float r = -INFINITY;
    for (int i = 0; i < nw; ++i) r = fmaxf(r, sh[i]);
    __syncthreads();
    return r;
}

template <typename T>
__device__ __forceinline__ T block_sum_int(T x, T *sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
    if (lane == 0) sh[wid] = x;
    __syncthreads();
    T r = 0;
    for (int i = 0; i < nw; ++i) r += sh[i];
    __syncthreads();
    return r;
}

__device__ __forceinline__ uint32_t block_min_u32(uint32_t x, uint32_t *sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x = min(x, __shfl_xor_sync(FULL, x, off));
    if (lane == 0) sh[wid] = x;
    __syncthreads();
    uint32_t r = 0xffffffffu;
    for (int i = 0; i < nw; ++i) r = min(r, sh[i]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ uint32_t block_max_u32(uint32_t x, uint32_t *sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x = max(x, __shfl_xor_sync(FULL, x, off));
    if (lane == 0) sh[wid] = x;
    __syncthreads();
    uint32_t r = 0u;
    for (int i = 0; i < nw; ++i) r = max(r, sh[i]);
    __syncthreads();
    return r;
}

}  // namespace zha

namespace zha {

// ---- helpers over the first 256 threads of a CTA (named barrier 1) ---------
//
// The decode kernel runs 9 warps per CTA; routing phases use warps 0-7 and
// synchronise them with `bar.sync 1, 256` while warp 8 stays out.

constexpr int GT = 256;  // threads of a group

__device__ __forceinline__ void gsync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ unsigned long long g_scan_u64(unsigned long long x, unsigned long long *sh,
                                                         unsigned long long *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    unsigned long long v = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        unsigned long long y = __shfl_up_sync(FULL, v, off);
        if (lane >= off) v += y;
    }
    if (lane == 31) sh[wid] = v;
    gsync();
    unsigned long long base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < GT / 32; ++w) {
        const unsigned long long s = sh[w];
        if (w < wid) base += s;
        tot += s;
    }
    gsync();
    *total = tot;
    return base + v;
}

__device__ __forceinline__ uint32_t g_scan_u32(uint32_t x, uint32_t *sh, uint32_t *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t v = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        uint32_t y = __shfl_up_sync(FULL, v, off);
        if (lane >= off) v += y;
    }
    if (lane == 31) sh[wid] = v;
    gsync();
    uint32_t base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < GT / 32; ++w) {
        const uint32_t s = sh[w];
        if (w < wid) base += s;
        tot += s;
    }
    gsync();
    *total = tot;
    return base + v;
}

__device__ __forceinline__ uint32_t g_min_u32(uint32_t x, uint32_t *sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x = min(x, __shfl_xor_sync(FULL, x, off));
    if (lane == 0) sh[wid] = x;
    gsync();
    uint32_t r = 0xffffffffu;
#pragma unroll
    for (int w = 0; w < GT / 32; ++w) r = min(r, sh[w]);
    gsync();
    return r;
}

__device__ __forceinline__ uint32_t g_max_u32(uint32_t x, uint32_t *sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x = max(x, __shfl_xor_sync(FULL, x, off));
    if (lane == 0) sh[wid] = x;
    gsync();
    uint32_t r = 0u;
#pragma unroll
    for (int w = 0; w < GT / 32; ++w) r = max(r, sh[w]);
    gsync();
    return r;
}

// Sums of NV u64 values per thread over the group (fixed tree order).
template <int NV>
__device__ __forceinline__ void g_sum_u64(unsigned long long (&v)[NV], unsigned long long *red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        unsigned long long x = v[i];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
        if (lane == 0) red[wid * NV + i] = x;
    }
    gsync();
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        unsigned long long s = 0;
#pragma unroll
        for (int w = 0; w < GT / 32; ++w) s += red[w * NV + i];
        v[i] = s;
    }
    gsync();
}

}  // namespace zha
